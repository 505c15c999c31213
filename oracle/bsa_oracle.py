"""CPU oracle for training-free block-sparse 3D attention — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this module. The CUDA library never calls it and shares no code
with it; when the CUDA extension is missing the product path fails instead of falling back
here.

Plain numpy, float64 arithmetic on the bf16 inputs (widened exactly). Every step is written
the slow, obvious way, in the order the pages describe the method:

1. ``block_layout``    — tile-major order of the 3D token grid, cut into query/key blocks
2. ``pool_blocks``     — per-block mean of Q or K over the block's real tokens
3. ``score_meanpool``  — softmax over key blocks of the pooled-query . pooled-key logits
   ``score_park``      — each query softmaxed over key blocks, then averaged in its block
4. ``select_topp``     — per-row top-p kept-block list (score descending, index ascending)
5. ``drift``           — per-head relative Q/K change since the cached reference
6. ``sparse_attention``— exact softmax attention restricted to the kept key blocks
7. ``reuse_run``       — the drift-gated mask-reuse loop across denoising steps
8. ``captured_mass``   — retrieval accuracy: the share of each query's exact (dense)
   attention mass that falls on its kept key blocks
9. ``rapid_run``       — one-shot block-importance estimate early in the run, cached scores
   and mask reused for the later steps, optional staged re-selection (Turbo)
10. ``recap_run``      — sparse attention corrected by a cached dense residual, refreshed
   per head when its query-key drift says the correction has aged
11. ``cluster_keys``   — PARK's key side: keys grouped by k-means in a metric built from the
   current queries, so that keys the queries score alike share a key block

Sources (page title, then the part of the page):
* PARK: Accurate Block Retrieval for Sparse Attention in Video Diffusion Transformers —
  Abstract: retrieval by averaged query/key block representations (the mean-pooled
  estimate), PARK's per-query normalisation over key blocks averaged within the query
  block, and attention computed only within the retrieved blocks.
* HASTE: Training-Free Video Diffusion Acceleration via Head-Wise Adaptive Sparse
  Attention — abstract: online top-p block selection, per-head thresholds, mask
  prediction skipped on small query-key drift.
* HEART: Exploiting Head Heterogeneity in Sparse Attention for Video Diffusion —
  abstract: Temporal Mask Reuse refreshes a head's cached mask only when its query-key
  drift exceeds a prescribed threshold.
* RAPID: Reusing Attention Sparsity with Inter-step Adaptation for Efficient Video
  Diffusion — English abstract: 3D attention, block importance estimated and the sparse
  mask cached for reuse across steps.
* RECAP: Reciprocal Sparse Attention and Hierarchical Caching for Efficient Video Diffusion
  — Abstract: a cached dense refinement corrects the interactions the current sparse
  estimate omits, and fresh sparse statistics track the inputs and regulate the aging
  correction.
* PARK — Abstract: inaccurate block retrieval either degrades quality or wastes computation;
  PARK is judged by its block retrieval accuracy (``captured_mass`` measures it without a
  model: how much of the exact attention the retrieved blocks hold).

Where the pages are silent the plainest reading is taken; each one is named at the point
of use (block shape/order, logit scale, top-p boundary, tie order, text blocks, drift
norm).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


# ----------------------------------------------------------------------------- helpers

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def default_tile(block: int):
    """Tile (t, h, w) that holds exactly one block: 1x8x8 for 64 tokens, 2x8x8 for 128.

    Reading: the pages speak of query and key blocks of a 3D token grid (PARK abstract;
    RAPID abstract, "3D attention") without a shape; a cube-like 3D tile is the plainest
    choice.
    """
    if block == 64:
        return (1, 8, 8)
    if block == 128:
        return (2, 8, 8)
    raise ValueError("block must be 64 or 128")


# ----------------------------------------------------------------------- 1. block layout

@dataclasses.dataclass
class Layout:
    perm: np.ndarray       # int64 [nb*B]: raster token index per slot, -1 for padding
    B: int
    nb: int                # total blocks
    nb_video: int          # video blocks (the last one may be partial)
    nb_text: int           # text blocks (after the padded video part)
    counts: np.ndarray     # int64 [nb]: real tokens per block

    @property
    def npad(self) -> int:
        return self.nb * self.B

    def rows(self, i: int) -> np.ndarray:
        """Raster token indices of the real tokens of block i, in block order."""
        s = self.perm[i * self.B:(i + 1) * self.B]
        return s[s >= 0]

    def is_text_block(self, i: int) -> bool:
        return i >= self.nb_video


def block_layout(T: int, H: int, W: int, text_tokens: int, block: int, tile=None) -> Layout:
    """Tile-major order of the video grid, cut into blocks of `block` tokens.

    Reading: tiles of shape (tt, th, tw) are visited in raster order of their tile
    coordinates; the tokens of a tile are taken in raster order (t, y, x; x fastest), edge
    tiles keep only the tokens inside the grid. The concatenated order is cut into blocks of
    B consecutive tokens, so only the last video block can be partial; it is padded. Text
    tokens (raster indices after the video tokens) follow as their own blocks, the last one
    padded.
    """
    tt, th, tw = tile if tile is not None else default_tile(block)
    order = []
    for a in range(0, T, tt):
        for b in range(0, H, th):
            for c in range(0, W, tw):
                for t in range(a, min(a + tt, T)):
                    for y in range(b, min(b + th, H)):
                        for x in range(c, min(c + tw, W)):
                            order.append((t * H + y) * W + x)
    nv = T * H * W
    nbv = -(-nv // block) if nv > 0 else 0
    nbt = -(-text_tokens // block) if text_tokens > 0 else 0
    nb = nbv + nbt
    perm = np.full(nb * block, -1, dtype=np.int64)
    perm[:nv] = np.asarray(order, dtype=np.int64)
    perm[nbv * block:nbv * block + text_tokens] = nv + np.arange(text_tokens, dtype=np.int64)
    counts = np.array([(perm[i * block:(i + 1) * block] >= 0).sum() for i in range(nb)],
                      dtype=np.int64)
    return Layout(perm, block, nb, nbv, nbt, counts)


# --------------------------------------------------------------------------- 2. pooling

def pool_blocks(X: np.ndarray, layout: Layout) -> np.ndarray:
    """Mean of X's rows over each block's real tokens (padding excluded; divide by the real
    count). X is float64 [N, d] in raster order; returns [nb, d].
    (PARK abstract: "averaged representations of query and key blocks".)"""
    out = np.zeros((layout.nb, X.shape[1]), dtype=np.float64)
    for i in range(layout.nb):
        r = layout.rows(i)
        out[i] = X[r].sum(axis=0) / len(r)
    return out


# --------------------------------------------------------------------------- 3. scoring

def _softmax_rows(L: np.ndarray) -> np.ndarray:
    """Row softmax, two passes: subtract the row max, exponentiate, divide by the sum."""
    m = L.max(axis=1, keepdims=True)
    e = np.exp(L - m)
    return e / e.sum(axis=1, keepdims=True)


def score_meanpool(Qh: np.ndarray, Kh: np.ndarray, layout: Layout) -> np.ndarray:
    """S[i, j] = softmax over j of (qbar_i . kbar_j) / sqrt(d), all key blocks j.

    The mean-pooled retrieval estimate the PARK abstract describes (query and key blocks
    represented by their averages). Reading: the logit scale is 1/sqrt(d), the same as the
    attention it predicts; no size correction for partial blocks.
    """
    d = Qh.shape[1]
    qbar = pool_blocks(Qh, layout)
    kbar = pool_blocks(Kh, layout)
    return _softmax_rows(qbar @ kbar.T / math.sqrt(d))


def score_park(Qh: np.ndarray, Kh: np.ndarray, layout: Layout) -> np.ndarray:
    """P[i, j] = mean over real queries q of block i of softmax_j(q . kbar_j / sqrt(d)).

    PARK abstract: every original query is kept, its attention over key blocks is
    normalised on its own, and those distributions are averaged within the query block.
    Reading: key blocks are represented by their mean key (the page's query-aware key
    clustering has no formula there and is not part of this scorer).
    """
    d = Qh.shape[1]
    kbar = pool_blocks(Kh, layout)
    P = np.zeros((layout.nb, layout.nb), dtype=np.float64)
    for i in range(layout.nb):
        q = Qh[layout.rows(i)]
        P[i] = _softmax_rows(q @ kbar.T / math.sqrt(d)).mean(axis=0)
    return P


# ------------------------------------------------------------------------ 4. top-p select

def sort_row(scores_row_f32: np.ndarray) -> np.ndarray:
    """Block indices ordered by score descending, then index ascending."""
    s = np.asarray(scores_row_f32, dtype=np.float32).astype(np.float64)
    j = np.arange(len(s))
    return np.lexsort((j, -s))


def select_row(scores_row_f32: np.ndarray, p: float, forced=()):
    """Top-p kept list for one (head, query-block) row.

    HASTE abstract (online top-p block selection, per-head thresholds). Readings:
    * blocks are ordered by score descending, ties by index ascending;
    * the kept prefix is the shortest one whose cumulative score reaches p (>= p), so at
      least one block is kept; p >= 1 keeps every block (float32 sums may stop short of 1);
    * the cumulative sum is taken in float32, sequentially in sorted order (float32 is the
      precision of the stored scores and of the kernel that makes the same decision);
    * forced blocks (text key blocks) are added to the kept set, and the union keeps the
      same order.
    Returns (kept list, sorted order, float32 cumulative masses in sorted order).
    """
    s32 = np.asarray(scores_row_f32, dtype=np.float32)
    order = sort_row(s32)
    cum = np.cumsum(s32[order], dtype=np.float32)
    n = len(order)
    if p >= 1.0:
        m = n
    else:
        hit = np.nonzero(cum >= np.float32(p))[0]
        m = int(hit[0]) + 1 if len(hit) else n
    keep = np.zeros(n, dtype=bool)
    keep[order[:m]] = True
    keep[np.asarray(list(forced), dtype=np.int64)] = True
    kept = [int(j) for j in order[keep[order]]]
    return kept, order, cum


def select_topp(scores_f32: np.ndarray, p: float, layout: Layout):
    """Kept-block lists for every query block of one head.

    Text query blocks keep every block; video query blocks keep their top-p set plus all
    text key blocks (reading of "text tokens always kept as dense key/query blocks").
    Returns idx int32 [nb, nb] (entries past cnt are -1) and cnt int32 [nb].
    """
    nb = layout.nb
    idx = np.full((nb, nb), -1, dtype=np.int32)
    cnt = np.zeros(nb, dtype=np.int32)
    text = list(range(layout.nb_video, nb))
    for i in range(nb):
        if layout.is_text_block(i):
            kept, _, _ = select_row(scores_f32[i], 1.0)
        else:
            kept, _, _ = select_row(scores_f32[i], p, forced=text)
        idx[i, :len(kept)] = kept
        cnt[i] = len(kept)
    return idx, cnt


# ------------------------------------------------------------------------------ 5. drift

def relative_change(X: np.ndarray, Xref: np.ndarray) -> float:
    """||X - Xref||_F / ||Xref||_F (0 when both are zero, +inf when only Xref is)."""
    num = math.sqrt(float(((X - Xref) ** 2).sum()))
    den = math.sqrt(float((Xref ** 2).sum()))
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return num / den


def drift(Qh, Kh, Qref_h, Kref_h) -> float:
    """Per-head query-key drift since the head's last refresh (HEART abstract, Temporal
    Mask Reuse). Reading: the larger of the relative Frobenius changes of Q and K over the
    head's real tokens."""
    return max(relative_change(Qh, Qref_h), relative_change(Kh, Kref_h))


def refresh_decision(delta: float, tau: float, have_cache: bool) -> bool:
    """Refresh when there is no cached mask yet or the drift is strictly above tau."""
    return (not have_cache) or (delta > tau)


# -------------------------------------------------------------------------- 6. attention

def sparse_attention_head(Qh, Kh, Vh, idx, cnt, layout: Layout, qblocks=None) -> np.ndarray:
    """O_t = sum over real keys u of the kept blocks of softmax_u(Q_t . K_u / sqrt(d)) V_u.

    The exact definition of attention restricted to the retrieved blocks (PARK abstract:
    attention computed only within the retrieved blocks). Logits over the kept real keys
    are materialised, softmaxed in two passes (max, then sum) and applied to V. Rows of
    query blocks not listed in `qblocks` are left as NaN. Returns float64 [N, d] in raster
    order.
    """
    N, d = Qh.shape
    O = np.full((N, Vh.shape[1]), np.nan, dtype=np.float64)
    scale = 1.0 / math.sqrt(d)
    for i in (range(layout.nb) if qblocks is None else qblocks):
        rows = layout.rows(i)
        keys = np.concatenate([layout.rows(int(j)) for j in idx[i, :cnt[i]]])
        L = (Qh[rows] @ Kh[keys].T) * scale
        m = L.max(axis=1, keepdims=True)
        e = np.exp(L - m)
        O[rows] = (e @ Vh[keys]) / e.sum(axis=1, keepdims=True)
    return O


# ----------------------------------------------------------------------- whole pipeline

def score_head(Qh, Kh, layout, mode: str) -> np.ndarray:
    if mode == "meanpool":
        return score_meanpool(Qh, Kh, layout)
    if mode == "park":
        return score_park(Qh, Kh, layout)
    raise ValueError(mode)


def pipeline_head(Qb, Kb, Vb, layout, p, mode="meanpool", qblocks=None):
    """Score -> select -> attend for one head (bf16 bit inputs [N, d]).
    Returns (scores float32 [nb, nb], idx, cnt, O float64 [N, d])."""
    Qh, Kh, Vh = bf16_to_f64(Qb), bf16_to_f64(Kb), bf16_to_f64(Vb)
    S = score_head(Qh, Kh, layout, mode).astype(np.float32)
    idx, cnt = select_topp(S, p, layout)
    O = sparse_attention_head(Qh, Kh, Vh, idx, cnt, layout, qblocks)
    return S, idx, cnt, O


# --------------------------------------------------------------------- 7. mask-reuse run

def reuse_run(steps_qk, V, layout, p, tau, mode="meanpool", attend=True):
    """Drift-gated mask reuse across denoising steps (HEART abstract, Temporal Mask Reuse;
    HASTE abstract; RAPID abstract: masks cached and reused across steps).

    `steps_qk` yields (Q, K) bf16 bits [heads, N, d] per step; V is fixed. At each step a
    head whose drift since its last refresh exceeds tau (or that has no cache yet) re-scores,
    re-selects and snapshots its Q, K as the new reference; the other heads reuse their
    cached kept lists. Returns a dict with per-step drift, refresh flags, the final masks
    and (if `attend`) the per-step outputs.
    """
    heads = V.shape[0]
    Vf = [bf16_to_f64(V[h]) for h in range(heads)]
    ref = [None] * heads
    masks = [None] * heads
    out = {"drift": [], "refresh": [], "O": []}
    for Q, K in steps_qk:
        deltas, flags, Os = [], [], []
        for h in range(heads):
            Qh, Kh = bf16_to_f64(Q[h]), bf16_to_f64(K[h])
            if ref[h] is None:
                delta = math.inf
            else:
                delta = drift(Qh, Kh, ref[h][0], ref[h][1])
            fresh = refresh_decision(delta, tau, ref[h] is not None)
            if fresh:
                S = score_head(Qh, Kh, layout, mode).astype(np.float32)
                masks[h] = select_topp(S, p[h], layout)
                ref[h] = (Qh, Kh)
            deltas.append(delta)
            flags.append(fresh)
            if attend:
                Os.append(sparse_attention_head(Qh, Kh, Vf[h], masks[h][0], masks[h][1], layout))
        out["drift"].append(deltas)
        out["refresh"].append(flags)
        if attend:
            out["O"].append(np.stack(Os))
    out["masks"] = masks
    return out


# ------------------------------------------------------------------ 8. retrieval accuracy

def captured_mass(Qh, Kh, idx, cnt, layout: Layout, qblocks=None) -> np.ndarray:
    """Share of the exact attention mass that each query block's kept key blocks capture.

    For a real query t of block i, its exact attention is softmax over ALL real keys u of
    Q_t . K_u / sqrt(d); the captured mass is the sum of that distribution over the real keys
    of the kept blocks idx[i, :cnt[i]] (PARK abstract: accurate block retrieval, where an
    inaccurate retrieval loses attention mass or spends computation on blocks that hold
    little). Returned per query block, as the mean over its real queries: float64 [nb]
    (NaN for blocks not in `qblocks`). Reading: the plain average over queries, every query
    weighted alike.
    """
    d = Qh.shape[1]
    scale = 1.0 / math.sqrt(d)
    real = np.concatenate([layout.rows(j) for j in range(layout.nb)])
    out = np.full(layout.nb, np.nan)
    for i in (range(layout.nb) if qblocks is None else qblocks):
        rows = layout.rows(i)
        L = (Qh[rows] @ Kh[real].T) * scale
        m = L.max(axis=1, keepdims=True)
        e = np.exp(L - m)
        p = e / e.sum(axis=1, keepdims=True)
        kept = np.zeros(Qh.shape[0], dtype=bool)
        for j in idx[i, :cnt[i]]:
            kept[layout.rows(int(j))] = True
        out[i] = p[:, kept[real]].sum(axis=1).mean()
    return out


# ---------------------------------------------------------------- 9. one-shot schedule

def rapid_run(steps_qk, V, layout, p0, estimate_step=0, stages=(), mode="meanpool", attend=True):
    """One-shot block-importance estimate with cached reuse, and Turbo staged pruning.

    RAPID English abstract: block importance is estimated once, early in the generation; the
    scores and the sparse mask are cached and reused by the later steps (no recalculation);
    the cached scores also allow an optional multi-stage adaptive pruning (Turbo mode), since
    the attention density the steps need decays as the generation proceeds. Readings (the
    abstract gives no schedule): steps before `estimate_step` attend densely (every key
    block); at `estimate_step` every head is scored and its kept lists are selected with p0
    (per head); `stages` is a sequence of (step, p) with increasing steps: from each such step
    on, the kept lists are selected anew from the CACHED scores with that p (no re-scoring).

    `steps_qk` yields (Q, K) bf16 bits [heads, N, d] per step; V is fixed. Returns a dict
    with per-step kept-block counts (None for dense steps), the selection each step used
    ('dense', 'estimate', 'reuse' or 'stage'), the final masks and scores and (if
    `attend`) the per-step outputs.
    """
    heads = V.shape[0]
    Vf = [bf16_to_f64(V[h]) for h in range(heads)]
    stage_p = {int(s): p for s, p in stages}
    scores = [None] * heads
    masks = [None] * heads
    out = {"kind": [], "cnt": [], "O": []}
    for s, (Q, K) in enumerate(steps_qk):
        if s < estimate_step:
            kind = "dense"
        elif s == estimate_step:
            kind = "estimate"
        elif s in stage_p:
            kind = "stage"
        else:
            kind = "reuse"
        Os, cnts = [], []
        for h in range(heads):
            Qh, Kh = bf16_to_f64(Q[h]), bf16_to_f64(K[h])
            if kind == "estimate":
                scores[h] = score_head(Qh, Kh, layout, mode).astype(np.float32)
                masks[h] = select_topp(scores[h], p0[h], layout)
            elif kind == "stage":
                masks[h] = select_topp(scores[h], stage_p[s], layout)
            if kind == "dense":
                idx = np.tile(np.arange(layout.nb, dtype=np.int32), (layout.nb, 1))
                cnt = np.full(layout.nb, layout.nb, dtype=np.int32)
                cnts.append(None)
            else:
                idx, cnt = masks[h]
                cnts.append(cnt.copy())
            if attend:
                Os.append(sparse_attention_head(Qh, Kh, Vf[h], idx, cnt, layout))
        out["kind"].append(kind)
        out["cnt"].append(cnts)
        if attend:
            out["O"].append(np.stack(Os))
    out["masks"] = masks
    out["scores"] = scores
    return out


# ------------------------------------------------------------ 10. cached dense correction

def dense_attention_head(Qh, Kh, Vh, layout: Layout) -> np.ndarray:
    """Attention over every key block (the kept list of every row is all blocks)."""
    idx = np.tile(np.arange(layout.nb, dtype=np.int32), (layout.nb, 1))
    cnt = np.full(layout.nb, layout.nb, dtype=np.int32)
    return sparse_attention_head(Qh, Kh, Vh, idx, cnt, layout)


def recap_run(steps_qk, V, layout, p, tau, mode="meanpool"):
    """Sparse attention with a cached dense correction, refreshed per head on drift.

    RECAP abstract: a cached dense refinement corrects the interactions that the current
    sparse estimate omits, while fresh sparse statistics follow the input changes and
    regulate the aging correction. Readings (the abstract gives no formula; the rest of RECAP,
    whole-step prediction reuse and its error feedback, is out of scope here):
    * the correction of head h is R_h = O_dense - O_sparse at the head's last refresh step;
    * the fresh statistics are the per-head query-key drift of Temporal Mask Reuse (HEART
      abstract): a head whose drift since its last refresh exceeds tau (or that has no cache
      yet) refreshes its mask, its dense output and its correction, and outputs the dense
      attention; every other head outputs its current sparse attention plus its cached R.

    `steps_qk` yields (Q, K) bf16 bits [heads, N, d] per step; V is fixed. Returns per-step
    refresh flags, outputs and the final corrections.
    """
    heads = V.shape[0]
    Vf = [bf16_to_f64(V[h]) for h in range(heads)]
    ref = [None] * heads
    masks = [None] * heads
    corr = [None] * heads
    out = {"refresh": [], "O": []}
    for Q, K in steps_qk:
        flags, Os = [], []
        for h in range(heads):
            Qh, Kh = bf16_to_f64(Q[h]), bf16_to_f64(K[h])
            delta = math.inf if ref[h] is None else drift(Qh, Kh, ref[h][0], ref[h][1])
            fresh = refresh_decision(delta, tau, ref[h] is not None)
            if fresh:
                S = score_head(Qh, Kh, layout, mode).astype(np.float32)
                masks[h] = select_topp(S, p[h], layout)
                ref[h] = (Qh, Kh)
            O_sparse = sparse_attention_head(Qh, Kh, Vf[h], masks[h][0], masks[h][1], layout)
            if fresh:
                O_dense = dense_attention_head(Qh, Kh, Vf[h], layout)
                corr[h] = O_dense - O_sparse
                Os.append(O_dense)
            else:
                Os.append(O_sparse + corr[h])
            flags.append(fresh)
        out["refresh"].append(flags)
        out["O"].append(np.stack(Os))
    out["R"] = corr
    return out


# ----------------------------------------------------------- 11. query-aware key blocks

def query_metric(Qh: np.ndarray, layout: Layout) -> np.ndarray:
    """M = (1/n) sum over the head's real queries q of q q^T (d x d).

    For two keys, (k1 - k2)^T M (k1 - k2) is the mean over the queries of (q.k1 - q.k2)^2: how
    differently the current queries score them. Reading of PARK abstract ("uses information
    from the current queries to transform keys before clustering, so that keys receiving
    similar QK scores are grouped together"): the transform is k -> L^T k with M = L L^T, under
    which Euclidean distance is exactly that score difference; clustering in the transformed
    space is clustering with the metric M.
    """
    rows = np.concatenate([layout.rows(i) for i in range(layout.nb)])
    Q = Qh[rows]
    return Q.T @ Q / len(rows)


def cluster_keys(Qh: np.ndarray, Kh: np.ndarray, layout: Layout, iters: int = 2, with_objective: bool = False):
    """Query-aware key blocks (PARK abstract, key-side clustering).

    Readings (the page gives no formula): the video keys are clustered by Lloyd's k-means
    with the metric M of `query_metric`, into as many clusters as there are video blocks,
    starting from the means of the 3D-tile blocks; each of `iters` rounds assigns every key
    to the centroid c_j minimising (k - c_j)^T M (k - c_j) (ties to the lowest j), then moves
    every non-empty cluster's centroid to the mean of its keys. The key blocks then follow the
    block rule of the query side: the video keys in order of (cluster, raster index), cut every
    B keys (so every key block keeps its tile-layout size); text key blocks are unchanged.
    Returns (key_perm int64 [nb*B] like Layout.perm, assignment int64 [Nv] of the last round)
    and, with `with_objective`, the last round's objective [Nv, nb_video] and the magnitude of
    its terms (|b_j| + 2 sum_c |k_c w_jc|, for error bounds).
    """
    if iters < 1:
        raise ValueError("iters >= 1")
    M = query_metric(Qh, layout)
    nv = layout.nb_video
    Nv = int(layout.counts[:nv].sum())
    Kv = Kh[:Nv]
    C = np.stack([Kh[layout.rows(j)].mean(axis=0) for j in range(nv)])
    a = obj = W = b = None
    for _ in range(iters):
        W = C @ M                                   # w_j = M c_j  (M symmetric)
        b = (C * W).sum(axis=1)                     # c_j^T M c_j
        obj = b[None, :] - 2.0 * (Kv @ W.T)         # (k - c_j)^T M (k - c_j) - k^T M k
        a = np.argmin(obj, axis=1)                  # first index on ties
        for j in range(nv):
            members = Kv[a == j]
            if len(members):
                C[j] = members.mean(axis=0)
    order = np.lexsort((np.arange(Nv), a))          # by cluster, then raster index
    key_perm = layout.perm.copy()
    key_perm[:Nv] = order
    if with_objective:
        scale = np.abs(b)[None, :] + 2.0 * (np.abs(Kv) @ np.abs(W).T)
        return key_perm, a, obj, scale
    return key_perm, a


def key_layout(layout: Layout, key_perm: np.ndarray) -> Layout:
    """The block layout of the key side after `cluster_keys` (same block sizes)."""
    return Layout(np.asarray(key_perm, dtype=np.int64), layout.B, layout.nb, layout.nb_video,
                  layout.nb_text, layout.counts.copy())


def score_park_keys(Qh, Kh, qlayout: Layout, klayout: Layout) -> np.ndarray:
    """PARK scores with separate query and key block layouts (key blocks from cluster_keys)."""
    d = Qh.shape[1]
    kbar = pool_blocks(Kh, klayout)
    P = np.zeros((qlayout.nb, klayout.nb), dtype=np.float64)
    for i in range(qlayout.nb):
        q = Qh[qlayout.rows(i)]
        P[i] = _softmax_rows(q @ kbar.T / math.sqrt(d)).mean(axis=0)
    return P


def sparse_attention_keys(Qh, Kh, Vh, idx, cnt, qlayout: Layout, klayout: Layout, qblocks=None):
    """sparse_attention_head with the key blocks of `klayout` (query blocks of `qlayout`)."""
    N, d = Qh.shape
    O = np.full((N, Vh.shape[1]), np.nan, dtype=np.float64)
    scale = 1.0 / math.sqrt(d)
    for i in (range(qlayout.nb) if qblocks is None else qblocks):
        rows = qlayout.rows(i)
        keys = np.concatenate([klayout.rows(int(j)) for j in idx[i, :cnt[i]]])
        L = (Qh[rows] @ Kh[keys].T) * scale
        e = np.exp(L - L.max(axis=1, keepdims=True))
        O[rows] = (e @ Vh[keys]) / e.sum(axis=1, keepdims=True)
    return O
