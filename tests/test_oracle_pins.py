"""Pins for the CPU oracle: checks against facts the pages and the mathematics fix, not
against the oracle itself (closed forms, brute force, library routines, invariants and
hand-derived cases). CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import bsa_oracle as O
from block_sparse_attention_query_b200 import inputs
from tests.conftest import GOLDEN


def _bf16_round_f64(x):
    return O.bf16_to_f64(inputs.f32_to_bf16_bits(np.asarray(x, np.float32)))


# ------------------------------------------------------------------------------ layout

def test_layout_golden_cases():
    with open(os.path.join(GOLDEN, "layout_small.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        L = O.block_layout(c["T"], c["H"], c["W"], c["text_tokens"], c["block"], tuple(c["tile"]))
        assert L.perm.tolist() == c["perm"], c["why"]


@pytest.mark.parametrize("T,H,W,text,B", [(4, 16, 16, 0, 64), (21, 30, 52, 0, 128),
                                          (3, 5, 7, 0, 64), (5, 9, 17, 40, 64), (3, 3, 3, 130, 128)])
def test_layout_is_permutation_with_tail_padding(T, H, W, text, B):
    L = O.block_layout(T, H, W, text, B)
    nv = T * H * W
    real = L.perm[L.perm >= 0]
    assert sorted(real.tolist()) == list(range(nv + text))
    assert L.nb == math.ceil(nv / B) + math.ceil(text / B)
    # padding only at the end of the video part and at the end of the text part
    vid = L.perm[:L.nb_video * B]
    assert (vid[:nv] >= 0).all() and (vid[nv:] == -1).all()
    txt = L.perm[L.nb_video * B:]
    assert (txt[:text] == nv + np.arange(text)).all() and (txt[text:] == -1).all()
    assert L.counts.sum() == nv + text


def test_layout_tiny_blocks_are_tiles():
    # 4x16x16 grid with 1x8x8 tiles and 64-token blocks: every block is exactly one tile
    L = O.block_layout(4, 16, 16, 0, 64)
    assert L.nb == 16
    for i in range(16):
        r = L.rows(i)
        t, y, x = r // 256, (r // 16) % 16, r % 16
        assert len(set(t.tolist())) == 1
        assert (y.max() - y.min()) == 7 and (x.max() - x.min()) == 7
        assert len(set((y // 8).tolist())) == 1 and len(set((x // 8).tolist())) == 1


def test_layout_wan_sizes():
    L = O.block_layout(21, 30, 52, 0, 128)
    assert (L.nb, L.counts[-1]) == (256, 120)
    L = O.block_layout(33, 45, 80, 256, 128)
    assert (L.nb, L.nb_video, L.nb_text, L.counts[L.nb_video - 1]) == (931, 929, 2, 16)


# ------------------------------------------------------------------------------ pooling

def test_pool_constant_within_block_is_exact():
    # 15 tokens, blocks of 4: ragged last block with 3 real tokens
    L = O.block_layout(1, 3, 5, 0, 4, (1, 2, 2))
    rng = np.random.default_rng(1)
    consts = rng.standard_normal((L.nb, 6))
    X = np.zeros((15, 6))
    for i in range(L.nb):
        X[L.rows(i)] = consts[i]
    got = O.pool_blocks(X, L)
    assert np.array_equal(got, consts)  # mean of equal values is exact


# ------------------------------------------------------------------------------ scoring

def _dense_probs(Qh, Kh):
    """Textbook softmax attention probabilities via torch (float64, CPU)."""
    q, k = torch.from_numpy(Qh), torch.from_numpy(Kh)
    return torch.softmax(q @ k.T / math.sqrt(Qh.shape[1]), dim=-1).numpy()


def _rand_qk(n, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (_bf16_round_f64(scale * rng.standard_normal((n, d))),
            _bf16_round_f64(scale * rng.standard_normal((n, d))))


@pytest.mark.parametrize("mode", ["meanpool", "park"])
def test_score_rows_sum_to_one(mode):
    L = O.block_layout(3, 5, 7, 9, 8, (1, 2, 2))
    Q, K = _rand_qk(3 * 5 * 7 + 9, 16, 2, 2.0)
    S = O.score_head(Q, K, L, mode)
    assert S.shape == (L.nb, L.nb)
    assert np.allclose(S.sum(axis=1), 1.0, atol=1e-12)
    assert (S >= 0).all()


def test_park_equals_exact_block_mass_when_keys_constant_in_blocks():
    # full blocks (no padding): with each block's keys all equal, the per-query softmax over
    # block means equals the exact attention mass that falls in each key block
    L = O.block_layout(2, 8, 8, 0, 16, (1, 4, 4))
    assert (L.counts == 16).all()
    rng = np.random.default_rng(3)
    Q = _bf16_round_f64(2.0 * rng.standard_normal((128, 32)))
    kc = _bf16_round_f64(2.0 * rng.standard_normal((L.nb, 32)))
    K = np.zeros((128, 32))
    for j in range(L.nb):
        K[L.rows(j)] = kc[j]
    P = _dense_probs(Q, K)
    exact = np.zeros((L.nb, L.nb))
    for i in range(L.nb):
        for j in range(L.nb):
            exact[i, j] = P[np.ix_(L.rows(i), L.rows(j))].sum(axis=1).mean()
    assert np.allclose(O.score_park(Q, K, L), exact, rtol=1e-10, atol=1e-14)


def test_meanpool_equals_park_equals_exact_when_q_and_k_constant_in_blocks():
    L = O.block_layout(2, 8, 8, 0, 16, (1, 4, 4))
    rng = np.random.default_rng(4)
    qc = _bf16_round_f64(2.0 * rng.standard_normal((L.nb, 32)))
    kc = _bf16_round_f64(2.0 * rng.standard_normal((L.nb, 32)))
    Q = np.zeros((128, 32))
    K = np.zeros((128, 32))
    for j in range(L.nb):
        Q[L.rows(j)] = qc[j]
        K[L.rows(j)] = kc[j]
    P = _dense_probs(Q, K)
    exact = np.array([[P[np.ix_(L.rows(i), L.rows(j))].sum(axis=1).mean() for j in range(L.nb)]
                      for i in range(L.nb)])
    assert np.allclose(O.score_meanpool(Q, K, L), exact, rtol=1e-10, atol=1e-14)
    assert np.allclose(O.score_park(Q, K, L), exact, rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("mode", ["meanpool", "park"])
def test_block_size_one_is_dense_softmax(mode):
    L = O.block_layout(1, 3, 7, 0, 1, (1, 1, 1))
    Q, K = _rand_qk(21, 16, 5, 1.5)
    perm = L.perm
    S = O.score_head(Q, K, L, mode)          # blocks in tile order
    P = _dense_probs(Q, K)                    # raster order
    assert np.allclose(S, P[np.ix_(perm, perm)], rtol=1e-12, atol=1e-15)


# -------------------------------------------------------------------------------- top-p

def test_topp_golden_cases():
    with open(os.path.join(GOLDEN, "topp_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        kept, _, _ = O.select_row(np.array(c["scores"], np.float32), c["p"], c["forced"])
        assert kept == c["kept"], c["why"]


def test_topp_is_minimum_cardinality_max_mass_set():
    # brute force over all subsets: the kept set is the smallest set whose mass reaches p,
    # and among sets of that size it has the largest mass
    rng = np.random.default_rng(6)
    checked = 0
    for trial in range(300):
        n = int(rng.integers(1, 11))
        s = rng.dirichlet(np.full(n, 0.7)).astype(np.float32)
        p = float(rng.choice([0.3, 0.5, 0.8, 0.9, 0.95]))
        exact = s.astype(np.float64)
        best = None
        for k in range(1, n + 1):
            masses = [sum(exact[list(c)]) for c in itertools.combinations(range(n), k)]
            if max(masses) >= p:
                best = (k, max(masses))
                break
        if best is None:
            best = (n, exact.sum())
        # skip rows where float32 summation could flip the decision
        if min(abs(np.cumsum(np.sort(exact)[::-1]) - p)) < 1e-6:
            continue
        kept, _, _ = O.select_row(s, p)
        assert len(kept) == best[0]
        assert abs(exact[kept].sum() - best[1]) < 1e-12
        checked += 1
    assert checked > 250


def test_topp_p_one_keeps_all_sorted():
    s = np.array([0.1, 0.4, 0.2, 0.3], np.float32)
    kept, _, _ = O.select_row(s, 1.0)
    assert kept == [1, 3, 2, 0]


def test_select_text_rows_dense_and_text_keys_forced():
    L = O.block_layout(2, 4, 4, 20, 8, (1, 2, 2))   # 32 video tokens -> 4 blocks; 20 text -> 3
    assert (L.nb_video, L.nb_text) == (4, 3)
    rng = np.random.default_rng(7)
    S = rng.dirichlet(np.ones(L.nb), size=L.nb).astype(np.float32)
    idx, cnt = O.select_topp(S, 0.5, L)
    for i in range(L.nb):
        kept = idx[i, :cnt[i]].tolist()
        if i >= 4:
            assert cnt[i] == L.nb
        else:
            assert {4, 5, 6} <= set(kept)
        order = O.sort_row(S[i]).tolist()
        assert kept == [j for j in order if j in kept]


# -------------------------------------------------------------------------------- drift

@pytest.mark.parametrize("c,expect", [(3.0, 2.0), (0.5, 0.5), (1.0, 0.0), (-1.0, 2.0)])
def test_drift_closed_form(c, expect):
    rng = np.random.default_rng(8)
    Qr = _bf16_round_f64(rng.standard_normal((40, 16)))
    Kr = _bf16_round_f64(rng.standard_normal((40, 16)))
    # Q = c * Q_ref (exact in bf16 for these c), K unchanged
    assert O.drift(c * Qr, Kr, Qr, Kr) == pytest.approx(expect, abs=1e-15)
    # the larger of the two changes is reported
    assert O.drift(Qr, c * Kr, Qr, Kr) == pytest.approx(expect, abs=1e-15)
    assert O.drift(c * Qr, 0.5 * c * Kr + 0.5 * Kr, Qr, Kr) == pytest.approx(
        max(abs(c - 1), abs(0.5 * c - 0.5)), abs=1e-15)


def test_refresh_is_strictly_above_tau():
    assert O.refresh_decision(0.05, 0.05, True) is False
    assert O.refresh_decision(0.0500001, 0.05, True) is True
    assert O.refresh_decision(0.0, 0.05, False) is True


# ---------------------------------------------------------------------------- attention

def _sdpa(Q, K, V, allowed=None):
    q, k, v = (torch.from_numpy(x)[None, None] for x in (Q, K, V))
    m = None if allowed is None else torch.from_numpy(allowed)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)[0, 0].numpy()


def _case(seed, T=2, H=5, W=6, text=7, B=8, tile=(1, 2, 4), d=16):
    L = O.block_layout(T, H, W, text, B, tile)
    n = T * H * W + text
    rng = np.random.default_rng(seed)
    Q = _bf16_round_f64(1.5 * rng.standard_normal((n, d)))
    K = _bf16_round_f64(1.5 * rng.standard_normal((n, d)))
    V = _bf16_round_f64(rng.standard_normal((n, d)))
    return L, Q, K, V


def test_attention_all_blocks_is_dense_attention():
    L, Q, K, V = _case(9)
    idx = np.tile(np.arange(L.nb, dtype=np.int32), (L.nb, 1))
    cnt = np.full(L.nb, L.nb, np.int32)
    got = O.sparse_attention_head(Q, K, V, idx, cnt, L)
    assert np.allclose(got, _sdpa(Q, K, V), rtol=1e-10, atol=1e-12)


def test_attention_any_mask_is_masked_dense_attention():
    L, Q, K, V = _case(10)
    rng = np.random.default_rng(11)
    idx = np.full((L.nb, L.nb), -1, np.int32)
    cnt = np.zeros(L.nb, np.int32)
    block_of = np.empty(len(Q), np.int64)
    for j in range(L.nb):
        block_of[L.rows(j)] = j
    allowed = np.zeros((len(Q), len(Q)), bool)
    for i in range(L.nb):
        k = int(rng.integers(1, L.nb + 1))
        sel = rng.permutation(L.nb)[:k]
        idx[i, :k] = sel
        cnt[i] = k
        allowed[np.ix_(L.rows(i), np.isin(block_of, sel).nonzero()[0])] = True
    got = O.sparse_attention_head(Q, K, V, idx, cnt, L)
    assert np.allclose(got, _sdpa(Q, K, V, allowed), rtol=1e-10, atol=1e-12)


def test_attention_constant_v_gives_constant_o():
    L, Q, K, V = _case(12)
    V[:] = 0.375
    idx = np.tile(np.arange(L.nb, dtype=np.int32), (L.nb, 1))
    cnt = np.array([1 + (i % L.nb) for i in range(L.nb)], np.int32)
    got = O.sparse_attention_head(Q, K, V, idx, cnt, L)
    assert np.allclose(got, 0.375, rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------- reuse run

def test_reuse_run_static_inputs_refresh_only_at_step_zero():
    walk = inputs.RandomWalk(2, 16, 2, 8, 8, 0, seed=3, sigma=0.0)
    L = O.block_layout(2, 8, 8, 0, 64)
    steps = []
    for _ in range(4):
        q, k, _ = walk.current()
        steps.append((q, k))
        walk.advance()
    out = O.reuse_run(steps, walk.V, L, [0.9, 0.9], 0.05, attend=False)
    assert out["refresh"] == [[True, True]] + [[False, False]] * 3
    assert all(d == 0.0 for row in out["drift"][1:] for d in row)


def test_reuse_run_refreshes_when_drift_exceeds_tau():
    L = O.block_layout(1, 8, 8, 0, 64)
    rng = np.random.default_rng(13)
    q0 = inputs.f32_to_bf16_bits(rng.standard_normal((1, 64, 16)).astype(np.float32))
    k0 = inputs.f32_to_bf16_bits(rng.standard_normal((1, 64, 16)).astype(np.float32))
    q2 = inputs.f32_to_bf16_bits(2.0 * O.bf16_to_f64(q0).astype(np.float32))   # drift 1.0
    V = k0.copy()
    out = O.reuse_run([(q0, k0), (q0, k0), (q2, k0), (q2, k0)], V, L, [0.9], 0.05)
    assert [r[0] for r in out["refresh"]] == [True, False, True, False]
    assert out["drift"][2][0] == pytest.approx(1.0, abs=1e-15)


# --------------------------------------------------------------------- retrieval accuracy

def _mass_case(T=2, H=8, W=12, text=20, B=16, tile=(1, 4, 4), d=8, seed=11):
    rng = np.random.default_rng(seed)
    L = O.block_layout(T, H, W, text, B, tile)
    N = T * H * W + text
    Q = _bf16_round_f64(rng.standard_normal((N, d)) * 1.5)
    K = _bf16_round_f64(rng.standard_normal((N, d)) * 1.5)
    return L, Q, K


def test_captured_mass_all_blocks_is_one():
    L, Q, K = _mass_case()
    idx = np.tile(np.arange(L.nb, dtype=np.int32), (L.nb, 1))
    cnt = np.full(L.nb, L.nb, np.int32)
    assert np.allclose(O.captured_mass(Q, K, idx, cnt, L), 1.0, atol=1e-12)


def test_captured_mass_equals_brute_force_softmax():
    # torch's softmax over the full logits, summed over the kept keys' columns
    L, Q, K = _mass_case()
    rng = np.random.default_rng(2)
    idx = np.full((L.nb, L.nb), -1, np.int32)
    cnt = rng.integers(1, L.nb + 1, L.nb).astype(np.int32)
    for i in range(L.nb):
        idx[i, :cnt[i]] = rng.permutation(L.nb)[:cnt[i]]
    got = O.captured_mass(Q, K, idx, cnt, L)
    P = torch.softmax(torch.from_numpy(Q @ K.T / math.sqrt(Q.shape[1])), dim=1).numpy()
    for i in range(L.nb):
        rows = L.rows(i)
        cols = np.concatenate([L.rows(int(j)) for j in idx[i, :cnt[i]]])
        assert got[i] == pytest.approx(P[np.ix_(rows, cols)].sum(axis=1).mean(), abs=1e-12)


def test_captured_mass_with_constant_keys_is_sum_of_park_scores():
    # keys constant within every block: PARK's score of block j is the exact mass of j, so the
    # captured mass is the sum of the kept blocks' PARK scores (and is additive over blocks)
    L, Q, K = _mass_case(text=0, B=16)
    rng = np.random.default_rng(4)
    for j in range(L.nb):
        K[L.rows(j)] = _bf16_round_f64(rng.standard_normal(K.shape[1]))
    P = O.score_park(Q, K, L)
    idx = np.full((L.nb, L.nb), -1, np.int32)
    cnt = np.zeros(L.nb, np.int32)
    for i in range(L.nb):
        keep = rng.permutation(L.nb)[:3]
        idx[i, :3] = keep
        cnt[i] = 3
    got = O.captured_mass(Q, K, idx, cnt, L)
    for i in range(L.nb):
        assert got[i] == pytest.approx(P[i, idx[i, :3]].sum(), abs=1e-12)


def test_captured_mass_grows_with_the_kept_set():
    L, Q, K = _mass_case()
    S = O.score_park(Q, K, L).astype(np.float32)
    prev = np.zeros(L.nb)
    for p in (0.3, 0.6, 0.9, 1.0):
        idx, cnt = O.select_topp(S, p, L)
        m = O.captured_mass(Q, K, idx, cnt, L)
        assert np.all(m >= prev - 1e-12) and np.all(m <= 1 + 1e-12)
        prev = m


# --------------------------------------------------------------------- one-shot schedule

def _walk_steps(n, shape=(2, 16, 2, 8, 16, 0, 32), tile=(1, 4, 8)):
    heads, d, T, H, W, text, B = shape
    walk = inputs.RandomWalk(heads, d, T, H, W, text, seed=5)
    steps = []
    for _ in range(n):
        q, k, v = walk.current()
        steps.append((q, k))
        walk.advance()
    return steps, v, O.block_layout(T, H, W, text, B, tile)


def test_rapid_dense_before_estimate_and_reuse_after():
    steps, V, L = _walk_steps(5)
    r = O.rapid_run(steps, V, L, [0.9, 0.8], estimate_step=2)
    assert r["kind"] == ["dense", "dense", "estimate", "reuse", "reuse"]
    # dense steps equal dense softmax attention (torch SDPA)
    for s in (0, 1):
        for h in range(V.shape[0]):
            q, k, v = (torch.from_numpy(O.bf16_to_f64(x[h])) for x in (steps[s][0], steps[s][1], V))
            ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
            assert np.allclose(r["O"][s][h], ref, atol=1e-10)
    # the estimate uses the scores of step 2's Q, K; later steps reuse that mask unchanged
    for h in range(V.shape[0]):
        S = O.score_meanpool(O.bf16_to_f64(steps[2][0][h]), O.bf16_to_f64(steps[2][1][h]), L).astype(np.float32)
        idx, cnt = O.select_topp(S, [0.9, 0.8][h], L)
        assert np.array_equal(r["cnt"][2][h], cnt) and np.array_equal(r["cnt"][4][h], cnt)
        assert np.array_equal(r["masks"][h][0], idx)


def test_rapid_turbo_stages_prune_the_cached_ranking():
    steps, V, L = _walk_steps(7)
    r = O.rapid_run(steps, V, L, [0.95, 0.95], estimate_step=0, stages=[(3, 0.8), (5, 0.6)], attend=False)
    assert r["kind"] == ["estimate", "reuse", "reuse", "stage", "reuse", "stage", "reuse"]
    for h in range(V.shape[0]):
        S = r["scores"][h]
        # each stage keeps a prefix of the same cached ranking, so kept sets only shrink
        for a, b in ((0, 3), (3, 5)):
            assert np.all(r["cnt"][b][h] <= r["cnt"][a][h])
        idx, cnt = O.select_topp(S, 0.6, L)
        assert np.array_equal(r["cnt"][6][h], cnt)
        for i in range(L.nb):
            order = O.sort_row(S[i])
            assert list(r["masks"][h][0][i, :cnt[i]]) == [int(j) for j in order[:cnt[i]]]


# ------------------------------------------------------------ cached dense correction

def test_recap_static_inputs_reproduce_dense_attention_every_step():
    # without drift the sparse output never changes, so sparse + cached correction is exactly
    # the dense attention of the refresh step, at every step
    steps, V, L = _walk_steps(1)
    steps = steps * 4
    r = O.recap_run(steps, V, L, [0.7, 0.7], tau=0.05)
    assert [list(f) for f in r["refresh"]] == [[True, True]] + [[False, False]] * 3
    for h in range(V.shape[0]):
        q, k, v = (torch.from_numpy(O.bf16_to_f64(x[h])) for x in (steps[0][0], steps[0][1], V))
        dense = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
        for s in range(4):
            assert np.allclose(r["O"][s][h], dense, atol=1e-12)
        assert np.abs(r["R"][h]).max() > 1e-3        # the correction is not trivial at p = 0.7


def test_recap_correction_is_zero_when_every_block_is_kept():
    steps, V, L = _walk_steps(3)
    r = O.recap_run(steps, V, L, [1.0, 1.0], tau=0.05)
    for h in range(V.shape[0]):
        assert np.abs(r["R"][h]).max() < 1e-12


def test_recap_between_refreshes_is_sparse_plus_cached_residual():
    steps, V, L = _walk_steps(4)
    r = O.recap_run(steps, V, L, [0.7, 0.7], tau=10.0)   # never refreshes after step 0
    for h in range(V.shape[0]):
        Q0, K0 = O.bf16_to_f64(steps[0][0][h]), O.bf16_to_f64(steps[0][1][h])
        Vh = O.bf16_to_f64(V[h])
        S = O.score_meanpool(Q0, K0, L).astype(np.float32)
        idx, cnt = O.select_topp(S, 0.7, L)
        R0 = O.dense_attention_head(Q0, K0, Vh, L) - O.sparse_attention_head(Q0, K0, Vh, idx, cnt, L)
        Q3, K3 = O.bf16_to_f64(steps[3][0][h]), O.bf16_to_f64(steps[3][1][h])
        expect = O.sparse_attention_head(Q3, K3, Vh, idx, cnt, L) + R0
        assert np.allclose(r["O"][3][h], expect, atol=1e-12)


# --------------------------------------------------------------- query-aware key blocks

def _cluster_case(seed=21, T=2, H=8, W=16, text=24, B=32, tile=(1, 4, 8), d=8):
    rng = np.random.default_rng(seed)
    L = O.block_layout(T, H, W, text, B, tile)
    N = T * H * W + text
    Q = _bf16_round_f64(rng.standard_normal((N, d)) * np.linspace(0.3, 2.0, d))
    K = _bf16_round_f64(rng.standard_normal((N, d)))
    return L, Q, K


def test_query_metric_is_mean_square_score_difference():
    L, Q, K = _cluster_case()
    M = O.query_metric(Q, L)
    k1, k2 = K[3], K[77]
    assert (k1 - k2) @ M @ (k1 - k2) == pytest.approx(np.mean((Q @ k1 - Q @ k2) ** 2), rel=1e-12)


def test_cluster_keys_is_kmeans_on_cholesky_transformed_keys():
    # a library routine on the transformed keys: sklearn's Lloyd k-means, same initial centres
    from sklearn.cluster import KMeans
    L, Q, K = _cluster_case()
    nv = L.nb_video
    Nv = int(L.counts[:nv].sum())
    Lc = np.linalg.cholesky(O.query_metric(Q, L))
    X = K[:Nv] @ Lc                                 # rows are (L^T k)^T
    init = np.stack([X[L.rows(j)].mean(axis=0) for j in range(nv)])
    for iters in (1, 2, 3):
        _, a = O.cluster_keys(Q, K, L, iters)
        km = KMeans(n_clusters=nv, init=init, n_init=1, max_iter=iters, tol=0.0, algorithm="lloyd").fit(X)
        # sklearn reports the labels of its last assignment after max_iter centre updates;
        # ours are the assignment of round `iters`: the same after one more assignment step
        C = km.cluster_centers_
        labels = np.argmin(((X[:, None, :] - C[None]) ** 2).sum(-1), axis=1)
        _, a_next = O.cluster_keys(Q, K, L, iters + 1)
        assert np.array_equal(a_next, labels), iters


def test_cluster_keys_invariant_to_query_scale_and_blocks_keep_sizes():
    L, Q, K = _cluster_case()
    kp, a = O.cluster_keys(Q, K, L, 2)
    kp2, a2 = O.cluster_keys(Q * 4.0, K, L, 2)
    assert np.array_equal(a, a2) and np.array_equal(kp, kp2)
    Nv = int(L.counts[:L.nb_video].sum())
    assert sorted(kp[:Nv].tolist()) == list(range(Nv))          # a permutation of the video keys
    assert np.array_equal(kp[Nv:], L.perm[Nv:])                 # padding and text unchanged
    KL = O.key_layout(L, kp)
    assert [len(KL.rows(j)) for j in range(L.nb)] == L.counts.tolist()
    # keys sorted by cluster: the cluster ids along the key order never decrease
    assert np.all(np.diff(a[kp[:Nv]]) >= 0)


def test_cluster_keys_keeps_block_constant_keys_in_their_blocks():
    # keys constant within each tile block and far apart across blocks: every key stays in its
    # own block's cluster, so the key blocks are the tile blocks (members in raster order)
    L, Q, K = _cluster_case(text=0)
    rng = np.random.default_rng(3)
    for j in range(L.nb):
        K[L.rows(j)] = rng.standard_normal(K.shape[1]) * 10.0
    kp, a = O.cluster_keys(Q, K, L, 3)
    for j in range(L.nb):
        assert set(a[L.rows(j)].tolist()) == {j}
        assert kp[j * L.B:j * L.B + L.counts[j]].tolist() == sorted(L.rows(j).tolist())


def test_keys_scored_alike_by_every_query_share_a_cluster():
    # queries confined to a 3-dimensional subspace: keys that differ only outside it receive
    # identical scores, are at distance 0 in the query metric, and must land in one cluster
    L, Q, K = _cluster_case(text=0)
    Q[:, 3:] = 0.0
    rng = np.random.default_rng(9)
    K[40, :] = K[17, :]
    K[40, 3:] = rng.standard_normal(K.shape[1] - 3) * 50.0
    _, a = O.cluster_keys(Q, K, L, 2)
    assert a[40] == a[17]
