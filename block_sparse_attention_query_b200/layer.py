"""Per-layer state for the block-sparse attention path across denoising steps, on top of the
C ABI. torch only allocates memory and provides the stream; every step of the path runs in
libbsa, with no host synchronisation.

`SparseAttentionLayer` — drift-gated mask reuse (HEART abstract, Temporal Mask Reuse; HASTE
abstract): each step runs

    drift_check (+ block means) -> score_blocks(refreshed heads) -> select_topp(refreshed heads)
    -> attention

`OneShotLayer` — one-shot estimate with cached reuse and optional Turbo stages (RAPID English
abstract): dense attention before the estimate step; at the estimate step every head is
scored once and its kept lists selected with p0; later steps reuse them; at each Turbo stage
the lists are selected anew from the cached scores with the stage's (smaller) p.
"""
from __future__ import annotations

import torch

from . import bsa


def _per_head(p, heads):
    return [float(p)] * heads if isinstance(p, (int, float)) else [float(v) for v in p]


class SparseAttentionLayer:
    def __init__(self, heads, d, T, H, W, text_tokens=0, block=128, p=0.9, tau=0.05,
                 score_mode=bsa.BSA_SCORE_MEANPOOL, tile=(0, 0, 0), device="cuda"):
        plan = bsa.bsa_plan(bsa.problem(heads, d, T, H, W, text_tokens, block, tile, score_mode))
        dev = torch.device(device)
        # the drift pass also writes the block means that the scores need (one read of Q, K)
        self.block_means = torch.empty(2, heads, plan.nb, d, dtype=torch.float32, device=dev)
        self.prob = bsa.problem(heads, d, T, H, W, text_tokens, block, tile, score_mode,
                                block_means=self.block_means)
        self.plan = bsa.bsa_plan(self.prob)
        self.heads, self.d, self.N = heads, d, self.prob.tokens
        nb = self.plan.nb
        self.nb = nb
        self.p = torch.tensor(_per_head(p, heads), dtype=torch.float32, device=dev)
        self.tau = float(tau)
        self.scores = torch.zeros(heads, nb, nb, dtype=torch.float32, device=dev)
        self.idx = torch.zeros(heads, nb, nb, dtype=torch.int32, device=dev)
        self.cnt = torch.zeros(heads, nb, dtype=torch.int32, device=dev)
        self.Q_ref = torch.zeros(heads, self.N, d, dtype=torch.bfloat16, device=dev)
        self.K_ref = torch.zeros(heads, self.N, d, dtype=torch.bfloat16, device=dev)
        self.drift = torch.zeros(heads, dtype=torch.float32, device=dev)
        self.refresh = torch.ones(heads, dtype=torch.int32, device=dev)
        self.ws_score = torch.empty(max(self.plan.score_workspace_bytes, 16), dtype=torch.uint8, device=dev)
        self.ws_drift = torch.empty(max(self.plan.drift_workspace_bytes, 16), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(max(self.plan.attention_workspace_bytes, 16), dtype=torch.uint8, device=dev)
        self.have_cache = False

    def step(self, Q, K, V, O, force_refresh=False):
        """One denoising step of this layer; O is written in place. Returns O."""
        force = force_refresh or not self.have_cache
        bsa.bsa_drift_check(self.prob, Q, K, self.Q_ref, self.K_ref, self.tau, force,
                            self.drift, self.refresh, self.ws_drift)
        bsa.bsa_score_blocks(self.prob, Q, K, self.refresh, self.scores, self.ws_score)
        bsa.bsa_select_topp(self.prob, self.scores, self.p, self.refresh, self.idx, self.cnt)
        bsa.bsa_sparse_attention(self.prob, Q, K, V, self.idx, self.cnt, O, self.ws_attn)
        self.have_cache = True
        return O


class OneShotLayer:
    """One-shot block-importance estimate, cached reuse and optional Turbo stages.

    estimate_step: the step (0-based) at which every head is scored, once; earlier steps
        attend densely. p: p0 per head (or one value) for the estimate's kept lists.
    stages: (step, p) pairs with steps after estimate_step, increasing: from that step on the
        kept lists are re-selected from the cached scores with that p (the same p for every
        head), with no re-scoring.
    """

    def __init__(self, heads, d, T, H, W, text_tokens=0, block=128, p=0.9, estimate_step=0, stages=(),
                 score_mode=bsa.BSA_SCORE_MEANPOOL, tile=(0, 0, 0), device="cuda"):
        self.prob = bsa.problem(heads, d, T, H, W, text_tokens, block, tile, score_mode)
        self.plan = bsa.bsa_plan(self.prob)
        self.heads, self.d, self.N = heads, d, self.prob.tokens
        nb = self.plan.nb
        self.nb = nb
        dev = torch.device(device)
        steps = [int(s) for s, _ in stages]
        if any(s <= estimate_step for s in steps) or steps != sorted(set(steps)):
            raise ValueError("stages must be increasing steps after the estimate step")
        self.estimate_step = int(estimate_step)
        self.p0 = torch.tensor(_per_head(p, heads), dtype=torch.float32, device=dev)
        self.stage_p = {int(s): torch.full((heads,), float(q), dtype=torch.float32, device=dev) for s, q in stages}
        self.scores = torch.zeros(heads, nb, nb, dtype=torch.float32, device=dev)
        self.idx = torch.zeros(heads, nb, nb, dtype=torch.int32, device=dev)
        self.cnt = torch.zeros(heads, nb, dtype=torch.int32, device=dev)
        self.ws_score = torch.empty(max(self.plan.score_workspace_bytes, 16), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(max(self.plan.attention_workspace_bytes, 16), dtype=torch.uint8, device=dev)
        self.step_index = 0
        self.kind = None

    def step(self, Q, K, V, O):
        """One denoising step; O is written in place. self.kind tells what the step did:
        'dense', 'estimate', 'stage' or 'reuse'. Returns O."""
        s = self.step_index
        if s < self.estimate_step:
            self.kind = "dense"
            bsa.bsa_sparse_attention(self.prob, Q, K, V, None, None, O, self.ws_attn)
        else:
            if s == self.estimate_step:
                self.kind = "estimate"
                bsa.bsa_score_blocks(self.prob, Q, K, None, self.scores, self.ws_score)
                bsa.bsa_select_topp(self.prob, self.scores, self.p0, None, self.idx, self.cnt)
            elif s in self.stage_p:
                self.kind = "stage"
                bsa.bsa_select_topp(self.prob, self.scores, self.stage_p[s], None, self.idx, self.cnt)
            else:
                self.kind = "reuse"
            bsa.bsa_sparse_attention(self.prob, Q, K, V, self.idx, self.cnt, O, self.ws_attn)
        self.step_index += 1
        return O


class CorrectedLayer(SparseAttentionLayer):
    """Drift-gated sparse attention with a cached dense correction (RECAP abstract: a cached
    dense refinement corrects what the sparse estimate omits; fresh statistics regulate the
    aging correction). Each step:

        drift_check -> score/select (refreshed heads) -> sparse attention
        -> dense_correction: refreshed heads get dense attention and a new correction
           R = dense - sparse; the others output sparse + their cached R

    The drift gate's refresh flags are the fresh statistics: a head refreshes its mask and its
    correction together, when its query-key drift since its last refresh exceeds tau.
    """

    def __init__(self, *args, **kwargs):
        super().__init__(*args, **kwargs)
        self.R = torch.zeros(self.heads, self.N, self.d, dtype=torch.bfloat16, device=self.p.device)

    def step(self, Q, K, V, O, force_refresh=False):
        super().step(Q, K, V, O, force_refresh)
        bsa.bsa_dense_correction(self.prob, Q, K, V, self.refresh, O, self.R, self.ws_attn)
        return O
