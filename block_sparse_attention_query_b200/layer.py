"""Per-layer state for the drift-gated block-sparse attention path, on top of the C ABI.

`SparseAttentionLayer` owns the device buffers one attention layer keeps across denoising
steps (cached scores and kept-block lists, Q/K reference snapshots, workspaces) and runs one
step as four library calls on the current stream, with no host synchronisation:

    drift_check -> score_blocks(refreshed heads) -> select_topp(refreshed heads) -> attention

torch only allocates memory and provides the stream; every step of the path runs in libbsa.
"""
from __future__ import annotations

import torch

from . import bsa


class SparseAttentionLayer:
    def __init__(self, heads, d, T, H, W, text_tokens=0, block=128, p=0.9, tau=0.05,
                 score_mode=bsa.BSA_SCORE_MEANPOOL, tile=(0, 0, 0), device="cuda"):
        self.prob = bsa.problem(heads, d, T, H, W, text_tokens, block, tile, score_mode)
        self.plan = bsa.bsa_plan(self.prob)
        self.heads, self.d, self.N = heads, d, self.prob.tokens
        nb = self.plan.nb
        self.nb = nb
        dev = torch.device(device)
        ps = [float(p)] * heads if isinstance(p, (int, float)) else [float(v) for v in p]
        self.p = torch.tensor(ps, dtype=torch.float32, device=dev)
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
