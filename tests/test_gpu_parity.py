"""CUDA path vs the CPU oracle on the same seeded inputs, call by call, through the C ABI.

Tolerances: attention max-abs <= 3e-2 and relative-L2 <= 1e-2 on the oracle's mask (bf16
inputs, float32 accumulation); scores within the float32 error bound of tests/parity.py
(score_bound), element by element; kept lists bit-exact except the rows the comparison rule
of tests/parity.py exempts (a cut within 1e-5 of p, or two blocks closer than their score
bounds), whose number every mask test prints and bounds."""
import math
import os

import numpy as np
import pytest
import torch

from block_sparse_attention_query_b200 import inputs
from oracle import bsa_oracle as O
from tests import parity as PT

pytestmark = pytest.mark.gpu

ATT_MAX_ABS = 3e-2
ATT_REL_L2 = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_query_b200 import build
    build.build()


def _bsa():
    from block_sparse_attention_query_b200 import bsa
    return bsa


class Case:
    """Inputs on host and device plus the problem descriptor."""

    def __init__(self, heads, d, T, H, W, text, B, p, mode="meanpool", seed=0, tile=(0, 0, 0)):
        bsa = _bsa()
        self.heads, self.d, self.B = heads, d, B
        big = heads * (T * H * W + text) > 4_000_000
        self.Qb, self.Kb, self.Vb = inputs.generate_qkv(heads, d, T, H, W, text, seed,
                                                        workers=min(os.cpu_count() or 1, 16) if big else 1)
        self.N = self.Qb.shape[1]
        self.p = np.array([p] * heads if np.isscalar(p) else p, dtype=np.float64)
        self.mode = mode
        smode = bsa.BSA_SCORE_PARK if mode == "park" else bsa.BSA_SCORE_MEANPOOL
        self.prob = bsa.problem(heads, d, T, H, W, text, B, tile, smode)
        self.plan = bsa.bsa_plan(self.prob)
        self.layout = O.block_layout(T, H, W, text, B, tile if tile != (0, 0, 0) else None)
        self.Q, self.K, self.V = (PT.to_dev_bf16(x) for x in (self.Qb, self.Kb, self.Vb))
        nb = self.plan.nb
        self.nb = nb
        self.p_dev = torch.tensor(self.p, dtype=torch.float32, device="cuda")

    def ws(self, nbytes):
        return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device="cuda")

    def gpu_scores(self):
        bsa = _bsa()
        S = torch.empty(self.heads, self.nb, self.nb, dtype=torch.float32, device="cuda")
        bsa.bsa_score_blocks(self.prob, self.Q, self.K, None, S, self.ws(self.plan.score_workspace_bytes))
        return S

    def gpu_select(self, S):
        bsa = _bsa()
        idx = torch.full((self.heads, self.nb, self.nb), -7, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(self.heads, self.nb, dtype=torch.int32, device="cuda")
        bsa.bsa_select_topp(self.prob, S, self.p_dev, None, idx, cnt)
        return idx, cnt

    def gpu_attention(self, idx, cnt):
        bsa = _bsa()
        Od = torch.full((self.heads, self.N, self.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        bsa.bsa_sparse_attention(self.prob, self.Q, self.K, self.V, idx, cnt, Od,
                                 self.ws(self.plan.attention_workspace_bytes))
        return Od

    def oracle_scores(self, h):
        return O.score_head(O.bf16_to_f64(self.Qb[h]), O.bf16_to_f64(self.Kb[h]), self.layout, self.mode)

    def oracle_scores_and_bound(self, h):
        """Exact scores (float64) of head h and the float32 kernel's error bound on them."""
        Qh, Kh = O.bf16_to_f64(self.Qb[h]), O.bf16_to_f64(self.Kb[h])
        S = O.score_head(Qh, Kh, self.layout, self.mode)
        return S, PT.score_bound(Qh, Kh, self.layout, self.mode, S if self.mode == "meanpool" else None)


def _check_scores(S_gpu_h, S, bnd, where):
    err = np.abs(S_gpu_h.astype(np.float64) - S)
    worst = float((err / bnd).max())
    print(f"\n[score bound] {where}: worst |error| / bound = {worst:.3f}")
    assert worst <= 1.0, (where, worst, float(err.max()))
    assert np.allclose(S_gpu_h.sum(axis=1), 1.0, atol=1e-5)
    return worst


def _report(tag, res):
    print(f"\n[mask parity] {tag}: rows={res['rows']} exact={res['exact']} window={res['window']} "
          f"tie={res['tie']} window_tie={res['window_tie']} mismatch={res['mismatch']}")


def _status_ok():
    assert _bsa().bsa_device_status() == 0


SMALL = {
    "tiny": dict(heads=2, d=64, T=4, H=16, W=16, text=0, B=64, p=0.9),
    # ragged last block with a single real token, d=128 with 64-token blocks
    "ragged_d128_b64": dict(heads=2, d=128, T=3, H=9, W=19, text=0, B=64, p=0.85),
    # text blocks (one partial), d=64 with 128-token blocks, odd grid
    "text_d64_b128": dict(heads=3, d=64, T=5, H=11, W=13, text=200, B=128, p=0.9),
    # d=128, B=128 with text, several tiles and a partial last video block
    "text_d128_b128": dict(heads=2, d=128, T=6, H=20, W=24, text=256, B=128, p=0.95),
    # a grid smaller than one block: nb = 1, one partial block (63 real tokens)
    "single_block": dict(heads=2, d=64, T=1, H=7, W=9, text=0, B=64, p=0.9),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("mode", ["meanpool", "park"])
def test_scores_match_oracle(name, mode):
    c = Case(**SMALL[name], mode=mode)
    S = c.gpu_scores().cpu().numpy()
    torch.cuda.synchronize()
    _status_ok()
    for h in range(c.heads):
        ref, bnd = c.oracle_scores_and_bound(h)
        _check_scores(S[h], ref, bnd, (name, mode, h))


# Enough 128-row items (heads x query tiles >= SM count) that the mean-pooled scores take the
# tensor-core path: several key tiles, a row count not a multiple of 4, text blocks.
MANY_HEADS = {
    "mh_d64_b64": dict(heads=150, d=64, T=5, H=32, W=52, text=0, B=64, p=0.9),
    "mh_d128_b128_text": dict(heads=150, d=128, T=3, H=16, W=40, text=130, B=128, p=0.9),
}


@pytest.mark.parametrize("name", list(MANY_HEADS))
def test_scores_tensor_core_path_match_oracle(name):
    c = Case(**MANY_HEADS[name], mode="meanpool")
    S = c.gpu_scores().cpu().numpy()
    torch.cuda.synchronize()
    _status_ok()
    for h in range(0, c.heads, 7):
        ref, bnd = c.oracle_scores_and_bound(h)
        _check_scores(S[h], ref, bnd, (name, h))


# PARK's one-pass kernel with the key blocks of a head split over a cluster of CTAs: nb above
# one CTA's share (160 key blocks), a partial last chunk, text blocks. The two-pass kernel runs on the same inputs, and a masked head stays untouched.
PARK_CLUSTER = {
    "c3_d128_b64_text": dict(heads=2, d=128, T=8, H=48, W=60, text=100, B=64, p=0.9),   # nb 362: 3 x 128
    "c2_d64_b64": dict(heads=2, d=64, T=9, H=32, W=60, text=0, B=64, p=0.9),             # nb 270: 2 x 144
}


@pytest.mark.parametrize("name", list(PARK_CLUSTER))
def test_park_cluster_kernel_matches_oracle_and_two_pass(name):
    bsa = _bsa()
    c = Case(**PARK_CLUSTER[name], mode="park")
    S1 = c.gpu_scores()
    try:
        assert bsa.bsa_set_park_kernel(bsa.PARK_TWO_PASS) == 0
        S2 = c.gpu_scores()
    finally:
        assert bsa.bsa_set_park_kernel(bsa.PARK_AUTO) == 0
    mask = torch.ones(c.heads, dtype=torch.int32, device="cuda")
    mask[1] = 0
    S3 = torch.full_like(S1, -1.0)
    bsa.bsa_score_blocks(c.prob, c.Q, c.K, mask, S3, c.ws(c.plan.score_workspace_bytes))
    torch.cuda.synchronize()
    _status_ok()
    assert (S3[1] == -1.0).all()
    assert torch.equal(S3[0], S1[0])          # same kernel, same inputs: the same bits
    S1, S2 = S1.cpu().numpy(), S2.cpu().numpy()
    for h in range(c.heads):
        ref, bnd = c.oracle_scores_and_bound(h)
        _check_scores(S1[h], ref, bnd, (name, "one-pass", h))
        _check_scores(S2[h], ref, bnd, (name, "two-pass", h))


@pytest.mark.parametrize("name", list(SMALL))
def test_select_on_oracle_scores_is_exact(name):
    # same float32 scores on both sides: only the cumulative-sum rounding may differ
    c = Case(**SMALL[name])
    S = np.stack([c.oracle_scores(h).astype(np.float32) for h in range(c.heads)])
    idx, cnt = c.gpu_select(torch.from_numpy(S).cuda())
    _status_ok()
    res = PT.compare_masks(idx.cpu().numpy(), cnt.cpu().numpy(), S, c.p, c.layout)
    _report(f"select on oracle scores, {name}", res)
    assert res["mismatch"] == 0 and res["tie"] == 0 and res["window_tie"] == 0, res
    assert res["window"] <= PT.exempt_limit(res["rows"]), res


@pytest.mark.parametrize("p", [1.0, 1e-6, 0.5])
def test_select_edge_p(p):
    c = Case(**{**SMALL["text_d64_b128"], "p": p})
    S = np.stack([c.oracle_scores(h).astype(np.float32) for h in range(c.heads)])
    idx, cnt = c.gpu_select(torch.from_numpy(S).cuda())
    cnt = cnt.cpu().numpy()
    if p == 1.0:
        assert (cnt == c.nb).all()
    if p == 1e-6:
        assert (cnt[:, :c.layout.nb_video] == 1 + c.layout.nb_text).all()
    res = PT.compare_masks(idx.cpu().numpy(), cnt, S, c.p, c.layout)
    assert res["mismatch"] == 0 and res["tie"] == 0 and res["window_tie"] == 0, res
    assert res["window"] <= PT.exempt_limit(res["rows"]), res


def test_select_hand_rows():
    # the hand-derived rows of tests/golden/topp_cases.json, padded into one head of 64 blocks
    import json, os
    from tests.conftest import GOLDEN
    bsa = _bsa()
    with open(os.path.join(GOLDEN, "topp_cases.json")) as f:
        cases = [c for c in json.load(f)["cases"] if not c["forced"]]
    prob = bsa.problem(1, 64, 1, 64, 64, 0, 64)       # 64 blocks, no text
    nb = bsa.bsa_plan(prob).nb
    for c in cases:
        row = np.zeros(nb, np.float32)
        row[:len(c["scores"])] = c["scores"]
        S = torch.from_numpy(np.tile(row, (nb, 1))[None]).cuda().contiguous()
        pd = torch.tensor([c["p"]], dtype=torch.float32, device="cuda")
        idx = torch.full((1, nb, nb), -7, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, nb, dtype=torch.int32, device="cuda")
        bsa.bsa_select_topp(prob, S, pd, None, idx, cnt)
        n = cnt[0, 0].item()
        got = idx[0, 0, :n].tolist()
        if c["p"] >= 1.0:
            assert got[:len(c["kept"])] == c["kept"]
        else:
            assert got == c["kept"], c["why"]


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("mode", ["meanpool", "park"])
def test_masks_end_to_end(name, mode):
    c = Case(**SMALL[name], mode=mode)
    idx, cnt = c.gpu_select(c.gpu_scores())
    _status_ok()
    sb = [c.oracle_scores_and_bound(h) for h in range(c.heads)]
    S = np.stack([x[0].astype(np.float32) for x in sb])
    res = PT.compare_masks(idx.cpu().numpy(), cnt.cpu().numpy(), S, c.p, c.layout,
                           bounds=[x[1] for x in sb])
    _report(f"end to end, {name}, {mode}", res)
    assert res["mismatch"] == 0, res
    assert res["exempt"] <= PT.exempt_limit(res["rows"]), res


def _oracle_mask(c):
    idxs, cnts = [], []
    for h in range(c.heads):
        S = c.oracle_scores(h).astype(np.float32)
        i_, c_ = O.select_topp(S, c.p[h], c.layout)
        idxs.append(i_)
        cnts.append(c_)
    return np.stack(idxs), np.stack(cnts)


@pytest.mark.parametrize("name", list(SMALL))
def test_attention_on_oracle_mask(name):
    c = Case(**SMALL[name])
    idx, cnt = _oracle_mask(c)
    Od = c.gpu_attention(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    _status_ok()
    got = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
    for h in range(c.heads):
        ref = O.sparse_attention_head(O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]),
                                      O.bf16_to_f64(c.Vb[h]), idx[h], cnt[h], c.layout)
        assert np.isfinite(got[h]).all()
        mx, rel = PT.attention_errors(got[h], ref, np.arange(c.N))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (h, mx, rel)


def test_attention_dense_mask_equals_dense_attention():
    # p = 1 keeps every block: the sparse kernel must reproduce dense softmax attention
    c = Case(**{**SMALL["text_d128_b128"], "p": 1.0})
    idx = np.tile(np.arange(c.nb, dtype=np.int32), (c.heads, c.nb, 1))
    cnt = np.full((c.heads, c.nb), c.nb, np.int32)
    Od = c.gpu_attention(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    _status_ok()
    got = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
    for h in range(c.heads):
        q, k, v = (torch.from_numpy(O.bf16_to_f64(x[h])) for x in (c.Qb, c.Kb, c.Vb))
        ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
        mx, rel = PT.attention_errors(got[h], ref, np.arange(c.N))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (h, mx, rel)


def test_attention_single_block_rows_and_constant_v():
    # cnt = 1 everywhere (each row attends its own block); V constant => O constant
    c = Case(**SMALL["ragged_d128_b64"])
    c.V = torch.full_like(c.V, 0.375)
    idx = np.tile(np.arange(c.nb, dtype=np.int32)[:, None], (c.heads, 1, c.nb))
    cnt = np.ones((c.heads, c.nb), np.int32)
    Od = c.gpu_attention(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    _status_ok()
    got = Od.float().cpu().numpy()
    assert np.all(got == 0.375)


def test_attention_bad_index_sets_device_error():
    # out-of-range kept index and count: the kernel's own checks flag them (no fault)
    bsa = _bsa()
    c = Case(**SMALL["tiny"])
    idx, cnt = _oracle_mask(c)
    idx[0, 3, 0] = c.nb + 5
    cnt[1, 2] = c.nb + 1
    c.gpu_attention(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    assert bsa.bsa_device_status() == bsa.BSA_ERR_DEVICE_ARG
    assert bsa.bsa_device_status() == 0   # cleared after reading


def test_drift_matches_oracle_and_snapshots():
    bsa = _bsa()
    c = Case(**SMALL["text_d64_b128"])
    rng = np.random.default_rng(5)
    scale = np.array([1.0, 1.03, 1.2])            # per-head drift 0, 0.03, 0.2 on Q
    Qref_bits = c.Qb.copy()
    Q2 = inputs.f32_to_bf16_bits((O.bf16_to_f64(c.Qb) * scale[:, None, None]).astype(np.float32))
    K2 = c.Kb.copy()
    K2[2, :10] = inputs.f32_to_bf16_bits(rng.standard_normal((10, c.d)).astype(np.float32))
    Qd, Kd = PT.to_dev_bf16(Q2), PT.to_dev_bf16(K2)
    Qr, Kr = PT.to_dev_bf16(Qref_bits), PT.to_dev_bf16(c.Kb)
    drift = torch.zeros(c.heads, dtype=torch.float32, device="cuda")
    refresh = torch.zeros(c.heads, dtype=torch.int32, device="cuda")
    bsa.bsa_drift_check(c.prob, Qd, Kd, Qr, Kr, 0.05, 0, drift, refresh, c.ws(c.plan.drift_workspace_bytes))
    _status_ok()
    for h in range(c.heads):
        ref = O.drift(O.bf16_to_f64(Q2[h]), O.bf16_to_f64(K2[h]), O.bf16_to_f64(Qref_bits[h]),
                      O.bf16_to_f64(c.Kb[h]))
        assert drift[h].item() == pytest.approx(ref, rel=1e-6, abs=1e-9)
        assert bool(refresh[h].item()) == (ref > 0.05)
    # refreshed heads now hold the new snapshot, the others the old one
    qr, kr = PT.from_dev_bf16(Qr), PT.from_dev_bf16(Kr)
    for h in range(c.heads):
        fresh = bool(refresh[h].item())
        assert np.array_equal(qr[h], Q2[h] if fresh else Qref_bits[h])
        assert np.array_equal(kr[h], K2[h] if fresh else c.Kb[h])
    # force_all refreshes everything and snapshots all heads
    bsa.bsa_drift_check(c.prob, Qd, Kd, Qr, Kr, 0.05, 1, drift, refresh, c.ws(c.plan.drift_workspace_bytes))
    assert refresh.cpu().tolist() == [1, 1, 1]
    assert np.array_equal(PT.from_dev_bf16(Qr), Q2) and np.array_equal(PT.from_dev_bf16(Kr), K2)
    # nothing changed since: zero drift, no refresh
    bsa.bsa_drift_check(c.prob, Qd, Kd, Qr, Kr, 0.05, 0, drift, refresh, c.ws(c.plan.drift_workspace_bytes))
    assert refresh.cpu().tolist() == [0, 0, 0]
    assert drift.cpu().tolist() == [0.0, 0.0, 0.0]


def test_reuse_run_tiny_50_steps():
    """Drift-gated mask reuse over 50 steps on the tiny shape: refresh decisions, kept lists
    and outputs follow the oracle step by step."""
    from block_sparse_attention_query_b200.layer import SparseAttentionLayer
    w = inputs.workload("tiny")
    walk = inputs.RandomWalk(w.heads, w.d, w.T, w.H, w.W, 0, seed=0)
    layer = SparseAttentionLayer(w.heads, w.d, w.T, w.H, w.W, 0, w.block, p=0.9, tau=0.05)
    L = O.block_layout(w.T, w.H, w.W, 0, w.block)
    Vd = PT.to_dev_bf16(walk.V)
    Od = torch.empty(w.heads, w.tokens, w.d, dtype=torch.bfloat16, device="cuda")
    steps = []
    gpu_flags, gpu_out = [], []
    for s in range(50):
        q, k, _ = walk.current()
        steps.append((q, k))
        layer.step(PT.to_dev_bf16(q), PT.to_dev_bf16(k), Vd, Od)
        gpu_flags.append(layer.refresh.cpu().tolist())
        if s in (0, 17, 49):
            gpu_out.append(PT.bf16_bits_f64(PT.from_dev_bf16(Od)))
        walk.advance()
    _status_ok()
    ref = O.reuse_run(steps, walk.V, L, [0.9] * w.heads, 0.05)
    flags_ref = [[int(x) for x in row] for row in ref["refresh"]]
    for s, (a, b, d) in enumerate(zip(gpu_flags, flags_ref, ref["drift"])):
        if a != b:  # only a drift within 1e-6 of tau may flip
            assert all(abs(x - 0.05) <= 1e-6 for x, u, v in zip(d, a, b) if u != v), (s, a, b, d)
    assert sum(map(sum, gpu_flags)) == sum(map(sum, flags_ref))
    assert sum(map(sum, flags_ref)) > w.heads       # the walk does trigger refreshes
    for o, s in zip(gpu_out, (0, 17, 49)):
        mx, rel = PT.attention_errors(o, ref["O"][s], np.arange(w.tokens))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (s, mx, rel)


# ------------------------------------------------------------------ full-size workloads

def _full_case(name, mode="meanpool"):
    w = inputs.workload(name)
    return Case(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block, list(w.p), mode=mode)


@pytest.mark.slow
@pytest.mark.parametrize("name,mode", [("wan13b_480p", "meanpool"), ("wan13b_480p", "park"),
                                       ("wan14b_720p", "meanpool"), ("wan14b_720p", "park"),
                                       ("hunyuan_720p", "meanpool"), ("hunyuan_720p", "park")])
def test_full_size_masks_and_sampled_attention(name, mode):
    c = _full_case(name, mode)
    S_gpu = c.gpu_scores()
    idx, cnt = c.gpu_select(S_gpu)
    _status_ok()
    heads = sorted(set([0, c.heads // 2, c.heads - 1]))
    S_gpu = S_gpu.cpu().numpy()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    rng = np.random.default_rng(0)
    S_or = np.zeros_like(S_gpu)
    bounds = {}
    for h in heads:
        ref, bounds[h] = c.oracle_scores_and_bound(h)
        S_or[h] = ref.astype(np.float32)
        _check_scores(S_gpu[h], ref, bounds[h], (name, mode, h))
    res = PT.compare_masks(idx_h, cnt_h, S_or, c.p, c.layout, heads=heads, bounds=bounds)
    _report(f"full size, {name}, {mode}, heads {heads}", res)
    assert res["mismatch"] == 0, res
    assert res["exempt"] <= PT.exempt_limit(res["rows"]), res
    # attention on the oracle's mask for sampled query blocks (text rows included)
    oi = {h: O.select_topp(S_or[h], c.p[h], c.layout) for h in heads}
    idx_o = idx.clone()
    cnt_o = cnt.clone()
    for h in heads:
        idx_o[h] = torch.from_numpy(oi[h][0]).cuda()
        cnt_o[h] = torch.from_numpy(oi[h][1]).cuda()
    Od = c.gpu_attention(idx_o, cnt_o)
    _status_ok()
    got = Od.float()
    for h in heads:
        qbl = sorted(set(rng.choice(c.layout.nb, 6, replace=False).tolist() + [c.layout.nb - 1]))
        ref = O.sparse_attention_head(O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]),
                                      O.bf16_to_f64(c.Vb[h]), oi[h][0], oi[h][1], c.layout, qblocks=qbl)
        rows = np.concatenate([c.layout.rows(i) for i in qbl])
        mx, rel = PT.attention_errors(got[h].cpu().double().numpy(), ref, rows)
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (h, mx, rel)
    # properties at full size on every row: finite, and each output is a convex
    # combination of V rows (bounded by the V range)
    vmax = float(np.abs(O.bf16_to_f64(c.Vb)).max())
    assert torch.isfinite(got).all() and float(got.abs().max()) <= vmax + 1e-2


@pytest.mark.parametrize("conc,p", [(50.0, 0.95), (0.3, 0.9), (5.0, 0.999)])
def test_select_flat_and_peaked_rows(conc, p):
    # flat rows need far more than the per-warp extraction cap and fall back to the full
    # sort; peaked rows stop early. Both must match the oracle's selection on the same
    # float32 scores (only the 1e-5 cumulative-mass window may differ).
    bsa = _bsa()
    L = O.block_layout(4, 64, 64, 0, 64)          # 256 blocks, no text
    heads = 3
    rng = np.random.default_rng(int(conc * 10) + int(p * 1000))
    S = rng.dirichlet(np.full(L.nb, conc), size=(heads, L.nb)).astype(np.float32)
    prob = bsa.problem(heads, 64, 4, 64, 64, 0, 64)
    pd = torch.full((heads,), p, dtype=torch.float32, device="cuda")
    idx = torch.full((heads, L.nb, L.nb), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(heads, L.nb, dtype=torch.int32, device="cuda")
    bsa.bsa_select_topp(prob, torch.from_numpy(S).cuda(), pd, None, idx, cnt)
    _status_ok()
    res = PT.compare_masks(idx.cpu().numpy(), cnt.cpu().numpy(), S, np.full(heads, p), L)
    assert res["mismatch"] == 0 and res["tie"] == 0 and res["window_tie"] == 0, res
    assert res["window"] <= PT.exempt_limit(res["rows"]), res
    if conc >= 5.0:
        assert cnt.cpu().numpy().mean() > 64       # the fallback path was exercised


# ------------------------------------------------------------------ retrieval accuracy
# Tolerance of the captured mass 2^(lse_kept - lse_all): each log-sum-exp carries the float32
# error of its logits (<= 4u * sum_c |q_c k_c| / sqrt(d), about 3e-5 for these inputs) and of
# its sum of up to N exponentials (relative (4 sqrt(n) + 32)u, about 1e-4 at n = 119k); the
# difference of two, through 2^x, stays under 2e-4 of a mass that is at most 1.
MASS_ATOL = 2e-4


def _gpu_mass(c, idx, cnt):
    bsa = _bsa()
    mass = torch.full((c.heads, c.nb), float("nan"), dtype=torch.float32, device="cuda")
    bsa.bsa_captured_mass(c.prob, c.Q, c.K, idx, cnt, mass, c.ws(c.plan.mass_workspace_bytes))
    _status_ok()
    return mass.cpu().numpy()


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("mode", ["meanpool", "park"])
def test_captured_mass_matches_oracle(name, mode):
    c = Case(**SMALL[name], mode=mode)
    idx, cnt = _oracle_mask(c)
    got = _gpu_mass(c, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    for h in range(c.heads):
        ref = O.captured_mass(O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]), idx[h], cnt[h], c.layout)
        err = np.abs(got[h] - ref)
        assert err.max() <= MASS_ATOL, (name, mode, h, float(err.max()))
    # text rows keep every block: all of the mass
    if c.layout.nb_text:
        assert np.allclose(got[:, c.layout.nb_video:], 1.0, atol=MASS_ATOL)


def test_captured_mass_all_blocks_is_one():
    c = Case(**SMALL["text_d128_b128"])
    idx = np.tile(np.arange(c.nb, dtype=np.int32), (c.heads, c.nb, 1))
    cnt = np.full((c.heads, c.nb), c.nb, np.int32)
    got = _gpu_mass(c, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    assert np.abs(got - 1.0).max() <= MASS_ATOL


@pytest.mark.slow
@pytest.mark.parametrize("name", ["wan13b_480p", "hunyuan_720p"])
def test_full_size_captured_mass_sampled(name):
    # the GPU's masks at full size; sampled query blocks (the last one, text rows included)
    # against the oracle's dense softmax
    c = _full_case(name)
    idx, cnt = c.gpu_select(c.gpu_scores())
    got = _gpu_mass(c, idx, cnt)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    rng = np.random.default_rng(1)
    for h in (0, c.heads - 1):
        qbl = sorted(set(rng.choice(c.layout.nb, 4, replace=False).tolist() + [c.layout.nb - 1]))
        ref = O.captured_mass(O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]), idx_h[h], cnt_h[h], c.layout,
                              qblocks=qbl)
        err = np.abs(got[h, qbl] - ref[qbl])
        assert err.max() <= MASS_ATOL, (name, h, float(err.max()))
    assert np.isfinite(got).all() and got.min() > 0 and got.max() <= 1 + MASS_ATOL


# ------------------------------------------------------------------ one-shot schedule

def test_one_shot_turbo_schedule_follows_oracle():
    """Dense steps, the one-shot estimate, reuse and two Turbo stages on the tiny random walk:
    what each step did, the kept lists and the outputs follow the oracle step by step."""
    from block_sparse_attention_query_b200.layer import OneShotLayer
    w = inputs.workload("tiny")
    walk = inputs.RandomWalk(w.heads, w.d, w.T, w.H, w.W, 0, seed=1)
    stages = [(5, 0.8), (8, 0.7)]
    layer = OneShotLayer(w.heads, w.d, w.T, w.H, w.W, 0, w.block, p=0.95, estimate_step=2, stages=stages)
    L = O.block_layout(w.T, w.H, w.W, 0, w.block)
    Vd = PT.to_dev_bf16(walk.V)
    Od = torch.empty(w.heads, w.tokens, w.d, dtype=torch.bfloat16, device="cuda")
    steps, kinds, cnts, outs = [], [], [], []
    for s in range(10):
        q, k, _ = walk.current()
        steps.append((q, k))
        layer.step(PT.to_dev_bf16(q), PT.to_dev_bf16(k), Vd, Od)
        kinds.append(layer.kind)
        cnts.append(layer.cnt.cpu().numpy().copy())
        outs.append(PT.bf16_bits_f64(PT.from_dev_bf16(Od)))
        walk.advance()
    _status_ok()
    ref = O.rapid_run(steps, walk.V, L, [0.95] * w.heads, estimate_step=2, stages=stages)
    assert kinds == ref["kind"]
    S = layer.scores.cpu().numpy()
    for h in range(w.heads):
        # the cached scores are those of the estimate step
        Qh, Kh = O.bf16_to_f64(steps[2][0][h]), O.bf16_to_f64(steps[2][1][h])
        Sx = O.score_meanpool(Qh, Kh, L)
        _check_scores(S[h], Sx, PT.score_bound(Qh, Kh, L, "meanpool", Sx), ("one-shot", h))
    for s in range(10):
        if ref["kind"][s] != "dense":
            assert all(np.array_equal(cnts[s][h], ref["cnt"][s][h]) for h in range(w.heads)), s
        mx, rel = PT.attention_errors(outs[s], ref["O"][s], np.arange(w.tokens))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (s, ref["kind"][s], mx, rel)
    # the stages pruned: fewer kept blocks at the end than at the estimate
    assert cnts[9].sum() < cnts[2].sum()


def test_dense_attention_without_lists():
    # idx = cnt = NULL keeps every block: dense softmax attention
    c = Case(**SMALL["text_d64_b128"])
    bsa = _bsa()
    Od = torch.full((c.heads, c.N, c.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    bsa.bsa_sparse_attention(c.prob, c.Q, c.K, c.V, None, None, Od, c.ws(c.plan.attention_workspace_bytes))
    _status_ok()
    got = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
    for h in range(c.heads):
        q, k, v = (torch.from_numpy(O.bf16_to_f64(x[h])) for x in (c.Qb, c.Kb, c.Vb))
        ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
        mx, rel = PT.attention_errors(got[h], ref, np.arange(c.N))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (h, mx, rel)


# --------------------------------------------------------------- cached dense correction

def test_dense_correction_follows_oracle():
    """Drift-gated sparse attention with a cached dense correction over 40 steps of the tiny
    random walk (refreshes at step 0 and again when the drift passes tau): refresh flags and
    outputs follow the oracle step by step. The correction is stored in bf16, so outputs are
    held to the attention tolerance."""
    from block_sparse_attention_query_b200.layer import CorrectedLayer
    w = inputs.workload("tiny")
    walk = inputs.RandomWalk(w.heads, w.d, w.T, w.H, w.W, 0, seed=2)
    layer = CorrectedLayer(w.heads, w.d, w.T, w.H, w.W, 0, w.block, p=0.8, tau=0.05)
    L = O.block_layout(w.T, w.H, w.W, 0, w.block)
    Vd = PT.to_dev_bf16(walk.V)
    Od = torch.empty(w.heads, w.tokens, w.d, dtype=torch.bfloat16, device="cuda")
    steps, flags, outs = [], [], {}
    check = (0, 1, 20, 39)
    for s in range(40):
        q, k, _ = walk.current()
        steps.append((q, k))
        layer.step(PT.to_dev_bf16(q), PT.to_dev_bf16(k), Vd, Od)
        flags.append(layer.refresh.cpu().tolist())
        if s in check:
            outs[s] = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
        walk.advance()
    _status_ok()
    ref = O.recap_run(steps, walk.V, L, [0.8] * w.heads, 0.05)
    flags_ref = [[int(x) for x in f] for f in ref["refresh"]]
    assert flags == flags_ref
    assert sum(map(sum, flags_ref)) > w.heads          # a second refresh happened
    for s in check:
        mx, rel = PT.attention_errors(outs[s], ref["O"][s], np.arange(w.tokens))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (s, mx, rel)
    # the cached correction itself (bf16) against the oracle's
    R = PT.bf16_bits_f64(PT.from_dev_bf16(layer.R))
    for h in range(w.heads):
        mx = float(np.abs(R[h] - ref["R"][h]).max())
        assert mx <= ATT_MAX_ABS, (h, mx)


def test_dense_correction_heads_masked():
    # refresh only head 1: head 0 gets O + R, head 1 the dense output and a new R
    c = Case(**SMALL["text_d64_b128"])
    bsa = _bsa()
    idx, cnt = _oracle_mask(c)
    Od = c.gpu_attention(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    sparse = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
    rng = np.random.default_rng(3)
    R0 = inputs.f32_to_bf16_bits((rng.standard_normal((c.heads, c.N, c.d)) * 0.01).astype(np.float32))
    Rd = PT.to_dev_bf16(R0)
    refresh = torch.tensor([0, 1, 0], dtype=torch.int32, device="cuda")
    bsa.bsa_dense_correction(c.prob, c.Q, c.K, c.V, refresh, Od, Rd, c.ws(c.plan.attention_workspace_bytes))
    _status_ok()
    out = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
    Rn = PT.bf16_bits_f64(PT.from_dev_bf16(Rd))
    R0f = O.bf16_to_f64(R0)
    for h in (0, 2):
        expect = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits((sparse[h] + R0f[h]).astype(np.float32)))
        assert np.array_equal(out[h], expect.astype(np.float64))
        assert np.array_equal(Rn[h], R0f[h])
    q, k, v = (torch.from_numpy(O.bf16_to_f64(x[1])) for x in (c.Qb, c.Kb, c.Vb))
    dense = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
    mx, rel = PT.attention_errors(out[1], dense, np.arange(c.N))
    assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2
    assert np.abs(Rn[1] - (out[1] - sparse[1])).max() <= 2 ** -8 * np.abs(out[1] - sparse[1]).max() + 1e-6


# ------------------------------------------------------------ query-aware key blocks
# The GPU's k-means rounds run in float32; a key may be assigned differently from the float64
# oracle only where the oracle's objective of the GPU's choice lies within 1e-4 of the terms'
# magnitude (|b_j| + 2 sum |k w_j|) of its own optimum: a float32 near-tie (such a flip can move
# a few other keys in later rounds, so at most 0.5% of the keys may differ).
CLUSTER_REL = 1e-4


def _gpu_cluster(c, iters):
    bsa = _bsa()
    table = torch.full((c.heads, c.nb * c.B), -9, dtype=torch.int32, device="cuda")
    nv = c.layout.nb_video
    Nv = int(c.layout.counts[:nv].sum())
    assign = torch.full((c.heads, Nv), -9, dtype=torch.int32, device="cuda")
    bsa.bsa_cluster_keys(c.prob, c.Q, c.K, iters, table, assign, c.ws(c.plan.cluster_workspace_bytes))
    _status_ok()
    return table, assign


def _check_clustering(c, h, table_h, assign_h, iters):
    L = c.layout
    kp, a, obj, scale = O.cluster_keys(O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]), L, iters, with_objective=True)
    Nv = len(a)
    # the table is the GPU's own assignment sorted by (cluster, raster index), then the tile
    # layout's padding and text slots: exactly
    assert np.array_equal(table_h[:Nv], np.lexsort((np.arange(Nv), assign_h)))
    assert np.array_equal(table_h[Nv:], L.perm[Nv:])
    diff = np.nonzero(assign_h != a)[0]
    u = np.arange(Nv)
    gap = obj[u, assign_h] - obj[u, a]
    near = gap <= CLUSTER_REL * scale[u, assign_h]
    assert np.all(near[diff]), (h, diff[~near[diff]][:5], gap[diff][:5])
    assert len(diff) <= max(2, Nv // 200), (h, len(diff))
    return len(diff), kp


@pytest.mark.parametrize("name", ["tiny", "text_d128_b128", "ragged_d128_b64"])
@pytest.mark.parametrize("iters", [1, 3])
def test_cluster_keys_matches_oracle(name, iters):
    c = Case(**SMALL[name])
    table, assign = _gpu_cluster(c, iters)
    table, assign = table.cpu().numpy(), assign.cpu().numpy()
    flips = [_check_clustering(c, h, table[h], assign[h], iters)[0] for h in range(c.heads)]
    print(f"\n[key clustering] {name}, {iters} rounds: assignments differing from the oracle {flips}")


@pytest.mark.parametrize("mode", ["park", "meanpool"])
def test_scores_and_attention_through_key_table(mode):
    # scores, masks and attention with the GPU's query-aware key blocks against the oracle on
    # the same key table
    bsa = _bsa()
    c = Case(**SMALL["text_d128_b128"], mode=mode)
    table, _ = _gpu_cluster(c, 2)
    smode = bsa.BSA_SCORE_PARK if mode == "park" else bsa.BSA_SCORE_MEANPOOL
    c.prob = bsa.problem(c.heads, c.d, 6, 20, 24, 256, c.B, score_mode=smode, key_table=table)
    S = c.gpu_scores()
    idx, cnt = c.gpu_select(S)
    _status_ok()
    S, idx_h, cnt_h, tab = S.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy(), table.cpu().numpy()
    S_or = np.zeros_like(S)
    bounds = []
    oracle_masks = []
    for h in range(c.heads):
        Qh, Kh = O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h])
        KL = O.key_layout(c.layout, tab[h])
        if mode == "park":
            ref = O.score_park_keys(Qh, Kh, c.layout, KL)
        else:
            ref = O._softmax_rows(O.pool_blocks(Qh, c.layout) @ O.pool_blocks(Kh, KL).T / math.sqrt(c.d))
        bnd = PT.score_bound(Qh, Kh, c.layout, mode, ref if mode == "meanpool" else None, klayout=KL)
        _check_scores(S[h], ref, bnd, ("key table", mode, h))
        S_or[h] = ref.astype(np.float32)
        bounds.append(bnd)
        oracle_masks.append(O.select_topp(S_or[h], c.p[h], c.layout))
    res = PT.compare_masks(idx_h, cnt_h, S_or, c.p, c.layout, bounds=bounds)
    _report(f"key table, {mode}", res)
    assert res["mismatch"] == 0 and res["exempt"] <= PT.exempt_limit(res["rows"]), res
    # attention on the oracle's mask, keys and values gathered through the table
    io = np.stack([m[0] for m in oracle_masks]); co = np.stack([m[1] for m in oracle_masks])
    Od = c.gpu_attention(torch.from_numpy(io).cuda(), torch.from_numpy(co).cuda())
    _status_ok()
    got = PT.bf16_bits_f64(PT.from_dev_bf16(Od))
    for h in range(c.heads):
        KL = O.key_layout(c.layout, tab[h])
        ref = O.sparse_attention_keys(O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]), O.bf16_to_f64(c.Vb[h]),
                                      io[h], co[h], c.layout, KL)
        mx, rel = PT.attention_errors(got[h], ref, np.arange(c.N))
        assert mx <= ATT_MAX_ABS and rel <= ATT_REL_L2, (h, mx, rel)


@pytest.mark.slow
def test_full_size_cluster_keys_sampled():
    # the 480p layer, 2 rounds: assignment near-tie rule on every key of two heads, the table
    # exact against the GPU's assignment
    c = _full_case("wan13b_480p", "park")
    table, assign = _gpu_cluster(c, 2)
    table, assign = table.cpu().numpy(), assign.cpu().numpy()
    for h in (0, c.heads - 1):
        n, _ = _check_clustering(c, h, table[h], assign[h], 2)
        print(f"\n[key clustering] wan13b_480p head {h}: {n} assignments differ from the oracle")


# ------------------------------------------------------ drift pass with the block means

@pytest.mark.parametrize("name", ["text_d64_b128", "ragged_d128_b64", "text_d128_b128"])
@pytest.mark.parametrize("force", [0, 1])
def test_drift_pass_writes_block_means(name, force):
    """bsa_problem.block_means set: the drift pass reads Q, K, Q_ref, K_ref block by block and
    also writes the block means. Drift, refresh flags and snapshots as without it (against the
    oracle), the means against the oracle's pooling (float32 sums of at most 128 bf16 values,
    bounded by 64 roundings of the mean absolute value), and the scores computed from them."""
    bsa = _bsa()
    c = Case(**SMALL[name])
    rng = np.random.default_rng(11)
    scale = np.linspace(1.0, 1.2, c.heads)
    Q2 = inputs.f32_to_bf16_bits((O.bf16_to_f64(c.Qb) * scale[:, None, None]).astype(np.float32))
    K2 = c.Kb.copy()
    K2[-1, :7] = inputs.f32_to_bf16_bits(rng.standard_normal((7, c.d)).astype(np.float32))
    means = torch.full((2, c.heads, c.nb, c.d), float("nan"), dtype=torch.float32, device="cuda")
    prob = bsa.problem(c.heads, c.d, *_grid(name), c.B, block_means=means)
    plan = bsa.bsa_plan(prob)
    Qd, Kd = PT.to_dev_bf16(Q2), PT.to_dev_bf16(K2)
    Qr, Kr = PT.to_dev_bf16(c.Qb), PT.to_dev_bf16(c.Kb)
    drift = torch.zeros(c.heads, dtype=torch.float32, device="cuda")
    refresh = torch.zeros(c.heads, dtype=torch.int32, device="cuda")
    bsa.bsa_drift_check(prob, Qd, Kd, Qr, Kr, 0.05, force, drift, refresh, c.ws(plan.drift_workspace_bytes))
    _status_ok()
    m = means.cpu().numpy()
    qr, kr = PT.from_dev_bf16(Qr), PT.from_dev_bf16(Kr)
    for h in range(c.heads):
        Qh, Kh = O.bf16_to_f64(Q2[h]), O.bf16_to_f64(K2[h])
        ref = O.drift(Qh, Kh, O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h]))
        assert drift[h].item() == pytest.approx(ref, rel=1e-6, abs=1e-9)
        fresh = bool(force) or ref > 0.05
        assert bool(refresh[h].item()) == fresh
        assert np.array_equal(qr[h], Q2[h] if fresh else c.Qb[h])
        assert np.array_equal(kr[h], K2[h] if fresh else c.Kb[h])
        for X, got in ((Qh, m[0, h]), (Kh, m[1, h])):
            exact = O.pool_blocks(X, c.layout)
            tol = 64 * PT.U32 * O.pool_blocks(np.abs(X), c.layout)
            assert np.all(np.abs(got - exact) <= tol), (h, float(np.abs(got - exact).max()))
    # the scores taken from these means equal those of a call that pools Q, K itself
    S1 = torch.empty(c.heads, c.nb, c.nb, dtype=torch.float32, device="cuda")
    bsa.bsa_score_blocks(prob, Qd, Kd, None, S1, c.ws(plan.score_workspace_bytes))
    S2 = torch.empty_like(S1)
    bsa.bsa_score_blocks(bsa.problem(c.heads, c.d, *_grid(name), c.B), Qd, Kd, None, S2,
                         c.ws(plan.score_workspace_bytes))
    _status_ok()
    for h in range(c.heads):
        Qh, Kh = O.bf16_to_f64(Q2[h]), O.bf16_to_f64(K2[h])
        ref = O.score_meanpool(Qh, Kh, c.layout)
        bnd = PT.score_bound(Qh, Kh, c.layout, "meanpool", ref)
        _check_scores(S1[h].cpu().numpy(), ref, bnd, ("block means", name, h))
        _check_scores(S2[h].cpu().numpy(), ref, bnd, ("pooled in the call", name, h))


def test_drift_block_means_through_key_table():
    """With a key table the drift pass pools K over the query-aware key blocks (and Q over the
    tile blocks); the scores taken from those means match the oracle on the same key layout."""
    bsa = _bsa()
    c = Case(**SMALL["text_d128_b128"])
    table, _ = _gpu_cluster(c, 2)
    means = torch.full((2, c.heads, c.nb, c.d), float("nan"), dtype=torch.float32, device="cuda")
    prob = bsa.problem(c.heads, c.d, 6, 20, 24, 256, c.B, key_table=table, block_means=means)
    plan = bsa.bsa_plan(prob)
    Qr, Kr = PT.to_dev_bf16(c.Qb), PT.to_dev_bf16(c.Kb)
    drift = torch.zeros(c.heads, dtype=torch.float32, device="cuda")
    refresh = torch.zeros(c.heads, dtype=torch.int32, device="cuda")
    bsa.bsa_drift_check(prob, c.Q, c.K, Qr, Kr, 0.05, 1, drift, refresh, c.ws(plan.drift_workspace_bytes))
    S = torch.empty(c.heads, c.nb, c.nb, dtype=torch.float32, device="cuda")
    bsa.bsa_score_blocks(prob, c.Q, c.K, None, S, c.ws(plan.score_workspace_bytes))
    _status_ok()
    m, tab, S = means.cpu().numpy(), table.cpu().numpy(), S.cpu().numpy()
    for h in range(c.heads):
        Qh, Kh = O.bf16_to_f64(c.Qb[h]), O.bf16_to_f64(c.Kb[h])
        KL = O.key_layout(c.layout, tab[h])
        for X, L, got in ((Qh, c.layout, m[0, h]), (Kh, KL, m[1, h])):
            exact = O.pool_blocks(X, L)
            tol = 64 * PT.U32 * O.pool_blocks(np.abs(X), L)
            assert np.all(np.abs(got - exact) <= tol), (h, float(np.abs(got - exact).max()))
        ref = O._softmax_rows(O.pool_blocks(Qh, c.layout) @ O.pool_blocks(Kh, KL).T / math.sqrt(c.d))
        bnd = PT.score_bound(Qh, Kh, c.layout, "meanpool", ref, klayout=KL)
        _check_scores(S[h], ref, bnd, ("block means, key table", h))


def _grid(name):
    s = SMALL[name]
    return s["T"], s["H"], s["W"], s["text"]
