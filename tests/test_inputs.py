"""The seeded input generator: determinism, bf16 rounding and workload shapes. CPU only."""
import numpy as np
import torch

from block_sparse_attention_query_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 7,
                        np.array([1.00390625, 1.01171875, -2.0078125, 0.0, 65504.0], np.float32)])
    ours = inputs.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(inputs.bf16_bits_to_f32(ours),
                          torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generator_is_seeded_and_shaped():
    a = inputs.generate_qkv(2, 16, 2, 3, 4, 5, seed=7)
    b = inputs.generate_qkv(2, 16, 2, 3, 4, 5, seed=7)
    c = inputs.generate_qkv(2, 16, 2, 3, 4, 5, seed=8)
    for x, y in zip(a, b):
        assert x.shape == (2, 2 * 3 * 4 + 5, 16) and x.dtype == np.uint16
        assert np.array_equal(x, y)
    assert not np.array_equal(a[0], c[0])


def test_structured_qk_dominate_noise():
    Q, K, V = inputs.generate_qkv(1, 64, 4, 16, 16, 0, seed=0)
    q = inputs.bf16_bits_to_f32(Q[0]).astype(np.float64)
    # 2.0 * unit-variance RFF + 0.5 * N(0,1): per-channel variance about 4.25
    assert 3.5 < q.var() < 5.0
    v = inputs.bf16_bits_to_f32(V[0]).astype(np.float64)
    assert 0.9 < v.var() < 1.1


def test_workloads():
    w = inputs.workload("wan14b_720p")
    assert w.heads == 40 and len(w.p) == 40 and set(w.p) <= set(inputs.TOP_P_CHOICES)
    assert inputs.workload("hunyuan_720p").tokens == 119056
    assert inputs.workload("wan13b_480p").tokens == 32760


def test_head_ranges_draw_the_same_heads():
    # one GPU's share of the heads (or heads drawn in parallel) equals that slice of the layer
    full = inputs.generate_qkv(5, 16, 2, 3, 4, 5, seed=3)
    part = inputs.generate_qkv(5, 16, 2, 3, 4, 5, seed=3, head_range=(2, 4))
    par = inputs.generate_qkv(5, 16, 2, 3, 4, 5, seed=3, workers=3)
    for x, y, z in zip(full, part, par):
        assert np.array_equal(x[2:4], y)
        assert np.array_equal(x, z)
