"""bsa_drift_check_noalloc: the drift check for callers that cannot allocate device memory.

Some host programs (servers and real-time pipelines that reserve all device memory at
start-up, plugin interfaces that pass only inputs and outputs) cannot hand the library a
workspace. This entry point keeps its scratch in a static device array inside the library
instead. Here it is called through the C ABI and checked against the workspace entry point
bsa_drift_check on the same inputs, for two calls in a row of different sizes (the second
call must not see the first call's leftovers in the shared array), and its size limit is
checked. Collected last on purpose, so a failure here comes after every other test ran.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_query_b200 import inputs

pytestmark = pytest.mark.gpu

DRIFT_RTOL = 1e-6     # the same tolerance the drift parity test uses


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_query_b200 import build
    build.build()
    from block_sparse_attention_query_b200 import bsa as lib
    return lib


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _case(bsa, heads, d, T, H, W, text, block, seed, scales):
    Qb, Kb, _ = inputs.generate_qkv(heads, d, T, H, W, text, seed)
    q = inputs.bf16_bits_to_f32(Qb) * np.asarray(scales, np.float32)[:, None, None]
    Q2 = inputs.f32_to_bf16_bits(q)
    prob = bsa.problem(heads, d, T, H, W, text, block)
    return prob, Q2, Kb, Qb


def _run_both(bsa, prob, Q2, K2, Qref, force):
    heads = prob.heads
    plan = bsa.bsa_plan(prob)
    out = []
    for which in ("workspace", "noalloc"):
        Qr, Kr = _dev(Qref), _dev(K2)
        drift = torch.full((heads,), -1.0, dtype=torch.float32, device="cuda")
        refresh = torch.full((heads,), -1, dtype=torch.int32, device="cuda")
        if which == "workspace":
            ws = torch.empty(max(plan.drift_workspace_bytes, 16), dtype=torch.uint8, device="cuda")
            bsa.bsa_drift_check(prob, _dev(Q2), _dev(K2), Qr, Kr, 0.05, force, drift, refresh, ws)
        else:
            bsa.bsa_drift_check_noalloc(prob, _dev(Q2), _dev(K2), Qr, Kr, 0.05, force, drift, refresh)
        torch.cuda.synchronize()
        assert bsa.bsa_device_status() == 0
        out.append((drift.cpu().numpy(), refresh.cpu().numpy(),
                    Qr.view(torch.int16).cpu().numpy(), Kr.view(torch.int16).cpu().numpy()))
    return out


def test_noalloc_matches_workspace_entry_point_two_calls(bsa):
    # call 1: 3 heads with drifts 0, ~0.03 and ~0.2 on Q
    prob, Q2, K2, Qref = _case(bsa, 3, 64, 5, 11, 13, 200, 128, 1, [1.0, 1.03, 1.2])
    (d_ws, r_ws, q_ws, k_ws), (d_na, r_na, q_na, k_na) = _run_both(bsa, prob, Q2, K2, Qref, 0)
    np.testing.assert_allclose(d_na, d_ws, rtol=DRIFT_RTOL, atol=1e-9)
    assert np.array_equal(r_na, r_ws) and r_ws.tolist() == [0, 0, 1]
    assert np.array_equal(q_na, q_ws) and np.array_equal(k_na, k_ws)
    # call 2, right after, on a smaller problem with different drifts
    prob, Q2, K2, Qref = _case(bsa, 2, 128, 3, 9, 19, 0, 64, 2, [1.1, 1.0])
    (d_ws, r_ws, q_ws, k_ws), (d_na, r_na, q_na, k_na) = _run_both(bsa, prob, Q2, K2, Qref, 0)
    np.testing.assert_allclose(d_na, d_ws, rtol=DRIFT_RTOL, atol=1e-9)
    assert np.array_equal(r_na, r_ws) and r_ws.tolist() == [1, 0]
    assert np.array_equal(q_na, q_ws) and np.array_equal(k_na, k_ws)


def test_noalloc_rejects_problems_beyond_its_scratch(bsa):
    # 64 heads x (2048 blocks * 128 tokens * 128 / 16384 = 2048 chunks) * 4 doubles > 2 MiB
    prob = bsa.problem(64, 128, 64, 64, 64, 0, 128)
    drift = torch.zeros(64, dtype=torch.float32, device="cuda")
    refresh = torch.zeros(64, dtype=torch.int32, device="cuda")
    dummy = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_drift_check_noalloc(prob, dummy, dummy, dummy, dummy, 0.05, 0, drift, refresh)
    assert e.value.status == bsa.BSA_ERR_SCRATCH_LIMIT
