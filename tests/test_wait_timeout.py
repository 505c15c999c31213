"""The bounded-wait timeout path of the attention kernel, on the GPU, without faulting it.

Every wait inside the library's kernels gives up after a cycle limit, raises BSA_ERR_TIMEOUT
in the device error word and lets every role of the CTA wind down (issued tensor-core work
and copies drained, TMEM freed), so that the context stays usable. This test uses the
test-only build libbsa_waittest.so (waits of about 10 ms instead of 2 s, plus a hook with
which CTA 0 withholds the arrival of its first query tile, a barrier phase that then never
completes) and checks that (1) a normal call succeeds and matches the oracle, (2) the call
with the withheld arrival returns within a fraction of a second and reports BSA_ERR_TIMEOUT,
(3) the next normal call succeeds and matches the oracle again."""
import ctypes
import time

import numpy as np
import pytest
import torch

from block_sparse_attention_query_b200 import inputs
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def waitlib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_query_b200 import build, bsa
    lib = ctypes.CDLL(build.build_wait_test())
    for name, (res, args) in bsa.EXPORTS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    lib.bsa_test_withhold_q_arrival.restype = ctypes.c_int
    lib.bsa_test_withhold_q_arrival.argtypes = [ctypes.c_int]
    return lib


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def test_withheld_arrival_times_out_and_the_next_call_recovers(waitlib):
    from block_sparse_attention_query_b200 import bsa
    w = inputs.workload("tiny")
    Qb, Kb, Vb = inputs.generate_qkv(w.heads, w.d, w.T, w.H, w.W, 0, seed=0)
    L = O.block_layout(w.T, w.H, w.W, 0, w.block)
    idx = np.zeros((w.heads, L.nb, L.nb), np.int32)
    cnt = np.zeros((w.heads, L.nb), np.int32)
    ref = []
    for h in range(w.heads):
        S = O.score_meanpool(O.bf16_to_f64(Qb[h]), O.bf16_to_f64(Kb[h]), L).astype(np.float32)
        idx[h], cnt[h] = O.select_topp(S, 0.9, L)
        ref.append(O.sparse_attention_head(O.bf16_to_f64(Qb[h]), O.bf16_to_f64(Kb[h]), O.bf16_to_f64(Vb[h]),
                                           idx[h], cnt[h], L))
    Q, K, V = _dev(Qb), _dev(Kb), _dev(Vb)
    idx_d, cnt_d = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    prob = bsa.problem(w.heads, w.d, w.T, w.H, w.W, 0, w.block)
    plan = bsa.bsa_plan(prob)
    ws = torch.empty(plan.attention_workspace_bytes, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        Od = torch.full((w.heads, w.tokens, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = waitlib.bsa_sparse_attention(ctypes.byref(prob), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                          idx_d.data_ptr(), cnt_d.data_ptr(), Od.data_ptr(), ws.data_ptr(),
                                          ws.numel(), stream)
        assert rc == bsa.BSA_OK
        return Od

    def matches(Od):
        got = Od.float().cpu().numpy()
        return all(np.abs(got[h] - ref[h]).max() <= 3e-2 for h in range(w.heads))

    assert waitlib.bsa_test_withhold_q_arrival(0) == bsa.BSA_OK
    assert waitlib.bsa_device_status(stream) == bsa.BSA_OK
    assert matches(call()) and waitlib.bsa_device_status(stream) == bsa.BSA_OK

    assert waitlib.bsa_test_withhold_q_arrival(1) == bsa.BSA_OK
    t0 = time.perf_counter()
    call()
    status = waitlib.bsa_device_status(stream)     # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert waitlib.bsa_test_withhold_q_arrival(0) == bsa.BSA_OK
    assert status == bsa.BSA_ERR_TIMEOUT
    assert elapsed < 2.0, elapsed                  # ~10 ms waits, not the product's 2 s
    assert waitlib.bsa_device_status(stream) == bsa.BSA_OK   # read once, then cleared

    # the context is intact: the same call works again, and so does the product library
    assert matches(call()) and waitlib.bsa_device_status(stream) == bsa.BSA_OK
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == bsa.BSA_OK
