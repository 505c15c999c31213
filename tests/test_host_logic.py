"""Host-side logic with no GPU: workspace sizes cover every buffer the kernels address, and
bench.py's roofline traffic is taken from the committed ncu summary only while the kernel
sources it was measured on are unchanged."""
import importlib.util
import os
import shutil

import pytest

from block_sparse_attention_query_b200 import build as bsa_build

bsa_build.build()
from block_sparse_attention_query_b200 import bsa  # noqa: E402
from block_sparse_attention_query_b200 import inputs  # noqa: E402
from tests.conftest import ROOT  # noqa: E402


def _up(x, m):
    return (x + m - 1) // m * m


@pytest.mark.parametrize("name", inputs.WORKLOADS)
def test_score_workspace_covers_every_buffer(name):
    w = inputs.workload(name)
    mp = bsa.bsa_plan(bsa.problem(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block, score_mode=bsa.BSA_SCORE_MEANPOOL))
    pk = bsa.bsa_plan(bsa.problem(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block, score_mode=bsa.BSA_SCORE_PARK))
    nb, d, h = mp.nb, w.d, w.heads
    pooled = 2 * h * nb * d * 4                  # q-bar, k-bar float32
    perm = nb * w.block * 4                      # block-slot table
    ksplit = h * 3 * _up(nb, 64) * d * 2         # hi/mid/lo bf16 of k-bar, key tiles of 64
    qsplit = h * 3 * _up(nb, 128) * d * 2        # hi/mid/lo bf16 of q-bar, query tiles of 128
    rowoff = h * nb * 4                          # one softmax offset per score row
    assert pk.score_workspace_bytes >= pooled + perm + ksplit
    assert mp.score_workspace_bytes >= pooled + perm + ksplit + qsplit + rowoff
    assert mp.score_workspace_bytes > pk.score_workspace_bytes
    # attention: block-slot table, plus text rows' float32 partial O and log-sum-exp
    assert mp.attention_workspace_bytes >= perm
    if w.text_tokens:
        assert mp.attention_workspace_bytes >= perm + mp.nb_text * h * 128 * d * 4


def _load_bench(root):
    spec = importlib.util.spec_from_file_location("bench_copy", os.path.join(root, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_profiled_traffic_only_for_matching_sources(tmp_path):
    bench = _load_bench(ROOT)
    t = bench._profiled_traffic("sparse_attention", "wan13b_480p")
    assert t is None or (isinstance(t, int) and t > 0)
    assert bench._profiled_traffic("sparse_attention", "no_such_workload") is None
    assert bench._profiled_traffic("drift_check", "wan13b_480p") is None
    # a copy of the tree whose kernel source differs by one byte gets no traffic figure
    csrc = os.path.join("block_sparse_attention_query_b200", "csrc")
    os.makedirs(tmp_path / csrc)
    shutil.copy(os.path.join(ROOT, "bench.py"), tmp_path / "bench.py")
    shutil.copytree(os.path.join(ROOT, "profiles"), tmp_path / "profiles")
    for f in ("attention.cuh", "bsa_common.cuh"):
        shutil.copy(os.path.join(ROOT, csrc, f), tmp_path / csrc / f)
    copy = _load_bench(str(tmp_path))
    assert copy._profiled_traffic("sparse_attention", "wan13b_480p") == t
    with open(tmp_path / csrc / "attention.cuh", "a") as f:
        f.write("\n")
    assert copy._profiled_traffic("sparse_attention", "wan13b_480p") is None
