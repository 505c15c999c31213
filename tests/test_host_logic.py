"""Host-side logic with no GPU: workspace sizes cover every buffer the kernels address, and
bench.py's roofline traffic is taken from the committed ncu figures (profiles/*.json) only
while the kernel sources they were measured on are unchanged."""
import importlib.util
import json
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
    rowoff = h * nb * 2 * 4                      # two log-sum-exps per score row (key-tile halves)
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
    assert bench._profiled_traffic("sparse_attention", "no_such_workload") is None
    assert bench._profiled_traffic("drift_check", "hunyuan_720p") is None
    # a copy of the tree with a profile written for its current kernel sources
    csrc = os.path.join("block_sparse_attention_query_b200", "csrc")
    os.makedirs(tmp_path / csrc)
    os.makedirs(tmp_path / "profiles")
    shutil.copy(os.path.join(ROOT, "bench.py"), tmp_path / "bench.py")
    for f in ("attention.cuh", "bsa_common.cuh"):
        shutil.copy(os.path.join(ROOT, csrc, f), tmp_path / csrc / f)
    copy = _load_bench(str(tmp_path))
    rec = {"workload": "hunyuan_720p", "traffic_bytes_per_launch": 123456789,
           "sources_sha256_16": copy._sources_hash(str(tmp_path))}
    with open(tmp_path / "profiles" / "sparse_attention_hunyuan_720p.json", "w") as f:
        json.dump(rec, f)
    assert copy._profiled_traffic("sparse_attention", "hunyuan_720p") == 123456789
    assert copy._profiled_traffic("sparse_attention", "wan13b_480p") is None
    # the traffic follows the kept blocks: a capture of mean-pooled masks says nothing of PARK's
    assert copy._profiled_traffic("sparse_attention", "hunyuan_720p", mode="park") is None
    # one byte more in a kernel source: the figure is stale and is not used
    with open(tmp_path / csrc / "attention.cuh", "a") as f:
        f.write("\n")
    assert copy._profiled_traffic("sparse_attention", "hunyuan_720p") is None
