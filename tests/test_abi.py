"""The C-ABI library on the host (no GPU): it loads, exports every symbol include/bsa.h
declares, plans sizes, reproduces the oracle's block layout exactly, and rejects bad
arguments before launching anything."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

from block_sparse_attention_query_b200 import build as bsa_build

bsa_build.build()
from block_sparse_attention_query_b200 import bsa  # noqa: E402
from block_sparse_attention_query_b200 import inputs  # noqa: E402
from oracle import bsa_oracle as O  # noqa: E402
from tests.conftest import GOLDEN, ROOT  # noqa: E402


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "bsa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^(?:const\s+)?(?:unsigned\s+)?(?:long\s+)*\w+\s*\*?\s*(bsa_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol():
    names = _declared_symbols()
    assert "bsa_sparse_attention" in names and "bsa_launch_count" in names and len(names) >= 12
    for n in names:
        assert hasattr(bsa.lib, n), n
        assert n in bsa.EXPORTS, n


def test_plan_reports_the_park_cluster_shape():
    # key blocks split over C CTAs of W (a multiple of 16, at most 160): (C - 1) * W < nb <= C * W
    for (T, H, W, text, heads), (C, cols) in {(21, 30, 52, 0, 12): (2, 128),      # nb 256
                                             (21, 45, 80, 0, 40): (4, 160),      # nb 591
                                             (33, 45, 80, 256, 24): (6, 160),    # nb 931
                                             (2, 8, 8, 0, 1): (1, 16)}.items():  # nb 1
        plan = bsa.bsa_plan(bsa.problem(heads, 128, T, H, W, text, 128, score_mode=bsa.BSA_SCORE_PARK))
        assert (plan.park_cluster, plan.park_cols) == (C, cols), (plan.nb, plan.park_cluster, plan.park_cols)
        assert (C - 1) * cols < plan.nb <= C * cols and cols % 16 == 0 and cols <= 160
    # above 8 x 160 key blocks the two-pass kernel runs
    plan = bsa.bsa_plan(bsa.problem(1, 64, 41, 64, 80, 0, 128, score_mode=bsa.BSA_SCORE_PARK))
    assert plan.nb > 1280 and plan.park_cluster == 0 and plan.park_cols == 0


def test_park_kernel_setting_is_checked_on_the_host():
    # a process-wide host setting: no CUDA call, so it runs without a GPU
    assert bsa.bsa_set_park_kernel(bsa.PARK_TWO_PASS) == 0
    assert bsa.bsa_set_park_kernel(2) == bsa.BSA_ERR_ARG
    assert bsa.bsa_set_park_kernel(-1) == bsa.BSA_ERR_ARG
    assert bsa.bsa_set_park_kernel(bsa.PARK_AUTO) == 0


def test_version_and_error_strings():
    assert "sm_100a" in bsa.bsa_version()
    for code in range(-7, 1):
        assert bsa.lib.bsa_error_string(code)
    assert bsa.lib.bsa_error_string(-99) == b"unknown status"


@pytest.mark.parametrize("name", inputs.WORKLOADS)
def test_plan_matches_oracle_layout(name):
    w = inputs.workload(name)
    prob = bsa.problem(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block)
    info = bsa.bsa_plan(prob)
    L = O.block_layout(w.T, w.H, w.W, w.text_tokens, w.block)
    assert (info.nb, info.nb_video, info.nb_text, info.npad) == (L.nb, L.nb_video, L.nb_text, L.npad)
    perm = np.array(bsa.bsa_block_layout(prob))
    assert np.array_equal(perm, L.perm)


def test_block_layout_golden_and_odd_tiles():
    with open(os.path.join(GOLDEN, "layout_small.json")) as f:
        cases = json.load(f)["cases"]
    # the library only accepts blocks of 64/128 tokens: scale the hand cases' grids up by
    # using tiles whose volume is the block size, and compare against the oracle
    for T, H, W, text, B, tile in [(3, 5, 7, 0, 64, (1, 8, 8)), (5, 9, 17, 40, 64, (4, 4, 4)),
                                   (7, 13, 11, 130, 128, (2, 8, 8)), (2, 3, 50, 5, 64, (1, 2, 32)),
                                   (9, 9, 9, 0, 128, (8, 4, 4))]:
        prob = bsa.problem(1, 64, T, H, W, text, B, tile)
        L = O.block_layout(T, H, W, text, B, tile)
        assert np.array_equal(np.array(bsa.bsa_block_layout(prob)), L.perm)
    assert len(cases) >= 3


def test_plan_rejects_bad_problems():
    good = bsa.problem(2, 64, 4, 16, 16, 0, 64)
    info = bsa.PlanInfo()
    assert bsa.lib.bsa_plan(ctypes.byref(good), ctypes.byref(info)) == bsa.BSA_OK
    bad = []
    p = bsa.problem(2, 96, 4, 16, 16, 0, 64); bad.append((p, bsa.BSA_ERR_UNSUPPORTED))
    p = bsa.problem(2, 64, 4, 16, 16, 0, 32); bad.append((p, bsa.BSA_ERR_UNSUPPORTED))
    p = bsa.problem(2, 64, 4, 16, 16, 0, 64); p.tokens += 1; bad.append((p, bsa.BSA_ERR_ARG))
    p = bsa.problem(0, 64, 4, 16, 16, 0, 64); bad.append((p, bsa.BSA_ERR_ARG))
    p = bsa.problem(2, 64, 4, 16, 16, 0, 64, tile=(2, 8, 8)); bad.append((p, bsa.BSA_ERR_ARG))
    p = bsa.problem(2, 64, 4, 16, 16, 0, 64, score_mode=7); bad.append((p, bsa.BSA_ERR_ARG))
    p = bsa.problem(2, 64, 64, 64, 64, 0, 64); bad.append((p, bsa.BSA_ERR_UNSUPPORTED))  # 4096 blocks
    for prob, code in bad:
        assert bsa.lib.bsa_plan(ctypes.byref(prob), ctypes.byref(info)) == code
    assert bsa.lib.bsa_plan(None, ctypes.byref(info)) == bsa.BSA_ERR_ARG
    assert bsa.lib.bsa_plan(ctypes.byref(good), None) == bsa.BSA_ERR_ARG


def test_calls_reject_bad_pointers_before_launch():
    # host-side validation only: no pointer is dereferenced and nothing is launched
    launches_before = bsa.bsa_launch_count()
    prob = bsa.problem(2, 64, 4, 16, 16, 0, 64)
    L = bsa.lib
    a = ctypes.c_void_p(4096)          # aligned, never dereferenced on these paths
    mis = ctypes.c_void_p(4096 + 2)
    pr = ctypes.byref(prob)
    assert L.bsa_score_blocks(pr, None, a, None, a, a, 1 << 20, None) == bsa.BSA_ERR_ARG
    assert L.bsa_score_blocks(pr, mis, a, None, a, a, 1 << 20, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_score_blocks(pr, a, a, None, a, a, 16, None) == bsa.BSA_ERR_WORKSPACE
    assert L.bsa_score_blocks(pr, a, a, None, a, None, 1 << 20, None) == bsa.BSA_ERR_WORKSPACE
    assert L.bsa_select_topp(pr, a, None, None, a, a, None) == bsa.BSA_ERR_ARG
    assert L.bsa_select_topp(pr, a, a, mis, a, a, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_drift_check(pr, a, a, a, a, ctypes.c_float(-1.0), 0, a, a, a, 1 << 20, None) == bsa.BSA_ERR_ARG
    assert L.bsa_drift_check(pr, a, a, a, a, ctypes.c_float(float("nan")), 0, a, a, a, 1 << 20, None) == bsa.BSA_ERR_ARG
    assert L.bsa_drift_check(pr, a, a, a, a, ctypes.c_float(0.05), 0, a, a, a, 8, None) == bsa.BSA_ERR_WORKSPACE
    assert L.bsa_drift_check(pr, a, a, a, None, ctypes.c_float(0.05), 0, a, a, a, 1 << 20, None) == bsa.BSA_ERR_ARG
    assert L.bsa_sparse_attention(pr, a, a, a, a, a, None, a, 1 << 20, None) == bsa.BSA_ERR_ARG
    assert L.bsa_sparse_attention(pr, a, a, a, None, a, a, a, 1 << 20, None) == bsa.BSA_ERR_ARG   # idx alone NULL
    assert L.bsa_sparse_attention(pr, a, a, a, a, None, a, a, 1 << 20, None) == bsa.BSA_ERR_ARG   # cnt alone NULL
    assert L.bsa_sparse_attention(pr, a, a, mis, a, a, a, a, 1 << 20, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_sparse_attention(pr, a, a, a, a, a, a, None, 1 << 20, None) == bsa.BSA_ERR_WORKSPACE
    text = bsa.problem(2, 64, 4, 16, 16, 64, 64)
    need = bsa.bsa_plan(text).attention_workspace_bytes
    assert need > 0
    assert L.bsa_sparse_attention(ctypes.byref(text), a, a, a, a, a, a, a, need - 1, None) == bsa.BSA_ERR_WORKSPACE
    # captured mass: the same host checks, and a workspace of plan.mass_workspace_bytes
    need = bsa.bsa_plan(prob).mass_workspace_bytes
    assert need > bsa.bsa_plan(prob).attention_workspace_bytes
    assert L.bsa_captured_mass(pr, a, a, a, a, None, a, need, None) == bsa.BSA_ERR_ARG
    assert L.bsa_captured_mass(pr, a, mis, a, a, a, a, need, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_captured_mass(pr, a, a, a, a, a, a, need - 1, None) == bsa.BSA_ERR_WORKSPACE
    # dense correction: pointers, alignment, workspace
    aw = bsa.bsa_plan(prob).attention_workspace_bytes
    assert L.bsa_dense_correction(pr, a, a, a, None, a, a, a, aw, None) == bsa.BSA_ERR_ARG
    assert L.bsa_dense_correction(pr, a, a, a, a, a, mis, a, aw, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_dense_correction(pr, a, a, a, a, a, a, a, aw - 1, None) == bsa.BSA_ERR_WORKSPACE
    # query-aware key blocks: iteration range, pointers, alignment, workspace; a misaligned key
    # table in the problem is refused by the calls that read it
    cw = bsa.bsa_plan(prob).cluster_workspace_bytes
    assert cw > 0
    assert L.bsa_cluster_keys(pr, a, a, 0, a, None, a, cw, None) == bsa.BSA_ERR_ARG
    assert L.bsa_cluster_keys(pr, a, a, 65, a, None, a, cw, None) == bsa.BSA_ERR_ARG
    assert L.bsa_cluster_keys(pr, a, a, 2, None, None, a, cw, None) == bsa.BSA_ERR_ARG
    assert L.bsa_cluster_keys(pr, a, a, 2, mis, None, a, cw, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_cluster_keys(pr, a, a, 2, a, mis, a, cw, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_cluster_keys(pr, a, a, 2, a, None, a, cw - 1, None) == bsa.BSA_ERR_WORKSPACE
    bad = bsa.problem(2, 64, 4, 16, 16, 0, 64)
    bad.key_table = 4096 + 4
    pb = ctypes.byref(bad)
    assert L.bsa_score_blocks(pb, a, a, None, a, a, 1 << 30, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_sparse_attention(pb, a, a, a, a, a, a, a, 1 << 30, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_captured_mass(pb, a, a, a, a, a, a, 1 << 30, None) == bsa.BSA_ERR_ALIGN
    # block means: a misaligned buffer is refused by both calls that use it
    bm = bsa.problem(2, 64, 4, 16, 16, 0, 64)
    bm.block_means = 4096 + 8
    pbm = ctypes.byref(bm)
    dw = bsa.bsa_plan(bm).drift_workspace_bytes
    assert L.bsa_drift_check(pbm, a, a, a, a, ctypes.c_float(0.05), 0, a, a, a, dw, None) == bsa.BSA_ERR_ALIGN
    assert L.bsa_score_blocks(pbm, a, a, None, a, a, 1 << 30, None) == bsa.BSA_ERR_ALIGN
    bm.block_means = 4096
    assert L.bsa_drift_check(pbm, a, a, a, a, ctypes.c_float(0.05), 0, a, a, a, dw - 1, None) == bsa.BSA_ERR_WORKSPACE
    assert bsa.bsa_launch_count() == launches_before     # none of the rejected calls launched
