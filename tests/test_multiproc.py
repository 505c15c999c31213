"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

With N GPUs the layer's heads are split into N contiguous ranges and every rank runs the
whole path on its own heads; nothing crosses ranks on the data path, only the timing (max over
ranks, the same collective at the same point on every rank) and, optionally, an all-gather of
the outputs. Here each rank draws only its own heads and runs the oracle on them; gathered, the
kept lists and outputs equal those of one process running every head, bit for bit."""
import importlib.util
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_mp", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


SHAPES = {"tiny": (2, 64, 4, 16, 16, 0, 64), "text": (3, 64, 3, 9, 19, 70, 64)}


def _oracle_heads(shape, h0, h1, p=0.9):
    from block_sparse_attention_query_b200 import inputs
    from oracle import bsa_oracle as O
    heads, d, T, H, W, text, B = shape
    Qb, Kb, Vb = inputs.generate_qkv(heads, d, T, H, W, text, seed=4, head_range=(h0, h1))
    L = O.block_layout(T, H, W, text, B)
    idx, cnt, out = [], [], []
    for h in range(h1 - h0):
        _, i_, c_, o_ = O.pipeline_head(Qb[h], Kb[h], Vb[h], L, p)
        idx.append(i_)
        cnt.append(c_)
        out.append(o_)
    return np.stack(idx), np.stack(cnt), np.stack(out)


def _rank_main(rank, ws, port, out_dir, shape_name):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    bench = _load_bench()
    shape = SHAPES[shape_name]
    h0, h1 = bench.head_range(shape[0], ws, rank)
    idx, cnt, out = _oracle_heads(shape, h0, h1)
    gathered = [None] * ws
    dist.all_gather_object(gathered, (h0, h1, idx, cnt, out))
    # per-rank step times: rank r is slower by r ms; every rank must see the slowest
    got = bench.max_over_ranks(10.0 + rank, ws, torch.device("cpu"))
    total = bench.sum_over_ranks(3 + rank, ws, torch.device("cpu"))
    if rank == 0:
        np.savez(os.path.join(out_dir, "gathered.npz"),
                 ranges=np.array([g[:2] for g in gathered]),
                 idx=np.concatenate([g[2] for g in gathered]), cnt=np.concatenate([g[3] for g in gathered]),
                 out=np.concatenate([g[4] for g in gathered]))
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": got, "sum": total, "range": [h0, h1]}, f)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("shape_name", list(SHAPES))
def test_head_split_equals_single_process(tmp_path, shape_name):
    ws = 2
    mp.start_processes(_rank_main, args=(ws, _free_port(), str(tmp_path), shape_name), nprocs=ws, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(ws)]
    for r in res:
        assert r["max"] == 11.0 and r["sum"] == 7.0
    shape = SHAPES[shape_name]
    g = np.load(tmp_path / "gathered.npz")
    # contiguous ranges that tile [0, heads)
    assert g["ranges"][0][0] == 0 and g["ranges"][-1][1] == shape[0]
    assert all(g["ranges"][k][1] == g["ranges"][k + 1][0] for k in range(ws - 1))
    idx, cnt, out = _oracle_heads(shape, 0, shape[0])
    assert np.array_equal(g["idx"], idx) and np.array_equal(g["cnt"], cnt)
    assert np.array_equal(g["out"], out, equal_nan=True)


def test_head_ranges():
    bench = _load_bench()
    for heads in (1, 2, 3, 12, 24, 40):
        for ws in (1, 2, 3, 4, 8):
            if ws > heads:
                continue
            rs = [bench.head_range(heads, ws, r) for r in range(ws)]
            assert rs[0][0] == 0 and rs[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    assert [bench.head_range(24, 8, r) for r in range(8)] == [(3 * r, 3 * r + 3) for r in range(8)]


def test_single_rank_helpers_need_no_process_group():
    bench = _load_bench()
    assert bench.max_over_ranks(7.25, 1, None) == 7.25
    assert bench.sum_over_ranks(7.25, 1, None) == 7.25


def test_reference_arm_under_torchrun_prints_one_line():
    # the reference arm (the oracle on host cores) under torchrun: rank 0 alone runs and prints
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "3", "--gpus", "2"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    # the steps it reports are the steps it ran: one head each
    assert d["steps"] == 2 and d["heads_timed_per_step"] == 1
    assert d["value"] == pytest.approx(d["ms_per_step"] * 2, rel=1e-3)
