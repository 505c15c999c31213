"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1). The GPU path runs
independent replicas per rank with no collective on the data path; what crosses ranks is the
timing (max over ranks, the same collective at the same point on every rank) and the single
JSON line that only rank 0 prints."""
import importlib.util
import json
import os
import socket
import subprocess
import sys

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


def _rank_main(rank, ws, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    bench = _load_bench()
    # per-rank step times: rank r is slower by r ms; every rank must see the slowest
    got = bench.max_over_ranks(10.0 + rank, ws, torch.device("cpu"))
    got_e2e = bench.max_over_ranks(3.5 - rank, ws, torch.device("cpu"))
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": got, "max_e2e": got_e2e, "job": bench.job_value(got, ws)}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo(tmp_path):
    ws = 2
    mp.start_processes(_rank_main, args=(ws, _free_port(), str(tmp_path)), nprocs=ws, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(ws)]
    for r in res:
        assert r["max"] == 11.0 and r["max_e2e"] == 3.5
        assert r["job"] == pytest.approx(11.0 / ws)


def test_single_rank_helpers_need_no_process_group():
    bench = _load_bench()
    assert bench.max_over_ranks(7.25, 1, None) == 7.25
    assert bench.job_value(4.0, 1) == 4.0


def test_reference_arm_under_torchrun_prints_one_line():
    # the reference arm (the oracle on host cores) under torchrun: rank 0 alone runs and prints
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "1", "--warmup", "3", "--gpus", "2"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
