"""Benchmark of the block-sparse 3D attention hot path on B200.

One step = one pass of the whole path over one attention layer of synthetic input resident in
HBM:
    drift check (forced refresh: every head re-scores) -> block scores -> top-p select
    -> block-sparse attention
on the HunyuanVideo-shaped 720p 5 s layer (24 heads, d=128, 33x45x80 grid + 256 text tokens,
128-token blocks, p=0.9; the largest layer of the five workloads) unless --workload says
otherwise. Its inputs (2.2 GB) are far larger than the 126 MB L2, so no step finds them in L2;
smaller layers rotate three input sets.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--mode meanpool|park] [--gather]

Prints one JSON line. Multi-GPU (torchrun, one rank per GPU): the layer's heads are split into
N contiguous ranges and rank r runs the same C-ABI calls on heads [r*H/N, (r+1)*H/N). Every
step of the path is per head, so the data path has no collective; --gather adds an NCCL
all-gather of O (for a caller that wants every head's output on every GPU). value = the
slowest rank's time per layer call (strong scaling: the layer is fixed and N GPUs share it).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms per sparse-attn call & % bf16 tensor peak (score+select+attend), 1 B200"
UNIT = "ms"
TAU = 0.05
L2_BYTES = 126 * 2 ** 20
DEFAULT_WORKLOAD = "hunyuan_720p"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def head_range(heads, ws, rank):
    """Contiguous heads [h0, h1) of rank `rank` when `heads` are split over `ws` ranks (sizes
    differ by at most one)."""
    return rank * heads // ws, (rank + 1) * heads // ws


def max_over_ranks(x, ws, device):
    """The slowest rank's value of a per-rank time (a collective over the process group when
    there is more than one rank; every rank calls it at the same point)."""
    if ws <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, ws, device):
    if ws <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- ours

def _sources_hash(root):
    src = b"".join(open(os.path.join(root, "block_sparse_attention_query_b200", "csrc", f), "rb").read()
                   for f in ("attention.cuh", "bsa_common.cuh"))
    return hashlib.sha256(src).hexdigest()[:16]


def _profiled_traffic(kernel, workload, root=None, mode="meanpool"):
    """DRAM bytes per launch of the attention kernel from the committed ncu figures
    (profiles/sparse_attention_<workload>.json), or None when the kernel sources changed since
    that capture, no capture exists for the workload, or the capture ran another scorer's masks
    (the traffic follows the kept blocks)."""
    if kernel != "sparse_attention":
        return None
    root = root or os.path.dirname(os.path.abspath(__file__))
    prof = os.path.join(root, "profiles", f"sparse_attention_{workload}.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        fields = json.load(f)
    if fields.get("workload") != workload or fields.get("sources_sha256_16") != _sources_hash(root):
        return None
    if fields.get("score_mode", "meanpool") != mode:
        return None
    return int(fields["traffic_bytes_per_launch"])


def _input_sets(w, h0, h1, n_sets, rank):
    from block_sparse_attention_query_b200 import inputs
    workers = max(1, min(os.cpu_count() or 1, 16, h1 - h0))
    return [inputs.generate_qkv(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, seed=s,
                                head_range=(h0, h1), workers=workers) for s in range(n_sets)]


def run_ours(args, ws, rank, local):
    import torch
    import torch.distributed as dist

    from block_sparse_attention_query_b200 import bsa, inputs
    from block_sparse_attention_query_b200.layer import SparseAttentionLayer

    w = inputs.workload(args.workload)
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads, p=tuple(w.p[:args.heads]))
    h0, h1 = head_range(w.heads, ws, rank)
    Hl = h1 - h0
    B, d, N = w.block, w.d, w.tokens
    elem = 2
    local_set_bytes = 3 * Hl * N * d * elem
    n_sets = 1 if local_set_bytes >= 4 * L2_BYTES else 3
    host_sets = _input_sets(w, h0, h1, n_sets, rank)   # drawn before the first CUDA call

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    mode = bsa.BSA_SCORE_PARK if args.mode == "park" else bsa.BSA_SCORE_MEANPOOL
    sets = [tuple(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in hs) for hs in host_sets]
    layer = SparseAttentionLayer(Hl, d, w.T, w.H, w.W, w.text_tokens, B, p=list(w.p[h0:h1]),
                                 tau=TAU, score_mode=mode, device=dev)
    O = torch.empty(Hl, N, d, dtype=torch.bfloat16, device=dev)
    O_all = torch.empty(ws, Hl, N, d, dtype=torch.bfloat16, device=dev) if (args.gather and ws > 1) else None
    stream = torch.cuda.current_stream(dev)
    prob, plan = layer.prob, layer.plan

    def step(k, ev=None):
        Q, K, V = sets[k % n_sets]
        if ev is not None:
            ev[0].record(stream)
        bsa.bsa_drift_check(prob, Q, K, layer.Q_ref, layer.K_ref, TAU, 1, layer.drift, layer.refresh, layer.ws_drift)
        if ev is not None:
            ev[1].record(stream)
        bsa.bsa_score_blocks(prob, Q, K, layer.refresh, layer.scores, layer.ws_score)
        if ev is not None:
            ev[2].record(stream)
        bsa.bsa_select_topp(prob, layer.scores, layer.p, layer.refresh, layer.idx, layer.cnt)
        if ev is not None:
            ev[3].record(stream)
        bsa.bsa_sparse_attention(prob, Q, K, V, layer.idx, layer.cnt, O, layer.ws_attn)
        if ev is not None:
            ev[4].record(stream)
        if O_all is not None:
            dist.all_gather_into_tensor(O_all.view(-1), O.view(-1))

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    st = bsa.bsa_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = bsa.bsa_launch_count()
    t0.record(stream)
    for k in range(args.steps):
        step(k, evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    launches = bsa.bsa_launch_count() - launches0
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t0.elapsed_time(t1)
    stage_ms = np.zeros(4)
    for e in evs:
        for s in range(4):
            stage_ms[s] += e[s].elapsed_time(e[s + 1])
    stage_ms /= args.steps
    total_ms = max_over_ranks(total_ms, ws, dev)
    stage_ms = np.array([max_over_ranks(x, ws, dev) for x in stage_ms])
    ms_step = total_ms / args.steps
    st = bsa.bsa_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")

    # work accounting from the masks the last step produced (all ranks' heads)
    cnt = layer.cnt.cpu().numpy().astype(np.int64)
    kept_pairs = int(sum_over_ranks(int(cnt.sum()), ws, dev))
    launches = int(sum_over_ranks(launches, ws, dev))
    H = w.heads
    att_flops = kept_pairs * 4.0 * B * B * d
    dense_flops = 4.0 * N * N * d * H
    bytes_qkvo = 4.0 * H * N * d * elem
    bytes_drift = 6.0 * H * N * d * elem              # read Q,K,Qref,Kref; write Qref,Kref (the same pass
                                                      # writes the block means the scores use)
    bytes_score = 4.0 * H * plan.nb * plan.nb         # the score matrix written (Q, K are not re-read)
    hbm, bf16_peak, bf16_sus, peak_src = _peaks()
    # per-GPU rates: each GPU does 1/ws of the work in the (slowest rank's) stage time
    per_gpu = 1.0 / ws

    stages = {}
    names = ["drift_check", "score_blocks", "select_topp", "sparse_attention"]
    for s, n in enumerate(names):
        stages[n] = {"ms": round(float(stage_ms[s]), 5), "share": round(float(stage_ms[s] / stage_ms.sum()), 4)}
    att_s = stage_ms[3] * 1e-3
    stages["sparse_attention"].update({
        "tflops_actual": round(att_flops / att_s / 1e12, 2),
        "tflops_dense_equiv": round(dense_flops / att_s / 1e12, 2),
        "frac_bf16_peak": round(att_flops * per_gpu / att_s / 1e12 / bf16_peak, 4),
        "hbm_gbs_compulsory": round(bytes_qkvo / att_s / 1e9, 1),
        "frac_hbm": round(bytes_qkvo * per_gpu / att_s / 1e9 / hbm, 4)})
    stages["drift_check"].update({"gbs": round(bytes_drift / (stage_ms[0] * 1e-3) / 1e9, 1),
                                  "frac_hbm": round(bytes_drift * per_gpu / (stage_ms[0] * 1e-3) / 1e9 / hbm, 4)})
    stages["drift_check"]["note"] = "one pass over Q, K, Q_ref, K_ref; also writes the block means of Q and K"
    stages["score_blocks"].update({"note": "block means from the drift pass; Q, K not read again",
                                   "score_matrix_gbs": round(bytes_score / (stage_ms[1] * 1e-3) / 1e9, 1)})
    # PARK: every query against every pooled key, three bf16 parts of the pooled keys, one pass
    park_flops = 3 * 2.0 * N * plan.nb * d * H if args.mode == "park" else 0.0
    if park_flops:
        sc_s = stage_ms[1] * 1e-3
        stages["score_blocks"].update({
            "note": "PARK, one pass: Q x (hi + mid + lo parts of the pooled keys); products issued = 3 x 2*N*nb*d",
            "tflops_issued": round(park_flops / sc_s / 1e12, 2),
            "frac_bf16_peak_issued": round(park_flops * per_gpu / sc_s / 1e12 / bf16_peak, 4)})

    # dominant kernel roofline (per GPU)
    dom = names[int(np.argmax(stage_ms))]
    if dom == "sparse_attention":
        t_tensor = att_flops / (bf16_peak * 1e12)
        t_hbm = bytes_qkvo / (hbm * 1e9)
        if t_tensor >= t_hbm:
            ach = att_flops * per_gpu / att_s / 1e12
            roof = {"bound": "tensor", "achieved": round(ach, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                    "frac": round(ach / bf16_peak, 4)}
        else:
            ach = bytes_qkvo * per_gpu / att_s / 1e9
            roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(ach / hbm, 4)}
    elif dom == "score_blocks" and park_flops:
        ach = park_flops * per_gpu / (stage_ms[1] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": round(ach / bf16_peak, 4)}
    else:
        b = bytes_drift if dom == "drift_check" else bytes_score
        ach = b * per_gpu / (stage_ms[names.index(dom)] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4)}
    traffic = args.traffic if args.traffic is not None else (_profiled_traffic(dom, w.name, mode=args.mode) if ws == 1 and not args.heads else None)
    roof.update({"kernel": dom,
                 "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured" else peak_src,
                 "traffic": traffic, "traffic_unit": "DRAM bytes per launch (ncu)",
                 "algorithmic_bytes": int((bytes_qkvo if dom == "sparse_attention" else
                                           bytes_drift if dom == "drift_check" else bytes_score) * per_gpu)})
    if dom == "sparse_attention":
        roof["algorithmic_flops"] = int(att_flops * per_gpu)
    elif dom == "score_blocks" and park_flops:
        roof["algorithmic_flops"] = int(park_flops * per_gpu)

    # end to end through the public API: every step copies its Q, K, V in from pinned host
    # memory and its O back out. The copies run on their own streams, so step k's output copy
    # and step k+1's input copy (opposite directions of the link) overlap step k's compute;
    # the inputs and O are double-buffered on the device.
    e2e = None
    if not args.no_e2e:
        hQ, hK, hV = (torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in sets[0])
        for hx, dx in zip((hQ, hK, hV), sets[0]):
            hx.copy_(dx)
        hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        bufs = [tuple(torch.empty_like(x) for x in sets[0]) for _ in range(2)]
        Obufs = [torch.empty_like(O) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(k):
            b = k & 1
            Qd, Kd, Vd = bufs[b]
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(ev_done[b])           # step k-2 has finished reading buffer b
                Qd.copy_(hQ, non_blocking=True); Kd.copy_(hK, non_blocking=True); Vd.copy_(hV, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if used[b]:
                stream.wait_event(ev_out[b])              # step k-2's output has left O buffer b
            layer.step(Qd, Kd, Vd, Obufs[b], force_refresh=True)
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                hO.copy_(Obufs[b], non_blocking=True)
                ev_out[b].record(s_out)
            used[b] = True

        e2e_steps = max(3, min(args.steps, 20))
        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_event(a)
        for k in range(2, 2 + e2e_steps):
            e2e_step(k)
        s_out.wait_event(ev_out[(1 + e2e_steps) & 1])
        b.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, ws, dev)
        e2e = {"value": round(e2e_ms, 4), "unit": UNIT,
               "h2d_bytes_per_step": int(3 * H * N * d * elem), "d2h_bytes_per_step": int(H * N * d * elem),
               "overlap": "input copies, compute and output copies of consecutive steps on three streams"}

    retrieval = None if args.no_retrieval else retrieval_accuracy(w, h0, h1, sets[0], dev, ws)

    line = {
        "metric": METRIC, "value": round(ms_step, 5), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded RFF-structured Q/K, Gaussian V; no model weights)",
        "config": {"workload": w.name + (f" (first {w.heads} heads)" if args.heads else ""), "heads": H, "d": d, "grid": [w.T, w.H, w.W],
                   "text_tokens": w.text_tokens, "tokens": N, "block": B, "blocks": plan.nb,
                   "top_p": sorted(set(float(x) for x in w.p)), "scorer": args.mode,
                   "parallelism": (f"heads split over {ws} GPUs, {Hl} per GPU, no data-path collective"
                                   + (", all-gather of O" if O_all is not None else "")) if ws > 1 else "single GPU",
                   "l2": (f"{n_sets} rotating input sets of {local_set_bytes / 1e6:.0f} MB per GPU "
                          f"(> 126 MB L2); no flush"),
                   "step": "drift_check(force) + score_blocks + select_topp + sparse_attention"},
        "call_ms_score_select_attend": round(float(stage_ms[1:].sum()), 5),
        "pct_bf16_peak_call": round(100.0 * att_flops * per_gpu / (ms_step * 1e-3) / 1e12 / bf16_peak, 3),
        "kept_blocks_per_row": round(kept_pairs / (H * plan.nb), 3),
        "kept_density": round(kept_pairs / (H * plan.nb * plan.nb), 5),
        "tflops_actual_call": round(att_flops / (ms_step * 1e-3) / 1e12, 2),
        "tflops_dense_equiv_call": round(dense_flops / (ms_step * 1e-3) / 1e12, 2),
        "stages": stages, "roofline": roof, "e2e": e2e, "retrieval": retrieval,
        "gpu_launches": launches, "gpu_launches_per_step": round(launches / args.steps / ws, 2),
        "clocks": clocks,
    }
    return line, (w, host_sets[0] if (rank == 0 and ws == 1) else None)


def retrieval_accuracy(w, h0, h1, qkv, dev, ws):
    """Retrieval accuracy of both scorers on this rank's heads (outside the timed region): the
    captured mass of their top-p masks (the share of each query's exact attention that the
    kept blocks hold), averaged over all query blocks of all heads, and their kept density."""
    import torch

    from block_sparse_attention_query_b200 import bsa
    Q, K, _ = qkv
    Hl = h1 - h0
    p = torch.tensor(list(w.p[h0:h1]), dtype=torch.float32, device=dev)
    out = {}
    # query-aware key blocks (PARK's key side): two k-means rounds, timed with CUDA events
    base = bsa.problem(Hl, w.d, w.T, w.H, w.W, w.text_tokens, w.block, score_mode=bsa.BSA_SCORE_PARK)
    bplan = bsa.bsa_plan(base)
    table = torch.empty(Hl, bplan.npad, dtype=torch.int32, device=dev)
    cws = torch.empty(bplan.cluster_workspace_bytes, dtype=torch.uint8, device=dev)
    bsa.bsa_cluster_keys(base, Q, K, 2, table, None, cws)            # warm-up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    bsa.bsa_cluster_keys(base, Q, K, 2, table, None, cws)
    e1.record()
    torch.cuda.synchronize()
    cluster_ms = max_over_ranks(e0.elapsed_time(e1), ws, dev)
    del cws
    for name, mode, ktab in (("meanpool", bsa.BSA_SCORE_MEANPOOL, None), ("park", bsa.BSA_SCORE_PARK, None),
                             ("park_query_aware_key_blocks", bsa.BSA_SCORE_PARK, table)):
        prob = bsa.problem(Hl, w.d, w.T, w.H, w.W, w.text_tokens, w.block, score_mode=mode, key_table=ktab)
        plan = bsa.bsa_plan(prob)
        nb = plan.nb
        S = torch.empty(Hl, nb, nb, dtype=torch.float32, device=dev)
        idx = torch.empty(Hl, nb, nb, dtype=torch.int32, device=dev)
        cnt = torch.empty(Hl, nb, dtype=torch.int32, device=dev)
        mass = torch.empty(Hl, nb, dtype=torch.float32, device=dev)
        bsa.bsa_score_blocks(prob, Q, K, None, S, torch.empty(plan.score_workspace_bytes, dtype=torch.uint8, device=dev))
        bsa.bsa_select_topp(prob, S, p, None, idx, cnt)
        wsm = torch.empty(plan.mass_workspace_bytes, dtype=torch.uint8, device=dev)
        bsa.bsa_captured_mass(prob, Q, K, idx, cnt, mass, wsm)
        del wsm
        torch.cuda.synchronize()
        st = bsa.bsa_device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} in the retrieval measurement")
        vid = mass[:, :plan.nb_video].double()
        tot = sum_over_ranks(float(vid.sum()), ws, dev)
        n = sum_over_ranks(float(vid.numel()), ws, dev)
        kept = sum_over_ranks(float(cnt[:, :plan.nb_video].double().sum()), ws, dev)
        mn = float(vid.min()) if ws == 1 else None
        out[name] = {"captured_mass_mean": round(tot / n, 5), "kept_blocks_per_video_row": round(kept / n, 3)}
        if mn is not None:
            out[name]["captured_mass_min_block"] = round(mn, 5)
    out["park_query_aware_key_blocks"]["cluster_ms"] = round(cluster_ms, 3)
    out["park_query_aware_key_blocks"]["cluster_rounds"] = 2
    out["definition"] = ("mean over video query blocks of the share of each query's exact softmax mass held by "
                         "its top-p kept blocks (bsa_captured_mass); park_query_aware_key_blocks: PARK scores "
                         "over the key blocks of bsa_cluster_keys")
    return out


# ------------------------------------------------------------------------- oracle

def oracle_head_ms(w, Qb, Kb, Vb, mode, h_local, h_global):
    """One head's drift + score + select + attention through the oracle; returns ms."""
    from oracle import bsa_oracle as O
    L = O.block_layout(w.T, w.H, w.W, w.text_tokens, w.block)
    t = time.perf_counter()
    Qh, Kh, Vh = O.bf16_to_f64(Qb[h_local]), O.bf16_to_f64(Kb[h_local]), O.bf16_to_f64(Vb[h_local])
    O.drift(Qh, Kh, Qh, Kh)
    S = O.score_head(Qh, Kh, L, mode).astype(np.float32)
    idx, cnt = O.select_topp(S, w.p[h_global], L)
    O.sparse_attention_head(Qh, Kh, Vh, idx, cnt, L)
    return (time.perf_counter() - t) * 1e3


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w, Qb, Kb, Vb, mode, seconds):
    """The oracle timed on the host cores on a bounded sample: whole heads (0, 1, ... in
    order) until `seconds` of CPU work have passed, at least one; mean per head x heads."""
    t = time.perf_counter()
    per = []
    while not per or time.perf_counter() - t < seconds:
        h = len(per) % Qb.shape[0]
        per.append(oracle_head_ms(w, Qb, Kb, Vb, mode, h, h))
    ms = float(np.mean(per)) * w.heads
    return {"value": round(ms, 3), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{len(per)} single-head calls (heads 0.. in order, cycling; {w.heads} heads per layer), "
                      f"full drift+score+select+attention, {time.perf_counter() - t:.1f} s of CPU work, "
                      f"mean per head x {w.heads}"}


def run_reference(args):
    """The oracle on the host cores, as it stands. Each step runs one head of the layer through
    the whole path (the next head each step); value = mean per-head time x heads, the same
    metric (ms per layer call) as the GPU arm."""
    from block_sparse_attention_query_b200 import inputs
    w = inputs.workload(args.workload)
    n_heads = min(w.heads, args.warmup + args.steps)
    Qb, Kb, Vb = inputs.generate_qkv(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, seed=0,
                                     head_range=(0, n_heads), workers=min(os.cpu_count() or 1, 16))
    mode = "park" if args.mode == "park" else "meanpool"
    per_step = []
    t_all = time.perf_counter()
    for k in range(args.warmup + args.steps):
        h = k % n_heads
        ms = oracle_head_ms(w, Qb, Kb, Vb, mode, h, h)
        if k >= args.warmup:
            per_step.append(ms)
    ms_head = float(np.mean(per_step))
    v = ms_head * w.heads
    cores = cpu_threads()
    sample = (f"{args.steps} timed steps, each one head of {w.heads} (heads cycling) through the whole path "
              f"(drift+score+select+attention); value = mean per-head time x {w.heads}")
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_head, 3),
        "step": "one head of the layer through the oracle", "heads_timed_per_step": 1,
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "scorer": mode, "parallelism": "single process (host cores)"},
        "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s_timed_and_warmup": round(time.perf_counter() - t_all, 1),
    }


def turbo_stages(n_steps, p_base):
    """Default Turbo stages of the one-shot schedule (the page gives none): re-select from the
    cached scores at 40% and 70% of the run with p lowered by 0.05 and 0.10."""
    return [(max(1, round(0.4 * n_steps)), round(p_base - 0.05, 4)),
            (max(2, round(0.7 * n_steps)), round(p_base - 0.10, 4))]


def run_reuse(args):
    """A multi-step run on a Q/K random walk (x_{s+1} = x_s + 0.02 N(0,1), V fixed) under one
    of the mask schedules:
      tmr      drift-gated reuse: a head's mask is recomputed only when its drift since the
               last refresh exceeds TAU (HEART abstract, Temporal Mask Reuse);
      oneshot  one estimate at --estimate-step (dense attention before it), the cached mask
               reused by every later step (RAPID English abstract);
      turbo    oneshot plus staged re-selection from the cached scores with smaller p.
    Reports amortised ms per step (CUDA events around all steps; all steps' inputs resident
    before timing) and what the steps did."""
    import torch

    from block_sparse_attention_query_b200 import inputs
    from block_sparse_attention_query_b200.layer import OneShotLayer, SparseAttentionLayer

    w = inputs.workload(args.workload)
    walk = inputs.RandomWalk(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, seed=0)
    dev = torch.device("cuda", 0)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    qs, ks = [], []
    for s in range(args.reuse):
        q, k, v = walk.current()
        qs.append(to_dev(q))
        ks.append(to_dev(k))
        walk.advance()
    V = to_dev(v)
    O = torch.empty(w.heads, w.tokens, w.d, dtype=torch.bfloat16, device=dev)
    flags = torch.zeros(args.reuse, w.heads, dtype=torch.int32, device=dev)
    kept = torch.zeros(args.reuse, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)
    stages = turbo_stages(args.reuse, float(np.mean(w.p))) if args.schedule == "turbo" else []
    kinds = []

    def make_layer():
        if args.schedule == "tmr":
            return SparseAttentionLayer(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block, p=list(w.p),
                                        tau=TAU, device=dev)
        return OneShotLayer(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block, p=list(w.p),
                            estimate_step=args.estimate_step, stages=stages, device=dev)

    def run(timed):
        layer = make_layer()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for s in range(args.reuse):
            layer.step(qs[s], ks[s], V, O)
            if timed:
                if args.schedule == "tmr":
                    flags[s].copy_(layer.refresh)
                    kept[s] = layer.cnt.sum()
                else:
                    if len(kinds) < args.reuse:
                        kinds.append(layer.kind)
                    if layer.kind != "dense":
                        kept[s] = layer.cnt.sum()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    for _ in range(max(1, args.warmup)):
        run(False)
    ms = [run(True) for _ in range(args.steps)]
    per_step = float(np.median(ms)) / args.reuse
    from block_sparse_attention_query_b200 import bsa
    nb = bsa.bsa_plan(bsa.problem(w.heads, w.d, w.T, w.H, w.W, w.text_tokens, w.block)).nb
    line = {
        "metric": f"amortised ms per denoising step ({args.reuse}-step {args.schedule} run)",
        "value": round(per_step, 5), "unit": UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic random walk x_{s+1} = x_s + 0.02 N(0,1) on Q, K (V fixed)",
        "config": {"workload": f"{w.name} {args.schedule} run", "denoising_steps": args.reuse,
                   "schedule": args.schedule, "timed_runs": args.steps, "statistic": "median over timed runs"},
        "kept_blocks_per_row_per_step": [round(float(x) / (w.heads * nb), 3) for x in kept.cpu().tolist()],
    }
    if args.schedule == "tmr":
        line["config"]["tau"] = TAU
        line.update({"refreshes": int(flags.sum().item()), "head_steps": args.reuse * w.heads,
                     "refreshed_per_step": [int(x) for x in flags.sum(dim=1).cpu().tolist()]})
    else:
        line["config"].update({"estimate_step": args.estimate_step, "stages": stages})
        line["step_kinds"] = kinds
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--mode", default="meanpool", choices=["meanpool", "park"])
    ap.add_argument("--gather", action="store_true", help="all-gather O over the ranks every step (N > 1)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first H heads of the layer (same shape per head; for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-retrieval", action="store_true", help="skip the retrieval-accuracy measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU seconds the oracle sample runs for (whole heads, at least one)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture (None if stale)")
    ap.add_argument("--reuse", type=int, default=0,
                    help="run an N-step random-walk run under --schedule instead (amortised ms per step)")
    ap.add_argument("--schedule", default="tmr", choices=["tmr", "oneshot", "turbo"],
                    help="mask schedule of the --reuse run: drift-gated reuse, one-shot estimate, one-shot + Turbo")
    ap.add_argument("--estimate-step", type=int, default=0, help="step of the one-shot estimate (oneshot/turbo)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    ws, rank, local = _dist()
    if args.gather and ws > 1:
        from block_sparse_attention_query_b200 import inputs
        if inputs.workload(args.workload).heads % ws:
            raise SystemExit("--gather needs the heads to split evenly over the GPUs")

    if args.reuse > 0:
        from block_sparse_attention_query_b200 import build
        build.build()
        print(json.dumps(run_reuse(args)), flush=True)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from block_sparse_attention_query_b200 import build
    if rank == 0 or ws == 1:
        build.build()
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    line, (w, host0) = run_ours(args, ws, rank, local)
    if rank == 0:
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, host0[0], host0[1], host0[2],
                                                "park" if args.mode == "park" else "meanpool", args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
