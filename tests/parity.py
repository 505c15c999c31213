"""Helpers for GPU-vs-oracle parity: device transfer and the kept-list comparison rule.

Kept-list rule (top-p lists, per row):
  * bit-exact lists pass;
  * a different cut length passes when the oracle's float32 cumulative mass at the
    boundary lies within WINDOW (1e-5) of p — the prefix must still be identical;
  * position-wise substitutions pass only between blocks whose oracle scores agree within
    the scorer's own float32 error (TIE_REL relative): the two scores are then not
    distinguishable by the kernel's arithmetic, so either order is correct.
Anything else is a true mismatch; the gate is zero true mismatches.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import bsa_oracle as O

WINDOW = 1e-5
# Relative error bound of a float32 block score: logits |x| <= ~60 carry <= ~1e-5 absolute
# float32 error after a 128-term dot product, i.e. <= ~2e-5 relative after exp; the bound
# below keeps a 2.5x margin.
TIE_REL = 5e-5
TIE_ABS = 1e-12


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_bits_f64(bits):
    return O.bf16_to_f64(bits)


def _expected(order, m, forced):
    keep = set(order[:m].tolist()) | set(forced)
    return [int(j) for j in order if int(j) in keep]


def compare_row(gpu_list, scores_f32, p, forced, text_row):
    """Classify one row: 'exact', 'window', 'tie' or 'mismatch'."""
    s = np.asarray(scores_f32, np.float32)
    n = len(s)
    kept_o, order, cum = O.select_row(s, 1.0 if text_row else p, forced)
    g = [int(x) for x in gpu_list]
    if g == kept_o:
        return "exact"
    if len(set(g)) != len(g) or not set(forced) <= set(g) or any(j < 0 or j >= n for j in g):
        return "mismatch"
    if text_row or p >= 1.0:
        allowed = [n]
    else:
        p32 = np.float32(p)
        allowed = [m for m in range(1, n + 1)
                   if cum[m - 1] >= p32 - WINDOW and (m == 1 or cum[m - 2] < p32 + WINDOW)]
    for m in allowed:
        if g == _expected(order, m, forced):
            return "window"
    s64 = s.astype(np.float64)
    for m in allowed + [len(g)]:
        e = _expected(order, m, forced)
        if len(e) != len(g):
            continue
        ok = True
        for a, b in zip(g, e):
            if a != b and abs(s64[a] - s64[b]) > TIE_REL * max(s64[a], s64[b]) + TIE_ABS:
                ok = False
                break
        if ok:
            return "tie"
    return "mismatch"


def compare_masks(gpu_idx, gpu_cnt, scores_f32, p_heads, layout, heads=None):
    """Compare every row of the GPU kept lists against the oracle's selection from the
    given float32 scores [heads, nb, nb]. Returns a dict of counts and the first
    mismatches."""
    counts = {"exact": 0, "window": 0, "tie": 0, "mismatch": 0}
    bad = []
    text = list(range(layout.nb_video, layout.nb))
    for h in (range(scores_f32.shape[0]) if heads is None else heads):
        for i in range(layout.nb):
            c = int(gpu_cnt[h, i])
            row = gpu_idx[h, i, :max(c, 0)]
            text_row = layout.is_text_block(i)
            kind = compare_row(row, scores_f32[h, i], float(p_heads[h]),
                               [] if text_row else text, text_row)
            counts[kind] += 1
            if kind == "mismatch" and len(bad) < 5:
                bad.append((h, i, row.tolist()[:12]))
    counts["first_mismatches"] = bad
    return counts


def attention_errors(gpu_o, ref_o, rows):
    """max-abs and relative-L2 error over the given raster rows (float64)."""
    a = gpu_o[:, rows] if gpu_o.ndim == 3 else gpu_o[rows]
    b = ref_o[:, rows] if ref_o.ndim == 3 else ref_o[rows]
    diff = a - b
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / np.linalg.norm(b))
