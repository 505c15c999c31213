"""Seeded synthetic inputs shaped like the video-DiT attention layers the pages benchmark.

This module draws random numbers and nothing else: it holds none of the block-sparse
method's arithmetic (no tiling, pooling, scoring, selection, drift or attention), so the
CPU oracle and the CUDA path can both take their inputs from it without sharing code.

Recipe (the pages give no input distribution; these stand in for Wan2.1 / HunyuanVideo
activations, which need trained weights we do not have):

* video tokens sit on a 3D grid (t, y, x) in raster order, x fastest;
* head h draws from its own stream, PCG64 seeded by SeedSequence(seed, spawn_key=(h,)), so
  any range of heads can be drawn alone (one GPU's share of the heads, or heads in parallel);
  in this order: omega_h ~ N(0, (1/8)^2) of shape [d, 3] (radians per grid unit),
  b_h ~ U[0, 2*pi)^d, then Q noise, K noise, V;
* RFF(t, y, x)_c = sqrt(2) * cos(omega_c . (t, y, x) + b_c)  (unit variance per channel);
* Q = 0.5 * N(0,1) + 2.0 * RFF,  K = 0.5 * N(0,1) + 2.0 * RFF (same RFF, fresh noise),
  V ~ N(0,1);
* text tokens (appended after the video tokens) have Q, K, V ~ N(0,1);
* every tensor is rounded once, round-to-nearest-even, to bfloat16.

Arrays are returned as numpy uint16 bfloat16 bit patterns of shape [heads, tokens, d].
"""
from __future__ import annotations

import dataclasses

import numpy as np

TOP_P_CHOICES = (0.80, 0.85, 0.90, 0.95, 0.98)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, nearest-even, returning uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention layer: shapes, block size and top-p per head."""

    name: str
    heads: int
    d: int
    T: int
    H: int
    W: int
    text_tokens: int
    block: int
    p: tuple  # per-head top-p thresholds

    @property
    def video_tokens(self) -> int:
        return self.T * self.H * self.W

    @property
    def tokens(self) -> int:
        return self.video_tokens + self.text_tokens


def _coords(T: int, H: int, W: int) -> np.ndarray:
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    return np.stack([t.ravel(), y.ravel(), x.ravel()], axis=1).astype(np.float64)


def _head_rng(seed: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(h,))))


def _generate_head(args):
    """Q, K, V bits (and the float32 pre-rounding Q, K) of head h."""
    h, d, T, H, W, text_tokens, seed = args
    rng = _head_rng(seed, h)
    nv = T * H * W
    n = nv + text_tokens
    xyz = _coords(T, H, W)
    omega = rng.normal(0.0, 1.0 / 8.0, size=(d, 3))
    b = rng.uniform(0.0, 2.0 * np.pi, size=d)
    rff = (np.sqrt(2.0) * np.cos(xyz @ omega.T + b)).astype(np.float32)
    qn = rng.standard_normal((n, d), dtype=np.float32)
    kn = rng.standard_normal((n, d), dtype=np.float32)
    vn = rng.standard_normal((n, d), dtype=np.float32)
    q = qn * np.float32(0.5)
    k = kn * np.float32(0.5)
    q[:nv] += np.float32(2.0) * rff
    k[:nv] += np.float32(2.0) * rff
    # text tokens: plain N(0,1), no 3D structure
    q[nv:] = qn[nv:]
    k[nv:] = kn[nv:]
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(vn), q, k


def generate_qkv(heads: int, d: int, T: int, H: int, W: int, text_tokens: int = 0,
                 seed: int = 0, state: bool = False, head_range=None, workers: int = 1):
    """Draw Q, K, V for one layer, or for the heads [h0, h1) of `head_range` only.

    Returns (Q, K, V) as uint16 bf16 bits [h1 - h0, tokens, d]. With ``state=True`` also
    returns the float32 pre-rounding Q and K (the random-walk state of the reuse run).
    ``workers`` > 1 draws heads in that many spawned processes (the result is the same).
    """
    h0, h1 = (0, heads) if head_range is None else head_range
    if not 0 <= h0 <= h1 <= heads:
        raise ValueError("head range outside the layer")
    jobs = [(h, d, T, H, W, text_tokens, seed) for h in range(h0, h1)]
    if workers > 1 and len(jobs) > 1:
        import concurrent.futures
        import multiprocessing
        with concurrent.futures.ProcessPoolExecutor(
                max_workers=min(workers, len(jobs)), mp_context=multiprocessing.get_context("spawn")) as ex:
            per_head = list(ex.map(_generate_head, jobs))
    else:
        per_head = [_generate_head(j) for j in jobs]
    n = T * H * W + text_tokens
    out = [np.empty((h1 - h0, n, d), np.uint16) for _ in range(3)]
    st = [np.empty((h1 - h0, n, d), np.float32) for _ in range(2)] if state else None
    for i, r in enumerate(per_head):
        for a in range(3):
            out[a][i] = r[a]
        if state:
            st[0][i] = r[3]
            st[1][i] = r[4]
    if state:
        return out[0], out[1], out[2], st[0], st[1]
    return out[0], out[1], out[2]


def draw_top_p(heads: int, seed: int = 0) -> np.ndarray:
    """Per-head top-p drawn uniformly from TOP_P_CHOICES (drawn after the tensors)."""
    rng = np.random.Generator(np.random.PCG64([seed, 1]))
    return rng.choice(np.array(TOP_P_CHOICES), heads)


class RandomWalk:
    """Q/K evolving across denoising steps: x_{s+1} = x_s + 0.02 * N(0,1) on the float32
    state, re-rounded to bf16 every step; V stays fixed."""

    def __init__(self, heads, d, T, H, W, text_tokens=0, seed=0, sigma=0.02):
        Q, K, V, Qs, Ks = generate_qkv(heads, d, T, H, W, text_tokens, seed, state=True)
        self.V = V
        self._q = Qs
        self._k = Ks
        self.sigma = np.float32(sigma)
        self.step_index = 0
        self._rng = np.random.Generator(np.random.PCG64([seed, 2]))

    def current(self):
        return f32_to_bf16_bits(self._q), f32_to_bf16_bits(self._k), self.V

    def advance(self):
        self._q = self._q + self.sigma * self._rng.standard_normal(self._q.shape, dtype=np.float32)
        self._k = self._k + self.sigma * self._rng.standard_normal(self._k.shape, dtype=np.float32)
        self.step_index += 1


# The five workloads: a tiny parity case, three layers shaped like Wan2.1-1.3B 480p,
# Wan2.1-14B 720p and HunyuanVideo 720p 5 s, and a 50-step reuse run on the tiny shape.
def workload(name: str, seed: int = 0) -> Workload:
    if name == "tiny":
        return Workload("tiny", 2, 64, 4, 16, 16, 0, 64, (0.9,) * 2)
    if name == "wan13b_480p":
        return Workload("wan13b_480p", 12, 128, 21, 30, 52, 0, 128, (0.9,) * 12)
    if name == "wan14b_720p":
        p = tuple(float(v) for v in draw_top_p(40, seed))
        return Workload("wan14b_720p", 40, 128, 21, 45, 80, 0, 128, p)
    if name == "hunyuan_720p":
        return Workload("hunyuan_720p", 24, 128, 33, 45, 80, 256, 128, (0.9,) * 24)
    raise KeyError(name)


WORKLOADS = ("tiny", "wan13b_480p", "wan14b_720p", "hunyuan_720p")
