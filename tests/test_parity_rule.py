"""The kept-list comparison rule and the score error bound of tests/parity.py, on the CPU.

The rule must pass exactly what the parity contract allows (an identical list; a cut within
1e-5 of p; a position-wise swap of two blocks whose scores are closer than their error
bounds) and nothing else: in particular not a shorter or longer prefix of the oracle's order
whose cut lies outside the window. The bound must cover a float32 evaluation of the scorers
and must not cover a real arithmetic mistake."""
import math

import numpy as np
import pytest

from block_sparse_attention_query_b200 import inputs
from oracle import bsa_oracle as O
from tests import parity as PT


def _row(scores):
    return np.asarray(scores, np.float32)


def test_prefix_of_wrong_length_is_a_mismatch():
    s = _row([.5, .3, .1, .05, .05])
    zero = np.zeros(5)
    assert PT.compare_row([0, 1, 2], s, zero, 0.9, [], False) == "exact"
    assert PT.compare_row([0], s, zero, 0.9, [], False) == "mismatch"
    assert PT.compare_row([0, 1, 2, 3, 4], s, zero, 0.9, [], False) == "mismatch"
    assert PT.compare_row([0, 1], s, zero, 0.9, [], False) == "mismatch"
    # here the float32 cumulative mass after three blocks is 0.9 itself, inside the window:
    # a fourth block is allowed, a fifth is not
    assert PT.compare_row([0, 1, 2, 3], s, zero, 0.9, [], False) == "window"
    # at p = 0.85 the cut (0.9) is far from p: only the exact three-block list passes
    assert PT.compare_row([0, 1, 2], s, zero, 0.85, [], False) == "exact"
    assert PT.compare_row([0, 1, 2, 3], s, zero, 0.85, [], False) == "mismatch"
    assert PT.compare_row([0, 1], s, zero, 0.85, [], False) == "mismatch"


def test_cut_within_window_only():
    # cumulative masses 0.5, 0.8, 0.9000001 ...: p = 0.9 cuts after three blocks; a kernel
    # whose float32 sum lands a hair lower may take a fourth block
    s = _row([.5, .3, .1000001, .05, .0499999])
    assert PT.compare_row([0, 1, 2, 3], s, None, 0.9, [], False) == "window"
    # the same row at p = 0.85: the cut (0.9) is 0.05 above p, outside the window
    assert PT.compare_row([0, 1, 2, 3], s, None, 0.85, [], False) == "mismatch"


def test_swap_only_between_blocks_within_their_bounds():
    s = _row([.4, .3, .3000002, .0, .0])
    s[3] = s[4] = np.float32(0.0)
    tight = np.full(5, 1e-8)
    loose = np.full(5, 2e-7)
    # oracle order: 0, 2, 1 (score desc); p = 0.65 keeps 0, 2
    assert PT.compare_row([0, 2], s, tight, 0.65, [], False) == "exact"
    assert PT.compare_row([0, 1], s, loose, 0.65, [], False) == "tie"
    assert PT.compare_row([0, 1], s, tight, 0.65, [], False) == "mismatch"
    # a swap with a block far away in score is never a tie
    assert PT.compare_row([0, 3], s, loose, 0.65, [], False) == "mismatch"
    # a swap at different positions (a reordered list) of non-tied blocks is a mismatch
    assert PT.compare_row([2, 0], s, loose, 0.65, [], False) == "mismatch"


def test_forced_and_text_rows():
    s = _row([.6, .3, .05, .05])
    assert PT.compare_row([0, 1, 3], s, None, 0.85, [3], False) == "exact"
    assert PT.compare_row([0, 1], s, None, 0.85, [3], False) == "mismatch"      # text block missing
    assert PT.compare_row([0, 1, 2, 3], s, None, 0.3, [], True) == "exact"     # text row keeps all
    assert PT.compare_row([0, 1, 2], s, None, 0.3, [], True) == "mismatch"


def _head(name_args, h=0):
    heads, d, T, H, W, text, B = name_args
    Qb, Kb, _ = inputs.generate_qkv(heads, d, T, H, W, text, seed=3)
    L = O.block_layout(T, H, W, text, B)
    return O.bf16_to_f64(Qb[h]), O.bf16_to_f64(Kb[h]), L


def _f32_meanpool(Qh, Kh, L, scale_factor=1.0):
    """The mean-pooled scores evaluated in float32 throughout (block sums, dot products,
    exponentials, normalisation)."""
    d = Qh.shape[1]
    q = np.stack([Qh[L.rows(i)].astype(np.float32).sum(axis=0) / np.float32(len(L.rows(i))) for i in range(L.nb)])
    k = np.stack([Kh[L.rows(i)].astype(np.float32).sum(axis=0) / np.float32(len(L.rows(i))) for i in range(L.nb)])
    x = (q @ k.T) * np.float32(scale_factor / math.sqrt(d))
    e = np.exp(x - x.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True, dtype=np.float32)


def _f32_park(Qh, Kh, L):
    d = Qh.shape[1]
    k = np.stack([Kh[L.rows(i)].astype(np.float32).sum(axis=0) / np.float32(len(L.rows(i))) for i in range(L.nb)])
    out = np.zeros((L.nb, L.nb), np.float32)
    for i in range(L.nb):
        x = (Qh[L.rows(i)].astype(np.float32) @ k.T) * np.float32(1.0 / math.sqrt(d))
        e = np.exp(x - x.max(axis=1, keepdims=True))
        out[i] = (e / e.sum(axis=1, keepdims=True, dtype=np.float32)).mean(axis=0, dtype=np.float32)
    return out


SHAPES = [(2, 64, 4, 16, 16, 0, 64), (2, 128, 6, 20, 24, 256, 128)]


@pytest.mark.parametrize("shape", SHAPES)
def test_bound_covers_float32_evaluation_meanpool(shape):
    Qh, Kh, L = _head(shape)
    S = O.score_meanpool(Qh, Kh, L)
    bnd = PT.score_bound(Qh, Kh, L, "meanpool", S)
    assert np.all(np.abs(_f32_meanpool(Qh, Kh, L) - S) <= bnd)
    # the bound is tight enough to matter: a relative logit-scale error of 1e-4 breaks it
    bad = _f32_meanpool(Qh, Kh, L, scale_factor=1.0 + 1e-4)
    assert (np.abs(bad - S) > bnd).mean() > 0.2


@pytest.mark.parametrize("shape", SHAPES)
def test_bound_covers_float32_evaluation_park(shape):
    Qh, Kh, L = _head(shape)
    S = O.score_park(Qh, Kh, L)
    bnd = PT.score_bound(Qh, Kh, L, "park")
    assert np.all(np.abs(_f32_park(Qh, Kh, L) - S) <= bnd)
    # a dropped real query in every block (the mean over n-1 rows) breaks it
    bad = np.zeros_like(S)
    for i in range(L.nb):
        r = L.rows(i)[1:]
        x = Qh[r] @ O.pool_blocks(Kh, L).T / math.sqrt(Qh.shape[1])
        e = np.exp(x - x.max(axis=1, keepdims=True))
        bad[i] = (e / e.sum(axis=1, keepdims=True)).mean(axis=0)
    assert (np.abs(bad - S) > bnd).mean() > 0.2


def test_bound_is_about_float32_sized():
    # the relative bound sits a few hundred float32 roundings above exact: far below a blanket
    # tolerance such as 5e-5 relative on every score
    Qh, Kh, L = _head(SHAPES[1])
    S = O.score_meanpool(Qh, Kh, L)
    rel = PT.score_bound(Qh, Kh, L, "meanpool", S) / S
    assert 16 * PT.U32 < np.median(rel) < 6e-5
