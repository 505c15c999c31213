"""Thin Python binding of libbsa (include/bsa.h): argument marshalling only.

Every function keeps the C name and signature; tensors are passed as device pointers
(torch is used for device memory and streams, nothing else). There is no fallback: if
libbsa.so is missing or cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

BSA_OK = 0
BSA_ERR_ARG = -1
BSA_ERR_UNSUPPORTED = -2
BSA_ERR_ALIGN = -3
BSA_ERR_WORKSPACE = -4
BSA_ERR_CUDA = -5
BSA_ERR_TIMEOUT = -6
BSA_ERR_DEVICE_ARG = -7
BSA_ERR_SCRATCH_LIMIT = -8

BSA_SCORE_MEANPOOL = 0
BSA_SCORE_PARK = 1


class Problem(ctypes.Structure):
    """Mirror of `bsa_problem`."""
    _fields_ = [
        ("heads", ctypes.c_int), ("tokens", ctypes.c_int), ("d", ctypes.c_int),
        ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("text_tokens", ctypes.c_int), ("block", ctypes.c_int),
        ("tile_t", ctypes.c_int), ("tile_h", ctypes.c_int), ("tile_w", ctypes.c_int),
        ("score_mode", ctypes.c_int),
        ("key_table", ctypes.c_void_p),
        ("block_means", ctypes.c_void_p),
    ]


class PlanInfo(ctypes.Structure):
    """Mirror of `bsa_plan_info`."""
    _fields_ = [
        ("nb", ctypes.c_int), ("nb_video", ctypes.c_int), ("nb_text", ctypes.c_int),
        ("npad", ctypes.c_int), ("tile_t", ctypes.c_int), ("tile_h", ctypes.c_int),
        ("tile_w", ctypes.c_int),
        ("score_workspace_bytes", ctypes.c_size_t),
        ("drift_workspace_bytes", ctypes.c_size_t),
        ("attention_workspace_bytes", ctypes.c_size_t),
        ("mass_workspace_bytes", ctypes.c_size_t),
        ("cluster_workspace_bytes", ctypes.c_size_t),
        ("park_cluster", ctypes.c_int), ("park_cols", ctypes.c_int),
    ]


EXPORTS = {
    # name: (restype, argtypes)
    "bsa_plan": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.POINTER(PlanInfo)]),
    "bsa_block_layout": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.POINTER(ctypes.c_int)]),
    "bsa_score_blocks": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p]),
    "bsa_select_topp": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p]),
    "bsa_drift_check": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p]),
    "bsa_drift_check_noalloc": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "bsa_sparse_attention": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]),
    "bsa_cluster_keys": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]),
    "bsa_dense_correction": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "bsa_captured_mass": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]),
    "bsa_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "bsa_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bsa_version": (ctypes.c_char_p, []),
    "bsa_launch_count": (ctypes.c_ulonglong, []),
    "bsa_set_park_kernel": (ctypes.c_int, [ctypes.c_int]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbsa.so not built ({LIB_PATH}); run "
                          "`python -m block_sparse_attention_query_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {lib.bsa_error_string(status).decode()} ({status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != BSA_OK:
        raise BsaError(status, where)


def problem(heads, d, T, H, W, text_tokens=0, block=128, tile=(0, 0, 0),
            score_mode=BSA_SCORE_MEANPOOL, key_table=None, block_means=None) -> Problem:
    """key_table: a device int32 tensor [heads, nb*block] from bsa_cluster_keys, or None.
    block_means: a device float32 tensor [2, heads, nb, d] (drift pass writes, scores read), or None."""
    return Problem(heads, T * H * W + text_tokens, d, T, H, W, text_tokens, block,
                   tile[0], tile[1], tile[2], score_mode,
                   None if key_table is None else key_table.data_ptr(),
                   None if block_means is None else block_means.data_ptr())


def bsa_plan(prob: Problem) -> PlanInfo:
    info = PlanInfo()
    check(lib.bsa_plan(ctypes.byref(prob), ctypes.byref(info)), "bsa_plan")
    return info


def bsa_block_layout(prob: Problem):
    """Host-side block layout: raster token per block slot (-1 = padding), as a list."""
    info = bsa_plan(prob)
    buf = (ctypes.c_int * info.npad)()
    check(lib.bsa_block_layout(ctypes.byref(prob), buf), "bsa_block_layout")
    return list(buf)


# ---------------------------------------------------------------------- device calls

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def bsa_score_blocks(prob, Q, K, head_mask, scores, ws, stream=None):
    check(lib.bsa_score_blocks(ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(head_mask), _ptr(scores),
                               _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
                               _stream(stream)), "bsa_score_blocks")


def bsa_select_topp(prob, scores, p, head_mask, idx, cnt, stream=None):
    check(lib.bsa_select_topp(ctypes.byref(prob), _ptr(scores), _ptr(p), _ptr(head_mask), _ptr(idx),
                              _ptr(cnt), _stream(stream)), "bsa_select_topp")


def bsa_drift_check(prob, Q, K, Q_ref, K_ref, tau, force_all, drift, refresh, ws, stream=None):
    check(lib.bsa_drift_check(ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(Q_ref), _ptr(K_ref),
                              ctypes.c_float(tau), int(force_all), _ptr(drift), _ptr(refresh), _ptr(ws),
                              ws.numel() * ws.element_size() if ws is not None else 0,
                              _stream(stream)), "bsa_drift_check")


def bsa_drift_check_noalloc(prob, Q, K, Q_ref, K_ref, tau, force_all, drift, refresh, stream=None):
    """bsa_drift_check with the library's static scratch instead of a caller workspace."""
    check(lib.bsa_drift_check_noalloc(ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(Q_ref), _ptr(K_ref),
                                      ctypes.c_float(tau), int(force_all), _ptr(drift), _ptr(refresh),
                                      _stream(stream)), "bsa_drift_check_noalloc")


def bsa_sparse_attention(prob, Q, K, V, idx, cnt, O, ws, stream=None):
    check(lib.bsa_sparse_attention(ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(cnt),
                                   _ptr(O), _ptr(ws),
                                   ws.numel() * ws.element_size() if ws is not None else 0,
                                   _stream(stream)), "bsa_sparse_attention")


def bsa_cluster_keys(prob, Q, K, iters, key_table, assignment, ws, stream=None):
    check(lib.bsa_cluster_keys(ctypes.byref(prob), _ptr(Q), _ptr(K), int(iters), _ptr(key_table), _ptr(assignment),
                               _ptr(ws),
                               ws.numel() * ws.element_size() if ws is not None else 0,
                               _stream(stream)), "bsa_cluster_keys")


def bsa_dense_correction(prob, Q, K, V, refresh, O, R, ws, stream=None):
    check(lib.bsa_dense_correction(ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(V), _ptr(refresh), _ptr(O), _ptr(R),
                                   _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
                                   _stream(stream)), "bsa_dense_correction")


def bsa_captured_mass(prob, Q, K, idx, cnt, mass, ws, stream=None):
    check(lib.bsa_captured_mass(ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(idx), _ptr(cnt), _ptr(mass), _ptr(ws),
                                ws.numel() * ws.element_size() if ws is not None else 0,
                                _stream(stream)), "bsa_captured_mass")


def bsa_device_status(stream=None) -> int:
    return lib.bsa_device_status(_stream(stream))


def bsa_version() -> str:
    return lib.bsa_version().decode()


def bsa_launch_count() -> int:
    return int(lib.bsa_launch_count())


PARK_AUTO = 0
PARK_TWO_PASS = 1


def bsa_set_park_kernel(which: int) -> int:
    return lib.bsa_set_park_kernel(which)
