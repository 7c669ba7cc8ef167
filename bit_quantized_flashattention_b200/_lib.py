"""ctypes view of libhifa4.so (include/hifa4.h). Loading fails loudly when the
library is missing: there is no fallback implementation."""
from __future__ import annotations

import ctypes
import os

from ._build import LIB

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4
NORM_P_REORDER, NORM_HIGH_PRECISION_L = 0, 1
F16, BF16, F32 = 0, 1, 2
CAUSAL = 1
SPLIT_KV = 2

EXPORTS = ["hifa4_packed_bytes", "hifa4_workspace_bytes", "hifa4_calibrate_smooth", "hifa4_quantize_qkv",
           "hifa4_quantize_kv", "hifa4_attention_fwd", "hifa4_attention_fwd_debug", "hifa4_get_status",
           "hifa4_debug_set_wait_limit", "hifa4_status_string", "hifa4_version", "hifa4_attention_fwd_noalloc",
           "hifa4_last_cuda_error", "hifa4_attention_splits", "hifa4_quantize_qkv_ex", "hifa4_q_mean",
           "hifa4_append_kv", "hifa4_attention_fwd_ex", "hifa4_tile_stats", "hifa4_attention_fwd_q",
           "hifa4_quantize_q"]


class Packed(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("qc", "qs", "kc", "ks", "vtc", "vts")]


class Prequant(ctypes.Structure):
    _fields_ = [("s", ctypes.c_void_p), ("s_inv", ctypes.c_void_p), ("rope_cos", ctypes.c_void_p),
                ("rope_sin", ctypes.c_void_p), ("q_pos", ctypes.c_void_p), ("k_pos", ctypes.c_void_p),
                ("n_pos", ctypes.c_int), ("q_mean", ctypes.c_void_p), ("s_bias", ctypes.c_void_p)]


class AttentionExtras(ctypes.Structure):
    _fields_ = [("s_bias", ctypes.c_void_p), ("p_codes", ctypes.c_void_p), ("p_scales", ctypes.c_void_p),
                ("tile_sums", ctypes.c_void_p)]


class HiFA4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = f" [{load().hifa4_last_cuda_error().decode()}]" if status == ERR_CUDA else ""
        super().__init__(f"{what}: {status_string(status)} (status {status}){detail}")


_lib = None


def load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise ImportError(f"libhifa4.so is not built ({LIB}); run __graft_entry__.build() or "
                          "python -m bit_quantized_flashattention_b200._build")
    L = ctypes.CDLL(LIB)
    vp, ci, cf, cu, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint, ctypes.c_size_t
    pk = ctypes.POINTER(Packed)
    L.hifa4_packed_bytes.argtypes = [ci] * 6 + [ctypes.POINTER(sz)]
    L.hifa4_packed_bytes.restype = sz
    L.hifa4_attention_splits.argtypes = [ci] * 6 + [cu]
    L.hifa4_attention_splits.restype = ci
    L.hifa4_workspace_bytes.argtypes = [ci] * 6
    L.hifa4_workspace_bytes.restype = sz
    L.hifa4_calibrate_smooth.argtypes = [vp, vp, ci, ci, ci, ci, ci, ci, cf, vp, vp, vp]
    L.hifa4_calibrate_smooth.restype = ci
    L.hifa4_quantize_qkv.argtypes = [vp, vp, vp, ci] + [ci] * 6 + [vp, vp, pk, vp]
    L.hifa4_quantize_qkv.restype = ci
    L.hifa4_quantize_kv.argtypes = [vp, vp, ci, ci, ci, ci, ci, vp, pk, vp]
    L.hifa4_quantize_kv.restype = ci
    L.hifa4_attention_fwd.argtypes = [pk] + [ci] * 6 + [cf, cu, ci, vp, ci, vp, vp, vp]
    L.hifa4_attention_fwd.restype = ci
    L.hifa4_attention_fwd_debug.argtypes = [pk] + [ci] * 6 + [cf, cu, ci, vp, ci, vp, vp, vp, vp, vp]
    L.hifa4_attention_fwd_debug.restype = ci
    L.hifa4_attention_fwd_noalloc.argtypes = [pk] + [ci] * 6 + [cf, cu, ci, vp, ci, vp, vp]
    L.hifa4_attention_fwd_noalloc.restype = ci
    pre = ctypes.POINTER(Prequant)
    L.hifa4_quantize_qkv_ex.argtypes = [vp, vp, vp, ci] + [ci] * 6 + [pre, pk, vp]
    L.hifa4_quantize_qkv_ex.restype = ci
    L.hifa4_quantize_q.argtypes = [vp, ci, ci, ci, ci, ci, ci, pre, pk, vp]
    L.hifa4_quantize_q.restype = ci
    L.hifa4_q_mean.argtypes = [vp, ci, ci, ci, ci, ci, ci, pre, vp, vp]
    L.hifa4_q_mean.restype = ci
    L.hifa4_append_kv.argtypes = [vp, vp, ci, ci, ci, ci, ci, pre, pk, ci, ci, vp]
    L.hifa4_append_kv.restype = ci
    L.hifa4_attention_fwd_ex.argtypes = [pk] + [ci] * 6 + [cf, cu, ci, vp, ci, vp, ctypes.POINTER(AttentionExtras),
                                                           vp, vp]
    L.hifa4_attention_fwd_ex.restype = ci
    L.hifa4_attention_fwd_q.argtypes = [vp, ci, vp, pk] + [ci] * 6 + [cf, cu, ci, vp, ci, vp, vp, vp]
    L.hifa4_attention_fwd_q.restype = ci
    L.hifa4_tile_stats.argtypes = [vp, ci, ci, ci, ci, vp, vp]
    L.hifa4_tile_stats.restype = ci
    L.hifa4_get_status.argtypes = [vp, vp]
    L.hifa4_get_status.restype = ci
    L.hifa4_debug_set_wait_limit.argtypes = [ctypes.c_longlong, ci]
    L.hifa4_debug_set_wait_limit.restype = ctypes.c_longlong
    L.hifa4_status_string.argtypes = [ci]
    L.hifa4_status_string.restype = ctypes.c_char_p
    L.hifa4_last_cuda_error.argtypes = []
    L.hifa4_last_cuda_error.restype = ctypes.c_char_p
    L.hifa4_version.argtypes = []
    L.hifa4_version.restype = ci
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().hifa4_status_string(int(status)).decode()


def check(status: int, what: str) -> None:
    if status != OK:
        raise HiFA4Error(status, what)
