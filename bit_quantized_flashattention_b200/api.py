"""PyTorch-facing binding of libhifa4.so.

Argument marshalling only: torch supplies device memory and the current CUDA
stream, every step of the computation runs in the library's kernels. The
function names follow the C ABI (include/hifa4.h) without the ``hifa4_``
prefix.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _lib as L

_DT = {torch.float16: L.F16, torch.bfloat16: L.BF16, torch.float32: L.F32}
_NORM = {"p_reorder": L.NORM_P_REORDER, "high_precision_l": L.NORM_HIGH_PRECISION_L,
         L.NORM_P_REORDER: L.NORM_P_REORDER, L.NORM_HIGH_PRECISION_L: L.NORM_HIGH_PRECISION_L}


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p | None:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_input(x: torch.Tensor, name: str, ndim: int = 4):
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if x.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


@dataclass
class PackedQKV:
    """Quantized operands (device uint8 buffers, layouts as in hifa4.h)."""
    qc: torch.Tensor
    qs: torch.Tensor
    kc: torch.Tensor
    ks: torch.Tensor
    vtc: torch.Tensor
    vts: torch.Tensor
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    D: int

    def struct(self) -> L.Packed:
        return L.Packed(*(ctypes.c_void_p(t.data_ptr()) for t in
                          (self.qc, self.qs, self.kc, self.ks, self.vtc, self.vts)))

    @property
    def shape(self):
        return (self.B, self.Hq, self.Hkv, self.Nq, self.Nkv, self.D)

    def tensors(self):
        return dict(qc=self.qc, qs=self.qs, kc=self.kc, ks=self.ks, vtc=self.vtc, vts=self.vts)


def packed_bytes(B, Hq, Hkv, Nq, Nkv, D) -> list[int]:
    out = (ctypes.c_size_t * 6)()
    total = L.load().hifa4_packed_bytes(B, Hq, Hkv, Nq, Nkv, D, out)
    if total == 0:
        raise L.HiFA4Error(L.ERR_UNSUPPORTED, "packed_bytes")
    return list(out)


def alloc_packed(B, Hq, Hkv, Nq, Nkv, D, device="cuda") -> PackedQKV:
    sizes = packed_bytes(B, Hq, Hkv, Nq, Nkv, D)
    bufs = [torch.empty(n, dtype=torch.uint8, device=device) for n in sizes]
    return PackedQKV(*bufs, B, Hq, Hkv, Nq, Nkv, D)


def workspace_bytes(B, Hq, Hkv, Nq, Nkv, D) -> int:
    return int(L.load().hifa4_workspace_bytes(B, Hq, Hkv, Nq, Nkv, D))


def alloc_workspace(B, Hq, Hkv, Nq, Nkv, D, device="cuda") -> torch.Tensor:
    return torch.zeros(workspace_bytes(B, Hq, Hkv, Nq, Nkv, D), dtype=torch.uint8, device=device)


def calibrate_smooth(q: torch.Tensor, k: torch.Tensor, alpha: float = 0.5, s=None, s_inv=None, stream=None):
    """Smooth-QK factors (s, s_inv), fp32 [Hkv, D], from calibration Q/K."""
    _check_input(q, "q")
    _check_input(k, "k")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D) or q.dtype != k.dtype:
        raise ValueError("q and k shapes / dtypes do not match")
    s = torch.empty(Hkv, D, dtype=torch.float32, device=q.device) if s is None else s
    s_inv = torch.empty_like(s) if s_inv is None else s_inv
    L.check(L.load().hifa4_calibrate_smooth(_ptr(q), _ptr(k), _DT[q.dtype], B, Hq, Hkv, N, D, float(alpha),
                                            _ptr(s), _ptr(s_inv), _stream(stream)), "calibrate_smooth")
    return s, s_inv


def quantize_qkv(q, k, v, s=None, s_inv=None, out: PackedQKV | None = None, stream=None) -> PackedQKV:
    """Smooth (when s/s_inv are given) and quantize Q, K, V to the packed 4-bit operands."""
    for x, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_input(x, n)
    B, Hq, Nq, D = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D or not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v shapes / dtypes do not match")
    if out is None:
        out = alloc_packed(B, Hq, Hkv, Nq, Nkv, D, q.device)
    st = out.struct()
    L.check(L.load().hifa4_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], B, Hq, Hkv, Nq, Nkv, D,
                                        _ptr(s), _ptr(s_inv), ctypes.byref(st), _stream(stream)), "quantize_qkv")
    return out


def quantize_kv(k, v, s_inv=None, out: PackedQKV | None = None, Hq: int | None = None, Nq: int = 16,
                stream=None) -> PackedQKV:
    """Quantize K and V only (e.g. when a KV cache is appended)."""
    _check_input(k, "k")
    _check_input(v, "v")
    B, Hkv, Nkv, D = k.shape
    if out is None:
        out = alloc_packed(B, Hq or Hkv, Hkv, Nq, Nkv, D, k.device)
    st = out.struct()
    L.check(L.load().hifa4_quantize_kv(_ptr(k), _ptr(v), _DT[k.dtype], B, Hkv, Nkv, D, _ptr(s_inv),
                                       ctypes.byref(st), _stream(stream)), "quantize_kv")
    return out


def attention_splits(B, Hq, Hkv, Nq, Nkv, D, causal=False, split_kv=False) -> int:
    """Number of kv ranges the attention calls use for this shape (1 = one pass)."""
    flags = (L.CAUSAL if causal else 0) | (L.SPLIT_KV if split_kv else 0)
    return int(L.load().hifa4_attention_splits(B, Hq, Hkv, Nq, Nkv, D, flags))


def _attn_args(packed, sm_scale, causal, norm, out_dtype, out, lse, workspace, want_lse=True, split_kv=False):
    B, Hq, Hkv, Nq, Nkv, D = packed.shape
    dev = packed.qc.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(B, Hq, Nq, D, dtype=out_dtype, device=dev)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, Nq, Nkv, D, dev)
    flags = (L.CAUSAL if causal else 0) | (L.SPLIT_KV if split_kv else 0)
    return sm_scale, flags, _NORM[norm], out, lse, workspace


def attention_fwd(packed: PackedQKV, sm_scale: float | None = None, causal: bool = False,
                  norm="p_reorder", out_dtype=torch.bfloat16, out=None, lse=None, workspace=None,
                  stream=None, want_lse: bool = True, split_kv: bool = False):
    """4-bit attention forward. Returns (O [B,Hq,Nq,D], LSE [B,Hq,Nq] fp32 or None).
    split_kv: allow the split-kv decode mode (see attention_splits)."""
    sm_scale, flags, nm, out, lse, workspace = _attn_args(packed, sm_scale, causal, norm, out_dtype, out, lse,
                                                          workspace, want_lse, split_kv)
    st = packed.struct()
    B, Hq, Hkv, Nq, Nkv, D = packed.shape
    L.check(L.load().hifa4_attention_fwd(ctypes.byref(st), B, Hq, Hkv, Nq, Nkv, D, float(sm_scale), flags, nm,
                                         _ptr(out), _DT[out.dtype], _ptr(lse), _ptr(workspace), _stream(stream)),
            "attention_fwd")
    return out, lse


def attention_fwd_noalloc(packed: PackedQKV, sm_scale: float | None = None, causal: bool = False,
                          norm="p_reorder", out_dtype=torch.bfloat16, out=None, lse=None, stream=None,
                          split_kv: bool = False):
    """attention_fwd for callers that cannot allocate device memory: the library
    uses its own fixed scratch (see hifa4_attention_fwd_noalloc in hifa4.h).
    ``out``/``lse`` are still the caller's buffers (allocated here when None)."""
    B, Hq, Hkv, Nq, Nkv, D = packed.shape
    dev = packed.qc.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(B, Hq, Nq, D, dtype=out_dtype, device=dev)
    if lse is None:
        lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=dev)
    st = packed.struct()
    L.check(L.load().hifa4_attention_fwd_noalloc(ctypes.byref(st), B, Hq, Hkv, Nq, Nkv, D, float(sm_scale),
                                                 (L.CAUSAL if causal else 0) | (L.SPLIT_KV if split_kv else 0),
                                                 _NORM[norm], _ptr(out), _DT[out.dtype],
                                                 _ptr(lse), _stream(stream)), "attention_fwd_noalloc")
    return out, lse


def attention_fwd_debug(packed: PackedQKV, sm_scale: float | None = None, causal: bool = False,
                        norm="p_reorder", out_dtype=torch.float32, workspace=None, stream=None, split_kv: bool = False):
    """attention_fwd plus the P_hat the PV GEMM consumed: (O, LSE, p_codes, p_scales)."""
    sm_scale, flags, nm, out, lse, workspace = _attn_args(packed, sm_scale, causal, norm, out_dtype, None, None,
                                                          workspace, True, split_kv)
    B, Hq, Hkv, Nq, Nkv, D = packed.shape
    pc = torch.zeros(B, Hq, Nq, Nkv // 2, dtype=torch.uint8, device=out.device)
    ps = torch.zeros(B, Hq, Nq, Nkv // 16, dtype=torch.uint8, device=out.device)
    st = packed.struct()
    L.check(L.load().hifa4_attention_fwd_debug(ctypes.byref(st), B, Hq, Hkv, Nq, Nkv, D, float(sm_scale), flags, nm,
                                               _ptr(out), _DT[out.dtype], _ptr(lse), _ptr(pc), _ptr(ps),
                                               _ptr(workspace), _stream(stream)), "attention_fwd_debug")
    return out, lse, pc, ps


def get_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return (and clear) the status a kernel recorded."""
    return int(L.load().hifa4_get_status(_ptr(workspace), _stream(stream)))


def debug_set_wait_limit(limit_ns: int, stall_loads: bool = False) -> int:
    return int(L.load().hifa4_debug_set_wait_limit(int(limit_ns), 1 if stall_loads else 0))
