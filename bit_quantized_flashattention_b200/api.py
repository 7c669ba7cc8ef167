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
    s_bias: torch.Tensor | None = None     # Q-Mean score bias written by quantize_qkv(q_mean=...)

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


@dataclass
class Rope:
    """RoPE inputs: fp32 tables [n_pos, D/2] and int32 positions of the query
    tokens [Nq] and key tokens [Nkv] (or the appended keys [n_new])."""
    cos: torch.Tensor
    sin: torch.Tensor
    q_pos: torch.Tensor | None = None
    k_pos: torch.Tensor | None = None


def _prequant(s=None, s_inv=None, rope: Rope | None = None, q_mean=None, s_bias=None) -> L.Prequant:
    pq = L.Prequant()
    pq.s, pq.s_inv, pq.q_mean, pq.s_bias = _ptr(s), _ptr(s_inv), _ptr(q_mean), _ptr(s_bias)
    if rope is not None:
        for t, n in ((rope.cos, "rope.cos"), (rope.sin, "rope.sin")):
            _check_input(t, n, 2)
            if t.dtype != torch.float32:
                raise ValueError(f"{n} must be float32")
        for t, n in ((rope.q_pos, "rope.q_pos"), (rope.k_pos, "rope.k_pos")):
            if t is not None and (t.dtype != torch.int32 or not t.is_contiguous()):
                raise ValueError(f"{n} must be a contiguous int32 tensor")
        pq.rope_cos, pq.rope_sin = _ptr(rope.cos), _ptr(rope.sin)
        pq.q_pos, pq.k_pos = _ptr(rope.q_pos), _ptr(rope.k_pos)
        pq.n_pos = int(rope.cos.shape[0])
    return pq


def quantize_qkv(q, k, v, s=None, s_inv=None, out: PackedQKV | None = None, stream=None, rope: Rope | None = None,
                 q_mean=None, s_bias=None) -> PackedQKV:
    """Quantize Q, K, V to the packed 4-bit operands, after (in order) RoPE
    (rope), Smooth-QK (s / s_inv) and the Q-Mean subtraction (q_mean, from
    q_mean(); the K pass then writes the score bias into s_bias [B,Hq,Nkv],
    allocated here when None and q_mean is given: read it from ``out.s_bias``)."""
    for x, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_input(x, n)
    B, Hq, Nq, D = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D or not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v shapes / dtypes do not match")
    if out is None:
        out = alloc_packed(B, Hq, Hkv, Nq, Nkv, D, q.device)
    if q_mean is not None and s_bias is None:
        s_bias = torch.empty(B, Hq, Nkv, dtype=torch.float32, device=q.device)
    st = out.struct()
    if rope is None and q_mean is None:
        L.check(L.load().hifa4_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], B, Hq, Hkv, Nq, Nkv, D,
                                            _ptr(s), _ptr(s_inv), ctypes.byref(st), _stream(stream)), "quantize_qkv")
    else:
        pq = _prequant(s, s_inv, rope, q_mean, s_bias)
        L.check(L.load().hifa4_quantize_qkv_ex(_ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], B, Hq, Hkv, Nq, Nkv, D,
                                               ctypes.byref(pq), ctypes.byref(st), _stream(stream)),
                "quantize_qkv_ex")
    out.s_bias = s_bias
    return out


def quantize_q(q, out: PackedQKV, s=None, rope: Rope | None = None, q_mean=None, stream=None) -> PackedQKV:
    """Quantize Q alone into ``out.qc`` / ``out.qs`` (e.g. a decode step's new
    queries into the Q buffers of a packed KV cache from quantize_kv), after
    RoPE (rope.q_pos), Smooth-QK (s) and the Q-Mean subtraction (q_mean), in
    that order; out's B, Hq, Hkv, Nq and D must match q."""
    _check_input(q, "q")
    B, Hq, Nq, D = q.shape
    if (B, Hq, Nq, D) != (out.B, out.Hq, out.Nq, out.D):
        raise ValueError("q does not match the packed operands' Q shape")
    pq = _prequant(s, s, rope, q_mean)
    st = out.struct()
    L.check(L.load().hifa4_quantize_q(_ptr(q), _DT[q.dtype], B, Hq, out.Hkv, Nq, D, ctypes.byref(pq),
                                      ctypes.byref(st), _stream(stream)), "quantize_q")
    return out


def q_mean(q, s=None, rope: Rope | None = None, out=None, Hkv: int | None = None, stream=None) -> torch.Tensor:
    """Q-Mean auxiliary: per-(b, h, channel) mean [B,Hq,D] fp32 of Q after RoPE
    and smoothing (s needs Hkv, the kv heads it is indexed by)."""
    _check_input(q, "q")
    B, Hq, Nq, D = q.shape
    if Hkv is None:
        Hkv = s.shape[0] if s is not None else Hq
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    pq = _prequant(s, s, rope)
    L.check(L.load().hifa4_q_mean(_ptr(q), _DT[q.dtype], B, Hq, Hkv, Nq, D, ctypes.byref(pq), _ptr(out),
                                  _stream(stream)), "q_mean")
    return out


def quantize_kv(k, v, s_inv=None, out: PackedQKV | None = None, Hq: int | None = None, Nq: int = 16,
                stream=None) -> PackedQKV:
    """Quantize K and V only (a whole KV cache at once; see append_kv)."""
    _check_input(k, "k")
    _check_input(v, "v")
    B, Hkv, Nkv, D = k.shape
    if out is None:
        out = alloc_packed(B, Hq or Hkv, Hkv, Nq, Nkv, D, k.device)
    st = out.struct()
    L.check(L.load().hifa4_quantize_kv(_ptr(k), _ptr(v), _DT[k.dtype], B, Hkv, Nkv, D, _ptr(s_inv),
                                       ctypes.byref(st), _stream(stream)), "quantize_kv")
    return out


def append_kv(cache: PackedQKV, k_new, v_new, start: int, s_inv=None, rope: Rope | None = None,
              stream=None) -> PackedQKV:
    """Quantize new K/V tokens [B,Hkv,n_new,D] into cache token slots
    [start, start + n_new) (both multiples of 16); RoPE uses rope.k_pos [n_new]."""
    _check_input(k_new, "k_new")
    _check_input(v_new, "v_new")
    B, Hkv, n_new, D = k_new.shape
    if v_new.shape != k_new.shape or (B, Hkv, D) != (cache.B, cache.Hkv, cache.D):
        raise ValueError("new tokens do not match the cache")
    pq = _prequant(s_inv, s_inv, rope)
    pq.s = None
    st = cache.struct()
    L.check(L.load().hifa4_append_kv(_ptr(k_new), _ptr(v_new), _DT[k_new.dtype], B, Hkv, n_new, D, ctypes.byref(pq),
                                     ctypes.byref(st), cache.Nkv, int(start), _stream(stream)), "append_kv")
    return cache


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


def attention_fwd_ex(packed: PackedQKV, sm_scale: float | None = None, causal: bool = False,
                     norm="p_reorder", out_dtype=torch.bfloat16, out=None, lse=None, workspace=None, stream=None,
                     split_kv: bool = False, s_bias=None, want_p: bool = False, want_tile_sums: bool = False,
                     tile_sums=None):
    """attention_fwd with the extras of hifa4_attention_fwd_ex: the score bias
    s_bias [B,Hq,Nkv] (Q-Mean), and optionally the P_hat dump and the
    per-(row, kv tile) sums (sum P_hat, sum P) [B,Hq,Nq,Nkv/128,2] (written
    into ``tile_sums`` when given, else into a zeroed new tensor).
    Returns dict(o, lse, p_codes, p_scales, tile_sums)."""
    sm_scale, flags, nm, out, lse, workspace = _attn_args(packed, sm_scale, causal, norm, out_dtype, out, lse,
                                                          workspace, True, split_kv)
    B, Hq, Hkv, Nq, Nkv, D = packed.shape
    dev = out.device
    pc = torch.zeros(B, Hq, Nq, Nkv // 2, dtype=torch.uint8, device=dev) if want_p else None
    ps = torch.zeros(B, Hq, Nq, Nkv // 16, dtype=torch.uint8, device=dev) if want_p else None
    ts = tile_sums
    if ts is None and want_tile_sums:
        ts = torch.zeros(B, Hq, Nq, Nkv // 128, 2, dtype=torch.float32, device=dev)
    if ts is not None and (ts.shape != (B, Hq, Nq, Nkv // 128, 2) or ts.dtype != torch.float32
                           or not ts.is_contiguous() or not ts.is_cuda):
        raise ValueError("tile_sums must be a contiguous float32 CUDA tensor [B, Hq, Nq, Nkv/128, 2]")
    if s_bias is not None and (s_bias.shape != (B, Hq, Nkv) or s_bias.dtype != torch.float32
                               or not s_bias.is_contiguous()):
        raise ValueError("s_bias must be a contiguous float32 [B, Hq, Nkv] tensor")
    ex = L.AttentionExtras(_ptr(s_bias), _ptr(pc), _ptr(ps), _ptr(ts))
    st = packed.struct()
    L.check(L.load().hifa4_attention_fwd_ex(ctypes.byref(st), B, Hq, Hkv, Nq, Nkv, D, float(sm_scale), flags, nm,
                                            _ptr(out), _DT[out.dtype], _ptr(lse), ctypes.byref(ex), _ptr(workspace),
                                            _stream(stream)), "attention_fwd_ex")
    return dict(o=out, lse=lse, p_codes=pc, p_scales=ps, tile_sums=ts)


def attention_fwd_q(q: torch.Tensor, kv: PackedQKV, s=None, sm_scale: float | None = None, causal: bool = False,
                    norm="p_reorder", out_dtype=torch.bfloat16, out=None, lse=None, workspace=None, stream=None):
    """Attention from unquantized Q (bf16/fp16 [B,Hq,Nq,D], D = 128) and packed K/V
    (``kv``: e.g. quantize_kv or append_kv): the kernel quantizes Q itself, with
    the optional Smooth-QK factors ``s`` [Hkv,D]. Same result as quantize_qkv +
    attention_fwd. Returns (O, LSE)."""
    _check_input(q, "q")
    B, Hq, Nq, D = q.shape
    if (B, D) != (kv.B, kv.D):
        raise ValueError("q does not match the packed K/V")
    Hkv, Nkv = kv.Hkv, kv.Nkv
    dev = q.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(B, Hq, Nq, D, dtype=out_dtype, device=dev)
    if lse is None:
        lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, Nq, Nkv, D, dev)
    st = kv.struct()
    L.check(L.load().hifa4_attention_fwd_q(_ptr(q), _DT[q.dtype], _ptr(s), ctypes.byref(st), B, Hq, Hkv, Nq, Nkv, D,
                                           float(sm_scale), L.CAUSAL if causal else 0, _NORM[norm], _ptr(out),
                                           _DT[out.dtype], _ptr(lse), _ptr(workspace), _stream(stream)),
            "attention_fwd_q")
    return out, lse


def tile_stats(tile_sums: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """Per-tile epsilon-bar [B,Hq,ceil(Nq/128),Nkv/128] (NaN: tile without mass)
    from the tile sums of attention_fwd_ex."""
    _check_input(tile_sums, "tile_sums", 5)
    B, Hq, Nq, T, two = tile_sums.shape
    if two != 2 or tile_sums.dtype != torch.float32:
        raise ValueError("tile_sums must be float32 [B, Hq, Nq, Nkv/128, 2]")
    if out is None:
        out = torch.empty(B, Hq, (Nq + 127) // 128, T, dtype=torch.float32, device=tile_sums.device)
    L.check(L.load().hifa4_tile_stats(_ptr(tile_sums), B, Hq, Nq, T * 128, _ptr(out), _stream(stream)), "tile_stats")
    return out


def get_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return (and clear) the status a kernel recorded."""
    return int(L.load().hifa4_get_status(_ptr(workspace), _stream(stream)))


def debug_set_wait_limit(limit_ns: int, stall_loads: bool = False) -> int:
    return int(L.load().hifa4_debug_set_wait_limit(int(limit_ns), 1 if stall_loads else 0))
