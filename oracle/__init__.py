"""CPU oracle of the 4-bit FlashAttention forward (HiFA4 reading), via ctypes.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use this package; the product package never
imports it. The arithmetic lives in ``hifa4_oracle.c`` (plain C, built with
``build()``); this file only marshals numpy arrays.

Parity status of each function (what pins it, see tests/test_oracle_pins.py):
  e2m1/e4m3 encode+decode  pinned: closed-form code tables, midpoint ties,
                           sweeps against ml_dtypes and torch float8 casts
  quantize_rows/_v         pinned: worked blocks in tests/golden, error bound,
                           independent NumPy restatement (np_ref)
  calibrate                pinned: hand-built 2-channel example, zero channel
  qk_row                   pinned: exact rational dot products (fractions)
  rope_neox                pinned: identity and quarter-turn tables (exact),
                           pair norms, relative-position invariance
  q_mean / sub_mean        pinned: hand-built means, exact shift
  q_mean_bias              pinned: K' = 1 closed form, brute force
  eps_bar                  pinned: hand-built per-row values with empty rows
  attention_rows           pinned: brute-force fp64 softmax attention with
                           quantization off (causal, GQA, ragged Nq), V = 1
                           invariants for both normalizer modes, convex-hull
                           bound, NumPy restatement on the tiny config;
                           with the Q-Mean bias: constant-Q rows against the
                           brute-force log-sum-exp of the exact scores
  The whole quantized output has no published values to compare with; beyond
  the pieces above its parity is pinned only through those pieces.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hifa4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

P_REORDER = 0
HIGH_PRECISION_L = 1


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        vp = ctypes.c_void_p
        ci, cf, cll = ctypes.c_int, ctypes.c_float, ctypes.c_longlong
        L.ora_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.ora_e2m1_decode.restype = ctypes.c_double
        L.ora_e2m1_encode.argtypes = [cf]
        L.ora_e2m1_encode.restype = ctypes.c_uint8
        L.ora_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.ora_e4m3_decode.restype = ctypes.c_double
        L.ora_e4m3_encode.argtypes = [cf]
        L.ora_e4m3_encode.restype = ctypes.c_uint8
        L.ora_scale_code.argtypes = [cf]
        L.ora_scale_code.restype = ctypes.c_uint8
        L.ora_quant_block16.argtypes = [f32p, u8p, u8p]
        L.ora_quant_block16.restype = None
        L.ora_calibrate.argtypes = [f32p, f32p, ci, ci, ci, ci, ci, cf, f32p, f32p]
        L.ora_calibrate.restype = None
        L.ora_quantize_rows.argtypes = [f32p, ci, ci, ci, ci, ci, vp, u8p, u8p]
        L.ora_quantize_rows.restype = None
        L.ora_quantize_v.argtypes = [f32p, ci, ci, ci, ci, u8p, u8p]
        L.ora_quantize_v.restype = None
        L.ora_qk_row.argtypes = [u8p, u8p, u8p, u8p, ci, ci, ci, ci, ci, cll, f32p]
        L.ora_qk_row.restype = None
        L.ora_attention_rows.argtypes = [vp] * 9 + [ci] * 6 + [cf, ci, ci, ci, ci, vp, i64p, cll] + [vp] * 7 + [ci]
        L.ora_attention_rows.restype = ci
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        L.ora_rope_neox.argtypes = [f32p, cll, ci, f32p, f32p, i32p]
        L.ora_rope_neox.restype = None
        L.ora_smooth_rows.argtypes = [f32p, ci, ci, ci, ci, ci, f32p]
        L.ora_smooth_rows.restype = None
        L.ora_q_mean.argtypes = [f32p, cll, ci, ci, f32p]
        L.ora_q_mean.restype = None
        L.ora_sub_mean.argtypes = [f32p, cll, ci, ci, f32p]
        L.ora_sub_mean.restype = None
        L.ora_q_mean_bias.argtypes = [f32p, f32p, ci, ci, ci, ci, ci, f64p]
        L.ora_q_mean_bias.restype = None
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------------ formats

def e2m1_encode(x) -> np.ndarray:
    L = lib()
    x = np.asarray(x, np.float32).ravel()
    return np.array([L.ora_e2m1_encode(float(v)) for v in x], np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.ora_e2m1_decode(int(c)) for c in np.asarray(codes).ravel()], np.float64)


def e4m3_encode(x) -> np.ndarray:
    L = lib()
    x = np.asarray(x, np.float32).ravel()
    return np.array([L.ora_e4m3_encode(float(v)) for v in x], np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.ora_e4m3_decode(int(c)) for c in np.asarray(codes).ravel()], np.float64)


def quant_block16(x):
    x = np.ascontiguousarray(x, np.float32)
    assert x.shape == (16,)
    codes = np.zeros(16, np.uint8)
    sf = np.zeros(1, np.uint8)
    lib().ora_quant_block16(x, codes, sf)
    return codes, int(sf[0])


# ----------------------------------------------------------- path steps

def calibrate(q: np.ndarray, k: np.ndarray, alpha: float = 0.5):
    """Smooth-QK factors s, s_inv [Hkv, D] from q [B,Hq,N,D], k [B,Hkv,N,D] (float32)."""
    q = np.ascontiguousarray(q, np.float32)
    k = np.ascontiguousarray(k, np.float32)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    s = np.zeros((Hkv, D), np.float32)
    si = np.zeros((Hkv, D), np.float32)
    lib().ora_calibrate(q, k, B, Hq, Hkv, N, D, float(alpha), s, si)
    return s, si


def quantize_rows(x: np.ndarray, scale: np.ndarray | None = None, group: int = 1):
    """Q or K [B,H,N,D] -> (codes [B,H,N,D/2], scales [B,H,N,D/16]); scale = s (Q) or s_inv (K)."""
    x = np.ascontiguousarray(x, np.float32)
    B, H, N, D = x.shape
    codes = np.zeros((B, H, N, D // 2), np.uint8)
    sf = np.zeros((B, H, N, D // 16), np.uint8)
    sc = None if scale is None else np.ascontiguousarray(scale, np.float32)
    lib().ora_quantize_rows(x, B, H, N, D, group, _ptr(sc), codes, sf)
    return codes, sf


def quantize_v(v: np.ndarray):
    """V [B,Hkv,N,D] -> (vtc [B,Hkv,D,N/2], vts [B,Hkv,D,N/16]), quantized along tokens."""
    v = np.ascontiguousarray(v, np.float32)
    B, H, N, D = v.shape
    vtc = np.zeros((B, H, D, N // 2), np.uint8)
    vts = np.zeros((B, H, D, N // 16), np.uint8)
    lib().ora_quantize_v(v, B, H, N, D, vtc, vts)
    return vtc, vts


def quantize_qkv(q, k, v, s=None, s_inv=None):
    Hq, Hkv = q.shape[1], k.shape[1]
    qc, qs = quantize_rows(q, s, Hq // Hkv)
    kc, ks = quantize_rows(k, s_inv, 1)
    vtc, vts = quantize_v(v)
    return dict(qc=qc, qs=qs, kc=kc, ks=ks, vtc=vtc, vts=vts)


# ------------------------------------------- steps before quantization

def rope_neox(x: np.ndarray, cos_t: np.ndarray, sin_t: np.ndarray, pos) -> np.ndarray:
    """RoPE with rotate-half pairing on x [B,H,N,D] (float32; returns a new array).

    Token i of every (b, h) sits at position pos[i]; cos_t / sin_t are the
    caller's tables [n_pos, D/2]. Op order in hifa4_oracle.c (ora_rope_neox).
    """
    x = np.array(x, np.float32, copy=True, order="C")
    B, H, N, D = x.shape
    pos = np.ascontiguousarray(np.asarray(pos, np.int32))
    assert pos.shape == (N,)
    rows_pos = np.ascontiguousarray(np.tile(pos, B * H))
    lib().ora_rope_neox(x, B * H * N, D, np.ascontiguousarray(cos_t, np.float32),
                        np.ascontiguousarray(sin_t, np.float32), rows_pos)
    return x


def smooth_rows(x: np.ndarray, scale: np.ndarray, group: int = 1) -> np.ndarray:
    """Smooth-QK multiply RN(x * scale[h/group]) on x [B,H,N,D] (new array)."""
    x = np.array(x, np.float32, copy=True, order="C")
    B, H, N, D = x.shape
    lib().ora_smooth_rows(x, B, H, N, D, int(group), np.ascontiguousarray(scale, np.float32))
    return x


def q_mean(x: np.ndarray) -> np.ndarray:
    """Q-Mean: per-(b, h, channel) mean over tokens of x [B,H,N,D] -> [B,H,D] float32."""
    x = np.ascontiguousarray(x, np.float32)
    B, H, N, D = x.shape
    m = np.zeros((B, H, D), np.float32)
    lib().ora_q_mean(x, B * H, N, D, m)
    return m


def sub_mean(x: np.ndarray, mean: np.ndarray) -> np.ndarray:
    """RN(x - mean[b,h]) on x [B,H,N,D] (new array)."""
    x = np.array(x, np.float32, copy=True, order="C")
    B, H, N, D = x.shape
    lib().ora_sub_mean(x, B * H, N, D, np.ascontiguousarray(mean, np.float32))
    return x


def prequant_rows(x: np.ndarray, *, rope=None, scale=None, group: int = 1, mean=None) -> np.ndarray:
    """The steps before quantization of Q or K, in order: RoPE (rope = (cos_t,
    sin_t, pos)), the Smooth-QK multiply (scale), the Q-Mean subtraction (mean)."""
    y = np.ascontiguousarray(x, np.float32)
    if rope is not None:
        y = rope_neox(y, *rope)
    if scale is not None:
        y = smooth_rows(y, scale, group)
    if mean is not None:
        y = sub_mean(y, mean)
    return y


def q_mean_bias(mean: np.ndarray, k_pre: np.ndarray, Hq: int) -> np.ndarray:
    """bias [B,Hq,Nkv] float64 = mean . K'^T per head, K' [B,Hkv,Nkv,D] the
    keys as they enter quantization (after RoPE / smoothing)."""
    mean = np.ascontiguousarray(mean, np.float32)
    kf = np.ascontiguousarray(k_pre, np.float32)
    B, Hkv, Nkv, D = kf.shape
    bias = np.zeros((B, Hq, Nkv), np.float64)
    lib().ora_q_mean_bias(mean, kf, B, Hq, Hkv, Nkv, D, bias)
    return bias


def eps_bar(eps_rows: np.ndarray, B: int, Hq: int, Nq: int) -> np.ndarray:
    """Per-tile mean of the per-(row, kv tile) epsilon (NaN = row without mass).

    eps_rows [B*Hq*Nq, T] (attention_rows(..., want_eps=True) over all rows).
    A tile is 128 query rows of one (b, h) x one 128-key tile; the mean runs
    over the tile's rows with mass, NaN when none has any.
    Returns [B, Hq, ceil(Nq/128), T] float64.
    """
    T = eps_rows.shape[1]
    e = np.asarray(eps_rows, np.float64).reshape(B, Hq, Nq, T)
    nqa = (Nq + 127) // 128
    out = np.full((B, Hq, nqa, T), np.nan)
    for a in range(nqa):
        blk = e[:, :, 128 * a:128 * (a + 1), :]
        cnt = np.sum(~np.isnan(blk), axis=2)
        tot = np.nansum(blk, axis=2)
        with np.errstate(invalid="ignore", divide="ignore"):
            out[:, :, a, :] = np.where(cnt > 0, tot / np.maximum(cnt, 1), np.nan)
    return out


def qk_row(packed, Hq, Hkv, Nq, Nkv, D, row):
    S = np.zeros(Nkv, np.float32)
    p = {k: np.ascontiguousarray(a) for k, a in packed.items()}
    lib().ora_qk_row(p["qc"], p["qs"], p["kc"], p["ks"], Hq, Hkv, Nq, Nkv, D, int(row), S)
    return S


def default_sm_scale(D: int) -> float:
    return float(np.float32(1.0 / np.sqrt(float(D))))


def attention_rows(shape, rows, *, packed=None, fp32=None, sm_scale=None, causal=False,
                   norm_mode=P_REORDER, want_eps=False, want_p=False, n_threads=0, n_splits=1,
                   s_bias=None):
    """Run the oracle on selected query rows.

    shape: (B, Hq, Hkv, Nq, Nkv, D). rows: flat ids (b*Hq + h)*Nq + i.
    packed: dict of canonical quantized operands (4-bit path), or
    fp32: (q, k, v) float32 operands (quantization off).
    n_splits: kv split count (contiguous ranges of 128-key tiles, each with its
    own online softmax, merged by log-sum-exp weights); 1 = one pass.
    l_hat / l_hp are reported in the frame of the merged max.
    s_bias: [B,Hq,Nkv] float64 score term added before the fp32 rounding of
    each score (the Q-Mean auxiliary, see q_mean_bias; 4-bit path only).
    Returns dict with O [n,D] f64, lse [n], l_hat [n], l_hp [n] and optionally
    eps [n, Nkv/128], p_codes [n, Nkv/2], p_sf [n, Nkv/16].
    """
    B, Hq, Hkv, Nq, Nkv, D = shape
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    n = rows.size
    if sm_scale is None:
        sm_scale = default_sm_scale(D)
    O = np.zeros((n, D), np.float64)
    lse = np.zeros(n, np.float64)
    lh = np.zeros(n, np.float64)
    lp = np.zeros(n, np.float64)
    eps = np.zeros((n, Nkv // 128), np.float64) if want_eps else None
    pc = np.zeros((n, Nkv // 2), np.uint8) if want_p else None
    ps = np.zeros((n, Nkv // 16), np.uint8) if want_p else None
    if packed is not None:
        p = {k: np.ascontiguousarray(a) for k, a in packed.items()}
        args = [_ptr(p["qc"]), _ptr(p["qs"]), _ptr(p["kc"]), _ptr(p["ks"]), _ptr(p["vtc"]), _ptr(p["vts"]),
                None, None, None]
        quant = 1
        keep = p
    else:
        qf, kf, vf = (np.ascontiguousarray(a, np.float32) for a in fp32)
        args = [None] * 6 + [_ptr(qf), _ptr(kf), _ptr(vf)]
        quant = 0
        keep = (qf, kf, vf)
    qm = None if s_bias is None else np.ascontiguousarray(s_bias, np.float64)
    if qm is not None:
        assert qm.shape == (B, Hq, Nkv)
    rc = lib().ora_attention_rows(*args, B, Hq, Hkv, Nq, Nkv, D, float(sm_scale), int(bool(causal)),
                                  int(norm_mode), quant, int(n_splits), _ptr(qm), rows, n,
                                  _ptr(O), _ptr(lse), _ptr(lh), _ptr(lp),
                                  _ptr(eps), _ptr(pc), _ptr(ps), int(n_threads))
    del keep
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    out = dict(O=O, lse=lse, l_hat=lh, l_hp=lp)
    if want_eps:
        out["eps"] = eps
    if want_p:
        out["p_codes"], out["p_sf"] = pc, ps
    return out


def all_rows(B, Hq, Nq):
    return np.arange(B * Hq * Nq, dtype=np.int64)
