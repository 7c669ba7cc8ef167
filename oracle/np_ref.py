"""Independent NumPy restatement of the quantized attention (small inputs only).

TEST INFRASTRUCTURE ONLY. It exists to cross-check the C oracle: it shares no
code with it and takes its format conversions from a different source
(``ml_dtypes`` float4_e2m1fn / float8_e4m3fn casts, both round-to-nearest-even).
It follows the same readings of the HiFA4 abstract (smooth, quantize per 16 along
the contraction dimension, one pass over 128-key tiles with the running max
updated per tile, P quantized per 16 keys, normalizer from P_hat or from P).
Vectorised over all query rows at once, so it is only for tiny shapes.
"""
from __future__ import annotations

import ml_dtypes
import numpy as np

_F4 = ml_dtypes.float4_e2m1fn
_F8 = ml_dtypes.float8_e4m3fn
_ONE_SIXTH = np.float32(1.0) / np.float32(6.0)


def _e4m3_sat(x32: np.ndarray) -> np.ndarray:
    # ml_dtypes maps values above the largest finite E4M3 to NaN; clamp first
    # (satfinite): any value >= 448 encodes to 448.
    return np.minimum(x32, np.float32(448.0)).astype(_F8)


def quantize_blocks(x: np.ndarray):
    """x float32 [..., n*16] grouped by 16 along the last axis.

    Returns (decoded float64 values, nibble codes uint8, scale codes uint8)."""
    x = np.asarray(x, np.float32)
    shp = x.shape
    xb = x.reshape(shp[:-1] + (shp[-1] // 16, 16))
    amax = np.abs(xb).max(axis=-1)
    sf8 = _e4m3_sat((amax * _ONE_SIXTH).astype(np.float32))
    S = sf8.astype(np.float32)
    with np.errstate(divide="ignore"):
        r = np.where(S == 0, np.float32(0), np.float32(1) / np.where(S == 0, np.float32(1), S)).astype(np.float32)
    y = (xb * r[..., None]).astype(np.float32)
    y = np.clip(y, np.float32(-6), np.float32(6))
    q4 = y.astype(_F4)
    codes = q4.view(np.uint8) & np.uint8(0xF)
    dec = q4.astype(np.float64) * S.astype(np.float64)[..., None]
    return dec.reshape(shp), codes.reshape(shp), sf8.view(np.uint8)


def pack(codes: np.ndarray) -> np.ndarray:
    c = codes.reshape(codes.shape[:-1] + (codes.shape[-1] // 2, 2))
    return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8)


def calibrate(q, k, alpha=0.5):
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    aq = np.abs(q).reshape(B, Hkv, G, N, D).max(axis=(0, 2, 3)).astype(np.float32)
    ak = np.abs(k).max(axis=(0, 2)).astype(np.float32)
    ok = (aq > 0) & (ak > 0)
    if alpha == 0.5:
        ratio = (ak.astype(np.float64) / np.where(ok, aq, 1).astype(np.float64)).astype(np.float32)
        s = np.sqrt(ratio.astype(np.float64)).astype(np.float32)
    else:
        s = (ak.astype(np.float64) ** alpha / np.where(ok, aq, 1).astype(np.float64) ** (1 - alpha)).astype(np.float32)
    s = np.where(ok, s, np.float32(1)).astype(np.float32)
    s_inv = (1.0 / s.astype(np.float64)).astype(np.float32)
    return s, s_inv


def attention(q, k, v, *, s=None, s_inv=None, causal=False, norm_mode=0, sm_scale=None, tile=128):
    """Full 4-bit path on q [B,Hq,Nq,D], k/v [B,Hkv,Nkv,D] (float32).

    Returns dict(O [B,Hq,Nq,D] f64, lse, q/k/v codes and scales in canonical
    layout, p_codes [B,Hq,Nq,Nkv/2], p_sf [B,Hq,Nq,Nkv/16])."""
    B, Hq, Nq, D = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = np.float32(1.0 / np.sqrt(float(D)))
    c = np.float32(np.float64(sm_scale) * np.log2(np.e))
    if s is not None:
        sq = np.repeat(s, G, axis=0)                       # [Hq, D]
        q = (q * sq[None, :, None, :]).astype(np.float32)
        k = (k * s_inv[None, :, None, :]).astype(np.float32)
    qd, qcodes, qsf = quantize_blocks(q)
    kd, kcodes, ksf = quantize_blocks(k)
    vt = np.swapaxes(v, 2, 3)                              # [B,Hkv,D,Nkv]
    vd_t, vcodes, vsf = quantize_blocks(vt)
    vd = np.swapaxes(vd_t, 2, 3)                           # [B,Hkv,Nkv,D]
    kd_h = np.repeat(kd, G, axis=1)                        # [B,Hq,Nkv,D]
    vd_h = np.repeat(vd, G, axis=1)
    S_all = np.einsum("bhid,bhjd->bhij", qd, kd_h).astype(np.float32)
    ii = np.arange(Nq)[:, None]
    jj = np.arange(Nkv)[None, :]
    visible = (jj <= ii + Nkv - Nq) if causal else np.ones((Nq, Nkv), bool)
    S_all = np.where(visible[None, None], S_all, np.float32(-np.inf))

    m = np.full((B, Hq, Nq), -np.inf, np.float32)
    mc = np.zeros((B, Hq, Nq), np.float32)
    oacc = np.zeros((B, Hq, Nq, D))
    l_hat = np.zeros((B, Hq, Nq))
    l_hp = np.zeros((B, Hq, Nq))
    p_codes = np.zeros((B, Hq, Nq, Nkv), np.uint8)
    p_sf = np.zeros((B, Hq, Nq, Nkv // 16), np.uint8)
    for t in range(Nkv // tile):
        sl = slice(t * tile, (t + 1) * tile)
        St = S_all[..., sl]
        live = np.isfinite(St).any(axis=-1)                # rows with a visible key in the tile
        m_new = np.maximum(m, St.max(axis=-1)).astype(np.float32)
        mc_new = (m_new.astype(np.float64) * np.float64(c)).astype(np.float32)
        with np.errstate(invalid="ignore", over="ignore"):
            alpha = np.where(np.isneginf(m), 0.0, np.exp2(mc.astype(np.float64) - mc_new.astype(np.float64)))
            # fma(S, c, -mc): S*c is exact in float64; the difference is rounded to
            # float64 and then to float32. That differs from a single rounding only
            # when the float64 result lands exactly on a float32 midpoint (odds of
            # about 2^-29 per element), so the cross-check tolerates no mismatch.
            t_arg = (St.astype(np.float64) * np.float64(c) - mc_new[..., None].astype(np.float64)).astype(np.float32)
            P = np.where(np.isneginf(St), np.float32(0), np.exp2(t_arg.astype(np.float64)).astype(np.float32))
        P = P.astype(np.float32)
        Pd, pcodes_t, psf_t = quantize_blocks(P)
        oacc_new = alpha[..., None] * oacc + np.einsum("bhij,bhjd->bhid", Pd, vd_h[..., sl, :])
        lh_new = alpha * l_hat + Pd.sum(axis=-1)
        lp_new = alpha * l_hp + P.astype(np.float64).sum(axis=-1)
        # rows with no visible key in this tile keep their state (the oracle skips the tile)
        oacc = np.where(live[..., None], oacc_new, oacc)
        l_hat = np.where(live, lh_new, l_hat)
        l_hp = np.where(live, lp_new, l_hp)
        p_codes[..., sl] = np.where(live[..., None], pcodes_t, 0)
        p_sf[..., t * tile // 16:(t + 1) * tile // 16] = np.where(live[..., None], psf_t, 0)
        m = np.where(live, m_new, m)
        mc = np.where(live, mc_new, mc)
    l = l_hat if norm_mode == 0 else l_hp
    O = oacc / l[..., None]
    lse = mc.astype(np.float64) * np.log(2.0) + np.log(l)
    return dict(O=O, lse=lse, l_hat=l_hat, l_hp=l_hp,
                qc=pack(qcodes), qs=qsf, kc=pack(kcodes), ks=ksf, vtc=pack(vcodes), vts=vsf,
                p_codes=pack(p_codes), p_sf=p_sf)
