"""Helpers shared by the GPU parity tests: uploading seeded inputs, and the
bijection between the library's MMA-ready scale layout and the canonical one
the oracle produces (see include/hifa4.h)."""
from __future__ import annotations

import numpy as np
import torch

import workloads as W

TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def to_device(x: np.ndarray, dtype: str) -> torch.Tensor:
    """float32 array holding exact bf16/fp16 values -> CUDA tensor of that dtype (bit-exact)."""
    bits = W.to_bits(x, dtype)
    t = torch.from_numpy(bits.view(np.int16).copy())
    return t.cuda().view(TORCH_DT[dtype])


def _atom(r):
    r = np.asarray(r)
    return 16 * (r % 32) + 4 * ((r // 32) % 4)


def qk_scale_index(B, H, Hkv, N, D):
    """Byte index into the MMA-ready Q/K scale buffer for every canonical scale [B,H,N,D/16]."""
    G = H // Hkv
    Tq = (G * N + 127) // 128
    KS = D // 64
    b, h, i, kb = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), np.arange(D // 16), indexing="ij")
    g = h // G
    p = (h % G) * N + i
    t, r = p // 128, p % 128
    s, k = kb // 4, kb % 4
    return (((b * Hkv + g) * Tq + t) * KS + s) * 512 + _atom(r) + k


def v_scale_index(B, Hkv, N, D):
    """Byte index into the MMA-ready V scale buffer for every canonical scale [B,Hkv,D,N/16]."""
    NT = N // 128
    NRB = (D + 127) // 128
    b, g, d, nb = np.meshgrid(np.arange(B), np.arange(Hkv), np.arange(D), np.arange(N // 16), indexing="ij")
    j, s, k = nb // 8, (nb % 8) // 4, nb % 4
    rb, r = d // 128, d % 128
    return ((((b * Hkv + g) * NT + j) * NRB + rb) * 2 + s) * 512 + _atom(r) + k


def canonical_vtc(vtc_tiled, B, Hkv, Nkv, D) -> np.ndarray:
    """Tiled V codes [B,Hkv,Nkv/128,D,64] (device or host) -> canonical Vtc [B,Hkv,D,Nkv/2]."""
    a = vtc_tiled.cpu().numpy() if hasattr(vtc_tiled, "cpu") else np.asarray(vtc_tiled)
    return np.ascontiguousarray(a.reshape(B, Hkv, Nkv // 128, D, 64).transpose(0, 1, 3, 2, 4).reshape(B, Hkv, D, Nkv // 2))


def canonical_scales(packed, B, Hq, Hkv, Nq, Nkv, D):
    """Device packed buffers -> canonical numpy (qs [B,Hq,Nq,D/16], ks, vts)."""
    qs_raw = packed.qs.cpu().numpy()
    ks_raw = packed.ks.cpu().numpy()
    vs_raw = packed.vts.cpu().numpy()
    qs = qs_raw[qk_scale_index(B, Hq, Hkv, Nq, D)]
    ks = ks_raw[qk_scale_index(B, Hkv, Hkv, Nkv, D)]
    vts = vs_raw[v_scale_index(B, Hkv, Nkv, D)]
    return qs, ks, vts


def padding_bytes_ok(packed, B, Hq, Hkv, Nq, Nkv, D) -> bool:
    """Bytes of the scale buffers that hold no canonical scale: zero, except the
    normalizer row (row 64 = 0x38) of the V atoms when D = 64."""
    qs_raw = packed.qs.cpu().numpy()
    used = np.zeros(qs_raw.size, bool)
    used[qk_scale_index(B, Hq, Hkv, Nq, D).ravel()] = True
    if np.any(qs_raw[~used] != 0):
        return False
    vs_raw = packed.vts.cpu().numpy()
    used = np.zeros(vs_raw.size, bool)
    used[v_scale_index(B, Hkv, Nkv, D).ravel()] = True
    pad = vs_raw[~used]
    if D >= 128:
        return pad.size == 0
    # rows 64..127 of every atom; row 64 holds 1.0 for all four scales
    atoms = vs_raw.reshape(-1, 512)
    row64 = atoms[:, [_atom(64) + k for k in range(4)]]
    others = np.ones(512, bool)
    others[[_atom(r) + k for r in range(64) for k in range(4)]] = False
    others[[_atom(64) + k for k in range(4)]] = False
    return bool(np.all(row64 == 0x38) and np.all(atoms[:, others] == 0))


def row_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    """Max abs error and per-row relative L2 (absolute where the row norm < 1e-6)."""
    diff = o_gpu.astype(np.float64) - o_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    num = np.linalg.norm(diff, axis=-1)
    den = np.linalg.norm(o_ref, axis=-1)
    rel = np.where(den < 1e-6, num, num / np.maximum(den, 1e-30))
    return max_abs, rel


def upload_config(cfg, device="cuda"):
    """Seeded inputs of a workload config on the device, built slice by slice.
    Returns (q, k, v, calib) with calib = (Qcal, Kcal) device tensors or None."""
    dt = TORCH_DT[cfg.dtype]
    gains = W.k_gains(cfg)

    def up(x):
        return torch.from_numpy(W.to_bits(x, cfg.dtype).view(np.int16).copy()).to(device).view(dt)

    q = torch.empty(cfg.B, cfg.Hq, cfg.Nq, cfg.D, dtype=dt, device=device)
    k = torch.empty(cfg.B, cfg.Hkv, cfg.Nkv, cfg.D, dtype=dt, device=device)
    v = torch.empty_like(k)
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            q[b, h] = up(W.q_slice(cfg, b, h))
        for g in range(cfg.Hkv):
            k[b, g] = up(W.k_slice(cfg, b, g, gains))
            v[b, g] = up(W.v_slice(cfg, b, g))
    calib = None
    if cfg.smooth == "calib":
        calib = (torch.stack([up(W.qcal_slice(cfg, h)) for h in range(cfg.Hq)])[None].contiguous(),
                 torch.stack([up(W.kcal_slice(cfg, g, gains)) for g in range(cfg.Hkv)])[None].contiguous())
    elif cfg.smooth == "self":
        calib = (q, k)
    return q, k, v, calib


def group_arrays(cfg, b, g):
    """Host copies (exact dtype values, float32) of one (batch, kv head) group:
    q [1,G,Nq,D], k [1,1,Nkv,D], v [1,1,Nkv,D]."""
    gains = W.k_gains(cfg)
    q = np.stack([W.q_slice(cfg, b, g * cfg.G + hh) for hh in range(cfg.G)])[None]
    k = W.k_slice(cfg, b, g, gains)[None, None]
    v = W.v_slice(cfg, b, g)[None, None]
    return q, k, v


def calib_arrays(cfg):
    """Host calibration tensors of a config (None when smoothing is off)."""
    if cfg.smooth == "off":
        return None
    if cfg.smooth == "self":
        q, k, _ = W.full(cfg)
        return q, k
    return W.calib_full(cfg)
