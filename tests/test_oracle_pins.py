"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: closed-form
code tables of E2M1/E4M3, independent conversions (ml_dtypes, torch float8),
hand-derived worked blocks (tests/golden), exact rational arithmetic, the
textbook softmax attention (quantization off), the P-Reordering invariants the
HiFA4 abstract states (normalizer and numerator from the same P_hat), and an
independent NumPy restatement on the tiny config.
"""
import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import np_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ formats

def test_e2m1_code_table_closed_form():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    want = mags + [-m for m in mags]
    got = oracle.e2m1_decode(np.arange(16))
    assert np.array_equal(got, np.array(want))
    assert np.signbit(got[8])                                   # code 8 is -0
    # every code is a fixed point of encode(decode(.))
    assert np.array_equal(oracle.e2m1_encode(got.astype(np.float32)), np.arange(16))


def test_e2m1_midpoints_round_to_even():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    want = [0, 2, 2, 4, 4, 6, 6]
    assert list(oracle.e2m1_encode(mids)) == want
    assert list(oracle.e2m1_encode(-mids)) == [w | 8 for w in want]
    # just above / below each midpoint
    up = np.nextafter(mids, np.float32(10))
    dn = np.nextafter(mids, np.float32(-10))
    assert list(oracle.e2m1_encode(up)) == [1, 2, 3, 4, 5, 6, 7]
    assert list(oracle.e2m1_encode(dn)) == [0, 1, 2, 3, 4, 5, 6]
    assert list(oracle.e2m1_encode(np.array([6.0, 7.0, 1e30, -1e30], np.float32))) == [7, 7, 7, 15]


def test_e2m1_sweep_matches_ml_dtypes():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-7, 7, 4000), rng.standard_normal(2000) * 0.3,
                        np.arange(-6.5, 6.5, 0.125)]).astype(np.float32)
    ref = np.clip(x, -6, 6).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(oracle.e2m1_encode(x), ref)


def _e4m3_closed_form(c):
    e, m = (c >> 3) & 15, c & 7
    return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)


def test_e4m3_code_table_closed_form():
    codes = np.arange(0x7F)
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(got, np.array([_e4m3_closed_form(int(c)) for c in codes]))
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0
    assert np.array_equal(oracle.e4m3_encode(got.astype(np.float32)), codes)
    assert np.isnan(oracle.e4m3_decode([0x7F])[0])


def test_e4m3_sweep_matches_torch_and_ml_dtypes():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-14, 6, 3000)),
                        rng.uniform(0, 2 ** -6, 1000)]).astype(np.float32)
    ours = oracle.e4m3_encode(x)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    m = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, t)
    assert np.array_equal(ours, m)


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e20], np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E] * 6


def test_scale_constant_is_rn_one_sixth():
    # 6 * 2^k times RN(1/6) rounds back to 2^k in fp32, so the scale is exactly 2^k
    for k in range(-9, 7):
        assert oracle.e4m3_decode([oracle.lib().ora_scale_code(float(6.0 * 2.0 ** k))])[0] == 2.0 ** k
    assert np.float32(1 / 6).view(np.uint32) == 0x3E2AAAAB


# ------------------------------------------------------------ quantization

def test_golden_worked_blocks():
    doc = json.load(open(os.path.join(GOLDEN, "quant_blocks.json")))
    for b in doc["blocks"]:
        codes, sf = oracle.quant_block16(np.array(b["x"], np.float32))
        assert sf == b["sf"], b["name"]
        assert list(codes) == b["codes"], b["name"]
        dec = oracle.e2m1_decode(codes) * oracle.e4m3_decode([sf])[0]
        assert np.array_equal(dec, np.array(b["decoded"])), b["name"]


def test_quantization_error_bound():
    rng = np.random.default_rng(2)
    for scale in [1e-3, 0.05, 1.0, 30.0, 300.0]:
        for _ in range(200):
            x = (rng.standard_normal(16) * scale).astype(np.float32)
            codes, sf = oracle.quant_block16(x)
            S = oracle.e4m3_decode([sf])[0]
            xh = oracle.e2m1_decode(codes) * S
            amax = np.abs(x).max()
            y = np.abs(x) / S if S > 0 else np.zeros(16)
            half_step = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0)) * S
            sat = np.maximum(np.abs(x) - 6 * S, 0)
            bound = half_step + sat + 1e-6 * amax
            if S == 0:
                bound = np.full(16, 6 * 2.0 ** -10 + 1e-12)
            assert np.all(np.abs(xh - x) <= bound)


def test_quantize_layouts_place_one_element():
    B, H, N, D = 2, 3, 32, 64
    x = np.zeros((B, H, N, D), np.float32)
    b, h, n, d = 1, 2, 17, 37
    x[b, h, n, d] = 3.0
    qc, qs = oracle.quantize_rows(x)
    nz = np.argwhere(qc)
    assert nz.tolist() == [[b, h, n, d // 2]]
    assert qc[b, h, n, d // 2] == (7 << 4 if d % 2 else 7)       # 3 -> sf 0.5, 3*2 = 6 -> code 7
    assert np.argwhere(qs).tolist() == [[b, h, n, d // 16]]
    vtc, vts = oracle.quantize_v(x)                              # treat x as V [B,Hkv,N,D]
    assert np.argwhere(vtc).tolist() == [[b, h, d, n // 2]]
    assert vtc[b, h, d, n // 2] == (7 << 4 if n % 2 else 7)
    assert np.argwhere(vts).tolist() == [[b, h, d, n // 16]]


def test_smoothing_uses_kv_head_of_each_q_head():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, N, D = 1, 4, 2, 16, 32
    q = rng.standard_normal((B, Hq, N, D)).astype(np.float32)
    s = rng.uniform(0.5, 4, (Hkv, D)).astype(np.float32)
    qc, qs = oracle.quantize_rows(q, s, Hq // Hkv)
    pre = (q * np.repeat(s, Hq // Hkv, axis=0)[None, :, None, :]).astype(np.float32)
    qc2, qs2 = oracle.quantize_rows(pre)
    assert np.array_equal(qc, qc2) and np.array_equal(qs, qs2)


# -------------------------------------------------------------- calibration

def test_calibration_hand_example():
    # one kv head, two q heads in its group, two channels
    q = np.array([[[[1.0, 2.0], [-3.0, 0.5]], [[0.5, -1.0], [2.0, 0.25]]]], np.float32)   # [1,2,2,2]
    k = np.array([[[[4.0, -8.0], [1.0, 2.0]]]], np.float32)                                # [1,1,2,2]
    s, si = oracle.calibrate(q, k, 0.5)
    # aQ = (3, 2), aK = (4, 8) -> s = sqrt(aK/aQ)
    assert s[0, 0] == np.float32(np.sqrt(np.float64(np.float32(4 / 3))))
    assert s[0, 1] == np.float32(2.0)
    assert si[0, 1] == np.float32(0.5)
    assert si[0, 0] == np.float32(1.0 / np.float64(s[0, 0]))
    # alpha = 1 moves all of K's range: s = aK
    s1, _ = oracle.calibrate(q, k, 1.0)
    assert np.array_equal(s1, np.array([[4.0, 8.0]], np.float32))


def test_calibration_zero_channel_gives_one():
    q = np.ones((1, 1, 4, 16), np.float32)
    k = np.ones((1, 1, 4, 16), np.float32)
    q[..., 3] = 0
    k[..., 5] = 0
    s, si = oracle.calibrate(q, k)
    assert s[0, 3] == 1 and s[0, 5] == 1 and si[0, 3] == 1 and np.all(s == 1)


def test_calibration_matches_numpy_restatement():
    cfg = W.get(1)
    q, k, _ = W.full(cfg)
    s, si = oracle.calibrate(q, k)
    s2, si2 = np_ref.calibrate(q, k)
    assert np.array_equal(s, s2) and np.array_equal(si, si2)


# ---------------------------------------------------------------- QK scores

def test_qk_row_is_exact_rational_sum():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, Nq, Nkv, D = 2, 4, 2, 8, 128, 64
    q = (rng.standard_normal((B, Hq, Nq, D)) * 2).astype(np.float32)
    k = (rng.standard_normal((B, Hkv, Nkv, D)) * 3).astype(np.float32)
    v = rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32)
    pk = oracle.quantize_qkv(q, k, v)

    def dec(codes, sf):
        nib = np.stack([codes & 15, codes >> 4], -1).reshape(codes.shape[:-1] + (-1,))
        return [Fraction(float(a)) * Fraction(float(b)) for a, b in
                zip(oracle.e2m1_decode(nib.ravel()), np.repeat(oracle.e4m3_decode(sf.ravel()), 16))]

    for (b, h, i) in [(0, 0, 0), (1, 3, 5), (1, 2, 7)]:
        row = (b * Hq + h) * Nq + i
        S = oracle.qk_row(pk, Hq, Hkv, Nq, Nkv, D, row)
        qv = dec(pk["qc"][b, h, i], pk["qs"][b, h, i])
        g = h // (Hq // Hkv)
        for n in [0, 1, 63, 127]:
            kv = dec(pk["kc"][b, g, n], pk["ks"][b, g, n])
            exact = sum(a * c for a, c in zip(qv, kv))
            assert S[n] == np.float32(float(exact))


# ------------------------------------------------------- attention pins

def _bruteforce(q, k, v, causal, sm_scale):
    B, Hq, Nq, D = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    kh = np.repeat(k.astype(np.float64), G, axis=1)
    vh = np.repeat(v.astype(np.float64), G, axis=1)
    s = np.einsum("bhid,bhjd->bhij", q.astype(np.float64), kh) * sm_scale
    if causal:
        mask = np.arange(Nkv)[None, :] > np.arange(Nq)[:, None] + (Nkv - Nq)
        s = np.where(mask, -np.inf, s)
    mx = s.max(-1, keepdims=True)
    e = np.exp(s - mx)
    l = e.sum(-1, keepdims=True)
    return np.einsum("bhij,bhjd->bhid", e / l, vh), (mx + np.log(l))[..., 0]


@pytest.mark.parametrize("shape,causal", [
    ((1, 1, 1, 256, 256, 64), False),
    ((1, 2, 1, 256, 256, 64), True),
    ((2, 4, 2, 64, 384, 128), True),        # Nq < Nkv: bottom-right causal alignment, GQA 2
    ((1, 2, 2, 48, 256, 256), False),
])
def test_quant_off_matches_bruteforce_softmax_attention(shape, causal):
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(5)
    q = (rng.standard_normal((B, Hq, Nq, D)) * 1.5).astype(np.float32)
    k = (rng.standard_normal((B, Hkv, Nkv, D)) * 1.5).astype(np.float32)
    v = rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32)
    sm = oracle.default_sm_scale(D)
    out = oracle.attention_rows(shape, oracle.all_rows(B, Hq, Nq), fp32=(q, k, v), sm_scale=sm, causal=causal,
                                norm_mode=oracle.HIGH_PRECISION_L)
    O_ref, lse_ref = _bruteforce(q, k, v, causal, sm)
    assert np.abs(out["O"] - O_ref.reshape(-1, D)).max() <= 1e-5
    assert np.abs(out["lse"] - lse_ref.ravel()).max() <= 1e-5


def _c2_like(Nq=512, Nkv=512, D=128, causal=True, seed=6):
    cfg = W.get(2).replace(B=1, Hq=2, Hkv=1, Nq=Nq, Nkv=Nkv, D=D, causal=causal)
    rng = np.random.default_rng(seed)
    q = W.round_to_dtype(rng.standard_normal((1, 2, Nq, D)).astype(np.float32), "bf16")
    g = W.k_gains(cfg)[:1]
    k = W.round_to_dtype((rng.standard_normal((1, 1, Nkv, D)) * g[0]).astype(np.float32), "bf16")
    return cfg, q, k


def test_p_reorder_constant_v_rows_equal_vhat():
    cfg, q, k = _c2_like()
    v = np.ones_like(k)
    s, si = oracle.calibrate(q, k)
    pk = oracle.quantize_qkv(q, k, v, s, si)
    vhat = 1.03125                                  # 1 -> sf 0x23, code 6 (see the golden constant block)
    assert np.all(pk["vtc"] == 0x77) and np.all(pk["vts"] == 0x23)
    shape = (1, 2, 1, cfg.Nq, cfg.Nkv, cfg.D)
    rows = oracle.all_rows(1, 2, cfg.Nq)
    pr = oracle.attention_rows(shape, rows, packed=pk, causal=True, norm_mode=oracle.P_REORDER, want_eps=True)
    hp = oracle.attention_rows(shape, rows, packed=pk, causal=True, norm_mode=oracle.HIGH_PRECISION_L)
    # numerator and denominator from the same P_hat: every row is exactly V_hat
    assert np.abs(pr["O"] / vhat - 1).max() <= 1e-12
    # the high-precision normalizer scales every row by (1 + eps_row), eps_row = l_hat/l - 1
    eps_row = pr["l_hat"] / pr["l_hp"] - 1
    assert np.abs(hp["O"] / vhat - (1 + eps_row)[:, None]).max() <= 1e-12
    assert np.abs(eps_row).max() > 1e-3                       # the error is real, not roundoff
    # net probability-mass change per tile: median below zero on this workload
    eps_tiles = pr["eps"][np.isfinite(pr["eps"])]
    assert np.median(eps_tiles) < 0


def test_p_reorder_output_in_convex_hull_of_vhat():
    cfg, q, k = _c2_like(Nq=256, Nkv=384, causal=True, seed=7)
    rng = np.random.default_rng(8)
    v = W.round_to_dtype(rng.standard_normal(k.shape).astype(np.float32), "bf16")
    pk = oracle.quantize_qkv(q, k, v)
    shape = (1, 2, 1, 256, 384, 128)
    out = oracle.attention_rows(shape, oracle.all_rows(1, 2, 256), packed=pk, causal=True)
    vt = oracle.e2m1_decode(np.stack([pk["vtc"] & 15, pk["vtc"] >> 4], -1).ravel()).reshape(128, 384)
    vt = vt * np.repeat(oracle.e4m3_decode(pk["vts"].ravel()).reshape(128, 24), 16, axis=1)
    lo, hi = vt.min(axis=1), vt.max(axis=1)
    assert np.all(out["O"] >= lo[None, :] - 1e-12) and np.all(out["O"] <= hi[None, :] + 1e-12)


def test_running_max_is_per_tile():
    # Row 0 sees tile 0 (keys 0..127) with a moderate max, then a much larger
    # score in tile 1. P of tile 0 is taken relative to the tile-0 running max,
    # so its largest element is quantized as P = 1 (code 7, scale 0x23); a
    # single global max would have pushed all of tile 0 towards zero.
    D = 64
    q = np.zeros((1, 1, 1, D), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, 256, D), np.float32)
    k[0, 0, :, 0] = 0.01
    k[0, 0, 5, 0] = 8.0
    k[0, 0, 200, 0] = 200.0
    v = np.ones_like(k)
    pk = oracle.quantize_qkv(q, k, v)
    out = oracle.attention_rows((1, 1, 1, 1, 256, D), [0], packed=pk, want_p=True, want_eps=True)
    codes, sf = out["p_codes"][0], out["p_sf"][0]
    assert (codes[2] >> 4) == 7 and sf[0] == 0x23           # key 5 = byte 2, high nibble
    assert np.all(codes[:64] != 0)                           # tile 0 keeps mass: P ~ 2^(c*(0.01-8))
    assert sf[200 // 16] == 0x23 and np.isfinite(out["eps"][0]).all()


def test_causal_masked_keys_get_zero_codes():
    cfg, q, k = _c2_like(Nq=128, Nkv=256, causal=True, seed=9)
    v = np.ones_like(k)
    pk = oracle.quantize_qkv(q, k, v)
    out = oracle.attention_rows((1, 2, 1, 128, 256, 128), oracle.all_rows(1, 2, 128), packed=pk,
                                causal=True, want_p=True)
    nib = np.stack([out["p_codes"] & 15, out["p_codes"] >> 4], -1).reshape(256, 256)
    i = np.arange(256) % 128
    masked = np.arange(256)[None, :] > (i[:, None] + 128)
    assert np.all(nib[masked] == 0)
    assert np.any(nib[~masked] != 0, axis=None)


def test_numpy_restatement_bit_exact_on_tiny_config():
    cfg = W.get(1)
    q, k, v = W.full(cfg)
    s, si = oracle.calibrate(q, k)
    pk = oracle.quantize_qkv(q, k, v, s, si)
    shape = (1, 1, 1, 256, 256, 64)
    for mode in (oracle.P_REORDER, oracle.HIGH_PRECISION_L):
        ref = np_ref.attention(q, k, v, s=s, s_inv=si, norm_mode=mode)
        for key in ("qc", "qs", "kc", "ks", "vtc", "vts"):
            assert np.array_equal(ref[key], pk[key]), key
        out = oracle.attention_rows(shape, oracle.all_rows(1, 1, 256), packed=pk, norm_mode=mode, want_p=True)
        assert np.array_equal(out["p_codes"], ref["p_codes"].reshape(256, -1))
        assert np.array_equal(out["p_sf"], ref["p_sf"].reshape(256, -1))
        assert np.abs(out["O"] - ref["O"].reshape(-1, 64)).max() <= 1e-12
        assert np.abs(out["lse"] - ref["lse"].ravel()).max() <= 1e-12


def test_smooth_qk_reduces_score_error_on_outlier_channels():
    cfg = W.get(1)
    q, k, v = W.full(cfg)
    exact = np.einsum("id,jd->ij", q[0, 0].astype(np.float64), k[0, 0].astype(np.float64))
    errs = {}
    for name, sc in (("off", None), ("on", oracle.calibrate(q, k))):
        pk = oracle.quantize_qkv(q, k, v, *(sc if sc else (None, None)))
        S = np.stack([oracle.qk_row(pk, 1, 1, 256, 256, 64, r) for r in range(0, 256, 8)])
        errs[name] = np.sqrt(np.mean((S - exact[::8]) ** 2))
    # same scores up to quantization error either way; smoothing lowers that error
    assert errs["on"] < errs["off"]
    assert errs["on"] < 0.1 * np.sqrt(np.mean(exact ** 2))


# ------------------------------------------------ Smooth-QK is an equivalence

def _exactly_smoothable(rng, B, Hq, Hkv, N, D):
    """Q = g * 2^-e, K = h * 2^e with g, h on the E2M1 grid, e per (kv head,
    channel), and a +-6 in every 16-element block of every row. Calibration then
    gives s = 2^e exactly, the smoothed rows are g and h, and 4-bit quantization
    of g and h is lossless (every block's scale is 1)."""
    G = Hq // Hkv
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e = rng.integers(-3, 4, (Hkv, D))

    def rows(H, n, group):
        x = rng.choice(grid, (B, H, n, D)) * rng.choice([-1.0, 1.0], (B, H, n, D))
        for blk in range(D // 16):
            x[:, :, np.arange(n), blk * 16 + np.arange(n) % 16] = 6.0 * rng.choice([-1.0, 1.0], (B, H, n))
        return x

    g, h = rows(Hq, N, G), rows(Hkv, N, 1)
    eq = np.repeat(e, G, axis=0)[None, :, None, :]
    q = (g * 2.0 ** -eq).astype(np.float32)
    k = (h * 2.0 ** e[None, :, None, :]).astype(np.float32)
    return q, k, e


@pytest.mark.parametrize("shape", [(2, 4, 2, 32, 64), (1, 8, 2, 48, 128), (1, 2, 1, 16, 256)])
def test_smooth_qk_leaves_qk_unchanged_exactly(shape):
    """HiFA4 abstract: Smooth-QK is an equivalent per-channel rescaling (Q*s,
    K/s), so QK^T is unchanged in exact arithmetic. On inputs where smoothing
    makes quantization lossless, the oracle's whole smoothing path (calibration,
    Q*s and K*s_inv per kv head and channel, quantization, QK^T) must give the
    exact unsmoothed scores bit for bit; without smoothing the same inputs are
    quantized lossily, so the check has teeth."""
    B, Hq, Hkv, N, D = shape
    G = Hq // Hkv
    rng = np.random.default_rng(31)
    q, k, e = _exactly_smoothable(rng, B, Hq, Hkv, N, D)
    s, si = oracle.calibrate(q, k, 0.5)
    assert np.array_equal(s, (2.0 ** e).astype(np.float32))
    v = np.zeros_like(k)
    on = oracle.quantize_qkv(q, k, v, s, si)
    off = oracle.quantize_qkv(q, k, v)
    exact = np.einsum("bhid,bhjd->bhij", q.astype(np.float64), np.repeat(k.astype(np.float64), G, axis=1))
    n_off_exact = 0
    for b in range(B):
        for hh in range(Hq):
            for i in (0, N // 2, N - 1):
                row = (b * Hq + hh) * N + i
                want = exact[b, hh, i].astype(np.float32)
                assert np.array_equal(oracle.qk_row(on, Hq, Hkv, N, N, D, row), want), (b, hh, i)
                n_off_exact += np.array_equal(oracle.qk_row(off, Hq, Hkv, N, N, D, row), want)
    assert n_off_exact == 0


def test_smooth_qk_factors_are_reciprocal_pairs_on_outlier_tensors():
    """On the tiny config's outlier tensors and on a GQA shape the calibration
    returns s_inv = RN(1/s), so (Q*s)(K*s_inv)^T equals QK^T up to one rounding
    of s*s_inv per channel (relative 2^-24), far below the 4-bit error."""
    cfg = W.get(1)
    q1, k1, _ = W.full(cfg)
    rng = np.random.default_rng(32)
    q2 = rng.standard_normal((2, 8, 64, 128)).astype(np.float32)
    k2 = (rng.standard_normal((2, 2, 64, 128)) * rng.lognormal(0, 1, (1, 2, 1, 128))).astype(np.float32)
    for q, k in ((q1, k1), (q2, k2)):
        s, si = oracle.calibrate(q, k)
        prod = s.astype(np.float64) * si.astype(np.float64)
        assert np.all(np.abs(prod - 1.0) <= 2.0 ** -24)
        assert np.all(si == (1.0 / s.astype(np.float64)).astype(np.float32))
        G = q.shape[1] // k.shape[1]
        sq = np.repeat(s.astype(np.float64), G, axis=0)[None, :, None, :]
        kk = np.repeat(k.astype(np.float64), G, axis=1)
        ref = np.einsum("bhid,bhjd->bhij", q.astype(np.float64), kk)
        sm = np.einsum("bhid,bhjd->bhij", q * sq, kk * np.repeat(si.astype(np.float64), G, axis=0)[None, :, None, :])
        assert np.abs(sm - ref).max() <= 1e-6 * np.abs(ref).max()


# ----------------------------------------------------- split kv (decoding)

@pytest.mark.parametrize("shape,causal,n_splits", [
    ((1, 2, 1, 16, 512, 64), False, 4),
    ((2, 4, 2, 64, 640, 128), True, 4),       # 5 tiles over 4 splits: ragged ranges, bottom-right causal
    ((1, 2, 2, 32, 384, 128), False, 2),
    ((1, 1, 1, 128, 512, 256), True, 3),
])
def test_split_kv_quant_off_matches_bruteforce(shape, causal, n_splits):
    """With quantization off, cutting the kv tiles into ranges with their own
    online softmax and merging by log-sum-exp weights is exactly softmax
    attention, so it must match the brute-force fp64 result."""
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(33)
    q = (rng.standard_normal((B, Hq, Nq, D)) * 1.5).astype(np.float32)
    k = (rng.standard_normal((B, Hkv, Nkv, D)) * 1.5).astype(np.float32)
    v = rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32)
    sm = oracle.default_sm_scale(D)
    for mode in (oracle.P_REORDER, oracle.HIGH_PRECISION_L):
        out = oracle.attention_rows(shape, oracle.all_rows(B, Hq, Nq), fp32=(q, k, v), sm_scale=sm, causal=causal,
                                    norm_mode=mode, n_splits=n_splits)
        O_ref, lse_ref = _bruteforce(q, k, v, causal, sm)
        assert np.abs(out["O"] - O_ref.reshape(-1, D)).max() <= 1e-5
        assert np.abs(out["lse"] - lse_ref.ravel()).max() <= 1e-5


def test_split_kv_p_reorder_constant_v_rows_equal_vhat():
    """P-Reordering with kv splits: every split's numerator and normalizer come
    from the same P_hat, and the merge weights are shared, so with V = 1 every
    row is exactly V_hat again."""
    cfg, q, k = _c2_like(Nq=64, Nkv=512, causal=False, seed=34)
    v = np.ones_like(k)
    pk = oracle.quantize_qkv(q, k, v)
    out = oracle.attention_rows((1, 2, 1, 64, 512, 128), oracle.all_rows(1, 2, 64), packed=pk,
                                norm_mode=oracle.P_REORDER, n_splits=4)
    assert np.abs(out["O"] / 1.03125 - 1).max() <= 1e-12


def test_split_kv_p_hat_is_relative_to_the_split_max():
    """Each split starts its own running max: a large score in tile 0 shrinks
    the P of tile 2 in one pass, but not when tile 2 starts the second of two
    splits, where its own maximum quantizes to P = 1 (code 7, scale 0x23)."""
    D = 64
    q = np.zeros((1, 1, 1, D), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, 512, D), np.float32)
    k[0, 0, :, 0] = 0.01
    k[0, 0, 3, 0] = 60.0                       # tile 0, dominant
    k[0, 0, 300, 0] = 2.0                      # tile 2's maximum
    v = np.ones_like(k)
    pk = oracle.quantize_qkv(q, k, v)
    one = oracle.attention_rows((1, 1, 1, 1, 512, D), [0], packed=pk, want_p=True)
    two = oracle.attention_rows((1, 1, 1, 1, 512, D), [0], packed=pk, want_p=True, n_splits=2)
    key = 300
    nib = lambda c: (c[key // 2] >> 4) if key % 2 else (c[key // 2] & 15)
    assert nib(two["p_codes"][0]) == 7 and two["p_sf"][0][key // 16] == 0x23
    assert nib(one["p_codes"][0]) == 0                    # 2^((2 - 60) c) flushes to zero in one pass
    # tiles 0 and 1 (the first split) are the same either way
    assert np.array_equal(one["p_codes"][0][:128], two["p_codes"][0][:128])


# ------------------------------------------------ RoPE (steps before the path)

def _rope_tables(n_pos, D, base=10000.0):
    """cos/sin of pos * base^(-2d/D) in fp64, rounded to fp32 (the caller's tables)."""
    inv = base ** (-np.arange(0, D // 2, dtype=np.float64) * 2.0 / D)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_rope_identity_and_quarter_turn_are_exact():
    """cos = 1, sin = 0 leaves x unchanged; cos = 0, sin = 1 is the quarter
    turn of rotate-half pairing: (x[d], x[d+D/2]) -> (-x[d+D/2], x[d]). A swapped
    sign or the interleaved (2i, 2i+1) pairing fails the second check."""
    D = 16
    rng = np.random.default_rng(40)
    x = rng.standard_normal((1, 1, 3, D)).astype(np.float32)
    cos_t = np.stack([np.ones(D // 2), np.zeros(D // 2)]).astype(np.float32)
    sin_t = np.stack([np.zeros(D // 2), np.ones(D // 2)]).astype(np.float32)
    same = oracle.rope_neox(x, cos_t, sin_t, [0, 0, 0])
    assert np.array_equal(same, x)
    turned = oracle.rope_neox(x, cos_t, sin_t, [1, 0, 1])
    want = np.concatenate([-x[..., D // 2:], x[..., :D // 2]], axis=-1)
    assert np.array_equal(turned[:, :, 0], want[:, :, 0]) and np.array_equal(turned[:, :, 2], want[:, :, 2])
    assert np.array_equal(turned[:, :, 1], x[:, :, 1])


def test_rope_preserves_pair_norms_and_depends_on_relative_position():
    """A rotation keeps |(x[d], x[d+D/2])|, and the score between a query at
    position m and a key at n depends only on m - n."""
    D = 64
    cos_t, sin_t = _rope_tables(64, D)
    rng = np.random.default_rng(41)
    q = rng.standard_normal((1, 1, 1, D)).astype(np.float32)
    k = rng.standard_normal((1, 1, 1, D)).astype(np.float32)
    y = oracle.rope_neox(q, cos_t, sin_t, [37]).astype(np.float64)
    n_in = np.hypot(q[..., :D // 2], q[..., D // 2:])
    n_out = np.hypot(y[..., :D // 2], y[..., D // 2:])
    assert np.abs(n_out / n_in - 1).max() <= 1e-6
    s = [float(np.sum(oracle.rope_neox(q, cos_t, sin_t, [m]).astype(np.float64)
                      * oracle.rope_neox(k, cos_t, sin_t, [n]).astype(np.float64)))
         for m, n in ((10, 3), (20, 13), (57, 50))]
    assert max(s) - min(s) <= 1e-5 * np.abs(q).sum() * np.abs(k).sum()


def test_prequant_smoothing_step_equals_quantize_rows_scale():
    """The separate Smooth-QK step followed by plain quantization gives the same
    codes as quantize_rows with the scale (one product, one rounding)."""
    rng = np.random.default_rng(42)
    x = rng.standard_normal((1, 4, 32, 64)).astype(np.float32)
    s = rng.lognormal(0, 1, (2, 64)).astype(np.float32)
    a = oracle.quantize_rows(x, s, 2)
    b = oracle.quantize_rows(oracle.prequant_rows(x, scale=s, group=2))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------------------------------------------------------------ Q-Mean

def test_q_mean_hand_values_and_exact_shift():
    N, D = 8, 16
    x = np.zeros((1, 2, N, D), np.float32)
    x[0, 0, :, 0] = np.arange(N) * 0.125            # mean 0.4375
    x[0, 1, :, 3] = [1, -1] * (N // 2)               # mean 0
    x[0, 1, :, 5] = 3.0
    m = oracle.q_mean(x)
    assert m[0, 0, 0] == np.float32(0.4375) and m[0, 1, 3] == 0 and m[0, 1, 5] == 3
    assert np.count_nonzero(m) == 2
    # adding a dyadic vector to every token moves the mean by exactly that vector
    rng = np.random.default_rng(43)
    y = W.round_to_dtype(rng.standard_normal((1, 2, 64, D)).astype(np.float32), "bf16")
    shift = (rng.integers(-8, 8, D) * 0.25).astype(np.float32)
    base = oracle.q_mean(y).astype(np.float64)
    moved = oracle.q_mean(y + shift).astype(np.float64)
    # y + shift is exact in fp32 (bf16 values plus quarter integers of small size)
    assert np.abs(moved - base - shift).max() <= 2 * np.spacing(np.float32(4))


def test_q_mean_residual_sums_to_zero():
    """sum_i (x_i - mean) = N (mean_exact - mean) is within rounding of zero."""
    rng = np.random.default_rng(44)
    x = W.round_to_dtype((rng.standard_normal((2, 2, 128, 64)) + 3).astype(np.float32), "bf16")
    r = oracle.sub_mean(x, oracle.q_mean(x)).astype(np.float64)
    assert np.abs(r.sum(axis=2)).max() <= 128 * 4 * np.spacing(np.float32(4))


def test_q_mean_bias_closed_form_and_bruteforce():
    """K' = 1 everywhere: the bias of every key is the sum of the mean's
    channels. Then random keys against a plain fp64 product with GQA heads."""
    B, Hq, Hkv, Nkv, D = 1, 4, 2, 128, 64
    rng = np.random.default_rng(45)
    mean = rng.standard_normal((B, Hq, D)).astype(np.float32)
    bias = oracle.q_mean_bias(mean, np.ones((B, Hkv, Nkv, D), np.float32), Hq)
    assert np.abs(bias - mean.astype(np.float64).sum(-1)[..., None]).max() <= 1e-12
    k = rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32)
    bias = oracle.q_mean_bias(mean, k, Hq)
    for h in range(Hq):
        want = k[0, h // 2].astype(np.float64) @ mean[0, h].astype(np.float64)
        assert np.abs(bias[0, h] - want).max() <= 1e-12 * np.abs(want).max()


def test_q_mean_constant_rows_give_exact_scores():
    """Every query row equal to u: the residual quantizes to zero codes, so the
    scores are u . K exactly (the bias term alone), and the log-sum-exp
    (high-precision l) equals the brute-force fp64 log-sum-exp of
    sm_scale * u . K^T. Dropping the bias, flipping its sign or taking it from
    the quantized keys fails."""
    B, Hq, Hkv, Nq, Nkv, D = 1, 2, 1, 16, 256, 64
    rng = np.random.default_rng(46)
    u = W.round_to_dtype(rng.standard_normal((1, Hq, 1, D)).astype(np.float32) * 2, "bf16")
    q = np.repeat(u, Nq, axis=2)
    k = W.round_to_dtype(rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32), "bf16")
    v = rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32)
    m = oracle.q_mean(q)
    assert np.array_equal(m[:, :, None, :], u)
    pk = oracle.quantize_qkv(oracle.sub_mean(q, m), k, v)
    assert not pk["qc"].any() and not pk["qs"].any()
    bias = oracle.q_mean_bias(m, k, Hq)
    out = oracle.attention_rows((B, Hq, Hkv, Nq, Nkv, D), oracle.all_rows(B, Hq, Nq), packed=pk, s_bias=bias,
                                norm_mode=oracle.HIGH_PRECISION_L)
    sm = oracle.default_sm_scale(D)
    for h in range(Hq):
        s = sm * (k[0, 0].astype(np.float64) @ u[0, h, 0].astype(np.float64))
        want = s.max() + np.log(np.exp(s - s.max()).sum())
        assert np.abs(out["lse"][h * Nq:(h + 1) * Nq] - want).max() <= 1e-5


def _dequant_rows(codes, sf):
    e2 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])
    el = np.stack([e2[codes & 15], e2[codes >> 4]], -1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    sc = np.array([_e4m3_closed_form(int(c)) for c in range(256)])[sf]
    return el * np.repeat(sc, 16, axis=-1)


def test_q_mean_reduces_score_error_with_a_common_offset():
    """Q with a shared per-channel offset (the case Q smoothing targets): the
    4-bit scores with the Q-Mean term are much closer to the fp64 scores of
    the unquantized operands than the plain 4-bit scores."""
    B, Hq, Hkv, Nq, Nkv, D = 1, 1, 1, 128, 256, 128
    rng = np.random.default_rng(47)
    off = rng.standard_normal(D).astype(np.float32) * 4
    q = W.round_to_dtype((rng.standard_normal((B, Hq, Nq, D)) + off).astype(np.float32), "bf16")
    k = W.round_to_dtype(rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32), "bf16")
    exact = np.einsum("id,jd->ij", q[0, 0].astype(np.float64), k[0, 0].astype(np.float64))
    plain = oracle.quantize_qkv(q, k, np.zeros_like(k))
    S_plain = _dequant_rows(plain["qc"], plain["qs"])[0, 0] @ _dequant_rows(plain["kc"], plain["ks"])[0, 0].T
    m = oracle.q_mean(q)
    pm = oracle.quantize_qkv(oracle.sub_mean(q, m), k, np.zeros_like(k))
    khat = _dequant_rows(pm["kc"], pm["ks"])[0, 0]
    S_qm = _dequant_rows(pm["qc"], pm["qs"])[0, 0] @ khat.T + oracle.q_mean_bias(m, k, Hq)[0, 0][None, :]
    e_plain = np.sqrt(np.mean((S_plain - exact) ** 2))
    e_qm = np.sqrt(np.mean((S_qm - exact) ** 2))
    assert e_qm < 0.5 * e_plain


# ------------------------------------------------------ epsilon-bar tiles

def test_eps_bar_hand_values():
    """Tile mean over the rows with mass (NaN rows skipped); NaN when no row has any."""
    B, Hq, Nq, T = 1, 1, 130, 2
    e = np.full((Nq, T), np.nan)
    e[0, 0], e[5, 0], e[127, 0] = -0.1, -0.2, 0.3      # q tile 0, kv tile 0: mean 0
    e[128, 1], e[129, 1] = -0.5, -0.25                 # q tile 1, kv tile 1
    out = oracle.eps_bar(e, B, Hq, Nq)
    assert out.shape == (1, 1, 2, 2)
    assert abs(out[0, 0, 0, 0]) <= 1e-15 and np.isnan(out[0, 0, 0, 1])
    assert np.isnan(out[0, 0, 1, 0]) and out[0, 0, 1, 1] == -0.375


def test_eps_rows_follow_definition_on_a_tiny_case():
    """Per (row, tile): sum P_hat / sum P - 1, from the P_hat codes the oracle
    dumps and the fp64 P of a brute-force online softmax."""
    B, Hq, Hkv, Nq, Nkv, D = 1, 1, 1, 4, 256, 64
    rng = np.random.default_rng(48)
    q = W.round_to_dtype(rng.standard_normal((B, Hq, Nq, D)).astype(np.float32), "bf16")
    k = W.round_to_dtype(rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32), "bf16")
    pk = oracle.quantize_qkv(q, k, np.zeros_like(k))
    out = oracle.attention_rows((B, Hq, Hkv, Nq, Nkv, D), oracle.all_rows(B, Hq, Nq), packed=pk,
                                want_eps=True, want_p=True)
    phat = _dequant_rows(out["p_codes"][:, None, None, :], out["p_sf"][:, None, None, :])[:, 0, 0]
    S = _dequant_rows(pk["qc"], pk["qs"])[0, 0] @ _dequant_rows(pk["kc"], pk["ks"])[0, 0].T
    c = np.float32(oracle.default_sm_scale(D) * np.log2(np.e))
    for i in range(Nq):
        m = -np.inf
        for t in range(2):
            s = S[i, 128 * t:128 * (t + 1)].astype(np.float32)
            m = max(m, float(s.max()))
            mc = np.float32(np.float32(m) * c)
            p = np.exp2((s * np.float64(c) - np.float64(mc)))
            want = phat[i, 128 * t:128 * (t + 1)].sum() / p.sum() - 1
            assert abs(out["eps"][i, t] - want) <= 1e-6
