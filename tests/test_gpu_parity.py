"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
the same seeded inputs.

Bars (hot-path specification of this build):
  quantized Q/K/V codes and scales  bit-exact
  calibration factors s, s_inv      bit-exact (alpha = 0.5: correctly rounded
                                    division and square root on both sides)
  P_hat codes                       mismatch rate <= 1e-4 (S accumulation order
                                    and the hardware exp2 differ from the oracle)
  O (fp32 output)                   max abs <= 5e-3 and per-row relative L2
                                    <= 1e-3 (absolute where ||O_row|| < 1e-6)
  LSE                               max abs <= 1e-3
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import hifa4_testutil as U

pytestmark = pytest.mark.gpu

O_MAX_ABS = 5e-3
O_ROW_REL = 1e-3
LSE_ABS = 1e-3
P_MISMATCH = 1e-4


@pytest.fixture(scope="module")
def H():
    import bit_quantized_flashattention_b200 as H
    H.load()
    return H


def _rand(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _gpu_quant(H, q, k, v, dtype, s=None, si=None):
    dq, dk, dv = (U.to_device(x, dtype) for x in (q, k, v))
    ds = None if s is None else torch.from_numpy(s).cuda()
    dsi = None if si is None else torch.from_numpy(si).cuda()
    pk = H.quantize_qkv(dq, dk, dv, ds, dsi)
    torch.cuda.synchronize()
    return pk


def _compare_packed(pk, ref, shape):
    B, Hq, Hkv, Nq, Nkv, D = shape
    qs, ks, vts = U.canonical_scales(pk, B, Hq, Hkv, Nq, Nkv, D)
    assert np.array_equal(pk.qc.cpu().numpy().reshape(ref["qc"].shape), ref["qc"])
    assert np.array_equal(qs, ref["qs"])
    assert np.array_equal(pk.kc.cpu().numpy().reshape(ref["kc"].shape), ref["kc"])
    assert np.array_equal(ks, ref["ks"])
    assert np.array_equal(U.canonical_vtc(pk.vtc, B, Hkv, Nkv, D), ref["vtc"])
    assert np.array_equal(vts, ref["vts"])
    assert U.padding_bytes_ok(pk, B, Hq, Hkv, Nq, Nkv, D)


# ------------------------------------------------------------ quantization

def test_quantize_format_sweep_matches_oracle(H):
    """Values spread over every E2M1 / E4M3 regime: midpoints, signed zeros,
    subnormal and saturating scales, flushed blocks."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, N, D = 1, 2, 1, 256, 64
    mag = np.exp(rng.uniform(np.log(1e-4), np.log(3e3), (B, Hq, N, D))).astype(np.float32)
    q = (mag * np.sign(rng.standard_normal(mag.shape))).astype(np.float32)
    # exact midpoints with a block max of 6 -> scale 1
    q[0, 0, :16, :] = np.float32(0.25)
    q[0, 0, :16, ::16] = np.float32(6.0)
    q[0, 0, 16:32, :] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5,
                                  -3.5, -5.0, 6.0, -0.1] * 4, np.float32)
    q[0, 0, 32:48, :] = np.float32(-1e-3)             # flushed: scale 0, codes -0
    q[0, 0, 48:64, :] = np.float32(1e4)               # saturating scale
    q = W.round_to_dtype(q, "bf16")
    k = W.round_to_dtype(_rand(rng, (B, Hkv, N, D), 3.0), "bf16")
    v = W.round_to_dtype(q[:, :1].copy(), "bf16")
    pk = _gpu_quant(H, q, k, v, "bf16")
    ref = oracle.quantize_qkv(q, k, v)
    _compare_packed(pk, ref, (B, Hq, Hkv, N, N, D))


@pytest.mark.parametrize("shape,dtype", [
    ((1, 1, 1, 256, 256, 64), "fp16"),
    ((2, 8, 2, 48, 384, 128), "bf16"),         # G*Nq = 192: a partly filled q tile per group
    ((1, 4, 2, 128, 256, 256), "bf16"),
    ((1, 6, 2, 16, 128, 128), "fp16"),         # G*Nq = 48
])
def test_quantize_with_smoothing_matches_oracle(H, shape, dtype):
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(12)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)), dtype)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)) * rng.lognormal(0, 1, (1, Hkv, 1, D)).astype(np.float32), dtype)
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), dtype)
    s, si = oracle.calibrate(q, k)
    pk = _gpu_quant(H, q, k, v, dtype, s, si)
    ref = oracle.quantize_qkv(q, k, v, s, si)
    _compare_packed(pk, ref, shape)


@pytest.mark.parametrize("shape,dtype,alpha", [
    ((1, 1, 1, 256, 256, 64), "fp16", 0.5),
    ((2, 8, 2, 512, 512, 128), "bf16", 0.5),
    ((1, 4, 4, 100, 100, 256), "bf16", 0.5),
])
def test_calibrate_matches_oracle(H, shape, dtype, alpha):
    B, Hq, Hkv, N, _, D = shape
    rng = np.random.default_rng(13)
    q = W.round_to_dtype(_rand(rng, (B, Hq, N, D)), dtype)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, N, D)) * rng.lognormal(0, 1, (1, Hkv, 1, D)).astype(np.float32), dtype)
    q[0, 0, :, 3] = 0                                   # a zero channel -> s = 1 there (if the whole group is 0)
    s, si = H.calibrate_smooth(U.to_device(q, dtype), U.to_device(k, dtype), alpha)
    rs, rsi = oracle.calibrate(q, k, alpha)
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(si.cpu().numpy(), rsi)


# --------------------------------------------------------------- attention

def _attention_case(H, shape, causal, norm, dtype="bf16", out_dtype=torch.float32, seed=14, gain=1.0,
                    smooth=True):
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(seed)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)), dtype)
    g = rng.lognormal(0, gain, (1, Hkv, 1, D)).astype(np.float32)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)) * g, dtype)
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), dtype)
    s, si = oracle.calibrate(q, k) if smooth else (None, None)
    pk = _gpu_quant(H, q, k, v, dtype, s, si)
    o, lse, pc, ps = H.attention_fwd_debug(pk, causal=causal, norm=norm, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref_p = oracle.quantize_qkv(q, k, v, s, si)
    rows = oracle.all_rows(B, Hq, Nq)
    ref = oracle.attention_rows(shape, rows, packed=ref_p, causal=causal,
                                norm_mode=0 if norm == "p_reorder" else 1, want_p=True)
    return o, lse, pc, ps, ref


def _check_attention(o, lse, pc, ps, ref, D, out_dtype=torch.float32):
    og = o.float().cpu().numpy().reshape(-1, D)
    ref_o = ref["O"]
    if out_dtype != torch.float32:
        ref_o = torch.from_numpy(ref_o).to(out_dtype).double().numpy()
    pcg = pc.cpu().numpy().reshape(ref["p_codes"].shape)
    nib_g = np.stack([pcg & 15, pcg >> 4], -1)
    nib_r = np.stack([ref["p_codes"] & 15, ref["p_codes"] >> 4], -1)
    mism = float(np.mean(nib_g != nib_r))
    sf_mism = float(np.mean(ps.cpu().numpy().reshape(ref["p_sf"].shape) != ref["p_sf"]))
    max_abs, rel = U.row_errors(og, ref_o)
    lse_err = float(np.abs(lse.cpu().numpy().ravel() - ref["lse"]).max())
    assert mism <= P_MISMATCH, f"P_hat code mismatch {mism:.2e} (scale mismatch {sf_mism:.2e})"
    assert max_abs <= O_MAX_ABS, f"O max abs {max_abs:.3e}"
    assert rel.max() <= O_ROW_REL, f"O row rel L2 {rel.max():.3e} (rows over: {(rel > O_ROW_REL).sum()})"
    assert lse_err <= LSE_ABS, f"LSE max abs {lse_err:.3e}"


@pytest.mark.parametrize("shape,causal", [
    ((1, 1, 1, 256, 256, 64), False),
    ((1, 2, 1, 256, 384, 128), False),
    ((1, 4, 2, 384, 384, 128), True),
    ((2, 4, 2, 176, 512, 128), True),          # Nq < Nkv, G*Nq = 352: tiles mix heads, ragged tail
    ((1, 2, 2, 256, 256, 256), True),
    ((1, 8, 2, 16, 512, 128), False),          # decode-style: 4 heads x 16 queries in one tile
    ((1, 4, 2, 512, 512, 128), True),          # Nq % 256 == 0: paired query tiles, longest first
    ((1, 2, 1, 384, 384, 64), True),
])
@pytest.mark.parametrize("norm", ["p_reorder", "high_precision_l"])
def test_attention_matches_oracle(H, shape, causal, norm):
    o, lse, pc, ps, ref = _attention_case(H, shape, causal, norm)
    _check_attention(o, lse, pc, ps, ref, shape[-1])


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float16])
def test_attention_low_precision_output(H, out_dtype):
    shape = (1, 2, 1, 256, 256, 128)
    o, lse, pc, ps, ref = _attention_case(H, shape, True, "p_reorder", out_dtype=out_dtype)
    og = o.float().cpu().numpy().reshape(-1, 128)
    ref_o = torch.from_numpy(ref["O"]).to(out_dtype).float().numpy()
    # one output ulp of either side
    tol = 2.0 ** (-7 if out_dtype == torch.bfloat16 else -10) * np.maximum(np.abs(ref_o), 2 ** -6)
    assert np.all(np.abs(og - ref_o) <= tol + O_MAX_ABS * 0.1)


def test_plain_and_debug_calls_agree(H):
    shape = (1, 4, 2, 256, 256, 128)
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(15)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)), "bf16")
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    pk = _gpu_quant(H, q, k, v, "bf16")
    o1, l1 = H.attention_fwd(pk, causal=True, out_dtype=torch.float32)
    o2, l2, _, _ = H.attention_fwd_debug(pk, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_timeout_path_reports_status(H):
    """Loads stalled on purpose: every wait runs out with nothing in flight; the
    kernel records the timeout, frees TMEM and returns; the context stays usable."""
    shape = (1, 2, 1, 128, 256, 128)
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(16)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)), "bf16")
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    pk = _gpu_quant(H, q, k, v, "bf16")
    ws = H.alloc_workspace(*shape)
    H.debug_set_wait_limit(20_000_000, stall_loads=True)       # 20 ms
    try:
        H.attention_fwd(pk, causal=True, workspace=ws)
        assert H.get_status(ws) == 4
    finally:
        H.debug_set_wait_limit(0, stall_loads=False)
    o, _ = H.attention_fwd(pk, causal=True, workspace=ws, out_dtype=torch.float32)
    assert H.get_status(ws) == 0
    assert torch.isfinite(o).all()


def test_quantize_timeout_path_reports_status(H):
    """Row copies of the quantize pass stalled on purpose: its bounded waits run
    out with nothing in flight, the pass records the timeout in its status word
    (reported by get_status) and stops; the next pass runs normally and matches
    the oracle."""
    shape = (1, 2, 1, 128, 256, 128)
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(18)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)), "bf16")
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    dq, dk, dv = (U.to_device(x, "bf16") for x in (q, k, v))
    ws = H.alloc_workspace(*shape)
    assert H.get_status(ws) == 0
    H.debug_set_wait_limit(20_000_000, stall_loads=True)       # 20 ms
    try:
        H.quantize_qkv(dq, dk, dv)
        assert H.get_status(ws) == 4
    finally:
        H.debug_set_wait_limit(0, stall_loads=False)
    pk = H.quantize_qkv(dq, dk, dv)
    assert H.get_status(ws) == 0
    _compare_packed(pk, oracle.quantize_qkv(q, k, v), shape)


@pytest.mark.parametrize("shape,dtype,smooth", [
    ((2, 2, 384, 128), "bf16", True),
    ((1, 3, 256, 64), "fp16", False),
    ((1, 2, 512, 256), "bf16", True),
])
def test_quantize_kv_matches_oracle(H, shape, dtype, smooth):
    """hifa4_quantize_kv (K and V only, as when a KV cache is appended): codes
    and MMA-ready scales bit-exact against the oracle, with and without the
    Smooth-QK factor on K."""
    B, Hkv, N, D = shape
    rng = np.random.default_rng(17)
    q = W.round_to_dtype(_rand(rng, (B, Hkv, N, D)), dtype)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, N, D)) * rng.lognormal(0, 1, (1, Hkv, 1, D)).astype(np.float32), dtype)
    v = W.round_to_dtype(_rand(rng, (B, Hkv, N, D)), dtype)
    s = si = None
    if smooth:
        s, si = oracle.calibrate(q, k)
    dsi = None if si is None else torch.from_numpy(si).cuda()
    pk = H.quantize_kv(U.to_device(k, dtype), U.to_device(v, dtype), dsi)
    torch.cuda.synchronize()
    kc, ks = oracle.quantize_rows(k, si, 1)
    vtc, vts = oracle.quantize_v(v)
    _, ks_g, vts_g = U.canonical_scales(pk, B, Hkv, Hkv, 16, N, D)
    assert np.array_equal(pk.kc.cpu().numpy().reshape(kc.shape), kc)
    assert np.array_equal(ks_g, ks)
    assert np.array_equal(U.canonical_vtc(pk.vtc, B, Hkv, N, D), vtc)
    assert np.array_equal(vts_g, vts)


@pytest.mark.parametrize("shape,causal", [
    ((1, 8, 2, 16, 512, 128), False),          # 4 heads x 16 queries = 64 rows per group, 4 ranges of 1 tile
    ((2, 4, 1, 16, 640, 64), True),            # 5 tiles over 4 ranges (ragged), causal, D = 64
    ((1, 2, 2, 32, 1024, 128), False),         # 32 rows per group (half of each range's lanes idle)
    ((1, 4, 1, 16, 384, 128), False),          # 3 tiles: too few for 4 ranges -> one pass
])
@pytest.mark.parametrize("norm", ["p_reorder", "high_precision_l"])
def test_attention_split_kv_matches_oracle(H, shape, causal, norm):
    """Split-kv decode mode (HIFA4_SPLIT_KV): the library reports its range
    count, and the oracle with that many ranges is the reference (P_hat relative
    to each range's own running max, ranges merged by log-sum-exp weights)."""
    B, Hq, Hkv, Nq, Nkv, D = shape
    n_splits = H.attention_splits(B, Hq, Hkv, Nq, Nkv, D, causal=causal, split_kv=True)
    assert n_splits == (1 if Nkv < 512 else 4)
    rng = np.random.default_rng(18)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)), "bf16")
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)) * rng.lognormal(0, 1, (1, Hkv, 1, D)).astype(np.float32), "bf16")
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), "bf16")
    s, si = oracle.calibrate(q, k)
    pk = _gpu_quant(H, q, k, v, "bf16", s, si)
    o, lse, pc, ps = H.attention_fwd_debug(pk, causal=causal, norm=norm, split_kv=True)
    torch.cuda.synchronize()
    ref_p = oracle.quantize_qkv(q, k, v, s, si)
    ref = oracle.attention_rows(shape, oracle.all_rows(B, Hq, Nq), packed=ref_p, causal=causal,
                                norm_mode=0 if norm == "p_reorder" else 1, want_p=True, n_splits=n_splits)
    _check_attention(o, lse, pc, ps, ref, D)


@pytest.mark.parametrize("shape,causal,dtype,smooth", [
    ((1, 4, 2, 384, 384, 128), True, "bf16", True),
    ((2, 4, 2, 176, 512, 128), True, "bf16", False),       # G*Nq = 352: tiles mix heads, ragged last tile
    ((1, 2, 1, 256, 384, 128), False, "fp16", True),
    ((1, 8, 2, 16, 512, 128), False, "bf16", True),         # decode-style rows, one pass
])
@pytest.mark.parametrize("norm", ["p_reorder", "high_precision_l"])
def test_attention_with_in_kernel_q_quantization(H, shape, causal, dtype, smooth, norm):
    """hifa4_attention_fwd_q quantizes Q inside the attention kernel with the
    quantize pass's rule: O and LSE equal those of quantize_qkv + attention_fwd
    bit for bit, and therefore the oracle within the attention bars."""
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(19)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D), 1.5), dtype)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)) * rng.lognormal(0, 1, (1, Hkv, 1, D)).astype(np.float32), dtype)
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), dtype)
    s, si = oracle.calibrate(q, k) if smooth else (None, None)
    dq, dk, dv = (U.to_device(x, dtype) for x in (q, k, v))
    ds = None if s is None else torch.from_numpy(s).cuda()
    dsi = None if si is None else torch.from_numpy(si).cuda()
    pk = H.quantize_qkv(dq, dk, dv, ds, dsi)
    o_ref, l_ref = H.attention_fwd(pk, causal=causal, norm=norm, out_dtype=torch.float32)
    kv = H.quantize_kv(dk, dv, dsi, Hq=Hq, Nq=Nq)
    o, lse = H.attention_fwd_q(dq, kv, ds, causal=causal, norm=norm, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    if shape == (1, 4, 2, 384, 384, 128):
        ref = oracle.attention_rows(shape, oracle.all_rows(B, Hq, Nq), packed=oracle.quantize_qkv(q, k, v, s, si),
                                    causal=causal, norm_mode=0 if norm == "p_reorder" else 1)
        max_abs, rel = U.row_errors(o.cpu().numpy().reshape(-1, D), ref["O"])
        assert max_abs <= O_MAX_ABS and rel.max() <= O_ROW_REL
        assert np.abs(lse.cpu().numpy().ravel() - ref["lse"]).max() <= LSE_ABS
