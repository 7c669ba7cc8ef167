"""GPU parity of the steps around the hot path against the CPU oracle:
fused RoPE -> Smooth-QK -> quantize (also of Q alone), the Q-Mean auxiliary (mean, residual
quantization, score bias, attention with the bias), KV-cache append
quantization, and the epsilon-bar tile statistics.

Bars:
  codes and scales (RoPE, Q-Mean residual, appends)  bit-exact
  Q-Mean mean                                        bit-exact (fp64 sums on both sides)
  Q-Mean score bias (fp32 sum vs fp64)               |err| <= 1e-5 * sum |mean| |K'|
  attention with the bias                            the attention bars (P_hat mismatch
                                                     <= 1e-4, O, LSE)
  per-(row, tile) epsilon                            |err| <= 1e-5 on >= 99.9 % of the visited
                                                     (row, tile) pairs (a P_hat code flip moves it)
  per-tile epsilon-bar                               |err| <= 1e-4 vs the oracle's tile means
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import hifa4_testutil as U
from tests.test_gpu_parity import _check_attention, _rand

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import bit_quantized_flashattention_b200 as H
    H.load()
    return H


def _inputs(shape, dtype="bf16", seed=60, gain=1.0, offset=0.0):
    B, Hq, Hkv, Nq, Nkv, D = shape
    rng = np.random.default_rng(seed)
    off = (rng.standard_normal(D) * offset).astype(np.float32)
    q = W.round_to_dtype(_rand(rng, (B, Hq, Nq, D)) + off, dtype)
    g = rng.lognormal(0, gain, (1, Hkv, 1, D)).astype(np.float32)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)) * g, dtype)
    v = W.round_to_dtype(_rand(rng, (B, Hkv, Nkv, D)), dtype)
    return q, k, v


def _rope(H, D, n_pos, q_pos, k_pos):
    cos_t, sin_t = W.rope_tables(n_pos, D)
    dev = H.Rope(torch.from_numpy(cos_t).cuda(), torch.from_numpy(sin_t).cuda(),
                 torch.from_numpy(np.asarray(q_pos, np.int32)).cuda() if q_pos is not None else None,
                 torch.from_numpy(np.asarray(k_pos, np.int32)).cuda() if k_pos is not None else None)
    return cos_t, sin_t, dev


def _check_rows(pk, B, Hq, Hkv, Nq, Nkv, D, qc, qs, kc, ks):
    qs_g, ks_g, _ = U.canonical_scales(pk, B, Hq, Hkv, Nq, Nkv, D)
    if qc is not None:
        assert np.array_equal(pk.qc.cpu().numpy().reshape(qc.shape), qc)
        assert np.array_equal(qs_g, qs)
    assert np.array_equal(pk.kc.cpu().numpy().reshape(kc.shape), kc)
    assert np.array_equal(ks_g, ks)


# -------------------------------------------------------------------- RoPE

@pytest.mark.parametrize("shape,dtype,smooth", [
    ((1, 4, 2, 256, 256, 128), "bf16", True),
    ((2, 2, 1, 96, 384, 64), "fp16", False),          # ragged G*Nq (192 rows: 1.5 tiles)
    ((1, 2, 2, 128, 256, 256), "bf16", True),
])
def test_fused_rope_quantize_matches_oracle(H, shape, dtype, smooth):
    """RoPE -> Smooth-QK -> quantize in one pass: Q and K codes and scales equal
    the oracle's RoPE, smoothing and quantization steps run one after another;
    V is quantized without rotation. Positions are bottom-right aligned decode
    positions for Q and include clamped out-of-range entries for K."""
    B, Hq, Hkv, Nq, Nkv, D = shape
    q, k, v = _inputs(shape, dtype)
    n_pos = Nkv + 64
    q_pos = np.arange(Nq) + (Nkv - Nq) + 17
    k_pos = np.arange(Nkv) + 17
    k_pos[3], k_pos[-1] = -5, n_pos + 100             # clamped to 0 and n_pos - 1
    cos_t, sin_t, rope = _rope(H, D, n_pos, q_pos, k_pos)
    s = si = None
    if smooth:
        s, si = oracle.calibrate(oracle.rope_neox(q, cos_t, sin_t, q_pos),
                                 oracle.rope_neox(k, cos_t, sin_t, np.clip(k_pos, 0, n_pos - 1)))
    dq, dk, dv = (U.to_device(x, dtype) for x in (q, k, v))
    ds = None if s is None else torch.from_numpy(s).cuda()
    dsi = None if si is None else torch.from_numpy(si).cuda()
    pk = H.quantize_qkv(dq, dk, dv, ds, dsi, rope=rope)
    torch.cuda.synchronize()
    qp = oracle.prequant_rows(q, rope=(cos_t, sin_t, q_pos), scale=s, group=Hq // Hkv)
    kp = oracle.prequant_rows(k, rope=(cos_t, sin_t, np.clip(k_pos, 0, n_pos - 1)), scale=si)
    qc, qs = oracle.quantize_rows(qp)
    kc, ks = oracle.quantize_rows(kp)
    _check_rows(pk, B, Hq, Hkv, Nq, Nkv, D, qc, qs, kc, ks)
    vtc, vts = oracle.quantize_v(v)
    _, _, vts_g = U.canonical_scales(pk, B, Hq, Hkv, Nq, Nkv, D)
    assert np.array_equal(U.canonical_vtc(pk.vtc, B, Hkv, Nkv, D), vtc) and np.array_equal(vts_g, vts)


@pytest.mark.parametrize("shape,dtype,smooth,rope,qmean", [
    ((1, 4, 2, 48, 256, 128), "bf16", True, False, False),     # ragged G*Nq = 192 rows: padding rows
    ((2, 8, 1, 16, 128, 64), "fp16", False, True, False),       # decode-like: 8 heads x 16 queries
    ((1, 2, 2, 128, 256, 256), "bf16", True, True, True),
])
def test_quantize_q_alone_matches_oracle(H, shape, dtype, smooth, rope, qmean):
    """hifa4_quantize_q writes Q codes and scales (padding bytes included) equal
    to the oracle's RoPE, smoothing, Q-Mean and quantization steps, into the Q
    buffers of a packed KV cache, and leaves the cache's K and V untouched."""
    B, Hq, Hkv, Nq, Nkv, D = shape
    q, k, v = _inputs(shape, dtype, seed=62, offset=1.0 if qmean else 0.0)
    q_pos = np.arange(Nq) + (Nkv - Nq)
    cos_t, sin_t, drope = _rope(H, D, Nkv, q_pos, None)
    s = oracle.calibrate(q, k)[0] if smooth else None
    ds = None if s is None else torch.from_numpy(s).cuda()
    dq = U.to_device(q, dtype)
    cache = H.quantize_kv(U.to_device(k, dtype), U.to_device(v, dtype), Hq=Hq, Nq=Nq)
    torch.cuda.synchronize()
    kv_before = {n: t.clone() for n, t in cache.tensors().items() if n not in ("qc", "qs")}
    m = H.q_mean(dq, s=ds, rope=drope if rope else None, Hkv=Hkv) if qmean else None
    H.quantize_q(dq, cache, s=ds, rope=drope if rope else None, q_mean=m)
    torch.cuda.synchronize()
    qp = oracle.prequant_rows(q, rope=(cos_t, sin_t, q_pos) if rope else None, scale=s, group=Hq // Hkv,
                              mean=m.cpu().numpy() if qmean else None)
    qc, qs = oracle.quantize_rows(qp)
    qs_g, _, _ = U.canonical_scales(cache, B, Hq, Hkv, Nq, Nkv, D)
    assert np.array_equal(cache.qc.cpu().numpy().reshape(qc.shape), qc)
    assert np.array_equal(qs_g, qs)
    assert U.padding_bytes_ok(cache, B, Hq, Hkv, Nq, Nkv, D)
    for n, t in kv_before.items():
        assert torch.equal(getattr(cache, n), t), n


# ------------------------------------------------------------------ Q-Mean

@pytest.mark.parametrize("shape,rope,smooth", [
    ((2, 4, 2, 256, 256, 128), False, False),
    ((1, 2, 1, 1000 - 1000 % 16, 1024, 64), True, False),
    ((1, 2, 2, 16, 128, 256), True, True),
])
def test_q_mean_matches_oracle(H, shape, rope, smooth):
    B, Hq, Hkv, Nq, Nkv, D = shape
    q, k, _ = _inputs(shape, offset=2.0, seed=61)
    q_pos = np.arange(Nq) + (Nkv - Nq)
    cos_t, sin_t, drope = _rope(H, D, Nkv, q_pos, None)
    s = oracle.calibrate(q, k)[0] if smooth else None
    m = H.q_mean(U.to_device(q, "bf16"), s=None if s is None else torch.from_numpy(s).cuda(),
                 rope=drope if rope else None, Hkv=Hkv)
    torch.cuda.synchronize()
    want = oracle.q_mean(oracle.prequant_rows(q, rope=(cos_t, sin_t, q_pos) if rope else None, scale=s,
                                              group=Hq // Hkv))
    assert np.array_equal(m.cpu().numpy(), want)


@pytest.mark.parametrize("shape,causal", [
    ((1, 4, 2, 256, 256, 128), True),
    ((2, 2, 1, 128, 384, 64), False),
    ((1, 2, 1, 256, 256, 256), True),
])
@pytest.mark.parametrize("norm", ["p_reorder", "high_precision_l"])
def test_q_mean_attention_matches_oracle(H, shape, causal, norm):
    """Q-Mean end to end (Smooth-QK off, a shared Q offset): mean, residual
    codes, score bias and the attention that adds the bias back."""
    B, Hq, Hkv, Nq, Nkv, D = shape
    q, k, v = _inputs(shape, offset=3.0, seed=62)
    dq, dk, dv = (U.to_device(x, "bf16") for x in (q, k, v))
    m = H.q_mean(dq)
    pk = H.quantize_qkv(dq, dk, dv, q_mean=m)
    r = H.attention_fwd_ex(pk, causal=causal, norm=norm, out_dtype=torch.float32, s_bias=pk.s_bias, want_p=True)
    torch.cuda.synchronize()
    m_ref = oracle.q_mean(q)
    assert np.array_equal(m.cpu().numpy(), m_ref)
    qc, qs = oracle.quantize_rows(oracle.sub_mean(q, m_ref))
    kc, ks = oracle.quantize_rows(k)
    _check_rows(pk, B, Hq, Hkv, Nq, Nkv, D, qc, qs, kc, ks)
    bias_ref = oracle.q_mean_bias(m_ref, k, Hq)
    bound = 1e-5 * np.einsum("bhd,bgjd->bhj", np.abs(m_ref).astype(np.float64),
                             np.repeat(np.abs(k).astype(np.float64), Hq // Hkv, axis=1))
    assert np.all(np.abs(pk.s_bias.cpu().numpy() - bias_ref) <= bound)
    ref_p = dict(qc=qc, qs=qs, kc=kc, ks=ks)
    ref_p["vtc"], ref_p["vts"] = oracle.quantize_v(v)
    ref = oracle.attention_rows(shape, oracle.all_rows(B, Hq, Nq), packed=ref_p, causal=causal, s_bias=bias_ref,
                                norm_mode=0 if norm == "p_reorder" else 1, want_p=True)
    _check_attention(r["o"], r["lse"], r["p_codes"], r["p_scales"], ref, D)


# ------------------------------------------------------------ KV append

@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "fp16"), (256, "bf16")])
def test_append_chunks_equal_whole_quantization(H, D, dtype):
    """Appending ragged 16-aligned chunks (crossing 64- and 128-token
    boundaries, in shuffled order) gives the same cache bytes as quantizing
    all tokens at once, and the oracle's codes."""
    B, Hkv, N = 2, 2, 384
    rng = np.random.default_rng(63)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, N, D)) * rng.lognormal(0, 1, (1, Hkv, 1, D)).astype(np.float32), dtype)
    v = W.round_to_dtype(_rand(rng, (B, Hkv, N, D)), dtype)
    si = rng.lognormal(0, 0.5, (Hkv, D)).astype(np.float32)
    dk, dv = U.to_device(k, dtype), U.to_device(v, dtype)
    dsi = torch.from_numpy(si).cuda()
    whole = H.quantize_kv(dk, dv, dsi)
    cache = H.alloc_packed(B, Hkv, Hkv, 16, N, D)
    for t in (cache.kc, cache.ks, cache.vtc, cache.vts):
        t.fill_(0)
    cuts = [0, 16, 48, 112, 144, 208, 256, 272, 384]
    chunks = list(zip(cuts[:-1], cuts[1:]))
    rng.shuffle(chunks)
    for a, b in chunks:
        H.append_kv(cache, dk[:, :, a:b].contiguous(), dv[:, :, a:b].contiguous(), a, s_inv=dsi)
    torch.cuda.synchronize()
    for name in ("kc", "ks", "vtc", "vts"):
        assert torch.equal(getattr(cache, name), getattr(whole, name)), name
    kc, ks = oracle.quantize_rows(k, si, 1)
    vtc, vts = oracle.quantize_v(v)
    _, ks_g, vts_g = U.canonical_scales(cache, B, Hkv, Hkv, 16, N, D)
    assert np.array_equal(cache.kc.cpu().numpy().reshape(kc.shape), kc) and np.array_equal(ks_g, ks)
    assert np.array_equal(U.canonical_vtc(cache.vtc, B, Hkv, N, D), vtc) and np.array_equal(vts_g, vts)


def test_append_leaves_other_slots_untouched_and_applies_rope(H):
    B, Hkv, N, D = 1, 2, 256, 128
    rng = np.random.default_rng(64)
    k = W.round_to_dtype(_rand(rng, (B, Hkv, 48, D)), "bf16")
    v = W.round_to_dtype(_rand(rng, (B, Hkv, 48, D)), "bf16")
    start = 80                                        # crosses the 128-token tile at 128
    k_pos = np.arange(48) + start
    cos_t, sin_t, rope = _rope(H, D, N, None, k_pos)
    cache = H.alloc_packed(B, Hkv, Hkv, 16, N, D)
    for t in (cache.kc, cache.ks, cache.vtc, cache.vts):
        t.fill_(0xA5)
    before = {n: getattr(cache, n).clone() for n in ("kc", "ks", "vtc", "vts")}
    H.append_kv(cache, U.to_device(k, "bf16"), U.to_device(v, "bf16"), start, rope=rope)
    torch.cuda.synchronize()
    # expected: the bytes of the whole-cache quantization of a tensor holding
    # the new tokens, spliced into the sentinel-filled cache at their slots
    kc, ks = oracle.quantize_rows(oracle.prequant_rows(k, rope=(cos_t, sin_t, k_pos)))
    vtc, vts = oracle.quantize_v(v)
    kc_g = cache.kc.cpu().numpy().reshape(B, Hkv, N, D // 2)
    assert np.array_equal(kc_g[:, :, start:start + 48], kc)
    assert np.all(np.delete(kc_g, np.s_[start:start + 48], axis=2) == 0xA5)
    ks_idx = U.qk_scale_index(B, Hkv, Hkv, N, D)
    ks_bytes = cache.ks.cpu().numpy()
    canon = ks_bytes[ks_idx]                          # [B, Hkv, N, D/16]
    assert np.array_equal(canon[:, :, start:start + 48], ks)
    mask = np.ones(ks_bytes.shape, bool)
    mask[ks_idx[:, :, start:start + 48]] = False
    assert np.all(ks_bytes[mask] == 0xA5)
    vt_g = U.canonical_vtc(cache.vtc, B, Hkv, N, D)
    assert np.array_equal(vt_g[..., start // 2:(start + 48) // 2], vtc)
    assert np.all(np.delete(vt_g, np.s_[start // 2:(start + 48) // 2], axis=3) == 0xA5)
    vs_idx = U.v_scale_index(B, Hkv, N, D)
    vs_bytes = cache.vts.cpu().numpy()
    assert np.array_equal(vs_bytes[vs_idx][..., start // 16:(start + 48) // 16], vts)
    mask = np.ones(vs_bytes.shape, bool)
    mask[vs_idx[..., start // 16:(start + 48) // 16]] = False
    assert np.all(vs_bytes[mask] == 0xA5)
    assert torch.equal(before["kc"].view(-1)[:start * D // 2], cache.kc.view(-1)[:start * D // 2])


# ------------------------------------------------------- epsilon-bar tiles

@pytest.mark.parametrize("shape,causal,split_kv", [
    ((1, 4, 2, 384, 384, 128), True, False),
    ((2, 2, 1, 176, 512, 64), True, False),
    ((1, 8, 2, 16, 1024, 128), False, True),          # decode mode: 4 ranges
])
def test_tile_sums_and_eps_bar_match_oracle(H, shape, causal, split_kv):
    B, Hq, Hkv, Nq, Nkv, D = shape
    q, k, v = _inputs(shape, seed=65)
    s, si = oracle.calibrate(q, k)
    dq, dk, dv = (U.to_device(x, "bf16") for x in (q, k, v))
    pk = H.quantize_qkv(dq, dk, dv, torch.from_numpy(s).cuda(), torch.from_numpy(si).cuda())
    plain_o, plain_lse = H.attention_fwd(pk, causal=causal, out_dtype=torch.float32, split_kv=split_kv)
    r = H.attention_fwd_ex(pk, causal=causal, out_dtype=torch.float32, split_kv=split_kv, want_tile_sums=True)
    eb = H.tile_stats(r["tile_sums"])
    torch.cuda.synchronize()
    # the statistics do not change the result
    assert torch.equal(plain_o, r["o"]) and torch.equal(plain_lse, r["lse"])
    n_splits = H.attention_splits(B, Hq, Hkv, Nq, Nkv, D, causal=causal, split_kv=split_kv)
    ref = oracle.attention_rows(shape, oracle.all_rows(B, Hq, Nq), packed=oracle.quantize_qkv(q, k, v, s, si),
                                causal=causal, want_eps=True, n_splits=n_splits)
    ts = r["tile_sums"].cpu().numpy().reshape(B * Hq * Nq, Nkv // 128, 2).astype(np.float64)
    visited = ts[..., 1] > 0
    assert np.array_equal(visited, ~np.isnan(ref["eps"]))
    eps_g = np.where(visited, ts[..., 0] / np.where(visited, ts[..., 1], 1) - 1, np.nan)
    diff = np.abs(eps_g - ref["eps"])[visited]
    assert np.mean(diff > 1e-5) <= 1e-3, f"eps mismatch fraction {np.mean(diff > 1e-5):.2e}"
    # the tile kernel against the definition applied to the same sums, and the oracle's tile means
    want_same = oracle.eps_bar(eps_g, B, Hq, Nq)
    got = eb.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(want_same))
    assert np.nanmax(np.abs(got - want_same)) <= 1e-6
    assert np.nanmax(np.abs(got - oracle.eps_bar(ref["eps"], B, Hq, Nq))) <= 1e-4
