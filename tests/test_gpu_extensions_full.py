"""Parity of the steps around the hot path at the full workload sizes, in the
launch configuration `bench.py --extensions` times, against the CPU oracle on
sampled (batch, kv head) groups, query rows and tiles.

  Q-Mean on the N = 16384 workload (Smooth-QK off): mean and residual codes
      bit-exact, score bias within 1e-5 of sum |mean| |K'|, attention with the
      bias (score-bias variant) within the attention bars, P_hat mismatch
      <= 1e-4 (from the full-extras variant, whose O equals the timed one).
  epsilon-bar on the Qwen3-8B workload: per-(row, tile) epsilon and whole
      128-row tiles of the tile statistics against the oracle.
  Fused RoPE quantize on the Qwen3-8B workload: codes and scales bit-exact.
  KV-cache appends on the decode workload's cache (B = 64, 8192 slots):
      appended chunks byte-identical to the whole-cache quantization, and the
      oracle's codes on sampled groups.
  Attention with Q quantized in the kernel on the Qwen3-8B workload: O and
      LSE equal the packed path's bit for bit, every row (the packed path is
      oracle-checked on every row in test_gpu_configs.py).
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


def _groups(cfg):
    return sorted({(0, 0), (cfg.B - 1, cfg.Hkv - 1)})


def _rows(cfg, rng, n=24):
    i = np.unique(np.concatenate([np.arange(4), cfg.Nq - 1 - np.arange(4), rng.integers(0, cfg.Nq, n)]))
    return np.sort(i)


def _nibbles(c):
    return np.stack([c & 15, c >> 4], -1)


def test_q_mean_full_size(H):
    cfg = W.get(4)
    rng = np.random.default_rng(70)
    q, k, v, _ = U.upload_config(cfg)
    m = H.q_mean(q)
    pk = H.quantize_qkv(q, k, v, q_mean=m)
    timed = H.attention_fwd_ex(pk, causal=True, out_dtype=torch.float32, s_bias=pk.s_bias)
    full = H.attention_fwd_ex(pk, causal=True, out_dtype=torch.float32, s_bias=pk.s_bias, want_p=True)
    torch.cuda.synchronize()
    assert torch.equal(timed["o"], full["o"]) and torch.equal(timed["lse"], full["lse"])
    G = cfg.G
    n_codes = n_mism = 0
    for b, g in _groups(cfg):
        qh, kh, vh = U.group_arrays(cfg, b, g)
        hs = slice(g * G, (g + 1) * G)
        m_ref = oracle.q_mean(qh)
        assert np.array_equal(m[b, hs].cpu().numpy(), m_ref[0])
        qc, qs = oracle.quantize_rows(oracle.sub_mean(qh, m_ref))
        kc, ks = oracle.quantize_rows(kh)
        vtc, vts = oracle.quantize_v(vh)
        qs_all, ks_all, _ = U.canonical_scales(pk, cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D)
        assert np.array_equal(pk.qc.view(cfg.B, cfg.Hq, cfg.Nq, -1)[b, hs].cpu().numpy(), qc[0])
        assert np.array_equal(qs_all[b, hs], qs[0])
        bias_ref = oracle.q_mean_bias(m_ref, kh, G)
        bound = 1e-5 * np.abs(m_ref[0]).astype(np.float64) @ np.abs(kh[0, 0]).astype(np.float64).T
        assert np.all(np.abs(pk.s_bias[b, hs].cpu().numpy() - bias_ref[0]) <= bound)
        idx = _rows(cfg, rng)
        rows_local = np.concatenate([hh * cfg.Nq + idx for hh in range(G)])
        ref = oracle.attention_rows((1, G, 1, cfg.Nq, cfg.Nkv, cfg.D), rows_local,
                                    packed=dict(qc=qc, qs=qs, kc=kc, ks=ks, vtc=vtc, vts=vts), causal=True,
                                    s_bias=bias_ref, want_p=True)
        og = timed["o"][b, hs][:, idx].reshape(-1, cfg.D).cpu().numpy()
        max_abs, rel = U.row_errors(og, ref["O"])
        assert max_abs <= O_MAX_ABS and rel.max() <= O_ROW_REL, (b, g, max_abs, rel.max())
        assert np.abs(timed["lse"][b, hs][:, idx].reshape(-1).cpu().numpy() - ref["lse"]).max() <= LSE_ABS
        pcg = full["p_codes"][b, hs][:, idx].reshape(len(rows_local), -1).cpu().numpy()
        n_codes += pcg.size * 2
        n_mism += int((_nibbles(pcg) != _nibbles(ref["p_codes"])).sum())
    print(f"Q-Mean full size: P_hat code mismatch {n_mism} of {n_codes}")
    assert n_mism <= P_MISMATCH * n_codes


def test_eps_bar_full_size(H):
    cfg = W.get(2)
    q, k, v, calib = U.upload_config(cfg)
    s, s_inv = H.calibrate_smooth(calib[0], calib[1], cfg.alpha)
    pk = H.quantize_qkv(q, k, v, s, s_inv)
    r = H.attention_fwd_ex(pk, causal=True, out_dtype=torch.float32, want_tile_sums=True)
    eb = H.tile_stats(r["tile_sums"]).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    ref_s, ref_si = oracle.calibrate(*U.calib_arrays(cfg), cfg.alpha)
    G = cfg.G
    T = cfg.Nkv // 128
    for b, g in _groups(cfg):
        qh, kh, vh = U.group_arrays(cfg, b, g)
        ref_p = oracle.quantize_qkv(qh, kh, vh, ref_s[g:g + 1], ref_si[g:g + 1])
        # whole 128-row query tiles: the first, a middle and the last one of one head
        hh = G - 1
        for a in (0, cfg.Nq // 256, cfg.Nq // 128 - 1):
            idx = np.arange(128 * a, 128 * a + 128)
            ref = oracle.attention_rows((1, G, 1, cfg.Nq, cfg.Nkv, cfg.D), hh * cfg.Nq + idx, packed=ref_p,
                                        causal=True, want_eps=True)
            ts = r["tile_sums"][b, g * G + hh, idx].cpu().numpy().astype(np.float64)
            visited = ts[..., 1] > 0
            assert np.array_equal(visited, ~np.isnan(ref["eps"]))
            eps_g = np.where(visited, ts[..., 0] / np.where(visited, ts[..., 1], 1) - 1, np.nan)
            diff = np.abs(eps_g - ref["eps"])[visited]
            assert np.mean(diff > 1e-5) <= 1e-3
            want = oracle.eps_bar(ref["eps"], 1, 1, 128)[0, 0, 0]
            got = eb[b, g * G + hh, a]
            assert np.array_equal(np.isnan(got), np.isnan(want))
            assert np.nanmax(np.abs(got - want)) <= 1e-4
    assert eb.shape == (cfg.B, cfg.Hq, cfg.Nq // 128, T)


def test_rope_quantize_full_size(H):
    cfg = W.get(2)
    q, k, v, calib = U.upload_config(cfg)
    s, s_inv = H.calibrate_smooth(calib[0], calib[1], cfg.alpha)
    cos_t, sin_t = W.rope_tables(cfg.Nkv, cfg.D)
    pos = np.arange(cfg.Nkv, dtype=np.int32)
    rope = H.Rope(torch.from_numpy(cos_t).cuda(), torch.from_numpy(sin_t).cuda(),
                  torch.from_numpy(pos[cfg.Nkv - cfg.Nq:]).cuda(), torch.from_numpy(pos).cuda())
    pk = H.quantize_qkv(q, k, v, s, s_inv, rope=rope)
    torch.cuda.synchronize()
    qs_all, ks_all, vts_all = U.canonical_scales(pk, cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D)
    s_h, si_h = s.cpu().numpy(), s_inv.cpu().numpy()
    G = cfg.G
    for b, g in _groups(cfg):
        qh, kh, vh = U.group_arrays(cfg, b, g)
        qc, qs = oracle.quantize_rows(oracle.prequant_rows(qh, rope=(cos_t, sin_t, pos[cfg.Nkv - cfg.Nq:]),
                                                           scale=s_h[g:g + 1], group=G))
        kc, ks = oracle.quantize_rows(oracle.prequant_rows(kh, rope=(cos_t, sin_t, pos), scale=si_h[g:g + 1]))
        hs = slice(g * G, (g + 1) * G)
        assert np.array_equal(pk.qc.view(cfg.B, cfg.Hq, cfg.Nq, -1)[b, hs].cpu().numpy(), qc[0])
        assert np.array_equal(qs_all[b, hs], qs[0])
        assert np.array_equal(pk.kc.view(cfg.B, cfg.Hkv, cfg.Nkv, -1)[b, g].cpu().numpy(), kc[0, 0])
        assert np.array_equal(ks_all[b, g], ks[0, 0])


def test_append_full_size(H):
    cfg = W.get(5)
    _, k, v, calib = U.upload_config(cfg)
    s, s_inv = H.calibrate_smooth(calib[0], calib[1], cfg.alpha)
    whole = H.quantize_kv(k, v, s_inv, Hq=cfg.Hq, Nq=cfg.Nq)
    cache = H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D)
    for t in (cache.kc, cache.ks, cache.vtc, cache.vts):
        t.fill_(0)
    # a prefill chunk, then ragged chunks, then 16-token decode appends
    cuts = [0, 4096, 6144, 7168, 7680, 7936, 8064] + list(range(8080, cfg.Nkv + 1, 16))
    for a, c in zip(cuts[:-1], cuts[1:]):
        H.append_kv(cache, k[:, :, a:c].contiguous(), v[:, :, a:c].contiguous(), a, s_inv=s_inv)
    torch.cuda.synchronize()
    for name in ("kc", "ks", "vtc", "vts"):
        assert torch.equal(getattr(cache, name), getattr(whole, name)), name
    _, ks_all, vts_all = U.canonical_scales(cache, cfg.B, cfg.Hkv, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D)
    si_h = s_inv.cpu().numpy()
    for b, g in _groups(cfg):
        _, kh, vh = U.group_arrays(cfg, b, g)
        kc, ks = oracle.quantize_rows(kh, si_h[g:g + 1])
        vtc, vts = oracle.quantize_v(vh)
        assert np.array_equal(cache.kc.view(cfg.B, cfg.Hkv, cfg.Nkv, -1)[b, g].cpu().numpy(), kc[0, 0])
        assert np.array_equal(ks_all[b, g], ks[0, 0])
        vt = U.canonical_vtc(cache.vtc.view(cfg.B, cfg.Hkv, -1)[b, g], 1, 1, cfg.Nkv, cfg.D)[0, 0]
        assert np.array_equal(vt, vtc[0, 0]) and np.array_equal(vts_all[b, g], vts[0, 0])


def test_in_kernel_q_quantization_full_size(H):
    """The Qwen3-8B workload through hifa4_attention_fwd_q (Q quantized in the
    attention kernel) equals quantize_qkv + attention_fwd bit for bit, every row."""
    cfg = W.get(2)
    q, k, v, calib = U.upload_config(cfg)
    s, s_inv = H.calibrate_smooth(calib[0], calib[1], cfg.alpha)
    pk = H.quantize_qkv(q, k, v, s, s_inv)
    kv = H.quantize_kv(k, v, s_inv, Hq=cfg.Hq, Nq=cfg.Nq)
    for norm in cfg.modes:
        o_ref, l_ref = H.attention_fwd(pk, causal=True, norm=norm)
        o, lse = H.attention_fwd_q(q, kv, s, causal=True, norm=norm)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref), norm
