"""Benchmark of the 4-bit attention forward hot path on B200.

One step = one pass of the hot path over the Qwen3-8B-shaped causal prefill
(B=1, 32 q heads / 8 kv heads, D=128, N=4096, bf16 inputs, Smooth-QK from a
512-token calibration batch, P-Reordering): smooth + quantize Q, K, V
(hifa4_quantize_qkv) and the fused 4-bit attention (hifa4_attention_fwd).
Calibration is offline (once per layer) and runs before the timed region.

value    attention FLOPs (4*B*Hq*Nq*Nkv*D/2 for causal) per second over the
         whole step, inputs resident in HBM, L2 flushed between steps
e2e      the same metric through the public API with host buffers: pinned
         host->device copy of Q, K, V, the step, device->host copy of O, LSE
roofline the attention kernel alone against its bound: the FP4 dense tensor
         peak (prefill), or the HBM copy bandwidth (split-kv decode chunks)
context  torch bf16 SDPA on the same inputs and GPU; error of the 4-bit
         output against unquantized fp32 attention (torch fp32 SDPA) on
         sampled groups; a measured NVFP4 GEMM peak (torch scaled_mm)
cpu_baseline  the CPU oracle on a bounded sample of the same workload, on all
         host cores and on one core

``--impl reference`` times the CPU oracle (the slow, plainly written CPU
implementation of the same computation) on the host cores instead.
``--all-configs`` times every workload (both normalizer modes where the
workload names two) and prints one JSON line each; ``--table PATH`` also
writes them as a markdown table. ``--ingest-ncu CSV --workload NAME`` records
the DRAM bytes per attention launch from an ncu CSV capture (with the
kernel-source hash it belongs to) in profiles/attn_traffic.json.
Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no exchange step); value sums the ranks' work over the max time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "4-bit attn fwd TFLOPS & % of B200 FP4 tensor peak, Qwen3-8B shape N=4096"
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Leave L2 cold and clean between steps: write a buffer twice the size of
    L2, then read another one, so no input of the step is cached and the step
    does not pay for writing back someone else's dirty lines."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self, i=0):
        self.w.fill_(i & 0xFF)
        return self.r.sum()


def peaks():
    """Measured HBM and bf16 peaks of this machine (driver-written); FP4 = 4 x bf16 (nominal 9 / 2.25)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return dict(hbm=float(m["hbm_gbs"]), bf16=float(m["bf16_tflops"]),
                    bf16_sus=float(m["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


ATTN_SOURCES = ("bit_quantized_flashattention_b200/csrc/attention.cu",
                "bit_quantized_flashattention_b200/csrc/hifa4_device.cuh")


def attention_source_hash() -> str:
    """sha256 over the attention kernel's sources (the kernel version a profile was taken on)."""
    import hashlib
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "attn_traffic.json")


def profiled_traffic(cfg):
    """DRAM bytes per attention launch of this workload as recorded from an ncu
    capture by --ingest-ncu, or None when there is none or the kernel sources
    changed since it was captured."""
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f).get(cfg.name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha256") != attention_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


def ingest_ncu(csv_path, workload, command, scale=1.0):
    """Sum dram__bytes_read/write of the attention kernel's captured launches in an
    ncu CSV (``ncu --csv --metrics dram__bytes_read.sum,dram__bytes_write.sum ...``)
    and record the per-launch mean, with the kernel-source hash, in the JSON.
    scale > 1: the capture ran a smaller batch of the workload whose traffic grows
    in proportion to the batch; the recorded bytes are scaled to the full launch."""
    import csv
    per_launch = {}
    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    for row in csv.DictReader(lines):
        if "attn_fwd_kernel" not in row.get("Kernel Name", ""):
            continue
        name, unit, val = row["Metric Name"], row.get("Metric Unit", ""), row["Metric Value"].replace(",", "")
        unit_scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(unit, 1)
        if name in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            per_launch.setdefault(row["ID"], 0.0)
            per_launch[row["ID"]] += float(val) * unit_scale
    if not per_launch:
        raise SystemExit(f"no attn_fwd_kernel DRAM counters in {csv_path}")
    rec = {}
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        pass
    rec[workload] = {"dram_bytes_per_launch": int(round(statistics.mean(per_launch.values()) * scale)),
                     "launches": len(per_launch), "source_sha256": attention_source_hash(), "command": command}
    if scale != 1.0:
        rec[workload]["scaled_from_capture_by"] = scale
    os.makedirs(os.path.dirname(TRAFFIC_JSON), exist_ok=True)
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(rec, f, indent=1, sort_keys=True)
    print(json.dumps({workload: rec[workload]}))


def max_over_ranks(x: float, device) -> float:
    """Maximum of x over the ranks of the default process group (x itself on one
    rank). Every rank calls it at the same points, error checks included."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix=f"hifa4_clocks{self.index}_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        try:
            with open(self.path) as f:
                rows = [r.split(",") for r in f.read().strip().splitlines()]
            os.unlink(self.path)
            rows = [[c.strip() for c in r] for r in rows if len(r) >= 9]
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ inputs

def make_inputs(cfg, device, rank=0):
    """Seeded inputs on the device, built slice by slice (rank > 0: other data seeds)."""
    import torch
    TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}
    if rank:
        cfg = cfg.replace(index=cfg.index + 100 * rank)
    gains = W.k_gains(cfg)
    dt = TORCH_DT[cfg.dtype]

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
    cal = None
    if cfg.smooth == "calib":
        cq = torch.stack([up(W.qcal_slice(cfg, h)) for h in range(cfg.Hq)])[None]
        ck = torch.stack([up(W.kcal_slice(cfg, g, gains)) for g in range(cfg.Hkv)])[None]
        cal = (cq.contiguous(), ck.contiguous())
    elif cfg.smooth == "self":
        cal = (q, k)
    return q, k, v, cal


# -------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, seconds_target=12.0, n_threads=0, rows_per_head=None, n_splits=1):
    """Time the CPU oracle on a bounded sample of the workload: kv groups'
    quantization plus the attention of a strided subset of their query rows
    (n_threads = 0: all host cores). The row count grows to the target CPU
    time; once a group's rows are all in, further groups are added.
    Returns (flops_of_sample / seconds, description, seconds)."""
    flops, dt, desc = _oracle_group(cfg, 0, seconds_target, n_threads, rows_per_head, n_splits)
    groups = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    n = 1
    while dt < 0.75 * seconds_target and n < len(groups) and "all rows" in desc:
        f1, d1, _ = _oracle_group(cfg, n, seconds_target, n_threads, cfg.Nq, n_splits)
        flops, dt, n = flops + f1, dt + d1, n + 1
    if n > 1:
        desc = f"{n} (b, kv head) groups, each: {desc}"
    return flops / dt, desc, dt


def _oracle_group(cfg, gi, seconds_target, n_threads, rows_per_head, n_splits):
    """One group of the oracle sample: (flops, seconds, description)."""
    import oracle
    gains = W.k_gains(cfg)
    b, g = divmod(gi, cfg.Hkv)
    G = cfg.G
    q = np.stack([W.q_slice(cfg, b, g * G + hh) for hh in range(G)])[None]
    k = W.k_slice(cfg, b, g, gains)[None, None]
    v = W.v_slice(cfg, b, g)[None, None]
    s = si = None
    if cfg.smooth == "calib":
        qc = np.stack([W.qcal_slice(cfg, g * G + hh) for hh in range(G)])[None]
        kc = W.kcal_slice(cfg, g, gains)[None, None]
        s, si = oracle.calibrate(qc, kc, cfg.alpha)
    elif cfg.smooth == "self":
        s, si = oracle.calibrate(q, k, cfg.alpha)
    shape = (1, G, 1, cfg.Nq, cfg.Nkv, cfg.D)
    # rows spread over the causal range (stride keeps the average key count of the full set)
    n_rows = rows_per_head or max(8, min(cfg.Nq, 64))
    idx = np.linspace(0, cfg.Nq - 1, n_rows).astype(np.int64)
    rows = np.concatenate([hh * cfg.Nq + idx for hh in range(G)])
    t0 = time.perf_counter()
    pk = oracle.quantize_qkv(q, k, v, s, si)
    oracle.attention_rows(shape, rows, packed=pk, causal=cfg.causal, n_threads=n_threads, n_splits=n_splits)
    dt = time.perf_counter() - t0
    if cfg.causal:
        keys = np.minimum(idx + cfg.Nkv - cfg.Nq + 1, cfg.Nkv)
    else:
        keys = np.full(idx.shape, cfg.Nkv)
    flops = 4.0 * cfg.D * float(keys.sum()) * G
    # grow the sample to the target CPU time
    if dt < seconds_target / 4 and n_rows < cfg.Nq:
        scale = min(cfg.Nq / n_rows, max(2.0, seconds_target / max(dt, 1e-3)))
        return _oracle_group(cfg, gi, seconds_target, n_threads, int(min(cfg.Nq, n_rows * scale)), n_splits)
    which = "all rows" if n_rows == cfg.Nq else f"{n_rows} per head, evenly spaced"
    desc = (f"quantize one (b, kv head) group (Q {G}x{cfg.Nq}x{cfg.D}, K/V {cfg.Nkv}x{cfg.D}) + attention of "
            f"{rows.size} query rows ({which}) of that group")
    return flops, dt, desc


# ----------------------------------------------------------------- our arm

def attn_bytes(cfg, H):
    """Algorithmic HBM bytes of one attention launch: the packed operands read
    once, O (bf16) and LSE written."""
    packed = sum(H.packed_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D))
    return packed + cfg.B * cfg.Hq * cfg.Nq * (cfg.D * 2 + 4)


def fp4_gemm_peak(device):
    """Dense block-scaled FP4 (NVFP4: E2M1, E4M3 per 16) GEMM throughput of this
    GPU, 8192^3 through torch's scaled_mm (cuBLASLt), best of 10; None when this
    torch cannot run it."""
    import torch
    import torch.nn.functional as F
    try:
        from torch.nn.functional import ScalingType, SwizzleType
        M = N = K = 8192
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=device).view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=device).view(torch.float4_e2m1fn_x2)
        sa = torch.full((M * (K // 16),), 1.0, device=device).to(torch.float8_e4m3fn)
        sb = torch.full((N * (K // 16),), 1.0, device=device).to(torch.float8_e4m3fn)

        def f():
            return F.scaled_mm(a, b.t(), sa, ScalingType.BlockWise1x16, sb, ScalingType.BlockWise1x16,
                               swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                               output_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        ts = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return 2.0 * M * N * K / (min(ts) * 1e-3) / 1e12
    except Exception:
        return None


def sdpa_context(q, k, v, cfg, flush):
    """torch bf16 scaled_dot_product_attention on the same inputs (same FLOP formula)."""
    import torch
    import torch.nn.functional as F
    ts = []
    for i in range(8):
        flush(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        F.scaled_dot_product_attention(q, k, v, is_causal=cfg.causal, enable_gqa=True)
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(e0.elapsed_time(e1))
    return round(cfg.flops() / (statistics.mean(ts) * 1e-3) / 1e12, 2)


def error_vs_fp32(H, packed, q, k, v, cfg, norm, split_kv, max_groups=2):
    """Error of the 4-bit output (fp32) against unquantized fp32 softmax attention
    of the same bf16 inputs (torch fp32 SDPA), on up to max_groups (b, kv head)
    groups: max abs error and max / median per-row relative L2. Context only."""
    import torch
    import torch.nn.functional as F
    o4, _ = H.attention_fwd(packed, causal=cfg.causal, norm=norm, out_dtype=torch.float32, split_kv=split_kv)
    G = cfg.G
    errs, rels = [], []
    groups = [(0, 0), (cfg.B - 1, cfg.Hkv - 1)][:max_groups]
    for b, g in sorted(set(groups)):
        hs = slice(g * G, (g + 1) * G)
        qq = q[b:b + 1, hs].float()
        kk = k[b:b + 1, g:g + 1].float().expand(1, G, cfg.Nkv, cfg.D)
        vv = v[b:b + 1, g:g + 1].float().expand(1, G, cfg.Nkv, cfg.D)
        ref = F.scaled_dot_product_attention(qq, kk, vv, is_causal=cfg.causal)
        d = (o4[b:b + 1, hs] - ref).double()
        errs.append(float(d.abs().max()))
        rels.append((d.norm(dim=-1) / ref.double().norm(dim=-1).clamp_min(1e-30)).flatten())
    rel = torch.cat(rels)
    return {"max_abs": round(max(errs), 6), "row_rel_l2_max": round(float(rel.max()), 6),
            "row_rel_l2_median": round(float(rel.median()), 6), "groups": len(rels),
            "reference": "torch fp32 SDPA on the bf16 inputs (unquantized)"}


def eps_stats(H, packed, cfg, norm, split_kv):
    """The epsilon-bar statistic of the HiFA4 abstract on this workload: per
    (128-query-row, 128-key) tile, the mean over its rows with mass of
    sum P_hat / sum P - 1, from the kernel's tile sums (one extra launch of the
    statistics variant, outside every timed region)."""
    import torch
    r = H.attention_fwd_ex(packed, causal=cfg.causal, norm=norm, out_dtype=torch.bfloat16, split_kv=split_kv,
                           want_tile_sums=True)
    eb = H.tile_stats(r["tile_sums"])
    x = eb[~torch.isnan(eb)].double()
    out = {"tiles": int(x.numel()), "negative_frac": round(float((x < 0).double().mean()), 6),
           "median": round(float(x.median()), 6), "mean": round(float(x.mean()), 6),
           "p05": round(float(torch.quantile(x.float(), 0.05)), 6),
           "p95": round(float(torch.quantile(x.float(), 0.95)), 6)}
    del r, eb
    return out


def time_fn(fn, n, flush, stream):
    """Mean device time (ms) of fn over n calls, L2 cold before each."""
    import torch
    fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush(i)
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def run_extensions(args, dev, H):
    """Timings of the steps around the hot path (one JSON line each): the
    Q-Mean auxiliary on the Smooth-QK-off workload, the fused RoPE quantize
    pass, KV-cache appends on the decode workload, and the epsilon statistics."""
    import torch
    import torch.nn.functional as F
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    n = args.steps
    rows = []

    def emit(rec):
        print(json.dumps(rec), flush=True)
        rows.append(rec)

    # Q-Mean on the N = 16384 workload (Smooth-QK off)
    cfg = W.get(4)
    q, k, v, _ = make_inputs(cfg, dev)
    packed = H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
    o = torch.empty(cfg.B, cfg.Hq, cfg.Nq, cfg.D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Nq, dtype=torch.float32, device=dev)
    wsp = H.alloc_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
    qm = torch.empty(cfg.B, cfg.Hq, cfg.D, dtype=torch.float32, device=dev)
    bias = torch.empty(cfg.B, cfg.Hq, cfg.Nkv, dtype=torch.float32, device=dev)
    t_plain_q = time_fn(lambda: H.quantize_qkv(q, k, v, out=packed), n, flush, stream)
    t_plain_a = time_fn(lambda: H.attention_fwd(packed, causal=True, out=o, lse=lse, workspace=wsp), n, flush, stream)
    t_mean = time_fn(lambda: H.q_mean(q, out=qm), n, flush, stream)
    t_qm_q = time_fn(lambda: H.quantize_qkv(q, k, v, out=packed, q_mean=qm, s_bias=bias), n, flush, stream)
    t_qm_a = time_fn(lambda: H.attention_fwd_ex(packed, causal=True, out=o, lse=lse, workspace=wsp, s_bias=bias),
                     n, flush, stream)
    errs = {}
    for name, use in (("plain", False), ("q_mean", True)):
        H.quantize_qkv(q, k, v, out=packed, q_mean=qm if use else None, s_bias=bias if use else None)
        o4 = H.attention_fwd_ex(packed, causal=True, out_dtype=torch.float32, s_bias=bias if use else None)["o"]
        b, g = 0, 0
        hs = slice(0, cfg.G)
        qq = q[b:b + 1, hs].float()
        kk = k[b:b + 1, g:g + 1].float().expand(1, cfg.G, cfg.Nkv, cfg.D)
        vv = v[b:b + 1, g:g + 1].float().expand(1, cfg.G, cfg.Nkv, cfg.D)
        ref = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
        d = (o4[b:b + 1, hs] - ref).double()
        rel = (d.norm(dim=-1) / ref.double().norm(dim=-1).clamp_min(1e-30)).flatten()
        errs[name] = {"max_abs": round(float(d.abs().max()), 6), "row_rel_l2_median": round(float(rel.median()), 6)}
    fl = cfg.flops()
    emit({"extension": "q_mean", "workload": cfg.name, "q_mean_ms": round(t_mean, 5),
          "quantize_ms": {"plain": round(t_plain_q, 5), "q_mean": round(t_qm_q, 5)},
          "attention_ms": {"plain": round(t_plain_a, 5), "q_mean_bias": round(t_qm_a, 5)},
          "attention_tflops": {"plain": round(fl / t_plain_a / 1e9, 1), "q_mean_bias": round(fl / t_qm_a / 1e9, 1)},
          "error_vs_fp32_group0": errs,
          "note": "attention with the bias runs the extras variant of the kernel"})
    del q, k, v, packed, o, lse, qm, bias
    torch.cuda.empty_cache()

    # fused RoPE -> Smooth-QK -> quantize on the headline workload
    cfg = W.get(2)
    q, k, v, cal = make_inputs(cfg, dev)
    s, s_inv = H.calibrate_smooth(cal[0], cal[1], cfg.alpha)
    cos_t, sin_t = W.rope_tables(cfg.Nkv, cfg.D)
    pos = torch.arange(cfg.Nkv, dtype=torch.int32, device=dev)
    rope = H.Rope(torch.from_numpy(cos_t).to(dev), torch.from_numpy(sin_t).to(dev), pos[cfg.Nkv - cfg.Nq:].contiguous(),
                  pos)
    packed = H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
    t0 = time_fn(lambda: H.quantize_qkv(q, k, v, s, s_inv, out=packed), n, flush, stream)
    t1 = time_fn(lambda: H.quantize_qkv(q, k, v, s, s_inv, out=packed, rope=rope), n, flush, stream)
    elems = cfg.B * cfg.Hq * cfg.Nq * cfg.D + 2 * cfg.B * cfg.Hkv * cfg.Nkv * cfg.D
    nbytes = elems * (2 + 0.5625)
    emit({"extension": "rope_quantize", "workload": cfg.name, "quantize_ms": round(t0, 5),
          "rope_quantize_ms": round(t1, 5), "quantize_gbs": round(nbytes / t0 / 1e6, 1),
          "rope_quantize_gbs": round(nbytes / t1 / 1e6, 1),
          "bytes": "algorithmic: 2 B read + 0.5625 B written per Q/K/V element (tables stay in L2)"})

    # epsilon statistics on the headline workload
    H.quantize_qkv(q, k, v, s, s_inv, out=packed)
    o = torch.empty(cfg.B, cfg.Hq, cfg.Nq, cfg.D, dtype=torch.bfloat16, device=dev)
    ts = torch.zeros(cfg.B, cfg.Hq, cfg.Nq, cfg.Nkv // 128, 2, dtype=torch.float32, device=dev)
    eb = torch.empty(cfg.B, cfg.Hq, cfg.Nq // 128, cfg.Nkv // 128, dtype=torch.float32, device=dev)
    ta = time_fn(lambda: H.attention_fwd(packed, causal=True, out=o), n, flush, stream)
    te = time_fn(lambda: H.attention_fwd_ex(packed, causal=True, out=o, tile_sums=ts), n, flush, stream)
    tt = time_fn(lambda: H.tile_stats(ts, out=eb), n, flush, stream)
    emit({"extension": "eps_statistics", "workload": cfg.name, "attention_ms": round(ta, 5),
          "attention_with_tile_sums_ms": round(te, 5), "tile_stats_ms": round(tt, 5),
          "eps_bar": eps_stats(H, packed, cfg, "p_reorder", False)})
    del q, k, v, packed, o, ts, eb
    torch.cuda.empty_cache()

    # the step with Q quantized inside the attention kernel (quantize K/V only)
    for ci in (2, 4):
        cfg = W.get(ci)
        q, k, v, cal = make_inputs(cfg, dev)
        s = s_inv = None
        if cal is not None:
            s, s_inv = H.calibrate_smooth(cal[0], cal[1], cfg.alpha)
        packed = H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
        o = torch.empty(cfg.B, cfg.Hq, cfg.Nq, cfg.D, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(cfg.B, cfg.Hq, cfg.Nq, dtype=torch.float32, device=dev)
        wsp = H.alloc_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
        tq = time_fn(lambda: H.quantize_qkv(q, k, v, s, s_inv, out=packed), n, flush, stream)
        ta = time_fn(lambda: H.attention_fwd(packed, causal=cfg.causal, out=o, lse=lse, workspace=wsp), n, flush,
                     stream)
        tkv = time_fn(lambda: H.quantize_kv(k, v, s_inv, out=packed), n, flush, stream)
        taq = time_fn(lambda: H.attention_fwd_q(q, packed, s, causal=cfg.causal, out=o, lse=lse, workspace=wsp), n,
                      flush, stream)
        emit({"extension": "in_kernel_q_quantization", "workload": cfg.name,
              "packed_path_ms": {"quantize_qkv": round(tq, 5), "attention_fwd": round(ta, 5),
                                 "sum": round(tq + ta, 5)},
              "fused_path_ms": {"quantize_kv": round(tkv, 5), "attention_fwd_q": round(taq, 5),
                                "sum": round(tkv + taq, 5)}})
        del q, k, v, packed, o, lse
        torch.cuda.empty_cache()

    # KV-cache append on the decode workload (B = 64, 8 kv heads, 8192 slots)
    cfg = W.get(5)
    cache = H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
    for n_new in (16, 1024):
        kn = torch.randn(cfg.B, cfg.Hkv, n_new, cfg.D, device=dev).to(torch.bfloat16)
        vn = torch.randn_like(kn)
        start = cfg.Nkv - n_new
        t = time_fn(lambda: H.append_kv(cache, kn, vn, start), n, flush, stream)
        nb = 2 * kn.numel() * (2 + 0.5625)
        emit({"extension": "append_kv", "workload": cfg.name, "new_tokens": n_new, "start": start,
              "ms": round(t, 5), "gbs": round(nb / t / 1e6, 1),
              "bytes": "algorithmic: new K and V, 2 B read + 0.5625 B written per element"})
    if args.table:
        with open(args.table, "w") as f:
            for rec in rows:
                f.write(json.dumps(rec) + "\n")


def measure(cfg, norm, args, dev, rank, ws, H, want_e2e=True):
    """Time one workload: the step (quantize + attention, one CUDA graph) with a
    cold L2, the two kernels separately, and (want_e2e) the end-to-end loop."""
    import torch
    import torch.distributed as dist
    q, k, v, cal = make_inputs(cfg, dev, rank)
    s = s_inv = None
    if cal is not None:
        s, s_inv = H.calibrate_smooth(cal[0], cal[1], cfg.alpha)
    split_kv = True               # decode-style chunks take the split-kv mode (one pass otherwise)
    n_splits = H.attention_splits(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, causal=cfg.causal, split_kv=True)
    packed = H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
    o = torch.empty(cfg.B, cfg.Hq, cfg.Nq, cfg.D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.B, cfg.Hq, cfg.Nq, dtype=torch.float32, device=dev)
    wsp = H.alloc_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    # fused_q: the attention kernel quantizes Q itself (D = 128 outside the
    # decode mode; same result, bit for bit) and the quantize pass covers K and
    # V only. Measured a tie on the Qwen3-8B step, so the step keeps the packed
    # path; --extensions times both.
    fused_q = getattr(args, "fused_q", False) and cfg.D == 128 and n_splits == 1

    def quant():
        if fused_q:
            H.quantize_kv(k, v, s_inv, out=packed)
        else:
            H.quantize_qkv(q, k, v, s, s_inv, out=packed)

    def attn():
        if fused_q:
            H.attention_fwd_q(q, packed, s, causal=cfg.causal, norm=norm, out=o, lse=lse, workspace=wsp)
        else:
            H.attention_fwd(packed, causal=cfg.causal, norm=norm, out=o, lse=lse, workspace=wsp, split_kv=split_kv)

    def step():
        quant()
        attn()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = max_over_ranks(H.get_status(wsp), dev)
    if st != 0:
        raise RuntimeError(f"kernel status {int(st)} during warm-up (max over ranks)")

    # The timed loop replays the step from a CUDA graph captured after the
    # warm-up calls: the device timeline then holds the two kernels back to
    # back (the attention launch overlaps the quantize tail through
    # programmatic dependent launch), without host-side gaps. A second loop
    # replays each kernel from its own graph to split the step's time.
    g_step, g_quant, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    with torch.cuda.graph(g_quant):
        quant()
    with torch.cuda.graph(g_attn):
        attn()
    for g in (g_step, g_quant, g_attn):
        g.replay()
    torch.cuda.synchronize()

    n = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        for i in range(n):
            flush(i)
            ev[i][0].record(stream)
            g_step.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # per-kernel split (same inputs, same L2 flush before each step)
    ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush(i)
        ev3[i][0].record(stream)
        g_quant.replay()
        ev3[i][1].record(stream)
        g_attn.replay()
        ev3[i][2].record(stream)
    torch.cuda.synchronize()
    attn_ms = [b.elapsed_time(c) for _, b, c in ev3]
    quant_ms = [a.elapsed_time(b) for a, b, _ in ev3]
    total_ms = max_over_ranks(float(sum(step_ms)), dev)
    st = max_over_ranks(H.get_status(wsp), dev)
    if st != 0:
        raise RuntimeError(f"kernel status {int(st)} in the timed region (max over ranks)")
    if fused_q:
        H.quantize_qkv(q, k, v, s, s_inv, out=packed)      # packed Q_hat for the untimed extras
    res = dict(q=q, k=k, v=v, s=s, s_inv=s_inv, packed=packed, o=o, lse=lse, wsp=wsp, flush=flush,
               total_ms=total_ms, attn_ms=statistics.mean(attn_ms), quant_ms=statistics.mean(quant_ms),
               clocks=clk.summary(), n_splits=n_splits, split_kv=split_kv, fused_q=fused_q)
    del g_step, g_quant, g_attn
    if not want_e2e:
        return res

    # End to end through the public API: every step copies its inputs from
    # pinned host memory and reads its results (O and the LSE) back to pinned
    # host memory. Consecutive steps overlap on three streams with
    # double-buffered device tensors: the inputs of step i+1 and the results of
    # step i-1 cross PCIe while step i computes.
    hq = q.cpu().pin_memory()
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    nb = 2
    dq, dk, dv = [q, torch.empty_like(q)], [k, torch.empty_like(k)], [v, torch.empty_like(v)]
    do, dl = [o, torch.empty_like(o)], [lse, torch.empty_like(lse)]
    dpk = [packed, H.alloc_packed(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)]
    dws = [wsp, H.alloc_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.Nq, cfg.Nkv, cfg.D, dev)]
    ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(nb)]
    hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(nb)]
    s_in, s_cp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in, ev_cp, ev_out = ([torch.cuda.Event() for _ in range(nb)] for _ in range(3))

    def e2e_step(i):
        b = i % nb
        with torch.cuda.stream(s_in):
            if i >= nb:
                s_in.wait_event(ev_cp[b])          # step i-2 has consumed this input buffer
            dq[b].copy_(hq, non_blocking=True)
            dk[b].copy_(hk, non_blocking=True)
            dv[b].copy_(hv, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cp):
            s_cp.wait_event(ev_in[b])
            if i >= nb:
                s_cp.wait_event(ev_out[b])         # step i-2's results have left this output buffer
            if fused_q:
                H.quantize_kv(dk[b], dv[b], s_inv, out=dpk[b], stream=s_cp)
                H.attention_fwd_q(dq[b], dpk[b], s, causal=cfg.causal, norm=norm, out=do[b], lse=dl[b],
                                  workspace=dws[b], stream=s_cp)
            else:
                H.quantize_qkv(dq[b], dk[b], dv[b], s, s_inv, out=dpk[b], stream=s_cp)
                H.attention_fwd(dpk[b], causal=cfg.causal, norm=norm, out=do[b], lse=dl[b], workspace=dws[b],
                                stream=s_cp, split_kv=split_kv)
            ev_cp[b].record(s_cp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cp[b])
            ho[b].copy_(do[b], non_blocking=True)
            hl[b].copy_(dl[b], non_blocking=True)
            ev_out[b].record(s_out)

    w_e2e = max(args.warmup, 3)
    for i in range(w_e2e):
        e2e_step(i)
    torch.cuda.synchronize()
    t_beg, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_beg.record(s_in)
    for i in range(w_e2e, w_e2e + n):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cp)
    t_end.record(s_out)
    torch.cuda.synchronize()
    st = max_over_ranks(max(H.get_status(w_) for w_ in dws), dev)
    if st != 0:
        raise RuntimeError(f"kernel status {int(st)} in the end-to-end loop (max over ranks)")
    res["e2e_ms"] = max_over_ranks(t_beg.elapsed_time(t_end), dev)
    res["h2d"] = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    res["d2h"] = ho[0].numel() * ho[0].element_size() + hl[0].numel() * hl[0].element_size()
    return res


def roofline(cfg, H, attn_ms, fp4_peak, hbm_peak):
    """The attention kernel against the bound of its workload: tensor (FLOPs over
    the FP4 peak) or HBM (algorithmic bytes over the copy bandwidth), whichever
    takes longer at peak."""
    flops = cfg.flops()
    nbytes = attn_bytes(cfg, H)
    t_tensor = flops / (fp4_peak * 1e12)
    t_hbm = nbytes / (hbm_peak * 1e9)
    if t_hbm > t_tensor:
        achieved = nbytes / (attn_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "algorithmic_bytes": nbytes}
    achieved = flops / (attn_ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / fp4_peak, 4), "algorithmic_flops": flops}


def mufu_roofline(cfg, attn_ms, dev, clocks):
    """The softmax's own bound: every visible (query, key) pair needs one exp2
    and every 16 keys one more for the block scale; MUFU ex2 runs at 16 per clock
    per SM (measured on this GPU), at the SM clock sampled during the run."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    pairs = cfg.flops() / (4.0 * cfg.D)
    ex2 = pairs * (1.0 + 1.0 / 16.0)
    peak = 16.0 * sms * mhz * 1e6
    achieved = ex2 / (attn_ms * 1e-3)
    return {"bound": "alu", "unit": "ex2/s", "achieved": round(achieved / 1e12, 4), "peak": round(peak / 1e12, 4),
            "scale": "1e12", "frac": round(achieved / peak, 4), "ex2_per_launch": int(ex2),
            "floor_us": round(ex2 / peak * 1e6, 2)}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import bit_quantized_flashattention_b200 as H
    ws, rank, local = dist_env()
    if ws > 1:
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pk = peaks()
    fp4_peak = 4.0 * pk["bf16"]                       # burst: the kernel is timed alone, per launch
    if args.extensions:
        if rank == 0:
            run_extensions(args, dev, H)
        if ws > 1:
            dist.destroy_process_group()
        return
    if args.all_configs:
        run_all_configs(args, dev, rank, ws, H, pk, fp4_peak)
        if ws > 1:
            dist.destroy_process_group()
        return
    cfg = W.get(args.config)
    if args.batch:
        cfg = cfg.replace(B=args.batch)      # smaller case of the same workload (profiling captures)
    norm = args.norm
    r = measure(cfg, norm, args, dev, rank, ws, H)
    n = args.steps
    flops = cfg.flops()
    value = ws * flops * n / (r["total_ms"] * 1e-3) / 1e12
    attn_tflops = flops / (r["attn_ms"] * 1e-3) / 1e12
    launches_per_step = 2          # quantize_qkv_kernel (Q, K and V), attn_fwd_kernel
    roof = roofline(cfg, H, r["attn_ms"], fp4_peak, pk["hbm"])
    roof.update({"traffic": profiled_traffic(cfg), "kernel": "attn_fwd_kernel",
                 "peak_source": (f"4 x {pk['src']} bf16 burst" if roof["bound"] == "tensor"
                                 else f"{pk['src']} HBM copy bandwidth")})
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOPS",
        "n_gpus": ws,
        "steps": n,
        "warmup": args.warmup,
        "ms_per_step": round(r["total_ms"] / n, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1",
        "data": "synthetic (seeded normal Q/K/V, lognormal K channel gains + outlier channels)",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "Nq": cfg.Nq, "Nkv": cfg.Nkv,
                   "D": cfg.D, "causal": cfg.causal, "norm": norm, "smooth_qk": cfg.smooth != "off",
                   "kv_splits": r["n_splits"],
                   "inputs": cfg.dtype, "output": "bf16", "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "l2": "cold and clean between steps (256 MiB write, then 256 MiB read)",
                   "step": ("quantize_kv + attention_fwd_q (Q quantized inside the attention kernel; "
                            "calibration offline)" if r["fused_q"] else "quantize_qkv + attention_fwd (calibration offline)"),
                   "launch": "the step replayed from a CUDA graph (programmatic dependent launch between its two kernels)"},
        "fp4_tensor_pct": round(100.0 * value / ws / fp4_peak, 2),
        "breakdown_ms": {"quantize": round(r["quant_ms"], 5), "attention": round(r["attn_ms"], 5)},
        "attention_only_tflops": round(attn_tflops, 2),
        "roofline": roof,
        "alu_roofline": mufu_roofline(cfg, r["attn_ms"], dev, r["clocks"]),
        "e2e": {"value": round(ws * flops * n / (r["e2e_ms"] * 1e-3) / 1e12, 3), "unit": "TFLOPS",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "ms_per_step": round(r["e2e_ms"] / n, 4),
                "pipeline": "H2D, compute and D2H of consecutive steps overlap (3 streams, 2 buffers)"},
        "gpu_launches": launches_per_step * n,
        "clocks": r["clocks"],
    }
    # the HBM-bound quantize pass: algorithmic bytes (read 2 B/elem, write 0.5625 B/elem)
    elems = (0 if r["fused_q"] else cfg.B * cfg.Hq * cfg.Nq * cfg.D) + 2 * cfg.B * cfg.Hkv * cfg.Nkv * cfg.D
    line["quantize_gbs"] = round(elems * (2 + 0.5625) / (r["quant_ms"] * 1e-3) / 1e9, 1)
    if rank == 0 and not args.no_extras:
        line["sdpa_bf16_tflops"] = sdpa_context(r["q"], r["k"], r["v"], cfg, r["flush"])
        line["error_vs_fp32"] = error_vs_fp32(H, r["packed"], r["q"], r["k"], r["v"], cfg, norm, r["split_kv"])
        line["eps_bar"] = eps_stats(H, r["packed"], cfg, norm, r["split_kv"])
        g = fp4_gemm_peak(dev)
        if g is not None:
            line["fp4_gemm_tflops_measured"] = round(g, 1)
            line["attention_frac_of_measured_fp4_gemm"] = round(attn_tflops / g, 4)
    if rank == 0 and not args.no_cpu:
        v_cpu, desc, secs = oracle_sample(cfg, n_splits=r["n_splits"])
        line["cpu_baseline"] = {"value": round(v_cpu / 1e12, 8), "unit": "TFLOPS", "cores": os.cpu_count(),
                                "kind": "oracle", "sample": desc, "seconds": round(secs, 2)}
        v1, desc1, secs1 = oracle_sample(cfg, seconds_target=4.0, n_threads=1, n_splits=r["n_splits"])
        line["cpu_baseline_1core"] = {"value": round(v1 / 1e12, 9), "unit": "TFLOPS", "cores": 1, "kind": "oracle",
                                      "sample": desc1, "seconds": round(secs1, 2)}
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_all_configs(args, dev, rank, ws, H, pk, fp4_peak):
    """Every workload, in the launch configuration of the main line; one JSON
    line per (workload, normalizer mode)."""
    import torch
    rows = []
    for cfg in W.CONFIGS:
        for norm in cfg.modes:
            r = measure(cfg, norm, args, dev, rank, ws, H, want_e2e=False)
            roof = roofline(cfg, H, r["attn_ms"], fp4_peak, pk["hbm"])
            rec = {"workload": cfg.name, "norm": norm, "kv_splits": r["n_splits"],
                   "step_ms": round(r["total_ms"] / args.steps, 5),
                   "step_tflops": round(cfg.flops() / (r["total_ms"] / args.steps * 1e-3) / 1e12, 2),
                   "attention_ms": round(r["attn_ms"], 5),
                   "attention_tflops": round(cfg.flops() / (r["attn_ms"] * 1e-3) / 1e12, 2),
                   "quantize_ms": round(r["quant_ms"], 5), "roofline": roof,
                   "alu_roofline": mufu_roofline(cfg, r["attn_ms"], dev, r["clocks"]), "clocks": r["clocks"]}
            if rank == 0 and not args.no_extras:
                rec["sdpa_bf16_tflops"] = sdpa_context(r["q"], r["k"], r["v"], cfg, r["flush"])
                rec["error_vs_fp32"] = error_vs_fp32(H, r["packed"], r["q"], r["k"], r["v"], cfg, norm, r["split_kv"])
                rec["eps_bar"] = eps_stats(H, r["packed"], cfg, norm, r["split_kv"])
            if rank == 0:
                print(json.dumps(rec), flush=True)
            rows.append(rec)
            del r
            torch.cuda.empty_cache()
    if rank == 0 and args.table:
        with open(args.table, "w") as f:
            f.write("| workload | norm | kv ranges | step ms | step TFLOP/s | attention ms | attention TFLOP/s | "
                    "bound | roofline frac | quantize ms | bf16 SDPA TFLOP/s | max abs err vs fp32 | "
                    "row rel L2 (median / max) | eps_bar median (tiles < 0) | SM MHz |\n")
            f.write("|" + "---|" * 15 + "\n")
            for x in rows:
                e = x.get("error_vs_fp32", {})
                f.write(f"| {x['workload']} | {x['norm']} | {x['kv_splits']} | {x['step_ms']:.4f} | "
                        f"{x['step_tflops']:.1f} | {x['attention_ms']:.4f} | {x['attention_tflops']:.1f} | "
                        f"{x['roofline']['bound']} | {x['roofline']['frac']:.3f} | {x['quantize_ms']:.4f} | "
                        f"{x.get('sdpa_bf16_tflops', '')} | {e.get('max_abs', '')} | "
                        f"{e.get('row_rel_l2_median', '')} / {e.get('row_rel_l2_max', '')} | "
                        f"{x.get('eps_bar', {}).get('median', '')} ({x.get('eps_bar', {}).get('negative_frac', '')}) | "
                        f"{(x['clocks'] or {}).get('sm_mhz', '')} |\n")


# ----------------------------------------------------------- reference arm

def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    cfg = W.get(args.config)
    for _ in range(args.warmup):
        oracle_sample(cfg, seconds_target=2.0)
    vals, secs = [], []
    desc = ""
    t_all = time.perf_counter()
    for _ in range(args.steps):
        v_cpu, desc, s = oracle_sample(cfg, seconds_target=2.0)
        vals.append(v_cpu)
        secs.append(s)
    total = time.perf_counter() - t_all
    value = statistics.mean(vals) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 8), "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e2m1", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "Nq": cfg.Nq, "Nkv": cfg.Nkv,
                   "D": cfg.D, "causal": cfg.causal, "norm": args.norm, "smooth_qk": cfg.smooth != "off"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 8), "unit": "TFLOPS", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"each step: {desc}"},
        "e2e": {"value": round(value, 8), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload index 1..5 (2 = the headline)")
    ap.add_argument("--norm", choices=["p_reorder", "high_precision_l"], default="p_reorder")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle samples")
    ap.add_argument("--no-extras", action="store_true", help="skip SDPA, fp32-error and FP4-GEMM context")
    ap.add_argument("--all-configs", action="store_true", help="time every workload (one JSON line each)")
    ap.add_argument("--fused-q", action="store_true",
                    help="time the step as quantize_kv + attention_fwd_q (Q quantized in the attention kernel)")
    ap.add_argument("--extensions", action="store_true",
                    help="time Q-Mean, fused RoPE quantize, KV appends and the epsilon statistics")
    ap.add_argument("--table", help="with --all-configs: also write a markdown table here")
    ap.add_argument("--ingest-ncu", help="record DRAM bytes per attention launch from this ncu CSV")
    ap.add_argument("--workload", help="with --ingest-ncu: the workload name the capture ran")
    ap.add_argument("--ncu-command", default="", help="with --ingest-ncu: the command that made the capture")
    ap.add_argument("--ncu-scale", type=float, default=1.0,
                    help="with --ingest-ncu: the capture ran 1/scale of the workload's batch")
    args = ap.parse_args()
    if args.ingest_ncu:
        ingest_ncu(args.ingest_ncu, args.workload or W.get(args.config).name, args.ncu_command, args.ncu_scale)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
