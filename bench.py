"""Benchmark of the 2-bit KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Headline workload (one GPU, replicas only for N > 1): LLM-style decode, batch 8,
32 query / 8 KV heads, d=128, 32,768 cached tokens per sequence, M=64 centroids,
QSAC candidates 4, PSAC rank 8, bf16 output. One step = quantize/append of the
new token of every sequence + decode attention over the packed cache, through
kv2_append_attention_decode (append kernel; split-K attention kernel launched
as its programmatic dependent; split merge). ``value`` = packed-cache bytes
read per step / step time
(GB/s); inputs already resident in HBM; the packed cache (237 MB) is larger
than L2, so successive steps re-read it from HBM.

Extra sections of the same JSON line: ``quantize`` (4,680 new tokens x 40
heads, M=256, C=8, r=8: tokens/s and GB/s), ``fit`` (PSAC basis fit) and
``chunk`` (video-world-model chunk attention, TFLOP/s) when available.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one launch of the split kernel on the LLM
# decode workload (237,390,336 read + 3,970,560 written, ncu capture of the
# current kernel); None whenever the kernel changes.
DECODE_SPLIT_TRAFFIC = 241360896
# fp32 FMA peak of the CUDA cores, derived from the B200's unit counts: 148 SMs
# x 128 FP32 lanes x one FMA per lane and clock (the packed f32x2 form halves
# the instructions, not the lane count), at the SM clock in MHz
FMA_PER_SM_CLOCK = 148 * 128
# packed bytes per (token, KV head): K and V code words, K and V scale/zero
# words (one per group of `group` channels), the centroid id, the PSAC
# coefficients (fp16, or int8 codes with one fp16 scale)
BYTES_PER_TOKEN_HEAD = lambda d, r, M, psac_fmt=0, group=32: (2 * (d // 16) * 4 + 2 * (d // group) * 4
                                                              + (1 if M <= 256 else 2)
                                                              + (2 * r if psac_fmt == 0 else (r + 2 if r else 0)))


def compression(d, r, M, T, psac_fmt=0, group=32):
    """KV-cache compression against bf16 K+V (4 d bytes per token-head): per
    token, and with the per-head tables (fp16 centres M x d, the fp32 basis
    d x r, w and W) counted over T cached tokens, as the method's compression
    figure accounts for centres, quantization parameters and compensation."""
    per = BYTES_PER_TOKEN_HEAD(d, r, M, psac_fmt, group)
    tables = M * d * 2 + d * r * 4 + d * 4 + (d // group) * 4
    return {"bytes_per_token_head": per, "ratio": round(4 * d / per, 3),
            "ratio_with_tables": round(4 * d / (per + tables / T), 3)}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    def __init__(self, index=0):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def setup_decode(torch, kv2, s: wl.Spec):
    """Packed cache of the LLM decode workload built on the GPU by the library:
    fit on the history queries, quantize/append of the 32,768-token prefix."""
    w = wl.make(s.name, with_chunk=False)
    dev = torch.device("cuda")
    Qh = torch.from_numpy(w.Qhist.view(np.int16)).to(dev)
    P, wt, Wg, en = kv2.kv2_fit_psac_basis(Qh, s.H_kv, s.r)
    cache = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, torch.from_numpy(w.centroids.view(np.int16)))
    cache.set_fit(P, wt, Wg)
    K = torch.from_numpy(np.ascontiguousarray(w.K[:, :s.T]).view(np.int16)).to(dev)
    V = torch.from_numpy(np.ascontiguousarray(w.V[:, :s.T]).view(np.int16)).to(dev)
    kv2.kv2_quantize_append(cache, K, V, 0, s.C)
    del K, V
    new_k = torch.from_numpy(np.ascontiguousarray(w.K[:, s.T:s.T + 1]).view(np.int16)).to(dev)
    new_v = torch.from_numpy(np.ascontiguousarray(w.V[:, s.T:s.T + 1]).view(np.int16)).to(dev)
    Q = torch.from_numpy(w.Qdec.view(np.int16)).to(dev)
    torch.cuda.synchronize()
    return w, cache, new_k, new_v, Q, Qh


METRIC = "2-bit KV attention: packed-cache GB/s (% of HBM peak); quantize tokens/s"


def decode_config(world: int) -> dict:
    """The workload both arms report (the LLM decode step, weak scaling over
    independent replicas)."""
    s = wl.spec("llm_decode")
    return {"workload": "llm_decode: B=8, H_q=32, H_kv=8, d=128, T=32768 cached, M=64, C=4, r=8, "
                        "bf16 out; step = append 1 token/seq + decode",
            "global_batch": s.B * world, "seq_len": s.T + 1, "parallelism": f"replicas x{world}",
            "l2": "packed cache 237 MB > 126 MB L2 (no flush)"}


def max_over_ranks(value: float, device: str = "cuda") -> float:
    """The largest of the ranks' values (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_gpu(args, rank, world):
    import torch
    import bit_kv_cache_centroid_b200 as kv2
    torch.cuda.set_device(rank % max(torch.cuda.device_count(), 1))
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod
    s = wl.spec("llm_decode")
    w, cache, new_k, new_v, Q, Qh = setup_decode(torch, kv2, s)
    length = s.T + 1
    scale = 1.0 / math.sqrt(s.d)
    out = torch.empty((s.B, s.H_q, s.d), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(kv2.kv2_decode_workspace_size(cache, s.H_q, length), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        # append of the new token of every sequence + attention over all tokens,
        # the attention kernel overlapping the append (programmatic dependent)
        kv2.kv2_append_attention_decode(cache, new_k, new_v, s.T, s.C, Q, scale, out_dtype=kv2.KV2_OUT_BF16,
                                        out=out, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        time.sleep(0.2)
    total_ms = max_over_ranks(t0.elapsed_time(t1))
    ms_step = total_ms / args.steps

    # the two parts on their own (breakdown; the decode alone feeds the roofline)
    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in ev:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)
    app_ms = timed(lambda: kv2.kv2_quantize_append(cache, new_k, new_v, s.T, s.C))
    dec_ms = timed(lambda: kv2.kv2_attention_decode(cache, length, Q, scale, out_dtype=kv2.KV2_OUT_BF16,
                                                    out=out, ws=ws))
    bytes_step = length * s.B * s.H_kv * BYTES_PER_TOKEN_HEAD(s.d, s.r, s.M)
    value = bytes_step * world / (ms_step * 1e-3) / 1e9

    # ---- end to end through host buffers (pinned), copies inside the timed region:
    # the step's inputs (new K, new V, Q) travel as one pinned buffer, the
    # output comes back as one copy
    nk, nv, nq = new_k.numel(), new_v.numel(), Q.numel()
    hin = torch.empty(nk + nv + nq, dtype=torch.int16).pin_memory()
    hin[:nk].copy_(new_k.view(-1).cpu())
    hin[nk:nk + nv].copy_(new_v.view(-1).cpu())
    hin[nk + nv:].copy_(Q.view(-1).cpu())
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    din = torch.empty_like(hin, device="cuda")
    dk = din[:nk].view(new_k.shape)
    dv = din[nk:nk + nv].view(new_v.shape)
    dq = din[nk + nv:].view(Q.shape)

    def e2e_step():
        din.copy_(hin, non_blocking=True)
        kv2.kv2_append_attention_decode(cache, dk, dv, s.T, s.C, dq, scale, out_dtype=kv2.KV2_OUT_BF16,
                                        out=out, ws=ws)
        hout.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / args.steps
    h2d = hin.numel() * 2
    d2h = hout.numel() * 2

    pk, src = peaks()
    achieved = bytes_step / (dec_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u2+f32", "data": "synthetic",
        "config": decode_config(world),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": DECODE_SPLIT_TRAFFIC,
                     "kernel": "kv2_attention_decode (decode_split + decode_combine)",
                     "peak_source": src, "decode_ms": round(dec_ms, 5)},
        "e2e": {"value": round(bytes_step / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5)},
        "compression": compression(s.d, s.r, s.M, s.T + 1),
        "step_ms": {"append_alone": round(app_ms, 5), "decode_alone": round(dec_ms, 5),
                    "step_overlapped": round(ms_step, 5)},
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }
    if not args.skip_extras and rank == 0:
        result["int8_psac_decode"] = variant_decode(torch, kv2, args, pk, w, s, Q, scale, out, psac_fmt=1)
        result["group128_decode"] = variant_decode(torch, kv2, args, pk, w, s, Q, scale, out, group=128)
        result["group128_int8_psac_decode"] = variant_decode(torch, kv2, args, pk, w, s, Q, scale, out,
                                                             psac_fmt=1, group=128)
        result.update(extras(torch, kv2, args, pk))
    if rank == 0 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(args, budget_s=args.cpu_seconds)
        if "quantize" in result:
            result["quantize"]["cpu_baseline"] = cpu_quantize()
        if "chunk" in result:
            result["chunk"]["cpu_baseline"] = cpu_chunk()
    return result


def variant_decode(torch, kv2, args, pk, w, s, Q, scale, out, psac_fmt=0, group=32):
    """The LLM decode workload in another cache format: PSAC coefficients as
    int8 codes with one fp16 scale per token (psac_fmt 1) and/or one scale and
    zero per `group` channels (decode alone, same timing as above). A format
    the library refuses is reported as skipped, with the library's reason."""
    dev = torch.device("cuda")
    try:
        P, wt, Wg, en = kv2.kv2_fit_psac_basis(torch.from_numpy(w.Qhist.view(np.int16)).to(dev), s.H_kv, s.r,
                                               group=group)
    except kv2.Kv2Error as e:
        return {"skipped": str(e)}
    cache = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, s.capacity, torch.from_numpy(w.centroids.view(np.int16)),
                      psac_fmt=psac_fmt, group=group)
    cache.set_fit(P, wt, Wg)
    K = torch.from_numpy(np.ascontiguousarray(w.K[:, :s.T + 1]).view(np.int16)).to(dev)
    V = torch.from_numpy(np.ascontiguousarray(w.V[:, :s.T + 1]).view(np.int16)).to(dev)
    kv2.kv2_quantize_append(cache, K, V, 0, s.C)
    del K, V
    length = s.T + 1
    ws = torch.zeros(kv2.kv2_decode_workspace_size(cache, s.H_q, length), dtype=torch.uint8, device=dev)
    f = lambda: kv2.kv2_attention_decode(cache, length, Q, scale, out_dtype=kv2.KV2_OUT_BF16, out=out, ws=ws)
    for _ in range(3):
        f()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        f()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    per = BYTES_PER_TOKEN_HEAD(s.d, s.r, s.M, psac_fmt, group)
    gbs = length * s.B * s.H_kv * per / (ms * 1e-3) / 1e9
    fmt = "int8 PSAC coefficients + fp16 scale per token" if psac_fmt == 1 else "fp16 PSAC coefficients"
    return {"workload": f"llm_decode with {fmt}, scale/zero per {group} channels",
            "bytes_per_token_head": per, "compression": compression(s.d, s.r, s.M, length, psac_fmt, group),
            "ms": round(ms, 5), "GBps": round(gbs, 1), "hbm_frac": round(gbs / pk["hbm_gbs"], 4)}


def retrieval_shift(torch, kv2, w, s, wt, Wg, P):
    """How often Key quantization moves a query's most-attended token: the
    quantize workload's keys (cached frame + new tokens, video statistics)
    quantized with QSAC (C candidates, fitted weights, PSAC rank r) and with
    the nearest centre (C = 1, unit weights, no PSAC), against the exact keys,
    for 128 history queries per head."""
    dev = torch.device("cuda")
    n = w.K.shape[1]
    Kd = torch.from_numpy(np.ascontiguousarray(w.K).view(np.int16)).to(dev)
    Vd = torch.from_numpy(np.ascontiguousarray(w.V).view(np.int16)).to(dev)
    Qr = torch.from_numpy(np.ascontiguousarray(w.Qhist[None, :128]).view(np.int16)).to(dev)
    dense = kv2.kv2_dense_top1(Kd, Qr)
    cap = (n + 15) // 16 * 16
    res = {"tokens": n, "queries": int(Qr.shape[1] * Qr.shape[2])}
    for name, C, r in (("qsac_psac", s.C, s.r), ("nearest_centre", 1, 0)):
        cache = kv2.Cache(1, s.H_kv, s.d, s.M, r, cap, torch.from_numpy(w.centroids.view(np.int16)))
        if r:
            cache.set_fit(P, wt, Wg)
        kv2.kv2_quantize_append(cache, Kd, Vd, 0, C)
        top = kv2.kv2_decode_top1(cache, n, Qr)
        res[name] = round(float((top != dense).float().mean().item()), 4)
    torch.cuda.synchronize()
    return res


def quantize_section(torch, kv2, args, pk):
    """Quantize/append throughput: 4,680 new tokens x 40 heads appended at
    37,440 (M=256, C=8, r=8), after the PSAC basis fit; 3 untimed calls, then
    the timed ones. Returns the section and what the later sections reuse."""
    s = wl.spec("quant_append")
    w = wl.make("quant_append", T=wl.FRAME_TOKENS, with_chunk=False)
    dev = torch.device("cuda")
    Qh = torch.from_numpy(w.Qhist.view(np.int16)).to(dev)
    cap = (s.capacity + 15) // 16 * 16
    cache = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, cap, torch.from_numpy(w.centroids.view(np.int16)))
    P, wt, Wg, en = kv2.kv2_fit_psac_basis(Qh, s.H_kv, s.r)
    cache.set_fit(P, wt, Wg)
    K = torch.from_numpy(np.ascontiguousarray(w.K_new).view(np.int16)).to(dev)
    V = torch.from_numpy(np.ascontiguousarray(w.V_new).view(np.int16)).to(dev)
    for _ in range(3):
        kv2.kv2_quantize_append(cache, K, V, s.T, s.C)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(5, args.steps // 2)
    a.record()
    for _ in range(n):
        kv2.kv2_quantize_append(cache, K, V, s.T, s.C)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    toks = s.n_new * s.B
    rd = K.numel() * 2 * 2
    wr = toks * s.H_kv * BYTES_PER_TOKEN_HEAD(s.d, s.r, s.M)
    fma = toks * s.H_kv * s.M * s.d
    sec = {"workload": "quant_append: 4680 new tokens x 40 heads, d=128, M=256, C=8, r=8",
           "ms": round(ms, 4), "tokens_per_s": round(toks / (ms * 1e-3), 1),
           "token_heads_per_s": round(toks * s.H_kv / (ms * 1e-3), 1),
           "GBps": round((rd + wr) / (ms * 1e-3) / 1e9, 2),
           "hbm_frac": round((rd + wr) / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
           "ranking_TFMAps": round(fma / (ms * 1e-3) / 1e12, 3),
           "alu_peak_TFMAps": round(FMA_PER_SM_CLOCK * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12, 2),
           "alu_frac": round(fma / (ms * 1e-3) / (FMA_PER_SM_CLOCK * pk.get("sm_max_mhz", 1965.0) * 1e6), 4),
           "alu_peak_source": "derived: 148 SMs x 128 fp32 lanes x 1 FMA/clock x max SM clock",
           "bound": "latency",
           "note": "alu_frac is the ranking rate against the fp32 FMA peak; the ranking products run on the "
                   "tensor cores (mma.sync) and the kernel is latency-bound at 16 warps per SM"}
    return sec, (s, w, K, Qh, P, wt, Wg, a, b)


def extras(torch, kv2, args, pk):
    """Quantize/append throughput and fit time (same JSON line)."""
    out = {}
    dev = torch.device("cuda")
    out["quantize"], (s, w, K, Qh, P, wt, Wg, a, b) = quantize_section(torch, kv2, args, pk)
    out["retrieval_shift"] = retrieval_shift(torch, kv2, w, s, wt, Wg, P)
    # QSAC-aware centre fitting on the chunk's new keys (5 iterations)
    X = K[0]
    cent0 = torch.from_numpy(w.centroids.view(np.int16)).to(dev)
    cent = cent0.clone()
    kv2.kv2_fit_centroids(X, cent, s.C, wt, Wg, 1)
    torch.cuda.synchronize()
    iters = 5
    cent.copy_(cent0)
    a.record()
    kv2.kv2_fit_centroids(X, cent, s.C, wt, Wg, iters)
    b.record()
    torch.cuda.synchronize()
    it_ms = a.elapsed_time(b) / iters
    nk = X.shape[0] * X.shape[1]
    out["fit_centroids"] = {"workload": f"{X.shape[0]} keys x {X.shape[1]} heads, d={s.d}, M={s.M}, C={s.C}, "
                                        f"{iters} iterations", "ms_per_iteration": round(it_ms, 4),
                            "ranking_TFMAps": round(nk * s.M * s.d / (it_ms * 1e-3) / 1e12, 3)}
    out["chunk"] = chunk_section(torch, kv2, args, pk)
    out["long_horizon"] = long_horizon_section(torch, kv2, args, pk)
    a.record()
    for _ in range(3):
        kv2.kv2_fit_psac_basis(Qh, s.H_kv, s.r)
    b.record()
    torch.cuda.synchronize()
    out["fit"] = {"workload": "40 heads x 512 history queries, d=128, r=8", "ms": round(a.elapsed_time(b) / 3, 3)}
    return out


def chunk_flops(s: wl.Spec, length: int) -> float:
    """Algorithmic FLOPs of one chunk call: 4 d per (query, visible key) for
    Q K^T and P V, plus 2 r per (query, cached key) for the PSAC term (qP).a
    (the kernel pads the r columns to a multiple of 16; the padding is not
    counted)."""
    F = s.frame_tokens
    f = np.arange(s.Nq) // F
    self_seen = np.minimum((f + 1) * F, s.Nq).astype(np.float64)
    per_head = (4.0 * s.d * (length + self_seen) + 2.0 * s.r * length).sum()
    return float(per_head * s.H_q * s.B)


def chunk_section(torch, kv2, args, pk):
    """Video world-model chunk attention: 40 heads, 37,440 cached tokens, 4,680
    queries (3 latent frames), block-causal by frame, M=256, r=8 (packed cache
    drawn directly in the packed format)."""
    s = wl.spec("video_chunk")
    pc = wl.random_packed_cache(s, T=s.T)
    cache = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, pc.capacity, torch.from_numpy(pc.centroids.view(np.int16)))
    cache.load_packed(pc)
    rng = np.random.default_rng(3)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    cache.P.copy_(torch.from_numpy(P))
    dev = lambda x: torch.from_numpy(wl.bf16_bits(x).view(np.int16)).cuda()
    Q = dev(rng.standard_normal((1, s.Nq, s.H_q, s.d)).astype(np.float32))
    Ks = dev(rng.standard_normal((1, s.Nq, s.H_kv, s.d)).astype(np.float32))
    Vs = dev(rng.standard_normal((1, s.Nq, s.H_kv, s.d)).astype(np.float32))
    out = torch.empty((1, s.Nq, s.H_q, s.d), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(kv2.kv2_chunk_workspace_size(cache, s.H_q, s.Nq), dtype=torch.uint8, device="cuda")
    scale = 1.0 / math.sqrt(s.d)
    run = lambda: kv2.kv2_attention_chunk(cache, s.T, Q, Ks, Vs, s.frame_tokens, scale,
                                          out_dtype=kv2.KV2_OUT_BF16, out=out, ws=ws)
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 3
    a.record()
    for _ in range(n):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    fl = chunk_flops(s, s.T)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "video_chunk: 40 heads, d=128, 37,440 cached + 4,680 queries (3 frames), "
                        "block-causal, M=256, r=8, bf16 out",
            "ms": round(ms, 3), "tflop": round(fl / 1e12, 4), "TFLOPs": round(tf, 1),
            "tensor_frac": round(tf / pk["bf16_tflops"], 4), "peak_tflops": pk["bf16_tflops"],
            "timeout_flag": int(ws[:4].view(torch.int32).item())}


def long_horizon_section(torch, kv2, args, pk):
    """Long-horizon world memory: 187,200 cached tokens (120 latent frames,
    frames 30/60/90 revisiting frame 0), 40 heads (MHA), d=128, M=512 (u16
    ids), r=16: decode with one query per head, and a 4,680-query chunk."""
    s = wl.spec("long_horizon")
    pc = wl.random_packed_cache(s, T=s.T, revisit_every=30)
    cache = kv2.Cache(s.B, s.H_kv, s.d, s.M, s.r, pc.capacity, torch.from_numpy(pc.centroids.view(np.int16)))
    cache.load_packed(pc)
    del pc
    rng = np.random.default_rng(5)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    cache.P.copy_(torch.from_numpy(P))
    dev = lambda x: torch.from_numpy(wl.bf16_bits(x).view(np.int16)).cuda()
    scale = 1.0 / math.sqrt(s.d)

    def timed(fn, n):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    Qd = dev(rng.standard_normal((s.B, s.H_q, s.d)).astype(np.float32))
    outd = torch.empty((s.B, s.H_q, s.d), dtype=torch.bfloat16, device="cuda")
    wsd = torch.zeros(kv2.kv2_decode_workspace_size(cache, s.H_q, s.T), dtype=torch.uint8, device="cuda")
    dms = timed(lambda: kv2.kv2_attention_decode(cache, s.T, Qd, scale, out_dtype=kv2.KV2_OUT_BF16,
                                                 out=outd, ws=wsd), 20)
    dbytes = s.T * s.B * s.H_kv * BYTES_PER_TOKEN_HEAD(s.d, s.r, s.M)
    dgbs = dbytes / (dms * 1e-3) / 1e9
    Q = dev(rng.standard_normal((1, s.Nq, s.H_q, s.d)).astype(np.float32))
    Ks = dev(rng.standard_normal((1, s.Nq, s.H_kv, s.d)).astype(np.float32))
    Vs = dev(rng.standard_normal((1, s.Nq, s.H_kv, s.d)).astype(np.float32))
    outc = torch.empty((1, s.Nq, s.H_q, s.d), dtype=torch.bfloat16, device="cuda")
    wsc = torch.zeros(kv2.kv2_chunk_workspace_size(cache, s.H_q, s.Nq), dtype=torch.uint8, device="cuda")
    cms = timed(lambda: kv2.kv2_attention_chunk(cache, s.T, Q, Ks, Vs, s.frame_tokens, scale,
                                                out_dtype=kv2.KV2_OUT_BF16, out=outc, ws=wsc), 3)
    fl = chunk_flops(s, s.T)
    tf = fl / (cms * 1e-3) / 1e12
    return {"workload": "long_horizon: 187,200 cached tokens, 40 heads (MHA), d=128, M=512, r=16, bf16 out",
            "decode": {"ms": round(dms, 4), "bytes": dbytes, "GBps": round(dgbs, 1),
                       "hbm_frac": round(dgbs / pk["hbm_gbs"], 4)},
            "chunk": {"queries": s.Nq, "ms": round(cms, 3), "tflop": round(fl / 1e12, 4), "TFLOPs": round(tf, 1),
                      "tensor_frac": round(tf / pk["bf16_tflops"], 4),
                      "timeout_flag": int(wsc[:4].view(torch.int32).item())}}


# ----------------------------------------------------------------------------
# CPU: the oracle as it stands
# ----------------------------------------------------------------------------

def host_info() -> dict:
    """The host the oracle runs on: logical CPUs and the CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def _llm_oracle_inputs():
    s = wl.spec("llm_decode")
    pc = wl.random_packed_cache(s.with_(B=1), T=s.T + 1)
    rng = np.random.default_rng(5)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    Q = wl.bf16_bits(rng.standard_normal((1, s.H_q, s.d)).astype(np.float32))
    return s, pc, P, Q


def cpu_baseline(args, budget_s=15.0):
    """Oracle decode (fp64, single thread) on whole sequences of the LLM decode
    workload until ~budget_s of CPU time; GB/s of packed cache attended."""
    import oracle
    oracle.build()
    s, pc, P, Q = _llm_oracle_inputs()
    seqs, t = 0, 0.0
    while t < budget_s and seqs < 64:
        t0 = time.perf_counter()
        oracle.decode(pc, P, s.T + 1, Q, 1.0 / math.sqrt(s.d))
        t += time.perf_counter() - t0
        seqs += 1
    bytes_ = seqs * (s.T + 1) * s.H_kv * BYTES_PER_TOKEN_HEAD(s.d, s.r, s.M)
    return {"value": round(bytes_ / t / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{seqs} sequence(s) x 8 KV heads x 32 query heads x 32,769 tokens (oracle decode, fp64)",
            "seconds": round(t, 2), "host": host_info()}


def cpu_quantize(budget_s=8.0):
    """Oracle quantize/append (single thread, fp32 decisions) on the first new
    tokens of the quant_append workload, all 40 heads, until ~budget_s."""
    import oracle
    oracle.build()
    s = wl.spec("quant_append")
    w = wl.make("quant_append", T=wl.FRAME_TOKENS, with_chunk=False)
    f = oracle.fit(w.Qhist, s.H_kv, s.r)
    pc = wl.PackedCache.empty(s.B, s.H_kv, s.d, s.M, s.r, (s.capacity + 15) // 16 * 16, w.centroids)
    done, t, step = 0, 0.0, 16
    while t < budget_s and done + step <= s.n_new:
        K = np.ascontiguousarray(w.K_new[:, done:done + step])
        V = np.ascontiguousarray(w.V_new[:, done:done + step])
        t0 = time.perf_counter()
        oracle.quantize(pc, K, V, s.T + done, s.C, f.P, f.w, f.Wg)
        t += time.perf_counter() - t0
        done += step
    return {"value": round(done / t, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} of the {s.n_new} new tokens x 40 heads (M=256, C=8, r=8)",
            "seconds": round(t, 2), "host": host_info()}


def cpu_chunk(budget_s=10.0):
    """Oracle chunk attention (fp64 attention, fp16 operand emulation, single
    thread) on query rows of one head of the video chunk workload, each over
    the 37,440 cached tokens plus its visible self part, until ~budget_s; the
    TFLOP/s of the sample and the full call's time extrapolated from it."""
    import oracle
    oracle.build()
    s = wl.spec("video_chunk")
    pc = wl.random_packed_cache(s, T=s.T)
    rng = np.random.default_rng(3)
    P = np.zeros((s.H_kv, s.d, s.r), np.float32)
    for h in range(s.H_kv):
        q, _ = np.linalg.qr(rng.standard_normal((s.d, s.d)))
        P[h] = q[:, :s.r]
    Q = wl.bf16_bits(rng.standard_normal((1, s.Nq, s.H_q, s.d)).astype(np.float32))
    Ks = wl.bf16_bits(rng.standard_normal((1, s.Nq, s.H_kv, s.d)).astype(np.float32))
    Vs = wl.bf16_bits(rng.standard_normal((1, s.Nq, s.H_kv, s.d)).astype(np.float32))
    F = s.frame_tokens
    order = rng.permutation(s.Nq)
    n, t, flop = 0, 0.0, 0.0
    while t < budget_s and n < s.Nq:
        i = int(order[n])
        t0 = time.perf_counter()
        oracle.chunk(pc, P, s.T, Q, Ks, Vs, F, 1.0 / math.sqrt(s.d), np.array([[0, i, 0]], np.int32))
        t += time.perf_counter() - t0
        seen = min((i // F + 1) * F, s.Nq)
        flop += 4.0 * s.d * (s.T + seen) + 2.0 * s.r * s.T
        n += 1
    full = chunk_flops(s, s.T)
    return {"value": round(flop / t / 1e12, 8), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} random query rows of head 0 (of {s.Nq} x {s.H_q}), each over the 37,440 cached "
                      f"tokens + its visible self tokens",
            "seconds": round(t, 2), "extrapolated_full_call_s": round(full / (flop / t), 1),
            "host": host_info()}


def run_reference(args, world: int = 1):
    """The oracle arm: W untimed and K timed steps, each step the oracle's
    decode of one of the 8 sequences of the LLM decode workload (all 8 KV heads
    x 32 query heads x 32,769 tokens, fp64, one host thread); value = packed
    bytes attended per second over the timed steps."""
    import oracle
    oracle.build()
    s, pc, P, Q = _llm_oracle_inputs()
    run = lambda: oracle.decode(pc, P, s.T + 1, Q, 1.0 / math.sqrt(s.d))
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    t = time.perf_counter() - t0
    ms = t * 1e3 / args.steps
    bytes_step = (s.T + 1) * s.H_kv * BYTES_PER_TOKEN_HEAD(s.d, s.r, s.M)
    value = round(bytes_step * args.steps / t / 1e9, 4)
    sample = ("each step: 1 of the 8 sequences of the LLM decode workload (8 KV heads x 32 query heads x "
              "32,769 tokens, oracle decode, fp64)")
    r = {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
         "seconds": round(t, 2), "extrapolated_full_step_ms": round(ms * s.B, 1), "host": host_info()}
    return {"impl": "reference",
            "metric": METRIC,
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": decode_config(world),
            "cpu_baseline": r,
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libkv2")
    ap.add_argument("--skip-extras", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--only", choices=["decode", "quantize", "chunk"], default=None,
                    help="run one section only (for profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # the CPU oracle on the host: rank 0 alone works and prints
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.only == "quantize":
        import torch
        import bit_kv_cache_centroid_b200 as kv2
        print(json.dumps(quantize_section(torch, kv2, args, peaks()[0])[0]), flush=True)
        return
    if args.only == "chunk":
        import torch
        import bit_kv_cache_centroid_b200 as kv2
        print(json.dumps(chunk_section(torch, kv2, args, peaks()[0])), flush=True)
        return
    if args.only == "decode":
        args.skip_extras, args.no_cpu = True, True
    res = run_gpu(args, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
