#!/usr/bin/env python3
"""Benchmark: TurboQuant-prod compressed-KV decode on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload batched|llama8b|qwen15b_16384|longctx]

A step is one pass of the whole hot path over one batch: quantize-append of
one new token per sequence (all KV heads) followed by one decode-attention
step (query rotation, split-K one-pass attention over the compressed cache,
combine).  The default workload is the batched decode case (batch 32,
H_kv=8, H_q=32, d=128, ragged lengths uniform in [16384, 32768], 3-bit keys,
2-bit values): the cache read per step (~630 MB) is larger than the 126 MB
L2, so no flush is needed between steps.

Multi-GPU (``torchrun --nproc-per-node N``): every rank holds its own batch
(weak scaling, no data-path collective); the time is the max over ranks.

``--impl reference`` times the float64 CPU oracle (test infrastructure) on
the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from kv_cache_quantization_turboquantprod_b200 import tq, workloads  # noqa: E402

METRIC = "decode attn ctx-tokens/s & HBM GB/s vs ~8 TB/s; quantize Mvec/s (1 B200)"
UNIT = "ctx-tokens/s"
DECODE_SRC = os.path.join(ROOT, "kv_cache_quantization_turboquantprod_b200", "csrc")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _bf16_peak():
    """Dense bf16 tensor peak in TFLOP/s (burst): measured, else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def _source_hash(files):
    h = hashlib.sha256()
    for f in sorted(files):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _decode_kernel_files():
    return [os.path.join(DECODE_SRC, f) for f in sorted(os.listdir(DECODE_SRC))
            if f.startswith("decode") or f in ("tq_common.cuh", "tq_kernels.h")]


def _traffic_from_profile(kernel_hash):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, if it was taken on this exact source; else None."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("source_hash") == kernel_hash:
            return d
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.4)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

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
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def _fill_cache(wl, layer, cache, device):
    """Quantize-append every sequence's synthetic K/V (8192-token chunks)."""
    nchunks = (wl.capacity + workloads.TOKEN_CHUNK - 1) // workloads.TOKEN_CHUNK
    lens = [0] * wl.batch
    for c in range(nchunks):
        t0 = c * workloads.TOKEN_CHUNK
        nnew = [max(0, min(wl.lengths[b] - t0, workloads.TOKEN_CHUNK)) for b in range(wl.batch)]
        if max(nnew) == 0:
            break
        T = max(nnew)
        ks, vs = [], []
        for b in range(wl.batch):
            k, v = workloads.kv_chunk(wl, b, c, device)
            ks.append(k[:T])
            vs.append(v[:T])
        k = torch.stack(ks).contiguous()
        v = torch.stack(vs).contiguous()
        tq.tq_quantize_append(layer, cache, k, v, lens, nnew)
        lens = [lens[b] + nnew[b] for b in range(wl.batch)]
        del k, v, ks, vs
    torch.cuda.synchronize()
    return lens


def aggregate_across_ranks(times, counts, world, device):
    """Max over ranks of the times, sum over ranks of the work counts (weak
    scaling: every rank processes its own batch).  Identity for one rank."""
    t = torch.tensor(times, dtype=torch.float64, device=device)
    c = torch.tensor(counts, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        torch.distributed.all_reduce(c, op=torch.distributed.ReduceOp.SUM)
    return t.tolist(), c.tolist()


def run_ours(args, rank, world, device):
    wl = workloads.by_name(args.workload)
    if args.batch:
        wl = workloads.scaled(wl, batch=args.batch, capacity=wl.capacity,
                              name=f"{wl.name}_b{args.batch}")
    _, pi32, s32 = workloads.layer_matrices(wl)
    layer = tq.Layer(pi32, s32, wl.key_bits, wl.value_bits, device=device)
    cache = tq.CompressedCache(layer, wl.batch, wl.h_kv, wl.capacity, device=device)
    lengths = list(wl.lengths)
    # leave one free slot per sequence for the per-step append
    lengths = [min(n, wl.capacity - 1) for n in lengths]
    wl_fill = workloads.scaled(wl, lengths=tuple(lengths), capacity=wl.capacity)
    _fill_cache(wl_fill, layer, cache, device)

    B, HQ, D, HKV = wl.batch, wl.h_q, wl.d, wl.h_kv
    gen = torch.Generator(device=device)
    gen.manual_seed(1234 + rank)
    dt = torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32
    q = torch.randn((B, HQ, D), generator=gen, device=device).to(dt)
    k_new = torch.randn((B, 1, HKV, D), generator=gen, device=device).to(dt)
    v_new = torch.randn((B, 1, HKV, D), generator=gen, device=device).to(dt)
    len_after = torch.tensor([n + 1 for n in lengths], dtype=torch.int32, device=device)
    max_len = max(lengths) + 1
    ws = tq.workspace_for(layer, cache, HQ, max_len, device=device)
    out = torch.empty((B, HQ, D), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    launches_per_step = 1 + 3

    def step():
        tq.tq_quantize_append(layer, cache, k_new, v_new, lengths)
        tq.tq_decode_attention(layer, cache, q, len_after, max_len, out, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", device.index or 0)))
    if rank == 0:
        sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if args.profile_steps:
        torch.cuda.profiler.start()  # ncu --profile-from-start off captures the timed steps only
    t_start.record(stream)
    for i in range(args.steps):
        step()
    t_end.record(stream)
    if args.profile_steps:
        torch.cuda.profiler.stop()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    # The decode call alone (for the roofline): timed over a loop of decode
    # calls right after the steps, with CUDA events on the launching stream.
    # Events inside the step loop would sit between the append and the
    # decode's first kernel and keep the two from overlapping.
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    d0.record(stream)
    for _ in range(args.steps):
        tq.tq_decode_attention(layer, cache, q, len_after, max_len, out, ws)
    d1.record(stream)
    torch.cuda.synchronize()
    dec_ms = d0.elapsed_time(d1) / args.steps

    # end to end through the public API with host buffers (pinned): every step
    # copies its inputs host -> device and reads its output back inside the
    # timed region, pipelined as a server would: two device buffer sets, the
    # H2D copy of step i+1 and the D2H copy of step i on their own streams,
    # overlapping the compute of step i (events order each buffer's reuse)
    q_h = q.cpu().pin_memory()
    k_h = k_new.cpu().pin_memory()
    v_h = v_new.cpu().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    q_d = [torch.empty_like(q) for _ in range(2)]
    k_d = [torch.empty_like(k_new) for _ in range(2)]
    v_d = [torch.empty_like(v_new) for _ in range(2)]
    out_d = [torch.empty_like(out) for _ in range(2)]
    h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n_steps, start_event=None):
        if start_event is not None:
            h2d_stream.wait_event(start_event)
            d2h_stream.wait_event(start_event)
        for i in range(n_steps):
            j = i % 2
            with torch.cuda.stream(h2d_stream):
                if i >= 2:
                    h2d_stream.wait_event(done[j])  # compute of step i-2 is off buffer set j
                q_d[j].copy_(q_h, non_blocking=True)
                k_d[j].copy_(k_h, non_blocking=True)
                v_d[j].copy_(v_h, non_blocking=True)
                ready[j].record(h2d_stream)
            stream.wait_event(ready[j])
            if i >= 2:
                stream.wait_event(drained[j])  # out_d[j] of step i-2 was read back
            tq.tq_quantize_append(layer, cache, k_d[j], v_d[j], lengths)
            tq.tq_decode_attention(layer, cache, q_d[j], len_after, max_len, out_d[j], ws)
            done[j].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(done[j])
                out_h[j].copy_(out_d[j], non_blocking=True)
                drained[j].record(d2h_stream)
        # the last read-back ends the run on the compute stream
        stream.wait_event(drained[(n_steps - 1) % 2])
        if n_steps > 1:
            stream.wait_event(drained[(n_steps - 2) % 2])

    e2e_run(args.warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    e2e_run(args.steps, start_event=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    ctx_tokens_step = float(sum(n + 1 for n in lengths))
    rec_bytes = layer.record_bytes()
    dec_bytes = ctx_tokens_step * HKV * rec_bytes

    (elapsed_ms, e2e_ms, dec_ms), (ctx_all, dec_bytes_all) = aggregate_across_ranks(
        [elapsed_ms, e2e_ms, dec_ms], [ctx_tokens_step, dec_bytes], world, device)
    if rank != 0:
        return None

    value = ctx_all * args.steps / (elapsed_ms / 1e3)
    e2e_value = ctx_all * args.steps / (e2e_ms / 1e3)
    peak, peak_kind = _peaks()
    achieved = (dec_bytes_all / world) / (dec_ms / 1e3) / 1e9
    khash = _source_hash(_decode_kernel_files())
    prof = _traffic_from_profile(khash)
    traffic = None
    if prof is not None:
        traffic = prof.get("dram_bytes_per_launch_scaled")
    clocks = sampler.summary()
    cpu = cpu_baseline(wl, pi32, s32, args) if (rank == 0 and world == 1 and not args.no_cpu) else None
    h2d = q.numel() * q.element_size() + k_new.numel() * k_new.element_size() * 2
    d2h = out.numel() * out.element_size()
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; bf16 K/V/q with lognormal channel scales and outlier channels; no model weights)",
        "config": {
            "workload": wl.name,
            "batch_per_gpu": B, "h_kv": HKV, "h_q": HQ, "d": D,
            "key_bits": wl.key_bits, "value_bits": wl.value_bits, "group": wl.group,
            "capacity": wl.capacity, "ctx_tokens_per_step_per_gpu": ctx_tokens_step,
            "lengths": "ragged uniform [16384, 32768]" if wl.name == "batched" else list(wl.lengths),
            "step": "quantize-append 1 token/sequence + decode (query blocks, split-K, combine)",
            "l2": "no flush: each step streams the whole compressed cache (> 126 MB L2)",
            "parallelism": f"dp{world} (independent batches per GPU)",
        },
        "decode_gbs": dec_bytes_all / world / (dec_ms / 1e3) / 1e9,
        "decode_ms": dec_ms,
        "record_bytes": rec_bytes,
        "roofline": {
            "kernel": "tq_decode_attention (query blocks + split-K + combine, timed as one call)",
            "bound": "hbm",
            "achieved": achieved,
            "peak": peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": traffic,
            "algorithmic_bytes_per_launch": dec_bytes_all / world,
        },
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if world == 1:
        line["window"] = bench_window(layer, cache, q, len_after, max_len, out, ws, wl, device,
                                      dec_bytes_all, dec_ms)
        line["prefill"] = bench_prefill(layer, cache, len_after, max_len, wl, device, dec_bytes_all)
    if args.quantize and world == 1:
        line["quantize"] = bench_quantize(args, device)
    if args.configs and world == 1:
        line["configs"] = bench_configs(device, peak)
    return line


def bench_window(layer, cache, q, len_dev, max_len, out, ws, wl, device, dec_bytes, dec_ms):
    """The same decode call with a full 128-token exact window (bf16 K and V)
    per sequence merged into the softmax: time and the window's cost."""
    B, HKV, D = wl.batch, wl.h_kv, wl.d
    gen = torch.Generator(device=device)
    gen.manual_seed(4321)
    wk = torch.randn((B, HKV, 128, D), generator=gen, device=device).to(torch.bfloat16)
    wv = torch.randn((B, HKV, 128, D), generator=gen, device=device).to(torch.bfloat16)
    wlen = torch.full((B,), 128, dtype=torch.int32, device=device)
    for _ in range(3):
        tq.tq_decode_attention_window(layer, cache, q, len_dev, max_len, wk, wv, wlen, out, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 20
    e0.record()
    for _ in range(n):
        tq.tq_decode_attention_window(layer, cache, q, len_dev, max_len, wk, wv, wlen, out, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    win_bytes = B * HKV * 128 * D * 2 * 2
    return {"win_cap": 128, "decode_ms": ms, "decode_ms_without_window": dec_ms,
            "gbs": (dec_bytes + win_bytes) / (ms / 1e3) / 1e9,
            "window_bytes": win_bytes}


def bench_prefill(layer, cache, len_dev, max_len, wl, device, dec_bytes, t_chunk=8):
    """Causal prefill of an 8-token chunk per sequence over the same cache (the
    chunk taken as the cache's last 8 tokens): each pass of the library's
    tokens-per-pass streams the records once.  Reports query tokens/s and the
    record bytes streamed per second."""
    B, HQ, D = wl.batch, wl.h_q, wl.d
    gen = torch.Generator(device=device)
    gen.manual_seed(777)
    qp = torch.randn((B, t_chunk, HQ, D), generator=gen, device=device).to(torch.bfloat16)
    out = torch.empty((B, t_chunk, HQ, D), dtype=torch.float32, device=device)
    ws = tq.prefill_workspace_for(layer, cache, HQ, t_chunk, max_len, device=device)
    for _ in range(3):
        tq.tq_prefill_attention(layer, cache, qp, len_dev, max_len, out, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 10
    e0.record()
    for _ in range(n):
        tq.tq_prefill_attention(layer, cache, qp, len_dev, max_len, out, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    per_pass = tq.tq_prefill_tokens_per_pass(layer, HQ, wl.h_kv, t_chunk)
    passes = 0
    left = t_chunk
    while left > 0:  # passes of per_pass tokens, the last of the largest power of two left
        n = per_pass
        while n > left:
            n //= 2
        left -= n
        passes += 1
    return {"t_chunk": t_chunk, "tokens_per_pass": per_pass, "passes": passes, "ms": ms,
            "query_tokens_s": B * t_chunk / (ms / 1e3),
            "record_gbs": passes * dec_bytes / (ms / 1e3) / 1e9}


def _time_ms(fn, n=20, warmup=3):
    """Median CUDA-event time of fn() over n runs after warm-up (ms)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return float(np.median(times))


def _decode_line(wl, layer, cache, lengths, device, peak):
    """Decode-call latency of a workload (median of 20) and its record bandwidth."""
    q = workloads.queries(wl, 0, device=device)
    len_dev = torch.tensor(lengths, dtype=torch.int32, device=device)
    ml = max(lengths)
    ws = tq.workspace_for(layer, cache, wl.h_q, ml, device=device)
    out = torch.empty((wl.batch, wl.h_q, wl.d), dtype=torch.float32, device=device)
    ms = _time_ms(lambda: tq.tq_decode_attention(layer, cache, q, len_dev, ml, out, ws))
    rec = layer.record_bytes()
    nbytes = float(sum(lengths)) * wl.h_kv * rec
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"decode_us": ms * 1e3, "ctx_tokens_s": sum(lengths) / (ms / 1e3),
            "record_bytes_per_call": nbytes, "gbs": gbs, "frac_of_8tbs": gbs / 8000.0,
            "frac_of_peak": gbs / peak}


def bench_configs(device, peak):
    """Every configuration of the measurement table at N = 1: tiny and
    Llama-shaped decode (latency-bound, records L2-resident), the
    Qwen-shaped context sweep 512 .. 16K, and the long-context decode at
    131,072 tokens (the cache filled by 16 quantize-append chunks)."""
    res = {}
    for name in ("tiny", "llama8b"):
        wl = workloads.by_name(name)
        _, pi32, s32 = workloads.layer_matrices(wl)
        layer = tq.Layer(pi32, s32, wl.key_bits, wl.value_bits, device=device)
        cache = tq.CompressedCache(layer, wl.batch, wl.h_kv, wl.capacity, device=device)
        k, v = workloads.kv_tokens(wl, 0, 0, wl.lengths[0], device=device)
        k, v = k[None].contiguous(), v[None].contiguous()
        q_ms = _time_ms(lambda: tq.tq_quantize_append(layer, cache, k, v, [0]))
        line = _decode_line(wl, layer, cache, list(wl.lengths), device, peak)
        line["quantize_us"] = q_ms * 1e3
        line["quantize_mvec_s"] = wl.lengths[0] * wl.h_kv / (q_ms / 1e3) / 1e6
        res[name] = line
    sweep = {}
    for n in workloads.QWEN_SWEEP:
        wl = workloads.qwen15b(n)
        _, pi32, s32 = workloads.layer_matrices(wl)
        layer = tq.Layer(pi32, s32, wl.key_bits, wl.value_bits, device=device)
        cache = tq.CompressedCache(layer, wl.batch, wl.h_kv, wl.capacity, device=device)
        _fill_cache(wl, layer, cache, device)
        sweep[str(n)] = _decode_line(wl, layer, cache, list(wl.lengths), device, peak)
    res["qwen15b"] = sweep
    wl = workloads.longctx()
    _, pi32, s32 = workloads.layer_matrices(wl)
    layer = tq.Layer(pi32, s32, wl.key_bits, wl.value_bits, device=device)
    cache = tq.CompressedCache(layer, wl.batch, wl.h_kv, wl.capacity, device=device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    _fill_cache(wl, layer, cache, device)
    e1.record()
    torch.cuda.synchronize()
    line = _decode_line(wl, layer, cache, list(wl.lengths), device, peak)
    line["fill_ms_16_chunks_with_input_generation"] = e0.elapsed_time(e1)
    res["longctx"] = line
    del cache
    torch.cuda.empty_cache()
    return res


def bench_quantize(args, device):
    """Quantize-append Mvec/s on one 8192-token chunk of the long-context
    workload (batch 4, H_kv=8, 3+1-bit keys, 2-bit values)."""
    wl = workloads.longctx()
    _, pi32, s32 = workloads.layer_matrices(wl)
    layer = tq.Layer(pi32, s32, wl.key_bits, wl.value_bits, device=device)
    cap = 2 * workloads.TOKEN_CHUNK
    cache = tq.CompressedCache(layer, wl.batch, wl.h_kv, cap, device=device)
    ks, vs = [], []
    for b in range(wl.batch):
        k, v = workloads.kv_chunk(wl, b, 0, device)
        ks.append(k)
        vs.append(v)
    k = torch.stack(ks).contiguous()
    v = torch.stack(vs).contiguous()
    lens = [workloads.TOKEN_CHUNK] * wl.batch
    for _ in range(3):
        tq.tq_quantize_append(layer, cache, k, v, lens)
    torch.cuda.synchronize()
    n = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        tq.tq_quantize_append(layer, cache, k, v, lens)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    vecs = wl.batch * workloads.TOKEN_CHUNK * wl.h_kv
    in_bytes = k.numel() * k.element_size() * 2
    out_bytes = vecs * layer.record_bytes()
    peak, peak_kind = _bf16_peak()
    # two d x d products a key vector: y = Pi u and the sketch S r = W (y - c)
    useful = vecs * 2 * 2 * 128 * 128 / (ms / 1e3) / 1e12
    # issued: 48 MMAs of 128 x 128 x 16 a 128-vector tile (GEMM1 three bf16
    # parts of Pi, GEMM2 three hi/lo products), 16-bit operands
    issued = vecs * (48 * 2 * 128 * 128 * 16 / 128) / (ms / 1e3) / 1e12
    return {"workload": "longctx chunk (4 x 8192 tokens x 8 heads, bf16)",
            "ms_per_chunk": ms, "mvec_s": vecs / (ms / 1e3) / 1e6,
            "gbs": (in_bytes + out_bytes) / (ms / 1e3) / 1e9,
            "useful_tflops": useful, "mma_tflops": issued,
            "tensor": {"peak_tflops": peak, "peak_kind": peak_kind, "useful_frac": useful / peak,
                       "mma_frac": issued / peak}}


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------

def _oracle_sample(wl, pi32, s32, pairs, max_tokens):
    """Prepare oracle-encoded records for sampled (b, h) pairs (not timed)."""
    from oracle import attention, codebook, quant  # test infrastructure
    pi = pi32.astype(np.float64)
    s = s32.astype(np.float64)
    cent, bnd, _ = codebook.lloyd_max_gaussian(wl.key_bits - 1, wl.d)
    samples = []
    for (b, h) in pairs:
        n = min(wl.lengths[b], max_tokens)
        k, v = workloads.kv_tokens(wl, b, 0, n, device="cpu")
        ke = quant.encode_keys(k[:, h].float().numpy(), pi, s, cent, bnd)
        ve = quant.encode_values(v[:, h].float().numpy(), wl.value_bits, wl.group)
        rec = {"idx": ke["idx"][:, None], "sign": ke["sign"][:, None],
               "nk16": ke["nk16"][:, None], "rn16": ke["rn16"][:, None],
               "codes": ve["codes"][:, None], "scale16": ve["scale16"][:, None],
               "zero16": ve["zero16"][:, None]}
        q = workloads.queries(wl, 0, device="cpu")[b, h * wl.gqa:(h + 1) * wl.gqa].float().numpy()
        samples.append((q, rec, n))
    return samples, (pi, s, cent, attention)


def _oracle_decode_samples(samples, consts, group):
    pi, s, cent, attention = consts
    for q, rec, _ in samples:
        attention.decode_one_sequence(q, rec, pi, s, cent, group)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return None


def cpu_baseline(wl, pi32, s32, args, budget_s=10.0):
    """Time the oracle's decode on host cores over a bounded sample of the
    workload: (b, h) pairs, each with all G query heads of that KV head."""
    rng = np.random.default_rng(0)
    pairs = [(int(rng.integers(wl.batch)), int(rng.integers(wl.h_kv))) for _ in range(64)]
    max_tokens = 8192
    samples, consts = _oracle_sample(wl, pi32, s32, pairs[:2], max_tokens)
    t0 = time.perf_counter()
    done_tokens = 0.0
    i = 0
    while True:
        _oracle_decode_samples(samples, consts, wl.group)
        done_tokens += sum(n for _, _, n in samples)
        i += 1
        if time.perf_counter() - t0 > budget_s or i >= 50:
            break
    dt = time.perf_counter() - t0
    # a ctx-token covers all H_kv heads: a (b, h) pair's n tokens are n / H_kv ctx-tokens
    value = done_tokens / wl.h_kv / dt
    # the same sample on one thread (BLAS limited to one thread in-process)
    one = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t1 = time.perf_counter()
            j, tok1 = 0, 0.0
            while True:
                _oracle_decode_samples(samples, consts, wl.group)
                tok1 += sum(n for _, _, n in samples)
                j += 1
                if time.perf_counter() - t1 > budget_s / 2 or j >= 20:
                    break
            one = {"value": tok1 / wl.h_kv / (time.perf_counter() - t1), "cores": 1,
                   "repeats": j}
    except Exception as e:  # threadpoolctl missing: report why
        one = {"unavailable": str(e)}
    return {"value": value, "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
            "blas_threads": _blas_threads(), "kind": "oracle",
            "sample": f"oracle decode of 2 (sequence, KV head) pairs x {max_tokens} tokens "
                      f"x {wl.gqa} query heads, repeated {i}x ({dt:.1f} s); "
                      f"ctx-tokens counted as tokens / H_kv",
            "single_thread": one}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = workloads.by_name(args.workload)
    _, pi32, s32 = workloads.layer_matrices(wl)
    rng = np.random.default_rng(1)
    pairs = [(int(rng.integers(wl.batch)), int(rng.integers(wl.h_kv))) for _ in range(4)]
    max_tokens = 4096
    samples, consts = _oracle_sample(wl, pi32, s32, pairs[:1], max_tokens)
    for _ in range(args.warmup):
        _oracle_decode_samples(samples, consts, wl.group)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_decode_samples(samples, consts, wl.group)
    dt = time.perf_counter() - t0
    tokens = sum(n for _, _, n in samples) * args.steps / wl.h_kv
    value = tokens / dt
    sample = (f"each step: oracle decode of 1 (sequence, KV head) pair x {max_tokens} tokens x "
              f"{wl.gqa} query heads of the {wl.name} workload; ctx-tokens = tokens / H_kv")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                             "cores": len(os.sched_getaffinity(0)), "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="batched")
    ap.add_argument("--batch", type=int, default=None,
                    help="use the first N sequences of the workload (profiling)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-quantize", dest="quantize", action="store_false",
                    help="skip the quantize-append Mvec/s measurement")
    ap.add_argument("--profile-steps", action="store_true",
                    help="bracket the timed steps with cudaProfilerStart/Stop (for ncu --profile-from-start off)")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the per-configuration latency table")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    tq.load()
    try:
        line = run_ours(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
