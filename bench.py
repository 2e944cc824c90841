#!/usr/bin/env python3
"""Benchmark of the RoPE + grouped-query KV-cache decode path on B200.

Headline workload: the Llama-3-8B-shaped single-layer decode (B=16, n_head=32,
n_kv_head=8, d=128, ragged cache lengths uniform in [1024, 8192], RoPE base
500000).  One step = attn_decode_gqa_rope: the batch's new queries rotated
at position len_b inside the decode kernel (cached keys were rotated when
written), then attention over the cache.  The same work as two launches
(rope_apply_qk, then attn_decode_gqa) is reported beside it.
Metric: effective HBM GB/s = algorithmic bytes (K/V rows read once, q read,
out and lse written) / step time; also tokens/s (= B / step time).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvattn|reference]
With --gpus N > 1 (launched by torch.distributed.run) every rank decodes its
own batch (weak scaling, no collective on the data path); value = bytes of
all ranks / max-over-ranks time.  --impl reference times the fp64 CPU oracle
on the host cores on a bounded sample of the same workload.
"""
import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mqa_kv_cache_b200 import workloads as W  # noqa: E402

METRIC = "decode-attn effective HBM GB/s (% of peak) & tok/s; prefill TFLOP/s"
L2_FLUSH_BYTES = 256 << 20
# The committed ncu summary of the headline decode kernel records its DRAM traffic per
# launch (dram__bytes_read.sum + dram__bytes_write.sum) together with a hash of the kernel
# sources it was captured from; the traffic is reported only while the sources still match.
DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_kernel_llama3_8b_ragged_B16_H32_Hk8.md")
DECODE_SOURCES = ["decode.cu", "decode_plan.cuh", "common.cuh", "kernels.h"]


def kernel_sources_sha256(names):
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "mqa_kv_cache_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profile_traffic(path, sources):
    """(bytes per launch, note): the traffic a committed ncu summary records, or None
    when the summary is missing or the kernel sources changed since its capture."""
    import re
    try:
        text = open(path).read()
    except OSError:
        return None, "no committed ncu summary"
    t = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    h = re.search(r"sources_sha256:\s*([0-9a-f]{64})", text)
    if not t or not h:
        return None, "the ncu summary records no traffic"
    if h.group(1) != kernel_sources_sha256(sources):
        return None, "kernel sources changed since the committed ncu capture"
    return int(t.group(1)), "ncu capture of the current kernel sources (" + os.path.basename(path) + ")"


def measure_read_stream(device, nbytes=4 << 30, reps=5):
    """Best read-only streaming rate (GB/s) of a plain reduction over nbytes: the
    read-side counterpart of the copy figure (which moves read + write bytes)."""
    x = torch.ones(nbytes // 4, dtype=torch.float32, device=device)
    best = float("inf")
    for _ in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        torch.sum(x)
        b.record()
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b))
    del x
    torch.cuda.empty_cache()
    return nbytes / (best * 1e-3) / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def decode_bytes(w, lens):
    """Algorithmic bytes of one decode over the batch: every valid K and V row
    once, the queries, the outputs and the lse values."""
    kv = int(lens.sum()) * w.Hk * w.d * 2 * 2
    return kv + w.B * w.H * w.d * 2 * 2 + w.B * w.H * 4


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period=0.005):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------- GPU arm

def packed(specs, device):
    """One uint8 buffer holding tensors of the given (shape, dtype) at 256-byte
    aligned offsets, and views of them: a step's inputs (or outputs) then cross
    the PCIe link as one copy."""
    offs, total = [], 0
    for shape, dt in specs:
        offs.append(total)
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dt).element_size()
        total += (nbytes + 255) // 256 * 256
    buf = torch.zeros(total, dtype=torch.uint8, device=device)
    views = []
    for (shape, dt), o in zip(specs, offs):
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dt).element_size()
        views.append(buf[o:o + nbytes].view(dt).view(shape))
    return buf, views


class DecodeStep:
    """Device-resident decode workload; step() = rope on q + decode.  The step's
    inputs (q, positions, lengths) and outputs (out, lse) each live in one buffer."""

    def __init__(self, K, w, device, seed):
        self.K, self.w = K, w
        inp = W.decode_inputs(w, device=device, seed=seed, lens=W.lengths(w.B, w.T_lo, w.T_hi, seed))
        r = w.rope
        p = K.rope_params(w.d, base=r.base, scaling=r.scaling, s=r.s, L_train=r.L_train, alpha=r.alpha,
                          beta=r.beta)
        self.cos, self.sin = K.rope_table_build(p, w.T_max + 1, device=device)
        self.k, self.v = inp["k"], inp["v"]
        # cached keys are rotated once, when they are written to the cache
        K.rope_apply_qk(None, None, self.k, inp["k_pos"].to(device), self.cos, self.sin, k_layout="bhtd")
        self.inbuf, (self.q, self.q_pos, self.lens) = packed(
            [(tuple(inp["q"].shape), torch.bfloat16), (tuple(inp["q_pos"].shape), torch.int32),
             (tuple(inp["seq_lens"].shape), torch.int32)], device)
        self.q.copy_(inp["q"])
        self.q_pos.copy_(inp["q_pos"])
        self.lens.copy_(inp["seq_lens"])
        self.lens_host = inp["seq_lens"].clone()
        self.outbuf, (self.out, self.lse) = packed(
            [(tuple(inp["q"].shape), torch.bfloat16), ((w.B, w.H), torch.float32)], device)
        self.ws = K.workspace(K.attn_decode_gqa_workspace_bytes(w.B, w.H, w.Hk, w.d, w.T_max), device)
        self.bytes = decode_bytes(w, inp["seq_lens"])
        # the decode kernel (RoPE of q inside); the tcgen05 path (d = 128 with 64 query heads
        # per KV head) adds its merge kernel, the mma.sync path merges inside the decode kernel
        self.launches_per_step = 2 if (w.d == 128 and w.g == 64) else 1
        self.q_work = self.q.clone()  # the unfused variant rotates a copy in place
        # queries rotated once, for the attention kernel alone (attn_decode_gqa)
        self.q_rot = self.q.clone()
        K.rope_apply_qk(self.q_rot, self.q_pos, None, None, self.cos, self.sin, q_layout="bhd")

    def step(self):
        """The fused step: queries rotated inside the decode kernel (q is not modified)."""
        self.K.attn_decode_gqa_rope(self.q, self.q_pos, self.cos, self.sin, self.k, self.v, self.lens,
                                    self.w.scale, out=self.out, lse=self.lse, ws=self.ws)

    def attn(self):
        """Attention alone on pre-rotated queries (attn_decode_gqa)."""
        self.K.attn_decode_gqa(self.q_rot, self.k, self.v, self.lens, self.w.scale, out=self.out, lse=self.lse,
                               ws=self.ws)

    def reset_work(self):
        self.q_work.copy_(self.q)

    def unfused(self):
        """The same work as two launches: rope_apply_qk on a copy, then attn_decode_gqa."""
        self.K.rope_apply_qk(self.q_work, self.q_pos, None, None, self.cos, self.sin, q_layout="bhd")
        self.K.attn_decode_gqa(self.q_work, self.k, self.v, self.lens, self.w.scale, out=self.out, lse=self.lse,
                               ws=self.ws)


def capture(fn):
    """Capture fn() (launches on the current stream) as a CUDA graph."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def flush_l2(buf):
    """Evict L2 by reading a buffer twice its size (clean lines: no write-back
    of flush data can land inside the next timed step)."""
    torch.sum(buf, dtype=torch.int32)


def time_steps(fn, steps, flush, before=None):
    """Per-step CUDA-event times (ms) on the current stream, L2 flushed between steps."""
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        if before is not None:
            before()
        flush_l2(flush)
        a.record(st)
        fn()
        b.record(st)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def run_gpu(args, rank, world, device):
    from mqa_kv_cache_b200 import kvattn as K
    peaks = load_peaks()
    w = W.LLAMA3_8B_DECODE
    job = DecodeStep(K, w, device, rank_seed(w, rank))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    for _ in range(args.warmup):
        job.step()
        job.reset_work()
        job.unfused()
    torch.cuda.synchronize()
    # the fused step and the unfused pair, captured once as CUDA graphs
    step_graph = capture(job.step)
    unfused_graph = capture(job.unfused)
    for _ in range(args.warmup):
        step_graph.replay()
        job.reset_work()
        unfused_graph.replay()
    torch.cuda.synchronize()

    # ---- timed region: K whole steps (graph replays, L2 flushed in between) ----
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device() if device.index is None else device.index)
    with sampler:
        step_ms = time_steps(step_graph.replay, args.steps, flush)
    barrier(world)
    torch.cuda.synchronize()
    total_bytes, ms = whole_job(job.bytes, float(np.mean(step_ms)), world, device)

    # ---- the step is one kernel: it is also the roofline's kernel.  For context: the same
    # work as two launches, and the fused step launched eagerly from Python ----
    attn_ms = ms
    unfused_ms = max_over_ranks(float(np.mean(time_steps(unfused_graph.replay, args.steps, flush,
                                                          before=job.reset_work))), world, device)
    eager_ms = max_over_ranks(float(np.mean(time_steps(job.step, args.steps, flush))), world, device)

    # ---- end to end through the public API with host buffers: the step's packed
    # inputs (raw q, positions, lengths) in, rope + decode, packed (out, lse) back ----
    in_host = job.inbuf.cpu().pin_memory()
    out_host = torch.empty(job.outbuf.shape, dtype=torch.uint8).pin_memory()

    def e2e():
        job.inbuf.copy_(in_host, non_blocking=True)
        job.step()
        out_host.copy_(job.outbuf, non_blocking=True)

    for _ in range(args.warmup):
        e2e()
    e2e_ms = max_over_ranks(float(np.mean(time_steps(e2e, args.steps, flush))), world, device)
    h2d = in_host.numel()
    d2h = out_host.numel()

    gbs = total_bytes / (ms * 1e-3) / 1e9
    attn_gbs = job.bytes / (attn_ms * 1e-3) / 1e9
    traffic, traffic_note = profile_traffic(DECODE_PROFILE, DECODE_SOURCES)
    read_gbs = measure_read_stream(device)
    line = {
        "metric": METRIC,
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, ragged lengths U[1024,8192])",
        "config": {"workload": w.name, "B": w.B, "global_batch": w.B * world, "n_head": w.H, "n_kv_head": w.Hk,
                   "head_dim": w.d, "T_max": w.T_max, "mean_len": float(job.lens_host.float().mean()),
                   "rope_base": w.rope.base,
                   "parallelism": f"dp{world} (independent batches)",
                   "l2": "flushed between timed steps (read of a 256 MB buffer), and inputs exceed L2"},
        "tok_per_s": round(w.B * world / (ms * 1e-3), 1),
        "step_launch": "CUDA graph replay (eager Python launch: %.4f ms/step)" % eager_ms,
        "unfused_ms_per_step": round(unfused_ms, 5),
        "pct_of_hbm_peak": round(100.0 * gbs / world / peaks["hbm_gbs"], 2),
        "pct_of_nominal_8tbs": round(100.0 * gbs / world / 8000.0, 2),
        "roofline": {"kernel": "decode_kernel (attn_decode_gqa_rope: RoPE of q, split-K decode, merge)",
                     "bound": "hbm",
                     "achieved": round(attn_gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(attn_gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "traffic_source": traffic_note,
                     "peak_source": peaks["source"], "algorithmic_bytes": job.bytes,
                     "read_stream_gbs": round(read_gbs, 1), "frac_of_read_stream": round(attn_gbs / read_gbs, 4),
                     "frac_of_nominal_8tbs": round(attn_gbs / 8000.0, 4)},
        "e2e": {"value": round(total_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": job.launches_per_step * args.steps,
        "clocks": sampler.summary(),
    }
    return line


# ---------------------------------------------------------------------------- other configurations

def _graph_ms(fn, steps, flush, warmup=3, before=None):
    for _ in range(warmup):
        if before is not None:
            before()
        fn()
    torch.cuda.synchronize()
    g = capture(fn)
    # the mean: CUDA-event times come in steps of about 2 us on this part, and the
    # mean over steps that start at unrelated phases of that tick resolves below it
    return float(np.mean(time_steps(g.replay, steps, flush, before=before)))


def measure_decode_config(K, w, device, steps, flush, peaks):
    job = DecodeStep(K, w, device, W.SEED_BASE + w.index)
    ms = _graph_ms(job.step, steps, flush)
    unfused_ms = _graph_ms(job.unfused, steps, flush, before=job.reset_work)
    attn_ms = _graph_ms(job.attn, steps, flush)
    out = {"workload": w.name, "ms_per_step": round(ms, 5), "unfused_ms_per_step": round(unfused_ms, 5),
           "attn_ms": round(attn_ms, 5), "algorithmic_bytes": job.bytes,
           "GB_s": round(job.bytes / (ms * 1e-3) / 1e9, 1),
           "pct_of_hbm_peak": round(100 * job.bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 1),
           "pct_of_nominal_8tbs": round(100 * job.bytes / (ms * 1e-3) / 1e9 / 8000.0, 1),
           "attn_pct_of_hbm_peak": round(100 * job.bytes / (attn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 1),
           "attn_pct_of_nominal_8tbs": round(100 * job.bytes / (attn_ms * 1e-3) / 1e9 / 8000.0, 1),
           "tok_per_s": round(w.B / (ms * 1e-3), 1)}
    del job
    torch.cuda.empty_cache()
    return out


def measure_prefill(K, device, steps, flush, peaks):
    w = W.PREFILL_8K
    gen = W.generator(W.SEED_BASE + w.index, device)
    q_raw = W.normal_bf16((w.B, w.T, w.H, w.d), gen, device)
    k_raw = W.normal_bf16((w.B, w.Hk, w.T, w.d), gen, device)
    v = W.normal_bf16((w.B, w.Hk, w.T, w.d), gen, device)
    q, k = q_raw.clone(), k_raw.clone()
    pos = torch.arange(w.T, dtype=torch.int32, device=device).repeat(w.B, 1)
    cos, sin = K.rope_table_build(K.rope_params(w.d, base=w.rope.base), w.T, device=device)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=device)

    def reset():
        q.copy_(q_raw)
        k.copy_(k_raw)

    def rope():
        K.rope_apply_qk(q, pos, k, pos, cos, sin, q_layout="bthd", k_layout="bhtd")

    def attn():
        K.attn_prefill_causal(q, k, v, w.scale, out=out, lse=lse)

    def step():
        rope()
        attn()

    flops = 4.0 * w.B * w.H * w.d * w.T * (w.T + 1) / 2
    attn_ms = _graph_ms(attn, max(10, steps // 10), flush)
    step_ms = _graph_ms(step, max(10, steps // 10), flush, before=reset)
    rope_ms = _graph_ms(rope, max(10, steps // 10), flush, before=reset)
    rope_bytes = 2 * 2 * (q.numel() + k.numel())
    tf = flops / (attn_ms * 1e-3) / 1e12
    return {"workload": w.name, "attn_ms": round(attn_ms, 4), "step_ms": round(step_ms, 4),
            "causal_flops": flops, "attn_TFLOP_s": round(tf, 1),
            "pct_of_bf16_peak_burst": round(100 * tf / peaks["bf16_tflops"], 1),
            "pct_of_bf16_peak_sustained": round(100 * tf / peaks["bf16_tflops_sustained"], 1),
            "rope_apply_ms": round(rope_ms, 4), "rope_apply_GB_s": round(rope_bytes / (rope_ms * 1e-3) / 1e9, 1),
            "tok_per_s": round(w.B * w.T / (step_ms * 1e-3), 1)}


def measure_prefill_window(K, device, steps, flush, peaks):
    """The prefill shape with a 2048-token window and 4 sink tokens
    (attn_prefill_causal_window); FLOPs counted over the rows' actual key sets."""
    w = W.PREFILL_8K
    n_sink, window = 4, 2048
    gen = W.generator(W.SEED_BASE + w.index + 9, device)
    q = W.normal_bf16((w.B, w.T, w.H, w.d), gen, device)
    k = W.normal_bf16((w.B, w.Hk, w.T, w.d), gen, device)
    v = W.normal_bf16((w.B, w.Hk, w.T, w.d), gen, device)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=device)

    def attn():
        K.attn_prefill_causal_window(q, k, v, w.scale, n_sink, window, out=out, lse=lse)

    ms = _graph_ms(attn, max(10, steps // 10), flush)
    i = np.arange(w.T) + 1  # keys a row's query could see (causal), then the window and the sinks
    seen = np.where(i > n_sink, np.minimum(i, n_sink) + i - np.maximum(n_sink, i - window), i)
    flops = 4.0 * w.B * w.H * w.d * float(seen.sum())
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": f"causal_prefill_B2_T8192_H32_Hk8_d128_sink{n_sink}_window{window}", "attn_ms": round(ms, 4),
            "flops": flops, "attn_TFLOP_s": round(tf, 1),
            "pct_of_bf16_peak_burst": round(100 * tf / peaks["bf16_tflops"], 1),
            "tok_per_s": round(w.B * w.T / (ms * 1e-3), 1)}


def measure_dsa(K, device, steps, flush, peaks):
    w = W.DSA_128K
    gen = W.generator(W.SEED_BASE + w.index, device)
    q_idx = W.normal_bf16((w.B, w.HI, w.dI), gen, device)
    wt = W.uniform_f32((w.B, w.HI), gen, device)
    k_idx = W.normal_bf16((w.B, w.L, w.dI), gen, device)
    q = W.normal_bf16((w.B, w.Hq, w.Dk), gen, device)
    latent = W.normal_bf16((w.B, w.L, w.Dk), gen, device)
    idx = torch.empty((w.B, w.k), dtype=torch.int32, device=device)
    scores = torch.empty((w.B, w.L), dtype=torch.float32, device=device)
    out = torch.empty((w.B, w.Hq, w.Dv), dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
    ws1 = K.workspace(K.dsa_index_topk_workspace_bytes(w.B, w.L, w.k), device)
    ws2 = K.workspace(K.attn_decode_sparse_workspace_bytes(w.B, w.Hq, w.Dv, w.k), device)

    def index():
        K.dsa_index_topk(q_idx, wt, k_idx, w.k, topk_idx=idx, scores_out=scores, ws=ws1)

    def sparse():
        K.attn_decode_sparse(q, latent, idx, w.Dv, w.sparse_scale, out=out, lse=lse, ws=ws2)

    def step():
        index()
        sparse()

    n = max(10, steps // 5)
    index_ms = _graph_ms(index, n, flush)
    sparse_ms = _graph_ms(sparse, n, flush)
    step_ms = _graph_ms(step, n, flush)
    idx_bytes = w.B * w.L * w.dI * 2
    sp_bytes = w.B * w.k * w.Dk * 2
    sp_flops = 2.0 * w.B * w.Hq * w.k * (w.Dk + w.Dv)

    # the same step on the FP8 cache: keys of 128 codes + one scale (132 B per token), latent
    # rows of 656 B (512 codes, 4 scales, the bf16 RoPE part); quantised once, untimed
    codes, kscales = K.idx_key_quant_fp8(k_idx)
    packed = K.latent_quant_fp8(latent)
    del k_idx, latent
    torch.cuda.empty_cache()

    def index8():
        K.dsa_index_topk_fp8(q_idx, wt, codes, kscales, w.k, topk_idx=idx, scores_out=scores, ws=ws1)

    def sparse8():
        K.attn_decode_sparse_fp8(q, packed, idx, w.Dv, w.sparse_scale, out=out, lse=lse, ws=ws2)

    def step8():
        index8()
        sparse8()

    index8_ms = _graph_ms(index8, n, flush)
    sparse8_ms = _graph_ms(sparse8, n, flush)
    step8_ms = _graph_ms(step8, n, flush)
    idx8_bytes = w.B * w.L * (w.dI + 4)
    sp8_bytes = w.B * w.k * 656

    def bound_ms(nbytes, flops):
        return max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12)) * 1e3

    return {"workload": w.name, "step_ms": round(step_ms, 4), "tok_per_s": round(w.B / (step_ms * 1e-3), 1),
            "index_topk_ms": round(index_ms, 4),
            "indexer_GB_s_incl_topk": round(idx_bytes / (index_ms * 1e-3) / 1e9, 1),
            "sparse_ms": round(sparse_ms, 4), "sparse_TFLOP_s": round(sp_flops / (sparse_ms * 1e-3) / 1e12, 1),
            "sparse_gathered_bytes": sp_bytes,
            "sparse_roofline_ms": round(bound_ms(sp_bytes, sp_flops), 5),
            "sparse_frac_of_roofline": round(bound_ms(sp_bytes, sp_flops) / sparse_ms, 3),
            "fp8": {"step_ms": round(step8_ms, 4), "tok_per_s": round(w.B / (step8_ms * 1e-3), 1),
                    "index_topk_ms": round(index8_ms, 4), "indexer_key_bytes": idx8_bytes,
                    "indexer_GB_s_incl_topk": round(idx8_bytes / (index8_ms * 1e-3) / 1e9, 1),
                    "sparse_ms": round(sparse8_ms, 4), "sparse_gathered_bytes": sp8_bytes,
                    "sparse_TFLOP_s": round(sp_flops / (sparse8_ms * 1e-3) / 1e12, 1),
                    "sparse_roofline_ms": round(bound_ms(sp8_bytes, sp_flops), 5),
                    "sparse_frac_of_roofline": round(bound_ms(sp8_bytes, sp_flops) / sparse8_ms, 3)}}


def measure_qsa(K, device, steps, flush, peaks, B=None):
    """Block-level indexer decode step (B 8, ragged lengths up to 131072 tokens): the
    key of the newest 4-token group (qsa_block_keys, one group per row), group scoring
    + top-512 + expansion with the trailing partial group (qsa_select), then GQA
    decode (H 32, Hk 8, d 128) over the <= 2051 selected tokens (attn_decode_gqa_sparse)."""
    w = W.QSA_128K if B is None else dataclasses.replace(W.QSA_128K, B=B)
    inp = W.qsa_inputs(w, device=device)
    lens = inp["seq_lens"].to(device)
    cos, sin = K.rope_table_build(K.rope_params(w.dI, base=w.rope.base), w.L, device=device)
    kb = K.qsa_block_keys(inp["k_idx"], lens, cos, sin)  # the stored keys of every complete group
    newest = (lens // 4 - 1).clamp(min=0).to(torch.int32)
    n_idx = 4 * w.n_top + 3
    tok = torch.empty((w.B, n_idx), dtype=torch.int32, device=device)
    cnt = torch.empty(w.B, dtype=torch.int32, device=device)
    out = torch.empty_like(inp["q"])
    lse = torch.empty((w.B, w.H), dtype=torch.float32, device=device)
    ws1 = K.workspace(K.qsa_select_workspace_bytes(w.B, w.L, w.n_top), device)
    ws2 = K.workspace(K.attn_decode_gqa_sparse_workspace_bytes(w.B, w.H, w.Hk, w.d, n_idx), device)

    def keys_new():
        K.qsa_block_keys(inp["k_idx"], lens, cos, sin, block_keys=kb, block_from=newest, max_new=1)

    def keys_all():
        K.qsa_block_keys(inp["k_idx"], lens, cos, sin, block_keys=kb)

    def select():
        K.qsa_select(inp["q_idx"], inp["w"], kb, lens, n_top=w.n_top, tok_idx=tok, tok_count=cnt, ws=ws1)

    def sparse():
        K.attn_decode_gqa_sparse(inp["q"], inp["k"], inp["v"], tok, w.scale, tok_count=cnt, out=out, lse=lse, ws=ws2)

    def step():
        keys_new()
        select()
        sparse()

    n = max(10, steps // 5)
    step_ms = _graph_ms(step, n, flush)
    select_ms = _graph_ms(select, n, flush)
    sparse_ms = _graph_ms(sparse, n, flush)
    keys_ms = _graph_ms(keys_all, n, flush)
    L = [int(x) for x in inp["seq_lens"]]
    nb = [x // 4 for x in L]
    counts = [4 * min(g, w.n_top) + x % 4 for g, x in zip(nb, L)]
    key_bytes = sum(nb) * w.dI * 2                                    # stored group keys read once
    kv_bytes = sum(counts) * w.Hk * w.d * 2 * 2                        # gathered K and V rows
    qo_bytes = w.B * w.H * w.d * 2 * 2 + w.B * w.H * 4
    step_bytes = key_bytes + kv_bytes + qo_bytes + w.B * (w.HI * w.dI * 2 + w.HI * 4)
    build_bytes = sum(L) * w.dI * 2 + key_bytes
    hbm = peaks["hbm_gbs"]
    return {"workload": w.name if B is None else w.name.replace("_B8_", f"_B{B}_"), "step_ms": round(step_ms, 4),
            "tok_per_s": round(w.B / (step_ms * 1e-3), 1), "step_algorithmic_bytes": step_bytes,
            "step_GB_s": round(step_bytes / (step_ms * 1e-3) / 1e9, 1),
            "step_pct_of_hbm_peak": round(100 * step_bytes / (step_ms * 1e-3) / 1e9 / hbm, 1),
            "select_ms": round(select_ms, 4), "group_key_bytes": key_bytes,
            "sparse_ms": round(sparse_ms, 4), "sparse_gathered_bytes": kv_bytes,
            "sparse_GB_s": round((kv_bytes + qo_bytes) / (sparse_ms * 1e-3) / 1e9, 1),
            "sparse_pct_of_hbm_peak": round(100 * (kv_bytes + qo_bytes) / (sparse_ms * 1e-3) / 1e9 / hbm, 1),
            "block_keys_full_build_ms": round(keys_ms, 4),
            "block_keys_full_build_GB_s": round(build_bytes / (keys_ms * 1e-3) / 1e9, 1)}


def measure_window(K, device, steps, flush, peaks):
    """Llama-3-8B-shaped decode at 32768 tokens over a rolling cache of 4 sinks +
    a 4092-token window (attn_decode_gqa_rope_window): 4096 rows per KV head read."""
    w = W.LLAMA3_8B_DECODE
    n_sink, window, length = 4, 4092, 32768
    cap = n_sink + window
    gen = W.generator(W.SEED_BASE + w.index + 7, device)
    q = W.normal_bf16((w.B, w.H, w.d), gen, device)
    kc = W.normal_bf16((w.B, w.Hk, cap, w.d), gen, device)
    vc = W.normal_bf16((w.B, w.Hk, cap, w.d), gen, device)
    lens = torch.full((w.B,), length, dtype=torch.int32, device=device)
    cos, sin = K.rope_table_build(K.rope_params(w.d, base=w.rope.base), length + 1, device=device)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H), dtype=torch.float32, device=device)
    ws = K.workspace(K.attn_decode_gqa_workspace_bytes(w.B, w.H, w.Hk, w.d, cap), device)

    def step():
        K.attn_decode_gqa_rope_window(q, lens, cos, sin, kc, vc, lens, w.scale, n_sink, window, out=out, lse=lse, ws=ws)

    ms = _graph_ms(step, steps, flush)
    nbytes = w.B * w.Hk * cap * w.d * 2 * 2 + w.B * w.H * w.d * 2 * 2 + w.B * w.H * 4
    return {"workload": f"llama3_8b_decode_B16_H32_Hk8_len{length}_sink{n_sink}_window{window}",
            "ms_per_step": round(ms, 5), "algorithmic_bytes": nbytes,
            "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "pct_of_hbm_peak": round(100 * nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 1),
            "pct_of_nominal_8tbs": round(100 * nbytes / (ms * 1e-3) / 1e9 / 8000.0, 1),
            "tok_per_s": round(w.B / (ms * 1e-3), 1)}


def measure_others(K, device, steps, flush, peaks):
    res = {}
    for w in (W.TINY_GQA, W.LLAMA2_70B_GQA_32K, W.LLAMA2_70B_MQA_32K, W.LLAMA2_70B_MHA_32K):
        res[w.name] = measure_decode_config(K, w, device, steps, flush, peaks)
    win = measure_window(K, device, steps, flush, peaks)
    res[win["workload"]] = win
    res[W.PREFILL_8K.name] = measure_prefill(K, device, steps, flush, peaks)
    pw = measure_prefill_window(K, device, steps, flush, peaks)
    res[pw["workload"]] = pw
    res[W.DSA_128K.name] = measure_dsa(K, device, steps, flush, peaks)
    torch.cuda.empty_cache()
    res[W.QSA_128K.name] = measure_qsa(K, device, steps, flush, peaks)
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------- CPU oracle

def oracle_decode_sample(w, n_units, seed, nthreads):
    """(seconds, algorithmic bytes) of the fp64 oracle on the first n_units
    (batch, head) pairs of the workload."""
    import oracle
    inp = W.decode_inputs(w, seed=seed, lens=W.lengths(w.B, w.T_lo, w.T_hi, seed))
    qb, kb, vb = W.bf16_bits(inp["q"]), W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"])
    lens = inp["seq_lens"].numpy()
    sel = [(u // w.H, u % w.H) for u in range(n_units)]
    t0 = time.perf_counter()
    oracle.attn_decode(qb, kb, vb, lens, w.scale, sel=sel, nthreads=nthreads)
    dt = time.perf_counter() - t0
    nbytes = sum(int(lens[b]) * w.d * 2 * 2 + w.d * 2 * 2 + 4 for b, _ in sel)
    return dt, nbytes, (qb, kb, vb, lens, sel)


def cpu_baseline(budget_s=20.0):
    import oracle
    w = W.LLAMA3_8B_DECODE
    nthreads = oracle.max_threads()
    seed = W.SEED_BASE + w.index
    dt, nbytes, (qb, kb, vb, lens, sel) = oracle_decode_sample(w, w.B * w.H, seed, nthreads)
    reps, total_t = 1, dt
    while total_t < min(budget_s, 10.0) and reps < 50:
        t0 = time.perf_counter()
        oracle.attn_decode(qb, kb, vb, lens, w.scale, sel=sel, nthreads=nthreads)
        total_t += time.perf_counter() - t0
        reps += 1
    return {"value": round(nbytes * reps / total_t / 1e9, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
            "sample": f"full {w.name} batch ({w.B * w.H} (batch, head) outputs), {reps} passes, fp64"}


def run_reference(args):
    import oracle
    w = W.LLAMA3_8B_DECODE
    nthreads = oracle.max_threads()
    seed = W.SEED_BASE + w.index
    # size one step so that warmup + steps fit in about two minutes
    dt_full, _, _ = oracle_decode_sample(w, w.B * w.H, seed, nthreads)
    frac = min(1.0, 120.0 / max(1, args.steps + args.warmup) / max(dt_full, 1e-6))
    n_units = max(1, int(frac * w.B * w.H))
    inp = W.decode_inputs(w, seed=seed, lens=W.lengths(w.B, w.T_lo, w.T_hi, seed))
    qb, kb, vb = W.bf16_bits(inp["q"]), W.bf16_bits(inp["k"]), W.bf16_bits(inp["v"])
    lens = inp["seq_lens"].numpy()
    sel = [(u // w.H, u % w.H) for u in range(n_units)]
    nbytes = sum(int(lens[b]) * w.d * 2 * 2 + w.d * 2 * 2 + 4 for b, _ in sel)
    for _ in range(args.warmup):
        oracle.attn_decode(qb, kb, vb, lens, w.scale, sel=sel, nthreads=nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attn_decode(qb, kb, vb, lens, w.scale, sel=sel, nthreads=nthreads)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    val = nbytes / dt / 1e9
    sample = f"{n_units} of {w.B * w.H} (batch, head) outputs of {w.name} per step, fp64"
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded workload)",
        "config": {"workload": w.name, "B": w.B, "n_head": w.H, "n_kv_head": w.Hk, "head_dim": w.d,
                   "T_max": w.T_max, "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------- distributed plumbing

def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _reduce(x, world, device, op):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x, world, device):
    return _reduce(x, world, device, torch.distributed.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x, world, device):
    return _reduce(x, world, device, torch.distributed.ReduceOp.SUM if world > 1 else None)


def rank_seed(w, rank):
    """Every rank draws its own batch (own ragged lengths) of the workload."""
    return W.SEED_BASE + w.index + rank


def whole_job(local_bytes, local_ms, world, device):
    """(bytes all ranks processed, max-over-ranks step time): the weak-scaling
    throughput is their ratio."""
    return sum_over_ranks(float(local_bytes), world, device), max_over_ranks(local_ms, world, device)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvattn", choices=["kvattn", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true", help="skip the other configurations")
    ap.add_argument("--only", choices=["tiny", "gqa32k", "mqa32k", "mha32k", "window", "prefill", "prefill_window", "dsa",
                                       "qsa"],
                    help="time one other configuration alone and print its JSON")
    ap.add_argument("--batch", type=int, default=None,
                    help="with --only qsa: batch rows (default 8; a smaller case for profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    if args.only:
        from mqa_kv_cache_b200 import kvattn as K
        device = torch.device("cuda", local_rank)
        torch.cuda.set_device(device)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        peaks = load_peaks()
        decode = {"tiny": W.TINY_GQA, "gqa32k": W.LLAMA2_70B_GQA_32K, "mqa32k": W.LLAMA2_70B_MQA_32K,
                  "mha32k": W.LLAMA2_70B_MHA_32K}
        if args.only in decode:
            res = measure_decode_config(K, decode[args.only], device, args.steps, flush, peaks)
        elif args.only == "prefill":
            res = measure_prefill(K, device, args.steps, flush, peaks)
        elif args.only == "window":
            res = measure_window(K, device, args.steps, flush, peaks)
        elif args.only == "prefill_window":
            res = measure_prefill_window(K, device, args.steps, flush, peaks)
        elif args.only == "qsa":
            res = measure_qsa(K, device, args.steps, flush, peaks, B=args.batch)
        else:
            res = measure_dsa(K, device, args.steps, flush, peaks)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    line = run_gpu(args, rank, world, device)
    if not args.headline_only:
        from mqa_kv_cache_b200 import kvattn as K
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        line["other_configs"] = measure_others(K, device, args.steps, flush, load_peaks())
        # the read side of the denominator: the best read-only streaming rate seen in this run
        # (a plain reduction, or a decode kernel that only reads K and V)
        rates = [line["roofline"]["read_stream_gbs"]] + [v["GB_s"] for v in line["other_configs"].values()
                                                          if isinstance(v, dict) and "GB_s" in v]
        rp = max(rates)
        line["roofline"]["read_peak_gbs"] = round(rp, 1)
        line["roofline"]["frac_of_read_peak"] = round(line["roofline"]["achieved"] / rp, 4)
    if world > 1:
        torch.distributed.destroy_process_group()
    # the oracle on the host cores: rank 0 of a single-GPU run only
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
