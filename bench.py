#!/usr/bin/env python
"""Benchmark of the exact attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one forward over one batch of the main workload (default: the
largest single-GPU configuration, dense non-causal MHA B=1 S=20480 H=56 D=128
bf16, the long video-DiT validation shape).  Rank 0 prints ONE JSON line with
the throughput in TFLOP/s (4 * q_len * k_len * D * Hq per sequence, halved for
causal), the roofline of the kernel, the CPU oracle baseline, an end-to-end
figure through host buffers, the SM clocks seen while timing, and the other
workloads measured the same way ("workloads"; among them the varlen causal
GQA 32/8 D=128 workload with a 256-wide relative bias, and fp16 twins of two
bf16 workloads).

Multi-GPU (launched by torchrun): every rank runs its own copy of the workload
(independent problems, no data-path collective: weak scaling); the time is the
maximum over ranks of the device-measured time.

``--impl reference`` times the CPU fp64 oracle instead (rank 0 only), on a
bounded sample of rows of the same workload per step.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s & % of BF16 tensor peak; split-KV decode HBM GB/s"
MAIN = "video_dit_20480"
EXTRAS = ["varlen_gqa_bias", "dense_257", "encoder_d256_seqused", "decode_splitkv", "dense_d64",
          "local_window_softcap", "tabpfn_d16", "vision_d72", "dense_d256"]
# the same shapes in fp16: a bf16 / fp16 pair per shape ("FlashAttention-4
# backend for Blackwell #1235", Benchmarking, reports a bf16 slow-down on sm_100)
FP16_TWINS = ["video_dit_20480", "dense_d64"]
L2_BYTES = 126 << 20  # B200; the device's own figure replaces it where CUDA is up
DESCR = {
    "dense_257": "dense non-causal MHA B=1 S=257 H=8 D=128 bf16",
    "varlen_gqa_bias": "varlen causal GQA 32/8 D=128, 4 seqs U[512,4096] (seeded), rel_bias R=256 bf16",
    "video_dit_20480": "dense non-causal MHA B=1 S=20480 H=56 D=128 bf16",
    "encoder_d256_seqused": "dense GQA 8/1 D=256 B=2 Sq=1024 Sk=1024 seqused_k=968 bf16",
    "decode_splitkv": "split-KV decode B=8 Sq=1 Sk=131072 Hq=32 Hkv=8 D=128 bf16",
    "dense_d64": "dense non-causal MHA B=4 S=4096 H=16 D=64 bf16",
    "local_window_softcap": "causal GQA 16/4 D=128 B=1 S=32768, window 4095 left, softcap 50 bf16",
    "tabpfn_d16": "dense non-causal MHA B=1 S=30000 H=8 D=16 fp16",
    "vision_d72": "dense non-causal MHA B=32 S=729 H=16 D=72 bf16",
    "dense_d256": "dense non-causal MHA B=4 S=4096 H=8 D=256 bf16 (CTA-pair kernel)",
}
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=MAIN)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--splits", type=int, default=0, help="split-KV count (0 = auto)")
    ap.add_argument("--decode-sk", type=int, default=131072,
                    help="keys of the decode workload (smaller values for profiling)")
    ap.add_argument("--dit-s", type=int, default=20480,
                    help="sequence length of the video workload (smaller values for profiling)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# peaks, profiles, clocks
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]), "hbm_gbs": float(d["hbm_gbs"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=FALLBACK_PEAKS["bf16_tflops"],
                    source="fallback")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "exact_attention_forward_flash_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the main kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"fa_fwd_{workload}.ncu.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line:
                    a, b = line.split(":", 1)
                    kv[a.strip()] = b.strip()
        if kv.get("kernel_source_sha256") != kernel_source_hash():
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self._read()  # first calls resolve the NVML entry points: keep them out of the region
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _read(self):
        """(SM clock in MHz, active clock-event reason bits)."""
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        return mhz, int(r)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz, r = self._read()
                self.samples.append(mhz)
                self.reasons |= r
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# workloads on the device
# ---------------------------------------------------------------------------
BIG = {"decode_splitkv"}


DECODE_SK = 131072


DIT_S = 20480


def build_problem(name: str, device, dtype=None):
    import torch
    import fa_inputs
    dtype = dtype or torch.bfloat16
    if name in BIG:
        return fa_inputs.make(name, dtype=dtype, device=device, decode_sk=DECODE_SK)
    return fa_inputs.make(name, dtype=dtype, dit_s=DIT_S).to(device)


def workload_config(name: str, p, world: int, l2_bytes: int = L2_BYTES) -> dict:
    """The `config` object of the JSON line: the workload and how it is timed.
    Both arms print the same one for the same workload."""
    small = p.hbm_bytes() < 2 * l2_bytes
    return {"workload": f"{name}: {DESCR[name]}", "global_batch": p.B * world,
            "seq_len": p.max_seqlen_q,
            "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
            "l2": (f"{p.hbm_bytes() / 1e6:.0f} MB touched per step < 2 x L2: a buffer of 4 x L2 "
                   "is overwritten before every step, outside its events; time = per-step "
                   "event mean" if small else
                   f"inputs larger than L2 ({p.hbm_bytes() / 1e6:.0f} MB per step), no flush")}


class Runner:
    """Preallocated outputs and one call per step through the C ABI."""

    def __init__(self, p, splits: int = 0):
        import torch
        import exact_attention_forward_flash_b200 as fa
        self.fa, self.p = fa, p
        self.out = torch.empty_like(p.q)
        if p.layout == "dense":
            self.lse = torch.empty((p.B, p.Hq, p.q.shape[1]), dtype=torch.float32, device=p.q.device)
        else:
            self.lse = torch.empty((p.Hq, p.q.shape[0]), dtype=torch.float32, device=p.q.device)
        self.ws = None
        self.launches = 1
        if p.splitkv:
            B, Sq, Hq, D = p.q.shape
            Sk, Hkv = p.k.shape[1], p.k.shape[2]
            n_sms = torch.cuda.get_device_properties(p.q.device).multi_processor_count
            self.ns = splits or fa.splitkv_default_splits(B, Sq, Sk, Hq, Hkv, D, n_sms)
            nbytes = fa.splitkv_workspace_bytes(B, Sq, Hq, D, self.ns)
            self.ws = torch.empty(nbytes, dtype=torch.uint8, device=p.q.device)
            self.launches = 2

    def __call__(self, q=None, k=None, v=None, rel_bias=None, cu=None):
        p, fa = self.p, self.fa
        q = p.q if q is None else q
        k = p.k if k is None else k
        v = p.v if v is None else v
        rb = p.rel_bias if rel_bias is None else rel_bias
        if p.splitkv:
            fa.fa_fwd_splitkv(q, k, v, num_splits=self.ns, causal=p.causal,
                              softmax_scale=p.softmax_scale, seqused_k=p.seqused_k,
                              rel_bias=rb, out=self.out, lse=self.lse, workspace=self.ws,
                              window=p.window, softcap=p.softcap)
        elif p.layout == "dense":
            fa.fa_fwd(q, k, v, causal=p.causal, softmax_scale=p.softmax_scale,
                      seqused_k=p.seqused_k, rel_bias=rb, out=self.out, lse=self.lse,
                      window=p.window, softcap=p.softcap)
        else:
            cq, ck = (p.cu_seqlens_q, p.cu_seqlens_k) if cu is None else cu
            fa.fa_fwd_varlen(q, k, v, cq, ck, p.max_seqlen_q, p.max_seqlen_k,
                             seqused_k=p.seqused_k, causal=p.causal,
                             softmax_scale=p.softmax_scale, rel_bias=rb, out=self.out,
                             lse=self.lse, window=p.window, softcap=p.softcap)


class nvtx_range:
    """A named NVTX range around a timed region, so that a profiler run can
    select it (ncu --nvtx); nothing when NVTX is unavailable."""

    def __init__(self, name: str):
        self.name, self.on = name, False

    def __enter__(self):
        try:
            import torch
            torch.cuda.nvtx.range_push(self.name)
            self.on = True
        except Exception:
            self.on = False
        return self

    def __exit__(self, *exc):
        if self.on:
            import torch
            torch.cuda.nvtx.range_pop()


def time_steps(step, steps: int, warmup: int, dist_on: bool, device_index: int,
               flush=None, label: str = "timed steps"):
    """W untimed steps, then K steps between barrier + synchronize; returns
    (total ms over K, mean per-step ms from per-step events, clocks).

    ``flush``: a device buffer larger than L2 that is overwritten before every
    step, outside that step's event pair, for workloads whose inputs fit in L2
    (their time is then the per-step event mean, cold L2)."""
    import torch
    import torch.distributed as dist
    # NVML is initialised before the warm-up, so that its first
    # initialisation (a host stall with the device idle) never sits between
    # the warm-up and the timed region.
    sampler = ClockSampler(device_index)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler as clk, nvtx_range(label):
        t0.record()
        for a, b in evs:
            if flush is not None:
                flush.zero_()
            a.record()
            step()
            b.record()
        t1.record()
        torch.cuda.synchronize()
    if dist_on:
        dist.barrier()
    total = t0.elapsed_time(t1)
    per = statistics.mean(a.elapsed_time(b) for a, b in evs)
    return total, per, clk.summary()


def time_e2e(p, p_cpu, splits: int, steps: int, dist_on: bool, world: int, unit: str):
    """End-to-end throughput through the public API with host buffers.

    Every step copies its inputs from pinned host memory to the device, runs
    the forward and copies O and LSE back to pinned host memory; all of it is
    inside the timed region.  Steps are software-pipelined over two buffer
    sets and three streams (copy-in, compute, copy-out), as a serving loop
    would be: step k's input copy overlaps step k-1's forward and output
    copy.  Events order each set's reuse (inputs are overwritten only after
    the forward two steps back has read them, outputs only after their copy
    to the host finished).  The time runs from before the first input copy
    to the end of the last output copy, over K steps."""
    import torch
    import torch.distributed as dist
    pin = lambda t: t.pin_memory() if t is not None else None  # noqa: E731
    h_in = [pin(p_cpu.q), pin(p_cpu.k), pin(p_cpu.v), pin(p_cpu.rel_bias),
            pin(p_cpu.cu_seqlens_q), pin(p_cpu.cu_seqlens_k)]
    d_in = [[torch.empty_like(t, device=p.q.device) if t is not None else None for t in h_in]
            for _ in range(2)]
    runners = [Runner(p, splits) for _ in range(2)]
    h_out = [(torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory(),
              torch.empty(r.lse.shape, dtype=torch.float32).pin_memory()) for r in runners]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_read = [torch.cuda.Event() for _ in range(2)]    # forward on set j done reading inputs
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of set j on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]    # O/LSE of set j on the host
    used = [False, False]

    def step(k):
        j = k % 2
        din, r = d_in[j], runners[j]
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ev_read[j])
            for d, h in zip(din, h_in):
                if d is not None:
                    d.copy_(h, non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[j])
            if used[j]:
                s_cmp.wait_event(ev_done[j])
            cu = (din[4], din[5]) if din[4] is not None else None
            r(din[0], din[1], din[2], din[3], cu)
            ev_read[j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_read[j])
            h_out[j][0].copy_(r.out, non_blocking=True)
            h_out[j][1].copy_(r.lse, non_blocking=True)
            ev_done[j].record(s_out)
        used[j] = True

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        dist.barrier()
    torch.cuda.synchronize()
    with nvtx_range("end to end"):
        t0.record(s_in)
        for k in range(steps):
            step(k)
        s_in.wait_stream(s_out)
        t1.record(s_in)
        torch.cuda.synchronize()
    if dist_on:
        dist.barrier()
    total = max_over_ranks(t0.elapsed_time(t1), dist_on)
    h2d = sum(t.numel() * t.element_size() for t in h_in if t is not None)
    d2h = sum(o.numel() * o.element_size() + l.numel() * 4 for o, l in h_out[:1])
    return {"value": round(world * workload_value(p, total / steps)[0], 3), "unit": unit,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(total / steps, 4),
            "pipeline": "2 buffer sets, copy-in / compute / copy-out streams"}


def time_short_calls(dev, n_calls: int = 2000, per_graph: int = 100, replays: int = 20):
    """Per-call cost of a short forward: the query block of a cached
    prediction (B=1, Sq=128, Sk=1024, MQA 8/1, D=64, fp16), called many times.
    Reports the wall time per call of eager calls through the public API,
    issued back to back (host marshalling + launch), and the device time per
    call when the same calls are replayed from one CUDA graph."""
    import torch
    import fa_inputs
    import exact_attention_forward_flash_b200 as fa
    p = fa_inputs.random_dense(900, 1, 128, 1024, 8, 1, 64, dtype=torch.float16).to(dev)
    out = torch.empty_like(p.q)
    lse = torch.empty((1, 8, 128), dtype=torch.float32, device=dev)

    ns = fa.splitkv_default_splits(1, 128, 1024, 8, 1, 64,
                                   torch.cuda.get_device_properties(dev).multi_processor_count)
    ws = torch.empty(max(16, fa.splitkv_workspace_bytes(1, 128, 8, 64, ns)), dtype=torch.uint8,
                     device=dev)

    def plain():
        fa.fa_fwd(p.q, p.k, p.v, softmax_scale=p.softmax_scale, out=out, lse=lse)

    def split():
        fa.fa_fwd_splitkv(p.q, p.k, p.v, num_splits=ns, softmax_scale=p.softmax_scale,
                          out=out, lse=lse, workspace=ws)

    def measure(call):
        for _ in range(20):
            call()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(n_calls):
            call()
        torch.cuda.synchronize()
        eager_us = (time.perf_counter() - t0) / n_calls * 1e6
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(per_graph):
                call()
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(replays):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        graph_us = e0.elapsed_time(e1) * 1e3 / (replays * per_graph)
        del graph
        return {"eager_us_per_call": round(eager_us, 2), "graph_us_per_call": round(graph_us, 2),
                "graph_tflops": round(p.flops() / (graph_us * 1e-6) / 1e12, 2)}

    with nvtx_range("short calls: fa_fwd"):
        plain_res = measure(plain)
    with nvtx_range("short calls: fa_fwd_splitkv"):
        split_res = measure(split)
    return {"shape": "dense B=1 Sq=128 Sk=1024 Hq=8 Hkv=1 D=64 fp16",
            "fa_fwd": plain_res, "fa_fwd_splitkv": dict(split_res, num_splits=ns)}


def time_context_parallel(dev, world: int, rank: int, local: int, dist_on: bool, steps: int,
                          warmup: int, peaks) -> dict:
    """The decode workload with its keys sharded across the ranks: each rank
    holds one contiguous shard of every sequence's keys, computes its fp32
    partial (split-KV kernel + merge into one partial), the ranks exchange the
    partials with one NCCL all-gather, and every rank merges them in the
    combine kernel (fa_fwd_context_parallel).  Total work is fixed as N grows
    (strong scaling); the value is the WHOLE problem's K/V bytes over the
    slowest rank's time.  With one rank there is no exchange."""
    import torch
    from exact_attention_forward_flash_b200.context_parallel import (
        fa_fwd_context_parallel, shard_bounds)
    full = build_problem("decode_splitkv", dev)
    B, Sk = full.B, full.k.shape[1]
    start, length, after = shard_bounds(Sk, world, rank)
    k = full.k[:, start:start + length].contiguous()
    v = full.v[:, start:start + length].contiguous()
    q, scale, nbytes = full.q, full.softmax_scale, full.hbm_bytes()
    del full
    torch.cuda.empty_cache()
    k_after = torch.full((B,), after, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, q.shape[2], q.shape[1]), dtype=torch.float32, device=dev)

    def step():
        fa_fwd_context_parallel(q, k, v, k_after=k_after, softmax_scale=scale, out=out, lse=lse)

    tt, pm, ck = time_steps(step, steps, max(3, warmup), dist_on, local,
                            label="timed steps: context parallel")
    tt = max_over_ranks(tt, dist_on)
    ms = tt / steps
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": DESCR["decode_splitkv"] + f", keys sharded over {world} rank(s), "
                                                 "one NCCL all-gather of the fp32 partials",
            "value": round(gbs, 1), "unit": "GB/s", "scaling": "strong",
            "ms_per_step": round(ms, 4), "frac_of_peak": round(gbs / peaks["hbm_gbs"] / world, 4),
            "keys_per_rank": length, "sm_mhz": ck.get("sm_mhz"),
            "gpu_launches_per_step": 3, "l2": "inputs larger than L2, no flush"}


def max_over_ranks(x: float, dist_on: bool) -> float:
    """The maximum of a per-rank time over all ranks (NCCL on the GPU, or a
    CPU tensor when the process group runs on gloo)."""
    if not dist_on:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(per_rank_units: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processes its own copy of the
    workload, so the units of all ranks are divided by the slowest rank's
    time (in ms), giving units per second."""
    return world * per_rank_units / (max_ms * 1e-3)


def roofline(p, per_launch_ms: float, peaks, traffic):
    if p.splitkv:
        achieved = p.hbm_bytes() / (per_launch_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": peaks["source"]}
    achieved = p.flops() / (per_launch_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    # the burst figure is the denominator; the sustained one (a GEMM looped
    # for seconds under the power cap) is shown beside it, for runs whose
    # clocks the cap holds down
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": peaks["source"] + " (burst)",
            "peak_sustained": peaks["bf16_tflops_sustained"],
            "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)}


def workload_value(p, ms):
    if p.splitkv:
        return p.hbm_bytes() / (ms * 1e-3) / 1e9, "GB/s"
    return p.flops() / (ms * 1e-3) / 1e12, "TFLOP/s"


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded row sample)
# ---------------------------------------------------------------------------
def oracle_rows_sample(p, n_rows: int, seed: int = 0):
    import numpy as np
    rng = np.random.default_rng(seed)
    lens = p.seq_lens()
    B = len(lens)
    rows, flops = [], 0.0
    for _ in range(n_rows):
        b = int(rng.integers(B))
        ql, kl = lens[b]
        while ql == 0:
            b = int(rng.integers(B))
            ql, kl = lens[b]
        i = int(rng.integers(ql))
        h = int(rng.integers(p.Hq))
        flops += 4.0 * p.D * p.admitted_keys(ql, kl, i)
        rows.append((b, h, i))
    return np.array(rows, dtype=np.int32), flops


def time_oracle(p_cpu, target_s: float):
    import oracle
    kw = dict(causal=p_cpu.causal, softmax_scale=p_cpu.softmax_scale,
              seqused_k=p_cpu.seqused_k, rel_bias=p_cpu.rel_bias, window=p_cpu.window,
              softcap=p_cpu.softcap)
    if p_cpu.layout == "varlen":
        kw.update(cu_seqlens_q=p_cpu.cu_seqlens_q, cu_seqlens_k=p_cpu.cu_seqlens_k)
    n = 64
    while True:
        rows, flops = oracle_rows_sample(p_cpu, n)
        t = time.perf_counter()
        oracle.attention_rows(p_cpu.q, p_cpu.k, p_cpu.v, rows, **kw)
        dt = time.perf_counter() - t
        if dt >= 0.5 * target_s or n >= 1 << 22:
            return flops / dt / 1e12, dt, n
        n = int(n * min(64.0, max(2.0, target_s / max(dt, 1e-3))))


# ---------------------------------------------------------------------------
def main():
    a = parse()
    global DECODE_SK, DIT_S
    DECODE_SK = a.decode_sk
    DIT_S = a.dit_s
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if a.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(a, world)

    import torch
    import torch.distributed as dist
    import exact_attention_forward_flash_b200 as fa
    fa.load_library()
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    peaks = load_peaks()

    # ---- main workload, device-resident inputs
    import fa_inputs
    p_cpu = fa_inputs.make(a.workload, dit_s=DIT_S) if a.workload not in BIG else None
    p = build_problem(a.workload, dev)
    run = Runner(p, a.splits)
    l2_bytes = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20)
    flush_buf = None
    main_small = p.hbm_bytes() < 2 * l2_bytes
    if main_small:
        flush_buf = torch.empty(4 * l2_bytes, dtype=torch.uint8, device=dev)
    total_ms, per_ms, clocks = time_steps(run, a.steps, a.warmup, dist_on, local,
                                          flush=flush_buf, label=f"timed steps: {a.workload}")
    if main_small:
        total_ms = per_ms * a.steps  # the flush between steps is not the workload's time
    total_ms = max_over_ranks(total_ms, dist_on)
    ms_step = total_ms / a.steps
    unit = workload_value(p, ms_step)[1]
    per_rank_units = p.hbm_bytes() / 1e9 if p.splitkv else p.flops() / 1e12
    value = weak_value(per_rank_units, world, ms_step)  # TFLOP/s or GB/s
    traffic = profiled_traffic(a.workload)
    roof = roofline(p, per_ms, peaks, traffic)

    # ---- end to end: pinned host inputs -> device -> library -> host outputs
    e2e = None
    if not p.splitkv and p_cpu is not None:
        e2e = time_e2e(p, p_cpu, a.splits, max(3, min(a.steps, 20)), dist_on, world, unit)

    # ---- the other workloads, same protocol (rank 0 reports its own)
    extras = {}
    if not a.no_extras:
        runs = [(n, False) for n in EXTRAS if n != a.workload]
        runs += [(n, True) for n in FP16_TWINS]
        for name, twin in runs:
            key = name + "_fp16" if twin else name
            q = build_problem(name, dev, torch.float16 if twin else None)
            r = Runner(q, a.splits)
            k_steps = max(5, min(a.steps, 30))
            small = q.hbm_bytes() < 2 * l2_bytes
            if small and flush_buf is None:
                flush_buf = torch.empty(4 * l2_bytes, dtype=torch.uint8, device=dev)
            tt, pm, ck = time_steps(r, k_steps, max(3, a.warmup), dist_on, local,
                                    flush=flush_buf if small else None,
                                    label=f"timed steps: {name}")
            if small:
                tt = pm * k_steps  # the flush between steps is not the workload's time
            tt = max_over_ranks(tt, dist_on)
            v, u = workload_value(q, tt / k_steps)
            rf = roofline(q, pm, peaks, None if twin else profiled_traffic(name))
            extras[key] = {"workload": DESCR[name] + (" (fp16 twin)" if twin else ""),
                           "value": round(world * v, 3), "unit": u,
                            "ms_per_step": round(tt / k_steps, 4), "frac_of_peak": rf["frac"],
                            "roofline": rf, "gpu_launches_per_step": r.launches,
                            "sm_mhz": ck.get("sm_mhz"),
                            "l2": ("flushed before every step (inputs fit in L2), per-step events"
                                   if small else "inputs larger than L2, no flush")}
            if q.splitkv:
                extras[key]["num_splits"] = r.ns
            del q, r
            torch.cuda.empty_cache()

    # ---- the decode workload with its keys sharded across the ranks (the one
    # form of the path with a data exchange between GPUs)
    if not a.no_extras:
        extras["decode_context_parallel"] = time_context_parallel(
            dev, world, rank, local, dist_on, max(5, min(a.steps, 30)), a.warmup, peaks)
        torch.cuda.empty_cache()

    # ---- many short calls: per-call overhead, eager and from a CUDA graph
    short = None
    if not a.no_extras:
        short = time_short_calls(dev)

    # ---- CPU oracle on this host (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and p_cpu is not None:
        import oracle
        v, secs, n = time_oracle(p_cpu, a.cpu_seconds)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
               "kind": "oracle",
               "sample": f"{n} random (b, h, i) rows of {a.workload}, fp64 C/OpenMP, {secs:.1f} s"}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
        "config": workload_config(a.workload, p, world, l2_bytes),
        "pct_of_bf16_peak": round(100 * roof["frac"], 2) if roof["bound"] == "tensor" else None,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": a.steps * run.launches,
        "clocks": clocks,
        "kernel_source_sha256": kernel_source_hash(),
        "workloads": extras,
        "short_calls": short,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_reference(a, world):
    """The CPU oracle as the reference arm: each step computes a bounded
    random sample of rows of the same workload."""
    import fa_inputs
    import oracle
    name = a.workload
    p = fa_inputs.make(name) if name not in BIG else None
    if p is None:
        print(json.dumps({"impl": "reference", "unavailable":
                          f"{name}: multi-GB inputs are drawn on the device only"}))
        return 0
    # size one step to ~cpu_seconds / steps of CPU work
    v0, secs0, n0 = time_oracle(p, max(0.5, a.cpu_seconds / max(1, a.steps + a.warmup)))
    kw = dict(causal=p.causal, softmax_scale=p.softmax_scale, seqused_k=p.seqused_k,
              rel_bias=p.rel_bias, window=p.window, softcap=p.softcap)
    if p.layout == "varlen":
        kw.update(cu_seqlens_q=p.cu_seqlens_q, cu_seqlens_k=p.cu_seqlens_k)
    samples = [oracle_rows_sample(p, n0, seed=s) for s in range(a.warmup + a.steps)]
    for rows, _ in samples[:a.warmup]:
        oracle.attention_rows(p.q, p.k, p.v, rows, **kw)
    flops = 0.0
    t = time.perf_counter()
    for rows, f in samples[a.warmup:]:
        oracle.attention_rows(p.q, p.k, p.v, rows, **kw)
        flops += f
    dt = time.perf_counter() - t
    value = flops / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(1e3 * dt / a.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
            "config": workload_config(name, p, world),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                             "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{n0} random rows per step of {name}, fp64 C/OpenMP"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
