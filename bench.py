#!/usr/bin/env python
"""MLA decode throughput on B200: latent-KV HBM GB/s and attended tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl xmla|reference]

A step is one decode step of the whole hot path over every layer of the
workload: RoPE on the queries and on the q_len new tokens, the append of those
tokens to the paged latent cache, and xmla_decode (q absorb, split-K latent
attention, LSE combine with W_UV).  The default workload is a single 256K
context (batch 1, q_len 1, 64-token pages in a shuffled order).

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by CUDA
events on the launching stream; the L2 is flushed before every step, outside
the events (a 256 MiB write, then a 256 MiB read so that no dirty lines are
left for the timed step to write back).  The K steps are bracketed by a barrier and a device
synchronise; the reported time is the max over ranks.  Under torchrun every
rank runs its own replica of the workload (independent sequences, no
collective on the data path): weak scaling.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MLA decode: latent-KV HBM GB/s (% of B200 peak) and attended tokens/s"
ROW_BYTES = 1152  # one cache row: [c_kv 512 | k_pe 64] bf16
Q8_ROW_BYTES = 608  # one 8-bit cache row: 576 codes, 18 exponents, 14 pad bytes
FALLBACK_HBM_GBS = 6650.0
# a device-side wait queued before a directly launched step, long enough for the
# host to queue the whole step behind it (~50 us at the B200's clock)
HOST_AHEAD_CYCLES = 100_000
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_256k")
    ap.add_argument("--impl", default="xmla", choices=["xmla", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "q8"],
                    help="q8: the 8-bit latent cache (int8 codes, a power-of-two scale per 32 "
                         "values, 608 B per token; decode only)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--shards", type=int, default=0,
                    help="sequence-parallel decode over this many page shards: with --gpus G "
                         "(torchrun) each rank holds one shard and the partials are all-gathered "
                         "over NCCL; on one GPU, rank 0's share is timed (its shard, the gathered "
                         "partials' combine; the all-gather becomes a local copy)")
    ap.add_argument("--workloads", default="decode_4k,step_40l_b32,verify_q4_b8,decode_512k_b4,prefill_4k",
                    help="other workloads measured in the same run (one GPU; step and split-K "
                         "kernel times and roofline fractions under the line's 'workloads' key); "
                         "empty to skip")
    ap.add_argument("--extra-steps", type=int, default=20)
    ap.add_argument("--with-producer", action="store_true",
                    help="the step starts from the new tokens' hidden states: "
                         "kv_a_proj_with_mqa + RoPE + append (xmla_kv_produce), then decode")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, device) -> float:
    """The largest per-rank value (a time) across all ranks of the job."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step: int, steps: int, max_total_ms: float, world: int) -> float:
    """Whole-job GB/s: what every rank streamed, over the slowest rank's time."""
    return bytes_per_rank_step * world * steps / (max_total_ms * 1e-3) / 1e9


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s): the measured burst figure for a kernel
    timed alone, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def workload_config(wl, world):
    return {
        "workload": wl.name,
        "batch_per_gpu": wl.batch,
        "q_len": wl.q_len,
        "context": wl.seqlens[0] if len(set(wl.seqlens)) == 1 else f"U[8192,65536] mean {sum(wl.seqlens) / len(wl.seqlens):.0f}",
        "layers": wl.layers,
        "heads": 32,
        "cache_row": "[c_kv 512 | k_pe 64] bf16",
        "paging": "64-token blocks, contiguous" if wl.contiguous else "64-token blocks, shuffled",
        "l2": "flushed before every timed step (256 MiB write, then 256 MiB read so no dirty lines remain)",
        "parallelism": f"dp{world} (independent replicas)",
    }


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls SM clock and clock-event (throttle) reasons through NVML every
    millisecond from a background thread while the timed region runs."""

    REASONS = {  # NVML clocks-event reason bits
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap",
    }

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.thread = None
        self.max_mhz = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
        except Exception:
            self.nvml = None
            return
        self.stop_flag = False

        def loop():
            get_r = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(self.nvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            while not self.stop_flag:
                try:
                    self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                    r = get_r(self.h)
                    for bit, name in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                time.sleep(0.001)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons), "source": "nvml"}


# ------------------------------------------------------------------ CPU oracle sample

def oracle_sample(wl, seconds: float, form: str = "expanded"):
    """Time the fp64 oracle (expanded, or absorbed over pre-rotated rope keys) on
    the first S tokens of sequence 0 (one query at position S-1, 32 heads), S
    chosen for about `seconds` of work."""
    import numpy as np
    import torch

    from mla_latent_kv_yarn_b200 import workloads
    from oracle import mla_oracle as om

    try:
        from threadpoolctl import threadpool_info
        cores = max([t.get("num_threads", 1) for t in threadpool_info()
                     if t.get("user_api") == "blas"] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    n_max = wl.seqlens[0]
    one = workloads.custom(1, 1, [n_max], seed=wl.seed, name=wl.name)
    inp = workloads.layer_inputs(one, 0, "cpu")
    c = inp.c_kv.double().numpy()
    kp = inp.k_pe.double().numpy()
    wk, wv = inp.W_UK.double().numpy(), inp.W_UV.double().numpy()
    q = inp.q[0].double().numpy()
    cfg = om.YarnConfig()

    kr = om.rope(kp, np.arange(n_max), cfg) if form == "absorbed" else None

    def run(n):
        t0 = time.perf_counter()
        if form == "absorbed":
            om.mla_attention_absorbed(q, c[:n], kr[:n], wk, wv, cfg)
        else:
            om.mla_attention_expanded(q, c[:n], kp[:n], wk, wv, cfg)
        return time.perf_counter() - t0

    probe_n = min(n_max, 4096)
    t_probe = run(probe_n)
    n = int(min(n_max, max(probe_n, probe_n * seconds / max(t_probe, 1e-6))))
    n = max(64, n // 64 * 64)
    return n, run, cores


# ------------------------------------------------------------------ reference arm

def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    per_step = max(1.0, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    n, run, cores = oracle_sample(wl, per_step)
    for _ in range(args.warmup):
        run(n)
    times = [run(n) for _ in range(args.steps)]
    total = sum(times)
    gbs = n * ROW_BYTES * args.steps / total / 1e9
    sample = (f"fp64 expanded oracle (numpy), sequence 0 of {wl.name}, first {n} tokens, "
              f"32 heads, q_len 1, one layer per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 6), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world),
        "attended_tokens_per_s": round(n * args.steps / total, 3),
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

# the translation unit of the timed kernel: its source and the headers it includes
# (the split-K kernel, or a prompt chunk's attention kernel)
KERNEL_SOURCES = ["mla_decode.cu", "split_kv.h", "xmla_device.cuh"]
PREFILL_SOURCES = ["prefill.cu", "prefill.h", "xmla_device.cuh"]


def kernel_sources_sha(names=None) -> str:
    h = hashlib.sha256()
    for name in names or KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mla_latent_kv_yarn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_record(kernel_src_sha: str, name: str, kernel: str = "mla_decode_kernel"):
    """DRAM bytes per launch of the timed kernel from a committed ncu summary,
    valid only while the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{name}_dram.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("kernel_sources_sha256") == kernel_src_sha:
            return float(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def roofline_line(wl, achieved, peak, peak_kind, traffic, cache_bytes, kernel_ms, flops, tpeak,
                  tpeak_kind, q8=False):
    """The split-K kernel against the HBM roofline (decode: every cache byte read
    once) and against the tensor roofline; a prefill chunk (q_len > 8) reads a
    few MB many times from L2 and is bound by the tensor side, which then leads."""
    tensor_achieved = flops / (kernel_ms * 1e-3) / 1e12
    hbm = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
           "frac": round(achieved / peak, 4), "traffic": traffic,
           "algorithmic_bytes_per_launch": cache_bytes, "peak_source": peak_kind}
    tensor = {"bound": "tensor", "achieved": round(tensor_achieved, 2), "peak": tpeak,
              "unit": "TFLOP/s", "frac": round(tensor_achieved / tpeak, 4),
              "flops_per_launch": flops, "peak_source": tpeak_kind}
    rows = 32 if wl.q_len == 1 or wl.q_len > 8 or wl.max_seqlen <= 4096 else 64
    lead, other = (tensor, hbm) if wl.q_len > 8 else (hbm, tensor)
    name = ("mla_decode_q8_kernel" if q8 else "prefill_attn_kernel" if wl.q_len >= PREFILL_MIN_CHUNK
            else f"mla_decode_kernel<{rows}>")
    line = dict(lead, kernel=name, kernel_ms=round(kernel_ms, 5))
    line[other["bound"]] = {k: v for k, v in other.items() if k != "bound"}
    if lead is tensor:
        line["traffic"] = traffic
    return line


# a chunk of at least this many new tokens per sequence runs the non-absorbed
# prompt path (the library's kPrefillMinChunk)
PREFILL_MIN_CHUNK = 64


def pair_flops(wl) -> int:
    """Algorithmic flop per attended (query, cache token) pair and head of the
    attention kernel that runs: absorbed (decode, short chunks) QK over 576 and
    PV over 512 dims, 2 x (576 + 512); non-absorbed (prompt chunks) QK over
    192 and PV over 128, 2 x (192 + 128)."""
    return 2 * (192 + 128) if wl.q_len >= PREFILL_MIN_CHUNK else 2 * (576 + 512)


def host_mapped(t) -> bool:
    """Whether pinned host tensor t is mapped into the device's address space at
    the same address (unified addressing), so kernels may use its pointer."""
    try:
        from cuda.bindings import runtime as rt
        err, dptr = rt.cudaHostGetDevicePointer(t.data_ptr(), 0)
        return int(err) == 0 and int(dptr) == t.data_ptr()
    except Exception:
        return False


def stage_tensors(tensors, dev):
    """One device buffer holding `tensors` back to back (each at a 256-byte
    boundary) and views into it carrying the same values, so that a step's
    inputs (or outputs) cross between host and device in a single copy."""
    import torch
    offs, total = [], 0
    for t in tensors:
        total = (total + 255) // 256 * 256
        offs.append(total)
        total += t.numel() * t.element_size()
    buf = torch.empty(total, dtype=torch.uint8, device=dev)
    views = []
    for t, o in zip(tensors, offs):
        v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views


def run_xmla(args, wl):
    import torch
    import torch.distributed as dist

    from mla_latent_kv_yarn_b200 import build, session, workloads, xmla

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    build.build()
    cfg = xmla.xmla_yarn_default()
    scale = xmla.xmla_softmax_scale(cfg, 192)

    # ---- set up every layer's cache and step inputs on this GPU
    layers = []
    for layer in range(wl.layers):
        inp = workloads.layer_inputs(wl, layer, dev)
        prefix, new = session.split_prefix(wl, inp)
        st = session.build_layer(cfg, wl, prefix, dev, cache=args.cache)
        L = {"st": st, "q": inp.q.clone(), "k_new": new.k_pe.clone(),
             "c_new": new.c_kv.clone(), "pos": new.positions.clone(),
             "sid": new.seq_ids.clone(),
             "out": torch.empty((wl.batch, wl.q_len, 32, 128), dtype=torch.bfloat16, device=dev)}
        if args.with_producer:
            L["hidden"], L["W_kva"] = workloads.producer_inputs(wl, layer, dev)
        layers.append(L)
        del inp, prefix, new
    # every layer's step inputs in one device buffer and the outputs in another:
    # the end-to-end loop moves each with a single copy
    step_inputs = ("q", "hidden", "pos", "sid") if args.with_producer else ("q", "k_new", "c_new", "pos", "sid")
    d_in, views = stage_tensors([L[k] for L in layers for k in step_inputs], dev)
    for n, v in enumerate(views):
        layers[n // len(step_inputs)][step_inputs[n % len(step_inputs)]] = v
    d_out, views = stage_tensors([L["out"] for L in layers], dev)
    for L, v in zip(layers, views):
        L["out"] = v
    torch.cuda.synchronize()
    dec = session.Decoder(wl.batch, wl.q_len, wl.max_seqlen, dev, cache=args.cache)
    ev_attn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in layers]
    for a, b in ev_attn:          # materialise the events before capture
        a.record()
        b.record()
    torch.cuda.synchronize()

    def step(events=True):
        for L, ev in zip(layers, ev_attn):
            if args.with_producer:
                dec.step_from_hidden(cfg, L["st"], L["q"], L["hidden"], L["W_kva"], L["pos"],
                                     L["sid"], scale, out=L["out"], events=ev if events else None)
            else:
                dec.step(cfg, L["st"], L["q"], L["c_new"], L["k_new"], L["pos"], L["sid"], scale,
                         out=L["out"], events=ev if events else None)

    # eager warm-up (loads modules), then capture the step: `graph` is what is timed
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(events=False)
    torch.cuda.synchronize()
    if dec.check_status() != 0:
        raise RuntimeError(f"device status {dec.check_status()} after warm-up")

    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2(i):
        # evict everything (write), then replace the now-dirty lines with clean
        # ones (read) so the timed step does not pay for their write-back
        flush_w.fill_(i & 0xFF)
        flush_r.sum()

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        flush_l2(i)
        graph.replay()
        flush_l2(i)
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        step(events=True)
    torch.cuda.synchronize()

    def timed(g):
        """K steps, each bracketed by events on the stream; L2 flushed between."""
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ms = []
        for i in range(args.steps):
            flush_l2(i + 1)
            e0[i].record(stream)
            g.replay()
            e1[i].record(stream)
            e1[i].synchronize()
            ms.append(e0[i].elapsed_time(e1[i]))
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return ms

    def timed_kernel():
        """Every layer's split-K kernel timed alone: CUDA events recorded on the
        stream immediately before and after it (xmla_decode_step's profiling
        events).  The step is launched directly for this, not replayed from the
        graph (an event-record node inside a graph breaks the programmatic launch
        chain and delays the next kernel by several microseconds), queued behind
        the L2 flush and a short device-side wait, so the device never waits for
        the host."""
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        attn = []
        for i in range(args.steps):
            flush_l2(i + 1)
            torch.cuda._sleep(HOST_AHEAD_CYCLES)
            step(events=True)
            torch.cuda.synchronize()
            attn.extend(a.elapsed_time(b) for a, b in ev_attn)
        if world > 1:
            dist.barrier()
        return attn

    # the clock sampler runs over every timed phase of this workload (the steps,
    # the kernel-timed steps and the end-to-end steps), so it takes many samples
    clocks = ClockSampler(local)
    clocks.start()
    step_ms = timed(graph)
    attn_ms = timed_kernel()
    total_ms = max_over_ranks(sum(step_ms), dev)
    status = dec.check_status()
    # a cache that fits in L2 is also timed warm: the same steps back to back with
    # no flush between them (the cache and weights stay resident)
    fits_l2 = sum(wl.seqlens) * wl.layers * ROW_BYTES < (96 << 20)
    warm_ms = None
    if fits_l2:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            graph.replay()
        w0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        w1.record(stream)
        w1.synchronize()
        warm_ms = max_over_ranks(w0.elapsed_time(w1), dev)

    # ---- end to end through the API: every step's inputs copied in from pinned host
    # memory (one staging buffer), the step run, its outputs copied back
    h_in = torch.empty_like(d_in, device="cpu").pin_memory()
    h_in.copy_(d_in)
    h_out = torch.empty_like(d_out, device="cpu").pin_memory()
    h2d = d_in.numel()
    d2h = d_out.numel()

    ee0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ee1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e2e_ms = []
    for i in range(args.steps):
        flush_l2(i + 7)
        ee0[i].record(stream)
        d_in.copy_(h_in, non_blocking=True)
        graph.replay()
        h_out.copy_(d_out, non_blocking=True)
        ee1[i].record(stream)
        ee1[i].synchronize()
        e2e_ms.append(ee0[i].elapsed_time(ee1[i]))
    e2e_copy_total = max_over_ranks(sum(e2e_ms), dev)

    # The same step with the kernels reading the step's inputs from, and writing
    # its outputs to, those pinned host buffers directly (mapped into the device's
    # address space): the bytes still cross the bus every step, without the two
    # copy operations and their fixed latency.  Only for small steps (at most 64 KiB
    # of inputs: a decode step of a few sequences; larger inputs move faster as
    # one copy), decode steps (a prompt chunk's tensor-core absorb reads the
    # query by TMA, which stays on device memory), and inputs read once: the
    # producer's 144 blocks each read every hidden state, which over the bus cost
    # more than one copy (2.73 vs 3.47 TB/s measured).
    zero_copy = (wl.q_len <= 8 and h2d <= 64 * 1024 and not args.with_producer and
                 host_mapped(h_in) and host_mapped(h_out))
    if world > 1:
        f = torch.tensor([1 if zero_copy else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(f, op=dist.ReduceOp.MIN)
        zero_copy = bool(f.item())
    e2e_total = e2e_copy_total
    if zero_copy:
        def remap(views, dbuf, hbuf):
            base = dbuf.data_ptr()
            return [hbuf[v.data_ptr() - base:v.data_ptr() - base + v.numel() * v.element_size()]
                    .view(v.dtype).view(v.shape) for v in views]
        in_views = [L[k] for L in layers for k in step_inputs]
        for n, v in enumerate(remap(in_views, d_in, h_in)):
            layers[n // len(step_inputs)][step_inputs[n % len(step_inputs)]] = v
        out_dev = [L["out"] for L in layers]
        for L, v in zip(layers, remap(out_dev, d_out, h_out)):
            L["out"] = v
        with torch.cuda.stream(side):
            step(events=False)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph_zc = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_zc):
            step(events=False)
        for i in range(args.warmup):
            flush_l2(i)
            graph_zc.replay()
        torch.cuda.synchronize()
        # the host-buffer step gives the same outputs as the device-buffer step
        graph.replay()
        torch.cuda.synchronize()
        if not torch.equal(d_out.cpu(), h_out):
            raise RuntimeError("zero-copy step output differs from the device-buffer step")
        zc_ms = []
        for i in range(args.steps):
            flush_l2(i + 11)
            ee0[i].record(stream)
            graph_zc.replay()
            ee1[i].record(stream)
            ee1[i].synchronize()
            zc_ms.append(ee0[i].elapsed_time(ee1[i]))
        e2e_total = max_over_ranks(sum(zc_ms), dev)
        del graph_zc
    clk = clocks.stop()

    q8 = args.cache == "q8"
    cache_bytes_layer = sum(wl.seqlens) * (Q8_ROW_BYTES if q8 else ROW_BYTES)
    tokens_step = sum(wl.seqlens) * wl.layers * world
    bytes_step = cache_bytes_layer * wl.layers * world
    gbs = job_throughput(cache_bytes_layer * wl.layers, args.steps, total_ms, world)
    peak, peak_kind = measured_peaks()
    tpeak, tpeak_kind = measured_tensor_peak()
    # query j of a sequence of n tokens attends n - q_len + j + 1 tokens (causal)
    pairs = sum(wl.q_len * (n - wl.q_len) + wl.q_len * (wl.q_len + 1) // 2 for n in wl.seqlens)
    flops_layer = pair_flops(wl) * 32 * pairs
    attn_mean_ms = statistics.mean(attn_ms)
    achieved = cache_bytes_layer / (attn_mean_ms * 1e-3) / 1e9
    if wl.q_len >= PREFILL_MIN_CHUNK:
        traffic = traffic_record(kernel_sources_sha(PREFILL_SOURCES), wl.name, "prefill_attn_kernel")
    else:
        traffic = None if q8 else traffic_record(kernel_sources_sha(), wl.name)
    # per layer and step: prologue (append or producer + q absorb), split-K
    # attention, combine; on the 8-bit cache the append is a kernel of its own; a
    # prompt chunk: query prep (+ append), K/V expansion, attention
    launches = (4 if q8 else 3) * wl.layers * args.steps

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(gbs, 3), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16" if q8 else "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl, world), **(
                {"step": "hidden states in: kv_a_proj_with_mqa + RoPE + append, then decode"}
                if args.with_producer else {}), **(
                {"cache_row": "q8: 576 int8 codes + 18 power-of-two block exponents (32 values "
                              "each), 608 B", "step": "8-bit append (quantise) + decode"}
                if q8 else {})),
            "attended_tokens_per_s": round(tokens_step * args.steps / (total_ms * 1e-3), 1),
            **({"attended_pairs_per_s": round(pairs * wl.layers * world * args.steps /
                                              (total_ms * 1e-3), 1)} if wl.q_len > 1 else {}),
            **({"warm": {"ms_per_step": round(warm_ms / args.steps, 5),
                         "value": round(job_throughput(cache_bytes_layer * wl.layers, args.steps,
                                                       warm_ms, world), 3),
                         "unit": "GB/s", "l2": "not flushed; steps back to back"}}
               if warm_ms is not None else {}),
            "pct_of_hbm_peak": round(100.0 * gbs / (peak * world), 2),
            "roofline": roofline_line(wl, achieved, peak, peak_kind, traffic, cache_bytes_layer,
                                      attn_mean_ms, flops_layer, tpeak, tpeak_kind, q8),
            "e2e": {"value": round(job_throughput(cache_bytes_layer * wl.layers, args.steps,
                                                  e2e_total, world), 3),
                    "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "transfer": "kernels read inputs from / write outputs to pinned host memory"
                                if zero_copy else "cudaMemcpyAsync in and out each step",
                    "with_copies": round(job_throughput(cache_bytes_layer * wl.layers, args.steps,
                                                        e2e_copy_total, world), 3)},
            "gpu_launches": launches,
            "splits": dec.splits,
            "device_status": status,
        }
        if clk is not None:
            # the step time scaled to the maximum SM clock, for runs whose clocks differ
            clk["ms_per_step_x_mhz_over_max"] = round(
                total_ms / args.steps * clk["sm_mhz"] / clk["sm_max_mhz"], 5) \
                if clk.get("sm_max_mhz") else None
            line["clocks"] = clk
        if world == 1 and not args.no_cpu_baseline and not q8:
            n, run, cores = oracle_sample(wl, args.cpu_seconds)
            t = run(n)
            line["cpu_baseline"] = {
                "value": round(n * ROW_BYTES / t / 1e9, 6), "unit": "GB/s", "cores": cores,
                "kind": "oracle",
                "sample": f"fp64 expanded oracle (numpy), sequence 0 of {wl.name}, first {n} "
                          f"tokens, 32 heads, q_len 1, one layer ({t:.1f} s)"}
            n2, run2, cores2 = oracle_sample(wl, args.cpu_seconds / 2, form="absorbed")
            t2 = run2(n2)
            line["cpu_baseline_absorbed"] = {
                "value": round(n2 * ROW_BYTES / t2 / 1e9, 6), "unit": "GB/s", "cores": cores2,
                "kind": "oracle",
                "sample": f"fp64 absorbed oracle (numpy, rope keys rotated beforehand), sequence 0 "
                          f"of {wl.name}, first {n2} tokens, 32 heads, q_len 1, one layer "
                          f"({t2:.1f} s)"}
    del graph
    if rank == 0:
        extra = [w for w in args.workloads.split(",") if w and w != wl.name]
        if extra and world == 1 and not q8 and not args.with_producer:
            layers.clear()
            del d_in, d_out, dec, flush_w, flush_r
            torch.cuda.empty_cache()
            line["workloads"] = {w: measure_other(workloads.workload(w), args, dev, cfg, scale)
                                 for w in extra}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def measure_other(wl, args, dev, cfg, scale):
    """Another workload in the same run, timed like the headline one (the step
    captured in a CUDA graph, L2 flushed before every step, CUDA events on the
    stream; the split-K kernel timed in a second graph with events around it),
    without the end-to-end and CPU legs.  Returns step and kernel times and the
    kernel's fractions of the HBM and tensor rooflines."""
    import torch

    from mla_latent_kv_yarn_b200 import session, workloads

    steps = max(3, args.extra_steps)
    layers = []
    for layer in range(wl.layers):
        inp = workloads.layer_inputs(wl, layer, dev)
        prefix, new = session.split_prefix(wl, inp)
        st = session.build_layer(cfg, wl, prefix, dev)
        layers.append({"st": st, "q": inp.q.clone(), "c": new.c_kv.clone(), "k": new.k_pe.clone(),
                       "pos": new.positions.clone(), "sid": new.seq_ids.clone(),
                       "out": torch.empty((wl.batch, wl.q_len, 32, 128), dtype=torch.bfloat16,
                                          device=dev)})
        del inp, prefix, new
    torch.cuda.synchronize()
    dec = session.Decoder(wl.batch, wl.q_len, wl.max_seqlen, dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in layers]
    for a, b in ev:
        a.record()
        b.record()

    def step(events):
        for L, e in zip(layers, ev):
            dec.step(cfg, L["st"], L["q"], L["c"], L["k"], L["pos"], L["sid"], scale,
                     out=L["out"], events=e if events else None)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(False)
        step(False)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(False)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush(i):
        flush_w.fill_(i & 0xFF)
        flush_r.sum()

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        flush(i)
        graph.replay()
        flush(i)
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        step(True)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_ms, attn_ms = [], []
    for i in range(steps):
        flush(i + 1)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        e1.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    for i in range(steps):  # the split-K kernels alone, as in run_xmla's timed_kernel
        flush(i + 1)
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        step(True)
        torch.cuda.synchronize()
        attn_ms.extend(a.elapsed_time(b) for a, b in ev)
    clk = clocks.stop()
    status = dec.check_status()
    del graph
    cache_bytes_layer = sum(wl.seqlens) * ROW_BYTES
    pairs = sum(wl.q_len * (n - wl.q_len) + wl.q_len * (wl.q_len + 1) // 2 for n in wl.seqlens)
    flops_layer = pair_flops(wl) * 32 * pairs
    peak, peak_kind = measured_peaks()
    tpeak, tpeak_kind = measured_tensor_peak()
    step_mean = statistics.mean(step_ms)
    kern = statistics.mean(attn_ms)
    res = {
        "config": {k: v for k, v in workload_config(wl, 1).items() if k not in ("l2", "parallelism")},
        "steps": steps,
        "ms_per_step": round(step_mean, 5),
        "value": round(cache_bytes_layer * wl.layers / (step_mean * 1e-3) / 1e9, 3), "unit": "GB/s",
        "pct_of_hbm_peak": round(100.0 * cache_bytes_layer * wl.layers / (step_mean * 1e-3) / 1e9
                                 / peak, 2),
        "attended_tokens_per_s": round(sum(wl.seqlens) * wl.layers / (step_mean * 1e-3), 1),
        "kernel_ms": round(kern, 5),
        "kernel_hbm_frac": round(cache_bytes_layer / (kern * 1e-3) / 1e9 / peak, 4),
        "kernel_tensor_frac": round(flops_layer / (kern * 1e-3) / 1e12 / tpeak, 4),
        "peak_source": {"hbm": peak_kind, "tensor": tpeak_kind},
        "gpu_launches": 3 * wl.layers * steps,
        "device_status": status,
    }
    if wl.q_len > 1:
        res["attended_pairs_per_s"] = round(pairs * wl.layers / (step_mean * 1e-3), 1)
    if clk is not None:
        res["clocks"] = clk
    layers.clear()
    del dec, flush_w, flush_r
    torch.cuda.empty_cache()
    return res


def run_shards(args, wl):
    """Sequence-parallel decode (no append): every layer's pages are dealt out
    over G shards; one timed step is, per layer, xmla_decode_shard on this
    rank's pages, the all-gather of the partials, and xmla_combine_shards."""
    import torch
    import torch.distributed as dist

    from mla_latent_kv_yarn_b200 import build, session, workloads, xmla
    from mla_latent_kv_yarn_b200 import seq_parallel as sp

    rank, world, local = dist_env()
    G = args.shards
    if world not in (1, G):
        raise SystemExit(f"--shards {G} runs on one GPU (emulated rank 0) or on {G} GPUs")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    build.build()
    cfg = xmla.xmla_yarn_default()
    scale = xmla.xmla_softmax_scale(cfg, 192)
    layers = []
    for layer in range(wl.layers):
        inp = workloads.layer_inputs(wl, layer, dev)
        full = session.build_layer(cfg, wl, inp, dev)
        sh = sp.ShardDecoder(wl.batch, wl.q_len, wl.max_seqlen, G, rank, dev)
        st = sp.shard_layer(full, sh.page_lo, sh.page_hi)
        if world == 1:
            # the other ranks' partials, computed once: the combine reads all G
            parts = []
            for r in range(G):
                o = sp.ShardDecoder(wl.batch, wl.q_len, wl.max_seqlen, G, r, dev)
                o.decode_shard(cfg, sp.shard_layer(full, o.page_lo, o.page_hi), inp.q, scale)
                parts.append(o.partial.clone())
                del o
            sh.gathered.copy_(torch.cat(parts))
        layers.append({"st": st, "sh": sh, "q": inp.q.clone(), "W_UV": full.W_UV})
        del inp, full
        torch.cuda.empty_cache()
    torch.cuda.synchronize()
    P = layers[0]["sh"].partial_floats

    def step():
        for L in layers:
            sh = L["sh"]
            sh.decode_shard(cfg, L["st"], L["q"], scale)
            if world > 1:
                sh.gather()
            else:
                sh.gathered[:P].copy_(sh.partial)   # stands in for the all-gather
            sh.combine(L["W_UV"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    status = max(int(L["sh"].status.item()) for L in layers)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2(i):
        flush_w.fill_(i & 0xFF)
        flush_r.sum()

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        flush_l2(i)
        graph.replay()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    ms = []
    for i in range(args.steps):
        flush_l2(i + 1)
        e0[i].record(stream)
        graph.replay()
        e1[i].record(stream)
        e1[i].synchronize()
        ms.append(e0[i].elapsed_time(e1[i]))
    clk = clocks.stop()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(ms), dev)

    # end to end: q in from pinned host memory, the output back, every step
    h_q = [L["q"].cpu().pin_memory() for L in layers]
    h_out = [torch.empty_like(L["sh"].out, device="cpu").pin_memory() for L in layers]
    ee0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ee1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e2e_ms = []
    for i in range(args.steps):
        flush_l2(i + 7)
        ee0[i].record(stream)
        for L, h in zip(layers, h_q):
            L["q"].copy_(h, non_blocking=True)
        graph.replay()
        for L, h in zip(layers, h_out):
            h.copy_(L["sh"].out, non_blocking=True)
        ee1[i].record(stream)
        ee1[i].synchronize()
        e2e_ms.append(ee0[i].elapsed_time(ee1[i]))
    e2e_total = max_over_ranks(sum(e2e_ms), dev)

    sh0 = layers[0]["sh"]
    tokens_shard = sum(max(0, min(n, 64 * sh0.page_hi) - min(n, 64 * sh0.page_lo))
                       for n in wl.seqlens)
    # whole-job throughput: the cache of every layer, all shards together, per step
    cache_bytes = sum(wl.seqlens) * ROW_BYTES * wl.layers
    own_bytes = tokens_shard * ROW_BYTES * wl.layers
    if rank == 0:
        gbs = cache_bytes * args.steps / (total_ms * 1e-3) / 1e9
        peak, peak_kind = measured_peaks()
        line = {
            "metric": METRIC, "value": round(gbs if world > 1 else
                                             own_bytes * args.steps / (total_ms * 1e-3) / 1e9, 3),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "strong" if world > 1 else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl, world), **{
                "seq_parallel": f"{G} page shards per sequence" + (
                    "; one GPU: rank 0's shard timed, the all-gather replaced by a local copy "
                    "(value = that shard's cache bytes per second)" if world == 1 else
                    "; partials all-gathered over NCCL")}),
            "pct_of_hbm_peak": round(100.0 * (gbs if world > 1 else own_bytes * args.steps /
                                              (total_ms * 1e-3) / 1e9) / (peak * world), 2),
            "e2e": {"value": round((cache_bytes if world > 1 else own_bytes) * args.steps /
                                   (e2e_total * 1e-3) / 1e9, 3), "unit": "GB/s",
                    "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_q),
                    "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in h_out)},
            "gpu_launches": 4 * wl.layers * args.steps,
            "shard_pages": [sh0.page_lo, sh0.page_hi],
            "partial_bytes_per_rank": sh0.partial_floats * 4,
            "device_status": status,
            "peak_source": peak_kind,
        }
        if clk is not None:
            line["clocks"] = clk
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    from mla_latent_kv_yarn_b200 import workloads
    wl = workloads.workload(args.workload)
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.cache == "q8" and (args.with_producer or args.shards > 0 or wl.q_len > 8):
        raise SystemExit("--cache q8 runs decode steps (q_len <= 8) without --with-producer "
                         "or --shards")
    if args.shards > 0:
        return run_shards(args, wl)
    return run_xmla(args, wl)


if __name__ == "__main__":
    sys.exit(main())
