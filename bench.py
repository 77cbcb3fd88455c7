#!/usr/bin/env python
"""Benchmark of the paged MLA decode on B200: TB/s, TFLOPS and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload dsv3_decode]

A step is one pass of the whole hot path over one batch: the split-KV
scheduler, the decode kernel and (for split sequences) the combine kernel, all
through the C ABI.  The default workload is DeepSeek-V3-shaped decode: batch
64, s_q 1, 128 heads, every sequence 4096 tokens, 64-token pages shuffled in
the block table, q and cache ~ N(0, 1) in bf16, scale 1/sqrt(192).

Timing: W untimed warm-up steps, then exactly K steps, each a replay of a CUDA
graph of the step captured after the warm-up (the same three kernels, no host
work inside the events; e2e below runs eagerly), each preceded by an L2
flush outside the step's event pair: a 256 MB device write, then a read of the
same 256 MB, which evicts the write's dirty lines so that their write-back is
not charged to the step (the step starts on a cold, clean L2); every
step is timed with CUDA events on the launching stream, with nothing between
the scheduler and decode calls (the decode kernel starts, as a programmatic
dependent, while the scheduler finishes); the K timed steps are
bracketed by a barrier and a device synchronise on both sides; the reported
time is the maximum over ranks.  With N > 1 every rank runs the same workload
on its own GPU (independent replicas; the decode has no cross-GPU exchange).
After the timed steps, up to 200 more steps, replaying graphs of the two calls
with an event between them, give the scheduler's time and the decode call's
(decode kernel + split combine), which the roofline uses; there the decode
starts only after the scheduler has finished.

The line also carries `workloads`: every configuration (tiny, dsv3_decode,
varlen_h16, spec_causal, skewed_long) measured in the same run, bf16 cache,
default launch configuration: median / p10 / p90 of the step and of the decode
call over --sweep-reps graph replays, each after an L2 flush, with bytes, flops
and the roofline of each.  NVML clock samples cover the timed steps through
the end of that sweep (`clocks`); the timed steps' own are `clocks_timed_region`.

`--impl reference` times the fp64 CPU oracle on this host instead (bounded
samples of the same workload), printing the same JSON line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_paged_latent_decode_b200 import synth  # noqa: E402

METRIC = "MLA decode TB/s and TFLOPS on one B200 (bf16, paged KV), % of roofline"
UNIT = "TB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "mla_decode_pair_kernel_dsv3_decode_traffic.md")
CSRC = os.path.join(ROOT, "mla_paged_latent_decode_b200", "csrc")
# more than 64 query rows per sequence run on CTA pairs, fewer on single CTAs
PAIR_SRC = os.path.join(CSRC, "mla_decode_pair_sm100.cu")
SINGLE_SRC = os.path.join(CSRC, "mla_decode_sm100.cu")


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def decode_source(workload: str) -> str:
    w = synth.WORKLOADS[workload]
    return PAIR_SRC if w.s_q * w.h_q > 64 else SINGLE_SRC


def decode_source_sha(workload: str):
    with open(decode_source(workload), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken on the current decode kernel source and this workload; else None."""
    if workload != "dsv3_decode" or not os.path.exists(TRAFFIC_FILE):
        return None
    fields = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                fields[k.strip()] = v.strip()
    if fields.get("decode_kernel_source_sha256_16") != decode_source_sha(workload):
        return None
    try:
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = torch.cuda.get_device_properties(device_index).uuid
            self._nvml = pynvml
            self._handle = None
            for k in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(k)
                hu = pynvml.nvmlDeviceGetUUID(h)
                hu = hu.decode() if isinstance(hu, bytes) else hu
                if str(uuid) in hu or hu.endswith(str(uuid)):
                    self._handle = h
            if self._handle is None:
                self._handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._handle = None
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                mask = get(self._handle)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._handle is not None:
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._handle is not None:
            self._thread.join()

    def mark(self) -> int:
        """Number of samples taken so far (to tell the timed region's apart)."""
        return len(self.samples)

    def summary(self, first: int = 0, last: int | None = None):
        xs = self.samples[first:last]
        if not xs:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(xs), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(xs), "reasons": sorted(self.reasons), "samples": len(xs)}


def workload_config(inp, extra=None):
    w = inp.workload
    cfg = {"workload": f"{w.name}: {w.description}", "batch": inp.batch, "s_q": inp.s_q,
           "h_q": inp.h_q, "d_qk": 576, "dv": 512, "page": 64,
           "total_cached_tokens": int(inp.cache_seqlens.sum()), "causal": bool(inp.causal),
           "scale": inp.scale, "seed": inp.seed,
           "l2": "flushed before every timed step (outside its events) by a 256 MB device "
                 "write followed by a read of the same 256 MB, so the step starts on a cold L2 "
                 "holding no dirty lines",
           "timing": "each timed step replays a CUDA graph of the step (scheduler, decode and "
                     "combine kernels) captured after the warm-up; e2e runs eagerly through the "
                     "public API"}
    if extra:
        cfg.update(extra)
    return cfg


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(inp, target_s: float):
    """Pick a sample of the workload that the fp64 oracle finishes in about
    target_s: first more heads of one sequence, then more whole sequences.
    Returns (sample inputs, seconds of the last trial, description)."""
    import oracle
    b, h_q = inp.batch, inp.h_q
    n_seq, n_head = 1, 1
    while True:
        sub = subset(inp, n_seq, n_head)
        t0 = time.perf_counter()
        oracle.decode(sub.q, sub.kcache, sub.block_table, sub.cache_seqlens, sub.scale, sub.causal)
        dt = time.perf_counter() - t0
        done = n_seq >= b and n_head >= h_q
        if dt >= target_s or done:
            what = (f"{n_seq} of {b} sequences x {n_head} of {h_q} heads "
                    f"(all query positions), fp64 C oracle")
            return sub, dt, what
        grow = max(2.0, 0.9 * target_s / max(dt, 1e-4))
        if n_head < h_q:
            n_head = min(h_q, int(n_head * grow))
        else:
            n_seq = min(b, int(n_seq * grow))


def subset(inp, n_seq, n_head=None):
    """The first n_seq sequences (and first n_head heads) of a workload."""
    import copy
    sub = copy.copy(inp)
    n_head = inp.h_q if n_head is None else n_head
    sub.q = inp.q[:n_seq, :, :n_head].contiguous()
    sub.block_table = inp.block_table[:n_seq].contiguous()
    sub.cache_seqlens = inp.cache_seqlens[:n_seq].contiguous()
    return sub


def oracle_rate(sub, seconds):
    nbytes, flops = synth.algorithmic_work(sub)
    return nbytes / seconds / 1e12, flops / seconds / 1e12


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}; launch with torchrun")
    return rank, local, world


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_max(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def percentiles(xs):
    """(median, p10, p90) of a list of numbers."""
    ys = sorted(xs)
    n = len(ys)

    def at(f):
        k = min(n - 1, max(0, int(round(f * (n - 1)))))
        return ys[k]
    return statistics.median(ys), at(0.10), at(0.90)


def roofline_of(nbytes, flops, seconds, peaks):
    """The bound (whichever of bytes / HBM peak and flops / bf16 peak is longer)
    and the achieved rate against it for a call taking `seconds`."""
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        achieved, peak, unit, bound = nbytes / seconds / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    else:
        achieved, peak, unit, bound = flops / seconds / 1e12, peaks["bf16_tflops"], "TFLOP/s", \
            "tensor"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "bound_us": max(t_hbm, t_tc) * 1e6}


def measure_workload(name, dev, stream, flush_l2, reps, peaks):
    """Every configuration of the decode measured the same way as the headline
    one (bf16 cache, default launch configuration): `reps` graph replays of the
    whole step and of the decode call alone, each after an L2 flush."""
    from mla_paged_latent_decode_b200 import binding
    inp = synth.make_inputs(name, seed=0)
    nbytes, flops = synth.algorithmic_work(inp)
    q, kc = inp.q.to(dev), inp.kcache.to(dev)
    bt, sl = inp.block_table.to(dev), inp.cache_seqlens.to(dev)
    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    nw, _ = binding.metadata_shape(b, h_q, s_q)
    out = torch.empty((b, s_q, h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    ws = torch.empty((binding.workspace_size(b, s_q, h_q, nw),), dtype=torch.uint8, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)

    def call(md, ns):
        binding.mla_decode_kvcache(q, kc, bt, sl, 512, md, ns, inp.scale, inp.causal, out=out,
                                   lse=lse, workspace=ws, device_status=status)

    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(3):
            call(*binding.get_mla_metadata(sl, h_q, s_q, nw))
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    g_step, g_meta, g_call = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        call(*binding.get_mla_metadata(sl, h_q, s_q, nw))
    with torch.cuda.graph(g_meta):
        md_g, ns_g = binding.get_mla_metadata(sl, h_q, s_q, nw)
    with torch.cuda.graph(g_call):
        call(md_g, ns_g)
    for k in range(3):
        flush_l2(k)
        g_step.replay()
    torch.cuda.synchronize(dev)
    step_ev, call_ev = [], []
    for k in range(reps):
        flush_l2(k)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g_step.replay()
        e1.record(stream)
        step_ev.append((e0, e1))
    for k in range(reps):
        flush_l2(k)
        g_meta.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g_call.replay()
        e1.record(stream)
        call_ev.append((e0, e1))
    torch.cuda.synchronize(dev)
    del g_step, g_meta, g_call
    if int(status.item()) != 0:
        raise RuntimeError(f"{name}: device status {int(status.item())}")
    step_us = percentiles([a.elapsed_time(z) * 1e3 for a, z in step_ev])
    call_us = percentiles([a.elapsed_time(z) * 1e3 for a, z in call_ev])
    kernel = "pair" if s_q * h_q > 64 else "single-CTA"
    return {
        "workload": f"{name}: {inp.workload.description}", "kernel": kernel, "num_workers": nw,
        "bytes": nbytes, "flops": flops,
        "decode_call_us": call_us[0], "decode_call_us_p10": call_us[1],
        "decode_call_us_p90": call_us[2],
        "step_us": step_us[0], "step_us_p10": step_us[1], "step_us_p90": step_us[2],
        "tb_s_step": nbytes / (step_us[0] * 1e-6) / 1e12,
        "tflops_step": flops / (step_us[0] * 1e-6) / 1e12,
        "roofline": roofline_of(nbytes, flops, call_us[0] * 1e-6, peaks),
        "roofline_frac_step": roofline_of(nbytes, flops, step_us[0] * 1e-6, peaks)["frac"],
        "reps": reps,
    }


# ----------------------------------------------------------------------------- arms
def run_reference(args, rank, world):
    """The oracle arm: rank 0 only, on this host's cores."""
    if rank != 0:
        return None
    import oracle
    inp = synth.make_inputs(args.workload, seed=0)
    # size the per-step sample once so that all steps together take about two minutes
    per_step_target = max(0.01, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    sub, _, sample = oracle_sample(inp, per_step_target)
    threads = oracle.threads()
    for _ in range(args.warmup):
        oracle.decode(sub.q, sub.kcache, sub.block_table, sub.cache_seqlens, sub.scale, sub.causal)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode(sub.q, sub.kcache, sub.block_table, sub.cache_seqlens, sub.scale, sub.causal)
        times.append(time.perf_counter() - t0)
    nbytes, flops = synth.algorithmic_work(sub)
    total = sum(times)
    value = nbytes * args.steps / total / 1e12
    sample = f"per step: {sample}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 inputs widened exactly to fp64)",
        "config": workload_config(inp, {"sample": sample}),
        "tflops": flops * args.steps / total / 1e12,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def run_cuda(args, rank, local, world):
    from mla_paged_latent_decode_b200 import binding
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(args.workload, seed=0)
    fp8 = args.kv == "fp8"
    sparse_idx = None
    if args.sparse_topk:
        if fp8:
            raise SystemExit("--sparse-topk runs on the bf16 cache")
        sparse_idx = synth.make_sparse_indices(inp, args.sparse_topk, seed=0)
        nbytes, flops = synth.sparse_algorithmic_work(inp, sparse_idx)
    else:
        nbytes, flops = synth.algorithmic_work(inp, 580 if fp8 else 1152)
    q = inp.q.to(dev)
    kc = inp.kcache.to(dev)
    bt = inp.block_table.to(dev)
    sl = inp.cache_seqlens.to(dev)
    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    num_workers, _ = binding.metadata_shape(b, h_q, s_q)
    kc8 = ks = None
    if fp8:
        kc8, ks = encode_cache_fp8(kc, dev)
        del kc
        kc = None
    out = torch.empty((b, s_q, h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
    ws = torch.empty((binding.workspace_size(b, s_q, h_q, num_workers),), dtype=torch.uint8,
                     device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    if sparse_idx is not None:
        idx_d = sparse_idx.to(dev)
        sp_workers, _ = binding.metadata_shape(b * s_q, h_q, 1)
        sp_ws = torch.empty((binding.lib.mla_sparse_workspace_size(b, s_q, h_q, sparse_idx.shape[2],
                                                                   sp_workers),),
                            dtype=torch.uint8, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    flush_max = torch.empty((), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2(k):
        # The write replaces every line of L2; the read that follows evicts the
        # write's dirty lines (their write-back happens here, not in the step).
        flush.fill_(k & 0xFF)
        torch.amax(flush.view(torch.int32), dim=0, out=flush_max)

    def metadata():
        if sparse_idx is not None:  # the sparse call runs its own scheduler
            return None, None
        return binding.get_mla_metadata(sl, h_q, s_q, num_workers)

    def decode_call(md, ns):
        if sparse_idx is not None:
            binding.mla_decode_sparse(q, kc, bt, sl, idx_d, inp.scale, inp.causal, out=out, lse=lse,
                                      workspace=sp_ws, device_status=status)
        elif fp8:
            binding.mla_decode_kvcache_fp8(q, kc8, ks, bt, sl, 512, md, ns, inp.scale, inp.causal,
                                           out=out, lse=lse, workspace=ws, device_status=status)
        else:
            binding.mla_decode_kvcache(q, kc, bt, sl, 512, md, ns, inp.scale, inp.causal, out=out,
                                       lse=lse, workspace=ws, device_status=status)

    def step():
        # nothing between the two calls: the decode kernel is a programmatic
        # dependent of the scheduler kernel and starts while it finishes
        decode_call(*metadata())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")

    # The timed steps replay CUDA graphs of the calls (captured once, after the
    # warm-up), as a serving loop would: the same three kernels per step, with
    # no host work (argument checks, tensor-map encoding, launches) inside the
    # events.  g_step is the whole step; g_meta and g_call are the two calls
    # captured apart, for the split below.
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(3):
            step()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    g_step, g_meta, g_call = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    if sparse_idx is None:
        with torch.cuda.graph(g_meta):
            md_g, ns_g = metadata()
    else:  # the sparse call runs its own scheduler: nothing to capture apart
        md_g, ns_g = None, None
    with torch.cuda.graph(g_call):
        decode_call(md_g, ns_g)
    for k in range(3):
        flush_l2(k)
        g_step.replay()
    torch.cuda.synchronize(dev)

    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    # NVML samples from here to the end of the per-workload sweep; the timed
    # region's own samples are reported apart
    clocks = ClockSampler(local).__enter__()
    t_wall0 = time.perf_counter()
    for k in range(args.steps):
        flush_l2(k)
        e0, e1 = events[k]
        e0.record(stream)
        g_step.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter() - t_wall0
    timed_samples = clocks.mark()
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    step_ms = [e0.elapsed_time(e1) for e0, e1 in events]
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during timing")

    # The two calls timed apart (an event between them, so here the decode kernel
    # starts only once the scheduler has finished): the scheduler's time, and the
    # decode call's (decode kernel + split combine) for the roofline.
    n_split = max(3, min(args.steps, 200))
    split_events = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
                    for _ in range(n_split)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    for k in range(n_split):
        flush_l2(k)
        e0, em, e1 = split_events[k]
        e0.record(stream)
        if sparse_idx is None:
            g_meta.replay()
        em.record(stream)
        g_call.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    del g_step, g_meta, g_call
    decode_ms = [m.elapsed_time(e1) for _, m, e1 in split_events]
    meta_ms = [e0.elapsed_time(m) for e0, m, _ in split_events]
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during timing")

    total_s = reduce_max(sum(step_ms) / 1e3, world, dev)
    all_bytes = reduce_sum(float(nbytes * args.steps), world, dev)
    all_flops = reduce_sum(float(flops * args.steps), world, dev)
    decode_avg_s = reduce_max(sum(decode_ms) / len(decode_ms) / 1e3, world, dev)

    # end to end through the public API, as a serving loop runs it: every step
    # copies its inputs in from pinned host memory and its outputs back, all
    # inside the timed region.  Three streams (copies in, compute, copies out)
    # and several sets of step buffers (--e2e-sets) let step k + 1's inputs
    # travel while step k computes and step k - 1's outputs travel back; the
    # latent cache (larger than L2) stays resident in HBM, as in serving.
    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, min(args.steps, 200))
        hq = inp.q.pin_memory()
        hbt = inp.block_table.pin_memory()
        hsl = inp.cache_seqlens.pin_memory()
        hidx = sparse_idx.pin_memory() if sparse_idx is not None else None
        sets = []
        n_sets = max(2, args.e2e_sets)
        for _ in range(n_sets):
            sets.append(dict(
                q=torch.empty_like(q), bt=torch.empty_like(bt), sl=torch.empty_like(sl),
                idx=torch.empty_like(idx_d) if sparse_idx is not None else None,
                out=torch.empty_like(out), lse=torch.empty_like(lse),
                hout=torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                hlse=torch.empty(lse.shape, dtype=lse.dtype).pin_memory()))
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

        host_enqueue_s = [0.0]

        def run_e2e(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_cmp = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for st in (s_in, s_cmp, s_out):
                st.wait_stream(stream)
            t0.record(s_in)
            h0 = time.perf_counter()
            for k in range(n):
                b = sets[k % n_sets]
                with torch.cuda.stream(s_in):
                    if k >= n_sets:  # the set's previous step has finished reading its inputs
                        s_in.wait_event(ev_cmp[k - n_sets])
                    b["q"].copy_(hq, non_blocking=True)
                    b["bt"].copy_(hbt, non_blocking=True)
                    b["sl"].copy_(hsl, non_blocking=True)
                    if hidx is not None:
                        b["idx"].copy_(hidx, non_blocking=True)
                    ev_in[k].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[k])
                    if k >= n_sets:  # the set's previous outputs have been copied out
                        s_cmp.wait_event(ev_out[k - n_sets])
                    if hidx is not None:
                        binding.mla_decode_sparse(b["q"], kc, b["bt"], b["sl"], b["idx"], inp.scale,
                                                  inp.causal, out=b["out"], lse=b["lse"],
                                                  workspace=sp_ws)
                    else:
                        md, ns = binding.get_mla_metadata(b["sl"], h_q, s_q, num_workers)
                        if fp8:
                            binding.mla_decode_kvcache_fp8(b["q"], kc8, ks, b["bt"], b["sl"], 512, md,
                                                           ns, inp.scale, inp.causal, out=b["out"],
                                                           lse=b["lse"], workspace=ws)
                        else:
                            binding.mla_decode_kvcache(b["q"], kc, b["bt"], b["sl"], 512, md, ns,
                                                       inp.scale, inp.causal, out=b["out"],
                                                       lse=b["lse"], workspace=ws)
                    ev_cmp[k].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[k])
                    b["hout"].copy_(b["out"], non_blocking=True)
                    b["hlse"].copy_(b["lse"], non_blocking=True)
                    ev_out[k].record(s_out)
            host_enqueue_s[0] = time.perf_counter() - h0  # the host's work for the n steps
            s_out.wait_stream(s_in)
            s_out.wait_stream(s_cmp)
            t1.record(s_out)
            torch.cuda.synchronize(dev)
            return t0.elapsed_time(t1) / 1e3

        run_e2e(3)  # warm-up
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        e2e_total = reduce_max(run_e2e(n_e2e), world, dev)
        e2e_bytes = reduce_sum(float(nbytes * n_e2e), world, dev)
        # the last step's outputs arrived intact
        if not torch.equal(sets[(n_e2e - 1) % n_sets]["hout"], out.cpu()):
            raise RuntimeError("end-to-end output differs from the device-timed output")
        h2d = hq.numel() * hq.element_size() + hbt.numel() * 4 + hsl.numel() * 4
        if sparse_idx is not None:
            h2d += sparse_idx.numel() * 4
        d2h = out.numel() * out.element_size() + lse.numel() * 4
        # the host link on its own: the step's input copy and output copy, each
        # alone and both at once (one per direction), best of five
        def link_us(copy_in, copy_out):
            best = float("inf")
            for _ in range(5):
                for st in (s_in, s_out):
                    st.wait_stream(stream)
                a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(s_in)
                s_out.wait_event(a)
                if copy_in:
                    with torch.cuda.stream(s_in):
                        sets[0]["q"].copy_(hq, non_blocking=True)
                if copy_out:
                    with torch.cuda.stream(s_out):
                        sets[0]["hout"].copy_(sets[0]["out"], non_blocking=True)
                s_in.wait_stream(s_out)
                z.record(s_in)
                torch.cuda.synchronize(dev)
                best = min(best, a.elapsed_time(z) * 1e3)
            return best
        h2d_us, d2h_us, both_us = link_us(True, False), link_us(False, True), link_us(True, True)
        e2e = {"value": e2e_bytes / e2e_total / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "us_per_step": e2e_total / n_e2e * 1e6, "buffer_sets": n_sets,
               "host_enqueue_us_per_step": host_enqueue_s[0] / n_e2e * 1e6,
               "link": {"q_in_us": h2d_us, "out_back_us": d2h_us, "both_us": both_us,
                        "h2d_gb_s": hq.numel() * hq.element_size() / h2d_us / 1e3,
                        "d2h_gb_s": out.numel() * out.element_size() / d2h_us / 1e3},
               "note": "through the public API: q, block_table and cache_seqlens copied in from "
                       "pinned host memory and out and lse copied back every step; copies in, "
                       f"compute and copies out on three streams with {n_sets} buffer sets, so "
                       "consecutive steps overlap; the latent cache stays resident in HBM as "
                       "in serving; link: the q copy in and the out copy back timed alone and "
                       "together"}

    append = None if args.no_append else measure_append(inp, dev, stream, flush_l2, fp8=fp8)

    peaks, peak_kind = load_peaks()
    workloads = None
    if not (args.no_workloads or fp8 or sparse_idx is not None):
        # every configuration, bf16 cache, from the same run (the headline one included)
        workloads = {}
        for name in synth.WORKLOADS:
            workloads[name] = measure_workload(name, dev, stream, flush_l2, args.sweep_reps, peaks)
            torch.cuda.empty_cache()
    clocks.__exit__(None, None, None)

    if rank != 0:
        return None
    ms_per_step = total_s / args.steps * 1e3
    value = all_bytes / total_s / 1e12
    tflops = all_flops / total_s / 1e12
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    rl = roofline_of(nbytes, flops, decode_avg_s, peaks)
    bound, achieved, peak, unit = rl["bound"], rl["achieved"], rl["peak"], rl["unit"]
    step_p = percentiles(step_ms)
    call_p = percentiles(decode_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q and latent cache, shuffled 64-token pages)",
        "config": workload_config(inp, {"parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                                        "num_workers": num_workers,
                                        "sparse_topk": args.sparse_topk or None,
                                        "kv_cache": ("fp8: E4M3 codes + one power-of-two fp32 scale "
                                                     "per token (580 B per token)") if fp8 else
                                                    "bf16 (1152 B per token)"}),
        "tflops": tflops,
        "roofline_frac": max(t_hbm, t_tc) / (ms_per_step / 1e3),
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "traffic": None if (fp8 or sparse_idx is not None)
                     else recorded_traffic(args.workload),
                     "kernel": "mla_decode_kvcache call (decode kernel + split combine)",
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s / 1.59 PFLOP/s"},
        "kernel_us": {"metadata": statistics.median(meta_ms) * 1e3,
                      "decode_call": call_p[0] * 1e3, "decode_call_p10": call_p[1] * 1e3,
                      "decode_call_p90": call_p[2] * 1e3,
                      "step": step_p[0] * 1e3, "step_p10": step_p[1] * 1e3,
                      "step_p90": step_p[2] * 1e3},
        "gpu_launches": ((5 + (s_q > 1)) if sparse_idx is not None else 3) * args.steps,
        "clocks": dict(clocks.summary(), window=(
            "NVML samples every 5 ms from the first timed step to the end of the per-workload "
            "sweep (graph replays of the same kernels); the timed region's own samples are in "
            "clocks_timed_region")),
        "clocks_timed_region": clocks.summary(0, timed_samples),
        "wall_s_timed_region": t_wall,
    }
    if workloads is not None:
        line["workloads"] = workloads
    if e2e is not None:
        line["e2e"] = e2e
    if append is not None:
        for case in append.values():
            case["frac_of_hbm_peak"] = case["gb_s"] / peaks["hbm_gbs"]
        line["append"] = append
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        sub, dt, what = oracle_sample(inp, args.cpu_seconds)
        tbs, tfl = oracle_rate(sub, dt)
        line["cpu_baseline"] = {
            "value": tbs, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{what}, {dt:.1f} s", "tflops": tfl}
    return line


def encode_cache_fp8(kc, dev):
    """The FP8 cache of a bf16 cache, written by the library's own quantising
    append: every page is one 64-token "sequence" appended into an empty
    block-table row, with the free stack ordered so that sequence p receives
    page p."""
    from mla_paged_latent_decode_b200 import binding
    nblk = kc.shape[0]
    kc8 = torch.empty((nblk, 64, 576), dtype=torch.uint8, device=dev)
    ks = torch.empty((nblk, 64), dtype=torch.float32, device=dev)
    bt = torch.zeros((nblk, 1), dtype=torch.int32, device=dev)
    lens = torch.zeros((nblk,), dtype=torch.int32, device=dev)
    free = torch.arange(nblk - 1, -1, -1, dtype=torch.int32, device=dev)
    fc = torch.tensor([nblk], dtype=torch.int32, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    for p0 in range(0, nblk, 65536):  # at most 65536 sequences per call
        n = min(65536, nblk - p0)
        binding.append_latent_fp8(kc[p0:p0 + n], kc8, ks, bt[p0:p0 + n], lens[p0:p0 + n], free,
                                  fc, status)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0 or int(fc.item()) != 0:
        raise RuntimeError("building the FP8 cache failed")
    if not torch.equal(bt[:, 0], torch.arange(nblk, dtype=torch.int32, device=dev)):
        raise RuntimeError("FP8 cache pages out of order")
    return kc8, ks


def measure_append(inp, dev, stream, flush_l2, calls=50, fp8=False):
    """Time mla_append_latent (the latent-cache append with page allocation) on
    the workload's batch: every sequence sits at a page boundary, so every call
    takes one new page per sequence (the costliest decode step), for s_new = s_q
    (one decode step) and for s_new = 1024 (a chunk, large enough to show the
    copy's bandwidth).  Each call replays a CUDA graph of the append after the
    cache state has been restored and L2 flushed, outside its events.
    Algorithmic bytes: the new rows read and written (1152 B each), plus 16 B
    per sequence of lengths, block-table entries and popped free-stack slots."""
    from mla_paged_latent_decode_b200 import binding
    b = inp.batch
    res = {}
    for name, s_new in (("decode_step", inp.s_q), ("chunk_1024", 1024)):
        new_pages = -(-s_new // 64)
        pool = b * (1 + new_pages)
        gen = torch.Generator().manual_seed(1)
        kc = torch.randn((pool, 64, 576), generator=gen).to(torch.bfloat16).to(dev)
        kc8 = torch.zeros((pool, 64, 576), dtype=torch.uint8, device=dev) if fp8 else None
        ks = torch.zeros((pool, 64), dtype=torch.float32, device=dev) if fp8 else None
        rows = torch.randn((b, s_new, 576), generator=gen).to(torch.bfloat16).to(dev)
        perm = torch.randperm(pool, generator=gen).to(torch.int32)
        bt0 = torch.zeros((b, 1 + new_pages), dtype=torch.int32)
        bt0[:, 0] = perm[:b]
        free0 = perm[b:].contiguous()
        bt0, free0 = bt0.to(dev), free0.to(dev)
        sl0 = torch.full((b,), 64, dtype=torch.int32, device=dev)
        fc0 = torch.tensor([pool - b], dtype=torch.int32, device=dev)
        bt, sl, free, fc = bt0.clone(), sl0.clone(), free0.clone(), fc0.clone()
        status = torch.zeros((1,), dtype=torch.int32, device=dev)

        def restore():
            bt.copy_(bt0)
            sl.copy_(sl0)
            fc.copy_(fc0)

        def call():
            if fp8:
                binding.append_latent_fp8(rows, kc8, ks, bt, sl, free, fc, status)
            else:
                binding.append_latent(rows, kc, bt, sl, free, fc, status)

        for _ in range(3):
            restore()
            call()
        torch.cuda.synchronize(dev)
        if int(status.item()) != 0 or int(fc.item()) != 0 or int(sl[0].item()) != 64 + s_new:
            raise RuntimeError(f"append check failed: status {int(status.item())}")
        graph = torch.cuda.CUDAGraph()
        restore()
        with torch.cuda.graph(graph):
            call()
        evs = []
        for k in range(calls):
            restore()
            flush_l2(k)
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            z.record(stream)
            evs.append((a, z))
        torch.cuda.synchronize(dev)
        del graph
        us = statistics.median(a.elapsed_time(z) for a, z in evs) * 1e3
        nbytes = b * s_new * (1152 + (580 if fp8 else 1152)) + 16 * b
        res[name] = {"s_new": s_new, "batch": b, "us": us, "bytes": nbytes,
                     "gb_s": nbytes / (us * 1e-6) / 1e9, "launches": 2,
                     "note": "every sequence takes a new page; L2 flushed before each call"}
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default=None, choices=sorted(synth.WORKLOADS),
                    help="default: dsv3_decode (bf16 cache) or varlen_h16 (fp8 cache)")
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="latent cache format (fp8: E4M3 codes + per-token scale)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end measurement")
    ap.add_argument("--e2e-sets", type=int, default=4,
                    help="step buffer sets of the end-to-end loop (copies of consecutive steps "
                         "overlap across them)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the oracle")
    ap.add_argument("--sparse-topk", type=int, default=0,
                    help="time the sparse decode with this many selected tokens per query "
                         "position (seeded uniform picks; bf16 cache)")
    ap.add_argument("--no-append", action="store_true",
                    help="skip timing the latent-cache append")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the sweep over every configuration")
    ap.add_argument("--sweep-reps", type=int, default=100,
                    help="graph replays per configuration in the sweep (each after an L2 flush)")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="approximate oracle time for the cpu_baseline sample")
    args = ap.parse_args()
    if args.workload is None:
        args.workload = "varlen_h16" if args.kv == "fp8" else "dsv3_decode"
    if args.warmup < 3 and args.impl == "cuda":
        raise SystemExit("--warmup must be at least 3")
    rank, local, world = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_cuda(args, rank, local, world)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
