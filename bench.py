#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200 (one JSON line on rank 0).

A step is one pass of the hot path over one batch of synthetic input:
  * prefill: one attn_fwd call on the headline workload, by default the MHA
    causal prefill at the page-1 shape (B=4, Hq=Hkv=32, N=8192, d=128, bf16
    in/out, fp32 LSE) — the headline `value`, in mask-adjusted TFLOP/s;
  * the two other prefill workloads as their own legs ("prefill_legs"): MHA
    causal N=2048 and GQA sliding window N=32768 (Hq=32, Hkv=8,
    window_left=4096), each with its own roofline;
  * decode: one attn_decode call (split + combine kernels) on the GQA decode
    workload (B=64, L=8192, Hq=32, Hkv=8, d=128), reported under "decode" in
    KV-read GB/s;
  * the later rows (backward, merge, packed prefill, paged decode) as legs.
Each leg is timed over the same number of steps; mean, median and min are
reported (the headline value uses the mean: total time over K steps).

Timing: W untimed warm-up steps, then K steps; each kernel is bracketed by
CUDA events on the launching stream, preceded by an L2 flush (256 MiB
memset) and a short device-side sleep so the events measure the kernel
alone. Barrier + synchronize on both sides; the max over ranks is reported.
With N > 1 every rank runs its own independent batch (no collective in the
data path): weak scaling.

`--impl reference` times the fp64 CPU oracle instead (the only other
implementation of this path): each step is one block of 512 query rows of one
(batch, head) of the headline workload.
"""

from __future__ import annotations

import argparse
import dataclasses
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

import torch  # noqa: E402

import attn_inputs as ai  # noqa: E402
from exact_softmax_attention_03_b200 import metrics  # noqa: E402

METRIC = "attn fwd TFLOP/s (mask-adjusted) & % bf16 peak; decode KV-read GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "attn_fwd_kernel": ["exact_softmax_attention_03_b200/csrc/" + f
                        for f in ("sm100_ptx.cuh", "prefill_kernel.cuh")],
    "decode": ["exact_softmax_attention_03_b200/csrc/" + f
               for f in ("sm100_ptx.cuh", "decode_kernels.cuh")],
    "decode_paged": ["exact_softmax_attention_03_b200/csrc/" + f
                     for f in ("sm100_ptx.cuh", "decode_kernels.cuh")],
    "bwd_main_kernel": ["exact_softmax_attention_03_b200/csrc/" + f
                        for f in ("sm100_ptx.cuh", "backward_kernels.cuh")],
    "merge": ["exact_softmax_attention_03_b200/csrc/" + f
              for f in ("sm100_ptx.cuh", "merge_kernel.cuh")],
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["mha2k", "mha8k", "gqa32k"], default="mha8k",
                    help="headline prefill workload (default: MHA causal N=8192, the page-1 shape)")
    ap.add_argument("--only-headline", action="store_true",
                    help="skip the other prefill workloads' legs")
    ap.add_argument("--decode-splits", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the prefill batch (profiling a smaller case only)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="override the decode batch (profiling a smaller case only)")
    ap.add_argument("--page-size", type=int, default=16,
                    help="keys per page in the paged-cache decode leg (16, 32, 64 or k*128)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


PREFILL = {"mha2k": ai.MHA_2K, "mha8k": ai.MHA_8K, "gqa32k": ai.GQA_SWA_32K}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    """Short hash of the device sources of one kernel family."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, resized: bool = False):
    """DRAM bytes per launch from a committed ncu summary, if taken on these sources.

    The recorded figures are per launch of the full workload: none is reported
    when the run overrides the workload's batch (``resized``).
    """
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if resized or not os.path.exists(path):
        return None
    want = kernel_source_hash(kernel)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel \
                    and parts[1] == workload and parts[3] == want:
                return float(parts[2])
    return None


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML, only while a timed
    region is open (``timed_kernel_loop`` opens one per leg): the median is the
    clock under load, per leg and over all legs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []                         # (leg label, MHz)
        self.label = None                         # open timed region, or None
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:                         # NVML unavailable: report nothing
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            label = self.label
            if label is not None:
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((label, mhz))
                    self.reasons |= int(r) & ~0x1
                except Exception:
                    pass
            time.sleep(self.period)

    def open(self, label):
        self.label = label

    def close(self):
        self.label = None

    def start(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        legs = {}
        for label, mhz in self.samples:
            legs.setdefault(label, []).append(mhz)
        return {"sm_mhz": statistics.median(m for _, m in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b],
                "samples": len(self.samples),
                "sm_mhz_per_leg": {k: statistics.median(v) for k, v in legs.items()},
                "scope": "timed regions only"}


SAMPLER = None          # the run's ClockSampler (timed_kernel_loop opens and closes it)


# -------------------------------------------------------------- dist setup --

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def shard_seed(rank: int) -> int:
    """Each rank draws its own batch: independent shards, no data exchanged."""
    return ai.SEED_Q + 17 * rank


def whole_job_rate(units_per_rank: float, ms_max: float, world: int) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


# ------------------------------------------------------------------ timing --

def timed_kernel_loop(fn, steps, warmup, world, flush=None, label="leg"):
    """Per-step CUDA-event times (ms) of fn() on the current stream; returns
    (times, launches of this library inside the timed region)."""
    import exact_softmax_attention_03_b200 as ea
    for _ in range(warmup):
        if flush is not None:
            flush()
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    n0 = ea.attn_launch_count()
    if SAMPLER is not None:
        SAMPLER.open(label)
    for s, e in ev:
        if flush is not None:
            flush()
        torch.cuda._sleep(100_000)              # hold the stream while the launch is queued
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    if SAMPLER is not None:
        SAMPLER.close()
    n1 = ea.attn_launch_count()
    barrier(world)
    status = ea.attn_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}: {ea.attn_last_error()}")
    return [s.elapsed_time(e) for s, e in ev], n1 - n0


def time_stats(times):
    """mean / median / min of per-step times (ms)."""
    return {"mean": statistics.mean(times), "median": statistics.median(times), "min": min(times)}


def e2e_loop(step_fn, steps, warmup):
    """Event-timed region per step including host<->device copies; ms/step."""
    for _ in range(warmup):
        step_fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        step_fn()
        e.record()
        e.synchronize()
        times.append(s.elapsed_time(e))
    return statistics.mean(times)


def e2e_pipelined(step_in, step_fwd, step_out, steps, warmup):
    """ms per step of K steps, each an H2D copy of the step's inputs, the kernel and
    a D2H copy of its outputs, on three streams with two device buffer sets: step
    k's D2H and step k + 1's H2D overlap with the kernels (PCIe carries both
    directions at once). Every step's copies run in full; the region is timed with
    CUDA events from the first H2D to the last D2H."""
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    started = [False, False]

    def step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(cmp_done[b])           # the kernel of step i - 2 read buffer b
            step_in(b)
            in_ready[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_ready[b])
            if started[b]:
                s_cmp.wait_event(out_done[b])          # step i - 2's outputs left buffer b
            step_fwd(b, s_cmp)
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            step_out(b)
            out_done[b].record(s_out)
        started[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(warmup, warmup + steps):
        step(i)
    t1.record(s_out)
    t1.synchronize()
    return t0.elapsed_time(t1) / steps


# ------------------------------------------------------------ cpu baseline --

def blas_info():
    """(threads, vendor string) of the BLAS NumPy calls into."""
    try:
        from threadpoolctl import threadpool_info
        infos = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if infos:
            i = max(infos, key=lambda x: x.get("num_threads", 0))
            vendor = f"{i.get('internal_api', '?')} {i.get('version', '')}".strip()
            return int(i.get("num_threads", 1)), vendor
    except Exception:
        pass
    return os.cpu_count() or 1, "unknown"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


ROW_BLOCK = 512


def oracle_row_blocks(w):
    """The sample unit of the CPU legs: (b, head, first row) of 512-row blocks,
    spread over the rows so that short and long causal rows both appear."""
    blocks = list(range(0, w.Nq, ROW_BLOCK))
    order = blocks[::-2] + blocks[-2::-2]                   # longest and shortest rows mixed
    return [(b, h, r0) for b in range(w.B) for h in range(w.Hq) for r0 in order]


def oracle_block(w, q, k, v, b, hq, r0):
    """One oracle call on rows [r0, r0 + 512) of one (batch, head); its FLOPs.

    The oracle is handed that head's slices only (it upcasts what it is given)."""
    import oracle
    rows = list(range(r0, min(r0 + ROW_BLOCK, w.Nq)))
    hk = hq // (w.Hq // w.Hkv)
    oracle.oracle_attention_rows(q[b:b + 1, :, hq:hq + 1], k[b:b + 1, :, hk:hk + 1],
                                 v[b:b + 1, :, hk:hk + 1], 0, 0, rows, causal=w.causal,
                                 window_left=w.window_left)
    per_row = metrics.allowed_pairs_per_row(w.Nq, w.Nk, w.causal, w.window_left)
    return 4.0 * w.d * float(per_row[rows[0]:rows[-1] + 1].sum())


def cpu_baseline_block(w, q, k, v, budget_s):
    """The fp64 oracle timed on 512-row blocks of the workload for ~budget_s."""
    units = oracle_row_blocks(w)
    flops, n = 0.0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and n < len(units):
        flops += oracle_block(w, q, k, v, *units[n])
        n += 1
    dt = time.perf_counter() - t0
    threads, vendor = blas_info()
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 NumPy oracle on {n} blocks of {ROW_BLOCK} query rows of "
                      f"'{w.name}' ({dt:.1f} s of CPU work), same mask-adjusted FLOP count",
            "host_cpus": os.cpu_count(), "cpu_model": cpu_model(), "blas": vendor}


# --------------------------------------------------------------- reference --

def run_reference(args, world, rank):
    if rank != 0:
        return
    w = PREFILL[args.workload]
    q, k, v = ai.make_for(w)
    units = oracle_row_blocks(w)
    for i in range(args.warmup):
        oracle_block(w, q, k, v, *units[i % len(units)])
    flops = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        flops += oracle_block(w, q, k, v, *units[(args.warmup + i) % len(units)])
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    threads, vendor = blas_info()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.Nq,
                   "d": w.d, "causal": w.causal, "window_left": w.window_left,
                   "step": f"one block of {ROW_BLOCK} query rows of one (batch, head)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{args.steps} blocks of {ROW_BLOCK} query rows, fp64 NumPy "
                                   f"oracle, mask-adjusted FLOPs",
                         "host_cpus": os.cpu_count(), "cpu_model": cpu_model(), "blas": vendor},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- ours --

def tensor_roofline(achieved, peaks, peak_src, kernel, traffic, alg_bytes=None):
    peak_t = peaks["bf16_tflops"]
    r = {"bound": "tensor", "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
         "frac": achieved / peak_t, "peak_source": f"{peak_src} bf16_tflops (burst)",
         "kernel": kernel, "traffic": traffic}
    if "bf16_tflops_sustained" in peaks:
        # the timed loop runs the kernel back to back, where the SM clock settles
        # below its burst value under the power cap: the sustained GEMM figure,
        # measured the same way, is the like-for-like denominator
        r["peak_sustained"] = peaks["bf16_tflops_sustained"]
        r["frac_sustained"] = achieved / peaks["bf16_tflops_sustained"]
    if alg_bytes is not None:
        r["algorithmic_bytes"] = alg_bytes
    return r


def hbm_roofline(achieved, peaks, peak_src, kernel, traffic, alg_bytes):
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs",
            "kernel": kernel, "algorithmic_bytes": alg_bytes, "traffic": traffic}


def prefill_leg(ea, key, w, args, world, rank, dev, flush, peaks, peak_src, resized=False):
    """Time attn_fwd on one prefill workload; returns (leg dict, device tensors)."""
    q_h, k_h, v_h = ai.make_for(w, seed=shard_seed(rank))
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty((w.B, w.Nq, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)

    def fwd():
        ea.attn_fwd(q, k, v, o=o, lse=lse, causal=w.causal, window_left=w.window_left)

    times, launches = timed_kernel_loop(fwd, args.steps, args.warmup, world, flush, label=key)
    st = time_stats(times)
    ms_max = max_over_ranks(st["mean"], world)
    flops = metrics.attn_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.causal, w.window_left)
    tiles = metrics.executed_tiles(w.Nq, w.Nk, w.causal, w.window_left) * w.B * w.Hq
    leg = {
        "workload": w.name, "key": key,
        "config": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.Nq, "d": w.d,
                   "causal": w.causal, "window_left": w.window_left},
        "value": whole_job_rate(flops, ms_max, world) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": ms_max, "ms": st,
        "flops_per_step": flops,
        "tflops_at_median": flops / (st["median"] * 1e-3) / 1e12,
        "tile_tflops": tiles * 4.0 * 128 * 128 * w.d / (st["mean"] * 1e-3) / 1e12,
        "roofline": tensor_roofline(flops / (st["mean"] * 1e-3) / 1e12, peaks, peak_src,
                                    "attn_fwd_kernel<128,false>",
                                    recorded_traffic("attn_fwd_kernel", key, resized),
                                    metrics.attn_fwd_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)),
        "gpu_launches": launches,
    }
    leg["pct_bf16_peak"] = 100.0 * leg["roofline"]["frac"]
    return leg, (q_h, k_h, v_h, q, k, v, o, lse)


def run_ours(args, world, rank, local):
    import exact_softmax_attention_03_b200 as ea
    from exact_softmax_attention_03_b200 import build
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    global SAMPLER
    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    SAMPLER = sampler
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    resized = bool(args.batch)
    w = PREFILL[args.workload]
    if args.batch:
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name} [batch {args.batch}]")

    sampler.start()
    # ---- headline prefill
    head, (q_h, k_h, v_h, q, k, v, o, lse) = prefill_leg(
        ea, args.workload, w, args, world, rank, dev, flush, peaks, peak_src, resized)
    launches = head["gpu_launches"]

    # ---- the other prefill workloads, each its own leg
    legs = []
    if not args.only_headline:
        for key in ("mha2k", "mha8k", "gqa32k"):
            if key == args.workload:
                continue
            wl = PREFILL[key]
            if args.batch and wl.B > 1:
                wl = dataclasses.replace(wl, B=min(wl.B, args.batch),
                                         name=f"{wl.name} [batch {min(wl.B, args.batch)}]")
            leg, tensors = prefill_leg(ea, key, wl, args, world, rank, dev, flush, peaks,
                                       peak_src, resized)
            legs.append(leg)
            del tensors

    # ---- backward on the headline workload: dQ, dK, dV from the forward's O and
    # LSE (2.5x the forward's mask-adjusted FLOPs: five products instead of two)
    flops = head["flops_per_step"]
    do_h = ai.make_dout(w.B, w.Nq, w.Hq, w.d, seed=shard_seed(rank) + 21)
    dout = do_h.to(dev)
    ea.attn_fwd(q, k, v, o=o, lse=lse, causal=w.causal, window_left=w.window_left)
    dq_t, dk_t, dv_t = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bws = torch.empty(ea.attn_bwd_workspace_bytes(w.B, w.Hq, w.Nq, w.d), dtype=torch.uint8,
                      device=dev)

    def bwd():
        ea.attn_bwd(q, k, v, o, lse, dout, causal=w.causal, window_left=w.window_left,
                    dq=dq_t, dk=dk_t, dv=dv_t, workspace=bws)

    btimes, blaunches = timed_kernel_loop(bwd, args.steps, args.warmup, world, flush, label="backward")
    bst = time_stats(btimes)
    bms_max = max_over_ranks(bst["mean"], world)
    b_flops = 2.5 * flops
    backward = {
        "workload": f"{w.name}, backward (dQ, dK, dV)",
        "value": whole_job_rate(b_flops, bms_max, world) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": bms_max, "ms": bst,
        "flop_count": "2.5 x the forward's mask-adjusted FLOPs",
        "roofline": dict(tensor_roofline(b_flops / (bst["mean"] * 1e-3) / 1e12, peaks, peak_src,
                                         "bwd_prep_kernel + bwd_main_kernel<128> + bwd_finalize_kernel",
                                         recorded_traffic("bwd_main_kernel", args.workload, resized)),
                         traffic_kernel="bwd_main_kernel<128>"),
        "gpu_launches": blaunches,
    }
    del dout, dq_t, dk_t, dv_t, bws

    # ---- merge leg (sequence-sharded attention's combine): 4 fp32 parts of the
    # MHA N=2048 output shape -> bf16 O and LSE; HBM-bound, inputs far above L2
    mw = ai.MHA_2K
    R_m = 4
    g_m = torch.Generator(device="cpu")
    g_m.manual_seed(shard_seed(rank) + 31)
    mo_parts = torch.randn((R_m, mw.B, mw.Nq, mw.Hq, mw.d), generator=g_m).to(dev)
    ml_parts = torch.randn((R_m, mw.B, mw.Hq, mw.Nq), generator=g_m).to(dev)
    m_out = torch.empty((mw.B, mw.Nq, mw.Hq, mw.d), dtype=torch.bfloat16, device=dev)
    m_lse = torch.empty((mw.B, mw.Hq, mw.Nq), dtype=torch.float32, device=dev)

    def merge():
        ea.attn_merge(mo_parts, ml_parts, o=m_out, lse=m_lse)

    mtimes, mlaunches = timed_kernel_loop(merge, args.steps, args.warmup, world, None, label="merge")
    mst = time_stats(mtimes)
    mms_max = max_over_ranks(mst["mean"], world)
    m_rows = mw.B * mw.Nq * mw.Hq
    m_bytes = R_m * m_rows * (mw.d + 1) * 4 + m_rows * (mw.d * 2 + 4)
    merge_leg = {
        "workload": f"merge of {R_m} fp32 parts, {mw.name} output shape",
        "value": whole_job_rate(m_bytes, mms_max, world) / 1e9, "unit": "GB/s",
        "ms_per_step": mms_max, "ms": mst,
        "roofline": hbm_roofline(m_bytes / (mst["mean"] * 1e-3) / 1e9, peaks, peak_src,
                                 "attn_merge_kernel<128>", recorded_traffic("merge", "merge4"),
                                 m_bytes),
        "gpu_launches": mlaunches,
    }
    del mo_parts, ml_parts, m_out, m_lse

    # ---- packed variable-length prefill leg: 16 causal sequences with seeded
    # lengths in [256, 4096], MHA H32 d128, no padding
    vl_lens = ai.varlen_lengths(16, 256, 4096, seed=shard_seed(rank) + 13)
    vq_h, vk_h, vv_h, vcq_h, vck_h = ai.make_varlen(vl_lens, vl_lens, 32, 32, 128,
                                                   seed=shard_seed(rank) + 17)
    vq, vk, vv, vcq, vck = (t.to(dev) for t in (vq_h, vk_h, vv_h, vcq_h, vck_h))
    vo = torch.empty_like(vq)
    vlse = torch.empty((32, vq.shape[0]), dtype=torch.float32, device=dev)
    vmax = max(vl_lens)

    def fwd_varlen():
        ea.attn_fwd_varlen(vq, vk, vv, vcq, vck, vmax, vmax, o=vo, lse=vlse, causal=True)

    vtimes, vlaunches = timed_kernel_loop(fwd_varlen, args.steps, args.warmup, world, flush, label="varlen")
    vst = time_stats(vtimes)
    vms_max = max_over_ranks(vst["mean"], world)
    v_flops = sum(metrics.attn_flops(1, 32, n, n, 128, True, -1) for n in vl_lens)
    varlen = {
        "workload": f"MHA causal packed prefill, 16 sequences of {min(vl_lens)}-{max(vl_lens)} "
                    f"tokens ({sum(vl_lens)} total) H32 d128",
        "value": whole_job_rate(v_flops, vms_max, world) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": vms_max, "ms": vst,
        "roofline": tensor_roofline(v_flops / (vst["mean"] * 1e-3) / 1e12, peaks, peak_src,
                                    "attn_fwd_kernel<128,false> (packed)",
                                    recorded_traffic("attn_fwd_kernel", "varlen")),
        "gpu_launches": vlaunches,
    }
    del vq, vk, vv, vo

    # ---- decode leg
    dw = ai.GQA_DECODE
    if args.decode_batch:
        dw = dataclasses.replace(dw, B=args.decode_batch, name=f"{dw.name} [batch {args.decode_batch}]")
    qd_h, kc_h, vc_h = ai.make_decode(dw.B, dw.Hq, dw.Hkv, dw.Nk, dw.d, seed=shard_seed(rank))
    qd, kc, vc = qd_h.to(dev), kc_h.to(dev), vc_h.to(dev)
    od = torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device=dev)
    lsed = torch.empty((dw.B, dw.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(ea.attn_decode_workspace_bytes(dw.B, dw.Hq, dw.d, args.decode_splits, dw.Nk),
                     dtype=torch.uint8, device=dev)

    def dec():
        ea.attn_decode(qd, kc, vc, o=od, lse=lsed, num_splits=args.decode_splits, workspace=ws)

    # the cache (2.1 GB) is far larger than L2, so no flush between decode steps
    dtimes, dlaunches = timed_kernel_loop(dec, args.steps, args.warmup, world, None, label="decode")
    dst = time_stats(dtimes)
    dms_max = max_over_ranks(dst["mean"], world)
    kv_bytes = metrics.decode_kv_bytes([dw.Nk] * dw.B, dw.Hkv, dw.d)
    d_all = metrics.decode_bytes(dw.B, dw.Hq, dw.Hkv, [dw.Nk] * dw.B, dw.d)
    decode = {
        "workload": dw.name, "value": whole_job_rate(kv_bytes, dms_max, world) / 1e9,
        "unit": "GB/s", "ms_per_step": dms_max, "ms": dst,
        "roofline": hbm_roofline(kv_bytes / (dst["mean"] * 1e-3) / 1e9, peaks, peak_src,
                                 "decode_split_kernel<128,4> + decode_combine_kernel<128>",
                                 recorded_traffic("decode", "decode", bool(args.decode_batch)),
                                 d_all),
        "gpu_launches": dlaunches,
    }

    # ---- paged decode leg: the same logical cache scattered into shuffled pages
    # of args.page_size keys (a seeded permutation; unused pool pages are never read)
    ps = args.page_size
    per_seq = dw.Nk // ps
    n_pages = dw.B * per_seq + 64
    gperm = torch.Generator(device="cpu")
    gperm.manual_seed(shard_seed(rank) + 11)
    perm = torch.randperm(n_pages, generator=gperm)[: dw.B * per_seq]
    bt = perm.reshape(dw.B, per_seq).to(torch.int32).to(dev)
    kpg = torch.empty((n_pages, ps, dw.Hkv, dw.d), dtype=torch.bfloat16, device=dev)
    vpg = torch.empty_like(kpg)
    kpg[perm.to(dev)] = kc.reshape(dw.B * per_seq, ps, dw.Hkv, dw.d)
    vpg[perm.to(dev)] = vc.reshape(dw.B * per_seq, ps, dw.Hkv, dw.d)
    del kc, vc

    def dec_paged():
        ea.attn_decode_paged(qd, kpg, vpg, bt, o=od, lse=lsed, num_splits=args.decode_splits,
                             workspace=ws)

    ptimes, plaunches = timed_kernel_loop(dec_paged, args.steps, args.warmup, world, None, label="decode_paged")
    pst = time_stats(ptimes)
    pms_max = max_over_ranks(pst["mean"], world)
    decode_paged = {
        "workload": f"{dw.name}, paged cache ({ps}-key pages, shuffled pool)", "page_size": ps,
        "value": whole_job_rate(kv_bytes, pms_max, world) / 1e9, "unit": "GB/s",
        "ms_per_step": pms_max, "ms": pst,
        "roofline": hbm_roofline(kv_bytes / (pst["mean"] * 1e-3) / 1e9, peaks, peak_src,
                                 "decode_split_kernel<128,4,paged> + decode_combine_kernel<128>",
                                 recorded_traffic("decode_paged", f"decode_p{ps}",
                                                  bool(args.decode_batch)),
                                 d_all),
        "gpu_launches": plaunches,
    }
    del kpg, vpg
    sampler.stop()

    # ---- end-to-end through the public API with host buffers (headline workload)
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        op = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lp = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

        def e2e_step():
            q.copy_(qp, non_blocking=True)
            k.copy_(kp, non_blocking=True)
            v.copy_(vp, non_blocking=True)
            ea.attn_fwd(q, k, v, o=o, lse=lse, causal=w.causal, window_left=w.window_left)
            op.copy_(o, non_blocking=True)
            lp.copy_(lse, non_blocking=True)

        serial_ms = max_over_ranks(e2e_loop(e2e_step, min(args.steps, 30), 2), world)
        # the same steps pipelined: a second device buffer set, three streams
        qkv2 = [(q, k, v), (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))]
        out2 = [(o, lse), (torch.empty_like(o), torch.empty_like(lse))]
        host_out = [(op, lp), (torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                               torch.empty(lse.shape, dtype=lse.dtype).pin_memory())]

        def p_in(b):
            for dst, src in zip(qkv2[b], (qp, kp, vp)):
                dst.copy_(src, non_blocking=True)

        def p_fwd(b, stream):
            qq, kk, vv = qkv2[b]
            ea.attn_fwd(qq, kk, vv, o=out2[b][0], lse=out2[b][1], causal=w.causal,
                        window_left=w.window_left, stream=stream)

        def p_out(b):
            host_out[b][0].copy_(out2[b][0], non_blocking=True)
            host_out[b][1].copy_(out2[b][1], non_blocking=True)

        e_ms = max_over_ranks(e2e_pipelined(p_in, p_fwd, p_out, min(args.steps, 30), 2), world)
        h2d = sum(t.numel() * t.element_size() for t in (qp, kp, vp))
        d2h = op.numel() * op.element_size() + lp.numel() * lp.element_size()
        e2e = {"value": whole_job_rate(flops, e_ms, world) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "mode": "pipelined: H2D, kernel and D2H of consecutive steps overlap on three "
                       "streams with two device buffer sets; every step's copies run in full",
               "serial_ms_per_step": serial_ms,
               "serial_value": whole_job_rate(flops, serial_ms, world) / 1e12}
        del qkv2, out2, host_out

    # ---- the oracle on the host cores: the headline workload, and the GQA
    # sliding-window workload once
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_block(w, q_h, k_h, v_h, budget_s=12.0)
        for leg in legs:
            if leg["key"] == "gqa32k":
                gw = ai.GQA_SWA_32K
                gq, gk, gv = ai.make_for(gw, seed=shard_seed(rank))
                leg["cpu_baseline"] = cpu_baseline_block(gw, gq, gk, gv, budget_s=6.0)
                del gq, gk, gv

    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.Nq,
                   "d": w.d, "causal": w.causal, "window_left": w.window_left,
                   "parallelism": f"independent batch per GPU x{world}",
                   "l2": "256 MiB memset flush before every timed prefill/backward step "
                         "(outside the events); decode and merge inputs exceed L2",
                   "flop_count": "4*d*allowed (i,j) pairs (mask-adjusted)"},
        "ms": head["ms"],
        "pct_bf16_peak": head["pct_bf16_peak"],
        "tile_tflops": head["tile_tflops"],
        "roofline": head["roofline"],
        "prefill_legs": legs,
        "decode": decode,
        "backward": backward,
        "merge": merge_leg,
        "varlen": varlen,
        "decode_paged": decode_paged,
        "clocks": sampler.summary(),
        "gpu_launches": launches,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "kernel_sources": {k: kernel_source_hash(k) for k in KERNEL_SOURCES},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
