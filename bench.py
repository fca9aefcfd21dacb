#!/usr/bin/env python
"""Benchmark of factorized sparse attention (forward + recomputing backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of the workload: the fused forward
kernel, then the backward pass's three phases (D_i and accumulator set-up, the recomputing
tcgen05 kernel, dQ conversion).  The layout is built and uploaded once, outside the timed region.
The step time comes from K steps with CUDA events at their boundaries only; K further steps with
an event between the phases give the per-phase breakdown and the backward kernel's duration.
Inputs are seeded synthetic tensors (workloads.py), resident in HBM when timing starts; L2 is
flushed (a 256 MiB write, then a 256 MiB read that evicts the written lines) before every timed
step, outside the step's CUDA events.

The metric counts active-block FLOPs: every 128 x 128 tile pair the kernels compute contributes
128 * 128 * 4 * d FLOPs to the forward and 2.5 times that to the backward (five matmuls, one of
them the recomputation of S), 3.5x in total.  `value` is the whole-job figure over all ranks
(replicas: every rank runs the full workload on its own GPU; time is the max over ranks).

The reference arm (--impl reference) is the fp64 CPU oracle, run on the host cores: each step is
its forward and backward over the whole workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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

from workloads import HEADLINE, WORKLOADS, make_inputs  # noqa: E402

METRIC = "active-block TFLOP/s fwd+bwd (bf16) at n=12288 and % of B200 tensor peak"
UNIT = "TFLOP/s"
TILE = 128
FLUSH_BYTES = 256 << 20

# Per-launch DRAM traffic of the kernels, from the committed ncu table (profiles/), valid while
# the kernel's sources hash to the value recorded beside it.
TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "traffic_by_workload.md")
KERNEL_SOURCES = {
    "bwd_kernel": ("bwd.cu", "tiles.cuh", "sm100.cuh", "frames.cuh", "kernels.h"),
    "fwd_bf16_kernel": ("fwd_bf16.cu", "tiles.cuh", "sm100.cuh", "frames.cuh", "kernels.h"),
}


def kernel_src_hash(kernel: str = "bwd_kernel") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_factorized_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str = "bwd_kernel", path: str = TRAFFIC_TABLE):
    """DRAM read + write bytes of one step's launches of `kernel` (summed over the passes) from the
    ncu table, or None when the table has no rows for the workload at the current source hash."""
    try:
        with open(path) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    src = kernel_src_hash(kernel)
    total, found = 0, False
    for ln in lines:
        cells = [c.strip() for c in ln.strip().strip("|").split("|")]
        if len(cells) >= 6 and cells[0] == workload and cells[1] == kernel and cells[3] == src:
            total += int(cells[4]) + int(cells[5])
            found = True
    return total if found else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode", action="store_true",
                    help="time the decode step (one query row per batch-head at the last position) "
                         "instead of the forward + backward step")
    return ap.parse_args()


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int, device=None):
    if world > 1:
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job(per_rank_units: float, times_s, world: int):
    """Aggregate of replicas: all ranks' units over the slowest rank's time."""
    return per_rank_units * world / max(times_s)


# ---------------------------------------------------------------- clocks during the timed region
class ClockSampler:
    """NVML samples of SM clock, power and throttle reasons every ~2 ms on a thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                uuid = None
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.h, self.ok = pynvml, h, True
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = n.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((mhz, reasons, pw))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        reasons = [name for b, name in self.REASONS.items() if bits & b]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "power_w_max": max(s[2] for s in self.samples)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------- oracle sample (CPU)
def oracle_sample(w, slabs, inputs=None):
    """Run the oracle's full forward + backward on the given (batch, head) slabs; return
    (seconds, threads).  Each slab is one (b, h): the oracle runs the whole n for that head.
    inputs: the workload's (q, k, v, do), drawn here when not given (outside the timing)."""
    import oracle
    q, k, v, do = inputs if inputs is not None else make_inputs(w)
    kinds, offs = oracle.head_kinds(w.family, w.head_mode, w.heads, w.l, w.c, w.offset_step)
    t0 = time.perf_counter()
    for b, h in slabs:
        p = oracle.Problem.from_kinds([kinds[h]], [offs[h]], w.l, w.c)
        sl = [t[b:b + 1, h:h + 1].double().numpy() for t in (q, k, v, do)]
        p.fwd(*sl[:3])
        p.bwd(*sl)
    return time.perf_counter() - t0, oracle.num_threads()


CPU_BASELINE_SECONDS = 10.0  # oracle time per CPU-baseline measurement


def cpu_baseline(w, flops, min_seconds=CPU_BASELINE_SECONDS):
    """The oracle, as it stands, on the host cores: the full forward + backward of one (batch,
    head) slab after another, cycling over the workload's slabs until at least min_seconds of
    oracle time have run (at most 64 passes over the workload).  value = the metric's FLOPs per
    workload x the workloads covered / the oracle time."""
    inputs = make_inputs(w)
    slabs = [(b, h) for b in range(w.batch) for h in range(w.heads)]
    done, secs, threads = 0, 0.0, 1
    while secs < min_seconds and done < 64 * len(slabs):
        s, threads = oracle_sample(w, [slabs[done % len(slabs)]], inputs)
        secs += s
        done += 1
    covered = done / len(slabs)
    return {"value": flops * covered / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"oracle fwd+bwd of {done} (batch, head) slabs at full n={w.n}, cycling over the "
                      f"workload's {len(slabs)} ({covered:.2f} workloads), {secs:.1f} s"}


def step_flops(w, info):
    tiles = info["exec_tiles"] * w.batch
    fwd = tiles * TILE * TILE * 4 * w.d
    return fwd * 3.5, fwd * 2.5, info["allowed_pairs"] * w.batch * 4 * w.d * 3.5


def step_bytes(w, lay):
    """Algorithmic HBM bytes of one forward and one backward pass (each tensor touched once):
    forward Q, O, the K and V rows some query reads, lse; backward adds dO, D, dQ and full dK,
    dV writes.  A fixed-pattern summary head (kind fA2) reads only n / l * c key rows."""
    import block_sparse_factorized_b200 as bsf
    row = w.d * (4 if w.dtype == "fp32" else 2)
    rows = w.batch * w.heads * w.n
    used = 0
    for h in range(w.heads):
        kind, _ = lay.head_kind(h)
        used += (w.n // w.l) * w.c if kind == bsf.ST_KIND_FA2 else w.n
    used *= w.batch
    fwd = 2 * rows * row + 2 * used * row + rows * 4
    bwd = fwd + rows * row + rows * 4 + 3 * rows * row
    return fwd, bwd


# ---------------------------------------------------------------- reference arm
# Active 128 x 128 tile pairs per batch element in the canonical execution frames (same-block and
# band heads natural, stride heads on grid columns, summary heads on compacted summary keys,
# merged heads as the two parts of their LSE merge).  The reference arm counts the metric's FLOPs
# from this table, so it never loads the CUDA library; tests/test_bench_host.py checks the table
# against the library's own census of every workload.
CANONICAL_TILES = {
    "strided_n256_l16_fp32": 5,
    "strided_merged_n3072_l64": 632,
    "fixed_n12288_l128_c32": 5184,
    "strided_n12288_l128": 2552,
    "strided_merged_n12288_l128": 5104,
    "strided_n65536_l256": 9204,
    "fixed_merged_n12288_l128_c32": 10176,
    "strided_n12288_l128_d32": 2552,
}


def canonical_flops(w):
    """The metric's FLOPs of one step (forward + backward over every active tile pair)."""
    return CANONICAL_TILES[w.name] * w.batch * TILE * TILE * 4 * w.d * 3.5


def run_reference(args, rank, world):
    """The fp64 oracle, as it stands, on the host cores: each step is its full forward and
    backward over the whole workload (every (batch, head) slab at full n).  Only rank 0 runs it."""
    w = WORKLOADS[args.workload]
    if rank != 0:
        return 0
    flops = canonical_flops(w)
    slabs_all = [(b, h) for b in range(w.batch) for h in range(w.heads)]
    per_step = []
    threads = 1
    inputs = make_inputs(w)
    for s in range(args.warmup + args.steps):
        secs, threads = oracle_sample(w, slabs_all, inputs)
        if s >= args.warmup:
            per_step.append(secs)
    ms = 1e3 * statistics.mean(per_step)
    value = flops / (ms / 1e3) / 1e12
    sample = (f"oracle fwd+bwd of the whole workload per step: all {len(slabs_all)} (batch, head) "
              f"slabs at full n={w.n}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "pattern": "fixed" if w.family == 2 else "strided",
            "heads_mode": {1: "alternating", 2: "merged", 3: "head1", 4: "head2"}[w.head_mode],
            "n": w.n, "l": w.l, "c": w.c, "batch": w.batch, "heads": w.heads, "d": w.d,
            "io_dtype": w.dtype, "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)",
            "parallelism": "replicas"}


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local):
    import block_sparse_factorized_b200 as bsf
    from block_sparse_factorized_b200 import _abi
    import ctypes

    w = WORKLOADS[args.workload]
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)

    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload(stream)
    info = lay.info()
    flops, bwd_flops, useful = step_flops(w, info)
    q, k, v, do = (t.to(device) for t in make_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    lib = _abi.load()
    desc = bsf._desc(q)
    ws_bytes = int(lib.st_attn_bwd_workspace_bytes(ctypes.byref(desc), lay.handle))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    # a second buffer, read after the write: it evicts the written (dirty) lines, so that their
    # write-back to HBM happens before the step rather than inside its first kernels
    flush_rd = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()
    P = ctypes.c_void_p

    def ptr(t):
        return P(t.data_ptr())

    fws_bytes = int(lib.st_attn_fwd_workspace_bytes(ctypes.byref(desc), lay.handle))
    fws = torch.empty(fws_bytes, dtype=torch.uint8, device=device)

    def fwd():
        _abi.check(lib.st_attn_fwd(ptr(q), ptr(k), ptr(v), lay.handle, ptr(o), ptr(lse), ptr(fws),
                                   fws_bytes, ctypes.byref(desc), sp), "st_attn_fwd")

    def prep():
        _abi.check(lib.st_attn_bwd_prepare(ptr(o), ptr(do), lay.handle, ptr(dk), ptr(dv), ptr(ws),
                                           ws_bytes, ctypes.byref(desc), sp), "st_attn_bwd_prepare")

    def main():
        _abi.check(lib.st_attn_bwd_main(ptr(q), ptr(k), ptr(v), ptr(lse), ptr(do), lay.handle,
                                        ptr(dq), ptr(dk), ptr(dv), ptr(ws), ws_bytes, ctypes.byref(desc), sp),
                   "st_attn_bwd_main")

    def finish():
        _abi.check(lib.st_attn_bwd_finish(lay.handle, ptr(dq), ptr(ws), ws_bytes,
                                          ctypes.byref(desc), sp), "st_attn_bwd_finish")

    for _ in range(args.warmup):
        flush_l2()
        fwd(); prep(); main(); finish()
    torch.cuda.synchronize(device)
    lay.check(stream)

    # Timed region: K steps bracketed by events at their boundaries only (events between the
    # kernels would hold each kernel back until the previous one has completed, and time the
    # gaps they add) -- the step time; then K more steps with an event between the phases -- the
    # per-phase times of the breakdown and the backward kernel's duration for the roofline.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier(world, device)
    torch.cuda.synchronize(device)
    with sampler:
        for s in range(args.steps):
            flush_l2()
            e = ev[s]
            e[0].record(stream); fwd(); prep(); main(); finish(); e[1].record(stream)
        for s in range(args.steps):
            flush_l2()
            e = evp[s]
            e[0].record(stream); fwd(); e[1].record(stream); prep(); e[2].record(stream)
            main(); e[3].record(stream); finish(); e[4].record(stream)
        torch.cuda.synchronize(device)
    barrier(world, device)
    lay.check(stream)
    t_step = [e[0].elapsed_time(e[1]) for e in ev]
    t_fwd = [e[0].elapsed_time(e[1]) for e in evp]
    t_prep = [e[1].elapsed_time(e[2]) for e in evp]
    t_main = [e[2].elapsed_time(e[3]) for e in evp]
    t_fin = [e[3].elapsed_time(e[4]) for e in evp]
    ms_local = statistics.mean(t_step)
    ms = max_over_ranks(ms_local, world, device)
    value = flops * world / (ms / 1e3) / 1e12
    # fwd per pass; bwd: prepare, the main kernel per pass, a summing pass per split pass, and
    # the convert pass unless every head's dQ is stored by the main kernel
    launches_per_step = (2 * info["passes"] + 1 + info["split_passes"] +
                         (1 if info["dq_direct_heads"] < w.heads else 0))
    peaks = measured_peaks()
    main_ms = statistics.mean(t_main)
    achieved = bwd_flops / (main_ms / 1e3) / 1e12
    src = kernel_src_hash("bwd_kernel")
    tr = recorded_traffic(w.name, "bwd_kernel")
    fwd_bytes, bwd_bytes = step_bytes(w, lay)
    hbm = {"bytes_fwd": fwd_bytes, "bytes_bwd": bwd_bytes,
           "achieved_gbs": (fwd_bytes + bwd_bytes) / (ms / 1e3) / 1e9, "peak_gbs": peaks["hbm_gbs"]}
    hbm["frac"] = hbm["achieved_gbs"] / peaks["hbm_gbs"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)  # flop per byte
    if flops / (fwd_bytes + bwd_bytes) >= ridge:
        roofline = {"kernel": "st_attn_bwd_main (bwd_kernel)", "bound": "tensor", "achieved": achieved,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                    "traffic": tr, "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)"}
    else:  # below the ridge point: the backward kernel's own bytes against the copy bandwidth
        bwd_kernel_bytes = bwd_bytes - fwd_bytes // 2  # O is read by the prepare pass, not the kernel
        gbs = bwd_kernel_bytes / (main_ms / 1e3) / 1e9
        roofline = {"kernel": "st_attn_bwd_main (bwd_kernel)", "bound": "hbm", "achieved": gbs,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                    "traffic": tr, "peak_source": f"{peaks['source']} copy bandwidth (MEASURED_PEAKS.json)"}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, lay, device, stream, flops, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, flops)

    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(w),
        "pct_of_tensor_peak": 100.0 * (value / world) / peaks["bf16_tflops"],
        "useful_tflops": useful * world / (ms / 1e3) / 1e12,
        "breakdown_ms": {"fwd": statistics.mean(t_fwd), "bwd_prepare": statistics.mean(t_prep),
                         "bwd_main": main_ms, "bwd_finish": statistics.mean(t_fin)},
        "fwd_tflops": flops / 3.5 / (statistics.mean(t_fwd) / 1e3) / 1e12,
        "roofline": roofline, "hbm": hbm, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * 2 * args.steps, "clocks": clocks,
        "exec_tiles": info["exec_tiles"] * w.batch, "kernel_src": src,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del lay
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_e2e(args, w, lay, device, stream, flops, world):
    """Same metric through the public API with pinned host buffers: every step copies its q, k,
    v, dO from host memory and its dq, dk, dv back.  The copies of neighbouring steps overlap the
    compute (a host-to-device stream, the compute stream, a device-to-host stream, two sets of
    device buffers), as a training loop that streams its batches would run them; the time is the
    whole sequence of steps over their number."""
    import block_sparse_factorized_b200 as bsf
    hq, hk, hv, hdo = (t.pin_memory() for t in make_inputs(w))
    dq_h, dk_h, dv_h = (torch.empty_like(hq).pin_memory() for _ in range(3))
    dev = [[torch.empty_like(hq, device=device) for _ in range(4)] for _ in range(2)]
    grads = [[torch.empty_like(hq, device=device) for _ in range(3)] for _ in range(2)]
    o = torch.empty_like(dev[0][0])
    lse = torch.empty(hq.shape[:3], dtype=torch.float32, device=device)
    ws = torch.empty(max(256, bsf.st_attn_bwd_workspace_bytes(dev[0][0], lay)), dtype=torch.uint8,
                     device=device)
    fws = torch.empty(max(256, bsf.st_attn_fwd_workspace_bytes(dev[0][0], lay)), dtype=torch.uint8,
                      device=device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def run(steps):
        ev = [{k: torch.cuda.Event() for k in ("in", "comp", "out")} for _ in range(steps)]
        for i in range(steps):
            b = i % 2
            # inputs of step i into buffer set b, once step i - 2 (same set) has read them
            if i >= 2:
                s_in.wait_event(ev[i - 2]["comp"])
            with torch.cuda.stream(s_in):
                for d_, h_ in zip(dev[b], (hq, hk, hv, hdo)):
                    d_.copy_(h_, non_blocking=True)
                ev[i]["in"].record(s_in)
            # compute, once the inputs are in and step i - 2's outputs have left the device
            stream.wait_event(ev[i]["in"])
            if i >= 2:
                stream.wait_event(ev[i - 2]["out"])
            q_, k_, v_, do_ = dev[b]
            bsf.st_attn_fwd(q_, k_, v_, lay, o=o, lse=lse, workspace=fws, stream=stream)
            bsf.st_attn_bwd(q_, k_, v_, o, lse, do_, lay, dq=grads[b][0], dk=grads[b][1], dv=grads[b][2],
                            workspace=ws, stream=stream)
            ev[i]["comp"].record(stream)
            # outputs back to host memory
            s_out.wait_event(ev[i]["comp"])
            with torch.cuda.stream(s_out):
                for h_, d_ in zip((dq_h, dk_h, dv_h), grads[b]):
                    h_.copy_(d_, non_blocking=True)
                ev[i]["out"].record(s_out)

    run(min(args.warmup, 3) + 1)
    torch.cuda.synchronize(device)
    steps = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    stream.wait_event(e0)
    s_out.wait_event(e0)
    run(steps)
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    e1.record(s_out)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, device)
    nbytes = hq.numel() * hq.element_size()
    return {"value": flops * world / (ms / 1e3) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "steps": steps, "h2d_bytes_per_step": 4 * nbytes, "d2h_bytes_per_step": 3 * nbytes,
            "api": "block_sparse_factorized_b200.st_attn_fwd / st_attn_bwd (C ABI), pinned host buffers, "
                   "copies of neighbouring steps overlapping the compute on separate streams"}


def run_decode(args, rank, world, local):
    """The decode step of the workload's pattern at the last position, pos = n - 1 (the largest
    allowed sets of the growing kinds): one query row per (batch, head) against the K/V caches.
    HBM-bound, so the metric is the algorithmic bytes per step (the allowed K and V rows, the
    query and output rows, lse) over its event time, against the measured copy bandwidth."""
    import ctypes

    import block_sparse_factorized_b200 as bsf
    w = WORKLOADS[args.workload]
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c)
    q, k, v, _ = (t.to(device) for t in make_inputs(w))
    pos = w.n - 1
    qrow = q[:, :, pos].contiguous()
    esz = q.element_size()
    rows = sum(len(lay.decode_row_keys(h, pos)) for h in range(w.heads)) * w.batch
    nbytes = rows * 2 * 64 * esz + w.batch * w.heads * (2 * 64 * esz + 4)
    o = torch.empty_like(qrow)
    lse = torch.empty(qrow.shape[:2], dtype=torch.float32, device=device)
    ws = torch.empty(max(256, int(lay._lib.st_attn_decode_workspace_bytes(ctypes.byref(bsf._desc(q)), lay.handle))),
                     dtype=torch.uint8, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        bsf.st_attn_decode(qrow, k, v, lay, pos, o=o, lse=lse, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush.zero_(); flush_rd.sum(); step()
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier(world, device)
    torch.cuda.synchronize(device)
    with sampler:
        for a, b in ev:
            flush.zero_(); flush_rd.sum()
            a.record(stream); step(); b.record(stream)
        torch.cuda.synchronize(device)
    barrier(world, device)
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world, device)
    peaks = measured_peaks()
    gbs = nbytes * world / (ms / 1e3) / 1e9
    line = {"metric": "decode step GB/s (allowed K/V rows + q, o, lse)", "value": gbs, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": f"decode_{w.name}", "pos": pos, "batch": w.batch, "heads": w.heads,
                       "kv_rows_read": rows, "l2": "flushed before every timed step"},
            "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / world / peaks["hbm_gbs"], "traffic": None},
            "gpu_launches": args.steps, "clocks": sampler.summary()}  # one kernel per step (after a memset)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del lay
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device; this benchmark times the B200 kernels"}))
        return 1
    if args.decode:
        return run_decode(args, rank, world, local)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
