#!/usr/bin/env python3
"""Benchmark: decode GEMV achieved HBM GB/s on B200 (plus the prefill GEMM
TFLOP/s and the MoE GEMV GB/s as secondary lines of the same JSON record).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One *step* = the decode workload once: y = x . dequant(W)^T at M = 1 for the
three weight shapes 4096x4096, 14336x4096 and 4096x14336 (4-bit affine,
group 64, bf16 activations, scales and biases).  `value` is the algorithmic
bytes of those three calls (packed codes + scales + biases + x + y) summed over
all steps of all ranks, divided by the timed device time (max over ranks).

Timing: W warm-up steps, then timed trials of exactly K steps each, every
trial behind an L2 flush and bracketed by barrier + cuda.synchronize, CUDA
events on the launching stream; trials repeat for --clock-window seconds so
that the NVML clock sampler sees the load, and the median trial is reported.
The steps are replayed from CUDA graphs (host launch overhead is larger than
the kernels) and rotate over weight copies larger than 3x L2.  Under torchrun
each rank runs the same workload on its own GPU (independent replicas, weak
scaling); the time is the max over ranks.

Secondary lines (rank 0): every other workload -- the 36-config bit-width
sweep, the MoE gate+up+SiLU and down GEMVs at T = 1, 16, 64 and the six
prefill GEMMs -- with the fraction of the measured and the datasheet peaks.
The oracle's CPU baseline is timed single-threaded (reported) and on all
affinity cores (beside it).

--impl reference times the CPU oracle (oracle/) on the same workload and
metric, on a bounded sample per step; rank 0 only.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode GEMV achieved HBM GB/s (% of peak); prefill GEMM TFLOP/s (% of bf16 peak)"
L2_BYTES = 126 * 1024 * 1024


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def decode_bytes(M, N, K, bits, gs):
    # packed codes + bf16 scales and biases + bf16 x + bf16 y
    return N * K * bits // 8 + N * (K // gs) * 4 + 2 * M * K + 2 * M * N


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    HW_SLOW, HW_THERM, SW_THERM, SW_POWER = 0x8, 0x40, 0x20, 0x4

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(device_index)
            self.h = None
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                busid = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), bus,
                                             getattr(props, "pci_device_id", 0))
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByPciBusId(busid)
                except Exception:
                    self.h = None
            if self.h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = device_index
                if vis and vis.split(",")[0].strip().isdigit():
                    idx = int(vis.split(",")[device_index].strip())
                self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((sm, int(r)))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = {self.HW_SLOW: "hw_slowdown", self.HW_THERM: "hw_thermal_slowdown",
                 self.SW_THERM: "sw_thermal_slowdown", self.SW_POWER: "sw_power_cap"}
        seen = set()
        for _, r in self.samples:
            for bit, n in names.items():
                if r & bit:
                    seen.add(n)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(seen), "samples": len(self.samples)}


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float) -> float:
    """The slowest rank's time (the job's time): one all-reduce(MAX)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job GB/s: every rank's bytes over the max-over-ranks time."""
    return bytes_per_step * steps * world / (ms_max * 1e-3) / 1e9


# ---------------------------------------------------------------- traffic record
def traffic_record(name):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (sha256 of each file listed in the summary)."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        txt = open(path).read()
    except OSError:
        return None, None
    rec = {}
    for line in txt.splitlines():
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            rec[k.strip()] = v.strip()
    srcs = [x.strip() for x in rec.get("source_files", "").split(",") if x.strip()]
    shas = [x.strip() for x in rec.get("source_sha256", "").split(",") if x.strip()]
    if not srcs or len(srcs) != len(shas):
        return None, None
    for src, sha in zip(srcs, shas):
        try:
            cur = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()
        except OSError:
            return None, None
        if cur != sha:
            return None, "stale"
    return rec, "current"


# ---------------------------------------------------------------- our arm
HBM_DATASHEET_GBS = 8000.0      # B200 HBM3e, datasheet
BF16_DATASHEET_TFLOPS = 2250.0  # B200 dense bf16, datasheet


def copies_for(nbytes: int) -> int:
    """weight copies whose rotation reads more than 3x the L2 between reuses"""
    return max(2, int(np.ceil(3 * L2_BYTES / nbytes)))


def clone_qw(api, qw):
    return api.QWeight(qw.packed.clone(), qw.scales.clone(), qw.biases.clone(), qw.rows, qw.cols,
                       qw.group_size, qw.bits)


def build_decode(torch, api, wl, n_sets, dev):
    cases = wl.WORKLOADS.decode
    sets = []
    base = []
    for c in cases:
        w = wl.gen_weight(c.N, c.K, c.seed)
        qw = api.qmm_quantize(w.to(dev), c.group_size, c.bits, torch.bfloat16)
        x = wl.gen_x(c.M, c.K, c.seed + 1).to(dev)
        base.append((c, qw, x))
    torch.cuda.synchronize()
    for s in range(n_sets):
        cur = []
        for c, qw, x in base:
            q2 = qw if s == 0 else clone_qw(api, qw)
            y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)
            cur.append((c, q2, x, y))
        sets.append(cur)
    torch.cuda.synchronize()
    return sets


class L2Flush:
    """Writes a buffer twice the size of L2 (between timed trials)."""

    def __init__(self, torch, dev):
        self.buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.n = 0

    def __call__(self):
        self.n += 1
        self.buf.fill_(float(self.n))


def capture(torch, fn, n, stream):
    """a CUDA graph of fn(0), ..., fn(n - 1) on `stream` (None when n == 0)"""
    if n == 0:
        return None
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in range(n):
            fn(s)
    return g


def run_ours(args):
    import torch

    from weight_only_quantized_qmm_b200 import api
    from weight_only_quantized_qmm_b200 import workloads as wl

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    hbm_peak, bf16_peak, bf16_sust, peak_src = peaks()
    assert api.qmm_device_check() == 0, "needs a compute capability 10.0 GPU"

    cases = wl.WORKLOADS.decode
    step_bytes = sum(decode_bytes(c.M, c.N, c.K, c.bits, c.group_size) for c in cases)
    n_sets = copies_for(step_bytes)  # the step's weights rotate over > 3x L2
    sets = build_decode(torch, api, wl, n_sets, dev)
    stream = torch.cuda.Stream(device=dev)
    launches_per_step = len(cases)
    flush = L2Flush(torch, dev)

    def one_step(s):
        for c, qw, x, y in sets[s % n_sets]:
            api.qmm_matmul(x, qw, True, out=y, stream=stream)

    K = args.steps
    W = max(args.warmup, 3)
    with torch.cuda.stream(stream):
        for s in range(W):  # eager warm-up steps (also configure the kernels)
            one_step(s)
    torch.cuda.synchronize()
    # exactly K steps per timed trial: `reps` replays of a one-rotation graph
    # (n_sets steps) and one graph of the remaining K mod n_sets steps
    reps, rem = divmod(K, n_sets)
    g_full = capture(torch, one_step, n_sets if reps else 0, stream)
    g_rem = capture(torch, one_step, rem, stream)
    torch.cuda.synchronize()

    def replay_k():
        for _ in range(reps):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()

    with torch.cuda.stream(stream):  # warm-up replays
        replay_k()
    torch.cuda.synchronize()

    # timed trials: each trial is exactly K steps behind an L2 flush, bracketed
    # by barrier + synchronize; trials repeat until the clock sampler has seen
    # at least `clock_window` seconds of them; the reported time is the median
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index, period_s=0.01)
    trial_ms = []
    with sampler:
        t_start = time.perf_counter()
        while True:
            with torch.cuda.stream(stream):
                flush()
            torch.cuda.synchronize()
            barrier(world)
            torch.cuda.synchronize()
            with torch.cuda.stream(stream):
                ev0.record(stream)
                replay_k()
                ev1.record(stream)
            torch.cuda.synchronize()
            barrier(world)
            trial_ms.append(ev0.elapsed_time(ev1))
            done = (time.perf_counter() - t_start >= args.clock_window and len(trial_ms) >= 3) \
                or len(trial_ms) >= 20000
            # every rank takes the same number of trials
            if world > 1:
                done = max_over_ranks(world, 1.0 if done else 0.0) > 0.5
            if done:
                break
    ms = max_over_ranks(world, statistics.median(trial_ms))
    ms_step = ms / K
    value = job_throughput(step_bytes, K, world, ms)

    # per-shape launch durations: one graph per shape rotating its own copies
    # (> 3x L2 each), timed from outside, so no event sits between two kernels
    per_shape = {}
    tot_b, tot_ms = 0.0, 0.0
    for i, c in enumerate(cases):
        b = decode_bytes(c.M, c.N, c.K, c.bits, c.group_size)
        n_i = copies_for(b)
        qws = [sets[s][i][1] if s < n_sets else clone_qw(api, sets[0][i][1]) for s in range(n_i)]
        _, _, x, y = sets[0][i]

        def shape_fn(qws=qws, x=x, y=y):
            for qw in qws:
                api.qmm_matmul(x, qw, True, out=y, stream=stream)
        d = time_graph(torch, shape_fn, stream, reps=10, inner=1) / n_i
        per_shape[c.name] = {"us": round(d * 1e3, 3), "GB/s": round(b / (d * 1e-3) / 1e9, 1),
                             "frac": round(b / (d * 1e-3) / 1e9 / hbm_peak, 3),
                             "copies": n_i}
        tot_b += b
        tot_ms += d
        del qws
    achieved = tot_b / (tot_ms * 1e-3) / 1e9
    rec, state = traffic_record("qgemv_decode_m1.txt")
    traffic = None
    if rec is not None and state == "current":
        try:
            traffic = float(rec["dram_bytes_per_launch_avg"])
        except (KeyError, ValueError):
            traffic = None

    # end to end through the public API with host buffers (pinned), per step:
    # H2D of the step's x, the three calls, D2H of its y, synchronize.  The
    # three x (and y) rows sit in one pinned buffer and one device buffer, so
    # that each direction is one copy.
    xlens = [c.M * c.K for c in cases]
    ylens = [c.M * c.N for c in cases]
    xs_h = torch.cat([x.reshape(-1).cpu() for (_, _, x, _) in sets[0]]).pin_memory()
    ys_h = torch.empty(sum(ylens), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(sum(xlens), dtype=torch.bfloat16, device=dev)
    y_dev = torch.empty(sum(ylens), dtype=torch.bfloat16, device=dev)
    x_views, y_views = [], []
    xo = yo = 0
    for c, xl, yl in zip(cases, xlens, ylens):
        x_views.append(x_dev[xo:xo + xl].view(c.M, c.K))
        y_views.append(y_dev[yo:yo + yl].view(c.M, c.N))
        xo, yo = xo + xl, yo + yl
    h2d = xs_h.numel() * xs_h.element_size()
    d2h = ys_h.numel() * ys_h.element_size()
    n_e2e = min(2000, max(50, 10 * K))

    def e2e_step(s):
        # the step's inputs in, its three GEMVs back to back (each may start
        # while the previous one finishes), its outputs out, then wait
        x_dev.copy_(xs_h, non_blocking=True)
        for i, (c, qw, _, _) in enumerate(sets[s % n_sets]):
            api.qmm_matmul(x_views[i], qw, True, out=y_views[i])
        ys_h.copy_(y_dev, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    for s in range(10):
        e2e_step(s)
    barrier(world)
    t0 = time.perf_counter()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(n_e2e):
        e2e_step(s)
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = max(e0.elapsed_time(e1), (time.perf_counter() - t0) * 1e3)
    ms_e2e = max_over_ranks(world, ms_e2e)
    e2e = {"value": round(step_bytes * n_e2e * world / (ms_e2e * 1e-3) / 1e9, 2),
           "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(ms_e2e / n_e2e, 4), "steps": n_e2e}

    secondary = {}
    if not args.no_secondary and rank == 0:
        secondary = run_secondary(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: W=0.02*randn quantized 4-bit g64, x=randn->bf16)",
        "config": {"workload": "decode GEMV M=1, 4-bit affine g64, bf16 x/scales/biases; "
                               "N x K = 4096x4096 + 14336x4096 + 4096x14336 per step",
                   "global_batch": world, "M": 1, "bits": 4, "group_size": 64,
                   "l2": f"L2 flushed (256 MB write) before every trial; within a trial the steps "
                         f"rotate {n_sets} weight copies ({n_sets * step_bytes / 1e6:.0f} MB > 3x L2)",
                   "launch": "CUDA graph replay", "parallelism": f"replicas x{world}",
                   "trials": len(trial_ms),
                   "trial_ms": {"median": round(statistics.median(trial_ms), 5),
                                "min": round(min(trial_ms), 5), "max": round(max(trial_ms), 5)}},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                     "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "peak_source": peak_src,
                     "frac_of_datasheet_8000": round(achieved / HBM_DATASHEET_GBS, 4),
                     "kernel": "qgemv_stream_kernel (decode GEMV, one token)",
                     "per_shape": per_shape},
        "e2e": e2e,
        "gpu_launches": K * launches_per_step,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "secondary": secondary,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_full, g_rem
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def time_graph(torch, fn, stream, reps=20, inner=4):
    """median per-call device time (ms) of fn, replayed from a CUDA graph of
    `inner` calls"""
    with torch.cuda.stream(stream):
        fn()
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(inner):
            fn()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(reps):
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / inner)
    del g
    return statistics.median(times)


def _gbs(nbytes, ms, hbm_peak):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"GB/s": round(gbs, 1), "frac": round(gbs / hbm_peak, 3),
            "frac_of_datasheet_8000": round(gbs / HBM_DATASHEET_GBS, 3), "us": round(ms * 1e3, 3)}


def run_secondary(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust):
    out = {}
    for name, fn in (("moe", secondary_moe), ("sweep", secondary_sweep),
                     ("prefill", secondary_prefill), ("moe_prefill", secondary_moe_prefill),
                     ("other_layouts", secondary_other_layouts)):
        try:
            out[name] = fn(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust)
        except Exception as e:  # pragma: no cover
            out[name + "_error"] = str(e)[:300]
        torch.cuda.empty_cache()
    return out


def secondary_moe(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust):
    """MoE decode: fused gate+up+SiLU then down, T = 1, 16, 64, top-8 of 128"""
    out = {}
    for case in wl.WORKLOADS.moe:
        E, dff, dm, T, k = case.num_experts, case.d_ff, case.d_model, case.tokens, case.top_k
        n_sets = 3
        stacks = []
        for s in range(n_sets):
            g = api.qmm_quantize(wl.gen_weight(E * dff, dm, case.seed + 10 * s).to(dev), 64, 4, torch.bfloat16)
            u = api.qmm_quantize(wl.gen_weight(E * dff, dm, case.seed + 10 * s + 1).to(dev), 64, 4, torch.bfloat16)
            d = api.qmm_quantize(wl.gen_weight(E * dm, dff, case.seed + 10 * s + 2).to(dev), 64, 4, torch.bfloat16)
            stacks.append((api.ExpertStack.from_qweight(g, E), api.ExpertStack.from_qweight(u, E),
                           api.ExpertStack.from_qweight(d, E)))
        a = wl.gen_x(T, dm, case.seed + 3).to(dev).reshape(-1)
        # id sets rotate with the weight sets so that the experts a call reads
        # are not still in L2 from the previous calls: for one token, 16
        # disjoint sets of 8 cover all 128 experts; otherwise independent draws
        n_ids = 16
        if T == 1:
            perm = torch.randperm(E, generator=torch.Generator().manual_seed(case.seed + 4)).to(torch.int32)
            id_sets = [perm[i * k:(i + 1) * k].reshape(1, k) for i in range(E // k)][:n_ids]
        else:
            id_sets = [wl.gen_moe_ids(T, E, k, case.seed + 4 + 100 * i) for i in range(n_ids)]
        n_dist = float(np.mean([len(np.unique(x.numpy())) for x in id_sets]))
        id_sets = [x.to(dev) for x in id_sets]
        h = torch.empty(T * k, dff, dtype=torch.bfloat16, device=dev)
        o = torch.empty(T * k, dm, dtype=torch.bfloat16, device=dev)
        it = [0]

        def gu():
            g, u, _ = stacks[it[0] % n_sets]
            ids = id_sets[it[0] % n_ids]
            it[0] += 1
            api.qmm_moe_gemv_id_gate_up_silu_batched(a, ids, T, k, dm, 0, g, u, out=h, stream=stream)

        def dn():
            _, _, d = stacks[it[0] % n_sets]
            ids = id_sets[it[0] % n_ids]
            it[0] += 1
            api.qmm_moe_gemv_id(h.reshape(-1), ids.reshape(-1), T * k, dff, d, out=o, stream=stream)
        t_gu = time_graph(torch, gu, stream, inner=n_ids)
        t_dn = time_graph(torch, dn, stream, inner=n_ids)
        b_gu = n_dist * 2 * (dff * dm // 2 + dff * (dm // 64) * 4) + 2 * T * dm + 2 * T * k * dff
        b_dn = n_dist * (dm * dff // 2 + dm * (dff // 64) * 4) + 2 * T * k * dff + 2 * T * k * dm
        out[f"moe_gate_up_silu_t{T}"] = dict(_gbs(b_gu, t_gu, hbm_peak), distinct_experts=round(n_dist, 1),
                                             rotation=f"{n_sets} weight sets x {n_ids} id sets")
        out[f"moe_down_t{T}"] = _gbs(b_dn, t_dn, hbm_peak)
        del stacks
    return out


def secondary_sweep(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust):
    """bit-width sweep: N = K = 8192, bits x group size x M, weights rotating
    over copies > 3x L2"""
    out = {}
    by_w = {}
    for c in wl.WORKLOADS.sweep:
        by_w.setdefault((c.bits, c.group_size), []).append(c)
    for (bits, gs), cs in by_w.items():
        qw = api.qmm_quantize(wl.gen_weight(8192, 8192, 2000 + 100 * bits + gs).to(dev), gs, bits,
                              torch.bfloat16)
        wbytes = 8192 * 8192 * bits // 8 + 8192 * (8192 // gs) * 4
        qws = [qw] + [clone_qw(api, qw) for _ in range(copies_for(wbytes) - 1)]
        for c in cs:
            x = wl.gen_x(c.M, c.K, c.seed + 1).to(dev)
            y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)

            def fn(x=x, y=y):
                for q in qws:
                    api.qmm_matmul(x, q, True, out=y, stream=stream)
            t = time_graph(torch, fn, stream, reps=10, inner=1) / len(qws)
            out[c.name] = _gbs(decode_bytes(c.M, c.N, c.K, c.bits, c.group_size), t, hbm_peak)
        del qws, qw
        torch.cuda.empty_cache()
    return out


def secondary_moe_prefill(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust):
    """MoE prefill (128 experts, top-8): device routing, then the expert-grouped
    GEMMs gate [768 x 2048] (token rows) and down [2048 x 768] (pair rows)"""
    out = {}
    E, dff, dm, k = 128, 768, 2048, 8
    g = api.ExpertStack.from_qweight(
        api.qmm_quantize(wl.gen_weight(E * dff, dm, 4600).to(dev), 64, 4, torch.bfloat16), E)
    d = api.ExpertStack.from_qweight(
        api.qmm_quantize(wl.gen_weight(E * dm, dff, 4601).to(dev), 64, 4, torch.bfloat16), E)
    for T in (256, 2048):
        P = T * k
        ids = wl.gen_moe_ids(T, E, k, 4602 + T).to(dev)
        a = wl.gen_x(T, dm, 4603 + T).to(dev)
        h = wl.gen_x(P, dff, 4604 + T).to(dev)
        ws = api.moe_workspace(P, E, dev, n_cols=max(dm, dff))  # with room for the gathered rows
        og = torch.empty(P, dff, dtype=torch.bfloat16, device=dev)
        od = torch.empty(P, dm, dtype=torch.bfloat16, device=dev)
        t_r = time_graph(torch, lambda: api.qmm_moe_compute_ids_tpe(ids, E, ws, stream=stream), stream,
                         reps=10, inner=5)
        t_g = time_graph(torch, lambda: api.qmm_moe_gemm_id(a, T, k, 1, ws, g, out=og, stream=stream),
                         stream, reps=10, inner=3)
        t_d = time_graph(torch, lambda: api.qmm_moe_gemm_id(h, T, k, k, ws, d, out=od, stream=stream),
                         stream, reps=10, inner=3)
        for name, t, n in (("gate", t_g, dff), ("down", t_d, dm)):
            kk = dm if name == "gate" else dff
            tf = 2 * P * n * kk / (t * 1e-3) / 1e12
            out[f"moe_prefill_t{T}_{name}"] = {"TFLOP/s": round(tf, 1),
                                               "frac_of_measured_burst": round(tf / bf16_peak, 3),
                                               "frac_of_datasheet_2250": round(tf / BF16_DATASHEET_TFLOPS, 3),
                                               "us": round(t * 1e3, 2)}
        out[f"moe_prefill_t{T}_routing"] = {"us": round(t_r * 1e3, 2), "pairs": P}
    return out


def secondary_prefill(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust):
    """prefill GEMMs (tensor-bound): TFLOP/s against the measured burst and the
    datasheet dense bf16 peak"""
    out = {}
    for c in wl.WORKLOADS.prefill:
        qw = api.qmm_quantize(wl.gen_weight(c.N, c.K, c.seed).to(dev), 64, 4, torch.bfloat16)
        x = wl.gen_x(c.M, c.K, c.seed + 1).to(dev)
        y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)
        t = time_graph(torch, lambda: api.qmm_matmul(x, qw, True, out=y, stream=stream), stream,
                       reps=10, inner=3)
        tf = 2 * c.M * c.N * c.K / (t * 1e-3) / 1e12
        out[c.name] = {"TFLOP/s": round(tf, 1), "frac_of_measured_burst": round(tf / bf16_peak, 3),
                       "frac_of_datasheet_2250": round(tf / BF16_DATASHEET_TFLOPS, 3),
                       "us": round(t * 1e3, 1)}
        del qw, x, y
    return out


def _rotating(torch, call, make, nbytes, stream):
    """per-call device time (ms) of `call(item)` over copies of `make()` whose
    rotation reads more than 3x L2 between reuses"""
    items = [make() for _ in range(copies_for(nbytes))]

    def fn():
        for it in items:
            call(it)
    t = time_graph(torch, fn, stream, reps=10, inner=1) / len(items)
    del items
    return t


def secondary_other_layouts(torch, api, wl, dev, stream, hbm_peak, bf16_peak, bf16_sust):
    """one-token decode in the other weight formats: the [K, N] layout
    (transpose = 0), per-tensor int8, the microscaled modes, and a fused
    three-part projection (4-bit q, 4-bit k, 6-bit v sharing K)"""
    out = {}
    K = 4096
    x = wl.gen_x(1, K, 7001).to(dev)
    for N in (4096, 14336):
        w = wl.gen_weight(K, N, 7002 + N).to(dev)
        qw = api.qmm_quantize(w, 64, 4, torch.bfloat16)  # stored [K, N]
        y = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
        b = K * N // 2 + K * (N // 64) * 4 + 2 * K + 2 * N
        t = _rotating(torch, lambda q: api.qmm_matmul(x, q, False, out=y, stream=stream),
                      lambda: clone_qw(api, qw), b, stream)
        out[f"transpose0_{K}x{N}"] = _gbs(b, t, hbm_peak)
        del w, qw
    for N in (4096, 14336):
        q, prm = api.qmm_quantize_dynamic_int8(wl.gen_weight(N, K, 7003 + N).to(dev))
        y = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
        b = N * K + 2 * K + 2 * N
        t = _rotating(torch, lambda qq: api.qmm_matmul_dynamic_int8(x, qq, prm, out=y, stream=stream),
                      lambda: q.clone(), b, stream)
        out[f"int8_per_tensor_{N}x{K}"] = _gbs(b, t, hbm_peak)
        del q
    N = 14336
    for name, mode in (("mxfp4", api.QMM_MODE_MXFP4), ("mxfp8", api.QMM_MODE_MXFP8), ("nvfp4", api.QMM_MODE_NVFP4)):
        bits, gs = api.MX_PARAMS[mode]
        g = torch.Generator(device=dev)
        g.manual_seed(7004 + mode)
        packed = torch.randint(-2**31, 2**31 - 1, (N, K * bits // 32), dtype=torch.int32, device=dev, generator=g)
        lo, hi = (0x20, 0x50) if mode == api.QMM_MODE_NVFP4 else (110, 130)
        sc = torch.randint(lo, hi, (N, K // gs), dtype=torch.uint8, device=dev, generator=g)
        y = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
        b = N * K * bits // 8 + N * (K // gs) + 2 * K + 2 * N
        t = _rotating(torch, lambda q: api.qmm_matmul(x, q, True, out=y, stream=stream),
                      lambda: api.mx_qweight(packed.clone(), sc.clone(), mode, N, K), b, stream)
        out[f"{name}_{N}x{K}"] = _gbs(b, t, hbm_peak)
        del packed, sc
    parts = [api.qmm_quantize(wl.gen_weight(4096, K, 7010).to(dev), 64, 4, torch.bfloat16),
             api.qmm_quantize(wl.gen_weight(1024, K, 7011).to(dev), 64, 4, torch.bfloat16),
             api.qmm_quantize(wl.gen_weight(1024, K, 7012).to(dev), 64, 6, torch.bfloat16)]
    y = torch.empty(1, 6144, dtype=torch.bfloat16, device=dev)
    b = sum(p.rows * K * p.bits // 8 + p.rows * (K // 64) * 4 for p in parts) + 2 * K + 2 * 6144
    t = _rotating(torch, lambda ps: api.qmm_matmul_parts(x, ps, out=y, stream=stream),
                  lambda: [clone_qw(api, p) for p in parts], b, stream)
    out["fused_parts_q4096_k1024_v1024b6"] = _gbs(b, t, hbm_peak)
    return out


# ---------------------------------------------------------------- oracle arms
def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_decode_inputs(wl, oracle):
    ins = []
    for c in wl.WORKLOADS.decode:
        w = wl.gen_weight(c.N, c.K, c.seed).numpy()
        p, s, b = oracle.quantize(w, oracle.F32, c.group_size, c.bits, oracle.BF16)
        x = wl.storage_numpy(wl.gen_x(c.M, c.K, c.seed + 1))
        ins.append((c, p, s, b, x))
    return ins


def _oracle_step(oracle, ins, threads, frac):
    """one sampled step: the first `frac` of the output rows of each decode call"""
    nbytes = 0.0
    for c, p, s, b, x in ins:
        n = max(1, int(c.N * frac))
        oracle.matmul(x, oracle.BF16, p[:n], s[:n], b[:n], oracle.BF16, n, c.group_size, c.bits,
                      n_threads=threads)
        nbytes += decode_bytes(c.M, c.N, c.K, c.bits, c.group_size) * n / c.N
    return nbytes


def _time_oracle(oracle, ins, threads, seconds):
    """bytes/s of the oracle over repeated sampled decode steps for ~seconds"""
    t0 = time.perf_counter()
    _oracle_step(oracle, ins, threads, 0.01)
    dt = time.perf_counter() - t0
    # size the sample so one pass takes about a tenth of the budget
    frac = min(1.0, max(0.002, 0.01 * (seconds / 10) / max(dt, 1e-4)))
    total_b, reps, t0 = 0.0, 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds and reps < 1000:
        total_b += _oracle_step(oracle, ins, threads, frac)
        reps += 1
    dt = time.perf_counter() - t0
    return total_b / dt / 1e9, frac, reps, dt


def cpu_baseline(wl, seconds):
    """The oracle as it stands on the host's cores, on a bounded sample of the
    decode step: single-threaded (the reported baseline) and over every
    affinity core beside it."""
    import oracle
    ins = _oracle_decode_inputs(wl, oracle)
    threads = cpu_threads()
    v1, f1, r1, d1 = _time_oracle(oracle, ins, 1, seconds / 2)
    vn, fn, rn, dn = _time_oracle(oracle, ins, threads, seconds / 2)
    return {"value": round(v1, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{r1} passes over the first {f1:.2%} of output rows of the 3 decode GEMVs "
                      f"(M=1), fp64 oracle, 1 thread, {d1:.1f} s",
            "all_cores": {"value": round(vn, 5), "unit": "GB/s", "cores": threads,
                          "sample": f"{rn} passes over the first {fn:.2%} of output rows, "
                                    f"{threads} threads, {dn:.1f} s"}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from weight_only_quantized_qmm_b200 import workloads as wl
    threads = cpu_threads()
    ins = _oracle_decode_inputs(wl, oracle)
    frac = 0.02  # bounded sample per step: 2% of the output rows
    for _ in range(max(args.warmup, 3)):
        _oracle_step(oracle, ins, threads, frac)
    steps = args.steps if args.steps_given else 5
    t0 = time.perf_counter()
    total_b = 0.0
    for _ in range(steps):
        total_b += _oracle_step(oracle, ins, threads, frac)
    dt = time.perf_counter() - t0
    value = total_b / dt / 1e9
    sample = (f"each step: first {frac:.0%} of the output rows of the 3 decode GEMVs (M=1), "
              f"fp64 oracle on {threads} threads")
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": round(dt * 1e3 / steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same bytes as the GPU arm)", "impl": "reference",
        "config": {"workload": "decode GEMV M=1, 4-bit affine g64, bf16 x/scales/biases; "
                               "N x K = 4096x4096 + 14336x4096 + 4096x14336 per step",
                   "global_batch": 1, "M": 1, "bits": 4, "group_size": 64},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """A few eager launches of one case, for ncu (no timing output)."""
    import torch

    from weight_only_quantized_qmm_b200 import api
    from weight_only_quantized_qmm_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.profile
    if name == "decode_all":
        # one launch of each decode shape per repetition (per-shape DRAM traffic)
        fns = []
        for c in wl.WORKLOADS.decode:
            qw = api.qmm_quantize(wl.gen_weight(c.N, c.K, c.seed).to(dev), c.group_size, c.bits,
                                  torch.bfloat16)
            x = wl.gen_x(c.M, c.K, c.seed + 1).to(dev)
            fns.append(lambda x=x, qw=qw: api.qmm_matmul(x, qw))

        def fn():
            for f in fns:
                f()
    elif name.startswith("decode"):
        c = [d for d in wl.WORKLOADS.decode if d.name == name][0]
        qw = api.qmm_quantize(wl.gen_weight(c.N, c.K, c.seed).to(dev), c.group_size, c.bits,
                              torch.bfloat16)
        x = wl.gen_x(c.M, c.K, c.seed + 1).to(dev)
        fn = lambda: api.qmm_matmul(x, qw)  # noqa: E731
    elif name.startswith("prefill"):
        c = [d for d in wl.WORKLOADS.prefill if d.name == name][0]
        qw = api.qmm_quantize(wl.gen_weight(c.N, c.K, c.seed).to(dev), c.group_size, c.bits,
                              torch.bfloat16)
        x = wl.gen_x(c.M, c.K, c.seed + 1).to(dev)
        fn = lambda: api.qmm_matmul(x, qw)  # noqa: E731
    elif name.startswith("transpose0_"):
        # one token against the [K, N] layout (quantized along N), K = 4096
        K, N = (int(v) for v in name[len("transpose0_"):].split("x"))
        qw = api.qmm_quantize(wl.gen_weight(K, N, 7002 + N).to(dev), 64, 4, torch.bfloat16)
        x = wl.gen_x(1, K, 7001).to(dev)
        fn = lambda: api.qmm_matmul(x, qw, False)  # noqa: E731
    elif name.split("_")[0] in ("mxfp4", "mxfp8", "nvfp4"):
        # one token against a microscaled [N, K] matrix (random codes and scales)
        mname, shape = name.split("_")
        N, K = (int(v) for v in shape.split("x"))
        mode = {"mxfp4": api.QMM_MODE_MXFP4, "mxfp8": api.QMM_MODE_MXFP8, "nvfp4": api.QMM_MODE_NVFP4}[mname]
        bits, gs = api.MX_PARAMS[mode]
        gen = torch.Generator(device=dev)
        gen.manual_seed(7004 + mode)
        packed = torch.randint(-2**31, 2**31 - 1, (N, K * bits // 32), dtype=torch.int32, device=dev, generator=gen)
        lo, hi = (0x20, 0x50) if mode == api.QMM_MODE_NVFP4 else (110, 130)
        sc = torch.randint(lo, hi, (N, K // gs), dtype=torch.uint8, device=dev, generator=gen)
        mq = api.mx_qweight(packed, sc, mode, N, K)
        x = wl.gen_x(1, K, 7001).to(dev)
        fn = lambda: api.qmm_matmul(x, mq, True)  # noqa: E731
    elif name.startswith("moe_prefill_t"):
        # the gate projection of a MoE prefill (128 experts, top-8, 768 x 2048),
        # routed once on the device, activation rows gathered in schedule order
        T = int(name[len("moe_prefill_t"):])
        E, dff, dm, k = 128, 768, 2048, 8
        g = api.ExpertStack.from_qweight(
            api.qmm_quantize(wl.gen_weight(E * dff, dm, 4600).to(dev), 64, 4, torch.bfloat16), E)
        ids = wl.gen_moe_ids(T, E, k, 4602 + T).to(dev)
        a = wl.gen_x(T, dm, 4603 + T).to(dev)
        ws = api.moe_workspace(T * k, E, dev, n_cols=dm)
        api.qmm_moe_compute_ids_tpe(ids, E, ws)
        og = torch.empty(T * k, dff, dtype=torch.bfloat16, device=dev)
        fn = lambda: api.qmm_moe_gemm_id(a, T, k, 1, ws, g, out=og)  # noqa: E731
    elif name.startswith("moe_down"):
        # the down projection of a one-token MoE step: 8 pairs, K = 768
        case = [d for d in wl.WORKLOADS.moe if d.name == name.replace("moe_down", "moe")][0]
        E, dff, dm, T, k = case.num_experts, case.d_ff, case.d_model, case.tokens, case.top_k
        d = api.ExpertStack.from_qweight(api.qmm_quantize(wl.gen_weight(E * dm, dff, case.seed + 2).to(dev), 64, 4, torch.bfloat16), E)
        h = wl.gen_x(T * k, dff, case.seed + 5).to(dev).reshape(-1)
        ids = wl.gen_moe_ids(T, E, k, case.seed + 4).to(dev).reshape(-1)
        fn = lambda: api.qmm_moe_gemv_id(h, ids, T * k, dff, d)  # noqa: E731
    elif name.startswith("moe"):
        case = [d for d in wl.WORKLOADS.moe if d.name == name][0]
        E, dff, dm, T, k = case.num_experts, case.d_ff, case.d_model, case.tokens, case.top_k
        g = api.ExpertStack.from_qweight(api.qmm_quantize(wl.gen_weight(E * dff, dm, case.seed).to(dev), 64, 4, torch.bfloat16), E)
        u = api.ExpertStack.from_qweight(api.qmm_quantize(wl.gen_weight(E * dff, dm, case.seed + 1).to(dev), 64, 4, torch.bfloat16), E)
        a = wl.gen_x(T, dm, case.seed + 3).to(dev).reshape(-1)
        ids = wl.gen_moe_ids(T, E, k, case.seed + 4).to(dev)
        fn = lambda: api.qmm_moe_gemv_id_gate_up_silu_batched(a, ids, T, k, dm, 0, g, u)  # noqa: E731
    else:
        raise SystemExit(f"unknown profile case {name}")
    for _ in range(args.profile_launches):
        fn()
    torch.cuda.synchronize()
    print(f"profiled {name}: {args.profile_launches} launches")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=16.0,
                    help="oracle CPU baseline budget (half single-thread, half all cores)")
    ap.add_argument("--clock-window", type=float, default=0.3,
                    help="seconds of repeated K-step trials the clock sampler sees")
    ap.add_argument("--profile", default=None,
                    help="run a few launches of one named case (e.g. decode_14336x4096) for ncu")
    ap.add_argument("--profile-launches", type=int, default=3)
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    args.steps_given = args.steps is not None
    if args.steps is None:
        args.steps = 200
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
