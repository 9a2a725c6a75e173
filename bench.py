#!/usr/bin/env python
"""Benchmark of the WKV forward on one batch of the 7B-shaped bf16 workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one wkv_forward_bf16 call over B=8, T=4096, C=4096 (k, v, r, y bf16; fp32
arithmetic; w = exp(U(-6,2)), u ~ U(-2,2), k ~ N(0,3) with 0.1% set to +60, v, r ~ N(0,1);
seeded synthetic inputs, see wkv_inputs.py). Inputs (805 MB) and output (268 MB) are
far larger than the 126 MB L2, so no flush is needed between steps.

Under torchrun (N > 1) every rank runs its own batch (seed = rank) with no collective on
the data path: weak scaling. Timing: CUDA events on the launching stream, barrier and
synchronize on both sides, max over ranks. Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on bounded samples of the same workload
instead, on all of the host's cores (a process pool over channel blocks; rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WKV fwd G(B·T·C)/s and HBM GB/s vs B200 peak at B=8,T=4096,C=4096"
UNIT = "G(B·T·C)/s"
B, T, C = 8, 4096, 4096
BYTES_PER_ELEM = 8          # read k, v, r and write y, 2 bytes each
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0       # B200 HBM3e, nominal
EXPS_PER_ELEM = 3           # two stabilised combines (ex2) and the gate's rcp: MUFU ops
SUSTAINED_S = 1.2           # length of the sustained launch loop
KERNEL = "wkv_fwd_tma_kernel<bf16, gate=1, TT=32, S=3, NW=1>"
KERNEL_SOURCES = ["rwkv_linear_attention_wkv_b200/csrc/wkv_fwd.cu",
                  "rwkv_linear_attention_wkv_b200/csrc/wkv_window.cuh",
                  "rwkv_linear_attention_wkv_b200/csrc/wkv_step.cuh",
                  "rwkv_linear_attention_wkv_b200/csrc/wkv_device.cuh"]
TRAFFIC_FILE = "profiles/wkv_fwd_tma_bf16__B8_T4096_C4096.md"


def kernel_digest() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel sources as they are now; else None."""
    path = os.path.join(ROOT, TRAFFIC_FILE)
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            key, _, val = line.strip()[2:].partition(":")
            fields[key.strip()] = val.strip().strip("`")
    try:
        if fields.get("source_digest") != kernel_digest():
            return None
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def peak_source():
    """Where the HBM denominator comes from, for the JSON line."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return {"file": "MEASURED_PEAKS.json", "hbm_gbs": j.get("hbm_gbs"),
                "how": j.get("how"), "when": j.get("when"), "gpu": j.get("gpu_name")}
    except (OSError, ValueError):
        return {"file": None, "hbm_gbs": FALLBACK_HBM_GBS,
                "how": "fallback: an earlier copy measurement on this GPU type"}


def sfu_peak(sm_max_mhz=None):
    """MUFU operations per second from unit counts: 148 SMs x 16 per clock x the maximum
    SM clock (the nominal figure, kept beside the one pipe_rate measures)."""
    mhz = sm_max_mhz or 1965.0
    return 148 * 16 * mhz * 1e6


def pipe_rate(W, pipe, iters, reps=3):
    """A pipe's throughput measured on this GPU by the library's probe
    (wkv_testing_pipe_rate: 0 = ex2 per second, 1 = fp32 flops per second through packed
    FMA); the best of `reps` runs, or None if the probe fails."""
    import ctypes
    best = None
    for _ in range(reps):
        rate = ctypes.c_double(0.0)
        rc = W.lib.wkv_testing_pipe_rate(pipe, iters, ctypes.byref(rate), None)
        if rc != 0:
            return None
        best = rate.value if best is None else max(best, rate.value)
    return best


def host_cores():
    """Cores this process may run on (what nproc reports)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_block(spec):
    """Pool worker: the fp64 recurrence oracle, unchanged, on one block of channels of one
    batch row, read from the memory-mapped inputs. Returns the elements computed."""
    import numpy as np

    import oracle
    d, b, c0, c1 = spec
    w = np.load(os.path.join(d, "w.npy"))[c0:c1]
    u = np.load(os.path.join(d, "u.npy"))[c0:c1]
    k, v, r = (np.ascontiguousarray(np.load(os.path.join(d, n + ".npy"),
                                            mmap_mode="r")[b:b + 1, :, c0:c1])
               for n in "kvr")
    oracle.wkv_recurrent(w, u, k, v, r)
    return k.size


class OraclePool:
    """The fp64 oracle on all host cores: a process pool (spawn start method, so nothing
    is forked from a process that holds a CUDA context), each task one block of channels
    of one batch row (channels are independent). The inputs go to .npy files in a
    temporary directory that the workers map."""

    def __init__(self, x, cores=None):
        import concurrent.futures as cf
        import multiprocessing as mp

        import numpy as np
        self.cores = cores or host_cores()
        self.dir = tempfile.mkdtemp(prefix="wkv_oracle_")
        for n in ("w", "u", "k", "v", "r"):
            np.save(os.path.join(self.dir, n + ".npy"), getattr(x, n))
        self.B, self.T, self.C = x.B, x.T, x.C
        self.pool = cf.ProcessPoolExecutor(self.cores, mp_context=mp.get_context("spawn"))
        # start every worker and load the oracle library before anything is timed
        list(self.pool.map(_oracle_block, [(self.dir, 0, 0, 1)] * self.cores))

    def run(self, b, c0, c1):
        """Channels [c0, c1) of batch row b, split over the cores. Returns elements done."""
        n = c1 - c0
        pieces = max(1, min(n, 4 * self.cores))
        cuts = [c0 + n * i // pieces for i in range(pieces + 1)]
        specs = [(self.dir, b, cuts[i], cuts[i + 1]) for i in range(pieces)
                 if cuts[i + 1] > cuts[i]]
        return sum(self.pool.map(_oracle_block, specs))

    def close(self):
        import shutil
        self.pool.shutdown()
        shutil.rmtree(self.dir, ignore_errors=True)


class InProcessOracle:
    """The same interface on one core in this process (when the pool cannot run)."""

    def __init__(self, x, note):
        self.x, self.cores, self.note = x, 1, note

    def run(self, b, c0, c1):
        import numpy as np

        import oracle
        x = self.x
        k, v, r = (np.ascontiguousarray(a[b:b + 1, :, c0:c1]) for a in (x.k, x.v, x.r))
        oracle.wkv_recurrent(x.w[c0:c1], x.u[c0:c1], k, v, r)
        return k.size

    def close(self):
        pass


def oracle_runner(x):
    """OraclePool on all cores, else InProcessOracle with the reason."""
    try:
        return OraclePool(x)
    except Exception as e:  # noqa: BLE001 - report, do not lose the line
        return InProcessOracle(x, f"process pool unavailable ({type(e).__name__}: {e})")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_indices):
        self.gpu_indices = gpu_indices
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    idx = int(parts[0])
                    sm, smax = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                if self.gpu_indices is not None and idx not in self.gpu_indices:
                    continue
                rows.append((sm, smax, parts[5:9]))
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for _, _, flags in rows for n, f in zip(names, flags)
                          if f.lower().startswith("active")})
        loaded = [r for r in rows if r[0] > 0.5 * r[1]] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def rank_batch(rank, Bn=B, Tn=T, Cn=C):
    """The batch one rank works on: the 7B-shaped bf16 workload's distributions, seeded by
    the rank, so every rank has its own independent batch (weak scaling, no collective on
    the data path)."""
    import wkv_inputs
    return wkv_inputs.long_bf16(seed=rank, B=Bn, T=Tn, C=Cn)


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks (identity without dist)."""
    if dist is None:
        return [float(x) for x in values]
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_rate(world, elems_per_rank, steps, elapsed_ms):
    """Whole-job throughput in G elements per second: every rank processed its own batch
    `steps` times; the job took the slowest rank's time."""
    return world * elems_per_rank * steps / (elapsed_ms / 1e3) / 1e9


def visible_gpu_indices(n):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return [int(x) for x in vis.split(",")][:n]
        except ValueError:
            return None
    return list(range(n))


def cpu_oracle_rate(x, budget_s=20.0):
    """fp64 recurrence oracle over whole batch rows of the workload, on all host cores,
    until the wall-clock budget is spent (at least one row). Returns (elements per second,
    rows done, cores, note). If the process pool cannot be used (e.g. no room for its
    input files), one row in this process on one core instead, with the reason in note."""
    pool = oracle_runner(x)
    if not isinstance(pool, OraclePool):
        budget_s = 0.0  # one row on one core
    try:
        rows = elems = 0
        t0 = time.perf_counter()
        while rows < x.B:
            elems += pool.run(rows, 0, x.C)
            rows += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
    finally:
        pool.close()
    return elems / dt, rows, pool.cores, getattr(pool, "note", None)


def run_reference(args, rank, world):
    """The oracle as it stands, timed on all of this host's cores."""
    if rank != 0:
        return
    import numpy as np

    import wkv_inputs
    x = wkv_inputs.long_bf16(seed=0, B=1)      # one batch row; steps sample channels of it
    pool = oracle_runner(x)
    try:
        # Size each step so that warm-up + timed steps take about a minute in total.
        t0 = time.perf_counter()
        probe_c = 16 * pool.cores
        pool.run(0, 0, probe_c)
        per_chan = (time.perf_counter() - t0) / probe_c
        budget = 60.0 / max(1, args.steps + args.warmup)
        nchan = int(max(min(x.C, pool.cores), min(x.C, budget / per_chan)))
        g = np.random.Generator(np.random.PCG64(1))
        times = []
        for s in range(args.warmup + args.steps):
            c0 = int(g.integers(0, x.C - nchan + 1))
            t0 = time.perf_counter()
            pool.run(0, c0, c0 + nchan)
            if s >= args.warmup:
                times.append(time.perf_counter() - t0)
    finally:
        pool.close()
    elems = nchan * x.T
    total = sum(times)
    value = elems * len(times) / total / 1e9
    how = ("process pool over channel blocks" if isinstance(pool, OraclePool)
           else f"in this process: {pool.note}")
    sample = (f"per step {nchan} channels x {x.T} tokens of batch row 0 of the B=8,T=4096,"
              f"C=4096 bf16 workload; fp64 recurrence on {pool.cores} host cores ({how})")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "WKV forward, B=8 T=4096 C=4096 (oracle on a sample)",
                   "B": B, "T": T, "C": C, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import rwkv_linear_attention_wkv_b200 as W
    import wkv_inputs

    dist = None
    if world > 1:
        import torch.distributed as dist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    Bn, Tn = args.batch, args.seq or T
    ELEMS = Bn * Tn * C
    x = rank_batch(rank, Bn, Tn)

    def to_bf16(bits, pin=False):
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        return t.pin_memory() if pin else t.to(dev)

    w = torch.from_numpy(x.w).to(dev)
    u = torch.from_numpy(x.u).to(dev)
    k, v, r = (to_bf16(x.bits[n]) for n in "kvr")
    y = torch.empty_like(k)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        W.wkv_forward_bf16(w, u, k, v, r, y=y)
    if W.wkv_stream_status() != 0:
        raise RuntimeError("device-side error during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(visible_gpu_indices(world) if rank == 0 else None)
    barrier()
    if rank == 0:
        sampler.__enter__()
    for i in range(args.steps):
        starts[i].record(stream)
        W.wkv_forward_bf16(w, u, k, v, r, y=y)
        ends[i].record(stream)
    barrier()
    if rank == 0:
        sampler.__exit__(None, None, None)
    if W.wkv_stream_status() != 0:
        raise RuntimeError("device-side error during the timed region")
    per_launch = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    elapsed_ms, launch_ms = max_over_ranks(
        [starts[0].elapsed_time(ends[-1]), statistics.mean(per_launch)], dist, dev)
    value = aggregate_rate(world, ELEMS, args.steps, elapsed_ms)

    # Sustained: back-to-back launches for at least SUSTAINED_S seconds (the power cap and
    # the clock it settles at show over such a loop, not over a short burst), with its
    # own clock record.
    n_sus = max(args.steps, int(SUSTAINED_S / (launch_ms / 1e3)) + 1)
    sus_sampler = ClockSampler(visible_gpu_indices(world) if rank == 0 else None)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    barrier()
    if rank == 0:
        sus_sampler.__enter__()
    s0.record(stream)
    for _ in range(n_sus):
        W.wkv_forward_bf16(w, u, k, v, r, y=y)
    s1.record(stream)
    barrier()
    if rank == 0:
        sus_sampler.__exit__(None, None, None)
    if W.wkv_stream_status() != 0:
        raise RuntimeError("device-side error during the sustained loop")
    (sus_ms,) = max_over_ranks([s0.elapsed_time(s1)], dist, dev)

    # End to end through the public API: pinned host k, v, r -> device, forward, y -> host,
    # every step. Steps are pipelined over two device buffer sets and three streams (copy
    # in, compute, copy out): PCIe is full duplex, so one step's inputs go up while the
    # previous step's output comes down. A set's inputs are overwritten only after the
    # kernel that read them has finished, and its y only after it has been copied out.
    e2e_steps = max(3, min(args.steps, 20))
    hk, hv, hr = (to_bf16(x.bits[n], pin=True) for n in "kvr")
    hy = torch.empty(hk.shape, dtype=torch.bfloat16).pin_memory()
    bufs = [tuple(torch.empty_like(k) for _ in range(4)) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    consumed = [None, None]  # set j's inputs read by its last kernel
    drained = [None, None]   # set j's y copied to the host

    def e2e_step(i):
        j = i % 2
        dk, dv, dr, dy_ = bufs[j]
        if consumed[j] is not None:
            s_in.wait_event(consumed[j])
        with torch.cuda.stream(s_in):
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dr.copy_(hr, non_blocking=True)
        loaded = torch.cuda.Event()
        loaded.record(s_in)
        stream.wait_event(loaded)
        if drained[j] is not None:
            stream.wait_event(drained[j])
        W.wkv_forward_bf16(w, u, dk, dv, dr, y=dy_, stream=stream)
        done = torch.cuda.Event()
        done.record(stream)
        consumed[j] = done
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            hy.copy_(dy_, non_blocking=True)
        out = torch.cuda.Event()
        out.record(s_out)
        drained[j] = out

    def e2e_drain():
        for ev in drained:
            if ev is not None:
                stream.wait_event(ev)

    for i in range(2):
        e2e_step(i)
    e2e_drain()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    e2e_drain()
    e1.record(stream)
    barrier()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], dist, dev)
    e2e_value = aggregate_rate(world, ELEMS, e2e_steps, e2e_ms)
    assert np.array_equal(hy.view(torch.int16).numpy(), y.view(torch.int16).cpu().numpy()), \
        "end-to-end result differs from the device-resident run"

    if rank != 0:
        return
    peak, peak_kind = hbm_peak()
    clocks = sampler.summary()
    sus_clocks = sus_sampler.summary()
    algo_bytes = ELEMS * BYTES_PER_ELEM
    achieved = algo_bytes / (launch_ms / 1e3) / 1e9
    # Roofline: max(bytes / HBM peak, MUFU operations / MUFU peak) against the mean launch.
    # The MUFU peak is measured now, on this GPU (ex2 chains on every SM, ~20 ms a run);
    # the unit-count figure is kept beside it.
    exps = EXPS_PER_ELEM * ELEMS
    sfu_nominal = sfu_peak(clocks.get("sm_max_mhz"))
    sfu_measured = pipe_rate(W, 0, 40000)
    sfu = sfu_measured if sfu_measured else sfu_nominal
    t_hbm_ms = algo_bytes / (peak * 1e9) * 1e3
    t_sfu_ms = exps / sfu * 1e3
    traffic = measured_traffic()
    sus_launch_ms = sus_ms / n_sus
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, rows, cores, note = cpu_oracle_rate(x, budget_s=20.0)
        how = (f"process pool over channel blocks on {cores} host cores" if note is None
               else f"1 thread: {note}")
        cpu = {"value": rate / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{rows} of {Bn} batch rows ({rows} x {Tn} x 4096 elements) of the "
                         f"same inputs, fp64 recurrence, {how}"}
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "storage_dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"WKV forward bf16 in/out, B={Bn} T={Tn} C=4096 (7B-shaped, "
                               "k spikes of +60), one batch per GPU",
                   "B": Bn, "T": Tn, "C": C, "storage": "bf16 k, v, r, y",
                   "arithmetic": "fp32 (w, u fp32)", "global_batch": Bn * world,
                   "seq_len": Tn, "parallelism": f"dp{world} (independent batches)",
                   "l2": f"inputs {3 * ELEMS * 2 / 1e6:.0f} MB + output {ELEMS * 2 / 1e6:.0f} MB "
                         "per step > 126 MB L2; no flush",
                   "kernel": KERNEL},
        "roofline": {"bound": "hbm" if t_hbm_ms >= t_sfu_ms else "sfu",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": max(t_hbm_ms, t_sfu_ms) / launch_ms,
                     "traffic": traffic,
                     "traffic_source": ("ncu dram__bytes_read.sum + dram__bytes_write.sum "
                                        f"from {TRAFFIC_FILE} (taken on these kernel sources)"
                                        if traffic is not None else None),
                     "peak_kind": peak_kind, "peak_source": peak_source(),
                     "frac_of_spec_8TBs": achieved / SPEC_HBM_GBS,
                     "algorithmic_bytes_per_launch": algo_bytes,
                     "hbm_time_ms": t_hbm_ms, "hbm_frac": t_hbm_ms / launch_ms,
                     "exps": exps, "sfu_peak_per_s": sfu,
                     "sfu_peak_kind": ("measured: ex2.approx chains on every SM, best of 3 "
                                       "runs after the timed region (wkv_testing_pipe_rate)"
                                       if sfu_measured else
                                       "unit counts: 148 SMs x 16 MUFU/clk x max SM clock"),
                     "sfu_peak_nominal_per_s": sfu_nominal,
                     "sfu_time_ms": t_sfu_ms, "sfu_frac": t_sfu_ms / launch_ms,
                     "launch_ms": launch_ms},
        "sustained": {"launches": n_sus, "seconds": sus_ms / 1e3,
                      "ms_per_launch": sus_launch_ms,
                      "value": aggregate_rate(world, ELEMS, n_sus, sus_ms),
                      "achieved_GBps": algo_bytes / (sus_launch_ms / 1e3) / 1e9,
                      "frac": algo_bytes / (sus_launch_ms / 1e3) / 1e9 / peak,
                      "clocks": sus_clocks},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": 3 * ELEMS * 2, "d2h_bytes_per_step": ELEMS * 2,
                "steps": e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    print(json.dumps(out), flush=True)


def _time_loop(fn, steps, warmup, stream):
    """Mean milliseconds per call of fn over `steps` calls after `warmup` (CUDA events)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_workload(args):
    """The other workloads the operator is checked on, measured on one GPU (one JSON line
    each; the headline line above is the bf16 forward)."""
    import numpy as np
    import torch

    import rwkv_linear_attention_wkv_b200 as W
    import wkv_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peak, peak_kind = hbm_peak()

    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    def line(name, work, ms, elems, algo_bytes, extra=None):
        gbs = algo_bytes / (ms / 1e3) / 1e9
        out = {"workload": name, "work": work, "ms": ms,
               "G_elem_per_s": elems / (ms / 1e3) / 1e9, "algorithmic_bytes": algo_bytes,
               "achieved_GBps": gbs, "hbm_peak_GBps": peak, "peak_kind": peak_kind,
               "frac": gbs / peak}
        out.update(extra or {})
        print(json.dumps(out), flush=True)

    if args.workload == "train_169m":
        x = wkv_inputs.training_shape(seed=0)
        w, u, k, v, r, dy = (d(a) for a in (x.w, x.u, x.k, x.v, x.r, x.dy))
        n = x.B * x.T * x.C
        y = torch.empty_like(k)
        ms = _time_loop(lambda: W.wkv_forward(w, u, k, v, r, y=y), args.steps, args.warmup, stream)
        line("train_169m", "forward fp32 16x1024x768 (streaming kernel)", ms, n, 16 * n)
        ws = torch.empty(W.wkv_backward_workspace_bytes(x.B, x.T, x.C), dtype=torch.uint8,
                         device=dev)
        out = {nm: torch.empty_like(k) for nm in ("dk", "dv", "dr")}
        out["dw"] = torch.empty(x.C, device=dev)
        out["du"] = torch.empty(x.C, device=dev)
        ms = _time_loop(lambda: W.wkv_backward(w, u, k, v, r, dy, workspace=ws, out=out),
                        args.steps, args.warmup, stream)
        line("train_169m", "backward fp32 16x1024x768 (dk, dv, dr, dw, du)", ms, n, 28 * n)
        # the same through an entering and a leaving state (one piece of a longer sequence)
        g = np.random.Generator(np.random.PCG64(1))
        st = (d(g.standard_normal((x.B, x.C)).astype(np.float32)),
              d(g.uniform(0.5, 2.0, (x.B, x.C)).astype(np.float32)),
              d(g.normal(0.0, 2.0, (x.B, x.C)).astype(np.float32)))
        _, st1 = W.wkv_forward_state(w, u, k, v, r, state=st)
        gs = (d(g.standard_normal((x.B, x.C)).astype(np.float32)),
              d(g.standard_normal((x.B, x.C)).astype(np.float32)), st1[2])
        for nm in ("da0", "db0", "dp0"):
            out[nm] = torch.empty((x.B, x.C), device=dev)
        ms = _time_loop(lambda: W.wkv_backward_state(w, u, k, v, r, dy, state=st, grad_state=gs,
                                                     workspace=ws, out=out),
                        args.steps, args.warmup, stream)
        line("train_169m", "backward_state fp32 16x1024x768 (with initial state and final-state "
             "gradients)", ms, n, 28 * n + 36 * x.B * x.C)
        # The checkpointed pair: the forward also writes the backward's chunk checkpoints
        # (one float4 per channel per 16 tokens: 1 byte per element), the backward reads
        # them instead of forming them in a pass of its own.
        ms_f = _time_loop(lambda: W.wkv_forward_checkpointed(w, u, k, v, r, y=y, workspace=ws),
                          args.steps, args.warmup, stream)
        line("train_169m", "forward_checkpointed fp32 16x1024x768 (y and the backward's "
             "checkpoints)", ms_f, n, 17 * n)
        ms_b = _time_loop(lambda: W.wkv_backward_checkpointed(w, u, k, v, r, dy, ws, out=out),
                          args.steps, args.warmup, stream)
        line("train_169m", "backward_checkpointed fp32 16x1024x768 (dk, dv, dr, dw, du; "
             "checkpoints read)", ms_b, n, 29 * n)

        def step_plain():
            W.wkv_forward(w, u, k, v, r, y=y)
            W.wkv_backward(w, u, k, v, r, dy, workspace=ws, out=out)

        def step_ckpt():
            W.wkv_forward_checkpointed(w, u, k, v, r, y=y, workspace=ws)
            W.wkv_backward_checkpointed(w, u, k, v, r, dy, ws, out=out)

        ms_p = _time_loop(step_plain, args.steps, args.warmup, stream)
        ms_c = _time_loop(step_ckpt, args.steps, args.warmup, stream)
        line("train_169m", "training step: wkv_forward + wkv_backward", ms_p, n, 16 * n + 28 * n)
        line("train_169m", "training step: wkv_forward_checkpointed + wkv_backward_checkpointed",
             ms_c, n, 17 * n + 29 * n)
        # The same step captured once in a CUDA graph and replayed: no host work and no
        # launch gaps between the kernels.
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step_ckpt()
        ms_g = _time_loop(graph.replay, args.steps, args.warmup, stream)
        line("train_169m", "training step: the checkpointed pair replayed from a CUDA graph",
             ms_g, n, 17 * n + 29 * n)
        del graph
    elif args.workload == "long_ctx":
        x = wkv_inputs.long_context(seed=0, T=args.seq or 32768)
        w, u, k, v, r = (d(a) for a in (x.w, x.u, x.k, x.v, x.r))
        n = x.B * x.T * x.C
        y = torch.empty_like(k)
        st = tuple(torch.empty((x.B, x.C), device=dev) for _ in range(3))
        ms = _time_loop(lambda: W.wkv_forward_state(w, u, k, v, r, y=y, state_out=st),
                        args.steps, args.warmup, stream)
        line("long_ctx", f"forward_state fp32 1x{x.T}x4096 (chunked kernel, final state)", ms, n,
             16 * n + 12 * x.B * x.C)
    elif args.workload == "decode":
        dd = wkv_inputs.decode_batch(seed=0, N=args.decode_seqs)
        n = dd.N * dd.L * dd.C
        w, u = d(dd.w), d(dd.u)
        a, b, p = d(dd.a), d(dd.b), d(dd.p)
        k, v, r = (d(t) for t in dd.step(0))
        y = torch.empty_like(k)
        ms = _time_loop(lambda: W.wkv_decode_step(w, u, k, v, r, a, b, p, y=y), args.steps,
                        args.warmup, stream)
        line("decode", f"decode step fp32 {dd.N} seq x 32 layers x 4096 (state in place)", ms, n,
             40 * n, {"tokens_per_s": dd.N / (ms / 1e3)})
        # S tokens per call with the state kept on chip (wkv_decode_steps): per token
        # 16 bytes per state (k, v, r in, y out) plus the state once per call (24 / S).
        S = args.seq or 64
        ks = torch.empty((S,) + tuple(k.shape), device=dev)
        vs, rs = torch.empty_like(ks), torch.empty_like(ks)
        for s_ in range(S):
            kk, vv, rr = dd.step(s_)
            ks[s_].copy_(torch.from_numpy(kk))
            vs[s_].copy_(torch.from_numpy(vv))
            rs[s_].copy_(torch.from_numpy(rr))
        ys = torch.empty_like(ks)
        steps = max(3, args.steps // S)
        ms = _time_loop(lambda: W.wkv_decode_steps(w, u, ks, vs, rs, a, b, p, y=ys), steps,
                        3, stream)
        line("decode", f"decode_steps fp32 {dd.N} seq x 32 layers x 4096, {S} tokens per call "
             "(state on chip between tokens); ms and rates per token", ms / S, n,
             int(16 * n + 24 * n / S), {"tokens_per_s": dd.N * S / (ms / 1e3),
                                        "ms_per_call": ms, "tokens_per_call": S})
    elif args.workload == "rwkv7":
        T7 = args.seq or 4096
        x = wkv_inputs.rwkv7_inputs(8, T7, 64, seed=0)
        t = {nm: d(getattr(x, nm)) for nm in ("r", "w", "k", "v", "a", "b")}
        s0 = d(x.S0)
        y = torch.empty_like(t["k"])
        s1 = torch.empty_like(s0)
        n = x.B * x.T * x.H * x.N
        ms = _time_loop(lambda: W.wkv7_forward(*(t[nm] for nm in "rwkvab"), state=s0, y=y,
                                               state_out=s1), args.steps, args.warmup, stream)
        # FP32 work per token and head: sa (N^2 FMA), update (N^2 FMUL + 2 N^2 FMA), y (N^2 FMA)
        flops = 9 * x.N * x.N * x.B * x.T * x.H
        # FP32 peak from unit counts: 148 SMs x 128 FMA lanes x 2 x the max SM clock (74.4
        # TFLOP/s), and measured now on this GPU (packed fp32x2 FMA chains on every SM)
        alu_peak = 148 * 128 * 2 * 1.965e9
        alu_measured = pipe_rate(W, 1, 200000) or alu_peak
        line("rwkv7", f"RWKV-7 recurrence fp32 8x{x.T}x64 heads x 64 (state in and out)", ms, n,
             28 * n + 8 * x.B * x.H * x.N * x.N,
             {"flops": flops, "achieved_TFLOPs": flops / (ms / 1e3) / 1e12,
              "alu_peak_TFLOPs": alu_peak / 1e12,
              "alu_peak_measured_TFLOPs": alu_measured / 1e12,
              "alu_frac": flops / (ms / 1e3) / alu_peak,
              "alu_frac_of_measured": flops / (ms / 1e3) / alu_measured})
    elif args.workload == "mstate":
        # Matrix-valued state without the delta term: the chunked tensor-core kernel and the
        # token-by-token recurrence kernel on the same inputs (a = b = 0).
        T7 = args.seq or 4096
        x = wkv_inputs.rwkv7_inputs(8, T7, 64, seed=0)
        x.a[...] = 0.0
        x.b[...] = 0.0
        t = {nm: d(getattr(x, nm)) for nm in ("r", "w", "k", "v", "a", "b")}
        s0 = d(x.S0)
        y = torch.empty_like(t["k"])
        s1 = torch.empty_like(s0)
        n = x.B * x.T * x.H * x.N
        # per token and head: A (N L), A V (N L / 2 on average), R~ S0^T (N^2), V^T K~
        # (N^2) multiply-adds with L = N = 64 as 3 tf32 products each
        tc_flops = 3 * 2 * (64 * 64 + 64 * 32 + 64 * 64 + 64 * 64) * x.B * x.T * x.H
        ms = _time_loop(lambda: W.wkv_mstate_forward(*(t[nm] for nm in "rwkv"), state=s0, y=y,
                                                     state_out=s1), args.steps, args.warmup,
                        stream)
        line("mstate", f"matrix-state WKV fp32 8x{x.T}x64 heads x 64, chunked on tcgen05 "
             "(3 x tf32 products)", ms, n, 20 * n + 8 * x.B * x.H * x.N * x.N,
             {"tf32_flops_issued": tc_flops,
              "tf32_TFLOPs": tc_flops / (ms / 1e3) / 1e12})
        ms = _time_loop(lambda: W.wkv7_forward(*(t[nm] for nm in "rwkvab"), state=s0, y=y,
                                               state_out=s1), args.steps, args.warmup, stream)
        line("mstate", f"same inputs through the recurrence kernel (wkv7_forward, a = b = 0)",
             ms, n, 28 * n + 8 * x.B * x.H * x.N * x.N)
    else:
        raise SystemExit(f"unknown workload {args.workload}")
    if W.wkv_stream_status() != 0:
        raise RuntimeError("device-side error")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=B,
                    help="batch rows per GPU (default 8, the measured workload; smaller "
                         "values are for profiler captures)")
    ap.add_argument("--workload", default="bf16_7b",
                    choices=["bf16_7b", "train_169m", "long_ctx", "decode", "rwkv7", "mstate"],
                    help="bf16_7b (default) prints the benchmark line; the others print "
                         "measurements of the other workloads, one GPU")
    ap.add_argument("--decode-seqs", type=int, default=256,
                    help="sequences of the decode workload (default 256, the measured one; "
                         "fewer for profiler captures)")
    ap.add_argument("--seq", type=int, default=None,
                    help="tokens per sequence (default: the workload's own, 4096 for the "
                         "benchmark; shorter sequences keep the occupancy of the full case "
                         "for profiler captures); for decode, tokens per wkv_decode_steps "
                         "call (default 64)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 runs under torchrun (one process per GPU)")
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        try:
            run_ours(args, rank, world, local_rank)
        finally:
            dist.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload != "bf16_7b":
        run_workload(args)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
