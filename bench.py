#!/usr/bin/env python
"""Benchmark of the Newton-solved diag-mix sLSTM training step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--newton-mode tol|fixed] [--newton-iters K_N] [--impl reference]

One step = the whole hot path on one batch of synthetic input already in HBM:
  input projection GEMM  ->  Newton solve to the workload's tolerance (the
  decoupled initial guess, then iterations with fused residual, Jacobian,
  blocked scan and update until max |F| / (1 + |s|) <= tol)  ->  backward
  (fused adjoint scan + cell VJP, dR/db reduction, dx and dW_x GEMMs).
Metric: B*T*d_h elements per second for forward + backward (the JSON
`value`), with the forward alone reported beside it.  Under torchrun each
rank runs its own replica of the workload (independent batches, no data-path
collective): `value` is the sum over ranks of elements divided by the slowest
rank's device time.

`roofline` is for the step's dominant kernel, newton_iter (the Newton
iteration: 48 algorithmic bytes per element per launch), over the average
duration of its working launches, taken from CUDA events that the library
records on its stream around each of its launches inside the timed steps; the
guess launch and the whole solve are reported beside it.

With no flags the line also carries, measured in the same run on rank 0: the
long-sequence workload's forward (B=4, T=65536, d=2048: input projection and
the converged Newton solve, and the fixed K=4 solve) with newton_iter's HBM
roofline fraction, the same solve at T = 4096 and 16384 (newton_sweep), and
the scan_block4 sweep at B=4, d=2048 over T = 4096, 16384, 65536.

`--impl reference` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of lanes of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nonlinear_rnn_pararnn_b200.workloads import (ORDER, WORKLOADS, as_f64, make_head_R, make_inputs,  # noqa: E402
                                                   scaled)

METRIC = "sLSTM Newton solve elems/s (B*T*d_h/s, fwd+bwd)"
METRIC_FWD = "sLSTM Newton solve elems/s (B*T*d_h/s, fwd)"
UNIT = "elems/s"
DEFAULT_WORKLOAD = "slstm_bf16_train_b8_t8192_d1024"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device=None):
    """Element-wise max of a list of timings over all ranks (identity when
    not distributed).  Only timings cross ranks, never data."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate(elems_per_rank, n_ranks, ms_per_step_max):
    """Whole-job throughput: every rank's elements over the slowest rank's time."""
    return n_ranks * elems_per_rank / (ms_per_step_max / 1e3)


# ---------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def _sample_lanes(w, n_lanes, seed):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(0, w.B)), int(rng.integers(0, w.d_h))) for _ in range(n_lanes)]


def oracle_lane(w, inp, b, j, newton):
    """The fp64 oracle, as it stands, on one (b, j) lane of the workload: its
    input-projection rows, the Newton solve (newton = ("tol", cap, sweeps) or
    ("fixed", K, sweeps), from the decoupled guess with that many refinement
    sweeps), BPTT and the lane's
    contributions to dx and dW_x."""
    import oracle
    bias = as_f64(inp["bias"])
    xb = as_f64(inp["x"][b])                                        # (T, d_in)
    rows = [g * w.d_h + j for g in range(4)]
    Wr = as_f64(inp["Wx"][rows])                                    # (4, d_in)
    P = oracle.gemm(xb, Wr, tb=True, bias=bias[:, j])[None]         # (1, T, 4)
    R = as_f64(inp["R"][:, j])[None]
    s0 = np.zeros((1, 4))
    mode, k, sweeps = newton
    S, st = oracle.newton(P, R, s0, w.forget, max_iters=k, fixed=(mode == "fixed"), tol=w.tol, sweeps=sweeps)
    dH = as_f64(inp["dH"][b, :, j])[None]
    dP, dR, db, ds0 = oracle.bptt(P, R, s0, S, dH, w.forget)
    oracle.gemm(dP[0], Wr)                                          # this lane's share of dx
    oracle.gemm(np.ascontiguousarray(dP[0].T), np.ascontiguousarray(xb.T), tb=True)  # its dW_x rows
    return st["iters"]


_POOL_STATE = {}
_SHARED_KEYS = ("x", "Wx", "R", "bias", "dH")


def _share_inputs(inp):
    """Copy the workload's input tensors into shared memory once, so that the
    oracle's worker processes read them instead of each drawing its own copy.
    Returns (segments to keep alive, metadata for the workers)."""
    import torch
    from multiprocessing import shared_memory
    segs, meta = [], {}
    for k in _SHARED_KEYS:
        t = inp[k].contiguous()
        raw = t.view(torch.int16) if t.dtype == torch.bfloat16 else t
        arr = raw.numpy()
        shm = shared_memory.SharedMemory(create=True, size=max(1, arr.nbytes))
        np.ndarray(arr.shape, dtype=arr.dtype, buffer=shm.buf)[...] = arr
        segs.append(shm)
        meta[k] = (shm.name, tuple(t.shape), str(t.dtype))
    return segs, meta


def _pool_init(name, T, meta):
    import torch
    from multiprocessing import shared_memory
    w = WORKLOADS[name] if T == WORKLOADS[name].T else scaled(WORKLOADS[name], T=T)
    inp, keep = {}, []
    for k, (shm_name, shape, dt) in meta.items():
        shm = shared_memory.SharedMemory(name=shm_name)
        keep.append(shm)
        if dt == "torch.bfloat16":
            arr = np.ndarray(shape, dtype=np.int16, buffer=shm.buf)
            inp[k] = torch.from_numpy(arr).view(torch.bfloat16)
        else:
            inp[k] = torch.from_numpy(np.ndarray(shape, dtype=np.float32, buffer=shm.buf))
    _POOL_STATE.update(w=w, inp=inp, keep=keep)


def _pool_lane(task):
    b, j, newton = task
    return oracle_lane(_POOL_STATE["w"], _POOL_STATE["inp"], b, j, newton)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_timing(w, inp, newton, single_lanes, seed=0, pool=None, pool_lanes=0):
    """Elements per second of the oracle on sampled lanes: on one core in this
    process, and (pool given) on every core with one worker process per core,
    each lane one task.  Returns a dict."""
    out = {}
    oracle_lane(w, inp, 0, 0, newton)                               # warm the oracle library
    lanes = _sample_lanes(w, single_lanes, seed)
    t0 = time.perf_counter()
    iters = [oracle_lane(w, inp, b, j, newton) for b, j in lanes]
    dt = time.perf_counter() - t0
    out["single"] = {"value": single_lanes * w.T / dt, "cores": 1, "seconds": dt, "lanes": single_lanes,
                     "newton_iters": iters}
    if pool is not None and pool_lanes:
        lanes = _sample_lanes(w, pool_lanes, seed + 1)
        pool.map(_pool_lane, [(0, 0, newton)] * pool.cores)                  # every worker warmed
        t0 = time.perf_counter()
        pool.map(_pool_lane, [(b, j, newton) for b, j in lanes])
        dt = time.perf_counter() - t0
        out["all_cores"] = {"value": pool_lanes * w.T / dt, "cores": pool.cores, "seconds": dt,
                            "lanes": pool_lanes}
    return out


class OraclePool:
    """One spawned worker process per host core (at most 64), reading the
    workload's inputs from shared memory.  Spawned, not forked, so that it is
    safe whether or not this process has touched the GPU."""

    def __init__(self, w, inp):
        import concurrent.futures
        import multiprocessing as mp
        self.cores = min(host_cores(), 64)
        self.segs, meta = _share_inputs(inp)
        base = w.name.split("_T")[0] if w.name not in WORKLOADS else w.name
        self.ex = concurrent.futures.ProcessPoolExecutor(max_workers=self.cores, mp_context=mp.get_context("spawn"),
                                                         initializer=_pool_init, initargs=(base, w.T, meta))

    def map(self, fn, tasks):
        return list(self.ex.map(fn, tasks))

    def shutdown(self):
        self.ex.shutdown()
        for s in self.segs:
            s.close()
            s.unlink()


def _newton_desc(newton):
    mode, k, sweeps = newton
    it = f"Newton to the workload's tolerance (cap {k})" if mode == "tol" else f"{k} fixed Newton iterations"
    return f"{it} from the decoupled guess with {sweeps} refinement sweeps"


def run_reference(args, w):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    newton = (("tol", w.max_iters) if args.newton_mode == "tol" else ("fixed", args.newton_iters)) + (args.guess_sweeps,)
    inp = make_inputs(w)
    pool = OraclePool(w, inp)
    cores = pool.cores
    lanes = _sample_lanes(w, cores, 99)
    pool.map(_pool_lane, [(b, j, newton) for b, j in lanes])   # warm-up: every worker ready
    for _ in range(args.warmup - 1):
        pool.map(_pool_lane, [(b, j, newton) for b, j in lanes])
    t0 = time.perf_counter()
    pool.map(_pool_lane, [(b, j, newton) for b, j in lanes])
    per_round = time.perf_counter() - t0
    # bounded sample: about a minute of wall time over all timed steps
    rounds = int(max(1, min(args.ref_lanes, 60.0 / max(1e-3, args.steps * per_round))))
    total_t, total_e = 0.0, 0
    for s_ in range(args.steps):
        lanes = _sample_lanes(w, rounds * cores, s_)
        t0 = time.perf_counter()
        pool.map(_pool_lane, [(b, j, newton) for b, j in lanes])
        total_t += time.perf_counter() - t0
        total_e += len(lanes) * w.T
    pool.shutdown()
    value = total_e / total_t
    sample = (f"{rounds * cores} random (b,j) lanes x T={w.T} per step on {cores} worker processes "
              f"({cpu_model()}): fp64 input-projection rows, {_newton_desc(newton)}, "
              f"BPTT, dx/dW_x contributions")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(w.describe(), newton_mode=newton[0], newton_max_iters=newton[1], guess_sweeps=newton[2]),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    from nonlinear_rnn_pararnn_b200 import _lib, api

    ws, rank, local = _dist()
    if ws > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    api._lib.load()

    tol_mode = args.newton_mode == "tol"
    K = w.max_iters if tol_mode else args.newton_iters
    forward_only = args.mode == "forward"
    inp = make_inputs(w)
    pool = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        pool = OraclePool(w, inp)            # spawned workers, started before the GPU work
    x, Wx, R, bias, s0, dH = (inp[k].to(dev) for k in ("x", "Wx", "R", "bias", "s0", "dH"))
    P = torch.empty(w.B, w.T, 4, w.d_h, device=dev)
    S = torch.empty_like(P)
    stats = api.new_stats(dev)
    ws_n = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD, w.B, w.T, 0, w.d_h, dev)
    ws_b = None if args.mode == "forward" else api.workspace(_lib.SLSTM_OP_NEWTON_BACKWARD, w.B, w.T, w.d_in,
                                                               w.d_h, dev)
    grads = {"dx": torch.empty(w.B, w.T, w.d_in, device=dev), "dWx": torch.empty(4 * w.d_h, w.d_in, device=dev),
             "dR": torch.empty(4, w.d_h, device=dev), "db": torch.empty(4, w.d_h, device=dev),
             "ds0": torch.empty(w.B, 4, w.d_h, device=dev)}

    dev_main = {"x": x, "Wx": Wx, "R": R, "bias": bias, "s0": s0, "dH": dH}

    n_launch = newton_launches(args.guess_sweeps, K, tol_mode)   # launches of work of one Newton call

    def step(ev=None, dv=None, gr=None, lev=None):
        dv = dev_main if dv is None else dv
        gr = grads if gr is None else gr
        if ev is not None:
            ev[0].record()
        api.preact_gemm(dv["x"], dv["Wx"], dv["bias"], P=P)
        if ev is not None:
            ev[1].record()
        api.newton_forward(P, dv["R"], dv["s0"], forget=w.forget, max_iters=K, fixed=not tol_mode, tol=w.tol, S=S,
                           stats=stats, ws=ws_n, guess_sweeps=args.guess_sweeps, events=lev)
        if ev is not None:
            ev[2].record()
        if not forward_only:
            api.newton_backward(dv["x"], dv["Wx"], P, dv["R"], dv["s0"], S, dv["dH"], forget=w.forget, out=gr,
                                ws=ws_b)
        if ev is not None:
            ev[3].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    # the library records these around each of its Newton launches (guess,
    # then one per iteration) inside the timed steps
    levs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)] for _ in range(args.steps)]
    for lv in levs:
        for e in lv:
            e.record()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    time.sleep(0.25)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for s_ in range(args.steps):
        step(evs[s_], lev=levs[s_])
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms_total = start.elapsed_time(end)
    ms_gemm = sum(e[0].elapsed_time(e[1]) for e in evs)
    ms_newton = sum(e[1].elapsed_time(e[2]) for e in evs)
    ms_bwd = sum(e[2].elapsed_time(e[3]) for e in evs)
    st = api.read_stats(stats)
    S_finite = bool(torch.isfinite(S).all().item())

    # ---- end to end through the public API from pinned host buffers ----
    # Every step copies its inputs (x, W_x, R, b, s0, dH) host -> device and
    # its results (dW_x, dR, db and the stats record) device -> host.  The
    # copies run on their own streams into double buffers, so step i+1's
    # inputs travel while step i computes; all of them lie inside the timed
    # region, which runs from the first input copy to the last result copy.
    keys_in = ("x", "Wx", "R", "bias", "s0") + (() if forward_only else ("dH",))
    keys_out = ("dWx", "dR", "db") if not forward_only else ()
    host_in = {k: inp[k].pin_memory() for k in keys_in}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    dev_bufs = [dev_main, {k: torch.empty_like(dev_main[k]) for k in keys_in}]
    grad_bufs = [grads, {k: torch.empty_like(v) for k, v in grads.items()}]
    host_out = [{k: torch.empty(grads[k].shape, dtype=grads[k].dtype).pin_memory() for k in keys_out}
                for _ in range(2)]
    host_stats = [torch.empty(stats.shape, dtype=stats.dtype).pin_memory() for _ in range(2)]
    stats_bufs = [torch.empty_like(stats) for _ in range(2)]   # the next step rewrites `stats`
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values()) + host_stats[0].numel()
    comp = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)

    def run_e2e(n):
        """n pipelined steps; returns (start, end) events spanning every copy."""
        in_ready = [torch.cuda.Event() for _ in range(2)]
        in_free = [torch.cuda.Event() for _ in range(2)]
        out_ready = [torch.cuda.Event() for _ in range(2)]
        out_free = [torch.cuda.Event() for _ in range(2)]
        for e in in_free + out_free:
            e.record(comp)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)

        def load(i):
            b = i & 1
            s_in.wait_event(in_free[b])
            with torch.cuda.stream(s_in):
                for k in keys_in:
                    dev_bufs[b][k].copy_(host_in[k], non_blocking=True)
            in_ready[b].record(s_in)

        load(0)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                load(i + 1)
            comp.wait_event(in_ready[b])
            comp.wait_event(out_free[b])
            step(dv=dev_bufs[b], gr=grad_bufs[b])
            stats_bufs[b].copy_(stats)
            in_free[b].record(comp)
            out_ready[b].record(comp)
            s_out.wait_event(out_ready[b])
            with torch.cuda.stream(s_out):
                for k in keys_out:
                    host_out[b][k].copy_(grad_bufs[b][k], non_blocking=True)
                host_stats[b].copy_(stats_bufs[b], non_blocking=True)
            out_free[b].record(s_out)
        comp.wait_stream(s_out)
        t1.record(comp)
        return t0, t1

    run_e2e(2)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e2e_steps = max(2, min(args.steps, 20))
    e_start, e_end = run_e2e(e2e_steps)
    torch.cuda.synchronize()
    ms_e2e = e_start.elapsed_time(e_end) / e2e_steps

    # max over ranks of the device times
    ms_total, ms_e2e, ms_gemm, ms_newton, ms_bwd = max_over_ranks(
        [ms_total, ms_e2e, ms_gemm, ms_newton, ms_bwd], device=dev)
    ms_step = ms_total / args.steps
    elems = w.elems
    value = aggregate(elems, ws, ms_step)
    fwd_ms = (ms_gemm + ms_newton) / args.steps

    hbm, peak_kind = _peaks()
    # The Newton solve is one C call: the guess launch, which runs the decoupled
    # guess and up to GUESS_FUSED_SWEEPS refinement sweeps tile by tile (reads
    # P, writes S: 32 algorithmic B/elem), one launch per further sweep (reads
    # P and h, writes S: 36 B/elem each) and n iterations (read P and the old
    # S, write S: 48 B/elem each); in tolerance mode the launches after
    # convergence return at once.  Its CUDA-event time over the timed region
    # against those bytes.
    n_it = st["iters"]
    sw = args.guess_sweeps
    newton_ms = ms_newton / args.steps
    newton_bytes = elems * solve_bytes_per_elem(n_it, sw)
    solve_gbs = newton_bytes / (newton_ms / 1e3) / 1e9
    # Per launch, from the library's events: the guess launch(es), then the
    # iterations launched one by one (in tolerance mode the first LOOP_FROM;
    # the rest of the cap is one launch that loops on the device and ends with
    # the solve, listed apart with whatever iterations it ran).
    g = guess_launches(sw)
    n_sep = separate_iterations(n_it, tol_mode)
    per_it = [float(np.mean([lv[g + i].elapsed_time(lv[g + i + 1]) for lv in levs])) for i in range(n_sep)]
    guess_ms = [lv[0].elapsed_time(lv[g]) for lv in levs]
    idle_ms = [lv[g + n_sep].elapsed_time(lv[-1]) for lv in levs]
    per_it = max_over_ranks(per_it, device=dev) if per_it else []
    it_ms = float(np.mean(per_it)) if per_it else 0.0
    guess_ms, idle_ms = max_over_ranks([float(np.mean(guess_ms)), float(np.mean(idle_ms))], device=dev)
    # the dominant kernel of the step (largest share of the ncu launch list):
    # newton_iter, 48 algorithmic bytes per element per launch
    achieved = 48.0 * elems / (it_ms / 1e3) / 1e9 if it_ms > 0 else 0.0
    traffic = args.traffic_bytes if args.traffic_bytes else newton_iter_traffic_bytes(elems)
    guess_bytes = 32.0 * elems
    roofline = {"kernel": "newton_iter", "bound": "hbm", "achieved": achieved, "peak": hbm, "peak_kind": peak_kind,
                "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                "algorithmic_bytes_per_launch": 48 * elems, "avg_launch_ms": it_ms,
                "launches_per_step": n_sep, "launch_ms": per_it,
                "timing": "CUDA events the library records on its stream around each launch, over the timed steps",
                "guess_kernel": {"launches_per_step": g, "ms": guess_ms, "algorithmic_bytes": guess_bytes,
                                 "achieved": guess_bytes / (guess_ms / 1e3) / 1e9,
                                 "frac": guess_bytes / (guess_ms / 1e3) / 1e9 / hbm,
                                 "stages_per_tile": 1 + min(sw, GUESS_FUSED_SWEEPS),
                                 "note": "one scan per stage over each tile; issue-bound"},
                "device_loop": {"launches_per_step": n_launch - g - n_sep, "iterations_inside": n_it - n_sep,
                                "ms": idle_ms, "note": "the rest of the iteration cap, one launch looping on the device"},
                "solve": {"ms": newton_ms, "algorithmic_bytes": newton_bytes, "achieved": solve_gbs,
                          "frac": solve_gbs / hbm}}

    cpu = None
    if pool is not None:
        newton = ("tol", w.max_iters, args.guess_sweeps) if tol_mode else ("fixed", K, args.guess_sweeps)
        t = oracle_timing(w, inp, newton, args.cpu_lanes, seed=123, pool=pool,
                          pool_lanes=args.cpu_lanes * pool.cores)
        pool.shutdown()
        cpu = {"value": t["all_cores"]["value"], "unit": UNIT, "cores": t["all_cores"]["cores"], "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"{t['all_cores']['lanes']} random (b,j) lanes x T={w.T} on {t['all_cores']['cores']} "
                         f"worker processes ({t['all_cores']['seconds']:.1f} s): fp64 input-projection rows, "
                         f"{_newton_desc(newton)}, BPTT, dx/dW_x contributions",
               "single_core": {"value": t["single"]["value"], "lanes": t["single"]["lanes"],
                               "seconds": t["single"]["seconds"]}}

    extra = {}
    if rank == 0 and ws == 1 and args.mode == "train" and not args.no_extra and args.seq_len is None:
        del P, S, grads, dev_bufs, grad_bufs, ws_n, ws_b
        torch.cuda.empty_cache()
        extra["long_forward"] = long_forward(args, dev, hbm, peak_kind)
        torch.cuda.empty_cache()
        extra["newton_sweep"] = newton_sweep(args, dev, hbm, peak_kind)
        torch.cuda.empty_cache()
        extra["scan_block4_sweep"] = scan_sweep(args, dev, hbm, peak_kind)

    # kernels launched per step: preact GEMM 1, Newton: the guess, the
    # iterations launched one by one and (tolerance mode) the device loop over
    # the rest of the cap, backward: adjoint 1 + dR/db reduction 1 + 2 GEMMs
    # (+ the split-K sum of the tensor-core path)
    launches_per_step = (1 + n_launch + (0 if forward_only else 4 + (1 if w.dtype == "bf16" else 0)))
    line = {
        "metric": METRIC_FWD if forward_only else METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "operand_dtype": "bf16 x/W_x, fp32 state and scans" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": dict(w.describe(), newton_mode=args.newton_mode, newton_max_iters=K, newton_init="decoupled",
                       guess_sweeps=args.guess_sweeps, gemm_tiles=args.gemm_tiles,
                       l2="inputs larger than L2 (P and S are %.2f GB each)" % (elems * 16 / 1e9),
                       parallelism=f"replicas x{ws}"),
        "fwd": {"value": aggregate(elems, ws, fwd_ms), "unit": UNIT, "ms_per_step": fwd_ms},
        "breakdown_ms_per_step": {"preact_gemm": ms_gemm / args.steps, "newton_forward": ms_newton / args.steps,
                                  "backward": ms_bwd / args.steps},
        "newton_stats_last_step": {"iters": st["iters"], "converged": st["converged"], "diverged": st["diverged"],
                                   "error": st["error"], "max_scaled_F": st["max_scaled_F"],
                                   "init_max_scaled_F": st["init_max_scaled_F"], "S_finite": S_finite},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate(elems, ws, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    line.update(extra)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def scan_sweep(args, dev, hbm, peak_kind, T_list=None):
    """scan_block4 alone: B=4, d=2048, T swept; 96 algorithmic bytes per
    element (read A 64, b 16, write y 16).  Inputs drawn on the device from a
    seeded generator (values only set the timing's data, not checked here)."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    B, d = 4, 2048
    sweep = []
    for T in (T_list or [int(v) for v in args.scan_T.split(",")]):
        g = torch.Generator(device=dev)
        g.manual_seed(T)
        A = torch.rand(B, T, 4, 4, d, generator=g, device=dev) * 0.6 - 0.3
        b = torch.randn(B, T, 4, d, generator=g, device=dev)
        y = torch.empty_like(b)
        ws = api.workspace(_lib.SLSTM_OP_SCAN_BLOCK4, B, T, 0, d, dev)
        for _ in range(args.warmup):
            api.scan_block4(A, b, None, y=y, ws=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(3, min(args.steps, 20))
        e0.record()
        for _ in range(n):
            api.scan_block4(A, b, None, y=y, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        elems = B * T * d
        gbs = elems * 96 / (ms / 1e3) / 1e9
        sweep.append({"workload": f"scan_block4_b{B}_t{T}_d{d}", "T": T, "ms": ms, "elems_per_s": elems / (ms / 1e3),
                      "achieved_GBs": gbs, "peak": hbm, "peak_kind": peak_kind, "frac": gbs / hbm, "steps": n})
        del A, b, y, ws
        torch.cuda.empty_cache()
    return sweep


def long_forward(args, dev, hbm, peak_kind):
    """The long-sequence workload's forward (B=4, T=65536, d_in=d_h=2048, bf16
    x/W_x, R ~ U(-0.3, 0.3)): input projection + the Newton solve, converged
    to its tolerance and with K=4 fixed iterations, timed with CUDA events;
    the Newton solve's roofline as for the training step."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    w = WORKLOADS["slstm_bf16_long_b4_t65536_d2048"]
    inp = make_inputs(w, with_dH=False)
    x, Wx, R, bias, s0 = (inp[k].to(dev) for k in ("x", "Wx", "R", "bias", "s0"))
    P = torch.empty(w.B, w.T, 4, w.d_h, device=dev)
    S = torch.empty_like(P)
    stats = api.new_stats(dev)
    ws_n = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD, w.B, w.T, 0, w.d_h, dev)
    out = {"workload": w.name, "B": w.B, "T": w.T, "d_h": w.d_h, "forget": w.forget, "tol": w.tol}
    g = guess_launches(args.guess_sweeps)
    for mode, K in (("tol", w.max_iters), ("fixed", (w.fixed_iters or (4,))[0])):
        def step(ev, lev=None):
            ev[0].record()
            api.preact_gemm(x, Wx, bias, P=P)
            ev[1].record()
            api.newton_forward(P, R, s0, forget=w.forget, max_iters=K, fixed=(mode == "fixed"), tol=w.tol, S=S,
                               stats=stats, ws=ws_n, guess_sweeps=args.guess_sweeps, events=lev)
            ev[2].record()
        n = 5
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.warmup + n)]
        levs = [[torch.cuda.Event(enable_timing=True) for _ in range(g + K + 1)] for _ in range(n)]
        for i in range(args.warmup):
            step(evs[i])
        torch.cuda.synchronize()
        for i in range(n):
            step(evs[args.warmup + i], levs[i])
        torch.cuda.synchronize()
        timed = evs[args.warmup:]
        gemm_ms = sum(e[0].elapsed_time(e[1]) for e in timed) / n
        newton_ms = sum(e[1].elapsed_time(e[2]) for e in timed) / n
        st = api.read_stats(stats)
        it = st["iters"]
        nbytes = w.elems * solve_bytes_per_elem(it, args.guess_sweeps)
        gbs = nbytes / (newton_ms / 1e3) / 1e9
        n_sep = separate_iterations(it, mode == "tol")
        it_ms = float(np.mean([lv[g + i].elapsed_time(lv[g + i + 1]) for lv in levs for i in range(n_sep)]))
        guess_ms = float(np.mean([lv[0].elapsed_time(lv[g]) for lv in levs]))
        it_gbs = 48.0 * w.elems / (it_ms / 1e3) / 1e9
        out[mode] = {"newton_mode": mode, "max_iters": K, "iters": it, "guess_sweeps": args.guess_sweeps,
                     "converged": st["converged"],
                     "error": st["error"], "max_scaled_F": st["max_scaled_F"],
                     "S_finite": bool(torch.isfinite(S).all().item()),
                     "fwd_elems_per_s": w.elems / ((gemm_ms + newton_ms) / 1e3), "ms_preact_gemm": gemm_ms,
                     "ms_newton": newton_ms, "steps": n,
                     "roofline": {"kernel": "newton_iter", "bound": "hbm", "achieved": it_gbs, "peak": hbm,
                                  "peak_kind": peak_kind, "unit": "GB/s", "frac": it_gbs / hbm,
                                  "avg_launch_ms": it_ms, "algorithmic_bytes_per_launch": 48 * w.elems,
                                  "guess_kernel_ms": guess_ms,
                                  "solve": {"achieved": gbs, "frac": gbs / hbm, "algorithmic_bytes": nbytes}}}
    del x, Wx, R, bias, s0, P, S, ws_n
    torch.cuda.empty_cache()
    return out


def newton_sweep(args, dev, hbm, peak_kind, T_list=(4096, 16384)):
    """The long-sequence workload's Newton solve (B=4, d=2048, bf16 x/W_x) at shorter T, to the
    workload's tolerance from the decoupled guess: iterations, solve time and newton_iter's HBM
    fraction per T (T = 65536 is the long_forward entry)."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    base = WORKLOADS["slstm_bf16_long_b4_t65536_d2048"]
    out = []
    g = guess_launches(args.guess_sweeps)
    for T in T_list:
        w = scaled(base, T=T, name=f"{base.name}_T{T}")
        inp = make_inputs(w, with_dH=False)
        x, Wx, R, bias, s0 = (inp[k].to(dev) for k in ("x", "Wx", "R", "bias", "s0"))
        P = api.preact_gemm(x, Wx, bias)
        del x
        S = torch.empty_like(P)
        stats = api.new_stats(dev)
        ws_n = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD, w.B, w.T, 0, w.d_h, dev)
        K = w.max_iters
        n = 10
        levs = [[torch.cuda.Event(enable_timing=True) for _ in range(g + K + 1)] for _ in range(n)]
        for _ in range(args.warmup):
            api.newton_forward(P, R, s0, forget=w.forget, max_iters=K, tol=w.tol, S=S, stats=stats, ws=ws_n,
                               guess_sweeps=args.guess_sweeps)
        torch.cuda.synchronize()
        for i in range(n):
            api.newton_forward(P, R, s0, forget=w.forget, max_iters=K, tol=w.tol, S=S, stats=stats, ws=ws_n,
                               guess_sweeps=args.guess_sweeps, events=levs[i])
        torch.cuda.synchronize()
        st = api.read_stats(stats)
        it = st["iters"]
        solve_ms = float(np.median([lv[0].elapsed_time(lv[-1]) for lv in levs]))
        it_ms = float(np.mean([lv[g + i].elapsed_time(lv[g + i + 1]) for lv in levs
                               for i in range(separate_iterations(it, True))]))
        gbs = 48.0 * w.elems / (it_ms / 1e3) / 1e9
        out.append({"workload": w.name, "T": T, "iters": it, "converged": st["converged"],
                    "solve_ms": solve_ms, "solve_elems_per_s": w.elems / (solve_ms / 1e3),
                    "newton_iter_ms": it_ms, "newton_iter_achieved_GBs": gbs, "peak": hbm, "peak_kind": peak_kind,
                    "newton_iter_frac": gbs / hbm, "steps": n})
        del P, S, ws_n
        torch.cuda.empty_cache()
    return out


def run_scan(args):
    import torch
    ws_n, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    hbm, peak_kind = _peaks()
    sweep = scan_sweep(args, dev, hbm, peak_kind)
    last = sweep[-1]
    line = {"metric": "scan_block4 elems/s (B*T*d/s)", "value": last["elems_per_s"], "unit": UNIT, "n_gpus": 1,
            "steps": last["steps"], "warmup": args.warmup, "ms_per_step": last["ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": last["workload"], "B": 4, "T": last["T"], "d": 2048,
                       "l2": "inputs larger than L2"},
            "roofline": {"kernel": "scan_kernel", "bound": "hbm", "achieved": last["achieved_GBs"], "peak": hbm,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": last["frac"], "traffic": None},
            "sweep": sweep}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_varlen(args, w):
    """Packed ragged sequences: the workload's B*T steps repacked into sequences whose lengths are
    drawn (seeded) uniformly from [T/8, 2T), the last one cut to fit; the same inputs, each
    sequence from s0 = 0.  A step is the input-projection GEMM, the Newton solve (to tolerance, or K fixed) and the
    backward, all through the packed entry points."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    _, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    tol_mode = args.newton_mode == "tol"
    K = w.max_iters if tol_mode else args.newton_iters
    total = w.B * w.T
    rng = np.random.default_rng(7)
    lengths = []
    while sum(lengths) < total:
        lengths.append(int(rng.integers(max(1, w.T // 8), 2 * w.T)))
    lengths[-1] -= sum(lengths) - total
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=dev)
    n_seq = len(lengths)
    inp = make_inputs(w)
    x = inp["x"].reshape(total, w.d_in).to(dev)
    Wx, R, bias = inp["Wx"].to(dev), inp["R"].to(dev), inp["bias"].to(dev)
    dH = inp["dH"].reshape(total, w.d_h).to(dev)
    s0 = torch.zeros(n_seq, 4, w.d_h, device=dev)
    P = torch.empty(1, total, 4, w.d_h, device=dev)
    S = torch.empty(total, 4, w.d_h, device=dev)
    stats = api.new_stats(dev)
    ws_f = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD_VARLEN, n_seq, total, 0, w.d_h, dev)
    ws_b = api.workspace(_lib.SLSTM_OP_NEWTON_BACKWARD_VARLEN, n_seq, total, w.d_in, w.d_h, dev)
    grads = {"dx": torch.empty(total, w.d_in, device=dev), "dWx": torch.empty(4 * w.d_h, w.d_in, device=dev),
             "dR": torch.empty(4, w.d_h, device=dev), "db": torch.empty(4, w.d_h, device=dev),
             "ds0": torch.empty(n_seq, 4, w.d_h, device=dev)}

    def step(ev=None):
        api.preact_gemm(x[None], Wx, bias, P=P)
        if ev is not None:
            ev[0].record()
        api.newton_forward_varlen(P[0], R, s0, cu, forget=w.forget, max_iters=K, fixed=not tol_mode, tol=w.tol, S=S,
                                  stats=stats, ws=ws_f, guess_sweeps=args.guess_sweeps)
        if ev is not None:
            ev[1].record()
        api.newton_backward_varlen(x, Wx, P[0], R, s0, cu, S, dH, forget=w.forget, out=grads, ws=ws_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        step(evs[i])
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    newton_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    hbm, peak_kind = _peaks()
    st = api.read_stats(stats)
    nbytes = total * w.d_h * solve_bytes_per_elem(st["iters"], args.guess_sweeps)
    gbs = nbytes / (newton_ms / 1e3) / 1e9
    line = {"metric": METRIC + ", packed ragged sequences", "value": total * w.d_h / (ms / 1e3), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{w.name}_packed", "total_T": total, "n_seq": n_seq,
                       "lengths": f"uniform integers in [{max(1, w.T // 8)}, {2 * w.T}), seed 7, last cut to fit",
                       "d_in": w.d_in, "d_h": w.d_h, "x_dtype": w.dtype, "forget": w.forget, "newton_max_iters": K,
                       "newton_mode": args.newton_mode, "guess_sweeps": args.guess_sweeps,
                       "l2": "inputs larger than L2"},
            "roofline": {"kernel": "newton solve, packed (guess_kernel x guess launches + newton_iter x iters)",
                         "bound": "hbm",
                         "achieved": gbs, "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": None, "solve_ms": newton_ms},
            "newton_stats": {"iters": st["iters"], "converged": st["converged"], "error": st["error"]}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_head(args, w):
    """Head mixing: the workload with block-diagonal R of d_head x d_head blocks (--head-dim, R
    drawn U(-r, r) / sqrt(d_head)) in place of the diagonal R.  A step is the input-projection GEMM,
    the head-mixing Newton solve from the decoupled guess (to the workload's tolerance, or K fixed)
    and its backward.  The head solve applies its linear solve step by step (one warp per batch row
    and head walks the sequence), so it is bound by that walk's latency, not by HBM; the roofline
    object still states the solve's algorithmic bytes against the copy bandwidth."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    _, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    tol_mode = args.newton_mode == "tol"
    K = w.max_iters if tol_mode else args.newton_iters
    dh = args.head_dim
    inp = make_inputs(w)
    x, Wx, bias = inp["x"].to(dev), inp["Wx"].to(dev), inp["bias"].to(dev)
    Rh = make_head_R(w, dh).to(dev)
    s0, dH = inp["s0"].to(dev), inp["dH"].to(dev)
    P = torch.empty(w.B, w.T, 4, w.d_h, device=dev)
    S = torch.empty_like(P)
    stats = api.new_stats(dev)
    ws_f = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD, w.B, w.T, 0, w.d_h, dev)
    ws_b = api.workspace(_lib.SLSTM_OP_NEWTON_BACKWARD_HEAD, w.B, w.T, w.d_in, w.d_h, dev)
    grads = {"dx": torch.empty(w.B, w.T, w.d_in, device=dev), "dWx": torch.empty(4 * w.d_h, w.d_in, device=dev),
             "dR_head": torch.empty_like(Rh), "db": torch.empty(4, w.d_h, device=dev),
             "ds0": torch.empty(w.B, 4, w.d_h, device=dev)}

    def step(ev=None):
        api.preact_gemm(x, Wx, bias, P=P)
        if ev is not None:
            ev[0].record()
        api.newton_forward_head(P, Rh, s0, forget=w.forget, max_iters=K, fixed=not tol_mode, tol=w.tol, S=S,
                                stats=stats, ws=ws_f)
        if ev is not None:
            ev[1].record()
        api.newton_backward_head(x, Wx, P, Rh, s0, S, dH, forget=w.forget, out=grads, ws=ws_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    e0.record()
    for i in range(args.steps):
        step(evs[i])
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    newton_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    hbm, peak_kind = _peaks()
    st = api.read_stats(stats)
    elems = w.B * w.T * w.d_h
    # the guess (reads P, writes S: 32 B/elem) and each iteration (reads P and
    # the old S, writes S: 48 B/elem)
    nbytes = elems * (32 + 48 * st["iters"])
    gbs = nbytes / (newton_ms / 1e3) / 1e9
    line = {"metric": METRIC + ", head mixing", "value": elems / (ms / 1e3), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "operand_dtype": f"{w.dtype} x/W_x, fp32 state", "data": "synthetic",
            "config": {"workload": f"{w.name}_head{dh}", "B": w.B, "T": w.T, "d_in": w.d_in, "d_h": w.d_h,
                       "d_head": dh, "n_heads": w.d_h // dh, "x_dtype": w.dtype, "forget": w.forget,
                       "R_head": f"U(-{w.r_scale}, {w.r_scale}) / sqrt({dh}), seed {w.seed + 1}",
                       "newton_mode": args.newton_mode, "newton_max_iters": K, "newton_init": "decoupled",
                       "l2": "inputs larger than L2"},
            "breakdown_ms_per_step": {"preact_gemm_and_newton_forward": newton_ms, "backward": ms - newton_ms},
            "roofline": {"kernel": "head newton solve (guess_kernel + head_newton_kernel x iters)", "bound": "latency",
                         "achieved": gbs, "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": None, "solve_ms": newton_ms,
                         "note": "one warp per (batch row, head) walks the sequence: bound by the walk's latency"},
            "newton_stats": {"iters": st["iters"], "converged": st["converged"], "diverged": st["diverged"],
                             "error": st["error"], "max_scaled_F": st["max_scaled_F"],
                             "S_finite": bool(torch.isfinite(S).all().item())},
            "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_decode(args, w):
    """Decode: the workload's B rows, d_in and d_h stepped one token at a time with the fused decode
    kernel (input projection + cell update); a step is 128 tokens replayed from one CUDA graph.
    The roofline counts the bytes a token must read: all of W_x, x and the state, and the new state
    written; W_x (8.4 MB at d_in = d_h = 1024, bf16) stays in L2 between tokens, so the achieved rate
    can exceed the HBM copy bandwidth."""
    import torch
    from nonlinear_rnn_pararnn_b200 import api
    _, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    T_dec = 128
    inp = make_inputs(w, with_dH=False)
    xs = inp["x"][:, :T_dec].transpose(0, 1).contiguous().to(dev)   # (T_dec, B, d_in)
    Wx, R, bias = inp["Wx"].to(dev), inp["R"].to(dev), inp["bias"].to(dev)
    s0 = inp["s0"].to(dev)
    S = torch.empty(T_dec, w.B, 4, w.d_h, device=dev)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        api.decode(xs, Wx, bias, R, s0, forget=w.forget, S=S)
    torch.cuda.current_stream().wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        api.decode(xs, Wx, bias, R, s0, forget=w.forget, S=S)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    us_token = ms * 1e3 / T_dec
    esz = 2 if w.dtype == "bf16" else 4
    nbytes = 4 * w.d_h * w.d_in * esz + w.B * w.d_in * esz + 2 * w.B * 4 * w.d_h * 4
    gbs = nbytes / (us_token / 1e6) / 1e9
    hbm, peak_kind = _peaks()
    launches = T_dec * ((w.B + 15) // 16)
    line = {"metric": "sLSTM decode tokens/s (B rows x steps / s)", "value": w.B * T_dec / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "operand_dtype": f"{w.dtype} x/W_x, fp32 state", "data": "synthetic",
            "config": {"workload": f"{w.name}_decode", "B": w.B, "d_in": w.d_in, "d_h": w.d_h,
                       "x_dtype": w.dtype, "forget": w.forget, "tokens_per_step": T_dec,
                       "us_per_token": us_token, "cuda_graph": True,
                       "l2": "W_x stays in L2 between tokens (decode reuses it every token)"},
            "roofline": {"kernel": "decode_kernel", "bound": "hbm", "achieved": gbs, "peak": hbm,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": gbs / hbm, "traffic": None,
                         "bytes_per_token": nbytes},
            "gpu_launches": launches * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_block(args, w):
    """The trunk layer's forward (RMSNorm -> cell -> residual -> RMSNorm -> SwiGLU -> residual) at the
    workload's B and T with d_model = d_h and d_ff = 4 d_model: one slstm_block_forward call per step
    (7 launches + the Newton launches), the Newton solve to the workload's tolerance (or fixed K).  There is no single dominant
    kernel, so the roofline line compares the step with its floor: the three GEMMs' flops at the
    sustained bf16 tensor peak plus the Newton and norm kernels' algorithmic bytes at the HBM copy
    bandwidth; frac = floor / measured step time."""
    import torch
    from nonlinear_rnn_pararnn_b200 import api
    _, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    tol_mode = args.newton_mode == "tol"
    K = w.max_iters if tol_mode else args.newton_iters
    B, T, D = w.B, w.T, w.d_h
    F = 4 * D
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn(B, T, D, generator=g).to(dev)
    w1 = (torch.rand(D, generator=g) + 0.5).to(dev)
    w2 = (torch.rand(D, generator=g) + 0.5).to(dev)
    Wx = (torch.randn(4 * D, D, generator=g) * D ** -0.5).to(torch.bfloat16).to(dev)
    bias = torch.zeros(4, D)
    bias[2] = torch.linspace(3.0, 6.0, D)
    bias = bias.to(dev)
    R = ((torch.rand(4, D, generator=g) * 2 - 1) * w.r_scale).to(dev)
    W_gu = (torch.randn(2 * F, D, generator=g) * D ** -0.5).to(torch.bfloat16).to(dev)
    W_down = (torch.randn(D, F, generator=g) * F ** -0.5).to(torch.bfloat16).to(dev)
    y = torch.empty_like(x)
    S = torch.empty(B, T, 4, D, device=dev)
    stats = api.new_stats(dev)
    wsb = api.block_workspace(B, T, D, F, dev)

    dY = torch.randn(B, T, D, generator=g).to(dev)
    grads = {"dx": torch.empty(B, T, D, device=dev), "dnorm1_w": torch.empty(D, device=dev),
             "dWx": torch.empty(4 * D, D, device=dev), "dbias": torch.empty(4, D, device=dev),
             "dR": torch.empty(4, D, device=dev), "dnorm2_w": torch.empty(D, device=dev),
             "dW_gu": torch.empty(2 * F, D, device=dev), "dW_down": torch.empty(D, F, device=dev)}
    wsbb = torch.empty(int(api.load().slstm_block_backward_workspace_size(B, T, D, F)), dtype=torch.uint8,
                       device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        api.block_forward(x, w1, Wx, bias, R, w2, W_gu, W_down, forget=w.forget, max_iters=K, fixed=not tol_mode,
                          tol=w.tol, y=y, S=S, stats=stats, ws=wsb, guess_sweeps=args.guess_sweeps)
        if ev is not None:
            ev[1].record()
        api.block_backward(x, w1, Wx, bias, R, w2, W_gu, W_down, S, dY, forget=w.forget, out=grads, ws=wsbb)
        if ev is not None:
            ev[2].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    time.sleep(0.25)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        step(evs[i])
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_all = e0.elapsed_time(e1) / args.steps
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    ms_bwd = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    st = api.read_stats(stats)
    M = B * T
    flops = 2.0 * M * D * (4 * D + 2 * F + F)
    nbytes = M * D * solve_bytes_per_elem(st["iters"], args.guess_sweeps) + M * D * (4 + 2) + M * D * (4 + 16 + 4 + 2)
    hbm, peak_kind = _peaks()
    try:
        with open(PEAKS_PATH) as f:
            tflops = float(json.load(f)["bf16_tflops_sustained"])
        tkind = "measured"
    except Exception:
        tflops, tkind = 1400.0, "fallback"
    floor_ms = flops / (tflops * 1e12) * 1e3 + nbytes / (hbm * 1e9) * 1e3
    # the backward: eight GEMMs on the tensor cores (the forward's two recomputed, the five of the
    # SwiGLU and norm gradients, the cell's dx and dW_x with the bf16 pair doubling their flops)
    bwd_flops = 2.0 * M * D * (4 * D + 2 * F) + 2.0 * 2 * M * D * (F + F + 2 * F + 2 * F) + 2.0 * 2 * M * D * (4 * D) * 2
    line = {"metric": "trunk-layer forward tokens/s (B*T / s)", "value": M / (ms / 1e3), "unit": "tokens/s",
            "fwd_bwd": {"value": M / (ms_all / 1e3), "unit": "tokens/s", "ms_per_step": ms_all,
                        "ms_backward": ms_bwd, "backward_gemm_tflop": bwd_flops / 1e12,
                        "backward_tensor_floor_ms": bwd_flops / (tflops * 1e12) * 1e3},
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "operand_dtype": "bf16 GEMM operands, fp32 accumulation, state and residual stream", "data": "synthetic",
            "config": {"workload": f"{w.name}_block", "B": B, "T": T, "d_model": D, "d_ff": F, "forget": w.forget,
                       "gemm_tiles": args.gemm_tiles,
                       "newton_max_iters": K, "newton_mode": args.newton_mode, "newton_iters": st["iters"],
                       "converged": st["converged"], "error": st["error"],
                       "l2": "inputs larger than L2"},
            "roofline": {"kernel": "whole layer (3 GEMMs + Newton + norms)", "bound": "tensor+hbm",
                         "achieved": floor_ms, "peak": ms, "unit": "ms (floor vs measured)",
                         "frac": floor_ms / ms, "traffic": None, "gemm_tflop_per_step": flops / 1e12,
                         "tensor_peak_tflops": tflops, "tensor_peak_kind": tkind, "hbm_gbs": hbm,
                         "hbm_peak_kind": peak_kind, "algorithmic_bytes_per_step": nbytes},
            "clocks": clocks,
            "gpu_launches": (5 + newton_launches(args.guess_sweeps, K, tol_mode) + 20) * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# DRAM bytes (read + write) per element of B*T*d_h of the Newton solve's kernels, from one ncu
# capture of the training workload shortened to T = 2048 (summarised under profiles/): the guess
# launch (the guess and two sweeps fused), a separate sweep launch (not captured: None) and a Newton
# iteration that evaluates its whole residual.  The counters describe the kernel sources with this
# SHA-256; other sources report traffic null.  Traffic per element does not depend on T (every
# tile moves the same bytes), so it scales to a full launch by the element count.
NEWTON_TRAFFIC = {"sources_sha256": "60725403a102fc65e60d077642cfd653092b1f5b85ccd2a3c71016a8c77cb7f7",
                  "guess": 30.9, "sweep": None, "iter": 46.3}
NEWTON_SOURCES = ("newton.cu", "lookback.cuh", "common.cuh", "tma.cuh", "launchers.h")


def newton_sources_sha256() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nonlinear_rnn_pararnn_b200", "csrc")
    for name in NEWTON_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# Refinement sweeps that the guess launch runs itself, tile by tile, after the
# decoupled guess; each further sweep is a launch of its own.
GUESS_FUSED_SWEEPS = 3


def guess_launches(sweeps: int) -> int:
    return 1 + max(0, sweeps - GUESS_FUSED_SWEEPS)


# Tolerance mode with the fused carry: the library launches the first
# LOOP_FROM iterations one by one (slstm_newton_config.loop_from, its default)
# and the rest of the cap as one launch that loops on the device.
LOOP_FROM = 2


def newton_launches(sweeps: int, K: int, tol_mode: bool) -> int:
    """Launches of work of one Newton call (fused carry)."""
    return guess_launches(sweeps) + (LOOP_FROM + 1 if tol_mode and K > LOOP_FROM else K)


def separate_iterations(iters: int, tol_mode: bool) -> int:
    """How many of a call's iterations ran as launches of their own."""
    return min(iters, LOOP_FROM) if tol_mode else iters


def solve_bytes_per_elem(iters: int, sweeps: int) -> int:
    """Algorithmic bytes per element of B*T*d_h of one Newton solve: the
    guess launch reads P and writes S (32) whatever number of sweeps it fuses,
    a sweep launch also reads the previous guess's h (36), an iteration reads
    P and the old S and writes S (48)."""
    return 32 + 36 * (guess_launches(sweeps) - 1) + 48 * iters


def newton_traffic_bytes(elems: int, iters: int, sweeps: int):
    """Measured DRAM bytes of one Newton solve (the guess, its sweeps and
    `iters` iterations), or None when the counters were taken on other kernel sources."""
    t = NEWTON_TRAFFIC
    if t["sources_sha256"] is None or newton_sources_sha256() != t["sources_sha256"]:
        return None
    if guess_launches(sweeps) > 1 and t["sweep"] is None:
        return None
    return (t["guess"] + (t["sweep"] or 0.0) * (guess_launches(sweeps) - 1) + t["iter"] * iters) * elems


def newton_iter_traffic_bytes(elems: int):
    """Measured DRAM bytes of one newton_iter launch, or None when the
    counters were taken on other kernel sources."""
    t = NEWTON_TRAFFIC
    if t["sources_sha256"] is None or newton_sources_sha256() != t["sources_sha256"]:
        return None
    return t["iter"] * elems


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=ORDER)
    ap.add_argument("--newton-mode", default="tol", choices=["tol", "fixed"],
                    help="tol: Newton to the workload's tolerance (its cap as max_iters); fixed: --newton-iters")
    ap.add_argument("--newton-iters", type=int, default=4)
    ap.add_argument("--guess-sweeps", type=int, default=2,
                    help="refinement sweeps of the decoupled initial guess (the library's Python default)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the long-sequence forward and the scan sweep that the default line carries")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-lanes", type=int, default=16)
    ap.add_argument("--ref-lanes", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="train",
                    choices=["train", "forward", "scan", "varlen", "decode", "block", "head"],
                    help="train: GEMM + Newton + backward (default); forward: GEMM + Newton; "
                         "scan: scan_block4 alone over T in --scan-T at B=4, d=2048; "
                         "varlen: the workload repacked into ragged sequences (cu_seqlens); "
                         "decode: T = 1 steps under a CUDA graph; block: the trunk layer's forward; "
                         "head: head mixing (block-diagonal R, --head-dim) forward + backward")
    ap.add_argument("--head-dim", type=int, default=32, help="d_head of --mode head (1 .. 32, dividing d_h)")
    ap.add_argument("--scan-T", default="4096,16384,65536")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="ncu dram read+write bytes per Newton launch, when captured for the current kernel sources")
    ap.add_argument("--gemm-tiles", default="auto", choices=["auto", "pair", "single"],
                    help="tile shape of the tensor-core GEMMs: auto (the library default: SM pairs for the gradient GEMMs), "
                         "256 x 256 on SM pairs, or 128 x 256 per SM")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="run the workload with T shortened to this length (small cases for ncu "
                         "captures; the bench line then names the shortened workload)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = WORKLOADS[args.workload]
    if args.seq_len is not None:
        if not 1 <= args.seq_len <= w.T:
            ap.error(f"--seq-len must be in [1, {w.T}]")
        w = scaled(w, T=args.seq_len, name=f"{w.name}_T{args.seq_len}")
    ws, _, _ = _dist()
    if ws != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={ws}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.gemm_tiles != "auto":
        from nonlinear_rnn_pararnn_b200 import api
        api.set_gemm_tiles(args.gemm_tiles)
    if args.mode == "scan":
        return run_scan(args)
    if args.mode == "varlen":
        return run_varlen(args, w)
    if args.mode == "decode":
        return run_decode(args, w)
    if args.mode == "block":
        return run_block(args, w)
    if args.mode == "head":
        return run_head(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
