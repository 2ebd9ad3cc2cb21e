#!/usr/bin/env python
"""Benchmark of the Newton-solved diag-mix sLSTM training step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--newton-iters K_N] [--impl reference]

One step = the whole hot path on one batch of synthetic input already in HBM:
  input projection GEMM  ->  K_N fixed Newton iterations (fused residual,
  Jacobian, blocked scan, update)  ->  backward (fused adjoint scan + cell
  VJP, dR/db reduction, dx and dW_x GEMMs).
Metric: B*T*d_h elements per second for forward + backward (the JSON
`value`), with the forward alone reported beside it.  Under torchrun each
rank runs its own replica of the workload (independent batches, no data-path
collective): `value` is the sum over ranks of elements divided by the slowest
rank's device time.

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

from nonlinear_rnn_pararnn_b200.workloads import ORDER, WORKLOADS, as_f64, make_inputs, scaled  # noqa: E402

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
def oracle_sample(w, inp, n_lanes, newton_iters, seed=0):
    """Run the fp64 oracle, as it stands, on n_lanes (b, j) lanes of the
    workload: input projection rows, K fixed Newton iterations, BPTT and the
    lanes' contributions to dx and dW_x.  Returns (seconds, elements)."""
    import oracle
    rng = np.random.default_rng(seed)
    lanes = [(int(rng.integers(0, w.B)), int(rng.integers(0, w.d_h))) for _ in range(n_lanes)]
    bias = as_f64(inp["bias"])
    t0 = time.perf_counter()
    for b, j in lanes:
        xb = as_f64(inp["x"][b])                                        # (T, d_in)
        rows = [g * w.d_h + j for g in range(4)]
        Wr = as_f64(inp["Wx"][rows])                                    # (4, d_in)
        P = oracle.gemm(xb, Wr, tb=True, bias=bias[:, j])[None]         # (1, T, 4)
        R = as_f64(inp["R"][:, j])[None]
        s0 = np.zeros((1, 4))
        S, _ = oracle.newton(P, R, s0, w.forget, max_iters=newton_iters, fixed=True, tol=w.tol)
        dH = as_f64(inp["dH"][b, :, j])[None]
        dP, dR, db, ds0 = oracle.bptt(P, R, s0, S, dH, w.forget)
        oracle.gemm(dP[0], Wr)                                          # this lane's share of dx
        oracle.gemm(np.ascontiguousarray(dP[0].T), np.ascontiguousarray(xb.T), tb=True)  # its dW_x rows
    dt = time.perf_counter() - t0
    return dt, n_lanes * w.T


def run_reference(args, w):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    inp = make_inputs(w)
    t_lane = 0.0
    for _ in range(args.warmup):
        t_lane, _ = oracle_sample(w, inp, 1, args.newton_iters, seed=99)
    # bounded sample: about a minute of CPU work over all timed steps
    lanes_per_step = int(max(1, min(args.ref_lanes, 60.0 / max(1e-3, args.steps * t_lane))))
    total_t, total_e = 0.0, 0
    for s in range(args.steps):
        dt, el = oracle_sample(w, inp, lanes_per_step, args.newton_iters, seed=s)
        total_t += dt
        total_e += el
    value = total_e / total_t
    sample = (f"{lanes_per_step} random (b,j) lanes x T={w.T} per step: fp64 input-projection rows, "
              f"{args.newton_iters} fixed Newton iterations, BPTT, dx/dW_x contributions")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(w.describe(), newton_iters=args.newton_iters, newton_mode="fixed"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
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

    K = args.newton_iters
    forward_only = args.mode == "forward"
    inp = make_inputs(w)
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

    def step(ev=None, dv=None, gr=None):
        dv = dev_main if dv is None else dv
        gr = grads if gr is None else gr
        if ev is not None:
            ev[0].record()
        api.preact_gemm(dv["x"], dv["Wx"], dv["bias"], P=P)
        if ev is not None:
            ev[1].record()
        api.newton_forward(P, dv["R"], dv["s0"], forget=w.forget, max_iters=K, fixed=True, tol=w.tol, S=S,
                           stats=stats, ws=ws_n)
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
    sampler = ClockSampler(dev.index)
    time.sleep(0.25)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for s_ in range(args.steps):
        step(evs[s_])
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
    newton_launch_ms = ms_newton / args.steps / K
    # algorithmic bytes of one Newton launch: iteration 1 reads P and writes S
    # (32 B/elem); later ones also read the old S (48 B/elem).  Averaged over
    # the K launches of a step.
    newton_bytes = elems * (32 + 48 * (K - 1)) / K
    achieved = newton_bytes / (newton_launch_ms / 1e3) / 1e9
    traffic = args.traffic_bytes if args.traffic_bytes else newton_traffic_bytes(elems, K)
    roofline = {"kernel": "newton_iter", "bound": "hbm", "achieved": achieved, "peak": hbm,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                "algorithmic_bytes_per_launch": newton_bytes, "avg_launch_ms": newton_launch_ms}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        oracle_sample(w, inp, 1, K, seed=123)              # warm the oracle library
        dt, el = oracle_sample(w, inp, args.cpu_lanes, K)
        cpu = {"value": el / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{args.cpu_lanes} random (b,j) lanes x T={w.T}: fp64 input-projection rows, {K} fixed "
                         f"Newton iterations, BPTT, dx/dW_x contributions ({dt:.1f} s, single thread)"}

    # kernels launched per step: preact GEMM 1, Newton K, backward: adjoint 1 +
    # dR/db reduction 1 + 2 GEMMs (+ the split-K sum of the tensor-core path)
    launches_per_step = 1 + K + (0 if forward_only else 4 + (1 if w.dtype == "bf16" else 0))
    line = {
        "metric": METRIC_FWD if forward_only else METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "operand_dtype": "bf16 x/W_x, fp32 state and scans" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": dict(w.describe(), newton_iters=K, newton_mode="fixed",
                       l2="inputs larger than L2 (P and S are %.2f GB each)" % (elems * 16 / 1e9),
                       parallelism=f"replicas x{ws}"),
        "fwd": {"value": aggregate(elems, ws, fwd_ms), "unit": UNIT, "ms_per_step": fwd_ms},
        "breakdown_ms_per_step": {"preact_gemm": ms_gemm / args.steps, "newton_forward": ms_newton / args.steps,
                                  "backward": ms_bwd / args.steps},
        "newton_stats_last_step": {"iters": st["iters"], "diverged": st["diverged"], "error": st["error"]},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate(elems, ws, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_scan(args):
    """scan_block4 alone: B=4, d=2048, T swept; 96 algorithmic bytes per
    element (read A 64, b 16, write y 16).  Inputs drawn on the device from a
    seeded generator (values only set the timing's data, not checked here)."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    ws_n, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    hbm, peak_kind = _peaks()
    B, d = 4, 2048
    sweep = []
    for T in [int(v) for v in args.scan_T.split(",")]:
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
        e0.record()
        for _ in range(args.steps):
            api.scan_block4(A, b, None, y=y, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        elems = B * T * d
        gbs = elems * 96 / (ms / 1e3) / 1e9
        sweep.append({"T": T, "ms": ms, "elems_per_s": elems / (ms / 1e3), "achieved_GBs": gbs,
                      "frac": gbs / hbm})
        del A, b, y, ws
        torch.cuda.empty_cache()
    last = sweep[-1]
    line = {"metric": "scan_block4 elems/s (B*T*d/s)", "value": last["elems_per_s"], "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": last["ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"scan_block4_b{B}_d{d}", "B": B, "T": last["T"], "d": d,
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
    sequence from s0 = 0.  A step is the input-projection GEMM, K fixed Newton iterations and the
    backward, all through the packed entry points."""
    import torch
    from nonlinear_rnn_pararnn_b200 import _lib, api
    _, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    K = args.newton_iters
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
        api.newton_forward_varlen(P[0], R, s0, cu, forget=w.forget, max_iters=K, fixed=True, tol=w.tol, S=S,
                                  stats=stats, ws=ws_f)
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
    newton_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps / K
    hbm, peak_kind = _peaks()
    nbytes = total * w.d_h * (32 + 48 * (K - 1)) / K
    gbs = nbytes / (newton_ms / 1e3) / 1e9
    st = api.read_stats(stats)
    line = {"metric": METRIC + ", packed ragged sequences", "value": total * w.d_h / (ms / 1e3), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{w.name}_packed", "total_T": total, "n_seq": n_seq,
                       "lengths": f"uniform integers in [{max(1, w.T // 8)}, {2 * w.T}), seed 7, last cut to fit",
                       "d_in": w.d_in, "d_h": w.d_h, "x_dtype": w.dtype, "forget": w.forget, "newton_iters": K,
                       "newton_mode": "fixed", "l2": "inputs larger than L2"},
            "roofline": {"kernel": "newton_iter (packed)", "bound": "hbm", "achieved": gbs, "peak": hbm,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": gbs / hbm, "traffic": None,
                         "avg_launch_ms": newton_ms},
            "newton_stats": {"iters": st["iters"], "error": st["error"]}}
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
    (7 launches + the Newton iterations), fixed K Newton iterations.  There is no single dominant
    kernel, so the roofline line compares the step with its floor: the three GEMMs' flops at the
    sustained bf16 tensor peak plus the Newton and norm kernels' algorithmic bytes at the HBM copy
    bandwidth; frac = floor / measured step time."""
    import torch
    from nonlinear_rnn_pararnn_b200 import api
    _, rank, _ = _dist()
    dev = torch.device("cuda", 0)
    K = args.newton_iters
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

    def step():
        api.block_forward(x, w1, Wx, bias, R, w2, W_gu, W_down, forget=w.forget, max_iters=K, fixed=True,
                          y=y, S=S, stats=stats, ws=wsb)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    time.sleep(0.25)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    st = api.read_stats(stats)
    M = B * T
    flops = 2.0 * M * D * (4 * D + 2 * F + F)
    nbytes = M * D * (32 + 48 * (K - 1)) + M * D * (4 + 2) + M * D * (4 + 16 + 4 + 2)
    hbm, peak_kind = _peaks()
    try:
        with open(PEAKS_PATH) as f:
            tflops = float(json.load(f)["bf16_tflops_sustained"])
        tkind = "measured"
    except Exception:
        tflops, tkind = 1400.0, "fallback"
    floor_ms = flops / (tflops * 1e12) * 1e3 + nbytes / (hbm * 1e9) * 1e3
    line = {"metric": "trunk-layer forward tokens/s (B*T / s)", "value": M / (ms / 1e3), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "operand_dtype": "bf16 GEMM operands, fp32 accumulation, state and residual stream", "data": "synthetic",
            "config": {"workload": f"{w.name}_block", "B": B, "T": T, "d_model": D, "d_ff": F, "forget": w.forget,
                       "newton_iters": K, "newton_mode": "fixed", "error": st["error"],
                       "l2": "inputs larger than L2"},
            "roofline": {"kernel": "whole layer (3 GEMMs + Newton + norms)", "bound": "tensor+hbm",
                         "achieved": floor_ms, "peak": ms, "unit": "ms (floor vs measured)",
                         "frac": floor_ms / ms, "traffic": None, "gemm_tflop_per_step": flops / 1e12,
                         "tensor_peak_tflops": tflops, "tensor_peak_kind": tkind, "hbm_gbs": hbm,
                         "hbm_peak_kind": peak_kind, "algorithmic_bytes_per_step": nbytes},
            "clocks": clocks,
            "gpu_launches": (5 + K) * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# DRAM bytes (read + write) per element of B*T*d_h of the newton_iter launches (first, middle and
# last iteration of a step), from one ncu capture of the training workload shortened to T = 2048
# (the newton_iter capture summarised under profiles/).  The counters describe the kernel sources with
# this SHA-256; any other build reports traffic null.  Traffic per element does not depend on T
# (every tile moves the same bytes), so it scales to a full launch by the element count.
NEWTON_TRAFFIC = {"sources_sha256": "a1354d490b4ffca0023f55f55b9b12a31166f1d56c4ea2ff2b1e91f2ce16bad2", "first": 29.95, "middle": 46.33, "last": 46.35}
NEWTON_SOURCES = ("newton.cu", "lookback.cuh", "common.cuh", "tma.cuh", "launchers.h")


def newton_sources_sha256() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nonlinear_rnn_pararnn_b200", "csrc")
    for name in NEWTON_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def newton_traffic_bytes(elems: int, K: int):
    """Measured DRAM bytes of one Newton launch averaged over the K launches of a step, or None."""
    if newton_sources_sha256() != NEWTON_TRAFFIC["sources_sha256"]:
        return None
    t = NEWTON_TRAFFIC
    per = t["first"] if K == 1 else (t["first"] + t["middle"] * (K - 2) + t["last"]) / K
    return per * elems


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=ORDER)
    ap.add_argument("--newton-iters", type=int, default=4)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-lanes", type=int, default=40)
    ap.add_argument("--ref-lanes", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="train", choices=["train", "forward", "scan", "varlen", "decode", "block"],
                    help="train: GEMM + Newton + backward (default); forward: GEMM + Newton; "
                         "scan: scan_block4 alone over T in --scan-T at B=4, d=2048; "
                         "varlen: the workload repacked into ragged sequences (cu_seqlens); "
                         "decode: T = 1 steps under a CUDA graph; block: the trunk layer's forward")
    ap.add_argument("--scan-T", default="4096,16384,65536")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="ncu dram read+write bytes per Newton launch, when captured for this build")
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
    if args.mode == "scan":
        return run_scan(args)
    if args.mode == "varlen":
        return run_varlen(args, w)
    if args.mode == "decode":
        return run_decode(args, w)
    if args.mode == "block":
        return run_block(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
