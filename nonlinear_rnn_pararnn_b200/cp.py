"""Time context parallelism ("sLSTM in this library", section "Tensor
parallel": context parallel splits time).

Rank r of n holds a contiguous slice of the time axis of every sequence (its
P and S are (B, T_r, 4, d_h); B and d_h are the same on every rank).  The
Newton solve keeps the single-GPU arithmetic; each of its scans (the
decoupled guess, every refinement sweep, every iteration's linear solve)
runs as three phases:

  1. every rank composes its slice into one map (the guess's run, or the
     affine map of the iteration's linear solve)      slstm_cp_*_run / _map
  2. the maps are all-gathered                        one all-gather
  3. every rank enters its slice through the maps of the ranks before it
     and finishes the scan on its own steps           slstm_cp_*_apply

Before a sweep or an iteration the ranks also all-gather their slices' last
states (the state just before rank r's slice is rank r - 1's last one), and
after an iteration they take the maximum of the residual over ranks (one
all-reduce) for the stopping test.  Exchanged per (b, j) and rank: 20 floats
per iteration and 5 per guess stage, plus the 4 of the last state; nothing
of size T crosses the link.

The collectives are functions the caller passes in, so that the same driver
runs one rank per process (torch.distributed, NCCL over NVLink: see
`collectives`) or every rank in one process on one GPU (`local_collectives`,
used by the tests: the ranks' phases then run one after another, and no rank
ever waits on another).  Everything here is argument marshalling around the
library's kernels plus those collectives.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib, api
from ._lib import check, load


class Slice:
    """One rank's part: its index, P and S (B, T_r, 4, d_h) and workspace."""

    def __init__(self, rank: int, P: torch.Tensor, S: torch.Tensor = None):
        B, T, four, d = P.shape
        self.rank = rank
        self.P = P
        self.S = torch.empty_like(P) if S is None else S
        n = int(load().slstm_workspace_size(_lib.SLSTM_OP_CONTEXT_PARALLEL, B, T, 0, d))
        if n == 0:
            raise ValueError(f"unsupported slice sizes B={B}, T={T}, d_h={d}")
        self.ws = torch.empty(n, dtype=torch.uint8, device=P.device)
        self.stats = api.new_stats(P.device)

    @property
    def dims(self):
        B, T, _, d = self.P.shape
        return B, T, d

    def last_state(self) -> torch.Tensor:
        return self.S[:, -1].contiguous()


def local_collectives():
    """All ranks in this process: gather = stack the ranks' tensors, in rank
    order; max = elementwise maximum."""
    def gather(tensors):
        return [torch.stack(tensors)] * len(tensors)

    def reduce_max(values):
        m = torch.stack(values).amax(dim=0)
        return [m] * len(values)
    return gather, reduce_max


def collectives(group=None):
    """One rank per process over torch.distributed (NCCL between GPUs)."""
    import torch.distributed as dist

    def gather(tensors):
        (t,) = tensors
        out = torch.empty((dist.get_world_size(group),) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return [out]

    def reduce_max(values):
        (v,) = values
        v = v.clone()
        dist.all_reduce(v, op=dist.ReduceOp.MAX, group=group)
        return [v]
    return gather, reduce_max


def _s_before(lasts: torch.Tensor, rank: int, s0):
    return s0 if rank == 0 else lasts[rank - 1].contiguous()


def _guess_stage(slices, R, s0, forget, sweep, gather):
    lib = load()
    stream = api._stream()
    befores = [None] * len(slices)
    if sweep:
        lasts = gather([sl.last_state() for sl in slices])
        befores = [_s_before(la, sl.rank, s0) for la, sl in zip(lasts, slices)]
    runs_local = []
    for sl, sb in zip(slices, befores):
        B, T, d = sl.dims
        run = torch.empty(B, 5, d, device=sl.P.device)
        check("slstm_cp_guess_run", lib.slstm_cp_guess_run(
            api._ptr(sl.P), api._ptr(R), api._ptr(sb), api._ptr(sl.S), 1 if sweep else 0, api.forget_code(forget),
            api._ptr(run), B, T, d, api._ptr(sl.ws), sl.ws.numel(), stream))
        runs_local.append(run)
    runs = gather(runs_local)
    for sl, sb, rn in zip(slices, befores, runs):
        B, T, d = sl.dims
        check("slstm_cp_guess_apply", lib.slstm_cp_guess_apply(
            api._ptr(sl.P), api._ptr(R), api._ptr(s0), api._ptr(sb), api._ptr(rn), sl.rank, api._ptr(sl.S),
            1 if sweep else 0, api.forget_code(forget), B, T, d, api._ptr(sl.ws), sl.ws.numel(), stream))


def _iteration(slices, R, s0, cfg, gather, reduce_max):
    lib = load()
    stream = api._stream()
    lasts = gather([sl.last_state() for sl in slices])
    befores = [_s_before(la, sl.rank, s0) for la, sl in zip(lasts, slices)]
    maps_local = []
    for sl, sb in zip(slices, befores):
        B, T, d = sl.dims
        mp = torch.empty(B, 20, d, device=sl.P.device)
        check("slstm_cp_newton_map", lib.slstm_cp_newton_map(
            api._ptr(sl.P), api._ptr(R), api._ptr(sb), api._ptr(sl.S), cfg.forget, api._ptr(mp), B, T, d,
            api._ptr(sl.ws), sl.ws.numel(), stream))
        maps_local.append(mp)
    maps = gather(maps_local)
    resid = []
    for sl, sb, mp in zip(slices, befores, maps):
        B, T, d = sl.dims
        check("slstm_cp_newton_apply", lib.slstm_cp_newton_apply(
            api._ptr(sl.P), api._ptr(R), api._ptr(sb), api._ptr(mp), sl.rank, api._ptr(sl.S), ctypes.byref(cfg),
            api._ptr(sl.stats), B, T, d, api._ptr(sl.ws), sl.ws.numel(), stream))
        # the slice's residual maxima: max_abs_F[0] and max_scaled_F[0] of the record
        f = sl.stats[16:].view(torch.float32)
        resid.append(torch.stack([f[0], f[_lib.SLSTM_STATS_HISTORY]]))
    return reduce_max(resid)


def newton_forward(slices, R: torch.Tensor, s0: torch.Tensor = None, *, forget="sigmoid", max_iters: int = 16,
                   tol: float = 1e-5, fixed: bool = False, guess_sweeps: int = api.DEFAULT_GUESS_SWEEPS,
                   residual_mode="scaled", gather=None, reduce_max=None) -> dict:
    """Newton solve of a sequence split over time: `slices` are the Slice
    objects this process holds (one per process under torch.distributed,
    all of them in one process with local_collectives); s0 (B, 4, d_h) is the
    sequences' initial state (or None).  Solves in place into each slice's S
    and returns the stats of the solve (the same on every rank):
    iters, converged, diverged, max_abs_F, max_scaled_F."""
    if gather is None or reduce_max is None:
        gather, reduce_max = local_collectives()
    cfg = api.newton_config(1, False, tol, forget, residual_mode=residual_mode)
    _guess_stage(slices, R, s0, forget, False, gather)
    for _ in range(guess_sweeps):
        _guess_stage(slices, R, s0, forget, True, gather)
    raw_h, sc_h = [], []
    converged = diverged = False
    it = 0
    for it in range(1, max_iters + 1):
        m = _iteration(slices, R, s0, cfg, gather, reduce_max)[0].tolist()
        raw_h.append(m[0])
        sc_h.append(m[1])
        bad = not (m[0] <= 3.4e38 and m[1] <= 3.4e38)
        test = m[0] if residual_mode == "raw" else m[1]
        if bad:
            break
        if not fixed and test <= tol:
            converged = True
            break
    if fixed and raw_h and (raw_h[-1] if residual_mode == "raw" else sc_h[-1]) <= tol:
        converged = True
    if raw_h and not converged and not (raw_h[-1] <= 1.0):
        diverged = True
    return {"iters": it, "converged": converged, "diverged": diverged, "max_abs_F": raw_h, "max_scaled_F": sc_h}


def split_time(T: int, world: int):
    """[t0, t1) of each of `world` contiguous slices of T steps, as even as
    possible (the first T % world slices one step longer)."""
    if world < 1 or T < world:
        raise ValueError(f"cannot split {T} steps over {world} ranks")
    q, r = divmod(T, world)
    out, t = [], 0
    for k in range(world):
        n = q + (1 if k < r else 0)
        out.append((t, t + n))
        t += n
    return out
