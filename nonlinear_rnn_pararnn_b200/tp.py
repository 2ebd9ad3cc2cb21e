"""Tensor parallelism over the hidden features d_h ("sLSTM in this library",
section "Tensor parallel": channelwise shards of d_h, each rank scans its own
features, one all-reduce where the features meet a dense projection).

With diagonal recurrent mixing ("sLSTM in this library", "Cell": R holds one
weight per gate and feature) feature j of the state depends only on its own
four pre-activation rows g d_h + j of P = x W_x^T + bias and on R[:, j].  A
rank that owns a contiguous range of features [j0, j1) therefore solves its
whole share of the forward pass (input projection, Newton iterations) without
exchanging anything, and the backward pass is local too except for

    dx = sum over ranks of dP_rank W_x,rank

the input gradient, which every rank holds as a partial sum over its own
features and which one all-reduce (sum) completes.  (The forward all-reduce
of that section sits on the output projection, after h, outside this
library's boundary x -> h.)  dW_x, dR, db and ds0 of a
rank are its own rows and columns of the full gradients.

Ranges are whole groups of 32 features (the feature width of one tile of the
kernels), split as evenly as the group count allows; the last range takes the
ragged tail, and ranks beyond the group count get an empty range (they still
take part in the all-reduce, with zeros).

Everything here is argument marshalling around the library's kernels plus the
one collective (torch.distributed, NCCL between GPUs).
"""
from __future__ import annotations

import torch

from . import api

GROUP = 32


def feature_range(d_h: int, world: int, rank: int, group: int = GROUP):
    """[j0, j1) of the features that `rank` of `world` owns."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if d_h < 0 or group < 1:
        raise ValueError("d_h must be >= 0 and group >= 1")
    n = (d_h + group - 1) // group
    g0 = (rank * n) // world
    g1 = ((rank + 1) * n) // world
    return min(d_h, g0 * group), min(d_h, g1 * group)


def shard_params(Wx: torch.Tensor, bias: torch.Tensor, R: torch.Tensor, j0: int, j1: int):
    """The rank's rows of W_x (4 d_h, d_in), gate-major: rows g d_h + j for
    j in [j0, j1) of each gate g become rows g (j1 - j0) + (j - j0); bias and
    R (4, d_h) keep columns [j0, j1).  Returns contiguous copies."""
    d_h = R.shape[1]
    if Wx.shape[0] != 4 * d_h or tuple(bias.shape) != (4, d_h) or R.shape[0] != 4:
        raise ValueError("W_x must be (4 d_h, d_in) and bias, R (4, d_h)")
    if not 0 <= j0 <= j1 <= d_h:
        raise ValueError(f"feature range [{j0}, {j1}) outside [0, {d_h})")
    Wl = Wx.view(4, d_h, Wx.shape[1])[:, j0:j1].reshape(4 * (j1 - j0), Wx.shape[1]).contiguous()
    return Wl, bias[:, j0:j1].contiguous(), R[:, j0:j1].contiguous()


def shard_state(s: torch.Tensor, j0: int, j1: int) -> torch.Tensor:
    """Features [j0, j1) of a state or state-like tensor (..., 4, d_h) or of
    h-shaped (..., d_h) tensors (the last axis is the feature axis)."""
    return s[..., j0:j1].contiguous()


def forward(x, Wx_loc, bias_loc, R_loc, s0_loc=None, *, forget="sigmoid", max_iters=8, fixed=False, tol=1e-5):
    """The rank's share of the forward pass: P_loc (B, T, 4, d_loc) and the
    Newton solution S_loc; no collective.  Returns (P_loc, S_loc, stats) with
    stats None for an empty range."""
    B, T, _ = x.shape
    d_loc = R_loc.shape[1]
    if d_loc == 0:
        empty = torch.empty(B, T, 4, 0, device=x.device)
        return empty, empty.clone(), None
    P = api.preact_gemm(x, Wx_loc, bias_loc)
    S, stats = api.newton_forward(P, R_loc, s0_loc, forget=forget, max_iters=max_iters, fixed=fixed, tol=tol)
    return P, S, stats


def all_reduce_dx(dx: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-rank partial input gradients in place over `group`."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dx, op=dist.ReduceOp.SUM, group=group)
    return dx


def backward(x, Wx_loc, P_loc, R_loc, s0_loc, S_loc, dH_loc, *, forget="sigmoid", group=None, reduce=True):
    """The rank's share of the backward pass.  dx is this rank's partial
    (its features' contribution) unless `reduce`, in which case it is summed
    over `group` and every rank holds the full input gradient; dWx, dR, db,
    ds0 are the rank's own slices of the full gradients."""
    B, T, d_in = x.shape
    d_loc = R_loc.shape[1]
    if d_loc == 0:
        out = {"dx": torch.zeros(B, T, d_in, device=x.device),
               "dWx": torch.empty(0, d_in, device=x.device), "dR": torch.empty(4, 0, device=x.device),
               "db": torch.empty(4, 0, device=x.device), "ds0": torch.empty(B, 4, 0, device=x.device)}
    else:
        out = api.newton_backward(x, Wx_loc, P_loc, R_loc, s0_loc, S_loc, dH_loc, forget=forget)
    if reduce:
        all_reduce_dx(out["dx"], group)
    return out
