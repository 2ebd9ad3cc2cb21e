"""The context-parallel decomposition of the Newton solve's linear scan,
with two gloo ranks on the CPU: each rank holds a time slice of an affine
recurrence y_t = A_t y_{t-1} + b_t, composes its slice into one map, the
maps are all-gathered, and each rank solves its slice from the carry that
the maps of the ranks before it give; the concatenation equals the oracle's
solve of the whole sequence.  (The GPU side of the same decomposition, the
library's phases through cp.py, is tests/test_gpu_cp.py.)"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from nonlinear_rnn_pararnn_b200 import cp


def _slice_map(A, b):
    """The slice's affine map (M, c): y_end = M y_in + c, composed step by
    step from the oracle's solve of the identity columns and of the offset."""
    L, T = b.shape[:2]
    M = np.zeros((L, 4, 4))
    for k in range(4):
        b0 = np.zeros_like(b)
        y0 = np.zeros((L, 4))
        y0[:, k] = 1.0
        M[:, :, k] = oracle.affine_solve(A, b0, y0)[:, -1]
    c = oracle.affine_solve(A, b)[:, -1]
    return M, c


def _worker(rank, world, port, T, seed, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(seed)
        L = 3
        A = rng.uniform(-0.4, 0.4, size=(L, T, 4, 4))
        b = rng.normal(size=(L, T, 4))
        t0, t1 = cp.split_time(T, world)[rank]
        M, c = _slice_map(A[:, t0:t1], b[:, t0:t1])
        mine = torch.from_numpy(np.concatenate([M.reshape(L, 16), c], axis=1))
        maps = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(maps, mine)
        carry = np.zeros((L, 4))
        for q in range(rank):
            mq = maps[q].numpy()
            carry = np.einsum("lij,lj->li", mq[:, :16].reshape(L, 4, 4), carry) + mq[:, 16:]
        y = oracle.affine_solve(A[:, t0:t1], b[:, t0:t1], carry)
        ys = [torch.empty(L, T, 4, dtype=torch.float64) for _ in range(world)]
        pad = torch.zeros(L, T, 4, dtype=torch.float64)
        pad[:, t0:t1] = torch.from_numpy(y)
        dist.all_gather(ys, pad)
        if rank == 0:
            full = oracle.affine_solve(A, b)
            got = sum(yy.numpy() for yy in ys)
            out.put(float(np.abs(got - full).max()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 37), (3, 50)])
def test_context_parallel_scan_composition_gloo(world, T):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + world * 7 + T % 5
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, 5, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert q.get(timeout=10) <= 1e-12
