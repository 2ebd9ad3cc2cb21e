"""Host logic of the d_h tensor-parallel split on CPU: the feature ranges,
the gate-major row selection of W_x, and, with two gloo ranks, that each
rank's oracle forward and backward on its shard plus the all-reduce of the
partial input gradients give the full problem's results (the oracle stands in
for the kernels, which need a GPU)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from nonlinear_rnn_pararnn_b200 import tp  # noqa: E402


@pytest.mark.parametrize("d", [1, 31, 32, 33, 72, 100, 1024])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_feature_ranges_partition_the_features(d, world):
    rs = [tp.feature_range(d, world, r) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == d
    for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
        assert a1 == b0 and a0 <= a1
    for j0, j1 in rs:
        assert j0 % 32 == 0 and (j1 % 32 == 0 or j1 == d)
    sizes = [j1 - j0 for j0, j1 in rs]
    groups = [(s + 31) // 32 for s in sizes]
    assert max(groups) - min(groups) <= 1     # whole 32-feature groups, balanced


def test_feature_range_rejects_bad_rank():
    with pytest.raises(ValueError):
        tp.feature_range(64, 2, 2)
    with pytest.raises(ValueError):
        tp.feature_range(64, 0, 0)


def test_shard_params_selects_gate_major_rows():
    d, d_in = 5, 3
    Wx = torch.arange(4 * d * d_in, dtype=torch.float32).reshape(4 * d, d_in)
    bias = torch.arange(4 * d, dtype=torch.float32).reshape(4, d) + 100
    R = -torch.arange(4 * d, dtype=torch.float32).reshape(4, d)
    Wl, bl, Rl = tp.shard_params(Wx, bias, R, 1, 3)
    dl = 2
    assert Wl.shape == (4 * dl, d_in) and bl.shape == (4, dl) and Rl.shape == (4, dl)
    for g in range(4):
        for jl in range(dl):
            assert torch.equal(Wl[g * dl + jl], Wx[g * d + 1 + jl])
            assert bl[g, jl] == bias[g, 1 + jl] and Rl[g, jl] == R[g, 1 + jl]
    with pytest.raises(ValueError):
        tp.shard_params(Wx, bias, R, 3, 6)


def _problem():
    g = torch.Generator().manual_seed(7)
    B, T, d_in, d = 2, 20, 12, 72
    x = torch.randn(B, T, d_in, generator=g, dtype=torch.float64)
    Wx = torch.randn(4 * d, d_in, generator=g, dtype=torch.float64) * d_in ** -0.5
    bias = torch.zeros(4, d, dtype=torch.float64)
    bias[2] = torch.linspace(3.0, 6.0, d, dtype=torch.float64)
    R = (torch.rand(4, d, generator=g, dtype=torch.float64) * 2 - 1) * 0.5
    s0 = torch.stack([torch.randn(B, d, generator=g, dtype=torch.float64),
                      torch.rand(B, d, generator=g, dtype=torch.float64) + 0.5,
                      torch.randn(B, d, generator=g, dtype=torch.float64),
                      torch.rand(B, d, generator=g, dtype=torch.float64) - 0.5], dim=1)
    dH = torch.randn(B, T, d, generator=g, dtype=torch.float64)
    return x, Wx, bias, R, s0, dH


def _oracle_pass(x, Wx, bias, R, s0, dH):
    import oracle
    P = oracle.preact(x.numpy(), Wx.numpy(), bias.numpy())
    S = oracle.sequential_btgd(P, R.numpy(), s0.numpy())
    g = oracle.backward_btgd(x.numpy(), Wx.numpy(), P, R.numpy(), s0.numpy(), S, dH.numpy())
    return S, g


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from datetime import timedelta
    from nonlinear_rnn_pararnn_b200 import tp as tpm
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    x, Wx, bias, R, s0, dH = _problem()
    j0, j1 = tpm.feature_range(R.shape[1], world, rank)
    Wl, bl, Rl = tpm.shard_params(Wx, bias, R, j0, j1)
    S, g = _oracle_pass(x, Wl, bl, Rl, tpm.shard_state(s0, j0, j1), tpm.shard_state(dH, j0, j1))
    dx = torch.from_numpy(np.ascontiguousarray(g["dx"]))
    tpm.all_reduce_dx(dx)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, j0, j1, S, dx.numpy(), g["dWx"], g["dR"], g["db"], g["ds0"]))


@pytest.mark.parametrize("world", [2, 3])
def test_tensor_parallel_shards_match_full_problem_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        item = q.get(timeout=240)
        got[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, Wx, bias, R, s0, dH = _problem()
    S, g = _oracle_pass(x, Wx, bias, R, s0, dH)
    d = R.shape[1]
    # 72 features = three 32-feature groups: [0, 32) + [32, 72) for two ranks,
    # [0, 32) + [32, 64) + [64, 72) for three
    want = {2: [(0, 32), (32, 72)], 3: [(0, 32), (32, 64), (64, 72)]}[world]
    assert [(got[r][0], got[r][1]) for r in range(world)] == want and want[-1][1] == d
    for r in range(world):
        j0, j1, Sr, dx, dWx, dR, db, ds0 = got[r]
        np.testing.assert_allclose(Sr, S[..., j0:j1], rtol=0, atol=1e-12)
        # every rank holds the full input gradient after the all-reduce
        np.testing.assert_allclose(dx, g["dx"], rtol=0, atol=1e-10 * (1 + np.abs(g["dx"]).max()))
        rows = np.concatenate([np.arange(gi * d + j0, gi * d + j1) for gi in range(4)])
        np.testing.assert_allclose(dWx, g["dWx"][rows], rtol=0, atol=1e-10)
        np.testing.assert_allclose(dR, g["dR"][:, j0:j1], rtol=0, atol=1e-10)
        np.testing.assert_allclose(db, g["db"][:, j0:j1], rtol=0, atol=1e-10)
        np.testing.assert_allclose(ds0, g["ds0"][..., j0:j1], rtol=0, atol=1e-10)
    # one rank's partial alone is not the full gradient (the all-reduce is needed)
    Wl, bl, Rl = tp.shard_params(Wx, bias, R, 0, 32)
    _, gp = _oracle_pass(x, Wl, bl, Rl, tp.shard_state(s0, 0, 32), tp.shard_state(dH, 0, 32))
    assert np.abs(gp["dx"] - g["dx"]).max() > 1e-3


def test_empty_shard_forward_and_backward_need_no_kernels():
    """A rank beyond the group count owns no features: its forward returns
    empty (B, T, 4, 0) tensors and its backward a zero input gradient of the
    full shape (its share of the all-reduce) without calling the library."""
    B, T, d_in = 2, 5, 8
    x = torch.randn(B, T, d_in)
    Wl, bl, Rl = tp.shard_params(torch.zeros(4 * 32, d_in), torch.zeros(4, 32), torch.zeros(4, 32), 32, 32)
    assert Wl.shape == (0, d_in) and bl.shape == (4, 0) and Rl.shape == (4, 0)
    P, S, st = tp.forward(x, Wl, bl, Rl)
    assert P.shape == (B, T, 4, 0) and S.shape == (B, T, 4, 0) and st is None
    out = tp.backward(x, Wl, P, Rl, None, S, torch.empty(B, T, 0))
    assert out["dx"].shape == (B, T, d_in) and not out["dx"].any()
    assert out["dWx"].shape == (0, d_in) and out["dR"].shape == (4, 0)
