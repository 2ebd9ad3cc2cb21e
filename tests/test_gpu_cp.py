"""Time context parallelism on one GPU: the ranks' time slices run one after
another in this process (local_collectives: every phase of every rank
completes before the exchange that follows it, and no rank waits on
another), through the same C-ABI phases and driver the multi-GPU path uses.
Checked against the single-GPU solve and the fp64 oracle on the same inputs:
the guess with its refinement sweeps, the fixed-K iterate, and the converged
solution, for 1 to 4 ranks with slices that are not multiples of the
kernels' 64-step tiles, ragged feature counts and both forget modes.
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api, cp
from nonlinear_rnn_pararnn_b200.workloads import Workload, as_f64, make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _case(B, T, d, forget, seed):
    w = Workload("cp", B, T, 16, d, "f32", forget, 0.5, seed, 1e-5, 16)
    inp = make_inputs(w, with_dH=False)
    g = torch.Generator().manual_seed(seed + 1)
    s0 = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                      torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    P32 = torch.from_numpy(Pref).float().cuda()
    return inp, s0.cuda(), Pref, P32


def _slices(P, world):
    T = P.shape[1]
    return [cp.Slice(r, P[:, t0:t1].contiguous()) for r, (t0, t1) in enumerate(cp.split_time(T, world))]


def _joined(slices):
    return torch.cat([sl.S for sl in slices], dim=1)


def _s_err(S, ref):
    return float((np.abs(S - ref) / (1 + np.abs(ref))).max())


def _h_err(S, ref):
    h = ref[:, :, 3, :]
    return float((np.abs(S[:, :, 3, :] - h) / (1 + np.abs(h))).max())


def test_split_time_partitions():
    for T, n in ((10, 3), (64, 4), (1000, 3), (5, 5)):
        sp = cp.split_time(T, n)
        assert sp[0][0] == 0 and sp[-1][1] == T and len(sp) == n
        assert all(a[1] == b[0] for a, b in zip(sp, sp[1:]))
        assert max(b - a for a, b in sp) - min(b - a for a, b in sp) <= 1
    with pytest.raises(ValueError):
        cp.split_time(3, 4)


@pytest.mark.parametrize("sweeps", [0, 2])
@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_cp_guess_matches_single_gpu_and_oracle(world, forget, sweeps, cuda_device):
    B, T, d = 2, 1000, 40
    inp, s0, Pref, P = _case(B, T, d, forget, 5 + world)
    R = inp["R"].cuda()
    slices = _slices(P, world)
    cp.newton_forward(slices, R, s0, forget=forget, max_iters=0, guess_sweeps=sweeps)
    S = as_f64(_joined(slices).cpu())
    S1, _ = api.newton_forward(P, R, s0, forget=forget, max_iters=0, guess_sweeps=sweeps)
    Sg, _ = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(s0), forget, 0, False, 1e-5, sweeps=sweeps)
    assert _s_err(S, Sg) <= TOL
    assert _s_err(S, as_f64(S1.cpu())) <= TOL


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("B,T,d,forget", [(2, 1000, 40, "sigmoid"), (3, 777, 64, "exp"), (1, 2500, 36, "sigmoid")])
def test_cp_newton_matches_single_gpu_and_oracle(world, B, T, d, forget, cuda_device):
    inp, s0, Pref, P = _case(B, T, d, forget, 11 + world)
    R = inp["R"].cuda()
    # the fixed-K iterate: the same arithmetic as the single-GPU solve, split over time
    K = 2
    slices = _slices(P, world)
    st = cp.newton_forward(slices, R, s0, forget=forget, max_iters=K, fixed=True)
    assert st["iters"] == K
    SK1, _ = api.newton_forward(P, R, s0, forget=forget, max_iters=K, fixed=True)
    SKo, _ = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(s0), forget, K, True, 1e-5,
                                sweeps=api.DEFAULT_GUESS_SWEEPS)
    SK = as_f64(_joined(slices).cpu())
    assert _s_err(SK, SKo) <= TOL
    assert _s_err(SK, as_f64(SK1.cpu())) <= TOL
    # converged: the sequential trajectory, in about as many iterations
    slices = _slices(P, world)
    st = cp.newton_forward(slices, R, s0, forget=forget, max_iters=16, tol=1e-5)
    S1, st1 = api.newton_forward(P, R, s0, forget=forget, max_iters=16, tol=1e-5)
    s1 = api.read_stats(st1)
    print("cp", st, "single", s1["iters"], s1["max_scaled_F"])
    assert st["converged"] and not st["diverged"], st
    assert abs(st["iters"] - s1["iters"]) <= 1
    ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(s0), forget)
    assert _h_err(as_f64(_joined(slices).cpu()), ref) <= TOL


def test_cp_world_one_equals_the_single_call(cuda_device):
    inp, s0, Pref, P = _case(2, 300, 64, "sigmoid", 3)
    R = inp["R"].cuda()
    slices = _slices(P, 1)
    st = cp.newton_forward(slices, R, s0, max_iters=16, tol=1e-5)
    # the context-parallel solve records every iteration's exact residual
    S1, st1 = api.newton_forward(P, R, s0, max_iters=16, tol=1e-5, exact_history=True)
    s1 = api.read_stats(st1)
    assert st["iters"] == s1["iters"]
    np.testing.assert_allclose(st["max_scaled_F"], s1["max_scaled_F"], rtol=1e-3, atol=1e-7)
    assert _s_err(as_f64(_joined(slices).cpu()), as_f64(S1.cpu())) <= TOL
