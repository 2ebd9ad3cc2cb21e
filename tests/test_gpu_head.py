"""GPU parity of the head-mixing calls ("sLSTM in this library", section
"Cell", row 'head': block-diagonal R (4, n_heads, d_head, d_head)) against the
fp64 oracle on the same seeded inputs: sequential stepping, the Newton solve
(converged, and the fixed-K iterate from the same guess), and every gradient.
Head widths 1 (diag mixing by another route), 3, 8, 12 and 32 (the largest a
warp serves); several warps per CTA and several CTAs.

Tolerances as the diag tests: max|dh| <= 1e-4 (1 + |h|) for fp32 inputs,
5e-3 for bf16 inputs; gradients 1e-4 (1 + max|g|) for fp32 inputs, 1e-3 for
bf16 inputs (the tensor-core GEMMs of dx and dW_x).
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import Workload, as_f64, make_inputs

pytestmark = pytest.mark.gpu


def _case(B, T, d, dh, forget, seed, dtype="f32", s0_random=True):
    w = Workload("head", B, T, 16, d, dtype, forget, 0.5, seed, 1e-6, 32)
    inp = make_inputs(w, with_dH=True)
    g = torch.Generator().manual_seed(seed + 1)
    H = d // dh
    # R ~ U(-a, a) per block entry, scaled by d_head^-1/2 so that a head's
    # recurrent input has the diag workloads' magnitude
    Rh = (torch.rand(4, H, dh, dh, generator=g) * 2 - 1) * (0.5 / dh ** 0.5)
    s0 = inp["s0"]
    if s0_random:
        s0 = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                          torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    P = api.preact_gemm(inp["x"].cuda(), inp["Wx"].cuda(), inp["bias"].cuda())
    return inp, Rh, s0, P, Pref


def _h_err(S, ref):
    h = ref[:, :, 3, :]
    return float((np.abs(S[:, :, 3, :] - h) / (1 + np.abs(h))).max())


def _s_err(S, ref):
    return float((np.abs(S - ref) / (1 + np.abs(ref))).max())


SHAPES = [(2, 40, 32, 8), (3, 33, 36, 12), (2, 50, 64, 32), (1, 20, 6, 3), (2, 30, 8, 1), (5, 17, 96, 32)]


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d,dh", SHAPES)
def test_head_sequential_matches_oracle(B, T, d, dh, forget, cuda_device):
    inp, Rh, s0, P, Pref = _case(B, T, d, dh, forget, 61)
    S = api.sequential_step_head(P, Rh.cuda(), s0.cuda(), forget=forget)
    torch.cuda.synchronize()
    ref = oracle.sequential_head(Pref, as_f64(Rh), as_f64(s0), forget)
    assert _h_err(as_f64(S.cpu()), ref) <= 1e-4


def test_head_sequential_long(cuda_device):
    inp, Rh, s0, P, Pref = _case(2, 1500, 16, 8, "sigmoid", 62)
    S = api.sequential_step_head(P, Rh.cuda(), s0.cuda())
    ref = oracle.sequential_head(Pref, as_f64(Rh), as_f64(s0))
    assert _h_err(as_f64(S.cpu()), ref) <= 1e-4


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d,dh", [(2, 40, 32, 8), (1, 20, 6, 3), (2, 30, 64, 32)])
def test_head_newton_converges_and_matches_fixed_k(B, T, d, dh, forget, cuda_device):
    inp, Rh, s0, P, Pref = _case(B, T, d, dh, forget, 63)
    Rd, s0d = Rh.cuda(), s0.cuda()
    S, st = api.newton_forward_head(P, Rd, s0d, forget=forget, max_iters=30, tol=1e-6)
    s = api.read_stats(st)
    ref = oracle.sequential_head(Pref, as_f64(Rh), as_f64(s0), forget)
    _, ost = oracle.newton_head(Pref, as_f64(Rh), as_f64(s0), forget, max_iters=30, tol=1e-6)
    print("gpu", s["iters"], s["max_scaled_F"], "oracle", ost["iters"])
    assert s["converged"] and s["error"] == 0, s
    assert ost["converged"] and abs(s["iters"] - ost["iters"]) <= 1
    assert _h_err(as_f64(S.cpu()), ref) <= 1e-4
    # the whole iterate after K fixed iterations from the same decoupled guess
    K = 2
    SK, stK = api.newton_forward_head(P, Rd, s0d, forget=forget, max_iters=K, fixed=True, tol=1e-6)
    assert api.read_stats(stK)["iters"] == K
    oK, _ = oracle.newton_head(Pref, as_f64(Rh), as_f64(s0), forget, max_iters=K, fixed=True)
    assert _s_err(as_f64(SK.cpu()), oK) <= 1e-4


def test_head_newton_zero_guess_prefix_exact(cuda_device):
    inp, Rh, s0, P, Pref = _case(2, 24, 32, 8, "sigmoid", 64)
    ref = oracle.sequential_head(Pref, as_f64(Rh), as_f64(s0))
    for K in (1, 3):
        S, st = api.newton_forward_head(P, Rh.cuda(), s0.cuda(), max_iters=K, fixed=True, init="zero")
        assert api.read_stats(st)["iters"] == K
        assert _h_err(as_f64(S[:, :K].cpu()), ref[:, :K]) <= 1e-4


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d,dh", [(2, 40, 32, 8), (3, 33, 36, 12), (2, 30, 64, 32), (1, 20, 6, 3)])
def test_head_backward_matches_oracle(B, T, d, dh, forget, dtype, cuda_device):
    inp, Rh, s0, P, Pref = _case(B, T, d, dh, forget, 65, dtype=dtype)
    S = api.sequential_step_head(P, Rh.cuda(), s0.cuda(), forget=forget)
    out = api.newton_backward_head(inp["x"].cuda(), inp["Wx"].cuda(), P, Rh.cuda(), s0.cuda(), S, inp["dH"].cuda(),
                                   forget=forget)
    torch.cuda.synchronize()
    Sref = oracle.sequential_head(Pref, as_f64(Rh), as_f64(s0), forget)
    ref = oracle.backward_head(as_f64(inp["x"]), as_f64(inp["Wx"]), Pref, as_f64(Rh), as_f64(s0), Sref,
                               as_f64(inp["dH"]), forget)
    tol = 1e-4 if dtype == "f32" else 1e-3
    for k, rk in (("dx", "dx"), ("dWx", "dWx"), ("dR_head", "dRh"), ("db", "db"), ("ds0", "ds0")):
        got = as_f64(out[k].cpu())
        err = np.abs(got - ref[rk]).max() / (1 + np.abs(ref[rk]).max())
        assert err <= tol, (k, err)


@pytest.mark.parametrize("forget,dtype", [("sigmoid", "bf16"), ("exp", "f32")])
def test_head_newton_long_sequence_sampled_heads(forget, dtype, cuda_device):
    """A long sequence (T = 4096, 8 heads of 32): the converged GPU solve
    against the oracle's sequential trajectory of two sampled heads over every
    step (the heads are independent, so the oracle runs each alone)."""
    B, T, d, dh = 2, 4096, 256, 32
    w = Workload("head_long", B, T, 64, d, dtype, forget, 0.5, 17, 1e-5, 16)
    inp = make_inputs(w, with_dH=False)
    g = torch.Generator().manual_seed(18)
    H = d // dh
    Rh = (torch.rand(4, H, dh, dh, generator=g) * 2 - 1) * (0.5 / dh ** 0.5)
    P = api.preact_gemm(inp["x"].cuda(), inp["Wx"].cuda(), inp["bias"].cuda())
    S, st = api.newton_forward_head(P, Rh.cuda(), inp["s0"].cuda(), forget=forget, max_iters=16, tol=1e-5)
    s = api.read_stats(st)
    print("gpu", s["iters"], s["max_scaled_F"])
    assert s["converged"] and not s["diverged"] and s["error"] == 0, s
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    S_gpu = as_f64(S.cpu())
    tol = 5e-3 if dtype == "bf16" else 1e-4
    for hd in (1, H - 1):
        cols = slice(hd * dh, (hd + 1) * dh)
        ref = oracle.sequential_head(Pref[:, :, :, cols], as_f64(Rh[:, hd:hd + 1]), as_f64(inp["s0"])[:, :, cols],
                                     forget)
        assert _h_err(S_gpu[:, :, :, cols], ref) <= tol, (hd, _h_err(S_gpu[:, :, :, cols], ref))
