"""The two tile shapes of the tensor-core GEMMs ("sLSTM in this library",
section "API notes": W_x is a GEMM): 256 x 256 tiles on SM pairs (clusters of
two CTAs, tcgen05 cta_group::2) and 128 x 256 tiles on single SMs (the
default setting takes pairs for long K only).  Every bf16 GEMM of the library runs in both shapes here: the input
projection against the fp64 oracle and across shapes, the gradient GEMMs of
the backward (dx, dW_x with split-K) and the trunk layer's GEMMs (SwiGLU and
residual epilogues, the FFN gradient GEMMs) across shapes.  Ragged M, N and K
(edge tiles of both shapes), several waves of work items (the two TMEM
accumulators and the ring reused many times), and exact multiples.

The input projection gives identical results in both shapes.  The backward
and the trunk layer are not bitwise reproducible from run to run (the
decoupled look-back of the adjoint composes the carry in an order that
depends on timing, and the split-K count of a weight gradient follows the
tile shape), so their outputs are compared within a bound:
|pair - single| <= 1e-5 (1 + max |g|), beside the oracle checks of the
backward and trunk-layer tests, which run in the default setting.
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import Workload, as_f64, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture
def tiles():
    prev = api.set_gemm_tiles("auto")
    yield
    api.set_gemm_tiles(prev)


def _close(a, b, tol=1e-5):
    err = float((a - b).abs().max()) / (1.0 + float(b.abs().max()))
    return err <= tol, err


def _both(fn):
    """fn() with every GEMM on SM pairs, then on single SMs."""
    api.set_gemm_tiles("pair")
    a = fn()
    torch.cuda.synchronize()
    api.set_gemm_tiles("single")
    b = fn()
    torch.cuda.synchronize()
    api.set_gemm_tiles("auto")
    return a, b


@pytest.mark.parametrize("B,T,d_in,d_h", [(2, 300, 64, 96), (3, 77, 24, 40), (4, 128, 512, 64), (1, 1000, 1032, 200)])
def test_preact_both_tile_shapes_match_oracle(B, T, d_in, d_h, tiles, cuda_device):
    w = Workload("t", B, T, d_in, d_h, "bf16", "sigmoid", 0.5, 7, 1e-6, 16)
    inp = make_inputs(w, with_dH=False)
    x, Wx, b = (inp[k].cuda() for k in ("x", "Wx", "bias"))
    Pp, Ps = _both(lambda: api.preact_gemm(x, Wx, b))
    assert torch.equal(Pp, Ps)
    ref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    err = np.abs(as_f64(Pp.cpu()) - ref).max() / (1 + np.abs(ref).max())
    assert err < 1e-5, err


def test_preact_both_tile_shapes_many_waves(tiles, cuda_device):
    """M = 16384, N = 4096, K = 1024: 1024 pair tiles over the persistent
    clusters; sampled rows against the oracle."""
    w = Workload("t", 8, 2048, 1024, 1024, "bf16", "sigmoid", 0.5, 8, 1e-6, 16)
    inp = make_inputs(w, with_dH=False)
    x, Wx, b = (inp[k].cuda() for k in ("x", "Wx", "bias"))
    Pp, Ps = _both(lambda: api.preact_gemm(x, Wx, b))
    assert torch.equal(Pp, Ps)
    rng = np.random.default_rng(3)
    for bi, t in zip(rng.integers(0, 8, 6), rng.integers(0, 2048, 6)):
        xr = as_f64(inp["x"][bi, t:t + 1])
        ref = oracle.gemm(xr, as_f64(inp["Wx"]), tb=True).reshape(4, 1024) + as_f64(inp["bias"])
        got = as_f64(Pp[bi, t].cpu())
        assert np.abs(got - ref).max() / (1 + np.abs(ref).max()) < 1e-5


@pytest.mark.parametrize("B,T,d_in,d_h", [(2, 300, 64, 96), (1, 517, 1024, 256)])
def test_backward_gemms_both_tile_shapes(B, T, d_in, d_h, tiles, cuda_device):
    w = Workload("t", B, T, d_in, d_h, "bf16", "sigmoid", 0.5, 9, 1e-6, 32)
    inp = make_inputs(w)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    P = api.preact_gemm(dev["x"], dev["Wx"], dev["bias"])
    S, st = api.newton_forward(P, dev["R"], dev["s0"], max_iters=32, tol=1e-6)
    assert api.read_stats(st)["converged"]

    def run():
        out = api.newton_backward(dev["x"], dev["Wx"], P, dev["R"], dev["s0"], S, dev["dH"])
        return {k: v.clone() for k, v in out.items()}

    gp, gs = _both(run)
    for k in ("dx", "dWx", "dR", "db", "ds0"):
        ok, err = _close(gp[k], gs[k])
        assert ok, (k, err)


@pytest.mark.parametrize("B,T,D,F", [(2, 40, 64, 256), (1, 300, 96, 384)])
def test_block_both_tile_shapes(B, T, D, F, tiles, cuda_device):
    g = torch.Generator().manual_seed(31)
    x = torch.randn(B, T, D, generator=g).cuda()
    w1 = (torch.rand(D, generator=g) + 0.5).cuda()
    w2 = (torch.rand(D, generator=g) + 0.5).cuda()
    Wx = (torch.randn(4 * D, D, generator=g) * D ** -0.5).to(torch.bfloat16).cuda()
    bias = torch.zeros(4, D).cuda()
    R = ((torch.rand(4, D, generator=g) * 2 - 1) * 0.5).cuda()
    Wg = (torch.randn(F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
    Wu = (torch.randn(F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
    W_gu = api.interleave_gate_up(Wg, Wu).contiguous().cuda()
    Wd = (torch.randn(D, F, generator=g) * F ** -0.5).to(torch.bfloat16).cuda()
    dY = torch.randn(B, T, D, generator=g).cuda()

    def run():
        y, S, _ = api.block_forward(x, w1, Wx, bias, R, w2, W_gu, Wd, max_iters=64, tol=1e-6)
        out = api.block_backward(x, w1, Wx, bias, R, w2, W_gu, Wd, S, dY)
        return y.clone(), {k: v.clone() for k, v in out.items()}

    (yp, gp), (ys, gs) = _both(run)
    ok, err = _close(yp, ys)
    assert ok, ("y", err)
    for k in gp:
        ok, err = _close(gp[k], gs[k])
        assert ok, (k, err)
