"""GPU parity of the trunk layer's forward (RMSNorm -> cell -> residual ->
RMSNorm -> SwiGLU -> residual) against the fp64 oracle with the same bf16
rounding of the GEMM operands.  Sizes ragged against the 32-feature tiles,
the 128 x 256 GEMM tiles and the 32-step time tiles; both forget modes;
in-place output.  Tolerance as for the bf16 path: |dy| <= 5e-3 (1 + |y|)."""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import as_f64

pytestmark = pytest.mark.gpu

TOL = 5e-3


def _params(B, T, D, F, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, D, generator=g)
    w1 = torch.rand(D, generator=g) + 0.5
    w2 = torch.rand(D, generator=g) + 0.5
    Wx = (torch.randn(4 * D, D, generator=g) * D ** -0.5).to(torch.bfloat16)
    bias = torch.zeros(4, D)
    bias[2] = torch.linspace(3.0, 6.0, D)
    R = (torch.rand(4, D, generator=g) * 2 - 1) * 0.5
    Wg = (torch.randn(F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
    Wu = (torch.randn(F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
    Wd = (torch.randn(D, F, generator=g) * F ** -0.5).to(torch.bfloat16)
    return x, w1, w2, Wx, bias, R, Wg, Wu, Wd


def _ref(p, forget, eps=1e-6):
    x, w1, w2, Wx, bias, R, Wg, Wu, Wd = p
    return oracle.block_forward(as_f64(x), as_f64(w1), as_f64(Wx), as_f64(bias), as_f64(R), as_f64(w2), as_f64(Wg),
                                as_f64(Wu), as_f64(Wd), forget, eps, bf16_operands=True)


def _run(p, forget, y=None, x_override=None):
    x, w1, w2, Wx, bias, R, Wg, Wu, Wd = [t.cuda() for t in p]
    if x_override is not None:
        x = x_override
    W_gu = api.interleave_gate_up(Wg, Wu).contiguous()
    return api.block_forward(x, w1, Wx, bias, R, w2, W_gu, Wd, forget=forget, max_iters=64, tol=1e-6, y=y)


@pytest.mark.parametrize("B,T,D,F,forget", [(2, 64, 64, 256, "sigmoid"), (2, 8, 96, 384, "exp"),
                                            (2, 300, 96, 384, "exp"), (2, 700, 64, 256, "sigmoid"),
                                            (3, 40, 136, 544, "sigmoid"), (1, 33, 264, 1056, "sigmoid"),
                                            (3, 60, 64, 256, "sigmoid")])
def test_block_forward_matches_oracle(B, T, D, F, forget, cuda_device):
    p = _params(B, T, D, F, 81)
    y, S, st = _run(p, forget)
    torch.cuda.synchronize()
    s = api.read_stats(st)
    assert s["error"] == 0 and s["converged"], s
    yref, Sref = _ref(p, forget)
    got = as_f64(y.cpu())
    err = float((np.abs(got - yref) / (1 + np.abs(yref))).max())
    assert err <= TOL, err
    h, hr = as_f64(S[:, :, 3].cpu()), Sref[:, :, 3]
    assert float((np.abs(h - hr) / (1 + np.abs(hr))).max()) <= TOL
    # the layer is not the identity: the FFN and the cell both moved y
    assert np.abs(yref - as_f64(p[0])).max() > 0.1


def test_block_forward_in_place(cuda_device):
    p = _params(2, 48, 64, 256, 82)
    y, _, _ = _run(p, "sigmoid")
    x = p[0].cuda()
    y2, _, _ = _run(p, "sigmoid", y=x, x_override=x)
    torch.cuda.synchronize()
    assert y2.data_ptr() == x.data_ptr() and torch.equal(y2, y)


@pytest.mark.parametrize("B,T,D,F,forget", [(2, 40, 64, 256, "sigmoid"), (1, 33, 96, 384, "sigmoid"),
                                            (2, 8, 64, 256, "exp")])
def test_block_backward_matches_oracle(B, T, D, F, forget, cuda_device):
    """Gradients of sum(dY * y) from the forward's S against the oracle's
    gradient of the unrounded layer; the GPU's recomputed z1, z2 are the
    forward's bf16 values, so the per-tensor bound is the bf16 one for
    gradients, 1e-2 (1 + max |g|)."""
    p = _params(B, T, D, F, 83)
    x, w1, w2, Wx, bias, R, Wg, Wu, Wd = p
    y, S, st = _run(p, forget)
    torch.cuda.synchronize()
    assert api.read_stats(st)["converged"]
    dY = torch.randn(B, T, D, generator=torch.Generator().manual_seed(84))
    d = [t.cuda() for t in (x, w1, Wx, bias, R, w2)]
    W_gu = api.interleave_gate_up(Wg, Wu).contiguous().cuda()
    out = api.block_backward(d[0], d[1], d[2], d[3], d[4], d[5], W_gu, Wd.cuda(), S, dY.cuda(), forget=forget)
    torch.cuda.synchronize()
    ref = oracle.block_backward(as_f64(x), as_f64(w1), as_f64(Wx), as_f64(bias), as_f64(R), as_f64(w2), as_f64(Wg),
                                as_f64(Wu), as_f64(Wd), as_f64(dY), forget)
    gu = as_f64(out["dW_gu"].cpu()).reshape(F // 32, 2, 32, D)
    got = {k: as_f64(out[k].cpu()) for k in ("dx", "dnorm1_w", "dWx", "dbias", "dR", "dnorm2_w", "dW_down")}
    got["dW_gate"] = gu[:, 0].reshape(F, D)
    got["dW_up"] = gu[:, 1].reshape(F, D)
    for k, g in got.items():
        r = ref[k]
        err = float(np.abs(g - r).max() / (1 + np.abs(r).max()))
        assert err <= 1e-2, (k, err)
