"""GPU parity of the d_h tensor-parallel split: the ranks' shares run one after
another on one GPU (they never wait on one another), their partial input
gradients are added, and everything is compared with the fp64 oracle on the
full problem.  Shards of whole 32-feature groups plus a ragged last shard;
three ranks over 72 features leave one rank with 32, one with 32 and one with
8 features, four ranks over 72 leave one rank empty."""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api, tp
from nonlinear_rnn_pararnn_b200.workloads import Workload, as_f64, make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4
TF = 60


def _case(B, T, d_in, d, dtype, seed):
    w = Workload("tp", B, T, d_in, d, dtype, "sigmoid", 0.5, seed, 1e-6, 64)
    inp = make_inputs(w, with_dH=True)
    g = torch.Generator().manual_seed(seed + 300)
    inp["s0"] = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                             torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    return inp


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("B,T,d_in,d,dtype", [(2, 300, 16, 72, "f32"), (2, 200, 64, 72, "bf16"),
                                              (1, 150, 32, 100, "bf16")])
def test_tensor_parallel_shards_match_oracle(world, B, T, d_in, d, dtype, cuda_device):
    inp = _case(B, T, d_in, d, dtype, 71)
    x = inp["x"].cuda()
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    Sref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]))
    gref = oracle.backward_btgd(as_f64(inp["x"]), as_f64(inp["Wx"]), Pref, as_f64(inp["R"]), as_f64(inp["s0"]),
                                Sref, as_f64(inp["dH"]))
    dx = torch.zeros(B, T, d_in, device="cuda")
    for r in range(world):
        j0, j1 = tp.feature_range(d, world, r)
        Wl, bl, Rl = tp.shard_params(inp["Wx"], inp["bias"], inp["R"], j0, j1)
        Wl, bl, Rl = Wl.cuda(), bl.cuda(), Rl.cuda()
        s0l = tp.shard_state(inp["s0"], j0, j1).cuda()
        # forward to convergence on the first TF steps (Newton from the zero
        # guess converges in fp32 there); the backward below runs on all T
        _, S, st = tp.forward(x[:, :TF].contiguous(), Wl, bl, Rl, s0l, max_iters=64, tol=1e-6)
        P, _, _ = tp.forward(x, Wl, bl, Rl, s0l, max_iters=1, fixed=True)
        torch.cuda.synchronize()
        if j1 == j0:
            assert st is None and S.shape[-1] == 0
        else:
            s = api.read_stats(st)
            assert s["error"] == 0 and s["converged"], (r, s)
            h, hr = as_f64(S[:, :, 3].cpu()), Sref[:, :TF, 3, j0:j1]
            assert float((np.abs(h - hr) / (1 + np.abs(hr))).max()) <= TOL, r
            p, pr = as_f64(P.cpu()), Pref[..., j0:j1]
            assert float((np.abs(p - pr) / (1 + np.abs(pr))).max()) <= 1e-5, r
        # backward from the oracle's solution so that only the gradient kernels are compared
        Sl = torch.from_numpy(np.ascontiguousarray(Sref[..., j0:j1])).float().cuda()
        out = tp.backward(x, Wl, P, Rl, s0l, Sl, tp.shard_state(inp["dH"], j0, j1).cuda(), reduce=False)
        dx += out["dx"]
        rows = np.concatenate([np.arange(gi * d + j0, gi * d + j1) for gi in range(4)])
        for k, ref in (("dWx", gref["dWx"][rows]), ("dR", gref["dR"][:, j0:j1]), ("db", gref["db"][:, j0:j1]),
                       ("ds0", gref["ds0"][..., j0:j1])):
            if ref.size:
                got = as_f64(out[k].cpu())
                err = np.abs(got - ref).max() / (1 + np.abs(ref).max())
                assert err <= TOL, (r, k, err)
    torch.cuda.synchronize()
    err = np.abs(as_f64(dx.cpu()) - gref["dx"]).max() / (1 + np.abs(gref["dx"]).max())
    assert err <= TOL, err
