"""GPU parity of the fused decode step (input projection + cell update, one
launch per step) against the fp64 oracle's input projection and sequential
solve, token by token; batch rows beyond one launch's 16, ragged feature
counts, the zero initial state, in-place stepping and replay under a CUDA
graph.  Tolerance as for the fp32 solve: |ds| <= 1e-4 (1 + |s|)."""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import Workload, as_f64, make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _case(B, T, d_in, d, dtype, forget, seed):
    w = Workload("dec", B, T, d_in, d, dtype, forget, 0.5, seed, 1e-6, 8)
    inp = make_inputs(w, with_dH=False)
    g = torch.Generator().manual_seed(seed + 500)
    s0 = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                      torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    return inp, s0


def _ref(inp, s0, forget):
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    B, T, _, d = Pref.shape
    S = oracle.sequential_btgd(Pref, as_f64(inp["R"]), np.zeros((B, 4, d)) if s0 is None else as_f64(s0), forget)
    return np.transpose(S, (1, 0, 2, 3))   # (T, B, 4, d)


def _err(got, ref):
    return float((np.abs(got - ref) / (1 + np.abs(ref))).max())


@pytest.mark.parametrize("B,d_in,d,dtype,forget", [(3, 16, 40, "f32", "sigmoid"), (8, 64, 64, "bf16", "sigmoid"),
                                                   (20, 32, 33, "f32", "exp"), (17, 128, 96, "bf16", "exp"),
                                                   (1, 8, 8, "bf16", "sigmoid")])
def test_decode_matches_oracle(B, d_in, d, dtype, forget, cuda_device):
    T = 12
    inp, s0 = _case(B, T, d_in, d, dtype, forget, 61)
    xs = inp["x"].transpose(0, 1).contiguous().cuda()
    S = api.decode(xs, inp["Wx"].cuda(), inp["bias"].cuda(), inp["R"].cuda(), s0.cuda(), forget=forget)
    torch.cuda.synchronize()
    assert _err(as_f64(S.cpu()), _ref(inp, s0, forget)) <= TOL


def test_decode_zero_state_and_in_place(cuda_device):
    B, T, d_in, d = 5, 6, 16, 40
    inp, _ = _case(B, T, d_in, d, "f32", "sigmoid", 62)
    xs = inp["x"].transpose(0, 1).contiguous().cuda()
    Wx, b, R = inp["Wx"].cuda(), inp["bias"].cuda(), inp["R"].cuda()
    S = api.decode(xs, Wx, b, R, None)
    # the same steps in place in one state buffer, starting from explicit zeros
    s = torch.zeros(B, 4, d, device="cuda")
    for t in range(T):
        api.decode_step(xs[t], Wx, b, R, s, out=s)
        assert torch.equal(s, S[t])
    torch.cuda.synchronize()
    assert _err(as_f64(S.cpu()), _ref(inp, None, "sigmoid")) <= TOL


def test_decode_replays_under_cuda_graph(cuda_device):
    B, T, d_in, d = 4, 8, 64, 64
    inp, s0 = _case(B, T, d_in, d, "bf16", "sigmoid", 63)
    xs = inp["x"].transpose(0, 1).contiguous().cuda()
    Wx, b, R, s0d = inp["Wx"].cuda(), inp["bias"].cuda(), inp["R"].cuda(), s0.cuda()
    eager = api.decode(xs, Wx, b, R, s0d)
    S = torch.empty_like(eager)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        api.decode(xs, Wx, b, R, s0d, S=S)   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    S.zero_()
    with torch.cuda.graph(graph):
        api.decode(xs, Wx, b, R, s0d, S=S)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(S, eager)
    # new inputs in the same buffers, replayed
    xs.copy_(torch.flip(xs, dims=[0]))
    graph.replay()
    ref = api.decode(xs, Wx, b, R, s0d)
    torch.cuda.synchronize()
    assert torch.equal(S, ref)
