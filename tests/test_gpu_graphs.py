"""The library's calls are stream-ordered, allocate nothing given their
buffers and never synchronise, so a whole training step (input projection,
Newton solve, backward) and a trunk-layer forward capture into one CUDA graph.
Replays must reproduce the eager results, also after new inputs are written
into the captured buffers.  The decoupled look-back may group a tile's
predecessor maps differently from run to run (which ones have published
their prefixes yet), so results are compared within the parity tolerance,
not bit for bit."""
import pytest
import torch

from nonlinear_rnn_pararnn_b200 import _lib, api
from nonlinear_rnn_pararnn_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _close(a, b, tol=1e-4):
    """Within the parity tolerance: |a - b| <= tol (1 + max |b|) (NaN fails)."""
    return float((a - b).abs().max()) <= tol * (1 + float(b.abs().max()))


def _capture(step):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                      # first call outside the capture (one-time set-up)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    return graph


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_training_step_replays_under_cuda_graph(dtype, cuda_device):
    # solved to convergence, so that replay and eager runs are compared on the
    # solution
    w = Workload("graph", 2, 64, 32, 64, dtype, "sigmoid", 0.5, 91, 1e-6, 64)
    inp = make_inputs(w)
    x, Wx, R, bias, s0, dH = (inp[k].cuda() for k in ("x", "Wx", "R", "bias", "s0", "dH"))
    B, T, d_in, d = w.B, w.T, w.d_in, w.d_h
    P = torch.empty(B, T, 4, d, device="cuda")
    S = torch.empty_like(P)
    stats = api.new_stats()
    ws_p = api.workspace(_lib.SLSTM_OP_PREACT_GEMM, B, T, d_in, d)
    ws_f = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD, B, T, 0, d)
    ws_b = api.workspace(_lib.SLSTM_OP_NEWTON_BACKWARD, B, T, d_in, d)
    out = {"dx": torch.empty(B, T, d_in, device="cuda"), "dWx": torch.empty(4 * d, d_in, device="cuda"),
           "dR": torch.empty(4, d, device="cuda"), "db": torch.empty(4, d, device="cuda"),
           "ds0": torch.empty(B, 4, d, device="cuda")}

    def step():
        api.preact_gemm(x, Wx, bias, P=P, ws=ws_p)
        api.newton_forward(P, R, s0, max_iters=64, tol=1e-6, S=S, stats=stats, ws=ws_f)
        api.newton_backward(x, Wx, P, R, s0, S, dH, out=out, ws=ws_b)

    def snapshot():
        torch.cuda.synchronize()
        return {"S": S.clone(), **{k: v.clone() for k, v in out.items()}}

    step()
    eager = snapshot()
    graph = _capture(step)
    for t in [S, *out.values()]:
        t.fill_(float("nan"))
    graph.replay()
    got = snapshot()
    for k in eager:
        assert _close(got[k], eager[k]), k
    st = api.read_stats(stats)
    assert st["converged"] and st["error"] == 0, st
    # new inputs in the captured buffers: the two batch rows swapped, so the
    # problems (and their convergence) are the same ones, in the other order
    x.copy_(torch.flip(x, dims=[0]))
    dH.copy_(torch.flip(dH, dims=[0]))
    graph.replay()
    got = snapshot()
    assert api.read_stats(stats)["converged"]
    for k in ("S", "dx", "ds0"):
        assert _close(got[k], torch.flip(eager[k], dims=[0])), k
    for k in ("dWx", "dR", "db"):      # sums over the rows
        assert _close(got[k], eager[k]), k
    step()
    again = snapshot()
    for k in again:
        assert _close(got[k], again[k]), k


def test_block_forward_replays_under_cuda_graph(cuda_device):
    g = torch.Generator().manual_seed(92)
    B, T, D, F = 2, 48, 64, 256
    x = torch.randn(B, T, D, generator=g).cuda()
    w1, w2 = (torch.rand(D, generator=g) + 0.5).cuda(), (torch.rand(D, generator=g) + 0.5).cuda()
    Wx = (torch.randn(4 * D, D, generator=g) * D ** -0.5).to(torch.bfloat16).cuda()
    bias = torch.zeros(4, D)
    bias[2] = torch.linspace(3.0, 6.0, D)
    bias = bias.cuda()
    R = ((torch.rand(4, D, generator=g) * 2 - 1) * 0.5).cuda()
    W_gu = (torch.randn(2 * F, D, generator=g) * D ** -0.5).to(torch.bfloat16).cuda()
    W_down = (torch.randn(D, F, generator=g) * F ** -0.5).to(torch.bfloat16).cuda()
    y = torch.empty_like(x)
    S = torch.empty(B, T, 4, D, device="cuda")
    stats = api.new_stats()
    ws = api.block_workspace(B, T, D, F)

    def step():
        api.block_forward(x, w1, Wx, bias, R, w2, W_gu, W_down, max_iters=64, tol=1e-6, y=y, S=S, stats=stats,
                          ws=ws)

    step()
    torch.cuda.synchronize()
    eager = y.clone()
    graph = _capture(step)
    y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert _close(y, eager)
    assert api.read_stats(stats)["converged"]
    x.mul_(0.75)
    graph.replay()
    torch.cuda.synchronize()
    got = y.clone()
    step()
    torch.cuda.synchronize()
    assert _close(got, y)
