"""The device loop over Newton iterations (slstm_newton_config.loop_from;
"pararnn-torch structure", section "Current surface": the residual early
stop).  In tolerance mode with the fused carry the iterations from loop_from
on run inside one cooperative launch, a grid-wide barrier between two of
them, and the loop ends with the stopping rule.  Checked here against the
same solve with one launch per iteration (loop_from = -1) and against the
oracle's sequential trajectory: the same iteration count and convergence, and
iterates that agree to the rounding of the decoupled look-back (whose
grouping depends on timing).  Cases: the zero guess (many iterations inside
the loop), a solve that has converged before the loop starts, packed
sequences, more tiles than resident CTAs (every CTA takes several tiles per
iteration), and the bounded barrier's self-test (one CTA leaves; the others'
wait runs out and the call reports SLSTM_ERR_TIMEOUT).
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import _lib, api
from nonlinear_rnn_pararnn_b200.workloads import WORKLOADS, as_f64, make_inputs, scaled

pytestmark = pytest.mark.gpu


def _case(w):
    inp = make_inputs(w, with_dH=False)
    P = api.preact_gemm(inp["x"].cuda(), inp["Wx"].cuda(), inp["bias"].cuda())
    return inp, P, inp["R"].cuda(), inp["s0"].cuda()


def _solve(P, R, s0, w, **kw):
    S, st = api.newton_forward(P, R, s0, forget=w.forget, fixed=False, tol=w.tol, carry_mode=1, **kw)
    torch.cuda.synchronize()
    return S, api.read_stats(st)


def _rel(a, b):
    return float(((a - b).abs() / (1 + b.abs())).max())


@pytest.mark.parametrize("loop_from", [1, 2])
def test_loop_matches_per_launch_and_the_sequential_solution(loop_from, cuda_device):
    """tiny_f32 (B = 2, T = 64, d = 8, tol 1e-6) from the decoupled guess
    without sweeps: several iterations, those from loop_from on inside the
    loop; converged on the sequential trajectory."""
    w = WORKLOADS["tiny_f32"]
    inp, P, R, s0 = _case(w)
    S_ref, st_ref = _solve(P, R, s0, w, max_iters=64, guess_sweeps=0, loop_from=-1)
    S, st = _solve(P, R, s0, w, max_iters=64, guess_sweeps=0, loop_from=loop_from)
    assert st_ref["converged"], st_ref
    assert st["converged"] and st["error"] == 0 and st["iters"] == st_ref["iters"], (st, st_ref)
    assert _rel(S, S_ref) <= 1e-5
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), w.forget)
    h = as_f64(S[:, :, 3].cpu())
    assert float((np.abs(h - ref[:, :, 3]) / (1 + np.abs(ref[:, :, 3]))).max()) <= 1e-4


def test_loop_status_from_the_zero_guess_matches_per_launch(cuda_device):
    """From S = 0 (many iterations, all but the first inside the loop): the
    loop ends with the same record as one launch per iteration, whatever the
    outcome (converged, or diverged at the cap)."""
    w = WORKLOADS["tiny_f32"]
    inp, P, R, s0 = _case(w)
    S_ref, st_ref = _solve(P, R, s0, w, max_iters=40, init="zero", loop_from=-1)
    S, st = _solve(P, R, s0, w, max_iters=40, init="zero", loop_from=1)
    for k in ("iters", "converged", "diverged", "error"):
        assert st[k] == st_ref[k], (k, st, st_ref)
    if st["converged"]:
        assert _rel(S, S_ref) <= 1e-5


def test_loop_after_convergence_returns_at_once(cuda_device):
    """From the decoupled guess with two sweeps the solve converges in two
    iterations; with the default loop_from (2) the loop launch finds the
    solve done, and the record is that of the per-launch solve."""
    w = scaled(WORKLOADS["slstm_f32_b8_t1024_d256"], B=2, T=700, d_in=64, d_h=64)
    inp, P, R, s0 = _case(w)
    S_ref, st_ref = _solve(P, R, s0, w, max_iters=16, loop_from=-1)
    for lf in (0, 1):
        S, st = _solve(P, R, s0, w, max_iters=16, loop_from=lf)
        assert st["converged"] and st["iters"] == st_ref["iters"], (lf, st, st_ref)
        assert st["max_scaled_F"][-1] <= w.tol
        assert _rel(S, S_ref) <= 1e-5


def test_loop_with_more_tiles_than_resident_ctas(cuda_device):
    """B = 4, T = 4096, d = 256: 2048 tiles over at most one CTA per SM, so
    each CTA takes many tiles per iteration and the barrier separates real
    work; no refinement sweeps, so several iterations run inside the loop."""
    w = scaled(WORKLOADS["slstm_f32_b8_t1024_d256"], B=4, T=4096, d_in=64, d_h=256)
    inp, P, R, s0 = _case(w)
    S_ref, st_ref = _solve(P, R, s0, w, max_iters=32, guess_sweeps=0, loop_from=-1)
    S, st = _solve(P, R, s0, w, max_iters=32, guess_sweeps=0, loop_from=1)
    assert st["converged"] and st_ref["converged"] and st["iters"] == st_ref["iters"] >= 3, (st, st_ref)
    assert _rel(S, S_ref) <= 1e-5
    assert st["max_scaled_F"][-1] <= w.tol


def test_loop_packed_sequences(cuda_device):
    w = scaled(WORKLOADS["slstm_f32_b8_t1024_d256"], B=1, T=600, d_in=32, d_h=64)
    inp, P, R, _ = _case(w)
    lengths = [100, 0, 257, 1, 242]
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32).cuda()
    g = torch.Generator().manual_seed(5)
    s0 = torch.stack([torch.randn(5, 64, generator=g), torch.rand(5, 64, generator=g) + 0.5,
                      torch.randn(5, 64, generator=g), torch.rand(5, 64, generator=g) - 0.5], dim=1).cuda()
    out = {}
    for lf in (-1, 1):
        S, st = api.newton_forward_varlen(P[0], R, s0, cu, forget=w.forget, max_iters=32, tol=w.tol, carry_mode=1,
                                          guess_sweeps=0, loop_from=lf)
        torch.cuda.synchronize()
        out[lf] = (S, api.read_stats(st))
    (S_ref, st_ref), (S, st) = out[-1], out[1]
    assert st["converged"] and st["iters"] == st_ref["iters"] >= 2, (st, st_ref)
    assert _rel(S, S_ref) <= 1e-5


def test_loop_barrier_wait_runs_out_and_reports(cuda_device):
    """debug_fault = 3: CTA 0 of the loop leaves before the first grid
    barrier; every other CTA's wait ends after wait_limit_us with the error
    word's bit 4 set, stats.error = SLSTM_ERR_TIMEOUT, and the call returns."""
    w = scaled(WORKLOADS["slstm_f32_b8_t1024_d256"], B=2, T=700, d_in=64, d_h=64)
    inp, P, R, s0 = _case(w)
    ws = api.workspace(_lib.SLSTM_OP_NEWTON_FORWARD, w.B, w.T, 0, w.d_h, P.device)
    S, st = api.newton_forward(P, R, s0, forget=w.forget, max_iters=8, fixed=False, tol=w.tol, carry_mode=1,
                               loop_from=1, debug_fault=3, wait_limit_us=20000, ws=ws)
    torch.cuda.synchronize()
    rec = api.read_stats(st)
    assert rec["error"] == _lib.SLSTM_ERR_TIMEOUT, rec
    word = int(ws[4:8].cpu().view(torch.int32).item())
    assert word & 4, word
    # the library stays usable: the same call without the fault converges
    S2, st2 = _solve(P, R, s0, w, max_iters=8, loop_from=1)
    assert st2["converged"] and st2["error"] == 0
