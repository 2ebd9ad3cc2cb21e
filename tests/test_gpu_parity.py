"""GPU parity: every C-ABI entry point against the fp64 CPU oracle on the same
seeded inputs, at sizes the oracle finishes in seconds that still span
several tiles (32 steps x 32 features) and ragged tails in both time and
features.

Tolerances: max|dh| <= 1e-4 (1 + |h|) for fp32 inputs and <= 5e-3 (1 + |h|)
for bf16 inputs (the oracle reads the same bf16-rounded values, widened
exactly).  Gradients: max|dg| <= 1e-4 (1 + max|g|) per tensor for fp32
inputs; scans: 1e-5 relative to the solution's scale.
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import WORKLOADS, Workload, as_f64, make_inputs, scaled

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 5e-3
# refinement sweeps of the decoupled guess that the library's Python calls use by default
SW = api.DEFAULT_GUESS_SWEEPS


def _dev(t):
    return None if t is None else t.to("cuda").contiguous()


def _h_err(S_gpu, S_ref):
    h = S_ref[:, :, 3, :]
    return float((np.abs(S_gpu[:, :, 3, :] - h) / (1 + np.abs(h))).max())


# ---------------------------------------------------------------------------
# scan_block4
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,T,d", [(2, 100, 40), (1, 1, 1), (3, 33, 32), (1, 3000, 64)])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("with_y0", [False, True])
def test_scan_block4_matches_sequential_solve(B, T, d, reverse, with_y0, cuda_device):
    g = torch.Generator().manual_seed(1000 + B * T + d)
    A = (torch.rand(B, T, 4, 4, d, generator=g) * 0.6 - 0.3)
    b = torch.randn(B, T, 4, d, generator=g)
    y0 = torch.randn(B, 4, d, generator=g) if with_y0 else None
    y = api.scan_block4(_dev(A), _dev(b), _dev(y0), reverse=reverse)
    torch.cuda.synchronize()
    Al = np.transpose(as_f64(A), (0, 4, 1, 2, 3)).reshape(B * d, T, 4, 4)
    bl = np.transpose(as_f64(b), (0, 3, 1, 2)).reshape(B * d, T, 4)
    y0l = None if y0 is None else np.transpose(as_f64(y0), (0, 2, 1)).reshape(B * d, 4)
    ref = oracle.affine_solve(Al, bl, y0l, reverse=reverse)
    ref = np.transpose(ref.reshape(B, d, T, 4), (0, 2, 3, 1))
    err = np.abs(as_f64(y.cpu()) - ref).max() / (1 + np.abs(ref).max())
    assert err < 1e-5, err


# ---------------------------------------------------------------------------
# sequential step
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d", [(2, 64, 8), (3, 200, 130), (1, 1, 5)])
def test_sequential_step_matches_oracle(forget, B, T, d, cuda_device):
    w = Workload("t", B, T, 8, d, "f32", forget, 0.5, 7, 1e-6, 64)
    inp = make_inputs(w, with_dH=False)
    g = torch.Generator().manual_seed(5)
    s0 = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                      torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    P = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    S = api.sequential_step(_dev(torch.from_numpy(P).float()), _dev(inp["R"]), _dev(s0), forget=forget)
    ref = oracle.sequential_btgd(as_f64(torch.from_numpy(P).float()), as_f64(inp["R"]), as_f64(s0), forget)
    assert _h_err(as_f64(S.cpu()), ref) <= TOL_F32


# ---------------------------------------------------------------------------
# input projection
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,d_in,d_h", [(2, 64, 8, 8), (3, 50, 24, 40), (2, 300, 64, 96)])
def test_preact_gemm_matches_oracle(dtype, B, T, d_in, d_h, cuda_device):
    w = Workload("t", B, T, d_in, d_h, dtype, "sigmoid", 0.5, 3, 1e-6, 64)
    inp = make_inputs(w, with_dH=False)
    P = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    ref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    err = np.abs(as_f64(P.cpu()) - ref).max() / (1 + np.abs(ref).max())
    assert err < 1e-5, err


# ---------------------------------------------------------------------------
# Newton forward
# ---------------------------------------------------------------------------
# carry modes: 1 = one fused launch per iteration (decoupled look-back),
# 2 = two passes with a scan of tile aggregates in between
CARRY_MODES = [1, 2]


def _newton_case(w: Workload, fixed_k=None, carry_mode=0, init="decoupled", residual_mode="scaled",
                 exact_history=False):
    inp = make_inputs(w, with_dH=False)
    Pt = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    if fixed_k is None:
        S, st = api.newton_forward(Pt, _dev(inp["R"]), _dev(inp["s0"]), forget=w.forget,
                                   max_iters=w.max_iters, fixed=False, tol=w.tol, carry_mode=carry_mode,
                                   init=init, residual_mode=residual_mode, exact_history=exact_history)
    else:
        S, st = api.newton_forward(Pt, _dev(inp["R"]), _dev(inp["s0"]), forget=w.forget,
                                   max_iters=fixed_k, fixed=True, tol=w.tol, carry_mode=carry_mode, init=init,
                                   residual_mode=residual_mode)
    stats = api.read_stats(st)
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    return inp, as_f64(S.cpu()), stats, Pref


def _check_status_against_oracle(st, ost):
    """A GPU run either converges (and then the fp64 run converged too) or it
    stops on a non-finite or large residual; in that case the exact-arithmetic
    iterate at the same iteration was also far from converged (scaled
    residual > 1), so the stop is the method's behaviour from that guess,
    not an artefact of the kernels."""
    if st["converged"]:
        assert ost["converged"], (st, ost)
        return True
    assert st["diverged"] and st["error"] == 3, st
    k = st["iters"] - 1
    hist = list(ost["max_scaled_F"])
    assert k < len(hist) and not (hist[k] <= 1.0), (st, hist[: k + 1])
    return False


@pytest.mark.parametrize("sweeps,carry_mode,loop_from", [(2, 1, -1), (5, 1, -1), (2, 2, -1), (2, 1, 0), (5, 1, 3)])
def test_newton_launch_events_bracket_every_launch(sweeps, carry_mode, loop_from, cuda_device):
    """The optional timing events: one before each launch of work (the guess
    launches, then one per iteration, or the device loop over the rest of
    the cap as one launch) and one after the last, the events past it
    recorded there too; the solution is that of the same call without them
    (up to the rounding order of the decoupled look-back, which depends on
    timing: a tile's carry comes from its predecessor's published state or
    from composing earlier runs)."""
    w = scaled(WORKLOADS["slstm_f32_b8_t1024_d256"], B=2, T=300, d_in=64, d_h=64)
    inp = make_inputs(w, with_dH=False)
    P = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    R, s0 = _dev(inp["R"]), _dev(inp["s0"])
    K = 6
    kw = dict(forget=w.forget, max_iters=K, fixed=False, tol=w.tol, carry_mode=carry_mode, guess_sweeps=sweeps,
              loop_from=loop_from)
    S_ref, st_ref = api.newton_forward(P, R, s0, **kw)
    g = 1 + max(0, sweeps - 3)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(g + K + 1)]
    S, st = api.newton_forward(P, R, s0, events=evs, **kw)
    torch.cuda.synchronize()

    def close(a, b):
        return ((a - b).abs() / (1 + b.abs())).max().item() <= 1e-5

    assert close(S, S_ref)
    a, b = api.read_stats(st), api.read_stats(st_ref)
    assert a["iters"] == b["iters"] and a["converged"] and b["converged"]
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(evs) - 1)]
    assert all(t >= 0.0 for t in times), times
    loops = carry_mode == 1 and loop_from != -1
    n_launch = g + ((loop_from or 2) + 1 if loops else K)
    # the events past the last launch's mark the end of the call with it
    assert all(t <= 0.05 for t in times[n_launch:]), times
    # fewer events than launches: only the first ones are recorded
    few = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    S2, _ = api.newton_forward(P, R, s0, events=few, **kw)
    torch.cuda.synchronize()
    assert close(S2, S_ref) and few[0].elapsed_time(few[1]) >= 0.0


def test_newton_tiny_converges_to_sequential(cuda_device):
    w = WORKLOADS["tiny_f32"]
    inp, S, st, Pref = _newton_case(w, exact_history=True)
    ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), w.forget)
    _, ost = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), w.forget, w.max_iters, False, w.tol,
                                sweeps=SW)
    print("gpu stats", st, "oracle iters", ost["iters"])
    assert st["error"] == 0 and not st["diverged"]
    assert st["converged"]
    assert abs(st["iters"] - ost["iters"]) <= 1
    assert _h_err(S, ref) <= TOL_F32
    # the residual of the guess and of the first iterates agrees with the fp64 run
    g, o = st["init_max_scaled_F"], ost["init_max_scaled_F"]
    assert abs(g - o) <= 1e-3 * (1 + o), (g, o)
    for k in range(min(2, len(st["max_scaled_F"]), len(ost["max_scaled_F"]))):
        g, o = st["max_scaled_F"][k], ost["max_scaled_F"][k]
        assert abs(g - o) <= 1e-3 * (1 + o), (k, g, o)


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("B,T,d", [(2, 50, 40), (1, 1, 1), (2, 31, 33), (3, 64, 70)])
def test_newton_converges_to_sequential_sigmoid(B, T, d, carry_mode, cuda_device):
    w = Workload("t", B, T, 16, d, "f32", "sigmoid", 0.5, 11, 1e-6, 64)
    inp, S, st, Pref = _newton_case(w, carry_mode=carry_mode)
    ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), "sigmoid")
    assert st["error"] == 0 and st["converged"], st
    assert _h_err(S, ref) <= TOL_F32


@pytest.mark.parametrize("init", ["decoupled", "zero"])
@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d", [(2, 16, 40), (2, 32, 40), (1, 100, 33), (2, 128, 64), (8, 64, 256), (1, 300, 36), (2, 200, 40)])
def test_newton_status_agrees_with_oracle(forget, B, T, d, carry_mode, init, cuda_device):
    w = Workload("t", B, T, 16, d, "f32", forget, 0.5, 11, 1e-6, 64)
    # exact history: the iteration at which a diverging run stops is compared
    # with the fp64 run's residual there
    inp, S, st, Pref = _newton_case(w, carry_mode=carry_mode, init=init, exact_history=True)
    _, ost = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), forget, w.max_iters, False, w.tol,
                                init=init, sweeps=SW)
    converged = _check_status_against_oracle(st, ost)
    if init == "decoupled":
        assert converged, (st, ost["iters"])
    if converged:
        ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), forget)
        assert _h_err(S, ref) <= TOL_F32


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("B,T,d,sweeps", [(2, 1000, 64, 0), (4, 2000, 96, 1), (8, 1024, 256, 2), (1, 300, 33, 0)])
def test_newton_bound_history_keeps_the_decisions(B, T, d, sweeps, carry_mode, cuda_device):
    """The default history (an iteration whose test already failed somewhere
    stops evaluating the rest of its residual) takes the same decisions as the
    exact one: the same iterations, converged, the same final residual; the
    earlier entries are lower bounds above the tolerance."""
    w = Workload("t", B, T, 16, d, "f32", "sigmoid", 0.5, 21, 1e-6, 32)
    inp = make_inputs(w, with_dH=False)
    P = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    kw = dict(forget=w.forget, max_iters=w.max_iters, fixed=False, tol=w.tol, carry_mode=carry_mode,
              guess_sweeps=sweeps)
    Sb, stb = api.newton_forward(P, _dev(inp["R"]), _dev(inp["s0"]), **kw)
    Se, ste = api.newton_forward(P, _dev(inp["R"]), _dev(inp["s0"]), exact_history=True, **kw)
    b, e = api.read_stats(stb), api.read_stats(ste)
    print("bound", b["iters"], b["max_scaled_F"], "exact", e["iters"], e["max_scaled_F"])
    assert b["converged"] and e["converged"] and b["iters"] == e["iters"] and b["error"] == 0
    # the last entry is at the fp32 rounding floor of the iterate, which the
    # look-back's timing-dependent rounding order moves between runs
    assert b["max_scaled_F"][-1] <= w.tol and e["max_scaled_F"][-1] <= w.tol
    assert abs(b["max_scaled_F"][-1] - e["max_scaled_F"][-1]) <= 1e-3 * e["max_scaled_F"][-1] + 5e-7
    for x, y in zip(b["max_scaled_F"][:-1], e["max_scaled_F"][:-1]):
        assert w.tol < x <= y * (1 + 1e-3), (x, y)
    assert ((Sb - Se).abs() / (1 + Se.abs())).max().item() <= 1e-5


def _s_err(S_gpu, S_ref):
    """max over every slot of |dS| / (1 + |S|)."""
    return float((np.abs(S_gpu - S_ref) / (1 + np.abs(S_ref))).max())


@pytest.mark.parametrize("sweeps", [0, 1, 2, 3, 5])
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d,s0_random", [(2, 50, 40, True), (1, 1, 1, False), (3, 64, 70, True),
                                              (1, 3000, 36, True), (2, 4100, 64, False)])
def test_newton_decoupled_guess_matches_oracle(forget, B, T, d, s0_random, sweeps, cuda_device):
    """The guess launches alone (max_iters = 0 returns the guess): every slot
    of the decoupled trajectory, and of its refinement sweeps, against the
    oracle's, across many tiles and the look-back over up to 65 chunks of 64
    steps (the TMA path for d % 4 == 0, the cp.async path otherwise).  Up to
    three sweeps run inside the guess launch, tile by tile; a fifth sweep
    also takes the separate sweep launch that reads the guess from S."""
    w = Workload("t", B, T, 16, d, "f32", forget, 0.5, 17, 1e-6, 4)
    inp = make_inputs(w, with_dH=False)
    s0 = inp["s0"]
    if s0_random:
        g = torch.Generator().manual_seed(19)
        s0 = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                          torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    Pt = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    S, st = api.newton_forward(Pt, _dev(inp["R"]), _dev(s0), forget=forget, max_iters=0, guess_sweeps=sweeps)
    s = api.read_stats(st)
    assert s["iters"] == 0 and not s["converged"] and s["error"] == 0 and s["init_max_abs_F"] == -1.0, s
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    Sg, ost = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(s0), forget, 0, False, 1e-6, sweeps=sweeps)
    assert ost["iters"] == 0
    assert _s_err(as_f64(S.cpu()), Sg) <= TOL_F32
    # the first iteration records the guess's residual
    _, st1 = api.newton_forward(Pt, _dev(inp["R"]), _dev(s0), forget=forget, max_iters=1, tol=1e-30,
                                guess_sweeps=sweeps)
    _, ost1 = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(s0), forget, 1, False, 1e-30, sweeps=sweeps)
    g, o = api.read_stats(st1)["init_max_scaled_F"], ost1["init_max_scaled_F"]
    assert abs(g - o) <= 1e-3 * (1 + o), (g, o)


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("forget,T", [("sigmoid", 1024), ("exp", 512), ("sigmoid", 2500)])
def test_newton_converges_where_zero_guess_diverges(forget, T, carry_mode, cuda_device):
    """Lengths at which the zero guess overflows: from the decoupled guess the
    GPU solve converges, to the sequential trajectory, in about as many
    iterations as the fp64 run."""
    w = Workload("t", 2, T, 16, 40, "f32", forget, 0.5, 23, 1e-5, 16)
    inp, S, st, Pref = _newton_case(w, carry_mode=carry_mode)
    _, ost = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), forget, w.max_iters, False, w.tol,
                                sweeps=SW)
    print("gpu", st["iters"], st["max_scaled_F"], "oracle", ost["iters"], list(ost["max_scaled_F"]))
    assert st["converged"] and st["error"] == 0, st
    assert ost["converged"] and abs(st["iters"] - ost["iters"]) <= 1
    ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), forget)
    assert _h_err(S, ref) <= TOL_F32


def test_newton_raw_residual_mode(cuda_device):
    """residual_mode 'raw': the stop uses max|F| (the pages' norm); the run
    stops where the fp64 run with the same rule stops, give or take one.  The
    tolerance is one fp32 can reach on max|F| (the normaliser n reaches tens,
    so |F| has a rounding floor of a few 1e-6)."""
    w = scaled(WORKLOADS["tiny_f32"], tol=1e-4)
    inp, S, st, Pref = _newton_case(w, residual_mode="raw")
    _, ost = oracle.newton_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), w.forget, w.max_iters, False, w.tol,
                                residual_mode="raw", sweeps=SW)
    print("gpu", st, "oracle", ost)
    assert st["converged"] and ost["converged"]
    assert st["max_abs_F"][-1] <= w.tol
    assert abs(st["iters"] - ost["iters"]) <= 1
    ref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(inp["s0"]), w.forget)
    assert _h_err(S, ref) <= TOL_F32


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_newton_given_guess_one_iteration(forget, carry_mode, cuda_device):
    """Warm start: S holds a guess near the solution (the sequential
    trajectory, perturbed); one iteration from it matches the fp64 iteration
    from the same guess at every step and slot."""
    w = Workload("t", 3, 700, 16, 40, "f32", forget, 0.5, 29, 1e-6, 1)
    inp = make_inputs(w, with_dH=False)
    # both sides read the same fp32 P and guess, made on the host by the oracle
    P32 = torch.from_numpy(oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))).float()
    Sseq = oracle.sequential_btgd(as_f64(P32), as_f64(inp["R"]), as_f64(inp["s0"]), forget)
    # relative noise of 1e-3 on c, n, h and absolute 1e-3 on the stabiliser m
    u = np.random.default_rng(31).uniform(-1, 1, size=Sseq.shape)
    g64 = Sseq * (1 + 1e-3 * u)
    g64[:, :, 2] = Sseq[:, :, 2] + 1e-3 * u[:, :, 2]
    guess32 = torch.from_numpy(g64).float()
    S = _dev(guess32)
    S, st = api.newton_forward(_dev(P32), _dev(inp["R"]), None, forget=forget, max_iters=1, fixed=True, tol=1e-6,
                               S=S, init="given", carry_mode=carry_mode)
    s = api.read_stats(st)
    assert s["iters"] == 1 and s["init_max_abs_F"] == -1.0
    So, ost = oracle.newton_btgd(as_f64(P32), as_f64(inp["R"]), as_f64(inp["s0"]), forget, 1, True, 1e-6,
                                 init="given", S_init=as_f64(guess32))
    assert _s_err(as_f64(S.cpu()), So) <= TOL_F32
    g_r, o_r = s["max_abs_F"][0], ost["max_abs_F"][0]
    assert abs(g_r - o_r) <= 1e-3 * (1 + o_r) + 1e-5, (g_r, o_r)


@pytest.mark.parametrize("carry_mode", CARRY_MODES)
@pytest.mark.parametrize("K", [1, 3])
def test_newton_fixed_k_prefix_exact(K, carry_mode, cuda_device):
    """After K Newton iterations the first K steps equal the sequential
    trajectory whatever the rest of the iterate looks like."""
    w = WORKLOADS["slstm_f32_b8_t1024_d256"]
    inp, S, st, Pref = _newton_case(w, fixed_k=K, carry_mode=carry_mode)
    assert st["iters"] == K
    ref = oracle.sequential_btgd(Pref[:, :K], as_f64(inp["R"]), as_f64(inp["s0"]), w.forget)
    assert _h_err(S[:, :K], ref) <= TOL_F32


def test_newton_stats_divergence_on_nan(cuda_device):
    P = torch.full((1, 40, 4, 8), float("nan"), device="cuda")
    S, st = api.newton_forward(P, torch.zeros(4, 8, device="cuda"), max_iters=3, fixed=False, tol=1e-5)
    s = api.read_stats(st)
    assert s["diverged"] and not s["converged"] and s["error"] == 3
    assert s["iters"] == 1      # a non-finite residual stops the run at once


def test_newton_cap_beyond_history(cuda_device):
    """More iterations than the 64-entry residual history: the run still
    converges and the record keeps the last 64 residuals."""
    w = Workload("t", 2, 64, 16, 32, "f32", "sigmoid", 0.5, 11, 1e-30, 100)
    inp = make_inputs(w, with_dH=False)
    Pt = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    S, st = api.newton_forward(Pt, _dev(inp["R"]), None, max_iters=100, fixed=True, tol=1e-6)
    s = api.read_stats(st)
    assert s["iters"] == 100 and s["converged"]
    assert len(s["max_scaled_F"]) == 64 and s["history_first_iter"] == 36
    assert s["max_scaled_F"][-1] <= 1e-6 and s["max_scaled_F"][0] == -1.0


def test_newton_bounded_wait_reports_timeout(cuda_device):
    """Fault injection on the host's request: one tile withholds its carry;
    its successor's bounded wait expires and the run reports a timeout
    instead of hanging."""
    w = Workload("t", 1, 256, 8, 32, "f32", "sigmoid", 0.5, 1, 1e-6, 4)
    inp = make_inputs(w, with_dH=False)
    Pt = api.preact_gemm(_dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["bias"]))
    S, st = api.newton_forward(Pt, _dev(inp["R"]), None, max_iters=2, fixed=True, tol=1e-6,
                               debug_fault=1, wait_limit_us=20000)
    s = api.read_stats(st)
    assert s["error"] == 4, s
    # the context is still usable afterwards
    S2, st2 = api.newton_forward(Pt, _dev(inp["R"]), None, max_iters=64, fixed=False, tol=1e-6)
    assert api.read_stats(st2)["converged"]


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
@pytest.mark.parametrize("B,T,d_in,d,dtype", [(2, 64, 8, 8, "f32"), (2, 75, 12, 40, "f32"), (2, 33, 8, 10, "f32"),
                                              (1, 16400, 16, 36, "bf16"),
                                              (2, 75, 16, 40, "bf16"), (3, 130, 64, 96, "bf16"),
                                              (2, 96, 16, 40, "bf16"), (2, 100, 24, 36, "bf16"),
                                              (2, 70, 16, 18, "bf16")])
def test_backward_matches_oracle_bptt(forget, B, T, d_in, d, dtype, cuda_device):
    """fp32 inputs take the CUDA-core GEMMs; bf16 inputs the tensor-core GEMMs
    with dP carried as a bf16 pair (transposed copy for the W_x gradient).
    d % 4 != 0 takes the cp.async tile path of the adjoint kernel, d % 4 == 0
    the TMA one; T % 4 == 0 writes the transposed pair in 8-byte pieces
    (with T % 32 != 0 the last tile starts before t = 0), other T per element."""
    w = Workload("t", B, T, d_in, d, dtype, forget, 0.5, 13, 1e-6, 64)
    inp = make_inputs(w, with_dH=True)
    g = torch.Generator().manual_seed(9)
    s0 = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                      torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1)
    x, Wx, R = _dev(inp["x"]), _dev(inp["Wx"]), _dev(inp["R"])
    Pt = api.preact_gemm(x, Wx, _dev(inp["bias"]))
    S = api.sequential_step(Pt, R, _dev(s0), forget=forget)
    out = api.newton_backward(x, Wx, Pt, R, _dev(s0), S, _dev(inp["dH"]), forget=forget)
    torch.cuda.synchronize()
    Pref = oracle.preact(as_f64(inp["x"]), as_f64(inp["Wx"]), as_f64(inp["bias"]))
    Sref = oracle.sequential_btgd(Pref, as_f64(inp["R"]), as_f64(s0), forget)
    ref = oracle.backward_btgd(as_f64(inp["x"]), as_f64(inp["Wx"]), Pref, as_f64(inp["R"]), as_f64(s0), Sref,
                               as_f64(inp["dH"]), forget)
    for k in ("dx", "dWx", "dR", "db", "ds0"):
        got = as_f64(out[k].cpu())
        err = np.abs(got - ref[k]).max() / (1 + np.abs(ref[k]).max())
        assert err <= 1e-4, (k, err)


@pytest.mark.parametrize("reverse", [False, True])
def test_scan_block4_bounded_wait_poisons_outputs(reverse, cuda_device):
    """Fault injection on the host's request: a tile withholds its carry; the
    successor's bounded wait expires and, instead of using a made-up carry,
    it makes every output that depends on the missing one NaN.  Nothing is
    silently wrong: every finite output equals the oracle's (tiles that a
    stalled CTA held back may have given up too, and are NaN as well), the
    steps before the withheld carry are finite, and the context stays
    usable."""
    B, T, d = 2, 200, 64
    g = torch.Generator().manual_seed(77)
    A = (torch.rand(B, T, 4, 4, d, generator=g) * 0.6 - 0.3)
    b = torch.randn(B, T, 4, d, generator=g)
    flags = api._lib.SLSTM_SCAN_DEBUG_WITHHOLD | (api._lib.SLSTM_SCAN_REVERSE_T if reverse else 0)
    Ad, bd = _dev(A), _dev(b)
    y = torch.empty_like(bd)
    ws = api.workspace(api._lib.SLSTM_OP_SCAN_BLOCK4, B, T, 0, d, bd.device)
    rc = api.load().scan_block4(api._ptr(Ad), api._ptr(bd), None, api._ptr(y), B, T, d, flags, api._ptr(ws),
                                ws.numel(), api._stream())
    assert rc == 0
    torch.cuda.synchronize()
    # the expired wait is reported in the workspace's error word (bytes 4..7)
    assert ws[4:8].view(torch.int32).item() != 0
    got = y.cpu()
    Al = np.transpose(as_f64(A), (0, 4, 1, 2, 3)).reshape(B * d, T, 4, 4)
    bl = np.transpose(as_f64(b), (0, 3, 1, 2)).reshape(B * d, T, 4)
    ref = np.transpose(oracle.affine_solve(Al, bl, None, reverse=reverse).reshape(B, d, T, 4), (0, 2, 3, 1))
    late = slice(0, T - 64) if reverse else slice(64, T)
    early = slice(T - 64, T) if reverse else slice(0, 64)
    assert torch.isnan(got[0, late, :, :32]).all()
    fin = np.isfinite(as_f64(got))
    err = np.abs(as_f64(got)[fin] - ref[fin]).max() / (1 + np.abs(ref).max())
    assert err < 1e-5, err
    assert np.isfinite(as_f64(got[0, early])).all()
    # a normal call afterwards is unaffected
    y2 = api.scan_block4(Ad, bd, None, reverse=reverse, ws=ws)
    torch.cuda.synchronize()
    assert np.abs(as_f64(y2.cpu()) - ref).max() / (1 + np.abs(ref).max()) < 1e-5
    assert ws[4:8].view(torch.int32).item() == 0
