"""Pins for the fp64 CPU oracle (CPU only).

Each test ties the oracle to something other than itself: a worked example
derived by hand from the cell equations, closed forms, invariants the pages
state (stabilised == unstabilised), brute force, finite differences, or a
library routine.  Sources: "xLSTM - a from-scratch, educational
reimplementation" (section "Exponential gating + the stabilizer"), "xLSTM:
Extended Long Short-Term Memory" (summary, section "Method": sLSTM step,
stabilizer, item 1 "stabilised and unstabilised forms give identical
outputs"), "sLSTM in this library" (pararnn-torch docs, sections "Cell",
"Backward"), "pararnn-torch structure" (section "Current surface").
"""
import json
import math
import os
import re

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "slstm_two_steps.json")


def _ev(s: str) -> float:
    expr = re.sub(r"ln(\d+)", r"math.log(\1)", s)
    return float(eval(expr, {"__builtins__": {}, "math": math}))


def _rand_lane_inputs(rng, L, T, forget="sigmoid", r_scale=0.5, s0_random=True):
    P = rng.normal(size=(L, T, 4))
    P[:, :, 2] += rng.uniform(3, 6, size=(L, 1))       # forget bias as in the workloads
    R = rng.uniform(-r_scale, r_scale, size=(L, 4))
    if s0_random:
        s0 = np.stack([rng.normal(size=L), rng.uniform(0.5, 2.0, size=L),
                       rng.normal(size=L), rng.uniform(-0.9, 0.9, size=L)], axis=1)
    else:
        s0 = np.zeros((L, 4))
    return P, R, s0


# ---------------------------------------------------------------------------
# worked example by hand
# ---------------------------------------------------------------------------
def test_golden_two_steps():
    g = json.load(open(GOLDEN))
    R = np.array(g["R"])[None]
    s0 = np.array(g["s0"])[None]
    P = np.array([[_ev(v) for v in row] for row in g["P"]])[None]
    for forget in ("sigmoid", "exp"):
        S = oracle.sequential(P, R, s0, forget)[0]
        exp = np.array([[_ev(v) for v in row] for row in g["expected"][forget]])
        np.testing.assert_allclose(S, exp, rtol=0, atol=1e-14)
    _, J, _ = oracle.step(np.array([_ev(v) for v in g["expected"]["sigmoid"][0]]), P[0, 1], R[0],
                          "sigmoid")
    expJ = np.array([[_ev(v) for v in row] for row in g["expected"]["sigmoid_J_step2"]])
    np.testing.assert_allclose(J, expJ, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# closed forms and invariants of the forward step
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_stabilised_equals_unstabilised(forget):
    rng = np.random.default_rng(11)
    T = 48 if forget == "exp" else 200
    P, R, s0 = _rand_lane_inputs(rng, 6, T, forget)
    S = oracle.sequential(P, R, s0, forget)
    cu, nu, h = oracle.sequential_unstabilised(P, R, s0, forget)
    np.testing.assert_allclose(S[:, :, 3], h, rtol=0, atol=1e-12 * (1 + np.abs(h)).max())
    # the stabilised state is the unstabilised one rescaled by exp(-m)
    np.testing.assert_allclose(S[:, :, 0], cu * np.exp(-S[:, :, 2]), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[:, :, 1], nu * np.exp(-S[:, :, 2]), rtol=1e-11, atol=1e-12)


def test_first_step_from_zero_state():
    rng = np.random.default_rng(3)
    for forget in ("sigmoid", "exp"):
        for _ in range(50):
            p = rng.normal(scale=3.0, size=4)
            r = rng.normal(size=4)
            m0 = rng.normal(scale=5.0)
            h0 = rng.normal()
            s, _, _ = oracle.step(np.array([0.0, 0.0, m0, h0]), p, r, forget)
            az, ao = p[0] + r[0] * h0, p[3] + r[3] * h0
            assert abs(s[3] - math.tanh(az) / (1 + math.exp(-ao))) < 1e-14


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_zero_recurrence_closed_form(forget):
    """R = 0, zero start: h_t = o_t * sum_s w_ts z_s / sum_s w_ts with
    log w_ts = a_i(s) + sum_{s<u<=t} log f_u (evaluated in log space)."""
    rng = np.random.default_rng(5)
    T = 40
    P, _, _ = _rand_lane_inputs(rng, 3, T, forget)
    R = np.zeros((3, 4))
    s0 = np.zeros((3, 4))
    S = oracle.sequential(P, R, s0, forget)
    for l in range(3):
        z = np.tanh(P[l, :, 0])
        o = 1 / (1 + np.exp(-P[l, :, 3]))
        lf = P[l, :, 2] if forget == "exp" else -np.logaddexp(0, -P[l, :, 2])
        cum = np.concatenate([[0.0], np.cumsum(lf)])
        for t in range(T):
            lw = P[l, : t + 1, 1] + (cum[t + 1] - cum[1 : t + 2])
            w = np.exp(lw - lw.max())
            h = o[t] * (w @ z[: t + 1]) / w.sum()
            assert abs(S[l, t, 3] - h) < 1e-12


def test_stabilised_gates_bounded_and_finite_under_huge_inputs():
    rng = np.random.default_rng(7)
    for forget in ("sigmoid", "exp"):
        P = rng.normal(scale=300.0, size=(4, 64, 4))
        R = rng.normal(scale=50.0, size=(4, 4))
        S = oracle.sequential(P, R, np.zeros((4, 4)), forget)
        assert np.isfinite(S).all()
        # i', f' in (0, 1] means n_t <= n_{t-1} + 1 and n_t > 0
        n = S[:, :, 1]
        assert (n > 0).all()
        assert (n[:, 1:] <= n[:, :-1] + 1 + 1e-12).all()
        assert (np.abs(S[:, :, 3]) <= 1 + 1e-12).all()


# ---------------------------------------------------------------------------
# Jacobians
# ---------------------------------------------------------------------------
def _fd_jacobian(sp, p, r, forget, eps=1e-6):
    J = np.zeros((4, 4))
    for k in range(4):
        e = np.zeros(4)
        e[k] = eps
        fp_, _, _ = oracle.step(sp + e, p, r, forget)
        fm_, _, _ = oracle.step(sp - e, p, r, forget)
        J[:, k] = (fp_ - fm_) / (2 * eps)
    return J


def _fd_gate_jacobian(sp, p, r, forget, eps=1e-6):
    G = np.zeros((4, 4))
    for k in range(4):
        e = np.zeros(4)
        e[k] = eps
        fp_, _, _ = oracle.step(sp, p + e, r, forget)
        fm_, _, _ = oracle.step(sp, p - e, r, forget)
        G[:, k] = (fp_ - fm_) / (2 * eps)
    return G


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_jacobians_match_finite_differences(forget):
    rng = np.random.default_rng(17)
    checked = 0
    while checked < 60:
        sp = np.array([rng.normal(), rng.uniform(0.3, 3.0), rng.normal(scale=2), rng.uniform(-1, 1)])
        p = rng.normal(scale=1.5, size=4)
        r = rng.uniform(-1, 1, size=4)
        s, J, G = oracle.step(sp, p, r, forget)
        # stay away from the tie of the max (non-differentiable there)
        h0 = sp[3]
        lf = (p[2] + r[2] * h0) if forget == "exp" else -np.logaddexp(0, -(p[2] + r[2] * h0))
        if abs(lf + sp[2] - (p[1] + r[1] * h0)) < 1e-3:
            continue
        Jfd = _fd_jacobian(sp, p, r, forget)
        Gfd = _fd_gate_jacobian(sp, p, r, forget)
        np.testing.assert_allclose(J, Jfd, rtol=1e-6, atol=1e-8)
        np.testing.assert_allclose(G, Gfd, rtol=1e-6, atol=1e-8)
        # h_{t-1} enters only through a_t = P_t + r h_{t-1}: J[:, h] = G r
        np.testing.assert_allclose(J[:, 3], G @ r, rtol=1e-12, atol=1e-14)
        checked += 1


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_gauge_identity(forget):
    """Rescaling the unstabilised state leaves h unchanged: with
    g = (-c, -n, 1, 0), J_t g_{t-1} = beta_t g_t exactly."""
    rng = np.random.default_rng(23)
    for _ in range(100):
        sp = np.array([rng.normal(), rng.uniform(0.3, 3.0), rng.normal(scale=2), rng.uniform(-1, 1)])
        p = rng.normal(scale=1.5, size=4)
        r = rng.uniform(-1, 1, size=4)
        s, J, _ = oracle.step(sp, p, r, forget)
        beta = J[2, 2]
        assert beta in (0.0, 1.0)
        g_prev = np.array([-sp[0], -sp[1], 1.0, 0.0])
        g_now = np.array([-s[0], -s[1], 1.0, 0.0])
        np.testing.assert_allclose(J @ g_prev, beta * g_now, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# affine scan
# ---------------------------------------------------------------------------
def _tree_compose(maps):
    """Compose affine maps (A, b), earliest first, by recursive halving."""
    if len(maps) == 1:
        return maps[0]
    mid = len(maps) // 2
    A1, b1 = _tree_compose(maps[:mid])
    A2, b2 = _tree_compose(maps[mid:])
    return A2 @ A1, A2 @ b1 + b2


def test_affine_solve_matches_brute_force_and_tree():
    rng = np.random.default_rng(29)
    L, T = 3, 37
    A = rng.normal(scale=0.5, size=(L, T, 4, 4))
    b = rng.normal(size=(L, T, 4))
    y0 = rng.normal(size=(L, 4))
    y = oracle.affine_solve(A, b, y0)
    yr = oracle.affine_solve(A, b, y0, reverse=True)
    for l in range(L):
        # forward: left fold of y -> A y + b
        v = y0[l].copy()
        for t in range(T):
            v = A[l, t] @ v + b[l, t]
            np.testing.assert_allclose(y[l, t], v, rtol=1e-12, atol=1e-12)
            At, bt = _tree_compose([(A[l, s], b[l, s]) for s in range(t + 1)])
            np.testing.assert_allclose(y[l, t], At @ y0[l] + bt, rtol=1e-11, atol=1e-11)
        # reverse-transposed: y_t = A_t^T y_{t+1} + b_t, y_T = y0
        v = y0[l].copy()
        for t in range(T - 1, -1, -1):
            v = A[l, t].T @ v + b[l, t]
            np.testing.assert_allclose(yr[l, t], v, rtol=1e-12, atol=1e-12)
    # missing y0 means zero
    np.testing.assert_allclose(oracle.affine_solve(A, b), oracle.affine_solve(A, b, np.zeros((L, 4))))


# ---------------------------------------------------------------------------
# Newton
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_newton_prefix_exact_after_k_iterations(forget):
    """After k Newton iterations the first k steps equal the sequential
    trajectory (by induction: step t only depends on exact earlier steps),
    and K = T iterations reproduce the whole trajectory."""
    rng = np.random.default_rng(31)
    T = 12
    P, R, s0 = _rand_lane_inputs(rng, 4, T, forget)
    Sseq = oracle.sequential(P, R, s0, forget)
    for k in (1, 2, 5):
        S, st = oracle.newton(P, R, s0, forget, max_iters=k, fixed=True)
        assert st["iters"] == k
        np.testing.assert_allclose(S[:, :k], Sseq[:, :k], rtol=0,
                                   atol=1e-12 * (1 + np.abs(Sseq).max()))
    S, st = oracle.newton(P, R, s0, forget, max_iters=T, fixed=True)
    np.testing.assert_allclose(S, Sseq, rtol=0, atol=1e-12 * (1 + np.abs(Sseq).max()))


def test_newton_converges_by_tolerance():
    rng = np.random.default_rng(37)
    P, R, s0 = _rand_lane_inputs(rng, 8, 64, "sigmoid", s0_random=False)
    Sseq = oracle.sequential(P, R, s0, "sigmoid")
    S, st = oracle.newton(P, R, s0, "sigmoid", max_iters=64, fixed=False, tol=1e-10)
    assert st["converged"] and not st["diverged"]
    assert st["iters"] < 64
    assert st["max_scaled_F"][-1] <= 1e-10
    # iteration k's recorded residual is the residual of the k-th iterate
    np.testing.assert_allclose(S, Sseq, rtol=0, atol=1e-9)


def test_newton_divergence_flag():
    P = np.full((1, 8, 4), np.nan)
    S, st = oracle.newton(P, np.zeros((1, 4)), np.zeros((1, 4)), "sigmoid", max_iters=3)
    assert st["diverged"] and not st["converged"]


def _closed_form_h_zero_recurrence(P, forget):
    """h of the R = 0 cell from the zero state, by the log-space weighted
    average h_t = o_t sum_s w_ts z_s / sum_s w_ts (the closed form pinned in
    test_zero_recurrence_closed_form), for every lane and step."""
    L, T, _ = P.shape
    H = np.zeros((L, T))
    for l in range(L):
        z = np.tanh(P[l, :, 0])
        o = 1 / (1 + np.exp(-P[l, :, 3]))
        lf = P[l, :, 2] if forget == "exp" else -np.logaddexp(0, -P[l, :, 2])
        cum = np.concatenate([[0.0], np.cumsum(lf)])
        for t in range(T):
            lw = P[l, : t + 1, 1] + (cum[t + 1] - cum[1 : t + 2])
            w = np.exp(lw - lw.max())
            H[l, t] = o[t] * (w @ z[: t + 1]) / w.sum()
    return H


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_decoupled_guess_is_the_zero_recurrence_solution(forget):
    """The default initial guess is the trajectory with R = 0.  With R = 0 it
    is therefore the solution itself: its residual is zero, one iteration
    leaves it where it is, and h is the closed form.  max_iters = 0 returns
    the guess."""
    rng = np.random.default_rng(71)
    P, _, _ = _rand_lane_inputs(rng, 3, 30, forget)
    R = np.zeros((3, 4))
    s0 = np.zeros((3, 4))
    S, st = oracle.newton(P, R, s0, forget, max_iters=5, tol=1e-12)
    assert st["iters"] == 1 and st["converged"] and not st["diverged"]
    assert st["init_max_abs_F"] == 0.0 and st["max_abs_F"][0] == 0.0
    H = _closed_form_h_zero_recurrence(P, forget)
    np.testing.assert_allclose(S[:, :, 3], H, rtol=0, atol=1e-12)
    # with R != 0 the guess keeps the R = 0 gates: its h is still the closed
    # form of the R = 0 cell, and its residual is nonzero
    R2 = rng.uniform(-0.5, 0.5, size=(3, 4))
    Sg, stg = oracle.newton(P, R2, s0, forget, max_iters=0)
    assert stg["iters"] == 0 and not stg["converged"] and not stg["diverged"]
    np.testing.assert_allclose(Sg[:, :, 3], H, rtol=0, atol=1e-12)
    _, st2 = oracle.newton(P, R2, s0, forget, max_iters=1, tol=1e-30)
    assert st2["init_max_abs_F"] > 1e-3
    # a fixed-K solve does not record the guess's residual
    _, st3 = oracle.newton(P, R2, s0, forget, max_iters=1, fixed=True)
    assert st3["iters"] == 1 and st3["init_max_abs_F"] == -1.0


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_guess_sweeps(forget):
    """Refinement sweeps of the guess: a sweep's gates see the previous
    guess's h, so (1) with R = 0 a sweep leaves the decoupled guess unchanged,
    (2) the solution is a fixed point of the sweep, (3) after k sweeps the
    first k steps are the sequential trajectory (prefix exactness of the
    fixed-point iteration), and (4) on the workloads' lanes each sweep shrinks
    the residual and the sweeps converge to the solution."""
    rng = np.random.default_rng(97)
    T = 40
    P, R, s0 = _rand_lane_inputs(rng, 3, T, forget)
    Sseq = oracle.sequential(P, R, s0, forget)
    Z = np.zeros((3, 4))
    g0, _ = oracle.newton(P, Z, s0, forget, max_iters=0)
    g2, _ = oracle.newton(P, Z, s0, forget, max_iters=0, sweeps=2)
    np.testing.assert_array_equal(g0, g2)
    for k in (1, 2, 5):
        gk, _ = oracle.newton(P, R, s0, forget, max_iters=0, sweeps=k)
        np.testing.assert_allclose(gk[:, :k], Sseq[:, :k], rtol=0, atol=1e-12 * (1 + np.abs(Sseq).max()))
        if k < T:
            assert np.abs(gk[:, k:] - Sseq[:, k:]).max() > 1e-12
    # the solution is the sweeps' fixed point: T sweeps and more reach it
    g_many, _ = oracle.newton(P, R, s0, forget, max_iters=0, sweeps=T + 5)
    np.testing.assert_allclose(g_many, Sseq, rtol=0, atol=1e-10 * (1 + np.abs(Sseq).max()))
    P2, R2, s02 = _workload_lanes(rng, 4, 512, forget, 0.5)
    res = []
    for k in range(4):
        _, st = oracle.newton(P2, R2, s02, forget, max_iters=1, tol=1e-30, sweeps=k)
        res.append(st["init_max_scaled_F"])
    assert all(b < a for a, b in zip(res, res[1:])), res


def _workload_lanes(rng, L, T, forget, r_scale):
    """Lanes drawn like the workloads: P ~ N(0, 1) per gate (x ~ N(0,1) through
    W_x ~ N(0, 1/d_in)), forget bias spread over [3, 6], R ~ U(-a, a)."""
    P = rng.normal(size=(L, T, 4))
    P[:, :, 2] += np.linspace(3.0, 6.0, L)[:, None]
    R = rng.uniform(-r_scale, r_scale, size=(L, 4))
    return P, R, np.zeros((L, 4))


@pytest.mark.parametrize("forget,T", [("sigmoid", 1024), ("exp", 512)])
def test_decoupled_guess_converges_where_the_zero_guess_diverges(forget, T):
    """From the zero guess the iterates blow up on these lengths; from the
    decoupled guess the solve converges in a few iterations, and a converged
    iterate is the unique sequential trajectory."""
    rng = np.random.default_rng(73)
    P, R, s0 = _workload_lanes(rng, 6, T, forget, 0.5)
    Sseq = oracle.sequential(P, R, s0, forget)
    _, stz = oracle.newton(P, R, s0, forget, max_iters=8, tol=1e-8, init="zero")
    assert not stz["converged"]
    S, st = oracle.newton(P, R, s0, forget, max_iters=8, tol=1e-8)
    assert st["converged"] and st["iters"] <= 6, st
    np.testing.assert_allclose(S, Sseq, rtol=0, atol=1e-7 * (1 + np.abs(Sseq)).max())


@pytest.mark.parametrize("init", ["decoupled", "zero", "given"])
def test_newton_prefix_exact_from_every_guess(init):
    """Prefix exactness holds whatever the guess: after k iterations the first
    k steps are the sequential trajectory."""
    rng = np.random.default_rng(79)
    T = 10
    P, R, s0 = _rand_lane_inputs(rng, 3, T, "sigmoid")
    Sseq = oracle.sequential(P, R, s0, "sigmoid")
    guess = np.abs(rng.normal(size=(3, T, 4))) + 0.5
    for k in (1, 3):
        S, st = oracle.newton(P, R, s0, "sigmoid", max_iters=k, fixed=True, init=init,
                              S_init=guess if init == "given" else None)
        assert st["iters"] == k
        np.testing.assert_allclose(S[:, :k], Sseq[:, :k], rtol=0, atol=1e-12 * (1 + np.abs(Sseq).max()))
        if init != "decoupled":   # from these guesses the rest is not exact yet
            assert np.abs(S[:, k:] - Sseq[:, k:]).max() > 1e-9


def test_newton_given_guess():
    rng = np.random.default_rng(83)
    P, R, s0 = _rand_lane_inputs(rng, 3, 16, "exp")
    Sseq = oracle.sequential(P, R, s0, "exp")
    # a guess at the solution stays there: F = 0, so delta = 0
    S, st = oracle.newton(P, R, s0, "exp", max_iters=1, fixed=True, init="given", S_init=Sseq)
    np.testing.assert_allclose(S, Sseq, rtol=0, atol=1e-12 * (1 + np.abs(Sseq).max()))
    assert st["max_abs_F"][0] <= 1e-12 * (1 + np.abs(Sseq).max())
    # a zero guess given explicitly is the zero init
    Sz, stz = oracle.newton(P, R, s0, "exp", max_iters=3, fixed=True, init="zero")
    Sg, stg = oracle.newton(P, R, s0, "exp", max_iters=3, fixed=True, init="given", S_init=np.zeros_like(P))
    np.testing.assert_array_equal(Sz, Sg)
    np.testing.assert_array_equal(stz["max_abs_F"], stg["max_abs_F"])


def test_newton_residual_modes():
    """residual_mode 'raw' stops at the first iteration with max|F| <= tol,
    'scaled' at the first with max |F|/(1+|s|) <= tol; both histories are
    the same iterates, so each stop is the first crossing of its column."""
    rng = np.random.default_rng(89)
    P, R, s0 = _workload_lanes(rng, 4, 256, "sigmoid", 0.5)
    _, full = oracle.newton(P, R, s0, "sigmoid", max_iters=8, fixed=True, tol=0.0)
    for mode, col in (("raw", "max_abs_F"), ("scaled", "max_scaled_F")):
        tol = 1e-6
        _, st = oracle.newton(P, R, s0, "sigmoid", max_iters=8, tol=tol, residual_mode=mode)
        first = int(np.argmax(full[col] <= tol)) + 1
        assert full[col][first - 1] <= tol
        assert st["converged"] and st["iters"] == first
        np.testing.assert_array_equal(st[col], full[col][:first])
    # the scaled residual never exceeds the raw one
    assert np.all(full["max_scaled_F"] <= full["max_abs_F"])


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
def _loss(x, Wx, bias, R, s0, dH, forget):
    P = oracle.preact(x, Wx, bias)
    S = oracle.sequential_btgd(P, R, s0, forget)
    return float((S[:, :, 3, :] * dH).sum())


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_bptt_matches_finite_differences(forget):
    rng = np.random.default_rng(41)
    B, T, d_in, d = 2, 10, 3, 2
    x = rng.normal(size=(B, T, d_in))
    Wx = rng.normal(size=(4 * d, d_in)) / math.sqrt(d_in)
    R = rng.uniform(-0.5, 0.5, size=(4, d))
    bias = np.zeros((4, d))
    bias[2] = np.linspace(3, 6, d)
    s0 = np.stack([rng.normal(size=(B, d)), rng.uniform(0.5, 2, size=(B, d)),
                   rng.normal(size=(B, d)), rng.uniform(-0.5, 0.5, size=(B, d))], axis=1)
    dH = rng.normal(size=(B, T, d))
    P = oracle.preact(x, Wx, bias)
    S = oracle.sequential_btgd(P, R, s0, forget)
    g = oracle.backward_btgd(x, Wx, P, R, s0, S, dH, forget)

    def check(name, arr, grad):
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = arr[idx]
            eps = 1e-6 * max(1.0, abs(old))
            arr[idx] = old + eps
            lp = _loss(x, Wx, bias, R, s0, dH, forget)
            arr[idx] = old - eps
            lm = _loss(x, Wx, bias, R, s0, dH, forget)
            arr[idx] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, grad[idx])

    check("x", x, g["dx"])
    check("Wx", Wx, g["dWx"])
    check("R", R, g["dR"])
    check("bias", bias, g["db"])
    check("s0", s0, g["ds0"])


def test_gemm_matches_numpy():
    rng = np.random.default_rng(43)
    A = rng.normal(size=(7, 5))
    Bm = rng.normal(size=(5, 3))
    bias = rng.normal(size=3)
    np.testing.assert_allclose(oracle.gemm(A, Bm, bias=bias), A @ Bm + bias, rtol=1e-13)
    np.testing.assert_allclose(oracle.gemm(A.T.copy(), Bm, ta=True), A @ Bm, rtol=1e-13)
    np.testing.assert_allclose(oracle.gemm(A, Bm.T.copy(), tb=True), A @ Bm, rtol=1e-13)


# ---------------------------------------------------------------------------
# packed ragged sequences: the packed problem is the independent problems of
# its sequences ("sLSTM in this library", section "Packed sequences").  These
# pin the cutting and gathering at the offsets against the batched functions.
# ---------------------------------------------------------------------------
def _packed_case(rng, B, T, d, d_in):
    x = rng.normal(size=(B, T, d_in))
    Wx = rng.normal(size=(4 * d, d_in)) / math.sqrt(d_in)
    bias = np.zeros((4, d))
    bias[2] = np.linspace(3, 6, d)
    R = rng.uniform(-0.5, 0.5, size=(4, d))
    s0 = np.stack([rng.normal(size=(B, d)), rng.uniform(0.5, 1.5, size=(B, d)), rng.normal(size=(B, d)),
                   rng.uniform(-0.5, 0.5, size=(B, d))], axis=1)
    dH = rng.normal(size=(B, T, d))
    return x, Wx, bias, R, s0, dH


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_varlen_equal_lengths_equals_batched(forget):
    rng = np.random.default_rng(51)
    B, T, d, d_in = 3, 7, 4, 5
    x, Wx, bias, R, s0, dH = _packed_case(rng, B, T, d, d_in)
    P = oracle.preact(x, Wx, bias)
    cu = np.arange(B + 1) * T
    pk = lambda a: a.reshape((B * T,) + a.shape[2:])
    S_b = oracle.sequential_btgd(P, R, s0, forget)
    np.testing.assert_array_equal(oracle.sequential_varlen(pk(P), R, s0, cu, forget), pk(S_b))
    N_b, _ = oracle.newton_btgd(P, R, s0, forget, max_iters=3, fixed=True, tol=0.0)
    np.testing.assert_array_equal(oracle.newton_varlen_fixed(pk(P), R, s0, cu, forget, 3), pk(N_b))
    g_b = oracle.backward_btgd(x, Wx, P, R, s0, S_b, dH, forget)
    g_v = oracle.backward_varlen(pk(x), Wx, pk(P), R, s0, pk(S_b), pk(dH), cu, forget)
    np.testing.assert_allclose(g_v["dx"], pk(g_b["dx"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g_v["ds0"], g_b["ds0"], rtol=0, atol=1e-12)
    for k in ("dWx", "dR", "db"):
        np.testing.assert_allclose(g_v[k], g_b[k], rtol=1e-12, atol=1e-12)


def test_varlen_empty_sequences_and_independence():
    rng = np.random.default_rng(52)
    d, d_in = 3, 4
    x, Wx, bias, R, s0, dH = _packed_case(rng, 5, 6, d, d_in)
    P = oracle.preact(x, Wx, bias)
    total = 13
    xp, Pp, dHp = x.reshape(-1, d_in)[:total], P.reshape(-1, 4, d)[:total], dH.reshape(-1, d)[:total]
    cu = np.array([0, 5, 5, 6, 13, 13])        # lengths 5, 0, 1, 7, 0
    S = oracle.sequential_varlen(Pp, R, s0, cu)
    # a sequence of length one is one step from its own s0
    one = oracle.sequential_btgd(Pp[None, 5:6], R, s0[2:3])[0]
    np.testing.assert_array_equal(S[5:6], one)
    # changing the initial state of sequence 3 changes nothing outside [6, 13)
    s0b = s0.copy()
    s0b[3] += 0.7
    S2 = oracle.sequential_varlen(Pp, R, s0b, cu)
    np.testing.assert_array_equal(S2[:6], S[:6])
    assert np.abs(S2[6:] - S[6:]).max() > 1e-6
    g = oracle.backward_varlen(xp, Wx, Pp, R, s0, S, dHp, cu)
    assert not g["ds0"][1].any() and not g["ds0"][4].any()    # empty sequences get no gradient
    # dropping the empty sequences changes no gradient of the others
    cu2 = np.array([0, 5, 6, 13])
    g2 = oracle.backward_varlen(xp, Wx, Pp, R, s0[[0, 2, 3]], S, dHp, cu2)
    np.testing.assert_array_equal(g2["dx"], g["dx"])
    np.testing.assert_array_equal(g2["ds0"], g["ds0"][[0, 2, 3]])


# ---------------------------------------------------------------------------
# the trunk layer: RMSNorm, SwiGLU, the block's wiring, bf16 rounding
# ---------------------------------------------------------------------------
def test_round_bf16_known_values():
    # bf16: 8 significant bits, so the spacing just above 1 is 2^-7
    v = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 3 * 2.0 ** -9, -2.0 ** -130, 0.1, 3.0e38])
    got = oracle.round_bf16(v)
    assert got[0] == 1.0                       # tie between 1 and 1 + 2^-7: to the even one
    assert got[1] == 1 + 2.0 ** -6             # tie between 1 + 2^-7 and 1 + 2^-6: to the even one
    assert got[2] == 1 + 2.0 ** -7             # nearest, no tie
    assert got[3] == -2.0 ** -130              # subnormals are kept
    assert got[4] == 0.10009765625             # bf16 0x3DCD
    assert abs(got[5] - 3.0e38) / 3.0e38 < 2.0 ** -8


def test_rmsnorm_closed_forms():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((5, 37)) * 3
    eps = 1e-6
    y = oracle.rmsnorm(v, np.ones(37), eps)
    ms = np.mean(v * v, axis=-1)
    # mean of squares after the norm is ms / (ms + eps)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-13)
    # positive scaling of a row leaves the output (eps = 0) unchanged, w scales columns
    w = rng.standard_normal(37)
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * v, w, 0.0), oracle.rmsnorm(v, w, 0.0), rtol=1e-13)
    np.testing.assert_allclose(oracle.rmsnorm(v, w, 0.0), oracle.rmsnorm(v, np.ones(37), 0.0) * w, rtol=1e-13)
    # one feature: v / |v| * w
    np.testing.assert_allclose(oracle.rmsnorm(np.array([[-2.5]]), np.array([0.5]), 0.0), [[-0.5]], rtol=1e-15)


def test_silu_and_swiglu_known_values():
    # logistic(1) = 1 / (1 + e^-1) = 0.7310585786300049
    np.testing.assert_allclose(oracle.silu(np.array([0.0, 1.0, -1.0, 40.0])),
                               [0.0, 0.7310585786300049, -0.2689414213699951, 40.0], rtol=1e-15)
    # identity projections: SwiGLU(z) = silu(z) * z elementwise
    z = np.array([[1.0, -1.0, 2.0]])
    I3 = np.eye(3)
    np.testing.assert_allclose(oracle.swiglu(z, I3, I3, I3), [[0.7310585786300049, 0.2689414213699951,
                                                               2.0 * 2.0 / (1 + math.exp(-2.0))]], rtol=1e-15)
    # F = 2 hidden units, D = 1: W_down mixes them, the gate and the up projection
    # are separate rows (a swapped gate/up would give another value)
    z = np.array([[2.0]])
    Wg, Wu, Wd = np.array([[1.0], [0.0]]), np.array([[3.0], [1.0]]), np.array([[1.0, 10.0]])
    want = (2.0 / (1 + math.exp(-2.0))) * 6.0 + 0.0
    np.testing.assert_allclose(oracle.swiglu(z, Wg, Wu, Wd), [[want]], rtol=1e-15)


def test_block_wiring():
    rng = np.random.default_rng(4)
    B, T, D, F = 2, 9, 6, 12
    x = rng.standard_normal((B, T, D))
    w1, w2 = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
    Wx = rng.standard_normal((4 * D, D)) / np.sqrt(D)
    bias = np.zeros((4, D))
    bias[2] = 3.0
    R = rng.uniform(-0.5, 0.5, (4, D))
    Wg, Wu, Wd = rng.standard_normal((F, D)), rng.standard_normal((F, D)), rng.standard_normal((D, F)) / F
    y, S = oracle.block_forward(x, w1, Wx, bias, R, w2, Wg, Wu, Wd)
    # the cell sees the normalised input and starts from zero
    P = oracle.preact(oracle.rmsnorm(x, w1), Wx, bias)
    np.testing.assert_allclose(S, oracle.sequential_btgd(P, R, np.zeros((B, 4, D))), rtol=0, atol=0)
    # W_down = 0: the block is x + h
    y0, _ = oracle.block_forward(x, w1, Wx, bias, R, w2, Wg, Wu, 0 * Wd)
    np.testing.assert_allclose(y0, x + S[:, :, 3, :], rtol=0, atol=0)
    # the FFN part is a function of the residual u = x + h alone: moving an
    # amount into x and the opposite into nothing else changes y by that amount
    # only through u (check: y - u equals SwiGLU(RMSNorm(u)))
    u = x + S[:, :, 3, :]
    ffn = oracle.swiglu(oracle.rmsnorm(u, w2).reshape(-1, D), Wg, Wu, Wd).reshape(B, T, D)
    np.testing.assert_allclose(y - u, ffn, rtol=1e-12, atol=1e-12)
    # a causal layer: changing x at step t leaves the outputs before t alone
    x2 = x.copy()
    x2[:, 5] += 1.0
    y2, _ = oracle.block_forward(x2, w1, Wx, bias, R, w2, Wg, Wu, Wd)
    assert np.array_equal(y2[:, :5], y[:, :5]) and np.abs(y2[:, 5:] - y[:, 5:]).max() > 1e-3
    # bf16 operands move the result by about the bf16 step, no more
    yb, _ = oracle.block_forward(x, w1, Wx, bias, R, w2, Wg, Wu, Wd, bf16_operands=True)
    assert 0 < np.abs(yb - y).max() < 2e-2


def test_block_backward_matches_finite_differences():
    """Central differences of L = sum(dY * y) along one random direction per
    argument pin every gradient of the trunk layer (norms, SwiGLU, the cell)."""
    rng = np.random.default_rng(5)
    B, T, D, F = 2, 6, 4, 8
    args = {"x": rng.standard_normal((B, T, D)), "norm1_w": rng.uniform(0.5, 1.5, D),
            "Wx": rng.standard_normal((4 * D, D)) / 2, "bias": np.zeros((4, D)), "R": rng.uniform(-0.5, 0.5, (4, D)),
            "norm2_w": rng.uniform(0.5, 1.5, D), "W_gate": rng.standard_normal((F, D)) / 2,
            "W_up": rng.standard_normal((F, D)) / 2, "W_down": rng.standard_normal((D, F)) / 3}
    args["bias"][2] = 3.0
    dY = rng.standard_normal((B, T, D))
    names = list(args)

    def loss(a):
        y, _ = oracle.block_forward(*[a[k] for k in names])
        return float(np.sum(dY * y))

    grads = oracle.block_backward(*[args[k] for k in names], dY)
    key = {"x": "dx", "norm1_w": "dnorm1_w", "Wx": "dWx", "bias": "dbias", "R": "dR", "norm2_w": "dnorm2_w",
           "W_gate": "dW_gate", "W_up": "dW_up", "W_down": "dW_down"}
    h = 1e-6
    for k in names:
        e = rng.standard_normal(args[k].shape)
        ap, am = dict(args), dict(args)
        ap[k] = args[k] + h * e
        am[k] = args[k] - h * e
        fd = (loss(ap) - loss(am)) / (2 * h)
        an = float(np.sum(grads[key[k]] * e))
        assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (k, fd, an)


# ---------------------------------------------------------------------------
# head-wise recurrent mixing (dense per-head Jacobians)
# ---------------------------------------------------------------------------
def _head_case(B=2, T=7, H=2, dh=3, seed=6, scale=0.4):
    rng = np.random.default_rng(seed)
    d = H * dh
    P = rng.standard_normal((B, T, 4, d))
    P[:, :, 2, :] += 3.0
    Rh = rng.uniform(-scale, scale, (4, H, dh, dh))
    s0 = np.stack([rng.standard_normal((B, d)), rng.uniform(0.5, 1.5, (B, d)), rng.standard_normal((B, d)),
                   rng.uniform(-0.5, 0.5, (B, d))], axis=1)
    return P, Rh, s0


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_head_mixing_with_diagonal_blocks_is_diag_mixing(forget):
    P, Rh, s0 = _head_case()
    _, H, dh, _ = Rh.shape
    r = np.stack([np.concatenate([np.diag(Rh[g, h]) for h in range(H)]) for g in range(4)])
    Rdiag = np.zeros_like(Rh)
    for g in range(4):
        for h in range(H):
            Rdiag[g, h] = np.diag(np.diag(Rh[g, h]))
    np.testing.assert_allclose(oracle.sequential_head(P, Rdiag, s0, forget), oracle.sequential_btgd(P, r, s0, forget),
                               rtol=1e-14, atol=1e-14)
    # d_head = 1 is diag mixing too
    P1, R1, s01 = _head_case(H=6, dh=1)
    np.testing.assert_allclose(oracle.sequential_head(P1, R1, s01, forget),
                               oracle.sequential_btgd(P1, R1[:, :, 0, 0], s01, forget), rtol=1e-14, atol=1e-14)


def test_head_mixing_direction_of_the_weight():
    """R[g, head, i, k] carries h of feature k into feature i: with only the
    (0, 1) entries set, feature 1 of the head has no recurrence at all (the diag
    cell with r = 0) while feature 0 depends on feature 1's trajectory."""
    P, _, s0 = _head_case(B=1, H=1, dh=2)
    Rh = np.zeros((4, 1, 2, 2))
    Rh[:, 0, 0, 1] = [0.3, -0.4, 0.5, 0.2]
    S = oracle.sequential_head(P, Rh, s0)
    free = oracle.sequential_btgd(P[..., 1:], np.zeros((4, 1)), s0[..., 1:])
    np.testing.assert_allclose(S[..., 1:], free, rtol=0, atol=1e-15)
    plain0 = oracle.sequential_btgd(P[..., :1], np.zeros((4, 1)), s0[..., :1])
    assert np.abs(S[..., 0] - plain0[..., 0]).max() > 1e-3


def test_head_jacobian_matches_finite_differences():
    P, Rh, s0 = _head_case(B=1, T=1)
    _, H, dh, _ = Rh.shape
    d = H * dh
    _, Jl, G = oracle._head_step_all(s0, P[:, 0], Rh, "sigmoid")
    J = oracle.head_jacobian(Jl, G, Rh)
    eps = 1e-6
    for hd in range(H):
        for e2 in range(4):
            for k in range(dh):
                sp, sm = s0.copy(), s0.copy()
                sp[0, e2, hd * dh + k] += eps
                sm[0, e2, hd * dh + k] -= eps
                fp, _, _ = oracle._head_step_all(sp, P[:, 0], Rh, "sigmoid")
                fm, _, _ = oracle._head_step_all(sm, P[:, 0], Rh, "sigmoid")
                col = (fp - fm)[0] / (2 * eps)          # (4, d)
                for e in range(4):
                    for i in range(dh):
                        got = J[0, hd, e * dh + i, e2 * dh + k]
                        assert abs(got - col[e, hd * dh + i]) <= 1e-6 * (1 + abs(got)), (hd, e, i, e2, k)
                # no coupling across heads
                other = [j for j in range(d) if j // dh != hd]
                assert np.abs(col[:, other]).max() == 0.0


def test_head_newton_prefix_exact_and_converges():
    P, Rh, s0 = _head_case(T=6)
    ref = oracle.sequential_head(P, Rh, s0)
    for K in (1, 3):
        S, _ = oracle.newton_head(P, Rh, s0, max_iters=K, fixed=True)
        np.testing.assert_allclose(S[:, :K], ref[:, :K], rtol=1e-12, atol=1e-12)
    S, st = oracle.newton_head(P, Rh, s0, max_iters=20, tol=1e-12)
    assert st["converged"] and not st["diverged"]
    np.testing.assert_allclose(S, ref, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("init", ["decoupled", "zero"])
def test_head_newton_from_either_guess(init):
    """Prefix exactness and convergence hold from both initial guesses; the
    decoupled guess is the diag cell's R = 0 trajectory whatever the mixing."""
    P, Rh, s0 = _head_case(T=9, seed=8)
    ref = oracle.sequential_head(P, Rh, s0)
    S1, _ = oracle.newton_head(P, Rh, s0, max_iters=1, fixed=True, init=init)
    np.testing.assert_allclose(S1[:, :1], ref[:, :1], rtol=1e-12, atol=1e-12)
    S, st = oracle.newton_head(P, Rh, s0, max_iters=30, tol=1e-12, init=init)
    assert st["converged"]
    np.testing.assert_allclose(S, ref, rtol=1e-10, atol=1e-10)


def _head_grad_case(B=2, T=5, H=2, dh=3, d_in=4, seed=12):
    rng = np.random.default_rng(seed)
    d = H * dh
    x = rng.standard_normal((B, T, d_in))
    Wx = rng.standard_normal((4 * d, d_in)) / math.sqrt(d_in)
    bias = np.zeros((4, d))
    bias[2] = np.linspace(3, 6, d)
    Rh = rng.uniform(-0.4, 0.4, (4, H, dh, dh))
    s0 = np.stack([rng.standard_normal((B, d)), rng.uniform(0.5, 1.5, (B, d)), rng.standard_normal((B, d)),
                   rng.uniform(-0.5, 0.5, (B, d))], axis=1)
    dH = rng.standard_normal((B, T, d))
    return x, Wx, bias, Rh, s0, dH


@pytest.mark.parametrize("forget", ["sigmoid", "exp"])
def test_head_backward_matches_finite_differences(forget):
    """Every gradient of L = sum dH * h for head mixing against central
    differences of the sequential head recurrence (step 1e-6)."""
    x, Wx, bias, Rh, s0, dH = _head_grad_case()

    def loss(x, Wx, bias, Rh, s0):
        P_ = oracle.preact(x, Wx, bias)
        return float((oracle.sequential_head(P_, Rh, s0, forget)[:, :, 3, :] * dH).sum())

    P = oracle.preact(x, Wx, bias)
    S = oracle.sequential_head(P, Rh, s0, forget)
    g = oracle.backward_head(x, Wx, P, Rh, s0, S, dH, forget)
    eps = 1e-6
    args = {"x": x, "Wx": Wx, "bias": bias, "Rh": Rh, "s0": s0}
    names = {"x": "dx", "Wx": "dWx", "bias": "db", "Rh": "dRh", "s0": "ds0"}
    rng = np.random.default_rng(3)
    for k, gname in names.items():
        a = args[k]
        idx = [tuple(rng.integers(0, n) for n in a.shape) for _ in range(6)]
        for ix in idx:
            ap, am = a.copy(), a.copy()
            ap[ix] += eps
            am[ix] -= eps
            fp = loss(**{**args, k: ap})
            fm = loss(**{**args, k: am})
            fd = (fp - fm) / (2 * eps)
            got = g[gname][ix]
            assert abs(got - fd) <= 1e-6 * (1 + abs(fd)), (k, ix, got, fd)


def test_head_backward_with_diagonal_blocks_is_the_diag_backward():
    x, Wx, bias, Rh, s0, dH = _head_grad_case(seed=14)
    _, H, dh, _ = Rh.shape
    Rdiag = np.zeros_like(Rh)
    for g_ in range(4):
        for h_ in range(H):
            Rdiag[g_, h_] = np.diag(np.diag(Rh[g_, h_]))
    r = np.stack([np.concatenate([np.diag(Rh[g_, h_]) for h_ in range(H)]) for g_ in range(4)])
    P = oracle.preact(x, Wx, bias)
    S = oracle.sequential_btgd(P, r, s0, "sigmoid")
    gh = oracle.backward_head(x, Wx, P, Rdiag, s0, S, dH, "sigmoid")
    gd = oracle.backward_btgd(x, Wx, P, r, s0, S, dH, "sigmoid")
    for k in ("dx", "dWx", "db", "ds0", "dP"):
        np.testing.assert_allclose(gh[k], gd[k], rtol=1e-12, atol=1e-12)
    dR_diag = np.stack([np.concatenate([np.diag(gh["dRh"][g_, h_]) for h_ in range(H)]) for g_ in range(4)])
    np.testing.assert_allclose(dR_diag, gd["dR"], rtol=1e-12, atol=1e-12)
