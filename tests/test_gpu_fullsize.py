"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark uses, on sampled outputs the oracle computes lane by lane.

Diag mixing makes every (batch row, feature) lane independent once P is
known, so the oracle only needs the rows of W_x and x that a sampled lane
touches.  Checked here:
  * the input projection on the sampled lanes (fp64 GEMM of the same
    bf16-rounded inputs),
  * slstm_sequential_step over the whole length T (the exact solution),
  * Newton after the workload's fixed K iterations from the decoupled guess,
    every step against the fp64 iterate after the same K,
  * the converged tolerance run, every step of h against the sequential
    trajectory, with the GPU's and the fp64 run's iteration counts,
  * one iteration from a given guess near the solution, in both carry
    modes, against the fp64 iteration from the same guess,
  * the backward at the exact solution (training workload): dR, db and the
    W_x-gradient rows of sampled features, summed over every batch row.
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import api
from nonlinear_rnn_pararnn_b200.workloads import WORKLOADS, as_f64, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 5e-3}


def _lanes(w, n, seed):
    rng = np.random.default_rng(seed)
    bs = rng.integers(0, w.B, size=n)
    js = rng.integers(0, w.d_h, size=n)
    bs[0], js[0] = w.B - 1, w.d_h - 1       # the last lane is always in the sample
    return list(zip(bs.tolist(), js.tolist()))


def _oracle_P_lanes(inp, w, lanes):
    """P for the sampled lanes, (L, T, 4), fp64 GEMM of the lane's rows."""
    out = np.zeros((len(lanes), w.T, 4))
    bias = as_f64(inp["bias"])
    by_b = {}
    for i, (b, j) in enumerate(lanes):
        by_b.setdefault(b, []).append((i, j))
    Wx = inp["Wx"]
    for b, items in by_b.items():
        xb = as_f64(inp["x"][b])                                    # (T, d_in)
        rows = [g * w.d_h + j for _, j in items for g in range(4)]
        Wr = as_f64(Wx[rows])                                       # (4n, d_in)
        bi = np.array([bias[g, j] for _, j in items for g in range(4)])
        Pb = oracle.gemm(xb, Wr, tb=True, bias=bi)                  # (T, 4n)
        for q, (i, _) in enumerate(items):
            out[i] = Pb[:, 4 * q: 4 * q + 4]
    return out


def _gather(S, lanes):
    """(B,T,4,d) device tensor -> (L, T, 4) fp64 for the sampled lanes."""
    idx_b = torch.tensor([b for b, _ in lanes], device=S.device)
    idx_j = torch.tensor([j for _, j in lanes], device=S.device)
    g = S[idx_b, :, :, idx_j]                                       # (L, T, 4)
    return as_f64(g.cpu())


def _herr(h, href):
    return float((np.abs(h - href) / (1 + np.abs(href))).max())


FULL = ["slstm_f32_b8_t1024_d256", "slstm_bf16_expgates_b16_t4096_d1024", "slstm_bf16_long_b4_t65536_d2048",
        "slstm_bf16_train_b8_t8192_d1024"]


def _serr(S, Sref):
    """max over every step and slot of |dS| / (1 + |S|)."""
    return float((np.abs(S - Sref) / (1 + np.abs(Sref))).max())


def _perturb(S, rng, eps=1e-3):
    """Seeded noise near a trajectory: relative eps on c, n and h, absolute
    eps on the stabiliser m (a relative change of m would rescale c and n by
    exp(eps |m|))."""
    u = rng.uniform(-1, 1, size=S.shape)
    out = S * (1 + eps * u)
    out[..., 2] = S[..., 2] + eps * u[..., 2]
    return out


def _setup(w):
    inp = make_inputs(w, with_dH=False)
    dev = torch.device("cuda")
    x, Wx, bias, R = (inp[k].to(dev) for k in ("x", "Wx", "bias", "R"))
    s0 = inp["s0"].to(dev)
    P = api.preact_gemm(x, Wx, bias)
    lanes = _lanes(w, 12, seed=w.seed)
    Pl = _oracle_P_lanes(inp, w, lanes)
    Rl = np.stack([as_f64(inp["R"][:, j]) for _, j in lanes])
    s0l = np.zeros((len(lanes), 4))
    return inp, P, R, s0, lanes, Pl, Rl, s0l


@pytest.mark.parametrize("name", FULL)
def test_fullsize_forward_sampled(name, cuda_device):
    """Every step of the sampled lanes: the sequential stepping, the Newton
    iterate after the fixed K of the workload (against the fp64 iterate after
    the same K from the same guess: the decoupled trajectory and its default
    refinement sweeps), and the converged tolerance run (against the
    sequential trajectory)."""
    w = WORKLOADS[name]
    inp, P, R, s0, lanes, Pl, Rl, s0l = _setup(w)
    Sseq = api.sequential_step(P, R, s0, forget=w.forget)
    torch.cuda.synchronize()
    Pg = _gather(P, lanes)
    perr = float(np.abs(Pg - Pl).max() / (1 + np.abs(Pl).max()))
    assert perr < 1e-5, perr
    Sref = oracle.sequential(Pl, Rl, s0l, w.forget)
    tol = TOL[w.dtype]
    e_seq = _herr(_gather(Sseq, lanes)[:, :, 3], Sref[:, :, 3])
    assert e_seq <= tol, e_seq
    del Sseq

    K = w.fixed_iters[0] if w.fixed_iters else 4
    Snt, st = api.newton_forward(P, R, s0, forget=w.forget, max_iters=K, fixed=True, tol=w.tol)
    stats = api.read_stats(st)
    assert stats["iters"] == K and stats["error"] == 0, stats
    SK, _ = oracle.newton(Pl, Rl, s0l, w.forget, max_iters=K, fixed=True, tol=w.tol, sweeps=api.DEFAULT_GUESS_SWEEPS)
    e_fix = _serr(_gather(Snt, lanes), SK)
    assert e_fix <= tol, e_fix
    del Snt

    Sc, stc = api.newton_forward(P, R, s0, forget=w.forget, max_iters=w.max_iters, fixed=False, tol=w.tol)
    cst = api.read_stats(stc)
    _, ost = oracle.newton(Pl, Rl, s0l, w.forget, max_iters=w.max_iters, tol=w.tol, sweeps=api.DEFAULT_GUESS_SWEEPS)
    print(f"{name}: P err {perr:.2e}, sequential h err {e_seq:.2e}, K={K} iterate err {e_fix:.2e}; "
          f"tolerance run: GPU {cst['iters']} iterations (all lanes) scaled residuals {cst['max_scaled_F']}, "
          f"fp64 {ost['iters']} iterations (sampled lanes) {list(ost['max_scaled_F'])}")
    assert cst["converged"] and cst["error"] == 0, cst
    assert ost["converged"] and cst["iters"] >= ost["iters"]
    e_conv = _herr(_gather(Sc, lanes)[:, :, 3], Sref[:, :, 3])
    assert e_conv <= tol, e_conv


@pytest.mark.parametrize("carry_mode", [1, 2])
@pytest.mark.parametrize("name", FULL)
def test_fullsize_warm_start_one_iteration(name, carry_mode, cuda_device):
    """One Newton iteration from a guess near the solution, at full size in
    both carry modes (the fused look-back over every chunk, and the two-pass
    scan), compared at every step and slot of the sampled lanes with the fp64
    iteration from the same guess.  The sampled lanes' guess is the oracle's
    sequential trajectory with seeded noise of 1e-3 (_perturb), rounded to
    fp32; the other lanes (independent of these) start from the GPU's
    stepping, perturbed the same way."""
    w = WORKLOADS[name]
    inp, P, R, s0, lanes, Pl, Rl, s0l = _setup(w)
    S = api.sequential_step(P, R, s0, forget=w.forget)
    gen = torch.Generator(device="cuda").manual_seed(7)
    u = torch.rand(S.shape, generator=gen, device="cuda") * 2 - 1
    S[:, :, (0, 1, 3), :] *= 1 + 1e-3 * u[:, :, (0, 1, 3), :]
    S[:, :, 2, :] += 1e-3 * u[:, :, 2, :]
    del u
    rng = np.random.default_rng(w.seed + 100)
    Sref = oracle.sequential(Pl, Rl, s0l, w.forget)
    gl = _perturb(Sref, rng).astype(np.float32)
    for i, (b, j) in enumerate(lanes):
        S[b, :, :, j] = torch.from_numpy(gl[i]).to("cuda")
    S, st = api.newton_forward(P, R, s0, forget=w.forget, max_iters=1, fixed=True, tol=w.tol, S=S, init="given",
                               carry_mode=carry_mode)
    stats = api.read_stats(st)
    assert stats["iters"] == 1 and stats["error"] == 0, stats
    S1, _ = oracle.newton(Pl, Rl, s0l, w.forget, max_iters=1, fixed=True, tol=w.tol, init="given",
                          S_init=gl.astype(np.float64))
    got = _gather(S, lanes)
    e = _serr(got, S1)
    # the step moved the guess: on average the result is much closer to the
    # solution (not at every element: where the stabiliser's max is near a
    # tie, the guess's noise can pick the other branch, and the error there
    # stays first order)
    dist = lambda a: float((np.abs(a - Sref) / (1 + np.abs(Sref))).mean())
    moved = dist(gl.astype(np.float64)) / max(dist(got), 1e-12)
    print(f"{name} carry {carry_mode}: one-iteration err {e:.2e}, guess/result mean distance to solution ratio {moved:.1f}")
    assert e <= TOL[w.dtype], e
    assert moved > 10.0


def test_fullsize_backward_sampled(cuda_device):
    w = WORKLOADS["slstm_bf16_train_b8_t8192_d1024"]
    inp = make_inputs(w, with_dH=True)
    dev = torch.device("cuda")
    x, Wx, bias, R, s0, dH = (inp[k].to(dev) for k in ("x", "Wx", "bias", "R", "s0", "dH"))
    P = api.preact_gemm(x, Wx, bias)
    S = api.sequential_step(P, R, s0, forget=w.forget)
    g = api.newton_backward(x, Wx, P, R, s0, S, dH, forget=w.forget)
    torch.cuda.synchronize()

    rng = np.random.default_rng(44)
    feats = sorted(set(rng.integers(0, w.d_h, size=6).tolist()) | {w.d_h - 1})
    lanes = [(b, j) for j in feats for b in range(w.B)]
    Pl = _oracle_P_lanes(inp, w, lanes)
    Rl = np.stack([as_f64(inp["R"][:, j]) for _, j in lanes])
    s0l = np.zeros((len(lanes), 4))
    Sl = oracle.sequential(Pl, Rl, s0l, w.forget)
    dHl = np.stack([as_f64(inp["dH"][b, :, j]) for b, j in lanes])
    dP, dR, db, ds0 = oracle.bptt(Pl, Rl, s0l, Sl, dHl, w.forget)
    nb = w.B
    dR_ref = dR.reshape(len(feats), nb, 4).sum(axis=1)       # (F, 4)
    db_ref = db.reshape(len(feats), nb, 4).sum(axis=1)
    dR_g = as_f64(g["dR"].cpu())[:, feats].T
    db_g = as_f64(g["db"].cpu())[:, feats].T
    xsT = np.ascontiguousarray(as_f64(inp["x"].reshape(w.B * w.T, w.d_in)).T)   # (d_in, B*T)
    dW_g = as_f64(g["dWx"].cpu())
    errs = {}
    errs["dR"] = np.abs(dR_g - dR_ref).max() / (1 + np.abs(dR_ref).max())
    errs["db"] = np.abs(db_g - db_ref).max() / (1 + np.abs(db_ref).max())
    for fi, j in enumerate(feats):
        # dP rows of feature j for all (b, t): (B*T, 4), lane order b-major
        dPjT = np.ascontiguousarray(dP[fi * nb:(fi + 1) * nb].reshape(nb * w.T, 4).T)  # (4, B*T)
        ref_rows = oracle.gemm(dPjT, xsT, tb=True)             # (4, d_in) = dP_j^T x
        got = dW_g[[gg * w.d_h + j for gg in range(4)]]
        e = np.abs(got - ref_rows).max() / (1 + np.abs(ref_rows).max())
        errs[f"dWx[{j}]"] = e
    print("backward errors", {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= 1e-3, (k, v)
