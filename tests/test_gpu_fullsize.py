"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark uses, on sampled outputs the oracle computes lane by lane.

Diag mixing makes every (batch row, feature) lane independent once P is
known, so the oracle only needs the rows of W_x and x that a sampled lane
touches.  Checked here:
  * the input projection on the sampled lanes (fp64 GEMM of the same
    bf16-rounded inputs),
  * slstm_sequential_step over the whole length T (the exact solution),
  * Newton after K fixed iterations: the first K steps are exact (a property
    of Newton from any guess), and the stats record K iterations,
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


@pytest.mark.parametrize("name", ["slstm_f32_b8_t1024_d256", "slstm_bf16_expgates_b16_t4096_d1024",
                                  "slstm_bf16_long_b4_t65536_d2048", "slstm_bf16_train_b8_t8192_d1024"])
def test_fullsize_forward_sampled(name, cuda_device):
    w = WORKLOADS[name]
    inp = make_inputs(w, with_dH=False)
    dev = torch.device("cuda")
    x, Wx, bias, R = (inp[k].to(dev) for k in ("x", "Wx", "bias", "R"))
    s0 = inp["s0"].to(dev)
    P = api.preact_gemm(x, Wx, bias)
    Sseq = api.sequential_step(P, R, s0, forget=w.forget)
    K = w.fixed_iters[0] if w.fixed_iters else 4
    Snt, st = api.newton_forward(P, R, s0, forget=w.forget, max_iters=K, fixed=True, tol=w.tol)
    torch.cuda.synchronize()
    stats = api.read_stats(st)
    assert stats["iters"] == K and stats["error"] in (0, 3)

    lanes = _lanes(w, 12, seed=w.seed)
    Pl = _oracle_P_lanes(inp, w, lanes)
    Pg = _gather(P, lanes)
    perr = float(np.abs(Pg - Pl).max() / (1 + np.abs(Pl).max()))
    assert perr < 1e-5, perr

    Rl = np.stack([as_f64(inp["R"][:, j]) for _, j in lanes])
    s0l = np.zeros((len(lanes), 4))
    Sref = oracle.sequential(Pl, Rl, s0l, w.forget)
    tol = TOL[w.dtype]
    e_seq = _herr(_gather(Sseq, lanes)[:, :, 3], Sref[:, :, 3])
    assert e_seq <= tol, e_seq
    e_pre = _herr(_gather(Snt, lanes)[:, :K, 3], Sref[:, :K, 3])
    assert e_pre <= tol, e_pre
    print(f"{name}: P err {perr:.2e}, sequential h err {e_seq:.2e}, Newton prefix err {e_pre:.2e}, "
          f"stats {stats['iters']} it, diverged={stats['diverged']}")


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
