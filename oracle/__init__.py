"""Plain fp64 CPU oracle for the Newton-solved diag-mix sLSTM.

TEST INFRASTRUCTURE ONLY.  The product library never imports, links or calls
anything here; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` do.  The arithmetic
lives in ``slstm_oracle.c`` (fp64, libm, one lane and one step at a time);
this module compiles it with gcc on first use and marshals numpy arrays.

Pins that tie the oracle to the pages and to mathematics (not to itself) are
in ``tests/test_oracle_pins.py``.  Every function below is pinned; the oracle
header in ``slstm_oracle.c`` lists the page sections each one follows.

Layout conversions: the library boundary uses (B, T, 4, d_h) for P and S,
(4, d_h) for R and bias, (B, 4, d_h) for s0, (B, T, d_h) for dH.  The C code
works lane-major: one lane is one (b, j) pair.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "slstm_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

FORGET_SIGMOID = 0
FORGET_EXP = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (no fast-math, IEEE fp64)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        D = ctypes.POINTER(ctypes.c_double)
        I = ctypes.c_int
        IP = ctypes.POINTER(ctypes.c_int)
        lib.oracle_step.argtypes = [D, D, D, I, D, D, D]
        lib.oracle_sequential.argtypes = [I, I, D, D, D, I, D]
        lib.oracle_sequential_unstabilised.argtypes = [I, I, D, D, D, I, D, D, D]
        lib.oracle_affine_solve.argtypes = [I, I, D, D, D, I, D]
        lib.oracle_newton.argtypes = [I, I, D, D, D, I, I, I, ctypes.c_double, I, I, I, D, D, D, D,
                                      IP, IP, IP]
        lib.oracle_bptt.argtypes = [I, I, D, D, D, D, D, I, D, D, D, D]
        lib.oracle_gemm.argtypes = [I, I, I, D, I, D, I, D, D]
        for f in ("oracle_step", "oracle_sequential", "oracle_sequential_unstabilised",
                  "oracle_affine_solve", "oracle_newton", "oracle_bptt", "oracle_gemm"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _forget_code(forget) -> int:
    if forget in (FORGET_SIGMOID, "sigmoid"):
        return FORGET_SIGMOID
    if forget in (FORGET_EXP, "exp"):
        return FORGET_EXP
    raise ValueError(f"unknown forget mode {forget!r}")


# ----------------------------------------------------------------------------
# layout helpers (boundary layout <-> lane-major)
# ----------------------------------------------------------------------------
def lanes_from_btgd(P: np.ndarray) -> np.ndarray:
    """(B, T, 4, d) -> (B*d, T, 4), lane index = b*d + j."""
    B, T, four, d = P.shape
    assert four == 4
    return _f64(np.transpose(P, (0, 3, 1, 2)).reshape(B * d, T, 4))


def btgd_from_lanes(X: np.ndarray, B: int, d: int) -> np.ndarray:
    """(B*d, T, 4) -> (B, T, 4, d)."""
    T = X.shape[1]
    return np.ascontiguousarray(np.transpose(X.reshape(B, d, T, 4), (0, 2, 3, 1)))


def lanes_from_gd(R: np.ndarray, B: int) -> np.ndarray:
    """(4, d) per-feature parameters -> (B*d, 4)."""
    four, d = R.shape
    return _f64(np.broadcast_to(np.transpose(R)[None], (B, d, 4)).reshape(B * d, 4))


def lanes_from_bgd(s0: np.ndarray) -> np.ndarray:
    """(B, 4, d) -> (B*d, 4)."""
    B, four, d = s0.shape
    return _f64(np.transpose(s0, (0, 2, 1)).reshape(B * d, 4))


def bgd_from_lanes(X: np.ndarray, B: int, d: int) -> np.ndarray:
    return np.ascontiguousarray(np.transpose(X.reshape(B, d, 4), (0, 2, 1)))


# ----------------------------------------------------------------------------
# lane-major entry points
# ----------------------------------------------------------------------------
def step(sp, p, r, forget="sigmoid"):
    """One stabilised step; returns (s_t, J (4x4), G (4x4))."""
    lib = _load()
    sp, p, r = _f64(sp), _f64(p), _f64(r)
    out = np.zeros(4)
    J = np.zeros(16)
    G = np.zeros(16)
    lib.oracle_step(_ptr(sp), _ptr(p), _ptr(r), _forget_code(forget), _ptr(out), _ptr(J), _ptr(G))
    return out, J.reshape(4, 4), G.reshape(4, 4)


def sequential(P, R, s0, forget="sigmoid") -> np.ndarray:
    """P (L,T,4), R (L,4), s0 (L,4) -> S (L,T,4) by stepping through time."""
    lib = _load()
    P, R, s0 = _f64(P), _f64(R), _f64(s0)
    L, T, _ = P.shape
    S = np.zeros((L, T, 4))
    lib.oracle_sequential(L, T, _ptr(P), _ptr(R), _ptr(s0), _forget_code(forget), _ptr(S))
    return S


def sequential_unstabilised(P, R, s0, forget="sigmoid"):
    """Unstabilised recurrence; returns (c_u, n_u, h), each (L, T)."""
    lib = _load()
    P, R, s0 = _f64(P), _f64(R), _f64(s0)
    L, T, _ = P.shape
    cu, nu, h = np.zeros((L, T)), np.zeros((L, T)), np.zeros((L, T))
    lib.oracle_sequential_unstabilised(L, T, _ptr(P), _ptr(R), _ptr(s0), _forget_code(forget),
                                       _ptr(cu), _ptr(nu), _ptr(h))
    return cu, nu, h


def affine_solve(A, b, y0=None, reverse=False) -> np.ndarray:
    """A (L,T,4,4), b (L,T,4) -> y (L,T,4); see oracle_affine_solve."""
    lib = _load()
    A, b = _f64(A), _f64(b)
    L, T = b.shape[:2]
    y = np.zeros((L, T, 4))
    y0p = None
    if y0 is not None:
        y0 = _f64(y0)
        y0p = _ptr(y0)
    lib.oracle_affine_solve(L, T, _ptr(A), _ptr(b), y0p, 1 if reverse else 0, _ptr(y))
    return y


INIT_DECOUPLED = 0
INIT_ZERO = 1
INIT_GIVEN = 2
_INITS = {"decoupled": INIT_DECOUPLED, "zero": INIT_ZERO, "given": INIT_GIVEN}
_RESIDUAL_MODES = {"scaled": 0, "raw": 1}


def newton(P, R, s0, forget="sigmoid", max_iters=8, fixed=False, tol=1e-5, init="decoupled",
           residual_mode="scaled", S_init=None, sweeps=0):
    """fp64 Newton; returns (S, stats dict).

    init: "decoupled" (the trajectory with R = 0, then `sweeps` refinement
    sweeps; the default), "zero", or "given" with S_init (L, T, 4) as the
    initial guess.  residual_mode: "scaled" (max |F| / (1 + |s|) <= tol) or
    "raw" (max |F| <= tol)."""
    lib = _load()
    P, R, s0 = _f64(P), _f64(R), _f64(s0)
    L, T, _ = P.shape
    code = _INITS[init]
    if code == INIT_GIVEN:
        if S_init is None:
            raise ValueError("init='given' needs S_init")
        S = _f64(S_init).copy()
        if S.shape != (L, T, 4):
            raise ValueError(f"S_init shape {S.shape} != {(L, T, 4)}")
    else:
        S = np.zeros((L, T, 4))
    hr = np.full(max(max_iters, 1), np.nan)
    hs = np.full(max(max_iters, 1), np.nan)
    ir = np.zeros(2)
    it, conv, div = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    lib.oracle_newton(L, T, _ptr(P), _ptr(R), _ptr(s0), _forget_code(forget), int(max_iters),
                      1 if fixed else 0, float(tol), code, int(sweeps), _RESIDUAL_MODES[residual_mode], _ptr(S),
                      _ptr(hr), _ptr(hs), _ptr(ir), ctypes.byref(it), ctypes.byref(conv), ctypes.byref(div))
    return S, {"iters": it.value, "converged": bool(conv.value), "diverged": bool(div.value),
               "max_abs_F": hr[: it.value].copy(), "max_scaled_F": hs[: it.value].copy(),
               "init_max_abs_F": float(ir[0]), "init_max_scaled_F": float(ir[1])}


def bptt(P, R, s0, S, dH, forget="sigmoid"):
    """Reverse-time adjoint + cell VJP; returns (dP (L,T,4), dR (L,4), db (L,4), ds0 (L,4))."""
    lib = _load()
    P, R, s0, S, dH = _f64(P), _f64(R), _f64(s0), _f64(S), _f64(dH)
    L, T, _ = P.shape
    dP = np.zeros((L, T, 4))
    dR, db, ds0 = np.zeros((L, 4)), np.zeros((L, 4)), np.zeros((L, 4))
    lib.oracle_bptt(L, T, _ptr(P), _ptr(R), _ptr(s0), _ptr(S), _ptr(dH), _forget_code(forget),
                    _ptr(dP), _ptr(dR), _ptr(db), _ptr(ds0))
    return dP, dR, db, ds0


def gemm(A, B, ta=False, tb=False, bias=None) -> np.ndarray:
    """C = op(A) op(B) (+ bias); op(A) is (M,K), op(B) is (K,N)."""
    lib = _load()
    A, B = _f64(A), _f64(B)
    M, K = (A.shape[1], A.shape[0]) if ta else A.shape
    K2, N = (B.shape[1], B.shape[0]) if tb else B.shape
    assert K == K2, (A.shape, B.shape, ta, tb)
    C = np.zeros((M, N))
    bp = None
    if bias is not None:
        bias = _f64(bias)
        bp = _ptr(bias)
    lib.oracle_gemm(M, N, K, _ptr(A), int(ta), _ptr(B), int(tb), bp, _ptr(C))
    return C


# ----------------------------------------------------------------------------
# boundary-layout conveniences (full tensors; small problems only)
# ----------------------------------------------------------------------------
def preact(x, Wx, bias) -> np.ndarray:
    """x (B,T,d_in), Wx (4 d_h, d_in), bias (4, d_h) -> P (B,T,4,d_h)."""
    B, T, d_in = x.shape
    d_h = Wx.shape[0] // 4
    P = gemm(np.asarray(x).reshape(B * T, d_in), Wx, tb=True, bias=np.asarray(bias).reshape(-1))
    return P.reshape(B, T, 4, d_h)


def sequential_btgd(P, R, s0, forget="sigmoid") -> np.ndarray:
    B, T, _, d = P.shape
    S = sequential(lanes_from_btgd(P), lanes_from_gd(R, B), lanes_from_bgd(s0), forget)
    return btgd_from_lanes(S, B, d)


def newton_btgd(P, R, s0, forget="sigmoid", max_iters=8, fixed=False, tol=1e-5, init="decoupled",
                residual_mode="scaled", S_init=None, sweeps=0):
    B, T, _, d = P.shape
    Si = lanes_from_btgd(S_init) if S_init is not None else None
    S, st = newton(lanes_from_btgd(P), lanes_from_gd(R, B), lanes_from_bgd(s0), forget,
                   max_iters, fixed, tol, init, residual_mode, Si, sweeps)
    return btgd_from_lanes(S, B, d), st


def backward_btgd(x, Wx, P, R, s0, S, dH, forget="sigmoid"):
    """Full gradients of L = sum dH * h: returns dict dx, dWx, dR, db, ds0, dP."""
    B, T, _, d = P.shape
    d_in = Wx.shape[1]
    dHl = _f64(np.transpose(dH, (0, 2, 1)).reshape(B * d, T))
    dP, dR, db, ds0 = bptt(lanes_from_btgd(P), lanes_from_gd(R, B), lanes_from_bgd(s0),
                           lanes_from_btgd(S), dHl, forget)
    dP_b = btgd_from_lanes(dP, B, d)                       # (B,T,4,d)
    dP2 = dP_b.reshape(B * T, 4 * d)
    dx = gemm(dP2, Wx).reshape(B, T, d_in)                  # dP W_x
    dWx = gemm(dP2, np.asarray(x).reshape(B * T, d_in), ta=True)  # dP^T x
    dR_g = dR.reshape(B, d, 4).sum(axis=0).T.copy()         # (4, d)
    db_g = db.reshape(B, d, 4).sum(axis=0).T.copy()
    return {"dx": dx, "dWx": dWx, "dR": dR_g, "db": db_g,
            "ds0": bgd_from_lanes(ds0, B, d), "dP": dP_b}


# ----------------------------------------------------------------------------
# packed ragged sequences ("sLSTM in this library", section "Packed sequences":
# sequences concatenated along time, exclusive-prefix offsets cu_seqlens, one
# initial state per sequence).  The packed problem is, by definition, the
# independent problems of its sequences; these functions cut the packed
# arrays at the offsets and run the pinned per-sequence functions above.
# ----------------------------------------------------------------------------
def _segments(cu):
    cu = [int(v) for v in np.asarray(cu).reshape(-1)]
    return [(k, cu[k], cu[k + 1]) for k in range(len(cu) - 1)]


def sequential_varlen(P, R, s0, cu, forget="sigmoid") -> np.ndarray:
    """P (total_T, 4, d) packed; s0 (n, 4, d) or None -> S (total_T, 4, d)."""
    P = _f64(P)
    d = P.shape[2]
    S = np.zeros_like(P)
    for k, a, b in _segments(cu):
        if b > a:
            s0k = np.zeros((1, 4, d)) if s0 is None else _f64(s0)[k:k + 1]
            S[a:b] = sequential_btgd(P[None, a:b], R, s0k, forget)[0]
    return S


def newton_varlen_fixed(P, R, s0, cu, forget="sigmoid", K=4, init="decoupled", sweeps=0) -> np.ndarray:
    """K Newton iterations from the given kind of guess ("decoupled" or "zero")
    on every sequence (fixed-K mode)."""
    P = _f64(P)
    d = P.shape[2]
    S = np.zeros_like(P)
    for k, a, b in _segments(cu):
        if b > a:
            s0k = np.zeros((1, 4, d)) if s0 is None else _f64(s0)[k:k + 1]
            S[a:b] = newton_btgd(P[None, a:b], R, s0k, forget, max_iters=K, fixed=True, tol=0.0,
                                  init=init, sweeps=sweeps)[0][0]
    return S


def backward_varlen(x, Wx, P, R, s0, S, dH, cu, forget="sigmoid"):
    """Gradients of L = sum dH * h over all sequences: dx (total_T, d_in), dWx, dR, db
    (summed over sequences) and ds0 (n, 4, d; zero for empty sequences)."""
    x, P, S, dH = _f64(x), _f64(P), _f64(S), _f64(dH)
    Wx = _f64(Wx)
    d = P.shape[2]
    segs = _segments(cu)
    out = {"dx": np.zeros_like(x), "dWx": np.zeros(Wx.shape), "dR": np.zeros((4, d)), "db": np.zeros((4, d)),
           "ds0": np.zeros((len(segs), 4, d)), "dP": np.zeros_like(P)}
    for k, a, b in segs:
        if b == a:
            continue
        s0k = np.zeros((1, 4, d)) if s0 is None else _f64(s0)[k:k + 1]
        g = backward_btgd(x[None, a:b], Wx, P[None, a:b], R, s0k, S[None, a:b], dH[None, a:b], forget)
        out["dx"][a:b] = g["dx"][0]
        out["dP"][a:b] = g["dP"][0]
        out["ds0"][k] = g["ds0"][0]
        for key in ("dWx", "dR", "db"):
            out[key] += g[key]
    return out


# ----------------------------------------------------------------------------
# the trunk layer ("sLSTM in this library", section "Stacking":
# RMSNorm -> ParaRNN(ParaSLSTM) -> residual -> RMSNorm -> SwiGLU -> residual).
# Readings where the section is silent: RMSNorm(v) = v / sqrt(mean(v^2) + eps)
# * w over the model axis; SwiGLU(z) = W_down (silu(W_gate z) * (W_up z)) with
# no biases; the cell has d_in = d_h = d_model and starts from the zero state.
# Its GEMM operands are bf16 (the library's compute type): with
# ``bf16_operands`` the normalised activations and the SwiGLU product are
# rounded to bf16 (nearest, ties to even) where they enter a GEMM.
# ----------------------------------------------------------------------------
def round_bf16(a) -> np.ndarray:
    """Nearest bf16 value of each fp64 entry (ties to even), as fp64."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(_f64(a))).to(torch.bfloat16).to(torch.float64).numpy()


def rmsnorm(v, w, eps=1e-6) -> np.ndarray:
    v = _f64(v)
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps) * _f64(w)


def silu(a) -> np.ndarray:
    a = _f64(a)
    return a / (1.0 + np.exp(-a))


def swiglu(z, W_gate, W_up, W_down, bf16_operands=False) -> np.ndarray:
    """z (M, D), W_gate / W_up (F, D), W_down (D, F) -> (M, D)."""
    z = _f64(z)
    g = gemm(z, W_gate, tb=True)
    u = gemm(z, W_up, tb=True)
    a = silu(g) * u
    if bf16_operands:
        a = round_bf16(a)
    return gemm(a, W_down, tb=True)


def block_forward(x, norm1_w, Wx, bias, R, norm2_w, W_gate, W_up, W_down, forget="sigmoid", eps=1e-6,
                  bf16_operands=False):
    """x (B, T, D) -> (y (B, T, D), S (B, T, 4, D)), the cell solved exactly
    (sequentially) from the zero state."""
    x = _f64(x)
    B, T, D = x.shape
    z1 = rmsnorm(x, norm1_w, eps)
    if bf16_operands:
        z1 = round_bf16(z1)
    P = preact(z1, Wx, bias)
    S = sequential_btgd(P, R, np.zeros((B, 4, D)), forget)
    u = x + S[:, :, 3, :]
    z2 = rmsnorm(u, norm2_w, eps)
    if bf16_operands:
        z2 = round_bf16(z2)
    y = u + swiglu(z2.reshape(B * T, D), W_gate, W_up, W_down, bf16_operands).reshape(B, T, D)
    return y, S


def rmsnorm_backward(v, w, dz, eps=1e-6):
    """Gradients of sum(dz * rmsnorm(v, w)) with respect to v and w.
    With r = (mean(v^2) + eps)^(-1/2) and z_i = w_i v_i r over the model axis
    of size D: dv_j = r w_j dz_j - (r^3 v_j / D) sum_i dz_i w_i v_i and
    dw_i = sum over rows of dz_i v_i r."""
    v, w, dz = _f64(v), _f64(w), _f64(dz)
    D = v.shape[-1]
    r = 1.0 / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    s = np.sum(dz * w * v, axis=-1, keepdims=True)
    dv = r * w * dz - (r ** 3) * v * s / D
    dw = np.sum((dz * v * r).reshape(-1, D), axis=0)
    return dv, dw


def block_backward(x, norm1_w, Wx, bias, R, norm2_w, W_gate, W_up, W_down, dY, forget="sigmoid", eps=1e-6):
    """Gradients of L = sum(dY * y) for y = block_forward(...) without operand
    rounding (the rounded forward is piecewise constant in its operands; its
    gradient is read as that of the unrounded function).  Returns dict dx,
    dnorm1_w, dWx, dbias, dR, dnorm2_w, dW_gate, dW_up, dW_down."""
    x, dY = _f64(x), _f64(dY)
    B, T, D = x.shape
    M = B * T
    z1 = rmsnorm(x, norm1_w, eps)
    P = preact(z1, Wx, bias)
    S = sequential_btgd(P, R, np.zeros((B, 4, D)), forget)
    u = x + S[:, :, 3, :]
    z2 = rmsnorm(u, norm2_w, eps).reshape(M, D)
    g = gemm(z2, W_gate, tb=True)
    v = gemm(z2, W_up, tb=True)
    sg = 1.0 / (1.0 + np.exp(-g))
    a = g * sg * v
    dY2 = dY.reshape(M, D)
    dW_down = gemm(dY2, a, ta=True)                       # (D, F)
    da = gemm(dY2, W_down)                                # (M, F)
    dg = da * v * sg * (1.0 + g * (1.0 - sg))             # silu'(g) = s (1 + g (1 - s))
    dv = da * g * sg
    dW_gate = gemm(dg, z2, ta=True)
    dW_up = gemm(dv, z2, ta=True)
    dz2 = gemm(dg, W_gate) + gemm(dv, W_up)
    du_n, dnorm2_w = rmsnorm_backward(u.reshape(M, D), norm2_w, dz2, eps)
    du = dY + du_n.reshape(B, T, D)
    cell = backward_btgd(z1, Wx, P, R, np.zeros((B, 4, D)), S, du, forget)
    dx_n, dnorm1_w = rmsnorm_backward(x, norm1_w, cell["dx"], eps)
    return {"dx": du + dx_n, "dnorm1_w": dnorm1_w, "dWx": cell["dWx"], "dbias": cell["db"], "dR": cell["dR"],
            "dnorm2_w": dnorm2_w, "dW_gate": dW_gate, "dW_up": dW_up, "dW_down": dW_down}


# ----------------------------------------------------------------------------
# head-wise recurrent mixing ("sLSTM in this library", section on mix='head':
# block-diagonal R of shape (4, n_heads, d_head, d_head) run through the same
# Newton loop; the dense-Jacobian form is the reference for factorised
# kernels).  The gate pre-activations of feature j = head * d_head + i are
#   a_g[j] = P_g[j] + sum_k R[g, head, i, k] h_{t-1}[head * d_head + k],
# and the rest of the step is the diag cell's: the pinned lane step is called
# with r = 0 on the mixed pre-activations.  Small problems only (Python loops).
# ----------------------------------------------------------------------------
def _head_mix(Rh, h):
    """Rh (4, H, dh, dh), h (B, d) -> (B, 4, d) recurrent contributions."""
    B, d = h.shape
    _, H, dh, _ = Rh.shape
    return np.einsum("ghik,bhk->bghi", Rh, h.reshape(B, H, dh)).reshape(B, 4, d)


def _head_step_all(S_prev, Pt, Rh, forget):
    """One step for every (b, j): returns s (B, 4, d), Jl (B, d, 4, 4) with the
    recurrent path left out, G (B, d, 4, 4)."""
    B, _, d = S_prev.shape
    A = Pt + _head_mix(Rh, S_prev[:, 3, :])
    s = np.zeros((B, 4, d))
    Jl = np.zeros((B, d, 4, 4))
    G = np.zeros((B, d, 4, 4))
    z = np.zeros(4)
    for b in range(B):
        for j in range(d):
            s[b, :, j], Jl[b, j], G[b, j] = step(S_prev[b, :, j], A[b, :, j], z, forget)
    return s, Jl, G


def sequential_head(P, Rh, s0, forget="sigmoid") -> np.ndarray:
    """P (B, T, 4, d), Rh (4, H, dh, dh) with H dh = d, s0 (B, 4, d) -> S (B, T, 4, d)."""
    P, Rh = _f64(P), _f64(Rh)
    B, T, _, d = P.shape
    S = np.zeros((B, T, 4, d))
    prev = np.zeros((B, 4, d)) if s0 is None else _f64(s0).copy()
    for t in range(T):
        prev, _, _ = _head_step_all(prev, P[:, t], Rh, forget)
        S[:, t] = prev
    return S


def head_jacobian(Jl, G, Rh):
    """Dense per-head Jacobian ds_t / ds_{t-1}: (B, H, 4 dh, 4 dh), state index
    e * dh + i for slot e of head feature i.  J = diag-lane part + G R routed
    into the h column: d s[e, i] / d h[k] += sum_g G[i][e, g] R[g, head, i, k]."""
    B, d = Jl.shape[:2]
    _, H, dh, _ = Rh.shape
    J = np.zeros((B, H, 4 * dh, 4 * dh))
    for hd in range(H):
        for i in range(dh):
            j = hd * dh + i
            for e in range(4):
                for e2 in range(4):
                    J[:, hd, e * dh + i, e2 * dh + i] += Jl[:, j, e, e2]
                for k in range(dh):
                    J[:, hd, e * dh + i, 3 * dh + k] += np.einsum("bg,g->b", G[:, j, e, :], Rh[:, hd, i, k])
    return J


def newton_head(P, Rh, s0, forget="sigmoid", max_iters=8, fixed=False, tol=1e-5, init="decoupled"):
    """Newton over time with dense per-head Jacobian blocks, the same update
    and stopping rule (max |F| / (1 + |s|) <= tol) as the diag oracle.  The
    initial guess is the decoupled trajectory (the cell with no recurrent
    input, which does not depend on the mixing) or, with init="zero", S = 0.
    Returns (S, stats)."""
    P, Rh = _f64(P), _f64(Rh)
    B, T, _, d = P.shape
    _, H, dh, _ = Rh.shape
    s0v = np.zeros((B, 4, d)) if s0 is None else _f64(s0)
    if init == "decoupled":
        S = sequential_btgd(P, np.zeros((4, d)), s0v, forget)
    elif init == "zero":
        S = np.zeros((B, T, 4, d))
    else:
        raise ValueError(f"unknown init {init!r}")
    hist = []
    conv = div = False
    it = 0

    def residual_and_jac(S):
        F = np.zeros_like(S)
        Js = []
        for t in range(T):
            prev = s0v if t == 0 else S[:, t - 1]
            f, Jl, G = _head_step_all(prev, P[:, t], Rh, forget)
            F[:, t] = S[:, t] - f
            Js.append(head_jacobian(Jl, G, Rh))
        return F, Js

    def to_heads(x):   # (B, 4, d) -> (B, H, 4 dh)
        return x.reshape(B, 4, H, dh).transpose(0, 2, 1, 3).reshape(B, H, 4 * dh)

    def from_heads(y):
        return y.reshape(B, H, 4, dh).transpose(0, 2, 1, 3).reshape(B, 4, d)

    F, Js = residual_and_jac(S)
    for it in range(1, max_iters + 1):
        delta = np.zeros((B, H, 4 * dh))
        for t in range(T):
            delta = (np.einsum("bhij,bhj->bhi", Js[t], delta) if t > 0 else 0.0) - to_heads(F[:, t])
            S[:, t] += from_heads(delta)
        F, Js = residual_and_jac(S)
        raw = float(np.max(np.abs(F)))
        scaled = float(np.max(np.abs(F) / (1.0 + np.abs(S))))
        hist.append((raw, scaled))
        if not np.isfinite(raw):
            div = True
            break
        if not fixed and scaled <= tol:
            conv = True
            break
    if not conv and hist and hist[-1][0] > 1.0:
        div = True
    return S, {"iters": it, "converged": conv, "diverged": div, "max_abs_F": [h[0] for h in hist]}


def backward_head(x, Wx, P, Rh, s0, S, dH, forget="sigmoid"):
    """Gradients of L = sum dH * h for head mixing at the trajectory S, by the
    reverse loop of the diag backward with the dense per-head Jacobian
    (head_jacobian) in place of the 4x4 one:
      lambda_t = e_h dH_t + J_{t+1}^T lambda_{t+1}
      dP_t = G_t^T lambda_t per feature (G = d s_t / d a_t, as step() gives it)
      dRh[g, head, i, k] = sum_{b,t} dP_t[g, (head, i)] h_{t-1}[(head, k)]
      db = sum dP, ds0 = J_0^T lambda_0, dx = dP W_x, dW_x = dP^T x.
    Returns dict dx, dWx, dRh (4, H, dh, dh), db (4, d), ds0 (B, 4, d), dP."""
    P, Rh, S, dH = _f64(P), _f64(Rh), _f64(S), _f64(dH)
    B, T, _, d = P.shape
    _, H, dh, _ = Rh.shape
    d_in = np.asarray(Wx).shape[1]
    s0v = np.zeros((B, 4, d)) if s0 is None else _f64(s0)

    def to_heads(v):     # (B, 4, d) -> (B, H, 4 dh), state index e * dh + i
        return v.reshape(B, 4, H, dh).transpose(0, 2, 1, 3).reshape(B, H, 4 * dh)

    def from_heads(y):
        return y.reshape(B, H, 4, dh).transpose(0, 2, 1, 3).reshape(B, 4, d)

    dP = np.zeros((B, T, 4, d))
    dRh = np.zeros_like(Rh)
    lam = np.zeros((B, 4, d))
    J_next = None
    for t in range(T - 1, -1, -1):
        prev = s0v if t == 0 else S[:, t - 1]
        _, Jl, G = _head_step_all(prev, P[:, t], Rh, forget)
        lam_t = np.zeros((B, 4, d))
        lam_t[:, 3, :] = dH[:, t]
        if J_next is not None:
            lam_t += from_heads(np.einsum("bhji,bhj->bhi", J_next, to_heads(lam)))
        dp = np.einsum("bjeg,bej->bgj", G, lam_t)                 # (B, 4, d)
        dP[:, t] = dp
        hp = prev[:, 3, :].reshape(B, H, dh)
        dRh += np.einsum("bghi,bhk->ghik", dp.reshape(B, 4, H, dh), hp)
        lam = lam_t
        J_next = head_jacobian(Jl, G, Rh)
    ds0 = from_heads(np.einsum("bhji,bhj->bhi", J_next, to_heads(lam)))
    dP2 = dP.reshape(B * T, 4 * d)
    x2 = _f64(x).reshape(B * T, d_in)
    return {"dx": (dP2 @ _f64(Wx)).reshape(B, T, d_in), "dWx": dP2.T @ x2, "dRh": dRh,
            "db": dP.sum(axis=(0, 1)), "ds0": ds0, "dP": dP}
