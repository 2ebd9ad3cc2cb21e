"""Python binding of libslstm: torch tensors in, torch tensors out.

Each function checks shapes, dtypes and devices, allocates outputs and
workspace with torch (device memory is the one thing torch provides here),
and calls the C ABI on the current CUDA stream.  Every step of the method
runs in the library's CUDA kernels; nothing here computes.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import NewtonConfig, check, load

_FORGET = {"sigmoid": _lib.SLSTM_FORGET_SIGMOID, "exp": _lib.SLSTM_FORGET_EXP}
_DTYPE = {torch.float32: _lib.SLSTM_F32, torch.bfloat16: _lib.SLSTM_BF16}


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, shape, dtype=torch.float32):
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def forget_code(forget) -> int:
    return _FORGET[forget] if isinstance(forget, str) else int(forget)


def workspace_size(op: int, B: int, T: int, d_in: int, d_h: int) -> int:
    return int(load().slstm_workspace_size(op, B, T, d_in, d_h))


def workspace(op: int, B: int, T: int, d_in: int, d_h: int, device=None) -> torch.Tensor:
    n = workspace_size(op, B, T, d_in, d_h)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def preact_gemm(x: torch.Tensor, Wx: torch.Tensor, bias: torch.Tensor, P: torch.Tensor = None,
                ws: torch.Tensor = None) -> torch.Tensor:
    B, T, d_in = x.shape
    d_h = Wx.shape[0] // 4
    dt = x.dtype
    _need(x, "x", (B, T, d_in), dt)
    _need(Wx, "Wx", (4 * d_h, d_in), dt)
    _need(bias, "bias", (4, d_h))
    if P is None:
        P = torch.empty(B, T, 4, d_h, dtype=torch.float32, device=x.device)
    _need(P, "P", (B, T, 4, d_h))
    n = workspace_size(_lib.SLSTM_OP_PREACT_GEMM, B, T, d_in, d_h)
    if n and ws is None:
        ws = workspace(_lib.SLSTM_OP_PREACT_GEMM, B, T, d_in, d_h, x.device)
    check("slstm_preact_gemm", load().slstm_preact_gemm(_ptr(x), _ptr(Wx), _DTYPE[dt], _ptr(bias), _ptr(P),
                                                        B, T, d_in, d_h, _ptr(ws), 0 if ws is None else ws.numel(),
                                                        _stream()))
    return P


_INIT = {"decoupled": _lib.SLSTM_INIT_DECOUPLED, "zero": _lib.SLSTM_INIT_ZERO, "given": _lib.SLSTM_INIT_GIVEN}
_RESIDUAL = {"scaled": _lib.SLSTM_RESIDUAL_SCALED, "raw": _lib.SLSTM_RESIDUAL_RAW}


# refinement sweeps of the decoupled guess used when the caller names none
DEFAULT_GUESS_SWEEPS = 2


def set_gemm_tiles(tiles: str) -> str:
    """Tile shape of the tensor-core GEMMs: "auto" (the default: SM pairs for
    the gradient GEMMs, whose work items span K >= 4096, single SMs for the
    others), "pair"
    (256 x 256 tiles on a pair of SMs) or "single" (128 x 256 per SM); returns
    the previous one.  The shapes agree to fp32 rounding (the input projection
    bit for bit)."""
    codes = {"auto": _lib.SLSTM_GEMM_TILES_AUTO, "pair": _lib.SLSTM_GEMM_TILES_PAIR,
             "single": _lib.SLSTM_GEMM_TILES_SINGLE}
    if tiles not in codes:
        raise ValueError(f"tiles must be 'auto', 'pair' or 'single', got {tiles!r}")
    prev = load().slstm_set_gemm_tiles(codes[tiles])
    return {v: k for k, v in codes.items()}[prev]


def newton_config(max_iters: int, fixed: bool, tol: float, forget, debug_fault: int = 0, wait_limit_us: int = 0,
                  carry_mode: int = 0, init="decoupled", residual_mode="scaled",
                  guess_sweeps: int = DEFAULT_GUESS_SWEEPS, events=None, exact_history: bool = False,
                  loop_from: int = 0) -> NewtonConfig:
    """The C ABI's slstm_newton_config.  init: "decoupled" (default; with
    guess_sweeps refinement sweeps), "zero" or "given" (S holds the guess on
    entry); residual_mode: "scaled" or "raw"; events: optional list of
    torch.cuda.Event (timing enabled) recorded before each launch of work and
    after the last (see slstm.h); exact_history: every iteration records its
    exact residual (else an iteration that fails the test may record a lower
    bound); loop_from: in tolerance mode, the iterations from this one on run
    in one launch that loops on the device (0: the library default, negative:
    never)."""
    cfg = NewtonConfig(int(max_iters), 1 if fixed else 0, float(tol), forget_code(forget), int(debug_fault),
                       int(wait_limit_us), int(carry_mode), _INIT[init] if isinstance(init, str) else int(init),
                       _RESIDUAL[residual_mode] if isinstance(residual_mode, str) else int(residual_mode),
                       int(guess_sweeps), _lib.SLSTM_HISTORY_EXACT if exact_history else _lib.SLSTM_HISTORY_BOUND,
                       0, None, int(loop_from))
    if events:
        handles = []
        for ev in events:
            if ev.cuda_event == 0:
                ev.record()   # torch creates the CUDA event on its first record
            handles.append(ev.cuda_event)
        arr = (ctypes.c_void_p * len(handles))(*handles)
        cfg.n_events = len(handles)
        cfg.events = ctypes.cast(arr, ctypes.c_void_p)
        cfg._keep = arr   # the array lives as long as the config
    return cfg


def new_stats(device=None) -> torch.Tensor:
    return torch.zeros(_lib.STATS_BYTES, dtype=torch.uint8, device=device or "cuda")


def read_stats(stats: torch.Tensor) -> dict:
    """Copy a device stats record to the host and decode it."""
    raw = stats.detach().to("cpu")
    ints = raw[:16].view(torch.int32).tolist()
    fl = raw[16:].view(torch.float32)
    it = ints[0]
    m = _lib.SLSTM_STATS_HISTORY
    ks = list(range(max(0, it - m), it))     # the iterations the ring still holds
    raw_h, sc_h = fl[:m].tolist(), fl[m:2 * m].tolist()
    return {"iters": it, "converged": bool(ints[1]), "diverged": bool(ints[2]), "error": ints[3],
            "history_first_iter": ks[0] if ks else 0,
            "max_abs_F": [raw_h[k % m] for k in ks], "max_scaled_F": [sc_h[k % m] for k in ks],
            "init_max_abs_F": float(fl[2 * m]), "init_max_scaled_F": float(fl[2 * m + 1])}


def newton_forward(P: torch.Tensor, R: torch.Tensor, s0: torch.Tensor = None, *, forget="sigmoid",
                   max_iters: int = 8, fixed: bool = False, tol: float = 1e-5, S: torch.Tensor = None,
                   stats: torch.Tensor = None, ws: torch.Tensor = None, debug_fault: int = 0,
                   wait_limit_us: int = 0, carry_mode: int = 0, init="decoupled", residual_mode="scaled",
                   guess_sweeps: int = DEFAULT_GUESS_SWEEPS, events=None, exact_history: bool = False,
                   loop_from: int = 0):
    """Newton solve; returns (S, stats) with stats a device record (see read_stats).
    With init="given", S must be passed and holds the initial guess.  events:
    optional torch.cuda.Event list bracketing the launches; exact_history,
    loop_from: see newton_config."""
    B, T, four, d_h = P.shape
    _need(P, "P", (B, T, 4, d_h))
    _need(R, "R", (4, d_h))
    if s0 is not None:
        _need(s0, "s0", (B, 4, d_h))
    if S is None:
        if init == "given":
            raise ValueError("init='given' needs S holding the initial guess")
        S = torch.empty_like(P)
    _need(S, "S", (B, T, 4, d_h))
    if stats is None:
        stats = new_stats(P.device)
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_NEWTON_FORWARD, B, T, 0, d_h, P.device)
    cfg = newton_config(max_iters, fixed, tol, forget, debug_fault, wait_limit_us, carry_mode, init, residual_mode,
                        guess_sweeps, events, exact_history, loop_from)
    check("slstm_newton_forward", load().slstm_newton_forward(_ptr(P), _ptr(R), _ptr(s0), _ptr(S),
                                                              ctypes.byref(cfg), _ptr(stats), B, T, d_h,
                                                              _ptr(ws), ws.numel(), _stream()))
    return S, stats


def scan_block4(A: torch.Tensor, b: torch.Tensor, y0: torch.Tensor = None, reverse: bool = False,
                y: torch.Tensor = None, ws: torch.Tensor = None) -> torch.Tensor:
    B, T, four, four2, d = A.shape
    _need(A, "A", (B, T, 4, 4, d))
    _need(b, "b", (B, T, 4, d))
    if y0 is not None:
        _need(y0, "y0", (B, 4, d))
    if y is None:
        y = torch.empty_like(b)
    _need(y, "y", (B, T, 4, d))
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_SCAN_BLOCK4, B, T, 0, d, A.device)
    flags = _lib.SLSTM_SCAN_REVERSE_T if reverse else 0
    check("scan_block4", load().scan_block4(_ptr(A), _ptr(b), _ptr(y0), _ptr(y), B, T, d, flags, _ptr(ws),
                                            ws.numel(), _stream()))
    return y


def sequential_step(P: torch.Tensor, R: torch.Tensor, s0: torch.Tensor = None, *, forget="sigmoid",
                    S: torch.Tensor = None) -> torch.Tensor:
    B, T, four, d_h = P.shape
    _need(P, "P", (B, T, 4, d_h))
    _need(R, "R", (4, d_h))
    if s0 is not None:
        _need(s0, "s0", (B, 4, d_h))
    if S is None:
        S = torch.empty_like(P)
    _need(S, "S", (B, T, 4, d_h))
    check("slstm_sequential_step", load().slstm_sequential_step(_ptr(P), _ptr(R), _ptr(s0), _ptr(S), B, T, d_h,
                                                                forget_code(forget), _stream()))
    return S


def decode_step(x: torch.Tensor, Wx: torch.Tensor, bias: torch.Tensor, R: torch.Tensor, s_prev: torch.Tensor = None,
                *, forget="sigmoid", out: torch.Tensor = None) -> torch.Tensor:
    """One decode step: x (B, d_in) and Wx (4 d_h, d_in) of one dtype, bias and R (4, d_h), s_prev
    (B, 4, d_h) or None (zero state); returns s_next (B, 4, d_h), written into `out` when given
    (`out` may be `s_prev`)."""
    B, d_in = x.shape
    d_h = Wx.shape[0] // 4
    dt = x.dtype
    _need(x, "x", (B, d_in), dt)
    _need(Wx, "Wx", (4 * d_h, d_in), dt)
    _need(bias, "bias", (4, d_h))
    _need(R, "R", (4, d_h))
    if s_prev is not None:
        _need(s_prev, "s_prev", (B, 4, d_h))
    if out is None:
        out = torch.empty(B, 4, d_h, device=x.device, dtype=torch.float32)
    _need(out, "out", (B, 4, d_h))
    check("slstm_decode_step", load().slstm_decode_step(_ptr(x), _ptr(Wx), _DTYPE[dt], _ptr(bias), _ptr(R),
                                                        _ptr(s_prev), _ptr(out), forget_code(forget), B, d_in, d_h,
                                                        _stream()))
    return out


def decode(xs: torch.Tensor, Wx: torch.Tensor, bias: torch.Tensor, R: torch.Tensor, s0: torch.Tensor = None, *,
           forget="sigmoid", S: torch.Tensor = None) -> torch.Tensor:
    """T decode steps over xs (T, B, d_in) from s0 (B, 4, d_h) or zero; returns S (T, B, 4, d_h), the
    state after every step.  One launch per step on the current stream (capturable in a CUDA graph)."""
    T, B, d_in = xs.shape
    d_h = Wx.shape[0] // 4
    if S is None:
        S = torch.empty(T, B, 4, d_h, device=xs.device, dtype=torch.float32)
    _need(S, "S", (T, B, 4, d_h))
    prev = s0
    for t in range(T):
        decode_step(xs[t], Wx, bias, R, prev, forget=forget, out=S[t])
        prev = S[t]
    return S


def newton_backward(x, Wx, P, R, s0, S, dH, *, forget="sigmoid", out: dict = None, ws: torch.Tensor = None):
    """Gradients of sum(dH * h); returns dict dx, dWx, dR, db, ds0."""
    B, T, d_in = x.shape
    d_h = Wx.shape[0] // 4
    dt = x.dtype
    _need(x, "x", (B, T, d_in), dt)
    _need(Wx, "Wx", (4 * d_h, d_in), dt)
    _need(P, "P", (B, T, 4, d_h))
    _need(R, "R", (4, d_h))
    if s0 is not None:
        _need(s0, "s0", (B, 4, d_h))
    _need(S, "S", (B, T, 4, d_h))
    _need(dH, "dH", (B, T, d_h))
    dev = x.device
    if out is None:
        out = {"dx": torch.empty(B, T, d_in, device=dev), "dWx": torch.empty(4 * d_h, d_in, device=dev),
               "dR": torch.empty(4, d_h, device=dev), "db": torch.empty(4, d_h, device=dev),
               "ds0": torch.empty(B, 4, d_h, device=dev)}
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_NEWTON_BACKWARD, B, T, d_in, d_h, dev)
    check("slstm_newton_backward", load().slstm_newton_backward(
        _ptr(x), _ptr(Wx), _DTYPE[dt], _ptr(P), _ptr(R), _ptr(s0), _ptr(S), _ptr(dH), _ptr(out["dx"]),
        _ptr(out["dWx"]), _ptr(out["dR"]), _ptr(out["db"]), _ptr(out.get("ds0")), forget_code(forget), B, T,
        d_in, d_h, _ptr(ws), ws.numel(), _stream()))
    return out


# ---------------------------------------------------------------------------
# packed ragged sequences (cu_seqlens)
# ---------------------------------------------------------------------------
def _need_cu(cu: torch.Tensor, n_seq: int):
    if cu.device.type != "cuda" or cu.dtype != torch.int32 or not cu.is_contiguous() or cu.dim() != 1 \
            or cu.numel() != n_seq + 1:
        raise ValueError(f"cu_seqlens must be a contiguous int32 CUDA tensor of {n_seq + 1} offsets")


def newton_forward_varlen(P: torch.Tensor, R: torch.Tensor, s0: torch.Tensor, cu_seqlens: torch.Tensor, *,
                          forget="sigmoid", max_iters: int = 8, fixed: bool = False, tol: float = 1e-5,
                          S: torch.Tensor = None, stats: torch.Tensor = None, ws: torch.Tensor = None,
                          carry_mode: int = 0, init="decoupled", residual_mode="scaled",
                          guess_sweeps: int = DEFAULT_GUESS_SWEEPS, events=None, exact_history: bool = False,
                          loop_from: int = 0):
    """Newton solve of packed sequences: P (total_T, 4, d_h), s0 (n_seq, 4, d_h) or None,
    cu_seqlens int32 (n_seq + 1,) exclusive-prefix offsets; returns (S, stats).
    events, exact_history, loop_from: as newton_forward."""
    total_T, four, d_h = P.shape
    n_seq = cu_seqlens.numel() - 1
    _need(P, "P", (total_T, 4, d_h))
    _need(R, "R", (4, d_h))
    _need_cu(cu_seqlens, n_seq)
    if s0 is not None:
        _need(s0, "s0", (n_seq, 4, d_h))
    if S is None:
        S = torch.empty_like(P)
    _need(S, "S", (total_T, 4, d_h))
    if stats is None:
        stats = new_stats(P.device)
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_NEWTON_FORWARD_VARLEN, n_seq, total_T, 0, d_h, P.device)
    cfg = newton_config(max_iters, fixed, tol, forget, 0, 0, carry_mode, init, residual_mode, guess_sweeps, events,
                        exact_history, loop_from)
    check("slstm_newton_forward_varlen", load().slstm_newton_forward_varlen(
        _ptr(P), _ptr(R), _ptr(s0), _ptr(cu_seqlens), n_seq, _ptr(S), ctypes.byref(cfg), _ptr(stats), total_T, d_h,
        _ptr(ws), ws.numel(), _stream()))
    return S, stats


def newton_backward_varlen(x, Wx, P, R, s0, cu_seqlens, S, dH, *, forget="sigmoid", out: dict = None,
                           ws: torch.Tensor = None):
    """Gradients of sum(dH * h) over packed sequences: x (total_T, d_in), P and S (total_T, 4, d_h),
    dH (total_T, d_h); returns dict dx, dWx, dR, db, ds0 (n_seq, 4, d_h)."""
    total_T, d_in = x.shape
    d_h = Wx.shape[0] // 4
    n_seq = cu_seqlens.numel() - 1
    dt = x.dtype
    _need(x, "x", (total_T, d_in), dt)
    _need(Wx, "Wx", (4 * d_h, d_in), dt)
    _need(P, "P", (total_T, 4, d_h))
    _need(R, "R", (4, d_h))
    _need_cu(cu_seqlens, n_seq)
    if s0 is not None:
        _need(s0, "s0", (n_seq, 4, d_h))
    _need(S, "S", (total_T, 4, d_h))
    _need(dH, "dH", (total_T, d_h))
    dev = x.device
    if out is None:
        out = {"dx": torch.empty(total_T, d_in, device=dev), "dWx": torch.empty(4 * d_h, d_in, device=dev),
               "dR": torch.empty(4, d_h, device=dev), "db": torch.empty(4, d_h, device=dev),
               "ds0": torch.empty(n_seq, 4, d_h, device=dev)}
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_NEWTON_BACKWARD_VARLEN, n_seq, total_T, d_in, d_h, dev)
    check("slstm_newton_backward_varlen", load().slstm_newton_backward_varlen(
        _ptr(x), _ptr(Wx), _DTYPE[dt], _ptr(P), _ptr(R), _ptr(s0), _ptr(cu_seqlens), n_seq, _ptr(S), _ptr(dH),
        _ptr(out["dx"]), _ptr(out["dWx"]), _ptr(out["dR"]), _ptr(out["db"]), _ptr(out.get("ds0")),
        forget_code(forget), total_T, d_in, d_h, _ptr(ws), ws.numel(), _stream()))
    return out


# ---------------------------------------------------------------------------
# the trunk layer (RMSNorm -> cell -> residual -> RMSNorm -> SwiGLU -> residual)
# ---------------------------------------------------------------------------
def interleave_gate_up(W_gate: torch.Tensor, W_up: torch.Tensor) -> torch.Tensor:
    """(d_ff, d_model) W_gate and W_up -> the (2 d_ff, d_model) W_gu of
    block_forward: blocks of 32 gate rows followed by the 32 up rows of the
    same hidden features.  A one-time weight layout change (d_ff % 32 == 0)."""
    F, D = W_gate.shape
    if tuple(W_up.shape) != (F, D) or F % 32:
        raise ValueError("W_gate and W_up must both be (d_ff, d_model) with d_ff % 32 == 0")
    return torch.stack([W_gate.reshape(F // 32, 32, D), W_up.reshape(F // 32, 32, D)], dim=1).reshape(2 * F, D)


def block_workspace(B: int, T: int, d_model: int, d_ff: int, device=None) -> torch.Tensor:
    n = int(load().slstm_block_workspace_size(B, T, d_model, d_ff))
    if n == 0:
        raise ValueError("unsupported trunk-layer sizes (d_model % 8, d_ff % 32)")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def block_forward(x, norm1_w, Wx, bias, R, norm2_w, W_gu, W_down, *, forget="sigmoid", max_iters: int = 8,
                  fixed: bool = False, tol: float = 1e-5, eps: float = 1e-6, y: torch.Tensor = None,
                  S: torch.Tensor = None, stats: torch.Tensor = None, ws: torch.Tensor = None, carry_mode: int = 0,
                  init="decoupled", residual_mode="scaled", guess_sweeps: int = DEFAULT_GUESS_SWEEPS):
    """The trunk layer's forward; returns (y, S, stats).  x (B, T, d_model)
    fp32; Wx, W_gu (interleave_gate_up), W_down bf16."""
    B, T, D = x.shape
    F = W_down.shape[1]
    _need(x, "x", (B, T, D))
    _need(norm1_w, "norm1_w", (D,))
    _need(norm2_w, "norm2_w", (D,))
    _need(Wx, "Wx", (4 * D, D), torch.bfloat16)
    _need(bias, "bias", (4, D))
    _need(R, "R", (4, D))
    _need(W_gu, "W_gu", (2 * F, D), torch.bfloat16)
    _need(W_down, "W_down", (D, F), torch.bfloat16)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", (B, T, D))
    if S is None:
        S = torch.empty(B, T, 4, D, dtype=torch.float32, device=x.device)
    _need(S, "S", (B, T, 4, D))
    if stats is None:
        stats = new_stats(x.device)
    if ws is None:
        ws = block_workspace(B, T, D, F, x.device)
    cfg = newton_config(max_iters, fixed, tol, forget, 0, 0, carry_mode, init, residual_mode, guess_sweeps)
    check("slstm_block_forward", load().slstm_block_forward(
        _ptr(x), _ptr(norm1_w), _ptr(Wx), _ptr(bias), _ptr(R), _ptr(norm2_w), _ptr(W_gu), _ptr(W_down), _ptr(y),
        _ptr(S), ctypes.byref(cfg), _ptr(stats), B, T, D, F, float(eps), _ptr(ws), ws.numel(), _stream()))
    return y, S, stats


def block_backward(x, norm1_w, Wx, bias, R, norm2_w, W_gu, W_down, S, dY, *, forget="sigmoid", eps: float = 1e-6,
                   out: dict = None, ws: torch.Tensor = None) -> dict:
    """Gradients of sum(dY * y) of the trunk layer at x, given the forward's S;
    returns dict dx, dnorm1_w, dWx, dbias, dR, dnorm2_w, dW_gu (interleaved
    like W_gu), dW_down."""
    B, T, D = x.shape
    F = W_down.shape[1]
    _need(x, "x", (B, T, D))
    _need(norm1_w, "norm1_w", (D,))
    _need(norm2_w, "norm2_w", (D,))
    _need(Wx, "Wx", (4 * D, D), torch.bfloat16)
    _need(bias, "bias", (4, D))
    _need(R, "R", (4, D))
    _need(W_gu, "W_gu", (2 * F, D), torch.bfloat16)
    _need(W_down, "W_down", (D, F), torch.bfloat16)
    _need(S, "S", (B, T, 4, D))
    _need(dY, "dY", (B, T, D))
    dev = x.device
    if out is None:
        out = {"dx": torch.empty(B, T, D, device=dev), "dnorm1_w": torch.empty(D, device=dev),
               "dWx": torch.empty(4 * D, D, device=dev), "dbias": torch.empty(4, D, device=dev),
               "dR": torch.empty(4, D, device=dev), "dnorm2_w": torch.empty(D, device=dev),
               "dW_gu": torch.empty(2 * F, D, device=dev), "dW_down": torch.empty(D, F, device=dev)}
    if ws is None:
        n = int(load().slstm_block_backward_workspace_size(B, T, D, F))
        if n == 0:
            raise ValueError("unsupported trunk-layer sizes (d_model % 8, d_ff % 32)")
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
    names = ("dx", "dnorm1_w", "dWx", "dbias", "dR", "dnorm2_w", "dW_gu", "dW_down")
    check("slstm_block_backward", load().slstm_block_backward(
        _ptr(x), _ptr(norm1_w), _ptr(Wx), _ptr(bias), _ptr(R), _ptr(norm2_w), _ptr(W_gu), _ptr(W_down), _ptr(S),
        _ptr(dY), *[_ptr(out[k]) for k in names], forget_code(forget), B, T, D, F, float(eps), _ptr(ws), ws.numel(),
        _stream()))
    return out


# ---------------------------------------------------------------------------
# head mixing: block-diagonal R (4, n_heads, d_head, d_head)
# ---------------------------------------------------------------------------
def _head_dims(R_head: torch.Tensor, d_h: int):
    if R_head.dim() != 4 or R_head.shape[0] != 4 or R_head.shape[2] != R_head.shape[3]:
        raise ValueError(f"R_head must be (4, n_heads, d_head, d_head), got {tuple(R_head.shape)}")
    H, dh = R_head.shape[1], R_head.shape[2]
    if H * dh != d_h:
        raise ValueError(f"n_heads * d_head = {H * dh} != d_h = {d_h}")
    _need(R_head, "R_head", (4, H, dh, dh))
    return H, dh


def sequential_step_head(P: torch.Tensor, R_head: torch.Tensor, s0: torch.Tensor = None, *, forget="sigmoid",
                         S: torch.Tensor = None) -> torch.Tensor:
    B, T, four, d_h = P.shape
    _need(P, "P", (B, T, 4, d_h))
    H, dh = _head_dims(R_head, d_h)
    if s0 is not None:
        _need(s0, "s0", (B, 4, d_h))
    if S is None:
        S = torch.empty_like(P)
    _need(S, "S", (B, T, 4, d_h))
    check("slstm_sequential_step_head", load().slstm_sequential_step_head(
        _ptr(P), _ptr(R_head), _ptr(s0), _ptr(S), B, T, d_h, dh, forget_code(forget), _stream()))
    return S


def newton_forward_head(P: torch.Tensor, R_head: torch.Tensor, s0: torch.Tensor = None, *, forget="sigmoid",
                        max_iters: int = 8, fixed: bool = False, tol: float = 1e-5, S: torch.Tensor = None,
                        stats: torch.Tensor = None, ws: torch.Tensor = None, init="decoupled", residual_mode="scaled"):
    """Newton solve with head mixing; returns (S, stats)."""
    B, T, four, d_h = P.shape
    _need(P, "P", (B, T, 4, d_h))
    H, dh = _head_dims(R_head, d_h)
    if s0 is not None:
        _need(s0, "s0", (B, 4, d_h))
    if S is None:
        if init == "given":
            raise ValueError("init='given' needs S holding the initial guess")
        S = torch.empty_like(P)
    _need(S, "S", (B, T, 4, d_h))
    if stats is None:
        stats = new_stats(P.device)
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_NEWTON_FORWARD, B, T, 0, d_h, P.device)
    cfg = newton_config(max_iters, fixed, tol, forget, 0, 0, 0, init, residual_mode, 0)
    check("slstm_newton_forward_head", load().slstm_newton_forward_head(
        _ptr(P), _ptr(R_head), _ptr(s0), _ptr(S), ctypes.byref(cfg), _ptr(stats), B, T, d_h, dh, _ptr(ws),
        ws.numel(), _stream()))
    return S, stats


def newton_backward_head(x, Wx, P, R_head, s0, S, dH, *, forget="sigmoid", out: dict = None,
                         ws: torch.Tensor = None):
    """Gradients of sum(dH * h) with head mixing; returns dict dx, dWx, dR_head, db, ds0."""
    B, T, d_in = x.shape
    d_h = Wx.shape[0] // 4
    dt = x.dtype
    _need(x, "x", (B, T, d_in), dt)
    _need(Wx, "Wx", (4 * d_h, d_in), dt)
    _need(P, "P", (B, T, 4, d_h))
    H, dh = _head_dims(R_head, d_h)
    if s0 is not None:
        _need(s0, "s0", (B, 4, d_h))
    _need(S, "S", (B, T, 4, d_h))
    _need(dH, "dH", (B, T, d_h))
    dev = x.device
    if out is None:
        out = {"dx": torch.empty(B, T, d_in, device=dev), "dWx": torch.empty(4 * d_h, d_in, device=dev),
               "dR_head": torch.empty(4, H, dh, dh, device=dev), "db": torch.empty(4, d_h, device=dev),
               "ds0": torch.empty(B, 4, d_h, device=dev)}
    if ws is None:
        ws = workspace(_lib.SLSTM_OP_NEWTON_BACKWARD_HEAD, B, T, d_in, d_h, dev)
    check("slstm_newton_backward_head", load().slstm_newton_backward_head(
        _ptr(x), _ptr(Wx), _DTYPE[dt], _ptr(P), _ptr(R_head), _ptr(s0), _ptr(S), _ptr(dH), _ptr(out["dx"]),
        _ptr(out["dWx"]), _ptr(out["dR_head"]), _ptr(out["db"]), _ptr(out.get("ds0")), forget_code(forget), B, T,
        d_in, d_h, dh, _ptr(ws), ws.numel(), _stream()))
    return out
