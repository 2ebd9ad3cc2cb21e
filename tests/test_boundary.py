"""C-ABI boundary checks that need no GPU: the library builds and loads, it
exports every function include/slstm.h declares, and host-side validation
rejects bad arguments before anything is enqueued (these calls never reach
the CUDA runtime)."""
import ctypes
import os
import re

import pytest

from nonlinear_rnn_pararnn_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")

FAKE = ctypes.c_void_p(0x10000)          # 16-byte aligned, never dereferenced
FAKE_MIS = ctypes.c_void_p(0x10004)      # misaligned
NULL = ctypes.c_void_p(0)


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([A-Za-z_]\w*)\s*\(", text, flags=re.M):
            if m.group(1) not in ("if", "while", "sizeof", "defined"):
                names.append(m.group(1))
    return names


def test_library_loads_and_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_functions()
    assert "slstm_newton_forward" in names and "scan_block4" in names
    for n in names:
        assert hasattr(lib, n), n
    # the binding covers exactly the declared set
    assert set(names) == set(_lib.SIGNATURES)


def test_status_strings():
    lib = _lib.load()
    assert lib.slstm_status_string(0) == b"SLSTM_OK"
    assert lib.slstm_status_string(1) == b"SLSTM_ERR_INVALID_ARG"
    assert lib.slstm_status_string(4) == b"SLSTM_ERR_TIMEOUT"
    assert lib.slstm_status_string(99) == b"SLSTM_UNKNOWN_STATUS"


def test_workspace_sizes():
    lib = _lib.load()
    small = lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD, 2, 64, 8, 8)
    big = lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD, 4, 65536, 2048, 2048)
    assert 0 < small < big
    assert big < 8 * 1024 ** 3
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_SCAN_BLOCK4, 2, 100, 0, 40) > 0
    bwd = lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_BACKWARD, 2, 64, 8, 8)
    assert bwd >= 2 * 64 * 4 * 8 * 4  # holds dP
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD, 0, 64, 8, 8) == 0
    assert lib.slstm_workspace_size(77, 2, 64, 8, 8) == 0
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD, 70000, 64, 8, 8) == 0


def _cfg(**kw):
    base = dict(max_iters=4, fixed_iters=0, tol=1e-5, forget=0, debug_fault=0, wait_limit_us=0, carry_mode=0,
                init=0, residual_mode=0, guess_sweeps=0)
    base.update(kw)
    return _lib.NewtonConfig(**base)


def test_checked_build_entry_points_in_the_normal_library():
    """The normal library exports the bounds-check calls too: checks off,
    nothing recorded, a null output rejected (no device access)."""
    lib = _lib.load()
    assert lib.slstm_check_enabled() == 0
    assert lib.slstm_check_status(None) == _lib.SLSTM_ERR_INVALID_ARG
    assert lib.slstm_check_site_file(1) == b"newton.cu"
    assert lib.slstm_check_site_file(0) is None and lib.slstm_check_site_file(99) is None


def test_newton_forward_rejects_bad_arguments():
    lib = _lib.load()
    E = _lib.SLSTM_ERR_INVALID_ARG
    ws = FAKE
    big = ctypes.c_size_t(1 << 40)

    def call(P=FAKE, R=FAKE, s0=NULL, S=FAKE, cfg=None, stats=FAKE, B=2, T=64, d=8, w=ws, wb=big):
        c = cfg if cfg is not None else _cfg()
        return lib.slstm_newton_forward(P, R, s0, S, ctypes.byref(c), stats, B, T, d, w, wb, NULL)

    assert call(B=0) == E
    assert call(T=0) == E
    assert call(d=-1) == E
    assert call(P=NULL) == E
    assert call(S=FAKE_MIS) == E
    assert call(s0=FAKE_MIS) == E
    assert call(stats=NULL) == E
    assert call(cfg=_cfg(max_iters=-1)) == E
    assert call(cfg=_cfg(max_iters=65537)) == E
    assert call(cfg=_cfg(forget=2)) == E
    assert call(cfg=_cfg(tol=float("nan"))) == E
    assert call(cfg=_cfg(carry_mode=3)) == E
    assert call(cfg=_cfg(carry_mode=-1)) == E
    assert call(cfg=_cfg(init=3)) == E
    assert call(cfg=_cfg(init=-1)) == E
    assert call(cfg=_cfg(residual_mode=2)) == E
    assert call(cfg=_cfg(guess_sweeps=-1)) == E
    assert call(cfg=_cfg(guess_sweeps=65)) == E
    assert call(cfg=_cfg(max_iters=0, init=1)) == E      # only the decoupled guess allows 0 iterations
    assert call(cfg=_cfg(n_events=-1)) == E
    assert call(cfg=_cfg(n_events=3)) == E               # timing events announced, array missing
    assert call(cfg=_cfg(history=2)) == E
    assert call(cfg=_cfg(debug_fault=4)) == E
    assert call(wb=ctypes.c_size_t(16)) == E          # workspace too small
    assert call(w=ctypes.c_void_p(0x10010)) == E      # workspace not 256-aligned
    assert lib.slstm_newton_forward(FAKE, FAKE, NULL, FAKE, None, FAKE, 2, 64, 8, ws, big, NULL) == E


def test_other_entry_points_reject_bad_arguments():
    lib = _lib.load()
    E = _lib.SLSTM_ERR_INVALID_ARG
    big = ctypes.c_size_t(1 << 40)
    assert lib.scan_block4(FAKE, FAKE, NULL, FAKE, 2, 100, 0, 0, FAKE, big, NULL) == E
    assert lib.scan_block4(FAKE, FAKE, NULL, FAKE, 2, 100, 40, 2, FAKE, big, NULL) == E   # unknown flag
    assert lib.scan_block4(FAKE, FAKE, NULL, FAKE, 2, 100, 40, 0, FAKE, big, NULL) == E   # y aliases A
    assert lib.slstm_sequential_step(FAKE, FAKE, NULL, FAKE, 2, 0, 8, 0, NULL) == E
    assert lib.slstm_sequential_step(FAKE, FAKE, NULL, FAKE, 2, 8, 8, 3, NULL) == E
    assert lib.slstm_preact_gemm(FAKE, FAKE, 7, FAKE, FAKE, 2, 8, 8, 8, FAKE, big, NULL) == E
    assert lib.slstm_preact_gemm(FAKE, FAKE, _lib.SLSTM_BF16, FAKE, FAKE, 2, 8, 6, 8, FAKE, big, NULL) == E
    assert lib.slstm_preact_gemm(FAKE_MIS, FAKE, 0, FAKE, FAKE, 2, 8, 8, 8, FAKE, big, NULL) == E
    args = [FAKE] * 13
    assert lib.slstm_newton_backward(args[0], args[1], 0, *args[2:12], 0, 2, 0, 8, 8, FAKE, big, NULL) == E
    assert lib.slstm_newton_backward(args[0], args[1], 5, *args[2:12], 0, 2, 8, 8, 8, FAKE, big, NULL) == E
    # decode: dtype, forget mode, sizes, 16-byte rows, alignment
    assert lib.slstm_decode_step(FAKE, FAKE, 7, FAKE, FAKE, NULL, FAKE, 0, 2, 8, 8, NULL) == E
    assert lib.slstm_decode_step(FAKE, FAKE, 0, FAKE, FAKE, NULL, FAKE, 3, 2, 8, 8, NULL) == E
    assert lib.slstm_decode_step(FAKE, FAKE, 0, FAKE, FAKE, NULL, FAKE, 0, 0, 8, 8, NULL) == E
    assert lib.slstm_decode_step(FAKE, FAKE, _lib.SLSTM_BF16, FAKE, FAKE, NULL, FAKE, 0, 2, 12, 8, NULL) == E
    assert lib.slstm_decode_step(FAKE, FAKE, 0, FAKE, FAKE, NULL, FAKE, 0, 2, 6, 8, NULL) == E
    assert lib.slstm_decode_step(FAKE_MIS, FAKE, 0, FAKE, FAKE, NULL, FAKE, 0, 2, 8, 8, NULL) == E
    assert lib.slstm_decode_step(FAKE, FAKE, 0, FAKE, FAKE, FAKE_MIS, FAKE, 0, 2, 8, 8, NULL) == E


def test_varlen_entry_points_reject_bad_arguments():
    lib = _lib.load()
    E = _lib.SLSTM_ERR_INVALID_ARG
    big = ctypes.c_size_t(1 << 40)
    cu = FAKE

    def fwd(P=FAKE, R=FAKE, s0=NULL, cu=cu, n=3, S=FAKE, cfg=None, stats=FAKE, total=64, d=8, wb=big):
        c = cfg if cfg is not None else _cfg()
        return lib.slstm_newton_forward_varlen(P, R, s0, cu, n, S, ctypes.byref(c), stats, total, d, FAKE, wb, NULL)

    assert fwd(cu=NULL) == E                          # offsets missing
    assert fwd(cu=ctypes.c_void_p(0x10002)) == E      # offsets not int32-aligned
    assert fwd(n=0) == E
    assert fwd(n=65, total=64) == E                   # more sequences than steps
    assert fwd(total=0) == E
    assert fwd(S=FAKE_MIS) == E
    assert fwd(cfg=_cfg(max_iters=-1)) == E
    assert fwd(wb=ctypes.c_size_t(64)) == E
    assert lib.slstm_newton_forward_varlen(FAKE, FAKE, NULL, cu, 3, FAKE, None, FAKE, 64, 8, FAKE, big, NULL) == E
    # (x, Wx, dtype, P, R, s0, cu, n_seq, S, dH, dx, dWx, dR, db, ds0, forget, total_T, d_in, d_h, ws, bytes, stream)

    def bwd(dtype=0, cu=cu, n=3, forget=0, total=64, d_in=8, d=8, ds0=NULL):
        return lib.slstm_newton_backward_varlen(FAKE, FAKE, dtype, FAKE, FAKE, NULL, cu, n, FAKE, FAKE, FAKE, FAKE,
                                                FAKE, FAKE, ds0, forget, total, d_in, d, FAKE, big, NULL)
    assert bwd(dtype=5) == E
    assert bwd(forget=3) == E
    assert bwd(cu=NULL) == E
    assert bwd(n=0) == E
    assert bwd(total=0) == E
    assert bwd(ds0=FAKE_MIS) == E
    ws_f = lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD_VARLEN, 3, 64, 0, 8)
    assert ws_f > lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD, 1, 64, 0, 8)
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_FORWARD_VARLEN, 65, 64, 0, 8) == 0
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_NEWTON_BACKWARD_VARLEN, 3, 64, 8, 8) > 0


def test_python_binding_validates_before_calling():
    import torch
    from nonlinear_rnn_pararnn_b200 import api
    P = torch.zeros(2, 8, 4, 8)
    with pytest.raises(ValueError):
        api.newton_forward(P, torch.zeros(4, 8))     # CPU tensors are refused


def test_block_entry_point_rejects_bad_arguments():
    lib = _lib.load()
    E = _lib.SLSTM_ERR_INVALID_ARG
    big = ctypes.c_size_t(1 << 40)
    # (x, norm1_w, Wx, bias, R, norm2_w, W_gu, W_down, y, S, cfg, stats, B, T, D, F, eps, ws, bytes, stream)

    def fwd(x=FAKE, y=ctypes.c_void_p(0x10000), S=ctypes.c_void_p(0x20000000), cfg=None, B=2, T=16, D=64, F=256,
            eps=1e-6, wb=big):
        c = cfg if cfg is not None else _cfg()
        return lib.slstm_block_forward(x, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, y, S, ctypes.byref(c), FAKE,
                                       B, T, D, F, eps, FAKE, wb, NULL)

    assert fwd(D=60) == E                       # d_model % 8
    assert fwd(F=250) == E                      # d_ff % 32
    assert fwd(B=0) == E and fwd(T=0) == E
    assert fwd(eps=-1.0) == E and fwd(eps=float("nan")) == E
    assert fwd(x=FAKE_MIS) == E
    assert fwd(cfg=_cfg(max_iters=-1)) == E
    assert fwd(wb=ctypes.c_size_t(64)) == E     # workspace too small
    assert fwd(S=ctypes.c_void_p(0x10000 + 256)) == E   # y and S overlap
    assert lib.slstm_block_workspace_size(2, 16, 60, 256) == 0
    assert lib.slstm_block_workspace_size(2, 16, 64, 250) == 0
    n = lib.slstm_block_workspace_size(2, 16, 64, 256)
    # at least the bf16 activations and the fp32 pre-activations
    assert n >= 2 * 16 * 64 * 2 + 2 * 16 * 4 * 64 * 4


def test_block_backward_entry_point_rejects_bad_arguments():
    lib = _lib.load()
    E = _lib.SLSTM_ERR_INVALID_ARG
    big = ctypes.c_size_t(1 << 40)

    def bwd(x=FAKE, forget=0, B=2, T=16, D=64, F=256, eps=1e-6, wb=big):
        return lib.slstm_block_backward(x, *([FAKE] * 17), forget, B, T, D, F, eps, FAKE, wb, NULL)

    assert bwd(forget=5) == E
    assert bwd(D=60) == E and bwd(F=100) == E and bwd(B=0) == E
    assert bwd(B=2, T=65535 * 128 + 1) == E           # more column-sum chunks than the grid's y axis
    assert bwd(eps=-1.0) == E
    assert bwd(x=FAKE_MIS) == E
    assert bwd(wb=ctypes.c_size_t(64)) == E
    assert lib.slstm_block_backward_workspace_size(2, 16, 64, 250) == 0
    assert lib.slstm_block_backward_workspace_size(2, 16, 64, 256) > lib.slstm_block_workspace_size(2, 16, 64, 256)


def test_interleave_gate_up_layout():
    """W_gu rows 64 k .. 64 k + 31 are W_gate rows 32 k .. 32 k + 31 and rows
    64 k + 32 .. 64 k + 63 the W_up rows of the same features."""
    import torch
    from nonlinear_rnn_pararnn_b200 import api
    F, D = 96, 5
    Wg = torch.arange(F * D, dtype=torch.float32).reshape(F, D)
    Wu = -1 - Wg
    W = api.interleave_gate_up(Wg, Wu)
    assert W.shape == (2 * F, D)
    for k in range(F // 32):
        assert torch.equal(W[64 * k:64 * k + 32], Wg[32 * k:32 * k + 32])
        assert torch.equal(W[64 * k + 32:64 * k + 64], Wu[32 * k:32 * k + 32])
    with pytest.raises(ValueError):
        api.interleave_gate_up(Wg[:40], Wu[:40])


def test_gemm_tile_shape_switch():
    """slstm_set_gemm_tiles takes the three settings, returns the previous one
    and refuses anything else without changing the setting (no GPU work)."""
    lib = _lib.load()
    prev = lib.slstm_set_gemm_tiles(_lib.SLSTM_GEMM_TILES_SINGLE)
    assert prev in (_lib.SLSTM_GEMM_TILES_AUTO, _lib.SLSTM_GEMM_TILES_PAIR, _lib.SLSTM_GEMM_TILES_SINGLE)
    assert lib.slstm_set_gemm_tiles(7) == -1
    assert lib.slstm_set_gemm_tiles(-1) == -1
    assert lib.slstm_set_gemm_tiles(_lib.SLSTM_GEMM_TILES_PAIR) == _lib.SLSTM_GEMM_TILES_SINGLE
    assert lib.slstm_set_gemm_tiles(_lib.SLSTM_GEMM_TILES_AUTO) == _lib.SLSTM_GEMM_TILES_PAIR
    assert api.set_gemm_tiles("single") == "auto"
    assert api.set_gemm_tiles("pair") == "single"
    assert api.set_gemm_tiles("auto") == "pair"
    with pytest.raises(ValueError):
        api.set_gemm_tiles("quad")
    lib.slstm_set_gemm_tiles(prev)
