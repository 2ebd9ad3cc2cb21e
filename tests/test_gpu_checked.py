"""The bounds-checked build (libslstm_checked.so, the kernels compiled with
SLSTM_CHECKED): every guarded global access tests its index against its
buffer's extent, skips and records it when outside.  These tests run the
hot path's calls through that build on small and ragged shapes (T not a
multiple of the tiles, d_h not a multiple of 4 so that the cp.async paths
run, B = 1, packed sequences with an empty one) and expect no violation;
one more makes a check fail on purpose (a boundary store checked against an
extent one short, debug_fault = 2) and expects exactly that report.
"""
import ctypes

import pytest
import torch

from nonlinear_rnn_pararnn_b200 import _lib, api
from nonlinear_rnn_pararnn_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _status(lib):
    out = (ctypes.c_longlong * 4)()
    assert lib.slstm_check_status(out) == _lib.SLSTM_OK
    return list(out)


def _describe(lib, st):
    f = lib.slstm_check_site_file(int(st[1] // 100000))
    return f"{st[0]} violations, first at {f and f.decode()}:{st[1] % 100000} index {st[2]} extent {st[3]}"


def _dense_case(B, T, d_in, d, dtype, forget, seed):
    w = Workload("c", B, T, d_in, d, dtype, forget, 0.5, seed, 1e-5, 16)
    inp = make_inputs(w)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    g = torch.Generator().manual_seed(seed)
    dev["s0"] = torch.stack([torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) + 0.5,
                             torch.randn(B, d, generator=g), torch.rand(B, d, generator=g) - 0.5], dim=1).cuda()
    return w, dev


def test_normal_build_has_no_checks():
    lib = _lib.load()
    assert lib.slstm_check_enabled() == 0
    assert _status(lib) == [0, 0, 0, 0]


@pytest.mark.parametrize("B,T,d_in,d,dtype,forget", [
    (2, 64, 8, 8, "f32", "sigmoid"),       # one tile per group
    (1, 67, 12, 10, "f32", "exp"),          # ragged T and d_h % 4 != 0: cp.async paths
    (3, 300, 24, 40, "bf16", "sigmoid"),    # TMA paths, tensor-core GEMMs, several chunks
    (1, 1000, 16, 33, "f32", "sigmoid"),    # B = 1, ragged d
])
def test_checked_build_runs_clean(B, T, d_in, d, dtype, forget, cuda_device):
    with _lib.checked_library() as lib:
        assert lib.slstm_check_enabled() == 1
        assert lib.slstm_check_clear() == _lib.SLSTM_OK
        w, dev = _dense_case(B, T, d_in, d, dtype, forget, 5)
        P = api.preact_gemm(dev["x"], dev["Wx"], dev["bias"])
        for carry_mode in (1, 2):
            S, st = api.newton_forward(P, dev["R"], dev["s0"], forget=forget, max_iters=16, tol=1e-5,
                                       carry_mode=carry_mode)
            S3, _ = api.newton_forward(P, dev["R"], dev["s0"], forget=forget, max_iters=3, fixed=True,
                                       carry_mode=carry_mode, guess_sweeps=5)
        S0, _ = api.newton_forward(P, dev["R"], dev["s0"], forget=forget, max_iters=4, fixed=True, init="zero")
        Sg, _ = api.newton_forward(P, dev["R"], dev["s0"], forget=forget, max_iters=1, fixed=True, init="given",
                                   S=S.clone())
        api.sequential_step(P, dev["R"], dev["s0"], forget=forget)
        api.newton_backward(dev["x"], dev["Wx"], P, dev["R"], dev["s0"], S, dev["dH"], forget=forget)
        A = (torch.rand(B, T, 4, 4, d) * 0.6 - 0.3).cuda()
        bb = torch.randn(B, T, 4, d).cuda()
        for reverse in (False, True):
            api.scan_block4(A, bb, dev["s0"], reverse=reverse)
        api.decode(dev["x"][:, :3].transpose(0, 1).contiguous(), dev["Wx"], dev["bias"], dev["R"], dev["s0"],
                   forget=forget)
        st = _status(lib)
        assert st[0] == 0, _describe(lib, st)


def test_checked_build_runs_clean_packed(cuda_device):
    with _lib.checked_library() as lib:
        assert lib.slstm_check_clear() == _lib.SLSTM_OK
        lengths = [5, 0, 130, 1, 64, 77]
        total = sum(lengths)
        w, dev = _dense_case(1, total, 12, 36, "f32", "sigmoid", 9)
        cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0)), dtype=torch.int32).cuda()
        s0 = torch.randn(len(lengths), 4, 36).cuda()
        s0[:, 1] = s0[:, 1].abs() + 0.5
        P = api.preact_gemm(dev["x"], dev["Wx"], dev["bias"])[0]
        for carry_mode in (1, 2):
            S, _ = api.newton_forward_varlen(P, dev["R"], s0, cu, max_iters=16, tol=1e-5, carry_mode=carry_mode)
        api.newton_backward_varlen(dev["x"][0], dev["Wx"], P, dev["R"], s0, cu, S, dev["dH"][0])
        st = _status(lib)
        assert st[0] == 0, _describe(lib, st)


@pytest.mark.parametrize("B,T,d,dh", [(2, 70, 36, 12), (1, 33, 64, 32), (3, 5, 8, 1)])
def test_checked_build_runs_clean_head(B, T, d, dh, cuda_device):
    with _lib.checked_library() as lib:
        assert lib.slstm_check_clear() == _lib.SLSTM_OK
        w, dev = _dense_case(B, T, 16, d, "f32", "sigmoid", 11)
        g = torch.Generator().manual_seed(12)
        Rh = ((torch.rand(4, d // dh, dh, dh, generator=g) * 2 - 1) * (0.5 / dh ** 0.5)).cuda()
        P = api.preact_gemm(dev["x"], dev["Wx"], dev["bias"])
        api.sequential_step_head(P, Rh, dev["s0"])
        S, _ = api.newton_forward_head(P, Rh, dev["s0"], max_iters=16, tol=1e-5)
        api.newton_forward_head(P, Rh, None, max_iters=3, fixed=True, init="zero")
        api.newton_backward_head(dev["x"], dev["Wx"], P, Rh, dev["s0"], S, dev["dH"])
        st = _status(lib)
        assert st[0] == 0, _describe(lib, st)


@pytest.mark.parametrize("B,T,D,F", [(2, 40, 64, 256), (1, 33, 96, 384)])
def test_checked_build_runs_clean_block(B, T, D, F, cuda_device):
    with _lib.checked_library() as lib:
        assert lib.slstm_check_clear() == _lib.SLSTM_OK
        g = torch.Generator().manual_seed(21)
        x = torch.randn(B, T, D, generator=g).cuda()
        w1 = (torch.rand(D, generator=g) + 0.5).cuda()
        w2 = (torch.rand(D, generator=g) + 0.5).cuda()
        Wx = (torch.randn(4 * D, D, generator=g) * D ** -0.5).to(torch.bfloat16).cuda()
        bias = torch.zeros(4, D).cuda()
        R = ((torch.rand(4, D, generator=g) * 2 - 1) * 0.5).cuda()
        Wg = (torch.randn(F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
        Wu = (torch.randn(F, D, generator=g) * D ** -0.5).to(torch.bfloat16)
        W_gu = api.interleave_gate_up(Wg, Wu).contiguous().cuda()
        Wd = (torch.randn(D, F, generator=g) * F ** -0.5).to(torch.bfloat16).cuda()
        y, S, _ = api.block_forward(x, w1, Wx, bias, R, w2, W_gu, Wd, max_iters=32, tol=1e-6)
        dY = torch.randn(B, T, D, generator=g).cuda()
        api.block_backward(x, w1, Wx, bias, R, w2, W_gu, Wd, S, dY)
        st = _status(lib)
        assert st[0] == 0, _describe(lib, st)


def test_checked_build_reports_a_planted_violation(cuda_device):
    """debug_fault = 2: the checked build checks each iteration's last tile
    boundary store against an extent one element short, so every iteration
    reports that one element (and skips it); nothing else is out of bounds."""
    with _lib.checked_library() as lib:
        assert lib.slstm_check_clear() == _lib.SLSTM_OK
        B, T, d = 2, 256, 64    # T a multiple of 64: the last tile stores its boundary state
        w, dev = _dense_case(B, T, 8, d, "f32", "sigmoid", 3)
        P = api.preact_gemm(dev["x"], dev["Wx"], dev["bias"])
        K = 3
        api.newton_forward(P, dev["R"], dev["s0"], max_iters=K, fixed=True, debug_fault=2, carry_mode=1)
        st = _status(lib)
        n_tiles = B * (d // 32) * (T // 64)
        assert st[0] == K, _describe(lib, st)
        assert lib.slstm_check_site_file(int(st[1] // 100000)) == b"newton.cu"
        assert st[2] == n_tiles * 128 - 1 and st[3] == n_tiles * 128 - 1, st
        assert lib.slstm_check_clear() == _lib.SLSTM_OK
        assert _status(lib) == [0, 0, 0, 0]
