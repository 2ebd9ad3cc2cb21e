"""scan_block4_noalloc: the allocation-free variant of scan_block4.

It exists for callers that cannot allocate device memory (their allocator
owns the whole GPU, they may not risk cudaMalloc's device synchronisation,
or they are plugins handed only input and output pointers), so it brings
its scratch from a fixed block of device memory inside the library.  This
test calls it through the C ABI twice in a row, on different problems and
directions, and checks each result against the workspace-taking scan_block4
within the scan tests' tolerance; it runs the largest problem the block
holds, in both directions, against the fp64 oracle, and checks that the size
limit is reported before any work is enqueued.  The file is named to run
last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_pararnn_b200 import _lib, api
from nonlinear_rnn_pararnn_b200.workloads import as_f64

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _noalloc(A, b, y0, y, reverse):
    B, T, _, _, d = A.shape
    flags = _lib.SLSTM_SCAN_REVERSE_T if reverse else 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _lib.load().scan_block4_noalloc(_ptr(A), _ptr(b), _ptr(y0), _ptr(y), B, T, d, flags, stream)


def _problem(B, T, d, seed, with_y0):
    g = torch.Generator().manual_seed(seed)
    A = (torch.rand(B, T, 4, 4, d, generator=g) * 0.6 - 0.3).cuda()
    b = torch.randn(B, T, 4, d, generator=g).cuda()
    y0 = torch.randn(B, 4, d, generator=g).cuda() if with_y0 else None
    return A, b, y0


def test_noalloc_matches_scan_block4_twice(cuda_device):
    cases = [((2, 1000, 72), 21, True, False), ((3, 257, 40), 22, False, True)]
    for (B, T, d), seed, with_y0, reverse in cases:
        A, b, y0 = _problem(B, T, d, seed, with_y0)
        ref = api.scan_block4(A, b, y0, reverse=reverse)
        y = torch.full_like(b, float("nan"))
        assert _noalloc(A, b, y0, y, reverse) == _lib.SLSTM_OK
        torch.cuda.synchronize()
        err = ((y - ref).abs().max() / (1 + ref.abs().max())).item()
        assert err < 1e-5, (B, T, d, err)


@pytest.mark.parametrize("reverse", [False, True])
def test_noalloc_largest_accepted_problem_matches_oracle(reverse, cuda_device):
    """The largest problem the fixed block holds (2337 tiles of 32 steps x 32
    features, within a few KB of the block's end), against the fp64
    sequential solve of the oracle over the full length."""
    B, T, d = 1, 2337 * 32, 32
    lib = _lib.load()
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_SCAN_BLOCK4, B, T, 0, d) <= _lib.SLSTM_NOALLOC_SCRATCH_BYTES
    assert lib.slstm_workspace_size(_lib.SLSTM_OP_SCAN_BLOCK4, B, T + 32, 0, d) > _lib.SLSTM_NOALLOC_SCRATCH_BYTES
    A, b, y0 = _problem(B, T, d, 23, True)
    y = torch.full_like(b, float("nan"))
    assert _noalloc(A, b, y0, y, reverse) == _lib.SLSTM_OK
    torch.cuda.synchronize()
    Al = np.transpose(as_f64(A.cpu()), (0, 4, 1, 2, 3)).reshape(B * d, T, 4, 4)
    bl = np.transpose(as_f64(b.cpu()), (0, 3, 1, 2)).reshape(B * d, T, 4)
    y0l = np.transpose(as_f64(y0.cpu()), (0, 2, 1)).reshape(B * d, 4)
    ref = np.transpose(oracle.affine_solve(Al, bl, y0l, reverse=reverse).reshape(B, d, T, 4), (0, 2, 3, 1))
    err = np.abs(as_f64(y.cpu()) - ref).max() / (1 + np.abs(ref).max())
    assert err < 1e-5, err


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    # 2338 tiles of 32 steps x 32 features need more than the fixed block;
    # rejected on the host, so the fake pointers are never touched
    fake = ctypes.c_void_p(0x10000)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    lib = _lib.load()
    assert lib.scan_block4_noalloc(fake, fake, None, ctypes.c_void_p(0x20000), 1, 2338 * 32, 32, 0,
                                   stream) == _lib.SLSTM_ERR_UNSUPPORTED
    assert lib.scan_block4_noalloc(fake, fake, None, ctypes.c_void_p(0x20000), 1, 0, 32, 0,
                                   stream) == _lib.SLSTM_ERR_INVALID_ARG
