"""ctypes loader for libslstm.so (the C ABI declared in include/slstm.h).

Argument marshalling only: no arithmetic of the method happens in Python.
Importing this module never falls back to anything: if the shared library is
missing it is built with nvcc, and if that fails the import raises.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

SLSTM_OK = 0
SLSTM_ERR_INVALID_ARG = 1
SLSTM_ERR_CUDA = 2
SLSTM_ERR_DIVERGED = 3
SLSTM_ERR_TIMEOUT = 4
SLSTM_ERR_UNSUPPORTED = 5

SLSTM_F32 = 0
SLSTM_BF16 = 1
SLSTM_FORGET_SIGMOID = 0
SLSTM_FORGET_EXP = 1
SLSTM_OP_PREACT_GEMM = 0
SLSTM_OP_NEWTON_FORWARD = 1
SLSTM_OP_SCAN_BLOCK4 = 2
SLSTM_OP_NEWTON_BACKWARD = 3
SLSTM_OP_NEWTON_FORWARD_VARLEN = 4
SLSTM_OP_NEWTON_BACKWARD_VARLEN = 5
SLSTM_OP_NEWTON_BACKWARD_HEAD = 6
SLSTM_OP_CONTEXT_PARALLEL = 7
SLSTM_MAX_HEAD_DIM = 32
SLSTM_MAX_GUESS_SWEEPS = 64
SLSTM_MAX_ITERS = 65536
SLSTM_STATS_HISTORY = 64
SLSTM_SCAN_REVERSE_T = 1
SLSTM_SCAN_DEBUG_WITHHOLD = 2
SLSTM_INIT_DECOUPLED = 0
SLSTM_INIT_ZERO = 1
SLSTM_INIT_GIVEN = 2
SLSTM_RESIDUAL_SCALED = 0
SLSTM_RESIDUAL_RAW = 1
SLSTM_HISTORY_BOUND = 0
SLSTM_HISTORY_EXACT = 1
SLSTM_DEFAULT_LOOP_FROM = 2
SLSTM_GEMM_TILES_AUTO = 0
SLSTM_GEMM_TILES_PAIR = 1
SLSTM_GEMM_TILES_SINGLE = 2
SLSTM_NOALLOC_SCRATCH_BYTES = 8 << 20


class NewtonConfig(ctypes.Structure):
    _fields_ = [("max_iters", ctypes.c_int), ("fixed_iters", ctypes.c_int), ("tol", ctypes.c_float),
                ("forget", ctypes.c_int), ("debug_fault", ctypes.c_int), ("wait_limit_us", ctypes.c_int),
                ("carry_mode", ctypes.c_int), ("init", ctypes.c_int), ("residual_mode", ctypes.c_int),
                ("guess_sweeps", ctypes.c_int), ("history", ctypes.c_int), ("n_events", ctypes.c_int),
                ("events", ctypes.c_void_p), ("loop_from", ctypes.c_int)]


STATS_BYTES = 4 * 4 + 2 * 4 * SLSTM_STATS_HISTORY + 2 * 4

_V = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t

# name -> (restype, argtypes); every function of include/slstm.h
SIGNATURES = {
    "slstm_status_string": (ctypes.c_char_p, [_I]),
    "slstm_check_enabled": (_I, []),
    "slstm_check_status": (_I, [ctypes.POINTER(ctypes.c_longlong)]),
    "slstm_check_clear": (_I, []),
    "slstm_check_site_file": (ctypes.c_char_p, [_I]),
    "slstm_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "slstm_preact_gemm": (_I, [_V, _V, _I, _V, _V, _I, _I, _I, _I, _V, _Z, _V]),
    "slstm_set_gemm_tiles": (_I, [_I]),
    "slstm_newton_forward": (_I, [_V, _V, _V, _V, ctypes.POINTER(NewtonConfig), _V, _I, _I, _I, _V, _Z, _V]),
    "scan_block4": (_I, [_V, _V, _V, _V, _I, _I, _I, _I, _V, _Z, _V]),
    "scan_block4_noalloc": (_I, [_V, _V, _V, _V, _I, _I, _I, _I, _V]),
    "slstm_sequential_step": (_I, [_V, _V, _V, _V, _I, _I, _I, _I, _V]),
    "slstm_sequential_step_head": (_I, [_V, _V, _V, _V, _I, _I, _I, _I, _I, _V]),
    "slstm_cp_guess_run": (_I, [_V, _V, _V, _V, _I, _I, _V, _I, _I, _I, _V, _Z, _V]),
    "slstm_cp_guess_apply": (_I, [_V, _V, _V, _V, _V, _I, _V, _I, _I, _I, _I, _I, _V, _Z, _V]),
    "slstm_cp_newton_map": (_I, [_V, _V, _V, _V, _I, _V, _I, _I, _I, _V, _Z, _V]),
    "slstm_cp_newton_apply": (_I, [_V, _V, _V, _V, _I, _V, ctypes.POINTER(NewtonConfig), _V, _I, _I, _I, _V, _Z,
                                   _V]),
    "slstm_newton_forward_head": (_I, [_V, _V, _V, _V, ctypes.POINTER(NewtonConfig), _V, _I, _I, _I, _I, _V, _Z,
                                       _V]),
    "slstm_newton_backward_head": (_I, [_V, _V, _I, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _I,
                                        _I, _V, _Z, _V]),
    "slstm_newton_backward": (_I, [_V, _V, _I, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _I,
                                   _V, _Z, _V]),
    "slstm_newton_forward_varlen": (_I, [_V, _V, _V, _V, _I, _V, ctypes.POINTER(NewtonConfig), _V, _I, _I, _V, _Z,
                                         _V]),
    "slstm_newton_backward_varlen": (_I, [_V, _V, _I, _V, _V, _V, _V, _I, _V, _V, _V, _V, _V, _V, _V, _I, _I, _I,
                                          _I, _V, _Z, _V]),
    "slstm_decode_step": (_I, [_V, _V, _I, _V, _V, _V, _V, _I, _I, _I, _I, _V]),
    "slstm_block_workspace_size": (_Z, [_I, _I, _I, _I]),
    "slstm_block_backward_workspace_size": (_Z, [_I, _I, _I, _I]),
    "slstm_block_backward": (_I, [_V] * 18 + [_I, _I, _I, _I, _I, ctypes.c_float, _V, _Z, _V]),
    "slstm_block_forward": (_I, [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V, ctypes.POINTER(NewtonConfig), _V,
                                 _I, _I, _I, _I, ctypes.c_float, _V, _Z, _V]),
}

_lib = None


def lib_path() -> str:
    return _build.LIB


def _open(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"the library was not built at {path}")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load() -> ctypes.CDLL:
    """The active library: libslstm.so (built first when missing or stale),
    or the bounds-checked one inside `checked_library()`."""
    global _lib
    if _lib is None:
        _lib = _open(_build.build())
    return _lib


_checked = None


def load_checked() -> ctypes.CDLL:
    """The bounds-checked diagnostic library, libslstm_checked.so."""
    global _checked
    if _checked is None:
        _checked = _open(_build.build(checked=True))
    return _checked


class checked_library:
    """Within this context every api call goes to the bounds-checked library."""

    def __enter__(self):
        global _lib
        self._saved = load()
        _lib = load_checked()
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


class SlstmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        name = load().slstm_status_string(status).decode()
        super().__init__(f"{fn} returned {name} ({status})")


def check(fn: str, status: int) -> None:
    if status != SLSTM_OK:
        raise SlstmError(fn, status)
