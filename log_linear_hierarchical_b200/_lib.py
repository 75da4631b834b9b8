"""ctypes loader for libllsa.so, the CUDA C-ABI library of the LLSA hot path.

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
There is no fallback; a missing library raises ``LLSAExtensionMissing``.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libllsa.so")

LLSA_BF16 = 0
LLSA_F32 = 1

STATUS_NAMES = {
    0: "LLSA_OK",
    1: "LLSA_ERR_INVALID_ARG",
    2: "LLSA_ERR_UNSUPPORTED",
    3: "LLSA_ERR_WORKSPACE",
    4: "LLSA_ERR_CUDA",
    5: "LLSA_ERR_INTERNAL",
    6: "LLSA_ERR_TIMEOUT",
}

# Every symbol include/llsa.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_S = ctypes.c_size_t
_I = ctypes.c_int


class LLSAShape(ctypes.Structure):
    """Mirror of ``llsa_shape``."""

    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("D", ctypes.c_int32),
                ("block", ctypes.c_int32), ("topk", ctypes.c_int32), ("levels", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32), ("n_valid", ctypes.c_int32)]


# llsa_shape.flags: log-count score bias on the coarse KV entries (ln 16^l at level l)
LLSA_FLAG_LOG_BIAS = 1
LLSA_FLAG_ALL_TOP = 2
LLSA_FLAG_LEVEL1 = 4
LLSA_FLAG_GRID_ORDER = 8
LLSA_FLAG_ONE_LAUNCH_SELECT = 16
LLSA_FLAG_CAUSAL = 32
LLSA_NO_PICK = 0x7FFFFFFF


_SP = ctypes.POINTER(LLSAShape)


class LLSAStepBuffers(ctypes.Structure):
    """Mirror of ``llsa_step_buffers``."""

    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "dO", "q_pyr", "k_pyr", "v_pyr", "idx", "row_ptr",
                                                 "col", "o", "lse", "dq", "dk", "dv")] + \
               [("transpose_workspace", ctypes.c_void_p), ("transpose_workspace_bytes", ctypes.c_size_t),
                ("backward_workspace", ctypes.c_void_p), ("backward_workspace_bytes", ctypes.c_size_t)]


_BP = ctypes.POINTER(LLSAStepBuffers)

SIGNATURES = {
    "llsa_status_string": (ctypes.c_char_p, [_I]),
    "llsa_validate_shape": (_I, [_SP]),
    "llsa_pyramid_elems": (_S, [_SP]),
    "llsa_index_elems": (_S, [_SP]),
    "llsa_row_ptr_elems": (_S, [_SP]),
    "llsa_transpose_workspace_bytes": (_S, [_SP]),
    "llsa_backward_workspace_bytes": (_S, [_SP]),
    "llsa_build_pyramid": (_I, [_SP, _P, _P, _P, _P, _P, _P, _P]),
    "llsa_select": (_I, [_SP, _P, _P, _P, _P]),
    "llsa_index_transpose": (_I, [_SP, _P, _P, _P, _P, _S, _P]),
    "llsa_index_transpose_noalloc": (_I, [_SP, _P, _P, _P, _P]),
    "llsa_forward": (_I, [_SP, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "llsa_backward": (_I, [_SP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "llsa_train_step": (_I, [_SP, _BP, _P, _P]),
    "llsa_plan_create": (_I, [_SP, _BP, ctypes.c_int32, ctypes.POINTER(_P)]),
    "llsa_plan_launch": (_I, [_P, _P]),
    "llsa_plan_destroy": (None, [_P]),
    "llsa_token_permute": (_I, [_SP, _P, _P, ctypes.c_int32, _P]),
    "llsa_device_status": (_I, [ctypes.POINTER(ctypes.c_int32), _P]),
    "llsa_check_bounded_wait": (_I, [ctypes.c_int64, _P]),
    "llsa_gather_probe": (_I, [_P, ctypes.c_int64, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P]),
    "llsa_trace_begin": (_I, [ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]),
    "llsa_trace_end": (_I, [ctypes.POINTER(ctypes.c_int32)]),
    "llsa_kernel_name": (ctypes.c_char_p, [ctypes.c_int32]),
}


class LLSAExtensionMissing(RuntimeError):
    pass


# Size of the fixed scratch array behind llsa_index_transpose_noalloc (LLSA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 8 << 20

_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (once) and return the library with every declared signature bound."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise LLSAExtensionMissing(
            f"{p} is missing: build it with `python -m log_linear_hierarchical_b200.build` "
            "(the LLSA path has no CPU fallback)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib
