"""ctypes loader for libqwha.so (the C ABI declared in include/qwha.h).

The shared library must have been built (``python walsh_hadamard_sparse_b200/build.py``
or ``__graft_entry__.build()``). There is no fallback: importing the binding
without the library raises, so nothing can silently run another code path.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqwha.so")

P = ctypes.c_void_p
i32, i64, f32, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class QwhaAdapter(ctypes.Structure):
    _fields_ = [
        ("d_in", i32),
        ("d_out", i32),
        ("had_block", i32),
        ("algo", i32),
        ("p", i64),
        ("row_ptr", P),
        ("col_idx", P),
        ("coef", P),
        ("col_ptr", P),
        ("row_idx", P),
        ("perm", P),
        ("tile_ptr", P),
        ("tile_pos", P),
        ("tile_rk", P),
        ("weff", P),
        ("z_given", i32),
    ]


class QwhaQweight(ctypes.Structure):
    _fields_ = [("bits", i32), ("group", i32), ("qweight", P), ("scales", P), ("zeros", P)]


_SIGNATURES = {
    "qwha_fwht": (ctypes.c_int, [ctypes.c_int, P, P, i64, i32, i32, P]),
    "qwha_adapter_fwd": (
        ctypes.c_int,
        [ctypes.POINTER(QwhaAdapter), ctypes.POINTER(QwhaQweight), ctypes.c_int, P, i64, f32, P, P, P, sz, P],
    ),
    "qwha_adapter_bwd": (
        ctypes.c_int,
        [ctypes.POINTER(QwhaAdapter), ctypes.POINTER(QwhaQweight), ctypes.c_int, P, P, i64, f32, P, P, P, sz, P],
    ),
    "qwha_coef_grad_noalloc": (ctypes.c_int, [ctypes.POINTER(QwhaAdapter), ctypes.c_int, P, P, i64, f32, P, P]),
    "qwha_init_alloc": (ctypes.c_int, [P, i32, i32, i32, i64, i32, ctypes.c_int, P, P, P, P, P, sz, P]),
    "qwha_init_norms": (ctypes.c_int, [P, i32, i32, P, P]),
    "qwha_calib_hessian": (ctypes.c_int, [P, i64, i32, P, P]),
    "qwha_refine_values": (ctypes.c_int, [P, i32, i32, i32, P, f32, P, P, i64, P, P, sz, P]),
    "qwha_init_select_global": (ctypes.c_int, [P, i32, i32, i32, i64, ctypes.c_int, ctypes.c_uint64, P, P, P, P, P, sz,
                                               P]),
    "qwha_init_budgets": (ctypes.c_int, [P, i32, i32, i64, i32, ctypes.c_int, P, P, P, sz, P]),
    "qwha_init_select": (ctypes.c_int, [P, i32, i32, i32, P, P, i64, P, P, P]),
    "qwha_plan_build": (ctypes.c_int, [i32, i32, i64, P, P, P, P, P, P, P, P, P, sz, P]),
    "qwha_energy_stats": (ctypes.c_int, [P, i32, i32, i32, i64, P, P, sz, P]),
    "qwha_pattern_stats": (ctypes.c_int, [i32, i32, i64, P, P, P, P, P, sz, P]),
    "qwha_plan_tiles": (i64, [i32, i32]),
    "qwha_workspace_size": (sz, [ctypes.c_int, i32, i32, i64, i64, i32]),
    "qwha_validate_plan": (ctypes.c_int, [ctypes.POINTER(QwhaAdapter), P]),
    "qwha_check_stream_status": (ctypes.c_int, [P]),
    "qwha_stage_timing": (None, [i32]),
    "qwha_stage_count": (i32, []),
    "qwha_stage_name": (ctypes.c_char_p, [i32]),
    "qwha_stage_report": (ctypes.c_int, [P, P, P]),
    "qwha_debug_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "qwha_debug_fail_cuda_checks": (None, [i32]),
    "qwha_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qwha_last_error": (ctypes.c_char_p, []),
    "qwha_version": (ctypes.c_char_p, []),
}


class QwhaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises ImportError when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build the CUDA library first "
                "(python walsh_hadamard_sparse_b200/build.py)"
            )
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def check(status: int, where: str) -> None:
    if status != 0:
        h = lib()
        raise QwhaError(status, where, (h.qwha_last_error() or b"").decode())


def exported_symbols() -> list[str]:
    return sorted(_SIGNATURES)
