"""ctypes binding of libtgd.so (the C ABI declared in include/tgd.h).

Argument marshalling only: every step of the optimizer runs in the CUDA
library. PyTorch supplies device memory and the current stream.
"""

from __future__ import annotations

import ctypes as C
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtgd.so")

MAX_NDIM = 8
TOPK_STATIC_MAX_N = 1 << 28  # TGD_TOPK_STATIC_MAX_N

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "OOM", 4: "CUDA", 5: "TIMEOUT",
          6: "STATE", 7: "NONFINITE"}
DTYPES = {"r32": 0, "c64": 1, "c32h": 2, "r16": 3}
PATHS = {"auto": 0, "generic": 1, "tcgen05": 2}
ELEM_BYTES = {"r32": 4, "c64": 8, "c32h": 4, "r16": 2}


class TgdError(RuntimeError):
    def __init__(self, status: int, msg: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"TGD_ERR_{self.name}: {msg}")


class Options(C.Structure):
    _fields_ = [("omega_mode", C.c_int), ("seed", C.c_uint64), ("sparse_scale", C.c_float),
                ("complex_adam", C.c_int), ("moments_on_refresh", C.c_int),
                ("auto_refresh", C.c_int), ("path", C.c_int), ("sm_budget", C.c_int),
                ("order", C.c_int), ("basis", C.c_int), ("wait_limit_ms", C.c_int),
                ("test_stall", C.c_int), ("sparse_k", C.c_int64), ("mode0_total", C.c_int64)]


class Info(C.Structure):
    _fields_ = [("ndim", C.c_int), ("shape", C.c_int64 * MAX_NDIM), ("ranks", C.c_int64 * MAX_NDIM),
                ("N", C.c_int64), ("k", C.c_int64), ("ncore", C.c_int64),
                ("core_m_len", C.c_int64), ("core_v_len", C.c_int64),
                ("sparse_m_len", C.c_int64), ("sparse_v_len", C.c_int64), ("path", C.c_int),
                ("device_bytes", C.c_size_t), ("t", C.c_int64), ("refreshes", C.c_int64),
                ("has_subspace", C.c_int)]


class StateView(C.Structure):
    _fields_ = [("t", C.c_int64), ("refreshes", C.c_int64), ("has_subspace", C.c_int),
                ("omega", C.c_void_p), ("omega_val", C.c_void_p),
                ("U", C.c_void_p * MAX_NDIM), ("core_m", C.c_void_p), ("core_v", C.c_void_p),
                ("sparse_m", C.c_void_p), ("sparse_v", C.c_void_p)]


class KernelTime(C.Structure):
    _fields_ = [("name", C.c_char * 40), ("launches", C.c_int64), ("total_ms", C.c_double)]


_lock = threading.Lock()
_lib = None

# name -> (restype, argtypes); the exported symbols of include/tgd.h
class Memory(C.Structure):
    _fields_ = [(n, C.c_int64) for n in ("N", "k", "core_elems", "factor_elems", "adamw_bytes",
                                         "core_bytes", "factor_bytes", "sparse_bytes",
                                         "total_bytes")]


SIGNATURES = {
    "tgd_state_memory": (C.c_int, [C.c_int, C.c_void_p, C.c_void_p, C.c_double, C.c_int, C.c_int,
                                   C.POINTER(Memory)]),
    "tgd_default_options": (None, [C.POINTER(Options)]),
    "tgd_create": (C.c_int, [C.POINTER(C.c_void_p), C.c_int, C.c_void_p, C.c_void_p, C.c_double,
                             C.c_int64, C.c_float, C.c_float, C.c_float, C.c_float, C.c_float,
                             C.c_int, C.c_int, C.POINTER(Options)]),
    "tgd_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "tgd_refresh": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "tgd_step_host": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "tgd_step_begin": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "tgd_core_buffer": (C.c_int, [C.c_void_p, C.POINTER(C.c_void_p), C.POINTER(C.c_int64)]),
    "tgd_step_end": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "tgd_sync": (C.c_int, [C.c_void_p, C.c_void_p]),
    "tgd_destroy": (C.c_int, [C.c_void_p]),
    "tgd_query": (C.c_int, [C.c_void_p, C.POINTER(Info)]),
    "tgd_get_state": (C.c_int, [C.c_void_p, C.POINTER(StateView), C.c_void_p]),
    "tgd_set_state": (C.c_int, [C.c_void_p, C.POINTER(StateView), C.c_void_p]),
    "tgd_topk_workspace_bytes": (C.c_size_t, [C.c_int64]),
    "tgd_topk_select": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                  C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "tgd_topk_select_static": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                         C.c_void_p, C.c_void_p]),
    "tgd_profile": (C.c_int, [C.c_void_p, C.c_int]),
    "tgd_profile_read": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.POINTER(C.c_int)]),
    "tgd_last_error": (C.c_char_p, [C.c_void_p]),
}


def lib():
    """Loads libtgd.so; raises if it has not been built (no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build the CUDA library first "
                    "(python -m rank_sparse_tensor_b200.build)")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def check(status: int, handle=None):
    if status != 0:
        msg = lib().tgd_last_error(handle)
        raise TgdError(status, msg.decode() if msg else "")
