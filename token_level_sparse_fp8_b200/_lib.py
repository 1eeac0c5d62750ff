"""ctypes loader for libjssa.so: symbol table and argument types matching include/jssa.h."""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjssa.so")

c_int, c_int64, c_size_t, c_float, c_void_p = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                                               ctypes.c_float, ctypes.c_void_p)
c_uint32_p = ctypes.POINTER(ctypes.c_uint32)
c_size_t_p = ctypes.POINTER(ctypes.c_size_t)
P = c_void_p  # every device pointer

JSSA_OK = 0
STATUS_NAMES = {
    -1: "JSSA_ERR_NULL",
    -2: "JSSA_ERR_SHAPE",
    -3: "JSSA_ERR_UNSUPPORTED",
    -4: "JSSA_ERR_ALIGN",
    -5: "JSSA_ERR_WORKSPACE",
    -6: "JSSA_ERR_DEVICE",
    -7: "JSSA_ERR_SCRATCH_LIMIT",
}
FN_SCORE_TOPK, FN_INDEXED_ATTEND, FN_DENSE_DECODE, FN_DECODE, FN_COMPUTE_BASIS = 1, 2, 3, 4, 5
FN_MLA_ATTEND, FN_MLA_DECODE, FN_DECODE_HOST = 6, 7, 8
DEVERR_PAGE, DEVERR_INDEX, DEVERR_SEQLEN = 1, 2, 4

# name -> (restype, argtypes), in header order
SIGNATURES = {
    "jssa_status_string": (ctypes.c_char_p, [c_int]),
    "jssa_version": (c_int, []),
    "jssa_set_wait_limit": (ctypes.c_longlong, [ctypes.c_longlong]),
    "jssa_workspace_size": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_size_t_p]),
    "jssa_workspace_init": (c_int, [P, c_size_t, P]),
    "jssa_calibrate_accumulate": (c_int, [P, c_int64, P, c_int64, c_int, c_int, c_int, c_int, P, P, P]),
    "jssa_mla_calibrate_accumulate": (c_int, [P, c_int64, c_int64, P, c_int64, c_int, c_int, P, P, P]),
    "jssa_compute_basis": (c_int, [P, P, c_int, c_int, c_int, P, P, P, c_size_t, P]),
    "jssa_store": (c_int, [P, c_int64, P, c_int, c_int, c_int, c_int, P, P, c_int64, c_int, P]),
    "jssa_score_topk": (c_int, [P, P, P, P, c_int, P, c_int, c_int, c_int, c_int, c_int, c_int64,
                                c_int, c_int, P, P, P, c_size_t, P]),
    "jssa_indexed_attend": (c_int, [P, P, P, c_int64, c_int64, c_int64, P, c_int, P, P, c_int, c_int,
                                    c_int, c_int, c_int, c_int64, c_int, c_float, P, P, c_size_t, P]),
    "jssa_dense_decode": (c_int, [P, P, P, c_int64, c_int64, c_int64, P, c_int, P, c_int, c_int, c_int,
                                  c_int, c_int64, c_int, c_int, c_float, P, P, c_size_t, P]),
    "jssa_store_bf16": (c_int, [P, c_int64, P, c_int, c_int, c_int, c_int, P, P, c_int64, c_int, P]),
    "jssa_score_topk_bf16": (c_int, [P, P, P, P, c_int, P, c_int, c_int, c_int, c_int, c_int,
                                     c_int64, c_int, c_int, P, P, P, c_size_t, P]),
    "jssa_mla_attend": (c_int, [P, P, c_int64, c_int64, P, c_int, P, P, c_int, c_int, c_int, c_int64,
                                c_int, c_float, P, P, c_size_t, P]),
    "jssa_mla_decode": (c_int, [P, P, P, c_int64, c_int64, P, P, P, c_int, P, c_int, c_int, c_int,
                                c_int64, c_int, c_int, c_float, P, P, P, P, c_size_t, P]),
    "jssa_gather_kv": (c_int, [P, P, c_int64, c_int64, c_int64, P, c_int, P, P, c_int, c_int, c_int,
                               c_int, c_int64, c_int, P, P, P, P]),
    "jssa_decode": (c_int, [P, P, P, P, P, c_int64, c_int64, c_int64, P, P, P, c_int, P, c_int, c_int,
                            c_int, c_int, c_int, c_int64, c_int, c_int, c_float, P, P, P, P, c_size_t,
                            P]),
    "jssa_decode_host": (c_int, [P, P, P, P, P, c_int64, c_int64, c_int64, P, P, P, c_int, P, c_int,
                                 c_int, c_int, c_int, c_int, c_int64, c_int, c_int, c_float, P, P, P,
                                 P, c_size_t, P]),
    "jssa_decode_host_join": (c_int, [P, P]),
    "jssa_indexed_attend_noalloc": (c_int, [P, P, P, c_int64, c_int64, c_int64, P, c_int, P, P, c_int,
                                            c_int, c_int, c_int, c_int, c_int64, c_int, c_float, P, P]),
    "jssa_device_error": (c_int, [c_uint32_p, c_int, P]),
}

_lock = threading.Lock()
_lib = None


class JSSAError(RuntimeError):
    """A libjssa entry point returned a non-zero status."""

    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: status {status} ({STATUS_NAMES.get(status, 'cuda error')}): {text}")
        self.status = status


def load() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built: there is no fallback path)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m token_level_sparse_fp8_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def status_string(status: int) -> str:
    return load().jssa_status_string(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != JSSA_OK:
        raise JSSAError(fn, status, status_string(status))


def call(name: str, *args) -> None:
    check(name, getattr(load(), name)(*args))
