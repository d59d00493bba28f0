"""ctypes binding of libkvq.so (include/kvq.h).  Argument marshalling only:
every step of the hot path runs in the library's CUDA kernels.  There is no
CPU fallback -- if the library is missing this module raises."""
from __future__ import annotations

import ctypes as C
import os
from pathlib import Path

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libkvq.so"

KVQ_OK = 0
KVQ_ERR_INVALID = 1
KVQ_ERR_BUDGET = 2
KVQ_ERR_STATE = 3
KVQ_ERR_OOM = 4
KVQ_ERR_CUDA = 5
KVQ_ERR_WORKSPACE = 6
KVQ_ERR_TIMEOUT = 7
STATUS_NAMES = {
    0: "KVQ_OK", 1: "KVQ_ERR_INVALID", 2: "KVQ_ERR_BUDGET", 3: "KVQ_ERR_STATE",
    4: "KVQ_ERR_OOM", 5: "KVQ_ERR_CUDA", 6: "KVQ_ERR_WORKSPACE", 7: "KVQ_ERR_TIMEOUT",
}
KVQ_DTYPE_BF16 = 0
KVQ_DTYPE_F32 = 1
KVQ_SHIFT_EQUIVALENT = 0
KVQ_SHIFT_DIRECT = 1
KVQ_OPT_SINK_WINDOW = 1
KVQ_OPT_KEY_CHANNEL = 2
KEY_BLOCK = 128
WINDOW_TOKENS = 128

# name -> (restype, argtypes); the exported symbols of include/kvq.h
P = C.c_void_p
I = C.c_int
SZ = C.c_size_t
SIGNATURES = {
    "kvq_pool_bytes": (SZ, [I, I, I, I, SZ, P]),
    "kvq_pool_bytes_ex": (SZ, [I, I, I, I, SZ, P, I]),
    "kvq_alloc": (I, [C.POINTER(P), I, I, I, I, SZ, P, P, SZ]),
    "kvq_alloc_ex": (I, [C.POINTER(P), I, I, I, I, SZ, P, P, SZ, I]),
    "kvq_set_lambda": (I, [P, I, P]),
    "kvq_append": (I, [P, I, P, P, I, I, P]),
    "kvq_shrink": (I, [P, I, P]),
    "kvq_set_shift_mode": (I, [P, I, I]),
    "kvq_decode_workspace": (SZ, [P, I, I]),
    "kvq_decode_attn": (I, [P, I, P, I, C.c_float, P, P, SZ, P]),
    "kvq_decode_attn_noalloc": (I, [P, I, P, I, C.c_float, P, P]),
    "kvq_append_decode": (I, [P, I, P, P, I, P, I, C.c_float, P, P, SZ, P]),
    "kvq_query": (I, [P, I, P, P, P, P]),
    "kvq_max_tokens": (I, [P]),
    "kvq_export": (I, [P, I, I, I, P, P, P, P, P]),
    "kvq_export_window": (I, [P, I, I, I, P, P, P, P, P, P]),
    "kvq_device_status": (I, [P, P]),
    "kvq_selftest_timeout": (I, [P, P]),
    "kvq_allocate_bits": (I, [I, I, P, P, I, I, I, C.c_longlong, SZ, P, P]),
    "kvq_last_error": (C.c_char_p, []),
    "kvq_free": (None, [P]),
}

_lib = None


class KVQError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


def load() -> C.CDLL:
    """Load libkvq.so (built in-tree by build.py).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m mixed_precision_kv_kvq_b200.build` "
                "(nvcc, sm_100a); there is no CPU fallback")
        lib = C.CDLL(os.fspath(LIB_PATH))
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(status: int) -> None:
    if status != KVQ_OK:
        msg = load().kvq_last_error()
        raise KVQError(status, msg.decode() if msg else "")
