"""Python face of the CPU oracle (``kvq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  The product package never
imports this module, and this module imports nothing from the product.

Every function cites the passage of the PM-KVQ note (papernotes.org,
"PM-KVQ: Progressive Mixed-Precision KV Cache Quantization for Long-CoT LLMs")
that it follows; the readings taken where the note is silent are listed at the
top of ``kvq_oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from pathlib import Path

import numpy as np

HEAD_DIM = 128
_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "kvq_oracle.c"
_LIB = _HERE / "liboracle.so"

# -O2 without fast-math, FMA contraction off: every fp32 step of the quantizer
# is a single IEEE round-to-nearest operation.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> Path:
    """Compile the oracle to ``oracle/liboracle.so`` (gcc)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.{os.getpid()}")
        subprocess.check_call(["gcc", *CFLAGS, str(_SRC), "-o", str(tmp), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class _Layer(C.Structure):
    _fields_ = [
        ("batch", C.c_int), ("kv_heads", C.c_int), ("fbit", C.c_int), ("n_f", C.c_int),
        ("bits", C.c_int), ("n", C.c_int), ("n_shrinks", C.c_int),
        ("shrink_at", C.c_int * 8),
        ("kc", C.POINTER(C.c_uint16)), ("vc", C.POINTER(C.c_uint16)),
        ("km", C.POINTER(C.c_uint16)), ("vm", C.POINTER(C.c_uint16)),
        ("shift_mode", C.c_int),
    ]


class _WLayer(C.Structure):
    _fields_ = [
        ("main", _Layer), ("n", C.c_int), ("n_max", C.c_int),
        ("kc", C.POINTER(C.c_uint16)), ("vc", C.POINTER(C.c_uint16)),
        ("km", C.POINTER(C.c_uint16)), ("vm", C.POINTER(C.c_uint16)),
    ]


class _CLayer(C.Structure):
    _fields_ = [
        ("main", _Layer), ("kmc", C.POINTER(C.c_uint16)), ("n", C.c_int),
        ("skc", C.POINTER(C.c_uint16)), ("svc", C.POINTER(C.c_uint16)),
        ("skm", C.POINTER(C.c_uint16)), ("svm", C.POINTER(C.c_uint16)),
    ]


WINDOW = 128
KBLOCK = 128


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(str(build()))
        L = _lib
        P = C.c_void_p
        L.orc_f16_to_f64.argtypes = [C.c_uint16]
        L.orc_f16_to_f64.restype = C.c_double
        L.orc_f16_from_f64.argtypes = [C.c_double, C.c_int]
        L.orc_f16_from_f64.restype = C.c_uint16
        L.orc_lambda_inv.argtypes = [C.c_float]
        L.orc_lambda_inv.restype = C.c_float
        L.orc_migrate.argtypes = [C.c_float, C.c_float]
        L.orc_migrate.restype = C.c_float
        L.orc_lambda_from_keys.argtypes = [P, C.c_int, C.c_int, C.c_double, P]
        L.orc_group_meta.argtypes = [P, C.c_int, P, P]
        L.orc_codes_with_meta.argtypes = [P, C.c_int, C.c_int, C.c_uint16, C.c_uint16, P]
        L.orc_quantize_group.argtypes = [P, C.c_int, C.c_int, P, P, P]
        L.orc_dequant.argtypes = [C.c_uint16, C.c_uint16, C.c_uint16, C.c_int]
        L.orc_dequant.restype = C.c_double
        L.orc_ers.argtypes = [C.c_uint32, C.c_int]
        L.orc_ers.restype = C.c_uint32
        L.orc_scale_after_shrink.argtypes = [C.c_double, C.c_int]
        L.orc_scale_after_shrink.restype = C.c_double
        L.orc_drs.argtypes = [C.c_uint32, C.c_int]
        L.orc_drs.restype = C.c_uint32
        L.orc_drs_range.argtypes = [C.c_uint16, C.c_int]
        L.orc_drs_range.restype = C.c_uint16
        L.orc_layer_set_shift_mode.argtypes = [P, C.c_int]
        L.orc_wlayer_sizeof.restype = C.c_size_t
        L.orc_wlayer_init.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int]
        L.orc_wlayer_free.argtypes = [P]
        L.orc_wlayer_append.argtypes = [P, P, P, C.c_int, P]
        L.orc_wlayer_window_tokens.argtypes = [P, P]
        L.orc_wattention.argtypes = [P, P, C.c_int, P, C.c_double, P]
        L.orc_layer_sizeof.restype = C.c_size_t
        L.orc_layer_capacity.argtypes = [P, C.c_int]
        L.orc_layer_init.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int]
        L.orc_layer_free.argtypes = [P]
        L.orc_layer_shrink.argtypes = [P]
        L.orc_layer_force_shrink.argtypes = [P]
        L.orc_layer_append.argtypes = [P, P, P, C.c_int, P]
        L.orc_attention.argtypes = [P, P, C.c_int, P, C.c_double, P]
        L.orc_attention_dense.argtypes = [P, P, P, C.c_int, C.c_int, C.c_int, C.c_int,
                                          C.c_double, P]
        L.orc_clayer_sizeof.restype = C.c_size_t
        L.orc_clayer_init.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int]
        L.orc_clayer_free.argtypes = [P]
        L.orc_clayer_append.argtypes = [P, P, P, C.c_int, P]
        L.orc_cattention.argtypes = [P, P, C.c_int, P, C.c_double, P]
        L.orc_int16_value.argtypes = [C.c_uint16, C.c_uint16, C.c_uint16]
        L.orc_int16_value.restype = C.c_float
        assert L.orc_layer_sizeof() == C.sizeof(_Layer)
        assert L.orc_wlayer_sizeof() == C.sizeof(_WLayer)
        assert L.orc_clayer_sizeof() == C.sizeof(_CLayer)
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


# --- binary16 --------------------------------------------------------------

def f16_to_f64(bits: int) -> float:
    """binary16 bit pattern -> value (IEEE-754 definition)."""
    return lib().orc_f16_to_f64(int(bits))


def f16_from_f64(x: float, mode: int) -> int:
    """value -> binary16 bits; mode 0 nearest-even, -1 down, +1 up."""
    return lib().orc_f16_from_f64(float(x), int(mode))


# --- migration (Key design 3) ------------------------------------------------

def lambda_from_keys(keys: np.ndarray, alpha: float) -> np.ndarray:
    """lambda_i = (max_m |K_{m,i}|)^alpha.  keys: [m][kv_heads][128] -> [kv_heads][128]."""
    keys = np.ascontiguousarray(keys, dtype=np.float32)
    m, h, d = keys.shape
    out = np.empty((h, d), np.float32)
    for j in range(h):
        kj = np.ascontiguousarray(keys[:, j, :])
        lib().orc_lambda_from_keys(_ptr(kj), m, d, float(alpha), _ptr(out[j]))
    return out


def migrate(k: np.ndarray, lam: np.ndarray) -> np.ndarray:
    """fp32(k * fp32(1/lambda)) elementwise (small arrays; one C call per value)."""
    k = np.asarray(k, np.float32)
    lam = np.broadcast_to(np.asarray(lam, np.float32), k.shape)
    out = np.empty(k.shape, np.float32)
    f = lib().orc_migrate
    for idx in np.ndindex(k.shape):
        out[idx] = f(float(k[idx]), float(lam[idx]))
    return out


# --- quantizer (training strategy: group 128, asymmetric) ------------------

def quantize_group(x: np.ndarray, bits: int):
    """-> (codes uint16[n], R bits, Z bits)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.empty(x.shape[0], np.uint16)
    r = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    lib().orc_quantize_group(_ptr(x), x.shape[0], bits, _ptr(codes), _ptr(r), _ptr(z))
    return codes, int(r[0]), int(z[0])


def codes_with_meta(x: np.ndarray, bits: int, r_bits: int, z_bits: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.empty(x.shape[0], np.uint16)
    lib().orc_codes_with_meta(_ptr(x), x.shape[0], bits, r_bits, z_bits, _ptr(codes))
    return codes


def dequant(code: int, r_bits: int, z_bits: int, bits: int) -> float:
    return lib().orc_dequant(int(code), int(r_bits), int(z_bits), int(bits))


def dequant_array(codes: np.ndarray, meta: np.ndarray, bits: int) -> np.ndarray:
    """Vectorised x^ = Z + q R/(2^b-1) for codes [..., 128] and meta [..., 2]."""
    r = meta[..., 0].astype(np.uint16).view(np.float16).astype(np.float64)
    z = meta[..., 1].astype(np.uint16).view(np.float16).astype(np.float64)
    return z[..., None] + codes.astype(np.float64) * (r / float((1 << bits) - 1))[..., None]


# --- Equivalent Right Shift (Key design 1) -------------------------------------

def ers(x2b: int, b: int) -> int:
    return lib().orc_ers(int(x2b), int(b))


def scale_after_shrink(s2b: float, b: int) -> float:
    return lib().orc_scale_after_shrink(float(s2b), int(b))


def drs(x2b: int, b: int) -> int:
    """Direct Right Shift (the note's ablation): keep the high b bits."""
    return lib().orc_drs(int(x2b), int(b))


def drs_range(r_bits: int, b: int) -> int:
    """Range after a Direct Right Shift: binary16 RN of fp32(R 2^b / (2^b + 1))."""
    return lib().orc_drs_range(int(r_bits), int(b))


# --- progressive cache model of one block -------------------------------------

class Layer:
    """One transformer block's progressive cache (Key design 1), logical order."""

    def __init__(self, batch: int, kv_heads: int, n_f: int, fbit: int):
        self._s = _Layer()
        rc = lib().orc_layer_init(C.byref(self._s), batch, kv_heads, n_f, fbit)
        if rc != 0:
            raise ValueError(f"orc_layer_init failed ({rc})")
        self.batch, self.kv_heads, self.n_f, self.fbit = batch, kv_heads, n_f, fbit

    def __del__(self):
        if getattr(self, "_view", False):  # owned by a WLayer
            return
        try:
            lib().orc_layer_free(C.byref(self._s))
        except Exception:
            pass

    @property
    def bits(self) -> int:
        return self._s.bits

    @property
    def n(self) -> int:
        return self._s.n

    @property
    def n_shrinks(self) -> int:
        return self._s.n_shrinks

    @property
    def shrink_at(self):
        return list(self._s.shrink_at[: min(8, self._s.n_shrinks)])

    def capacity(self, bits: int | None = None) -> int:
        return lib().orc_layer_capacity(C.byref(self._s), bits or self.bits)

    def append(self, k: np.ndarray, v: np.ndarray, lam: np.ndarray | None) -> int:
        """k, v: [batch][n][kv_heads][128] fp32.  Returns 0 or 1 (budget full)."""
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        assert k.shape == v.shape and k.shape[0] == self.batch and k.shape[2] == self.kv_heads
        lp = None
        if lam is not None:
            lam = np.ascontiguousarray(lam, dtype=np.float32)
            lp = _ptr(lam)
        return lib().orc_layer_append(C.byref(self._s), _ptr(k), _ptr(v), k.shape[1], lp)

    def shrink(self) -> int:
        return lib().orc_layer_force_shrink(C.byref(self._s))

    def set_shift_mode(self, mode: int) -> int:
        """0: Equivalent Right Shift (default), 1: Direct Right Shift; before the first shrink."""
        return lib().orc_layer_set_shift_mode(C.byref(self._s), int(mode))

    def _arr(self, p, last):
        shape = (self.batch, self.kv_heads, self.n_f, last)
        a = np.ctypeslib.as_array(p, shape=(int(np.prod(shape)),)).reshape(shape)
        return a[:, :, : self.n]

    def k_codes(self):
        """[batch][kv_heads][n][128] uint16 (a copy)."""
        return self._arr(self._s.kc, HEAD_DIM).copy()

    def v_codes(self):
        return self._arr(self._s.vc, HEAD_DIM).copy()

    def k_meta(self):
        """[batch][kv_heads][n][2] uint16: (R bits, Z bits)."""
        return self._arr(self._s.km, 2).copy()

    def v_meta(self):
        return self._arr(self._s.vm, 2).copy()

    def attention(self, q: np.ndarray, lam: np.ndarray | None, sm_scale: float) -> np.ndarray:
        """q: [batch][q_heads][128] fp32 -> fp64 [batch][q_heads][128]."""
        q = np.ascontiguousarray(q, dtype=np.float32)
        out = np.empty(q.shape, np.float64)
        lp = None
        if lam is not None:
            lam = np.ascontiguousarray(lam, dtype=np.float32)
            lp = _ptr(lam)
        rc = lib().orc_attention(C.byref(self._s), _ptr(q), q.shape[1], lp, float(sm_scale),
                                 _ptr(out))
        if rc != 0:
            raise ValueError(f"orc_attention failed ({rc})")
        return out


def attention_dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, sm_scale: float) -> np.ndarray:
    """fp64 attention on real-valued K/V.  q [Hq][d], k/v [T][Hkv][d]."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    T, hkv, d = k.shape
    out = np.empty(q.shape, np.float64)
    lib().orc_attention_dense(_ptr(q), _ptr(k), _ptr(v), T, q.shape[0], hkv, d, float(sm_scale),
                              _ptr(out))
    return out


def block_bytes(bits: int, batch: int, kv_heads: int, max_tokens: int) -> int:
    """KV-cache bytes of one block at `bits` for max_tokens tokens: codes
    (16 bits bytes per token-head, K and V) plus binary16 (R, Z) per group."""
    return batch * kv_heads * 2 * max_tokens * (16 * bits + 4)


def allocate_bits_brute(sens, bits, batch: int, kv_heads: int, max_tokens: int, budget: int):
    """Block-wise bit allocation of the PM-KVQ note (key design 2), by
    enumeration: every assignment of one width per block whose total KV
    memory fits the budget M, and the least  sum_i s_{i,b_i}.  Returns
    (objective, [every optimal assignment as a tuple of widths]) or
    (None, []) if nothing fits.  Small cases only (n_opts ** layers)."""
    import itertools

    sens = np.asarray(sens, dtype=np.float64)
    layers, n_opts = sens.shape
    cost = [block_bytes(b, batch, kv_heads, max_tokens) for b in bits]
    best, arg = None, []
    for choice in itertools.product(range(n_opts), repeat=layers):
        if sum(cost[o] for o in choice) > budget:
            continue
        obj = 0.0
        for i, o in enumerate(choice):
            obj += float(sens[i, o])
        if best is None or obj < best - 1e-12 * max(1.0, abs(best)):
            best, arg = obj, [tuple(bits[o] for o in choice)]
        elif abs(obj - best) <= 1e-12 * max(1.0, abs(best)):
            arg.append(tuple(bits[o] for o in choice))
    return best, arg


class WLayer:
    """A block with the sink token and the recent-128 window held at INT16
    (training strategy of the PM-KVQ note: the KIVI trick it keeps); older
    tokens live in the block's progressive cache (`main`, a Layer view)."""

    def __init__(self, batch: int, kv_heads: int, n_f: int, fbit: int):
        self._s = _WLayer()
        rc = lib().orc_wlayer_init(C.byref(self._s), batch, kv_heads, n_f, fbit)
        if rc != 0:
            raise ValueError(f"orc_wlayer_init failed ({rc})")
        self.batch, self.kv_heads, self.n_f, self.fbit = batch, kv_heads, n_f, fbit
        self.main = Layer.__new__(Layer)  # a view of the embedded progressive cache
        self.main._s = self._s.main
        self.main.batch, self.main.kv_heads, self.main.n_f, self.main.fbit = batch, kv_heads, n_f, fbit
        self.main._view = True

    def __del__(self):
        try:
            lib().orc_wlayer_free(C.byref(self._s))
        except Exception:
            pass

    @property
    def n(self) -> int:
        return self._s.n

    def set_shift_mode(self, mode: int) -> int:
        return lib().orc_layer_set_shift_mode(C.byref(self._s.main), int(mode))

    def append(self, k: np.ndarray, v: np.ndarray, lam: np.ndarray | None) -> int:
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        assert k.shape == v.shape and k.shape[0] == self.batch and k.shape[2] == self.kv_heads
        lp = None
        if lam is not None:
            lam = np.ascontiguousarray(lam, dtype=np.float32)
            lp = _ptr(lam)
        return lib().orc_wlayer_append(C.byref(self._s), _ptr(k), _ptr(v), k.shape[1], lp)

    def window_tokens(self) -> list:
        """Token indices held at INT16: the sink, then the window oldest first."""
        out = (C.c_int * (WINDOW + 1))()
        n = lib().orc_wlayer_window_tokens(C.byref(self._s), out)
        return list(out[:n])

    def _all(self, p, last):
        shape = (self.batch, self.kv_heads, self._s.n_max, last)
        return np.ctypeslib.as_array(p, shape=(int(np.prod(shape)),)).reshape(shape)

    def int16_codes(self):
        """(k codes, v codes, k meta, v meta) of every appended token at INT16,
        [batch][kv_heads][n][...] (tokens since moved keep their INT16 record)."""
        n = self.n
        return tuple(self._all(p, d)[:, :, :n].copy() for p, d in
                     ((self._s.kc, HEAD_DIM), (self._s.vc, HEAD_DIM), (self._s.km, 2), (self._s.vm, 2)))

    def window_codes(self):
        """The sink and window tokens' INT16 codes and meta, oldest first."""
        idx = self.window_tokens()
        return tuple(a[:, :, idx] for a in self.int16_codes())

    def attention(self, q: np.ndarray, lam: np.ndarray | None, sm_scale: float) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.float32)
        out = np.empty(q.shape, np.float64)
        lp = None
        if lam is not None:
            lam = np.ascontiguousarray(lam, dtype=np.float32)
            lp = _ptr(lam)
        rc = lib().orc_wattention(C.byref(self._s), _ptr(q), q.shape[1], lp, float(sm_scale), _ptr(out))
        if rc != 0:
            raise ValueError(f"orc_wattention failed ({rc})")
        return out


def int16_value(code: int, r_bits: int, z_bits: int) -> float:
    """fp32 value of an INT16 record: Z + code * (R / 65535), three RN steps
    (how a staged Key re-enters the quantizer of a per-channel block)."""
    return lib().orc_int16_value(int(code), int(r_bits), int(z_bits))


class CLayer:
    """A block whose Keys are grouped per channel over blocks of 128 tokens
    (KIVI's axis, the other reading of the PM-KVQ note's group size 128);
    Values per token.  The block being filled is staged at INT16; complete
    blocks live in the progressive cache (`main`, a Layer view whose Key meta
    is unused: the per-channel ranges are in `k_meta_channel`)."""

    def __init__(self, batch: int, kv_heads: int, n_f: int, fbit: int):
        self._s = _CLayer()
        rc = lib().orc_clayer_init(C.byref(self._s), batch, kv_heads, n_f, fbit)
        if rc != 0:
            raise ValueError(f"orc_clayer_init failed ({rc})")
        self.batch, self.kv_heads, self.n_f, self.fbit = batch, kv_heads, n_f, fbit
        self.main = Layer.__new__(Layer)
        self.main._s = self._s.main
        self.main.batch, self.main.kv_heads, self.main.n_f, self.main.fbit = batch, kv_heads, n_f, fbit
        self.main._view = True

    def __del__(self):
        try:
            lib().orc_clayer_free(C.byref(self._s))
        except Exception:
            pass

    @property
    def n(self) -> int:
        return self._s.n

    @property
    def n_staged(self) -> int:
        return self._s.n - self._s.main.n

    def set_shift_mode(self, mode: int) -> int:
        return lib().orc_layer_set_shift_mode(C.byref(self._s.main), int(mode))

    def append(self, k: np.ndarray, v: np.ndarray, lam: np.ndarray | None) -> int:
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        assert k.shape == v.shape and k.shape[0] == self.batch and k.shape[2] == self.kv_heads
        lp = None
        if lam is not None:
            lam = np.ascontiguousarray(lam, dtype=np.float32)
            lp = _ptr(lam)
        return lib().orc_clayer_append(C.byref(self._s), _ptr(k), _ptr(v), k.shape[1], lp)

    def k_meta_channel(self):
        """[batch][kv_heads][blocks][128][2] uint16: (R bits, Z bits) of each
        Key channel of each complete block."""
        nb = self.n_f // KBLOCK
        shape = (self.batch, self.kv_heads, nb, HEAD_DIM, 2)
        a = np.ctypeslib.as_array(self._s.kmc, shape=(int(np.prod(shape)),)).reshape(shape)
        return a[:, :, : self._s.main.n // KBLOCK].copy()

    def staged_codes(self):
        """(k codes, v codes, k meta, v meta) of the staged tokens at INT16,
        oldest first: [batch][kv_heads][n_staged][...]."""
        ns = self.n_staged
        out = []
        for p, d in ((self._s.skc, HEAD_DIM), (self._s.svc, HEAD_DIM), (self._s.skm, 2), (self._s.svm, 2)):
            shape = (self.batch, self.kv_heads, KBLOCK, d)
            a = np.ctypeslib.as_array(p, shape=(int(np.prod(shape)),)).reshape(shape)
            out.append(a[:, :, :ns].copy())
        return tuple(out)

    def attention(self, q: np.ndarray, lam: np.ndarray | None, sm_scale: float) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.float32)
        out = np.empty(q.shape, np.float64)
        lp = None
        if lam is not None:
            lam = np.ascontiguousarray(lam, dtype=np.float32)
            lp = _ptr(lam)
        rc = lib().orc_cattention(C.byref(self._s), _ptr(q), q.shape[1], lp, float(sm_scale), _ptr(out))
        if rc != 0:
            raise ValueError(f"orc_cattention failed ({rc})")
        return out
