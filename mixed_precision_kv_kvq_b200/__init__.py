"""libkvq for Python: the B200 hot path of PM-KVQ's progressive
mixed-precision KV cache (quantize-on-append, Equivalent Right Shift shrink,
GQA decode attention over packed codes).

The functions named ``kvq_*`` mirror the C ABI of include/kvq.h one to one
(torch tensors in, raw pointers out).  ``KVQCache`` is the same API as an
object that owns its device pool and workspace as torch tensors.  PyTorch is
used for device memory and streams only; all arithmetic runs in libkvq.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional, Sequence

import numpy as np
import torch

from ._lib import (KVQ_DTYPE_BF16, KVQ_DTYPE_F32, KVQ_OPT_KEY_CHANNEL, KVQ_OPT_SINK_WINDOW, KVQ_SHIFT_DIRECT,  # noqa: F401
                   KVQ_SHIFT_EQUIVALENT, KEY_BLOCK, WINDOW_TOKENS, KVQError, check, load)

HEAD_DIM = 128

__all__ = [
    "KVQCache", "KVQError", "load",
    "kvq_pool_bytes", "kvq_pool_bytes_ex", "kvq_alloc", "kvq_alloc_ex", "kvq_export_window", "kvq_set_lambda", "kvq_append", "kvq_shrink", "kvq_set_shift_mode",
    "kvq_decode_workspace", "kvq_decode_attn", "kvq_decode_attn_noalloc", "kvq_append_decode", "kvq_query", "kvq_max_tokens", "kvq_export",
    "kvq_device_status", "kvq_selftest_timeout", "kvq_last_error", "kvq_free", "kvq_allocate_bits",
]


def _stream_ptr(stream) -> C.c_void_p:
    if stream is None:
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return C.c_void_p(torch.cuda.current_stream().cuda_stream)
        return C.c_void_p(None)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _fbit_array(fbit: Sequence[int]):
    arr = (C.c_int * len(fbit))(*[int(f) for f in fbit])
    return arr


def _dptr(t: torch.Tensor) -> C.c_void_p:
    return C.c_void_p(t.data_ptr())


# ---------------------------------------------------------------- C ABI mirror

def kvq_pool_bytes(layers: int, batch: int, kv_heads: int, head_dim: int, budget_bytes: int,
                   fbit: Sequence[int]) -> int:
    return load().kvq_pool_bytes(layers, batch, kv_heads, head_dim, budget_bytes, _fbit_array(fbit))


def kvq_pool_bytes_ex(layers: int, batch: int, kv_heads: int, head_dim: int, budget_bytes: int,
                      fbit: Sequence[int], options: int) -> int:
    return load().kvq_pool_bytes_ex(layers, batch, kv_heads, head_dim, budget_bytes, _fbit_array(fbit), options)


def kvq_alloc(layers: int, batch: int, kv_heads: int, head_dim: int, budget_bytes: int,
              fbit: Sequence[int], dev_pool: Optional[torch.Tensor] = None) -> C.c_void_p:
    return kvq_alloc_ex(layers, batch, kv_heads, head_dim, budget_bytes, fbit, dev_pool, 0)


def kvq_alloc_ex(layers: int, batch: int, kv_heads: int, head_dim: int, budget_bytes: int,
                 fbit: Sequence[int], dev_pool: Optional[torch.Tensor] = None, options: int = 0) -> C.c_void_p:
    h = C.c_void_p()
    pool_ptr = _dptr(dev_pool) if dev_pool is not None else C.c_void_p(None)
    pool_bytes = dev_pool.numel() * dev_pool.element_size() if dev_pool is not None else 0
    check(load().kvq_alloc_ex(C.byref(h), layers, batch, kv_heads, head_dim, budget_bytes,
                              _fbit_array(fbit), pool_ptr, pool_bytes, options))
    return h


def kvq_set_lambda(cache, layer: int, lam: np.ndarray) -> None:
    lam = np.ascontiguousarray(lam, dtype=np.float32)
    check(load().kvq_set_lambda(cache, layer, lam.ctypes.data_as(C.c_void_p)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KVQ_DTYPE_BF16
    if t.dtype == torch.float32:
        return KVQ_DTYPE_F32
    raise TypeError(f"k/v must be bf16 or fp32, got {t.dtype}")


def kvq_append(cache, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
    """k, v: device [batch][n][kv_heads][128], bf16 or fp32, contiguous."""
    if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4 or k.shape[-1] != HEAD_DIM:
        raise ValueError("k and v must both be [batch][n][kv_heads][128] of one dtype")
    if not (k.is_cuda and v.is_cuda and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k and v must be contiguous CUDA tensors")
    check(load().kvq_append(cache, layer, _dptr(k), _dptr(v), _dtype_code(k), k.shape[1],
                            _stream_ptr(stream)))


def kvq_shrink(cache, layer: int, stream=None) -> None:
    check(load().kvq_shrink(cache, layer, _stream_ptr(stream)))


def kvq_set_shift_mode(cache, layer: int, mode: int) -> None:
    """KVQ_SHIFT_EQUIVALENT (default) or KVQ_SHIFT_DIRECT, before the block's first shrink."""
    check(load().kvq_set_shift_mode(cache, layer, int(mode)))


def kvq_decode_workspace(cache, layer: int, q_heads: int) -> int:
    return load().kvq_decode_workspace(cache, layer, q_heads)


def kvq_decode_attn(cache, layer: int, q: torch.Tensor, sm_scale: float, out: torch.Tensor,
                    workspace: torch.Tensor, stream=None) -> None:
    """q: device bf16 [batch][q_heads][128]; out: device fp32, same shape."""
    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.shape[-1] != HEAD_DIM or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 [batch][q_heads][128] tensor")
    if out.dtype != torch.float32 or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous fp32 tensor shaped like q")
    if not (q.is_cuda and out.is_cuda and workspace.is_cuda):
        raise ValueError("q, out and workspace must be CUDA tensors")
    ws_bytes = workspace.numel() * workspace.element_size()
    check(load().kvq_decode_attn(cache, layer, _dptr(q), q.shape[1], float(sm_scale), _dptr(out),
                                 _dptr(workspace), ws_bytes, _stream_ptr(stream)))


def kvq_append_decode(cache, layer: int, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor, sm_scale: float,
                      out: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """One decode step in one launch: append k, v (device [batch][1][kv_heads][128])
    then attend with q (device bf16 [batch][q_heads][128]) into out (fp32)."""
    if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4 or k.shape[1] != 1 or k.shape[-1] != HEAD_DIM:
        raise ValueError("k and v must both be [batch][1][kv_heads][128] of one dtype")
    if not (k.is_cuda and v.is_cuda and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("k and v must be contiguous CUDA tensors")
    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.shape[-1] != HEAD_DIM or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 [batch][q_heads][128] tensor")
    if out.dtype != torch.float32 or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous fp32 tensor shaped like q")
    ws_bytes = workspace.numel() * workspace.element_size()
    check(load().kvq_append_decode(cache, layer, _dptr(k), _dptr(v), _dtype_code(k), _dptr(q), q.shape[1],
                                   float(sm_scale), _dptr(out), _dptr(workspace), ws_bytes, _stream_ptr(stream)))


def kvq_decode_attn_noalloc(cache, layer: int, q: torch.Tensor, sm_scale: float, out: torch.Tensor,
                            stream=None) -> None:
    """Decode attention without a workspace: for callers that cannot allocate
    device memory where they run decode.  The library's own fixed 24 MiB
    scratch buffer (one per GPU, kept until exit) holds the split partials;
    calls that can overlap on the GPU share it and must be serialised."""
    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.shape[-1] != HEAD_DIM or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 [batch][q_heads][128] tensor")
    if out.dtype != torch.float32 or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous fp32 tensor shaped like q")
    if not (q.is_cuda and out.is_cuda):
        raise ValueError("q and out must be CUDA tensors")
    check(load().kvq_decode_attn_noalloc(cache, layer, _dptr(q), q.shape[1], float(sm_scale), _dptr(out),
                                         _stream_ptr(stream)))


def kvq_query(cache, layer: int) -> dict:
    t, b, cap, ns = C.c_int(), C.c_int(), C.c_int(), C.c_int()
    check(load().kvq_query(cache, layer, C.byref(t), C.byref(b), C.byref(cap), C.byref(ns)))
    return {"tokens": t.value, "bits": b.value, "capacity": cap.value, "n_shrinks": ns.value}


def kvq_max_tokens(cache) -> int:
    return load().kvq_max_tokens(cache)


def kvq_export(cache, layer: int, b: int, j: int, stream=None, sink_window: bool = False,
               key_channel: bool = False):
    """-> (k_codes [T][128], v_codes [T][128], k_meta [T][2], v_meta [T][2]) uint16 numpy.
    With the sink + window option (sink_window=True) T counts the
    progressive cache only: tokens 1 .. n - 129.  With per-channel Key
    groups (key_channel=True) T counts the progressive cache (whole blocks of
    128) and k_meta row 128 k + c is Key channel c of block k."""
    T = kvq_query(cache, layer)["tokens"]
    if sink_window:
        T = max(0, T - WINDOW_TOKENS - 1)
    if key_channel:
        T = T // KEY_BLOCK * KEY_BLOCK
    kc = np.zeros((T, HEAD_DIM), np.uint16)
    vc = np.zeros((T, HEAD_DIM), np.uint16)
    km = np.zeros((T, 2), np.uint16)
    vm = np.zeros((T, 2), np.uint16)
    p = lambda a: a.ctypes.data_as(C.c_void_p)  # noqa: E731
    check(load().kvq_export(cache, layer, b, j, p(kc), p(vc), p(km), p(vm), _stream_ptr(stream)))
    return kc, vc, km, vm


def kvq_export_window(cache, layer: int, b: int, j: int, stream=None):
    """-> (k_codes [n][128], v_codes, k_meta [n][2], v_meta) uint16 numpy: the
    sink and window tokens (or, with per-channel Key groups, the staged
    tokens) at 16 bits, oldest first."""
    n1 = WINDOW_TOKENS + 1
    kc = np.zeros((n1, HEAD_DIM), np.uint16)
    vc = np.zeros((n1, HEAD_DIM), np.uint16)
    km = np.zeros((n1, 2), np.uint16)
    vm = np.zeros((n1, 2), np.uint16)
    n = C.c_int()
    p = lambda a: a.ctypes.data_as(C.c_void_p)  # noqa: E731
    check(load().kvq_export_window(cache, layer, b, j, p(kc), p(vc), p(km), p(vm), C.byref(n), _stream_ptr(stream)))
    return kc[:n.value], vc[:n.value], km[:n.value], vm[:n.value]


def kvq_device_status(cache, stream=None) -> None:
    check(load().kvq_device_status(cache, _stream_ptr(stream)))


def kvq_selftest_timeout(cache, stream=None) -> None:
    check(load().kvq_selftest_timeout(cache, _stream_ptr(stream)))


def kvq_allocate_bits(sens, bits: Sequence[int], batch: int, kv_heads: int, max_tokens: int,
                      budget_bytes: int, head_dim: int = HEAD_DIM):
    """sens: [layers][n_opts] sensitivities (host).  -> (fbit list, objective)."""
    sens = np.ascontiguousarray(sens, dtype=np.float64)
    if sens.ndim != 2 or sens.shape[1] != len(bits):
        raise ValueError("sens must be [layers][len(bits)]")
    layers = sens.shape[0]
    b = (C.c_int * len(bits))(*[int(x) for x in bits])
    out = (C.c_int * layers)()
    obj = C.c_double()
    check(load().kvq_allocate_bits(layers, len(bits), b, sens.ctypes.data_as(C.c_void_p), batch, kv_heads,
                                   head_dim, max_tokens, budget_bytes, out, C.byref(obj)))
    return list(out), obj.value


def kvq_last_error() -> str:
    m = load().kvq_last_error()
    return m.decode() if m else ""


def kvq_free(cache) -> None:
    load().kvq_free(cache)


# ---------------------------------------------------------------- object API

class KVQCache:
    """A progressive mixed-precision KV cache for `layers` transformer blocks.

    The device pool is a torch uint8 tensor sized by kvq_pool_bytes; the
    decode workspace is a torch tensor sized by kvq_decode_workspace.
    Host (CPU) inputs are copied to the device on the current stream before
    the call (pinned memory makes the copy asynchronous)."""

    def __init__(self, layers: int, batch: int, kv_heads: int, budget_bytes: int,
                 fbit: Sequence[int], head_dim: int = HEAD_DIM, device=None, sink_window: bool = False,
                 key_channel: bool = False):
        self.layers, self.batch, self.kv_heads = layers, batch, kv_heads
        self.fbit = list(fbit)
        self.device = torch.device(device if device is not None else "cuda")
        self.sink_window = sink_window
        self.key_channel = key_channel
        options = (KVQ_OPT_SINK_WINDOW if sink_window else 0) | (KVQ_OPT_KEY_CHANNEL if key_channel else 0)
        nbytes = kvq_pool_bytes_ex(layers, batch, kv_heads, head_dim, budget_bytes, fbit, options)
        if nbytes == 0:
            raise KVQError(1, "invalid cache parameters or budget too small")
        self.pool = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.handle = kvq_alloc_ex(layers, batch, kv_heads, head_dim, budget_bytes, fbit, self.pool, options)
        self._ws = {}
        self._stage = {}

    # -- helpers
    def _dev(self, t: torch.Tensor) -> torch.Tensor:
        if t.is_cuda:
            return t if t.is_contiguous() else t.contiguous()
        return t.to(self.device, non_blocking=True)

    def workspace(self, layer: int, q_heads: int) -> torch.Tensor:
        n = kvq_decode_workspace(self.handle, layer, q_heads)
        if n == 0:
            raise KVQError(1, f"no workspace size for layer {layer}, q_heads {q_heads}")
        ws = self._ws.get(n)
        if ws is None:
            ws = torch.empty((n + 3) // 4, dtype=torch.float32, device=self.device)
            self._ws[n] = ws
        return ws

    # -- the hot path
    def set_lambda(self, layer: int, lam) -> None:
        if isinstance(lam, torch.Tensor):
            lam = lam.detach().float().cpu().numpy()
        kvq_set_lambda(self.handle, layer, lam)

    def append(self, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        kvq_append(self.handle, layer, self._dev(k), self._dev(v), stream)

    def shrink(self, layer: int, stream=None) -> None:
        kvq_shrink(self.handle, layer, stream)

    def set_shift_mode(self, layer: int, mode: int) -> None:
        kvq_set_shift_mode(self.handle, layer, mode)

    def decode_attn(self, layer: int, q: torch.Tensor, sm_scale: Optional[float] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        q = self._dev(q)
        if sm_scale is None:
            sm_scale = HEAD_DIM ** -0.5
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        kvq_decode_attn(self.handle, layer, q, sm_scale, out, self.workspace(layer, q.shape[1]), stream)
        return out

    def append_decode(self, layer: int, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                      sm_scale: Optional[float] = None, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """append(layer, k, v) of one token per sequence, then decode_attn(layer, q), in one launch."""
        k, v, q = self._dev(k), self._dev(v), self._dev(q)
        if sm_scale is None:
            sm_scale = HEAD_DIM ** -0.5
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        kvq_append_decode(self.handle, layer, k, v, q, sm_scale, out, self.workspace(layer, q.shape[1]), stream)
        return out

    def query(self, layer: int) -> dict:
        return kvq_query(self.handle, layer)

    @property
    def max_tokens(self) -> int:
        return kvq_max_tokens(self.handle)

    def export(self, layer: int, b: int, j: int, stream=None):
        return kvq_export(self.handle, layer, b, j, stream, self.sink_window, self.key_channel)

    def export_window(self, layer: int, b: int, j: int, stream=None):
        return kvq_export_window(self.handle, layer, b, j, stream)

    def device_status(self, stream=None) -> None:
        kvq_device_status(self.handle, stream)

    def free(self) -> None:
        if getattr(self, "handle", None) is not None and self.handle.value:
            kvq_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass
