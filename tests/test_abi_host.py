"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol include/kvq.h declares, sizes the pool by the budget rule, and rejects
bad calls before touching the device."""
import ctypes as C
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def kvq():
    from mixed_precision_kv_kvq_b200 import build

    build.build()
    import mixed_precision_kv_kvq_b200 as m

    m.load()
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", src)))


def test_header_symbols_exported(kvq):
    lib = kvq.load()
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    from mixed_precision_kv_kvq_b200 import _lib
    assert set(names) == set(_lib.SIGNATURES)


def test_python_binding_has_same_names(kvq):
    for n in declared_functions():
        assert callable(getattr(kvq, n)), n


def _per_token(batch, kv_heads, fbit):
    return batch * kv_heads * 2 * sum(16 * f + 4 for f in fbit)


def test_pool_bytes_budget_rule(kvq):
    # tiny config: 1 block, batch 1, 2 KV heads, Fbit 4, room for 4096 tokens
    budget = 4096 * 2 * 2 * (64 + 4)
    assert budget == 1_114_112
    nb = kvq.kvq_pool_bytes(1, 1, 2, 128, budget, [4])
    codes_meta = 4096 * _per_token(1, 2, [4])
    assert codes_meta <= nb <= codes_meta + 8192
    # one byte less: the block drops to the next multiple of 512 tokens
    nb2 = kvq.kvq_pool_bytes(1, 1, 2, 128, budget - 1, [4])
    assert nb2 < nb and nb2 >= 3584 * _per_token(1, 2, [4])
    # 7B decode shape: 28 blocks, 4-bit for block 0 and the last 8, else 2-bit
    fbit = [4 if (l == 0 or l >= 20) else 2 for l in range(28)]
    per = _per_token(16, 4, fbit)
    nb = kvq.kvq_pool_bytes(28, 16, 4, 128, 32768 * per, fbit)
    assert 32768 * per <= nb <= 32768 * per + 28 * 8192 + 256


@pytest.mark.parametrize("args", [
    (0, 1, 2, 128, 10**9, [4]),        # no layers
    (1, 1, 2, 64, 10**9, [4]),         # head_dim != 128
    (1, 1, 2, 128, 10**9, [3]),        # fbit not a power of two in {2,4,8,16}
    (1, 1, 2, 128, 1000, [4]),         # budget below one 512-token tile
])
def test_pool_bytes_rejects(kvq, args):
    assert kvq.kvq_pool_bytes(*args) == 0


class HostPool:
    """A 256-byte aligned host buffer standing in for the device pool: with a
    caller pool, kvq_alloc and the validation paths make no CUDA call."""

    def __init__(self, nbytes):
        self.buf = np.zeros(nbytes + 512, np.uint8)
        base = self.buf.ctypes.data
        self.ptr = C.c_void_p(base + (-base) % 256)
        self.nbytes = nbytes


def _host_cache(kvq, layers=1, batch=1, kv_heads=2, budget=1_114_112, fbit=(4,)):
    lib = kvq.load()
    nb = kvq.kvq_pool_bytes(layers, batch, kv_heads, 128, budget, list(fbit))
    pool = HostPool(nb)
    h = C.c_void_p()
    fb = (C.c_int * layers)(*fbit)
    st = lib.kvq_alloc(C.byref(h), layers, batch, kv_heads, 128, budget, fb, pool.ptr, nb)
    assert st == 0, kvq.kvq_last_error()
    return h, pool


def test_alloc_initial_state_and_validation(kvq):
    lib = kvq.load()
    h, pool = _host_cache(kvq)
    try:
        assert kvq.kvq_max_tokens(h) == 4096
        assert kvq.kvq_query(h, 0) == {"tokens": 0, "bits": 16, "capacity": 1024, "n_shrinks": 0}
        dummy = C.c_void_p(pool.ptr.value)  # never dereferenced: every call below fails validation
        # more tokens than fit at Fbit -> BUDGET, nothing changes
        assert lib.kvq_append(h, 0, dummy, dummy, 0, 4097, None) == 2
        assert "4097" in kvq.kvq_last_error()
        assert kvq.kvq_query(h, 0)["tokens"] == 0
        # bad layer / dtype / negative count / null inputs -> INVALID
        assert lib.kvq_append(h, 1, dummy, dummy, 0, 1, None) == 1
        assert lib.kvq_append(h, 0, dummy, dummy, 7, 1, None) == 1
        assert lib.kvq_append(h, 0, dummy, dummy, 0, -1, None) == 1
        assert lib.kvq_append(h, 0, None, dummy, 0, 1, None) == 1
        assert lib.kvq_append(h, 0, dummy, dummy, 0, 0, None) == 0  # empty append is a no-op
        # shrink of a block that is not full -> STATE
        assert lib.kvq_shrink(h, 0, None) == 3
        # decode on an empty block -> STATE; GQA group above 8 -> INVALID
        assert lib.kvq_decode_attn(h, 0, dummy, 4, C.c_float(0.1), dummy, dummy, 1 << 30, None) == 3
        assert lib.kvq_decode_attn(h, 0, dummy, 18, C.c_float(0.1), dummy, dummy, 1 << 30, None) == 1
        assert lib.kvq_decode_attn(h, 0, dummy, 3, C.c_float(0.1), dummy, dummy, 1 << 30, None) == 1
        assert kvq.kvq_decode_workspace(h, 0, 18) == 0
        assert kvq.kvq_decode_workspace(h, 0, 4) > 0
        # lambda must be finite and positive (checked before any copy)
        bad = np.ones((2, 128), np.float32)
        bad[1, 5] = 0.0
        assert lib.kvq_set_lambda(h, 0, bad.ctypes.data_as(C.c_void_p)) == 1
        bad[1, 5] = np.nan
        assert lib.kvq_set_lambda(h, 0, bad.ctypes.data_as(C.c_void_p)) == 1
        # export of an out-of-range stream
        assert lib.kvq_export(h, 0, 1, 0, None, None, None, None, None) == 1
        # shift mode: two known modes, per block, before the first shrink
        assert lib.kvq_set_shift_mode(h, 0, 2) == 1
        assert lib.kvq_set_shift_mode(h, 1, 1) == 1
        assert lib.kvq_set_shift_mode(h, 0, kvq.KVQ_SHIFT_DIRECT) == 0
        assert lib.kvq_set_shift_mode(h, 0, kvq.KVQ_SHIFT_EQUIVALENT) == 0
    finally:
        kvq.kvq_free(h)


def test_alloc_rejects_small_pool(kvq):
    lib = kvq.load()
    nb = kvq.kvq_pool_bytes(1, 1, 2, 128, 1_114_112, [4])
    pool = HostPool(nb)
    h = C.c_void_p()
    fb = (C.c_int * 1)(4)
    assert lib.kvq_alloc(C.byref(h), 1, 1, 2, 128, 1_114_112, fb, pool.ptr, nb - 1) == 1
    assert lib.kvq_alloc(C.byref(h), 1, 1, 2, 128, 1_114_112, fb, C.c_void_p(pool.ptr.value + 8), nb) == 1
    assert lib.kvq_alloc(C.byref(h), 1, 1, 2, 128, 1000, fb, pool.ptr, nb) == 2


def test_per_layer_capacities(kvq):
    fbit = [2, 4, 8, 16]
    budget = 4096 * _per_token(2, 3, fbit)
    h, pool = _host_cache(kvq, layers=4, batch=2, kv_heads=3, budget=budget, fbit=fbit)
    try:
        assert kvq.kvq_max_tokens(h) == 4096
        # capacity at 16 bits is N * Fbit / 16
        assert [kvq.kvq_query(h, l)["capacity"] for l in range(4)] == [512, 1024, 2048, 4096]
    finally:
        kvq.kvq_free(h)


def test_window_option_host_side(kvq):
    """The sink + window option adds 5 tiles of 16 KiB and 1,280 bytes of meta
    per (sequence, KV head) and block to the pool, keeps the budget rule for
    the progressive cache, and rejects unknown option bits."""
    lib = kvq.load()
    budget = 4096 * _per_token(2, 3, [2, 4])
    plain = kvq.kvq_pool_bytes(2, 2, 3, 128, budget, [2, 4])
    win = kvq.kvq_pool_bytes_ex(2, 2, 3, 128, budget, [2, 4], kvq.KVQ_OPT_SINK_WINDOW)
    per_block = 2 * 3 * (5 * 16384 + 5 * 32 * 8)
    assert plain < win <= plain + 2 * (per_block + 2 * 256)
    assert kvq.kvq_pool_bytes_ex(2, 2, 3, 128, budget, [2, 4], 0) == plain
    assert kvq.kvq_pool_bytes_ex(2, 2, 3, 128, budget, [2, 4], 4) == 0
    pool = HostPool(win)
    h = C.c_void_p()
    fb = (C.c_int * 2)(2, 4)
    assert lib.kvq_alloc_ex(C.byref(h), 2, 2, 3, 128, budget, fb, pool.ptr, win, 4) == 1
    assert lib.kvq_alloc_ex(C.byref(h), 2, 2, 3, 128, budget, fb, pool.ptr, plain, 1) == 1  # pool too small
    assert lib.kvq_alloc_ex(C.byref(h), 2, 2, 3, 128, budget, fb, pool.ptr, win, 1) == 0
    try:
        assert kvq.kvq_max_tokens(h) == 4096 + 129
        assert kvq.kvq_query(h, 1) == {"tokens": 0, "bits": 16, "capacity": 1024 + 129, "n_shrinks": 0}
        n = C.c_int()
        assert lib.kvq_export_window(h, 0, 2, 0, None, None, None, None, C.byref(n), None) == 1  # stream
    finally:
        kvq.kvq_free(h)
    h2, pool2 = _host_cache(kvq)
    try:
        n = C.c_int()
        assert lib.kvq_export_window(h2, 0, 0, 0, None, None, None, None, C.byref(n), None) == 1  # no window
    finally:
        kvq.kvq_free(h2)


def test_key_channel_option_host_side(kvq):
    """Per-channel Key groups: N rounds down to a multiple of 1024, the pool
    adds the staging (the window storage) and one (R, Z) word per Key channel
    and 128-token block per stream; the option does not combine with the sink
    + window; capacity and max tokens count the staged block (127 more)."""
    lib = kvq.load()
    budget = 4096 * _per_token(2, 3, [2, 4])
    plain = kvq.kvq_pool_bytes(2, 2, 3, 128, budget, [2, 4])
    win = kvq.kvq_pool_bytes_ex(2, 2, 3, 128, budget, [2, 4], kvq.KVQ_OPT_SINK_WINDOW)
    ch = kvq.kvq_pool_bytes_ex(2, 2, 3, 128, budget, [2, 4], kvq.KVQ_OPT_KEY_CHANNEL)
    kmc = 2 * 2 * 3 * 4096 * 4  # layers * streams * N words
    assert ch == win + kmc or abs(ch - (win + kmc)) <= 2 * 256
    assert kvq.kvq_pool_bytes_ex(2, 2, 3, 128, budget, [2, 4], 3) == 0
    # 3584 tokens' budget: N = 3072 (a multiple of 1024), not 3584
    b2 = 3584 * _per_token(2, 3, [2, 4])
    pool = HostPool(kvq.kvq_pool_bytes_ex(2, 2, 3, 128, b2, [2, 4], kvq.KVQ_OPT_KEY_CHANNEL))
    h = C.c_void_p()
    fb = (C.c_int * 2)(2, 4)
    assert lib.kvq_alloc_ex(C.byref(h), 2, 2, 3, 128, b2, fb, pool.ptr, pool.nbytes, kvq.KVQ_OPT_KEY_CHANNEL) == 0
    try:
        assert kvq.kvq_max_tokens(h) == 3072 + 127
        assert kvq.kvq_query(h, 0) == {"tokens": 0, "bits": 16, "capacity": 3072 * 2 // 16 + 127, "n_shrinks": 0}
        n = C.c_int()
        assert lib.kvq_export_window(h, 0, 2, 0, None, None, None, None, C.byref(n), None) == 1  # stream
    finally:
        kvq.kvq_free(h)


def test_injected_allocation_failure(kvq, monkeypatch):
    """KVQ_FAULT_ALLOC makes the library's own pool allocation fail on the
    host, before any CUDA call: kvq_alloc returns KVQ_ERR_OOM, hands back no
    cache and says the failure was injected; a caller-owned pool is not
    affected (the library allocates nothing then), and "0" turns it off."""
    lib = kvq.load()
    fb = (C.c_int * 1)(4)
    monkeypatch.setenv("KVQ_FAULT_ALLOC", "1")
    h = C.c_void_p(1234)
    assert lib.kvq_alloc(C.byref(h), 1, 1, 2, 128, 1_114_112, fb, None, 0) == 4
    assert h.value is None
    msg = kvq.kvq_last_error()
    assert "injected" in msg and "KVQ_FAULT_ALLOC" in msg
    hc, pool = _host_cache(kvq)  # caller pool: succeeds with the hook set
    kvq.kvq_free(hc)
    monkeypatch.setenv("KVQ_FAULT_ALLOC", "0")
    st = lib.kvq_alloc(C.byref(h), 1, 1, 2, 128, 1_114_112, fb, None, 0)
    if st == 0:  # a GPU is present: the real allocation went through
        kvq.kvq_free(h)
    else:
        assert st == 4 and "injected" not in kvq.kvq_last_error()
