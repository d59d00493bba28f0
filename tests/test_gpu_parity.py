"""GPU parity: libkvq (through its C ABI) against the CPU oracle on the same
seeded inputs.  Codes and meta must be bit-exact; attention output must be
within a max relative error of 2e-3 per (sequence, query head):
    max_c |o - o*| / max_c |o*|  <=  2e-3
(the oracle attends over its own codes, which equal the GPU's)."""
import math

import numpy as np
import pytest
import torch

import kvq_synth as S

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixed_precision_kv_kvq_b200 import build

    build.build()
    import mixed_precision_kv_kvq_b200 as m

    m.load()
    return m


def per_token(batch, kv_heads, fbit):
    return batch * kv_heads * 2 * sum(16 * f + 4 for f in fbit)


class Pair:
    """A GPU cache and the oracle's model of the same block, fed identically."""

    def __init__(self, kvq, orc, batch, kv_heads, n_f, fbit, lam=None, shift_mode=0):
        self.batch, self.kv_heads, self.n_f, self.fbit = batch, kv_heads, n_f, fbit
        self.gpu = kvq.KVQCache(1, batch, kv_heads, n_f * per_token(batch, kv_heads, [fbit]), [fbit])
        assert self.gpu.max_tokens == n_f
        self.orc = orc.Layer(batch, kv_heads, n_f, fbit)
        self.lam = lam
        if lam is not None:
            self.gpu.set_lambda(0, lam)
        if shift_mode:
            self.gpu.set_shift_mode(0, shift_mode)
            assert self.orc.set_shift_mode(shift_mode) == 0

    def append(self, k, v):
        """k, v: CPU tensors [batch][n][kv_heads][128] (bf16 or fp32)."""
        self.gpu.append(0, k.cuda(), v.cuda())
        rc = self.orc.append(k.float().numpy(), v.float().numpy(), self.lam)
        assert rc == 0

    def check_codes(self, streams=None):
        q = self.gpu.query(0)
        assert q["tokens"] == self.orc.n and q["bits"] == self.orc.bits
        assert q["n_shrinks"] == self.orc.n_shrinks
        okc, ovc, okm, ovm = self.orc.k_codes(), self.orc.v_codes(), self.orc.k_meta(), self.orc.v_meta()
        streams = streams or [(b, j) for b in range(self.batch) for j in range(self.kv_heads)]
        for b, j in streams:
            kc, vc, km, vm = self.gpu.export(0, b, j)
            assert np.array_equal(km, okm[b, j]), (b, j, "k meta")
            assert np.array_equal(vm, ovm[b, j]), (b, j, "v meta")
            if not np.array_equal(kc, okc[b, j]):
                bad = np.argwhere(kc != okc[b, j])
                raise AssertionError(f"K codes differ at {len(bad)} places, first {bad[:5].tolist()}")
            if not np.array_equal(vc, ovc[b, j]):
                bad = np.argwhere(vc != ovc[b, j])
                raise AssertionError(f"V codes differ at {len(bad)} places, first {bad[:5].tolist()}")

    def check_attention(self, q, sm_scale=None):
        """q: CPU bf16 [batch][q_heads][128]."""
        sm_scale = sm_scale if sm_scale is not None else 1 / math.sqrt(128)
        out = self.gpu.decode_attn(0, q.cuda(), sm_scale).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        self.gpu.device_status()
        ref = self.orc.attention(q.float().numpy(), self.lam, sm_scale)
        err = np.abs(out - ref).max(axis=-1) / np.abs(ref).max(axis=-1)
        assert np.isfinite(out).all()
        assert err.max() <= TOL, f"max rel err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"
        return float(err.max())


def lam_for(k):
    from oracle import oracle as orc
    return orc.lambda_from_keys(k.float()[0].numpy(), 0.5)


def test_tiny_config_progressive_one_by_one(kvq, orc):
    """1 block, batch 1, 2 KV heads, 4 query heads, Fbit 4, 4096 fp32 tokens
    appended one at a time: 16 bits to 1024, 8 bits to 2048, then 4 bits.
    Codes/meta bit-exact and attention within tolerance after every shrink."""
    T = 4096
    k, v = S.keys_values(0, 0, 1, T, 2, 0, 4, dtype=torch.float32)
    lam = lam_for(k)
    P = Pair(kvq, orc, 1, 2, 4096, 4, lam)
    checkpoints = {1000, 1024, 1025, 1500, 2048, 2049, 3000, 4096}
    step = 0
    for t in range(T):
        P.append(k[:, t:t + 1], v[:, t:t + 1])
        if t + 1 in checkpoints:
            P.check_codes()
            q = S.queries(0, 0, step, 1, 4, t + 1, dtype=torch.bfloat16)
            P.check_attention(q)
            step += 1
    assert P.orc.shrink_at == [1024, 2048]
    assert kvq.kvq_query(P.gpu.handle, 0) == {"tokens": 4096, "bits": 4, "capacity": 4096, "n_shrinks": 2}
    for s in range(16):  # 16 decode queries at the end
        P.check_attention(S.queries(0, 0, 100 + s, 1, 4, T, dtype=torch.bfloat16))
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.append(0, k[:, :1].cuda(), v[:, :1].cuda())
    assert e.value.status == 2


@pytest.mark.parametrize("fbit,chunks", [
    (2, [700, 300, 600, 1000, 1000, 400, 96]),   # crosses 16->8->4->2 inside chunks
    (8, [1, 15, 16, 17, 2000]),
    (16, [63, 65, 512, 1]),
])
def test_chunked_append_bit_exact(kvq, orc, fbit, chunks):
    B, H = 2, 3
    n_f = 4096
    P = Pair(kvq, orc, B, H, n_f, fbit, None)
    pos = 0
    for i, n in enumerate(chunks):
        if pos + n > n_f:
            break
        k, v = S.keys_values(1, i, B, n, H, pos, 3, dtype=torch.bfloat16)
        P.append(k, v)
        pos += n
        P.check_codes(streams=[(0, 0), (1, 2)])
    P.check_codes()


@pytest.mark.parametrize("fbit", [2, 4, 8])
def test_chunked_append_fp32_group_mode(kvq, orc, fbit):
    """fp32 inputs with lambda in chunks whose whole 16-token groups take the
    group-mode append at 8, 4 and 2 bits (and whose unaligned heads and tails
    take the per-token path): codes and meta bit-exact, attention within 2e-3."""
    B, H, n_f = 2, 3, 4096
    cap16 = n_f * fbit // 16
    k, v = S.keys_values(17, fbit, B, n_f, H, 0, 4, dtype=torch.float32)
    lam = lam_for(k)
    P = Pair(kvq, orc, B, H, n_f, fbit, lam)
    pos = 0
    for n in (cap16, 5, 250, 37, 1000, 333, n_f):
        n = min(n, n_f - pos)
        if n <= 0:
            break
        P.append(k[:, pos:pos + n], v[:, pos:pos + n])
        pos += n
        P.check_codes(streams=[(0, 0), (1, 2)])
    assert pos == n_f and P.gpu.query(0)["bits"] == fbit
    P.check_codes()
    P.check_attention(S.queries(17, fbit, 0, B, 4 * H, n_f, dtype=torch.bfloat16))


@pytest.mark.parametrize("G", [1, 2, 3, 5, 7, 8])
@pytest.mark.parametrize("T,fbit", [(1, 2), (17, 2), (300, 4), (1500, 4), (3000, 2), (4096, 2)])
def test_decode_attention(kvq, orc, G, T, fbit):
    B, H = 2, 2
    k, v = S.keys_values(2, T, B, T, H, 0, 3, dtype=torch.bfloat16)
    lam = lam_for(k)
    P = Pair(kvq, orc, B, H, 4096, fbit, lam)
    P.append(k, v)
    q = S.queries(2, T, 0, B, H * G, T, dtype=torch.bfloat16)
    P.check_attention(q)


def test_forced_shrink_matches_oracle(kvq, orc):
    B, H = 1, 2
    P = Pair(kvq, orc, B, H, 4096, 2, None)
    k, v = S.keys_values(3, 0, B, 512, H, 0, 2, dtype=torch.float32)
    P.append(k, v)  # 512 = capacity at 16 bits for Fbit 2
    assert P.gpu.query(0)["capacity"] == 512
    P.gpu.shrink(0)
    assert P.orc.shrink() == 0
    P.check_codes()
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.shrink(0)  # not full at 8 bits
    assert e.value.status == 3
    P.check_attention(S.queries(3, 0, 0, B, 4, 512))


def test_bounded_wait_gives_up_and_reports(kvq, orc):
    """The decode kernel's bounded wait, run on a barrier no copy completes
    (kvq_selftest_timeout): after its time limit the kernel returns, the
    next device status is KVQ_ERR_TIMEOUT, and the cache keeps working."""
    import time
    P = Pair(kvq, orc, 1, 2, 4096, 4, None)
    k, v = S.keys_values(18, 0, 1, 300, 2, 0, 2, dtype=torch.bfloat16)
    P.append(k, v)
    t0 = time.time()
    kvq.kvq_selftest_timeout(P.gpu.handle)
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.device_status()
    assert e.value.status == 7 and time.time() - t0 >= 1.5
    P.gpu.device_status()  # cleared
    P.check_codes()
    P.check_attention(S.queries(18, 0, 0, 1, 4, 300, dtype=torch.bfloat16))


def test_decode_rejects_small_workspace(kvq, orc):
    P = Pair(kvq, orc, 1, 2, 4096, 4, None)
    k, v = S.keys_values(4, 0, 1, 10, 2, 0, 1, dtype=torch.float32)
    P.append(k, v)
    q = S.queries(4, 0, 0, 1, 4, 10).cuda()
    out = torch.empty(1, 4, 128, device="cuda")
    ws = torch.empty(16, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attn(P.gpu.handle, 0, q, 0.1, out, ws)
    assert e.value.status == 6


def test_empty_block_and_full_budget_edges(kvq, orc):
    """Empty block: decode is refused (STATE) and writes nothing; a zero-token
    append is a no-op.  A block filled to exactly its Fbit capacity matches the
    oracle (two shrinks on the way); one token more -- alone or fused with a
    decode -- is refused (BUDGET) and changes neither codes, meta nor state."""
    n_f, B, H, Hq = 1024, 2, 2, 6
    P = Pair(kvq, orc, B, H, n_f, 4, None)
    q = S.queries(21, 0, 0, B, Hq, n_f, dtype=torch.bfloat16)
    out = torch.full((B, Hq, 128), 7.0, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.decode_attn(0, q.cuda(), out=out)
    assert e.value.status == 3
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    empty = torch.empty(B, 0, H, 128, dtype=torch.bfloat16, device="cuda")
    P.gpu.append(0, empty, empty)
    assert P.gpu.query(0)["tokens"] == 0
    k, v = S.keys_values(21, 0, B, n_f + 1, H, 0, 3, dtype=torch.bfloat16)
    for a0, a1 in [(0, 200), (200, 300), (300, 550), (550, n_f)]:
        P.append(k[:, a0:a1], v[:, a0:a1])
    assert P.orc.shrink_at == [256, 512]  # a chunk is split where the next token would not fit
    P.check_codes()
    P.check_attention(q)
    before = [P.gpu.export(0, b, j) for b in range(B) for j in range(H)]
    assert P.orc.append(k[:, n_f:].float().numpy(), v[:, n_f:].float().numpy(), None) == 1
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.append(0, k[:, n_f:].cuda(), v[:, n_f:].cuda())
    assert e.value.status == 2
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.append_decode(0, k[:, n_f:, :, :].cuda(), v[:, n_f:].cuda(), q.cuda(), out=out)
    assert e.value.status == 2
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    qs = P.gpu.query(0)
    assert qs["tokens"] == n_f and qs["bits"] == 4 and qs["n_shrinks"] == 2
    after = [P.gpu.export(0, b, j) for b in range(B) for j in range(H)]
    for x, y in zip(before, after):
        for a, b in zip(x, y):
            assert np.array_equal(a, b)
    P.check_codes()
    P.check_attention(q)


@pytest.mark.parametrize("fbit", [2, 4])
@pytest.mark.parametrize("bad", [float("inf"), -70000.0])
def test_group_append_contains_a_non_finite_group(kvq, orc, fbit, bad):
    """A chunk taken in group mode holds groups outside the append contract:
    a Value with an infinite channel (R = inf, NaN scaled values) or a minimum
    below -65504 (Z = -inf), and a Key with an infinite channel.  Their own
    codes are unspecified; every other token's codes and meta must equal the
    oracle's (fed the finite originals) and a one-token-at-a-time append of the
    same chunk."""
    B, H, n_f = 1, 2, 4096
    pre = n_f // 2  # the capacity at 2 * fbit bits: the chunk shrinks the block to fbit first
    k, v = S.keys_values(23, fbit, B, pre + 48, H, 0, 3, dtype=torch.float32)
    P = Pair(kvq, orc, B, H, n_f, fbit, None)
    one = kvq.KVQCache(1, B, H, n_f * per_token(B, H, [fbit]), [fbit])
    P.append(k[:, :pre], v[:, :pre])
    one.append(0, k[:, :pre].cuda(), v[:, :pre].cuda())
    kb, vb = k[:, pre:].clone(), v[:, pre:].clone()
    bad_v, bad_k = 21, 30  # tokens of the chunk; the V of token 21 shares its words with token 20's
    vb[0, bad_v, 1, 9] = bad
    kb[0, bad_k, 0, 3] = float("inf")
    P.gpu.append(0, kb.cuda(), vb.cuda())  # the non-finite chunk goes to the GPU only
    assert P.orc.append(k[:, pre:].numpy(), v[:, pre:].numpy(), None) == 0
    for t in range(48):
        one.append(0, kb[:, t:t + 1].cuda(), vb[:, t:t + 1].cuda())
    torch.cuda.synchronize()
    assert P.gpu.query(0)["bits"] == fbit and P.gpu.query(0)["tokens"] == pre + 48
    okc, ovc, okm, ovm = P.orc.k_codes(), P.orc.v_codes(), P.orc.k_meta(), P.orc.v_meta()
    for j in range(H):
        kc, vc, km, vm = P.gpu.export(0, 0, j)
        kc1, vc1, km1, vm1 = one.export(0, 0, j)
        keep_k = np.ones(pre + 48, bool)
        keep_v = np.ones(pre + 48, bool)
        if j == 0:
            keep_k[pre + bad_k] = False
        if j == 1:
            keep_v[pre + bad_v] = False
        for got, ref, keep in ((kc, okc[0, j], keep_k), (km, okm[0, j], keep_k), (vc, ovc[0, j], keep_v),
                               (vm, ovm[0, j], keep_v), (kc1, okc[0, j], keep_k), (vc1, ovc[0, j], keep_v)):
            assert np.array_equal(got[keep], ref[keep])
        assert int(vc[~keep_v].max(initial=0)) < (1 << fbit) and int(kc[~keep_k].max(initial=0)) < (1 << fbit)
    one.free()


# ---------------------------------------------------- Direct Right Shift (ablation)

def test_direct_shift_tiny_config_one_by_one(kvq, orc):
    """The tiny configuration with the ablation's Direct Right Shift: the same
    schedule (16 -> 8 at 1024, 8 -> 4 at 2048); codes = X >> b and rescaled
    ranges bit-exact after every shrink; attention within tolerance."""
    T = 2100
    k, v = S.keys_values(5, 0, 1, T, 2, 0, 4, dtype=torch.float32)
    lam = lam_for(k)
    P = Pair(kvq, orc, 1, 2, 4096, 4, lam, shift_mode=kvq.KVQ_SHIFT_DIRECT)
    checkpoints = {1024, 1025, 2048, 2049, 2100}
    for t in range(T):
        P.append(k[:, t:t + 1], v[:, t:t + 1])
        if t + 1 in checkpoints:
            P.check_codes()
            P.check_attention(S.queries(5, 0, t, 1, 4, t + 1, dtype=torch.bfloat16))
    assert P.orc.shrink_at == [1024, 2048]
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.set_shift_mode(0, kvq.KVQ_SHIFT_EQUIVALENT)  # fixed once the block has shrunk
    assert e.value.status == 3


@pytest.mark.parametrize("fbit", [2, 8])
def test_direct_shift_chunked_bf16(kvq, orc, fbit):
    """Chunks crossing every shrink of a 2-bit block (16 -> 8 -> 4 -> 2) and an
    8-bit one, batch 3, 4 KV heads, bf16 inputs, Direct Right Shift."""
    B, H, n_f = 3, 4, 4096
    cap16 = n_f * fbit // 16
    k, v = S.keys_values(6, fbit, B, n_f, H, 0, 5, dtype=torch.bfloat16)
    lam = lam_for(k)
    P = Pair(kvq, orc, B, H, n_f, fbit, lam, shift_mode=kvq.KVQ_SHIFT_DIRECT)
    pos = 0
    for n in (cap16 - 7, 300, 900, 1600, n_f):
        n = min(n, n_f - pos)
        if n <= 0:
            break
        P.append(k[:, pos:pos + n], v[:, pos:pos + n])
        pos += n
    assert P.gpu.query(0)["bits"] == fbit and pos == n_f
    P.check_codes()
    P.check_attention(S.queries(6, fbit, 0, B, 4 * H, n_f, dtype=torch.bfloat16))


# ------------------------------------------ sink token + recent window at INT16

class WPair:
    """A GPU cache made with the sink + window option and the oracle's
    windowed block, fed identically."""

    def __init__(self, kvq, orc, batch, kv_heads, n_f, fbit, lam=None, shift_mode=0):
        self.kvq = kvq
        self.batch, self.kv_heads = batch, kv_heads
        self.gpu = kvq.KVQCache(1, batch, kv_heads, n_f * per_token(batch, kv_heads, [fbit]), [fbit],
                                sink_window=True)
        assert self.gpu.max_tokens == n_f + 129
        self.orc = orc.WLayer(batch, kv_heads, n_f, fbit)
        self.lam = lam
        if lam is not None:
            self.gpu.set_lambda(0, lam)
        if shift_mode:
            self.gpu.set_shift_mode(0, shift_mode)
            assert self.orc.set_shift_mode(shift_mode) == 0

    def append(self, k, v):
        self.gpu.append(0, k.cuda(), v.cuda())
        assert self.orc.append(k.float().numpy(), v.float().numpy(), self.lam) == 0

    def check_codes(self):
        q = self.gpu.query(0)
        m = self.orc.main
        assert (q["tokens"], q["bits"], q["n_shrinks"]) == (self.orc.n, m.bits, m.n_shrinks), (q, m.shrink_at)
        okc, ovc, okm, ovm = m.k_codes(), m.v_codes(), m.k_meta(), m.v_meta()
        wkc, wvc, wkm, wvm = self.orc.window_codes()
        for b in range(self.batch):
            for j in range(self.kv_heads):
                kc, vc, km, vm = self.gpu.export(0, b, j)
                assert kc.shape[0] == m.n
                for name, got, want in (("K", kc, okc[b, j]), ("V", vc, ovc[b, j]), ("K meta", km, okm[b, j]),
                                        ("V meta", vm, ovm[b, j])):
                    assert np.array_equal(got, want), (b, j, name, np.argwhere(got != want)[:4].tolist())
                kc, vc, km, vm = self.gpu.export_window(0, b, j)
                for name, got, want in (("window K", kc, wkc[b, j]), ("window V", vc, wvc[b, j]),
                                        ("window K meta", km, wkm[b, j]), ("window V meta", vm, wvm[b, j])):
                    assert np.array_equal(got, want), (b, j, name, np.argwhere(got != want)[:4].tolist())

    def check_attention(self, q, sm_scale=1 / math.sqrt(128)):
        out = self.gpu.decode_attn(0, q.cuda(), sm_scale).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        self.gpu.device_status()
        ref = self.orc.attention(q.float().numpy(), self.lam, sm_scale)
        err = np.abs(out - ref).max(axis=-1) / np.abs(ref).max(axis=-1)
        assert np.isfinite(out).all()
        assert err.max() <= TOL, f"max rel err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"


def test_window_tiny_one_by_one(kvq, orc):
    """Token by token through: window filling (progressive cache empty),
    the first move (token 129), and two shrinks of the progressive cache
    (at 128 and 256 of its tokens); codes bit-exact, attention within 2e-3."""
    T = 600
    k, v = S.keys_values(7, 0, 1, T, 2, 0, 4, dtype=torch.float32)
    lam = lam_for(k)
    P = WPair(kvq, orc, 1, 2, 512, 4, lam)
    checkpoints = {1, 2, 128, 129, 130, 131, 257, 258, 385, 386, 600}
    for t in range(T):
        P.append(k[:, t:t + 1], v[:, t:t + 1])
        if t + 1 in checkpoints:
            P.check_codes()
            P.check_attention(S.queries(7, 0, t, 1, 4, t + 1, dtype=torch.bfloat16))
    assert P.orc.main.shrink_at == [128, 256]


@pytest.mark.parametrize("fbit,mode", [(2, 0), (2, 1), (8, 0)])
def test_window_chunked_bf16(kvq, orc, fbit, mode):
    """Chunks of every size around the window (1 .. 700 tokens: launches are
    cut at 128 tokens and at the progressive cache's capacity), batch 3,
    4 KV heads, through every shrink of the block, either shift."""
    B, H, n_f = 3, 4, 1024
    total = n_f + 129
    k, v = S.keys_values(8, fbit, B, total, H, 0, 5, dtype=torch.bfloat16)
    lam = lam_for(k)
    P = WPair(kvq, orc, B, H, n_f, fbit, lam, shift_mode=mode)
    pos = 0
    for n in (1, 127, 1, 129, 300, 5, 700, total):
        n = min(n, total - pos)
        if n <= 0:
            break
        P.append(k[:, pos:pos + n], v[:, pos:pos + n])
        pos += n
        if pos in (1, 128, 258, 563):
            P.check_codes()
    assert pos == total and P.gpu.query(0)["bits"] == fbit
    P.check_codes()
    P.check_attention(S.queries(8, fbit, 0, B, 4 * H, total, dtype=torch.bfloat16))
    with pytest.raises(kvq.KVQError) as e:  # the progressive cache is full at Fbit
        P.gpu.append(0, k[:, :1].cuda(), v[:, :1].cuda())
    assert e.value.status == 2


def test_window_noalloc_matches_workspace_entry(kvq, orc):
    """The no-workspace entry point on a cache with the sink + window: the same
    two launches, the same result as kvq_decode_attn."""
    B, H, G = 2, 2, 4
    T = 700
    k, v = S.keys_values(9, 0, B, T, H, 0, 3, dtype=torch.bfloat16)
    P = WPair(kvq, orc, B, H, 1024, 2, lam_for(k))
    P.append(k, v)
    q = S.queries(9, 0, 0, B, H * G, T, dtype=torch.bfloat16).cuda()
    ref = P.gpu.decode_attn(0, q)
    out = torch.empty_like(ref)
    kvq.kvq_decode_attn_noalloc(P.gpu.handle, 0, q, 128 ** -0.5, out)
    torch.cuda.synchronize()
    assert torch.allclose(out, ref, rtol=0, atol=0)
    P.check_attention(q.cpu())


# ------------------------------------------------ per-channel Key groups

class CPair:
    """A GPU cache with per-channel Key groups (KVQ_OPT_KEY_CHANNEL) and the
    oracle's channel block, fed identically."""

    def __init__(self, kvq, orc, batch, kv_heads, n_f, fbit, lam=None, shift_mode=0):
        self.kvq = kvq
        self.batch, self.kv_heads = batch, kv_heads
        self.gpu = kvq.KVQCache(1, batch, kv_heads, n_f * per_token(batch, kv_heads, [fbit]), [fbit],
                                key_channel=True)
        assert self.gpu.max_tokens == n_f + 127
        self.orc = orc.CLayer(batch, kv_heads, n_f, fbit)
        self.lam = lam
        if lam is not None:
            self.gpu.set_lambda(0, lam)
        if shift_mode:
            self.gpu.set_shift_mode(0, shift_mode)
            assert self.orc.set_shift_mode(shift_mode) == 0

    def append(self, k, v):
        self.gpu.append(0, k.cuda(), v.cuda())
        assert self.orc.append(k.float().numpy(), v.float().numpy(), self.lam) == 0

    def check_codes(self):
        q = self.gpu.query(0)
        m = self.orc.main
        assert (q["tokens"], q["bits"], q["n_shrinks"]) == (self.orc.n, m.bits, m.n_shrinks), (q, m.shrink_at)
        okc, ovc, ovm = m.k_codes(), m.v_codes(), m.v_meta()
        okm = self.orc.k_meta_channel().reshape(self.batch, self.kv_heads, -1, 2)
        skc, svc, skm, svm = self.orc.staged_codes()
        for b in range(self.batch):
            for j in range(self.kv_heads):
                kc, vc, km, vm = self.gpu.export(0, b, j)
                assert kc.shape[0] == m.n
                for name, got, want in (("K", kc, okc[b, j]), ("V", vc, ovc[b, j]),
                                        ("K channel meta", km, okm[b, j]), ("V meta", vm, ovm[b, j])):
                    assert np.array_equal(got, want), (b, j, name, np.argwhere(got != want)[:4].tolist())
                kc, vc, km, vm = self.gpu.export_window(0, b, j)
                for name, got, want in (("staged K", kc, skc[b, j]), ("staged V", vc, svc[b, j]),
                                        ("staged K meta", km, skm[b, j]), ("staged V meta", vm, svm[b, j])):
                    assert np.array_equal(got, want), (b, j, name, np.argwhere(got != want)[:4].tolist())

    def check_attention(self, q, sm_scale=1 / math.sqrt(128)):
        out = self.gpu.decode_attn(0, q.cuda(), sm_scale).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        self.gpu.device_status()
        ref = self.orc.attention(q.float().numpy(), self.lam, sm_scale)
        err = np.abs(out - ref).max(axis=-1) / np.abs(ref).max(axis=-1)
        assert np.isfinite(out).all()
        assert err.max() <= TOL, f"max rel err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"
        return out


def test_key_channel_tiny_one_by_one(kvq, orc):
    """Token by token: the staged block alone, the first block entering the
    progressive cache at 16 bits, and the cache shrinking as the 2nd, 3rd and
    5th blocks arrive (N = 1024, Fbit 2), up to the last token that fits;
    codes and meta bit-exact, attention within 2e-3."""
    T = 1024 + 127
    k, v = S.keys_values(11, 0, 1, T, 2, 0, 4, dtype=torch.float32)
    lam = lam_for(k)
    P = CPair(kvq, orc, 1, 2, 1024, 2, lam)
    checkpoints = {1, 2, 127, 128, 129, 255, 256, 257, 384, 512, 513, 640, 1024, 1025, T}
    for t in range(T):
        P.append(k[:, t:t + 1], v[:, t:t + 1])
        if t + 1 in checkpoints:
            P.check_codes()
            P.check_attention(S.queries(11, 0, t, 1, 4, t + 1, dtype=torch.bfloat16))
    assert P.orc.main.shrink_at == [128, 256, 512]
    with pytest.raises(kvq.KVQError) as e:  # the 9th block does not fit at Fbit
        P.gpu.append(0, k[:, :1].cuda(), v[:, :1].cuda())
    assert e.value.status == 2


@pytest.mark.parametrize("fbit,mode", [(2, 0), (2, 1), (4, 0), (8, 1)])
def test_key_channel_chunked_bf16(kvq, orc, fbit, mode):
    """Chunks of 1 .. 700 tokens (launches are cut at block ends), batch 3,
    4 KV heads, through every shrink of the block with either shift; then
    the budget refuses a block that does not fit at Fbit."""
    B, H, n_f = 3, 4, 2048
    total = n_f + 127
    k, v = S.keys_values(12, fbit, B, total, H, 0, 5, dtype=torch.bfloat16)
    lam = lam_for(k)
    P = CPair(kvq, orc, B, H, n_f, fbit, lam, shift_mode=mode)
    pos = 0
    for n in (1, 126, 1, 129, 300, 5, 700, total):
        n = min(n, total - pos)
        if n <= 0:
            break
        P.append(k[:, pos:pos + n], v[:, pos:pos + n])
        pos += n
        if pos in (1, 128, 257, 562):
            P.check_codes()
            P.check_attention(S.queries(12, fbit, pos, B, 4 * H, pos, dtype=torch.bfloat16))
    assert pos == total and P.gpu.query(0)["bits"] == fbit
    P.check_codes()
    P.check_attention(S.queries(12, fbit, 0, B, 4 * H, total, dtype=torch.bfloat16))
    with pytest.raises(kvq.KVQError) as e:
        P.gpu.append(0, k[:, :1].cuda(), v[:, :1].cuda())
    assert e.value.status == 2


@pytest.mark.parametrize("mode", [0, 1])
def test_key_channel_whole_blocks_fp32(kvq, orc, mode):
    """fp32 inputs in calls of whole, aligned blocks (each block goes from the
    input straight into the progressive cache, nothing staged), through the
    shrinks of a Fbit-4 block with either shift, then a partial call that
    stages tokens: codes, meta and staged records bit-exact, attention within
    2e-3."""
    B, H, n_f = 2, 3, 1024
    T = n_f + 77
    k, v = S.keys_values(21, mode, B, T, H, 0, 3, dtype=torch.float32)
    P = CPair(kvq, orc, B, H, n_f, 4, lam_for(k), shift_mode=mode)
    pos = 0
    for n in (128, 256, 128, 512, 77):
        P.append(k[:, pos:pos + n], v[:, pos:pos + n])
        pos += n
        if n != 512:
            P.check_codes()
            P.check_attention(S.queries(21, mode, pos, B, 2 * H, pos, dtype=torch.bfloat16))
    assert pos == T and P.gpu.query(0)["bits"] == 4 and P.orc.main.shrink_at
    P.check_codes()
    P.check_attention(S.queries(21, mode, 0, B, 2 * H, T, dtype=torch.bfloat16))


@pytest.mark.parametrize("G", [1, 5, 8])
def test_key_channel_many_blocks_and_splits(kvq, orc, G):
    """A longer block (N = 8192 at Fbit 2, every epoch present, several CTAs
    per stream with warps on different blocks), GQA group sizes 1, 5, 8; the
    no-workspace entry point gives the same output."""
    B, H, n_f = 2, 2, 8192
    T = n_f + 100
    k, v = S.keys_values(13, G, B, T, H, 0, 3, dtype=torch.bfloat16)
    P = CPair(kvq, orc, B, H, n_f, 2, lam_for(k))
    for t0 in range(0, T, 4096):
        P.append(k[:, t0:t0 + 4096], v[:, t0:t0 + 4096])
    P.check_codes()
    q = S.queries(13, G, 0, B, H * G, T, dtype=torch.bfloat16)
    ref = P.check_attention(q)
    out = torch.empty(B, H * G, 128, device="cuda")
    kvq.kvq_decode_attn_noalloc(P.gpu.handle, 0, q.cuda(), 128 ** -0.5, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("mode", [0, 1])
def test_key_channel_explicit_shrink(kvq, orc, mode):
    """kvq_shrink on a full progressive cache with per-channel Key groups (the
    step the next block would take; the direct shift also rescales the
    per-channel ranges): after the next block the cache equals the oracle's,
    which shrinks when that block arrives; a shrink of a cache that is not
    full, or at Fbit, is refused."""
    B, H = 2, 2
    k, v = S.keys_values(15, mode, B, 400, H, 0, 3, dtype=torch.bfloat16)
    P = CPair(kvq, orc, B, H, 1024, 2, lam_for(k), shift_mode=mode)  # 128 tokens at 16 bits
    P.append(k[:, :100], v[:, :100])
    with pytest.raises(kvq.KVQError) as e:  # the progressive cache is empty, not full
        P.gpu.shrink(0)
    assert e.value.status == 3
    P.append(k[:, 100:200], v[:, 100:200])  # block 0 in the cache: full at 16 bits
    P.gpu.shrink(0)
    assert P.gpu.query(0)["bits"] == 8 and P.orc.main.bits == 16
    P.append(k[:, 200:300], v[:, 200:300])  # block 1 completes at 256: no second shrink on the GPU
    assert P.gpu.query(0)["n_shrinks"] == 1 and P.orc.main.n_shrinks == 1
    P.check_codes()
    P.check_attention(S.queries(15, mode, 0, B, 4 * H, 300, dtype=torch.bfloat16))


def test_key_channel_append_decode_is_two_calls(kvq, orc):
    """kvq_append_decode on a cache with per-channel Key groups runs the two
    calls: same output and state as append then decode, across a block end."""
    B, H, G, n_f = 2, 2, 4, 1024
    t0, steps = 250, 10
    k, v = S.keys_values(14, 0, B, t0 + steps, H, 0, 3, dtype=torch.bfloat16)
    lam = lam_for(k)
    P = CPair(kvq, orc, B, H, n_f, 4, lam)
    F = kvq.KVQCache(1, B, H, n_f * per_token(B, H, [4]), [4], key_channel=True)
    F.set_lambda(0, lam)
    P.append(k[:, :t0], v[:, :t0])
    F.append(0, k[:, :t0].cuda(), v[:, :t0].cuda())
    for s_ in range(steps):
        t = t0 + s_
        q = S.queries(14, 0, s_, B, H * G, t + 1, dtype=torch.bfloat16)
        P.append(k[:, t:t + 1], v[:, t:t + 1])
        ref = P.check_attention(q)
        out = F.append_decode(0, k[:, t:t + 1].cuda(), v[:, t:t + 1].cuda(), q.cuda())
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)
    assert F.query(0) == P.gpu.query(0)
    F.free()


# ------------------------------------------------ one stream: the most CTAs per stream

@pytest.mark.parametrize("mode", ["plain", "window", "chan"])
def test_single_stream_most_splits(kvq, orc, mode):
    """Batch 1 and one KV head: a long block is cut into the largest number
    of CTAs per stream (64 partials, or 61 plus the window's or staged
    block's 3), and the merge over all of them matches the oracle."""
    B, H, G, n_f, fbit = 1, 1, 8, 65536, 4  # 4096 groups at 4 bits: the split model wants more than 64
    T = n_f + (100 if mode == "chan" else (129 if mode == "window" else 0))
    k, v = S.keys_values(16, 1, B, T, H, 0, 2, dtype=torch.bfloat16)
    lam = lam_for(k)
    if mode == "window":
        P = WPair(kvq, orc, B, H, n_f, fbit, lam)
    elif mode == "chan":
        P = CPair(kvq, orc, B, H, n_f, fbit, lam)
    else:
        P = Pair(kvq, orc, B, H, n_f, fbit, lam)
    for t0 in range(0, T, 8192):
        P.append(k[:, t0:t0 + 8192], v[:, t0:t0 + 8192])
    P.check_attention(S.queries(16, 1, 0, B, H * G, T, dtype=torch.bfloat16))


# ------------------------------------------------ fused single-token append + decode

@pytest.mark.parametrize("fbit,t0,steps,dtype", [(2, 509, 6, torch.bfloat16), (2, 1021, 5, torch.bfloat16),
                                                 (4, 3000, 4, torch.bfloat16), (16, 250, 4, torch.bfloat16),
                                                 (4, 1020, 6, torch.float32)])
def test_append_decode_equals_two_calls(kvq, orc, fbit, t0, steps, dtype):
    """kvq_append_decode (one launch: the decode kernel writes the new token)
    gives the same codes, meta and output, bit for bit, as kvq_append then
    kvq_decode_attn -- including across a shrink, for bf16 and fp32 inputs --
    and matches the oracle."""
    B, H, G, n_f = 2, 3, 4, 4096
    k, v = S.keys_values(10, fbit, B, t0 + steps, H, 0, 3, dtype=dtype)
    lam = lam_for(k)
    P = Pair(kvq, orc, B, H, n_f, fbit, lam)  # separate calls, and the oracle
    F = kvq.KVQCache(1, B, H, n_f * per_token(B, H, [fbit]), [fbit])
    F.set_lambda(0, lam)
    P.append(k[:, :t0], v[:, :t0])
    F.append(0, k[:, :t0].cuda(), v[:, :t0].cuda())
    for i in range(steps):
        t = t0 + i
        kt, vt = k[:, t:t + 1].contiguous(), v[:, t:t + 1].contiguous()
        q = S.queries(10, fbit, i, B, H * G, t + 1, dtype=torch.bfloat16).cuda()
        P.append(kt, vt)
        o_sep = P.gpu.decode_attn(0, q)
        o_fus = F.append_decode(0, kt.cuda(), vt.cuda(), q)
        torch.cuda.synchronize()
        assert torch.equal(o_sep, o_fus), (i, (o_sep - o_fus).abs().max().item())
        assert F.query(0) == P.gpu.query(0)
    F.device_status()
    for b in range(B):
        for j in range(H):
            for x, y in zip(P.gpu.export(0, b, j), F.export(0, b, j)):
                assert np.array_equal(x, y), (b, j)
    P.check_codes()
    P.check_attention(S.queries(10, fbit, 99, B, H * G, t0 + steps, dtype=torch.bfloat16))
    F.free()
