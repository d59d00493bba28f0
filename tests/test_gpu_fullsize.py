"""GPU parity at the full sizes of the four model-shaped workloads, through
the same C-ABI calls and launch configuration the benchmark times.

The whole cache is built on the GPU; the oracle replays sampled (sequence,
KV head) streams -- every stream of the 32B 2-bit and the 70B 4-bit blocks --
from the same inputs (copied to the host chunk by chunk) and checks, for each
replayed stream: codes and meta bit-exact against kvq_export, the block's
shrink schedule, and decode attention of every query head of that KV head
within 2e-3 (max_c |o - o*| / max_c |o*|).

Workloads (synthetic RoPE'd bf16 K/V with x20 outlier Key channels on 1% of
the layer's channels, lambda = sqrt(max |K|) from the first chunk):
  7B decode      batch 16, 4 KV / 28 Q heads, 32768 tokens, Fbit 2 and 4,
                 N_F = 36864 (as the benchmark sizes it)
  7B progressive batch 8, 4 KV heads, 32768 tokens appended one at a time
                 from empty, N_F = 32768, Fbit 2 (16->8->4->2) and 4
  32B decode     batch 16, 8 KV / 40 Q heads, 32768 tokens, Fbit 2 and 4,
                 N_F = 55296 (a 40 GB budget split evenly in tokens over
                 48 two-bit and 16 four-bit blocks)
  70B long-CoT   batch 8, 8 KV / 64 Q heads, 131072 tokens; a Fbit-4 block
                 at N_F = 131072, and a Fbit-2 block with N_F = 262144
                 holding 131072 tokens at 4 bits, then the forced final
                 4 -> 2 shrink, then decode.
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import kvq_synth as S

pytestmark = pytest.mark.gpu

TOL = 2e-3
SEED = 0


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
    return batch * kv_heads * 2 * (16 * fbit + 4)


class Sampled:
    """A full-size GPU block plus oracle replays of a few of its streams."""

    def __init__(self, kvq, orc, batch, kv_heads, n_f, fbit, streams, layer, seed=SEED, shift_mode=0,
                 window=False, chan=False):
        self.kvq, self.orc_mod = kvq, orc
        self.batch, self.kv_heads, self.n_f, self.fbit = batch, kv_heads, n_f, fbit
        self.streams, self.layer, self.seed = streams, layer, seed
        self.window, self.chan = window, chan
        self.gpu = kvq.KVQCache(1, batch, kv_heads, n_f * per_token(batch, kv_heads, fbit), [fbit],
                                sink_window=window, key_channel=chan)
        assert self.gpu.max_tokens == n_f + (129 if window else (127 if chan else 0))
        cls = orc.WLayer if window else (orc.CLayer if chan else orc.Layer)
        self.orc = {s: cls(1, 1, n_f, fbit) for s in streams}
        self.lam = None
        self.pos = 0
        self.n_out = S.outliers_for(kv_heads)
        if shift_mode:
            self.gpu.set_shift_mode(0, shift_mode)
            for o in self.orc.values():
                assert o.set_shift_mode(shift_mode) == 0

    def _set_lambda(self, k):
        self.lam = self.orc_mod.lambda_from_keys(k[0].float().cpu().numpy(), 0.5)
        self.gpu.set_lambda(0, self.lam)

    def _replay(self, k, v):
        for (b, j), o in self.orc.items():
            kb = k[b:b + 1, :, j:j + 1].float().cpu().numpy()
            vb = v[b:b + 1, :, j:j + 1].float().cpu().numpy()
            assert o.append(kb, vb, self.lam[j:j + 1]) == 0

    def fill(self, tokens, chunk=4096):
        """Chunked appends (the benchmark's way of building the cache)."""
        while self.pos < tokens:
            n = min(chunk, tokens - self.pos)
            k, v = S.keys_values(self.seed, self.layer, self.batch, n, self.kv_heads, self.pos, self.n_out,
                                 dtype=torch.bfloat16, device="cuda")
            if self.lam is None:
                self._set_lambda(k)
            self.gpu.append(0, k, v)
            self._replay(k, v)
            self.pos += n

    def fill_one_by_one(self, tokens, chunk=4096):
        """One token per append call, as in generation."""
        while self.pos < tokens:
            n = min(chunk, tokens - self.pos)
            k, v = S.keys_values(self.seed, self.layer, self.batch, n, self.kv_heads, self.pos, self.n_out,
                                 dtype=torch.bfloat16, device="cuda")
            if self.lam is None:
                self._set_lambda(k)
            kt = k.transpose(0, 1).contiguous()  # [n][batch][kv_heads][128]
            vt = v.transpose(0, 1).contiguous()
            for t in range(n):
                self.kvq.kvq_append(self.gpu.handle, 0, kt[t].unsqueeze(1), vt[t].unsqueeze(1))
            self._replay(k, v)
            self.pos += n

    def check_state(self):
        st = self.gpu.query(0)
        for o in self.orc.values():
            m = o.main if self.window or self.chan else o
            assert (st["tokens"], st["bits"], st["n_shrinks"]) == (o.n, m.bits, m.n_shrinks), (st, m.shrink_at)
        return st

    def check_codes(self):
        for (b, j), w in self.orc.items():
            o = w.main if self.window or self.chan else w
            if self.window or self.chan:
                got = self.gpu.export_window(0, b, j)
                want = w.window_codes() if self.window else w.staged_codes()
                for name, x, y in zip(("wK", "wV", "wKm", "wVm"), got, want):
                    assert np.array_equal(x, y[0, 0]), (b, j, name)
            kc, vc, km, vm = self.gpu.export(0, b, j)
            want_km = w.k_meta_channel()[0, 0].reshape(-1, 2) if self.chan else o.k_meta()[0, 0]
            assert np.array_equal(km, want_km), (b, j, "K meta")
            assert np.array_equal(vm, o.v_meta()[0, 0]), (b, j, "V meta")
            for name, got, want in (("K", kc, o.k_codes()[0, 0]), ("V", vc, o.v_codes()[0, 0])):
                if not np.array_equal(got, want):
                    bad = np.argwhere(got != want)
                    raise AssertionError(f"stream {(b, j)} {name} codes differ at {len(bad)} places, "
                                         f"first {bad[:4].tolist()}")

    def check_attention(self, q_heads, step=0):
        G = q_heads // self.kv_heads
        q = S.queries(self.seed, self.layer, step, self.batch, q_heads, self.pos, dtype=torch.bfloat16,
                      device="cuda")
        sm = 1 / math.sqrt(128)
        out = self.gpu.decode_attn(0, q, sm).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        self.gpu.device_status()
        assert np.isfinite(out).all()
        qc = q.float().cpu().numpy()

        def stream_err(item):
            (b, j), o = item
            ref = o.attention(qc[b:b + 1, j * G:(j + 1) * G], self.lam[j:j + 1], sm)[0]
            got = out[b, j * G:(j + 1) * G]
            return float((np.abs(got - ref).max(axis=-1) / np.abs(ref).max(axis=-1)).max())

        # the oracle's C attention runs without the Python lock: many streams go in threads
        with ThreadPoolExecutor(max_workers=min(len(self.orc), os.cpu_count() or 1)) as pool:
            worst = max(pool.map(stream_err, self.orc.items()))
        assert worst <= TOL, f"max rel err {worst:.3e}"
        return worst

    def free(self):
        self.gpu.free()


def corners(batch, kv_heads):
    return [(0, 0), (batch // 2, kv_heads // 2 - 1), (batch - 1, kv_heads - 1)]


def every(batch, kv_heads):
    return [(b, j) for b in range(batch) for j in range(kv_heads)]


@pytest.mark.parametrize("fbit,layer", [(2, 1), (4, 0)])
def test_7b_decode_fullsize(kvq, orc, fbit, layer):
    B, H, HQ, T = 16, 4, 28, 32768
    x = Sampled(kvq, orc, B, H, T + 4096, fbit, corners(B, H), layer)
    x.fill(T)
    st = x.check_state()
    assert st["bits"] == fbit
    x.check_codes()
    x.check_attention(HQ)
    x.check_attention(HQ, step=1)
    x.free()


@pytest.mark.parametrize("fbit,shrinks", [(2, [4096, 8192, 16384]), (4, [8192, 16384])])
def test_7b_progressive_one_token_per_step(kvq, orc, fbit, shrinks):
    B, H, HQ, T = 8, 4, 28, 32768
    x = Sampled(kvq, orc, B, H, T, fbit, [(0, 0), (B - 1, H - 1)], 27 if fbit == 4 else 5)
    for stop in shrinks + [T]:
        x.fill_one_by_one(stop + (0 if stop == T else 1))
        x.check_state()
        x.check_codes()
        x.check_attention(HQ, step=stop)
    o = next(iter(x.orc.values()))
    assert o.shrink_at == shrinks and o.bits == fbit
    x.free()


@pytest.mark.parametrize("fbit,layer", [(2, 3), (4, 60)])
def test_32b_decode_fullsize(kvq, orc, fbit, layer):
    """At 2 bits every one of the 128 (sequence, KV head) streams is replayed
    through the oracle (codes bit-exact, all 40 query heads within 2e-3);
    at 4 bits three streams."""
    B, H, HQ, T = 16, 8, 40, 32768
    x = Sampled(kvq, orc, B, H, 55296, fbit, every(B, H) if fbit == 2 else corners(B, H), layer)
    x.fill(T, chunk=8192)
    st = x.check_state()
    assert st["bits"] == fbit
    x.check_codes()
    x.check_attention(HQ)
    x.free()


def test_70b_fbit4_decode_fullsize(kvq, orc):
    """Every one of the 64 streams of the 128K-token block replayed through the
    oracle: codes bit-exact, all 64 query heads (G = 8) within 2e-3."""
    B, H, HQ, T = 8, 8, 64, 131072
    x = Sampled(kvq, orc, B, H, T, 4, every(B, H), 0)
    x.fill(T, chunk=8192)
    st = x.check_state()
    assert (st["bits"], st["capacity"]) == (4, T)
    x.check_codes()
    x.check_attention(HQ)
    x.free()


def test_70b_final_4to2_shrink_then_decode(kvq, orc):
    B, H, HQ, T = 8, 8, 64, 131072
    x = Sampled(kvq, orc, B, H, 2 * T, 2, corners(B, H), 1)
    x.fill(T, chunk=8192)
    st = x.check_state()
    assert (st["bits"], st["capacity"]) == (4, T)  # full at 4 bits
    x.gpu.shrink(0)
    for o in x.orc.values():
        assert o.shrink() == 0
    st = x.check_state()
    assert st["bits"] == 2
    x.check_codes()
    x.check_attention(HQ)
    x.free()


def test_70b_final_4to2_direct_shift_then_decode(kvq, orc):
    """The same 128K-token 4 -> 2 event with the ablation's Direct Right Shift
    (codes X >> 2, every stored range rescaled by 4/5)."""
    B, H, HQ, T = 8, 8, 64, 131072
    x = Sampled(kvq, orc, B, H, 2 * T, 2, corners(B, H), 2, shift_mode=kvq.KVQ_SHIFT_DIRECT)
    x.fill(T, chunk=8192)
    assert x.check_state()["bits"] == 4
    x.gpu.shrink(0)
    for o in x.orc.values():
        assert o.shrink() == 0
    assert x.check_state()["bits"] == 2
    x.check_codes()
    x.check_attention(HQ)
    x.free()


def test_7b_decode_sink_window_fullsize(kvq, orc):
    """The 7B block with the pages' deployed configuration: the sink and the
    latest 128 tokens at INT16, 32768 + 129 tokens, Fbit 2."""
    B, H, HQ, T = 16, 4, 28, 32768 + 129
    x = Sampled(kvq, orc, B, H, 32768, 2, corners(B, H), 9, window=True)
    x.fill(T, chunk=4096)
    st = x.check_state()
    assert st["bits"] == 2 and st["tokens"] == T
    x.check_codes()
    x.check_attention(HQ)
    x.free()


@pytest.mark.parametrize("fbit,layer", [(2, 5), (4, 0)])
def test_7b_decode_key_channel_fullsize(kvq, orc, fbit, layer):
    """The 7B block with per-channel Key groups: 32768 + 100 tokens (the last
    100 staged at INT16), built from empty through the shrinks, sampled
    streams bit-exact and within 2e-3."""
    B, H, HQ, T = 16, 4, 28, 32768 + 100
    x = Sampled(kvq, orc, B, H, 32768, fbit, corners(B, H), layer, chan=True)
    x.fill(T, chunk=4096)
    st = x.check_state()
    assert st["bits"] == fbit and st["tokens"] == T
    x.check_codes()
    x.check_attention(HQ)
    x.check_attention(HQ, step=1)
    x.free()


def test_7b_fused_decode_steps_fullsize(kvq, orc):
    """The benchmark's step on a full 7B block: three single-token
    kvq_append_decode calls on top of 32768 tokens (2 bits), sampled streams
    against the oracle after each."""
    B, H, HQ, T = 16, 4, 28, 32768
    x = Sampled(kvq, orc, B, H, T + 4096, 2, corners(B, H), 11)
    x.fill(T)
    for step in range(3):
        k, v = S.keys_values(x.seed, x.layer, B, 1, H, x.pos, x.n_out, dtype=torch.bfloat16, device="cuda")
        q = S.queries(x.seed, x.layer, 50 + step, B, HQ, x.pos + 1, dtype=torch.bfloat16, device="cuda")
        out = x.gpu.append_decode(0, k, v, q).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        x._replay(k, v)
        x.pos += 1
        x.check_state()
        qc = q.float().cpu().numpy()
        for (b, j), o in x.orc.items():
            G = HQ // H
            ref = o.attention(qc[b:b + 1, j * G:(j + 1) * G], x.lam[j:j + 1], 1 / math.sqrt(128))[0]
            err = np.abs(out[b, j * G:(j + 1) * G] - ref).max(axis=-1) / np.abs(ref).max(axis=-1)
            assert err.max() <= TOL, (step, b, j, err.max())
    x.check_codes()
    x.free()
