"""Pins for the CPU oracle: each test checks an oracle function against something
other than itself -- a value the pages print, a closed form, a library
routine, exact rational arithmetic or an invariant of the mathematics.

Pages: "PM-KVQ: Progressive Mixed-Precision KV Cache Quantization for
Long-CoT LLMs" (papernotes.org note) and the ChanMix note on the same site
(key design 1: S = (max - min)/(2^b - 1), worst-case error S/2).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- binary16

def test_f16_decode_matches_numpy_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isinf(got), np.isinf(ref))
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_f16_round_nearest_matches_numpy(orc):
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.standard_normal(3000) * 10.0,
        rng.standard_normal(1000) * 1e-5,   # subnormal range
        rng.uniform(60000, 70000, 200),     # overflow boundary
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 2.0**-24, 2.0**-25, 3 * 2.0**-26]),
    ])
    with np.errstate(over="ignore"):  # values past 65520 round to inf on both sides
        for x in xs:
            assert orc.f16_from_f64(float(x), 0) == int(np.float16(x).view(np.uint16)), x


def test_f16_directed_rounding_brackets(orc):
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.standard_normal(3000) * 7.0, rng.standard_normal(300) * 1e-6])
    for x in xs:
        d = orc.f16_from_f64(float(x), -1)
        u = orc.f16_from_f64(float(x), +1)
        vd, vu = orc.f16_to_f64(d), orc.f16_to_f64(u)
        assert vd <= x <= vu
        rn = int(np.float16(x).view(np.uint16))
        assert rn in (d, u)
        if vd == x:
            assert d == u
        else:
            # adjacent binary16 values: nothing representable strictly between
            mid = np.float16(x)
            assert vd < vu
            nxt = np.nextafter(np.float16(vd), np.float16(np.inf))
            assert float(nxt) == vu, (x, vd, vu, mid)
    # exactly representable values are fixed points of both directions
    for b in (0x3C00, 0xBC00, 0x0001, 0x7BFF, 0x4248):
        v = orc.f16_to_f64(b)
        assert orc.f16_from_f64(v, -1) == b and orc.f16_from_f64(v, +1) == b


# ---------------------------------------------------------------- quantizer

def test_quantizer_golden_examples(orc):
    with open(os.path.join(GOLDEN, "quantizer_example.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        codes, r, z = orc.quantize_group(np.array(case["x"], np.float32), case["bits"])
        assert list(codes) == case["codes"]
        assert r == case["r_bits"] and z == case["z_bits"]


def _exact_code(x32: float, r_bits: int, z_bits: int, bits: int, orc) -> Fraction:
    """(x - Z) (2^b - 1) / R + 1/2 in exact rational arithmetic."""
    z = Fraction(orc.f16_to_f64(z_bits))
    r = Fraction(orc.f16_to_f64(r_bits))
    return (Fraction(float(x32)) - z) * ((1 << bits) - 1) / r + Fraction(1, 2)


@pytest.mark.parametrize("bits", [2, 4, 8, 16])
def test_quantizer_matches_exact_rounding(orc, bits):
    """Codes equal floor((x - Z)/S + 1/2) computed exactly, except within fp32
    noise of a rounding boundary, where they may differ by one."""
    rng = np.random.default_rng(bits)
    n_near = 0
    for trial in range(40):
        scale = float(np.exp(rng.uniform(-3, 3)))
        x = (rng.standard_normal(128) * scale + rng.uniform(-2, 2)).astype(np.float32)
        codes, r, z = orc.quantize_group(x, bits)
        qmax = (1 << bits) - 1
        for c in range(128):
            e = _exact_code(x[c], r, z, bits, orc)
            want = min(qmax, max(0, math.floor(e)))
            if codes[c] != want:
                frac = e - math.floor(e)
                dist = min(frac, 1 - frac)
                assert abs(int(codes[c]) - want) == 1
                assert dist < Fraction(qmax * 4, 1 << 24) + Fraction(1, 1 << 20)
                n_near += 1
    assert n_near < 40  # boundary cases are rare


@pytest.mark.parametrize("bits", [2, 4, 8, 16])
def test_quantizer_range_and_error_bound(orc, bits):
    """ChanMix key design 1: |x - x^| <= S/2 with S = R/(2^b-1) (plus the fp32
    rounding of the code computation); Z <= min, Z + R >= max; the min maps to
    round((min - Z)/S) (0 unless binary16 rounding of Z moved it) and, for
    b <= 8, the max maps to 2^b - 1 (R is rounded up by at most 2^-10 of itself)."""
    rng = np.random.default_rng(100 + bits)
    qmax = (1 << bits) - 1
    for trial in range(60):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 30)).astype(np.float32)
        if trial % 5 == 0:
            x[rng.integers(0, 128, 3)] *= 20  # outliers
        codes, r, z = orc.quantize_group(x, bits)
        R, Z = orc.f16_to_f64(r), orc.f16_to_f64(z)
        assert Z <= float(x.min()) and Z + R >= float(x.max())
        assert codes.max() <= qmax
        S = R / qmax
        # the min lands on 0 unless rounding Z down to binary16 moved it by S/2 or more
        off = (float(x.min()) - Z) / S
        assert codes[np.argmin(x)] == math.floor(off + 0.5) or abs(off % 1 - 0.5) < 1e-3
        if off < 0.25:
            assert codes[np.argmin(x)] == 0
        if bits <= 8:
            assert codes[np.argmax(x)] == qmax
        xhat = Z + codes.astype(np.float64) * S
        err = np.abs(xhat - x.astype(np.float64))
        assert err.max() <= S * (0.5 + 4 * qmax * 2.0**-24) + 1e-12


def test_quantizer_constant_group(orc):
    for v in (0.0, 1.0, -3.5, 0.1):
        x = np.full(128, v, np.float32)
        codes, r, z = orc.quantize_group(x, 4)
        assert orc.dequant(int(codes[0]), r, z, 4) == pytest.approx(v, abs=1e-3)
        if orc.f16_to_f64(z) == v:
            assert r == 0 and not codes.any()


def test_migration_rounds_in_fp32(orc):
    """fp32(k * fp32(1/lambda)) -- the stored Key of key design 3."""
    for k, lam in [(3.0, 2.0), (1.0, 3.0), (-7.25, 0.5), (20.0, 4.47213595)]:
        linv = np.float32(1.0 / np.float64(np.float32(lam)))
        assert orc.migrate(np.array([k]), np.array([lam]))[0] == np.float32(np.float32(k) * linv)


def test_lambda_rule_flattens_outliers(orc):
    """Key design 3: lambda_i = (max|K_i|)^alpha; with alpha = 1/2 the migrated
    key K/lambda has per-channel max |K_i|^(1/2), and (q lambda).(k/lambda) = q.k."""
    rng = np.random.default_rng(5)
    keys = rng.standard_normal((64, 2, 128)).astype(np.float32)
    keys[:, :, [3, 77]] *= 20
    lam = orc.lambda_from_keys(keys, 0.5)
    mx = np.abs(keys).max(axis=0)
    assert np.allclose(np.abs(keys / lam).max(axis=0), np.sqrt(mx), rtol=1e-5)
    q = rng.standard_normal(128)
    for j in range(2):
        a = float(np.dot(q * lam[j], keys[5, j] / lam[j].astype(np.float64)))
        assert a == pytest.approx(float(np.dot(q, keys[5, j])), rel=1e-12, abs=1e-12)


# ---------------------------------------------------------------- ERS

@pytest.mark.parametrize("b", [1, 2, 4, 8])
def test_ers_equals_dequant_requant_exhaustive(orc, b):
    """Key design 1: the shift is mathematically equal to dequantising the 2b-bit
    code and requantising to b bits with Z_b = Z_2b, S_b = (2^b+1) S_2b.
    (X^ - Z)/S_b = X/(2^b+1), rounded half up = floor((2X + 2^b + 1) / (2(2^b+1)))."""
    d = (1 << b) + 1
    mism, maxdiff = 0, 0
    for X in range(1 << (2 * b)):
        want = (2 * X + d) // (2 * d)
        got = orc.ers(X, b)
        if got != want:
            mism += 1
            maxdiff = max(maxdiff, abs(got - want))
    print(f"ERS b={b}: mismatches={mism} max_code_diff={maxdiff} over {1 << (2 * b)} codes")
    assert mism == 0 and maxdiff == 0
    assert orc.ers(0, b) == 0 and orc.ers((1 << (2 * b)) - 1, b) == (1 << b) - 1


@pytest.mark.parametrize("b", [2, 4, 8])
def test_ers_equals_fp64_requant_with_oracle_dequant(orc, b):
    """Same statement through the oracle's own dequantiser, in fp64, for random
    binary16 (R, Z): q_b = floor((X^ - Z)/S_b + 1/2)."""
    rng = np.random.default_rng(b)
    for trial in range(4):
        z = orc.f16_from_f64(float(rng.normal() * 3), -1)
        r = orc.f16_from_f64(float(abs(rng.normal()) * 5 + 0.01), +1)
        Z = orc.f16_to_f64(z)
        Sb = orc.f16_to_f64(r) / ((1 << b) - 1)
        xs = range(1 << (2 * b)) if b < 8 else rng.integers(0, 1 << 16, 4096)
        for X in xs:
            xh = orc.dequant(int(X), r, z, 2 * b)
            want = math.floor((xh - Z) / Sb + 0.5)
            assert orc.ers(int(X), b) == want


@pytest.mark.parametrize("b", [2, 4, 8])
def test_scale_zero_identities(orc, b):
    """Z_b = Z_2b and S_b = (2^b+1) S_2b: with the range R held fixed,
    R/(2^b-1) = (2^b+1) R/(2^2b-1) since 2^2b - 1 = (2^b-1)(2^b+1)."""
    rng = np.random.default_rng(7)
    for _ in range(500):
        R = orc.f16_to_f64(orc.f16_from_f64(float(rng.uniform(1e-3, 100)), +1))
        s2b = R / ((1 << (2 * b)) - 1)
        sb = orc.scale_after_shrink(s2b, b)
        assert sb == pytest.approx(R / ((1 << b) - 1), rel=4e-16)


# ---------------------------------------------------------------- cache model

def _cfg0_inputs(n, seed=0):
    import kvq_synth as S
    k, v = S.keys_values(seed, 0, 1, n, 2, 0, 4, dtype=torch.float32)
    return k.numpy(), v.numpy()


def test_progressive_schedule_tiny_config(orc):
    """1 layer, batch 1, 2 KV heads, Fbit 4, room for 4096 tokens at 4 bits:
    16 bits until the block is full at 1024 tokens, 8 bits until 2048, then 4."""
    k, v = _cfg0_inputs(4096)
    L = orc.Layer(1, 2, 4096, 4)
    assert (L.capacity(16), L.capacity(8), L.capacity(4)) == (1024, 2048, 4096)
    bits_seen = []
    for t in range(0, 4096, 256):
        assert L.append(k[:, t:t + 256], v[:, t:t + 256], None) == 0
        bits_seen.append(L.bits)
    assert L.shrink_at == [1024, 2048] and L.n_shrinks == 2 and L.bits == 4 and L.n == 4096
    assert bits_seen[:4] == [16] * 4 and bits_seen[4:8] == [8] * 4 and bits_seen[8:] == [4] * 8
    before = L.k_codes()
    assert L.append(k[:, :1], v[:, :1], None) == 1  # full at Fbit: refused, nothing written
    assert L.n == 4096 and np.array_equal(L.k_codes(), before)
    assert L.shrink() == -1  # never below Fbit


def test_chunked_append_equals_token_by_token(orc):
    k, v = _cfg0_inputs(1500, seed=3)
    lam = np.exp(np.random.default_rng(0).uniform(0, 1.5, (2, 128))).astype(np.float32)
    A = orc.Layer(1, 2, 4096, 4)
    B = orc.Layer(1, 2, 4096, 4)
    for t in range(1500):
        A.append(k[:, t:t + 1], v[:, t:t + 1], lam)
    for t0 in range(0, 1500, 333):
        B.append(k[:, t0:t0 + 333], v[:, t0:t0 + 333], lam)
    for f in ("k_codes", "v_codes", "k_meta", "v_meta"):
        assert np.array_equal(getattr(A, f)(), getattr(B, f)())


def test_shrink_is_elementwise_ers_and_keeps_meta(orc):
    k, v = _cfg0_inputs(1024, seed=4)
    L = orc.Layer(1, 2, 4096, 4)
    L.append(k, v, None)
    assert L.bits == 16 and L.n == 1024
    kc, vc, km, vm = L.k_codes(), L.v_codes(), L.k_meta(), L.v_meta()
    assert L.shrink() == 0 and L.bits == 8
    ers = np.vectorize(lambda x: orc.ers(int(x), 8))
    sub = (slice(None), slice(None), slice(0, 40))
    assert np.array_equal(L.k_codes()[sub], ers(kc[sub]))
    assert np.array_equal(L.v_codes()[sub], ers(vc[sub]))
    assert np.array_equal(L.k_meta(), km) and np.array_equal(L.v_meta(), vm)
    # a shrink needs a full block
    assert L.shrink() == -2


def test_direct_quantize_agrees_with_shrunk_cache_roughly(orc):
    """A token kept at 16 bits and shifted down to 4 is within one 4-bit step of
    quantising it directly at 4 bits (same Z, R)."""
    k, v = _cfg0_inputs(1024, seed=5)
    L = orc.Layer(1, 2, 4096, 4)
    L.append(k, v, None)
    L.shrink()
    L2 = orc.Layer(1, 2, 4096, 4)
    L2.append(k[:, :1024], v[:, :1024], None)
    # second layer: quantise the same groups directly at 4 bits
    direct = np.stack([orc.codes_with_meta(v[0, t, 0], 8, *L.v_meta()[0, 0, t]) for t in range(64)])
    assert np.abs(direct.astype(int) - L.v_codes()[0, 0, :64].astype(int)).max() <= 1


# ---------------------------------------------------- Direct Right Shift (ablation)

@pytest.mark.parametrize("b", [1, 2, 4, 8])
def test_drs_keeps_the_high_bits_exhaustive(orc, b):
    """The ablation's Direct Right Shift keeps only the high b bits of every
    2b-bit code: integer division by 2^b, over every code."""
    for x in range(1 << (2 * b)):
        assert orc.drs(x, b) == x // (1 << b)


@pytest.mark.parametrize("b", [1, 2, 4, 8])
def test_drs_range_is_ieee_fp32_then_binary16(orc, b):
    """R_b = binary16_RN(fp32(fp32(R * 2^b) / (2^b + 1))), checked against
    numpy's IEEE float32 / float16 arithmetic on random positive ranges."""
    rng = np.random.default_rng(b)
    bits = rng.integers(0x0001, 0x7bff, 400).astype(np.uint16)  # positive finite binary16
    for rb in bits:
        r = np.float32(np.uint16(rb).view(np.float16))
        want = np.float16((r * np.float32(2 ** b)) / np.float32(2 ** b + 1)).view(np.uint16)
        assert orc.drs_range(int(rb), b) == int(want)


@pytest.mark.parametrize("b", [2, 4, 8])
def test_drs_scale_is_the_truncation_scale(orc, b):
    """S_b = R_b / (2^b - 1) equals 2^b S_2b = 2^b R / (2^2b - 1) up to the one
    binary16 rounding of R_b (relative 2^-11)."""
    rng = np.random.default_rng(10 + b)
    for rb in rng.integers(0x2000, 0x6000, 200):
        r = orc.f16_to_f64(int(rb))
        s_b = orc.f16_to_f64(orc.drs_range(int(rb), b)) / (2 ** b - 1)
        s_trunc = (2 ** b) * r / (2 ** (2 * b) - 1)
        assert abs(s_b - s_trunc) <= 2 ** -11 * s_trunc


def test_drs_is_less_accurate_than_ers(orc):
    """The note's ablation ranks the Direct Right Shift well below the
    Equivalent Right Shift.  On Gaussian groups quantized at 2b and shifted
    to b, the mean reconstruction error of DRS exceeds ERS's, and a direct
    b-bit quantization is matched by ERS within one step."""
    rng = np.random.default_rng(21)
    for b in (2, 4, 8):
        e_ers, e_drs = [], []
        for _ in range(40):
            x = rng.standard_normal(128).astype(np.float32)
            codes, r, z = orc.quantize_group(x, 2 * b)
            ers = np.array([orc.ers(int(c), b) for c in codes])
            drs = np.array([orc.drs(int(c), b) for c in codes])
            x_ers = orc.dequant_array(ers, np.array([r, z]), b)
            x_drs = orc.dequant_array(drs, np.array([orc.drs_range(r, b), z]), b)
            e_ers.append(np.abs(x_ers - x).mean())
            e_drs.append(np.abs(x_drs - x).mean())
        # uniform data would give 2^(b+1) / (2^b + 1) (truncation vs rounding
        # of a step (2^b + 1)/2^b wider); Gaussian groups measure 1.27 / 1.81 / 2.05
        assert np.mean(e_drs) > 1.2 * np.mean(e_ers), (b, np.mean(e_drs), np.mean(e_ers))


def test_progressive_model_with_drs(orc):
    """Shift mode 1: the same schedule; at each shrink every stored code is
    X >> b and every stored R is rescaled, Z kept; tokens after a shrink
    are quantized directly at the new width."""
    k, v = _cfg0_inputs(1100, seed=6)
    L = orc.Layer(1, 2, 4096, 4)
    assert L.set_shift_mode(1) == 0
    L.append(k[:, :1024], v[:, :1024], None)
    kc, km, vm = L.k_codes(), L.k_meta(), L.v_meta()
    L.append(k[:, 1024:], v[:, 1024:], None)
    assert L.shrink_at == [1024] and L.bits == 8
    assert np.array_equal(L.k_codes()[:, :, :1024], kc >> 8)
    rr = np.vectorize(lambda r: orc.drs_range(int(r), 8))
    assert np.array_equal(L.k_meta()[:, :, :1024, 0], rr(km[..., 0]))
    assert np.array_equal(L.v_meta()[:, :, :1024, 0], rr(vm[..., 0]))
    assert np.array_equal(L.k_meta()[:, :, :1024, 1], km[..., 1])
    E = orc.Layer(1, 2, 4096, 4)  # the ERS block differs only in the shifted tokens
    E.append(k, v, None)
    assert np.array_equal(E.k_codes()[:, :, 1024:], L.k_codes()[:, :, 1024:])
    assert L.set_shift_mode(0) == -2  # fixed once the block has shrunk


# ------------------------------------------ sink token + recent window at INT16

def _chain(orc, codes, bits, mode=0):
    """Shift INT16 codes down to `bits` one level at a time (Python, from the
    operators pinned above)."""
    out = codes.astype(np.int64)
    b = 8
    while b >= bits:
        f = (lambda x, b=b: orc.drs(int(x), b)) if mode else (lambda x, b=b: orc.ers(int(x), b))
        out = np.vectorize(f)(out)
        b //= 2
    return out


def test_window_short_block_is_all_int16(orc):
    """Up to 129 tokens everything is held at INT16: the progressive cache is
    empty and attention equals that of a 16-bit block of the same tokens."""
    k, v = _cfg0_inputs(129, seed=7)
    W = orc.WLayer(1, 2, 4096, 4)
    P = orc.Layer(1, 2, 4096, 16)
    assert W.append(k, v, None) == 0 and P.append(k, v, None) == 0
    assert W.main.n == 0 and W.window_tokens() == list(range(129))
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(1)).numpy()
    np.testing.assert_allclose(W.attention(q, None, 0.1), P.attention(q, None, 0.1), rtol=1e-13, atol=1e-13)
    kc, vc, km, vm = W.window_codes()
    assert np.array_equal(kc, P.k_codes()) and np.array_equal(km, P.k_meta())


def test_window_fbit16_block_equals_plain_block(orc):
    """A 16-bit block never shrinks, so moving a token out of the window
    changes nothing: codes and attention equal the plain block's."""
    k, v = _cfg0_inputs(700, seed=8)
    W = orc.WLayer(1, 2, 1024, 16)
    P = orc.Layer(1, 2, 1024, 16)
    W.append(k, v, None)
    P.append(k, v, None)
    assert W.main.n == 700 - 129
    assert np.array_equal(W.main.k_codes(), P.k_codes()[:, :, 1:1 + W.main.n])
    assert np.array_equal(W.main.v_meta(), P.v_meta()[:, :, 1:1 + W.main.n])
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(2)).numpy()
    np.testing.assert_allclose(W.attention(q, None, 0.1), P.attention(q, None, 0.1), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mode", [0, 1])
def test_window_moved_tokens_are_the_shift_chain(orc, mode):
    """Tokens that left the window hold the block's shift chain of their INT16
    codes (ERS; or the direct shift with its range chain), whatever the
    shrinks in between; Z is kept."""
    k, v = _cfg0_inputs(900, seed=9)
    W = orc.WLayer(1, 2, 1024, 2)  # shrinks at progressive counts 128, 256, 512
    assert W.set_shift_mode(mode) == 0
    for t0 in range(0, 900, 150):
        assert W.append(k[:, t0:t0 + 150], v[:, t0:t0 + 150], None) == 0
    m = W.main
    assert m.n == 900 - 129 and m.bits == 2 and m.shrink_at == [128, 256, 512]
    kc16, vc16, km16, vm16 = W.int16_codes()
    sel = slice(1, 1 + m.n)
    assert np.array_equal(m.k_codes(), _chain(orc, kc16[:, :, sel], m.bits, mode))
    assert np.array_equal(m.v_codes(), _chain(orc, vc16[:, :, sel], m.bits, mode))
    assert np.array_equal(m.k_meta()[..., 1], km16[:, :, sel, 1])
    if mode:
        rr = km16[:, :, sel, 0].astype(np.int64)
        for b in (8, 4, 2):
            rr = np.vectorize(lambda r, b=b: orc.drs_range(int(r), b))(rr)
        assert np.array_equal(m.k_meta()[..., 0], rr)
    else:
        assert np.array_equal(m.k_meta(), km16[:, :, sel])
    assert W.window_tokens() == [0] + list(range(900 - 128, 900))


def test_window_chunked_equals_token_by_token(orc):
    k, v = _cfg0_inputs(700, seed=10)
    lam = np.exp(np.random.default_rng(3).uniform(0, 1.5, (2, 128))).astype(np.float32)
    A = orc.WLayer(1, 2, 1024, 4)
    B = orc.WLayer(1, 2, 1024, 4)
    for t in range(700):
        assert A.append(k[:, t:t + 1], v[:, t:t + 1], lam) == 0
    for t0 in range(0, 700, 97):
        assert B.append(k[:, t0:t0 + 97], v[:, t0:t0 + 97], lam) == 0
    assert A.main.n_shrinks == B.main.n_shrinks == 2
    for x, y in zip(A.int16_codes() + (A.main.k_codes(), A.main.v_codes(), A.main.k_meta()),
                    B.int16_codes() + (B.main.k_codes(), B.main.v_codes(), B.main.k_meta())):
        assert np.array_equal(x, y)


def test_window_attention_over_three_segments(orc):
    """Attention of a windowed block = dense fp64 attention over the
    dequantized sink, progressive cache and window, assembled here."""
    k, v = _cfg0_inputs(400, seed=11)
    lam = np.exp(np.random.default_rng(4).uniform(0, 1.0, (2, 128))).astype(np.float32)
    W = orc.WLayer(1, 2, 512, 4)
    W.append(k, v, lam)
    m = W.main
    wk, wv, wkm, wvm = W.window_codes()
    K = np.concatenate([orc.dequant_array(m.k_codes(), m.k_meta(), m.bits), orc.dequant_array(wk, wkm, 16)], axis=2)
    V = np.concatenate([orc.dequant_array(m.v_codes(), m.v_meta(), m.bits), orc.dequant_array(wv, wvm, 16)], axis=2)
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(5)).numpy()
    qp = q[0].astype(np.float64) * np.repeat(lam.astype(np.float64), 2, axis=0)
    want = orc.attention_dense(qp, K[0].transpose(1, 0, 2), V[0].transpose(1, 0, 2), 0.1)
    np.testing.assert_allclose(W.attention(q, lam, 0.1)[0], want, rtol=1e-11, atol=1e-12)


def test_window_budget(orc):
    """The progressive cache holds N_F tokens at Fbit; with the sink and the
    window the block refuses the (N_F + 130)-th token."""
    k, v = _cfg0_inputs(512 + 130, seed=12)
    W = orc.WLayer(1, 2, 512, 4)
    assert W.append(k[:, :512 + 129], v[:, :512 + 129], None) == 0
    assert W.main.n == 512 and W.main.bits == 4
    assert W.append(k[:, -1:], v[:, -1:], None) == 1 and W.n == 512 + 129


# ------------------------------- per-channel Key groups over 128-token blocks

def _int16_records(orc, x):
    """INT16 per-token records of rows x [T][128] (the quantizer pinned above)."""
    codes, meta = [], []
    for row in x:
        c, r, z = orc.quantize_group(row, 16)
        codes.append(c)
        meta.append((r, z))
    return np.array(codes), np.array(meta)


def test_channel_int16_value_is_three_fp32_steps(orc):
    """A staged Key re-enters the quantizer as Z + code * (R / 65535) in fp32,
    one IEEE round-to-nearest per step (numpy's float32 arithmetic here)."""
    rng = np.random.default_rng(20)
    f32 = np.float32
    for _ in range(3000):
        r = int(orc.f16_from_f64(float(rng.uniform(0.01, 40.0)), 1))
        z = int(orc.f16_from_f64(float(rng.uniform(-20.0, 5.0)), -1))
        code = int(rng.integers(0, 65536))
        rf, zf = f32(orc.f16_to_f64(r)), f32(orc.f16_to_f64(z))
        want = zf + f32(code) * (rf / f32(65535.0))
        assert orc.int16_value(code, r, z) == want
    assert orc.int16_value(0, r, z) == f32(orc.f16_to_f64(z))


def test_channel_short_block_is_all_int16(orc):
    """Fewer than 128 tokens: everything is staged at INT16, so codes and
    attention equal those of a 16-bit per-token block of the same tokens."""
    k, v = _cfg0_inputs(127, seed=21)
    Cl = orc.CLayer(1, 2, 1024, 4)
    P = orc.Layer(1, 2, 1024, 16)
    assert Cl.append(k, v, None) == 0 and P.append(k, v, None) == 0
    assert Cl.main.n == 0 and Cl.n_staged == 127
    kc, vc, km, vm = Cl.staged_codes()
    assert np.array_equal(kc, P.k_codes()) and np.array_equal(km, P.k_meta())
    assert np.array_equal(vc, P.v_codes()) and np.array_equal(vm, P.v_meta())
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(22)).numpy()
    np.testing.assert_allclose(Cl.attention(q, None, 0.1), P.attention(q, None, 0.1), rtol=1e-13, atol=1e-13)


def test_channel_ramp_block_codes_run_along_tokens(orc):
    """Keys that rise linearly along the tokens in every channel (each channel
    with its own offset and slope): per-channel groups over the block put the
    first token at code 0 and the last at 2^b - 1 in every channel and the
    codes never fall along the tokens; a per-token (transposed) grouping
    would not.  Z <= the channel's smallest INT16 value, Z + R >= its largest,
    and every code is within half a step of it."""
    t = np.arange(128, dtype=np.float64)[:, None]
    a = np.linspace(-3.0, 2.0, 128)[None, :]
    d = np.linspace(0.002, 0.05, 128)[None, :]
    x = (a + d * t).astype(np.float32)  # [token][channel]
    k = np.stack([x, x[:, ::-1]], axis=1)[None]  # [1][128][2 heads][128]
    v = np.zeros_like(k)
    for bits in (4, 2):
        Cl = orc.CLayer(1, 2, 2048 if bits == 2 else 1024, bits)
        # fill until the cache has shrunk to `bits`, then check the latest block
        while Cl.main.bits != bits or Cl.main.n == 0:
            assert Cl.append(k, v, None) == 0
        blk = Cl.main.n // 128 - 1
        kc = Cl.main.k_codes()[0, :, 128 * blk:]
        kmc = Cl.k_meta_channel()[0, :, blk]
        for h in range(2):
            codes16, meta16 = _int16_records(orc, k[0, :, h])
            xv = np.array([[orc.int16_value(int(codes16[i, c]), int(meta16[i, 0]), int(meta16[i, 1]))
                            for c in range(128)] for i in range(128)], dtype=np.float64)
            assert (kc[h, 0] == 0).all() and (kc[h, -1] == (1 << bits) - 1).all()
            assert (np.diff(kc[h].astype(np.int64), axis=0) >= 0).all()
            R = np.array([orc.f16_to_f64(int(r)) for r in kmc[h, :, 0]])
            Z = np.array([orc.f16_to_f64(int(z)) for z in kmc[h, :, 1]])
            assert (Z <= xv.min(axis=0)).all() and (Z + R >= xv.max(axis=0)).all()
            S = R / ((1 << bits) - 1)
            err = np.abs(xv - (Z[None] + kc[h] * S[None]))
            assert (err <= S[None] / 2 * (1 + 1e-3) + 1e-6).all()
            # the quantizer of the column, applied here to the same values
            for c in (0, 37, 127):
                want, r, z = orc.quantize_group(xv[:, c].astype(np.float32), bits)
                assert np.array_equal(kc[h, :, c], want) and (r, z) == tuple(kmc[h, c])


def test_channel_constant_channel(orc):
    """Keys constant over a block (every INT16 record then has range 0 and
    zero 1.25, so each channel's staged values are exactly 1.25): every
    channel gets range 0, zero 1.25 and all codes 0."""
    k, v = _cfg0_inputs(128, seed=23)
    k[:] = 1.25
    Cl = orc.CLayer(1, 2, 1024, 4)
    assert Cl.append(k, v, None) == 0 and Cl.main.n == 128
    kmc = Cl.k_meta_channel()[0, :, 0]
    assert (kmc[..., 0] == 0).all() and (Cl.main.k_codes() == 0).all()
    assert all(orc.f16_to_f64(int(z)) == 1.25 for z in kmc[..., 1].ravel())


@pytest.mark.parametrize("mode", [0, 1])
def test_channel_schedule_values_and_shifted_blocks(orc, mode):
    """N = 1024 tokens at Fbit 2 (128 at 16 bits): the progressive cache
    shrinks when the 2nd, 3rd and 5th blocks arrive (at 128, 256, 512
    tokens), the 9th block is refused.  Values are the shift chain of their
    INT16 codes (range chained under the direct shift, Z kept); the first
    block's Keys are its 16-bit per-channel codes shifted down with the block
    (ranges kept, or chained under the direct shift)."""
    k, v = _cfg0_inputs(1152, seed=24)
    Cl = orc.CLayer(1, 2, 1024, 2)
    assert Cl.set_shift_mode(mode) == 0
    assert Cl.append(k[:, :1151], v[:, :1151], None) == 0
    m = Cl.main
    assert (m.n, m.bits, m.shrink_at, Cl.n_staged) == (1024, 2, [128, 256, 512], 127)
    assert Cl.append(k[:, 1151:], v[:, 1151:], None) == 1 and Cl.n == 1151
    for h in range(2):
        vc16, vm16 = _int16_records(orc, v[0, :1024, h])
        assert np.array_equal(m.v_codes()[0, h], _chain(orc, vc16, 2, mode))
        assert np.array_equal(m.v_meta()[0, h, :, 1], vm16[:, 1])
        rr = vm16[:, 0].astype(np.int64)
        if mode:
            for b in (8, 4, 2):
                rr = np.vectorize(lambda r, b=b: orc.drs_range(int(r), b))(rr)
        assert np.array_equal(m.v_meta()[0, h, :, 0], rr)
        # block 0 entered at 16 bits
        kc16, km16 = _int16_records(orc, k[0, :128, h])
        xv = np.array([[orc.int16_value(int(kc16[i, c]), int(km16[i, 0]), int(km16[i, 1]))
                        for c in range(128)] for i in range(128)], dtype=np.float32)
        for c in (0, 64, 127):
            c16, r, z = orc.quantize_group(xv[:, c], 16)
            assert np.array_equal(m.k_codes()[0, h, :128, c], _chain(orc, c16, 2, mode))
            rw = r
            if mode:
                for b in (8, 4, 2):
                    rw = orc.drs_range(rw, b)
            assert tuple(Cl.k_meta_channel()[0, h, 0, c]) == (rw, z)


def test_channel_capacity_must_be_whole_blocks(orc):
    with pytest.raises(ValueError):
        orc.CLayer(1, 2, 512, 2)  # 64 tokens at 16 bits: not a whole block
    orc.CLayer(1, 2, 512, 4)


def test_channel_chunked_equals_token_by_token(orc):
    k, v = _cfg0_inputs(700, seed=25)
    lam = np.exp(np.random.default_rng(6).uniform(0, 1.5, (2, 128))).astype(np.float32)
    A = orc.CLayer(1, 2, 1024, 4)
    B = orc.CLayer(1, 2, 1024, 4)
    for t in range(700):
        assert A.append(k[:, t:t + 1], v[:, t:t + 1], lam) == 0
    for t0 in range(0, 700, 97):
        assert B.append(k[:, t0:t0 + 97], v[:, t0:t0 + 97], lam) == 0
    assert A.main.n_shrinks == B.main.n_shrinks == 2 and A.main.n == 640
    for x, y in zip(A.staged_codes() + (A.main.k_codes(), A.main.v_codes(), A.main.v_meta(), A.k_meta_channel()),
                    B.staged_codes() + (B.main.k_codes(), B.main.v_codes(), B.main.v_meta(), B.k_meta_channel())):
        assert np.array_equal(x, y)


def test_channel_attention_over_two_segments(orc):
    """Attention = dense fp64 attention over the progressive cache (each Key
    channel dequantized with its block's range and zero) and the staged INT16
    tokens, assembled here."""
    k, v = _cfg0_inputs(600, seed=26)
    lam = np.exp(np.random.default_rng(7).uniform(0, 1.0, (2, 128))).astype(np.float32)
    Cl = orc.CLayer(1, 2, 1024, 4)
    Cl.append(k, v, lam)
    m = Cl.main
    nb = m.n // 128
    kmc = Cl.k_meta_channel()[0]  # [2][nb][128][2]
    R = np.vectorize(orc.f16_to_f64)(kmc[..., 0].astype(np.int64))
    Z = np.vectorize(orc.f16_to_f64)(kmc[..., 1].astype(np.int64))
    blk = np.repeat(np.arange(nb), 128)
    Km = Z[:, blk] + m.k_codes()[0] * (R[:, blk] / ((1 << m.bits) - 1))
    sk, sv, skm, svm = Cl.staged_codes()
    K = np.concatenate([Km, orc.dequant_array(sk, skm, 16)[0]], axis=1)
    V = np.concatenate([orc.dequant_array(m.v_codes(), m.v_meta(), m.bits)[0], orc.dequant_array(sv, svm, 16)[0]],
                       axis=1)
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(27)).numpy()
    qp = q[0].astype(np.float64) * np.repeat(lam.astype(np.float64), 2, axis=0)
    want = orc.attention_dense(qp, K.transpose(1, 0, 2), V.transpose(1, 0, 2), 0.1)
    np.testing.assert_allclose(Cl.attention(q, lam, 0.1)[0], want, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- attention

def _small_layer(orc, T, bits_target=4, seed=0, lam=None):
    k, v = _cfg0_inputs(T, seed)
    n_f = 4096
    L = orc.Layer(1, 2, n_f, bits_target)
    L.append(k, v, lam)
    return L


def test_attention_matches_torch_sdpa_fp64(orc):
    rng = np.random.default_rng(9)
    lam = np.exp(rng.uniform(0, 1.5, (2, 128))).astype(np.float32)
    L = _small_layer(orc, 1500, lam=lam)  # 8-bit after one shrink
    assert L.bits == 8
    q = rng.standard_normal((1, 4, 128)).astype(np.float32)
    scale = 1 / math.sqrt(128)
    got = L.attention(q, lam, scale)
    kh = orc.dequant_array(L.k_codes(), L.k_meta(), L.bits)[0]  # [2][T][128]
    vh = orc.dequant_array(L.v_codes(), L.v_meta(), L.bits)[0]
    qp = q[0].astype(np.float64) * np.repeat(lam.astype(np.float64), 2, axis=0)
    Kt = torch.from_numpy(np.repeat(kh, 2, axis=0))[None]  # GQA: head h -> h // 2
    Vt = torch.from_numpy(np.repeat(vh, 2, axis=0))[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qp)[None, :, None, :], Kt, Vt, scale=scale)[0, :, 0].numpy()
    assert np.allclose(got[0], ref, rtol=1e-11, atol=1e-12)


def test_attention_single_token_returns_value(orc):
    L = _small_layer(orc, 1)
    q = np.random.default_rng(1).standard_normal((1, 4, 128)).astype(np.float32)
    out = L.attention(q, None, 0.1)
    vh = orc.dequant_array(L.v_codes(), L.v_meta(), L.bits)[0]
    for h in range(4):
        assert np.allclose(out[0, h], vh[h // 2, 0], rtol=0, atol=1e-14)


def test_attention_equal_keys_is_mean_of_values(orc):
    rng = np.random.default_rng(2)
    T = 37
    k = np.repeat(rng.standard_normal((1, 1, 2, 128)).astype(np.float32), T, axis=1)
    v = rng.standard_normal((1, T, 2, 128)).astype(np.float32)
    L = orc.Layer(1, 2, 4096, 4)
    L.append(k, v, None)
    out = L.attention(rng.standard_normal((1, 4, 128)).astype(np.float32), None, 0.2)
    vh = orc.dequant_array(L.v_codes(), L.v_meta(), L.bits)[0]
    for h in range(4):
        assert np.allclose(out[0, h], vh[h // 2].mean(axis=0), atol=1e-13)


def test_attention_brute_force_tiny(orc):
    """T <= 8: direct softmax-weighted sum with Python floats."""
    rng = np.random.default_rng(11)
    for T in (1, 2, 5, 8):
        k = rng.standard_normal((1, T, 2, 128)).astype(np.float32)
        v = rng.standard_normal((1, T, 2, 128)).astype(np.float32)
        L = orc.Layer(1, 2, 4096, 4)
        L.append(k, v, None)
        q = rng.standard_normal((1, 4, 128)).astype(np.float32)
        out = L.attention(q, None, 0.09)
        kh = orc.dequant_array(L.k_codes(), L.k_meta(), 16)[0]
        vh = orc.dequant_array(L.v_codes(), L.v_meta(), 16)[0]
        for hq in range(4):
            j = hq // 2
            s = [0.09 * sum(float(q[0, hq, c]) * kh[j, t, c] for c in range(128)) for t in range(T)]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            tot = sum(w)
            for c in (0, 17, 127):
                o = sum(w[t] / tot * vh[j, t, c] for t in range(T))
                assert out[0, hq, c] == pytest.approx(o, rel=1e-12, abs=1e-13)


def test_migration_invariance_fp64(orc):
    """Key design 3 / QServe: softmax((q lambda)(K/lambda)^T) = softmax(q K^T)."""
    rng = np.random.default_rng(3)
    T, hq, hkv = 50, 4, 2
    q = rng.standard_normal((hq, 128))
    k = rng.standard_normal((T, hkv, 128))
    k[:, :, [5, 9]] *= 20
    v = rng.standard_normal((T, hkv, 128))
    lam = np.abs(k).max(axis=0) ** 0.5
    a = orc.attention_dense(q, k, v, 0.088)
    b = orc.attention_dense(q * np.repeat(lam, 2, axis=0), k / lam[None], v, 0.088)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- generator

def test_rope_lowest_period_matches_note():
    import kvq_synth as S
    with open(os.path.join(GOLDEN, "rope_period.json")) as f:
        g = json.load(f)
    assert round(S.lowest_period(g["head_dim"], g["rope_theta"])) == g["lowest_period_tokens"]


def test_rope_preserves_pair_norms():
    import kvq_synth as S
    x = torch.randn(3, 9, 2, 128)
    y = S.apply_rope(x, torch.arange(100, 109))
    n0 = x[..., :64] ** 2 + x[..., 64:] ** 2
    n1 = y[..., :64] ** 2 + y[..., 64:] ** 2
    assert torch.allclose(n0, n1, rtol=1e-5, atol=1e-5)
    assert torch.equal(S.apply_rope(x, torch.zeros(9, dtype=torch.long)), x)
