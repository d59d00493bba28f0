"""Block-wise bit allocation (PM-KVQ note, key design 2): the oracle's
enumeration pinned against a closed form, and libkvq's exact solver
(`kvq_allocate_bits`, host code, no GPU) against the oracle."""
import numpy as np
import pytest

from oracle import oracle as orc


def greedy_two_widths(sens, batch, kv_heads, max_tokens, budget, lo=2, hi=4):
    """Closed form for two widths with the same cost for every block: the
    blocks that move from lo to hi are the K with the largest positive
    gains s_lo - s_hi, K = how many upgrades the budget leaves room for."""
    layers = sens.shape[0]
    c_lo = orc.block_bytes(lo, batch, kv_heads, max_tokens)
    c_hi = orc.block_bytes(hi, batch, kv_heads, max_tokens)
    if layers * c_lo > budget:
        return None
    k = min(layers, (budget - layers * c_lo) // (c_hi - c_lo))
    gains = np.sort(sens[:, 0] - sens[:, 1])[::-1]
    gains = gains[:k]
    return float(sens[:, 0].sum() - gains[gains > 0].sum())


@pytest.mark.parametrize("seed", range(6))
def test_oracle_enumeration_matches_closed_form(seed):
    rng = np.random.default_rng(seed)
    layers = int(rng.integers(1, 11))
    sens = rng.random((layers, 2)) * 10
    sens[:, 1] *= rng.random(layers)  # the wider width is usually, not always, better
    if seed % 2:
        sens[0, 1] = sens[0, 0] + 1.0  # one block where the wide width is worse
    B, H, N = 2, 3, 1024
    c2, c4 = orc.block_bytes(2, B, H, N), orc.block_bytes(4, B, H, N)
    for k in range(layers + 1):
        budget = layers * c2 + k * (c4 - c2) + int(rng.integers(0, c4 - c2))
        best, args = orc.allocate_bits_brute(sens, [2, 4], B, H, N, budget)
        want = greedy_two_widths(sens, B, H, N, budget)
        assert best == pytest.approx(want, rel=1e-12, abs=1e-12)
        assert args


def test_oracle_budget_extremes():
    sens = np.array([[3.0, 1.0, 0.5], [2.0, 1.5, 0.1]])
    B, H, N = 1, 1, 512
    bits = [2, 4, 8]
    # everything fits: the best width per block
    best, args = orc.allocate_bits_brute(sens, bits, B, H, N, 10 ** 12)
    assert best == pytest.approx(0.6) and args == [(8, 8)]
    # only the narrowest fits
    best, args = orc.allocate_bits_brute(sens, bits, B, H, N, 2 * orc.block_bytes(2, B, H, N))
    assert best == pytest.approx(5.0) and args == [(2, 2)]
    # nothing fits
    assert orc.allocate_bits_brute(sens, bits, B, H, N, 2 * orc.block_bytes(2, B, H, N) - 1) == (None, [])


@pytest.fixture(scope="module")
def kvq():
    from mixed_precision_kv_kvq_b200 import build

    build.build()
    import mixed_precision_kv_kvq_b200 as m

    m.load()
    return m


def objective(sens, bits, fbit):
    return float(sum(sens[i, bits.index(b)] for i, b in enumerate(fbit)))


def total_bytes(fbit, B, H, N):
    return sum(orc.block_bytes(b, B, H, N) for b in fbit)


@pytest.mark.parametrize("seed", range(12))
def test_solver_matches_enumeration(kvq, seed):
    rng = np.random.default_rng(100 + seed)
    layers = int(rng.integers(1, 9))
    bits = [int(b) for b in rng.choice([2, 4, 8, 16], size=int(rng.integers(2, 4)), replace=False)]
    sens = rng.random((layers, len(bits))) * 5
    B, H, N = int(rng.integers(1, 5)), int(rng.integers(1, 9)), int(rng.integers(1, 9)) * 512
    lo = layers * orc.block_bytes(min(bits), B, H, N)
    hi = layers * orc.block_bytes(max(bits), B, H, N)
    for budget in (lo, (lo + hi) // 2, int(lo + (hi - lo) * rng.random()), hi, 2 * hi):
        best, args = orc.allocate_bits_brute(sens, bits, B, H, N, budget)
        fbit, obj = kvq.kvq_allocate_bits(sens, bits, B, H, N, budget)
        assert total_bytes(fbit, B, H, N) <= budget
        assert obj == pytest.approx(best, rel=1e-12, abs=1e-12)
        assert objective(sens, bits, fbit) == pytest.approx(best, rel=1e-12, abs=1e-12)
        assert tuple(fbit) in args


def test_solver_80_blocks_two_widths(kvq):
    """A 70B-shaped model (80 blocks, widths {2, 4}): the closed form."""
    rng = np.random.default_rng(7)
    sens = np.stack([rng.random(80) * 10, rng.random(80) * 3], axis=1)
    B, H, N = 8, 8, 131072
    c2, c4 = orc.block_bytes(2, B, H, N), orc.block_bytes(4, B, H, N)
    for k in (0, 1, 20, 55, 80):
        budget = 80 * c2 + k * (c4 - c2)
        fbit, obj = kvq.kvq_allocate_bits(sens, [2, 4], B, H, N, budget)
        assert sum(1 for b in fbit if b == 4) <= k
        assert obj == pytest.approx(greedy_two_widths(sens, B, H, N, budget), rel=1e-12)
        # the result goes straight into the cache's budget rule
        assert kvq.kvq_pool_bytes(80, B, H, 128, budget, fbit) > 0


def test_solver_rejects(kvq):
    sens = np.ones((3, 2))
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_allocate_bits(sens, [2, 4], 1, 1, 512, 3 * orc.block_bytes(2, 1, 1, 512) - 1)
    assert e.value.status == 2  # BUDGET
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_allocate_bits(sens, [2, 3], 1, 1, 512, 10 ** 12)
    assert e.value.status == 1
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_allocate_bits(sens, [4, 4], 1, 1, 512, 10 ** 12)
    assert e.value.status == 1
    bad = sens.copy()
    bad[1, 0] = np.nan
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_allocate_bits(bad, [2, 4], 1, 1, 512, 10 ** 12)
    assert e.value.status == 1
