"""Randomised GPU parity: seeded random shapes, widths, options, input dtypes
and append schedules (single tokens, short runs, long chunks in any mix),
each checked against the oracle -- codes and meta bit-exact, attention
within 2e-3 -- at a random point on the way and at the end.  The fixed cases
of test_gpu_parity.py cover one feature each; these mix them."""
import os

import numpy as np
import pytest
import torch

import kvq_synth as S
from test_gpu_parity import CPair, Pair, WPair, kvq, lam_for  # noqa: F401  (kvq: the fixture)

pytestmark = pytest.mark.gpu

MODES = ("plain", "window", "chan", "direct")
# the case seeds: 7000 .. 7047 by default; KVQ_FUZZ_SEED and KVQ_FUZZ_CASES run others
SEED0 = int(os.environ.get("KVQ_FUZZ_SEED", "7000"))
CASES = int(os.environ.get("KVQ_FUZZ_CASES", "48"))


def schedule(rng, total):
    """Chunk sizes summing to total: 30% single tokens, 40% runs of 2-39,
    30% chunks of 40-1199."""
    sizes, left = [], total
    while left > 0:
        r = rng.random()
        n = 1 if r < 0.3 else int(rng.integers(2, 40)) if r < 0.7 else int(rng.integers(40, 1200))
        n = min(n, left)
        sizes.append(n)
        left -= n
    return sizes


@pytest.mark.parametrize("case", range(CASES))
def test_random_mix(kvq, orc, case):
    rng = np.random.default_rng(SEED0 + case)
    mode = MODES[case % len(MODES)]
    B = int(rng.integers(1, 4))
    H = int(rng.choice([1, 2, 4]))
    G = int(rng.integers(1, 9))
    fbit = int(rng.choice([2, 2, 4, 8] if mode in ("chan", "direct") else [2, 2, 4, 8, 16]))
    dtype = torch.float32 if rng.random() < 0.4 else torch.bfloat16
    if mode == "chan":
        n_f = int(rng.choice([1024, 2048]))
        cap = n_f + 127
    else:
        n_f = int(rng.choice([512, 1024, 2048]))
        cap = n_f + 129 if mode == "window" else n_f
    T = int(rng.integers(cap // 2, cap + 1))
    seed = 300 + SEED0 - 7000 + case
    k, v = S.keys_values(seed, fbit, B, T, H, 0, int(rng.integers(1, 6)), dtype=dtype)
    lam = lam_for(k) if rng.random() < 0.7 else None
    shift = kvq.KVQ_SHIFT_DIRECT if mode == "direct" else 0
    if mode == "window":
        P = WPair(kvq, orc, B, H, n_f, fbit, lam, shift_mode=shift)
    elif mode == "chan":
        P = CPair(kvq, orc, B, H, n_f, fbit, lam, shift_mode=int(rng.integers(0, 2)))
    else:
        P = Pair(kvq, orc, B, H, n_f, fbit, lam, shift_mode=shift)
    sizes = schedule(rng, T)
    mid = int(rng.integers(0, len(sizes)))
    pos = 0
    for i, n in enumerate(sizes):
        P.append(k[:, pos:pos + n], v[:, pos:pos + n])
        pos += n
        if i == mid or pos == T:
            P.check_codes()
            P.check_attention(S.queries(seed, fbit, i, B, H * G, pos, dtype=torch.bfloat16))
    assert pos == T
