"""kvq_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory where they run decode (an allocator owned by a host framework,
a serving loop that must not allocate after start-up).  It keeps its split
partials in a fixed scratch buffer inside the library instead of a caller
workspace.  Its result must match kvq_decode_attn's, call after call.

This file is collected last on purpose; it builds everything it needs itself,
so it also passes when run alone in a fresh process."""
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


def _rel_err(out, ref):
    out = out.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float((np.abs(out - ref).max(axis=-1) / np.abs(ref).max(axis=-1)).max())


@pytest.mark.parametrize("fbit,tokens,G", [(2, 3000, 7), (4, 1500, 8), (16, 200, 5)])
def test_noalloc_matches_workspace_entry_point(kvq, fbit, tokens, G):
    B, H, n_f = 4, 2, 4096
    budget = n_f * B * H * 2 * (16 * fbit + 4)
    cache = kvq.KVQCache(1, B, H, budget, [fbit])
    k, v = S.keys_values(7, fbit, B, tokens, H, 0, 3, dtype=torch.bfloat16)
    cache.set_lambda(0, k.float().abs().amax(dim=(0, 1)).clamp_min(1e-6).pow(0.5))
    cache.append(0, k.cuda(), v.cuda())
    q = S.queries(7, fbit, 0, B, H * G, tokens).cuda()
    scale = 1 / math.sqrt(128)
    ref = cache.decode_attn(0, q, scale)
    outs = []
    for _ in range(2):  # two calls in a row share the same scratch buffer
        o = torch.full_like(ref, float("nan"))
        kvq.kvq_decode_attn_noalloc(cache.handle, 0, q, scale, o)
        outs.append(o)
    torch.cuda.synchronize()
    cache.device_status()
    for o in outs:
        assert torch.isfinite(o).all()
        assert _rel_err(o, ref) <= TOL
    cache.free()


def test_noalloc_rejects_blocks_beyond_its_scratch(kvq):
    # 512 sequences x 16 KV heads = 8192 streams need ~34 MB of partials
    B, H = 512, 16
    budget = 512 * B * H * 2 * (16 * 2 + 4)
    cache = kvq.KVQCache(1, B, H, budget, [2])
    k = torch.zeros(B, 1, H, 128, dtype=torch.bfloat16, device="cuda")
    cache.append(0, k, k)
    q = torch.zeros(B, H, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(B, H, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attn_noalloc(cache.handle, 0, q, 0.1, out)
    assert e.value.status == 6 and "built-in buffer" in str(e.value)
    cache.free()
