"""kvq_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory where they run decode (an allocator owned by a host framework,
a serving loop that must not allocate after start-up).  It keeps its split
partials in a fixed scratch buffer inside the library instead of a caller
workspace.  Its result must equal kvq_decode_attn's, call after call.

This file is collected last on purpose; it builds everything it needs itself,
so it also passes when run alone in a fresh process."""
import math

import pytest
import torch

import kvq_synth as S

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixed_precision_kv_kvq_b200 import build

    build.build()
    import mixed_precision_kv_kvq_b200 as m

    m.load()
    return m


@pytest.mark.parametrize("fbit,tokens,G", [(2, 3000, 7), (4, 1500, 8), (16, 200, 5)])
def test_noalloc_matches_workspace_entry_point(kvq, fbit, tokens, G):
    """Same kernel, same split plan, same inputs: the output must equal the
    workspace entry point's bit for bit, on two calls in a row (the second
    finds the first call's partials still in the shared scratch)."""
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
    for _ in range(2):
        o = torch.full_like(ref, float("nan"))
        kvq.kvq_decode_attn_noalloc(cache.handle, 0, q, scale, o)
        outs.append(o)
    torch.cuda.synchronize()
    cache.device_status()
    assert torch.isfinite(ref).all()
    for o in outs:
        assert torch.equal(o, ref)
    cache.free()


def test_noalloc_one_slice_per_stream_needs_no_scratch(kvq):
    """8192 streams of one token each: every stream is one slice, whose result
    goes straight to the output, so the call is accepted even though that
    many partials would not fit the scratch, and equals the workspace call."""
    B, H = 512, 16
    budget = 512 * B * H * 2 * (16 * 2 + 4)
    cache = kvq.KVQCache(1, B, H, budget, [2])
    k, v = S.keys_values(9, 0, B, 1, H, 0, 3, dtype=torch.bfloat16)
    cache.append(0, k.cuda(), v.cuda())
    q = S.queries(9, 0, 0, B, H, 1).cuda()
    ref = cache.decode_attn(0, q, 0.1)
    out = torch.full_like(ref, float("nan"))
    kvq.kvq_decode_attn_noalloc(cache.handle, 0, q, 0.1, out)
    torch.cuda.synchronize()
    cache.device_status()
    assert torch.equal(out, ref)
    cache.free()


def test_noalloc_rejects_blocks_beyond_its_scratch(kvq):
    """2048 streams with the sink + window: 71 tokens in the progressive cache
    (one slice per stream) and the 129-token window in three slices, four
    partials per stream, 34 MB in all -- more than the 24 MiB scratch: the
    call is refused, writes nothing, and the workspace entry point still
    serves the block."""
    B, H, T = 256, 8, 200
    budget = 512 * B * H * 2 * (16 * 2 + 4)
    cache = kvq.KVQCache(1, B, H, budget, [2], sink_window=True)
    k, v = S.keys_values(11, 0, B, T, H, 0, 3, dtype=torch.bfloat16)
    cache.append(0, k.cuda(), v.cuda())
    q = S.queries(11, 0, 0, B, H, T).cuda()
    out = torch.full((B, H, 128), 7.0, dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attn_noalloc(cache.handle, 0, q, 0.1, out)
    assert e.value.status == 6 and "built-in buffer" in str(e.value)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    ref = cache.decode_attn(0, q, 0.1)
    torch.cuda.synchronize()
    cache.device_status()
    assert torch.isfinite(ref).all()
    cache.free()
