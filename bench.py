"""Benchmark of the PM-KVQ hot path on B200.

Workload (one step): a decode step of a DeepSeek-R1-Distill-Qwen-7B-shaped
model -- 28 blocks, 28 query / 4 KV heads, head_dim 128, batch 16, about
32768 cached tokens per sequence, Fbit 4 for block 0 and the last 8 blocks and
2 elsewhere.  Per block: quantize-on-append of the new token's K/V (with the
budget-triggered shrink check) and GQA decode attention over the packed cache.
Inputs are synthetic (seeded Gaussian K/V/Q with RoPE and x20 outlier Key
channels); the cache (~5.4 GB) is far larger than L2, and every block's read
(151-285 MB) exceeds L2, so no flush is needed between steps.

Printed: one JSON line.  `value` is the step's algorithmic HBM bytes
(attention reads of codes + meta + Q/O, append reads/writes) divided by the
device time of the step.  `roofline` reports the decode-attention kernel
alone; `shrink` the Equivalent-Right-Shift kernel on a full 128K-token block
of a Llama-70B-shaped layer (4 -> 2 bits) and on the 7B progressive-stream
events; `cpu_baseline` the CPU oracle on a bounded sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kvq_synth as S  # noqa: E402

METRIC = "decode-attn HBM GB/s & % of B200 peak over packed mixed-bit KV; shrink GB/s"
HEAD_DIM = 128
SEED = 0

# 7B decode workload
L7, HQ7, HKV7, B7, T7 = 28, 28, 4, 16, 32768
FBIT7 = [4 if (l == 0 or l >= L7 - 8) else 2 for l in range(L7)]
ROOM = 4096  # tokens of head-room for the appended decode tokens
# Llama-70B long-CoT workload
L70, HQ70, HKV70, B70, T70 = 80, 64, 8, 8, 131072
FBIT70 = [4 if l % 4 == 0 else 2 for l in range(L70)]
ROOM70 = 512
WORKLOAD70 = ("Llama-70B-shape long-CoT decode: 80 layers, 64 Q / 8 KV heads, head_dim 128, batch 8, context 131072, "
              "Fbit 4 for every 4th layer (0, 4, ...) else 2; one decode step = append + attention per layer")
WORKLOAD = ("DeepSeek-R1-Distill-Qwen-7B-shape decode: 28 layers, 28 Q / 4 KV heads, head_dim 128, "
            "batch 16, context 32768, Fbit 4 for layer 0 and the last 8 layers else 2; one decode step "
            "= append + attention per layer")


def per_token_bytes(batch, kv_heads, fbit):
    return batch * kv_heads * 2 * sum(16 * f + 4 for f in fbit)


def decode_bytes(batch, kv_heads, q_heads, tokens, bits):
    """Algorithmic bytes of one decode-attention call: every cached code and
    meta word once, Q (bf16) in, O (fp32) out."""
    return (batch * kv_heads * tokens * 2 * (16 * bits + 4)
            + batch * q_heads * HEAD_DIM * (2 + 4))


def append_bytes(batch, kv_heads, n, bits):
    """bf16 K/V in, codes + meta out."""
    return batch * kv_heads * n * 2 * (HEAD_DIM * 2 + 16 * bits + 4)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def code_tokens(text):
    """C/CUDA source with comments removed and whitespace runs collapsed, so
    that an edit to comments or layout leaves the digest unchanged.  String
    and character literals are kept verbatim."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif c.isspace():
            while i < n and text[i].isspace():
                i += 1
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest():
    """sha256 of the decode kernel's code (kvq_decode.cu, kvq_decode_common.cuh
    and kvq_internal.cuh, comments and whitespace removed): ncu counters stay valid only while it
    matches the digest recorded with them."""
    import hashlib
    h = hashlib.sha256()
    for name in ("kvq_decode.cu", "kvq_decode_common.cuh", "kvq_internal.cuh"):
        with open(os.path.join(ROOT, "mixed_precision_kv_kvq_b200", "csrc", name)) as f:
            h.update(code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")


def decode_traffic(fbit, path=TRAFFIC_FILE):
    """DRAM bytes per decode launch (ncu dram__bytes_read.sum +
    dram__bytes_write.sum, averaged over the layers' bit widths) from the
    committed traffic record, or None when the kernel changed since."""
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None, "no ncu traffic record"
    if rec.get("source_digest") != source_digest():
        return None, "kernel changed since the ncu capture"
    per = rec.get("bytes_per_launch", {})
    if not all(f"{b}bit" in per for b in fbit):
        return None, "no capture for some bit width"
    return int(sum(per[f"{b}bit"] for b in fbit) / len(fbit)), "profiles/decode_traffic.json"


def calib_lambda(k):
    """Migration factor from the first chunk of a block's keys (the note's
    calibration rule lambda_i = (max_m |K_m,i|)^alpha, alpha = 1/2)."""
    return k.float().abs().amax(dim=(0, 1)).clamp_min(1e-6).pow(0.5)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- GPU arm

def build_cache(kvq, dev, layers, batch, kv_heads, fbit, tokens, n_f, seed, n_out, chunk=4096, shift_mode=None,
                sink_window=False, key_channel=False):
    budget = n_f * per_token_bytes(batch, kv_heads, fbit)
    cache = kvq.KVQCache(layers, batch, kv_heads, budget, fbit, device=dev, sink_window=sink_window,
                         key_channel=key_channel)
    assert cache.max_tokens == n_f + (129 if sink_window else (127 if key_channel else 0)), (cache.max_tokens, n_f)
    if shift_mode is not None:
        for l in range(layers):
            cache.set_shift_mode(l, shift_mode)
    for l in range(layers):
        pos = 0
        while pos < tokens:
            n = min(chunk, tokens - pos)
            k, v = S.keys_values(seed, l, batch, n, kv_heads, pos, n_out, dtype=torch.bfloat16, device=dev)
            if pos == 0:
                cache.set_lambda(l, calib_lambda(k))
            cache.append(l, k, v)
            pos += n
    torch.cuda.synchronize(dev)
    return cache


def flush_l2(buf):
    buf.add_(1)


def measure_shrink(kvq, dev, flush_buf, blocks_7b=20, blocks_70b=3):
    """Shrink kernel GB/s (algorithmic: the block's code region read, half of
    it written; the Direct Right Shift also reads and rewrites the meta of
    every token).  Each event is timed on several blocks of one cache, each
    filled to the point where its next token would shrink it: the blocks are
    shrunk back to back (one launch each, every launch on a block no other
    launch touches) with CUDA events around the batch after an L2 flush, and
    the time per launch is the batch time over the blocks.
    (a) Llama-70B-shape layer (batch 8, 8 KV heads), Fbit 2, a block full with
    131072 tokens at 4 bits shrinking to 2 bits, with either shift.  (b) the
    7B progressive stream (batch 8, 4 KV heads, 32768 tokens at Fbit 2):
    events 16->8 at 4096, 8->4 at 8192, 4->2 at 16384 tokens."""
    res = {}
    stream = torch.cuda.current_stream(dev)

    def one(batch, kv_heads, n_f, fbit, fill_tokens, tag, blocks, direct=False):
        cache = build_cache(kvq, dev, blocks, batch, kv_heads, [fbit] * blocks, fill_tokens, n_f, SEED + 17, 10,
                            chunk=8192, shift_mode=kvq.KVQ_SHIFT_DIRECT if direct else None)
        st = [cache.query(l) for l in range(blocks)]
        assert all(x["tokens"] == x["capacity"] == fill_tokens for x in st), st
        region = batch * kv_heads * 2 * n_f * 16 * fbit  # code bytes of one block
        nbytes = region + region // 2
        if direct:  # the meta of every stored token is read and rewritten too
            nbytes += 2 * batch * kv_heads * fill_tokens * 2 * 4
        flush_l2(flush_buf)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("timed")
        e0.record(stream)
        for l in range(blocks):
            cache.shrink(l)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_pop()
        cache.device_status()
        t = e0.elapsed_time(e1) / 1e3 / blocks
        bits_from = st[0]["bits"]
        assert all(cache.query(l)["bits"] == bits_from // 2 for l in range(blocks))
        cache.free()
        del cache
        res[tag] = {"gbs": round(nbytes / t / 1e9, 1), "us": round(t * 1e6, 2), "bytes": nbytes,
                    "bits": f"{bits_from}->{bits_from // 2}", "launches": blocks,
                    "timing": f"{blocks} blocks shrunk back to back after an L2 flush, CUDA events around the "
                              "batch, time per launch"}

    one(8, 8, 262144, 2, 131072, "llama70b_128k_4to2", blocks_70b)
    one(8, 8, 262144, 2, 131072, "llama70b_128k_4to2_direct_shift", blocks_70b, direct=True)
    for tokens, tag in ((4096, "qwen7b_16to8"), (8192, "qwen7b_8to4"), (16384, "qwen7b_4to2")):
        one(8, 4, 32768, 2, tokens, tag, blocks_7b)
    return res


def measure_append_chunk(kvq, dev, flush_buf, reps=15):
    """Chunked appends of 4096 tokens (7B shape, batch 8, 4 KV heads) into a
    2-bit block: `reps` back-to-back calls, each with its own input chunk (so
    every input is read from HBM), CUDA events around the batch after an L2
    flush; time per call."""
    batch, kv_heads, n = 8, 4, 4096
    n_f = 131072
    pre = n_f // 2 + n  # past the 4 -> 2 shrink at n_f / 2 tokens
    assert pre + reps * n <= n_f
    cache = build_cache(kvq, dev, 1, batch, kv_heads, [2], pre, n_f, SEED + 5, 5, chunk=8192)
    st = cache.query(0)
    assert st["bits"] == 2
    chunks = [S.keys_values(SEED, 99, batch, n, kv_heads, pre + r * n, 5, dtype=torch.bfloat16, device=dev)
              for r in range(reps)]
    torch.cuda.synchronize(dev)
    flush_l2(flush_buf)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    e0.record(stream)
    for k, v in chunks:
        cache.append(0, k, v)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    cache.device_status()
    assert cache.query(0)["bits"] == 2 and cache.query(0)["tokens"] == pre + reps * n
    cache.free()
    nb = append_bytes(batch, kv_heads, n, 2)
    t = e0.elapsed_time(e1) / 1e3 / reps
    return {"gbs": round(nb / t / 1e9, 1), "us": round(t * 1e6, 2), "bytes": nb, "bits": 2, "tokens": n,
            "batch": batch, "timing": f"{reps} back-to-back appends of distinct chunks after an L2 flush, CUDA events "
                                      "around the batch, time per call"}


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's device time (every rank passes its own)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank: int, ms: float, world: int) -> float:
    """Replicas: every rank moves the same bytes; the job's rate is all
    ranks' bytes over the slowest rank's time."""
    return world * bytes_per_rank / (ms / 1e3) / 1e9


def _decode_args(kvq, cache, q, out, ws, stream):
    import ctypes as C
    return (cache.handle, 0, C.c_void_p(q.data_ptr()), q.shape[1], C.c_float(HEAD_DIM ** -0.5),
            C.c_void_p(out.data_ptr()), C.c_void_p(ws.data_ptr()), ws.numel() * 4, C.c_void_p(stream.cuda_stream))


def measure_decode_configs(kvq, dev, reps=20):
    """Decode attention of one block of each model-shaped workload at both of
    its widths: `reps` back-to-back launches on one block (CUDA events around
    the batch; the block's read exceeds L2), mean per launch."""
    lib = kvq.load()
    stream = torch.cuda.current_stream(dev)
    res = {}
    cfgs = (("qwen7b", 16, 4, 28, 32768, 32768 + ROOM),
            ("qwen32b", 16, 8, 40, 32768, 55296),
            ("llama70b", 8, 8, 64, 131072, 131072))
    runs = [(c, fbit, "") for c in cfgs for fbit in (2, 4)]
    runs.append((("qwen7b_sink_window", 16, 4, 28, 32768 + 129, 32768), 2, "window"))
    runs += [(("qwen7b_key_channel", 16, 4, 28, 32768 + 100, 32768), fbit, "chan") for fbit in (2, 4)]
    for (name, batch, kv_heads, q_heads, tokens, n_f), fbit, mode in runs:
        window = mode == "window"
        cache = build_cache(kvq, dev, 1, batch, kv_heads, [fbit], tokens, n_f, SEED + 31, S.outliers_for(kv_heads),
                            chunk=8192, sink_window=window, key_channel=mode == "chan")
        assert cache.query(0)["bits"] == fbit
        q = S.queries(SEED, 0, 0, batch, q_heads, tokens, dtype=torch.bfloat16, device=dev)
        out = torch.empty((batch, q_heads, HEAD_DIM), dtype=torch.float32, device=dev)
        ws = cache.workspace(0, q_heads)
        a = _decode_args(kvq, cache, q, out, ws, stream)
        for _ in range(3):
            kvq.check(lib.kvq_decode_attn(*a))
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            lib.kvq_decode_attn(*a)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        cache.device_status()
        us = e0.elapsed_time(e1) / reps * 1e3
        nb = decode_bytes(batch, kv_heads, q_heads, tokens, fbit)
        if window or mode == "chan":  # the sink and the window, or the staged tokens, are read at 16 bits
            w = 129 if window else tokens % 128
            nb = decode_bytes(batch, kv_heads, q_heads, tokens - w, fbit) + \
                decode_bytes(batch, kv_heads, q_heads, w, 16) - batch * q_heads * HEAD_DIM * (2 + 4)
        res[f"{name}_{fbit}bit"] = {"us": round(us, 2), "gbs": round(nb / us / 1e3, 1), "bytes": nb,
                                    "batch": batch, "kv_heads": kv_heads, "q_heads": q_heads, "tokens": tokens}
        cache.free()
        del cache
    res["timing"] = (f"{reps} back-to-back calls on one block, CUDA events around the batch, mean per call "
                     "(with the sink + window or per-channel Key groups: two launches a call, the window or the "
                     "staged block at 16 bits and the rest; per-channel Key groups count their (R, Z) per channel "
                     "and 128-token block, the same bytes as per token)")
    return res


def measure_block_append_key_channel(kvq, dev, reps=50):
    """Per-channel Key groups: appends of 128 tokens that each complete a
    block with nothing staged, so the block goes from the input straight into
    the progressive cache in one launch (each token quantized to INT16 as the
    staging would hold it, then Keys quantized per channel over the block and
    Values shift-chained) on a 7B-shaped 2-bit block (batch 16, 4 KV heads)
    holding 16384 tokens; `reps` back-to-back calls, mean."""
    import ctypes as C
    lib = kvq.load()
    stream = torch.cuda.current_stream(dev)
    cache = build_cache(kvq, dev, 1, B7, HKV7, [2], 16384, 32768, SEED + 51, S.outliers_for(HKV7), chunk=8192,
                        key_channel=True)
    g = torch.Generator(device=dev)
    g.manual_seed(SEED + 53)
    kin = torch.randn((B7, 128, HKV7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    vin = torch.randn((B7, 128, HKV7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    sp = C.c_void_p(stream.cuda_stream)
    args = (cache.handle, 0, C.c_void_p(kin.data_ptr()), C.c_void_p(vin.data_ptr()), kvq.KVQ_DTYPE_BF16, 128, sp)
    for _ in range(3):
        kvq.check(lib.kvq_append(*args))
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        lib.kvq_append(*args)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    cache.device_status()
    us = e0.elapsed_time(e1) / reps * 1e3
    st = cache.query(0)
    assert st["tokens"] == 16384 + 128 * (reps + 3) and st["bits"] == 2
    cache.free()
    streams = B7 * HKV7
    # bf16 K/V in, codes at 2 bits + meta out (per-token Value meta; the Keys'
    # per-channel meta is one word per channel of the block, as many bytes)
    nb = append_bytes(B7, HKV7, 128, 2)
    return {"us": round(us, 2), "gbs": round(nb / us / 1e3, 1), "bytes": nb, "tokens": 128, "batch": B7,
            "kv_heads": HKV7, "bits": 2, "streams": streams,
            "timing": f"{reps} back-to-back 128-token appends (one launch each), CUDA events around the batch"}


def measure_append_token(kvq, dev, reps=200, sink_window=False):
    """Single-token append on a 7B-shaped block (batch 16, 4 KV heads, 2-bit,
    32768 tokens cached): `reps` back-to-back calls through the C ABI, mean.
    With the sink + window every call also moves the token leaving the window."""
    import ctypes as C
    lib = kvq.load()
    stream = torch.cuda.current_stream(dev)
    cache = build_cache(kvq, dev, 1, B7, HKV7, [2], T7, T7 + ROOM, SEED + 41, S.outliers_for(HKV7), chunk=8192,
                        sink_window=sink_window)
    g = torch.Generator(device=dev)
    g.manual_seed(SEED + 43)
    kin = torch.randn((reps + 3, B7, 1, HKV7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    vin = torch.randn((reps + 3, B7, 1, HKV7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    sp = C.c_void_p(stream.cuda_stream)
    for i in range(3):
        kvq.check(lib.kvq_append(cache.handle, 0, C.c_void_p(kin[i].data_ptr()), C.c_void_p(vin[i].data_ptr()),
                                 kvq.KVQ_DTYPE_BF16, 1, sp))
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(3, reps + 3):
        lib.kvq_append(cache.handle, 0, C.c_void_p(kin[i].data_ptr()), C.c_void_p(vin[i].data_ptr()),
                       kvq.KVQ_DTYPE_BF16, 1, sp)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) / reps * 1e3
    assert cache.query(0)["tokens"] == T7 + reps + 3
    cache.free()
    nb = append_bytes(B7, HKV7, 1, 2)
    return {"us": round(us, 2), "gbs": round(nb / us / 1e3, 2), "bytes": nb, "batch": B7, "kv_heads": HKV7,
            "bits": 2, "timing": f"{reps} back-to-back single-token appends, CUDA events around the batch; "
                                 "launch-latency bound"}


def serve_steps(cache, kh, vh, qh, oh, sm_scale, dev, stream):
    """A serving loop's decode steps through the public API, end to end:
    step i's K, V, Q (kh[i], vh[i], qh[i]: pinned host [layers][...]) go to
    the device, every block runs KVQCache.append_decode on device views, and
    the step's outputs come back to pinned host memory (oh).  Double-buffered
    on a copy stream: step i+1's inputs arrive and step i-1's outputs leave
    while step i computes.  Returns the device time in ms of all the steps,
    every copy included (CUDA events on `stream`)."""
    E, layers = kh.shape[0], kh.shape[1]
    cs = torch.cuda.Stream(dev)
    bufs = [(torch.empty(kh.shape[1:], dtype=kh.dtype, device=dev), torch.empty(vh.shape[1:], dtype=vh.dtype, device=dev),
             torch.empty(qh.shape[1:], dtype=qh.dtype, device=dev), torch.empty(oh.shape, dtype=oh.dtype, device=dev))
            for _ in range(2)]
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]      # step's compute finished (inputs read, output written)
    drained = [torch.cuda.Event() for _ in range(2)]   # step's output copied out

    def fetch(i):
        b = i % 2
        with torch.cuda.stream(cs):
            if i >= 2:
                cs.wait_event(done[b])  # the step that last read these buffers
            kd, vd, qd, _ = bufs[b]
            kd.copy_(kh[i], non_blocking=True)
            vd.copy_(vh[i], non_blocking=True)
            qd.copy_(qh[i], non_blocking=True)
            in_ready[b].record(cs)

    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    cs.wait_event(f0)
    fetch(0)
    for i in range(E):
        b = i % 2
        if i + 1 < E:
            fetch(i + 1)
        kd, vd, qd, od = bufs[b]
        stream.wait_event(in_ready[b])
        if i >= 2:
            stream.wait_event(drained[b])  # output buffer b copied out by then
        for l in range(layers):
            cache.append_decode(l, kd[l], vd[l], qd[l], sm_scale, out=od[l])
        done[b].record(stream)
        with torch.cuda.stream(cs):
            cs.wait_event(done[b])
            oh.copy_(od, non_blocking=True)
            drained[b].record(cs)
    stream.wait_stream(cs)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    return f0.elapsed_time(f1)


def measure_step_70b(kvq, dev, K, W, E, cpu=True, peak=None):
    """The Llama-70B long-CoT decode step as a whole: 80 blocks (every 4th at
    4 bits, the rest at 2), batch 8, 64 query / 8 KV heads, 131072 cached
    tokens per sequence (the cache holds 59 GB), one kvq_append_decode per
    block.  W warm-up steps, then K steps with CUDA events around the region
    only; E more steps end to end through the public API with host buffers
    (serve_steps); the CPU oracle on 70B-shaped streams beside it."""
    import ctypes as C
    lib = kvq.load()
    stream = torch.cuda.current_stream(dev)
    layers = L70
    n_f = T70 + ROOM70
    if K + W + E > ROOM70:
        raise SystemExit(f"70B step: steps + warm-up + e2e steps must be <= {ROOM70}")
    t_build = time.perf_counter()
    cache = build_cache(kvq, dev, layers, B70, HKV70, FBIT70, T70, n_f, SEED + 70, S.outliers_for(HKV70), chunk=8192)
    t_build = time.perf_counter() - t_build
    for l in range(layers):
        assert cache.query(l)["bits"] == FBIT70[l]
    sm_scale = HEAD_DIM ** -0.5
    nsteps = W + K + E
    g = torch.Generator(device=dev)
    g.manual_seed(SEED + 71)
    kin = torch.randn((nsteps, layers, B70, 1, HKV70, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    vin = torch.randn((nsteps, layers, B70, 1, HKV70, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    qin = torch.randn((nsteps, layers, B70, HQ70, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((layers, B70, HQ70, HEAD_DIM), dtype=torch.float32, device=dev)
    ws = [cache.workspace(l, HQ70) for l in range(layers)]
    sp = C.c_void_p(stream.cuda_stream)
    h = cache.handle
    scale_c = C.c_float(sm_scale)
    args = [[(h, l, C.c_void_p(kin[i, l].data_ptr()), C.c_void_p(vin[i, l].data_ptr()), kvq.KVQ_DTYPE_BF16,
              C.c_void_p(qin[i, l].data_ptr()), HQ70, scale_c, C.c_void_p(out[l].data_ptr()),
              C.c_void_p(ws[l].data_ptr()), ws[l].numel() * 4, sp) for l in range(layers)] for i in range(W + K)]

    def step(i):
        for l in range(layers):
            st = lib.kvq_append_decode(*args[i][l])
            if st:
                kvq.check(st)

    def step_bytes(t_before):
        return sum(append_bytes(B70, HKV70, 1, FBIT70[l]) + decode_bytes(B70, HKV70, HQ70, t_before + 1, FBIT70[l])
                   for l in range(layers))

    for i in range(W):
        step(i)
    torch.cuda.synchronize(dev)
    t0 = cache.query(0)["tokens"]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        e0.record(stream)
        for i in range(K):
            step(W + i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    cache.device_status()
    ms = e0.elapsed_time(e1)
    nb = sum(step_bytes(t0 + i) for i in range(K))
    value = nb / (ms / 1e3) / 1e9
    if peak is None:
        peak = peaks()[0]
    n_dec = K * layers
    res = {"value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms / K, 4), "steps": K, "warmup": W,
           "config": {"workload": WORKLOAD70, "layers": layers, "batch": B70, "q_heads": HQ70, "kv_heads": HKV70,
                      "head_dim": HEAD_DIM, "context": T70, "fbit": "4 if layer % 4 == 0 else 2",
                      "cache_gb": round(cache.pool.numel() / 1e9, 2), "build_s": round(t_build, 1),
                      "l2": "no flush: every block's cache read (0.6-1.1 GB) exceeds the 126 MB L2"},
           "roofline": {"bound": "hbm", "achieved": round(value, 1), "peak": peak, "unit": "GB/s",
                        "frac": round(value / peak, 4), "kernel": "decode_kernel (kvq_append_decode)",
                        "avg_launch_us": round(ms * 1e3 / n_dec, 2), "bytes_per_launch": int(nb / n_dec),
                        "timing": f"CUDA events around the {n_dec} launches of the timed region, all this kernel"},
           "gpu_launches": n_dec, "clocks": clk.summary()}
    if E > 0:
        kh = kin[W + K:].cpu().pin_memory()
        vh = vin[W + K:].cpu().pin_memory()
        qh = qin[W + K:].cpu().pin_memory()
        oh = torch.empty((layers, B70, HQ70, HEAD_DIM), dtype=torch.float32).pin_memory()
        t1 = cache.query(0)["tokens"]
        e2e_ms = serve_steps(cache, kh, vh, qh, oh, sm_scale, dev, stream)
        cache.device_status()
        eb = sum(step_bytes(t1 + i) for i in range(E))
        res["e2e"] = {"value": round(eb / (e2e_ms / 1e3) / 1e9, 1), "unit": "GB/s",
                      "h2d_bytes_per_step": layers * (2 * kin[0, 0].numel() * 2 + qin[0, 0].numel() * 2),
                      "d2h_bytes_per_step": layers * out[0].numel() * 4, "steps": E}
    cache.free()
    del cache, kin, vin, qin, args
    torch.cuda.empty_cache()
    if cpu:
        res["cpu_baseline"] = cpu_baseline(tokens=T70, g=HQ70 // HKV70, n_out=S.outliers_for(HKV70),
                                           budget_s=12.0, single_s=4.0, max_threads=16)
    return res


def run_gpu(args, rank, world):
    from mixed_precision_kv_kvq_b200 import build as kbuild

    kbuild.build()
    import mixed_precision_kv_kvq_b200 as kvq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    layers = args.layers
    fbit = FBIT7 if layers == L7 else [4 if l % 2 == 1 else 2 for l in range(layers)]
    K, W = args.steps, args.warmup
    if 4 * K + W > ROOM:
        raise SystemExit(f"4 * --steps + --warmup must be <= {ROOM}")
    n_f = T7 + ROOM
    n_out = S.outliers_for(HKV7)
    seed = SEED + 1000 * rank
    cache = build_cache(kvq, dev, layers, B7, HKV7, fbit, T7, n_f, seed, n_out)
    sm_scale = HEAD_DIM ** -0.5

    # per-step inputs, generated up front on the device
    nsteps = 3 * K + W  # warm-up, timed steps, per-launch-event steps, two-call steps
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 7)
    kin = torch.randn((nsteps, layers, B7, 1, HKV7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    vin = torch.randn((nsteps, layers, B7, 1, HKV7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    qin = torch.randn((nsteps, layers, B7, HQ7, HEAD_DIM), generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((layers, B7, HQ7, HEAD_DIM), dtype=torch.float32, device=dev)
    ws = [cache.workspace(l, HQ7) for l in range(layers)]
    stream = torch.cuda.current_stream(dev)

    # Raw C-ABI calls with pre-built arguments keep the host well ahead of the GPU.
    import ctypes as C
    lib = kvq.load()
    sp = C.c_void_p(stream.cuda_stream)
    h = cache.handle
    kp = [[C.c_void_p(kin[i, l].data_ptr()) for l in range(layers)] for i in range(nsteps)]
    vp = [[C.c_void_p(vin[i, l].data_ptr()) for l in range(layers)] for i in range(nsteps)]
    qp = [[C.c_void_p(qin[i, l].data_ptr()) for l in range(layers)] for i in range(nsteps)]
    op = [C.c_void_p(out[l].data_ptr()) for l in range(layers)]
    wp = [(C.c_void_p(w.data_ptr()), w.numel() * 4) for w in ws]
    scale_c = C.c_float(sm_scale)

    def step(i, ev=None):
        # one decode step per block: the new token's append and the attention
        # in one launch (kvq_append_decode)
        for l in range(layers):
            if ev is not None:
                ev[l][0].record(stream)
            st = lib.kvq_append_decode(h, l, kp[i][l], vp[i][l], kvq.KVQ_DTYPE_BF16, qp[i][l], HQ7, scale_c, op[l],
                                       wp[l][0], wp[l][1], sp)
            if st:
                kvq.check(st)
            if ev is not None:
                ev[l][1].record(stream)

    def step_two_calls(i):
        # the same step as kvq_append then kvq_decode_attn (two launches per block)
        for l in range(layers):
            st = lib.kvq_append(h, l, kp[i][l], vp[i][l], kvq.KVQ_DTYPE_BF16, 1, sp)
            if st:
                kvq.check(st)
            st = lib.kvq_decode_attn(h, l, qp[i][l], HQ7, scale_c, op[l], wp[l][0], wp[l][1], sp)
            if st:
                kvq.check(st)

    def bytes_of_step(t_before):
        """Algorithmic bytes of one step given the token count before it."""
        tot, dec = 0, 0
        for l in range(layers):
            bits = fbit[l]
            a = append_bytes(B7, HKV7, 1, bits)
            d = decode_bytes(B7, HKV7, HQ7, t_before + 1, bits)
            tot += a + d
            dec += d
        return tot, dec

    for i in range(W):
        step(i)
    torch.cuda.synchronize(dev)
    for l in range(layers):
        st = cache.query(l)
        assert st["bits"] == fbit[l], (l, st)
    t0_tokens = cache.query(0)["tokens"]

    # ---- timed region (device-only inputs) ----
    # No events between launches here: an event record between two kernels
    # would break the programmatic dependent launch of append -> decode.
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        torch.cuda.nvtx.range_push("timed")
        e_start.record(stream)
        for i in range(K):
            step(W + i)
        e_end.record(stream)
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_pop()
    cache.device_status()
    total_ms = e_start.elapsed_time(e_end)
    tot_bytes = 0
    for i in range(K):
        tot_bytes += bytes_of_step(t0_tokens + i)[0]
    total_ms = max_over_ranks(total_ms, world, dev)
    value = whole_job_gbs(tot_bytes, total_ms, world)
    launches = K * layers  # one kvq_append_decode launch per block (no shrink in the timed steps)

    # ---- per-launch decode durations: the same step again, K more times,
    # with CUDA events on the launch stream around every decode launch ----
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(layers)] for _ in range(K)]
    torch.cuda.synchronize(dev)
    r_start, r_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r_start.record(stream)
    for i in range(K):
        step(W + K + i, evs[i])
    r_end.record(stream)
    torch.cuda.synchronize(dev)
    cache.device_status()
    dec_ms = sum(evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(K) for l in range(layers))
    dec_ms_bits = {}
    for i in range(K):
        for l in range(layers):
            dec_ms_bits.setdefault(fbit[l], []).append(evs[i][l][0].elapsed_time(evs[i][l][1]))
    ev_step_ms = r_start.elapsed_time(r_end) / K

    # ---- the same steps as two calls per block (append, then attention) ----
    t2_tokens = cache.query(0)["tokens"]
    torch.cuda.synchronize(dev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for i in range(K):
        step_two_calls(W + 2 * K + i)
    c1.record(stream)
    torch.cuda.synchronize(dev)
    cache.device_status()
    two_ms = c0.elapsed_time(c1) / K
    two_bytes = sum(bytes_of_step(t2_tokens + i)[0] for i in range(K)) / K
    two_calls = {"ms_per_step": round(two_ms, 4), "gbs": round(two_bytes / two_ms / 1e6, 1),
                 "what": "the step as kvq_append + kvq_decode_attn per block (two launches)"}

    # ---- the decode half of the step captured in one CUDA graph ----
    graph = None
    if not args.no_shrink:
        gs = torch.cuda.Stream(dev)
        gsp = C.c_void_p(gs.cuda_stream)
        qg = qin[W + 2 * K - 1]
        gargs = [(h, l, C.c_void_p(qg[l].data_ptr()), HQ7, scale_c, op[l], wp[l][0], wp[l][1], gsp)
                 for l in range(layers)]
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            for l in range(layers):  # warm the side stream
                kvq.check(lib.kvq_decode_attn(*gargs[l]))
        gs.synchronize()
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=gs):
            for l in range(layers):
                lib.kvq_decode_attn(*gargs[l])
        torch.cuda.synchronize(dev)
        nrep = max(K, 20)
        for _ in range(3):
            cg.replay()
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(nrep):
            cg.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        graph_ms = g0.elapsed_time(g1) / nrep
        # the same launches without the graph
        n0, n1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        plain = [(h, l, C.c_void_p(qg[l].data_ptr()), HQ7, scale_c, op[l], wp[l][0], wp[l][1], sp)
                 for l in range(layers)]
        n0.record(stream)
        for _ in range(nrep):
            for l in range(layers):
                lib.kvq_decode_attn(*plain[l])
        n1.record(stream)
        torch.cuda.synchronize(dev)
        plain_ms = n0.elapsed_time(n1) / nrep
        cache.device_status()
        dbytes = sum(decode_bytes(B7, HKV7, HQ7, cache.query(l)["tokens"], fbit[l]) for l in range(layers))
        graph = {"ms_per_step": round(graph_ms, 4), "gbs": round(dbytes / graph_ms / 1e6, 1),
                 "ms_per_step_no_graph": round(plain_ms, 4), "gbs_no_graph": round(dbytes / plain_ms / 1e6, 1),
                 "what": f"the {layers} decode launches of one step in one CUDA graph, {nrep} replays "
                         "(appends cannot be replayed: the host scheduler state moves with every token)"}
        del cg

    # ---- e2e: the same step through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        kh = kin.cpu().pin_memory()
        vh = vin.cpu().pin_memory()
        qh = qin.cpu().pin_memory()
        oh = torch.empty((layers, B7, HQ7, HEAD_DIM), dtype=torch.float32).pin_memory()
        E = min(K, ROOM - 3 * K - W)
        if E > 0:
            torch.cuda.synchronize(dev)
            if world > 1:
                torch.distributed.barrier()
            e2e_ms = serve_steps(cache, kh[:E], vh[:E], qh[:E], oh, sm_scale, dev, stream)
            e2e_ms = max_over_ranks(e2e_ms, world, dev)
            eb = 0
            t1 = cache.query(0)["tokens"] - E
            for i in range(E):
                eb += bytes_of_step(t1 + i)[0]
            e2e = {"value": whole_job_gbs(eb, e2e_ms, world), "unit": "GB/s",
                   "h2d_bytes_per_step": layers * (kin[0, 0].numel() * 2 * 2 + qin[0, 0].numel() * 2),
                   "d2h_bytes_per_step": layers * out[0].numel() * 4, "steps": E}

    # ---- roofline of the decode kernel ----
    # Every launch of the timed region is this kernel (kvq_append_decode: one
    # launch per block, no shrink in the timed steps), so its average launch
    # duration over the timed region is the region's time over its launches.
    # The event pass above brackets each launch instead; its events break the
    # dependent-launch overlap of consecutive launches, so it is reported as a
    # breakdown by width, not as the kernel's duration.
    peak, peak_kind = peaks()
    n_dec = K * layers
    avg_ms = total_ms / n_dec
    bytes_per_launch = tot_bytes / n_dec
    achieved = bytes_per_launch / (avg_ms / 1e3) / 1e9
    traffic, traffic_src = decode_traffic(fbit)
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs (copy)",
            "traffic": traffic, "traffic_source": traffic_src,
            "kernel": "decode_kernel (kvq_append_decode: the step's new token and the attention)",
            "avg_launch_us": round(avg_ms * 1e3, 2),
            "bytes_per_launch": int(bytes_per_launch),
            "timing": f"CUDA events around the timed region, whose {n_dec} launches are all this kernel "
                      "(slowest rank): region time / launches",
            "per_launch_events": {
                "avg_launch_us": round(dec_ms * 1e3 / n_dec, 2),
                "per_bits_us": {f"{b}bit": round(statistics.mean(v) * 1e3, 2) for b, v in sorted(dec_ms_bits.items())},
                "what": f"CUDA events around each of {n_dec} launches in {K} more steps ({ev_step_ms:.4f} ms/step "
                        "with the events, which serialise the launches)"}}

    extra = {}
    if not args.no_shrink and rank == 0:
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        cache.free()
        del cache, kin, vin, qin
        torch.cuda.empty_cache()
        extra["shrink"] = measure_shrink(kvq, dev, flush)
        extra["shrink"]["unit"] = "GB/s"
        extra["append_chunk"] = measure_append_chunk(kvq, dev, flush)
        extra["append_token"] = measure_append_token(kvq, dev)
        extra["append_token_sink_window"] = measure_append_token(kvq, dev, sink_window=True)
        extra["decode_configs"] = measure_decode_configs(kvq, dev)
        extra["block_append_key_channel"] = measure_block_append_key_channel(kvq, dev)
        extra["decode_graph"] = graph
    if not args.no_70b and rank == 0:
        if not args.no_shrink:
            del flush
        else:
            cache.free()
            del cache, kin, vin, qin
        torch.cuda.empty_cache()
        k70 = min(K, 100)
        extra["llama70b_step"] = measure_step_70b(kvq, dev, k70, 3, 0 if args.no_e2e else min(k70, 20),
                                                  cpu=world == 1 and not args.no_cpu)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(total_ms / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": layers, "batch": B7, "q_heads": HQ7, "kv_heads": HKV7,
                   "head_dim": HEAD_DIM, "context": T7, "fbit": fbit, "parallelism": f"replicas x{world}",
                   "l2": "no flush: every block's cache read (151-285 MB) exceeds the 126 MB L2",
                   "decode_ms_share": round(dec_ms / (ev_step_ms * K), 3),
                   "headline": "the 7B-shape decode step, the model-shaped workload the metric is quoted on; the "
                               "largest one-GPU workload (Llama-70B shape, 128K context) is measured the same way "
                               "as the llama70b_step entry"},
        "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clk.summary(),
        "two_call_step": two_calls,
        **extra,
    }
    return res


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(tokens, fbit=2, g=HQ7 // HKV7, seed=SEED, n_out=None):
    """One (sequence, KV head) stream of a model-shaped block, replayed
    through the oracle's progressive cache; returns (layer, q, lam)."""
    from oracle import oracle as orc

    if n_out is None:
        n_out = S.outliers_for(HKV7)
    # a block sized for exactly `tokens` (a multiple of 512) ends full at its Fbit
    tokens = (tokens + 511) // 512 * 512
    L = orc.Layer(1, 1, tokens, fbit)
    lam = None
    pos = 0
    while pos < tokens:
        n = min(4096, tokens - pos)
        k, v = S.keys_values(seed, 1, 1, n, 1, pos, n_out, dtype=torch.bfloat16)
        if lam is None:
            lam = calib_lambda(k).numpy().reshape(1, HEAD_DIM).astype(np.float32)
        assert L.append(k.float().numpy(), v.float().numpy(), lam) == 0
        pos += n
    q = S.queries(seed, 1, 0, 1, g, tokens, dtype=torch.bfloat16).float().numpy()
    return L, q, lam


def host_cores(cap=64, cpu_max="/sys/fs/cgroup/cpu.max"):
    """CPUs this process may run on: its affinity set, capped by a cgroup v2
    CPU quota when one is set ("quota period" in `cpu_max`, "max" for none),
    and at `cap` (one oracle stream, ~17 MB, per thread)."""
    n = min(cap, len(os.sched_getaffinity(0)))
    try:
        with open(cpu_max) as f:
            quota, period = f.read().split()[:2]
        if quota != "max":
            n = min(n, max(1, math.ceil(int(quota) / int(period))))
    except (OSError, ValueError):
        pass
    return n


def oracle_threads(threads, tokens, warmup, run, g=HQ7 // HKV7, n_out=None):
    """Run the oracle's fp64 attention on `threads` threads at once, each over
    its own stream sample (the oracle's C code runs without the Python lock
    and keeps no global state).  After `warmup` calls per thread and a
    barrier, run(call) times the thread's measured calls and returns
    (calls, seconds).  Returns (total calls, slowest thread's seconds)."""
    import concurrent.futures as cf

    barrier = threading.Barrier(threads)

    def one(i):
        L, q, lam = oracle_sample(tokens, g=g, seed=SEED + i, n_out=n_out)
        assert L.bits == 2, "the sample block ends full at its Fbit of 2"
        call = lambda: L.attention(q, lam, HEAD_DIM ** -0.5)  # noqa: E731
        for _ in range(warmup):
            call()
        barrier.wait()
        return run(call)

    with cf.ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(one, range(threads)))
    return sum(r[0] for r in res), max(r[1] for r in res)


def cpu_baseline(budget_s=15.0, single_s=5.0, tokens=T7, g=HQ7 // HKV7, n_out=None, max_threads=64):
    """The oracle's fp64 attention over sampled (sequence, KV head) streams of
    a 2-bit block at the full context (7B shape by default): on one thread,
    then on every host core at once (one stream per thread)."""
    cores = min(host_cores(), max_threads)

    def timed(budget):
        def run(call):
            t0 = time.perf_counter()
            n = 0
            while True:
                call()
                n += 1
                if time.perf_counter() - t0 > budget:
                    return n, time.perf_counter() - t0
        return run

    nb = decode_bytes(1, 1, g, tokens, 2)
    n1, dt1 = oracle_threads(1, tokens, 0, timed(single_s), g=g, n_out=n_out)
    n, dt = oracle_threads(cores, tokens, 0, timed(budget_s), g=g, n_out=n_out)
    return {"value": round(n * nb / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} x one (sequence, KV head) stream of a 2-bit block, {tokens} tokens, "
                      f"{g} query heads, fp64 attention, {cores} threads each on its own stream; {dt:.1f} s",
            "single_thread": {"value": round(n1 * nb / dt1 / 1e9, 5), "unit": "GB/s", "cores": 1,
                              "sample": f"{n1} x the same stream on one thread; {dt1:.1f} s"}}


def run_reference(args, world=1):
    K, W = args.steps, args.warmup
    tokens = T7  # the GPU arm's context; a step is one call per thread
    cores = host_cores()

    def run(call):
        t0 = time.perf_counter()
        for _ in range(K):
            call()
        return K, time.perf_counter() - t0

    n, dt = oracle_threads(cores, tokens, W, run)
    nb = decode_bytes(1, 1, HQ7 // HKV7, tokens, 2)
    v = n * nb / dt / 1e9
    sample = (f"each step: {cores} (sequence, KV head) streams of a 2-bit 7B-shape block at once, one per "
              f"thread, {tokens} tokens, {HQ7 // HKV7} query heads, fp64 attention in the CPU oracle")
    return {"impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(dt * 1e3 / K, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "layers": L7, "batch": B7, "q_heads": HQ7, "kv_heads": HKV7,
                       "head_dim": HEAD_DIM, "context": T7, "fbit": FBIT7, "parallelism": f"replicas x{world}",
                       "reference": "the CPU oracle on rank 0 only (the other ranks exit without work)"},
            "cpu_baseline": {"value": round(v, 5), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_part(args):
    """One measurement alone on cuda:0 (for profiling): the shrink events, or
    the Llama-70B step (args.steps timed steps, no end-to-end pass)."""
    from mixed_precision_kv_kvq_b200 import build as kbuild

    kbuild.build()
    import mixed_precision_kv_kvq_b200 as kvq

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.part == "append":
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        return {"part": "append", **measure_append_chunk(kvq, dev, flush)}
    if args.part == "shrink":
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        n = args.shrink_blocks
        return {"part": "shrink", **measure_shrink(kvq, dev, flush, blocks_7b=n or 20, blocks_70b=n or 3)}
    return {"part": "step70b",
            **measure_step_70b(kvq, dev, args.steps, args.warmup, 0 if args.no_e2e else min(args.steps, 20),
                               cpu=not args.no_cpu)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--layers", type=int, default=L7, help="blocks of the 7B shape to run (profiling cases)")
    ap.add_argument("--no-shrink", action="store_true", help="skip the separate shrink/append measurements")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--no-70b", action="store_true", help="skip the Llama-70B decode step")
    ap.add_argument("--part", choices=["all", "shrink", "append", "step70b"], default="all",
                    help="run one measurement alone (profiling cases): the shrink events, the chunked append or "
                         "the 70B step")
    ap.add_argument("--shrink-blocks", type=int, default=0,
                    help="with --part shrink: blocks per event (0: 20 for the 7B events, 3 for the 70B ones)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "kvq":
        print("note: warm-up raised to 3", file=sys.stderr)
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if args.part != "all":
        if rank == 0:
            print(json.dumps(run_part(args)), flush=True)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_gpu(args, rank, world)
        if rank == 0:
            if world == 1 and not args.no_cpu:
                res["cpu_baseline"] = cpu_baseline()
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
