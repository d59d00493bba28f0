/*
 * kvq.h -- C ABI of libkvq, a B200 (sm_100a) implementation of the online hot
 * path of PM-KVQ's progressive mixed-precision KV cache.
 *
 * Method source: "PM-KVQ: Progressive Mixed-Precision KV Cache Quantization
 * for Long-CoT LLMs" (papernotes.org note on the ICLR 2026 paper):
 *   - key design 1, progressive quantization: every transformer block keeps
 *     its KV cache at 16 bits until the block's memory budget is full, then
 *     shrinks the whole block one level 16 -> 8 -> 4 -> 2 with the Equivalent
 *     Right Shift  X_b = ((2^{2b} - 2^b + 1)(X_{2b} + 2^{b-1})) >> 3b,
 *     Z_b = Z_{2b}, S_b = (2^b + 1) S_{2b}, stopping at the block's Fbit;
 *   - key design 2: each block has its own Fbit (chosen offline; an input);
 *   - key design 3: Key outliers move to the Query per channel (K / lambda,
 *     Q * lambda; lambda is calibrated offline and is an input here);
 *   - training strategy: asymmetric quantization with groups of 128.
 *
 * Conventions for every call:
 *   - head_dim is 128; one quantization group is one token's 128 channels of
 *     one KV head.  Codes are unsigned; x^ = Z + q * R / (2^b - 1) with R and
 *     Z binary16 per group.
 *   - "device" pointers are CUDA global-memory addresses on the device that
 *     was current when the cache was created; "host" pointers are ordinary
 *     CPU memory.  The caller owns every buffer it passes (inputs, outputs,
 *     workspace, the optional pool).  The library owns the cache's host state
 *     and, when it allocated it, the device pool.
 *   - stream: a cudaStream_t (NULL = legacy default stream).  Calls that take
 *     a stream enqueue work on it and return without waiting, unless stated.
 *   - A call that returns an error other than KVQ_ERR_CUDA has changed
 *     nothing.  kvq_last_error() describes the last failure on the calling
 *     thread.
 *   - Calls on one cache are not thread-safe; serialise them.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kvq_cache kvq_cache; /* opaque, host-owned */
typedef struct CUstream_st* kvq_stream_t; /* same type as cudaStream_t */

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID = 1,   /* bad argument (null pointer, range, shape) */
  KVQ_ERR_BUDGET = 2,    /* the block is full at its Fbit: the tokens do not fit */
  KVQ_ERR_STATE = 3,     /* the call is not allowed in the block's current state */
  KVQ_ERR_OOM = 4,       /* device allocation failed */
  KVQ_ERR_CUDA = 5,      /* a CUDA call or kernel launch failed */
  KVQ_ERR_WORKSPACE = 6, /* workspace missing or smaller than kvq_decode_workspace() */
  KVQ_ERR_TIMEOUT = 7    /* a kernel gave up waiting on one of its own copies */
} kvq_status;

enum { KVQ_DTYPE_BF16 = 0, KVQ_DTYPE_F32 = 1 };

/* Size in bytes of the device pool a cache with these parameters needs, or 0
 * if the parameters are invalid.  Pure host computation.
 *
 * Budget split (key designs 1 and 2): every block can hold the same number of
 * tokens N at its own Fbit, the largest multiple of 512 with
 *   batch * kv_heads * 2 * N * sum_l (16 * fbit[l] + 4)  <=  budget_bytes
 * (16*F bytes of codes and 4 bytes of binary16 (R, Z) per token, head and
 * K-or-V).  The pool is exactly that many bytes plus a few KiB of per-layer
 * lambda tables and counters. */
size_t kvq_pool_bytes(int layers, int batch, int kv_heads, int head_dim, size_t budget_bytes,
                      const int* fbit /* host [layers], each 2, 4, 8 or 16 */);

/* Options of kvq_pool_bytes_ex / kvq_alloc_ex.
 *   KVQ_OPT_SINK_WINDOW  the deployed configuration of the pages (training
 *     strategy, the KIVI trick the note keeps): every block holds token 0
 *     (the sink) and its latest 128 tokens at 16 bits; a token that leaves
 *     the window moves into the block's progressive cache at that cache's
 *     current width by the block's shift applied 16 -> 8 -> ... -> b (R and Z
 *     kept; R rescaled under KVQ_SHIFT_DIRECT) -- the codes it would have had
 *     had it been stored at 16 bits and shrunk with the block.  The budget
 *     rule (N tokens per block) applies to the progressive cache; the window
 *     adds 5 tiles of 16 KiB plus 1,280 bytes of meta per (sequence, KV head)
 *     and block to the pool, outside the budget.  With the option: kvq_query
 *     reports every token (tokens), the progressive cache's width (bits) and
 *     capacity + 129; kvq_max_tokens is N + 129; kvq_export returns the
 *     progressive cache (tokens 1 .. n-129) and kvq_export_window the sink
 *     and the window; kvq_shrink needs the progressive cache full;
 *     attention covers all three. */
/*   KVQ_OPT_KEY_CHANNEL  Key groups along the tokens (KIVI's per-channel Key,
 *     per-token Value split, which the pages' comparison with KIVI names; the
 *     pages' "group size 128" names no axis): a Key group is one channel of one
 *     KV head over a block of 128 consecutive tokens.  The block being filled
 *     (the latest n mod 128 tokens) is staged at 16 bits, each token quantized
 *     per token as the pages store recent tokens at INT16.  When a block's
 *     128th token arrives the block enters the progressive cache at its
 *     current width: every staged Key is read back in fp32 as
 *     Z + code * (R / 65535) (one division, one multiply, one add, each
 *     round-to-nearest) and each channel's 128 values are quantized directly
 *     at that width with the quantizer of this file; every staged Value moves
 *     by the block's shift chain 16 -> ... -> b (R and Z kept; R rescaled
 *     under KVQ_SHIFT_DIRECT).  A shrink treats the per-channel Key ranges as
 *     the per-token ones.  N is a multiple of 1024 (so the progressive cache
 *     takes whole blocks at every width); the staging adds 5 tiles of 16 KiB
 *     plus 1,280 bytes of meta per (sequence, KV head) and block to the pool,
 *     outside the budget, and the per-channel Key meta takes the place of the
 *     per-token Key meta in the budget.  With the option: kvq_query reports
 *     every token (tokens) and capacity + 127; kvq_max_tokens is N + 127;
 *     kvq_export returns the progressive cache (tokens 0 .. n - (n mod 128) - 1)
 *     with k_meta[2 (128 k + c) + {0, 1}] = (R, Z) of Key channel c of block
 *     k; kvq_export_window returns the staged tokens; kvq_shrink needs the
 *     progressive cache full; kvq_append_decode runs the two calls.  Not
 *     combinable with KVQ_OPT_SINK_WINDOW. */
enum { KVQ_OPT_SINK_WINDOW = 1, KVQ_OPT_KEY_CHANNEL = 2 };
size_t kvq_pool_bytes_ex(int layers, int batch, int kv_heads, int head_dim, size_t budget_bytes,
                         const int* fbit, int options);

/* Create a cache.  fbit: host [layers].  dev_pool: a device buffer of at least
 * kvq_pool_bytes(...) bytes, owned by the caller and kept alive until
 * kvq_free; or NULL, and the library cudaMallocs the pool itself.  With a
 * caller pool this call makes no CUDA call.  Every block starts empty at 16
 * bits.  Errors: INVALID (shape -- batch <= 65535 and kv_heads <= 4096 --,
 * fbit, head_dim != 128), BUDGET (budget smaller than 512 tokens), OOM. */
kvq_status kvq_alloc(kvq_cache** out, int layers, int batch, int kv_heads, int head_dim,
                     size_t budget_bytes, const int* fbit, void* dev_pool, size_t pool_bytes);

/* kvq_alloc with options (KVQ_OPT_*; 0 = kvq_alloc).  dev_pool, when given,
 * must hold kvq_pool_bytes_ex(..., options) bytes.  Errors as kvq_alloc;
 * INVALID for unknown option bits. */
kvq_status kvq_alloc_ex(kvq_cache** out, int layers, int batch, int kv_heads, int head_dim,
                        size_t budget_bytes, const int* fbit, void* dev_pool, size_t pool_bytes, int options);

/* Per-channel migration factor of one block (key design 3).  lambda_host:
 * host float [kv_heads][128], every value finite and > 0.  Stored Keys become
 * fp32(k * fp32(1/lambda)) and queries are multiplied by lambda inside the
 * attention kernel.  Until it is called a block uses lambda = 1.  Copies
 * synchronously; must not be called while kernels on this block are in
 * flight. */
kvq_status kvq_set_lambda(kvq_cache* c, int layer, const float* lambda_host);

/* Quantize-on-append (key design 1): append n_tokens tokens to every
 * sequence of the batch.  k, v: device [batch][n_tokens][kv_heads][128],
 * dtype KVQ_DTYPE_BF16 or KVQ_DTYPE_F32, 16-byte aligned, every value
 * finite (the codes of a non-finite value are unspecified).  A group's
 * minimum and range must fit binary16 (magnitudes up to 65,504): beyond that
 * Z or R overflows to infinity, and the group's codes and attention over it
 * are unspecified (not checked, as on the oracle).  Each token is
 * quantized at the block's current width; when the block is full the block
 * is first shrunk one level (never below its Fbit).  n tokens behave exactly
 * like n single-token appends.  Errors: BUDGET when the block cannot hold
 * them at its Fbit (nothing is written), INVALID, CUDA. */
kvq_status kvq_append(kvq_cache* c, int layer, const void* k, const void* v, int dtype,
                      int n_tokens, kvq_stream_t stream);

/* Shrink a full block one level now (the step its next append would take):
 * every stored code goes through the Equivalent Right Shift, in place.  Meta
 * is not touched: with R = (2^b - 1) S, S_b = (2^b + 1) S_{2b} leaves R
 * unchanged.  Errors: STATE if the block is not full at its current width or
 * is already at its Fbit. */
kvq_status kvq_shrink(kvq_cache* c, int layer, kvq_stream_t stream);

/* Shift a block uses when it shrinks (before its first shrink; the default
 * is the Equivalent Right Shift):
 *   KVQ_SHIFT_EQUIVALENT  key design 1: X_b = ((2^2b - 2^b + 1)(X_2b + 2^(b-1)))
 *                         >> 3b, Z_b = Z_2b, S_b = (2^b + 1) S_2b (meta untouched);
 *   KVQ_SHIFT_DIRECT      the "Direct Right Shift" row of the note's ablation:
 *                         keep the high b bits, X_b = X_2b >> b, Z_b = Z_2b and
 *                         the truncation's scale S_b = 2^b S_2b, i.e. every
 *                         stored range becomes binary16_RN(fp32(R 2^b) / (2^b + 1))
 *                         (the shrink also rewrites the block's meta).
 * The ablation's "Modified Right Shift" has no definition on the pages and is
 * not offered.  Errors: INVALID (mode), STATE (the block has already shrunk
 * with the other shift). */
enum { KVQ_SHIFT_EQUIVALENT = 0, KVQ_SHIFT_DIRECT = 1 };
kvq_status kvq_set_shift_mode(kvq_cache* c, int layer, int mode);

/* Bytes of device workspace kvq_decode_attn needs for this block and number
 * of query heads (any token count).  0 on invalid arguments. */
size_t kvq_decode_workspace(const kvq_cache* c, int layer, int q_heads);

/* GQA decode attention over the block's quantized cache:
 *   out[b][h] = sum_t softmax_t(sm_scale * (q[b][h] * lambda) . k^_t) v^_t
 * over every cached token, query head h reading KV head h / (q_heads /
 * kv_heads).  q: device bf16 [batch][q_heads][128], 16-byte aligned; out:
 * device fp32 [batch][q_heads][128]; workspace: device buffer of at least
 * kvq_decode_workspace(c, layer, q_heads) bytes (contents need no
 * initialisation; the call owns it until it completes on the stream).
 * q_heads must be a multiple of kv_heads with at most 8 query heads per KV
 * head.  Errors: STATE if the block is empty, WORKSPACE, INVALID, CUDA. */
kvq_status kvq_decode_attn(kvq_cache* c, int layer, const void* q, int q_heads, float sm_scale,
                           float* out, void* workspace, size_t ws_bytes, kvq_stream_t stream);

/* One decode step of a block in one launch: kvq_append of one token per
 * sequence (k, v: device [batch][1][kv_heads][128], dtype as kvq_append,
 * 16-byte aligned) followed by kvq_decode_attn over every token including it
 * (q, q_heads, sm_scale, out, workspace as kvq_decode_attn) -- the same codes,
 * meta and output as the two calls.  The token is quantized and written by
 * the attention kernel itself (by the warp whose share of the block holds the
 * token's group, before it reads that group), which saves the append launch
 * on the decode path.  A full block is first shrunk one level as kvq_append
 * would (a separate launch).  With KVQ_OPT_SINK_WINDOW the call runs the two
 * calls.  Errors: those of kvq_append (BUDGET, INVALID) and of
 * kvq_decode_attn (WORKSPACE, INVALID, CUDA); on an error before a launch
 * nothing has changed. */
kvq_status kvq_append_decode(kvq_cache* c, int layer, const void* k, const void* v, int dtype, const void* q,
                             int q_heads, float sm_scale, float* out, void* workspace, size_t ws_bytes,
                             kvq_stream_t stream);

/* Decode attention that allocates nothing and takes no workspace; same
 * arguments, result and errors as kvq_decode_attn otherwise.  The paper has
 * no counterpart to this call: it exists for callers that cannot allocate device
 * memory where they run decode (an allocator owned by a host framework, a
 * serving loop that must not allocate after start-up, a host that only hands
 * out inputs and outputs).  When a stream of the block is cut into several
 * slices, their partials go to a 24 MiB buffer that is part of the library:
 * every GPU that loads the library holds it until the process exits.  A
 * block whose batch * kv_heads streams need more than that is rejected with
 * KVQ_ERR_WORKSPACE (use kvq_decode_attn); a block whose streams take one
 * slice each needs no scratch at all.  Each call looks up the buffer's
 * device address on the current device (a CUDA runtime query, no
 * allocation); the first call on a device may also load the library's
 * device code there, so make that first call before any stream capture.
 * All calls on one device share the buffer, so calls that can overlap on
 * the GPU (different streams, or different caches) race: serialise them. */
kvq_status kvq_decode_attn_noalloc(kvq_cache* c, int layer, const void* q, int q_heads, float sm_scale,
                                   float* out, kvq_stream_t stream);

/* Host-side state of one block.  Any output pointer may be NULL.
 * capacity: tokens that fit at the current width. */
kvq_status kvq_query(const kvq_cache* c, int layer, int* tokens, int* bits, int* capacity,
                     int* n_shrinks);

/* Tokens every block can hold at its Fbit (N in kvq_pool_bytes). */
int kvq_max_tokens(const kvq_cache* c);

/* Copy one (sequence b, KV head j) stream of a block to host memory in
 * logical token order (the order tokens were appended):
 *   k_codes, v_codes: host uint16 [tokens][128] (codes at the current width)
 *   k_meta,  v_meta : host uint16 [tokens][2]   (binary16 bits of R, Z)
 * Any of the four may be NULL.  Synchronous: waits for the stream. */
kvq_status kvq_export(const kvq_cache* c, int layer, int b, int j, uint16_t* k_codes,
                      uint16_t* v_codes, uint16_t* k_meta, uint16_t* v_meta,
                      kvq_stream_t stream);

/* The sink and window tokens of one stream (caches made with
 * KVQ_OPT_SINK_WINDOW), oldest first: token 0, then the latest min(n - 1,
 * 128) tokens, at 16 bits:
 *   k_codes, v_codes: host uint16 [129][128]; k_meta, v_meta: host uint16 [129][2]
 * (buffers for 129 tokens; the first *n_tokens rows are written).  With
 * KVQ_OPT_KEY_CHANNEL: the staged tokens of the block being filled (n mod
 * 128 of them), oldest first, in the same buffers.  Any of the four may be
 * NULL.  Synchronous.  Errors: INVALID (neither option, stream). */
kvq_status kvq_export_window(const kvq_cache* c, int layer, int b, int j, uint16_t* k_codes,
                             uint16_t* v_codes, uint16_t* k_meta, uint16_t* v_meta, int* n_tokens,
                             kvq_stream_t stream);

/* Wait for the stream and report whether a kernel of this cache gave up on a
 * bounded wait (KVQ_ERR_TIMEOUT) since the last check; clears the flag. */
kvq_status kvq_device_status(kvq_cache* c, kvq_stream_t stream);

/* Self-test of that path: enqueues a one-warp kernel whose bulk-copy barrier
 * waits for bytes no copy will bring, with the attention kernel's bounded
 * wait; after its time limit (2 s) the wait gives up, raises the cache's
 * error flag and the kernel returns normally (nothing faults, no copy is in
 * flight).  The next kvq_device_status then reports KVQ_ERR_TIMEOUT and the
 * cache stays usable.  Asynchronous.  Errors: INVALID, CUDA. */
kvq_status kvq_selftest_timeout(kvq_cache* c, kvq_stream_t stream);

/* Block-wise bit allocation (key design 2): choose one width per block from
 * the candidate widths bits[0..n_opts) (each 2, 4, 8 or 16, distinct;
 * n_opts <= 4) minimising  sum_i sens[i][o_i]  subject to the cache's budget
 * rule for max_tokens tokens in every block:
 *   batch * kv_heads * 2 * max_tokens * sum_i (16 * bits[o_i] + 4) <= budget_bytes.
 * sens: host double [layers][n_opts], the sensitivity s_{i,b} of block i at
 * width bits[o] (computed offline from gradients; an input here).  The
 * solution is exact (dynamic programming over the budget in units of
 * batch * kv_heads * 2 * max_tokens * 4 bytes); among assignments of equal
 * objective the first found (blocks in order, options in the given order)
 * is returned.  fbit_out: host int [layers], ready for kvq_pool_bytes /
 * kvq_alloc; objective_out (may be NULL): the minimal sum.  Pure host
 * computation.  Errors: INVALID (arguments), BUDGET (no assignment fits). */
kvq_status kvq_allocate_bits(int layers, int n_opts, const int* bits, const double* sens, int batch,
                             int kv_heads, int head_dim, long long max_tokens, size_t budget_bytes,
                             int* fbit_out, double* objective_out);

/* Message of the last failed call on this thread ("" if none). */
const char* kvq_last_error(void);

/* Release the cache (and the pool if the library allocated it).  Waits for
 * the device.  NULL is ignored. */
void kvq_free(kvq_cache* c);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
