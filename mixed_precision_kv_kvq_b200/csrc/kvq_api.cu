// kvq_api.cu -- the C ABI of libkvq (include/kvq.h): cache allocation, the
// budget-triggered shrink scheduler, the slot map, export and error state.
//
// Scheduler (PM-KVQ note, key design 1): a block starts at 16 bits; a token
// that arrives while the block holds cap(b) = N * Fbit / b tokens first
// shrinks the whole block one level (16 -> 8 -> 4 -> 2, never below Fbit).
// The host keeps every counter, so deciding to shrink never reads device
// memory and nothing synchronises.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/kvq.h"
#include "kvq_internal.cuh"

using namespace kvq;

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
kvq_status fail(kvq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}
kvq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// NVTX range around one entry point (a profiler's timeline shows the calls
// around their kernels; with no tool attached a push and a pop cost a few ns).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

// Host-side fault injection: with KVQ_FAULT_ALLOC set to anything but "" or
// "0", the library's own device allocation reports failure without calling
// CUDA, so the out-of-memory path can be tested on any machine.
bool fault_alloc() {
  const char* f = getenv("KVQ_FAULT_ALLOC");
  return f && *f && strcmp(f, "0") != 0;
}

}  // namespace

namespace kvq {
// Records the message of a failed call (for the host-only entry points in
// other files).
kvq_status api_fail(kvq_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace kvq

namespace {

constexpr size_t kAlign = 256;
constexpr int kTokenRound = 512;  // tokens per tile at 2 bits: a multiple for every width
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool valid_fbit(int f) { return f == 2 || f == 4 || f == 8 || f == 16; }

struct LayerState {
  int fbit;
  int bits;
  long long n;
  int n_shrinks;
  // Tokens whose slots no library kernel still in flight can be writing when
  // a later kernel on the same stream starts early (programmatic dependent
  // launch): the append kernel triggers its dependents only after its own
  // predecessors completed, and the shrink kernel never triggers early, so
  // only the most recent append kernel of the block can still be running.
  long long n_stable;
  int shift_mode;  // KVQ_SHIFT_EQUIVALENT or KVQ_SHIFT_DIRECT
  int nt;  // tiles per stream
  int pf;  // meta slots per tile
  bool counters_zeroed;
  size_t off_lam, off_lam_inv, off_counters, off_codes, off_meta;
  // sink + window option: n counts the progressive cache; n_all every token
  bool window;
  long long n_all;
  size_t off_wcodes, off_wmeta;
  // per-channel Key groups (uses the window storage for the staged block):
  // n counts the progressive cache (whole blocks), n_all every token
  bool chan;
  size_t off_kmc;
  bool lambda_set;
};

struct Plan {
  long long n_f;
  size_t bytes;
  std::vector<LayerState> layers;
};

// Budget split: every block holds the same N tokens at its own Fbit.
bool make_plan(int layers, int batch, int kv_heads, int head_dim, size_t budget, const int* fbit, int options,
               Plan& p, kvq_status* why) {
  *why = KVQ_ERR_INVALID;
  if (layers < 1 || batch < 1 || kv_heads < 1 || head_dim != kHeadDim || !fbit) return false;
  if (batch > 65535 || kv_heads > 4096) return false;  // kernel grid limits
  if (options & ~(KVQ_OPT_SINK_WINDOW | KVQ_OPT_KEY_CHANNEL)) return false;
  const bool chan = (options & KVQ_OPT_KEY_CHANNEL) != 0;
  if (chan && (options & KVQ_OPT_SINK_WINDOW)) return false;
  const bool window = (options & KVQ_OPT_SINK_WINDOW) != 0;
  // whole 128-token blocks at every width: N * Fbit / 16 divisible by 128
  const long long round = chan ? 2 * kTokenRound : kTokenRound;
  unsigned long long per_token = 0;  // bytes per token over all blocks
  const unsigned long long streams = (unsigned long long)batch * kv_heads * 2;
  for (int l = 0; l < layers; l++) {
    if (!valid_fbit(fbit[l])) return false;
    per_token += streams * (16ull * fbit[l] + 4ull);
  }
  const unsigned long long n_raw = budget / per_token;
  const long long n_f = (long long)(n_raw / round) * round;
  if (n_f < round || n_f > (1ll << 30)) {
    *why = KVQ_ERR_BUDGET;
    return false;
  }
  p.n_f = n_f;
  p.layers.assign(layers, LayerState{});
  size_t off = kAlign;  // [0, 256): device error flag
  const size_t n_streams = (size_t)batch * kv_heads;
  for (int l = 0; l < layers; l++) {
    LayerState& L = p.layers[l];
    L.fbit = fbit[l];
    L.bits = 16;
    L.n = 0;
    L.n_shrinks = 0;
    L.n_stable = 0;
    L.shift_mode = KVQ_SHIFT_EQUIVALENT;
    L.pf = slots_per_tile(L.fbit);
    L.nt = (int)(n_f / L.pf);
    L.counters_zeroed = false;
    L.lambda_set = false;
    L.off_lam = off;
    off += align_up((size_t)kv_heads * kHeadDim * 4);
    L.off_lam_inv = off;
    off += align_up((size_t)kv_heads * kHeadDim * 4);
    L.off_counters = off;
    off += align_up(n_streams * 4);
    L.off_codes = off;
    off += align_up(n_streams * (size_t)L.nt * kTileBytes);
    L.off_meta = off;
    off += align_up(n_streams * (size_t)L.nt * L.pf * 8);
    L.window = window;
    L.chan = chan;
    L.n_all = 0;
    L.off_wcodes = L.off_wmeta = L.off_kmc = 0;
    if (chan) {  // per-channel Key meta: (R, Z) of 128 channels per block of 128 tokens
      L.off_kmc = off;
      off += align_up(n_streams * (size_t)n_f * 4);
    }
    if (window || chan) {  // window: token 0 and the latest 128 tokens at 16 bits; chan: the staged block
      L.off_wcodes = off;
      off += align_up(n_streams * (size_t)kWindowTiles * kTileBytes);
      L.off_wmeta = off;
      off += align_up(n_streams * (size_t)kWindowTiles * slots_per_tile(16) * 8);
    }
  }
  p.bytes = off;
  *why = KVQ_OK;
  return true;
}

long long capacity(const LayerState& L, long long n_f, int bits) { return n_f * L.fbit / bits; }

}  // namespace

struct kvq_cache {
  int layers, batch, kv_heads;
  long long n_f;
  uint8_t* pool;
  size_t pool_bytes;
  bool owns_pool;
  int num_sms;
  bool err_zeroed;
  std::vector<LayerState> L;

  // The error flag lives in the pool; clear it once, stream-ordered, before
  // the first kernel of this cache can set it.
  cudaError_t ensure_err(cudaStream_t s) {
    if (err_zeroed) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(pool, 0, 4, s);
    if (e == cudaSuccess) err_zeroed = true;
    return e;
  }

  int sms() {
    if (num_sms <= 0) {
      int dev = 0, n = 0;
      if (cudaGetDevice(&dev) == cudaSuccess &&
          cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) {
        num_sms = n;
      } else {
        cudaGetLastError();
        num_sms = 148;  // B200
      }
    }
    return num_sms;
  }
  uint8_t* codes(int l) { return pool + L[l].off_codes; }
  uint32_t* meta(int l) { return reinterpret_cast<uint32_t*>(pool + L[l].off_meta); }
  uint8_t* wcodes(int l) { return pool + L[l].off_wcodes; }
  uint32_t* wmeta(int l) { return reinterpret_cast<uint32_t*>(pool + L[l].off_wmeta); }
  uint32_t* kmc(int l) { return reinterpret_cast<uint32_t*>(pool + L[l].off_kmc); }
  int blocks_max() const { return (int)(n_f / kKeyBlock); }
  float* lam(int l) { return reinterpret_cast<float*>(pool + L[l].off_lam); }
  float* lam_inv(int l) { return reinterpret_cast<float*>(pool + L[l].off_lam_inv); }
  int* counters(int l) { return reinterpret_cast<int*>(pool + L[l].off_counters); }
  int* err() { return reinterpret_cast<int*>(pool); }
};

namespace {

kvq_status check_layer(const kvq_cache* c, int layer) {
  if (!c) return fail(KVQ_ERR_INVALID, "cache is NULL");
  if (layer < 0 || layer >= c->layers) return fail(KVQ_ERR_INVALID, "layer %d out of range [0, %d)", layer, c->layers);
  return KVQ_OK;
}

// Slot of logical token i: the epoch it was appended in fixes its tile/slot.
void slot_of(const LayerState& L, long long i, int* tile, int* slot) {
  int e = 0;
  int bits = 16;
  while (e < L.n_shrinks) {
    const long long end = (long long)L.nt * slots_per_tile(bits);  // cap at this width
    if (i < end) break;
    bits >>= 1;
    e++;
  }
  const int p = slots_per_tile(bits);
  const int h = e > 0 ? p / 2 : 0;
  const int ee = p - h;
  const long long m = i - (long long)L.nt * h;
  *tile = (int)(m / ee);
  *slot = h + (int)(m % ee);
}

// Shrink of block `layer` from its current width to half of it.
ShrinkArgs shrink_args(kvq_cache* c, int layer) {
  const LayerState& L = c->L[layer];
  ShrinkArgs sa{};
  sa.codes = c->codes(layer);
  sa.n_tiles = (long long)c->batch * c->kv_heads * L.nt;
  sa.bits_to = L.bits / 2;
  sa.direct = L.shift_mode == KVQ_SHIFT_DIRECT;
  sa.meta = c->meta(layer);
  sa.pf = L.pf;
  sa.p_from = slots_per_tile(L.bits);
  if (L.chan) {
    sa.kmc = c->kmc(layer);
    sa.kmc_words = (long long)c->batch * c->kv_heads * c->blocks_max() * kHeadDim;
  }
  return sa;
}

// Groups (in the kernels' group order, see locate_group) of every stream
// that hold only slots of tokens before n_stable.
long long stable_groups(const LayerState& L, const Fill& f) {
  if (L.n_stable >= L.n) return f.gps;
  int tile, slot;
  slot_of(L, L.n_stable, &tile, &slot);
  return (long long)tile * f.gpt + slot / kGroupTokens;
}

// The decode launches of one call: the progressive cache (if it holds
// tokens) and, with the sink + window option, the window, or with
// per-channel Key groups the staged block (up to three CTAs per stream, 16
// bits); every CTA leaves one partial and the last to finish a stream merges
// them all.
struct DecodePlan {
  Fill fill, wfill;
  int splits = 0, wsplits = 0, nparts = 0;
};

DecodePlan plan_decode(kvq_cache* c, const LayerState& L) {
  DecodePlan d;
  const int n_streams = c->batch * c->kv_heads;
  if (L.n > 0) {
    d.fill = make_fill(L.bits, L.nt, L.pf, L.n_shrinks, L.n);
    d.splits = decode_splits(c->sms(), n_streams, d.fill.gps);
    if (L.chan) d.splits = (int)std::min<long long>(d.splits, d.fill.gps / 8);  // whole blocks per CTA
  }
  if (L.chan && L.n_all > L.n) {  // the staged block at 16 bits, token t in slot t mod 128
    d.wfill = make_fill(16, kWindowTiles, slots_per_tile(16), 0, L.n_all - L.n);
    d.wsplits = (int)std::min<long long>(3, d.wfill.gps);
    if (d.splits > kMaxSplits - 3) d.splits = kMaxSplits - 3;
  }
  if (L.window) {
    d.wfill = make_fill(16, kWindowTiles, slots_per_tile(16), 0, std::min<long long>(L.n_all, kWindowTokens + 1));
    // up to 9 16-bit groups: 3 CTAs so the window's copies overlap; every CTA gets a group
    d.wsplits = (int)std::min<long long>(3, d.wfill.gps);
    if (d.splits > kMaxSplits - 3) d.splits = kMaxSplits - 3;
  }
  d.nparts = d.splits + d.wsplits;
  return d;
}

// The new token of a fused single-token append (kvq_append_decode).
struct AppendOne {
  long long group = -1;  // its group in the kernels' group order; < 0: no append
  int tile = 0, slot = 0;
  const void* k = nullptr;
  const void* v = nullptr;
  int dtype = 0;
};

cudaError_t enqueue_decode(kvq_cache* c, int layer, const DecodePlan& d, const void* q, int q_heads, float sm_scale,
                           float* out, float* parts, cudaStream_t s, const AppendOne& app = AppendOne()) {
  const LayerState& L = c->L[layer];
  DecodeArgs a{};
  a.app_group = -1;
  a.q = q;
  a.lam = L.lambda_set ? c->lam(layer) : nullptr;
  a.out = out;
  a.parts = parts;
  a.counters = c->counters(layer);
  a.err = c->err();
  a.batch = c->batch;
  a.kv_heads = c->kv_heads;
  a.q_heads = q_heads;
  a.group = q_heads / c->kv_heads;
  a.qscale = sm_scale * 1.4426950408889634f;
  a.nparts = d.nparts;
  // The progressive cache first; the window launch follows it.  The first
  // launch triggers its dependents only after its own dependency wait, so
  // the window launch needs none: it runs in the shadow of the first one's
  // merge.  The last CTA of a stream, in either launch, merges all partials.
  // Per-channel Key groups take the other order: the staged block (a few
  // 16-bit groups) first, then the progressive cache without a wait at its
  // start (measured on the 7B 2-bit block: 92 us a call against 125 us with
  // the progressive cache first, whose early trigger let the staged block's
  // CTAs sit on SMs the next call's CTAs needed).
  if (L.chan && d.splits && d.wsplits) {
    DecodeArgs w = a;
    w.codes = c->wcodes(layer);
    w.meta = c->wmeta(layer);
    w.fill = d.wfill;
    w.splits = d.wsplits;
    w.part_base = d.splits;
    w.safe = 0;
    w.trigger_early = true;
    if (cudaError_t e = launch_decode(w, s)) return e;
    a.codes = c->codes(layer);
    a.meta = c->meta(layer);
    a.fill = d.fill;
    a.splits = d.splits;
    a.part_base = 0;
    a.safe = 0;
    a.chan = true;
    a.kmc = c->kmc(layer);
    a.blocks_max = c->blocks_max();
    a.ep = make_epochs(L.nt, L.n_shrinks);
    a.after_decode = true;  // everything before the staged block's launch is complete
    return launch_decode(a, s);
  }
  if (d.splits) {
    a.codes = c->codes(layer);
    a.meta = c->meta(layer);
    a.fill = d.fill;
    a.splits = d.splits;
    a.part_base = 0;
    a.safe = L.chan ? 0 : stable_groups(L, d.fill);  // the block-move kernel may still run: no early copies
    if (L.chan) {
      a.chan = true;
      a.kmc = c->kmc(layer);
      a.blocks_max = c->blocks_max();
      a.ep = make_epochs(L.nt, L.n_shrinks);
    }
    a.trigger_early = d.wsplits > 0;
    a.rank_sms = !L.chan && d.wsplits == 0 ? c->sms() : 0;  // the block's only launch: arrival-weighted slices
    if (app.group >= 0) {  // this launch writes the new token itself: keep the pre-wait copies clear of it
      a.app_group = app.group;
      a.app_tile = app.tile;
      a.app_slot = app.slot;
      a.ak = app.k;
      a.av = app.v;
      a.adtype = app.dtype;
      a.lam_inv = L.lambda_set ? c->lam_inv(layer) : nullptr;
      a.safe = std::min(a.safe, app.group);
    }
    if (cudaError_t e = launch_decode(a, s)) return e;
    a.trigger_early = false;
    a.app_group = -1;
    a.rank_sms = 0;
  }
  if (d.wsplits) {
    DecodeArgs w = a;
    w.chan = false;
    w.codes = c->wcodes(layer);
    w.meta = c->wmeta(layer);
    w.fill = d.wfill;
    w.splits = d.wsplits;
    w.part_base = d.splits;
    w.after_decode = d.splits > 0;
    w.safe = w.after_decode ? d.wfill.gps : 0;  // alone, every window slot may be rewritten by an append in flight
    if (cudaError_t e = launch_decode(w, s)) return e;
  }
  return cudaSuccess;
}

// Per-channel Key groups: append into the staged block (16 bits, slot
// t mod 128); each completed block enters the progressive cache, which is
// shrunk first when the block does not fit at its width.
kvq_status append_chan(kvq_cache* c, int layer, const void* k, const void* v, int dtype, int n_tokens,
                       cudaStream_t s) {
  LayerState& L = c->L[layer];
  int off = 0;
  while (off < n_tokens) {
    const int staged = (int)(L.n_all - L.n);
    const int cnt = std::min(n_tokens - off, kKeyBlock - staged);
    // a whole block with nothing staged goes straight from the input into
    // the progressive cache (the block move quantizes it as the append would
    // have staged it); otherwise the tokens are staged first
    const bool direct_block = staged == 0 && cnt == kKeyBlock;
    if (!direct_block) {
      AppendArgs a{};
      a.k = k;
      a.v = v;
      a.dtype = dtype;
      a.n_call = n_tokens;
      a.tok_off = off;
      a.cnt = cnt;
      a.n0 = L.n;
      a.bits = L.bits;
      a.nt = L.nt;
      a.pf = L.pf;
      a.batch = c->batch;
      a.kv_heads = c->kv_heads;
      a.codes = c->codes(layer);
      a.meta = c->meta(layer);
      a.lam_inv = L.lambda_set ? c->lam_inv(layer) : nullptr;
      a.window = true;
      a.stage = true;
      a.direct = L.shift_mode == KVQ_SHIFT_DIRECT;
      a.t0 = L.n_all;
      a.wcodes = c->wcodes(layer);
      a.wmeta = c->wmeta(layer);
      if (cudaError_t e = launch_append(a, s)) return cuda_fail(e, "append launch");
    }
    L.n_all += cnt;
    off += cnt;
    if (L.n_all - L.n < kKeyBlock) continue;
    // the block is complete: make room at the current width, then move it
    while (L.n + kKeyBlock > capacity(L, c->n_f, L.bits)) {  // the budget check keeps bits > fbit here
      const ShrinkArgs sa = shrink_args(c, layer);
      if (cudaError_t e = launch_shrink(sa, s)) return cuda_fail(e, "shrink launch");
      L.bits /= 2;
      L.n_shrinks++;
    }
    BlockMoveArgs m{};
    m.wcodes = c->wcodes(layer);
    m.wmeta = c->wmeta(layer);
    m.codes = c->codes(layer);
    m.meta = c->meta(layer);
    m.kmc = c->kmc(layer);
    m.blocks_max = c->blocks_max();
    m.blk = (int)(L.n / kKeyBlock);
    m.nt = L.nt;
    m.pf = L.pf;
    m.bits = L.bits;
    m.direct = L.shift_mode == KVQ_SHIFT_DIRECT;
    m.from_input = direct_block;
    m.k = k;
    m.v = v;
    m.dtype = dtype;
    m.n_call = n_tokens;
    m.tok_off = off - cnt;
    m.kv_heads = c->kv_heads;
    m.lam_inv = L.lambda_set ? c->lam_inv(layer) : nullptr;
    for (int gi = 0; gi < kKeyBlock / kGroupTokens; gi++) slot_of(L, L.n + kGroupTokens * gi, &m.g_tile[gi], &m.g_slot[gi]);
    if (cudaError_t e = launch_block_move(m, c->batch * c->kv_heads, s)) return cuda_fail(e, "block move launch");
    L.n += kKeyBlock;
    L.n_stable = L.n;
  }
  return KVQ_OK;
}

uint32_t rd32(const uint8_t* p) {
  uint32_t w;
  memcpy(&w, p, 4);
  return w;
}

}  // namespace

extern "C" {

size_t kvq_pool_bytes_ex(int layers, int batch, int kv_heads, int head_dim, size_t budget_bytes, const int* fbit,
                         int options) {
  Plan p;
  kvq_status why;
  if (!make_plan(layers, batch, kv_heads, head_dim, budget_bytes, fbit, options, p, &why)) return 0;
  return p.bytes;
}

size_t kvq_pool_bytes(int layers, int batch, int kv_heads, int head_dim, size_t budget_bytes, const int* fbit) {
  return kvq_pool_bytes_ex(layers, batch, kv_heads, head_dim, budget_bytes, fbit, 0);
}

kvq_status kvq_alloc_ex(kvq_cache** out, int layers, int batch, int kv_heads, int head_dim, size_t budget_bytes,
                        const int* fbit, void* dev_pool, size_t pool_bytes, int options) {
  if (!out) return fail(KVQ_ERR_INVALID, "out is NULL");
  *out = nullptr;
  Plan p;
  kvq_status why;
  if (!make_plan(layers, batch, kv_heads, head_dim, budget_bytes, fbit, options, p, &why)) {
    if (why == KVQ_ERR_BUDGET) return fail(why, "budget of %zu bytes holds fewer than %d tokens per block", budget_bytes, kTokenRound);
    return fail(why, "invalid shape, fbit or options (layers=%d batch=%d kv_heads=%d head_dim=%d options=%d; fbit must be "
                "2/4/8/16, head_dim 128)", layers, batch, kv_heads, head_dim, options);
  }
  if (dev_pool && pool_bytes < p.bytes)
    return fail(KVQ_ERR_INVALID, "pool of %zu bytes is smaller than the %zu bytes needed", pool_bytes, p.bytes);
  if (dev_pool && (reinterpret_cast<uintptr_t>(dev_pool) % kAlign))
    return fail(KVQ_ERR_INVALID, "pool must be %zu-byte aligned", kAlign);
  kvq_cache* c = new (std::nothrow) kvq_cache();
  if (!c) return fail(KVQ_ERR_OOM, "host allocation failed");
  c->layers = layers;
  c->batch = batch;
  c->kv_heads = kv_heads;
  c->n_f = p.n_f;
  c->L = p.layers;
  c->num_sms = 0;
  c->err_zeroed = false;
  if (dev_pool) {
    c->pool = static_cast<uint8_t*>(dev_pool);
    c->owns_pool = false;
  } else {
    if (fault_alloc()) {
      delete c;
      return fail(KVQ_ERR_OOM, "cudaMalloc(%zu): injected failure (KVQ_FAULT_ALLOC)", p.bytes);
    }
    void* ptr = nullptr;
    cudaError_t e = cudaMalloc(&ptr, p.bytes);
    if (e != cudaSuccess) {
      cudaGetLastError();
      delete c;
      return fail(KVQ_ERR_OOM, "cudaMalloc(%zu): %s", p.bytes, cudaGetErrorString(e));
    }
    c->pool = static_cast<uint8_t*>(ptr);
    c->owns_pool = true;
  }
  c->pool_bytes = p.bytes;
  *out = c;
  return KVQ_OK;
}

kvq_status kvq_alloc(kvq_cache** out, int layers, int batch, int kv_heads, int head_dim, size_t budget_bytes,
                     const int* fbit, void* dev_pool, size_t pool_bytes) {
  return kvq_alloc_ex(out, layers, batch, kv_heads, head_dim, budget_bytes, fbit, dev_pool, pool_bytes, 0);
}

kvq_status kvq_set_lambda(kvq_cache* c, int layer, const float* lambda_host) {
  if (kvq_status s = check_layer(c, layer)) return s;
  if (!lambda_host) return fail(KVQ_ERR_INVALID, "lambda is NULL");
  const size_t n = (size_t)c->kv_heads * kHeadDim;
  std::vector<float> inv(n);
  for (size_t i = 0; i < n; i++) {
    const float v = lambda_host[i];
    if (!(v > 0.0f) || !std::isfinite(v)) return fail(KVQ_ERR_INVALID, "lambda[%zu] = %g is not finite and > 0", i, (double)v);
    inv[i] = (float)(1.0 / (double)v);
  }
  if (c->L[layer].n != 0) return fail(KVQ_ERR_STATE, "layer %d already holds tokens; set lambda before the first append", layer);
  cudaError_t e = cudaMemcpy(c->lam(layer), lambda_host, n * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(c->lam_inv(layer), inv.data(), n * 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "lambda upload");
  c->L[layer].lambda_set = true;
  return KVQ_OK;
}

kvq_status kvq_append(kvq_cache* c, int layer, const void* k, const void* v, int dtype, int n_tokens,
                      kvq_stream_t stream) {
  const Range range("kvq_append");
  if (kvq_status s = check_layer(c, layer)) return s;
  if (n_tokens < 0) return fail(KVQ_ERR_INVALID, "n_tokens %d < 0", n_tokens);
  if (n_tokens == 0) return KVQ_OK;
  if (!k || !v) return fail(KVQ_ERR_INVALID, "k or v is NULL");
  if (dtype != KVQ_DTYPE_BF16 && dtype != KVQ_DTYPE_F32) return fail(KVQ_ERR_INVALID, "dtype %d unknown", dtype);
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) % 16)
    return fail(KVQ_ERR_INVALID, "k and v must be 16-byte aligned");
  LayerState& L = c->L[layer];
  const long long W1 = kWindowTokens + 1;  // sink + window
  if (L.chan) {
    if ((L.n_all + n_tokens) / kKeyBlock * kKeyBlock > c->n_f)
      return fail(KVQ_ERR_BUDGET, "layer %d holds %lld tokens (%lld staged); %d more complete blocks that do not fit at "
                  "Fbit %d", layer, L.n_all, L.n_all - L.n, n_tokens, L.fbit);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
    return append_chan(c, layer, k, v, dtype, n_tokens, s);
  }
  if (!L.window && L.n + n_tokens > c->n_f)
    return fail(KVQ_ERR_BUDGET, "layer %d holds %lld of %lld tokens at Fbit %d; %d more do not fit", layer, L.n, c->n_f,
                L.fbit, n_tokens);
  if (L.window && std::max(0LL, L.n_all + n_tokens - W1) > c->n_f)
    return fail(KVQ_ERR_BUDGET, "layer %d holds %lld tokens (%lld in the window); %d more do not fit at Fbit %d", layer,
                L.n_all, std::min(L.n_all, W1), n_tokens, L.fbit);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
  int off = 0;
  while (off < n_tokens) {
    const long long cap = capacity(L, c->n_f, L.bits);
    // tokens this launch moves into the progressive cache: with the window,
    // token t >= 129 moves token t - 128 (to index t - 129)
    const long long t0 = L.window ? L.n_all : 0;
    const bool moves_next = L.window ? t0 >= W1 : true;
    if (L.n == cap && moves_next) {  // full: shrink one level first (bits > fbit is implied by the budget check)
      const ShrinkArgs sa = shrink_args(c, layer);
      cudaError_t e = launch_shrink(sa, s);
      if (e != cudaSuccess) return cuda_fail(e, "shrink launch");
      L.bits /= 2;
      L.n_shrinks++;
      continue;
    }
    int cnt;
    if (L.window) {
      // at most 128 tokens a launch (their window slots are distinct), and no
      // more moves than the progressive cache holds at this width
      long long lim = std::min<long long>(n_tokens - off, kWindowTokens);
      lim = std::min(lim, cap + W1 - t0);  // keeps t0 + cnt - 129 <= cap
      cnt = (int)lim;
    } else {
      cnt = (int)std::min<long long>(n_tokens - off, cap - L.n);
    }
    AppendArgs a{};
    a.k = k;
    a.v = v;
    a.dtype = dtype;
    a.n_call = n_tokens;
    a.tok_off = off;
    a.cnt = cnt;
    a.n0 = L.n;
    a.bits = L.bits;
    const int p = slots_per_tile(L.bits);
    a.h = L.n_shrinks > 0 ? p / 2 : 0;
    a.e = p - a.h;
    a.nt = L.nt;
    a.pf = L.pf;
    a.batch = c->batch;
    a.kv_heads = c->kv_heads;
    a.codes = c->codes(layer);
    a.meta = c->meta(layer);
    a.lam_inv = L.lambda_set ? c->lam_inv(layer) : nullptr;
      a.window = L.window;
    a.direct = L.shift_mode == KVQ_SHIFT_DIRECT;
    a.t0 = t0;
    a.wcodes = L.window ? c->wcodes(layer) : nullptr;
    a.wmeta = L.window ? c->wmeta(layer) : nullptr;
    cudaError_t e = launch_append(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    L.n_stable = L.n;
    if (L.window) {
      L.n_all += cnt;
      L.n = std::max(0LL, L.n_all - W1);
    } else {
      L.n += cnt;
    }
    off += cnt;
  }
  return KVQ_OK;
}

kvq_status kvq_shrink(kvq_cache* c, int layer, kvq_stream_t stream) {
  const Range range("kvq_shrink");
  if (kvq_status s = check_layer(c, layer)) return s;
  LayerState& L = c->L[layer];
  if (L.bits <= L.fbit) return fail(KVQ_ERR_STATE, "layer %d is at its Fbit %d", layer, L.fbit);
  const long long cap = capacity(L, c->n_f, L.bits);
  if (L.n != cap)
    return fail(KVQ_ERR_STATE, "layer %d holds %lld tokens; a shrink needs the block full (%lld at %d bits)", layer, L.n, cap,
                L.bits);
  const ShrinkArgs sa = shrink_args(c, layer);
  cudaError_t e = launch_shrink(sa, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "shrink launch");
  L.bits /= 2;
  L.n_shrinks++;
  L.n_stable = L.n;
  return KVQ_OK;
}

kvq_status kvq_set_shift_mode(kvq_cache* c, int layer, int mode) {
  if (kvq_status s = check_layer(c, layer)) return s;
  if (mode != KVQ_SHIFT_EQUIVALENT && mode != KVQ_SHIFT_DIRECT) return fail(KVQ_ERR_INVALID, "shift mode %d unknown", mode);
  LayerState& L = c->L[layer];
  if (L.n_shrinks > 0 && mode != L.shift_mode)
    return fail(KVQ_ERR_STATE, "layer %d has already shrunk; its shift is fixed", layer);
  L.shift_mode = mode;
  return KVQ_OK;
}

size_t kvq_decode_workspace(const kvq_cache* c, int layer, int q_heads) {
  if (!c || layer < 0 || layer >= c->layers || q_heads <= 0 || q_heads % c->kv_heads) return 0;
  const int G = q_heads / c->kv_heads;
  if (G > 8) return 0;
  return decode_parts_bytes(c->batch * c->kv_heads, G);
}

kvq_status kvq_decode_attn(kvq_cache* c, int layer, const void* q, int q_heads, float sm_scale, float* out,
                           void* workspace, size_t ws_bytes, kvq_stream_t stream) {
  const Range range("kvq_decode_attn");
  if (kvq_status s = check_layer(c, layer)) return s;
  if (!q || !out) return fail(KVQ_ERR_INVALID, "q or out is NULL");
  if (q_heads <= 0 || q_heads % c->kv_heads)
    return fail(KVQ_ERR_INVALID, "q_heads %d is not a positive multiple of kv_heads %d", q_heads, c->kv_heads);
  const int G = q_heads / c->kv_heads;
  if (G > 8) return fail(KVQ_ERR_INVALID, "%d query heads per KV head; at most 8 are supported", G);
  if (!std::isfinite(sm_scale)) return fail(KVQ_ERR_INVALID, "sm_scale is not finite");
  if ((reinterpret_cast<uintptr_t>(q) % 16) || (reinterpret_cast<uintptr_t>(out) % 4))
    return fail(KVQ_ERR_INVALID, "q must be 16-byte aligned and out 4-byte aligned");
  LayerState& L = c->L[layer];
  if ((L.window || L.chan ? L.n_all : L.n) <= 0) return fail(KVQ_ERR_STATE, "layer %d is empty", layer);
  const int n_streams = c->batch * c->kv_heads;
  const size_t need = decode_parts_bytes(n_streams, G);
  if (!workspace || ws_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace of %zu bytes; %zu needed", workspace ? ws_bytes : (size_t)0, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
  if (!L.counters_zeroed) {
    cudaError_t e = cudaMemsetAsync(c->counters(layer), 0, (size_t)n_streams * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "counter reset");
    L.counters_zeroed = true;
  }
  const DecodePlan d = plan_decode(c, L);
  cudaError_t e = enqueue_decode(c, layer, d, q, q_heads, sm_scale, out, static_cast<float*>(workspace), s);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return KVQ_OK;
}

kvq_status kvq_append_decode(kvq_cache* c, int layer, const void* k, const void* v, int dtype, const void* q,
                             int q_heads, float sm_scale, float* out, void* workspace, size_t ws_bytes,
                             kvq_stream_t stream) {
  const Range range("kvq_append_decode");
  if (kvq_status s = check_layer(c, layer)) return s;
  LayerState& L = c->L[layer];
  if (L.window || L.chan) {  // the window's moves and the staged blocks need the append kernels: the two calls
    if (kvq_status st = kvq_append(c, layer, k, v, dtype, 1, stream)) return st;
    return kvq_decode_attn(c, layer, q, q_heads, sm_scale, out, workspace, ws_bytes, stream);
  }
  if (!k || !v || !q || !out) return fail(KVQ_ERR_INVALID, "k, v, q or out is NULL");
  if (dtype != KVQ_DTYPE_BF16 && dtype != KVQ_DTYPE_F32) return fail(KVQ_ERR_INVALID, "dtype %d unknown", dtype);
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) % 16)
    return fail(KVQ_ERR_INVALID, "k and v must be 16-byte aligned");
  if (q_heads <= 0 || q_heads % c->kv_heads)
    return fail(KVQ_ERR_INVALID, "q_heads %d is not a positive multiple of kv_heads %d", q_heads, c->kv_heads);
  const int G = q_heads / c->kv_heads;
  if (G > 8) return fail(KVQ_ERR_INVALID, "%d query heads per KV head; at most 8 are supported", G);
  if (!std::isfinite(sm_scale)) return fail(KVQ_ERR_INVALID, "sm_scale is not finite");
  if ((reinterpret_cast<uintptr_t>(q) % 16) || (reinterpret_cast<uintptr_t>(out) % 4))
    return fail(KVQ_ERR_INVALID, "q must be 16-byte aligned and out 4-byte aligned");
  if (L.n + 1 > c->n_f)
    return fail(KVQ_ERR_BUDGET, "layer %d holds %lld of %lld tokens at Fbit %d; 1 more does not fit", layer, L.n, c->n_f,
                L.fbit);
  const int n_streams = c->batch * c->kv_heads;
  const size_t need = decode_parts_bytes(n_streams, G);
  if (!workspace || ws_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace of %zu bytes; %zu needed", workspace ? ws_bytes : (size_t)0, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
  if (!L.counters_zeroed) {
    cudaError_t e = cudaMemsetAsync(c->counters(layer), 0, (size_t)n_streams * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "counter reset");
    L.counters_zeroed = true;
  }
  if (L.n == capacity(L, c->n_f, L.bits)) {  // full: shrink one level first, as kvq_append would
    const ShrinkArgs sa = shrink_args(c, layer);
    if (cudaError_t e = launch_shrink(sa, s)) return cuda_fail(e, "shrink launch");
    L.bits /= 2;
    L.n_shrinks++;
  }
  // the new token's slot (the append kernel's formula) and its group
  const int p = slots_per_tile(L.bits);
  const int h = L.n_shrinks > 0 ? p / 2 : 0;
  const long long m = L.n - (long long)L.nt * h;
  AppendOne app;
  app.tile = (int)(m / (p - h));
  app.slot = h + (int)(m % (p - h));
  app.group = (long long)app.tile * (p / kGroupTokens) + app.slot / kGroupTokens;
  app.k = k;
  app.v = v;
  app.dtype = dtype;
  L.n += 1;  // the plan covers the new token
  const DecodePlan d = plan_decode(c, L);
  L.n -= 1;
  cudaError_t e = enqueue_decode(c, layer, d, q, q_heads, sm_scale, out, static_cast<float*>(workspace), s, app);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  L.n_stable = L.n;
  L.n += 1;
  return KVQ_OK;
}

// ---- decode attention without a caller workspace ----------------------------
//
// Some callers cannot allocate device memory at the point where they run
// decode: code inside a framework whose allocator owns all device memory,
// a serving loop that must not allocate after start-up (allocation can
// stall, fragment or fail under memory pressure), or a host that only hands
// out input and output buffers.  For them this entry point keeps the split
// partials in a fixed buffer of device memory that is part of the library
// itself: every GPU that loads the library holds it until the process exits.
// Nothing is allocated per call.
constexpr size_t kNoAllocScratchBytes = (size_t)24 << 20;  // 24 MiB per device
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
// Device address of the scratch buffer on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with the device current, on every call: a runtime query that allocates
// nothing, and that stays right after a device reset or a new context (which
// may load the library's device code at another address).
cudaError_t noalloc_scratch(void** out) {
  *out = nullptr;
  return cudaGetSymbolAddress(out, g_noalloc_scratch);
}
}  // namespace

kvq_status kvq_decode_attn_noalloc(kvq_cache* c, int layer, const void* q, int q_heads, float sm_scale,
                                   float* out, kvq_stream_t stream) {
  const Range range("kvq_decode_attn_noalloc");
  if (kvq_status s = check_layer(c, layer)) return s;
  if (!q || !out) return fail(KVQ_ERR_INVALID, "q or out is NULL");
  if (q_heads <= 0 || q_heads % c->kv_heads)
    return fail(KVQ_ERR_INVALID, "q_heads %d is not a positive multiple of kv_heads %d", q_heads, c->kv_heads);
  const int G = q_heads / c->kv_heads;
  if (G > 8) return fail(KVQ_ERR_INVALID, "%d query heads per KV head; at most 8 are supported", G);
  if (!std::isfinite(sm_scale)) return fail(KVQ_ERR_INVALID, "sm_scale is not finite");
  if ((reinterpret_cast<uintptr_t>(q) % 16) || (reinterpret_cast<uintptr_t>(out) % 4))
    return fail(KVQ_ERR_INVALID, "q must be 16-byte aligned and out 4-byte aligned");
  LayerState& L = c->L[layer];
  if ((L.window || L.chan ? L.n_all : L.n) <= 0) return fail(KVQ_ERR_STATE, "layer %d is empty", layer);
  const int n_streams = c->batch * c->kv_heads;
  const DecodePlan d = plan_decode(c, L);
  // A single partial per stream goes straight to `out`: the scratch is used
  // only when a stream is cut into several.
  const size_t need = d.nparts > 1 ? decode_parts_used(n_streams, d.nparts) : 0;
  if (need > kNoAllocScratchBytes)
    return fail(KVQ_ERR_WORKSPACE,
                "this block needs %zu bytes of scratch (batch*kv_heads=%d x %d splits); the built-in buffer holds "
                "%zu bytes -- use kvq_decode_attn with a workspace",
                need, n_streams, d.nparts, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (cudaError_t e = noalloc_scratch(&scratch)) return cuda_fail(e, "scratch address");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
  if (!L.counters_zeroed) {  // the ticket counters live in the cache pool and must start at zero
    cudaError_t e = cudaMemsetAsync(c->counters(layer), 0, (size_t)n_streams * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "counter reset");
    L.counters_zeroed = true;
  }
  // the scratch is fully written before it is read: it needs no clearing
  cudaError_t e = enqueue_decode(c, layer, d, q, q_heads, sm_scale, out, static_cast<float*>(scratch), s);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return KVQ_OK;
}

kvq_status kvq_query(const kvq_cache* c, int layer, int* tokens, int* bits, int* cap, int* n_shrinks) {
  if (kvq_status s = check_layer(c, layer)) return s;
  const LayerState& L = c->L[layer];
  const int w = L.window ? kWindowTokens + 1 : (L.chan ? kKeyBlock - 1 : 0);
  if (tokens) *tokens = (int)(L.window || L.chan ? L.n_all : L.n);
  if (bits) *bits = L.bits;
  if (cap) *cap = (int)capacity(L, c->n_f, L.bits) + w;
  if (n_shrinks) *n_shrinks = L.n_shrinks;
  return KVQ_OK;
}

int kvq_max_tokens(const kvq_cache* c) {
  if (!c) return 0;
  if (c->layers > 0 && c->L[0].chan) return (int)c->n_f + kKeyBlock - 1;
  return (int)c->n_f + (c->layers > 0 && c->L[0].window ? kWindowTokens + 1 : 0);
}

kvq_status kvq_export(const kvq_cache* c, int layer, int b, int j, uint16_t* k_codes, uint16_t* v_codes,
                      uint16_t* k_meta, uint16_t* v_meta, kvq_stream_t stream) {
  if (kvq_status s = check_layer(c, layer)) return s;
  if (b < 0 || b >= c->batch || j < 0 || j >= c->kv_heads)
    return fail(KVQ_ERR_INVALID, "stream (%d, %d) out of range", b, j);
  const LayerState& L = c->L[layer];
  kvq_cache* m = const_cast<kvq_cache*>(c);
  const size_t code_bytes = (size_t)L.nt * kTileBytes, meta_words = (size_t)L.nt * L.pf * 2;
  const size_t st = (size_t)b * c->kv_heads + j;
  std::vector<uint8_t> cb(code_bytes);
  std::vector<uint32_t> mw(meta_words);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(cb.data(), m->codes(layer) + st * code_bytes, code_bytes, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(mw.data(), m->meta(layer) + st * meta_words, meta_words * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "export copy");
  const int bits = L.bits, ppw = 16 / bits;
  const uint32_t mask = bits == 16 ? 0xffffu : ((1u << bits) - 1u);
  std::vector<uint32_t> kw;  // per-channel Key meta of the stream's blocks
  if (L.chan && k_meta && L.n > 0) {
    kw.resize((size_t)L.n);  // (L.n / 128) blocks of 128 words
    const size_t base = st * (size_t)c->blocks_max() * kHeadDim;
    e = cudaMemcpyAsync(kw.data(), m->kmc(layer) + base, kw.size() * 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "export copy");
  }
  for (long long i = 0; i < L.n; i++) {
    int tile, slot;
    slot_of(L, i, &tile, &slot);
    const int grp = slot >> 4, tok = slot & 15;
    const size_t gbase = (size_t)tile * kTileBytes + (size_t)grp * group_bytes(bits);
    if (k_codes) {
      const int g = tok & 7, x = tok >> 3;
      for (int kp = 0; kp < kHeadDim; kp++) {
        // channel 32s + 16r + 4t + i: member i of quad p = 2s + r in unit 4g + t
        const int p = 2 * (kp >> 5) + ((kp >> 4) & 1), t = (kp >> 2) & 3, mi = kp & 3;
        int word, shift;
        if (bits == 16) {
          word = x * bits + 2 * p + (mi >> 1);
          shift = 16 * (mi & 1);
        } else {
          const int qpw = 8 / bits;
          word = x * bits + p / qpw;
          shift = 8 * mi + bits * (p % qpw);
        }
        const uint32_t w = rd32(&cb[gbase + (size_t)(4 * g + t) * unit_bytes(bits) + 4 * word]);
        k_codes[i * kHeadDim + kp] = (uint16_t)((w >> shift) & mask);
      }
    }
    if (v_codes) {
      const int t = (tok & 7) >> 1, mb = tok & 1, u = tok >> 3;
      for (int ch = 0; ch < kHeadDim; ch++) {
        const int sb = ch >> 4, rem = ch & 15, r = rem >> 3, g = rem & 7;
        const int p = 2 * sb + r, word = u * bits + p / ppw, pos = p % ppw;
        const uint32_t w = rd32(&cb[gbase + part_bytes(bits) + (size_t)(4 * g + t) * unit_bytes(bits) + 4 * word]);
        v_codes[i * kHeadDim + ch] = (uint16_t)((w >> (16 * mb + bits * pos)) & mask);
      }
    }
    const size_t mi = ((size_t)tile * L.pf + slot) * 2;
    if (k_meta) {  // per-channel Key groups: entry 128 k + c is channel c of block k
      const uint32_t w = L.chan ? kw[i] : mw[mi];
      k_meta[2 * i] = (uint16_t)(w & 0xffffu);
      k_meta[2 * i + 1] = (uint16_t)(w >> 16);
    }
    if (v_meta) {
      v_meta[2 * i] = (uint16_t)(mw[mi + 1] & 0xffffu);
      v_meta[2 * i + 1] = (uint16_t)(mw[mi + 1] >> 16);
    }
  }
  return KVQ_OK;
}

kvq_status kvq_export_window(const kvq_cache* c, int layer, int b, int j, uint16_t* k_codes, uint16_t* v_codes,
                             uint16_t* k_meta, uint16_t* v_meta, int* n_tokens, kvq_stream_t stream) {
  if (kvq_status s = check_layer(c, layer)) return s;
  if (b < 0 || b >= c->batch || j < 0 || j >= c->kv_heads)
    return fail(KVQ_ERR_INVALID, "stream (%d, %d) out of range", b, j);
  const LayerState& L = c->L[layer];
  if (!L.window && !L.chan)
    return fail(KVQ_ERR_INVALID, "the cache was made without KVQ_OPT_SINK_WINDOW or KVQ_OPT_KEY_CHANNEL");
  kvq_cache* m = const_cast<kvq_cache*>(c);
  constexpr int P16 = slots_per_tile(16);
  const size_t code_bytes = (size_t)kWindowTiles * kTileBytes, meta_words = (size_t)kWindowTiles * P16 * 2;
  const size_t st = (size_t)b * c->kv_heads + j;
  std::vector<uint8_t> cb(code_bytes);
  std::vector<uint32_t> mw(meta_words);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(cb.data(), m->wcodes(layer) + st * code_bytes, code_bytes, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(mw.data(), m->wmeta(layer) + st * meta_words, meta_words * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "export copy");
  // window: tokens 0, then max(1, n - 128) .. n - 1; token t >= 1 sits in slot 1 + (t - 1) mod 128.
  // per-channel Key groups: the staged tokens, token t in slot t mod 128.
  std::vector<long long> toks;
  if (L.chan) {
    for (long long t = L.n; t < L.n_all; t++) toks.push_back(t);
  } else {
    if (L.n_all > 0) toks.push_back(0);
    for (long long t = std::max(1LL, L.n_all - kWindowTokens); t < L.n_all; t++) toks.push_back(t);
  }
  constexpr int kUnit = 8 * 16;  // unit bytes at 16 bits
  for (size_t i = 0; i < toks.size(); i++) {
    const long long t = toks[i];
    const int rs = L.chan ? (int)(t % kKeyBlock) : (t == 0 ? 0 : 1 + (int)((t - 1) % kWindowTokens));
    const int tile = rs / P16, slot = rs % P16, grp = slot >> 4, tok = slot & 15;
    const size_t gbase = (size_t)tile * kTileBytes + (size_t)grp * group_bytes(16);
    if (k_codes) {
      const int g = tok & 7, x = tok >> 3;
      for (int kp = 0; kp < kHeadDim; kp++) {
        const int p = 2 * (kp >> 5) + ((kp >> 4) & 1), tt = (kp >> 2) & 3, mi = kp & 3;
        const int word = x * 16 + 2 * p + (mi >> 1);
        const uint32_t w = rd32(&cb[gbase + (size_t)(4 * g + tt) * kUnit + 4 * word]);
        k_codes[i * kHeadDim + kp] = (uint16_t)(w >> (16 * (mi & 1)));
      }
    }
    if (v_codes) {
      const int tt = (tok & 7) >> 1, mb = tok & 1, u = tok >> 3;
      for (int ch = 0; ch < kHeadDim; ch++) {
        const int sb = ch >> 4, r = (ch >> 3) & 1, g = ch & 7;
        const int word = u * 16 + 2 * sb + r;
        const uint32_t w = rd32(&cb[gbase + part_bytes(16) + (size_t)(4 * g + tt) * kUnit + 4 * word]);
        v_codes[i * kHeadDim + ch] = (uint16_t)(w >> (16 * mb));
      }
    }
    const size_t mi = ((size_t)tile * P16 + slot) * 2;
    if (k_meta) {
      k_meta[2 * i] = (uint16_t)(mw[mi] & 0xffffu);
      k_meta[2 * i + 1] = (uint16_t)(mw[mi] >> 16);
    }
    if (v_meta) {
      v_meta[2 * i] = (uint16_t)(mw[mi + 1] & 0xffffu);
      v_meta[2 * i + 1] = (uint16_t)(mw[mi + 1] >> 16);
    }
  }
  if (n_tokens) *n_tokens = (int)toks.size();
  return KVQ_OK;
}

kvq_status kvq_device_status(kvq_cache* c, kvq_stream_t stream) {
  if (!c) return fail(KVQ_ERR_INVALID, "cache is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
  int flag = 0;
  cudaError_t e = cudaMemcpyAsync(&flag, c->err(), 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "device status");
  if (flag) {
    const int zero = 0;
    e = cudaMemcpy(c->err(), &zero, 4, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "device status reset");
    return fail(KVQ_ERR_TIMEOUT, "a kernel gave up waiting on its own bulk copies");
  }
  return KVQ_OK;
}

kvq_status kvq_selftest_timeout(kvq_cache* c, kvq_stream_t stream) {
  if (!c) return fail(KVQ_ERR_INVALID, "cache is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = c->ensure_err(s)) return cuda_fail(e, "error flag reset");
  if (cudaError_t e = launch_wait_probe(c->err(), s)) return cuda_fail(e, "wait probe launch");
  return KVQ_OK;
}

const char* kvq_last_error(void) { return g_last_error.c_str(); }

void kvq_free(kvq_cache* c) {
  if (!c) return;
  if (c->owns_pool && c->pool) {
    cudaDeviceSynchronize();
    cudaFree(c->pool);
  }
  delete c;
}

}  // extern "C"
