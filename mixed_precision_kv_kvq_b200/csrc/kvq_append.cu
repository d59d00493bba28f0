// kvq_append.cu -- quantize-on-append (PM-KVQ note, key design 1: each new
// token is stored at the block's current width; key design 3: Keys are
// divided by the per-channel migration factor lambda first; training
// strategy: asymmetric groups of 128).
//
// One warp quantizes the groups (128 channels of one KV head, K or V) of a
// few consecutive tokens with the quantizer of kvq_quant.cuh (Keys divided by
// lambda first), scatters the codes into the lane units of the group's K or V
// part (see kvq_internal.cuh) and writes (R, Z) to the slot's K or V meta word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "kvq_quant.cuh"

namespace kvq {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kTokensPerWarp = 4;

// BITS: the block's current width (the progressive cache's, with the window).
template <int BITS>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) append_kernel(AppendArgs a) {
  __shared__ uint16_t codes_sh[kWarpsPerBlock][kHeadDim];
  __shared__ float4 x_sh[kWarpsPerBlock][kTokensPerWarp][32];
  pdl_wait();  // k/v and the cache may come from earlier kernels in the stream
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  // grid: x over (token block, head, K/V) of one sequence, y = sequence; a
  // warp takes kTokensPerWarp consecutive tokens (their inputs are loaded
  // together, so more bytes are in flight).  The host keeps the counts below
  // 2^31, so the index math is 32-bit.
  const unsigned nblk = ((unsigned)a.cnt + kTokensPerWarp - 1) / kTokensPerWarp;
  const unsigned w = blockIdx.x * kWarpsPerBlock + wib;
  if (w >= nblk * (unsigned)a.kv_heads * 2u) return;  // warp-uniform
  const int b = blockIdx.y;
  const int kv = (int)(w & 1u);
  const unsigned rest = w >> 1;
  const int tb = (int)(rest / (unsigned)a.kv_heads);
  const int j = (int)(rest - (unsigned)tb * (unsigned)a.kv_heads);
  const int tk0 = tb * kTokensPerWarp;
  const int ntk = min(kTokensPerWarp, a.cnt - tk0);
  const size_t stream = (size_t)b * a.kv_heads + j;
  uint16_t* sc = codes_sh[wib];

  // ---- load 4 channels per lane of every token of this warp, migrate Keys ----
  const void* src = kv ? a.v : a.k;
  {
    float4 xv[kTokensPerWarp];
#pragma unroll
    for (int tt = 0; tt < kTokensPerWarp; tt++) {  // every load issued before any is used
      if (tt < ntk) {
        const size_t in_off =
            (((size_t)b * a.n_call + (size_t)(a.tok_off + tk0 + tt)) * a.kv_heads + j) * kHeadDim + 4 * lane;
        if (a.dtype == 1) {
          xv[tt] = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + in_off);
        } else {
          const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(src) + in_off);
          xv[tt] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                               __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
        }
      }
    }
    float4 li = make_float4(1.f, 1.f, 1.f, 1.f);
    const bool mig = kv == 0 && a.lam_inv;
    if (mig) li = *reinterpret_cast<const float4*>(a.lam_inv + (size_t)j * kHeadDim + 4 * lane);
#pragma unroll
    for (int tt = 0; tt < kTokensPerWarp; tt++) {
      if (tt < ntk) {
        float4 v = xv[tt];
        if (mig) {
          v.x = __fmul_rn(v.x, li.x); v.y = __fmul_rn(v.y, li.y);
          v.z = __fmul_rn(v.z, li.z); v.w = __fmul_rn(v.w, li.w);
        }
        x_sh[wib][tt][lane] = v;
      }
    }
  }

  // progressive-cache slot of index li at the block's current width
  auto main_group = [&](long long li, int* slot_out, size_t* tile_out) {
    const unsigned m = (unsigned)(li - (long long)a.nt * a.h);  // < 2^30: tokens per stream
    const int tile = (int)(m / (unsigned)a.e);
    const int slot = a.h + (int)(m - (unsigned)tile * (unsigned)a.e);
    *slot_out = slot;
    *tile_out = stream * a.nt + tile;
    return a.codes + *tile_out * (size_t)kTileBytes + (size_t)(slot >> 4) * group_bytes(BITS) +
           (size_t)kv * part_bytes(BITS);
  };

  for (int tt = 0; tt < ntk; tt++) {  // warp-uniform
    const int tkn = tk0 + tt;
    const float4 xv4 = x_sh[wib][tt][lane];  // written by this lane
    const float x[4] = {xv4.x, xv4.y, xv4.z, xv4.w};

    // ---- sink + window: the slot token t uses is the one its leaving token frees ----
    uint8_t* wg = nullptr;
    size_t wmi = 0;
    int wtok = 0;
    if (a.window) {
      const long long t = a.t0 + tkn;
      const int rs = a.stage ? (int)((unsigned long long)t & (kKeyBlock - 1))
                             : (t == 0 ? 0 : 1 + (int)((unsigned long long)(t - 1) & (kWindowTokens - 1)));
      const int wtile = rs / slots_per_tile(16), wslot = rs % slots_per_tile(16);
      wtok = wslot & 15;
      wg = a.wcodes + (stream * kWindowTiles + wtile) * (size_t)kTileBytes + (size_t)(wslot >> 4) * group_bytes(16) +
           (size_t)kv * part_bytes(16);
      wmi = ((stream * kWindowTiles + wtile) * (size_t)slots_per_tile(16) + wslot) * 2 + kv;
      if (!a.stage && t >= kWindowTokens + 1) {
        // token t - 128 leaves the window: its INT16 codes go to the progressive
        // cache at the current width (index t - 129) by the block's shift chain
        unpack_codes16(wg, wtok, kv, sc, lane);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; i++) sc[4 * lane + i] = (uint16_t)shift_chain<BITS>(sc[4 * lane + i], a.direct);
        const uint32_t old = a.wmeta[wmi];
        __syncwarp();
        int slot;
        size_t tile;
        uint8_t* gbase = main_group(t - (kWindowTokens + 1), &slot, &tile);
        pack_codes<BITS>(gbase, slot & 15, kv, sc, lane);
        if (lane == 0) {
          const uint32_t mw = (uint32_t)range_chain<BITS>((uint16_t)(old & 0xffffu), a.direct) | (old & 0xffff0000u);
          a.meta[(tile * (size_t)a.pf + slot) * 2 + kv] = mw;
        }
        __syncwarp();  // sc is reused below
      }
    }

    // ---- group meta and codes (window tokens are held at INT16) ----
    const uint32_t mw = quantize_group(x, a.window ? 65535u : (1u << BITS) - 1u, sc, lane);
    __syncwarp();

    if (a.window) {
      pack_codes<16>(wg, wtok, kv, sc, lane);
      if (lane == 0) a.wmeta[wmi] = mw;
    } else {
      int slot;
      size_t tile;
      uint8_t* gbase = main_group(a.n0 + tkn, &slot, &tile);
      pack_codes<BITS>(gbase, slot & 15, kv, sc, lane);
      if (lane == 0) a.meta[(tile * (size_t)a.pf + slot) * 2 + kv] = mw;
    }
    __syncwarp();  // sc is rewritten by the next token
  }
}

// Group mode (chunked appends at b <= 8 bits): one warp quantizes the 16
// tokens of one slot group (one KV head, K or V) with the same quantizer
// (four tokens at a time, 8 lanes each),
// keeps their codes in shared memory as bytes, token-major, and then writes
// the group part lane unit by lane unit: lane L builds unit L's 2b words
// from byte quads (Keys) or token pairs (Values) and stores them with 16-byte
// stores -- instead of every token scattering its codes with shuffles and
// 4- or 2-byte stores.  The group's 16 tokens are consecutive in the call
// and fill the group (the host cuts a chunk at 16-token boundaries).
constexpr int kGroupWarps = 4;
constexpr int kRowBytes = 144;  // 128 codes + pad: quad reads of lanes (g, t) hit 32 distinct banks
// Three-input min / max (one instruction on sm_100), same result as two
// nested two-input ones.
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// floor(y) for 0 <= y < 2^23 in the low bits of the result: y + 2^23 rounded
// down is exactly 2^23 + floor(y), since the spacing of floats in
// [2^23, 2^24) is 1.
__device__ __forceinline__ uint32_t floor_bits(float y) {
  return __float_as_uint(__fadd_rd(y, 8388608.0f));
}
template <int BITS>
__global__ void __launch_bounds__(kGroupWarps * 32) append_group_kernel(AppendArgs a) {
  static_assert(BITS <= 8, "16-bit codes take the per-token path");
  __shared__ __align__(16) uint8_t cs[kGroupWarps][kGroupTokens][kRowBytes];
  __shared__ uint32_t ms[kGroupWarps][kGroupTokens];
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const unsigned ngroups = (unsigned)a.cnt / kGroupTokens;
  const unsigned w = blockIdx.x * kGroupWarps + wib;
  if (w >= ngroups * (unsigned)a.kv_heads * 2u) return;  // warp-uniform
  const int b = blockIdx.y;
  const int kv = (int)(w & 1u);
  const unsigned rest = w >> 1;
  const int gi = (int)(rest / (unsigned)a.kv_heads);
  const int j = (int)(rest - (unsigned)gi * (unsigned)a.kv_heads);
  const size_t stream = (size_t)b * a.kv_heads + j;
  const int tk0 = gi * kGroupTokens;  // first token of the group within this launch
  constexpr unsigned qmax = (1u << BITS) - 1u;

  // ---- quantize the 16 tokens, four at a time: lane L takes token 4 step + L / 8
  // and its channels 16 (L % 8) .. + 15, so a token's min / max needs three
  // shuffle levels over its 8 lanes and one division serves 16 values ----
  const void* src = kv ? a.v : a.k;
  const int sub = lane & 7, tq = lane >> 3;
  const bool mig = kv == 0 && a.lam_inv;
  float li[16];
#pragma unroll
  for (int c = 0; c < 16; c++) li[c] = 1.0f;
  if (mig) {
#pragma unroll
    for (int c4 = 0; c4 < 4; c4++) {
      const float4 l4 = *reinterpret_cast<const float4*>(a.lam_inv + (size_t)j * kHeadDim + 16 * sub + 4 * c4);
      li[4 * c4] = l4.x; li[4 * c4 + 1] = l4.y; li[4 * c4 + 2] = l4.z; li[4 * c4 + 3] = l4.w;
    }
  }
  uint4 rawb[kGroupTokens / 4][2];  // bf16 inputs of every step, loaded before any is used
  if (a.dtype != 1) {
#pragma unroll
    for (int step = 0; step < kGroupTokens / 4; step++) {
      const size_t off = (((size_t)b * a.n_call + (size_t)(a.tok_off + tk0 + 4 * step + tq)) * a.kv_heads + j) *
                         kHeadDim + 16 * sub;
#pragma unroll
      for (int c8 = 0; c8 < 2; c8++)
        rawb[step][c8] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + off + 8 * c8);
    }
  }
#pragma unroll
  for (int step = 0; step < kGroupTokens / 4; step++) {
    const int tok = 4 * step + tq;
    const size_t in_off =
        (((size_t)b * a.n_call + (size_t)(a.tok_off + tk0 + tok)) * a.kv_heads + j) * kHeadDim + 16 * sub;
    float x[16];
    if (a.dtype == 1) {
#pragma unroll
      for (int c4 = 0; c4 < 4; c4++) {
        const float4 f4 = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + in_off + 4 * c4);
        x[4 * c4] = f4.x; x[4 * c4 + 1] = f4.y; x[4 * c4 + 2] = f4.z; x[4 * c4 + 3] = f4.w;
      }
    } else {
#pragma unroll
      for (int c8 = 0; c8 < 2; c8++) {
        const uint4 raw = rawb[step][c8];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int q = 0; q < 4; q++) {
          x[8 * c8 + 2 * q] = __uint_as_float(w[q] << 16);
          x[8 * c8 + 2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
      }
    }
    if (mig) {
#pragma unroll
      for (int c = 0; c < 16; c++) x[c] = __fmul_rn(x[c], li[c]);
    }
    // the quantizer of kvq_quant.cuh over the token's 8 lanes, codes kept in registers
    float mn = fminf(fmin3(fmin3(x[0], x[1], x[2]), fmin3(x[3], x[4], x[5]), fmin3(x[6], x[7], x[8])),
                     fmin3(fmin3(x[9], x[10], x[11]), fmin3(x[12], x[13], x[14]), x[15]));
    float mx = fmaxf(fmax3(fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmax3(x[6], x[7], x[8])),
                     fmax3(fmax3(x[9], x[10], x[11]), fmax3(x[12], x[13], x[14]), x[15]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const __half zh = __float2half_rd(mn);
    const float z = __half2float(zh);
    const __half rh = __float2half_ru(__fsub_rn(mx, z));
    const float r = __half2float(rh);
    uint32_t wq[4] = {0u, 0u, 0u, 0u};
    if (r != 0.0f) {
      const float inv = __fdiv_rn((float)qmax, r);
      // code = clamp(floor(y), 0, qmax), and for finite groups within
      // binary16 range the clamp never binds: y >= 1/2 as x >= Z, and
      // fl(x - Z) <= fl(max - Z) <= R, inv <= (qmax / R)(1 + 2^-24), so
      // y < qmax (1 + 2^-24)^3 + 1/2 < qmax + 1 for qmax < 2^16.  The code is
      // the low byte of floor_bits; four bytes go into a word by byte
      // permutes.  A group outside that contract (an infinite Value gives
      // R = inf, inv = 0 and inf * 0 = NaN; a minimum below -65504 gives
      // Z = -inf) can yield NaN, whose low byte is 0xff: the mask keeps every
      // byte inside its b-bit field, so such a group's codes, unspecified as
      // they are, never reach the fields of the tokens packed beside them.
      uint32_t fb[16];
#pragma unroll
      for (int c = 0; c < 16; c++) fb[c] = floor_bits(__fadd_rn(__fmul_rn(__fsub_rn(x[c], z), inv), 0.5f));
#pragma unroll
      for (int c4 = 0; c4 < 4; c4++)
        wq[c4] = __byte_perm(__byte_perm(fb[4 * c4], fb[4 * c4 + 1], 0x0040),
                             __byte_perm(fb[4 * c4 + 2], fb[4 * c4 + 3], 0x0040), 0x5410) &
                 (qmax * 0x01010101u);
    }
    *reinterpret_cast<uint4*>(&cs[wib][tok][16 * sub]) = make_uint4(wq[0], wq[1], wq[2], wq[3]);  // one byte per channel
    if (sub == 0) ms[wib][tok] = (uint32_t)__half_as_ushort(rh) | ((uint32_t)__half_as_ushort(zh) << 16);
  }
  __syncwarp();

  // ---- the group part, lane unit L = 4g + t ----
  const unsigned m = (unsigned)(a.n0 + tk0 - (long long)a.nt * a.h);  // the group's first token, this epoch
  const int tile = (int)(m / (unsigned)a.e);
  const int slot0 = a.h + (int)(m - (unsigned)tile * (unsigned)a.e);  // a multiple of 16
  const size_t tl = stream * a.nt + tile;
  uint8_t* gbase = a.codes + tl * kTileBytes + (size_t)(slot0 >> 4) * group_bytes(BITS) + (size_t)kv * part_bytes(BITS);
  const int g = lane >> 2, t = lane & 3;
  uint32_t wd[2 * BITS];
  if (kv == 0) {
    // word x b + jw holds quads p = jw (8/b) + k (field k) of token g + 8x:
    // channels 32 (p/2) + 16 (p%2) + 4t + i, member i in byte i
#pragma unroll
    for (int x = 0; x < 2; x++)
#pragma unroll
      for (int jw = 0; jw < BITS; jw++) {
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < 8 / BITS; k++) {
          const int p = jw * (8 / BITS) + k;
          word |= *reinterpret_cast<const uint32_t*>(&cs[wib][g + 8 * x][32 * (p >> 1) + 16 * (p & 1) + 4 * t])
                  << (BITS * k);
        }
        wd[x * BITS + jw] = word;
      }
  } else {
    // word u b + jw holds pairs p = jw (16/b) + k (field k): channel
    // 16 (p/2) + g + 8 (p%2) of tokens 2t + 8u (low half) and 2t + 8u + 1 (high half)
#pragma unroll
    for (int u = 0; u < 2; u++)
#pragma unroll
      for (int jw = 0; jw < BITS; jw++) {
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < 16 / BITS; k++) {
          const int p = jw * (16 / BITS) + k;
          const int ch = 16 * (p >> 1) + g + 8 * (p & 1);
          word |= ((uint32_t)cs[wib][2 * t + 8 * u][ch] | ((uint32_t)cs[wib][2 * t + 8 * u + 1][ch] << 16)) << (BITS * k);
        }
        wd[u * BITS + jw] = word;
      }
  }
  uint4* dst = reinterpret_cast<uint4*>(gbase + (size_t)lane * unit_bytes(BITS));
#pragma unroll
  for (int i = 0; i < BITS / 2; i++) dst[i] = make_uint4(wd[4 * i], wd[4 * i + 1], wd[4 * i + 2], wd[4 * i + 3]);
  if (lane < kGroupTokens) a.meta[(tl * a.pf + slot0 + lane) * 2 + kv] = ms[wib][lane];
}

// Per-channel Key groups (KIVI's axis): the staged block of 128 tokens of
// one stream enters the progressive cache at width BITS.  Keys: every staged
// INT16 Key is read back in fp32 as Z + code * (R / 65535) and each channel's
// 128 values go through the quantizer of kvq_quant.cuh; Values: each token's
// INT16 codes take the block's shift chain, R and Z kept (R rescaled by the
// direct shift).  Six CTAs of 256 threads per stream: two take the Keys of
// one half of the channels each (a half's codes fill whole words of the
// packed layout at every width, so the two never write the same word), four
// take the Values of 32 tokens each.  In a Key CTA thread (quarter, c) finds
// channel c's min / max over tokens 32 quarter .. +31 and the quarters
// combine them.
constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / 32;
constexpr int kMoveRoles = 6;  // 2 Key halves, 4 Value quarters
constexpr int kHalf = kHeadDim / 2;
struct MoveKeySmem {
  uint16_t kc[kKeyBlock][kHalf];       // [token][channel of the half]: INT16 codes, then the new codes
  float z[kKeyBlock], step[kKeyBlock];  // staged Keys: Z and R / 65535 of each token
  float mn[4][kHalf], mx[4][kHalf];
};
static_assert(kMoveWarps * 4 * (kHeadDim * 2 + 4) <= (int)sizeof(MoveKeySmem), "the Value rows fit the Key state");
template <int BITS>
__global__ void __launch_bounds__(kMoveThreads) block_move_kernel(BlockMoveArgs a) {
  // the Key roles' state; the Value roles keep per warp their tokens' codes
  // (and meta words) here instead
  __shared__ __align__(16) uint8_t sm_raw[sizeof(MoveKeySmem)];
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t stream = blockIdx.x / kMoveRoles;
  const int role = (int)(blockIdx.x % kMoveRoles);
  // From the call's input, four tokens per warp step: lane L takes token
  // 4 step + L / 8 of the warp's tokens and its channels 16 (L % 8) .. + 15,
  // and each token gets the INT16 quantization the append would stage (Keys
  // divided by lambda first; the steps of quantize_group, the min / max over
  // the token's 8 lanes in three shuffle levels).
  const int sub = lane & 7, tq = lane >> 3;
  const int bq = (int)(stream / (size_t)a.kv_heads), jq = (int)(stream % (size_t)a.kv_heads);
  auto in_ptr = [&](int t, int kv) {  // this lane's 16 values of token t
    const size_t off = (((size_t)bq * a.n_call + (size_t)(a.tok_off + t)) * a.kv_heads + jq) * kHeadDim + 16 * sub;
    return a.dtype == 1 ? static_cast<const void*>(static_cast<const float*>(kv ? a.v : a.k) + off)
                        : static_cast<const void*>(static_cast<const __nv_bfloat16*>(kv ? a.v : a.k) + off);
  };
  auto widen_bf16 = [](const uint4 (&r)[2], float (&x)[16]) {
#pragma unroll
    for (int c8 = 0; c8 < 2; c8++) {
      const uint32_t w[4] = {r[c8].x, r[c8].y, r[c8].z, r[c8].w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        x[8 * c8 + 2 * i] = __uint_as_float(w[i] << 16);
        x[8 * c8 + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  };
  auto load_f32 = [](const void* p, float (&x)[16]) {
#pragma unroll
    for (int c4 = 0; c4 < 4; c4++) {
      const float4 f4 = reinterpret_cast<const float4*>(p)[c4];
      x[4 * c4] = f4.x; x[4 * c4 + 1] = f4.y; x[4 * c4 + 2] = f4.z; x[4 * c4 + 3] = f4.w;
    }
  };
  auto quant16 = [&](float (&x)[16], int kv, uint16_t (&c)[16]) -> uint32_t {
    if (kv == 0 && a.lam_inv) {
      const float4* l4 = reinterpret_cast<const float4*>(a.lam_inv + (size_t)jq * kHeadDim + 16 * sub);
#pragma unroll
      for (int c4 = 0; c4 < 4; c4++) {
        const float4 li = l4[c4];
        x[4 * c4] = __fmul_rn(x[4 * c4], li.x); x[4 * c4 + 1] = __fmul_rn(x[4 * c4 + 1], li.y);
        x[4 * c4 + 2] = __fmul_rn(x[4 * c4 + 2], li.z); x[4 * c4 + 3] = __fmul_rn(x[4 * c4 + 3], li.w);
      }
    }
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < 16; i++) {
      mn = fminf(mn, x[i]);
      mx = fmaxf(mx, x[i]);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const __half zh = __float2half_rd(mn);
    const float z = __half2float(zh);
    const __half rh = __float2half_ru(__fsub_rn(mx, z));
    const float r = __half2float(rh);
    const float inv = r == 0.0f ? 0.0f : __fdiv_rn(65535.0f, r);
#pragma unroll
    for (int i = 0; i < 16; i++)
      c[i] = r == 0.0f ? (uint16_t)0
                       : (uint16_t)min(__float2uint_rd(__fadd_rn(__fmul_rn(__fsub_rn(x[i], z), inv), 0.5f)), 65535u);
    return (uint32_t)__half_as_ushort(rh) | ((uint32_t)__half_as_ushort(zh) << 16);
  };
  constexpr int P16 = slots_per_tile(16);
  auto staged = [&](int t, int kv) {  // group part holding staged token t
    return a.wcodes + (stream * kWindowTiles + t / P16) * (size_t)kTileBytes +
           (size_t)((t % P16) >> 4) * group_bytes(16) + (size_t)kv * part_bytes(16);
  };
  auto staged_meta = [&](int t, int kv) {
    return ((stream * kWindowTiles + t / P16) * (size_t)P16 + t % P16) * 2 + kv;
  };
  if (role >= 2) {  // ---- Values of tokens 32 q .. 32 q + 31 ----
    const int q = role - 2;
    if (a.from_input) {  // warp w: tokens 32 q + 4 w .. + 3, one step
      uint16_t (*rows)[kHeadDim] = reinterpret_cast<uint16_t (*)[kHeadDim]>(sm_raw) + 4 * warp;  // [4][128]
      uint32_t* wm = reinterpret_cast<uint32_t*>(sm_raw + kMoveWarps * 4 * kHeadDim * 2) + 4 * warp;
      const int t0 = 32 * q + 4 * warp;
      float x[16];
      if (a.dtype == 1) {
        load_f32(in_ptr(t0 + tq, 1), x);
      } else {
        const uint4* p = reinterpret_cast<const uint4*>(in_ptr(t0 + tq, 1));
        const uint4 r[2] = {p[0], p[1]};
        widen_bf16(r, x);
      }
      uint16_t c[16];
      const uint32_t mw = quant16(x, 1, c);
#pragma unroll
      for (int i = 0; i < 16; i++) rows[tq][16 * sub + i] = (uint16_t)shift_chain<BITS>(c[i], a.direct);
      if (sub == 0) wm[tq] = mw;
      __syncwarp();
#pragma unroll 1
      for (int r = 0; r < 4; r++) {
        const int t = t0 + r, gi = t >> 4, slot = a.g_slot[gi] + (t & 15);
        const size_t tile = stream * a.nt + a.g_tile[gi];
        uint8_t* gbase = a.codes + tile * kTileBytes + (size_t)(slot >> 4) * group_bytes(BITS);
        pack_codes<BITS>(gbase + part_bytes(BITS), slot & 15, 1, rows[r], lane);
        if (lane == 0)
          a.meta[(tile * a.pf + slot) * 2 + 1] =
              (uint32_t)range_chain<BITS>((uint16_t)(wm[r] & 0xffffu), a.direct) | (wm[r] & 0xffff0000u);
      }
      return;
    }
    uint16_t* sc = reinterpret_cast<uint16_t*>(sm_raw) + warp * kHeadDim;
    for (int t = 32 * q + warp; t < 32 * q + 32; t += kMoveWarps) {
      const int gi = t >> 4, slot = a.g_slot[gi] + (t & 15);
      const size_t tile = stream * a.nt + a.g_tile[gi];
      uint8_t* gbase = a.codes + tile * kTileBytes + (size_t)(slot >> 4) * group_bytes(BITS);
      unpack_codes16(staged(t, 1), t & 15, 1, sc, lane);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; i++) sc[4 * lane + i] = (uint16_t)shift_chain<BITS>(sc[4 * lane + i], a.direct);
      __syncwarp();
      pack_codes<BITS>(gbase + part_bytes(BITS), slot & 15, 1, sc, lane);
      if (lane == 0) {
        const uint32_t old = a.wmeta[staged_meta(t, 1)];
        a.meta[(tile * a.pf + slot) * 2 + 1] =
            (uint32_t)range_chain<BITS>((uint16_t)(old & 0xffffu), a.direct) | (old & 0xffff0000u);
      }
      __syncwarp();  // sc is rewritten by the next token
    }
    return;
  }
  // ---- Keys of channels 64 h .. 64 h + 63 ----
  MoveKeySmem& sh = *reinterpret_cast<MoveKeySmem*>(sm_raw);
  const int h = role;
  // staged INT16 Key codes of the half: channel ch of token t is member i = ch % 4
  // of quad p = 2 (ch / 32) + (ch / 16) % 2 in unit 4 (t % 8) + (ch / 4) % 4, word
  // 16 x + 2 p + i / 2 (x = (t % 16) / 8), half-word i % 2 (the 16-bit layout)
  if (a.from_input) {  // warp w: tokens 16 w .. 16 w + 15, four steps, every load in flight first
    const int t0 = 16 * warp;
    uint4 raw[4][2];
    if (a.dtype != 1) {
#pragma unroll
      for (int st = 0; st < 4; st++) {
        const uint4* p = reinterpret_cast<const uint4*>(in_ptr(t0 + 4 * st + tq, 0));
        raw[st][0] = p[0];
        raw[st][1] = p[1];
      }
    }
#pragma unroll
    for (int st = 0; st < 4; st++) {
      const int t = t0 + 4 * st + tq;
      float x[16];
      if (a.dtype == 1) load_f32(in_ptr(t, 0), x);
      else widen_bf16(raw[st], x);
      uint16_t c[16];
      const uint32_t w = quant16(x, 0, c);
      if ((sub >> 2) == h) {  // this lane's channels lie in the half
        uint4* d = reinterpret_cast<uint4*>(&sh.kc[t][16 * (sub & 3)]);
        d[0] = make_uint4(c[0] | ((uint32_t)c[1] << 16), c[2] | ((uint32_t)c[3] << 16), c[4] | ((uint32_t)c[5] << 16),
                          c[6] | ((uint32_t)c[7] << 16));
        d[1] = make_uint4(c[8] | ((uint32_t)c[9] << 16), c[10] | ((uint32_t)c[11] << 16),
                          c[12] | ((uint32_t)c[13] << 16), c[14] | ((uint32_t)c[15] << 16));
      }
      if (sub == 0) {
        sh.z[t] = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
        sh.step[t] = __fdiv_rn(__half2float(__ushort_as_half((unsigned short)(w & 0xffffu))), 65535.0f);
      }
    }
  } else {
    for (int e = threadIdx.x; e < kKeyBlock * kHalf; e += kMoveThreads) {
      const int t = e / kHalf, cc = e % kHalf, ch = kHalf * h + cc;
      const int tok = t & 15, g = tok & 7, x = tok >> 3;
      const int p = 2 * (ch >> 5) + ((ch >> 4) & 1), tt = (ch >> 2) & 3, mi = ch & 3;
      const uint16_t* u16 = reinterpret_cast<const uint16_t*>(staged(t, 0));
      sh.kc[t][cc] = u16[(4 * g + tt) * (unit_bytes(16) / 2) + 2 * (x * 16 + 2 * p + (mi >> 1)) + (mi & 1)];
    }
    if (threadIdx.x < kKeyBlock) {
      const int t = threadIdx.x;
      const uint32_t w = a.wmeta[staged_meta(t, 0)];
      sh.z[t] = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
      sh.step[t] = __fdiv_rn(__half2float(__ushort_as_half((unsigned short)(w & 0xffffu))), 65535.0f);
    }
  }
  __syncthreads();
  {
    const int cc = threadIdx.x & (kHalf - 1), qt = threadIdx.x / kHalf;  // channel of the half, token quarter
    const int t0 = 32 * qt;
    auto value = [&](int t) { return __fadd_rn(sh.z[t], __fmul_rn((float)sh.kc[t][cc], sh.step[t])); };
    float mn = value(t0), mx = mn;
    for (int t = t0 + 1; t < t0 + 32; t++) {
      const float x = value(t);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    sh.mn[qt][cc] = mn;
    sh.mx[qt][cc] = mx;
    __syncthreads();
    mn = fminf(fminf(sh.mn[0][cc], sh.mn[1][cc]), fminf(sh.mn[2][cc], sh.mn[3][cc]));
    mx = fmaxf(fmaxf(sh.mx[0][cc], sh.mx[1][cc]), fmaxf(sh.mx[2][cc], sh.mx[3][cc]));
    const __half zh = __float2half_rd(mn);
    const float z = __half2float(zh);
    const __half rh = __float2half_ru(__fsub_rn(mx, z));
    const float r = __half2float(rh);
    constexpr unsigned qmax = BITS == 16 ? 65535u : (1u << BITS) - 1u;
    const float inv = r == 0.0f ? 0.0f : __fdiv_rn((float)qmax, r);
    for (int t = t0; t < t0 + 32; t++) {
      uint16_t q = 0;
      if (r != 0.0f) {
        const float y = __fadd_rn(__fmul_rn(__fsub_rn(value(t), z), inv), 0.5f);
        q = (uint16_t)min(__float2uint_rd(y), qmax);
      }
      sh.kc[t][cc] = q;  // only this thread reads or writes this token's channel cc
    }
    if (qt == 0)
      a.kmc[(stream * a.blocks_max + a.blk) * kHeadDim + kHalf * h + cc] =
          (uint32_t)__half_as_ushort(rh) | ((uint32_t)__half_as_ushort(zh) << 16);
  }
  __syncthreads();
  // the half's Key words of every token: unit 4 g + t4 of the token's group,
  // words x b + jw for jw in [h b / 2, (h + 1) b / 2) (b <= 8; at 16 bits the
  // half's quads 4h .. 4h + 3 fill words 8h .. 8h + 7); word x b + jw holds quads
  // p = jw (8/b) + k at field k, member i (channel 32 (p/2) + 16 (p%2) + 4 t4 + i) in byte i
  constexpr int kWords = BITS == 16 ? 8 : BITS / 2;  // per (token, unit) and half
  for (int e = threadIdx.x; e < kKeyBlock * 4 * kWords; e += kMoveThreads) {
    const int t = e / (4 * kWords), t4 = (e / kWords) % 4, wl = e % kWords;
    const int gi = t >> 4, slot = a.g_slot[gi] + (t & 15);
    const size_t tile = stream * a.nt + a.g_tile[gi];
    const int tok = slot & 15, g = tok & 7, x = tok >> 3;
    uint32_t* unit = reinterpret_cast<uint32_t*>(a.codes + tile * kTileBytes + (size_t)(slot >> 4) * group_bytes(BITS) +
                                                 (size_t)(4 * g + t4) * unit_bytes(BITS));
    uint32_t word = 0;
    int widx;
    if constexpr (BITS == 16) {
      const int wi = 8 * h + wl, p = wi >> 1, mi0 = 2 * (wi & 1);  // members mi0, mi0 + 1 as half-words
      const int cb = 32 * (p >> 1) + 16 * (p & 1) + 4 * t4 - kHalf * h;
      word = (uint32_t)sh.kc[t][cb + mi0] | ((uint32_t)sh.kc[t][cb + mi0 + 1] << 16);
      widx = x * 16 + wi;
    } else {
      const int jw = h * (BITS / 2) + wl;
#pragma unroll
      for (int k = 0; k < 8 / BITS; k++) {
        const int p = jw * (8 / BITS) + k;
        const int cb = 32 * (p >> 1) + 16 * (p & 1) + 4 * t4 - kHalf * h;
#pragma unroll
        for (int i = 0; i < 4; i++) word |= (uint32_t)sh.kc[t][cb + i] << (8 * i + BITS * k);
      }
      widx = x * BITS + jw;
    }
    unit[widx] = word;
  }
}

}  // namespace

cudaError_t launch_block_move(const BlockMoveArgs& a, int n_streams, cudaStream_t s) {
  if (n_streams <= 0) return cudaSuccess;
  if ((long long)n_streams * kMoveRoles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)n_streams * kMoveRoles), block(kMoveThreads);
  switch (a.bits) {
    case 16: return launch_pdl(block_move_kernel<16>, grid, block, 0, s, a);
    case 8: return launch_pdl(block_move_kernel<8>, grid, block, 0, s, a);
    case 4: return launch_pdl(block_move_kernel<4>, grid, block, 0, s, a);
    case 2: return launch_pdl(block_move_kernel<2>, grid, block, 0, s, a);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
  // A chunk of a per-token cache at b <= 8 bits: its whole 16-token groups
  // go through the group mode, the tokens before the first and after the
  // last whole group through the per-token path (three launches at most,
  // disjoint slots).
  if (!a.window && a.bits <= 8 && a.cnt >= kGroupTokens) {
    const int head = std::min(a.cnt, (int)((kGroupTokens - a.n0 % kGroupTokens) % kGroupTokens));
    const int body = (a.cnt - head) / kGroupTokens * kGroupTokens;
    if (body > 0) {
      AppendArgs p = a;
      p.cnt = head;
      if (head > 0)
        if (cudaError_t e = launch_append(p, s)) return e;
      p = a;
      p.tok_off = a.tok_off + head;
      p.n0 = a.n0 + head;
      p.cnt = body;
      const long long gw = (long long)(body / kGroupTokens) * a.kv_heads * 2;  // warps per sequence
      if (gw >= (1ll << 31) || a.batch > 65535) return cudaErrorInvalidValue;
      const dim3 grid((unsigned)((gw + kGroupWarps - 1) / kGroupWarps), (unsigned)a.batch), block(kGroupWarps * 32);
      cudaError_t e = cudaSuccess;
      switch (a.bits) {
        case 8: e = launch_pdl(append_group_kernel<8>, grid, block, 0, s, p); break;
        case 4: e = launch_pdl(append_group_kernel<4>, grid, block, 0, s, p); break;
        case 2: e = launch_pdl(append_group_kernel<2>, grid, block, 0, s, p); break;
        default: return cudaErrorInvalidValue;
      }
      if (e != cudaSuccess) return e;
      p = a;
      p.tok_off = a.tok_off + head + body;
      p.n0 = a.n0 + head + body;
      p.cnt = a.cnt - head - body;
      return p.cnt > 0 ? launch_append(p, s) : cudaSuccess;
    }
  }
  const long long warps = ((long long)a.cnt + kTokensPerWarp - 1) / kTokensPerWarp * a.kv_heads * 2;  // per sequence
  if (warps <= 0 || a.batch <= 0) return cudaSuccess;
  if (warps >= (1ll << 31) || a.batch > 65535) return cudaErrorInvalidValue;
  const long long blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const dim3 grid((unsigned)blocks, (unsigned)a.batch), block(kWarpsPerBlock * 32);
  switch (a.bits) {
    case 16: return launch_pdl(append_kernel<16>, grid, block, 0, s, a);
    case 8: return launch_pdl(append_kernel<8>, grid, block, 0, s, a);
    case 4: return launch_pdl(append_kernel<4>, grid, block, 0, s, a);
    case 2: return launch_pdl(append_kernel<2>, grid, block, 0, s, a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
