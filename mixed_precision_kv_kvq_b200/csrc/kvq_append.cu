// kvq_append.cu -- quantize-on-append (PM-KVQ note, key design 1: each new
// token is stored at the block's current width; key design 3: Keys are
// divided by the per-channel migration factor lambda first; training
// strategy: asymmetric groups of 128).
//
// One warp quantizes the groups (128 channels of one KV head, K or V) of a
// few consecutive tokens.  Per group, with every step a single IEEE fp32
// round-to-nearest
// operation (no contraction):
//   x_c = k_c * lambda_inv_c            (K only)
//   Z   = binary16 round-down(min x)    R = binary16 round-up(max x - Z)
//   q_c = clamp(floor((x_c - Z) * ((2^b - 1) / R) + 1/2), 0, 2^b - 1)
// (R = 0: all codes 0), then scatters the codes into the lane units of the
// group's K or V part (see kvq_internal.cuh) and writes (R, Z) to the slot's
// K or V meta word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kTokensPerWarp = 4;

__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Scatter one token's 128 codes (sc, channel order) into its group's K or V
// part at gbase, as slot `tok` (0..15) of the group, at `bits` bits.
//
// At b <= 8 bits the token's part holds 16 b bytes and lane L builds bytes
// L, L + 32, ...: each byte packs 8/b codes.  The four bytes of a 32-bit word
// (Keys) or the two of a 16-bit half (Values) sit in neighbouring lanes and
// are joined with shuffles; one lane stores the word or half.
//   K: token tok -> g = tok % 8, x = tok / 8.  Byte B -> unit 4g + t, word
//      x*b + jw, member i (t = B / 4b, jw = (B / 4) % b, i = B % 4); it holds
//      member i of quads p = jw*(8/b) + k (k = 0 .. 8/b-1) at bits b*k, quad
//      p = 2s + r being positions 32s + 16r + 4t + i, mapped to channels by
//      the block's Key channel order.
//   V: token tok -> t = (tok % 8) / 2, member mb = tok % 2, u = tok / 8.  Byte
//      B -> unit 4g + t, word u*b + jw, half mb, byte hb of the half
//      (g = B / 2b, jw = (B / 2) % b, hb = B % 2); it holds pairs p = jw*(16/b)
//      + hb*(8/b) + k of channel 16(p/2) + g + 8(p%2) at bits b*k.
template <int bits>
__device__ __forceinline__ void pack_codes(uint8_t* gbase, int tok, int kv, const uint16_t* sc, const uint8_t* pm,
                                           int lane) {
  if constexpr (bits == 16) {  // two codes per 32-bit word
    if (kv == 0) {
      const int g = tok & 7, xs = tok >> 3;
      for (int wi = lane; wi < 64; wi += 32) {
        const int t = wi >> 4, jw = wi & 15;
        const int p = jw >> 1;
        const int pos = 32 * (p >> 1) + 16 * (p & 1) + 4 * t + 2 * (jw & 1);
        const uint32_t word = (uint32_t)sc[pm ? pm[pos] : pos] | ((uint32_t)sc[pm ? pm[pos + 1] : pos + 1] << 16);
        reinterpret_cast<uint32_t*>(gbase + (4 * g + t) * unit_bytes(16))[xs * 16 + jw] = word;
      }
    } else {
      const int t = (tok & 7) >> 1, mb = tok & 1, u = tok >> 3;
      for (int hw = lane; hw < 128; hw += 32) {
        const int g = hw >> 4, jw = hw & 15;
        const int ch = 16 * (jw >> 1) + g + 8 * (jw & 1);
        reinterpret_cast<uint16_t*>(gbase + (4 * g + t) * unit_bytes(16))[2 * (u * 16 + jw) + mb] = sc[ch];
      }
    }
  } else {
  constexpr int per_byte = 8 / bits;
#pragma unroll
  for (int B = lane; B < 16 * bits; B += 32) {  // warp-uniform: 16 b is a multiple of 32 for b = 2, 4, 8
    uint32_t byte = 0;
    if (kv == 0) {
      const int t = B / (4 * bits), jw = (B >> 2) % bits, i = B & 3;
#pragma unroll
      for (int k = 0; k < per_byte; k++) {
        const int p = jw * per_byte + k;
        const int pos = 32 * (p >> 1) + 16 * (p & 1) + 4 * t + i;
        byte |= (uint32_t)sc[pm ? pm[pos] : pos] << (bits * k);
      }
      // join the 4 bytes of the word (lanes 4w .. 4w+3)
      uint32_t word = byte << (8 * i);
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      if (i == 0) {
        const int g = tok & 7, xs = tok >> 3;
        reinterpret_cast<uint32_t*>(gbase + (4 * g + t) * unit_bytes(bits))[xs * bits + jw] = word;
      }
    } else {
      const int g = B / (2 * bits), jw = (B >> 1) % bits, hb = B & 1;
      constexpr int ppw = 16 / bits;
#pragma unroll
      for (int k = 0; k < per_byte; k++) {
        const int p = jw * ppw + hb * per_byte + k;
        byte |= (uint32_t)sc[16 * (p >> 1) + g + 8 * (p & 1)] << (bits * k);
      }
      uint32_t half = byte << (8 * hb);
      half |= __shfl_xor_sync(0xffffffffu, half, 1);
      if (hb == 0) {
        const int t = (tok & 7) >> 1, mb = tok & 1, u = tok >> 3;
        reinterpret_cast<uint16_t*>(gbase + (4 * g + t) * unit_bytes(bits))[2 * (u * bits + jw) + mb] = (uint16_t)half;
      }
    }
  }
  }
}

// Read one token's 16-bit codes back from its group part (the inverse of
// pack_codes at 16 bits) into sc, channel order.
__device__ __forceinline__ void unpack_codes16(const uint8_t* gbase, int tok, int kv, uint16_t* sc,
                                               const uint8_t* pm, int lane) {
  const uint16_t* u16 = reinterpret_cast<const uint16_t*>(gbase);
  constexpr int kUnitHalves = 8 * 16 / 2;  // 128-byte units
  if (kv == 0) {
    const int g = tok & 7, xs = tok >> 3;
    for (int pos = lane; pos < kHeadDim; pos += 32) {
      const int p = 2 * (pos >> 5) + ((pos >> 4) & 1), t = (pos >> 2) & 3, i = pos & 3;
      const int word = xs * 16 + 2 * p + (i >> 1);
      sc[pm ? pm[pos] : pos] = u16[(4 * g + t) * kUnitHalves + 2 * word + (i & 1)];
    }
  } else {
    const int t = (tok & 7) >> 1, mb = tok & 1, u = tok >> 3;
    for (int ch = lane; ch < kHeadDim; ch += 32) {
      const int s = ch >> 4, r = (ch >> 3) & 1, g = ch & 7;
      const int word = u * 16 + 2 * s + r;
      sc[ch] = u16[(4 * g + t) * kUnitHalves + 2 * word + mb];
    }
  }
}

// One INT16 code brought to `bits` by the block's shift, one level at a time.
template <int bits>
__device__ __forceinline__ uint32_t shift_chain(uint32_t x, bool direct) {
#pragma unroll
  for (int b = 8; b >= bits; b >>= 1) {
    if (direct) {
      x >>= b;
    } else {
      const uint32_t mul = (1u << (2 * b)) - (1u << b) + 1u;
      x = (x + (1u << (b - 1))) * mul >> (3 * b);  // max (65535 + 128) * 65281 < 2^32
    }
  }
  return x;
}
// The range of a group under the same chain (rescaled by the direct shift only).
template <int bits>
__device__ __forceinline__ uint16_t range_chain(uint16_t rbits, bool direct) {
  if (direct) {
#pragma unroll
    for (int b = 8; b >= bits; b >>= 1) {
      const float r = __half2float(__ushort_as_half(rbits));
      const float q = __fdiv_rn(__fmul_rn(r, (float)(1u << b)), (float)((1u << b) + 1u));
      rbits = __half_as_ushort(__float2half_rn(q));
    }
  }
  return rbits;
}

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
  const uint8_t* pm = (kv == 0 && a.perm) ? a.perm + (size_t)j * kHeadDim : nullptr;
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
      const int rs = t == 0 ? 0 : 1 + (int)((unsigned long long)(t - 1) & (kWindowTokens - 1));
      const int wtile = rs / slots_per_tile(16), wslot = rs % slots_per_tile(16);
      wtok = wslot & 15;
      wg = a.wcodes + (stream * kWindowTiles + wtile) * (size_t)kTileBytes + (size_t)(wslot >> 4) * group_bytes(16) +
           (size_t)kv * part_bytes(16);
      wmi = ((stream * kWindowTiles + wtile) * (size_t)slots_per_tile(16) + wslot) * 2 + kv;
      if (t >= kWindowTokens + 1) {
        // token t - 128 leaves the window: its INT16 codes go to the progressive
        // cache at the current width (index t - 129) by the block's shift chain
        unpack_codes16(wg, wtok, kv, sc, pm, lane);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; i++) sc[4 * lane + i] = (uint16_t)shift_chain<BITS>(sc[4 * lane + i], a.direct);
        const uint32_t old = a.wmeta[wmi];
        __syncwarp();
        int slot;
        size_t tile;
        uint8_t* gbase = main_group(t - (kWindowTokens + 1), &slot, &tile);
        pack_codes<BITS>(gbase, slot & 15, kv, sc, pm, lane);
        if (lane == 0) {
          const uint32_t mw = (uint32_t)range_chain<BITS>((uint16_t)(old & 0xffffu), a.direct) | (old & 0xffff0000u);
          a.meta[(tile * (size_t)a.pf + slot) * 2 + kv] = mw;
        }
        __syncwarp();  // sc is reused below
      }
    }

    // ---- group meta ----
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mn = warp_min(mn);
    mx = warp_max(mx);
    const __half zh = __float2half_rd(mn);
    const float z = __half2float(zh);
    const __half rh = __float2half_ru(__fsub_rn(mx, z));
    const float r = __half2float(rh);
    const unsigned qmaxu = a.window ? 65535u : (1u << BITS) - 1u;  // window tokens are held at INT16
    if (r == 0.0f) {
#pragma unroll
      for (int i = 0; i < 4; i++) sc[4 * lane + i] = 0;
    } else {
      const float inv = __fdiv_rn((float)qmaxu, r);
#pragma unroll
      for (int i = 0; i < 4; i++) {
        // clamp(floor(y), 0, qmax) as an integer: float -> uint conversion
        // rounding down saturates negatives to 0; same value as the float form
        const float y = __fadd_rn(__fmul_rn(__fsub_rn(x[i], z), inv), 0.5f);
        sc[4 * lane + i] = (uint16_t)min(__float2uint_rd(y), qmaxu);
      }
    }
    __syncwarp();
    const uint32_t mw = (uint32_t)__half_as_ushort(rh) | ((uint32_t)__half_as_ushort(zh) << 16);

    if (a.window) {
      pack_codes<16>(wg, wtok, kv, sc, pm, lane);
      if (lane == 0) a.wmeta[wmi] = mw;
    } else {
      int slot;
      size_t tile;
      uint8_t* gbase = main_group(a.n0 + tkn, &slot, &tile);
      pack_codes<BITS>(gbase, slot & 15, kv, sc, pm, lane);
      if (lane == 0) a.meta[(tile * (size_t)a.pf + slot) * 2 + kv] = mw;
    }
    __syncwarp();  // sc is rewritten by the next token
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
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
