// kvq_quant.cuh -- one group's quantizer and the packing of a token's codes
// into the lane-unit layout (kvq_internal.cuh); used by the append kernel and
// by the decode kernel's fused single-token append.
//
// Quantizer (PM-KVQ note, key design 1; training strategy: asymmetric groups
// of 128), every step a single IEEE fp32 round-to-nearest operation:
//   Z   = binary16 round-down(min x)    R = binary16 round-up(max x - Z)
//   q_c = clamp(floor((x_c - Z) * ((2^b - 1) / R) + 1/2), 0, 2^b - 1)
// (R = 0: all codes 0).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

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
//      p = 2s + r being channels 32s + 16r + 4t + i.
//   V: token tok -> t = (tok % 8) / 2, member mb = tok % 2, u = tok / 8.  Byte
//      B -> unit 4g + t, word u*b + jw, half mb, byte hb of the half
//      (g = B / 2b, jw = (B / 2) % b, hb = B % 2); it holds pairs p = jw*(16/b)
//      + hb*(8/b) + k of channel 16(p/2) + g + 8(p%2) at bits b*k.
template <int bits>
__device__ __forceinline__ void pack_codes(uint8_t* gbase, int tok, int kv, const uint16_t* sc, int lane) {
  if constexpr (bits == 16) {  // two codes per 32-bit word
    if (kv == 0) {
      const int g = tok & 7, xs = tok >> 3;
      for (int wi = lane; wi < 64; wi += 32) {
        const int t = wi >> 4, jw = wi & 15;
        const int p = jw >> 1;
        const int pos = 32 * (p >> 1) + 16 * (p & 1) + 4 * t + 2 * (jw & 1);
        const uint32_t word = (uint32_t)sc[pos] | ((uint32_t)sc[pos + 1] << 16);
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
        byte |= (uint32_t)sc[pos] << (bits * k);
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
__device__ __forceinline__ void unpack_codes16(const uint8_t* gbase, int tok, int kv, uint16_t* sc, int lane) {
  const uint16_t* u16 = reinterpret_cast<const uint16_t*>(gbase);
  constexpr int kUnitHalves = 8 * 16 / 2;  // 128-byte units
  if (kv == 0) {
    const int g = tok & 7, xs = tok >> 3;
    for (int pos = lane; pos < kHeadDim; pos += 32) {
      const int p = 2 * (pos >> 5) + ((pos >> 4) & 1), t = (pos >> 2) & 3, i = pos & 3;
      const int word = xs * 16 + 2 * p + (i >> 1);
      sc[pos] = u16[(4 * g + t) * kUnitHalves + 2 * word + (i & 1)];
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

// Quantize one group: this lane's four values x (channels 4 lane .. 4 lane + 3,
// Keys already divided by lambda) with codes in [0, qmax] into sc (channel
// order).  Returns the meta word: binary16 R (low half), Z (high half).
__device__ __forceinline__ uint32_t quantize_group(const float (&x)[4], unsigned qmaxu, uint16_t* sc, int lane) {
  float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
  float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  mn = warp_min(mn);
  mx = warp_max(mx);
  const __half zh = __float2half_rd(mn);
  const float z = __half2float(zh);
  const __half rh = __float2half_ru(__fsub_rn(mx, z));
  const float r = __half2float(rh);
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
  return (uint32_t)__half_as_ushort(rh) | ((uint32_t)__half_as_ushort(zh) << 16);
}

}  // namespace
}  // namespace kvq
