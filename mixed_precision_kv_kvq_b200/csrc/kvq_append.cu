// kvq_append.cu -- quantize-on-append (PM-KVQ note, key design 1: each new
// token is stored at the block's current width; key design 3: Keys are
// divided by the per-channel migration factor lambda first; training
// strategy: asymmetric groups of 128).
//
// One warp quantizes one group = one token's 128 channels of one KV head, K
// or V.  Per group, with every step a single IEEE fp32 round-to-nearest
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
__device__ __forceinline__ void pack_codes(uint8_t* gbase, int bits, int tok, int kv, const uint16_t* sc,
                                           const uint8_t* pm, int lane) {
  if (kv == 0) {
    // Token tok: g = tok % 8, x = tok / 8.  Lane units 4g + t (t = 0..3) each
    // get `bits` words of this token, unit words x*bits + jw, holding its
    // quads Q = 8x + p, p = 2s + r: positions 32s + 16r + 4t + i (member i
    // in byte i).  Positions map to channels through the block's Key
    // channel order.
    const int g = tok & 7, xs = tok >> 3;
    for (int wi = lane; wi < 4 * bits; wi += 32) {
      const int t = wi / bits, jw = wi - t * bits;
      uint32_t word = 0;
      if (bits == 16) {  // half a quad: members 2(jw%2), 2(jw%2)+1 of quad p = jw/2
        const int p = jw >> 1;
        const int pos = 32 * (p >> 1) + 16 * (p & 1) + 4 * t + 2 * (jw & 1);
        word = (uint32_t)sc[pm ? pm[pos] : pos] | ((uint32_t)sc[pm ? pm[pos + 1] : pos + 1] << 16);
      } else {
        const int qpw = 8 / bits;  // quads per word
        for (int kk = 0; kk < qpw; kk++) {
          const int p = jw * qpw + kk;
          const int pos0 = 32 * (p >> 1) + 16 * (p & 1) + 4 * t;
#pragma unroll
          for (int i = 0; i < 4; i++) {
            const int c = pm ? pm[pos0 + i] : pos0 + i;
            word |= (uint32_t)sc[c] << (8 * i + bits * kk);
          }
        }
      }
      uint32_t* dst = reinterpret_cast<uint32_t*>(gbase + (4 * g + t) * unit_bytes(bits)) + xs * bits + jw;
      *dst = word;
    }
  } else {
    // Token tok: t = (tok % 8) / 2, member mb = tok % 2, pair set u = tok / 8.
    // Units 4g + t (g = 0..7): word u*bits + jw, half mb, pairs p = 2s + rr of
    // channel 16s + g + 8rr.
    const int t = (tok & 7) >> 1, mb = tok & 1, u = tok >> 3;
    const int ppw = 16 / bits;  // pairs per 32-bit word (per 16-bit half)
    for (int hw = lane; hw < 8 * bits; hw += 32) {
      const int g = hw / bits, jw = hw - g * bits;
      uint32_t half = 0;
      for (int kk = 0; kk < ppw; kk++) {
        const int p = jw * ppw + kk;
        const int ch = 16 * (p >> 1) + g + 8 * (p & 1);
        half |= (uint32_t)sc[ch] << (bits * kk);
      }
      uint16_t* dst = reinterpret_cast<uint16_t*>(gbase + (4 * g + t) * unit_bytes(bits)) +
                      2 * (u * bits + jw) + mb;
      *dst = (uint16_t)half;
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
__device__ __forceinline__ uint32_t shift_chain(uint32_t x, int bits, bool direct) {
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
__device__ __forceinline__ uint16_t range_chain(uint16_t rbits, int bits, bool direct) {
  if (direct) {
    for (int b = 8; b >= bits; b >>= 1) {
      const float r = __half2float(__ushort_as_half(rbits));
      const float q = __fdiv_rn(__fmul_rn(r, (float)(1u << b)), (float)((1u << b) + 1u));
      rbits = __half_as_ushort(__float2half_rn(q));
    }
  }
  return rbits;
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32) append_kernel(AppendArgs a) {
  __shared__ uint16_t codes_sh[kWarpsPerBlock][kHeadDim];
  pdl_wait();  // k/v and the cache may come from earlier kernels in the stream
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const long long w = (long long)blockIdx.x * kWarpsPerBlock + wib;
  const long long total = (long long)a.batch * a.cnt * a.kv_heads * 2;
  if (w >= total) return;  // warp-uniform

  const int kv = (int)(w & 1);
  long long rest = w >> 1;
  const int j = (int)(rest % a.kv_heads);
  rest /= a.kv_heads;
  const int tkn = (int)(rest % a.cnt);
  const int b = (int)(rest / a.cnt);
  const size_t stream = (size_t)b * a.kv_heads + j;
  const uint8_t* pm = (kv == 0 && a.perm) ? a.perm + (size_t)j * kHeadDim : nullptr;
  uint16_t* sc = codes_sh[wib];

  // progressive-cache slot of index li at the block's current width
  auto main_group = [&](long long li, int* slot_out, size_t* tile_out) {
    const long long m = li - (long long)a.nt * a.h;
    const int tile = (int)(m / a.e);
    const int slot = a.h + (int)(m - (long long)tile * a.e);
    *slot_out = slot;
    *tile_out = stream * a.nt + tile;
    return a.codes + *tile_out * (size_t)kTileBytes + (size_t)(slot >> 4) * group_bytes(a.bits) +
           (size_t)kv * part_bytes(a.bits);
  };

  // ---- sink + window: the slot token t uses is the one its leaving token frees ----
  uint8_t* wg = nullptr;
  size_t wmi = 0;
  int wtok = 0;
  if (a.window) {
    const long long t = a.t0 + tkn;
    const int rs = t == 0 ? 0 : 1 + (int)((t - 1) % kWindowTokens);
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
      for (int i = 0; i < 4; i++) sc[4 * lane + i] = (uint16_t)shift_chain(sc[4 * lane + i], a.bits, a.direct);
      const uint32_t old = a.wmeta[wmi];
      __syncwarp();
      int slot;
      size_t tile;
      uint8_t* gbase = main_group(t - (kWindowTokens + 1), &slot, &tile);
      pack_codes(gbase, a.bits, slot & 15, kv, sc, pm, lane);
      if (lane == 0) {
        const uint32_t mw = (uint32_t)range_chain((uint16_t)(old & 0xffffu), a.bits, a.direct) | (old & 0xffff0000u);
        a.meta[(tile * (size_t)a.pf + slot) * 2 + kv] = mw;
      }
      __syncwarp();  // sc is reused below
    }
  }

  // ---- load 4 channels per lane, migrate Keys ----
  const size_t in_off =
      (((size_t)b * a.n_call + (size_t)(a.tok_off + tkn)) * a.kv_heads + j) * kHeadDim + 4 * lane;
  const void* src = kv ? a.v : a.k;
  float x[4];
  if (a.dtype == 1) {
    float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + in_off);
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  } else {
    uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(src) + in_off);
    __nv_bfloat162 p0 = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
    __nv_bfloat162 p1 = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
    x[0] = __low2float(p0); x[1] = __high2float(p0);
    x[2] = __low2float(p1); x[3] = __high2float(p1);
  }
  if (kv == 0 && a.lam_inv) {
    float4 li = *reinterpret_cast<const float4*>(a.lam_inv + (size_t)j * kHeadDim + 4 * lane);
    x[0] = __fmul_rn(x[0], li.x); x[1] = __fmul_rn(x[1], li.y);
    x[2] = __fmul_rn(x[2], li.z); x[3] = __fmul_rn(x[3], li.w);
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
  const int bits = a.window ? 16 : a.bits;  // window tokens are held at INT16
  const float qmax = (float)((1u << bits) - 1u);
  if (r == 0.0f) {
#pragma unroll
    for (int i = 0; i < 4; i++) sc[4 * lane + i] = 0;
  } else {
    const float inv = __fdiv_rn(qmax, r);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      float t = __fmul_rn(__fsub_rn(x[i], z), inv);
      float f = floorf(__fadd_rn(t, 0.5f));
      f = fminf(fmaxf(f, 0.0f), qmax);
      sc[4 * lane + i] = (uint16_t)f;
    }
  }
  __syncwarp();
  const uint32_t mw = (uint32_t)__half_as_ushort(rh) | ((uint32_t)__half_as_ushort(zh) << 16);

  if (a.window) {
    pack_codes(wg, 16, wtok, kv, sc, pm, lane);
    if (lane == 0) a.wmeta[wmi] = mw;
  } else {
    int slot;
    size_t tile;
    uint8_t* gbase = main_group(a.n0 + tkn, &slot, &tile);
    pack_codes(gbase, bits, slot & 15, kv, sc, pm, lane);
    if (lane == 0) a.meta[(tile * (size_t)a.pf + slot) * 2 + kv] = mw;
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
  const long long warps = (long long)a.batch * a.cnt * a.kv_heads * 2;
  if (warps <= 0) return cudaSuccess;
  const long long blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
  return launch_pdl(append_kernel, dim3((unsigned)blocks), dim3(kWarpsPerBlock * 32), 0, s, a);
}

}  // namespace kvq
