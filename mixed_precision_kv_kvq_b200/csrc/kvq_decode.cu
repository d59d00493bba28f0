// kvq_decode.cu -- split-K GQA decode attention over the packed low-bit cache.
//
// For one block (layer) and every (sequence b, KV head j), the G = q_heads /
// kv_heads query heads h of that KV head attend over every cached token:
//   out_h = sum_t softmax_t(sm_scale * (q_h * lambda) . k^_t) v^_t,
//   k^_t = Z_t + c_t R_t / (2^b - 1)   (dequantised migrated Key),
// the online half of the PM-KVQ note (key design 1 keeps the cache packed at
// the block's width; key design 3 folds the migration factor into the
// query).  Dequantisation is folded out of the inner loop:
//   q'.k^_t = (R_t / (2^b-1)) (q'.c_t) + Z_t sum(q'),
//   sum_t p_t v^_t = (sum_t p_t R_t c_t) / (2^b-1) + sum_t p_t Z_t,
// so the raw codes go straight into mma.sync.m16n8k16 operands (fp16, exact
// for codes < 2^11; 16-bit codes as two bytes): QK^T with A = 16 tokens x 16
// channels of codes and B = q' (N = 8 query heads; q' is carried as a hi + lo
// pair of fp16 values, two MMAs on the same A registers, because one fp16
// rounding of q' alone moves large outlier-channel scores by up to ~2^-12 of
// their size, enough to break a 2e-3 output tolerance), PV with A = 16 channels x
// 16 tokens of V codes and B = p R (transposed from the score fragment with
// movmatrix).  Codes are widened to fp16 in registers with the 0x6400 exponent
// trick (integer c in the low mantissa bits of 1024.0; one lop3 + one hfma2
// per code pair).
//
// Work split: the groups (16 tokens) of all streams of the block form one
// list; CTA c takes the contiguous slice [c*tot/grid, (c+1)*tot/grid).  One
// producer warp streams the slice's codes and meta into a ring of shared-
// memory stages with cp.async.bulk (TMA bulk copies) on mbarriers; eight
// consumer warps take alternate groups of each stage and keep their own
// online-softmax state, merged through shared memory when a stream segment
// ends.  A stream split over several CTAs leaves one partial (max, sum,
// unnormalised output) per CTA in the workspace; the last CTA to finish the
// stream (atomic ticket, no waiting) merges them with log-sum-exp weights.
// Every wait on an mbarrier is bounded in time; a kernel that gives up sets
// the cache's error flag and carries on without hanging.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 4;
constexpr int kChunkBytes = 8192;                 // K (and V) code bytes per stage
constexpr int kMaxChunkGroups = kChunkBytes / 512; // 16 groups at 2 bits
constexpr int kMetaBytes = kMaxChunkGroups * 64;  // 16 tokens * 4 B per group
constexpr int kStageBytes = 2 * kChunkBytes + 2 * kMetaBytes;
constexpr int kMaxGroup = 8;                      // query heads per KV head (MMA N)
constexpr int kSmemBytes = kStages * kStageBytes + kMaxGroup * kHeadDim * 4 +
                           3 * kConsumerWarps * kMaxGroup * 4 + 2 * kStages * 8 + 16;
constexpr int kCtasPerSm = 2;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: true when the phase completed, false after kWaitNs (the
// error flag is then set and *abort raised so later waits give up at once).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* err, volatile int* abort) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned it = 0;; it++) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63) == 63) {
      if (*abort || global_ns() - t0 > kWaitNs) {
        *abort = 1;
        atomicExch(err, 1);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(d) : "r"(a), "r"(mask), "r"(orv));  // (a & b) | c
  return d;
}
__device__ __forceinline__ uint32_t hfma2_u(uint32_t x, uint32_t m, uint32_t a) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(x), "r"(m), "r"(a));
  return d;
}
__device__ __forceinline__ void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                    uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(x));
  return d;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// --------------------------------------------------------- code widening
// Pair at field position POS of a word packed at BITS (BITS <= 8): the two
// codes sit at bits [BITS*POS, +BITS) of each half-word.  Result: half2 of the
// two codes as exact fp16 values.
template <int BITS, int POS>
__device__ __forceinline__ uint32_t widen(uint32_t w, uint32_t w8) {
  constexpr int kPerByte = 8 / BITS;
  constexpr int kp = POS % kPerByte;
  constexpr uint32_t m = (1u << BITS) - 1u;
  constexpr uint32_t mask = (m << (BITS * kp)) | (m << (16 + BITS * kp));
  const uint32_t x = lop_and_or(POS >= kPerByte ? w8 : w, mask, 0x64006400u);  // 1024 + c*2^e
  constexpr int e = BITS * kp;
  constexpr uint32_t sc = (uint32_t)(15 - e) << 10;               // 2^-e
  constexpr uint32_t bi = 0x8000u | ((uint32_t)(25 - e) << 10);   // -1024 * 2^-e
  return hfma2_u(x, sc | (sc << 16), bi | (bi << 16));
}
// 16-bit codes: whole word is the pair; split each code into high and low byte.
__device__ __forceinline__ uint32_t widen16_hi(uint32_t w) {
  return hfma2_u(lop_and_or(w >> 8, 0x00ff00ffu, 0x64006400u), 0x3c003c00u, 0xe400e400u);
}
__device__ __forceinline__ uint32_t widen16_lo(uint32_t w) {
  return hfma2_u(lop_and_or(w, 0x00ff00ffu, 0x64006400u), 0x3c003c00u, 0xe400e400u);
}

// Word of a lane unit holding pair p (0..15) of half x at BITS, and its
// position.
template <int BITS>
struct PairAddr {
  static constexpr int ppw = 16 / BITS;
  __device__ static constexpr int word(int x, int p) { return x * BITS + p / ppw; }
  __device__ static constexpr int pos(int p) { return p % ppw; }
};

// A-fragment registers for MMA block s (channels or tokens 16s..16s+15).
// K: a0a1 = (x=0, p=2s), a2a3 = (x=1, p=2s), a4a5 = (x=0, p=2s+1), a6a7 = (x=1, p=2s+1)
// V: a0a1 = (x=0, p=2s), a2a3 = (x=0, p=2s+1), a4a5 = (x=1, p=2s), a6a7 = (x=1, p=2s+1)
template <int BITS, int S>
__device__ __forceinline__ uint32_t pair_at(const uint32_t* u, const uint32_t* u8, int x, int r) {
  const int p = 2 * S + r;
  const int wi = x * BITS + p / PairAddr<BITS>::ppw;
  // POS must be a compile-time constant: expand over r.
  if (r == 0) return widen<BITS, (2 * S) % (16 / BITS)>(u[wi], u8[wi]);
  return widen<BITS, (2 * S + 1) % (16 / BITS)>(u[wi], u8[wi]);
}

// ------------------------------------------------------------ work list

struct Chunk {
  int s;          // stream (b * kv_heads + j)
  int tile, grp0, ng, tile_valid;
};

struct ChunkIter {
  long long gidx, gend;
  __device__ bool next(const Fill& f, int max_groups, Chunk& c) {
    if (gidx >= gend) return false;
    const long long s = gidx / f.gps;
    const long long v = gidx - s * f.gps;
    const GroupLoc loc = locate_group(f, v);
    long long ng = loc.tile_groups - loc.grp;
    if (ng > max_groups) ng = max_groups;
    if (ng > gend - gidx) ng = gend - gidx;
    c.s = (int)s;
    c.tile = loc.tile;
    c.grp0 = loc.grp;
    c.ng = (int)ng;
    c.tile_valid = loc.tile < f.k ? f.p : (loc.tile == f.k ? f.h + f.r : f.h);
    gidx += ng;
    return true;
  }
};

__device__ __forceinline__ long long cta_of(long long x, long long tot, int grid) {
  return ((x + 1) * grid - 1) / tot;
}

// ------------------------------------------------------------------ kernel

template <int BITS>
__global__ void __maxnreg__(112) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* o_acc = reinterpret_cast<float*>(smem + kStages * kStageBytes);  // [8][128]
  float* w_m = o_acc + kMaxGroup * kHeadDim;                               // [warps][8]
  float* w_l = w_m + kConsumerWarps * kMaxGroup;
  float* w_pz = w_l + kConsumerWarps * kMaxGroup;
  uint64_t* bars = reinterpret_cast<uint64_t*>(w_pz + kConsumerWarps * kMaxGroup);
  volatile int* flags = reinterpret_cast<volatile int*>(bars + 2 * kStages);  // [0] abort, [1] last
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kStages);

  constexpr int kGroupBytes = 256 * BITS;
  constexpr int kChunkGroups = kChunkBytes / kGroupBytes;
  constexpr float kCScale = (BITS == 16 ? 256.0f : 1.0f) / (float)((1u << BITS) - 1u);

  const Fill f = a.fill;
  const int n_streams = a.batch * a.kv_heads;
  const long long tot = (long long)n_streams * f.gps;
  const int cta = blockIdx.x;
  const long long g_begin = tot * cta / a.grid, g_end = tot * (cta + 1) / a.grid;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; i++) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kConsumerWarps);
    }
    flags[0] = 0;
    flags[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i < kMaxGroup * kHeadDim; i += kThreads) o_acc[i] = 0.f;
  __syncthreads();
  if (g_begin >= g_end) return;

  if (warp == kConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      ChunkIter it{g_begin, g_end};
      Chunk c;
      for (int ci = 0; it.next(f, kChunkGroups, c); ci++) {
        const int st = ci % kStages;
        if (ci >= kStages) {
          if (!mbar_wait(empty0 + 8 * st, ((ci / kStages) - 1) & 1, a.err, flags)) break;
        }
        const uint32_t kb = (uint32_t)c.ng * kGroupBytes, mb = (uint32_t)c.ng * 64u;
        mbar_expect_tx(full0 + 8 * st, 2 * kb + 2 * mb);
        uint8_t* sb = smem + st * kStageBytes;
        const size_t sk = (size_t)c.s * 2, sv = sk + 1;
        const uint8_t* kc = a.codes + (sk * f.nt + c.tile) * (size_t)kTileBytes + (size_t)c.grp0 * kGroupBytes;
        const uint8_t* vc = a.codes + (sv * f.nt + c.tile) * (size_t)kTileBytes + (size_t)c.grp0 * kGroupBytes;
        const uint32_t* km = a.meta + (sk * f.nt + c.tile) * (size_t)f.pf + (size_t)c.grp0 * 16;
        const uint32_t* vm = a.meta + (sv * f.nt + c.tile) * (size_t)f.pf + (size_t)c.grp0 * 16;
        bulk_g2s(smem_u32(sb), kc, kb, full0 + 8 * st);
        bulk_g2s(smem_u32(sb + kChunkBytes), vc, kb, full0 + 8 * st);
        bulk_g2s(smem_u32(sb + 2 * kChunkBytes), km, mb, full0 + 8 * st);
        bulk_g2s(smem_u32(sb + 2 * kChunkBytes + kMetaBytes), vm, mb, full0 + 8 * st);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, t = lane & 3;
  const int G = a.group;
  uint32_t bq[8][2];      // q' B fragments (fp16x2), high part
  uint32_t bqo[8][2];     // q' - high part, rounded to fp16 (low part)
  uint32_t bql[8][2];     // high part / 256 (16-bit codes only)
  float sig0 = 0.f, sig1 = 0.f;  // sum of q' for heads 2t, 2t+1
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, pz0 = 0.f, pz1 = 0.f;
  float o[8][4];
  int cur = -1;

  auto start_stream = [&](int s) {
    const int b = s / a.kv_heads, j = s - b * a.kv_heads;
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.q_heads + (size_t)j * G) * kHeadDim;
    const float* lam = a.lam ? a.lam + (size_t)j * kHeadDim : nullptr;
    float part = 0.f;
#pragma unroll
    for (int sb = 0; sb < 8; sb++) {
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
        const int c0 = 16 * sb + 2 * t + 8 * hf;
        float v0 = 0.f, v1 = 0.f;
        if (g < G) {
          const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162*>(qb + (size_t)g * kHeadDim + c0);
          v0 = __low2float(qq) * a.qscale;
          v1 = __high2float(qq) * a.qscale;
          if (lam) {
            v0 *= lam[c0];
            v1 *= lam[c0 + 1];
          }
        }
        const __half2 h = __floats2half2_rn(v0, v1);
        const __half2 lo = __floats2half2_rn(v0 - __low2float(h), v1 - __high2float(h));
        bq[sb][hf] = *reinterpret_cast<const uint32_t*>(&h);
        bqo[sb][hf] = *reinterpret_cast<const uint32_t*>(&lo);
        part += (__low2float(h) + __low2float(lo)) + (__high2float(h) + __high2float(lo));
        if (BITS == 16) {
          const __half2 hl = __hmul2(h, __float2half2_rn(1.0f / 256.0f));
          bql[sb][hf] = *reinterpret_cast<const uint32_t*>(&hl);
        }
      }
    }
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);  // lanes 4g..4g+3: sum for head g
    sig0 = __shfl_sync(0xffffffffu, part, 4 * (2 * t));
    sig1 = __shfl_sync(0xffffffffu, part, 4 * (2 * t + 1));
    m0 = m1 = -INFINITY;
    l0 = l1 = pz0 = pz1 = 0.f;
#pragma unroll
    for (int sb = 0; sb < 8; sb++) o[sb][0] = o[sb][1] = o[sb][2] = o[sb][3] = 0.f;
  };

  auto finish_stream = [&](int s) {
    // per-warp totals for heads 2t, 2t+1 (reduce the thread partials over g)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      pz0 += __shfl_xor_sync(0xffffffffu, pz0, off);
      pz1 += __shfl_xor_sync(0xffffffffu, pz1, off);
    }
    if (g == 0) {
      w_m[warp * kMaxGroup + 2 * t] = m0;
      w_m[warp * kMaxGroup + 2 * t + 1] = m1;
      w_l[warp * kMaxGroup + 2 * t] = l0;
      w_l[warp * kMaxGroup + 2 * t + 1] = l1;
      w_pz[warp * kMaxGroup + 2 * t] = pz0;
      w_pz[warp * kMaxGroup + 2 * t + 1] = pz1;
    }
    consumer_sync();
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; w++) {
      M0 = fmaxf(M0, w_m[w * kMaxGroup + 2 * t]);
      M1 = fmaxf(M1, w_m[w * kMaxGroup + 2 * t + 1]);
    }
    const float sc0 = ex2(m0 - M0), sc1 = ex2(m1 - M1);
    if (2 * t < G) {
#pragma unroll
      for (int sb = 0; sb < 8; sb++) {
        atomicAdd(&o_acc[(2 * t) * kHeadDim + 16 * sb + g], sc0 * o[sb][0]);
        atomicAdd(&o_acc[(2 * t) * kHeadDim + 16 * sb + g + 8], sc0 * o[sb][2]);
      }
    }
    if (2 * t + 1 < G) {
#pragma unroll
      for (int sb = 0; sb < 8; sb++) {
        atomicAdd(&o_acc[(2 * t + 1) * kHeadDim + 16 * sb + g], sc1 * o[sb][1]);
        atomicAdd(&o_acc[(2 * t + 1) * kHeadDim + 16 * sb + g + 8], sc1 * o[sb][3]);
      }
    }
    consumer_sync();
    const long long first = cta_of((long long)s * f.gps, tot, a.grid);
    const long long last = cta_of((long long)(s + 1) * f.gps - 1, tot, a.grid);
    const int nparts = (int)(last - first + 1);
    const int b = s / a.kv_heads, j = s - b * a.kv_heads;
    float* outp = a.out + ((size_t)b * a.q_heads + (size_t)j * G) * kHeadDim;
    float* mypart = a.parts + (size_t)(cta + s) * G * (kHeadDim + 2);
    for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kConsumerWarps * 32) {
      const int h = idx / kHeadDim, c = idx - h * kHeadDim;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; w++) M = fmaxf(M, w_m[w * kMaxGroup + h]);
      float L = 0.f, PZ = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; w++) {
        const float e = ex2(w_m[w * kMaxGroup + h] - M);
        L += e * w_l[w * kMaxGroup + h];
        PZ += e * w_pz[w * kMaxGroup + h];
      }
      const float O = o_acc[idx] * kCScale + PZ;
      o_acc[idx] = 0.f;
      if (nparts == 1) {
        outp[idx] = O / L;
      } else {
        float* pr = mypart + (size_t)h * (kHeadDim + 2);
        pr[2 + c] = O;
        if (c == 0) {
          pr[0] = M;
          pr[1] = L;
        }
      }
    }
    if (nparts > 1) {
      __threadfence();  // this thread's partial is visible device-wide before the ticket
      consumer_sync();
      if (threadIdx.x == 0) {
        __threadfence();
        const int old = atomicAdd(a.counters + s, 1);
        flags[1] = (old == nparts - 1);
      }
      consumer_sync();
      if (flags[1]) {
        __threadfence();
        const float* p0 = a.parts + (size_t)(first + s) * G * (kHeadDim + 2);
        for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kConsumerWarps * 32) {
          const int h = idx / kHeadDim, c = idx - h * kHeadDim;
          float M = -INFINITY;
          for (int k = 0; k < nparts; k++) M = fmaxf(M, __ldcg(p0 + ((size_t)k * G + h) * (kHeadDim + 2)));
          float L = 0.f, O = 0.f;
          for (int k = 0; k < nparts; k++) {
            const float* pr = p0 + ((size_t)k * G + h) * (kHeadDim + 2);
            const float e = ex2(__ldcg(pr) - M);
            L += e * __ldcg(pr + 1);
            O += e * __ldcg(pr + 2 + c);
          }
          outp[idx] = O / L;
        }
        if (threadIdx.x == 0) a.counters[s] = 0;
      }
    }
    consumer_sync();
  };

  ChunkIter it{g_begin, g_end};
  Chunk c;
  for (int ci = 0; it.next(f, kChunkGroups, c); ci++) {
    if (c.s != cur) {
      if (cur >= 0) finish_stream(cur);
      start_stream(c.s);
      cur = c.s;
    }
    const int st = ci % kStages;
    const bool ok = mbar_wait(full0 + 8 * st, (ci / kStages) & 1, a.err, flags);
    const uint8_t* sb = smem + st * kStageBytes;
    for (int gi = warp; ok && gi < c.ng; gi += kConsumerWarps) {
      const int valid = min(16, c.tile_valid - 16 * (c.grp0 + gi));
      // ---- K unit -> scores ----
      const uint32_t* ku = reinterpret_cast<const uint32_t*>(sb + (size_t)gi * kGroupBytes + lane * unit_bytes(BITS));
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (BITS == 16) {
#pragma unroll
        for (int sb2 = 0; sb2 < 8; sb2++) {
          const uint2 w0 = *reinterpret_cast<const uint2*>(ku + 2 * sb2);        // token g: pairs 2s, 2s+1
          const uint2 w1 = *reinterpret_cast<const uint2*>(ku + 16 + 2 * sb2);   // token g+8
          const uint32_t h0 = widen16_hi(w0.x), h1 = widen16_hi(w1.x), h2 = widen16_hi(w0.y), h3 = widen16_hi(w1.y);
          mma(d, h0, h1, h2, h3, bq[sb2][0], bq[sb2][1]);
          mma(d, h0, h1, h2, h3, bqo[sb2][0], bqo[sb2][1]);
          mma(d, widen16_lo(w0.x), widen16_lo(w1.x), widen16_lo(w0.y), widen16_lo(w1.y), bql[sb2][0], bql[sb2][1]);
        }
      } else {
        uint32_t u[2 * BITS], u8[2 * BITS];
#pragma unroll
        for (int i = 0; i < 2 * BITS; i += 4) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(ku + i);
          u[i] = q4.x; u[i + 1] = q4.y; u[i + 2] = q4.z; u[i + 3] = q4.w;
        }
#pragma unroll
        for (int i = 0; i < 2 * BITS; i++) u8[i] = u[i] >> 8;
#define KVQ_QK(S)                                                                                     \
  {                                                                                                     \
    const uint32_t a0 = pair_at<BITS, S>(u, u8, 0, 0), a1 = pair_at<BITS, S>(u, u8, 1, 0);             \
    const uint32_t a2 = pair_at<BITS, S>(u, u8, 0, 1), a3 = pair_at<BITS, S>(u, u8, 1, 1);             \
    mma(d, a0, a1, a2, a3, bq[S][0], bq[S][1]);                                                         \
    mma(d, a0, a1, a2, a3, bqo[S][0], bqo[S][1]);                                                       \
  }
        KVQ_QK(0) KVQ_QK(1) KVQ_QK(2) KVQ_QK(3) KVQ_QK(4) KVQ_QK(5) KVQ_QK(6) KVQ_QK(7)
#undef KVQ_QK
      }
      // ---- meta for tokens g, g+8 ----
      const uint32_t* kmeta = reinterpret_cast<const uint32_t*>(sb + 2 * kChunkBytes) + gi * 16;
      const uint32_t* vmeta = reinterpret_cast<const uint32_t*>(sb + 2 * kChunkBytes + kMetaBytes) + gi * 16;
      const bool va = g < valid, vb = g + 8 < valid;
      const float2 ka = __half22float2(*reinterpret_cast<const __half2*>(kmeta + g));
      const float2 kb = __half22float2(*reinterpret_cast<const __half2*>(kmeta + g + 8));
      const float2 vma = __half22float2(*reinterpret_cast<const __half2*>(vmeta + g));
      const float2 vmb = __half22float2(*reinterpret_cast<const __half2*>(vmeta + g + 8));
      const float rka = ka.x * kCScale, rkb = kb.x * kCScale;
      const float s00 = va ? fmaf(rka, d[0], ka.y * sig0) : -INFINITY;
      const float s01 = va ? fmaf(rka, d[1], ka.y * sig1) : -INFINITY;
      const float s10 = vb ? fmaf(rkb, d[2], kb.y * sig0) : -INFINITY;
      const float s11 = vb ? fmaf(rkb, d[3], kb.y * sig1) : -INFINITY;
      float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      if (__any_sync(0xffffffffu, (n0 > m0) | (n1 > m1))) {
        const float a0 = ex2(m0 - n0), a1 = ex2(m1 - n1);
#pragma unroll
        for (int sb2 = 0; sb2 < 8; sb2++) {
          o[sb2][0] *= a0; o[sb2][2] *= a0;
          o[sb2][1] *= a1; o[sb2][3] *= a1;
        }
        l0 *= a0; pz0 *= a0;
        l1 *= a1; pz1 *= a1;
        m0 = n0;
        m1 = n1;
      }
      const float p00 = ex2(s00 - m0), p01 = ex2(s01 - m1), p10 = ex2(s10 - m0), p11 = ex2(s11 - m1);
      const float rva = va ? vma.x : 0.f, zva = va ? vma.y : 0.f;
      const float rvb = vb ? vmb.x : 0.f, zvb = vb ? vmb.y : 0.f;
      l0 += p00 + p10;
      l1 += p01 + p11;
      pz0 = fmaf(p00, zva, fmaf(p10, zvb, pz0));
      pz1 = fmaf(p01, zva, fmaf(p11, zvb, pz1));
      const uint32_t b0 = movmatrix_t(pack_h2(p00 * rva, p01 * rva));  // tokens 2t,2t+1 of head g
      const uint32_t b1 = movmatrix_t(pack_h2(p10 * rvb, p11 * rvb));  // tokens 2t+8, 2t+9
      // ---- V unit -> output ----
      const uint32_t* vu = reinterpret_cast<const uint32_t*>(sb + kChunkBytes + (size_t)gi * kGroupBytes + lane * unit_bytes(BITS));
      if constexpr (BITS == 16) {
        const uint32_t b0l = hfma2_u(b0, 0x1c001c00u, 0u), b1l = hfma2_u(b1, 0x1c001c00u, 0u);  // /256
#pragma unroll
        for (int sb2 = 0; sb2 < 8; sb2++) {
          const uint2 w0 = *reinterpret_cast<const uint2*>(vu + 2 * sb2);        // u = 0
          const uint2 w1 = *reinterpret_cast<const uint2*>(vu + 16 + 2 * sb2);   // u = 1
          mma(o[sb2], widen16_hi(w0.x), widen16_hi(w0.y), widen16_hi(w1.x), widen16_hi(w1.y), b0, b1);
          mma(o[sb2], widen16_lo(w0.x), widen16_lo(w0.y), widen16_lo(w1.x), widen16_lo(w1.y), b0l, b1l);
        }
      } else {
        uint32_t u[2 * BITS], u8[2 * BITS];
#pragma unroll
        for (int i = 0; i < 2 * BITS; i += 4) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(vu + i);
          u[i] = q4.x; u[i + 1] = q4.y; u[i + 2] = q4.z; u[i + 3] = q4.w;
        }
#pragma unroll
        for (int i = 0; i < 2 * BITS; i++) u8[i] = u[i] >> 8;
#define KVQ_PV(S)                                                                                       \
  mma(o[S], pair_at<BITS, S>(u, u8, 0, 0), pair_at<BITS, S>(u, u8, 0, 1), pair_at<BITS, S>(u, u8, 1, 0), \
      pair_at<BITS, S>(u, u8, 1, 1), b0, b1);
        KVQ_PV(0) KVQ_PV(1) KVQ_PV(2) KVQ_PV(3) KVQ_PV(4) KVQ_PV(5) KVQ_PV(6) KVQ_PV(7)
#undef KVQ_PV
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * st);
  }
  if (cur >= 0) finish_stream(cur);
}

template <int BITS>
cudaError_t launch_bits(const DecodeArgs& a, cudaStream_t s) {
  static bool attr_set = false;  // per process; set before the first launch
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  decode_kernel<BITS><<<a.grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_grid(int num_sms) { return num_sms * kCtasPerSm; }

size_t decode_parts_bytes(int grid, int n_streams, int group) {
  return (size_t)(grid + n_streams) * group * (kHeadDim + 2) * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.group < 1 || a.group > kMaxGroup) return cudaErrorInvalidValue;
  switch (a.fill.bits) {
    case 2: return launch_bits<2>(a, s);
    case 4: return launch_bits<4>(a, s);
    case 8: return launch_bits<8>(a, s);
    case 16: return launch_bits<16>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
