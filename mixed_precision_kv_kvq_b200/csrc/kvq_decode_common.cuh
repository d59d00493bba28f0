// kvq_decode_common.cuh -- pieces of the split-K GQA decode kernel
// (kvq_decode.cu) kept apart from its main loop: PTX wrappers, bounded
// mbarrier waits, bulk copies, the widening of packed codes into MMA
// operands, and the split merge that ends every CTA of a stream.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kMaxGroup = 8;                            // query heads per KV head (MMA N)
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait
constexpr int kPartFloats = 2 * kMaxGroup + kHeadDim * kMaxGroup;  // one CTA's partial record
// Largest amount (log2 units) a score may exceed the running max before the
// max is moved: p <= 2^8, and p * R stays well inside fp16 for R < 255.
constexpr float kRebase = 8.0f;

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
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, int* err, volatile int* abort) {
  const unsigned long long t0 = global_ns();
  for (unsigned it = 0;; it++) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 15) == 15) {
      if (*abort || global_ns() - t0 > kWaitNs) {
        *abort = 1;
        atomicExch(err, 1);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* err, volatile int* abort) {
  if (mbar_try(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, err, abort);
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
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
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
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
// int8 MMA, A = u8 codes, B = s8 (hi byte of q') or u8 (lo byte of q').
__device__ __forceinline__ void imma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void imma_u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// w * 2^SH as an integer multiply (keeps the shift off the logic pipe)
template <int SH>
__device__ __forceinline__ uint32_t shl_mul(uint32_t w) {
  if constexpr (SH == 0) {
    return w;
  } else {
    uint32_t d;
    asm("mul.lo.u32 %0, %1, %2;" : "=r"(d) : "r"(w), "n"(1 << SH));
    return d;
  }
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
// Bit offset, within its byte, of the codes at field position POS of a word
// packed at BITS (BITS <= 8); positions past the first byte are read from
// the word shifted right by 8.
template <int BITS, int POS>
__host__ __device__ constexpr int field_shift() {
  return BITS * ((POS % (16 / BITS)) % (8 / BITS));
}
// Pair at field position POS: the two codes sit at bits [BITS*POS, +BITS) of
// each half-word.  Result: half2 (c0 2^(e-24), c1 2^(e-24)), exact, with
// e = field_shift: the code bits, masked in place, are the mantissa of a
// binary16 subnormal (exponent field zero: the value is the 10-bit mantissa
// times 2^-24), which the fp16 MMA takes as it is.  One AND per pair; the
// 2^(e-24) is undone outside the inner loop, in the output rows.  The legacy
// MMA rounds products with a subnormal operand (up to ~2^-12.5 of the sum of
// the terms' sizes, measured), the same order as the fp16 rounding of P; the
// caller centres the codes afterwards (sum_t P_t (c_t - h) = sum_t P_t c_t -
// h sum_t P_t) so neither error is weighted by the uncentred code.
template <int BITS, int POS>
__device__ __forceinline__ uint32_t widen(uint32_t w, uint32_t w8) {
  constexpr int kPerByte = 8 / BITS;
  constexpr int e = field_shift<BITS, POS>();
  constexpr uint32_t m = (1u << BITS) - 1u;
  static_assert(((m << e) >> 10) == 0u, "the code lies in the mantissa field");
  return ((POS % (16 / BITS)) >= kPerByte ? w8 : w) & ((m << e) | (m << (16 + e)));
}
// field_shift of pair p (any p in 0..15) at BITS <= 8.
template <int BITS>
__host__ __device__ constexpr int pair_shift(int p) {
  return BITS >= 16 ? 0 : BITS * ((p % (16 / BITS)) % (8 / BITS));
}
// 16-bit codes: the whole word is the pair; split each code into high and low
// byte, c - 2^15 = 256 (hi - 128) + lo.  Each byte x goes in as the binary16
// 1024 + x (0x6400 | x), and one fma.f16x2 takes the offset off exactly; the
// codes are centred so the high-byte MMA sum stays near the output.
__device__ __forceinline__ uint32_t widen16_hi(uint32_t w) {
  return hfma2_u(lop_and_or(w >> 8, 0x00ff00ffu, 0x64006400u), 0x3c003c00u, 0xe480e480u);  // - 1152
}
__device__ __forceinline__ uint32_t widen16_lo(uint32_t w) {
  return hfma2_u(lop_and_or(w, 0x00ff00ffu, 0x64006400u), 0x3c003c00u, 0xe400e400u);
}

// Pair p = 2S + r of half x of a lane unit at BITS (<= 8), widened.
template <int BITS, int S, int X, int R>
__device__ __forceinline__ uint32_t pair_at(const uint32_t* u, const uint32_t* u8) {
  constexpr int ppw = 16 / BITS;
  constexpr int p = 2 * S + R;
  constexpr int wi = X * BITS + p / ppw;
  return widen<BITS, p % ppw>(u[wi], u8[wi]);
}

// Packed fp32 pairs (add / mul / fma .f32x2): one instruction for the two
// heads a lane holds, each lane an ordinary IEEE round-to-nearest operation.
__device__ __forceinline__ unsigned long long f2_bits(float2 v) { return *reinterpret_cast<unsigned long long*>(&v); }
__device__ __forceinline__ float2 f2_from(unsigned long long b) { return *reinterpret_cast<float2*>(&b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_from(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_from(d);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return f2_from(d);
}
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// Key quads.  A quad is the 4 codes of one token at 4 consecutive Key
// positions, one int8 A-fragment register of mma.m16n8k32; member i sits in
// byte i of its word at the quad's field (kvq_internal.cuh).  quad_reg gives
// the register of quad (k-block S, token half X, column half R), its codes
// moved to the top bits of each byte: c * 2^(8 - BITS), exact in u8.
template <int BITS, int F>
__device__ __forceinline__ uint32_t quad_field(uint32_t w) {
  constexpr uint32_t top = (((1u << BITS) - 1u) << (8 - BITS)) * 0x01010101u;
  return shl_mul<8 - BITS - BITS * F>(w) & top;
}
template <int BITS, int S, int X, int R>
__device__ __forceinline__ uint32_t quad_reg(const uint32_t* u) {
  constexpr int qpw = 8 / BITS;  // quads per word
  constexpr int Q = 8 * X + 2 * S + R;
  return quad_field<BITS, Q % qpw>(u[Q / qpw]);
}

// The end of every CTA of a stream.  Oc, Mh, Lh: this CTA's unnormalised
// output for channel c = threadIdx.x (one channel per thread, 128 threads),
// running max and sum for every head.  A stream cut into one slice writes its
// output; otherwise the CTA leaves a partial record (M[8], L[8], O[128][8])
// and the CTA that takes the stream's last ticket (atomic, no waiting) merges
// all partials with log-sum-exp weights.  flags[1]: CTA-shared scratch word;
// scratch: kScratchFloats floats of free shared memory.
constexpr int kScratchFloats = 2 * kMaxSplits * kMaxGroup + 2 * kMaxGroup;
__device__ __forceinline__ void finish_stream(const DecodeArgs& a, int s, int split, const float (&Oc)[kMaxGroup],
                                              const float (&Mh)[kMaxGroup], const float (&Lh)[kMaxGroup],
                                              volatile int* flags, float* scratch) {
  const int b = s / a.kv_heads, j = s - b * a.kv_heads;
  const int G = a.group;
  float* outp = a.out + ((size_t)b * a.q_heads + (size_t)j * G) * kHeadDim;
  const int nparts = a.nparts;  // partials of this stream over every launch of the call
  const int c = threadIdx.x;    // one channel per thread
  if (nparts == 1) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; h++)
      if (h < G) outp[h * kHeadDim + c] = Oc[h] / Lh[h];
    return;
  }
  // Partial record of this CTA: M[8], L[8], then O[128 channels][8 heads].
  float* mypart = a.parts + ((size_t)s * nparts + a.part_base + split) * kPartFloats;
  if (c == 0) {
#pragma unroll
    for (int h = 0; h < kMaxGroup; h += 4) {
      *reinterpret_cast<float4*>(mypart + h) = make_float4(Mh[h], Mh[h + 1], Mh[h + 2], Mh[h + 3]);
      *reinterpret_cast<float4*>(mypart + kMaxGroup + h) = make_float4(Lh[h], Lh[h + 1], Lh[h + 2], Lh[h + 3]);
    }
  }
  *reinterpret_cast<float4*>(mypart + 2 * kMaxGroup + c * kMaxGroup) = make_float4(Oc[0], Oc[1], Oc[2], Oc[3]);
  *reinterpret_cast<float4*>(mypart + 2 * kMaxGroup + c * kMaxGroup + 4) = make_float4(Oc[4], Oc[5], Oc[6], Oc[7]);
  // Ticket: after the CTA barrier one thread takes it with an
  // acquire-release atomic at GPU scope (it publishes the CTA's partial, which
  // the barrier ordered before it, and the CTA that takes the last ticket sees
  // every other partial); that CTA merges.
  __syncthreads();
  if (threadIdx.x == 0) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(a.counters + s) : "memory");
    flags[1] = old == nparts - 1;
  }
  __syncthreads();
  // A launch that skipped its dependency wait still completes only after the
  // launch before it (so kernels after this one are ordered behind both).
  // No deadlock: this grid started only once every CTA of that launch had
  // triggered, i.e. was resident.
  if (a.after_decode) pdl_wait();
  if (!flags[1]) return;
  const float* p0 = a.parts + (size_t)s * nparts * kPartFloats;
  // The first kPre partials' outputs for this thread's channel are loaded
  // now, in flight while the weights are formed from every partial's M, L.
  constexpr int kPre = 8;
  const float* oc = p0 + 2 * kMaxGroup + c * kMaxGroup;
  float4 ov[kPre][2];
#pragma unroll
  for (int k = 0; k < kPre; k++) {
    if (k < nparts) {
      ov[k][0] = __ldcg(reinterpret_cast<const float4*>(oc + (size_t)k * kPartFloats));
      ov[k][1] = __ldcg(reinterpret_cast<const float4*>(oc + (size_t)k * kPartFloats + 4));
    }
  }
  float* wk = scratch;  // [nparts][8] M, then [nparts][8] L
  float* lk = wk + kMaxSplits * kMaxGroup;
  for (int i = threadIdx.x; i < nparts * 2 * kMaxGroup / 4; i += kHeadDim) {  // every partial's M, L at once
    const int k = i / (2 * kMaxGroup / 4), q4 = i - k * (2 * kMaxGroup / 4);
    const float4 v = __ldcg(reinterpret_cast<const float4*>(p0 + (size_t)k * kPartFloats) + q4);
    float* dst = q4 < 2 ? wk + k * kMaxGroup + 4 * q4 : lk + k * kMaxGroup + 4 * (q4 - 2);
    dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
  }
  __syncthreads();
  // Log-sum-exp weights, formed once: thread h takes head h's max M over the
  // partials, then thread (k, h) the weight w_k = e^(M_k - M) (in place of
  // M_k), then thread h the sum of w_k L_k; out = sum_k w_k O_k / sum_k w_k L_k.
  float* mxs = lk + kMaxSplits * kMaxGroup;  // [8] M, then [8] sum w L
  if (threadIdx.x < kMaxGroup) {
    float m = -INFINITY;
    for (int k = 0; k < nparts; k++) m = fmaxf(m, wk[k * kMaxGroup + threadIdx.x]);
    mxs[threadIdx.x] = m;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nparts * kMaxGroup; i += kHeadDim) wk[i] = ex2(wk[i] - mxs[i % kMaxGroup]);
  __syncthreads();
  if (threadIdx.x < kMaxGroup) {
    float l = 0.f;
    for (int k = 0; k < nparts; k++) l = fmaf(wk[k * kMaxGroup + threadIdx.x], lk[k * kMaxGroup + threadIdx.x], l);
    mxs[kMaxGroup + threadIdx.x] = l;
  }
  float acc[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; h++) acc[h] = 0.f;
  auto add = [&](int k, const float4& o0, const float4& o1) {
    const float4 w0 = *reinterpret_cast<const float4*>(wk + k * kMaxGroup);
    const float4 w1 = *reinterpret_cast<const float4*>(wk + k * kMaxGroup + 4);
    acc[0] = fmaf(w0.x, o0.x, acc[0]); acc[1] = fmaf(w0.y, o0.y, acc[1]);
    acc[2] = fmaf(w0.z, o0.z, acc[2]); acc[3] = fmaf(w0.w, o0.w, acc[3]);
    acc[4] = fmaf(w1.x, o1.x, acc[4]); acc[5] = fmaf(w1.y, o1.y, acc[5]);
    acc[6] = fmaf(w1.z, o1.z, acc[6]); acc[7] = fmaf(w1.w, o1.w, acc[7]);
  };
#pragma unroll
  for (int k = 0; k < kPre; k++)
    if (k < nparts) add(k, ov[k][0], ov[k][1]);
#pragma unroll 4
  for (int k = kPre; k < nparts; k++) {
    const float4 v0 = __ldcg(reinterpret_cast<const float4*>(oc + (size_t)k * kPartFloats));
    const float4 v1 = __ldcg(reinterpret_cast<const float4*>(oc + (size_t)k * kPartFloats + 4));
    add(k, v0, v1);
  }
  __syncthreads();  // the sums of w L
#pragma unroll
  for (int h = 0; h < kMaxGroup; h++)
    if (h < G) outp[h * kHeadDim + c] = acc[h] / mxs[kMaxGroup + h];
  if (threadIdx.x == 0) a.counters[s] = 0;
}

}  // namespace
}  // namespace kvq
