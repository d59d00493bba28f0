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
//   sum_t p_t v^_t = (sum_t p_t R_t (c_t - h)) / (2^b-1) + sum_t p_t Z'_t,
//   h = 2^(b-1), Z'_t = Z_t + R_t h / (2^b-1)  (codes centred: the MMAs sum
//   P_t c_t and the h sum_t P_t over the same fp16 P_t is taken off in fp32),
// so the raw codes go straight into tensor-core operands:
//   QK^T: int8 mma.sync.m16n8k32, A = 16 tokens x 32 Key channels of codes
//   (byte quads, each code moved to the top of its byte: c 2^(8-b), exact in
//   u8), B = the query as an exact per-head int16, q' = s_h (256 hi + lo)
//   with hi s8 and lo u8, two MMAs on the same A registers, int32
//   accumulation (no rounding until one int -> float conversion per score);
//   PV: fp16 mma.sync.m16n8k16, A = 16 channels x 16 tokens of V codes,
//   each pair masked in place by one AND and read as binary16 subnormals
//   (c 2^(e-24): the code bits are the mantissa of a number whose exponent
//   field is zero),
//   B = p R (transposed from the score fragment with movmatrix).
// 16-bit codes go in as two bytes (Keys) or two fp16 halves (Values).

// Work split: each stream is cut into `splits` slices of 16-token groups,
// one CTA per slice (the host picks `splits` so the grid fills the GPU in
// whole waves; the slices are equal, or weighted as described below).  The CTA's four warps take contiguous quarters of the
// slice; each warp streams its quarter through its own ring of shared-memory
// stages filled by cp.async.bulk (TMA bulk copies) on mbarriers, a few KiB
// ahead of its math, and keeps its own online-softmax state.  The warps merge
// in shared memory; a stream cut into several slices leaves one partial
// (max, sum, unnormalised output) per CTA in the workspace, and the last CTA
// to finish the stream (atomic ticket, no waiting) merges them with
// log-sum-exp weights.  Every mbarrier wait is bounded in time; a kernel that
// gives up sets the cache's error flag and returns normally.
//
// Per-channel Key groups (CHAN = true): a Key's range and zero belong to a
// channel of a 128-token block, so they move from the token side of the dot
// product to the query side.  Warps take whole blocks and walk them in
// logical order; per block a warp rebuilds the query operand (a 24-bit
// integer per head, see chan_block) from the block's (R, Z) words, which the
// block's first chunk brings along with its codes.  Values are unchanged.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_decode_common.cuh"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 2;                 // per warp
constexpr int kStageCode = 4096;           // code bytes per stage (K and V parts of whole groups)
constexpr int kStageMeta = 512;            // meta bytes per stage (128 per group)
constexpr int kWarpSmem = kStages * (kStageCode + kStageMeta);
constexpr int kCtasPerSm = 4;
constexpr int kQfBytes = 4 * 32 * 16;      // q' B fragments: [k-block][lane] x (hi b0, hi b1, lo b0, lo b1)
constexpr int kSmemBytes = kWarps * kWarpSmem + kQfBytes + 3 * kWarps * kMaxGroup * 4 + kWarps * kStages * 8 + 16 +
                           2 * kMaxGroup * 4;
// Per-channel Key groups: q' = q lambda qscale in fp32 for the whole kernel,
// and per warp the int16 B fragments, scales and zero terms of its block.
constexpr int kChanSmem = kMaxGroup * kHeadDim * 4 + kWarps * kQfBytes + kWarps * kQfBytes / 2 + 2 * kWarps * kMaxGroup * 4;
static_assert(kSmemBytes % 16 == 0, "the channel area starts 16-byte aligned");
static_assert(kQfBytes >= kWarps * kHeadDim * 4, "per-warp block (R, Z) words fit the per-token fragment area");
// Scratch of the fused append in a warp's second code stage (unused until the
// main loop; warp 0's holds q, lambda and the channel order below this).
constexpr int kAppScratch = 3072;
static_assert(kAppScratch >= 2 * kMaxGroup * kHeadDim + 4 * kHeadDim + kHeadDim, "clear of q, lambda, order");
static_assert(kAppScratch + 2 * kHeadDim <= kStageCode, "the scratch fits the stage");

// -------------------------------------------------------- group pieces

// Scores of NG 16-token groups: D[n][token][head] = sum over Key channels of
// A * q'_int, with A = c 2^(8 - BITS) (BITS <= 8) or the 16-bit code itself,
// and q'_int = 256 hi + lo the per-head int16 query (hi: s8, lo: u8); every
// product and sum is exact in int32.  The k-block loop is outermost so each
// q' fragment is loaded once for all groups.
// QP = 3 (per-channel Key groups): the query operand is a 24-bit integer
// 65536 hi + 256 mid + lo (hi s8; mid, lo u8 in qfl3), three MMAs per A.
template <int BITS, int NG, int QP>
__device__ __forceinline__ void qk_groups(const uint32_t* const (&ku)[NG], const uint4* qfl, const uint2* qfl3,
                                          float (&d)[NG][4]) {
  if constexpr (BITS == 16 && QP == 3) {
    int hh[NG][4], hm[NG][4], hl[NG][4], lh[NG][4], lm[NG][4], ll[NG][4];
#pragma unroll
    for (int n = 0; n < NG; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) hh[n][e] = hm[n][e] = hl[n][e] = lh[n][e] = lm[n][e] = ll[n][e] = 0;
#pragma unroll
    for (int sb = 0; sb < 4; sb++) {
      const uint4 q4 = qfl[32 * sb];
      const uint2 q2 = qfl3[32 * sb];
#pragma unroll
      for (int n = 0; n < NG; n++) {
        const uint2 w00 = *reinterpret_cast<const uint2*>(ku[n] + 4 * sb);
        const uint2 w01 = *reinterpret_cast<const uint2*>(ku[n] + 4 * sb + 2);
        const uint2 w10 = *reinterpret_cast<const uint2*>(ku[n] + 16 + 4 * sb);
        const uint2 w11 = *reinterpret_cast<const uint2*>(ku[n] + 16 + 4 * sb + 2);
        const uint32_t l0 = __byte_perm(w00.x, w00.y, 0x6420), h0 = __byte_perm(w00.x, w00.y, 0x7531);
        const uint32_t l1 = __byte_perm(w10.x, w10.y, 0x6420), h1 = __byte_perm(w10.x, w10.y, 0x7531);
        const uint32_t l2 = __byte_perm(w01.x, w01.y, 0x6420), h2 = __byte_perm(w01.x, w01.y, 0x7531);
        const uint32_t l3 = __byte_perm(w11.x, w11.y, 0x6420), h3 = __byte_perm(w11.x, w11.y, 0x7531);
        imma_s8(hh[n], h0, h1, h2, h3, q4.x, q4.y);
        imma_u8(hm[n], h0, h1, h2, h3, q4.z, q4.w);
        imma_u8(hl[n], h0, h1, h2, h3, q2.x, q2.y);
        imma_s8(lh[n], l0, l1, l2, l3, q4.x, q4.y);
        imma_u8(lm[n], l0, l1, l2, l3, q4.z, q4.w);
        imma_u8(ll[n], l0, l1, l2, l3, q2.x, q2.y);
      }
    }
#pragma unroll
    for (int n = 0; n < NG; n++)
#pragma unroll
      for (int e = 0; e < 4; e++)
        d[n][e] = 256.0f * ((float)hh[n][e] * 65536.0f + (float)hm[n][e] * 256.0f + (float)hl[n][e]) +
                  ((float)lh[n][e] * 65536.0f + (float)lm[n][e] * 256.0f + (float)ll[n][e]);
  } else if constexpr (BITS == 16) {
    int hh[NG][4], hl[NG][4], lh[NG][4], ll[NG][4];
#pragma unroll
    for (int n = 0; n < NG; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) hh[n][e] = hl[n][e] = lh[n][e] = ll[n][e] = 0;
#pragma unroll
    for (int sb = 0; sb < 4; sb++) {
      const uint4 q4 = qfl[32 * sb];
#pragma unroll
      for (int n = 0; n < NG; n++) {
        // quad Q = 8x + 2s + r spans words 2Q (members 0, 1) and 2Q + 1 (members 2, 3)
        const uint2 w00 = *reinterpret_cast<const uint2*>(ku[n] + 4 * sb);            // x 0, r 0
        const uint2 w01 = *reinterpret_cast<const uint2*>(ku[n] + 4 * sb + 2);        // x 0, r 1
        const uint2 w10 = *reinterpret_cast<const uint2*>(ku[n] + 16 + 4 * sb);       // x 1, r 0
        const uint2 w11 = *reinterpret_cast<const uint2*>(ku[n] + 16 + 4 * sb + 2);   // x 1, r 1
        const uint32_t l0 = __byte_perm(w00.x, w00.y, 0x6420), h0 = __byte_perm(w00.x, w00.y, 0x7531);
        const uint32_t l1 = __byte_perm(w10.x, w10.y, 0x6420), h1 = __byte_perm(w10.x, w10.y, 0x7531);
        const uint32_t l2 = __byte_perm(w01.x, w01.y, 0x6420), h2 = __byte_perm(w01.x, w01.y, 0x7531);
        const uint32_t l3 = __byte_perm(w11.x, w11.y, 0x6420), h3 = __byte_perm(w11.x, w11.y, 0x7531);
        imma_s8(hh[n], h0, h1, h2, h3, q4.x, q4.y);
        imma_u8(hl[n], h0, h1, h2, h3, q4.z, q4.w);
        imma_s8(lh[n], l0, l1, l2, l3, q4.x, q4.y);
        imma_u8(ll[n], l0, l1, l2, l3, q4.z, q4.w);
      }
    }
#pragma unroll
    for (int n = 0; n < NG; n++)
#pragma unroll
      for (int e = 0; e < 4; e++)
        d[n][e] = 256.0f * (float)(hh[n][e] * 256 + hl[n][e]) + (float)(lh[n][e] * 256 + ll[n][e]);
  } else {
    uint32_t u[NG][2 * BITS];
#pragma unroll
    for (int n = 0; n < NG; n++) {
#pragma unroll
      for (int i = 0; i < 2 * BITS; i += 4) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(ku[n] + i);
        u[n][i] = w4.x; u[n][i + 1] = w4.y; u[n][i + 2] = w4.z; u[n][i + 3] = w4.w;
      }
    }
    int ah[NG][4], al[NG][4], a3[QP == 3 ? NG : 1][4];
#pragma unroll
    for (int n = 0; n < NG; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) ah[n][e] = al[n][e] = 0;
    if constexpr (QP == 3) {
#pragma unroll
      for (int n = 0; n < NG; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) a3[n][e] = 0;
    }
#define KVQ_QK(S)                                                                                    \
  {                                                                                                  \
    const uint4 q4 = qfl[32 * S];                                                                    \
    _Pragma("unroll") for (int n = 0; n < NG; n++) {                                                \
      const uint32_t a0 = quad_reg<BITS, S, 0, 0>(u[n]), a1 = quad_reg<BITS, S, 1, 0>(u[n]);         \
      const uint32_t a2 = quad_reg<BITS, S, 0, 1>(u[n]), a3r = quad_reg<BITS, S, 1, 1>(u[n]);        \
      imma_s8(ah[n], a0, a1, a2, a3r, q4.x, q4.y);                                                   \
      imma_u8(al[n], a0, a1, a2, a3r, q4.z, q4.w);                                                   \
      if constexpr (QP == 3) {                                                                       \
        const uint2 q2 = qfl3[32 * S];                                                               \
        imma_u8(a3[n], a0, a1, a2, a3r, q2.x, q2.y);                                                 \
      }                                                                                              \
    }                                                                                                \
  }
    KVQ_QK(0) KVQ_QK(1) KVQ_QK(2) KVQ_QK(3)
#undef KVQ_QK
#pragma unroll
    for (int n = 0; n < NG; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) {
        if constexpr (QP == 3)
          d[n][e] = (float)ah[n][e] * 65536.0f + (float)al[n][e] * 256.0f + (float)a3[n][e];
        else
          d[n][e] = (float)(ah[n][e] * 256 + al[n][e]);
      }
  }
}

// o[channel rows][heads] += V^T codes x P for NG groups (B fragments b0[n]:
// tokens 2t, 2t+1, b1[n]: tokens 2t+8, 2t+9 of head g).
template <int BITS, int NG>
__device__ __forceinline__ void pv_groups(const uint32_t* const (&vu)[NG], const uint32_t (&b0)[NG],
                                          const uint32_t (&b1)[NG], float (&o)[8][4]) {
  if constexpr (BITS == 16) {
    uint32_t b0l[NG], b1l[NG];
#pragma unroll
    for (int n = 0; n < NG; n++) {
      b0l[n] = hfma2_u(b0[n], 0x1c001c00u, 0u);  // / 256
      b1l[n] = hfma2_u(b1[n], 0x1c001c00u, 0u);
    }
#pragma unroll
    for (int sb = 0; sb < 8; sb++) {
#pragma unroll
      for (int n = 0; n < NG; n++) {
        const uint2 w0 = *reinterpret_cast<const uint2*>(vu[n] + 2 * sb);       // u = 0
        const uint2 w1 = *reinterpret_cast<const uint2*>(vu[n] + 16 + 2 * sb);  // u = 1
        mma(o[sb], widen16_hi(w0.x), widen16_hi(w0.y), widen16_hi(w1.x), widen16_hi(w1.y), b0[n], b1[n]);
        mma(o[sb], widen16_lo(w0.x), widen16_lo(w0.y), widen16_lo(w1.x), widen16_lo(w1.y), b0l[n], b1l[n]);
      }
    }
  } else {
    uint32_t u[NG][2 * BITS], u8[NG][2 * BITS];
#pragma unroll
    for (int n = 0; n < NG; n++) {
#pragma unroll
      for (int i = 0; i < 2 * BITS; i += 4) {
        const uint4 q4 = *reinterpret_cast<const uint4*>(vu[n] + i);
        u[n][i] = q4.x; u[n][i + 1] = q4.y; u[n][i + 2] = q4.z; u[n][i + 3] = q4.w;
      }
#pragma unroll
      for (int i = 0; i < 2 * BITS; i++) u8[n][i] = u[n][i] >> 8;
    }
#define KVQ_PV(S)                                                                                      \
  _Pragma("unroll") for (int n = 0; n < NG; n++) {                                                    \
    mma(o[S], pair_at<BITS, S, 0, 0>(u[n], u8[n]), pair_at<BITS, S, 0, 1>(u[n], u8[n]),               \
        pair_at<BITS, S, 1, 0>(u[n], u8[n]), pair_at<BITS, S, 1, 1>(u[n], u8[n]), b0[n], b1[n]);         \
  }
    KVQ_PV(0) KVQ_PV(1) KVQ_PV(2) KVQ_PV(3) KVQ_PV(4) KVQ_PV(5) KVQ_PV(6) KVQ_PV(7)
#undef KVQ_PV
  }
}

// Online-softmax state of one warp for the heads 2t, 2t+1 of its lanes.
struct Soft {
  float m0, m1;
  float2 l, pz;  // heads 2t, 2t+1
  float o[8][4];
};

// NG consecutive groups of one stage (cs, ms point at the first): scores,
// one shared running-max update, probabilities, then P V.  valid0: valid
// tokens from the first group on (FULL: all NG groups are full).  FIRST: the
// warp's first group (no running max yet: scores are taken relative to 0 and
// the max is set from them; o, l and pz are still zero).
template <int BITS, int NG, bool FULL, bool CHAN, bool FIRST = false>
__device__ __forceinline__ void process_groups(const uint8_t* cs, const uint2* ms, int valid0, int lane,
                                               const uint4* qfl, const uint2* qfl3, float ks0, float ks1, float sig0,
                                               float sig1, Soft& st) {
  constexpr int kGroupBytes = 512 * BITS, kPart = 256 * BITS;
  constexpr float kVMid = (float)(1u << (BITS - 1)) / (float)((1u << BITS) - 1u);
  const int g = lane >> 2;
  const uint32_t* ku[NG];
  const uint32_t* vu[NG];
#pragma unroll
  for (int n = 0; n < NG; n++) {
    ku[n] = reinterpret_cast<const uint32_t*>(cs + n * kGroupBytes + lane * unit_bytes(BITS));
    vu[n] = reinterpret_cast<const uint32_t*>(cs + n * kGroupBytes + kPart + lane * unit_bytes(BITS));
  }
  float d[NG][4];
  qk_groups<BITS, NG, CHAN ? 3 : 2>(ku, qfl, qfl3, d);
  // Scores relative to the running max: x = R ks_h d + (Z sum(q'_h) - m),
  // ks_h = (q' scale of head h) / (code scale).  Per-channel Key groups: the
  // block's ranges are inside the query operand and its zeros in sig, so
  // x = ks_h d + sig_h - m (R and Z of the token read as 1).
  // The warp's first group takes its scores relative to 0.
  const float me0 = FIRST ? 0.f : st.m0, me1 = FIRST ? 0.f : st.m1;
  float x[NG][4], zv[NG][2];
  uint32_t rv2[NG][2];  // (R^V, R^V) of tokens g and g+8 as half2
  const float2 ks = make_float2(ks0, ks1), sg = make_float2(sig0, sig1), nme = make_float2(-me0, -me1);
#pragma unroll
  for (int n = 0; n < NG; n++) {
    const uint2 mga = ms[n * 16 + g], mgb = ms[n * 16 + g + 8];
    const float2 ka = CHAN ? make_float2(1.f, 1.f) : __half22float2(*reinterpret_cast<const __half2*>(&mga.x));
    const float2 kb = CHAN ? make_float2(1.f, 1.f) : __half22float2(*reinterpret_cast<const __half2*>(&mgb.x));
    // heads 2t, 2t+1 at once: x = (R ks) d + (Z sig - m), the same IEEE steps as one head at a time
    const float2 xa = fma2(mul2(splat2(ka.x), ks), make_float2(d[n][0], d[n][1]), fma2(splat2(ka.y), sg, nme));  // token g
    const float2 xb = fma2(mul2(splat2(kb.x), ks), make_float2(d[n][2], d[n][3]), fma2(splat2(kb.y), sg, nme));  // token g+8
    x[n][0] = xa.x; x[n][1] = xa.y;
    x[n][2] = xb.x; x[n][3] = xb.y;
    // Value zero of tokens g, g+8 for centred codes: Z + R 2^(b-1) / (2^b - 1)
    const float2 va = __half22float2(*reinterpret_cast<const __half2*>(&mga.y));
    const float2 vb = __half22float2(*reinterpret_cast<const __half2*>(&mgb.y));
    const float2 z2 = fma2(make_float2(va.x, vb.x), splat2(kVMid), make_float2(va.y, vb.y));
    zv[n][0] = z2.x;
    zv[n][1] = z2.y;
    rv2[n][0] = __byte_perm(mga.y, 0, 0x1010);  // low half twice
    rv2[n][1] = __byte_perm(mgb.y, 0, 0x1010);
  }
  if constexpr (!FULL) {
    if (valid0 < 16 * NG) {  // warp-uniform: only the last group of a stream's partial tile
#pragma unroll
      for (int n = 0; n < NG; n++) {
        const int valid = valid0 - 16 * n;
        if (g >= valid) {
          x[n][0] = x[n][1] = -INFINITY;
          rv2[n][0] = 0u;
          zv[n][0] = 0.f;
        }
        if (g + 8 >= valid) {
          x[n][2] = x[n][3] = -INFINITY;
          rv2[n][1] = 0u;
          zv[n][1] = 0.f;
        }
      }
    }
  }
  float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
#pragma unroll
  for (int n = 1; n < NG; n++) {
    mx0 = fmaxf(mx0, fmaxf(x[n][0], x[n][2]));
    mx1 = fmaxf(mx1, fmaxf(x[n][1], x[n][3]));
  }
  // Lazy rebase: the running max moves only when a score exceeds it by more
  // than kRebase (log2 units), so p = 2^(s - m) <= 2^kRebase.  Whether any
  // lane needs it is one vote; the maxima over the tokens are only formed
  // when it does.
  if (FIRST || __any_sync(0xffffffffu, fmaxf(mx0, mx1) > kRebase)) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    // new max = old max + shift (the first group: its own max, relative to 0)
    const float d0 = FIRST ? mx0 : fmaxf(mx0, 0.f);
    const float d1 = FIRST ? mx1 : fmaxf(mx1, 0.f);
    if constexpr (!FIRST) {
      const float a0 = ex2(-d0), a1 = ex2(-d1);  // in (0, 1]
#pragma unroll
      for (int sb = 0; sb < 8; sb++) {
        st.o[sb][0] *= a0; st.o[sb][2] *= a0;
        st.o[sb][1] *= a1; st.o[sb][3] *= a1;
      }
      st.l = mul2(st.l, make_float2(a0, a1));
      st.pz = mul2(st.pz, make_float2(a0, a1));
    }
    st.m0 = me0 + d0;
    st.m1 = me1 + d1;
#pragma unroll
    for (int n = 0; n < NG; n++) {
      x[n][0] -= d0; x[n][2] -= d0;
      x[n][1] -= d1; x[n][3] -= d1;
    }
  }
  uint32_t b0[NG], b1[NG];
#pragma unroll
  for (int n = 0; n < NG; n++) {
    const float p00 = ex2(x[n][0]), p01 = ex2(x[n][1]);
    const float p10 = ex2(x[n][2]), p11 = ex2(x[n][3]);
    const float2 pa = make_float2(p00, p01), pb = make_float2(p10, p11);  // tokens g, g+8
    st.l = add2(st.l, add2(pa, pb));
    st.pz = fma2(pa, splat2(zv[n][0]), fma2(pb, splat2(zv[n][1]), st.pz));
    // P = p R^V in fp16, transposed to the B fragment (tokens 2t, 2t+1 / 2t+8, 2t+9 of head g)
    const uint32_t Pa = hmul2_u(pack_h2(p00, p01), rv2[n][0]), Pb = hmul2_u(pack_h2(p10, p11), rv2[n][1]);
    if constexpr (BITS <= 8) {
      // the P V MMAs take the codes uncentred: sum_t P_t (c_t - h) = sum_t P_t c_t
      // - h sum_t P_t, the second sum over the same fp16 P
      const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&Pa));
      const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&Pb));
      st.pz = fma2(add2(fa, fb), splat2(-kVMid), st.pz);
    }
    b0[n] = movmatrix_t(Pa);
    b1[n] = movmatrix_t(Pb);
  }
  pv_groups<BITS, NG>(vu, b0, b1, st.o);
}

// Per-channel Key groups: the query operand of one 128-token block.  The
// block's Key channel c is Z_c + code R_c / (2^b - 1), so
//   q'.k^_t = sum_c q'_c Z_c + sum_c (q'_c R_c / (2^b - 1)) code_t,c
// and w_c = q'_c R_c / (2^b - 1) takes the place of q' as an exact per-head
// 24-bit integer (scale max|w| / (2^22 - 2)); the first sum is the head's
// zero term.  24 bits, not the 16 of the per-token operand: w carries both
// the migrated query's outlier channels and the same channels' wider ranges,
// so its largest entry is far above the typical one and 16 bits left the
// ordinary channels too coarse (2.4e-3 output error on 2-bit blocks).  The
// warp writes its own B fragments (hi and mid bytes in the per-token layout,
// lo bytes in qfw3), and per head the score scale ks (w scale times the code
// scale of the A operand) and the zero term.  km: the block's 128 (R, Z)
// words, in shared memory.
template <int BITS>
__device__ __forceinline__ void chan_block(const float* s_qp, const uint32_t* km, uint4* qfw, uint2* qfw3, float* wks,
                                        float* wsig, int lane) {
  constexpr float kInvQ = 1.0f / (float)((1u << BITS) - 1u);
  constexpr float kA = BITS >= 8 ? 1.0f : 1.0f / (float)(1 << (8 - BITS));  // A = c 2^(8 - BITS) at b <= 8
  const int tq = (lane >> 2) & 3, sq = lane & 3, hsel = lane >> 4;
  // this lane's channels: 32 sq + 16 hf + 4 tq + i
  float R[2][4], Z[2][4];
#pragma unroll
  for (int hf = 0; hf < 2; hf++) {
    const uint4 w4 = *reinterpret_cast<const uint4*>(km + 32 * sq + 16 * hf + 4 * tq);
    const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      R[hf][i] = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xffffu))) * kInvQ;
      Z[hf][i] = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
    }
  }
#pragma unroll 2
  for (int hp = 0; hp < kMaxGroup / 2; hp++) {
    const int gq = 2 * hp + hsel;  // the 16 lanes of a head cover its 128 channels
    float v[2][4];
    float m = 0.f, zs = 0.f;
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      const float4 q4 = *reinterpret_cast<const float4*>(s_qp + gq * kHeadDim + 32 * sq + 16 * hf + 4 * tq);
      const float q[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        v[hf][i] = q[i] * R[hf][i];
        m = fmaxf(m, fabsf(v[hf][i]));
        zs = fmaf(q[i], Z[hf][i], zs);
      }
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      zs += __shfl_xor_sync(0xffffffffu, zs, o);
    }
    constexpr float kQMax = 4194302.0f;  // 2^22 - 2
    // any inv close to kQMax / m works: |w inv| < 2^22 - 1 then, and the score
    // scale below is the same m / kQMax the MMAs' integers are read with
    // (qi / inv ~ w up to half a step, ks d = sum w c up to the rounding of
    // inv).  qi = w inv rounded to an integer by one fma with 1.5 * 2^23: the
    // sum lies in [2^23, 2^24), where floats are the integers, and its bits
    // minus those of 1.5 * 2^23 are qi as a 32-bit two's-complement integer.
    const float inv = m > 0.f ? kQMax * __frcp_rn(m) : 0.f;
    uint32_t hb[2], mb[2], lb[2];
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      uint32_t q[4];
#pragma unroll
      for (int i = 0; i < 4; i++) q[i] = __float_as_uint(fmaf(v[hf][i], inv, 12582912.0f)) - 0x4B400000u;
      // bytes 0, 1, 2 of the four 24-bit two's-complement integers (byte 2 is the s8 high part)
      const uint32_t ab = __byte_perm(q[0], q[1], 0x5140), cd = __byte_perm(q[2], q[3], 0x5140);
      lb[hf] = __byte_perm(ab, cd, 0x5410);
      mb[hf] = __byte_perm(ab, cd, 0x7632);
      hb[hf] = __byte_perm(__byte_perm(q[0], q[1], 0x0062), __byte_perm(q[2], q[3], 0x0062), 0x5410);
    }
    qfw[sq * 32 + 4 * gq + tq] = make_uint4(hb[0], hb[1], mb[0], mb[1]);
    qfw3[sq * 32 + 4 * gq + tq] = make_uint2(lb[0], lb[1]);
    if ((lane & 15) == 0) {
      wks[gq] = m / kQMax * kA;
      wsig[gq] = zs;
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ kernel

struct WarpSmem {
  uint8_t code[kStages][kStageCode];
  uint8_t meta[kStages][kStageMeta];
};

template <int BITS, bool CHAN>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  WarpSmem* ws = reinterpret_cast<WarpSmem*>(smem);
  uint4* qf = reinterpret_cast<uint4*>(smem + kWarps * kWarpSmem);     // [8][32]
  float* w_m = reinterpret_cast<float*>(qf + 4 * 32);                 // [warps][8]
  float* w_l = w_m + kWarps * kMaxGroup;
  float* w_pz = w_l + kWarps * kMaxGroup;
  uint64_t* bars = reinterpret_cast<uint64_t*>(w_pz + kWarps * kMaxGroup);  // [warps][stages]
  volatile int* flags = reinterpret_cast<volatile int*>(bars + kWarps * kStages);  // [0] abort, [1] last
  unsigned* s_amax = reinterpret_cast<unsigned*>(const_cast<int*>(flags) + 4);  // [8] bits of max|q'| per head
  int* s_isum = reinterpret_cast<int*>(s_amax + kMaxGroup);                     // [8] sum of q_int per head
  // per-channel Key groups only (the launch sizes the area): q' [8][128],
  // per-warp B fragments [warps][4][32], scales and zero terms [warps][8]
  float* s_qp = reinterpret_cast<float*>(smem + kSmemBytes);
  uint4* qfw = reinterpret_cast<uint4*>(s_qp + kMaxGroup * kHeadDim);
  uint2* qfw3 = reinterpret_cast<uint2*>(qfw + kWarps * 4 * 32);
  float* w_ks = reinterpret_cast<float*>(qfw3 + kWarps * 4 * 32);
  float* w_sig = w_ks + kWarps * kMaxGroup;

  constexpr int kGroupBytes = 512 * BITS;
  constexpr bool kWide = BITS == 16;            // a 16-bit group (8 KiB) takes every code stage
  constexpr int kS = kWide ? 1 : kStages;       // stages in use
  constexpr int kChunkGroups = kWide ? 1 : kStageCode / kGroupBytes;
  constexpr float kCScale = (BITS == 16 ? 256.0f : 1.0f) / (float)((1u << BITS) - 1u);
  // QK products carry the code as A = c 2^(8 - BITS) (BITS <= 8) or c (16)
  constexpr float kKCode = 1.0f / ((float)((1u << BITS) - 1u) * (float)(BITS >= 8 ? 1 : 1 << (8 - BITS)));

  const Fill f = a.fill;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = a.group;
  const int s = blockIdx.x / a.splits, split = blockIdx.x - s * a.splits;
  // Per-channel Key groups split the stream by whole 128-token blocks (8 groups).
  const long long units = CHAN ? f.gps / 8 : f.gps, per = CHAN ? 8 : 1;
  // Slices are equal, or, in a one-wave launch (a.rank_sms > 0), weighted by
  // the order in which the CTAs reach their SMs: CTA i is the (i / SMs)-th on
  // its SM, and the warp schedulers favour older warps, so with equal slices an
  // SM's first CTA ends its loop well before its fourth.  Weights 20 : 19 : 18 :
  // 17 even that out; the host asks for them only with >= 2 units per CTA, so
  // every slice still holds at least one.
  long long ca, cb;
  if (a.rank_sms > 0) {
    long long wsum = 0, wpre = 0;
    for (int k = 0; k < a.splits; k++) {
      const int w = 20 - min(3, (s * a.splits + k) / a.rank_sms);
      wpre += k < split ? w : 0;
      wsum += w;
    }
    ca = units * wpre / wsum;
    cb = units * (wpre + 20 - min(3, (int)blockIdx.x / a.rank_sms)) / wsum;
  } else {
    ca = units * split / a.splits;
    cb = units * (split + 1) / a.splits;
  }
  const long long wa = per * (ca + (cb - ca) * warp / kWarps), wb = per * (ca + (cb - ca) * (warp + 1) / kWarps);
  WarpSmem& my = ws[warp];
  const uint32_t bar0 = smem_u32(bars + warp * kStages);
  // per-channel Key groups: this warp's copy of its block's (R, Z) words, in
  // the per-token query fragments' area (unused then)
  uint32_t* kmcb = reinterpret_cast<uint32_t*>(qf) + warp * kHeadDim;

  if (threadIdx.x == 0) {
    flags[0] = 0;
    flags[1] = 0;
  }
  if (lane == 0) {
    for (int i = 0; i < kS; i++) mbar_init(bar0 + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // lambda is fixed while kernels run on the block, so it is fetched before
  // waiting for the previous kernel.  Per-channel Key groups stage q and
  // lambda in shared memory (in warp 0's second code stage, unused until the
  // main loop starts); otherwise each lane loads the channels it quantizes:
  // head gq = 2 warp + lane / 16, channels 32 sq + 16 hf + 4 tq + i.
  const int b = s / a.kv_heads, j = s - b * a.kv_heads;
  __nv_bfloat16* s_q = reinterpret_cast<__nv_bfloat16*>(ws[0].code[kStages - 1]);  // [8][128]
  float* s_lam = reinterpret_cast<float*>(s_q + kMaxGroup * kHeadDim);               // [128]
  const int gq = 2 * warp + (lane >> 4), tq = (lane >> 2) & 3, sq = lane & 3;
  float4 lam4[2] = {make_float4(1.f, 1.f, 1.f, 1.f), make_float4(1.f, 1.f, 1.f, 1.f)};
  if constexpr (CHAN) {
    if (warp == 1) {
      const float4 lv = a.lam ? __ldg(reinterpret_cast<const float4*>(a.lam + (size_t)j * kHeadDim) + lane)
                              : make_float4(1.f, 1.f, 1.f, 1.f);
      reinterpret_cast<float4*>(s_lam)[lane] = lv;
    }
  } else if (a.lam) {
#pragma unroll
    for (int hf = 0; hf < 2; hf++)
      lam4[hf] = __ldg(reinterpret_cast<const float4*>(a.lam + (size_t)j * kHeadDim + 32 * sq + 16 * hf + 4 * tq));
  }
  // ---- chunk iterator: the warp walks its groups tile by tile (per-channel
  // Key groups: lane 0, in logical order, publishing per-stage descriptors) ----
  int left = (int)(wb - wa);  // groups this warp still has to issue
  int it_tile = 0, it_grp = 0, it_tgroups = 0, it_tvalid = 0;
  long long v_next = wa;  // per-channel Key groups: next group in logical order
  if (!CHAN && left > 0) {
    const GroupLoc loc = locate_group(f, wa);
    it_tile = loc.tile;
    it_grp = loc.grp;
    it_tgroups = loc.tile_groups;
    it_tvalid = loc.tile < f.k ? f.p : (loc.tile == f.k ? f.h + f.r : f.h);
  }
  const uint8_t* sbase = a.codes + (size_t)s * f.nt * kTileBytes;
  const uint32_t* mbase = a.meta + (size_t)s * f.nt * f.pf * 2;
  // Per-channel Key groups: all lanes step the same iterator in logical order.
  // Group v holds tokens 16v .. 16v+15, which arrived in epoch e and sit in
  // slots [h_e, h_e + ee_e) of tile (16v - start_e) / ee_e.  A chunk gathers
  // whole or partial runs (one tile's slots of an epoch, contiguous) up to
  // kChunkGroups groups without leaving its 128-token block (runs never
  // straddle blocks: epochs start on block boundaries and a run is 32, 64 or
  // 128 tokens at a multiple of its length); x = groups, y = block, and
  // `first` when it starts the block (it then also fetches the block's Key
  // (R, Z) words).  ep_e, the epoch of v_next, only moves forward.
  int ep_e = 0;
  struct Runs {
    uint32_t r[kChunkGroups];  // tile << 10 | first group << 4 | groups (tiles per stream < 2^22)
    bool first;
  };
  auto next_chunk_chan = [&](Runs& ru) -> int2 {
    int ng = 0;
    const long long v0 = v_next;
#pragma unroll
    for (int r = 0; r < kChunkGroups; r++) {
      ru.r[r] = 0u;
      if (ng < kChunkGroups && left > 0 && (ng == 0 || (v_next & 7) != 0)) {
        const int i = 16 * (int)v_next;
        while (ep_e + 1 < a.ep.n && i >= a.ep.start[ep_e + 1]) ep_e++;
        const int m = i - a.ep.start[ep_e], lg = a.ep.lg_ee[ep_e];
        const int tile = m >> lg, off = m & ((1 << lg) - 1);
        int take = ((1 << lg) - off) >> 4;
        take = min(min(take, kChunkGroups - ng), left);
        take = min(take, 8 - (int)(v_next & 7));  // stay inside the block
        ru.r[r] = ((uint32_t)tile << 10) | ((uint32_t)((a.ep.h[ep_e] + off) >> 4) << 4) | (uint32_t)take;
        ng += take;
        left -= take;
        v_next += take;
      }
    }
    ru.first = (v0 & 7) == 0;
    return make_int2(ng, (int)(v0 >> 3));
  };
  auto copy_chunk_chan = [&](int st, int2 d, const Runs& ru) {
    if (lane == 0 && d.x > 0) {
      const uint32_t bar = bar0 + 8 * st;
      mbar_expect_tx(bar, (uint32_t)d.x * (kGroupBytes + 128u) + (ru.first ? 4u * kHeadDim : 0u));
      int done = 0;
#pragma unroll
      for (int r = 0; r < kChunkGroups; r++) {
        const uint32_t n = ru.r[r] & 15u, g = (ru.r[r] >> 4) & 63u;
        const size_t tile = ru.r[r] >> 10;
        if (n > 0) {
          bulk_g2s(smem_u32(my.code[st] + done * kGroupBytes), sbase + tile * kTileBytes + (size_t)g * kGroupBytes,
                   n * kGroupBytes, bar);
          bulk_g2s(smem_u32(my.meta[st] + done * 128), mbase + (tile * f.pf + (size_t)g * 16) * 2, n * 128u, bar);
          done += (int)n;
        }
      }
      if (ru.first)  // one buffer per warp: a block spans at least two chunks, so the previous block's words are used
        bulk_g2s(smem_u32(kmcb), a.kmc + ((size_t)s * a.blocks_max + (size_t)d.y) * kHeadDim, 4u * kHeadDim, bar);
    }
  };
  // Every other layout: all lanes step the same iterator (the values are
  // warp-uniform) and lane 0 alone issues the copies.  A chunk is up to
  // kChunkGroups groups of one tile; x = groups, y = valid tokens from its
  // first group; coff, moff: its code byte and meta word offsets in the stream.
  auto next_chunk = [&](size_t& coff, size_t& moff) -> int2 {
    if (left <= 0) return make_int2(0, 0);
    const int ng = min(min(it_tgroups - it_grp, kChunkGroups), left);
    const int2 d = make_int2(ng, it_tvalid - 16 * it_grp);
    coff = (size_t)it_tile * kTileBytes + (size_t)it_grp * kGroupBytes;
    moff = ((size_t)it_tile * f.pf + (size_t)it_grp * 16) * 2;
    left -= ng;
    it_grp += ng;
    if (it_grp == it_tgroups) {  // next tile: full, the partial tile k, or a base tile
      it_tile++;
      it_grp = 0;
      it_tgroups = it_tile < f.k ? f.gpt : (it_tile == f.k ? f.gk : f.gh);
      it_tvalid = it_tile < f.k ? f.p : (it_tile == f.k ? f.h + f.r : f.h);
    }
    return d;
  };
  auto copy_chunk = [&](int st, int2 d, size_t coff, size_t moff) {
    if (lane == 0 && d.x > 0) {
      const uint32_t cbytes = (uint32_t)d.x * kGroupBytes, mbytes = (uint32_t)d.x * 128u;
      const uint32_t bar = bar0 + 8 * st;
      mbar_expect_tx(bar, cbytes + mbytes);
      bulk_g2s(smem_u32(my.code[st]), sbase + coff, cbytes, bar);
      bulk_g2s(smem_u32(my.meta[st]), mbase + moff, mbytes, bar);
    }
  };

  // A first chunk that lies wholly in groups no kernel still in flight can
  // be writing (a.safe: before the slots of the most recent append) is
  // fetched before waiting for the previous kernel.
  bool pre = false;
  int2 d0 = make_int2(0, 0);  // the first chunk (double-buffered layouts)
  size_t c0 = 0, m0off = 0;
  if constexpr (!kWide && !CHAN) {
    d0 = next_chunk(c0, m0off);
    if (d0.x > 0 && wa + d0.x <= a.safe) {
      copy_chunk(0, d0, c0, m0off);
      pre = true;
    }
  }
  // the rest of the cache, q and the counters may be written by earlier
  // kernels -- unless this launch directly follows another decode launch of
  // the same call, which triggers this one only after its own wait (then
  // everything before that launch is complete).
  // q may be written by an earlier kernel, so it is read only after the wait;
  // an L2 prefetch of its lines before the wait is a hint that reads nothing
  // into registers (the loads after the wait see whatever q holds then).
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.q_heads + (size_t)j * G) * kHeadDim;
  if (CHAN ? (int)threadIdx.x < G * (kHeadDim / 8) : gq < G)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(CHAN ? qb + 8 * threadIdx.x : qb + (size_t)gq * kHeadDim + 32 * sq + 4 * tq));
  if (!a.after_decode) pdl_wait();
  if (a.trigger_early) pdl_launch_dependents();  // a window launch follows: let it fill free SMs now
  uint4 qv = make_uint4(0u, 0u, 0u, 0u);  // per-channel Key groups: 8 bf16 of q, head threadIdx/16, channels 8 (threadIdx%16) ..
  uint2 qv2[2] = {make_uint2(0u, 0u), make_uint2(0u, 0u)};  // otherwise this lane's channels of head gq
  if constexpr (CHAN) {
    if ((int)threadIdx.x < G * (kHeadDim / 8)) qv = reinterpret_cast<const uint4*>(qb)[threadIdx.x];
  } else if (gq < G) {
#pragma unroll
    for (int hf = 0; hf < 2; hf++)
      qv2[hf] = *reinterpret_cast<const uint2*>(qb + (size_t)gq * kHeadDim + 32 * sq + 16 * hf + 4 * tq);
  }

  // ---- fused single-token append: the warp whose range holds the new
  // token's group quantizes and writes the token (K, then V) before it
  // copies any group (a.safe kept the pre-wait copy away from that group) ----
  if (!CHAN && a.app_group >= 0 && wa <= a.app_group && a.app_group < wb) {  // warp-uniform
    uint16_t* sc = reinterpret_cast<uint16_t*>(ws[warp].code[kStages - 1] + kAppScratch);
    const size_t tile = (size_t)s * f.nt + a.app_tile;
#pragma unroll 1
    for (int kv = 0; kv < 2; kv++) {
      const size_t in_off = (((size_t)b * a.kv_heads + j) * kHeadDim) + 4 * lane;  // token 0 of a 1-token call
      const void* src = kv ? a.av : a.ak;
      float x[4];
      if (a.adtype == 1) {
        const float4 f4 = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + in_off);
        x[0] = f4.x; x[1] = f4.y; x[2] = f4.z; x[3] = f4.w;
      } else {
        const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(src) + in_off);
        x[0] = __uint_as_float(raw.x << 16); x[1] = __uint_as_float(raw.x & 0xffff0000u);
        x[2] = __uint_as_float(raw.y << 16); x[3] = __uint_as_float(raw.y & 0xffff0000u);
      }
      if (kv == 0 && a.lam_inv) {
        const float4 li = *reinterpret_cast<const float4*>(a.lam_inv + (size_t)j * kHeadDim + 4 * lane);
        x[0] = __fmul_rn(x[0], li.x); x[1] = __fmul_rn(x[1], li.y);
        x[2] = __fmul_rn(x[2], li.z); x[3] = __fmul_rn(x[3], li.w);
      }
      const uint32_t mw = quantize_group(x, BITS == 16 ? 65535u : (1u << BITS) - 1u, sc, lane);
      __syncwarp();
      uint8_t* gbase = a.codes + tile * kTileBytes + (size_t)(a.app_slot >> 4) * kGroupBytes + (size_t)kv * (kGroupBytes / 2);
      pack_codes<BITS>(gbase, a.app_slot & 15, kv, sc, lane);
      if (lane == 0) a.meta[(tile * f.pf + a.app_slot) * 2 + kv] = mw;
      __syncwarp();  // sc is rewritten for V
    }
    // this warp's own bulk copies (async proxy) must see these writes
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
  }

  // start streaming before the q' set-up so DRAM latency overlaps it
  if constexpr (CHAN) {
    if constexpr (!kWide) {
      Runs ru;
      d0 = next_chunk_chan(ru);
      copy_chunk_chan(0, d0, ru);
    }
  } else if constexpr (!kWide) {
    if (!pre) copy_chunk(0, d0, c0, m0off);
  }
  __syncwarp();

  // ---- q' for this stream: exact int16 per head, as int8 MMA B fragments ----
  // q'_h = q_h * lambda * qscale at the Key channels, then per head h
  //   s_h = max|q'_h| / 32767,  q_int = round(q'_h / s_h) = 256 hi + lo
  // (hi: s8, lo: u8).  The MMAs compute sum A q_int exactly, and sum(q'_h)
  // is taken as s_h sum(q_int), over exactly the values the MMAs use, so
  // (R/(2^b-1)) q'.c + Z sum(q') is the dot product of s_h q_int with the
  // dequantised key.
  if constexpr (CHAN) {  // q' in fp32 for the per-block operands
    reinterpret_cast<uint4*>(s_q)[threadIdx.x] = qv;  // heads >= G are zero
    __syncthreads();
    for (int idx = threadIdx.x; idx < kMaxGroup * kHeadDim; idx += kThreads)
      s_qp[idx] = __bfloat162float(s_q[idx]) * a.qscale * s_lam[idx & (kHeadDim - 1)];
  } else {
    // Warp w quantizes heads 2w and 2w+1: lane L takes head gq = 2w + L/16
    // and writes the B fragment of k-block sq = L%4 for MMA lane 4 gq + tq,
    // tq = (L/4)%4: channels 32 sq + 16 hf + 4 tq + i (hf = 0..1, i = 0..3).
    // The 16 lanes of a head cover its 128 channels.
    float v[2][4];
    float m = 0.f;
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      const float qx[4] = {__uint_as_float(qv2[hf].x << 16), __uint_as_float(qv2[hf].x & 0xffff0000u),
                           __uint_as_float(qv2[hf].y << 16), __uint_as_float(qv2[hf].y & 0xffff0000u)};
      const float lx[4] = {lam4[hf].x, lam4[hf].y, lam4[hf].z, lam4[hf].w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        v[hf][i] = qx[i] * a.qscale * lx[i];
        m = fmaxf(m, fabsf(v[hf][i]));
      }
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float inv = m > 0.f ? 32767.0f / m : 0.f;
    uint32_t hb[2] = {0u, 0u}, lb[2] = {0u, 0u};
    int part = 0;
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int qi = max(-32767, min(32767, __float2int_rn(v[hf][i] * inv)));
        part += qi;
        hb[hf] |= (uint32_t)((qi >> 8) & 0xff) << (8 * i);
        lb[hf] |= (uint32_t)(qi & 0xff) << (8 * i);
      }
    }
    qf[sq * 32 + 4 * gq + tq] = make_uint4(hb[0], hb[1], lb[0], lb[1]);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((lane & 15) == 0) {
      s_amax[gq] = __float_as_uint(m);
      s_isum[gq] = part;
    }
  }
  __syncthreads();
  float ks0 = 0.f, ks1 = 0.f, sig0 = 0.f, sig1 = 0.f;  // heads 2t, 2t+1 (per block with per-channel Keys)
  if constexpr (!CHAN) {
    const float s0 = __uint_as_float(s_amax[2 * t]) / 32767.0f, s1 = __uint_as_float(s_amax[2 * t + 1]) / 32767.0f;
    ks0 = s0 * kKCode;
    ks1 = s1 * kKCode;
    sig0 = s0 * (float)s_isum[2 * t];
    sig1 = s1 * (float)s_isum[2 * t + 1];
  }
  const uint4* qfl = CHAN ? qfw + warp * 4 * 32 + lane : qf + lane;
  const uint2* qfl3 = qfw3 + warp * 4 * 32 + lane;  // per-channel Key groups only
  int cur_blk = -1;  // per-channel Key groups: the block whose operand is in qfw
  // The staging areas (second code stages) are refilled by bulk copies from
  // the first loop iteration on: order the generic accesses before them.
  if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");

  Soft sm;
  sm.m0 = sm.m1 = -INFINITY;
  sm.l = sm.pz = make_float2(0.f, 0.f);
#pragma unroll
  for (int sb = 0; sb < 8; sb++) sm.o[sb][0] = sm.o[sb][1] = sm.o[sb][2] = sm.o[sb][3] = 0.f;

  int2 dA = d0, dB = make_int2(0, 0);  // chunks in stages 0 and 1 (not per-channel Key groups)
  for (int ci = 0;; ci++) {
    const int st = kWide ? 0 : (ci & 1);
    int2 dsc;
    if constexpr (CHAN) {
      Runs ru;
      if constexpr (kWide) {  // one stage: the chunk is fetched and waited for in turn
        dsc = next_chunk_chan(ru);
        copy_chunk_chan(0, dsc, ru);
      } else {  // chunk ci+1 into the stage chunk ci-1 used
        const int2 dn = next_chunk_chan(ru);
        copy_chunk_chan(st ^ 1, dn, ru);
        dsc = st ? dB : dA;
        if (st) dA = dn; else dB = dn;
      }
    } else if constexpr (kWide) {  // one stage: the chunk is fetched and waited for in turn
      size_t co = 0, mo = 0;
      dsc = next_chunk(co, mo);
      copy_chunk(0, dsc, co, mo);
    } else {  // chunk ci+1 into the stage chunk ci-1 used
      size_t co = 0, mo = 0;
      const int2 dn = next_chunk(co, mo);
      copy_chunk(st ^ 1, dn, co, mo);
      dsc = st ? dB : dA;
      if (st) dA = dn; else dB = dn;
    }
    if (dsc.x == 0) break;
    const uint32_t parity = kWide ? (ci & 1) : ((ci >> 1) & 1);
    if (!mbar_wait(bar0 + 8 * st, parity, a.err, flags)) break;
    const uint8_t* cs = my.code[st];
    const uint2* ms = reinterpret_cast<const uint2*>(my.meta[st]);
    // the warp's first group (chunk 0 holds at least one) sets the running max
    const int gi0 = ci == 0 ? 1 : 0;
    if constexpr (CHAN) {  // every group full; dsc.y is the chunk's 128-token block
      if (dsc.y != cur_blk) {
        cur_blk = dsc.y;
        float* wks = w_ks + warp * kMaxGroup;
        float* wsig = w_sig + warp * kMaxGroup;
        chan_block<BITS>(s_qp, kmcb, qfw + warp * 4 * 32, qfw3 + warp * 4 * 32, wks, wsig, lane);
        ks0 = wks[2 * t];
        ks1 = wks[2 * t + 1];
        sig0 = wsig[2 * t];
        sig1 = wsig[2 * t + 1];
      }
      if (ci == 0)
        process_groups<BITS, 1, true, true, true>(cs, ms, 16, lane, qfl, qfl3, ks0, ks1, sig0, sig1, sm);
      int gi = gi0;
      if constexpr (kChunkGroups >= 2) {
        for (; gi + 2 <= dsc.x; gi += 2)
          process_groups<BITS, 2, true, true>(cs + gi * kGroupBytes, ms + gi * 16, 32, lane, qfl, qfl3, ks0, ks1, sig0,
                                              sig1, sm);
      }
      if (gi < dsc.x)
        process_groups<BITS, 1, true, true>(cs + gi * kGroupBytes, ms + gi * 16, 16, lane, qfl, qfl3, ks0, ks1, sig0,
                                            sig1, sm);
    } else if (ci > 0 && dsc.x == kChunkGroups && dsc.y >= 16 * kChunkGroups) {
      // full chunk: fixed offsets, no masking
      // unrolled: one pair's P V and the next pair's QK share a basic block
      constexpr int kNG = kChunkGroups >= 2 ? 2 : 1;
#pragma unroll
      for (int gi = 0; gi < kChunkGroups; gi += kNG)
        process_groups<BITS, kNG, true, false>(cs + gi * kGroupBytes, ms + gi * 16, 16 * kNG, lane, qfl, qfl3, ks0, ks1, sig0,
                                        sig1, sm);
    } else {
      if (ci == 0)
        process_groups<BITS, 1, false, false, true>(cs, ms, dsc.y, lane, qfl, qfl3, ks0, ks1, sig0, sig1, sm);
      for (int gi = gi0; gi < dsc.x; gi++)
        process_groups<BITS, 1, false, false>(cs + gi * kGroupBytes, ms + gi * 16, dsc.y - 16 * gi, lane, qfl, qfl3, ks0,
                                       ks1, sig0, sig1, sm);
    }
    __syncwarp();  // every lane is done with this stage before lane 0 refills it
  }
  float m0 = sm.m0, m1 = sm.m1, l0 = sm.l.x, l1 = sm.l.y, pz0 = sm.pz.x, pz1 = sm.pz.y;
  float (&o)[8][4] = sm.o;

  if (!a.trigger_early) pdl_launch_dependents();  // the next kernel may start to launch while this one merges
  // ---- merge the four warps ----
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
  __syncthreads();  // also: every stage of every warp is consumed (no copy in flight)
  {
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
      M0 = fmaxf(M0, w_m[w * kMaxGroup + 2 * t]);
      M1 = fmaxf(M1, w_m[w * kMaxGroup + 2 * t + 1]);
    }
    const float sc0 = ex2(m0 - M0), sc1 = ex2(m1 - M1);
    float* ob = reinterpret_cast<float*>(my.code[0]);  // this warp's scaled o: [8][128]
#pragma unroll
    for (int sb = 0; sb < 8; sb++) {
      // rows 16sb+g (pair 2sb) and 16sb+g+8 (pair 2sb+1) carry 2^(field_shift - 24) at BITS <= 8
      const float r0 = BITS == 16 ? 1.0f : (float)(1 << (24 - pair_shift<BITS>(2 * sb)));
      const float r1 = BITS == 16 ? 1.0f : (float)(1 << (24 - pair_shift<BITS>(2 * sb + 1)));
      ob[(2 * t) * kHeadDim + 16 * sb + g] = sc0 * r0 * o[sb][0];
      ob[(2 * t + 1) * kHeadDim + 16 * sb + g] = sc1 * r0 * o[sb][1];
      ob[(2 * t) * kHeadDim + 16 * sb + g + 8] = sc0 * r1 * o[sb][2];
      ob[(2 * t + 1) * kHeadDim + 16 * sb + g + 8] = sc1 * r1 * o[sb][3];
    }
  }
  // Per head h (thread h): the CTA's max M over its warps and the
  // e^(m_w - M)-weighted sums L and PZ, in warp 0's free second stage.
  float* fin = reinterpret_cast<float*>(ws[0].code[1]);  // M[8], L[8], PZ[8]
  if (threadIdx.x < kMaxGroup) {
    const int h = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, w_m[w * kMaxGroup + h]);
    float L = 0.f, PZ = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
      const float e = ex2(w_m[w * kMaxGroup + h] - M);
      L += e * w_l[w * kMaxGroup + h];
      PZ += e * w_pz[w * kMaxGroup + h];
    }
    fin[h] = M;
    fin[kMaxGroup + h] = L;
    fin[2 * kMaxGroup + h] = PZ;
  }
  __syncthreads();
  // Final state of this CTA for every head h < G and channel c = thread:
  //   O = sum of the warps' scaled rows (times 2^-e and 1/(2^b-1)) + PZ
  //   (unnormalised), with the head's M and L.
  const int c = threadIdx.x;  // one channel per thread
  static_assert(kThreads == kHeadDim, "one channel per thread");
  float Oc[kMaxGroup], Mh[kMaxGroup], Lh[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; h++) {
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) O += reinterpret_cast<const float*>(ws[w].code[0])[h * kHeadDim + c];
    Oc[h] = O * kCScale + fin[2 * kMaxGroup + h];
    Mh[h] = fin[h];
    Lh[h] = fin[kMaxGroup + h];
  }
  // warp 0's two code stages (free now; the merge weights above are in registers)
  static_assert(kScratchFloats * 4 <= kStages * kStageCode, "the merge scratch fits");
  finish_stream(a, s, split, Oc, Mh, Lh, flags, reinterpret_cast<float*>(ws[0].code[0]));
}

template <int BITS, bool CHAN>
cudaError_t launch_bits(const DecodeArgs& a, cudaStream_t s) {
  constexpr int kBytes = kSmemBytes + (CHAN ? kChanSmem : 0);
  static bool attr_set = false;  // per process and kernel; set before the first launch
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS, CHAN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<BITS, CHAN>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const unsigned grid = (unsigned)(a.batch * a.kv_heads) * (unsigned)a.splits;
  return launch_pdl(decode_kernel<BITS, CHAN>, dim3(grid), dim3(kThreads), kBytes, s, a);
}

template <bool CHAN>
cudaError_t launch_width(const DecodeArgs& a, cudaStream_t s) {
  switch (a.fill.bits) {
    case 2: return launch_bits<2, CHAN>(a, s);
    case 4: return launch_bits<4, CHAN>(a, s);
    case 8: return launch_bits<8, CHAN>(a, s);
    case 16: return launch_bits<16, CHAN>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

// Self-test of the bounded wait: a barrier that expects 16 bytes no copy will
// bring.  The decode kernel's own wait gives up after its time limit, raises
// the device error flag and the kernel returns normally; no copy is in flight,
// so nothing touches shared memory after the kernel ends.
__global__ void wait_probe_kernel(int* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(smem_u32(&bar), 16u);
    (void)mbar_wait(smem_u32(&bar), 0, err, &abort_flag);
  }
}

}  // namespace

cudaError_t launch_wait_probe(int* err, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

int decode_splits(int num_sms, int n_streams, long long gps) {
  // Smallest modelled makespan  waves(s) * (gps / s + c0)  over
  // s = 1..min(kMaxSplits, gps), where a wave is num_sms * kCtasPerSm CTAs
  // and c0 (in groups) stands for a CTA's fixed cost: pipeline fill, q'
  // set-up, the warp merge and its share of the split merge.  Every CTA gets
  // at least one group; ties go to fewer splits (fewer partials).
  const long long slots = (long long)num_sms * kCtasPerSm;
  const double c0 = 8.0;
  const int smax = (int)(gps < kMaxSplits ? gps : kMaxSplits);
  int best = 1;
  double best_t = 1e300;
  for (int sp = 1; sp <= smax; sp++) {
    const long long waves = ((long long)n_streams * sp + slots - 1) / slots;
    const double tm = (double)waves * ((double)gps / sp + c0 + (sp > 1 ? 0.25 * sp : 0.0));
    if (tm < best_t * (1.0 - 1e-9)) {
      best_t = tm;
      best = sp;
    }
  }
  return best;
}

size_t decode_parts_bytes(int n_streams, int group) {
  (void)group;
  return (size_t)n_streams * kMaxSplits * kPartFloats * sizeof(float);
}

size_t decode_parts_used(int n_streams, int splits) {
  return (size_t)n_streams * splits * kPartFloats * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.group < 1 || a.group > kMaxGroup || a.splits < 1 || a.nparts > kMaxSplits || a.part_base < 0 ||
      a.part_base + a.splits > a.nparts)
    return cudaErrorInvalidValue;
  if (a.chan && (!a.kmc || a.blocks_max < 1 || a.fill.gps % 8 != 0 || a.splits > a.fill.gps / 8))
    return cudaErrorInvalidValue;
  if (a.rank_sms < 0) return cudaErrorInvalidValue;
  DecodeArgs b = a;
  // weighted slices only where they are meant: one wave, >= 2 units per CTA
  const long long units = a.chan ? a.fill.gps / 8 : a.fill.gps;
  if ((long long)a.batch * a.kv_heads * a.splits > (long long)a.rank_sms * kCtasPerSm || units < 2LL * a.splits)
    b.rank_sms = 0;
  return b.chan ? launch_width<true>(b, s) : launch_width<false>(b, s);
}

}  // namespace kvq
