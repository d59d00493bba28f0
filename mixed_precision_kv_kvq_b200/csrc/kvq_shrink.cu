// kvq_shrink.cu -- the Equivalent Right Shift of the PM-KVQ note (key design
// 1):  X_b = ((2^{2b} - 2^b + 1)(X_{2b} + 2^{b-1})) >> 3b, applied to every
// code of a block, in place; and, as a per-block option, the Direct Right
// Shift of the note's ablation (X_b = X_2b >> b, S_b = 2^b S_2b).  The bracket around the product on the page is
// garbled; the product of integers is already an integer, so it is read as a
// plain multiply followed by a logical right shift.  Meta is not touched
// (R = (2^b - 1) S is invariant under S_b = (2^b + 1) S_{2b}, Z_b = Z_{2b}).
//
// Data movement: the packed layout (kvq_internal.cuh) maps input words
// (2J, 2J+1) of a 16 KiB tile to output word J of the same tile, so one CTA
// loads a whole tile into registers, waits at a barrier and writes the
// compacted tile into the tile's first half.  No CTA ever writes bytes
// another CTA reads.  Pure HBM streaming: 16 KiB read + 8 KiB written per
// tile.
//
// SWAR: the product never leaves the lane it is computed in --
//   16 -> 8: one code per 32-bit lane, max (65535+128)*65281 < 2^32;
//    8 -> 4: two codes in 16-bit lanes, max (255+8)*241 = 63383 < 2^16;
//    4 -> 2: four codes in 8-bit lanes, max (15+2)*13 = 221 < 2^8.
#include <cuda_fp16.h>

#include <type_traits>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kShrinkThreads = 256;

// Per-lane shift operators.  Ers: the Equivalent Right Shift; Drs: the
// Direct Right Shift of the note's ablation (keep the high b bits).
//   c16: one 16-bit code in a 32-bit lane -> 8 bits
//   c8:  8-bit codes in the two 16-bit lanes of a word -> 4 bits each
//   c4:  4-bit codes in the four 8-bit lanes of a word -> 2 bits each
struct Ers {
  static __device__ __forceinline__ uint32_t c16(uint32_t x) { return (x + 128u) * 65281u >> 24; }
  static __device__ __forceinline__ uint32_t c8(uint32_t x) { return ((x + 0x00080008u) * 241u >> 12) & 0x000f000fu; }
  static __device__ __forceinline__ uint32_t c4(uint32_t x) { return ((x + 0x02020202u) * 13u >> 6) & 0x03030303u; }
};
struct Drs {
  static __device__ __forceinline__ uint32_t c16(uint32_t x) { return x >> 8; }
  static __device__ __forceinline__ uint32_t c8(uint32_t x) { return (x >> 4) & 0x000f000fu; }
  static __device__ __forceinline__ uint32_t c4(uint32_t x) { return (x >> 2) & 0x03030303u; }
};

// Value parts: in0, in1 are two consecutive input words (each half-word
// packs 16/(2b) codes of width 2b).  Returns the output word: half-word h of
// the output is the shifted codes of half h of in0 (low byte) and of in1
// (high byte).
template <int BTO, class Op>
__device__ __forceinline__ uint32_t shift_pairs(uint32_t in0, uint32_t in1) {
  if constexpr (BTO == 8) {  // one 16-bit code per half-word
    const uint32_t a = Op::c16(in0 & 0xffffu), b = Op::c16(in0 >> 16);
    const uint32_t c = Op::c16(in1 & 0xffffu), d = Op::c16(in1 >> 16);
    return a | (c << 8) | (b << 16) | (d << 24);
  } else if constexpr (BTO == 4) {  // two 8-bit codes per half-word
    auto half = [](uint32_t in) {
      return Op::c8(in & 0x00ff00ffu) | (Op::c8((in >> 8) & 0x00ff00ffu) << 4);
    };
    return half(in0) | (half(in1) << 8);
  } else {  // four 4-bit codes per half-word
    auto half = [](uint32_t in) {
      const uint32_t a = Op::c4(in & 0x0f0f0f0fu);          // fields 0, 2
      const uint32_t b = Op::c4((in >> 4) & 0x0f0f0f0fu);   // fields 1, 3
      const uint32_t t = a | (b << 2);  // fields 0,1 at bits 0-3; fields 2,3 at bits 8-11 (per half)
      return (t | (t >> 4)) & 0x00ff00ffu;
    };
    return half(in0) | (half(in1) << 8);
  }
}

// Key parts hold byte quads (member i of a quad in byte i of its word, see
// kvq_internal.cuh): output byte i gets the shifted member i of the input
// quads, in field order.
template <int BTO, class Op>
__device__ __forceinline__ uint32_t shift_quads(uint32_t in0, uint32_t in1) {
  if constexpr (BTO == 8) {  // one quad spans two input words (members 0, 1 in in0; 2, 3 in in1)
    const uint32_t a = Op::c16(in0 & 0xffffu), b = Op::c16(in0 >> 16);
    const uint32_t c = Op::c16(in1 & 0xffffu), d = Op::c16(in1 >> 16);
    return a | (b << 8) | (c << 16) | (d << 24);
  } else if constexpr (BTO == 4) {  // in0 holds quad 2J (-> low nibbles), in1 quad 2J+1 (-> high nibbles)
    const uint32_t ev = Op::c8(in0 & 0x00ff00ffu) | (Op::c8(in1 & 0x00ff00ffu) << 4);
    const uint32_t od = Op::c8((in0 >> 8) & 0x00ff00ffu) | (Op::c8((in1 >> 8) & 0x00ff00ffu) << 4);
    return ev | (od << 8);
  } else {  // in0 holds quads 4J, 4J+1 (nibbles), in1 quads 4J+2, 4J+3 -> fields 0..3
    return Op::c4(in0 & 0x0f0f0f0fu) | (Op::c4((in0 >> 4) & 0x0f0f0f0fu) << 2) |
           (Op::c4(in1 & 0x0f0f0f0fu) << 4) | (Op::c4((in1 >> 4) & 0x0f0f0f0fu) << 6);
  }
}

template <int BTO, class Op>
__device__ __forceinline__ uint4 shift_uint4(uint4 a, uint4 b, bool key) {
  uint4 o;
  if (key) {
    o.x = shift_quads<BTO, Op>(a.x, a.y);
    o.y = shift_quads<BTO, Op>(a.z, a.w);
    o.z = shift_quads<BTO, Op>(b.x, b.y);
    o.w = shift_quads<BTO, Op>(b.z, b.w);
  } else {
    o.x = shift_pairs<BTO, Op>(a.x, a.y);
    o.y = shift_pairs<BTO, Op>(a.z, a.w);
    o.z = shift_pairs<BTO, Op>(b.x, b.y);
    o.w = shift_pairs<BTO, Op>(b.z, b.w);
  }
  return o;
}

// Direct Right Shift keeps the scale of the kept bits, S_b = 2^b S_2b; in the
// range form R = (2^b - 1) S that is R_b = 2^b R_2b / (2^b + 1), computed in
// fp32 (exact product, one rounded division) and rounded to binary16.  Z is
// kept.  Word: binary16 R in the low half, Z in the high half.
template <int BTO>
__device__ __forceinline__ uint32_t drs_meta(uint32_t w) {
  const float r = __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
  const float q = __fdiv_rn(__fmul_rn(r, (float)(1u << BTO)), (float)((1u << BTO) + 1u));
  return (uint32_t)__half_as_ushort(__float2half_rn(q)) | (w & 0xffff0000u);
}

template <int BTO, class Op>
__global__ void __launch_bounds__(kShrinkThreads) shrink_kernel(uint8_t* codes, uint32_t* meta, int pf, int p_from,
                                                               uint32_t* kmc, long long kmc_words) {
  // Tile = 1024 uint4 in, 512 uint4 out.  Thread i produces output uint4
  // u = i and u = i + 256 from input uint4 2u and 2u + 1.
  uint4* tile = reinterpret_cast<uint4*>(codes + (size_t)blockIdx.x * kTileBytes);
  const int i = threadIdx.x;
  // Launched with programmatic dependent launch so its launch overlaps the
  // previous kernel's tail; it waits for that kernel before touching the
  // block, and never triggers its dependents early (they start when it ends).
  pdl_wait();
  uint4 in[4];
  in[0] = __ldcs(tile + 2 * i);
  in[1] = __ldcs(tile + 2 * i + 1);
  in[2] = __ldcs(tile + 2 * (i + 256));
  in[3] = __ldcs(tile + 2 * (i + 256) + 1);
  __syncthreads();  // every read of the tile is done before any write
  // Output uint4 u lies in a Key part when (u mod 32*BTO) < 16*BTO (a group
  // at BTO bits is 32*BTO uint4: Key part, then Value part); warp-uniform.
  constexpr int kGroupU4 = 32 * BTO, kPartU4 = 16 * BTO;
  const uint4 o0 = shift_uint4<BTO, Op>(in[0], in[1], (i % kGroupU4) < kPartU4);
  const uint4 o1 = shift_uint4<BTO, Op>(in[2], in[3], ((i + 256) % kGroupU4) < kPartU4);
  tile[i] = o0;
  tile[i + 256] = o1;
  if constexpr (std::is_same<Op, Drs>::value) {
    // the tile's p_from slots (all valid: a shrink needs a full block), K and V words
    uint32_t* mt = meta + (size_t)blockIdx.x * pf * 2;
    for (int w = i; w < 2 * p_from; w += kShrinkThreads) mt[w] = drs_meta<BTO>(mt[w]);
    // per-channel Key ranges (blocks with per-channel Key groups)
    for (long long w = (long long)blockIdx.x * kShrinkThreads + i; w < kmc_words;
         w += (long long)gridDim.x * kShrinkThreads)
      kmc[w] = drs_meta<BTO>(kmc[w]);
  }
}

template <int BTO>
cudaError_t launch_to(const ShrinkArgs& a, unsigned grid, cudaStream_t s) {
  const dim3 g(grid), blk(kShrinkThreads);
  if (a.direct) return launch_pdl(shrink_kernel<BTO, Drs>, g, blk, 0, s, a.codes, a.meta, a.pf, a.p_from, a.kmc, a.kmc_words);
  return launch_pdl(shrink_kernel<BTO, Ers>, g, blk, 0, s, a.codes, a.meta, a.pf, a.p_from, (uint32_t*)nullptr, 0LL);
}

}  // namespace

cudaError_t launch_shrink(const ShrinkArgs& a, cudaStream_t s) {
  if (a.n_tiles <= 0) return cudaSuccess;
  if (a.n_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)a.n_tiles;
  switch (a.bits_to) {
    case 8: return launch_to<8>(a, grid, s);
    case 4: return launch_to<4>(a, grid, s);
    case 2: return launch_to<2>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
