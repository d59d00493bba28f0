// kvq_shrink.cu -- the Equivalent Right Shift of the PM-KVQ note (key design
// 1):  X_b = ((2^{2b} - 2^b + 1)(X_{2b} + 2^{b-1})) >> 3b, applied to every
// code of a block, in place.  The bracket around the product on the page is
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
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kShrinkThreads = 256;

// Value parts: in0, in1 are two consecutive input words (each half-word
// packs 16/(2b) codes of width 2b).  Returns the output word: half-word h of
// the output is the shifted codes of half h of in0 (low byte) and of in1
// (high byte).
template <int BTO>
__device__ __forceinline__ uint32_t ers_pair(uint32_t in0, uint32_t in1);

template <>
__device__ __forceinline__ uint32_t ers_pair<8>(uint32_t in0, uint32_t in1) {
  // one 16-bit code per half-word
  const uint32_t mul = 65281u;  // 2^16 - 2^8 + 1
  uint32_t a = ((in0 & 0xffffu) + 128u) * mul >> 24;
  uint32_t b = ((in0 >> 16) + 128u) * mul >> 24;
  uint32_t c = ((in1 & 0xffffu) + 128u) * mul >> 24;
  uint32_t d = ((in1 >> 16) + 128u) * mul >> 24;
  return a | (c << 8) | (b << 16) | (d << 24);
}

__device__ __forceinline__ uint32_t ers_half_words_4(uint32_t in) {
  // two 8-bit codes per half-word -> two 4-bit codes in the low byte of each half
  uint32_t lo = (((in & 0x00ff00ffu) + 0x00080008u) * 241u >> 12) & 0x000f000fu;
  uint32_t hi = ((((in >> 8) & 0x00ff00ffu) + 0x00080008u) * 241u >> 12) & 0x000f000fu;
  return lo | (hi << 4);
}

template <>
__device__ __forceinline__ uint32_t ers_pair<4>(uint32_t in0, uint32_t in1) {
  return ers_half_words_4(in0) | (ers_half_words_4(in1) << 8);
}

__device__ __forceinline__ uint32_t ers_half_words_2(uint32_t in) {
  // four 4-bit codes per half-word -> four 2-bit codes in the low byte of each half
  uint32_t a = (((in & 0x0f0f0f0fu) + 0x02020202u) * 13u >> 6) & 0x03030303u;          // fields 0, 2
  uint32_t b = ((((in >> 4) & 0x0f0f0f0fu) + 0x02020202u) * 13u >> 6) & 0x03030303u;   // fields 1, 3
  uint32_t t = a | (b << 2);  // fields 0,1 at bits 0-3; fields 2,3 at bits 8-11 (per half)
  return (t | (t >> 4)) & 0x00ff00ffu;
}

template <>
__device__ __forceinline__ uint32_t ers_pair<2>(uint32_t in0, uint32_t in1) {
  return ers_half_words_2(in0) | (ers_half_words_2(in1) << 8);
}

// Key parts hold byte quads (member i of a quad in byte i of its word, see
// kvq_internal.cuh): output byte i gets the shifted member i of the input
// quads, in field order.
template <int BTO>
__device__ __forceinline__ uint32_t ers_quads(uint32_t in0, uint32_t in1);

template <>
__device__ __forceinline__ uint32_t ers_quads<8>(uint32_t in0, uint32_t in1) {
  // one quad spans two input words (members 0, 1 in in0; 2, 3 in in1)
  const uint32_t mul = 65281u;
  uint32_t a = ((in0 & 0xffffu) + 128u) * mul >> 24;
  uint32_t b = ((in0 >> 16) + 128u) * mul >> 24;
  uint32_t c = ((in1 & 0xffffu) + 128u) * mul >> 24;
  uint32_t d = ((in1 >> 16) + 128u) * mul >> 24;
  return a | (b << 8) | (c << 16) | (d << 24);
}

__device__ __forceinline__ uint32_t ers_lanes16_4(uint32_t x) {  // 8-bit codes in 16-bit lanes -> 4 bits
  return ((x + 0x00080008u) * 241u >> 12) & 0x000f000fu;
}

template <>
__device__ __forceinline__ uint32_t ers_quads<4>(uint32_t in0, uint32_t in1) {
  // in0 holds quad 2J (-> low nibbles), in1 quad 2J+1 (-> high nibbles)
  const uint32_t ev = ers_lanes16_4(in0 & 0x00ff00ffu) | (ers_lanes16_4(in1 & 0x00ff00ffu) << 4);
  const uint32_t od = ers_lanes16_4((in0 >> 8) & 0x00ff00ffu) | (ers_lanes16_4((in1 >> 8) & 0x00ff00ffu) << 4);
  return ev | (od << 8);
}

__device__ __forceinline__ uint32_t ers_lanes8_2(uint32_t x) {  // 4-bit codes in 8-bit lanes -> 2 bits
  return ((x + 0x02020202u) * 13u >> 6) & 0x03030303u;
}

template <>
__device__ __forceinline__ uint32_t ers_quads<2>(uint32_t in0, uint32_t in1) {
  // in0 holds quads 4J, 4J+1 (nibbles), in1 quads 4J+2, 4J+3 -> fields 0..3
  return ers_lanes8_2(in0 & 0x0f0f0f0fu) | (ers_lanes8_2((in0 >> 4) & 0x0f0f0f0fu) << 2) |
         (ers_lanes8_2(in1 & 0x0f0f0f0fu) << 4) | (ers_lanes8_2((in1 >> 4) & 0x0f0f0f0fu) << 6);
}

template <int BTO>
__device__ __forceinline__ uint4 ers_uint4(uint4 a, uint4 b, bool key) {
  uint4 o;
  if (key) {
    o.x = ers_quads<BTO>(a.x, a.y);
    o.y = ers_quads<BTO>(a.z, a.w);
    o.z = ers_quads<BTO>(b.x, b.y);
    o.w = ers_quads<BTO>(b.z, b.w);
  } else {
    o.x = ers_pair<BTO>(a.x, a.y);
    o.y = ers_pair<BTO>(a.z, a.w);
    o.z = ers_pair<BTO>(b.x, b.y);
    o.w = ers_pair<BTO>(b.z, b.w);
  }
  return o;
}

template <int BTO>
__global__ void __launch_bounds__(kShrinkThreads) shrink_kernel(uint8_t* codes) {
  // Tile = 1024 uint4 in, 512 uint4 out.  Thread i produces output uint4
  // u = i and u = i + 256 from input uint4 2u and 2u + 1.
  uint4* tile = reinterpret_cast<uint4*>(codes + (size_t)blockIdx.x * kTileBytes);
  const int i = threadIdx.x;
  uint4 in[4];
  in[0] = __ldcs(tile + 2 * i);
  in[1] = __ldcs(tile + 2 * i + 1);
  in[2] = __ldcs(tile + 2 * (i + 256));
  in[3] = __ldcs(tile + 2 * (i + 256) + 1);
  __syncthreads();  // every read of the tile is done before any write
  // Output uint4 u lies in a Key part when (u mod 32*BTO) < 16*BTO (a group
  // at BTO bits is 32*BTO uint4: Key part, then Value part); warp-uniform.
  constexpr int kGroupU4 = 32 * BTO, kPartU4 = 16 * BTO;
  const uint4 o0 = ers_uint4<BTO>(in[0], in[1], (i % kGroupU4) < kPartU4);
  const uint4 o1 = ers_uint4<BTO>(in[2], in[3], ((i + 256) % kGroupU4) < kPartU4);
  tile[i] = o0;
  tile[i + 256] = o1;
}

}  // namespace

cudaError_t launch_shrink(const ShrinkArgs& a, cudaStream_t s) {
  if (a.n_tiles <= 0) return cudaSuccess;
  if (a.n_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)a.n_tiles;
  switch (a.bits_to) {
    case 8: shrink_kernel<8><<<grid, kShrinkThreads, 0, s>>>(a.codes); break;
    case 4: shrink_kernel<4><<<grid, kShrinkThreads, 0, s>>>(a.codes); break;
    case 2: shrink_kernel<2><<<grid, kShrinkThreads, 0, s>>>(a.codes); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kvq
