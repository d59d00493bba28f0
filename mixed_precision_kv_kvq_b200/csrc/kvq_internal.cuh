// kvq_internal.cuh -- packed layout, block fill pattern and launch interfaces
// shared by the libkvq kernels and the host scheduler.
//
// Packed layout.  A "stream" is one (layer, sequence b, KV head j); it owns a
// region of NT tiles of 16 KiB holding both its Keys and its Values.  At b
// bits a tile holds P_b = 512 / b token slots (32 at 16 bits ... 256 at 2
// bits) in 16-token groups of 512*b bytes: the group's K part (256*b bytes)
// followed by its V part (256*b bytes).  Each part is 32 "lane units" of 8*b
// bytes; unit L (lane L = 4g + t of a warp) holds exactly the 64 codes that
// lane needs as its MMA A-fragment registers:
//   K (QK^T, int8 mma.m16n8k32, A = K[token][channel]): tokens g and g+8
//     of the group, channels 32s + 16r + 4t + i (k-block s = 0..3, column
//     half r = 0..1, member i = 0..3).  The 4 codes (i = 0..3) of one token,
//     k-block and column half form a "quad" = one A register of 4 bytes.  A
//     unit holds 16 quads, quad index Q = 8x + 2s + r with x = 0 for token
//     g and 1 for token g+8.  At b <= 8 bits quad Q lives in 32-bit word
//     Q / (8/b) of the unit at field k = Q % (8/b): member i at bits
//     [8i + b*k, 8i + b*k + b), so each byte packs 8/b codes.  At 16 bits
//     quad Q spans words 2Q (members 0, 1 as half-words) and 2Q + 1
//     (members 2, 3).
//   V (P V, fp16 mma.m16n8k16, A = V^T[channel][token]): channels
//     16s + g + 8r, tokens 2t + {0,1} + 8u (s = 0..7, r, u = 0..1).  Codes
//     come in pairs that fill one half2 register: the same channel of tokens
//     2t+8u and 2t+8u+1.  A unit holds 32 pairs, pair index P = 16u + 2s + r.
//     At b bits pair P lives in 32-bit word P / (16/b) of the unit at field
//     k = P % (16/b): the first member at bits [b*k, b*k+b), the second at
//     bits [16 + b*k, 16 + b*k + b), so each 16-bit half-word packs 16/b
//     codes.
//   In both parts the order of quads (pairs) is the same at every width, so
//   the shift 2b -> b maps input words (2J, 2J+1) of a tile to output word J
//   of the same tile (the K/V interleave of the groups is preserved too),
//   with no data moving between tiles: a shrink compacts every tile into its
//   first half in place and token slots keep their indices.  Every word of
//   a Key part belongs to one token (x is the outermost quad index), so a
//   single-token append writes whole words there.

// Fill pattern of a block (the slot map): before the first shrink tokens
// fill tile 0, tile 1, ... (P_16 each).  A shrink happens only when every
// tile is full, so afterwards every tile is exactly half full (h = P_b / 2)
// and new tokens fill the free halves tile by tile.  At any time the block is
// therefore: tiles < k full, tile k holding h + r, tiles > k holding h.
// Attention does not depend on token order, so nothing is ever reordered.
//
// Meta: two 32-bit words per (stream, tile, slot), the Key's then the
// Value's, each binary16 R (low half) and binary16 Z (high half); P_F slots
// per tile (F = the block's Fbit, the widest a tile ever gets).  A shrink
// never touches meta.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kTileBytes = 16384;
constexpr int kGroupTokens = 16;
// Sink + window option: token 0 and the latest kWindowTokens tokens held at
// 16 bits in kWindowTiles tiles per stream: slot 0 the sink, slot
// 1 + (t - 1) mod kWindowTokens token t >= 1 (the slot its leaving token frees).
constexpr int kWindowTokens = 128;
constexpr int kWindowTiles = 5;  // 129 slots at 32 per 16-bit tile
static_assert((kWindowTokens & (kWindowTokens - 1)) == 0, "window slots are taken modulo a power of two");

__host__ __device__ constexpr int slots_per_tile(int bits) { return 512 / bits; }
__host__ __device__ constexpr int group_bytes(int bits) { return 512 * bits; }  // K part + V part
__host__ __device__ constexpr int part_bytes(int bits) { return 256 * bits; }   // offset of the V part
__host__ __device__ constexpr int unit_bytes(int bits) { return 8 * bits; }

// Fill pattern of one block at its current width (identical for every stream
// of the block, since all sequences of a batch have the same length).
struct Fill {
  int bits;  // current width
  int nt;    // tiles per stream
  int pf;    // meta slots per tile (P at Fbit)
  int p;     // slots per tile at `bits`
  int h;     // base valid slots of every tile (0 before the first shrink)
  int e;     // free slots per tile in this epoch (p - h)
  int k;     // tiles completely full
  int r;     // extra valid slots in tile k (beyond h)
  int gpt;   // groups in a full tile
  int gk;    // groups in tile k (0 if k == nt)
  int gh;    // groups in a tile holding h
  long long gps;  // groups per stream
};

inline Fill make_fill(int bits, int nt, int pf, int n_shrinks, long long n_tokens) {
  Fill f;
  f.bits = bits;
  f.nt = nt;
  f.pf = pf;
  f.p = slots_per_tile(bits);
  f.h = n_shrinks > 0 ? f.p / 2 : 0;
  f.e = f.p - f.h;
  long long m = n_tokens - (long long)nt * f.h;
  f.k = (int)(m / f.e);
  f.r = (int)(m % f.e);
  f.gpt = f.p / kGroupTokens;
  f.gh = f.h / kGroupTokens;
  if (f.k >= nt) {
    f.k = nt;
    f.r = 0;
    f.gk = 0;
  } else {
    f.gk = (f.h + f.r + kGroupTokens - 1) / kGroupTokens;
  }
  f.gps = (long long)f.k * f.gpt + (f.k < nt ? (long long)f.gk + (long long)(nt - f.k - 1) * f.gh : 0);
  return f;
}

// vgroup index within a stream -> tile, group in tile, valid tokens, groups
// in that tile.
struct GroupLoc {
  int tile, grp, valid, tile_groups;
};

__host__ __device__ inline GroupLoc locate_group(const Fill& f, long long v) {
  GroupLoc g;
  long long full = (long long)f.k * f.gpt;
  if (v < full) {
    g.tile = (int)(v / f.gpt);
    g.grp = (int)(v - (long long)g.tile * f.gpt);
    g.valid = kGroupTokens;
    g.tile_groups = f.gpt;
    return g;
  }
  v -= full;
  if (v < f.gk) {
    g.tile = f.k;
    g.grp = (int)v;
    int rem = f.h + f.r - kGroupTokens * g.grp;
    g.valid = rem < kGroupTokens ? rem : kGroupTokens;
    g.tile_groups = f.gk;
    return g;
  }
  v -= f.gk;
  long long t = v / f.gh;
  g.tile = f.k + 1 + (int)t;
  g.grp = (int)(v - t * f.gh);
  g.valid = kGroupTokens;
  g.tile_groups = f.gh;
  return g;
}

// ---------------------------------------------------------------- launches

struct AppendArgs {
  const void* k;
  const void* v;
  int dtype;          // 0 bf16, 1 f32
  int n_call;         // tokens in the caller's k/v arrays (batch stride)
  int tok_off;        // first token of this launch within the call
  int cnt;            // tokens in this launch (all in one epoch)
  long long n0;       // logical index of the first token of this launch
  int bits, h, e, nt, pf;
  int batch, kv_heads;
  uint8_t* codes;     // layer base: [batch][kv_heads][nt][16 KiB]
  uint32_t* meta;     // layer base: [batch][kv_heads][nt][pf][2]
  const float* lam_inv;  // [kv_heads][128] or null
  // sink + window (the block keeps token 0 and the latest kWindowTokens at 16 bits)
  bool window;           // tokens enter the window; n0/bits/h/e/nt describe the progressive cache
  bool stage;            // with window: per-channel Key staging -- token t takes slot t mod 128, nothing leaves
  bool direct;           // the block shrinks with the Direct Right Shift
  long long t0;          // token index (all tokens) of the first token of this launch
  uint8_t* wcodes;       // window codes: [batch][kv_heads][kWindowTiles][16 KiB]
  uint32_t* wmeta;       // window meta:  [batch][kv_heads][kWindowTiles][32][2]
};

struct ShrinkArgs {
  uint8_t* codes;     // layer base
  long long n_tiles;  // batch * kv_heads * nt
  int bits_to;        // 8, 4 or 2
  bool direct;        // Direct Right Shift (also rescales the ranges in meta)
  uint32_t* meta;     // layer base of the meta (used when direct)
  int pf;             // meta slots per tile
  int p_from;         // valid slots per tile before the shrink (the tile is full)
  uint32_t* kmc;      // per-channel Key meta words rescaled too when direct, or null
  long long kmc_words;
};

// Per-channel Key groups: a full staged block of 128 tokens enters the
// progressive cache (one CTA per stream).
constexpr int kKeyBlock = 128;
struct BlockMoveArgs {
  const uint8_t* wcodes;  // staging codes: [streams][kWindowTiles][16 KiB], token t of the block in slot t
  const uint32_t* wmeta;  // staging meta:  [streams][kWindowTiles][32][2]
  uint8_t* codes;         // progressive cache (layer base)
  uint32_t* meta;
  uint32_t* kmc;          // per-channel Key meta: [streams][blocks_max][128] words (R low, Z high)
  int blocks_max, blk;    // blocks per stream; the block being moved
  int nt, pf, bits;       // progressive cache: tiles per stream, meta slots per tile, current width
  bool direct;            // the block shrinks with the Direct Right Shift
  int g_tile[kKeyBlock / kGroupTokens], g_slot[kKeyBlock / kGroupTokens];  // where its 8 groups go
  // from_input: the block arrives whole in one append call with nothing
  // staged, and is read from the call's k, v (as the append would stage it:
  // Keys divided by lambda, each token quantized to INT16) instead of the
  // staging area, which it never touches
  bool from_input;
  const void* k;
  const void* v;
  int dtype, n_call, tok_off, kv_heads;
  const float* lam_inv;  // [kv_heads][128] or null
};

// Logical order of a block's progressive cache, epoch by epoch: tokens
// [start_e, start_{e+1}) arrived at width 16 >> e and sit in slots
// [h_e, h_e + ee_e) of tiles 0, 1, ... (ee_e per tile).
struct Epochs {
  int n;                  // epochs so far (shrinks + 1)
  int start[4];           // tokens per stream stay below 2^30
  int h[4], lg_ee[4];     // ee_e = 1 << lg_ee[e] (32, 32, 64, 128 slots)
};
inline Epochs make_epochs(int nt, int n_shrinks) {
  Epochs ep{};
  ep.n = n_shrinks + 1;
  for (int e = 0; e < ep.n && e < 4; e++) {
    const int p = slots_per_tile(16 >> e);
    ep.h[e] = e > 0 ? p / 2 : 0;
    int lg = 0;
    while ((1 << lg) < p - ep.h[e]) lg++;
    ep.lg_ee[e] = lg;
    ep.start[e] = nt * ep.h[e];
  }
  return ep;
}

struct DecodeArgs {
  uint8_t* codes;       // the block's (or window's) codes; written only by a fused append
  uint32_t* meta;
  const void* q;        // bf16 [batch][q_heads][128]
  const float* lam;     // [kv_heads][128] or null
  float* out;           // fp32 [batch][q_heads][128]
  float* parts;         // workspace partials: [batch*kv_heads][splits] records of M[8], L[8], O[128][8]
  int* counters;        // [batch*kv_heads] ticket counters (zero between calls)
  int* err;             // device error flag
  Fill fill;
  int batch, kv_heads, q_heads, group;
  float qscale;         // sm_scale * log2(e)
  int splits;           // CTAs per stream in this launch
  int nparts;           // partials per stream over every launch of the call (the ticket counts them all)
  int part_base;        // index of this launch's first partial
  long long safe;       // groups [0, safe) of every stream are not written by kernels still in flight
  bool after_decode;    // launched right after another decode launch of the same call: no dependency wait
  int rank_sms;         // > 0: the GPU's SM count, slices weighted by arrival order (one-wave launches); 0: equal
  bool trigger_early;   // another decode launch of the call follows: trigger it right after the wait
  // fused single-token append (kvq_append_decode): the warp whose groups
  // include group app_group writes the new token (slot app_slot of tile
  // app_tile of every stream) before copying its groups; app_group < 0: none
  long long app_group;
  int app_tile, app_slot;
  const void* ak;        // [batch][1][kv_heads][128] new Keys (bf16 or f32)
  const void* av;        // new Values
  int adtype;            // 0 bf16, 1 f32
  const float* lam_inv;  // [kv_heads][128] or null
  // per-channel Key groups: groups are walked in logical order (ep) and
  // each 128-token block's Key ranges and zeros come from kmc
  bool chan;
  const uint32_t* kmc;   // [streams][blocks_max][128]
  int blocks_max;
  Epochs ep;
};

// CTAs per stream for a launch over n_streams streams on num_sms SMs.
int decode_splits(int num_sms, int n_streams, long long groups_per_stream);
constexpr int kMaxSplits = 64;
size_t decode_parts_bytes(int n_streams, int group);
// Workspace bytes one launch with `splits` CTAs per stream actually touches.
size_t decode_parts_used(int n_streams, int splits);

// Programmatic dependent launch: kernels of libkvq are launched so that the
// next kernel in the stream may be scheduled while the previous one drains;
// each kernel waits (griddepcontrol.wait) before it touches memory an earlier
// kernel may have written, so results are exactly as with plain launches.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename Kernel, typename... Args>
inline cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);
cudaError_t launch_block_move(const BlockMoveArgs& a, int n_streams, cudaStream_t s);
cudaError_t launch_shrink(const ShrinkArgs& a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);

cudaError_t launch_wait_probe(int* err, cudaStream_t s);

}  // namespace kvq
