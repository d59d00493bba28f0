// kvq_bitalloc.cu -- block-wise bit allocation (PM-KVQ note, key design 2):
// choose one width b_i per transformer block from a candidate set so that
//   sum_i s_{i, b_i}  is minimal  subject to  sum_i mem_i(b_i) <= M,
// the integer program the note solves with CVXPY.  Here it is solved exactly
// on the host by dynamic programming over memory units (a multiple-choice
// knapsack), which needs no solver library.
//
// Memory model: the cache's budget rule (include/kvq.h, kvq_pool_bytes): a
// block at width b holding N tokens takes batch * kv_heads * 2 * N * (16 b + 4)
// bytes, i.e. (4 b + 1) units of batch * kv_heads * 2 * N * 4 bytes.  The
// capacity in units is at most layers * 65 (every block at 16 bits), so the
// table is small.  Ties between assignments of equal objective go to the one
// the DP meets first (blocks in order, options in the caller's order).
#include <cmath>
#include <cstdint>
#include <vector>

#include "kvq.h"

namespace kvq {
kvq_status api_fail(kvq_status s, const char* msg);
}

extern "C" kvq_status kvq_allocate_bits(int layers, int n_opts, const int* bits, const double* sens, int batch,
                                        int kv_heads, int head_dim, long long max_tokens, size_t budget_bytes,
                                        int* fbit_out, double* objective_out) {
  using kvq::api_fail;
  if (layers <= 0 || n_opts <= 0 || n_opts > 4 || !bits || !sens || !fbit_out)
    return api_fail(KVQ_ERR_INVALID, "bad layers / options / pointers");
  if (batch <= 0 || kv_heads <= 0 || head_dim != 128 || max_tokens <= 0)
    return api_fail(KVQ_ERR_INVALID, "bad shape or token count");
  for (int o = 0; o < n_opts; o++) {
    if (bits[o] != 2 && bits[o] != 4 && bits[o] != 8 && bits[o] != 16)
      return api_fail(KVQ_ERR_INVALID, "candidate widths must be 2, 4, 8 or 16");
    for (int p = 0; p < o; p++)
      if (bits[p] == bits[o]) return api_fail(KVQ_ERR_INVALID, "candidate widths must be distinct");
  }
  for (long long i = 0; i < (long long)layers * n_opts; i++)
    if (!std::isfinite(sens[i])) return api_fail(KVQ_ERR_INVALID, "a sensitivity is not finite");

  // one unit = batch * kv_heads * 2 * N * 4 bytes
  const long double unit = (long double)batch * kv_heads * 2 * (long double)max_tokens * 4;
  const long double cap_ld = std::floor((long double)budget_bytes / unit);
  int min_u = 1 << 30, max_u = 0;
  std::vector<int> u(n_opts);
  for (int o = 0; o < n_opts; o++) {
    u[o] = 4 * bits[o] + 1;
    min_u = u[o] < min_u ? u[o] : min_u;
    max_u = u[o] > max_u ? u[o] : max_u;
  }
  if (cap_ld < (long double)min_u * layers)
    return api_fail(KVQ_ERR_BUDGET, "the budget does not hold every block at the narrowest candidate width");
  const long long cap_all = (long long)max_u * layers;
  const int C = (int)(cap_ld > (long double)cap_all ? cap_all : (long long)cap_ld);

  // dp[c]: least objective of the blocks so far using at most c units
  const double inf = INFINITY;
  std::vector<double> dp(C + 1, 0.0), nx(C + 1);
  std::vector<uint8_t> choice((size_t)layers * (C + 1), 0xff);
  for (int i = 0; i < layers; i++) {
    for (int c = 0; c <= C; c++) {
      double best = inf;
      uint8_t arg = 0xff;
      for (int o = 0; o < n_opts; o++) {
        if (c < u[o] || dp[c - u[o]] == inf) continue;
        const double v = dp[c - u[o]] + sens[(size_t)i * n_opts + o];
        if (v < best) {
          best = v;
          arg = (uint8_t)o;
        }
      }
      nx[c] = best;
      choice[(size_t)i * (C + 1) + c] = arg;
    }
    dp.swap(nx);
  }
  if (dp[C] == inf) return api_fail(KVQ_ERR_BUDGET, "no assignment fits the budget");
  int c = C;
  for (int i = layers - 1; i >= 0; i--) {
    const uint8_t o = choice[(size_t)i * (C + 1) + c];
    fbit_out[i] = bits[o];
    c -= u[o];
  }
  if (objective_out) *objective_out = dp[C];
  return KVQ_OK;
}
