/*
 * kvq_oracle.c -- plain, slow CPU oracle for the PM-KVQ progressive
 * mixed-precision KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * reads this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Sources (the PM-KVQ note on papernotes.org, "PM-KVQ: Progressive
 * Mixed-Precision KV Cache Quantization for Long-CoT LLMs"):
 *   - Key design 1 (progressive quantization): every block starts at 16 bits
 *     and, when its memory budget is full, the whole block's cache is shrunk
 *     one level 16 -> 8 -> 4 -> 2 by the Equivalent Right Shift
 *       X_b = ((2^{2b} - 2^b + 1) (X_{2b} + 2^{b-1})) >> 3b,
 *     with Z_b = Z_{2b} and S_b = (2^b + 1) S_{2b}.
 *   - Key design 3 / QServe reparameterisation: Key outliers are migrated to
 *     the Query per channel, K / lambda and Q * lambda.
 *   - Loss function / training strategy: asymmetric group quantization,
 *     group size 128.
 * And the ChanMix note on the same site, key design 1: an asymmetric
 * quantizer has scale S = (Cmax - Cmin) / (2^b - 1) and worst-case error S/2.
 *
 * Readings where the pages are silent:
 *   - One group = one token's 128 channels of one KV head (K and V alike).
 *   - Dequantisation is  x^ = Z + S * q  with Z a real-valued zero (the group
 *     minimum rounded down to binary16), which is what keeps Z_b = Z_{2b}
 *     meaningful.  The scale is held as the range R = (2^b - 1) * S, also a
 *     binary16 value, rounded up; S = R / (2^b - 1).
 *   - Codes:  q = clamp(floor(fp32(fp32(x - Z) * fp32((2^b-1)/R)) + 1/2), 0, 2^b-1)
 *     with every step an IEEE fp32 round-to-nearest operation and no fused
 *     multiply-add (build with -ffp-contract=off).  A group with R = 0 has all
 *     codes 0.
 *   - The 16-bit stage stores 16-bit integer codes (the shift needs integer
 *     X_16).  The garbled bracket around the shift formula is read as a plain
 *     integer product followed by a logical right shift.
 *   - A block shrinks when a token arrives and the block holds as many tokens
 *     as fit at its current width; it never shrinks below its allocated Fbit.
 *     An append of n tokens behaves exactly like n appends of one token.
 *   - Attention: s_t = sm_scale * (q * lambda) . k^_t, softmax over every
 *     cached token, o = sum_t p_t v^_t, all in fp64.  Query head h reads KV
 *     head h / G.
 */
#pragma STDC FP_CONTRACT OFF
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 128

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16, written from the format's definition:                   */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; exponent field 0  */
/* encodes subnormals m * 2^-24, field 31 encodes inf / NaN.                  */
/* ------------------------------------------------------------------------ */

double orc_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 31;
  int m = h & 1023;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp(1024.0 + (double)m, e - 25);
  }
  return sign ? -v : v;
}

/* Encode a non-negative magnitude that is exactly representable (or inf). */
static uint16_t f16_encode_mag(double a) {
  if (a == 0.0) return 0;
  if (isinf(a) || a > 65504.0) return 0x7c00;
  if (a < ldexp(1.0, -14)) {
    return (uint16_t)(a / ldexp(1.0, -24)); /* subnormal: exact multiple of 2^-24 */
  }
  int E;
  double fr = frexp(a, &E); /* a = fr * 2^E, fr in [0.5, 1) */
  int e = E - 1;            /* a in [2^e, 2^{e+1}) */
  double mant = ldexp(a, -e) - 1.0; /* in [0, 1) */
  (void)fr;
  return (uint16_t)(((e + 15) << 10) | (uint16_t)(mant * 1024.0));
}

/* x -> binary16 bits.  mode 0: nearest, ties to even; -1: toward -inf;
 * +1: toward +inf. */
uint16_t orc_f16_from_f64(double x, int mode) {
  if (isnan(x)) return 0x7e00;
  int neg = signbit(x) ? 1 : 0;
  double a = fabs(x);
  if (a == 0.0) return neg ? 0x8000 : 0;
  /* spacing of binary16 values around a */
  double ulp;
  if (a < ldexp(1.0, -14)) {
    ulp = ldexp(1.0, -24);
  } else {
    int E;
    frexp(a, &E);
    ulp = ldexp(1.0, (E - 1) - 10);
  }
  double lo = floor(a / ulp) * ulp; /* largest multiple <= a (exact) */
  double hi = (lo == a) ? lo : lo + ulp;
  double mag;
  if (lo == hi) {
    mag = lo;
  } else if (mode == 0) {
    double dlo = a - lo, dhi = hi - a;
    if (dlo < dhi) mag = lo;
    else if (dhi < dlo) mag = hi;
    else {
      /* tie: pick the one whose last fraction bit is 0 */
      double k = lo / ulp;
      mag = (fmod(k, 2.0) == 0.0) ? lo : hi;
    }
  } else {
    /* directed: toward +inf means larger magnitude for positives */
    int up_mag = (mode > 0) ? !neg : neg;
    mag = up_mag ? hi : lo;
  }
  uint16_t bits;
  if (mag > 65504.0) {
    /* overflow: RN goes to inf; directed goes to inf only away from zero */
    if (mode == 0) bits = 0x7c00;
    else {
      int up_mag = (mode > 0) ? !neg : neg;
      bits = up_mag ? 0x7c00 : 0x7bff;
    }
  } else {
    bits = f16_encode_mag(mag);
  }
  return (uint16_t)(bits | (neg ? 0x8000 : 0));
}

/* ------------------------------------------------------------------------ */
/* Outlier migration (Key design 3): the stored Key is k / lambda per channel */
/* (lambda is folded into the Query).  fp32 product with the fp32 value of    */
/* 1 / lambda.                                                               */
/* ------------------------------------------------------------------------ */

float orc_lambda_inv(float lambda) { return (float)(1.0 / (double)lambda); }

float orc_migrate(float k, float lambda) {
  volatile float linv = orc_lambda_inv(lambda);
  volatile float x = k * linv;
  return x;
}

/* Migration factor from calibration keys (Key design 3):
 * lambda_i = (max_m |K_{m,i}|)^alpha over the m calibration tokens of one
 * KV head.  keys: [m][n_ch]. */
void orc_lambda_from_keys(const float* keys, int m, int n_ch, double alpha, float* lambda) {
  for (int i = 0; i < n_ch; i++) {
    double mx = 0.0;
    for (int t = 0; t < m; t++) {
      double a = fabs((double)keys[(size_t)t * n_ch + i]);
      if (a > mx) mx = a;
    }
    lambda[i] = (float)pow(mx, alpha);
  }
}

/* ------------------------------------------------------------------------ */
/* Asymmetric group quantizer (training strategy: group 128, asymmetric;     */
/* ChanMix key design 1: S = (max - min) / (2^b - 1)).                        */
/* ------------------------------------------------------------------------ */

/* Step 1: the group's zero and range as binary16 bit patterns. */
void orc_group_meta(const float* x, int n, uint16_t* r_bits, uint16_t* z_bits) {
  float mn = x[0], mx = x[0];
  for (int c = 1; c < n; c++) {
    if (x[c] < mn) mn = x[c];
    if (x[c] > mx) mx = x[c];
  }
  uint16_t zb = orc_f16_from_f64((double)mn, -1); /* Z <= min */
  volatile float z = (float)orc_f16_to_f64(zb);
  volatile float diff = mx - z; /* fp32, round to nearest */
  uint16_t rb = orc_f16_from_f64((double)diff, +1); /* Z + R >= max */
  *r_bits = rb;
  *z_bits = zb;
}

/* Step 2: codes for given (R, Z) at `bits`. */
void orc_codes_with_meta(const float* x, int n, int bits, uint16_t r_bits, uint16_t z_bits,
                         uint16_t* codes) {
  volatile float r = (float)orc_f16_to_f64(r_bits);
  volatile float z = (float)orc_f16_to_f64(z_bits);
  float qmax = (float)((1u << bits) - 1u);
  if (r == 0.0f) {
    for (int c = 0; c < n; c++) codes[c] = 0;
    return;
  }
  volatile float inv = qmax / r; /* fp32 division, round to nearest */
  for (int c = 0; c < n; c++) {
    volatile float d = x[c] - z;
    volatile float t = d * inv;
    volatile float u = t + 0.5f;
    float f = floorf(u);
    if (f < 0.0f) f = 0.0f;
    if (f > qmax) f = qmax;
    codes[c] = (uint16_t)f;
  }
}

void orc_quantize_group(const float* x, int n, int bits, uint16_t* codes, uint16_t* r_bits,
                        uint16_t* z_bits) {
  orc_group_meta(x, n, r_bits, z_bits);
  orc_codes_with_meta(x, n, bits, *r_bits, *z_bits, codes);
}

/* x^ = Z + q * R / (2^b - 1), in fp64 (binary16 meta is exact in fp64). */
double orc_dequant(uint16_t code, uint16_t r_bits, uint16_t z_bits, int bits) {
  double r = orc_f16_to_f64(r_bits);
  double z = orc_f16_to_f64(z_bits);
  return z + (double)code * (r / (double)((1u << bits) - 1u));
}

/* ------------------------------------------------------------------------ */
/* Equivalent Right Shift (Key design 1): 2b-bit code -> b-bit code.           */
/* ------------------------------------------------------------------------ */

uint32_t orc_ers(uint32_t x2b, int b) {
  uint64_t mul = (1ull << (2 * b)) - (1ull << b) + 1ull;
  uint64_t prod = mul * ((uint64_t)x2b + (1ull << (b - 1)));
  return (uint32_t)(prod >> (3 * b));
}

/* Scale after a shrink, as a function of the scale before it (S_b = (2^b+1) S_2b). */
double orc_scale_after_shrink(double s2b, int b) { return (double)((1u << b) + 1u) * s2b; }

/* Direct Right Shift (the first row of the note's ablation): keep only the
 * high b bits of the 2b-bit code, X_b = X_2b >> b, with Z_b = Z_2b and the
 * scale of the kept bits S_b = 2^b S_2b (reading: the plain scale of a
 * truncation; the note gives no formula).  In the range form R = (2^b - 1) S
 * that is R_b = 2^b R_2b / (2^b + 1), computed as fp32(fp32(R 2^b) / (2^b + 1))
 * and rounded to binary16 to nearest (reading: the meta format is binary16). */
uint32_t orc_drs(uint32_t x2b, int b) { return x2b >> b; }

uint16_t orc_drs_range(uint16_t r_bits, int b) {
  const float r = (float)orc_f16_to_f64(r_bits);
  const float num = r * (float)(1u << b); /* exact: a power of two */
  const float q = num / (float)((1u << b) + 1u);
  return orc_f16_from_f64((double)q, 0);
}

/* ------------------------------------------------------------------------ */
/* Progressive cache model of one transformer block (Key design 1).          */
/* Codes and meta are kept in logical token order.                          */
/* ------------------------------------------------------------------------ */

typedef struct {
  int batch, kv_heads, fbit, n_f; /* n_f: tokens that fit at fbit */
  int bits, n, n_shrinks;
  int shrink_at[8]; /* token count when each shrink happened */
  uint16_t* kc;     /* [batch][kv_heads][n_f][128] */
  uint16_t* vc;
  uint16_t* km; /* [batch][kv_heads][n_f][2]  (R bits, Z bits) */
  uint16_t* vm;
  int shift_mode; /* 0: Equivalent Right Shift, 1: Direct Right Shift */
} orc_layer;

size_t orc_layer_sizeof(void) { return sizeof(orc_layer); }

int orc_layer_capacity(const orc_layer* L, int bits) {
  return (int)((int64_t)L->n_f * L->fbit / bits);
}

int orc_layer_init(orc_layer* L, int batch, int kv_heads, int n_f, int fbit) {
  memset(L, 0, sizeof(*L));
  if (fbit != 2 && fbit != 4 && fbit != 8 && fbit != 16) return -1;
  L->batch = batch;
  L->kv_heads = kv_heads;
  L->fbit = fbit;
  L->n_f = n_f;
  L->bits = 16;
  size_t ncode = (size_t)batch * kv_heads * n_f * ORC_D;
  size_t nmeta = (size_t)batch * kv_heads * n_f * 2;
  L->kc = (uint16_t*)calloc(ncode, 2);
  L->vc = (uint16_t*)calloc(ncode, 2);
  L->km = (uint16_t*)calloc(nmeta, 2);
  L->vm = (uint16_t*)calloc(nmeta, 2);
  if (!L->kc || !L->vc || !L->km || !L->vm) return -2;
  return 0;
}

void orc_layer_free(orc_layer* L) {
  free(L->kc);
  free(L->vc);
  free(L->km);
  free(L->vm);
  memset(L, 0, sizeof(*L));
}

static size_t orc_slot(const orc_layer* L, int b, int h, int t) {
  return ((size_t)b * L->kv_heads + h) * L->n_f + t;
}

/* Shrink every stored code one level (2b -> b).  Equivalent Right Shift:
 * meta is untouched (with the range form R = (2^b - 1) S, S_b = (2^b + 1) S_2b
 * keeps R fixed).  Direct Right Shift: every stored R is rescaled. */
int orc_layer_shrink(orc_layer* L) {
  if (L->bits <= L->fbit) return -1;
  int b = L->bits / 2;
  for (int bb = 0; bb < L->batch; bb++)
    for (int h = 0; h < L->kv_heads; h++)
      for (int t = 0; t < L->n; t++) {
        size_t slot = orc_slot(L, bb, h, t);
        size_t base = slot * ORC_D;
        for (int c = 0; c < ORC_D; c++) {
          if (L->shift_mode == 1) {
            L->kc[base + c] = (uint16_t)orc_drs(L->kc[base + c], b);
            L->vc[base + c] = (uint16_t)orc_drs(L->vc[base + c], b);
          } else {
            L->kc[base + c] = (uint16_t)orc_ers(L->kc[base + c], b);
            L->vc[base + c] = (uint16_t)orc_ers(L->vc[base + c], b);
          }
        }
        if (L->shift_mode == 1) {
          L->km[slot * 2] = orc_drs_range(L->km[slot * 2], b);
          L->vm[slot * 2] = orc_drs_range(L->vm[slot * 2], b);
        }
      }
  if (L->n_shrinks < 8) L->shrink_at[L->n_shrinks] = L->n;
  L->n_shrinks++;
  L->bits = b;
  return 0;
}

/* Append n tokens.  k, v: [batch][n][kv_heads][128] (fp32 values; bf16 inputs
 * are passed as their exact fp32 values).  lambda: [kv_heads][128] or NULL
 * (no migration).  Returns 0, or 1 when the block cannot hold the tokens at
 * its Fbit (nothing is written in that case). */
int orc_layer_append(orc_layer* L, const float* k, const float* v, int n, const float* lambda) {
  if (n < 0) return -1;
  if ((int64_t)L->n + n > (int64_t)L->n_f) return 1;
  float x[ORC_D];
  for (int t = 0; t < n; t++) {
    if (L->n == orc_layer_capacity(L, L->bits)) {
      if (orc_layer_shrink(L) != 0) return 1; /* unreachable after the check above */
    }
    for (int bb = 0; bb < L->batch; bb++)
      for (int h = 0; h < L->kv_heads; h++) {
        size_t in = (((size_t)bb * n + t) * L->kv_heads + h) * ORC_D;
        size_t slot = orc_slot(L, bb, h, L->n);
        for (int c = 0; c < ORC_D; c++)
          x[c] = lambda ? orc_migrate(k[in + c], lambda[h * ORC_D + c]) : k[in + c];
        orc_quantize_group(x, ORC_D, L->bits, L->kc + slot * ORC_D, L->km + slot * 2,
                           L->km + slot * 2 + 1);
        orc_quantize_group(v + in, ORC_D, L->bits, L->vc + slot * ORC_D, L->vm + slot * 2,
                           L->vm + slot * 2 + 1);
      }
    L->n++;
  }
  return 0;
}

/* Choose the shift of a block before its first shrink (0 ERS, 1 DRS). */
int orc_layer_set_shift_mode(orc_layer* L, int mode) {
  if (mode != 0 && mode != 1) return -1;
  if (L->n_shrinks > 0) return -2;
  L->shift_mode = mode;
  return 0;
}

/* Eager shrink of a full block (the step the next append would take). */
int orc_layer_force_shrink(orc_layer* L) {
  if (L->bits <= L->fbit) return -1;
  if (L->n != orc_layer_capacity(L, L->bits)) return -2;
  return orc_layer_shrink(L);
}

/* ------------------------------------------------------------------------ */
/* Sink token + recent window (training strategy: the KIVI trick the note    */
/* keeps -- the first token and the most recent 128 tokens are stored as     */
/* INT16).  Readings: a token is quantized at 16 bits when it arrives; when  */
/* it leaves the window (token t arrives, t - 128 >= 1 leaves) it moves into */
/* the block's progressive cache at that cache's current width by the        */
/* block's own shift applied 16 -> 8 -> ... -> b, R and Z kept (rescaled R   */
/* under the Direct Right Shift) -- the same codes it would have if it had   */
/* been stored at 16 bits and shrunk with the block; the sink never leaves.  */
/* The progressive cache (tokens 1 .. n - 129) follows the budget schedule   */
/* on its own token count.                                                   */
/* ------------------------------------------------------------------------ */

#define ORC_WINDOW 128

typedef struct {
  orc_layer main; /* the progressive cache: token 1 + m at index m */
  int n;          /* tokens appended */
  int n_max;      /* main.n_f + 1 + ORC_WINDOW */
  uint16_t* kc;   /* [batch][kv_heads][n_max][128]: INT16 codes of every token */
  uint16_t* vc;
  uint16_t* km; /* [batch][kv_heads][n_max][2] */
  uint16_t* vm;
} orc_wlayer;

size_t orc_wlayer_sizeof(void) { return sizeof(orc_wlayer); }

int orc_wlayer_init(orc_wlayer* W, int batch, int kv_heads, int n_f, int fbit) {
  memset(W, 0, sizeof(*W));
  int rc = orc_layer_init(&W->main, batch, kv_heads, n_f, fbit);
  if (rc) return rc;
  W->n_max = n_f + 1 + ORC_WINDOW;
  size_t ncode = (size_t)batch * kv_heads * W->n_max * ORC_D;
  size_t nmeta = (size_t)batch * kv_heads * W->n_max * 2;
  W->kc = (uint16_t*)calloc(ncode, 2);
  W->vc = (uint16_t*)calloc(ncode, 2);
  W->km = (uint16_t*)calloc(nmeta, 2);
  W->vm = (uint16_t*)calloc(nmeta, 2);
  if (!W->kc || !W->vc || !W->km || !W->vm) return -2;
  return 0;
}

void orc_wlayer_free(orc_wlayer* W) {
  orc_layer_free(&W->main);
  free(W->kc);
  free(W->vc);
  free(W->km);
  free(W->vm);
  memset(W, 0, sizeof(*W));
}

static size_t orc_wslot(const orc_wlayer* W, int b, int h, int t) {
  return ((size_t)b * W->main.kv_heads + h) * W->n_max + t;
}

/* One INT16 code (and its group's range) brought down to `bits` by the
 * block's shift, one level at a time. */
static uint32_t orc_chain_code(uint32_t x, int bits, int mode) {
  for (int b = 8; b >= bits; b /= 2) x = mode == 1 ? orc_drs(x, b) : orc_ers(x, b);
  return x;
}
static uint16_t orc_chain_range(uint16_t r, int bits, int mode) {
  if (mode == 1)
    for (int b = 8; b >= bits; b /= 2) r = orc_drs_range(r, b);
  return r;
}

/* Move token e (>= 1) from the INT16 store into the progressive cache. */
static void orc_wlayer_evict(orc_wlayer* W, int e) {
  orc_layer* L = &W->main;
  if (L->n == orc_layer_capacity(L, L->bits)) orc_layer_shrink(L); /* budget checked by the caller */
  for (int bb = 0; bb < L->batch; bb++)
    for (int h = 0; h < L->kv_heads; h++) {
      size_t src = orc_wslot(W, bb, h, e), dst = orc_slot(L, bb, h, L->n);
      for (int c = 0; c < ORC_D; c++) {
        L->kc[dst * ORC_D + c] = (uint16_t)orc_chain_code(W->kc[src * ORC_D + c], L->bits, L->shift_mode);
        L->vc[dst * ORC_D + c] = (uint16_t)orc_chain_code(W->vc[src * ORC_D + c], L->bits, L->shift_mode);
      }
      L->km[dst * 2] = orc_chain_range(W->km[src * 2], L->bits, L->shift_mode);
      L->km[dst * 2 + 1] = W->km[src * 2 + 1];
      L->vm[dst * 2] = orc_chain_range(W->vm[src * 2], L->bits, L->shift_mode);
      L->vm[dst * 2 + 1] = W->vm[src * 2 + 1];
    }
  L->n++;
}

/* Append n tokens (same arguments as orc_layer_append).  Returns 1 when the
 * progressive cache could not hold its share at Fbit (nothing written). */
int orc_wlayer_append(orc_wlayer* W, const float* k, const float* v, int n, const float* lambda) {
  orc_layer* L = &W->main;
  if (n < 0) return -1;
  int64_t main_after = (int64_t)W->n + n - 1 - ORC_WINDOW;
  if (main_after > (int64_t)L->n_f) return 1;
  float x[ORC_D];
  for (int i = 0; i < n; i++) {
    int t = W->n;
    for (int bb = 0; bb < L->batch; bb++)
      for (int h = 0; h < L->kv_heads; h++) {
        size_t in = (((size_t)bb * n + i) * L->kv_heads + h) * ORC_D;
        size_t slot = orc_wslot(W, bb, h, t);
        for (int c = 0; c < ORC_D; c++)
          x[c] = lambda ? orc_migrate(k[in + c], lambda[h * ORC_D + c]) : k[in + c];
        orc_quantize_group(x, ORC_D, 16, W->kc + slot * ORC_D, W->km + slot * 2, W->km + slot * 2 + 1);
        orc_quantize_group(v + in, ORC_D, 16, W->vc + slot * ORC_D, W->vm + slot * 2, W->vm + slot * 2 + 1);
      }
    W->n++;
    if (t - ORC_WINDOW >= 1) orc_wlayer_evict(W, t - ORC_WINDOW);
  }
  return 0;
}

/* Tokens held at INT16: the sink and the window, oldest first. */
int orc_wlayer_window_tokens(const orc_wlayer* W, int* tokens) {
  int c = 0;
  if (W->n > 0) tokens[c++] = 0;
  int lo = W->n - ORC_WINDOW > 1 ? W->n - ORC_WINDOW : 1;
  for (int t = lo; t < W->n; t++) tokens[c++] = t;
  return c;
}

/* ------------------------------------------------------------------------ */
/* Per-channel Key groups (KIVI's axis; the PM-KVQ note's training strategy  */
/* names group size 128 without an axis, and its comparison with KIVI names  */
/* KIVI's per-channel Key / per-token Value split).  Readings:               */
/*   - A Key group is one channel of one KV head over a block of 128         */
/*     consecutive tokens; Value groups stay one token's 128 channels.       */
/*   - The tokens of the block being filled (the last n mod 128) are held at */
/*     INT16, each quantized per token (Keys after the migration), as the    */
/*     note stores recent tokens at INT16.                                   */
/*   - When a block's 128th token arrives the block enters the progressive   */
/*     cache.  Keys: every staged INT16 Key is dequantized in fp32 as         */
/*     x = Z + code * (R / 65535) (one division, one multiply, one add, each */
/*     round-to-nearest, no fused multiply-add) and each channel's 128       */
/*     values are quantized by the affine quantizer directly at the cache's  */
/*     current width (tokens reach the cache directly at its width, as new   */
/*     tokens do after a shrink).  Values move by the block's shift chain    */
/*     from their INT16 codes, R and Z kept (R rescaled by the direct        */
/*     shift), as tokens leaving the sink + window store do.                 */
/*   - The progressive cache takes whole blocks: a block that does not fit   */
/*     at the current width shrinks the cache first.  Its capacity at every  */
/*     width is a multiple of 128 tokens (N * Fbit / 16 divisible by 128),   */
/*     so a shrink always finds the cache full.  A shrink treats the         */
/*     per-channel Key ranges as the per-token ones (kept by the Equivalent  */
/*     Right Shift, rescaled by the Direct Right Shift).                     */
/* ------------------------------------------------------------------------ */

#define ORC_KBLOCK 128

typedef struct {
  orc_layer main; /* codes and Value meta per token; its Key meta is unused */
  uint16_t* kmc;  /* [batch][kv_heads][n_f / 128][128][2]: per-channel Key (R, Z) per block */
  int n;          /* tokens appended */
  uint16_t* skc;  /* staging: [batch][kv_heads][128][128] INT16 codes, token t in slot t mod 128 */
  uint16_t* svc;
  uint16_t* skm; /* [batch][kv_heads][128][2] */
  uint16_t* svm;
} orc_clayer;

size_t orc_clayer_sizeof(void) { return sizeof(orc_clayer); }

int orc_clayer_init(orc_clayer* C, int batch, int kv_heads, int n_f, int fbit) {
  memset(C, 0, sizeof(*C));
  if (n_f <= 0 || ((int64_t)n_f * fbit / 16) % ORC_KBLOCK != 0 || ((int64_t)n_f * fbit) % 16 != 0) return -1;
  int rc = orc_layer_init(&C->main, batch, kv_heads, n_f, fbit);
  if (rc) return rc;
  size_t streams = (size_t)batch * kv_heads;
  C->kmc = (uint16_t*)calloc(streams * (size_t)n_f * 2, 2);
  C->skc = (uint16_t*)calloc(streams * ORC_KBLOCK * ORC_D, 2);
  C->svc = (uint16_t*)calloc(streams * ORC_KBLOCK * ORC_D, 2);
  C->skm = (uint16_t*)calloc(streams * ORC_KBLOCK * 2, 2);
  C->svm = (uint16_t*)calloc(streams * ORC_KBLOCK * 2, 2);
  if (!C->kmc || !C->skc || !C->svc || !C->skm || !C->svm) return -2;
  return 0;
}

void orc_clayer_free(orc_clayer* C) {
  orc_layer_free(&C->main);
  free(C->kmc);
  free(C->skc);
  free(C->svc);
  free(C->skm);
  free(C->svm);
  memset(C, 0, sizeof(*C));
}

static size_t orc_cstage(const orc_clayer* C, int b, int h, int s) {
  return ((size_t)b * C->main.kv_heads + h) * ORC_KBLOCK + s;
}
/* (R, Z) of channel c of block blk: index of its pair */
static size_t orc_ckm(const orc_clayer* C, int b, int h, int blk, int c) {
  return ((((size_t)b * C->main.kv_heads + h) * (C->main.n_f / ORC_KBLOCK) + blk) * ORC_D + c) * 2;
}

/* fp32 value of an INT16 code: Z + code * (R / 65535), three RN steps. */
float orc_int16_value(uint16_t code, uint16_t r_bits, uint16_t z_bits) {
  volatile float r = (float)orc_f16_to_f64(r_bits);
  volatile float z = (float)orc_f16_to_f64(z_bits);
  volatile float step = r / 65535.0f;
  volatile float p = (float)code * step;
  volatile float x = z + p;
  return x;
}

static int orc_clayer_shrink(orc_clayer* C) {
  orc_layer* L = &C->main;
  int rc = orc_layer_shrink(L);
  if (rc) return rc;
  if (L->shift_mode == 1) {
    int blocks = L->n / ORC_KBLOCK;
    for (int bb = 0; bb < L->batch; bb++)
      for (int h = 0; h < L->kv_heads; h++)
        for (int k = 0; k < blocks; k++)
          for (int c = 0; c < ORC_D; c++) {
            size_t i = orc_ckm(C, bb, h, k, c);
            C->kmc[i] = orc_drs_range(C->kmc[i], L->bits);
          }
  }
  return 0;
}

/* The full staged block enters the progressive cache. */
static void orc_clayer_move_block(orc_clayer* C) {
  orc_layer* L = &C->main;
  while (L->n + ORC_KBLOCK > orc_layer_capacity(L, L->bits))
    if (orc_clayer_shrink(C) != 0) return; /* unreachable: the caller checked the budget */
  const int blk = L->n / ORC_KBLOCK;
  float col[ORC_KBLOCK];
  uint16_t codes[ORC_KBLOCK];
  for (int bb = 0; bb < L->batch; bb++)
    for (int h = 0; h < L->kv_heads; h++) {
      for (int c = 0; c < ORC_D; c++) {
        for (int t = 0; t < ORC_KBLOCK; t++) {
          size_t s = orc_cstage(C, bb, h, t);
          col[t] = orc_int16_value(C->skc[s * ORC_D + c], C->skm[s * 2], C->skm[s * 2 + 1]);
        }
        size_t mi = orc_ckm(C, bb, h, blk, c);
        orc_quantize_group(col, ORC_KBLOCK, L->bits, codes, &C->kmc[mi], &C->kmc[mi + 1]);
        for (int t = 0; t < ORC_KBLOCK; t++) L->kc[orc_slot(L, bb, h, L->n + t) * ORC_D + c] = codes[t];
      }
      for (int t = 0; t < ORC_KBLOCK; t++) {
        size_t s = orc_cstage(C, bb, h, t), dst = orc_slot(L, bb, h, L->n + t);
        for (int c = 0; c < ORC_D; c++)
          L->vc[dst * ORC_D + c] = (uint16_t)orc_chain_code(C->svc[s * ORC_D + c], L->bits, L->shift_mode);
        L->vm[dst * 2] = orc_chain_range(C->svm[s * 2], L->bits, L->shift_mode);
        L->vm[dst * 2 + 1] = C->svm[s * 2 + 1];
      }
    }
  L->n += ORC_KBLOCK;
}

/* Append n tokens (same arguments as orc_layer_append).  Returns 1 when the
 * progressive cache could not hold the blocks completed by the call at Fbit
 * (nothing written). */
int orc_clayer_append(orc_clayer* C, const float* k, const float* v, int n, const float* lambda) {
  orc_layer* L = &C->main;
  if (n < 0) return -1;
  if (((int64_t)C->n + n) / ORC_KBLOCK * ORC_KBLOCK > (int64_t)L->n_f) return 1;
  float x[ORC_D];
  for (int i = 0; i < n; i++) {
    int t = C->n;
    for (int bb = 0; bb < L->batch; bb++)
      for (int h = 0; h < L->kv_heads; h++) {
        size_t in = (((size_t)bb * n + i) * L->kv_heads + h) * ORC_D;
        size_t s = orc_cstage(C, bb, h, t % ORC_KBLOCK);
        for (int c = 0; c < ORC_D; c++)
          x[c] = lambda ? orc_migrate(k[in + c], lambda[h * ORC_D + c]) : k[in + c];
        orc_quantize_group(x, ORC_D, 16, C->skc + s * ORC_D, C->skm + s * 2, C->skm + s * 2 + 1);
        orc_quantize_group(v + in, ORC_D, 16, C->svc + s * ORC_D, C->svm + s * 2, C->svm + s * 2 + 1);
      }
    C->n++;
    if (C->n % ORC_KBLOCK == 0) orc_clayer_move_block(C);
  }
  return 0;
}

/* Decode attention over a block with per-channel Key groups: the progressive
 * cache (Key channel c of token t dequantized with its block's (R_c, Z_c))
 * and the staged tokens at INT16, every token attended in fp64. */
int orc_cattention(const orc_clayer* C, const float* q, int q_heads, const float* lambda, double sm_scale,
                   double* out) {
  const orc_layer* L = &C->main;
  if (C->n <= 0 || q_heads % L->kv_heads) return -1;
  int g = q_heads / L->kv_heads;
  int T = C->n; /* main tokens 0 .. L->n - 1, then the staged ones */
  double* s = (double*)malloc(sizeof(double) * (size_t)T);
  double qp[ORC_D];
  if (!s) return -2;
  for (int bb = 0; bb < L->batch; bb++)
    for (int hq = 0; hq < q_heads; hq++) {
      int h = hq / g;
      const float* qq = q + ((size_t)bb * q_heads + hq) * ORC_D;
      for (int c = 0; c < ORC_D; c++)
        qp[c] = (double)qq[c] * (lambda ? (double)lambda[h * ORC_D + c] : 1.0);
      double mx = -INFINITY;
      for (int t = 0; t < T; t++) {
        double acc = 0.0;
        if (t < L->n) {
          size_t slot = orc_slot(L, bb, h, t);
          for (int c = 0; c < ORC_D; c++) {
            size_t mi = orc_ckm(C, bb, h, t / ORC_KBLOCK, c);
            acc += qp[c] * orc_dequant(L->kc[slot * ORC_D + c], C->kmc[mi], C->kmc[mi + 1], L->bits);
          }
        } else {
          size_t st = orc_cstage(C, bb, h, t % ORC_KBLOCK);
          for (int c = 0; c < ORC_D; c++)
            acc += qp[c] * orc_dequant(C->skc[st * ORC_D + c], C->skm[st * 2], C->skm[st * 2 + 1], 16);
        }
        s[t] = sm_scale * acc;
        if (s[t] > mx) mx = s[t];
      }
      double den = 0.0;
      for (int t = 0; t < T; t++) {
        s[t] = exp(s[t] - mx);
        den += s[t];
      }
      double* o = out + ((size_t)bb * q_heads + hq) * ORC_D;
      for (int c = 0; c < ORC_D; c++) o[c] = 0.0;
      for (int t = 0; t < T; t++) {
        const uint16_t *vc, *vm;
        int bits;
        if (t < L->n) {
          size_t slot = orc_slot(L, bb, h, t);
          vc = L->vc + slot * ORC_D, vm = L->vm + slot * 2, bits = L->bits;
        } else {
          size_t st = orc_cstage(C, bb, h, t % ORC_KBLOCK);
          vc = C->svc + st * ORC_D, vm = C->svm + st * 2, bits = 16;
        }
        double p = s[t] / den;
        for (int c = 0; c < ORC_D; c++) o[c] += p * orc_dequant(vc[c], vm[0], vm[1], bits);
      }
    }
  free(s);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode attention over the quantized cache, fp64.                          */
/* q: [batch][q_heads][128] (fp32 values of the bf16 queries).               */
/* lambda: [kv_heads][128] or NULL.  out: [batch][q_heads][128].             */
/* ------------------------------------------------------------------------ */

int orc_attention(const orc_layer* L, const float* q, int q_heads, const float* lambda,
                  double sm_scale, double* out) {
  if (L->n <= 0 || q_heads % L->kv_heads) return -1;
  int g = q_heads / L->kv_heads;
  int T = L->n;
  double* s = (double*)malloc(sizeof(double) * (size_t)T);
  double qp[ORC_D];
  if (!s) return -2;
  for (int bb = 0; bb < L->batch; bb++)
    for (int hq = 0; hq < q_heads; hq++) {
      int h = hq / g;
      const float* qq = q + ((size_t)bb * q_heads + hq) * ORC_D;
      for (int c = 0; c < ORC_D; c++)
        qp[c] = (double)qq[c] * (lambda ? (double)lambda[h * ORC_D + c] : 1.0);
      double mx = -INFINITY;
      for (int t = 0; t < T; t++) {
        size_t slot = orc_slot(L, bb, h, t);
        uint16_t rb = L->km[slot * 2], zb = L->km[slot * 2 + 1];
        double acc = 0.0;
        for (int c = 0; c < ORC_D; c++)
          acc += qp[c] * orc_dequant(L->kc[slot * ORC_D + c], rb, zb, L->bits);
        s[t] = sm_scale * acc;
        if (s[t] > mx) mx = s[t];
      }
      double den = 0.0;
      for (int t = 0; t < T; t++) {
        s[t] = exp(s[t] - mx);
        den += s[t];
      }
      double* o = out + ((size_t)bb * q_heads + hq) * ORC_D;
      for (int c = 0; c < ORC_D; c++) o[c] = 0.0;
      for (int t = 0; t < T; t++) {
        size_t slot = orc_slot(L, bb, h, t);
        uint16_t rb = L->vm[slot * 2], zb = L->vm[slot * 2 + 1];
        double p = s[t] / den;
        for (int c = 0; c < ORC_D; c++)
          o[c] += p * orc_dequant(L->vc[slot * ORC_D + c], rb, zb, L->bits);
      }
    }
  free(s);
  return 0;
}

/* Decode attention over a block with the sink + window: every token the
 * block holds -- the sink and the window at 16 bits, the progressive cache
 * at its width -- dequantized and attended in fp64. */
int orc_wattention(const orc_wlayer* W, const float* q, int q_heads, const float* lambda, double sm_scale,
                   double* out) {
  const orc_layer* L = &W->main;
  if (W->n <= 0 || q_heads % L->kv_heads) return -1;
  int g = q_heads / L->kv_heads;
  int* wt = (int*)malloc(sizeof(int) * (ORC_WINDOW + 1));
  int nw = orc_wlayer_window_tokens(W, wt);
  int T = L->n + nw;
  double* s = (double*)malloc(sizeof(double) * (size_t)T);
  double qp[ORC_D];
  if (!s || !wt) return -2;
  for (int bb = 0; bb < L->batch; bb++)
    for (int hq = 0; hq < q_heads; hq++) {
      int h = hq / g;
      const float* qq = q + ((size_t)bb * q_heads + hq) * ORC_D;
      for (int c = 0; c < ORC_D; c++)
        qp[c] = (double)qq[c] * (lambda ? (double)lambda[h * ORC_D + c] : 1.0);
      double mx = -INFINITY;
      for (int t = 0; t < T; t++) {
        const uint16_t *kc, *km;
        int bits;
        if (t < L->n) {
          size_t slot = orc_slot(L, bb, h, t);
          kc = L->kc + slot * ORC_D, km = L->km + slot * 2, bits = L->bits;
        } else {
          size_t slot = orc_wslot(W, bb, h, wt[t - L->n]);
          kc = W->kc + slot * ORC_D, km = W->km + slot * 2, bits = 16;
        }
        double acc = 0.0;
        for (int c = 0; c < ORC_D; c++) acc += qp[c] * orc_dequant(kc[c], km[0], km[1], bits);
        s[t] = sm_scale * acc;
        if (s[t] > mx) mx = s[t];
      }
      double den = 0.0;
      for (int t = 0; t < T; t++) {
        s[t] = exp(s[t] - mx);
        den += s[t];
      }
      double* o = out + ((size_t)bb * q_heads + hq) * ORC_D;
      for (int c = 0; c < ORC_D; c++) o[c] = 0.0;
      for (int t = 0; t < T; t++) {
        const uint16_t *vc, *vm;
        int bits;
        if (t < L->n) {
          size_t slot = orc_slot(L, bb, h, t);
          vc = L->vc + slot * ORC_D, vm = L->vm + slot * 2, bits = L->bits;
        } else {
          size_t slot = orc_wslot(W, bb, h, wt[t - L->n]);
          vc = W->vc + slot * ORC_D, vm = W->vm + slot * 2, bits = 16;
        }
        double p = s[t] / den;
        for (int c = 0; c < ORC_D; c++) o[c] += p * orc_dequant(vc[c], vm[0], vm[1], bits);
      }
    }
  free(s);
  free(wt);
  return 0;
}

/* Plain fp64 attention over given real-valued K and V (no quantization):
 * q [q_heads][d], k, v [T][kv_heads][d]; used for the migration-invariance
 * and brute-force pins. */
void orc_attention_dense(const double* q, const double* k, const double* v, int T, int q_heads,
                         int kv_heads, int d, double sm_scale, double* out) {
  int g = q_heads / kv_heads;
  double* s = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  for (int hq = 0; hq < q_heads; hq++) {
    int h = hq / g;
    double mx = -INFINITY;
    for (int t = 0; t < T; t++) {
      double acc = 0.0;
      for (int c = 0; c < d; c++) acc += q[hq * d + c] * k[((size_t)t * kv_heads + h) * d + c];
      s[t] = sm_scale * acc;
      if (s[t] > mx) mx = s[t];
    }
    double den = 0.0;
    for (int t = 0; t < T; t++) {
      s[t] = exp(s[t] - mx);
      den += s[t];
    }
    for (int c = 0; c < d; c++) {
      double o = 0.0;
      for (int t = 0; t < T; t++) o += s[t] / den * v[((size_t)t * kv_heads + h) * d + c];
      out[hq * d + c] = o;
    }
  }
  free(s);
}
