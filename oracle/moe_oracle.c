/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle of the Step-3.5-Flash
 * routed-expert MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this
 * file: only the test suite, the package's smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or constant generator with the CUDA
 * library; both sides read the same seeded inputs and nothing else.
 *
 * What the layer computes (sources, all on the llm-atlas page "Step-3.5-Flash",
 * table "Champs bruts du config.json" unless noted):
 *   - moe_num_experts = 288, moe_top_k = 8: every token is routed to 8 of 288 experts;
 *   - norm_expert_weight = true: the weights of the chosen experts are renormalised so
 *     that they sum to 1;
 *   - need_fp32_gate = true: router scores are fp32 values;
 *   - moe_intermediate_size = 1280, share_expert_dim = 1280: the routed experts and the
 *     always-on shared expert are gated FFNs of width 1280 on hidden size 4096;
 *   - the same page's "FFN / MoE" paragraph: a sparse mixture of 288 routed experts with
 *     top-8 routing.
 * The pages leave the score function and the activation open; this oracle takes a
 * softmax router, ties broken toward the lower expert index, and SiLU(gate)*up.
 *
 * Precision:
 *   - router score s[t,e] = the EXACT real value of sum_h x[t,h]*W_r[e,h], rounded
 *     once to fp32, nearest-even (every product of two bf16 or two fp32 numbers is an
 *     exact dyadic rational; they are summed without error in integer bins);
 *   - key[t,e] = fp32(s[t,e] + b[e]) when a router bias is given, else s[t,e];
 *   - selection by (key descending, expert index ascending), stored by ascending index;
 *   - routing weights: softmax over the selected keys, in fp64;
 *   - expert FFNs and the combine: fp64, sequential accumulation;
 *   - SwiGLU limits (same table: swiglu_limits "0.0x46 + 7x2" for the routed experts,
 *     swiglu_limits_shared "0.0x47 + 16x1" for the shared one): the page gives only the
 *     values.  Read here as a clamp of the activation inputs when the limit L > 0:
 *     gate <- min(gate, L), up <- min(max(up, -L), L), then SiLU(gate)*up; L = 0 means
 *     no clamp (the value of almost every layer).
 *
 * The router as configured (sigmoid scores, selection-only bias, weights scaled by the
 * routing factor) is a second routing mode, described above oracle_route_mode().
 *
 * Parity status: every function here is pinned by tests (exact rational sums,
 * brute-force subset enumeration, closed forms, high-precision decimal values and
 * invariants); none is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_F32 0
#define OR_BF16 1

/* ------------------------------------------------------------------------------------
 * Exact dot product.
 *
 * Every finite bf16 or fp32 value v is m * 2^q with an integer m (|m| < 2^24) and an
 * integer q.  A product of two such values is (m1*m2) * 2^(q1+q2), exact.  We add each
 * product's integer mantissa into a bin indexed by its exponent (int64 bins; a bf16
 * product has |m1*m2| < 2^16, an fp32 product is split into two 24-bit halves), then
 * turn the bins into one big binary integer by carry propagation and round it once to
 * the nearest fp32 (ties to even), with subnormal results handled.
 * ---------------------------------------------------------------------------------- */

/* smallest product exponent: fp32 subnormal * subnormal = 2^-149 * 2^-149 */
#define BIN_EMIN (-298)
/* largest exponent a bin can receive: bf16 max 2^120*2^120 = 2^240, fp32 hi half 2^232,
   bf16 x fp32 hi half 2^248 */
#define BIN_EMAX 249
#define NBINS (BIN_EMAX - BIN_EMIN + 1)
/* room for the carries of up to 2^62 in magnitude above the top bin */
#define NBITS (NBINS + 72)

typedef struct {
  int32_t m; /* signed integer mantissa */
  int32_t q; /* exponent: value = m * 2^q */
  int finite;
} dyadic;

static dyadic decode_f32(uint32_t bits) {
  dyadic d;
  uint32_t sign = bits >> 31, ex = (bits >> 23) & 0xFF, fr = bits & 0x7FFFFF;
  d.finite = (ex != 0xFF);
  if (ex == 0) {
    d.m = (int32_t)fr;
    d.q = -149;
  } else {
    d.m = (int32_t)(fr | 0x800000u);
    d.q = (int32_t)ex - 150;
  }
  if (sign) d.m = -d.m;
  return d;
}

static dyadic decode_bf16(uint16_t bits) {
  dyadic d;
  uint32_t sign = bits >> 15, ex = (bits >> 7) & 0xFF, fr = bits & 0x7F;
  d.finite = (ex != 0xFF);
  if (ex == 0) {
    d.m = (int32_t)fr;
    d.q = -133;
  } else {
    d.m = (int32_t)(fr | 0x80u);
    d.q = (int32_t)ex - 134;
  }
  if (sign) d.m = -d.m;
  return d;
}

/* Round the integer  sum_b bins[b] * 2^(b + BIN_EMIN)  to the nearest fp32. */
static float round_bins_to_f32(const int64_t* bins) {
  /* 1. two's-complement bit string of the sum by carry propagation (floor division) */
  static __thread uint8_t bit[NBITS];
  int64_t carry = 0;
  int nb = 0;
  for (int b = 0; b < NBINS; ++b) {
    /* v = bins[b] + carry may overflow only if |bins| ~ 2^63: excluded by the
       caller's length limit */
    int64_t v = bins[b] + carry;
    bit[nb++] = (uint8_t)(v & 1);
    carry = (v - (v & 1)) / 2; /* exact floor(v/2) */
  }
  while (carry != 0 && carry != -1) {
    bit[nb++] = (uint8_t)(carry & 1);
    carry = (carry - (carry & 1)) / 2;
  }
  int negative = (carry == -1);
  if (negative) { /* magnitude = two's complement of the bit string */
    int c = 1;
    for (int i = 0; i < nb; ++i) {
      int v = (bit[i] ^ 1) + c;
      bit[i] = (uint8_t)(v & 1);
      c = v >> 1;
    }
    /* c == 1 here would mean the magnitude is 2^nb: append it */
    if (c) bit[nb++] = 1;
  }
  /* 2. highest set bit */
  int top = -1;
  for (int i = nb - 1; i >= 0; --i)
    if (bit[i]) { top = i; break; }
  if (top < 0) return negative ? -0.0f : 0.0f; /* exact zero: +0 (carry 0) */
  int e_top = top + BIN_EMIN; /* value of the top bit is 2^e_top */
  /* 3. position of the last kept bit: 24 significant bits for normals, 2^-149 floor */
  int keep_lsb_exp = e_top - 23;
  if (keep_lsb_exp < -149) keep_lsb_exp = -149;
  int lsb = keep_lsb_exp - BIN_EMIN; /* bit index of the last kept bit (>= 0) */
  uint64_t mant = 0;
  for (int i = top; i >= lsb; --i) mant = (mant << 1) | bit[i];
  int round_bit = (lsb - 1 >= 0) ? bit[lsb - 1] : 0;
  int sticky = 0;
  for (int i = lsb - 2; i >= 0; --i)
    if (bit[i]) { sticky = 1; break; }
  if (round_bit && (sticky || (mant & 1))) mant += 1;
  /* mant * 2^keep_lsb_exp is exact in fp32 unless it overflows the range */
  double v = ldexp((double)mant, keep_lsb_exp);
  if (v > 3.4028234663852886e38) v = INFINITY; /* beyond FLT_MAX after rounding */
  float f = (float)v; /* exact: mant has <= 25 bits and the exponent is in range */
  return negative ? -f : f;
}

/* Exact sum_h x[h]*w[h] rounded once to fp32, x and w each bf16 or fp32.  Returns 0 on
   success, -1 on a non-finite input, -2 if the length could overflow a bin. */
static int exact_dot_mixed(int dtype_x, int dtype_w, int n, const void* x, const void* w, float* out) {
  int64_t bins[NBINS];
  memset(bins, 0, sizeof(bins));
  if (n > (1 << 30)) return -2;
  for (int h = 0; h < n; ++h) {
    dyadic a = dtype_x == OR_BF16 ? decode_bf16(((const uint16_t*)x)[h]) : decode_f32(((const uint32_t*)x)[h]);
    dyadic b = dtype_w == OR_BF16 ? decode_bf16(((const uint16_t*)w)[h]) : decode_f32(((const uint32_t*)w)[h]);
    if (!a.finite || !b.finite) return -1;
    if (a.m == 0 || b.m == 0) continue;
    int64_t p = (int64_t)a.m * (int64_t)b.m; /* |p| < 2^48 */
    int q = a.q + b.q;
    int64_t mag = p < 0 ? -p : p;
    int64_t sgn = p < 0 ? -1 : 1;
    int64_t lo = mag & 0xFFFFFF, hi = mag >> 24; /* both < 2^24 */
    bins[q - BIN_EMIN] += sgn * lo;
    if (hi) bins[q + 24 - BIN_EMIN] += sgn * hi;
  }
  *out = round_bins_to_f32(bins);
  return 0;
}

static int exact_dot_f32(int dtype, int n, const void* x, const void* w, float* out) {
  return exact_dot_mixed(dtype, dtype, n, x, w, out);
}

/* Exposed for the tests that pin the exact dot product on its own. */
int oracle_exact_dot(int dtype, int n, const void* x, const void* w, float* out) {
  return exact_dot_f32(dtype, n, x, w, out);
}
int oracle_exact_dot_mixed(int dtype_x, int dtype_w, int n, const void* x, const void* w, float* out) {
  return exact_dot_mixed(dtype_x, dtype_w, n, x, w, out);
}

static size_t esize(int dtype) { return dtype == OR_BF16 ? 2 : 4; }

static double to_f64(int dtype, const void* base, size_t i) {
  if (dtype == OR_BF16) {
    uint32_t b = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &b, 4);
    return (double)f;
  }
  return (double)((const float*)base)[i];
}

/* ------------------------------------------------------------------------------------
 * Router scores: s[t,e] = RN32(exact sum_h x[t,h] W_r[e,h]) for every token and expert
 * (router logits; fp32 scores per need_fp32_gate).  The router matrix may be fp32 with
 * bf16 tokens (need_fp32_gate read as fp32 router weights).
 * ---------------------------------------------------------------------------------- */
int oracle_router_scores_mixed(int dtype_x, int dtype_w, int64_t T, int H, int E, const void* x,
                               const void* Wr, float* s_out, int nthreads) {
  int err = 0;
  size_t es = esize(dtype_x), ews = esize(dtype_w);
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 16) reduction(| : err)
  for (int64_t te = 0; te < T * (int64_t)E; ++te) {
    int64_t t = te / E;
    int e = (int)(te % E);
    const char* xr = (const char*)x + (size_t)t * H * es;
    const char* wr = (const char*)Wr + (size_t)e * H * ews;
    float s;
    if (exact_dot_mixed(dtype_x, dtype_w, H, xr, wr, &s) != 0) err |= 1;
    s_out[te] = s;
  }
  return err ? -1 : 0;
}

int oracle_router_scores(int dtype, int64_t T, int H, int E, const void* x, const void* Wr,
                         float* s_out, int nthreads) {
  return oracle_router_scores_mixed(dtype, dtype, T, H, E, x, Wr, s_out, nthreads);
}

/* ------------------------------------------------------------------------------------
 * Routing of one token (softmax router, top-k, renormalised weights).
 *   key[e] = fp32(s[e] + b[e])   (b = 0 when no bias is given)
 *   S = the k experts first in the order (key descending, index ascending)
 *   stored by ascending expert index;
 *   w_j = exp(key_j - m) / sum_{i in S} exp(key_i - m), m = max_{i in S} key_i, fp64.
 * The full-softmax denominator over all E experts cancels under the renormalisation
 * that norm_expert_weight asks for, so it is never formed.
 * ---------------------------------------------------------------------------------- */
static int beats(float ka, int a, float kb, int b) { /* a is ordered before b */
  return (ka > kb) || (ka == kb && a < b);
}

/* ------------------------------------------------------------------------------------
 * The router as configured on the llm-atlas page "Step-3.5-Flash", table "Champs bruts
 * du config.json": moe_router_activation = sigmoid, use_moe_router_bias = true,
 * moe_router_scaling_factor = 3, norm_expert_weight = true, need_fp32_gate = true.
 * Reading (the page gives the fields only): the fp32 score of expert e is
 *   p_e = sigma32(s_e) = fp32(1 / (1 + e^(-s_e))),
 * the bias only steers the selection, key_e = fp32(p_e + b_e), and the weights are the
 * chosen scores renormalised and scaled: w_j = scale * p_j / sum_{i in S} p_i (fp64).
 *
 * e^z is evaluated by a fixed sequence of IEEE fp64 operations, so that any IEEE
 * implementation of the same steps (the CUDA library's own is one) returns the same
 * bits: z = n ln2 + r with n = round(z / ln 2) and ln 2 split in two (the first part
 * has 42 significant bits, so n * ln2_hi is exact for the |n| < 2^11 used here),
 * |r| <= ln2/2 + tiny, then the degree-13 Taylor polynomial of e^r in Horner form with
 * fused multiply-adds (truncation < 6e-18 relative), then an exact scaling by 2^n.
 * The file is compiled with -ffp-contract=off: no other operation is fused.
 * ---------------------------------------------------------------------------------- */
static double exp_fixed(double z) {
  const double inv_ln2 = 0x1.71547652b82fep+0; /* RN(1 / ln 2) */
  const double ln2_hi = 0x1.62e42fefa3800p-1;  /* ln 2 = 0.693147180559945309417... cut to 42 bits */
  const double ln2_lo = 0x1.ef35793c76730p-45; /* RN(ln 2 - ln2_hi) */
  double n = nearbyint(z * inv_ln2);
  double r = (z - n * ln2_hi) - n * ln2_lo;
  double q = 1.0 / 6227020800.0; /* 1/13! */
  q = fma(q, r, 1.0 / 479001600.0);
  q = fma(q, r, 1.0 / 39916800.0);
  q = fma(q, r, 1.0 / 3628800.0);
  q = fma(q, r, 1.0 / 362880.0);
  q = fma(q, r, 1.0 / 40320.0);
  q = fma(q, r, 1.0 / 5040.0);
  q = fma(q, r, 1.0 / 720.0);
  q = fma(q, r, 1.0 / 120.0);
  q = fma(q, r, 1.0 / 24.0);
  q = fma(q, r, 1.0 / 6.0);
  q = fma(q, r, 0.5);
  q = fma(q, r, 1.0);
  q = fma(q, r, 1.0);
  uint64_t bits = (uint64_t)((int64_t)n + 1023) << 52; /* 2^n, a normal number here */
  double two_n;
  memcpy(&two_n, &bits, sizeof two_n);
  return q * two_n;
}

/* sigma32(s): 0 below s = -110 (sigma < 2e-48 rounds to 0 in fp32), 1 above s = 40
 * (1 - sigma < 5e-18 rounds to 1), else fp32(1 / (1 + e^(-s))). */
static float sigmoid32(float sv) {
  double z = (double)sv;
  if (z < -110.0) return 0.0f;
  if (z > 40.0) return 1.0f;
  return (float)(1.0 / (1.0 + exp_fixed(-z)));
}

int oracle_sigmoid32(int64_t n, const float* s, float* p) {
  for (int64_t i = 0; i < n; ++i) p[i] = sigmoid32(s[i]);
  return 0;
}

/* mode 0: softmax router (above); mode 1: sigmoid router with selection-only bias and
   weights scale * p / sum p. */
int oracle_route_mode(int64_t T, int E, int k, const float* s, const float* bias, int mode,
                      double scale, int32_t* idx_out, float* w_out, double* w64_out) {
  if (k < 1 || k > E || (mode != 0 && mode != 1)) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    float* key = (float*)malloc(sizeof(float) * E);
    float* prob = (float*)malloc(sizeof(float) * E);
    int* chosen = (int*)calloc(E, sizeof(int));
    for (int e = 0; e < E; ++e) {
      float v = s[t * E + e];
      if (mode == 1) v = sigmoid32(v);
      prob[e] = v;
      key[e] = bias ? (float)(v + bias[e]) : v; /* fp32 + fp32 -> RN fp32 */
    }
    /* k passes of "pick the best not yet chosen" */
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (chosen[e]) continue;
        if (best < 0 || beats(key[e], e, key[best], best)) best = e;
      }
      chosen[best] = 1;
    }
    /* ascending expert index */
    int j = 0;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
      if (chosen[e]) {
        idx_out[t * k + j++] = e;
        if ((double)key[e] > m) m = (double)key[e];
      }
    double z = 0.0;
    if (mode == 0) {
      for (j = 0; j < k; ++j) z += exp((double)key[idx_out[t * k + j]] - m);
      for (j = 0; j < k; ++j) {
        double w = exp((double)key[idx_out[t * k + j]] - m) / z;
        if (w64_out) w64_out[t * k + j] = w;
        if (w_out) w_out[t * k + j] = (float)w;
      }
    } else {
      for (j = 0; j < k; ++j) z += (double)prob[idx_out[t * k + j]];
      for (j = 0; j < k; ++j) {
        double w = z > 0.0 ? scale * (double)prob[idx_out[t * k + j]] / z : scale / k;
        if (w64_out) w64_out[t * k + j] = w;
        if (w_out) w_out[t * k + j] = (float)w;
      }
    }
    free(key);
    free(prob);
    free(chosen);
  }
  return 0;
}

int oracle_route(int64_t T, int E, int k, const float* s, const float* bias, int32_t* idx_out,
                 float* w_out, double* w64_out) {
  return oracle_route_mode(T, E, k, s, bias, 0, 1.0, idx_out, w_out, w64_out);
}

/* ------------------------------------------------------------------------------------
 * Dispatch bookkeeping by plain counting:
 *   counts[e]  = number of (token, slot) assignments routed to e;
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e];
 *   perm[offsets[e] + r] = t*k + j for the r-th token (ascending t) routed to e;
 *   inv_perm[t*k + j]    = position of that assignment in perm.
 * ---------------------------------------------------------------------------------- */
int oracle_dispatch(int64_t T, int E, int k, const int32_t* idx, int32_t* counts,
                    int32_t* offsets, int32_t* perm, int32_t* inv_perm) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < T * k; ++a) {
    int e = idx[a];
    if (e < 0 || e >= E) return -1;
    counts[e]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* fill = (int32_t*)calloc(E, sizeof(int32_t));
  for (int64_t t = 0; t < T; ++t)  /* token order makes the pass stable */
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      int32_t pos = offsets[e] + fill[e]++;
      perm[pos] = (int32_t)(t * k + j);
      if (inv_perm) inv_perm[t * k + j] = pos;
    }
  free(fill);
  return 0;
}

/* ------------------------------------------------------------------------------------
 * One gated FFN on one token, fp64:
 *   g_i = sum_h x_h Wgu[i, h],  u_i = sum_h x_h Wgu[I + i, h]     (gate rows, then up rows)
 *   a_i = SiLU(g_i) * u_i,      SiLU(z) = z / (1 + exp(-z))
 *   out_h += scale * sum_i a_i Wd[h, i]
 * ---------------------------------------------------------------------------------- */
/* SiLU(gate) * up with the SwiGLU limit L (0: none) applied to the inputs. */
static double swiglu(double g, double u, double limit) {
  if (limit > 0.0) {
    if (g > limit) g = limit;
    if (u > limit) u = limit;
    if (u < -limit) u = -limit;
  }
  return g / (1.0 + exp(-g)) * u;
}

static void gated_ffn_acc(int dtype, int H, int I, const void* xrow, const void* Wgu,
                          const void* Wd, double scale, double limit, double* out,
                          double* a /*[I]*/) {
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      double xv = to_f64(dtype, xrow, h);
      g += xv * to_f64(dtype, Wgu, (size_t)i * H + h);
      u += xv * to_f64(dtype, Wgu, (size_t)(I + i) * H + h);
    }
    a[i] = swiglu(g, u, limit);
  }
  for (int h = 0; h < H; ++h) {
    double o = 0.0;
    for (int i = 0; i < I; ++i) o += a[i] * to_f64(dtype, Wd, (size_t)h * I + i);
    out[h] += scale * o;
  }
}

/* The intermediate activation of one token through one expert (exposed so that the
   tests can pin the gate/up/SiLU step on its own). */
int oracle_expert_act(int dtype, int H, int I, const void* xrow, const void* Wgu_e,
                      double limit, double* act_out) {
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      double xv = to_f64(dtype, xrow, h);
      g += xv * to_f64(dtype, Wgu_e, (size_t)i * H + h);
      u += xv * to_f64(dtype, Wgu_e, (size_t)(I + i) * H + h);
    }
    act_out[i] = swiglu(g, u, limit);
  }
  return 0;
}

/* ------------------------------------------------------------------------------------
 * Blockwise FP8 expert weights (the low-precision expert weights for decode).
 *
 * A weight matrix W [R, K] is stored as one byte per element, an FP8 E4M3 code, plus one
 * scale byte per 128 x 128 block, an E8M0 power of two; the weight it stands for is
 *   W[r, c] = e4m3(q[r, c]) * e8m0(s[r / 128, c / 128]),  s laid out [ceil(R/128), ceil(K/128)].
 * Formats (OCP 8-bit floating point and microscaling formats):
 *   E4M3: sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
 *         subnormals m/8 * 2^-6; no infinities; S.1111.111 is NaN; largest finite 448;
 *   E8M0: an unsigned biased exponent, 2^(v - 127); v = 255 is NaN.
 * Every such product is exact in fp64.  The layer is then the same gated FFNs on these
 * weights (the tokens stay bf16), in fp64 as above.
 * ---------------------------------------------------------------------------------- */
static double decode_e4m3(uint8_t c) {
  int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9); /* m/8 * 2^-6 */
  else
    v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return sgn ? -v : v;
}

static double decode_e8m0(uint8_t v) { return v == 255 ? NAN : ldexp(1.0, (int)v - 127); }

/* the two decodings of every byte, filled once (before any parallel region) */
static double e4m3_val[256], e8m0_val[256];
static int fp8_tables_ready = 0;
static void fp8_tables(void) {
  if (fp8_tables_ready) return;
  for (int c = 0; c < 256; ++c) {
    e4m3_val[c] = decode_e4m3((uint8_t)c);
    e8m0_val[c] = decode_e8m0((uint8_t)c);
  }
  fp8_tables_ready = 1;
}

typedef struct {
  const uint8_t* q; /* [R, K] codes */
  const uint8_t* s; /* [ceil(R/128), ceil(K/128)] scales */
  int K;
} fp8_mat;

static double fp8_at(fp8_mat w, size_t r, int c) {
  int kb = (w.K + 127) / 128;
  return e4m3_val[w.q[r * (size_t)w.K + c]] * e8m0_val[w.s[(r / 128) * (size_t)kb + c / 128]];
}

int oracle_dequant_e4m3(int64_t R, int K, const uint8_t* q, const uint8_t* s, double* out) {
  fp8_mat w = {q, s, K};
  fp8_tables();
  for (int64_t r = 0; r < R; ++r)
    for (int c = 0; c < K; ++c) out[r * (int64_t)K + c] = fp8_at(w, (size_t)r, c);
  return 0;
}

/* gated_ffn_acc with FP8 weights: gu is [2I, H] (gate rows, then up rows), d is [H, I] */
static void gated_ffn_acc_fp8(int H, int I, const uint16_t* xrow, fp8_mat gu, fp8_mat d, double scale,
                              double limit, double* out, double* a /*[I]*/) {
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      double xv = to_f64(OR_BF16, xrow, h);
      g += xv * fp8_at(gu, (size_t)i, h);
      u += xv * fp8_at(gu, (size_t)(I + i), h);
    }
    a[i] = swiglu(g, u, limit);
  }
  for (int h = 0; h < H; ++h) {
    double o = 0.0;
    for (int i = 0; i < I; ++i) o += a[i] * fp8_at(d, (size_t)h, i);
    out[h] += scale * o;
  }
}

/* oracle_moe_tokens with bf16 tokens and FP8 weights.  Per routed expert e the codes are
   Wgu_q[e] [2I, H] and Wd_q[e] [H, I]; the scale tables are Wgu_s[e] [ceil(2I/128),
   ceil(H/128)] and Wd_s[e] [ceil(H/128), ceil(I/128)], stacked by expert like the codes. */
int oracle_moe_tokens_fp8(int64_t ntok, const int64_t* tok, int H, int E, int k, int I, int Is,
                          const uint16_t* x, const int32_t* idx, const double* w,
                          const uint8_t* Wgu_q, const uint8_t* Wgu_s, const uint8_t* Wd_q,
                          const uint8_t* Wd_s, const uint8_t* Wsgu_q, const uint8_t* Wsgu_s,
                          const uint8_t* Wsd_q, const uint8_t* Wsd_s, double limit,
                          double limit_shared, double* y, int nthreads) {
  const size_t gu_sc = (size_t)((2 * I + 127) / 128) * ((H + 127) / 128);
  const size_t d_sc = (size_t)((H + 127) / 128) * ((I + 127) / 128);
  int bad = 0;
  fp8_tables();
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t n = 0; n < ntok; ++n) {
    int64_t t = tok[n];
    const uint16_t* xr = x + (size_t)t * H;
    double* out = y + (size_t)n * H;
    int Imax = I > Is ? I : Is;
    double* a = (double*)malloc(sizeof(double) * (Imax > 0 ? Imax : 1));
    for (int h = 0; h < H; ++h) out[h] = 0.0;
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      if (e < 0 || e >= E) {
        bad |= 1;
        continue;
      }
      fp8_mat gu = {Wgu_q + (size_t)e * 2 * I * H, Wgu_s + (size_t)e * gu_sc, H};
      fp8_mat d = {Wd_q + (size_t)e * H * I, Wd_s + (size_t)e * d_sc, I};
      gated_ffn_acc_fp8(H, I, xr, gu, d, w[t * k + j], limit, out, a);
    }
    if (Wsgu_q && Wsd_q && Is > 0) {
      fp8_mat gu = {Wsgu_q, Wsgu_s, H};
      fp8_mat d = {Wsd_q, Wsd_s, Is};
      gated_ffn_acc_fp8(H, Is, xr, gu, d, 1.0, limit_shared, out, a);
    }
    free(a);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------------------
 * Layer output for a list of tokens, given their routing:
 *   y_t = sum_j w[t,j] * FFN_{idx[t,j]}(x_t) + FFN_shared(x_t)      (fp64)
 * The shared expert (share_expert_dim) is always on with weight 1; pass NULL shared
 * weights for a layer without one.  Weight layouts: Wgu [E, 2I, H], Wd [E, H, I],
 * Wsgu [2Is, H], Wsd [H, Is].  tok[n] is the token whose output goes to y[n, :];
 * idx/w are indexed by token.  limit / limit_shared: SwiGLU limits of the routed and the
 * shared experts (0: none).
 * ---------------------------------------------------------------------------------- */
int oracle_moe_tokens(int dtype, int64_t ntok, const int64_t* tok, int H, int E, int k, int I,
                      int Is, const void* x, const int32_t* idx, const double* w,
                      const void* Wgu, const void* Wd, const void* Wsgu, const void* Wsd,
                      double limit, double limit_shared, double* y, int nthreads) {
  size_t es = esize(dtype);
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t n = 0; n < ntok; ++n) {
    int64_t t = tok[n];
    const char* xr = (const char*)x + (size_t)t * H * es;
    double* out = y + (size_t)n * H;
    int Imax = I > Is ? I : Is;
    double* a = (double*)malloc(sizeof(double) * (Imax > 0 ? Imax : 1));
    for (int h = 0; h < H; ++h) out[h] = 0.0;
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      if (e < 0 || e >= E) {
        bad |= 1;
        continue;
      }
      const char* gu = (const char*)Wgu + (size_t)e * 2 * I * H * es;
      const char* d = (const char*)Wd + (size_t)e * H * I * es;
      gated_ffn_acc(dtype, H, I, xr, gu, d, w[t * k + j], limit, out, a);
    }
    if (Wsgu && Wsd && Is > 0) gated_ffn_acc(dtype, H, Is, xr, Wsgu, Wsd, 1.0, limit_shared, out, a);
    free(a);
  }
  return bad ? -1 : 0;
}
