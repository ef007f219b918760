// router.cu -- router scores, certified top-k selection and renormalised softmax weights.
//
// The routing decision must equal the one made on the exact fp32 router score
// s[t,e] = RN32(sum_h x[t,h] W_r[e,h]) (llm-atlas page "Step-3.5-Flash", table "Champs
// bruts du config.json": need_fp32_gate true, moe_top_k 8, norm_expert_weight true).
// A fast score s^ comes with a rigorous bound |s^ - s_real| <= delta, so the fp32 key of
// an expert lies in [key(s^ - delta), key(s^ + delta)].  Each candidate is classified as
// certainly chosen, certainly not chosen, or undecided; only undecided ones are
// recomputed, in fp64 (delta ~ 2^-41 relative) and, if that is still not conclusive, with
// an exact integer dot product.
//
//   bf16 tokens: a tcgen05 GEMM (fp32 accumulation over short slices, the slices added in
//                fp64; small batches split the reduction over blocks) scores, then a
//                selection kernel;
//   fp32 tokens, or more experts than tensor memory holds: one kernel computes fp64 scores
//                on the CUDA cores; the last block of each token group selects for them.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <limits.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr double kU53 = 1.1102230246251565e-16;  // 2^-53
constexpr double kU23 = 1.1920928955078125e-07;  // 2^-23

// ---------------------------------------------------------------------------------------
// Upper bounds of row 2-norms, fp64: sqrt(sum v^2) rounded up, with the fp64 summation
// error (at most n*2^-53 relative for n terms) covered by a factor (1 + 2 n 2^-53).
// One warp per row.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ double norm_ub_from_sumsq(double ss, int H) {
  const double infl = __dadd_ru(1.0, __dmul_ru(2.0 * H, kU53));
  return __dsqrt_ru(__dmul_ru(ss, infl));
}

template <typename T>
__device__ double warp_sumsq(const T* __restrict__ p, int H) {
  const int lane = threadIdx.x & 31;
  constexpr int V = Vec16<T>::N;
  double ss = 0.0;
  const int nv = H / V;
  for (int vb = lane; vb < nv; vb += 4 * 32) {
    Vec16<T> a[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (vb + 32 * u < nv) a[u] = ld16(p + (vb + 32 * u) * V);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (vb + 32 * u >= nv) break;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const double d = static_cast<double>(to_f32(a[u].v[j]));
        ss = fma(d, d, ss);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  return ss;
}

// rows [0, rows_a) of A then [0, rows_b) of B, one warp per row
template <typename T>
__global__ void row_norm_ub_kernel(const T* __restrict__ A, int64_t rows_a, double* __restrict__ out_a,
                                   const T* __restrict__ B, int64_t rows_b, double* __restrict__ out_b,
                                   int H) {
  pdl_wait();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row < rows_a + rows_b) {
    const bool first = row < rows_a;
    const int64_t r = first ? row : row - rows_a;
    const double ss = warp_sumsq((first ? A : B) + r * H, H);
    if ((threadIdx.x & 31) == 0) (first ? out_a : out_b)[r] = norm_ub_from_sumsq(ss, H);
  }
}

// ---------------------------------------------------------------------------------------
// Exact dot product of one (token, expert) pair by one warp, rounded once to fp32.
// Every bf16/fp32 value is m * 2^q with an integer m.  Each lane adds its products
// exactly into a 128-bit fixed-point accumulator anchored 60 bits below its largest
// product exponent; products further below go straight into int64 exponent bins in
// shared memory.  The lane accumulators are then added into the bins (three 42-bit
// pieces each), the bins are folded into 32-bit limbs, and the integer is rounded to the
// nearest fp32 (ties to even, subnormals included).
// ---------------------------------------------------------------------------------------
constexpr int kQMin = -298;               // smallest product exponent (fp32 subnormal^2)
constexpr int kQMax = 270;                // largest bin needed (anchor + 84 for bf16 max^2)
constexpr int kNBins = kQMax - kQMin + 1;
constexpr int kNLimbs = (kNBins + 31) / 32 + 4;

__device__ __forceinline__ void decode(float v, int& m, int& q) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t ex = (b >> 23) & 0xFF, fr = b & 0x7FFFFF;
  m = ex ? static_cast<int>(fr | 0x800000u) : static_cast<int>(fr);
  q = ex ? static_cast<int>(ex) - 150 : -149;
  if (b >> 31) m = -m;
}
__device__ __forceinline__ void decode(__nv_bfloat16 v, int& m, int& q) {
  const uint32_t b = __bfloat16_as_ushort(v);
  const uint32_t ex = (b >> 7) & 0xFF, fr = b & 0x7F;
  m = ex ? static_cast<int>(fr | 0x80u) : static_cast<int>(fr);
  q = ex ? static_cast<int>(ex) - 134 : -133;
  if (b >> 15) m = -m;
}

__device__ float round_limbs_rn32(const uint32_t* d, int nl, bool negative) {
  int top_limb = -1;
  for (int j = nl - 1; j >= 0; --j)
    if (d[j]) { top_limb = j; break; }
  if (top_limb < 0) return 0.0f;
  const int P = top_limb * 32 + (31 - __clz(d[top_limb]));  // index of the top set bit
  const int e_top = P + kQMin;
  int lsb_exp = e_top - 23;
  if (lsb_exp < -149) lsb_exp = -149;
  const int lsb = lsb_exp - kQMin;  // >= 0
  auto bit = [&](int i) -> uint32_t { return (i < 0) ? 0u : (d[i >> 5] >> (i & 31)) & 1u; };
  uint32_t mant = 0;
  for (int i = P; i >= lsb; --i) mant = (mant << 1) | bit(i);
  const uint32_t rb = bit(lsb - 1);
  bool sticky = false;
  const int sb = lsb - 2;  // bits [0, sb] are sticky
  if (sb >= 0) {
    for (int j = 0; j < (sb >> 5); ++j) sticky |= (d[j] != 0);
    const uint32_t partial =
        d[sb >> 5] & (((sb & 31) == 31) ? 0xFFFFFFFFu : ((2u << (sb & 31)) - 1u));
    sticky |= (partial != 0);
  }
  if (rb && (sticky || (mant & 1u))) mant += 1;
  const double v = ldexp(static_cast<double>(mant), lsb_exp);
  const float f = (v > static_cast<double>(FLT_MAX)) ? __int_as_float(0x7f800000) : static_cast<float>(v);
  return negative ? -f : f;
}

__device__ __forceinline__ void bin_add(long long* bins, int q, long long v) {
  atomicAdd(reinterpret_cast<unsigned long long*>(&bins[q - kQMin]), static_cast<unsigned long long>(v));
}

template <typename TA, typename TB>
__device__ __noinline__ float warp_exact_dot_rn32(const TA* __restrict__ a, const TB* __restrict__ b, int H,
                                     long long* bins /* kNBins, warp-private smem */,
                                     uint32_t* limbs /* kNLimbs, warp-private smem */) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < kNBins; i += 32) bins[i] = 0;
  __syncwarp();
  // pass 1: this lane's largest product exponent
  int qmax = INT_MIN;
  for (int h = lane; h < H; h += 32) {
    int m1, q1, m2, q2;
    decode(a[h], m1, q1);
    decode(b[h], m2, q2);
    if (m1 != 0 && m2 != 0) qmax = max(qmax, q1 + q2);
  }
  if (qmax != INT_MIN) {
    const int anchor = max(qmax - 60, kQMin);
    __int128 acc = 0;
    for (int h = lane; h < H; h += 32) {
      int m1, q1, m2, q2;
      decode(a[h], m1, q1);
      decode(b[h], m2, q2);
      const long long p = static_cast<long long>(m1) * m2;  // |p| < 2^48 (bf16 x fp32: < 2^32)
      if (p == 0) continue;
      const int q = q1 + q2;
      if (q >= anchor) {
        acc += static_cast<__int128>(p) << (q - anchor);  // < 2^108 per term, < 2^115 summed
      } else {  // far below this lane's largest product: straight into the bins
        const long long sg = p < 0 ? -1 : 1, mag = p < 0 ? -p : p;
        bin_add(bins, q, sg * (mag & 0xFFFFFF));
        if (mag >> 24) bin_add(bins, q + 24, sg * (mag >> 24));
      }
    }
    // acc = p0 + p1 2^42 + p2 2^84 with 0 <= p0, p1 < 2^42 (floor semantics)
    const long long mask42 = (1ll << 42) - 1;
    const long long p0 = static_cast<long long>(acc & mask42);
    const __int128 r1 = (acc - p0) >> 42;
    const long long p1 = static_cast<long long>(r1 & mask42);
    const long long p2 = static_cast<long long>((r1 - p1) >> 42);
    if (p0) bin_add(bins, anchor, p0);
    if (p1) bin_add(bins, anchor + 42, p1);
    if (p2) bin_add(bins, anchor + 84, p2);
  }
  __syncwarp();
  // limb j = sum of bins 32j .. 32j+31, each shifted into place (lane j computes limb j)
  __int128 L = 0;
  for (int j = lane; j < kNLimbs; j += 32) {
    L = 0;
    for (int i = 32 * j; i < 32 * j + 32 && i < kNBins; ++i)
      L += static_cast<__int128>(bins[i]) << (i & 31);
    // store as 4 x 32-bit two's-complement words next to each other (lane j: words 4j..4j+3)
    const unsigned __int128 u = static_cast<unsigned __int128>(L);
    limbs[4 * j + 0] = static_cast<uint32_t>(u);
    limbs[4 * j + 1] = static_cast<uint32_t>(u >> 32);
    limbs[4 * j + 2] = static_cast<uint32_t>(u >> 64);
    limbs[4 * j + 3] = static_cast<uint32_t>(u >> 96);
  }
  __syncwarp();
  float result = 0.0f;
  if (lane == 0) {
    uint32_t d[kNLimbs];
    __int128 carry = 0;
    for (int j = 0; j < kNLimbs; ++j) {
      const unsigned __int128 u = static_cast<unsigned __int128>(limbs[4 * j]) |
                                  (static_cast<unsigned __int128>(limbs[4 * j + 1]) << 32) |
                                  (static_cast<unsigned __int128>(limbs[4 * j + 2]) << 64) |
                                  (static_cast<unsigned __int128>(limbs[4 * j + 3]) << 96);
      const __int128 v = static_cast<__int128>(u) + carry;
      d[j] = static_cast<uint32_t>(static_cast<unsigned __int128>(v) & 0xFFFFFFFFu);
      carry = v >> 32;  // arithmetic shift: floor division
    }
    const bool negative = (carry < 0);  // carry is 0 or -1: the limbs hold the full value
    if (negative) {                     // two's complement of the limb string
      uint64_t c = 1;
      for (int j = 0; j < kNLimbs; ++j) {
        const uint64_t v = static_cast<uint64_t>(~d[j]) + c;
        d[j] = static_cast<uint32_t>(v);
        c = v >> 32;
      }
    }
    result = round_limbs_rn32(d, kNLimbs, negative);
  }
  __syncwarp();
  return __shfl_sync(0xffffffffu, result, 0);
}

// ---------------------------------------------------------------------------------------
// Certified selection of one token by one warp.  Lane l holds experts l, l+32, l+64, ...
// (EPL of them) in registers: the two ends of each key interval, the best-estimate key
// and a status.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ordered(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// e^z for the sigmoid router, z in [-41, 111]: the fixed sequence of IEEE fp64 steps that
// defines the router's sigmoid (Cody-Waite reduction z = n ln2 + r with ln 2 split into a
// 42-bit head, so that n * ln2_hi is exact, and a tail; the degree-13 Taylor polynomial of
// e^r by fused multiply-adds; an exact scaling by 2^n).  Every operation is an explicit
// round-to-nearest intrinsic, so nothing is contracted or approximated and the result is
// the same on any IEEE implementation of these steps.
__device__ __forceinline__ double exp_fixed(double z) {
  const double inv_ln2 = 0x1.71547652b82fep+0;  // RN(1 / ln 2)
  const double ln2_hi = 0x1.62e42fefa3800p-1;   // ln 2 = 0.693147180559945309417..., 42 bits
  const double ln2_lo = 0x1.ef35793c76730p-45;  // RN(ln 2 - ln2_hi)
  const double n = rint(__dmul_rn(z, inv_ln2));
  const double r = __dsub_rn(__dsub_rn(z, __dmul_rn(n, ln2_hi)), __dmul_rn(n, ln2_lo));
  double q = 1.0 / 6227020800.0;  // 1/13!
  q = __fma_rn(q, r, 1.0 / 479001600.0);
  q = __fma_rn(q, r, 1.0 / 39916800.0);
  q = __fma_rn(q, r, 1.0 / 3628800.0);
  q = __fma_rn(q, r, 1.0 / 362880.0);
  q = __fma_rn(q, r, 1.0 / 40320.0);
  q = __fma_rn(q, r, 1.0 / 5040.0);
  q = __fma_rn(q, r, 1.0 / 720.0);
  q = __fma_rn(q, r, 1.0 / 120.0);
  q = __fma_rn(q, r, 1.0 / 24.0);
  q = __fma_rn(q, r, 1.0 / 6.0);
  q = __fma_rn(q, r, 0.5);
  q = __fma_rn(q, r, 1.0);
  q = __fma_rn(q, r, 1.0);
  const double two_n = __longlong_as_double((static_cast<long long>(n) + 1023) << 52);
  return __dmul_rn(q, two_n);
}

// The router's fp32 sigmoid score of an fp32 logit: 0 below -110, 1 above 40, else
// fp32(1 / (1 + e^-s)), within a few fp64 ulps of the exact sigmoid before the rounding.
__device__ __forceinline__ float sigmoid32(float s32) {
  const double z = static_cast<double>(s32);
  if (z < -110.0) return 0.0f;
  if (z > 40.0) return 1.0f;
  return __double2float_rn(__ddiv_rn(1.0, __dadd_rn(1.0, exp_fixed(-z))));
}

// How router logits become selection keys and weights.
//   softmax (sigmoid = 0): key = fp32(s) (+ bias), weights = softmax of the chosen keys;
//   sigmoid (sigmoid = 1): p = sigmoid32(fp32(s)), key = fp32(p + bias) with the bias
//     steering the choice only, weights = scale * p / sum of the chosen p
//     (llm-atlas page "Step-3.5-Flash", table "Champs bruts du config.json":
//     moe_router_activation, use_moe_router_bias, moe_router_scaling_factor).
struct Keys {
  const float* bias;
  int sigmoid;
  float scale;
  __device__ __forceinline__ float score(double s) const {  // p, or the logit itself
    const float s32 = __double2float_rn(s);
    return sigmoid ? sigmoid32(s32) : s32;
  }
  // the bias of expert e (0 without one), for the *_b forms below that take it loaded
  __device__ __forceinline__ float bias_of(int e) const { return bias ? bias[e] : 0.0f; }
  // the key of a logit (exact when s is the exact logit rounded to fp32); b = bias_of(e)
  __device__ __forceinline__ float key_b(double s, float b) const {
    const float v = score(s);
    return bias ? __fadd_rn(v, b) : v;
  }
  __device__ __forceinline__ float key(double s, int e) const { return key_b(s, bias_of(e)); }
  // Lower / upper ends of the keys of all logits >= s_lo / <= s_hi.  For the sigmoid the
  // ends come from an fp32 evaluation, 1 / (1 + expf(-z)) (expf within 2 ulps over its whole
  // range, as CUDA documents it; one rounding each for the add and the IEEE division), widened
  // by a relative 2^-20: that covers its error against the exact sigmoid and the fp64
  // definition's rounding to fp32, at a tenth of the cost of the fp64 evaluation.  Below
  // z = -80 the ends are 0 and 2^-115 > sigma(-80).
  __device__ __forceinline__ float key_lo_b(double s_lo, float b) const {
    if (!sigmoid) return key_b(s_lo, b);
    const float z = __double2float_rd(s_lo);
    const float p = z < -80.0f ? 0.0f : __fmul_rd(__fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-z))), 1.0f - 0x1p-20f);
    return bias ? __fadd_rd(p, b) : p;
  }
  __device__ __forceinline__ float key_hi_b(double s_hi, float b) const {
    if (!sigmoid) return key_b(s_hi, b);
    const float z = __double2float_ru(s_hi);
    const float p = z < -80.0f ? 0x1p-115f : __fmul_ru(__fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-z))), 1.0f + 0x1p-20f);
    return bias ? __fadd_ru(p, b) : p;
  }
  __device__ __forceinline__ float key_lo(double s_lo, int e) const { return key_lo_b(s_lo, bias_of(e)); }
  __device__ __forceinline__ float key_hi(double s_hi, int e) const { return key_hi_b(s_hi, bias_of(e)); }
  // The same ends for a refined (fp64) score, tight: the fp64 definition itself, widened by
  // one ulp of p for its at most one-ulp departure from monotonicity.
  __device__ __forceinline__ float key_lo_ref(double s_lo, int e) const {
    if (!sigmoid) return key(s_lo, e);
    const float p = nextafterf(sigmoid32(__double2float_rd(s_lo)), -INFINITY);
    return bias ? __fadd_rd(p, bias[e]) : p;
  }
  __device__ __forceinline__ float key_hi_ref(double s_hi, int e) const {
    if (!sigmoid) return key(s_hi, e);
    const float p = nextafterf(sigmoid32(__double2float_ru(s_hi)), INFINITY);
    return bias ? __fadd_ru(p, bias[e]) : p;
  }
};

// a is ranked before b: larger key, then lower index
__device__ __forceinline__ bool better(float ka, int a, float kb, int b) {
  return (ka > kb) || (ka == kb && a < b);
}

enum : int { ST_OUT = 0, ST_CAND = 1, ST_IN = 2, ST_UNDECIDED = 3 };

// per-warp shared scratch of the exact dot product
constexpr size_t kExactScratch =
    ((sizeof(long long) * kNBins + sizeof(uint32_t) * 4 * kNLimbs + 15) / 16) * 16;

// experts per lane of the register-resident selection
inline int select_epl(int E) { return E <= 128 ? 4 : (E <= 384 ? 12 : 32); }

// register-array access with a run-time index, without spilling the array to memory
template <int EPL, typename V>
__device__ __forceinline__ V pick(const V (&a)[EPL], int i) {
  V r = a[0];
#pragma unroll
  for (int j = 1; j < EPL; ++j)
    if (j == i) r = a[j];
  return r;
}
template <int EPL, typename V>
__device__ __forceinline__ void put(V (&a)[EPL], int i, V v) {
#pragma unroll
  for (int j = 0; j < EPL; ++j)
    if (j == i) a[j] = v;
}

// fp64 dot with four 16-byte loads per operand in flight per lane
// eight consecutive elements as floats (one 16-byte load of bf16, two of fp32)
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&o)[8]) {
  const Vec16<__nv_bfloat16> v = ld16(p);
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j] = __bfloat162float(v.v[j]);
}
__device__ __forceinline__ void load8(const float* p, float (&o)[8]) {
  const Vec16<float> v0 = ld16(p), v1 = ld16(p + 4);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o[j] = v0.v[j];
    o[4 + j] = v1.v[j];
  }
}

// fp64 dot of two rows of different types (bf16 tokens, fp32 router weights): exact
// products, fp64 accumulation; H a multiple of 8
template <typename TA, typename TB>
__device__ double warp_dot_f64_prefetch(const TA* __restrict__ a, const TB* __restrict__ b, int H) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
  const int n8 = H / 8;
  for (int v = lane; v < n8; v += 64) {
    float av[2][8], bv[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (v + 32 * u < n8) {
        load8(a + (v + 32 * u) * 8, av[u]);
        load8(b + (v + 32 * u) * 8, bv[u]);
      }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (v + 32 * u >= n8) break;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc = fma(static_cast<double>(av[u][j]), static_cast<double>(bv[u][j]), acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

template <typename T>
__device__ double warp_dot_f64_prefetch(const T* __restrict__ a, const T* __restrict__ b, int H) {
  const int lane = threadIdx.x & 31;
  constexpr int V = Vec16<T>::N;
  const int nv = H / V;
  double acc = 0.0;
  int v = lane;
  for (; v + 96 < nv; v += 128) {
    Vec16<T> av[4], bv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      av[u] = ld16(a + (v + 32 * u) * V);
      bv[u] = ld16(b + (v + 32 * u) * V);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < V; ++j)
        acc = fma(static_cast<double>(to_f32(av[u].v[j])), static_cast<double>(to_f32(bv[u].v[j])), acc);
  }
  for (; v < nv; v += 32) {
    const Vec16<T> av = ld16(a + v * V), bv = ld16(b + v * V);
#pragma unroll
    for (int j = 0; j < V; ++j)
      acc = fma(static_cast<double>(to_f32(av.v[j])), static_cast<double>(to_f32(bv.v[j])), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// srow: score estimates of the token (fp64 values); |s^ - s| <= delta_coef ||x|| ||w_e||
// + delta_abs.  refine_f64: recompute undecided candidates in fp64 before the exact pass
// (the estimates are not fp64-accurate).  Norms ||w_e||: wnorm[e], or computed from the
// sums of squares wss[e] when wss is given.
// Fast path of the selection of one token by one warp.
// srow: score estimates of the token (fp64 values), |s^ - s| <= delta_coef ||x|| ||w_e||
// + delta_abs.  refine_f64: recompute undecided candidates in fp64 (the estimates are
// not fp64 sums).  Norms ||w_e||: wnorm[e], or from the sums of squares wss[e].
//   1. lower key bounds lo_e in registers (lane l holds experts l, l+32, ...);
//   2. Lk, the k-th largest lower bound, by k rounds of warp max-extraction;
//   3. candidates hi_e >= Lk compacted, in ascending expert order, into a 32-entry list
//      in shared memory (only they can be chosen, and a candidate can only be beaten for
//      certain by candidates);
//   4. lane j classifies candidate j: chosen for certain if fewer than k candidates can be
//      ranked before it, rejected for certain if k are ranked before it for certain;
//   5. undecided ones are recomputed in fp64 by the whole warp, then classified again;
//   6. open slots, renormalised softmax, outputs.
// Returns false, writing nothing, if more than 32 candidates remain or a key is still
// undecided; select_token_slow() then redoes the token.
struct CandList {
  int e[32];
  float lo[32], hi[32], mid[32];
  float p[32];  // sigmoid router: the score of the best estimate (weights)
};

// SIG: the router mode as a compile-time constant (the softmax path carries no sigmoid code)
template <typename T, typename TW, int EPL, bool SIG>
__device__ __forceinline__ bool select_token(const double* __restrict__ srow, double delta_coef,
                                             double delta_abs, bool refine_f64, double nx,
                                             const double* __restrict__ wnorm,
                                             const double* __restrict__ wss,
                                             const Keys kf_in, const T* __restrict__ xt,
                                             const TW* __restrict__ Wr, int H, int E, int k, int64_t t,
                                             int32_t* __restrict__ idx_ws, float* __restrict__ w_ws,
                                             int32_t* __restrict__ idx_user, float* __restrict__ w_user,
                                             CandList& C, Ctrl* ctrl) {
  Keys kf = kf_in;
  kf.sigmoid = SIG ? 1 : 0;
  const int lane = threadIdx.x & 31;
  auto nw = [&](int e) -> double { return wss ? norm_ub_from_sumsq(wss[e], H) : wnorm[e]; };
  const double cdx = __dmul_ru(delta_coef, nx);
  // 1. lower bounds (the estimates and their error bounds stay in registers for step 3)
  uint32_t u[EPL];
  double sh_r[EPL], d_r[EPL];
  float b_r[EPL];  // the experts' biases, loaded once
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    sh_r[i] = (e < E) ? srow[e] : 0.0;
    d_r[i] = (e < E) ? __dadd_ru(__dmul_ru(cdx, nw(e)), delta_abs) : 0.0;
    b_r[i] = (e < E) ? kf.bias_of(e) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    u[i] = (e < E) ? ordered(kf.key_lo_b(__dadd_rd(sh_r[i], -d_r[i]), b_r[i])) : 0u;
  }
  // 2. Lk: each lane sorts its lower bounds in descending order; each of k rounds takes the
  //    warp's largest head and shifts that lane's list by one (0 marks an empty slot)
  uint32_t lk = 0;
  {
#pragma unroll
    for (int i = 0; i < EPL; ++i)
#pragma unroll
      for (int j = i + 1; j < EPL; ++j) {
        const uint32_t a = u[i], b = u[j];
        u[i] = max(a, b);
        u[j] = min(a, b);
      }
    for (int r = 0; r < k; ++r) {
      const uint32_t gbest = __reduce_max_sync(0xffffffffu, u[0]);
      const unsigned holders = __ballot_sync(0xffffffffu, u[0] == gbest);
      if (lane == __ffs(holders) - 1) {
#pragma unroll
        for (int i = 0; i + 1 < EPL; ++i) u[i] = u[i + 1];
        u[EPL - 1] = 0;
      }
      lk = gbest;
    }
  }
  // 3. candidates, compacted in ascending expert order (their keys first, then the places)
  int cn = 0;
  bool cand_r[EPL];
  float hi_r[EPL];
  unsigned m_r[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    hi_r[i] = (e < E) ? kf.key_hi_b(__dadd_ru(sh_r[i], d_r[i]), b_r[i]) : 0.f;
    cand_r[i] = (e < E) && ordered(hi_r[i]) >= lk;
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) m_r[i] = __ballot_sync(0xffffffffu, cand_r[i]);  // independent ballots
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    const int pos = cn + __popc(m_r[i] & ((1u << lane) - 1u));
    if (cand_r[i] && pos < 32) {
      C.e[pos] = e;
      C.lo[pos] = kf.key_lo_b(__dadd_rd(sh_r[i], -d_r[i]), b_r[i]);
      C.hi[pos] = hi_r[i];
      C.mid[pos] = kf.key_b(sh_r[i], b_r[i]);
      if (SIG) C.p[pos] = kf.score(sh_r[i]);
    }
    cn += __popc(m_r[i]);
  }
  if (cn > 32) return false;
  __syncwarp();
  // 4. classification, lane j <-> candidate j
  const bool mine = lane < cn;
  const int my_e = mine ? C.e[lane] : 0;
  float my_lo = mine ? C.lo[lane] : 0.f, my_hi = mine ? C.hi[lane] : 0.f, my_mid = mine ? C.mid[lane] : 0.f;
  float my_p = (SIG && mine) ? C.p[lane] : 0.f;
  // (the whole warp runs it: lane j's candidate reaches the others by shuffles; cn <= 32)
  auto classify = [&]() -> int {
    int cp = 0, cc = 0;
#pragma unroll 4
    for (int j = 0; j < cn; ++j) {
      const int f = __shfl_sync(0xffffffffu, my_e, j);
      const float hf = __shfl_sync(0xffffffffu, my_hi, j), lf = __shfl_sync(0xffffffffu, my_lo, j);
      const bool other = j != lane;
      cp += other && ((hf > my_lo) || (hf == my_lo && f < my_e));
      cc += other && ((lf > my_hi) || (lf == my_hi && f < my_e));
    }
    return !mine ? ST_OUT : (cp < k) ? ST_IN : (cc >= k ? ST_OUT : ST_UNDECIDED);
  };
  int st = classify();
  // 5. fp64 recompute of the undecided candidates
  int n_ref = 0;
  if (refine_f64) {
    unsigned need = __ballot_sync(0xffffffffu, st == ST_UNDECIDED && my_lo != my_hi);
    if (need) {
      while (need) {
        const int src = __ffs(need) - 1;
        need &= need - 1;
        const int e = __shfl_sync(0xffffffffu, my_e, src);
        const double s64 = warp_dot_f64_prefetch(xt, Wr + static_cast<size_t>(e) * H, H);
        if (lane == src) {
          const double d = __dmul_ru(__dmul_ru(1.01 * H * kU53, nx), nw(e));
          my_lo = kf.key_lo_ref(__dadd_rd(s64, -d), e);
          my_hi = kf.key_hi_ref(__dadd_ru(s64, d), e);
          my_mid = kf.key(s64, e);
          if (SIG) my_p = kf.score(s64);
          C.lo[lane] = my_lo;
          C.hi[lane] = my_hi;
          C.mid[lane] = my_mid;
        }
        ++n_ref;
      }
      __syncwarp();
      st = classify();
    }
  }
  if (__any_sync(0xffffffffu, st == ST_UNDECIDED && my_lo != my_hi)) {
    if (lane == 0 && n_ref) atomicAdd(&ctrl->n_refined, static_cast<unsigned long long>(n_ref));
    return false;
  }
  // 6. open slots go to the best undecided candidates (their keys are exact)
  int n_in = __popc(__ballot_sync(0xffffffffu, st == ST_IN));
  for (int j = n_in; j < k; ++j) {
    float bk = my_mid;
    int be = (st == ST_UNDECIDED) ? my_e : -1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (oe >= 0 && (be < 0 || better(ok, oe, bk, be))) {
        bk = ok;
        be = oe;
      }
    }
    if (be < 0) {  // only with non-finite keys (outside the contract)
      if (lane == 0) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      break;
    }
    if (mine && my_e == be) st = ST_IN;
  }
  // 7. weights: renormalised softmax over the chosen keys, or (sigmoid router) the chosen
  //    scores renormalised and scaled; outputs in ascending expert order
  const bool in = st == ST_IN;
  float m = in ? my_mid : -FLT_MAX;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float ex = in ? (kf.sigmoid ? my_p : expf(my_mid - m)) : 0.0f;
  float z = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const unsigned in_mask = __ballot_sync(0xffffffffu, in);
  if (in) {
    const int pos = __popc(in_mask & ((1u << lane) - 1u));
    if (pos < k) {
      const float w = !kf.sigmoid ? ex / z : (z > 0.0f ? kf.scale * ex / z : kf.scale / k);
      idx_ws[t * k + pos] = my_e;
      w_ws[t * k + pos] = w;
      if (idx_user) idx_user[t * k + pos] = my_e;
      if (w_user) w_user[t * k + pos] = w;
    }
  }
  if (lane == 0) {
    if (__popc(in_mask) != k) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
    if (n_ref) {
      atomicAdd(&ctrl->n_refined, static_cast<unsigned long long>(n_ref));
      atomicAdd(&ctrl->n_tokens_refined, 1ull);
    }
  }
  return true;
}

// key state of one token in the workspace, for the rare path
struct KeySpill {
  float* lo;
  float* hi;
  float* mid;
  int* st;
  float* p;  // sigmoid router: scores of the best estimates
};

__device__ __forceinline__ KeySpill key_spill(float* base, int64_t T, int E, int64_t t) {
  const int64_t n = T * E;
  KeySpill s;
  s.lo = base + t * E;
  s.hi = base + n + t * E;
  s.mid = base + 2 * n + t * E;
  s.st = reinterpret_cast<int*>(base + 3 * n) + t * E;
  s.p = base + 4 * n + t * E;
  return s;
}

// Rare path: the whole selection of one token with its key state in global memory (one
// warp): intervals from the score estimates, fp64 recompute (when the estimates are not
// fp64 sums) and exact dots for what stays undecided, classification, open slots,
// weights and outputs.
template <typename T, typename TW, bool SIG>
__device__ __noinline__ void select_token_slow(const double* __restrict__ srow, int64_t sstride,
                                               double delta_coef,
                                               double delta_abs, bool refine_f64, double nx,
                                               const double* __restrict__ wnorm,
                                               const double* __restrict__ wss, KeySpill sp,
                                               const Keys kf_in,
                                               const T* __restrict__ xt, const TW* __restrict__ Wr,
                                               int H, int E, int k, int64_t t,
                                               int32_t* __restrict__ idx_ws, float* __restrict__ w_ws,
                                               int32_t* __restrict__ idx_user, float* __restrict__ w_user,
                                               unsigned char* exact_scratch, Ctrl* ctrl) {
  Keys kf = kf_in;
  kf.sigmoid = SIG ? 1 : 0;
  const int lane = threadIdx.x & 31;
  auto nw = [&](int e) -> double { return wss ? norm_ub_from_sumsq(wss[e], H) : wnorm[e]; };
  long long* bins = reinterpret_cast<long long*>(exact_scratch);
  uint32_t* limbs = reinterpret_cast<uint32_t*>(exact_scratch + sizeof(long long) * kNBins);
  for (int e = lane; e < E; e += 32) {
    const double sh = srow[e * sstride];
    const double d = __dadd_ru(__dmul_ru(__dmul_ru(delta_coef, nx), nw(e)), delta_abs);
    sp.lo[e] = kf.key_lo(__dadd_rd(sh, -d), e);
    sp.hi[e] = kf.key_hi(__dadd_ru(sh, d), e);
    sp.mid[e] = kf.key(sh, e);
    sp.p[e] = kf.score(sh);
    sp.st[e] = ST_CAND;
  }
  __syncwarp();
  int n_ref = 0, n_exact = 0, n_in = 0;
  for (int pass = refine_f64 ? 0 : 1; pass < 3; ++pass) {
    // classify every remaining candidate
    n_in = 0;
    for (int base = 0; base < E; base += 32) {
      const int e0 = base + lane;
      unsigned mask = __ballot_sync(0xffffffffu, e0 < E && sp.st[e0] != ST_OUT);
      while (mask) {
        const int e = base + __ffs(mask) - 1;
        mask &= mask - 1;
        const float le = sp.lo[e], he = sp.hi[e];
        int cp = 0, cc = 0;
        for (int f = lane; f < E; f += 32) {
          if (f == e) continue;
          const float hf = sp.hi[f], lf = sp.lo[f];
          cp += (hf > le) || (hf == le && f < e);
          cc += (lf > he) || (lf == he && f < e);
        }
        cp = __reduce_add_sync(0xffffffffu, cp);
        cc = __reduce_add_sync(0xffffffffu, cc);
        const int st = (cp < k) ? ST_IN : (cc >= k ? ST_OUT : ST_UNDECIDED);
        n_in += (st == ST_IN);
        __syncwarp();
        if (lane == 0) sp.st[e] = st;
        __syncwarp();
      }
    }
    if (pass == 2) break;  // keys of the undecided ones are exact now
    // recompute the undecided ones whose key is not yet exact: fp64, then exactly
    for (int base = 0; base < E; base += 32) {
      const int e0 = base + lane;
      unsigned mask = __ballot_sync(0xffffffffu, e0 < E && sp.st[e0] == ST_UNDECIDED && sp.lo[e0] != sp.hi[e0]);
      while (mask) {
        const int e = base + __ffs(mask) - 1;
        mask &= mask - 1;
        const TW* we = Wr + static_cast<size_t>(e) * H;
        float klo, khi, kmid, kp;
        if (pass == 0) {
          const double s64 = warp_dot_f64_prefetch(xt, we, H);
          const double d = __dmul_ru(__dmul_ru(1.01 * H * kU53, nx), nw(e));
          klo = kf.key_lo_ref(__dadd_rd(s64, -d), e);
          khi = kf.key_hi_ref(__dadd_ru(s64, d), e);
          kmid = kf.key(s64, e);
          kp = kf.score(s64);
          ++n_ref;
        } else {
          const float s32 = warp_exact_dot_rn32(xt, we, H, bins, limbs);
          klo = khi = kmid = kf.key(s32, e);
          kp = kf.score(s32);
          ++n_exact;
        }
        __syncwarp();
        if (lane == 0) {
          sp.lo[e] = klo;
          sp.hi[e] = khi;
          sp.mid[e] = kmid;
          sp.p[e] = kp;
        }
        __syncwarp();
      }
    }
    for (int e = lane; e < E; e += 32)
      if (sp.st[e] == ST_UNDECIDED) sp.st[e] = ST_CAND;
    __syncwarp();
  }
  // open slots: best undecided by (exact key desc, index asc)
  for (int j = n_in; j < k; ++j) {
    float bk = 0.0f;
    int be = -1;
    for (int e = lane; e < E; e += 32)
      if (sp.st[e] == ST_UNDECIDED && (be < 0 || better(sp.mid[e], e, bk, be))) {
        bk = sp.mid[e];
        be = e;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (oe >= 0 && (be < 0 || better(ok, oe, bk, be))) {
        bk = ok;
        be = oe;
      }
    }
    if (be < 0) {
      if (lane == 0) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      break;
    }
    __syncwarp();
    if (lane == 0) sp.st[be] = ST_IN;
    __syncwarp();
  }
  float m = -FLT_MAX;
  for (int e = lane; e < E; e += 32)
    if (sp.st[e] == ST_IN) m = fmaxf(m, sp.mid[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.0f;
  for (int e = lane; e < E; e += 32)
    if (sp.st[e] == ST_IN) z += kf.sigmoid ? sp.p[e] : expf(sp.mid[e] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  int written = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const bool ch = (e < E) && sp.st[e] == ST_IN;
    const unsigned mask = __ballot_sync(0xffffffffu, ch);
    if (ch) {
      const int pos = written + __popc(mask & ((1u << lane) - 1u));
      if (pos < k) {
        const float w = !kf.sigmoid ? expf(sp.mid[e] - m) / z
                                    : (z > 0.0f ? kf.scale * sp.p[e] / z : kf.scale / k);
        idx_ws[t * k + pos] = e;
        w_ws[t * k + pos] = w;
        if (idx_user) idx_user[t * k + pos] = e;
        if (w_user) w_user[t * k + pos] = w;
      }
    }
    written += __popc(mask);
  }
  if (lane == 0) {
    if (written != k) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
    if (n_ref) atomicAdd(&ctrl->n_refined, static_cast<unsigned long long>(n_ref));
    if (n_exact) atomicAdd(&ctrl->n_exact, static_cast<unsigned long long>(n_exact));
    atomicAdd(&ctrl->n_tokens_refined, 1ull);
  }
}

// ---------------------------------------------------------------------------------------
// Selection kernel for the tensor-core scores: one warp per token.
// ---------------------------------------------------------------------------------------
constexpr int kSelectWarps = 4;

template <typename T, typename TW, int EPL, bool SIG>
__global__ void __launch_bounds__(32 * kSelectWarps) route_select_kernel(
    const double* __restrict__ scores, double delta_coef, double delta_abs,
    const double* __restrict__ xnorm, const double* __restrict__ wnorm,
    const Keys kf, const T* __restrict__ x, const TW* __restrict__ Wr,
    int64_t T_, int H, int E, int k, int32_t* __restrict__ idx_ws, float* __restrict__ w_ws,
    int32_t* __restrict__ idx_user, float* __restrict__ w_user, float* __restrict__ spill,
    Ctrl* ctrl) {
  __shared__ __align__(16) unsigned char exact_scratch[kSelectWarps][kExactScratch];
  __shared__ CandList cands[kSelectWarps];
  pdl_wait();
  const int warp = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kSelectWarps + warp;
  if (t < T_) {
    if (!select_token<T, TW, EPL, SIG>(scores + t * E, delta_coef, delta_abs, true, xnorm[t], wnorm, nullptr,
                              kf, x + t * H, Wr, H, E, k, t, idx_ws, w_ws, idx_user, w_user,
                              cands[warp], ctrl))
      select_token_slow<T, TW, SIG>(scores + t * E, 1, delta_coef, delta_abs, true, xnorm[t], wnorm, nullptr,
                           key_spill(spill, T_, E, t), kf, x + t * H, Wr, H, E, k, t, idx_ws, w_ws,
                           idx_user, w_user, exact_scratch[warp], ctrl);
  }
}

// ---------------------------------------------------------------------------------------
// Small batches: fused fp64 scores, norms and selection.  Block (b, g, z) adds, for the
// experts [16b, 16b+16), the tokens [16g, 16g+16) and the z-th quarter of the hidden
// dimension, the fp64 partial scores into scores[t, e] and the partial sums of squares
// of W_r rows into wss[g, e] (both zeroed before the launch; products exact in fp64, any
// summation order).  Warp w owns experts 16b+2w and 16b+2w+1.  The last block of token
// group g to finish (a counter in the workspace) then selects for the group's tokens, one
// warp per token.
// ---------------------------------------------------------------------------------------
constexpr int kDecodeTok = 16;
constexpr int kDecodeExp = 16;
constexpr int kDecodeSplit = 4;
constexpr int kDecodeThreads = 256;

template <typename T, int EPL, bool SIG>
__global__ void __launch_bounds__(kDecodeThreads, 1) router_decode_kernel(
    const T* __restrict__ x, const T* __restrict__ Wr, const Keys kf, int64_t T_,
    int H, int E, int k, double* __restrict__ scores, double* __restrict__ wss,
    unsigned int* __restrict__ group_done, int32_t* __restrict__ idx_ws, float* __restrict__ w_ws,
    int32_t* __restrict__ idx_user, float* __restrict__ w_user, float* __restrict__ spill, Ctrl* ctrl) {
  __shared__ __align__(16) unsigned char exact_scratch[kDecodeThreads / 32][kExactScratch];
  __shared__ CandList cands[kDecodeThreads / 32];
  __shared__ int is_last;
  pdl_wait();
  const int g = blockIdx.y;
  const int64_t t0 = static_cast<int64_t>(g) * kDecodeTok;
  const int nt = static_cast<int>(min64(kDecodeTok, T_ - t0));
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = blockIdx.x * kDecodeExp + 2 * warp;
  const bool has0 = e0 < E, has1 = e0 + 1 < E;
  const int nv = H / V;
  const int per = (nv + kDecodeSplit - 1) / kDecodeSplit;
  const int v_begin = blockIdx.z * per, v_end = min(nv, v_begin + per);
  double* wss_g = wss + static_cast<int64_t>(g) * E;
  if (has0) {
    double acc0[kDecodeTok], acc1[kDecodeTok];
    double ss0 = 0.0, ss1 = 0.0;
#pragma unroll
    for (int j = 0; j < kDecodeTok; ++j) acc0[j] = acc1[j] = 0.0;
    const T* w0 = Wr + static_cast<size_t>(e0) * H;
    const T* w1 = Wr + static_cast<size_t>(has1 ? e0 + 1 : e0) * H;
    for (int vb = v_begin + lane; vb < v_end; vb += 2 * 32) {
      Vec16<T> a0[2], a1[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int v = vb + 32 * u;
        if (v < v_end) {
          a0[u] = ld16(w0 + v * V);
          a1[u] = ld16(w1 + v * V);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int v = vb + 32 * u;
        if (v >= v_end) break;
        double d0[V], d1[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
          d0[j] = static_cast<double>(to_f32(a0[u].v[j]));
          d1[j] = static_cast<double>(to_f32(a1[u].v[j]));
          ss0 = fma(d0[j], d0[j], ss0);
          ss1 = fma(d1[j], d1[j], ss1);
        }
#pragma unroll
        for (int tt = 0; tt < kDecodeTok; ++tt) {
          if (tt < nt) {
            const Vec16<T> xv = ld16(x + (t0 + tt) * H + v * V);
#pragma unroll
            for (int j = 0; j < V; ++j) {
              const double xd = static_cast<double>(to_f32(xv.v[j]));
              acc0[tt] = fma(xd, d0[j], acc0[tt]);
              acc1[tt] = fma(xd, d1[j], acc1[tt]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss0 += __shfl_xor_sync(0xffffffffu, ss0, o);
      ss1 += __shfl_xor_sync(0xffffffffu, ss1, o);
#pragma unroll
      for (int tt = 0; tt < kDecodeTok; ++tt) {
        acc0[tt] += __shfl_xor_sync(0xffffffffu, acc0[tt], o);
        acc1[tt] += __shfl_xor_sync(0xffffffffu, acc1[tt], o);
      }
    }
    if (lane == 0) {
      atomicAdd(&wss_g[e0], ss0);
      if (has1) atomicAdd(&wss_g[e0 + 1], ss1);
#pragma unroll
      for (int tt = 0; tt < kDecodeTok; ++tt) {
        if (tt < nt) {
          atomicAdd(&scores[(t0 + tt) * E + e0], acc0[tt]);
          if (has1) atomicAdd(&scores[(t0 + tt) * E + e0 + 1], acc1[tt]);
        }
      }
    }
  }
  // last block of the token group?
  fence_acq_rel_gpu();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&group_done[g], 1u);
    is_last = (prev == gridDim.x * gridDim.z - 1);
  }
  __syncthreads();
  if (is_last) {
    fence_acq_rel_gpu();
    for (int tt = warp; tt < nt; tt += kDecodeThreads / 32) {
      const int64_t t = t0 + tt;
      const T* xt = x + t * H;
      const double nx = norm_ub_from_sumsq(warp_sumsq(xt, H), H);
      // fp64 scores: |s^ - s| <= 1.01 * H * 2^-53 * ||x|| ||w|| (any summation order)
      if (!select_token<T, T, EPL, SIG>(scores + t * E, 1.01 * H * kU53, 0.0, false, nx, nullptr, wss_g, kf,
                                xt, Wr, H, E, k, t, idx_ws, w_ws, idx_user, w_user, cands[warp], ctrl))
        select_token_slow<T, T, SIG>(scores + t * E, 1, 1.01 * H * kU53, 0.0, false, nx, nullptr, wss_g,
                             key_spill(spill, T_, E, t), kf, xt, Wr, H, E, k, t, idx_ws, w_ws,
                             idx_user, w_user, exact_scratch[warp], ctrl);
    }
  }
}

// ---------------------------------------------------------------------------------------
// tcgen05 router GEMM.  Block (m, n, z) scores the tokens [128m, 128m+128) against the
// experts [64n, 64n+64) over chunk z of the reduction.  Every slice of kRtSliceSteps
// 64-product steps is accumulated in fp32 in one of two tensor-memory buffers and then
// drained by the epilogue warps, so the fp32 accumulation error of each partial is
// bounded by the slice; the partials add up in fp64, in slice order.  Only the token
// rows that exist are loaded (16-row boxes); rows of the A tile beyond them are never
// read back.  Warp 0 issues TMA copies, warp 1 the MMAs, warps 2-5 (one thread per
// token) drain.
//
// Unsplit (one chunk): the epilogue adds the slices in fp64 registers and writes the
// scores.  Split (a batch whose tiles do not fill the GPU): each block writes its slices'
// fp32 partials and the sums of squares of its x / W_router columns (for the norm bounds
// of the selection); the last block of each (m, n) tile, found by a counter, adds the
// partials in the same slice order -- the scores are bit-identical to the unsplit ones --
// and finishes the norms of its rows.
// ---------------------------------------------------------------------------------------
constexpr int kRtExperts = 64;
constexpr int kRtStages = 8;
constexpr int kRtSliceSteps = 4;                     // slice = 256 products
constexpr int kRtABytes = kTileM * kTileK * 2;       // 16 KB of x (at most)
constexpr int kRtBBytes = kRtExperts * kTileK * 2;   // 8 KB of W_router
constexpr int kRtStageBytes = kRtABytes + kRtBBytes;
constexpr int kRtSmem = kRtStages * kRtStageBytes + 1024 + 256;
constexpr int kRtRowBox = 16;                        // token rows per TMA box
constexpr int kRtMaxChunks = 16;                      // a tile's last block adds them in one pass
constexpr int kRtSmTarget = 148;                     // blocks that fill the GPU

struct RouterTcParams {
  CUtensorMap tmX;   // x [T, Hx], box {64, 16}
  CUtensorMap tmX128;  // x [T, Hx], box {64, 128}: one copy per k-step for a full token tile
  CUtensorMap tmW;   // W_router [E, H] (fp32 weights: their bf16 split [E, 3 Hx]), box {64, 64}
  int64_t T;
  int H, E;          // H: length of the reduction (Hx, or 3 Hx for split fp32 weights)
  int Hx;            // tokens' hidden size; reduction step kb reads x columns (kb mod Hx/64)
  int w_given;       // W_router norms precomputed (split fp32 weights): no W sums of squares
  double* scores;    // [T, E]
  // split only
  int chunks, chunk_slices;
  int last_block_reduces;  // 1: the last block of each tile adds the partials (T <= 32); 0:
                           // router_reduce_kernel does, after this launch
  const __nv_bfloat16* x;
  const __nv_bfloat16* Wr;
  float* part;       // [slices, T, E] fp32 slice partials
  double* xss;       // [chunks, T] partial sums of squares
  double* wss;       // [chunks, E]
  unsigned int* tile_done;   // [tiles m x n], zero before the launch
  double* xnorm;     // [T]
  double* wnorm;     // [E]
  Ctrl* ctrl;
};

// Sum of squares of rows [0, nrows) of a bf16 matrix over columns [c0, c1) (multiples of
// 8), by the four epilogue warps (w = 0..3), eight rows per warp at a time; out[r].
__device__ void sumsq_rows_bf16(const __nv_bfloat16* __restrict__ base, int64_t ld, int nrows, int c0,
                                int c1, double* __restrict__ out, int w, int lane) {
  const int nv = (c1 - c0) / 8;
  for (int r0 = w; r0 < nrows; r0 += 4 * 8) {
    double ss[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) ss[u] = 0.0;
#pragma unroll 2
    for (int v = lane; v < nv; v += 32) {
      Vec16<__nv_bfloat16> a[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (r0 + 4 * u < nrows) a[u] = ld16(base + (r0 + 4 * u) * ld + c0 + v * 8);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (r0 + 4 * u >= nrows) break;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const double d = static_cast<double>(__bfloat162float(a[u].v[j]));
          ss[u] = fma(d, d, ss[u]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
      if (lane == 0 && r0 + 4 * u < nrows) out[r0 + 4 * u] = ss[u];
    }
  }
}

__global__ void __launch_bounds__(192, 1) router_gemm_tc_kernel(const __grid_constant__ RouterTcParams p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRtStages * kRtStageBytes);
  uint64_t* empty = full + kRtStages;
  uint64_t* tfull = empty + kRtStages;   // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;
  constexpr uint32_t kCols = 128;  // two 64-column accumulators

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // blocks are numbered expert tile fastest: the blocks that share a token tile run side by
  // side, so its rows of x are read from HBM once and then from L2
  const int n_tiles = (p.E + kRtExperts - 1) / kRtExperts;
  const int mi = static_cast<int>(blockIdx.x / n_tiles), ni = static_cast<int>(blockIdx.x % n_tiles);
  const int64_t t0 = static_cast<int64_t>(mi) * kTileM;
  const int e0 = ni * kRtExperts;
  const int ne = min(kRtExperts, p.E - e0);
  const int kb_all = p.H / kTileK;
  const int n_sl_all = (kb_all + kRtSliceSteps - 1) / kRtSliceSteps;
  const bool split = p.chunks > 1;
  const int sl_begin = blockIdx.z * p.chunk_slices;
  const int sl_end = min(n_sl_all, sl_begin + p.chunk_slices);
  const int kb_begin = sl_begin * kRtSliceSteps;
  const int kb_end = min(kb_all, sl_end * kRtSliceSteps);
  const int n_sl = sl_end - sl_begin;
  const int rows = static_cast<int>(min64(kTileM, p.T - t0));
  const int nbox = (rows + kRtRowBox - 1) / kRtRowBox;
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(rows == kTileM ? &p.tmX128 : &p.tmX);
      tma_prefetch_desc(&p.tmW);
      const uint32_t bytes = nbox * kRtRowBox * kTileK * 2 + kRtBBytes;
      int stage = 0;
      uint32_t phase = 0, used = 0;
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.ctrl, abort_flag)) break;
        unsigned char* st = smem + stage * kRtStageBytes;
        mbar_arrive_expect_tx(&full[stage], bytes);
        const int xcol = (kb % (p.Hx / kTileK)) * kTileK;
        if (rows == kTileM) {
          tma_load_2d(st, &p.tmX128, xcol, static_cast<int32_t>(t0), &full[stage]);
        } else {
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(st + b * kRtRowBox * kTileK * 2, &p.tmX, xcol,
                        static_cast<int32_t>(t0 + b * kRtRowBox), &full[stage]);
        }
        tma_load_2d(st + kRtABytes, &p.tmW, kb * kTileK, e0, &full[stage]);
        used |= 1u << stage;
        if (++stage == kRtStages) { stage = 0; phase ^= 1u; }
      }
      for (int s = 0; s < kRtStages; ++s)
        if (used & (1u << s)) {
          const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
          const uint64_t tw = globaltimer_ns();
          while (!mbar_try_wait(&full[s], par))
            if (globaltimer_ns() - tw > kWaitLimitNs) { set_status(p.ctrl, MOE_ERR_DEVICE_TIMEOUT); break; }
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileM, (ne + 15) & ~15);
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        const int sl = (kb - kb_begin) / kRtSliceSteps;   // slice within the chunk
        const bool first = (kb % kRtSliceSteps) == 0;
        const bool last = (kb % kRtSliceSteps) == kRtSliceSteps - 1 || kb == kb_end - 1;
        const int b = sl & 1;
        if (first && !mbar_wait(&tempty[b], ((sl >> 1) & 1) ^ 1u, p.ctrl, abort_flag)) break;
        if (!mbar_wait(&full[stage], phase, p.ctrl, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + stage * kRtStageBytes);
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk)
          mma_bf16(tmem_base + b * kRtExperts, sw128_kmajor_desc(a0 + kk * 32),
                   sw128_kmajor_desc(a0 + kRtABytes + kk * 32), idesc, (first && kk == 0) ? 0u : 1u);
        mma_commit(&empty[stage]);
        if (last) mma_commit(&tfull[b]);
        if (++stage == kRtStages) { stage = 0; phase ^= 1u; }
      }
      mma_commit(drain);
      const uint64_t tw = globaltimer_ns();
      while (!mbar_try_wait(drain, 0))
        if (globaltimer_ns() - tw > kWaitLimitNs) { set_status(p.ctrl, MOE_ERR_DEVICE_TIMEOUT); break; }
    }
  } else {
    const int quarter = warp & 3;
    const int64_t t = t0 + quarter * 32 + lane;
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    bool ok = true;
    if (!split) {
      double acc[kRtExperts];
#pragma unroll
      for (int j = 0; j < kRtExperts; ++j) acc[j] = 0.0;
      for (int sl = 0; sl < n_sl && ok; ++sl) {
        const int b = sl & 1;
        if (!mbar_wait(&tfull[b], (sl >> 1) & 1, p.ctrl, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[kRtExperts];
#pragma unroll
        for (int j0 = 0; j0 < kRtExperts; j0 += 16) tmem_ld16_nowait(trow + b * kRtExperts + j0, r + j0);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kRtExperts; ++j) acc[j] += static_cast<double>(__uint_as_float(r[j]));
        tc_fence_before();
        mbar_arrive(&tempty[b]);
      }
      if (ok && t < p.T) {
        double* dst = p.scores + t * p.E + e0;
#pragma unroll
        for (int j = 0; j < kRtExperts; ++j)
          if (j < ne) dst[j] = acc[j];
      }
    } else {
      // sums of squares of this chunk's columns while the MMAs run: the x rows once per
      // m tile (n == 0), the W_router rows once per n tile (m == 0)
      const int c0 = kb_begin * kTileK, c1 = kb_end * kTileK;
      if (ni == 0)  // x columns once (the split fp32 weights repeat them)
        sumsq_rows_bf16(p.x + t0 * p.Hx, p.Hx, rows, min(c0, p.Hx), min(c1, p.Hx),
                        p.xss + blockIdx.z * p.T + t0, quarter, lane);
      if (mi == 0 && !p.w_given)
        sumsq_rows_bf16(p.Wr + static_cast<int64_t>(e0) * p.H, p.H, ne, c0, c1,
                        p.wss + static_cast<int64_t>(blockIdx.z) * p.E + e0, quarter, lane);
      for (int sl = 0; sl < n_sl && ok; ++sl) {
        const int b = sl & 1;
        if (!mbar_wait(&tfull[b], (sl >> 1) & 1, p.ctrl, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[kRtExperts];
#pragma unroll
        for (int j0 = 0; j0 < kRtExperts; j0 += 16) tmem_ld16_nowait(trow + b * kRtExperts + j0, r + j0);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[b]);
        if (t < p.T) {
          float* dst = p.part + (static_cast<int64_t>(sl_begin + sl) * p.T + t) * p.E + e0;
#pragma unroll
          for (int j = 0; j < kRtExperts; ++j)
            if (j < ne) dst[j] = __uint_as_float(r[j]);
        }
      }
      // the last block of this (m, n) tile adds the partials of every chunk (below)
      if (p.last_block_reduces) {
        fence_acq_rel_gpu();
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) {
          const unsigned int done = atomicAdd(p.tile_done + blockIdx.x, 1u);
          *last_flag = (done == static_cast<unsigned int>(p.chunks - 1)) ? 1 : 0;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kCols);
  if (!split || !*last_flag) return;
  // Last block of the tile: the scores (each the fp64 sum of its slices' fp32 partials, in
  // slice order: the unsplit kernel's result bit for bit) and the norm bounds (fp64 sums of
  // the chunks' sums of squares, in chunk order), by all six warps.  Every load of a thread
  // is issued before the first of its values is used: first the sums of squares of the norm
  // bound it owns (threads from the last one down), then two scores at a time.
  fence_acq_rel_gpu();
  const int np = rows * ne, nxj = (ni == 0) ? rows : 0, nwj = (mi == 0 && !p.w_given) ? ne : 0;
  const int nthr = static_cast<int>(blockDim.x);
  const int jn = nthr - 1 - static_cast<int>(threadIdx.x);  // this thread's norm bound, if < nxj + nwj
  const bool has_norm = jn < nxj + nwj;  // every bound has its thread: rows + ne <= 32 + 64 < 192
  const bool norm_x = jn < nxj;
  double nv[16];
  if (has_norm) {  // 16 loads, none of them conditional (chunks past the last repeat it, unused)
    const double* src = norm_x ? p.xss + t0 + jn : p.wss + e0 + (jn - nxj);
    const int64_t nst = norm_x ? p.T : static_cast<int64_t>(p.E);
#pragma unroll
    for (int z = 0; z < 16; ++z) nv[z] = __ldcg(src + min(z, p.chunks - 1) * nst);
  }
  const int64_t sstride = p.T * p.E;
  for (int j0 = threadIdx.x; j0 < np; j0 += 2 * nthr) {
    const int j1 = j0 + nthr;
    const bool h1 = j1 < np;
    const int ta = j0 / ne, ea = j0 - ta * ne;
    const int tb = h1 ? j1 / ne : ta, eb = h1 ? j1 - tb * ne : ea;
    const float* pa = p.part + (t0 + ta) * p.E + e0 + ea;
    const float* pb = p.part + (t0 + tb) * p.E + e0 + eb;
    double acc_a = 0.0, acc_b = 0.0;
    int b = 0;
    for (; b + 16 <= n_sl_all; b += 16) {  // 32 unconditional loads, then the sums in slice order
      float va[16], vb[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        va[q] = __ldcg(pa + (b + q) * sstride);
        vb[q] = __ldcg(pb + (b + q) * sstride);
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        acc_a += static_cast<double>(va[q]);
        acc_b += static_cast<double>(vb[q]);
      }
    }
    for (; b < n_sl_all; ++b) {
      acc_a += static_cast<double>(__ldcg(pa + b * sstride));
      acc_b += static_cast<double>(__ldcg(pb + b * sstride));
    }
    p.scores[(t0 + ta) * p.E + e0 + ea] = acc_a;
    if (h1) p.scores[(t0 + tb) * p.E + e0 + eb] = acc_b;
  }
  if (has_norm) {
    double ss = 0.0;
#pragma unroll
    for (int z = 0; z < 16; ++z)
      if (z < p.chunks) ss += nv[z];
    if (norm_x)
      p.xnorm[t0 + jn] = norm_ub_from_sumsq(ss, p.Hx);
    else
      p.wnorm[e0 + jn - nxj] = norm_ub_from_sumsq(ss, p.H);
  }
}

// The reduction-split router's sums for batches of 33..128 tokens, whose tiles' last blocks
// would each have thousands of scores to add: one thread per score (the fp64 sum of its
// slices' fp32 partials in slice order, as the last block forms it: the unsplit kernel's
// result bit for bit) or norm bound (the fp64 sum of the chunks' sums of squares in chunk
// order), over the whole grid.
__global__ void __launch_bounds__(256) router_reduce_kernel(const __grid_constant__ RouterTcParams p) {
  pdl_wait();
  const int64_t ns = p.T * p.E, nx = p.T, nw = p.w_given ? 0 : p.E;
  const int n_sl_all = (p.H / kTileK + kRtSliceSteps - 1) / kRtSliceSteps;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < ns + nx + nw;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (j < ns) {
      const float* src = p.part + j;  // part[sl][t][e], j = t E + e
      double acc = 0.0;
      int b = 0;
      for (; b + 16 <= n_sl_all; b += 16) {
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = __ldcg(src + (b + q) * ns);
#pragma unroll
        for (int q = 0; q < 16; ++q) acc += static_cast<double>(v[q]);
      }
      for (; b < n_sl_all; ++b) acc += static_cast<double>(__ldcg(src + b * ns));
      p.scores[j] = acc;
    } else {
      const bool is_x = j < ns + nx;
      const int64_t i = is_x ? j - ns : j - ns - nx;
      const double* src = is_x ? p.xss + i : p.wss + i;
      const int64_t st = is_x ? p.T : static_cast<int64_t>(p.E);
      double ss = 0.0;
      for (int z = 0; z < p.chunks; ++z) ss += __ldcg(src + z * st);
      if (is_x)
        p.xnorm[i] = norm_ub_from_sumsq(ss, p.Hx);
      else
        p.wnorm[i] = norm_ub_from_sumsq(ss, p.H);
    }
  }
}

// ---------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------
static bool encode_bf16_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                             uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 batches score on the tensor cores (fp32 accumulation over slices, certified band,
// fp64 / exact recompute near the top-k boundary); fp32 inputs, or more experts than one
// tensor-memory row of accumulators allows, score in fp64 on the CUDA cores.
constexpr int64_t kTcRouterMinTokens = 1;

static bool router_tc_supported(bool bf16, int64_t T, int E, int H) {
  return bf16 && T >= kTcRouterMinTokens && E <= 512 && H % kTileK == 0;
}

bool router_scores_f32(const moe_layer_shape& s) {
  return router_tc_supported(s.dtype == MOE_BF16, s.T, s.E, s.H);
}

template <typename K>
static cudaError_t allow_smem(K kern, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
}

int router_slice_len(int /*H*/) { return kRtSliceSteps * kTileK; }

// Reduction chunks of the tensor-core router: 1 when the (m, n) tiles fill the GPU or the
// batch is too large for one block per tile to add the partials quickly, else the fewest
// (at most 16, at least one slice each) that bring the blocks to one per SM.
constexpr int64_t kRtSplitMaxTokens = 32;        // the tiles' last blocks add the partials
constexpr int64_t kRtSplitReduceMaxTokens = 128; // router_reduce_kernel adds them
static_assert(kRtSplitMaxTokens + kRtExperts <= 192, "one thread per norm bound in a tile's last block");
static int router_chunks(int64_t T, int E, int H) {
  if (T > kRtSplitReduceMaxTokens) return 1;
  const int64_t tiles = ((T + kTileM - 1) / kTileM) * ((E + kRtExperts - 1) / kRtExperts);
  const int n_sl = (H / kTileK + kRtSliceSteps - 1) / kRtSliceSteps;
  int c = 1;
  while (c < kRtMaxChunks && tiles * c < kRtSmTarget && 2 * c <= n_sl) c *= 2;
  if (c == 1) return 1;
  const int per = (n_sl + c - 1) / c;
  return (n_sl + per - 1) / per;
}

static size_t split_bytes_for(int64_t T, int E, int K) {
  const int c = router_chunks(T, E, K);
  if (c == 1) return 0;
  const size_t n_sl = static_cast<size_t>((K / kTileK + kRtSliceSteps - 1) / kRtSliceSteps);
  return static_cast<size_t>(c) * (static_cast<size_t>(T) + E) * 8 + n_sl * static_cast<size_t>(T) * E * 4;
}

// room for both reduction lengths: H, and 3H for split fp32 router weights
size_t router_split_bytes(const moe_layer_shape& s) {
  if (!router_tc_supported(s.dtype == MOE_BF16, s.T, s.E, s.H)) return 0;
  return std::max(split_bytes_for(s.T, s.E, s.H), split_bytes_for(s.T, s.E, 3 * s.H));
}

bool router_w32_supported(const moe_layer_shape& s) {
  return router_tc_supported(s.dtype == MOE_BF16, s.T > 0 ? s.T : 1, s.E, s.H);
}

size_t router_w3_bytes(const moe_layer_shape& s) {
  if (!router_tc_supported(s.dtype == MOE_BF16, s.T, s.E, s.H)) return 0;
  return static_cast<size_t>(s.E) * 3 * s.H * 2;
}

// fp32 router weights on the bf16 tensor cores: W = hi + mid + lo, each part bf16, so that
// x . W is the bf16 GEMM of x against [hi | mid | lo] over 3H (every part is an exact fp32
// difference; lo is exact unless W falls below the bf16 normal range, and whatever it misses
// goes into the norm bound).  One warp per expert row also bounds the row's norm for the
// selection: ||hi|| + ||mid|| + ||lo|| (all products of the split counted), plus the
// unrepresented rest scaled by 1/coef, so that coef * |x| * bound still covers it.
__global__ void __launch_bounds__(256) split_w32_kernel(const float* __restrict__ W, int E, int H,
                                                         __nv_bfloat16* __restrict__ W3,
                                                         double* __restrict__ wnorm, double rest_scale) {
  __shared__ double red[8][4];
  pdl_wait();
  const int e = blockIdx.x;  // one block per expert row, four floats per thread and step
  const float* w = W + static_cast<int64_t>(e) * H;
  __nv_bfloat16* out = W3 + static_cast<int64_t>(e) * 3 * H;
  double ss[4] = {0.0, 0.0, 0.0, 0.0};
  for (int v = threadIdx.x; v < H / 4; v += blockDim.x) {
    const Vec16<float> w4 = ld16(w + v * 4);
    __nv_bfloat16 part[3][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x0 = w4.v[j];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x0);
      const float r1 = __fsub_rn(x0, __bfloat162float(hi));
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const float r2 = __fsub_rn(r1, __bfloat162float(mid));
      const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
      const double r3 = static_cast<double>(r2) - static_cast<double>(__bfloat162float(lo));
      part[0][j] = hi;
      part[1][j] = mid;
      part[2][j] = lo;
      const double dh = __bfloat162float(hi), dm = __bfloat162float(mid), dl = __bfloat162float(lo);
      ss[0] = fma(dh, dh, ss[0]);
      ss[1] = fma(dm, dm, ss[1]);
      ss[2] = fma(dl, dl, ss[2]);
      ss[3] = fma(r3, r3, ss[3]);
    }
#pragma unroll
    for (int q = 0; q < 3; ++q)
      *reinterpret_cast<uint2*>(out + static_cast<int64_t>(q) * H + v * 4) = *reinterpret_cast<const uint2*>(part[q]);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss[q] += __shfl_xor_sync(0xffffffffu, ss[q], o);
    if (lane == 0) red[warp][q] = ss[q];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t[4] = {0.0, 0.0, 0.0, 0.0};
    for (int w8 = 0; w8 < static_cast<int>(blockDim.x >> 5); ++w8)
      for (int q = 0; q < 4; ++q) t[q] += red[w8][q];
    double b = __dadd_ru(norm_ub_from_sumsq(t[0], H), norm_ub_from_sumsq(t[1], H));
    b = __dadd_ru(b, norm_ub_from_sumsq(t[2], H));
    b = __dadd_ru(b, __dmul_ru(norm_ub_from_sumsq(t[3], H), rest_scale));
    wnorm[e] = b;
  }
}

// The selection of the tensor-core scores: one warp per token.
template <typename TW, int EPL, bool SIG>
static cudaError_t launch_select(const RouterArgs& a, const TW* Wsel, double coef, int Kg, cudaStream_t st) {
  using bf16 = __nv_bfloat16;
  const double delta_abs = Kg * 2.350988701644575e-38;
  const bf16* x = static_cast<const bf16*>(a.x);
  const Keys kf{a.bias, a.sigmoid, a.scale};
  const unsigned sgrid = static_cast<unsigned>((a.T + kSelectWarps - 1) / kSelectWarps);
  return launch_pdl(route_select_kernel<bf16, TW, EPL, SIG>, dim3(sgrid), dim3(32 * kSelectWarps), 0, st,
                    static_cast<const double*>(a.scores64), coef, delta_abs, static_cast<const double*>(a.xnorm),
                    static_cast<const double*>(a.wnorm), kf, x, Wsel, a.T, a.H, a.E, a.k, a.idx_ws, a.w_ws,
                    a.idx_user, a.w_user, a.spill, a.ctrl);
}

template <typename TW, bool SIG>
static cudaError_t launch_select_epl(const RouterArgs& a, const TW* Wsel, double coef, int Kg, cudaStream_t st) {
  const int epl = select_epl(a.E);
  return epl == 4    ? launch_select<TW, 4, SIG>(a, Wsel, coef, Kg, st)
         : epl == 12 ? launch_select<TW, 12, SIG>(a, Wsel, coef, Kg, st)
                     : launch_select<TW, 32, SIG>(a, Wsel, coef, Kg, st);
}

static cudaError_t launch_router_tc(const RouterArgs& a, cudaStream_t st) {
  using bf16 = __nv_bfloat16;
  RouterTcParams p{};
  const int Kg = a.w32 ? 3 * a.H : a.H;  // length of the GEMM's reduction
  p.T = a.T;
  p.H = Kg;
  p.Hx = a.H;
  p.E = a.E;
  p.w_given = a.w32 ? 1 : 0;
  p.scores = a.scores64;
  p.ctrl = a.ctrl;
  const bf16* x = static_cast<const bf16*>(a.x);
  const bf16* Wg = static_cast<const bf16*>(a.w32 ? a.w3 : a.Wr);  // the GEMM's B operand
  if (!encode_bf16_rows(&p.tmX, a.x, a.T, a.H, kRtRowBox) ||
      (a.T >= kTileM && !encode_bf16_rows(&p.tmX128, a.x, a.T, a.H, kTileM)) ||
      !encode_bf16_rows(&p.tmW, Wg, a.E, Kg, kRtExperts))
    return cudaErrorInvalidValue;
  if (a.T < kTileM) p.tmX128 = p.tmX;  // no full token tile: never used
  cudaError_t e = allow_smem(router_gemm_tc_kernel, kRtSmem);
  if (e != cudaSuccess) return e;
  // Each slice of L = 256 products is accumulated in fp32 from exact products, at most
  // 2^-23 relative per accumulation step (truncation included), so its error is
  // <= 2 L 2^-23 * sum|x w| over the slice; adding the K/L partials in fp64 costs at most
  // 2 (K/L) 2^-53 more; K 2^-125 covers partial sums flushed below the normal range.
  const double slice = static_cast<double>(kRtSliceSteps) * kTileK;
  const double coef = 2.0 * slice * kU23 + 2.0 * (Kg / slice + 1) * kU53;
  int launches = 2;
  if (a.w32) {
    e = launch_pdl(split_w32_kernel, dim3(static_cast<unsigned>(a.E)), dim3(256), 0, st,
                   static_cast<const float*>(a.Wr), a.E, a.H, static_cast<bf16*>(a.w3), a.wnorm,
                   (1.0 / coef) * (1.0 + 0x1p-40));  // >= 1 / coef
    if (e != cudaSuccess) return e;
    ++launches;
  }
  const int n_sl = (Kg / kTileK + kRtSliceSteps - 1) / kRtSliceSteps;
  const int chunks = a.rsplit ? router_chunks(a.T, a.E, Kg) : 1;
  p.chunks = chunks;
  p.chunk_slices = (n_sl + chunks - 1) / chunks;
  if (chunks > 1) {
    // the split blocks also produce the norm bounds
    double* d = static_cast<double*>(a.rsplit);
    p.x = x;
    p.Wr = Wg;
    p.xss = d;
    p.wss = d + static_cast<int64_t>(chunks) * a.T;
    p.part = reinterpret_cast<float*>(p.wss + static_cast<int64_t>(chunks) * a.E);
    p.tile_done = a.group_done;
    p.xnorm = a.xnorm;
    p.wnorm = a.wnorm;
    p.last_block_reduces = a.T <= kRtSplitMaxTokens ? 1 : 0;
  } else {
    const int64_t wrows = a.w32 ? 0 : a.E;  // split fp32 weights come with their norm bounds
    e = launch_pdl(row_norm_ub_kernel<bf16>, dim3(static_cast<unsigned>(((a.T + wrows) * 32 + 255) / 256)),
                   dim3(256), 0, st, x, a.T, a.xnorm, Wg, wrows, a.wnorm, a.H);
    if (e != cudaSuccess) return e;
    ++launches;
  }
  e = launch_pdl(router_gemm_tc_kernel,
                 dim3(static_cast<unsigned>(((a.T + kTileM - 1) / kTileM) * ((a.E + kRtExperts - 1) / kRtExperts)), 1,
                      static_cast<unsigned>(chunks)),
                 dim3(192), static_cast<size_t>(kRtSmem), st, p);
  if (e != cudaSuccess) return e;
  if (chunks > 1 && !p.last_block_reduces) {
    const int64_t jobs = a.T * a.E + a.T + a.E;
    e = launch_pdl(router_reduce_kernel, dim3(static_cast<unsigned>(std::min<int64_t>((jobs + 255) / 256, 148 * 4))),
                   dim3(256), 0, st, p);
    if (e != cudaSuccess) return e;
    ++launches;
  }
  const float* Wf = static_cast<const float*>(a.Wr);
  if (a.w32)  // the recomputations read the fp32 weights themselves
    e = a.sigmoid ? launch_select_epl<float, true>(a, Wf, coef, Kg, st)
                  : launch_select_epl<float, false>(a, Wf, coef, Kg, st);
  else
    e = a.sigmoid ? launch_select_epl<bf16, true>(a, static_cast<const bf16*>(a.Wr), coef, Kg, st)
                  : launch_select_epl<bf16, false>(a, static_cast<const bf16*>(a.Wr), coef, Kg, st);
  count_launches(launches);
  return e;
}

template <typename T>
static cudaError_t launch_router_decode(const RouterArgs& a, cudaStream_t st) {
  const dim3 grid((a.E + kDecodeExp - 1) / kDecodeExp, static_cast<unsigned>((a.T + kDecodeTok - 1) / kDecodeTok),
                  kDecodeSplit);
  auto go = [&](auto kern) {
    return launch_pdl(kern, grid, dim3(kDecodeThreads), 0, st, static_cast<const T*>(a.x),
                      static_cast<const T*>(a.Wr), Keys{a.bias, a.sigmoid, a.scale}, a.T, a.H, a.E, a.k,
                      a.scores64, a.wss,
                      a.group_done, a.idx_ws, a.w_ws, a.idx_user, a.w_user, a.spill, a.ctrl);
  };
  const int epl = select_epl(a.E);
  cudaError_t e;
  if (a.sigmoid)
    e = epl == 4 ? go(router_decode_kernel<T, 4, true>)
        : epl == 12 ? go(router_decode_kernel<T, 12, true>) : go(router_decode_kernel<T, 32, true>);
  else
    e = epl == 4 ? go(router_decode_kernel<T, 4, false>)
        : epl == 12 ? go(router_decode_kernel<T, 12, false>) : go(router_decode_kernel<T, 32, false>);
  count_launches(1);
  return e;
}

int64_t router_group_counters(int64_t T, int E) {
  const int64_t tiles = ((T + kTileM - 1) / kTileM) * ((E + kRtExperts - 1) / kRtExperts);
  return std::max<int64_t>((T + kDecodeTok - 1) / kDecodeTok, tiles);
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (router_tc_supported(a.bf16, a.T, a.E, a.H)) return launch_router_tc(a, st);
  if (a.bf16) return launch_router_decode<__nv_bfloat16>(a, st);
  return launch_router_decode<float>(a, st);
}

}  // namespace moe
