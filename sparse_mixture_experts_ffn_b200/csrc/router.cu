// router.cu -- router scores, certified top-k selection and renormalised softmax weights.
//
// The routing decision must equal the one made on the exact fp32 router score
// s[t,e] = RN32(sum_h x[t,h] W_r[e,h]) (llm-atlas page "Step-3.5-Flash", table "Champs
// bruts du config.json": need_fp32_gate true, moe_top_k 8, norm_expert_weight true).
// A fast score s^ comes with a rigorous bound |s^ - s_real| <= delta; the fp32 key of an
// expert is then known to lie in [key(s^-delta), key(s^+delta)].  Experts whose interval
// can matter for the top-k set are recomputed in fp64 (delta ~ 2^-41 relative) and, if
// that is still not conclusive, with an exact integer dot product.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------------------
// Upper bounds of row 2-norms, fp64: sqrt(sum v^2) rounded up, with the fp64 summation
// error (at most n*2^-53 relative for n terms) covered by a factor (1 + 2 n 2^-53).
// One warp per row.
// ---------------------------------------------------------------------------------------
template <typename T>
__global__ void row_norm_ub_kernel(const T* __restrict__ A, int64_t rows, int H,
                                   double* __restrict__ out) {
  int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int V = Vec16<T>::N;
  const T* p = A + row * H;
  double ss = 0.0;
  for (int v = lane; v < H / V; v += 32) {
    Vec16<T> a = ld16(p + v * V);
#pragma unroll
    for (int j = 0; j < V; ++j) {
      double d = static_cast<double>(to_f32(a.v[j]));
      ss = fma(d, d, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) {
    double infl = __dadd_ru(1.0, __dmul_ru(2.0 * H, 1.1102230246251565e-16));  // 2^-53
    out[row] = __dsqrt_ru(__dmul_ru(ss, infl));
  }
}

// ---------------------------------------------------------------------------------------
// fp64 router scores: products exact in fp64, fp64 accumulation in any order.
// One block (256 threads) per (expert, group of TT tokens).
// ---------------------------------------------------------------------------------------
template <typename T, int TT>
__global__ void __launch_bounds__(256) router_scores_f64_kernel(
    const T* __restrict__ x, const T* __restrict__ Wr, int64_t T_, int H, int E,
    double* __restrict__ scores) {
  const int e = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * TT;
  const int nt = static_cast<int>(min64(TT, T_ - t0));
  constexpr int V = Vec16<T>::N;
  double acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.0;
  const T* w = Wr + static_cast<size_t>(e) * H;
  for (int v = threadIdx.x; v < H / V; v += blockDim.x) {
    Vec16<T> wv = ld16(w + v * V);
    double wd[V];
#pragma unroll
    for (int j = 0; j < V; ++j) wd[j] = static_cast<double>(to_f32(wv.v[j]));
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (t < nt) {
        Vec16<T> xv = ld16(x + (t0 + t) * H + v * V);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[t] = fma(static_cast<double>(to_f32(xv.v[j])), wd[j], acc[t]);
      }
    }
  }
  __shared__ double red[8][TT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    double v = acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][t] = v;
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    double v = 0.0;
    for (int w8 = 0; w8 < (blockDim.x >> 5); ++w8) v += red[w8][threadIdx.x];
    scores[(t0 + threadIdx.x) * E + e] = v;
  }
}

// ---------------------------------------------------------------------------------------
// Exact dot product of one (token, expert) pair by one warp, rounded once to fp32.
// Every bf16/fp32 value is m * 2^q with integer m; each product's integer mantissa is
// added into an int64 bin for its exponent (fp32 products are split in two 24-bit
// halves).  Lane 0 then folds the bins into 32-bit limbs, resolves the sign and rounds
// the integer to the nearest fp32 (ties to even, subnormals included).
// ---------------------------------------------------------------------------------------
constexpr int kQMin = -298;               // smallest product exponent (fp32 subnormal^2)
constexpr int kNBins = 241 - kQMin + 1;   // up to 2^241 (bf16 max^2 / fp32 upper halves)
constexpr int kNLimbs = (kNBins + 31) / 32 + 4;

__device__ __forceinline__ void decode(float v, int& m, int& q) {
  uint32_t b = __float_as_uint(v);
  uint32_t ex = (b >> 23) & 0xFF, fr = b & 0x7FFFFF;
  m = ex ? static_cast<int>(fr | 0x800000u) : static_cast<int>(fr);
  q = ex ? static_cast<int>(ex) - 150 : -149;
  if (b >> 31) m = -m;
}
__device__ __forceinline__ void decode(__nv_bfloat16 v, int& m, int& q) {
  uint32_t b = __bfloat16_as_ushort(v);
  uint32_t ex = (b >> 7) & 0xFF, fr = b & 0x7F;
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
  uint32_t rb = bit(lsb - 1);
  bool sticky = false;
  const int sb = lsb - 2;  // bits [0, sb] are sticky
  if (sb >= 0) {
    for (int j = 0; j < (sb >> 5); ++j) sticky |= (d[j] != 0);
    uint32_t partial = d[sb >> 5] & (((sb & 31) == 31) ? 0xFFFFFFFFu : ((2u << (sb & 31)) - 1u));
    sticky |= (partial != 0);
  }
  if (rb && (sticky || (mant & 1u))) mant += 1;
  double v = ldexp(static_cast<double>(mant), lsb_exp);
  float f = (v > static_cast<double>(FLT_MAX)) ? __int_as_float(0x7f800000) : static_cast<float>(v);
  return negative ? -f : f;
}

template <typename T>
__device__ float warp_exact_dot_rn32(const T* __restrict__ a, const T* __restrict__ b, int H,
                                     long long* bins /* kNBins, warp-private smem */) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < kNBins; i += 32) bins[i] = 0;
  __syncwarp();
  for (int h = lane; h < H; h += 32) {
    int m1, q1, m2, q2;
    decode(a[h], m1, q1);
    decode(b[h], m2, q2);
    long long p = static_cast<long long>(m1) * m2;
    if (p == 0) continue;
    const int q = q1 + q2;
    const long long sg = p < 0 ? -1 : 1;
    const long long mag = p < 0 ? -p : p;
    atomicAdd(reinterpret_cast<unsigned long long*>(&bins[q - kQMin]),
              static_cast<unsigned long long>(sg * (mag & 0xFFFFFF)));
    if (mag >> 24)
      atomicAdd(reinterpret_cast<unsigned long long*>(&bins[q + 24 - kQMin]),
                static_cast<unsigned long long>(sg * (mag >> 24)));
  }
  __syncwarp();
  float result = 0.0f;
  if (lane == 0) {
    __int128 L[kNLimbs];
    for (int j = 0; j < kNLimbs; ++j) L[j] = 0;
    for (int i = 0; i < kNBins; ++i) L[i >> 5] += static_cast<__int128>(bins[i]) << (i & 31);
    uint32_t d[kNLimbs];
    __int128 carry = 0;
    for (int j = 0; j < kNLimbs; ++j) {
      __int128 v = L[j] + carry;
      d[j] = static_cast<uint32_t>(static_cast<unsigned __int128>(v) & 0xFFFFFFFFu);
      carry = v >> 32;  // arithmetic shift: floor division
    }
    const bool negative = (carry < 0);  // carry is 0 or -1: the limbs hold the full value
    if (negative) {  // two's complement of the limb string
      uint64_t c = 1;
      for (int j = 0; j < kNLimbs; ++j) {
        uint64_t v = static_cast<uint64_t>(~d[j]) + c;
        d[j] = static_cast<uint32_t>(v);
        c = v >> 32;
      }
    }
    result = round_limbs_rn32(d, kNLimbs, negative);
  }
  __syncwarp();
  return __shfl_sync(0xffffffffu, result, 0);
}

template <typename T>
__device__ double warp_dot_f64(const T* __restrict__ a, const T* __restrict__ b, int H) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
  for (int h = lane; h < H; h += 32)
    acc = fma(static_cast<double>(to_f32(a[h])), static_cast<double>(to_f32(b[h])), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// ---------------------------------------------------------------------------------------
// Certified selection.  One warp per token.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ordered(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_of(double s, const float* bias, int e) {
  float s32 = __double2float_rn(s);
  return bias ? __fadd_rn(s32, bias[e]) : s32;
}

// a is ranked before b: larger key, then lower index
__device__ __forceinline__ bool better(float ka, int a, float kb, int b) {
  return (ka > kb) || (ka == kb && a < b);
}

constexpr int kSelectWarps = 4;

template <typename T, typename S>
__global__ void __launch_bounds__(32 * kSelectWarps) route_select_kernel(
    const S* __restrict__ scores, double delta_coef, double delta_abs,
    const double* __restrict__ xnorm, const double* __restrict__ wnorm,
    const float* __restrict__ bias, const T* __restrict__ x, const T* __restrict__ Wr,
    int64_t T_, int H, int E, int k, int32_t* __restrict__ idx_ws, float* __restrict__ w_ws,
    int32_t* __restrict__ idx_user, float* __restrict__ w_user, Ctrl* ctrl) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kSelectWarps + warp;
  // per warp: lo[E], hi[E] floats, flags[E] bytes, bins[kNBins] int64
  const size_t per_warp = (static_cast<size_t>(E) * 9 + 15) / 16 * 16 + sizeof(long long) * kNBins;
  unsigned char* mine = smem_raw + per_warp * warp;
  long long* bins = reinterpret_cast<long long*>(mine);
  float* lo = reinterpret_cast<float*>(mine + sizeof(long long) * kNBins);
  float* hi = lo + E;
  unsigned char* flag = reinterpret_cast<unsigned char*>(hi + E);  // 1 = candidate, 2 = chosen
  if (t >= T_) return;

  const T* xt = x + t * H;
  const double nx = xnorm[t];
  // 1. key intervals
  for (int e = lane; e < E; e += 32) {
    const double sh = static_cast<double>(scores[t * E + e]);
    const double d = __dadd_ru(__dmul_ru(__dmul_ru(delta_coef, nx), wnorm[e]), delta_abs);
    lo[e] = key_of(__dadd_rd(sh, -d), bias, e);
    hi[e] = key_of(__dadd_ru(sh, d), bias, e);
  }
  __syncwarp();
  // 2. Lk = k-th largest lower bound: largest u with #{e : ordered(lo_e) >= u} >= k
  uint32_t u = 0;
  for (int bitpos = 31; bitpos >= 0; --bitpos) {
    const uint32_t cand = u | (1u << bitpos);
    int c = 0;
    for (int e = lane; e < E; e += 32) c += (ordered(lo[e]) >= cand);
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= k) u = cand;
  }
  // 3. candidates: hi_e >= Lk; everything else is beaten by >= k experts for certain
  for (int e = lane; e < E; e += 32) flag[e] = (ordered(hi[e]) >= u) ? 1 : 0;
  __syncwarp();
  // 4. recompute the candidates whose key is not yet certain
  int n_ref = 0, n_exact = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const bool need = (e < E) && flag[e] && (lo[e] != hi[e]);
    unsigned mask = __ballot_sync(0xffffffffu, need);
    while (mask) {
      const int src = __ffs(mask) - 1;
      mask &= mask - 1;
      const int ee = base + src;
      const T* we = Wr + static_cast<size_t>(ee) * H;
      float klo, khi;
      if constexpr (sizeof(S) == 4) {  // scores came from the fp32 pass: fp64 recompute first
        const double s64 = warp_dot_f64(xt, we, H);
        const double d = __dmul_ru(__dmul_ru(1.01 * H * 1.1102230246251565e-16, nx), wnorm[ee]);
        klo = key_of(__dadd_rd(s64, -d), bias, ee);
        khi = key_of(__dadd_ru(s64, d), bias, ee);
        ++n_ref;
      } else {
        klo = lo[ee];
        khi = hi[ee];
      }
      if (klo != khi) {
        const float s32 = warp_exact_dot_rn32(xt, we, H, bins);
        klo = khi = bias ? __fadd_rn(s32, bias[ee]) : s32;
        ++n_exact;
      }
      if (lane == 0) {
        lo[ee] = klo;
        hi[ee] = khi;
      }
      __syncwarp();
    }
  }
  // 5. pick the top k candidates by (key desc, index asc); all their keys are exact now
  for (int j = 0; j < k; ++j) {
    float bk = 0.0f;
    int be = -1;
    for (int e = lane; e < E; e += 32)
      if (flag[e] == 1 && (be < 0 || better(lo[e], e, bk, be))) {
        bk = lo[e];
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
    if (be < 0) {  // only with non-finite keys (outside the contract): stay in bounds
      if (lane == 0) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      for (int e = 0; e < E; ++e)
        if (flag[e] != 2) { be = e; break; }
    }
    if (lane == 0) flag[be] = 2;
    __syncwarp();
  }
  // 6. renormalised softmax over the chosen keys, fp64; write in ascending expert order
  float m = -FLT_MAX;
  for (int e = lane; e < E; e += 32)
    if (flag[e] == 2) m = fmaxf(m, lo[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  double z = 0.0;
  for (int e = lane; e < E; e += 32)
    if (flag[e] == 2) z += exp(static_cast<double>(lo[e]) - static_cast<double>(m));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  int written = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const bool ch = (e < E) && flag[e] == 2;
    const unsigned mask = __ballot_sync(0xffffffffu, ch);
    if (ch) {
      const int pos = written + __popc(mask & ((1u << lane) - 1u));
      const float w = static_cast<float>(exp(static_cast<double>(lo[e]) - static_cast<double>(m)) / z);
      idx_ws[t * k + pos] = e;
      w_ws[t * k + pos] = w;
      if (idx_user) idx_user[t * k + pos] = e;
      if (w_user) w_user[t * k + pos] = w;
    }
    written += __popc(mask);
  }
  if (lane == 0 && (n_ref | n_exact)) {
    if (n_ref) atomicAdd(&ctrl->n_refined, static_cast<unsigned long long>(n_ref));
    if (n_exact) atomicAdd(&ctrl->n_exact, static_cast<unsigned long long>(n_exact));
    atomicAdd(&ctrl->n_tokens_refined, 1ull);
  }
}

// ---------------------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------------------
template <typename T>
static cudaError_t launch_router_f64_t(const RouterArgs& a, cudaStream_t st) {
  const T* x = static_cast<const T*>(a.x);
  const T* Wr = static_cast<const T*>(a.Wr);
  {
    const int64_t rows = a.T;
    row_norm_ub_kernel<T><<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(x, rows, a.H, a.xnorm);
    row_norm_ub_kernel<T><<<static_cast<unsigned>((a.E * 32 + 255) / 256), 256, 0, st>>>(Wr, a.E, a.H, a.wnorm);
  }
  constexpr int TT = 8;
  dim3 grid(a.E, static_cast<unsigned>((a.T + TT - 1) / TT));
  router_scores_f64_kernel<T, TT><<<grid, 256, 0, st>>>(x, Wr, a.T, a.H, a.E, a.scores64);
  const size_t per_warp = (static_cast<size_t>(a.E) * 9 + 15) / 16 * 16 + sizeof(long long) * kNBins;
  const size_t smem = per_warp * kSelectWarps;
  auto kern = route_select_kernel<T, double>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // fp64 scores: |s^ - s| <= 1.01 * H * 2^-53 * ||x|| ||w|| (any summation order)
  const double coef = 1.01 * a.H * 1.1102230246251565e-16;
  kern<<<static_cast<unsigned>((a.T + kSelectWarps - 1) / kSelectWarps), 32 * kSelectWarps, smem, st>>>(
      a.scores64, coef, 0.0, a.xnorm, a.wnorm, a.bias, x, Wr, a.T, a.H, a.E, a.k, a.idx_ws,
      a.w_ws, a.idx_user, a.w_user, a.ctrl);
  count_launches(4);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (a.bf16) return launch_router_f64_t<__nv_bfloat16>(a, st);
  return launch_router_f64_t<float>(a, st);
}

}  // namespace moe
