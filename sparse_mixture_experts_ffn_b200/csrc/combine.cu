// combine.cu -- unpermute and combine: y_t = sum_{j<k} o[inv_perm[t*k+j]] + o_shared[t],
// accumulated in fp32 in fixed slot order (deterministic), stored in the working dtype.
// The rows of o already carry their routing weight (fused in the down projection); the
// shared expert (share_expert_dim on the llm-atlas page "Step-3.5-Flash") has weight 1.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// BATCHED: the slots' row indices and rows are loaded eight at a time (short latency chains
// for small batches); otherwise one slot at a time (more threads resident for large ones).
template <typename T, bool BATCHED>
__global__ void combine_kernel(const int32_t* __restrict__ inv_perm, const T* __restrict__ o,
                               const T* __restrict__ o_shared, int64_t Tn, int H, int k,
                               T* __restrict__ y, Ctrl* ctrl) {
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  constexpr int V = Vec16<T>::N;
  const int vpr = H / V;
  const int64_t total = Tn * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vpr;
    const int v = static_cast<int>(i - t * vpr);
    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.f;
    if (!BATCHED) {
      for (int s = 0; s < k; ++s) {
        const int64_t row = __ldg(inv_perm + t * k + s);
        if (row < 0 || row >= Tn * k) {
          set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
          continue;
        }
        const Vec16<T> r = ld16(o + row * H + v * V);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] += to_f32(r.v[j]);
      }
    }
    // slots in groups of 8: the row indices, then the rows, each group's loads in flight
    // together; the sum stays in slot order
    for (int s0 = 0; BATCHED && s0 < k; s0 += 8) {
      int64_t row[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        row[u] = (s0 + u < k) ? __ldg(inv_perm + t * k + s0 + u) : 0;
        if (row[u] < 0 || row[u] >= Tn * k) {
          set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
          row[u] = -1;
        }
      }
      Vec16<T> r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (s0 + u < k && row[u] >= 0) r[u] = ld16(o + row[u] * H + v * V);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (s0 + u < k && row[u] >= 0) {
#pragma unroll
          for (int j = 0; j < V; ++j) acc[j] += to_f32(r[u].v[j]);
        }
    }
    if (o_shared) {
      const Vec16<T> r = ld16(o_shared + t * H + v * V);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] += to_f32(r.v[j]);
    }
    Vec16<T> out;
#pragma unroll
    for (int j = 0; j < V; ++j) out.v[j] = from_f32<T>(acc[j]);
    reinterpret_cast<uint4*>(y + t * H)[v] = *reinterpret_cast<const uint4*>(&out);
  }
}

// Expert parallelism: one rank's fp32 share of the output,
//   y_partial[t] = sum_{j: row(t, j) in [p_lo, p_hi)} o[row(t, j)] + [sh_lo <= t < sh_hi] o_shared[t],
// where rows [p_lo, p_hi) = [offsets[e_lo], offsets[e_hi]) are those of this rank's experts
// (the only rows of o its GEMMs wrote).  Slots are added in slot order; the ranks' shares
// are added afterwards (moe_layer_sum_partials, or a reduce-scatter).
template <typename T>
__global__ void combine_partial_kernel(const int32_t* __restrict__ inv_perm, const int32_t* __restrict__ offsets,
                                       int e_lo, int e_hi, const T* __restrict__ o,
                                       const T* __restrict__ o_shared, int64_t sh_lo, int64_t sh_hi,
                                       int64_t Tn, int H, int k, float* __restrict__ y, Ctrl* ctrl) {
  pdl_wait();
  pdl_trigger();
  constexpr int V = Vec16<T>::N;
  const int vpr = H / V;
  const int64_t total = Tn * vpr;
  const int64_t p_lo = __ldg(offsets + e_lo), p_hi = __ldg(offsets + e_hi);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vpr;
    const int v = static_cast<int>(i - t * vpr);
    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.f;
    for (int s = 0; s < k; ++s) {
      const int64_t row = __ldg(inv_perm + t * k + s);
      if (row < 0 || row >= Tn * k) {
        set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
        continue;
      }
      if (row < p_lo || row >= p_hi) continue;  // another rank's expert
      const Vec16<T> r = ld16(o + row * H + v * V);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] += to_f32(r.v[j]);
    }
    if (o_shared && t >= sh_lo && t < sh_hi) {
      const Vec16<T> r = ld16(o_shared + t * H + v * V);
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] += to_f32(r.v[j]);
    }
    float4* dst = reinterpret_cast<float4*>(y + t * H + v * V);
#pragma unroll
    for (int j = 0; j < V / 4; ++j) dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
  }
}

// y = sum_{r < n} parts[r], fp32 in rank order, stored in the working dtype.  The parts may
// be other GPUs' buffers mapped into this process (peer pointers over NVLink): the reduction
// of the ranks' shares then reads each peer's memory once.
struct PartsArg {
  const float* p[kMaxParts];
};

template <typename T>
__global__ void sum_partials_kernel(const __grid_constant__ PartsArg parts, int n, int64_t count4,
                                    T* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 acc = __ldcs(reinterpret_cast<const float4*>(parts.p[0]) + i);
    for (int r = 1; r < n; ++r) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(parts.p[r]) + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if constexpr (sizeof(T) == 4) {
      reinterpret_cast<float4*>(y)[i] = acc;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 out;
      out.x = *reinterpret_cast<uint32_t*>(&lo);
      out.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(y)[i] = out;
    }
  }
}

cudaError_t launch_sum_partials(const float* const* parts, int n, int64_t count, bool bf16, void* y,
                                cudaStream_t st) {
  if (count == 0) return cudaSuccess;
  PartsArg pa{};
  for (int r = 0; r < n; ++r) pa.p[r] = parts[r];
  const int64_t count4 = count / 4;
  const int blocks = static_cast<int>(std::min<int64_t>((count4 + 255) / 256, 148 * 8));
  cudaError_t e = bf16 ? launch_pdl(sum_partials_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, pa, n,
                                    count4, static_cast<__nv_bfloat16*>(y))
                       : launch_pdl(sum_partials_kernel<float>, dim3(blocks), dim3(256), 0, st, pa, n, count4,
                                    static_cast<float*>(y));
  count_launches(1);
  return e;
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t vec = a.T * (a.H / (a.bf16 ? 8 : 4));
  const int blocks = static_cast<int>(std::min<int64_t>((vec + 255) / 256, 148 * 16));
  cudaError_t e;
  const bool batched = vec <= 148 * 256;  // fewer rows than one thread each on a full GPU
  auto go = [&](auto kern, auto* o, auto* o_shared, auto* y) {
    return launch_pdl(kern, dim3(blocks), dim3(256), 0, st, a.inv_perm, o, a.has_shared ? o_shared : nullptr,
                      a.T, a.H, a.k, y, a.ctrl);
  };
  using bf = __nv_bfloat16;
  if (a.y_partial) {  // expert parallelism: this rank's fp32 share (bf16 layers only)
    e = launch_pdl(combine_partial_kernel<bf>, dim3(blocks), dim3(256), 0, st, a.inv_perm, a.offsets, a.e_lo,
                   a.e_hi, static_cast<const bf*>(a.o), a.has_shared ? static_cast<const bf*>(a.o_shared) : nullptr,
                   a.shared_lo, a.shared_hi, a.T, a.H, a.k, a.y_partial, a.ctrl);
    count_launches(1);
    return e;
  }
  if (a.bf16) {
    const bf* o = static_cast<const bf*>(a.o);
    const bf* os = static_cast<const bf*>(a.o_shared);
    bf* y = static_cast<bf*>(a.y);
    e = batched ? go(combine_kernel<bf, true>, o, os, y) : go(combine_kernel<bf, false>, o, os, y);
  } else {
    const float* o = static_cast<const float*>(a.o);
    const float* os = static_cast<const float*>(a.o_shared);
    float* y = static_cast<float*>(a.y);
    e = batched ? go(combine_kernel<float, true>, o, os, y) : go(combine_kernel<float, false>, o, os, y);
  }
  count_launches(1);
  return e;
}

}  // namespace moe
