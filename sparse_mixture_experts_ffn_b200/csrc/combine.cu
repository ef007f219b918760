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
