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

template <typename T>
__global__ void combine_kernel(const int32_t* __restrict__ inv_perm, const T* __restrict__ o,
                               const T* __restrict__ o_shared, int64_t Tn, int H, int k,
                               T* __restrict__ y, Ctrl* ctrl) {
  pdl_wait();
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
  pdl_trigger();
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t vec = a.T * (a.H / (a.bf16 ? 8 : 4));
  const int blocks = static_cast<int>(std::min<int64_t>((vec + 255) / 256, 148 * 16));
  cudaError_t e;
  if (a.bf16)
    e = launch_pdl(combine_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, a.inv_perm,
                   static_cast<const __nv_bfloat16*>(a.o),
                   a.has_shared ? static_cast<const __nv_bfloat16*>(a.o_shared) : nullptr, a.T, a.H,
                   a.k, static_cast<__nv_bfloat16*>(a.y), a.ctrl);
  else
    e = launch_pdl(combine_kernel<float>, dim3(blocks), dim3(256), 0, st, a.inv_perm,
                   static_cast<const float*>(a.o),
                   a.has_shared ? static_cast<const float*>(a.o_shared) : nullptr, a.T, a.H, a.k,
                   static_cast<float*>(a.y), a.ctrl);
  count_launches(1);
  return e;
}

}  // namespace moe
