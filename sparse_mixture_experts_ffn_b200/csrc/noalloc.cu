// noalloc.cu -- routing of a token batch for callers that cannot allocate device memory.
//
// moe_layer_forward() takes a caller-provided workspace.  Some callers have no way to
// provide one: an inference runtime whose memory planner owns every device buffer and
// hands each layer only its inputs and outputs; a host program that must not call
// cudaMalloc on its latency-critical path (the allocation can synchronise the device);
// a plugin that a host framework calls with tensors but without an allocator.  For them,
// moe_layer_route_noalloc() runs the routing step (router scores, certified top-k and
// renormalised softmax weights) with its scratch in a fixed device array compiled into
// this library: kNoAllocScratchBytes on every GPU that loads it, held until the process
// exits.  It allocates nothing and calls no allocating routine.
//
// The array is shared by every call: calls that may overlap on the GPU (other streams,
// other host threads) race on it and must be serialised by the caller.  The part that
// must start at zero (status word and counters) is cleared by each call on its stream.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe_layer.h"

namespace moe {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

// Device address of g_route_scratch on the current device.  The symbol name is only a
// host-side stand-in; the address must come from the runtime, once per device, with that
// device current.  The first call on a device does this set-up.
static cudaError_t scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

static size_t align_up(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_layer_route_noalloc(const moe_layer_shape* shape, const void* x,
                                              const void* W_router, const float* router_bias,
                                              int32_t* topk_idx, float* topk_w, void* stream) {
  if (!shape) return MOE_ERR_INVALID_ARG;
  const moe_layer_shape& s = *shape;
  if (s.dtype != MOE_F32 && s.dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (s.T < 0 || s.H < 1 || s.E < 1 || s.top_k < 1 || s.top_k > s.E) return MOE_ERR_INVALID_ARG;
  if (s.E > 1024 || s.H % 8 || s.H > (1 << 20) ||
      s.T * static_cast<int64_t>(s.top_k) >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.T == 0) return MOE_OK;
  if (!x || !W_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(W_router)) & 15u ||
      (reinterpret_cast<uintptr_t>(router_bias) | reinterpret_cast<uintptr_t>(topk_idx) |
       reinterpret_cast<uintptr_t>(topk_w)) & 3u)
    return MOE_ERR_INVALID_ARG;

  // carve the scratch: control block and counters (cleared each call), then the scores,
  // norms and the key spill of the rare exact path
  const size_t T = static_cast<size_t>(s.T), E = static_cast<size_t>(s.E);
  const bool tc = router_scores_f32(s);
  const size_t groups = static_cast<size_t>(router_group_counters(s.T, s.E));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  const size_t o_ctrl = take(sizeof(Ctrl));
  const size_t o_group = take(groups * 4);
  const size_t o_wss = take(tc ? 0 : groups * E * 8);
  const size_t o_scores = take(T * E * 8);
  const size_t zero_end = tc ? o_scores : off;
  const size_t o_xnorm = take(T * 8);
  const size_t o_wnorm = take(E * 8);
  const size_t o_spill = take(T * E * 20);
  if (off > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
  char* ws = static_cast<char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, zero_end, st) != cudaSuccess) return MOE_ERR_CUDA;

  RouterArgs ra{};
  ra.bf16 = s.dtype == MOE_BF16;
  ra.T = s.T;
  ra.H = s.H;
  ra.E = s.E;
  ra.k = s.top_k;
  ra.x = x;
  ra.Wr = W_router;
  ra.bias = router_bias;
  ra.scores64 = reinterpret_cast<double*>(ws + o_scores);
  ra.wss = reinterpret_cast<double*>(ws + o_wss);
  ra.xnorm = reinterpret_cast<double*>(ws + o_xnorm);
  ra.wnorm = reinterpret_cast<double*>(ws + o_wnorm);
  ra.group_done = reinterpret_cast<unsigned int*>(ws + o_group);
  ra.idx_ws = topk_idx;
  ra.w_ws = topk_w;
  ra.idx_user = nullptr;
  ra.w_user = nullptr;
  ra.spill = reinterpret_cast<float*>(ws + o_spill);
  ra.rsplit = nullptr;  // the scratch holds no reduction-split partials
  ra.sigmoid = 0;       // the softmax router
  ra.scale = 1.0f;
  ra.ctrl = reinterpret_cast<Ctrl*>(ws + o_ctrl);
  return launch_router(ra, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
