// kernels.h -- host-side launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "moe_layer.h"

namespace moe {

struct Ctrl;

// tokens per block of the histogram / permutation kernels
constexpr int kTokBlock = 256;
// rows of weights per tcgen05 tile (MMA M) and reduction elements per pipeline stage
constexpr int kTileM = 128;
constexpr int kTileK = 64;
// tokens per tcgen05 tile of the gate/up GEMM (MMA N upper bound): 16 when experts hold a
// few tokens each (decode), 128 otherwise
inline int choose_tile_n(int64_t T, int k, int E) {
  return (T * k <= static_cast<int64_t>(6) * E) ? 16 : 128;
}
// tokens per tile of the down GEMM: as gate/up, but 256 when experts hold 256 or more on
// average (long prefill: a third less operand traffic per MMA cycle; its accumulators stay
// double-buffered in tensor memory, unlike gate/up's pair of 256-column ones)
inline int choose_tile_n_down(int64_t T, int k, int E) {
  const int bn = choose_tile_n(T, k, E);
  return (bn == 128 && T * k >= static_cast<int64_t>(256) * E) ? 256 : bn;
}
// long prefill (256 or more tokens per expert on average) with bf16 weights whose sizes are
// multiples of 256: both GEMMs use 256 x 256 tiles over pairs of SMs
inline bool choose_pair(int64_t T, int k, int E, int H, int I, int Is) {
  return T * k >= static_cast<int64_t>(256) * E && H % 256 == 0 && I % 256 == 0 && Is % 256 == 0;
}

struct RouterArgs {
  bool bf16;
  int64_t T;
  int H, E, k;
  const void* x;
  const void* Wr;
  const float* bias;
  int sigmoid;       // 0: softmax router; 1: sigmoid router (bias for the selection only)
  float scale;       // sigmoid router: routed scaling factor of the weights
  double* scores64;  // [T, E], zero before the forward on the small-batch path
  double* wss;       // [router_group_counters(T), E] zero before the forward
  double* xnorm;     // [T]
  double* wnorm;     // [E]
  unsigned int* group_done;  // [router_group_counters(T)], zero before the forward
  int32_t* idx_ws;   // [T, k]
  float* w_ws;       // [T, k]
  int32_t* idx_user;
  float* w_user;
  float* spill;      // [5, T, E] key state of tokens that need exact dots
  void* rsplit;      // router_split_bytes(shape) bytes, or null: the reduction is not split
  bool w32;          // bf16 tokens with fp32 router weights (Wr is float [E, H])
  void* w3;          // router_w3_bytes(shape): the fp32 weights split into 3 bf16 parts
  Ctrl* ctrl;
};
cudaError_t launch_router(const RouterArgs& a, cudaStream_t st);
// counters of the router kernels, zero before the forward
int64_t router_group_counters(int64_t T, int E);
// scratch of the reduction-split tensor-core router (0 when a batch fills the GPU unsplit)
size_t router_split_bytes(const moe_layer_shape& s);
// the bf16 split of fp32 router weights for the tensor-core router (0 when it is not used)
size_t router_w3_bytes(const moe_layer_shape& s);
// whether fp32 router weights can be used with this shape (bf16 tokens, tensor-core router)
bool router_w32_supported(const moe_layer_shape& s);
// whether the router scores of this shape come from the tensor cores (else fp64)
bool router_scores_f32(const moe_layer_shape& s);
// products per fp32-accumulated slice of the tensor-core router scores
int router_slice_len(int H);

struct DispatchArgs {
  bool bf16;
  int64_t T;
  int H, E, k;
  int I, Is;        // expert widths (Is = 0: no shared expert)
  bool pair_dn;     // down GEMM on 256-row x 256-token tiles over pairs of SMs
  int bn;           // tokens per gate/up GEMM tile
  int bn_dn;        // tokens per down GEMM tile
  int ksplit;       // gate/up reduction slices
  int e_lo, e_hi;   // routed experts whose rows are computed: [0, E), or one rank's range
  int shared_rows;  // rows of the shared-expert group (T, or one rank's token slice)
  bool need_x_perm; // the GEMMs read a permuted copy of x (fp32; FP8 weights with 128-token tiles)
  const void* x;
  const int32_t* idx;   // [T, k]
  const float* w;       // [T, k]
  int32_t* blk_hist;    // [nblk, E]
  int32_t* counts;      // [E]
  int32_t* offsets;     // [E + 1]
  int32_t* group_order;     // [G]   groups sorted by row count, descending
  int32_t* item_start_gu;   // [G+1] tcgen05 tiles of the gate/up GEMM per group (prefix)
  int32_t* item_start_dn;   // [G+1] tiles of the down GEMM
  int4* info_gu;            // [cap_gu] one descriptor per gate/up tile, in schedule order
  int4* info_dn;            // [cap_dn] the same for the down GEMM
  int cap_gu, cap_dn;
  int32_t* perm;        // [T*k]
  int32_t* inv_perm;    // [T*k]
  float* row_w;         // [T*k]
  int32_t* row_tok;     // [T*k]
  void* x_perm;         // [T*k, H]
  int32_t* counts_user;
  int32_t* offsets_user;
  int32_t* perm_user;
  Ctrl* ctrl;
};
cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t st);

struct ExpertArgs {
  bool bf16;
  int64_t T;
  int H, E, k, I, Is;
  int e_lo, e_hi;          // routed experts whose weights Wgu / Wd hold: [e_lo, e_hi)
  int64_t shared_base;     // token rows [shared_base, shared_base + shared_rows) get the
  int64_t shared_rows;     // shared expert (all T rows without expert parallelism)
  const void* x;
  const void* Wgu;   // [E, 2I, H]
  const void* Wd;    // [E, H, I]
  const void* Wsgu;  // [2Is, H] or null
  const void* Wsd;   // [H, Is]
  bool w8;           // the four weight matrices are FP8 E4M3 codes with E8M0 block scales
  const void* Wgu_scale;   // FP8: [E, 2I/128, H/128]
  const void* Wd_scale;    // FP8: [E, H/128, I/128]
  const void* Wsgu_scale;  // FP8: [2Is/128, H/128]
  const void* Wsd_scale;   // FP8: [H/128, Is/128]
  const int32_t* offsets;
  const int32_t* group_order;
  const int32_t* item_start_gu;
  const int32_t* item_start_dn;
  const int4* info_gu;
  const int4* info_dn;
  const float* row_w;
  const int32_t* row_tok;  // [T*k] token of each routed row (bf16: gathered from x)
  const void* x_perm;      // fp32 path: routed rows of x in expert order
  bool pair_dn;     // long prefill: down on 256-row x 256-token tiles over pairs of SMs
  int bn;           // tokens per gate/up GEMM tile (16 or 128)
  int bn_dn;        // tokens per down GEMM tile (16, 128 or 256)
  int ksplit;       // gate/up reduction slices (1, 2 or 4)
  float* partial;   // split partial sums (ksplit > 1)
  unsigned int* tile_done;  // per-tile slice counters, zero before the forward
  unsigned int* item_counters;  // [2] dynamic item claims of the two GEMMs, zero before the forward
  unsigned int* gu_done;   // [E + 1] gate/up tiles finished per group, zero before the forward
  const int32_t* counts;   // [E] rows per routed expert
  float swiglu_limit;          // routed experts: gate <= L, up in [-L, L] before SiLU*up (0: none)
  float swiglu_limit_shared;   // the same for the shared expert
  void* h;          // [T*k, I]
  void* h_shared;   // [T, Is]
  void* o;          // [T*k, H]
  void* o_shared;   // [T, H]
  int num_sms;
  Ctrl* ctrl;
  void (*stage_mark)(void* ctx, int stage, cudaStream_t st) = nullptr;  // between the GEMMs
  void* stage_mark_ctx = nullptr;
};
cudaError_t launch_experts(const ExpertArgs& a, cudaStream_t st);
int64_t expert_tile_bound(int64_t T, int k, int E, int rows, int rows_shared, int bn);

// reduction slices of the gate/up GEMM: split when a 16-token tiling leaves fewer than
// about six tiles per SM of a 148-SM B200 (small decode batches)
inline int choose_ksplit(int64_t T, int k, int E, int I, int Is, int bn) {
  if (bn != 16) return 1;
  const int64_t touched = std::min<int64_t>(static_cast<int64_t>(T) * k, E);
  const int64_t tiles = touched * (I / kTileM) + (Is ? ((T + 15) / 16) * (Is / kTileM) : 0);
  for (int ks = 1; ks < 4; ks *= 2)
    if (tiles * ks >= 6 * 148) return ks;
  return 4;
}

struct CombineArgs {
  bool bf16;
  int64_t T;
  int H, k;
  bool has_shared;
  const int32_t* inv_perm;
  const void* o;
  const void* o_shared;
  void* y;
  Ctrl* ctrl;
  // expert parallelism: when y_partial is set, the fp32 share of the experts [e_lo, e_hi)
  // and of the shared expert on token rows [shared_lo, shared_hi) is written there instead
  float* y_partial = nullptr;
  const int32_t* offsets = nullptr;
  int e_lo = 0, e_hi = 0;
  int64_t shared_lo = 0, shared_hi = 0;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);

// the most partial outputs that moe_layer_sum_partials adds in one call
constexpr int kMaxParts = 16;
// y = sum of n fp32 buffers of `count` elements (count a multiple of 4), in order, as bf16 or fp32
cudaError_t launch_sum_partials(const float* const* parts, int n, int64_t count, bool bf16, void* y,
                                cudaStream_t st);

// adds n to the process-wide count of kernels launched by this library
void count_launches(int n);

// resolves cuTensorMapEncodeTiled through the runtime's driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace moe
