// api.cu -- the C ABI declared in include/moe_layer.h: validation, workspace carving and
// the kernel sequence of one forward pass:
//   router scores + certified top-k + softmax  (router.cu)
//   histogram, scan, permutation, row gather    (dispatch.cu)
//   grouped gate/up GEMM + SiLU*up, grouped down GEMM + routing weight  (experts.cu)
//   unpermute-combine                           (combine.cu)
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <float.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "moe_layer.h"

namespace moe {

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

static std::atomic<long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// ------------------------------ stage timing --------------------------------------------
constexpr int kStages = 5;
struct Profiler {
  std::mutex mu;
  bool enabled = false;
  std::vector<cudaEvent_t> pool;      // free events
  std::vector<cudaEvent_t> recorded;  // (kStages + 1) per forward call
};
static Profiler& profiler() {
  static Profiler p;
  return p;
}
static cudaEvent_t take_event(Profiler& p) {
  if (!p.pool.empty()) {
    cudaEvent_t e = p.pool.back();
    p.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
struct StageMarks {
  cudaEvent_t ev[kStages + 1] = {};
  bool on = false;
  void mark(int i, cudaStream_t st) {
    if (on && ev[i]) cudaEventRecord(ev[i], st);
  }
};
static void begin_marks(StageMarks& m) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.enabled) return;
  m.on = true;
  for (int i = 0; i <= kStages; ++i) m.ev[i] = take_event(p);
}
static void end_marks(StageMarks& m) {
  if (!m.on) return;
  Profiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  for (int i = 0; i <= kStages; ++i) p.recorded.push_back(m.ev[i]);
}

static int num_sms_current_device() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

static size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct Layout {
  size_t ctrl, group_done, tile_done, item_counters, gu_done, wss, zero_end, scores, xnorm, wnorm, idx, w, blk_hist, counts,
      offsets, group_order, item_start_gu, item_start_dn, info_gu, info_dn, perm, inv_perm, row_w, row_tok, partial, spill, rsplit, w3,
      x_perm, h, h_shared, o, o_shared, total;
  int bn, bn_dn, ksplit;
  int64_t max_tiles, cap_gu, cap_dn;
};

static bool make_layout(const moe_layer_shape* s, Layout& L) {
  const size_t T = static_cast<size_t>(s->T), H = s->H, E = s->E, k = s->top_k, I = s->I,
               Is = s->I_shared;
  const size_t es = s->dtype == MOE_BF16 ? 2 : 4;
  const size_t P = T * k;
  const size_t nblk = (T + kTokBlock - 1) / kTokBlock;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.bn = choose_tile_n(s->T, s->top_k, s->E);
  L.bn_dn = choose_tile_n_down(s->T, s->top_k, s->E);
  L.ksplit = s->dtype == MOE_BF16 ? choose_ksplit(s->T, s->top_k, s->E, s->I, s->I_shared, L.bn) : 1;
  // every slice of the reduction keeps at least one 64-column k-block (H = 128 has two)
  while (L.ksplit > 1 && L.ksplit > s->H / kTileK) L.ksplit /= 2;
  L.max_tiles = expert_tile_bound(s->T, s->top_k, s->E, s->I, s->I_shared, L.bn);
  // control block and counters first: one memset per forward clears them
  const bool tc_scores = router_scores_f32(*s);
  const size_t groups = static_cast<size_t>(router_group_counters(s->T, s->E));
  L.ctrl = take(sizeof(Ctrl));
  L.group_done = take(groups * 4);
  L.tile_done = take(L.ksplit > 1 ? static_cast<size_t>(L.max_tiles) * 4 : 0);
  L.item_counters = take(2 * 4);
  L.gu_done = take((E + 1) * 4);  // gate/up tiles finished per group (one launch for both GEMMs)
  // the small-batch router accumulates scores and row sums of squares atomically
  L.wss = take(tc_scores ? 0 : groups * E * 8);
  L.scores = take(T * E * 8);
  L.zero_end = tc_scores ? L.scores : off;
  L.spill = take(T * E * 20);
  L.rsplit = take(router_split_bytes(*s));
  L.w3 = take(router_w3_bytes(*s));
  L.xnorm = take(T * 8);
  L.wnorm = take(E * 8);
  L.idx = take(P * 4);
  L.w = take(P * 4);
  L.blk_hist = take((nblk ? nblk : 1) * E * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.group_order = take((E + 1) * 4);
  L.item_start_gu = take((E + 2) * 4);
  L.item_start_dn = take((E + 2) * 4);
  // tile descriptors: room for the longest schedules (128-row tiles; the down GEMM's
  // narrowest token tiles, which FP8 weights use)
  L.cap_gu = L.max_tiles * L.ksplit;
  L.cap_dn = expert_tile_bound(s->T, s->top_k, s->E, s->H, Is ? s->H : 0, std::min(L.bn_dn, 128));
  L.info_gu = take(static_cast<size_t>(L.cap_gu) * 16);
  L.info_dn = take(static_cast<size_t>(L.cap_dn) * 16);
  L.perm = take(P * 4);
  L.inv_perm = take(P * 4);
  L.row_w = take(P * 4);
  L.row_tok = take(P * 4);
  L.partial = take(L.ksplit > 1 ? static_cast<size_t>(L.max_tiles) * L.ksplit * L.bn * 256 * 4 : 0);
  // bf16 GEMMs gather their token rows from x; fp32, and FP8 weights with 128-token tiles,
  // read a permuted copy (the workspace size does not depend on the weight format)
  L.x_perm = take(s->dtype == MOE_BF16 && L.bn == 16 ? 0 : P * H * es);
  L.h = take(P * I * es);
  L.h_shared = take(T * Is * es);
  L.o = take(P * H * es);
  L.o_shared = take(Is ? T * H * es : 0);
  L.total = off;
  return true;
}

static moe_status validate_shape(const moe_layer_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->dtype != MOE_F32 && s->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H < 1 || s->E < 1 || s->I < 1 || s->I_shared < 0) return MOE_ERR_INVALID_ARG;
  if (s->top_k < 1 || s->top_k > s->E) return MOE_ERR_INVALID_ARG;
  if (s->H > (1 << 20)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->E > 1024) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->T * static_cast<int64_t>(s->top_k) >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(s->E) * 2 * s->I >= (int64_t(1) << 31) ||
      static_cast<int64_t>(s->E) * s->H >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->dtype == MOE_BF16) {
    if (s->H % kTileM || s->I % kTileM || s->I_shared % kTileM) return MOE_ERR_UNSUPPORTED_SHAPE;
  } else {
    if (s->H % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  return MOE_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace moe

using namespace moe;

extern "C" size_t moe_layer_workspace_bytes(const moe_layer_shape* shape) {
  if (validate_shape(shape) != MOE_OK) return 0;
  Layout L;
  make_layout(shape, L);
  return L.total;
}

extern "C" moe_status moe_layer_workspace_layout(const moe_layer_shape* shape,
                                                 moe_workspace_layout* out) {
  if (!out || validate_shape(shape) != MOE_OK) return MOE_ERR_INVALID_ARG;
  Layout L;
  make_layout(shape, L);
  out->x_perm = L.x_perm;
  out->h = L.h;
  out->h_shared = L.h_shared;
  out->o = L.o;
  out->o_shared = L.o_shared;
  out->row_w = L.row_w;
  out->scores = L.scores;
  // fp32 slices on the tensor-core router; fp64 sums on the CUDA-core router
  out->scores_slice = router_scores_f32(*shape) ? router_slice_len(shape->H) : 0;
  return MOE_OK;
}

extern "C" moe_status moe_layer_forward(const moe_layer_shape* shape, const void* x,
                                        const void* W_router, const float* router_bias,
                                        const void* W_gate_up, const void* W_down,
                                        const void* Ws_gate_up, const void* Ws_down, void* y,
                                        moe_routing_out* routing, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  return moe_layer_forward_ex(shape, x, W_router, router_bias, W_gate_up, W_down, Ws_gate_up, Ws_down,
                              y, routing, nullptr, workspace, workspace_bytes, stream);
}

namespace moe {

// The four expert weight matrices: bf16/fp32 in the layer's dtype, or FP8 codes with their
// block scales.
struct ExpertWeights {
  const void* Wgu;
  const void* Wd;
  const void* Wsgu;
  const void* Wsd;
  bool w8;
  const void* scale[4];  // FP8: of Wgu, Wd, Wsgu, Wsd
};

// ep = nullptr: the whole layer into y.  Otherwise (expert parallelism) the weights hold the
// routed experts [ep->expert_begin, ep->expert_end) only, and this rank's fp32 share of the
// output goes to y_partial (y is not used).
static moe_status forward_impl(const moe_layer_shape* shape, const void* x, const void* W_router,
                               const float* router_bias, const ExpertWeights& wt, void* y,
                               moe_routing_out* routing, const moe_layer_options* options,
                               void* workspace, size_t workspace_bytes, void* stream,
                               const moe_ep_range* ep = nullptr, float* y_partial = nullptr) {
  const void* W_gate_up = wt.Wgu;
  const void* W_down = wt.Wd;
  const void* Ws_gate_up = wt.Wsgu;
  const void* Ws_down = wt.Wsd;
  const moe_layer_options opt = options ? *options : moe_layer_options{0.0f, 0.0f, MOE_ROUTER_SOFTMAX, 0.0f, 0};
  if (!(opt.swiglu_limit >= 0.0f && opt.swiglu_limit <= FLT_MAX) ||
      !(opt.swiglu_limit_shared >= 0.0f && opt.swiglu_limit_shared <= FLT_MAX) ||
      !(opt.routed_scaling_factor >= 0.0f && opt.routed_scaling_factor <= FLT_MAX))
    return MOE_ERR_INVALID_ARG;  // negative, infinite or NaN
  if (opt.router != MOE_ROUTER_SOFTMAX && opt.router != MOE_ROUTER_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (opt.router_weights_fp32 != 0 && opt.router_weights_fp32 != 1) return MOE_ERR_INVALID_ARG;
  const moe_status vs = validate_shape(shape);
  if (vs != MOE_OK) return vs;
  const moe_layer_shape& s = *shape;
  // fp32 router weights with bf16 tokens run on the tensor-core router only
  if (opt.router_weights_fp32 && s.dtype == MOE_BF16 && !router_w32_supported(s)) return MOE_ERR_UNSUPPORTED_SHAPE;
  int e_lo = 0, e_hi = s.E;
  int64_t sh_lo = 0, sh_hi = s.T;
  if (ep) {
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED_SHAPE;
    e_lo = ep->expert_begin;
    e_hi = ep->expert_end;
    sh_lo = ep->shared_begin;
    sh_hi = ep->shared_end;
    if (e_lo < 0 || e_hi > s.E || e_lo >= e_hi || sh_lo < 0 || sh_hi > s.T || sh_lo > sh_hi)
      return MOE_ERR_INVALID_ARG;
  }
  if (s.T == 0) return MOE_OK;  // empty batch: nothing to read or write
  if (!x || !W_router || !W_gate_up || !W_down || !workspace) return MOE_ERR_INVALID_ARG;
  if (ep ? (!y_partial || !aligned16(y_partial)) : !y) return MOE_ERR_INVALID_ARG;
  const bool has_shared = s.I_shared > 0;
  if (has_shared != (Ws_gate_up != nullptr) || has_shared != (Ws_down != nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_router) || !aligned16(W_gate_up) || !aligned16(W_down) ||
      (!ep && !aligned16(y)) || (has_shared && (!aligned16(Ws_gate_up) || !aligned16(Ws_down))) ||
      (reinterpret_cast<uintptr_t>(router_bias) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return MOE_ERR_INVALID_ARG;
  if (wt.w8 && (!wt.scale[0] || !wt.scale[1] || (has_shared && (!wt.scale[2] || !wt.scale[3]))))
    return MOE_ERR_INVALID_ARG;
  Layout L;
  make_layout(shape, L);
  if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  // FP8 weights run on 16- and 128-token tiles only
  const int bn_dn = wt.w8 ? std::min(L.bn_dn, 128) : L.bn_dn;
  // long prefill: the down projection on 256-row x 256-token tiles over pairs of SMs (the
  // gate/up GEMM stays on one SM a tile, where its gather warps read the token rows from x)
  const bool pair = s.dtype == MOE_BF16 && !wt.w8 && L.ksplit == 1 &&
                    choose_pair(s.T, s.top_k, s.E, s.H, s.I, s.I_shared);
  const bool pair_dn = pair;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
  Ctrl* ctrl = static_cast<Ctrl*>(at(L.ctrl));
  const bool bf16 = s.dtype == MOE_BF16;
  const int64_t P = s.T * s.top_k;
  (void)P;

  if (cudaMemsetAsync(ctrl, 0, L.zero_end, st) != cudaSuccess) return MOE_ERR_CUDA;
  StageMarks marks;
  begin_marks(marks);
  struct EndMarks {
    StageMarks& m;
    ~EndMarks() { end_marks(m); }
  } end_guard{marks};
  marks.mark(0, st);

  RouterArgs ra{};
  ra.bf16 = bf16;
  ra.T = s.T;
  ra.H = s.H;
  ra.E = s.E;
  ra.k = s.top_k;
  ra.x = x;
  ra.Wr = W_router;
  ra.bias = router_bias;
  ra.scores64 = static_cast<double*>(at(L.scores));
  ra.wss = static_cast<double*>(at(L.wss));
  ra.spill = static_cast<float*>(at(L.spill));
  ra.sigmoid = opt.router == MOE_ROUTER_SIGMOID ? 1 : 0;
  ra.w32 = bf16 && opt.router_weights_fp32;
  ra.w3 = at(L.w3);
  ra.scale = opt.routed_scaling_factor > 0.0f ? opt.routed_scaling_factor : 1.0f;
  ra.rsplit = router_split_bytes(*shape) ? at(L.rsplit) : nullptr;
  ra.xnorm = static_cast<double*>(at(L.xnorm));
  ra.wnorm = static_cast<double*>(at(L.wnorm));
  ra.group_done = static_cast<unsigned int*>(at(L.group_done));
  ra.idx_ws = static_cast<int32_t*>(at(L.idx));
  ra.w_ws = static_cast<float*>(at(L.w));
  ra.idx_user = routing ? routing->topk_idx : nullptr;
  ra.w_user = routing ? routing->topk_w : nullptr;
  ra.ctrl = ctrl;

  DispatchArgs da{};
  da.bf16 = bf16;
  da.T = s.T;
  da.H = s.H;
  da.E = s.E;
  da.k = s.top_k;
  da.I = s.I;
  da.Is = s.I_shared;
  da.bn = L.bn;
  da.bn_dn = bn_dn;
  da.ksplit = L.ksplit;
  da.pair_dn = pair_dn;
  da.e_lo = e_lo;
  da.e_hi = e_hi;
  da.shared_rows = static_cast<int>(sh_hi - sh_lo);
  da.need_x_perm = !bf16 || (wt.w8 && L.bn == 128);
  da.x = x;
  da.idx = ra.idx_ws;
  da.w = ra.w_ws;
  da.blk_hist = static_cast<int32_t*>(at(L.blk_hist));
  da.counts = static_cast<int32_t*>(at(L.counts));
  da.offsets = static_cast<int32_t*>(at(L.offsets));
  da.group_order = static_cast<int32_t*>(at(L.group_order));
  da.item_start_gu = static_cast<int32_t*>(at(L.item_start_gu));
  da.item_start_dn = static_cast<int32_t*>(at(L.item_start_dn));
  da.info_gu = static_cast<int4*>(at(L.info_gu));
  da.info_dn = static_cast<int4*>(at(L.info_dn));
  da.cap_gu = static_cast<int>(L.cap_gu);
  da.cap_dn = static_cast<int>(L.cap_dn);
  da.perm = static_cast<int32_t*>(at(L.perm));
  da.inv_perm = static_cast<int32_t*>(at(L.inv_perm));
  da.row_w = static_cast<float*>(at(L.row_w));
  da.row_tok = static_cast<int32_t*>(at(L.row_tok));
  da.x_perm = at(L.x_perm);
  da.counts_user = routing ? routing->counts : nullptr;
  da.offsets_user = routing ? routing->offsets : nullptr;
  da.perm_user = routing ? routing->perm : nullptr;
  da.ctrl = ctrl;
  if (launch_router(ra, st) != cudaSuccess) return MOE_ERR_CUDA;
  marks.mark(1, st);
  if (launch_dispatch(da, st) != cudaSuccess) return MOE_ERR_CUDA;
  marks.mark(2, st);

  ExpertArgs ea{};
  ea.bf16 = bf16;
  ea.T = s.T;
  ea.H = s.H;
  ea.E = s.E;
  ea.k = s.top_k;
  ea.I = s.I;
  ea.Is = s.I_shared;
  ea.e_lo = e_lo;
  ea.e_hi = e_hi;
  ea.shared_base = sh_lo;
  ea.shared_rows = sh_hi - sh_lo;
  ea.x = x;
  ea.Wgu = W_gate_up;
  ea.Wd = W_down;
  ea.Wsgu = Ws_gate_up;
  ea.Wsd = Ws_down;
  ea.w8 = wt.w8;
  ea.Wgu_scale = wt.scale[0];
  ea.Wd_scale = wt.scale[1];
  ea.Wsgu_scale = wt.scale[2];
  ea.Wsd_scale = wt.scale[3];
  ea.offsets = da.offsets;
  ea.group_order = da.group_order;
  ea.item_start_gu = da.item_start_gu;
  ea.item_start_dn = da.item_start_dn;
  ea.info_gu = da.info_gu;
  ea.info_dn = da.info_dn;
  ea.row_w = da.row_w;
  ea.x_perm = da.x_perm;
  ea.row_tok = da.row_tok;
  ea.pair_dn = pair_dn;
  ea.bn = L.bn;
  ea.bn_dn = bn_dn;
  ea.ksplit = L.ksplit;
  ea.partial = static_cast<float*>(at(L.partial));
  ea.tile_done = static_cast<unsigned int*>(at(L.tile_done));
  ea.swiglu_limit = opt.swiglu_limit;
  ea.swiglu_limit_shared = opt.swiglu_limit_shared;
  ea.item_counters = static_cast<unsigned int*>(at(L.item_counters));
  ea.gu_done = static_cast<unsigned int*>(at(L.gu_done));
  ea.counts = static_cast<const int32_t*>(at(L.counts));
  ea.h = at(L.h);
  ea.h_shared = at(L.h_shared);
  ea.o = at(L.o);
  ea.o_shared = at(L.o_shared);
  ea.num_sms = num_sms_current_device();
  ea.ctrl = ctrl;
  ea.stage_mark = [](void* m, int i, cudaStream_t s2) { static_cast<StageMarks*>(m)->mark(i, s2); };
  ea.stage_mark_ctx = &marks;
  if (launch_experts(ea, st) != cudaSuccess) return MOE_ERR_CUDA;
  marks.mark(4, st);

  CombineArgs ca{};
  ca.bf16 = bf16;
  ca.T = s.T;
  ca.H = s.H;
  ca.k = s.top_k;
  ca.has_shared = has_shared;
  ca.inv_perm = da.inv_perm;
  ca.o = ea.o;
  ca.o_shared = ea.o_shared;
  ca.y = y;
  ca.ctrl = ctrl;
  if (ep) {
    ca.y_partial = y_partial;
    ca.offsets = da.offsets;
    ca.e_lo = e_lo;
    ca.e_hi = e_hi;
    ca.shared_lo = sh_lo;
    ca.shared_hi = sh_hi;
  }
  if (launch_combine(ca, st) != cudaSuccess) return MOE_ERR_CUDA;
  marks.mark(5, st);
  return MOE_OK;
}

}  // namespace moe

extern "C" moe_status moe_layer_forward_ex(const moe_layer_shape* shape, const void* x,
                                           const void* W_router, const float* router_bias,
                                           const void* W_gate_up, const void* W_down,
                                           const void* Ws_gate_up, const void* Ws_down, void* y,
                                           moe_routing_out* routing, const moe_layer_options* options,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  const ExpertWeights wt{W_gate_up, W_down, Ws_gate_up, Ws_down, false, {nullptr, nullptr, nullptr, nullptr}};
  return forward_impl(shape, x, W_router, router_bias, wt, y, routing, options, workspace, workspace_bytes,
                      stream);
}

extern "C" moe_status moe_layer_forward_fp8(const moe_layer_shape* shape, const void* x,
                                            const void* W_router, const float* router_bias,
                                            const moe_fp8_weights* weights, void* y,
                                            moe_routing_out* routing, const moe_layer_options* options,
                                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape || !weights) return MOE_ERR_INVALID_ARG;
  const moe_layer_shape& s = *shape;
  if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED_SHAPE;
  // the GEMM producer keeps one item's block scales in two registers per lane: at most
  // 64 scale blocks (8192 columns) along a reduction
  if (s.H > 8192 || s.I > 8192 || s.I_shared > 8192 || s.H % 128 || s.I % 128 || s.I_shared % 128)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const moe_fp8_weights& w = *weights;
  const ExpertWeights wt{w.W_gate_up, w.W_down, w.Ws_gate_up, w.Ws_down, true,
                         {w.W_gate_up_scale, w.W_down_scale, w.Ws_gate_up_scale, w.Ws_down_scale}};
  return forward_impl(shape, x, W_router, router_bias, wt, y, routing, options, workspace, workspace_bytes,
                      stream);
}

extern "C" moe_status moe_layer_forward_ep(const moe_layer_shape* shape, const void* x,
                                           const void* W_router, const float* router_bias,
                                           const void* W_gate_up, const void* W_down,
                                           const void* Ws_gate_up, const void* Ws_down,
                                           const moe_ep_range* range, float* y_partial,
                                           moe_routing_out* routing, const moe_layer_options* options,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!range) return MOE_ERR_INVALID_ARG;
  const ExpertWeights wt{W_gate_up, W_down, Ws_gate_up, Ws_down, false, {nullptr, nullptr, nullptr, nullptr}};
  return forward_impl(shape, x, W_router, router_bias, wt, nullptr, routing, options, workspace, workspace_bytes,
                      stream, range, y_partial);
}

extern "C" moe_status moe_layer_sum_partials(int64_t T, int32_t H, int32_t dtype, int32_t n_parts,
                                             const float* const* parts, void* y, void* stream) {
  if (T < 0 || H < 1 || H % 8 || (dtype != MOE_F32 && dtype != MOE_BF16)) return MOE_ERR_INVALID_ARG;
  if (n_parts < 1 || n_parts > kMaxParts || !parts) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  for (int r = 0; r < n_parts; ++r)
    if (!parts[r] || !aligned16(parts[r])) return MOE_ERR_INVALID_ARG;
  return launch_sum_partials(parts, n_parts, T * static_cast<int64_t>(H), dtype == MOE_BF16, y,
                             static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

extern "C" moe_status moe_layer_check_status(void* workspace, void* stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, &static_cast<Ctrl*>(workspace)->status, sizeof(int),
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  return static_cast<moe_status>(status);
}

extern "C" moe_status moe_layer_route_stats(void* workspace, moe_route_stats* out, void* stream) {
  if (!workspace || !out) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  Ctrl c;
  if (cudaMemcpy(&c, workspace, sizeof(Ctrl), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  out->n_refined = static_cast<int64_t>(c.n_refined);
  out->n_exact = static_cast<int64_t>(c.n_exact);
  out->n_tokens_refined = static_cast<int64_t>(c.n_tokens_refined);
  out->n_weight_keys = static_cast<int64_t>(c.n_weight_keys);
  return MOE_OK;
}

extern "C" moe_status moe_layer_profile_enable(int enable) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  p.enabled = enable != 0;
  return MOE_OK;
}

extern "C" int moe_layer_profile_read(float* ms, int n_stages) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  const int calls = static_cast<int>(p.recorded.size() / (kStages + 1));
  int rc = calls;
  for (int c = 0; c < calls; ++c) {
    cudaEvent_t* ev = &p.recorded[static_cast<size_t>(c) * (kStages + 1)];
    if (cudaEventSynchronize(ev[kStages]) != cudaSuccess) rc = -1;
    for (int i = 0; i < kStages && i < n_stages; ++i) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, ev[i], ev[i + 1]) != cudaSuccess) rc = -1;
      if (ms) ms[i] += t;
    }
  }
  for (cudaEvent_t e : p.recorded) p.pool.push_back(e);
  p.recorded.clear();
  return rc;
}

extern "C" int64_t moe_layer_launch_count(void) { return g_launches.load(); }

extern "C" const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE: unsupported layer shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL: workspace too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a device-side wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS: a device-side index check failed";
  }
  return "unknown moe_status";
}
