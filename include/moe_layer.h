/*
 * moe_layer.h -- C ABI of the B200 (sm_100a) routed-expert MoE FFN layer of Step-3.5-Flash.
 *
 * The layer (llm-atlas page "Step-3.5-Flash", table "Champs bruts du config.json":
 * moe_num_experts 288, moe_top_k 8, norm_expert_weight true, need_fp32_gate true,
 * moe_intermediate_size 1280, share_expert_dim 1280, hidden_size 4096; and the page's
 * "FFN / MoE" paragraph: a sparse mixture of 288 routed experts with top-8 routing):
 *
 *   s[t,e]   = sum_h x[t,h] * W_router[e,h]      exact sum, rounded once to fp32
 *   key[t,e] = fp32(s[t,e] + router_bias[e])     (router_bias optional)
 *   S_t      = the top_k experts by (key descending, expert index ascending)
 *   w[t,j]   = softmax of the keys over S_t      (renormalised: sums to 1)
 *   y_t      = sum_{e in S_t} w * (SiLU(x_t Wg_e^T) * (x_t Wu_e^T)) Wd_e^T
 *            + (SiLU(x_t Wsg^T) * (x_t Wsu^T)) Wsd^T      (shared expert, weight 1)
 *
 * The pages leave the score function and the activation open: this library uses a
 * softmax router and SiLU(gate)*up.  Routing is decided on the exact fp32 score, so the
 * chosen experts do not depend on summation order.
 *
 * Conventions for every entry point:
 *   - all tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous, 16-byte aligned; the library never allocates or frees device memory;
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream);
 *     work is enqueued asynchronously and the call returns without synchronising;
 *   - the return value reports argument validation and launch errors only; errors found
 *     on the device (a bounded wait that timed out) are written to a status word in the
 *     workspace and read back by moe_layer_check_status();
 *   - inputs must be finite; NaN/Inf give an unspecified result but never a hang;
 *   - y must not alias any input; the workspace must not be shared by calls that may
 *     run concurrently.
 */
#ifndef MOE_LAYER_H
#define MOE_LAYER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null pointer, bad top_k, misaligned pointer, ... */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* sizes outside what the kernels tile (see below) */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < moe_layer_workspace_bytes() */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime/driver call or launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait gave up */
  MOE_ERR_DEVICE_BOUNDS = 6        /* a device-side index check failed */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Layer sizes.  T tokens, hidden size H, E routed experts, expert width I, shared
 * expert width I_shared (0 = no shared expert), top_k experts per token.
 * Supported: T >= 0 (T = 0 is a no-op), 1 <= top_k <= E <= 1024, T*top_k < 2^31.
 *   MOE_BF16: H, I and I_shared (if nonzero) multiples of 128.
 *   MOE_F32 : H a multiple of 8; I, I_shared >= 1.                                  */
typedef struct {
  int64_t T;
  int32_t H, E, I, I_shared, top_k;
  int32_t dtype; /* moe_dtype */
} moe_layer_shape;

/* Optional routing outputs (any field may be NULL; the struct pointer may be NULL).
 *   topk_idx [T, top_k] int32  chosen experts of each token, ascending expert index
 *   topk_w   [T, top_k] fp32   their renormalised softmax weights (same order)
 *   counts   [E]        int32  number of tokens routed to each expert
 *   offsets  [E + 1]    int32  exclusive prefix sum of counts (offsets[E] = T*top_k)
 *   perm     [T*top_k]  int32  assignments t*top_k + j sorted by (expert, token):
 *                              perm[offsets[e] + r] is the r-th token routed to e     */
typedef struct {
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
} moe_routing_out;

/* Device workspace needed by moe_layer_forward for this shape, in bytes (0 on an
 * invalid shape).  Pure host computation. */
MOE_API size_t moe_layer_workspace_bytes(const moe_layer_shape* shape);

/* Forward pass of the MoE layer.
 *   x          [T, H]          dtype   input tokens
 *   W_router   [E, H]          dtype   router matrix
 *   router_bias[E]             fp32    added to the router scores, or NULL
 *   W_gate_up  [E, 2*I, H]     dtype   per expert: I gate rows, then I up rows
 *   W_down     [E, H, I]       dtype   per expert down projection
 *   Ws_gate_up [2*I_shared, H] dtype   shared expert gate rows then up rows (NULL iff
 *                                      I_shared == 0)
 *   Ws_down    [H, I_shared]   dtype   shared expert down projection
 *   y          [T, H]          dtype   output (written, never read)
 *   routing    optional routing outputs (see moe_routing_out)
 *   workspace  device scratch of at least moe_layer_workspace_bytes(shape) bytes,
 *              256-byte aligned, owned by the caller; its contents need no
 *              initialisation and are overwritten.
 * T = 0 returns MOE_OK at once (pointers are not inspected).
 * Errors: MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_SHAPE / MOE_ERR_WORKSPACE_TOO_SMALL
 * before anything is enqueued; MOE_ERR_CUDA if a launch fails. */
MOE_API moe_status moe_layer_forward(const moe_layer_shape* shape, const void* x, const void* W_router,
                             const float* router_bias, const void* W_gate_up, const void* W_down,
                             const void* Ws_gate_up, const void* Ws_down, void* y,
                             moe_routing_out* routing, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Per-layer options of moe_layer_forward_ex().  All zero = moe_layer_forward().
 *   swiglu_limit, swiglu_limit_shared: the SwiGLU limits of the routed experts and of the
 *   shared expert (llm-atlas page "Step-3.5-Flash", table "Champs bruts du config.json":
 *   swiglu_limits "0.0x46 + 7x2", swiglu_limits_shared "0.0x47 + 16x1"; the page gives
 *   the values only).  A limit L > 0 clamps the activation inputs, gate to <= L and up to
 *   [-L, L], before SiLU(gate)*up; 0 means no clamp.  Limits must be finite and >= 0.
 *   router: MOE_ROUTER_SOFTMAX (0) or MOE_ROUTER_SIGMOID (1), the router as configured on
 *   the same table (moe_router_activation = sigmoid, use_moe_router_bias,
 *   moe_router_scaling_factor = 3): p_e = fp32(1 / (1 + e^-s_e)) of the fp32 logit s_e,
 *   with e^z evaluated by a fixed sequence of fp64 operations (Cody-Waite reduction by a
 *   42-bit ln 2 head and its tail, the degree-13 Taylor polynomial in fused
 *   multiply-adds, scaling by 2^n; p = 0 below s = -110 and 1 above 40); the router bias
 *   only steers the selection (key_e = fp32(p_e + b_e)); the weights are
 *   routed_scaling_factor * p_j / sum of the chosen p (uniform if that sum is 0).
 *   routed_scaling_factor: sigmoid router only; 0 is read as 1; else finite and > 0.
 *   router_weights_fp32: 1 = W_router is fp32 [E, H] while the tokens and experts are bf16
 *   (need_fp32_gate on the same table, read as fp32 router weights).  The scores stay the
 *   exact dot rounded once to fp32; the weights are split into three bf16 parts for the
 *   tensor cores.  Needs E <= 512 and H a multiple of 64 (else MOE_ERR_UNSUPPORTED_SHAPE);
 *   ignored for fp32 layers, whose router is fp32 already. */
enum { MOE_ROUTER_SOFTMAX = 0, MOE_ROUTER_SIGMOID = 1 };
typedef struct {
  float swiglu_limit;
  float swiglu_limit_shared;
  int32_t router;
  float routed_scaling_factor;
  int32_t router_weights_fp32;
} moe_layer_options;

/* moe_layer_forward() with per-layer options; options = NULL is moe_layer_forward().
 * Errors as moe_layer_forward(), plus MOE_ERR_INVALID_ARG for a negative or non-finite
 * limit, an unknown router or a negative or non-finite scaling factor. */
MOE_API moe_status moe_layer_forward_ex(const moe_layer_shape* shape, const void* x,
                                        const void* W_router, const float* router_bias,
                                        const void* W_gate_up, const void* W_down,
                                        const void* Ws_gate_up, const void* Ws_down, void* y,
                                        moe_routing_out* routing, const moe_layer_options* options,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Expert weights in the blockwise FP8 format, for moe_layer_forward_fp8().  Each weight
 * matrix W [R, K] of the layer is given as
 *   codes  [R, K] bytes: FP8 E4M3 (OCP 8-bit floating point: sign, 4 exponent bits with
 *          bias 7, 3 mantissa bits, subnormals at exponent 0, largest finite 448; the two
 *          NaN codes S.1111.111 are outside the contract);
 *   scales [R/128, K/128] bytes: one E8M0 scale per 128 x 128 block (OCP microscaling
 *          formats: the power of two 2^(v - 127)), codes v in [10, 134];
 * and stands for W[r, c] = e4m3(codes[r, c]) * 2^(scales[r/128, c/128] - 127).  Every such
 * value is exact in bf16, so the layer computes exactly what moe_layer_forward() computes
 * on bf16 weights holding the decoded values.  Matrices, as in moe_layer_forward():
 *   W_gate_up  [E, 2*I, H]      scales [E, 2*I/128, H/128]
 *   W_down     [E, H, I]        scales [E, H/128, I/128]
 *   Ws_gate_up [2*I_shared, H]  scales [2*I_shared/128, H/128]   (NULL iff I_shared == 0)
 *   Ws_down    [H, I_shared]    scales [H/128, I_shared/128]     (NULL iff I_shared == 0)
 * Code arrays 16-byte aligned; scale arrays any alignment; all device memory owned by
 * the caller and read only.  This format is the low-precision expert-weight option for
 * decode; the source pages deploy 4-bit weights in a third-party format instead. */
typedef struct {
  const void* W_gate_up;
  const void* W_gate_up_scale;
  const void* W_down;
  const void* W_down_scale;
  const void* Ws_gate_up;
  const void* Ws_gate_up_scale;
  const void* Ws_down;
  const void* Ws_down_scale;
} moe_fp8_weights;

/* moe_layer_forward_ex() with FP8 expert weights (moe_fp8_weights).  The shape's dtype
 * must be MOE_BF16 (x, W_router and y as before); H, I and I_shared must be multiples of
 * 128 and at most 8192.  The workspace is that of moe_layer_workspace_bytes(shape).
 * Errors as moe_layer_forward_ex(), plus MOE_ERR_UNSUPPORTED_SHAPE for another dtype or
 * sizes outside those bounds and MOE_ERR_INVALID_ARG for a missing or misaligned array. */
MOE_API moe_status moe_layer_forward_fp8(const moe_layer_shape* shape, const void* x,
                                         const void* W_router, const float* router_bias,
                                         const moe_fp8_weights* weights, void* y,
                                         moe_routing_out* routing, const moe_layer_options* options,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* Expert parallelism: the layer split over G GPUs (one process per GPU), each holding a
 * contiguous range of the routed experts.  The source pages say only that multi-GPU setups
 * serve the model (q4km.ai model page, hardware section); the split is this library's.
 * Every rank sees the same tokens (for example after an all-gather of the ranks' batches),
 * routes them over all E experts as moe_layer_forward() does, computes the routed experts
 * it holds and, on a range of token rows, the shared expert, and writes its fp32 share:
 *   y_partial[t] = sum_{j: expert_begin <= idx[t,j] < expert_end} w[t,j] FFN_idx[t,j](x_t)
 *                + [shared_begin <= t < shared_end] shared(x_t)
 * The sum of the shares over the ranks (in rank order: moe_layer_sum_partials(), or a
 * reduce-scatter) is the layer's output, when the ranks' expert ranges partition [0, E)
 * and their shared ranges partition [0, T).                                               */
typedef struct {
  int32_t expert_begin;  /* first routed expert held by this rank */
  int32_t expert_end;    /* one past the last; 0 <= begin < end <= E */
  int64_t shared_begin;  /* token rows [shared_begin, shared_end) get the shared expert */
  int64_t shared_end;    /* 0 <= begin <= end <= T (an empty range adds no shared expert) */
} moe_ep_range;

/* One rank's share of the layer (see moe_ep_range).  As moe_layer_forward_ex(), except:
 *   W_gate_up  [expert_end - expert_begin, 2*I, H] bf16: this rank's routed experts only
 *   W_down     [expert_end - expert_begin, H, I]   bf16
 *   y_partial  [T, H] fp32, written (16-byte aligned); there is no y argument
 * x, W_router (all E experts), router_bias, the shared expert's matrices, routing,
 * options and the workspace (moe_layer_workspace_bytes(shape)) are as for
 * moe_layer_forward_ex(); the routing outputs cover all E experts.  The shape's dtype must
 * be MOE_BF16 (else MOE_ERR_UNSUPPORTED_SHAPE); a range outside the bounds above returns
 * MOE_ERR_INVALID_ARG before anything is enqueued. */
MOE_API moe_status moe_layer_forward_ep(const moe_layer_shape* shape, const void* x, const void* W_router,
                                        const float* router_bias, const void* W_gate_up, const void* W_down,
                                        const void* Ws_gate_up, const void* Ws_down, const moe_ep_range* range,
                                        float* y_partial, moe_routing_out* routing,
                                        const moe_layer_options* options, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* y = sum_{r < n_parts} parts[r], the n_parts fp32 [T, H] buffers added element by element
 * in index order (fp32), stored in `dtype` (MOE_BF16 or MOE_F32).  `parts` is a HOST array
 * of n_parts device pointers (1 <= n_parts <= 16), each 16-byte aligned; they may point to
 * other GPUs' memory mapped into this process (peer access over NVLink), so the ranks'
 * shares of moe_layer_forward_ep() can be added where they lie.  H must be a multiple of 8.
 * Used by expert parallelism; no counterpart on the source pages. */
MOE_API moe_status moe_layer_sum_partials(int64_t T, int32_t H, int32_t dtype, int32_t n_parts,
                                          const float* const* parts, void* y, void* stream);

/* Synchronises `stream`, then returns the device status word of the most recent
 * moe_layer_forward() that used this workspace (MOE_OK, MOE_ERR_DEVICE_TIMEOUT or
 * MOE_ERR_DEVICE_BOUNDS), or MOE_ERR_CUDA if the stream itself reports an error. */
MOE_API moe_status moe_layer_check_status(void* workspace, void* stream);

/* Routing diagnostics of the most recent forward on this workspace (synchronises):
 *   n_refined : (token, expert) scores recomputed in fp64 because their fp32 key was not
 *               certain and could change the chosen set;
 *   n_exact   : scores that needed the exact (integer) dot product after that;
 *   n_tokens_refined : tokens that needed any recomputation;
 *   n_weight_keys : keys of chosen experts recomputed in fp64 so that the routing
 *               weights are computed from exact (or 1-ulp) keys.                        */
typedef struct {
  int64_t n_refined;
  int64_t n_exact;
  int64_t n_tokens_refined;
  int64_t n_weight_keys;
} moe_route_stats;
MOE_API moe_status moe_layer_route_stats(void* workspace, moe_route_stats* out, void* stream);

/* Byte offsets of the intermediate buffers inside the workspace (for inspection by
 * tests; layout is private and may change between versions).  Sizes in elements:
 *   x_perm [T*top_k, H] dtype (no bytes when the bf16 GEMMs use 16-token tiles; written only
 *   for fp32 layers and FP8 weights with 128-token tiles: bf16 GEMMs gather their token rows
 *   from x), h [T*top_k, I] dtype, h_shared [T, I_shared] dtype,
 *   o [T*top_k, H] dtype, o_shared [T, H] dtype, row_w [T*top_k] fp32 (routing weight
 *   of each row of x_perm/h/o in expert order), scores: the fp64 router score estimates
 *   before selection.  scores_slice > 0 for tensor-core scoring (bf16): the H products
 *   are accumulated in fp32 over consecutive slices of scores_slice products and the
 *   slices added in fp64; scores_slice = 0 means fp64 accumulation.  Token-major [T, E].
 *   Returns MOE_ERR_INVALID_ARG on a bad shape. */
typedef struct {
  size_t x_perm, h, h_shared, o, o_shared, row_w, scores;
  int32_t scores_slice;
} moe_workspace_layout;
MOE_API moe_status moe_layer_workspace_layout(const moe_layer_shape* shape, moe_workspace_layout* out);

/* Stage timing for benchmarks.  While enabled, every moe_layer_forward() also records
 * CUDA events on its stream at the boundaries of its five stages:
 *   0 routing  (router scores, certified top-k, softmax weights)
 *   1 dispatch (histogram, scan, stable permutation, row gather)
 *   2 gate/up  (grouped GEMM with the SiLU(gate)*up epilogue; with 16-token tiles, bf16
 *              weights, both GEMMs, which then run as one launch)
 *   3 down     (grouped GEMM with the routing-weight epilogue; empty when stage 2 ran both)
 *   4 combine  (unpermute and sum)
 * moe_layer_profile_read() waits for the recorded events, adds each stage's elapsed
 * milliseconds since the previous read into ms[0..n_stages), forgets them and returns
 * the number of forward calls covered (or -1 on a CUDA error).  Process-wide; not meant
 * for concurrent forwards on several threads. */
MOE_API moe_status moe_layer_profile_enable(int enable);
MOE_API int moe_layer_profile_read(float* ms, int n_stages);

/* Number of kernels this library has launched in this process so far. */
MOE_API int64_t moe_layer_launch_count(void);

/* Routing of a batch without a workspace argument, for callers that cannot allocate
 * device memory (a runtime whose memory planner owns every buffer and hands a layer only
 * its inputs and outputs; a host loop that must not call cudaMalloc, which can
 * synchronise the device; a plugin called with tensors but no allocator).  This entry
 * point has no counterpart on the source pages: it is a deployment convenience.
 *
 * Computes what moe_layer_forward() computes for routing -- router scores, the top_k
 * experts of each token (ascending index, same certified selection) and their
 * renormalised softmax weights -- and writes
 *   topk_idx [T, top_k] int32 and topk_w [T, top_k] fp32 (device pointers, caller-owned).
 * x, W_router and router_bias are as for moe_layer_forward() without options: W_router has
 * the shape's dtype (fp32 router weights with bf16 tokens are not accepted here, since
 * nothing tells this call they are fp32), and the router is the softmax router, with
 * router_bias added to the score for both the selection and the weights.  The sigmoid
 * router of moe_layer_forward_ex() is not available through this entry point.  The I and
 * I_shared fields of the shape are not used.
 *
 * Scratch: a 16 MiB device array inside this library (present on every GPU that loads the
 * library, until the process exits).  The call needs about T * (28 * E + 8) bytes of it
 * (plus E / 2 per token for fp32 inputs), so batches of up to about 2000 tokens fit at
 * E = 288.  Larger batches return MOE_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
 * The array is shared by all calls: calls that may overlap on the GPU (several streams or
 * host threads) race and must be serialised by the caller.  Each call clears the part
 * that must start at zero on its stream.
 * The first call on a device looks up the array's device address (once per device, with
 * that device current); make that first call before any stream capture.
 * Returns validation and launch errors; device-side statuses are not reported. */
MOE_API moe_status moe_layer_route_noalloc(const moe_layer_shape* shape, const void* x,
                                           const void* W_router, const float* router_bias,
                                           int32_t* topk_idx, float* topk_w, void* stream);

/* Self-test of the device-side failure detection.  Every wait of the library's kernels
 * gives up after 2 s, records MOE_ERR_DEVICE_TIMEOUT in the workspace's status word and
 * lets its kernel return, so a stalled pipeline ends with an error that
 * moe_layer_check_status() reports instead of a hang.  This call clears the status word of
 * `workspace` (at least 256-byte aligned, >= 64 bytes) and runs one kernel whose wait, the
 * same code, is on a barrier that nothing completes: about 2 s later the status reads
 * MOE_ERR_DEVICE_TIMEOUT and the stream and context remain usable.  No counterpart on the
 * source pages. */
MOE_API moe_status moe_layer_selftest_wait_timeout(void* workspace, size_t workspace_bytes, void* stream);

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_LAYER_H */
