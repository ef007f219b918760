// experts.cu -- grouped expert GEMMs of the MoE layer.
//
// bf16: one persistent, warp-specialised tcgen05 kernel per projection (with 16-token tiles,
// at decode, one launch for both: each down tile starts once its group's gate/up tiles have
// stored their h rows).  Weights are the A operand (128 rows per tile, "swap-AB"), the tokens
// routed to an expert the B operand (16, 128 or 256 per tile), so an expert's few tokens never
// pad a 128-row tile; the long prefill's down GEMM runs 256-row x 256-token tiles over pairs of
// SMs (cta_group::2):
//   gate/up:  h[p, i]  = SiLU(x_p . Wg[e, i]) * (x_p . Wu[e, i])     (SiLU(gate) * up)
//   down:     o[p, c]  = w_p * (h_p . Wd[e, c])                     (routing weight fused)
// with fp32 accumulators in tensor memory and bf16 outputs.  The shared expert
// (share_expert_dim, always on, weight 1) is one more group over all T tokens.
//
// FP8 weights (the low-precision expert weights for decode): each weight matrix is
// E4M3 codes plus one E8M0 power-of-two scale per 128 x 128 block.  TMA brings the codes
// (half the bytes of bf16); eight more warps, in two groups taking alternate k-blocks, turn
// each 128 x 64 code tile into the bf16 tile the MMA reads, scale applied, in the layout
// 128-byte-swizzled TMA would have written.  Every decoded weight is exact in bf16, so the
// GEMM is the bf16 GEMM of the decoded weights, with bf16 tokens as before.
// Sources: llm-atlas page "Step-3.5-Flash", "Champs bruts du config.json":
// moe_intermediate_size 1280, share_expert_dim 1280, hidden_size 4096, norm_expert_weight.
//
// fp32: plain CUDA-core kernels (fp32 FMA), same data flow.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------------------
// tcgen05 grouped GEMM
// ---------------------------------------------------------------------------------------
struct TcParams {
  CUtensorMap tmA[2];  // weights: [0] routed (all experts stacked), [1] shared expert
  CUtensorMap tmB[2];  // activations: [0] routed rows in expert order (gather: x rows,
                       // one-row box), [1] shared rows
  const int32_t* item_start;   // [G + 1] tiles per group slot (prefix); [G] = schedule length
  const int4* item_info;       // [schedule length] tile descriptors {g, m, first row, rows | ks << 16}
  const float* row_w;          // routing weight per routed row (down projection only)
  const int32_t* row_tok;      // token of each routed row (gather)
  int gather;                  // routed token rows gathered from x by tmB[0] (gate/up)
  const __nv_bfloat16* x;      // tokens [T, H] (gate/up with 128-token tiles: rows gathered
                               // by the gather warps, routed and shared alike)
  __nv_bfloat16* out[2];       // [0] routed rows, [1] shared rows
  int ld_out[2];               // row stride of out (elements), routed and shared
  int E, G;
  int64_t T;
  int g_lo, g_hi;              // routed experts held in the weight matrices: [g_lo, g_hi)
                               // (all E, or one rank's range under expert parallelism)
  int sh_base, sh_rows;        // rows of the shared-expert group: [sh_base, sh_base + sh_rows)
  int kblocks[2];              // reduction length / kTileK, routed and shared
  int a_rows_per_group;        // rows of one routed expert's weight matrix
  int a_up_offset[2];          // gate/up: row offset of the up block (I or Is)
  int mt[2];                   // weight row tiles per group, routed and shared
  int rows_out[2];             // rows of out[0] (T*k) and out[1] (T)
  int max_items;               // upper bound of the schedule length (host-computed)
  int ksplit;                  // gate/up: slices of the reduction per tile (1 = no split)
  float limit[2];              // gate/up: SwiGLU limits, routed and shared (0: none)
  int max_tiles;               // bound of tile ids (split partial buffers)
  float* partial;              // [max_tiles][ksplit][BN][256] fp32 gate|up partial sums
  unsigned int* tile_done;     // [max_tiles] slices finished per tile, zero before the launch
  unsigned int* item_counter;  // items claimed beyond the first gridDim.x, zero before the launch
  // gate/up: the down GEMM's schedule and weights, so that a block out of work brings the
  // weight rows of the down GEMM's item blockIdx.x into L2 (null: no prefetch)
  const int32_t* pf_item_start;    // [G + 1] item prefix of the down GEMM
  const int4* pf_info;             // its tile descriptors
  const unsigned char* pf_w[2];    // W_down (this launch's experts), Ws_down
  int pf_mt;                       // weight tiles per group of the down GEMM
  int64_t pf_rows_per_group;       // rows of one routed expert's down matrix (H)
  int64_t pf_row_bytes[2];         // bytes of one row: routed (I), shared (I_shared)
  // both projections in one launch (16-token tiles): a down item of group g waits until
  // every gate/up tile of g has written its h rows
  unsigned int* gu_done;           // [G] gate/up tiles finished per group, zero before the launch
  const int32_t* counts;           // [E] rows per routed expert (its gate/up token tiles)
  const uint8_t* scaleA[2];    // FP8 weights: E8M0 block scales of the A matrices, routed
                               // (stacked by expert) and shared
  int s_rows_per_group;        // FP8 weights: scale rows (128-row blocks) per routed expert
  int s_ld[2];                 // FP8 weights: scale columns (128-column blocks), routed and shared
  Ctrl* ctrl;
};

constexpr int kMaxDynSmem = 232448;  // 227 KB per block on sm_100
constexpr int kConvGroups = 2;       // FP8: converter groups of four warps
constexpr int kRing = 4;             // item slots between the producer and the other roles

template <bool GATED, int BN, bool W8 = false, bool FUSED = false>
struct TcCfg {
  static constexpr int kMats = GATED ? 2 : 1;           // weight tiles per stage (gate, up)
  // k-blocks (64 columns, one 128-byte swizzle atom wide) per stage.  bf16 16-token tiles
  // stream their weights from HBM: two adjacent k-blocks per stage, so that each weight row
  // is requested 256 contiguous bytes at a time rather than 128
  static constexpr int kKB = (BN == 16 && !W8) ? 2 : 1;
  // both GEMMs in one launch: a down tile has no up rows, so it fills a stage's weight room
  // with four k-blocks of its one matrix (and the token-row room holds four k-blocks too)
  static constexpr int kDnKB = FUSED ? 2 * kKB : kKB;
  static constexpr int kAtomA = kTileM * kTileK * 2;   // one k-block of 128 weight rows (16 KB)
  static constexpr int kAtomB = BN * kTileK * 2;       // one k-block of the token rows
  static constexpr int kABytes = kKB * kAtomA;         // bf16 weights per operand tile and stage
  static constexpr int kA8Bytes = kTileM * kTileK;     // one k-block as FP8 codes
  static constexpr int kBBytes = kDnKB * kAtomB;       // token rows
  // one TMA stage: the weight tiles as loaded (bf16, or FP8 codes), then the token rows
  static constexpr int kBOffset = kMats * (W8 ? kA8Bytes : kABytes);
  static constexpr int kStageBytes = kBOffset + kBBytes;
  static constexpr int kKBytes = kMats * (W8 ? kA8Bytes : kAtomA) + kAtomB;  // bytes of one k-block
  // FP8: stages of converted bf16 weight tiles plus a copy of the token rows, between the
  // converters and the MMA.  The converters free each TMA stage as soon as they have read
  // it, so every TMA stage is either in flight or waiting for conversion.  More converted
  // stages than converter groups let a group start its next step before the MMA has
  // finished its previous one (16-token tiles; 128-token ones lack the room).
  static constexpr int kConvStages = W8 ? (BN <= 16 ? (GATED ? 3 : 4) : 2) : 0;
  static constexpr int kConvBOffset = kMats * kABytes;
  static constexpr int kConvBytes = kConvBOffset + kBBytes;
  // bf16 gate/up with 128-token tiles: four more warps gather the tiles' token rows from x
  // (cp.async, 16 bytes per lane), so no permuted copy of x is written and read back
  static constexpr bool kCpGather = GATED && BN == 128 && !W8;
  // bf16 tiles of 128 or more tokens: a stage-watcher warp (the last) waits for each stage's
  // operands and hands the stage to the MMA warp at a named barrier.  A thread that has
  // tcgen05.mma in flight stalls on its next shared-memory read (an mbarrier poll included)
  // for about as long as one stage of MMAs takes, so the issuing warp reads no shared memory
  // between the stages of a tile; the watcher also waits for the accumulator and walks the
  // item ring for it.
  static constexpr bool kWatch = BN >= 128 && !W8;
  static constexpr int kThreads = (W8 ? 192 + 128 * kConvGroups : (kCpGather ? 192 + 128 : 192)) + (kWatch ? 32 : 0);
  static constexpr int kConvMod = kConvStages > 0 ? kConvStages : 1;  // a divisor in every variant
  // tiles of up to 128 tokens stage the output tile [BN][128] bf16 in shared memory for
  // 16-byte stores; 256-token tiles store straight from registers (each warp writes 64
  // contiguous bytes per token) to leave shared memory to the pipeline
  static constexpr bool kStaged = BN <= 128;
  static constexpr int kStagingBytes = kStaged ? BN * kTileM * 2 : 0;
  static constexpr int kAuxBytes = 512 + (BN * 4 > 512 ? BN * 4 : 512);  // barriers, TMEM slot | row weights
  static constexpr int kFit =
      (kMaxDynSmem - kStagingBytes - 1024 - kAuxBytes - kConvStages * kConvBytes) / kStageBytes;
  static constexpr int kStages = kFit > 12 ? 12 : kFit;
  static constexpr int kAccCols = (GATED ? 2 : 1) * BN;  // TMEM columns per accumulator
  static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;  // double-buffered when it fits
  static constexpr int kTmemNeed = kAccBufs * kAccCols;
  static constexpr int kTmemCols = (kTmemNeed <= 32) ? 32 : (kTmemNeed <= 64) ? 64
                                 : (kTmemNeed <= 128) ? 128 : (kTmemNeed <= 256) ? 256 : 512;
  static constexpr int kSmemBytes =
      kStages * kStageBytes + kConvStages * kConvBytes + kStagingBytes + 1024 + kAuxBytes;
  static_assert(kStages >= 2, "pipeline too shallow");
  static_assert(kStageBytes % 1024 == 0 && kBOffset % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(!W8 || BN <= 128, "FP8 weights: staged tiles only");
  static_assert(kConvStages <= 6 && kStages <= 12, "barrier and scale slots in the aux block");
  static_assert(kConvBytes % 1024 == 0, "converted stages keep the 1024-byte swizzle alignment");
  static_assert(kStages >= kConvStages, "the converters' wait order relies on it");
  static_assert(kTmemNeed <= 512, "accumulators exceed tensor memory");
  static_assert(kSmemBytes <= kMaxDynSmem, "shared memory budget");
  static_assert(BN % 16 == 0 && BN <= 256, "tile width");
  static_assert(!FUSED || (GATED && kDnKB * kAtomA <= kBOffset), "a down stage fits the gate/up weight room");
};

struct Item {
  int valid;   // 0: the schedule entry is inconsistent (reported; skipped by every role)
  int ks;      // slice of the reduction (split gate/up tiles), else 0
  int tile;    // tile id (items of one tile share it)
  int sh;      // 0 routed expert, 1 shared expert
  int g;       // group (expert id, or E for the shared expert)
  int m;       // weight row tile
  int row0;    // first activation row of the tile (in the routed or the shared row space)
  int nvalid;  // tokens in the tile
};

// Tile `it` of the schedule from its descriptor (written by the dispatch step), checked
// against this launch's bounds: an inconsistent descriptor is reported and skipped.
template <int BN>
__device__ __forceinline__ Item decode_item_info(const TcParams& p, const int4 d, int it) {
  Item r;
  r.g = d.x;
  r.sh = (r.g == p.E) ? 1 : 0;
  r.m = d.y;
  r.row0 = d.z + (r.sh ? p.sh_base : 0);
  r.nvalid = d.w & 0xFFFF;
  r.ks = d.w >> 16;
  r.tile = it / p.ksplit;  // every group's item count is a multiple of ksplit
  r.valid = (r.g >= 0 && r.g < p.G && (r.sh || (r.g >= p.g_lo && r.g < p.g_hi)) && r.m >= 0 &&
             r.m < p.mt[r.sh] && r.nvalid >= 1 && r.nvalid <= BN && r.ks < p.ksplit &&
             r.row0 >= 0 && r.row0 + r.nvalid <= p.rows_out[r.sh] &&
             (p.ksplit == 1 || (r.tile >= 0 && r.tile < p.max_tiles))) ? 1 : 0;
  if (!r.valid) {
    r.nvalid = 0;
    r.sh = 0;
  }
  return r;
}
template <int BN>
__device__ __forceinline__ Item decode_item(const TcParams& p, int it) {
  return decode_item_info<BN>(p, __ldg(p.item_info + it), it);
}

// The shape of a valid tile as a number 1..32 for the MMA warp: (shared expert) * 16 +
// (16-token MMA columns - 1); 0 ends the schedule.  Tiles of up to 256 tokens.
__device__ __forceinline__ uint32_t tile_code(const Item& t) {
  return static_cast<uint32_t>(t.sh) * 16u + static_cast<uint32_t>((t.nvalid + 15) >> 4);
}

// schedule length, clamped to the host bound (a larger value is reported, not run)
__device__ __forceinline__ int schedule_length(const TcParams& p) {
  const int total = __ldg(p.item_start + p.G);
  if (total < 0 || total > p.max_items) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(p.ctrl, MOE_ERR_DEVICE_BOUNDS);
    return 0;
  }
  return total;
}

// SiLU(gate) * up; a SwiGLU limit L > 0 first clamps gate to <= L and up to [-L, L]
// (limits of llm-atlas page "Step-3.5-Flash", table "Champs bruts du config.json":
// swiglu_limits, swiglu_limits_shared)
__device__ __forceinline__ float swiglu(float g, float u, float L) {
  if (L > 0.0f) {
    g = fminf(g, L);
    u = fminf(fmaxf(u, -L), L);
  }
  return g / (1.0f + __expf(-g)) * u;
}

// Two E4M3 codes (bytes `sel` picks from w) -> two bf16 bit patterns, the low code in
// the low half, each standing for its code times 2^-120.  An E4M3 code is a sign, a
// 4-bit exponent e (bias 7) and a 3-bit mantissa m; moving its exponent and mantissa
// fields into bf16's (bias 127) gives 2^(e-127) (1 + m/8) for e > 0 and, for e = 0, the
// bf16 subnormal 2^-126 m/8 = the code's subnormal m/8 * 2^-6 times the same 2^-120.
__device__ __forceinline__ uint32_t e4m3x2_bits(uint32_t w, uint32_t sel) {
  const uint32_t v = __byte_perm(w, 0u, sel);  // one code in the high byte of each half
  return (v & 0x80008000u) | ((v >> 4) & 0x07F007F0u);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 r = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&r);
}

// One 128 x 64 FP8 code tile (rows of 64 bytes, as TMA loads it without swizzling) ->
// the bf16 tile [128][64] the MMA reads: rows of 128 bytes whose 16-byte chunk c sits at
// chunk c ^ (row % 8), the layout of a 128-byte-swizzled TMA load.  `scale` is the
// block's E8M0 code v: the weights are code * 2^(v - 127) = bits * 2^(v - 7), a product
// exact in bf16 for v <= 134.  128 threads, four 16-code chunks each.
__device__ __forceinline__ void fp8_tile_to_bf16(const unsigned char* src, unsigned char* dst, int ct,
                                                 uint32_t scale) {
  const uint32_t mb = (scale + 120u) << 7;  // bf16 2^(v - 7)
  const uint32_t mult = mb | (mb << 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qd = ct + 128 * i;  // row qd / 4, codes 16 (qd % 4) .. + 15 of the row
    const int r = qd >> 2, j = qd & 3;
    const uint4 w = *reinterpret_cast<const uint4*>(src + r * 64 + j * 16);
    uint4 o0, o1;
    o0.x = bf16x2_mul(e4m3x2_bits(w.x, 0x1404u), mult);
    o0.y = bf16x2_mul(e4m3x2_bits(w.x, 0x3424u), mult);
    o0.z = bf16x2_mul(e4m3x2_bits(w.y, 0x1404u), mult);
    o0.w = bf16x2_mul(e4m3x2_bits(w.y, 0x3424u), mult);
    o1.x = bf16x2_mul(e4m3x2_bits(w.z, 0x1404u), mult);
    o1.y = bf16x2_mul(e4m3x2_bits(w.z, 0x3424u), mult);
    o1.z = bf16x2_mul(e4m3x2_bits(w.w, 0x1404u), mult);
    o1.w = bf16x2_mul(e4m3x2_bits(w.w, 0x3424u), mult);
    unsigned char* row = dst + r * 128;
    *reinterpret_cast<uint4*>(row + (((2 * j) ^ (r & 7)) << 4)) = o0;
    *reinterpret_cast<uint4*>(row + (((2 * j + 1) ^ (r & 7)) << 4)) = o1;
  }
}

// Wait without looking at the abort flag (teardown: in-flight copies must land).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, Ctrl* ctrl) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_status(ctrl, MOE_ERR_DEVICE_TIMEOUT);
      return;
    }
  }
}

// An epilogue thread's stores of h rows, ordered before the release of the group's count
// (after a barrier of the four epilogue warps) and before the TMA loads that read them on
// other SMs once the count is acquired.
__device__ __forceinline__ void release_rows_stored() {
  fence_proxy_async_global();
  fence_acq_rel_gpu();
}

// Persistent grouped GEMM, one block per SM.
//   warp 0      TMA producer (one lane): weight tiles (gate and up for GATED) and token rows
//   warp 1      allocates tensor memory; one lane issues the tcgen05 MMAs
//   warps 2..5  epilogue: tensor memory -> registers -> shared staging tile -> global
//   warps 6..9  bf16 gate/up with 128-token tiles: token-row gather (cp.async)
//   warps 6..13 FP8 weights only: code tiles -> bf16 tiles, two groups of four warps
//               taking alternate k-steps
//   last warp   bf16 tiles of 128 or 256 tokens: stage watcher (waits, hands stages over)
// Accumulators are double-buffered in tensor memory, so the epilogue of one tile overlaps
// the main loop of the next.  Items are claimed dynamically: block b starts with item b and
// then takes the next unclaimed one from a global counter, so blocks that draw short tiles
// take more of them; the producer publishes each claimed item to the MMA and epilogue warps
// through a ring of kRing shared-memory slots (index -1 ends the schedule).
// 16 bytes global -> shared, bypassing L1; `bytes` = 0 fills the 16 bytes with zeros
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src),
               "r"(bytes)
               : "memory");
}
// the mbarrier receives one arrival once every cp.async issued so far by this thread has
// landed (counted in the barrier's expected arrivals)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// FUSED (bf16 16-token tiles): one launch runs both projections.  p holds the gate/up
// GEMM's parameters and pdn the down GEMM's; items [0, n_gu) of the schedule are gate/up
// tiles, the rest down tiles (item n_gu + i is down tile i).  A down item's producer waits
// until every gate/up tile of its group has written its h rows (gu_done, released after the
// rows are stored) before it loads them; the weights of the down GEMM need no wait.
template <bool GATED, int BN, bool W8, bool FUSED = false>
__global__ void __launch_bounds__(TcCfg<GATED, BN, W8, FUSED>::kThreads, 1)
    expert_gemm_tc_kernel(const __grid_constant__ TcParams p, const __grid_constant__ TcParams pdn) {
  using C = TcCfg<GATED, BN, W8, FUSED>;
  static_assert(!FUSED || (GATED && BN == 16 && !W8), "one launch for both projections: bf16 16-token tiles");
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  unsigned char* conv = smem + C::kStages * C::kStageBytes;  // FP8: converted weight tiles
  __nv_bfloat16* staging = reinterpret_cast<__nv_bfloat16*>(conv + C::kConvStages * C::kConvBytes);
  unsigned char* aux = conv + C::kConvStages * C::kConvBytes + C::kStagingBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* hand = abort_flag + 1;  // [2] items handed from the watcher to the MMA warp
  uint64_t* cfull = reinterpret_cast<uint64_t*>(aux + 256);  // FP8: [kConvStages] converted
  uint64_t* cempty = cfull + 6;                              // FP8: [kConvStages] consumed
  volatile uint32_t* sc_stage = reinterpret_cast<volatile uint32_t*>(aux + 464);  // FP8: [kStages]
                                                         // scale codes of each stage's tiles
  uint64_t* ring_full = reinterpret_cast<uint64_t*>(aux + 384);  // [kRing]
  uint64_t* ring_empty = ring_full + kRing;                     // [kRing]
  volatile int* ring = reinterpret_cast<volatile int*>(ring_empty + kRing);  // [kRing] item ids
  float* sw = reinterpret_cast<float*>(aux + 512);  // [BN] routing weights of the tile rows

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], C::kCpGather ? 1 + 128 : 1);  // + one per gather thread
      mbar_init(&empty[s], W8 ? 4 : 1);  // the MMA commit, or (FP8) the four converter warps
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4 * 32);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < kRing; ++q) {
      mbar_init(&ring_full[q], 1);
      // the MMA thread (or the watcher) and one lane per epilogue, converter and gather warp
      mbar_init(&ring_empty[q], 1 + 4 + (W8 ? 4 * kConvGroups : 0) + (C::kCpGather ? 4 : 0));
    }
    for (int c = 0; c < C::kConvStages; ++c) {
      mbar_init(&cfull[c], 4);    // one lane per warp of the converter group
      mbar_init(&cempty[c], 1);   // the MMA commit
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA[0]);
    tma_prefetch_desc(&p.tmB[0]);
    tma_prefetch_desc(&p.tmA[1]);
    tma_prefetch_desc(&p.tmB[1]);
    if (FUSED) {
      tma_prefetch_desc(&pdn.tmA[0]);
      tma_prefetch_desc(&pdn.tmB[0]);
      tma_prefetch_desc(&pdn.tmA[1]);
      tma_prefetch_desc(&pdn.tmB[1]);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  // the producer requests its first item's descriptor (item blockIdx.x, within the table's
  // capacity) together with the schedule length, so that both arrive in one round trip
  int4 first_info = make_int4(-1, 0, 0, 0);
  if (warp == 0 && static_cast<int>(blockIdx.x) < p.max_items) first_info = __ldg(p.item_info + blockIdx.x);
  int n_gu, total;  // gate/up items, all items
  if constexpr (FUSED) {
    const int a = __ldg(p.item_start + p.G), b = __ldg(pdn.item_start + pdn.G);
    const bool lengths_ok = a >= 0 && a <= p.max_items && b >= 0 && b <= pdn.max_items;
    if (!lengths_ok && threadIdx.x == 0 && blockIdx.x == 0) set_status(p.ctrl, MOE_ERR_DEVICE_BOUNDS);
    n_gu = lengths_ok ? a : 0;
    total = lengths_ok ? a + b : 0;
  } else {
    n_gu = total = schedule_length(p);
  }
  // the launch parameters of item `it` (gate/up or down) and its index in that schedule
  auto prm_of = [&](int it) -> const TcParams& { return (FUSED && it >= n_gu) ? pdn : p; };
  auto local_of = [&](int it) { return (FUSED && it >= n_gu) ? it - n_gu : it; };
  // FP8: waiting threads sleep in their polls, leaving the issue slots to the converters
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return W8 ? mbar_wait_sleep(bar, parity, p.ctrl, abort_flag) : mbar_wait(bar, parity, p.ctrl, abort_flag);
  };

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------------
    // Lane 0 waits for free stages and loads the weight tiles; routed token rows of the
    // gate/up GEMM come straight from x, four rows per lane and copy (row-gather TMA).
    int stage = 0;
    uint32_t phase = 0;
    uint32_t used = 0;  // stages that ever received a copy
    bool ok = true;
    int q = 0;
    uint32_t qphase = 0;
    // FP8: block scales of an item (one 128-column block per lane, and lane + 32)
    auto load_scales = [&](const Item& t, uint32_t* g, uint32_t* u) {
      const int kbn = p.kblocks[t.sh];
      const int k0 = t.ks * kbn / p.ksplit, k1 = (t.ks + 1) * kbn / p.ksplit;
      const int c0 = k0 >> 1, nblk = k1 > k0 ? ((k1 - 1) >> 1) - c0 + 1 : 0;
      const int ld = p.s_ld[t.sh];
      const uint8_t* sbase = p.scaleA[t.sh] + static_cast<int64_t>(t.sh ? 0 : t.g - p.g_lo) * p.s_rows_per_group * ld;
      const uint8_t* srow_g = sbase + static_cast<int64_t>(t.m) * ld;
      const uint8_t* srow_u = sbase + static_cast<int64_t>(t.m + p.a_up_offset[t.sh] / kTileM) * ld;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        g[h] = u[h] = 0u;
        if (lane + 32 * h < nblk) {
          g[h] = __ldg(srow_g + c0 + lane + 32 * h);
          if (GATED) u[h] = __ldg(srow_u + c0 + lane + 32 * h);
        }
      }
    };
    int pf_it = -1;  // FP8: the item whose scales pf_sg / pf_su hold
    uint32_t pf_sg[2] = {0u, 0u}, pf_su[2] = {0u, 0u};
    // the item after the current one is claimed, and its descriptor loaded, while the
    // current one streams
    int it = static_cast<int>(blockIdx.x);
    int4 info = first_info;  // descriptor of item `it`
    if (FUSED && it >= n_gu && it < total) info = __ldg(pdn.item_info + (it - n_gu));  // a down item first
    int claimed = (lane == 0) ? static_cast<int>(atomicAdd(p.item_counter, 1u) + gridDim.x) : 0;
    // fused launch: the gate/up tiles finished in the group of the next (down) item, read
    // during the current item's second stage so that the next item seldom waits for it
    int pre_g = -1;
    unsigned int pre_seen = 0;
    for (;;) {
      if (it >= total || !ok) it = -1;
      // publish the item (or the end) to the MMA and epilogue warps
      int pub = 1;
      if (lane == 0) {
        pub = wait(&ring_empty[q], qphase ^ 1u) ? 1 : 0;
        if (pub) {
          ring[q] = it;
          mbar_arrive(&ring_full[q]);
        }
      }
      pub = __shfl_sync(0xffffffffu, pub, 0);
      if (++q == kRing) { q = 0; qphase ^= 1u; }
      if (!pub || it < 0) break;
      const int cur = it;
      const bool dn = FUSED && cur >= n_gu;  // a down item of the fused launch
      const TcParams& pp = prm_of(cur);
      const Item t = decode_item_info<BN>(pp, info, local_of(cur));
      // the next item's claim and descriptor, taken once this item's first stage is issued
      // (at the first item the claim is still in flight)
      bool next_taken = false;
      auto take_next = [&]() {
        if (next_taken) return;
        next_taken = true;
        it = __shfl_sync(0xffffffffu, claimed, 0);
        if (lane == 0 && it < total) claimed = static_cast<int>(atomicAdd(p.item_counter, 1u) + gridDim.x);
        if (it < total) info = __ldg(prm_of(it).item_info + local_of(it));
      };
      if (!t.valid) {
        if (blockIdx.x == 0 && lane == 0) set_status(p.ctrl, MOE_ERR_DEVICE_BOUNDS);
        take_next();
        continue;
      }
      const bool gated = GATED && !dn;
      // a down item of the fused launch (lane 0): every gate/up tile of its group has stored
      // its h rows -- ceil(rows / BN) token tiles times the group's gate/up weight tiles
      auto rows_ready = [&]() -> bool {
        const int rows = t.sh ? p.sh_rows : __ldg(p.counts + t.g);
        const unsigned int need = static_cast<unsigned int>((rows + BN - 1) / BN * p.mt[t.sh]);
        if (pre_g == t.g && pre_seen >= need) {
          fence_proxy_async_global();
          return true;
        }
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(p.gu_done + t.g) < need) {
          if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
            set_status(p.ctrl, MOE_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
          }
          __nanosleep(100);
        }
        fence_proxy_async_global();  // the h rows, stored by other SMs, before the TMA reads
        return true;
      };
      const bool gath = gated && pp.gather && !t.sh;
      int tok[4] = {0, 0, 0, 0};
      if (gath && lane < BN / 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int n = lane * 4 + q;
          const int v = __ldg(p.row_tok + t.row0 + (n < t.nvalid ? n : 0));
          if (v < 0 || v >= p.T) set_status(p.ctrl, MOE_ERR_DEVICE_BOUNDS);
          tok[q] = (v < 0 || v >= p.T) ? 0 : v;  // padding rows repeat the first token
        }
      }
      const int arow = t.sh ? t.m * kTileM : (t.g - pp.g_lo) * pp.a_rows_per_group + t.m * kTileM;
      const int kb_n = pp.kblocks[t.sh];
      const int kb0 = t.ks * kb_n / pp.ksplit, kb1 = (t.ks + 1) * kb_n / pp.ksplit;
      // bytes of one k-block of a stage (a down item of the fused launch has no up rows)
      const uint32_t kbytes = (FUSED && dn) ? C::kAtomA + C::kAtomB : C::kKBytes;
      // FP8: the item's block scales, one 128-column block per lane (and lane + 32),
      // loaded one item ahead so that their latency overlaps the previous item's stream
      uint32_t sg[2] = {0u, 0u}, su[2] = {0u, 0u};
      const int sc0 = kb0 >> 1;  // 128-column scale blocks hold two 64-column k-blocks
      if (W8) {
        take_next();  // the next item's scales are loaded now
        if (pf_it == cur) {
          sg[0] = pf_sg[0]; sg[1] = pf_sg[1]; su[0] = pf_su[0]; su[1] = pf_su[1];
        } else {
          load_scales(t, sg, su);
        }
        pf_it = -1;
        if (it < total) {
          const Item tn = decode_item<BN>(p, it);
          if (tn.valid) {
            load_scales(tn, pf_sg, pf_su);
            pf_it = it;
          }
        }
      }
      const int kstep = (FUSED && dn) ? C::kDnKB : C::kKB;  // k-blocks per stage
      for (int kb = kb0; kb < kb1; kb += kstep) {
        unsigned char* st = smem + stage * C::kStageBytes;
        const int nk = min(kstep, kb1 - kb);  // k-blocks in this stage
        uint32_t scw = 0;
        if (W8) {
          const int rel = (kb >> 1) - sc0;  // < 64: the host bounds K by 64 scale blocks
          scw = __shfl_sync(0xffffffffu, rel < 32 ? sg[0] : sg[1], rel & 31);
          if (GATED) scw |= __shfl_sync(0xffffffffu, rel < 32 ? su[0] : su[1], rel & 31) << 8;
        }
        int good = 1;
        if (lane == 0) {
          good = wait(&empty[stage], phase ^ 1u) ? 1 : 0;
          if (good) {
            if (W8) sc_stage[stage] = scw;  // published by the arrive below
            mbar_arrive_expect_tx(&full[stage], C::kCpGather ? C::kBOffset : nk * kbytes);
            for (int j = 0; j < nk; ++j) {
              tma_load_2d(st + j * C::kAtomA, &pp.tmA[t.sh], (kb + j) * kTileK, arow, &full[stage]);
              if (gated)
                tma_load_2d(st + (W8 ? C::kA8Bytes : C::kABytes) + j * C::kAtomA, &pp.tmA[t.sh],
                            (kb + j) * kTileK, arow + pp.a_up_offset[t.sh], &full[stage]);
            }
            // a down item's h rows once its group's gate/up tiles are done (its first
            // weight k-blocks are in flight meanwhile)
            if (FUSED && dn && kb == kb0 && !rows_ready()) good = 0;
            if (good && !gath && !C::kCpGather)
              for (int j = 0; j < nk; ++j)
                tma_load_2d(st + C::kBOffset + j * C::kAtomB, &pp.tmB[t.sh], (kb + j) * kTileK, t.row0,
                            &full[stage]);
          }
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) { ok = false; break; }
        if (gath && lane < BN / 4)
          for (int j = 0; j < nk; ++j)
            tma_gather4_2d(st + C::kBOffset + j * C::kAtomB + lane * 4 * kTileK * 2, &p.tmB[0], (kb + j) * kTileK,
                           tok[0], tok[1], tok[2], tok[3], &full[stage]);
        used |= 1u << stage;
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        if (kb == kb0) take_next();
        if (FUSED && lane == 0 && kb == kb0 + kstep) {
          pre_g = -1;
          if (it >= n_gu && it < total && info.x >= 0 && info.x <= p.E) {  // the next item is a down item
            pre_g = info.x;
            pre_seen = ld_acquire_gpu(p.gu_done + pre_g);
          }
        }
      }
      take_next();
    }
    __syncwarp();
    if (GATED && !W8 && p.pf_item_start && lane == 0 && static_cast<int>(blockIdx.x) < __ldg(p.pf_item_start + p.G)) {
      // out of work: the rows of the down GEMM's item blockIdx.x (its first wave) into L2
      const int4 d = __ldg(p.pf_info + blockIdx.x);
      const int g = d.x, m = d.y;
      const int sh = (g == p.E) ? 1 : 0;
      if (g >= 0 && m >= 0 && m < p.pf_mt && (sh || (g >= p.g_lo && g < p.g_hi))) {
        const int64_t row = (sh ? 0 : (g - p.g_lo) * p.pf_rows_per_group) + static_cast<int64_t>(m) * kTileM;
        prefetch_l2(p.pf_w[sh] + row * p.pf_row_bytes[sh], static_cast<uint64_t>(kTileM) * p.pf_row_bytes[sh]);
      }
    }
    // every copy issued must have landed before the block exits
    if (lane == 0)
      for (int s = 0; s < C::kStages; ++s) {
        if (!(used & (1u << s))) continue;
        // the last phase issued on stage s: stages before `stage` were last issued in the
        // current pass (parity phase), the others in the previous pass (phase ^ 1)
        const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait_drain(&full[s], par, p.ctrl);
      }
  } else if (C::kWatch && warp == 1) {
    // ------------------------- MMA issuer (stages handed over) -------------------------
    // The whole warp takes the hand-overs at named barrier 2; lane 0 issues.  The item of
    // each tile is read once (hand[n & 1]); every stage after it costs the warp one barrier
    // and no shared-memory read.  (The pause that the read and the decode cost once a tile
    // measured faster here than passing the tile in the barrier, as the pair kernel does:
    // it lets the copies into shared memory, which compete with the tensor cores' operand
    // reads, catch up.)  After a failed wait the watcher goes on handing over the
    // stages of the current tile (their MMAs read stale operands; the status is set) and
    // then ends the schedule.
    int stage = 0, acc = 0, n = 0;
    for (;; ++n) {
      __syncwarp();
      named_bar_sync(2, 64);  // item hand-over: hand[n & 1], accumulator `acc` free
      const int it = hand[n & 1];
      if (it < 0) break;
      const Item t = decode_item<BN>(p, it);  // valid: the watcher skips the others
      const uint32_t idesc = idesc_bf16_f32(kTileM, (t.nvalid + 15) & ~15);
      const uint32_t d0 = tmem_base + acc * C::kAccCols;
      const int kb_n = p.kblocks[t.sh];
      const int kb0 = t.ks * kb_n / p.ksplit, kb1 = (t.ks + 1) * kb_n / p.ksplit;
      for (int kb = kb0; kb < kb1; ++kb) {
        __syncwarp();
        named_bar_sync(2, 64);  // stage hand-over: its operands are in shared memory
        if (lane == 0) {
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b0 = a0 + C::kBOffset;
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            const uint32_t accum = (kb != kb0 || kk) ? 1u : 0u;
            const uint64_t bdesc = sw128_kmajor_desc(b0 + kk * 32);
            mma_bf16(d0, sw128_kmajor_desc(a0 + kk * 32), bdesc, idesc, accum);
            if (GATED)
              mma_bf16(d0 + BN, sw128_kmajor_desc(a0 + C::kABytes + kk * 32), bdesc, idesc, accum);
          }
          mma_commit(&empty[stage]);
        }
        if (++stage == C::kStages) stage = 0;
      }
      if (lane == 0) mma_commit(&tfull[acc]);
      if (++acc == C::kAccBufs) acc = 0;
    }
    // all MMAs issued by this thread complete before the accumulators are freed
    if (lane == 0) {
      mma_commit(drain);
      mbar_wait_drain(drain, 0, p.ctrl);
    }
  } else if (C::kWatch && warp == C::kThreads / 32 - 1) {
    // ------------------------------- stage watcher ------------------------------------
    // Walks the item ring like the MMA warp would: per item it waits for a free
    // accumulator and hands the item over, per stage it waits for the operands (TMA bytes
    // and, with gather warps, their cp.async rows made visible to the tensor cores' proxy)
    // and hands the stage over.
    int stage = 0, acc = 0, n = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool failed = false;
    int q = 0;
    uint32_t qphase = 0;
    for (;; ++n) {
      int it = -1;
      Item t{};
      while (!failed) {
        if (!wait(&ring_full[q], qphase)) { failed = true; break; }
        it = ring[q];
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring_empty[q]);
        if (++q == kRing) { q = 0; qphase ^= 1u; }
        if (it < 0) break;
        t = decode_item<BN>(p, it);
        if (t.valid) break;
        it = -1;  // inconsistent entry (reported by the producer): the next one
      }
      if (failed) it = -1;
      if (it >= 0 && !wait(&tempty[acc], acc_phase ^ 1u)) { failed = true; it = -1; }
      if (lane == 0) hand[n & 1] = it;
      __syncwarp();
      named_bar_sync(2, 64);
      if (it < 0) break;
      const int kb_n = p.kblocks[t.sh];
      const int kb0 = t.ks * kb_n / p.ksplit, kb1 = (t.ks + 1) * kb_n / p.ksplit;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!failed && !wait(&full[stage], phase)) failed = true;
        // token rows written by the gather warps' cp.async: order them before the tensor
        // cores' (async-proxy) reads of the stage
        if (C::kCpGather) fence_proxy_async_smem();
        __syncwarp();
        named_bar_sync(2, 64);
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
      if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
    }
  } else if (warp == 1) {
    // ------------------------------- MMA issuer ---------------------------------------
    if (lane == 0) {
      int stage = 0, acc = 0, cs = 0;
      uint32_t phase = 0, acc_phase = 0, cphase = 0;
      bool ok = true;
      int q = 0;
      uint32_t qphase = 0;
      while (ok) {
        if (!wait(&ring_full[q], qphase)) break;
        const int it = ring[q];
        mbar_arrive(&ring_empty[q]);
        if (++q == kRing) { q = 0; qphase ^= 1u; }
        if (it < 0) break;
        const TcParams& pp = prm_of(it);
        const bool gated = GATED && !(FUSED && it >= n_gu);
        const Item t = decode_item<BN>(pp, local_of(it));
        if (!t.valid) continue;
        const int n_mma = (t.nvalid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kTileM, n_mma);
        if (!wait(&tempty[acc], acc_phase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::kAccCols;
        const int kb_n = pp.kblocks[t.sh];
        const int kb0 = t.ks * kb_n / pp.ksplit, kb1 = (t.ks + 1) * kb_n / pp.ksplit;
        const int kstep = gated ? C::kKB : C::kDnKB;  // k-blocks per stage
        for (int kb = kb0; kb < kb1; kb += kstep) {
          if (!(W8 ? wait(&cfull[cs], cphase) : wait(&full[stage], phase))) { ok = false; break; }
          tc_fence_after();
          // token rows written by the gather warps' cp.async: order them before the
          // tensor cores' (async-proxy) reads of the stage
          if (C::kCpGather) fence_proxy_async_smem();
          const uint32_t s0 = W8 ? smem_u32(conv + cs * C::kConvBytes) : smem_u32(smem + stage * C::kStageBytes);
          const int nk = min(kstep, kb1 - kb);
          for (int j = 0; j < nk; ++j) {
            const uint32_t a0 = s0 + j * C::kAtomA;
            const uint32_t b0 = s0 + (W8 ? C::kConvBOffset : C::kBOffset) + j * C::kAtomB;
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              const uint32_t accum = (kb != kb0 || j || kk) ? 1u : 0u;
              const uint64_t bdesc = sw128_kmajor_desc(b0 + kk * 32);
              mma_bf16(d0, sw128_kmajor_desc(a0 + kk * 32), bdesc, idesc, accum);
              if (gated)
                mma_bf16(d0 + BN, sw128_kmajor_desc(a0 + C::kABytes + kk * 32), bdesc, idesc, accum);
            }
          }
          if (W8) {
            mma_commit(&cempty[cs]);
            if (++cs == C::kConvStages) { cs = 0; cphase ^= 1u; }
          } else {
            mma_commit(&empty[stage]);
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread complete before the accumulators are freed
      mma_commit(drain);
      mbar_wait_drain(drain, 0, p.ctrl);
    }
  } else if (C::kCpGather && warp >= 6) {
    // --------------------- token-row gather (warps 6..9, 128-token tiles) ---------------
    // Each k-step's B tile is 128 token rows x 64 columns (128 bytes a row), written where a
    // 128-byte-swizzled TMA load would put them: chunk c of row n at chunk c ^ (n % 8).
    // Lane l of gather warp w copies chunk l % 8 of rows 32w + 4i + l / 8 (i = 0..7), so a
    // warp's eight lanes per row read one 128-byte line.  Rows past the tile's tokens are
    // zero-filled.  Routed rows come from x[row_tok[row]], shared-expert rows from x[row].
    const int gw = warp - 6;
    const int c = lane & 7;
    int stage = 0;
    uint32_t phase = 0;
    int q = 0;
    uint32_t qphase = 0;
    bool ok = true;
    while (ok) {
      if (!wait(&ring_full[q], qphase)) break;
      const int it = ring[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring_empty[q]);
      if (++q == kRing) { q = 0; qphase ^= 1u; }
      if (it < 0) break;
      const Item t = decode_item<BN>(p, it);
      if (!t.valid) continue;
      const __nv_bfloat16* src[8];
      uint32_t nbytes[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int n = 32 * gw + 4 * i + (lane >> 3);
        int64_t tok = 0;
        nbytes[i] = 0;
        if (n < t.nvalid) {
          tok = t.sh ? static_cast<int64_t>(t.row0 + n) : static_cast<int64_t>(__ldg(p.row_tok + t.row0 + n));
          if (tok < 0 || tok >= p.T) {
            set_status(p.ctrl, MOE_ERR_DEVICE_BOUNDS);
            tok = 0;
          } else {
            nbytes[i] = 16;
          }
        }
        src[i] = p.x + tok * (static_cast<int64_t>(p.kblocks[0]) * kTileK) + c * 8;
      }
      const int kb_n = p.kblocks[t.sh];
      const int kb0 = t.ks * kb_n / p.ksplit, kb1 = (t.ks + 1) * kb_n / p.ksplit;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait(&empty[stage], phase ^ 1u)) { ok = false; break; }
        unsigned char* bt = smem + stage * C::kStageBytes + C::kBOffset;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int n = 32 * gw + 4 * i + (lane >> 3);
          cp_async16(bt + n * 128 + ((c ^ (n & 7)) << 4), src[i] + kb * kTileK, nbytes[i]);
        }
        cp_async_arrive_noinc(&full[stage]);
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait_all();  // this thread's copies land before the block exits
  } else if (W8 && warp >= 6) {
    // ------------------------ FP8 code tiles -> bf16 (warps 6..13) --------------------
    // Group g converts the block's k-steps n with n % 2 == g, so one group's waits and
    // fences overlap the other group's conversion.
    const uint32_t grp = static_cast<uint32_t>(warp - 6) >> 2;  // < kConvGroups
    const int ct = threadIdx.x - 192 - 128 * static_cast<int>(grp);  // 0..127 within the group
    uint32_t n = 0;  // k-steps of this block so far, over all items
    int q = 0;
    uint32_t qphase = 0;
    bool ok = true;
    while (ok) {
      if (!wait(&ring_full[q], qphase)) break;
      const int it = ring[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring_empty[q]);
      if (++q == kRing) { q = 0; qphase ^= 1u; }
      if (it < 0) break;
      const Item t = decode_item<BN>(p, it);
      if (!t.valid) continue;
      const int kb_n = p.kblocks[t.sh];
      const int kb0 = t.ks * kb_n / p.ksplit, kb1 = (t.ks + 1) * kb_n / p.ksplit;
      for (int kb = kb0; kb < kb1; ++kb, ++n) {
        if (n % kConvGroups != grp) continue;
        const int stage = static_cast<int>(n % C::kStages), cs = static_cast<int>(n % C::kConvMod);
        const uint32_t phase = (n / C::kStages) & 1u, cphase = (n / C::kConvMod) & 1u;
        // the converted stage first: once the MMA has consumed step n - kConvStages, every
        // earlier use of this TMA stage (n - kStages <= n - kConvStages) has completed, so
        // the parity wait on it below cannot mistake an older phase for this one, whichever
        // group took the stage's previous use
        if (!wait(&cempty[cs], cphase ^ 1u) || !wait(&full[stage], phase)) { ok = false; break; }
        const uint32_t scw = sc_stage[stage];
        const unsigned char* src = smem + stage * C::kStageBytes;
        unsigned char* dst = conv + cs * C::kConvBytes;
        fp8_tile_to_bf16(src, dst, ct, scw & 0xFFu);
        if (GATED) fp8_tile_to_bf16(src + C::kA8Bytes, dst + C::kABytes, ct, (scw >> 8) & 0xFFu);
        // the token rows, byte for byte (both copies sit at 1024-byte-aligned offsets, so the
        // 128-byte swizzle TMA wrote them in stays valid)
        for (int i = ct; i < C::kBBytes / 16; i += 128)
          reinterpret_cast<uint4*>(dst + C::kConvBOffset)[i] =
              reinterpret_cast<const uint4*>(src + C::kBOffset)[i];
        fence_proxy_async_smem();  // the tensor cores read these bytes next
        __syncwarp();              // the warp's reads and writes, then one arrival each
        if (lane == 0) {
          mbar_arrive(&empty[stage]);  // the TMA stage may be refilled
          mbar_arrive(&cfull[cs]);
        }
      }
    }
  } else {
    // ------------------------------- epilogue (warps 2..5) ----------------------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access: 32*quarter ..
    const int r = quarter * 32 + lane;  // weight row within the tile = output column
    const int et = threadIdx.x - 64;    // 0..127
    int acc = 0;
    uint32_t acc_phase = 0;
    int q = 0;
    uint32_t qphase = 0;
    for (;;) {
      if (!wait(&ring_full[q], qphase)) break;
      const int it = ring[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring_empty[q]);
      if (++q == kRing) { q = 0; qphase ^= 1u; }
      if (it < 0) break;
      const TcParams& pp = prm_of(it);
      const bool gated = GATED && !(FUSED && it >= n_gu);
      const Item t = decode_item<BN>(pp, local_of(it));
      if (!t.valid) continue;
      if (!gated)
        for (int n = et; n < BN; n += 128)
          sw[n] = (t.sh || n >= t.nvalid) ? 1.0f : __ldg(pp.row_w + t.row0 + n);
      if (!wait(&tfull[acc], acc_phase)) break;
      tc_fence_after();
      named_bar_sync(1, 128);  // staging free (previous tile copied out), sw visible
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * C::kAccCols;
      if (!C::kStaged) {
        // rows of this thread's output column, one token at a time, straight to global
        const int ld = p.ld_out[t.sh];
        __nv_bfloat16* out = p.out[t.sh] + static_cast<int64_t>(t.row0) * ld + t.m * kTileM + r;
        for (int c0 = 0; c0 < t.nvalid; c0 += 16) {
          uint32_t a[16];
          tmem_ld16_nowait(trow + c0, a);
          float v[16];
          if (GATED) {
            uint32_t u[16];
            tmem_ld16_nowait(trow + BN + c0, u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = swiglu(__uint_as_float(a[j]), __uint_as_float(u[j]), p.limit[t.sh]);
          } else {
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(a[j]) * sw[c0 + j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < t.nvalid) out[static_cast<int64_t>(c0 + j) * ld] = __float2bfloat16_rn(v[j]);
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
        named_bar_sync(1, 128);  // sw free for the next tile
        continue;
      }
      if (gated && C::kStaged && p.ksplit > 1) {
        // this slice's gate|up partial sums -> its own fp32 slab; the last slice of the
        // tile adds the slabs, applies SiLU(gate)*up and writes the tile
        float* slab = p.partial + (static_cast<int64_t>(t.tile) * p.ksplit + t.ks) * BN * 256;
        for (int c0 = 0; c0 < t.nvalid; c0 += 16) {
          uint32_t a[16], u[16];
          tmem_ld16_nowait(trow + c0, a);
          tmem_ld16_nowait(trow + BN + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < t.nvalid) {
              slab[(c0 + j) * 256 + r] = __uint_as_float(a[j]);
              slab[(c0 + j) * 256 + 128 + r] = __uint_as_float(u[j]);
            }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
        fence_acq_rel_gpu();
        named_bar_sync(1, 128);
        if (et == 0) sw[0] = (atomicAdd(p.tile_done + t.tile, 1u) == static_cast<unsigned>(p.ksplit - 1)) ? 1.f : 0.f;
        named_bar_sync(1, 128);
        const bool last_slice = sw[0] != 0.f;
        named_bar_sync(1, 128);  // the flag is read by all before it can be rewritten
        if (!last_slice) continue;  // another slice finishes this tile
        fence_acq_rel_gpu();
        const float* tile_slabs = p.partial + static_cast<int64_t>(t.tile) * p.ksplit * BN * 256;
        for (int n = 0; n < t.nvalid; ++n) {
          float gs = 0.f, us = 0.f;
          for (int q = 0; q < p.ksplit; ++q) {
            gs += __ldcg(tile_slabs + (static_cast<int64_t>(q) * BN + n) * 256 + r);
            us += __ldcg(tile_slabs + (static_cast<int64_t>(q) * BN + n) * 256 + 128 + r);
          }
          staging[n * kTileM + r] = __float2bfloat16_rn(swiglu(gs, us, p.limit[t.sh]));
        }
        named_bar_sync(1, 128);
        const int ld = p.ld_out[t.sh];
        __nv_bfloat16* out = p.out[t.sh] + static_cast<int64_t>(t.row0) * ld + t.m * kTileM;
        const uint4* src = reinterpret_cast<const uint4*>(staging);
        for (int i = et; i < t.nvalid * 16; i += 128) {
          const int n = i >> 4, c = i & 15;
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(n) * ld + c * 8) = src[n * 16 + c];
        }
        if (FUSED) release_rows_stored();
        named_bar_sync(1, 128);  // staging and sw[0] free for the next tile
        if (FUSED && et == 0) atomicAdd(p.gu_done + t.g, 1u);  // the tile's h rows are stored
        continue;
      }
      for (int c0 = 0; c0 < t.nvalid; c0 += 16) {
        uint32_t a[16];
        tmem_ld16_nowait(trow + c0, a);
        if (gated) {
          uint32_t u[16];
          tmem_ld16_nowait(trow + BN + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < t.nvalid)
              staging[(c0 + j) * kTileM + r] =
                  __float2bfloat16_rn(swiglu(__uint_as_float(a[j]), __uint_as_float(u[j]), pp.limit[t.sh]));
        } else {
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < t.nvalid)
              staging[(c0 + j) * kTileM + r] = __float2bfloat16_rn(__uint_as_float(a[j]) * sw[c0 + j]);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);  // the accumulator may be overwritten now
      if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      named_bar_sync(1, 128);  // staging tile complete
      // rows of 128 bf16 (256 B) -> out[row0 + n][m*128 ...], 16-byte coalesced stores
      const int ld = pp.ld_out[t.sh];
      __nv_bfloat16* out = pp.out[t.sh] + static_cast<int64_t>(t.row0) * ld + t.m * kTileM;
      const uint4* src = reinterpret_cast<const uint4*>(staging);
      for (int i = et; i < t.nvalid * 16; i += 128) {
        const int n = i >> 4, c = i & 15;
        *reinterpret_cast<uint4*>(out + static_cast<int64_t>(n) * ld + c * 8) = src[n * 16 + c];
      }
      if (FUSED && gated) {
        release_rows_stored();
        named_bar_sync(1, 128);
        if (et == 0) atomicAdd(p.gu_done + t.g, 1u);  // the tile's h rows are stored
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------------------------------
// Pair tiles for the down GEMM of long prefill (on average 256 or more tokens per expert): a
// cluster of two CTAs on two SMs computes one 256-row weight tile x 256-token tile with
// tcgen05.mma cta_group::2.  CTA c of the pair holds weight rows [128c, 128c + 128) of the
// tile and token rows [128c, 128c + 128) in its own shared memory; the even CTA's MMA warp
// multiplies the pair's 256 x 256 tile, each CTA's tensor memory receiving its own 128 weight
// rows for all 256 tokens (two 256-column accumulators).  Each SM thus loads, and its tensor
// cores read, half the token rows a single-SM tile of the same shape would.  The routing
// weight is applied in the epilogue.
// Work items (group, 256-row weight tile, token tile) are taken in a fixed order, pair q
// doing items q, q + pairs, ...; both CTAs walk the same sequence.  TMA loads of both CTAs
// complete on the even CTA's barrier; the MMA commits arrive on both CTAs' barriers; both
// epilogues release an accumulator on the even CTA's barrier.
// ---------------------------------------------------------------------------------------
struct PairCfg {
  static constexpr int BN = 256;                       // tokens per pair tile
  static constexpr int kABytes = kTileM * kTileK * 2;  // this CTA's 128 weight rows
  static constexpr int kBRows = BN / 2;                // this CTA's token rows
  static constexpr int kBBytes = kBRows * kTileK * 2;
  static constexpr int kBOffset = kABytes;
  static constexpr int kStageBytes = kBOffset + kBBytes;
  static constexpr int kThreads = 192 + 32;            // + the stage watcher (even CTA)
  static constexpr int kChunk = 32;                    // tokens per epilogue chunk
  static constexpr int kStagingBytes = kChunk * kTileM * 2;
  static constexpr int kAuxBytes = 2048;               // barriers, TMEM slot, row weights
  static constexpr int kFit = (kMaxDynSmem - kStagingBytes - 1024 - kAuxBytes) / kStageBytes;
  static constexpr int kStages = kFit > 8 ? 8 : kFit;
  static constexpr int kAccCols = BN;
  static constexpr int kAccBufs = 2;
  static constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes + 1024 + kAuxBytes;
  static_assert(kStages >= 3 && kSmemBytes <= kMaxDynSmem, "shared memory budget");
  static_assert(kStageBytes % 1024 == 0 && kBOffset % 1024 == 0, "stages keep the swizzle alignment");
  static_assert(kAccBufs * kAccCols <= 512, "tensor memory");
};

__global__ void __launch_bounds__(PairCfg::kThreads, 1) expert_gemm_pair_kernel(const __grid_constant__ TcParams p) {
  using C = PairCfg;
  constexpr int BN = C::BN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  __nv_bfloat16* staging = reinterpret_cast<__nv_bfloat16*>(smem + C::kStages * C::kStageBytes);
  unsigned char* aux = smem + C::kStages * C::kStageBytes + C::kStagingBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(aux);   // [kStages], used on the even CTA
  uint64_t* empty = full + 8;                          // [kStages]
  uint64_t* tfull = empty + 8;                         // [2]
  uint64_t* tempty = tfull + 2;                        // [2], used on the even CTA
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sw = reinterpret_cast<float*>(aux + 1024);    // [256] routing weights of the tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();             // 0: the pair's MMA issuer
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);   // the even CTA's expect_tx; bytes of both CTAs
      mbar_init(&empty[s], 1);  // the pair's MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 4);  // one lane per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  cluster_sync();  // barriers initialised in both CTAs before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();
  const int total = schedule_length(p);
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);

  if (warp == 0) {
    // ------------------------------- TMA producer (both CTAs) -------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = pair; it < total && ok; it += npairs) {
        const Item t = decode_item<BN>(p, it);
        if (!t.valid) {
          if (blockIdx.x == 0) set_status(p.ctrl, MOE_ERR_DEVICE_BOUNDS);
          continue;
        }
        const int arow = (t.sh ? 0 : (t.g - p.g_lo) * p.a_rows_per_group) + t.m * 256 + static_cast<int>(rank) * 128;
        const int brow = t.row0 + static_cast<int>(rank) * C::kBRows;
        for (int kb = 0; kb < p.kblocks[t.sh]; ++kb) {
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, p.ctrl, abort_flag)) { ok = false; break; }
          unsigned char* st = smem + stage * C::kStageBytes;
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
          tma_load_2d_pair(st, &p.tmA[t.sh], kb * kTileK, arow, fb);
          tma_load_2d_pair(st + C::kBOffset, &p.tmB[t.sh], kb * kTileK, brow, fb);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ----------------------------- MMA issuer (even CTA) ----------------------------
      // The whole warp takes the hand-overs of the watcher at named barrier 2 (per tile a
      // free accumulator and tile_code(), per stage the operands of both CTAs) and reads no
      // memory; lane 0 issues.  Pair tiles always run all BN columns.
      const uint32_t idesc = idesc_bf16_f32(256, BN);
      const int kb_routed = p.kblocks[0], kb_shared = p.kblocks[1];  // in registers before any MMA
      int stage = 0, acc = 0;
      for (;;) {
        __syncwarp();
        const uint32_t code = named_bar_popc(2, 64, false);  // accumulator `acc` free
        if (code == 0) break;
        const int kb_n = code > 16 ? kb_shared : kb_routed;
        const uint32_t d0 = tmem_base + acc * C::kAccCols;
        for (int kb = 0; kb < kb_n; ++kb) {
          __syncwarp();
          named_bar_sync(2, 64);  // both CTAs' operands of this stage have landed
          if (lane == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
            const uint32_t b0 = a0 + C::kBOffset;
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              const uint32_t accum = (kb || kk) ? 1u : 0u;
              const uint64_t bdesc = sw128_kmajor_desc(b0 + kk * 32);
              mma_bf16_pair(d0, sw128_kmajor_desc(a0 + kk * 32), bdesc, idesc, accum);
            }
            mma_commit_pair(&empty[stage]);
          }
          if (++stage == C::kStages) stage = 0;
        }
        if (lane == 0) mma_commit_pair(&tfull[acc]);
        if (++acc == C::kAccBufs) acc = 0;
      }
      if (lane == 0) {
        mma_commit_pair(drain);  // every MMA of the pair done before the accumulators are freed
        mbar_wait_drain(drain, 0, p.ctrl);
      }
    }
  } else if (warp == C::kThreads / 32 - 1) {
    if (rank == 0) {
      // ------------------------- stage watcher (even CTA) ------------------------------
      // Walks the same items; waits for each accumulator and stage and hands them to the
      // MMA warp.  After a failed wait (status set) it goes on handing over without
      // waiting, so that the MMA warp reaches the end of the schedule.
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool failed = false;
      for (int it = pair; it < total; it += npairs) {
        const Item t = decode_item<BN>(p, it);
        if (!t.valid) continue;
        if (!failed && !mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, p.ctrl, abort_flag)) failed = true;
        __syncwarp();
        named_bar_popc(2, 64, static_cast<uint32_t>(lane) < tile_code(t));
        for (int kb = 0; kb < p.kblocks[t.sh]; ++kb) {
          if (!failed && !mbar_wait_cluster(&full[stage], phase, p.ctrl, abort_flag)) failed = true;
          __syncwarp();
          named_bar_sync(2, 64);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      __syncwarp();
      named_bar_popc(2, 64, false);  // the end of the schedule
    }
  } else {
    // ------------------------------- epilogue (warps 2..5, both CTAs) -----------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // this CTA's weight row = output column
    const int et = threadIdx.x - 64;
    const uint32_t tempty_even0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_even1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = pair; it < total; it += npairs) {
      const Item t = decode_item<BN>(p, it);
      if (!t.valid) continue;
      for (int n = et; n < BN; n += 128) sw[n] = (t.sh || n >= t.nvalid) ? 1.0f : __ldg(p.row_w + t.row0 + n);
      named_bar_sync(1, 128);
      if (!mbar_wait_cluster(&tfull[acc], acc_phase, p.ctrl, abort_flag)) break;
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * C::kAccCols;
      const int ld = p.ld_out[t.sh];
      __nv_bfloat16* out = p.out[t.sh] + static_cast<int64_t>(t.row0) * ld + t.m * 256 + static_cast<int>(rank) * 128;
      for (int c0 = 0; c0 < t.nvalid; c0 += C::kChunk) {
        uint32_t a[32];
        tmem_ld16_nowait(trow + c0, a);
        tmem_ld16_nowait(trow + c0 + 16, a + 16);
        tmem_wait_ld();
        if (c0 + C::kChunk >= t.nvalid) {  // the accumulator has been read: release it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(acc ? tempty_even1 : tempty_even0);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j)
          staging[j * kTileM + r] = __float2bfloat16_rn(__uint_as_float(a[j]) * sw[c0 + j]);
        named_bar_sync(1, 128);
        // rows of 128 bf16 (256 B) -> out[row0 + c0 + j][...], 16-byte coalesced stores
        const int rows = min(C::kChunk, t.nvalid - c0);
        const uint4* src = reinterpret_cast<const uint4*>(staging);
        for (int i = et; i < rows * 16; i += 128) {
          const int j = i >> 4, cc = i & 15;
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(c0 + j) * ld + cc * 8) = src[j * 16 + cc];
        }
        named_bar_sync(1, 128);  // staging (and sw) free again
      }
      if (++acc == C::kAccBufs) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs may still read its operands
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

// ---------------------------------------------------------------------------------------
// fp32 CUDA-core path
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int group_of_row(const int32_t* offsets, int E, int p) {
  int lo = 0, hi = E - 1;  // last expert e with offsets[e] <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= p) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void gate_up_f32_kernel(const float* __restrict__ x_perm, const float* __restrict__ x,
                                   const int32_t* __restrict__ offsets,
                                   const float* __restrict__ Wgu, const float* __restrict__ Wsgu,
                                   int64_t P, int64_t T, int H, int E, int I, int Is,
                                   float limit, float limit_shared,
                                   float* __restrict__ h, float* __restrict__ hs) {
  const int64_t n_routed = P * I, total = n_routed + T * Is;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float *xr, *wg, *wu;
    float* dst;
    float L = limit;
    if (q < n_routed) {
      const int64_t p = q / I;
      const int i = static_cast<int>(q - p * I);
      const int e = group_of_row(offsets, E, static_cast<int>(p));
      xr = x_perm + p * H;
      wg = Wgu + (static_cast<int64_t>(e) * 2 * I + i) * H;
      wu = wg + static_cast<int64_t>(I) * H;
      dst = h + q;
    } else {
      const int64_t qs = q - n_routed;
      const int64_t t = qs / Is;
      const int i = static_cast<int>(qs - t * Is);
      xr = x + t * H;
      wg = Wsgu + static_cast<int64_t>(i) * H;
      wu = wg + static_cast<int64_t>(Is) * H;
      dst = hs + qs;
      L = limit_shared;
    }
    float g = 0.f, u = 0.f;
    for (int k = 0; k < H; ++k) {
      const float xv = __ldg(xr + k);
      g = fmaf(xv, __ldg(wg + k), g);
      u = fmaf(xv, __ldg(wu + k), u);
    }
    if (L > 0.0f) {
      g = fminf(g, L);
      u = fminf(fmaxf(u, -L), L);
    }
    *dst = g / (1.0f + expf(-g)) * u;
  }
}

__global__ void down_f32_kernel(const float* __restrict__ h, const float* __restrict__ hs,
                                const int32_t* __restrict__ offsets, const float* __restrict__ row_w,
                                const float* __restrict__ Wd, const float* __restrict__ Wsd,
                                int64_t P, int64_t T, int H, int E, int I, int Is,
                                float* __restrict__ o, float* __restrict__ os) {
  const int64_t n_routed = P * H, total = n_routed + (Is > 0 ? T * H : 0);
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float *hr, *wr;
    float scale, *dst;
    int n;
    if (q < n_routed) {
      const int64_t p = q / H;
      const int c = static_cast<int>(q - p * H);
      const int e = group_of_row(offsets, E, static_cast<int>(p));
      hr = h + p * I;
      wr = Wd + (static_cast<int64_t>(e) * H + c) * I;
      scale = row_w[p];
      dst = o + q;
      n = I;
    } else {
      const int64_t qs = q - n_routed;
      const int64_t t = qs / H;
      const int c = static_cast<int>(qs - t * H);
      hr = hs + t * Is;
      wr = Wsd + static_cast<int64_t>(c) * Is;
      scale = 1.0f;
      dst = os + qs;
      n = Is;
    }
    float acc = 0.f;
    for (int i = 0; i < n; ++i) acc = fmaf(__ldg(hr + i), __ldg(wr + i), acc);
    *dst = scale * acc;
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
static bool encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// FP8 code matrix [rows, cols] (bytes): 128-row x 64-byte boxes, no swizzling (the
// converters read the rows and write the swizzled bf16 layout themselves)
static bool encode_2d_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(kTileM)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool GATED, int BN, bool W8>
static cudaError_t launch_tc(const TcParams& prm_in, int num_sms, cudaStream_t st) {
  using C = TcCfg<GATED, BN, W8>;
  auto kern = expert_gemm_tc_kernel<GATED, BN, W8>;
  TcParams prm = prm_in;
  const size_t smem = C::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(num_sms), dim3(C::kThreads), smem, st, prm, prm);
  count_launches(1);
  return e;
}

// both projections of bf16 16-token tiles in one launch (gu: gate/up, dn: down)
static cudaError_t launch_fused(const TcParams& gu, const TcParams& dn, int num_sms, cudaStream_t st) {
  using C = TcCfg<true, 16, false, true>;
  auto kern = expert_gemm_tc_kernel<true, 16, false, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmemBytes));
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(num_sms), dim3(C::kThreads), static_cast<size_t>(C::kSmemBytes), st, gu, dn);
  count_launches(1);
  return e;
}

static cudaError_t launch_pair(const TcParams& prm, int num_sms, cudaStream_t st) {
  using C = PairCfg;
  auto kern = expert_gemm_pair_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, prm);
  count_launches(1);
  return e;
}

template <bool GATED>
static cudaError_t launch_tc_bn(const TcParams& prm, int bn, bool w8, int num_sms, cudaStream_t st) {
  if (w8) {  // FP8 weights: 16- and 128-token tiles
    if (bn == 16) return launch_tc<GATED, 16, true>(prm, num_sms, st);
    return launch_tc<GATED, 128, true>(prm, num_sms, st);
  }
  if (bn == 16) return launch_tc<GATED, 16, false>(prm, num_sms, st);
  if constexpr (!GATED) {
    if (bn == 256) return launch_tc<false, 256, false>(prm, num_sms, st);
  }
  return launch_tc<GATED, 128, false>(prm, num_sms, st);
}

// Upper bound of the tiles of one grouped GEMM whose weight matrices have `rows` rows per
// routed expert and `rows_shared` for the shared one: every touched expert contributes
// ceil(count / bn) token tiles, with at most min(T*k, E) partial ones.
int64_t expert_tile_bound(int64_t T, int k, int E, int rows, int rows_shared, int bn) {
  const int64_t P = T * k;
  const int64_t routed = (P / bn + std::min<int64_t>(P, E) + 1) * (rows / kTileM);
  const int64_t shared = rows_shared ? (T / bn + 1) * (rows_shared / kTileM) : 0;
  return routed + shared + 1;
}

cudaError_t launch_experts(const ExpertArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t P = a.T * a.k;
  const bool has_shared = a.Is > 0;
  if (!a.bf16) {
    const int64_t n1 = P * a.I + (has_shared ? a.T * a.Is : 0);
    gate_up_f32_kernel<<<static_cast<unsigned>(std::min<int64_t>((n1 + 255) / 256, 148 * 32)), 256, 0, st>>>(
        static_cast<const float*>(a.x_perm), static_cast<const float*>(a.x), a.offsets,
        static_cast<const float*>(a.Wgu), static_cast<const float*>(a.Wsgu), P,
        has_shared ? a.T : 0, a.H, a.E, a.I, a.Is, a.swiglu_limit, a.swiglu_limit_shared,
        static_cast<float*>(a.h), static_cast<float*>(a.h_shared));
    count_launches(2);
    if (a.stage_mark) a.stage_mark(a.stage_mark_ctx, 3, st);
    const int64_t n2 = P * a.H + (has_shared ? a.T * a.H : 0);
    down_f32_kernel<<<static_cast<unsigned>(std::min<int64_t>((n2 + 255) / 256, 148 * 32)), 256, 0, st>>>(
        static_cast<const float*>(a.h), static_cast<const float*>(a.h_shared), a.offsets, a.row_w,
        static_cast<const float*>(a.Wd), static_cast<const float*>(a.Wsd), P,
        has_shared ? a.T : 0, a.H, a.E, a.I, a.Is, static_cast<float*>(a.o),
        static_cast<float*>(a.o_shared));
    return cudaGetLastError();
  }
  const int G = a.E + (has_shared ? 1 : 0);
  // gate/up: A = W_gate_up viewed as [E*2I, H]; B = rows of x [T, H] gathered by token
  // (row-gather TMA for 16-token tiles, gather warps for 128-token tiles) or, for FP8 weights
  // with 128-token tiles, x_perm [P, H]; the shared expert's rows are x [T, H] in order
  TcParams g{};
  const bool gather = a.bn == 16;
  // bf16 128-token tiles gather their token rows inside the kernel (no x_perm); FP8 weights
  // read the permuted copy
  const bool cp_gather = a.bn == 128 && !a.w8;
  // token rows per B copy (down pair tiles: each CTA's half)
  const uint32_t box_gu = static_cast<uint32_t>(a.bn);
  const uint32_t box_dn = a.pair_dn ? 128 : static_cast<uint32_t>(a.bn_dn);
  // weight matrices: bf16 rows, or FP8 code rows with their block scales
  auto encode_w = [&](CUtensorMap* m, const void* w, uint64_t rows, uint64_t cols) {
    return a.w8 ? encode_2d_u8(m, w, rows, cols) : encode_2d_bf16(m, w, rows, cols, kTileM);
  };
  const uint64_t n_local = static_cast<uint64_t>(a.e_hi - a.e_lo);  // routed experts held
  bool ok = encode_w(&g.tmA[0], a.Wgu, n_local * 2 * a.I, a.H) &&
            (gather ? encode_2d_bf16(&g.tmB[0], a.x, a.T, a.H, 1)
                    : encode_2d_bf16(&g.tmB[0], cp_gather ? a.x : a.x_perm, cp_gather ? a.T : P, a.H, box_gu));
  if (has_shared)
    ok = ok && encode_w(&g.tmA[1], a.Wsgu, 2ull * a.Is, a.H) &&
         encode_2d_bf16(&g.tmB[1], a.x, a.T, a.H, box_gu);
  else {
    g.tmA[1] = g.tmA[0];
    g.tmB[1] = g.tmB[0];
  }
  if (!ok) return cudaErrorInvalidValue;
  g.item_start = a.item_start_gu;
  g.item_info = a.info_gu;
  g.row_w = a.row_w;
  g.row_tok = a.row_tok;
  g.limit[0] = a.swiglu_limit;
  g.limit[1] = a.swiglu_limit_shared;
  g.gather = gather ? 1 : 0;
  g.x = static_cast<const __nv_bfloat16*>(a.x);
  // bf16 16-token tiles (decode): both projections in one launch, each down tile starting
  // as soon as its group's gate/up tiles are done
  const bool fused = !a.w8 && !a.pair_dn && a.bn == 16 && a.bn_dn == 16 && a.gu_done && a.counts;
  g.gu_done = a.gu_done;
  g.counts = a.counts;
  if (!a.w8 && !a.pair_dn && !fused) {
    g.pf_item_start = a.item_start_dn;
    g.pf_info = a.info_dn;
    g.pf_w[0] = static_cast<const unsigned char*>(a.Wd);
    g.pf_w[1] = static_cast<const unsigned char*>(has_shared ? a.Wsd : a.Wd);
    g.pf_mt = a.H / kTileM;
    g.pf_rows_per_group = a.H;
    g.pf_row_bytes[0] = static_cast<int64_t>(a.I) * 2;
    g.pf_row_bytes[1] = static_cast<int64_t>(a.Is) * 2;
  }
  g.out[0] = static_cast<__nv_bfloat16*>(a.h);
  g.out[1] = static_cast<__nv_bfloat16*>(a.h_shared);
  g.E = a.E;
  g.G = G;
  g.T = a.T;
  g.g_lo = a.e_lo;
  g.g_hi = a.e_hi;
  g.sh_base = static_cast<int>(a.shared_base);
  g.sh_rows = static_cast<int>(a.shared_rows);
  g.kblocks[0] = g.kblocks[1] = a.H / kTileK;
  g.a_rows_per_group = 2 * a.I;
  g.a_up_offset[0] = a.I;
  g.a_up_offset[1] = a.Is;
  g.mt[0] = a.I / kTileM;
  g.mt[1] = a.Is / kTileM;
  g.rows_out[0] = static_cast<int>(P);
  g.rows_out[1] = static_cast<int>(a.T);
  g.ksplit = a.ksplit;
  g.max_tiles = static_cast<int>(expert_tile_bound(a.T, a.k, a.E, a.I, a.Is, a.bn));
  g.max_items = g.max_tiles * a.ksplit;
  g.partial = a.partial;
  g.tile_done = a.tile_done;
  g.item_counter = a.item_counters;
  g.ctrl = a.ctrl;
  g.ld_out[0] = a.I;
  g.ld_out[1] = a.Is;
  g.scaleA[0] = static_cast<const uint8_t*>(a.Wgu_scale);
  g.scaleA[1] = static_cast<const uint8_t*>(a.Wsgu_scale);
  g.s_rows_per_group = 2 * a.I / kTileM;
  g.s_ld[0] = g.s_ld[1] = (a.H + 127) / 128;
  if (!fused) {
    cudaError_t e = launch_tc_bn<true>(g, a.bn, a.w8, a.num_sms, st);
    if (e != cudaSuccess) return e;
    if (a.stage_mark) a.stage_mark(a.stage_mark_ctx, 3, st);
  }
  // down: A = W_down viewed as [E*H, I]; B = h [P, I] (shared: Ws_down [H, Is], h_shared)
  TcParams d{};
  ok = encode_w(&d.tmA[0], a.Wd, n_local * a.H, a.I) &&
       encode_2d_bf16(&d.tmB[0], a.h, P, a.I, box_dn);
  if (has_shared)
    ok = ok && encode_w(&d.tmA[1], a.Wsd, a.H, a.Is) &&
         encode_2d_bf16(&d.tmB[1], a.h_shared, a.T, a.Is, box_dn);
  else {
    d.tmA[1] = d.tmA[0];
    d.tmB[1] = d.tmB[0];
  }
  if (!ok) return cudaErrorInvalidValue;
  d.item_start = a.item_start_dn;
  d.item_info = a.info_dn;
  d.row_w = a.row_w;
  d.out[0] = static_cast<__nv_bfloat16*>(a.o);
  d.out[1] = static_cast<__nv_bfloat16*>(a.o_shared);
  d.ld_out[0] = d.ld_out[1] = a.H;
  d.E = a.E;
  d.G = G;
  d.T = a.T;
  d.g_lo = a.e_lo;
  d.g_hi = a.e_hi;
  d.sh_base = static_cast<int>(a.shared_base);
  d.sh_rows = static_cast<int>(a.shared_rows);
  d.kblocks[0] = a.I / kTileK;
  d.kblocks[1] = has_shared ? a.Is / kTileK : 0;
  d.a_rows_per_group = a.H;
  d.a_up_offset[0] = d.a_up_offset[1] = 0;
  d.mt[0] = d.mt[1] = a.H / kTileM;
  d.rows_out[0] = static_cast<int>(P);
  d.rows_out[1] = static_cast<int>(a.T);
  d.ksplit = 1;
  d.max_tiles = static_cast<int>(expert_tile_bound(a.T, a.k, a.E, a.H, a.Is > 0 ? a.H : 0, a.bn_dn));
  d.max_items = d.max_tiles;
  d.item_counter = a.item_counters + 1;
  d.ctrl = a.ctrl;
  d.scaleA[0] = static_cast<const uint8_t*>(a.Wd_scale);
  d.scaleA[1] = static_cast<const uint8_t*>(a.Wsd_scale);
  d.s_rows_per_group = a.H / kTileM;
  d.s_ld[0] = (a.I + 127) / 128;
  d.s_ld[1] = (a.Is + 127) / 128;
  if (a.pair_dn) {
    d.mt[0] = d.mt[1] = a.H / 256;
    d.max_tiles = static_cast<int>(expert_tile_bound(a.T, a.k, a.E, a.H / 2, a.Is > 0 ? a.H / 2 : 0, 256));
    d.max_items = d.max_tiles;
    return launch_pair(d, a.num_sms, st);
  }
  if (fused) {
    const cudaError_t e = launch_fused(g, d, a.num_sms, st);
    if (e == cudaSuccess && a.stage_mark) a.stage_mark(a.stage_mark_ctx, 3, st);  // no boundary between them
    return e;
  }
  return launch_tc_bn<false>(d, a.bn_dn, a.w8, a.num_sms, st);
}

}  // namespace moe
