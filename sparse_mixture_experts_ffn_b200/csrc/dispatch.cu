// dispatch.cu -- per-expert histogram, exclusive scan, stable permutation of the
// (token, slot) assignments by (expert, token), the tile schedule of the grouped expert
// GEMMs, and the gather of token rows into expert order.
//
// Definitions (the routing of llm-atlas page "Step-3.5-Flash", "Champs bruts du
// config.json": moe_num_experts, moe_top_k): counts[e] = #{(t,j): idx[t,j] = e};
// offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e]; perm[offsets[e] + r] = t*k + j for
// the r-th token (ascending t) routed to e; inv_perm is its inverse.
//
// Small batches run one single-block kernel (histogram in shared memory, scans, stable
// placement); large batches a block histogram, a scan kernel and a block-parallel
// placement.  Both then gather the token rows into expert order.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "dispatch_common.cuh"
#include "kernels.h"

namespace moe {

// block-local histogram of the assignments of kTokBlock tokens
__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int64_t T,
                                                   int k, int E, int32_t* __restrict__ blk_hist,
                                                   Ctrl* ctrl) {
  extern __shared__ int sh_hist[];
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh_hist[e] = 0;
  __syncthreads();
  const int64_t a0 = static_cast<int64_t>(blockIdx.x) * kTokBlock * k;
  const int64_t a1 = min64(a0 + static_cast<int64_t>(kTokBlock) * k, T * k);
  for (int64_t a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) {
      set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    atomicAdd(&sh_hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    blk_hist[static_cast<int64_t>(blockIdx.x) * E + e] = sh_hist[e];
}

// One block of 1024 threads: per-expert block prefixes, counts and the schedule.
__global__ void __launch_bounds__(1024) scan_kernel(ScheduleArgs sa, int k, int nblk,
                                                    int32_t* __restrict__ blk_hist,
                                                    int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ counts_user) {
  __shared__ int cnt[2048];
  __shared__ int order[2048];
  __shared__ unsigned long long warp_tot[33];
  __shared__ ScheduleSmem ss;
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  const int E = sa.E;
  // thread e scans the block counts of expert e (loads coalesced across experts), sixteen
  // blocks' counts in flight at a time
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0, b = 0;
    for (; b + 16 <= nblk; b += 16) {
      int v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = blk_hist[static_cast<int64_t>(b + j) * E + e];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        blk_hist[static_cast<int64_t>(b + j) * E + e] = run;
        run += v[j];
      }
    }
    for (; b < nblk; ++b) {
      const int64_t i = static_cast<int64_t>(b) * E + e;
      const int c = blk_hist[i];
      blk_hist[i] = run;
      run += c;
    }
    cnt[e] = run;
    counts[e] = run;
    if (counts_user) counts_user[e] = run;
  }
  if (sa.has_shared && threadIdx.x == 0) cnt[E] = sa.shared_rows;
  __syncthreads();
  build_schedule<true>(sa, cnt, order, warp_tot, ss);  // the tile descriptors: permute_kernel
}

// Placement for large batches: block b owns the assignments of tokens [256b, 256b+256);
// its 8 warps split them into 8 consecutive ranges, count per warp, prefix the counts per
// expert across warps, then place.
constexpr int kPermWarps = 8;

__global__ void __launch_bounds__(32 * kPermWarps) permute_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, int64_t T, int k, int E,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ blk_hist,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm, float* __restrict__ row_w,
    int32_t* __restrict__ row_tok, int32_t* __restrict__ perm_user, const ScheduleArgs sa,
    const int32_t* __restrict__ counts) {
  extern __shared__ int wcnt[];  // [kPermWarps][E], then the schedule tables
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  {
    // the tile descriptors of both GEMMs, spread over every block: first the schedule
    // tables into shared memory (G <= E + 1 groups)
    const int G = E + (sa.has_shared ? 1 : 0);
    int* t_cnt = wcnt + kPermWarps * E;  // [E + 1]
    int* t_off = t_cnt + E + 1;          // [E + 1]
    int* t_order = t_off + E + 1;        // [G]
    int* t_gu = t_order + G;             // [G + 1]
    int* t_dn = t_gu + G + 1;            // [G + 1]
    for (int i = threadIdx.x; i <= E; i += blockDim.x) {
      t_cnt[i] = i < E ? counts[i] : sa.shared_rows;
      t_off[i] = offsets[i];
    }
    for (int i = threadIdx.x; i <= G; i += blockDim.x) {
      if (i < G) t_order[i] = sa.group_order[i];
      t_gu[i] = sa.item_start_gu[i];
      t_dn[i] = sa.item_start_dn[i];
    }
    __syncthreads();
    write_item_tables(sa, t_cnt, t_order, t_off, t_gu, t_dn, blockIdx.x * blockDim.x + threadIdx.x,
                      gridDim.x * blockDim.x);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kTokBlock * k;
  const int64_t b1 = min64(b0 + static_cast<int64_t>(kTokBlock) * k, T * k);
  const int64_t per = (((b1 - b0) + kPermWarps - 1) / kPermWarps + 31) / 32 * 32;
  const int64_t a0 = min64(b0 + warp * per, b1), a1 = min64(a0 + per, b1);
  int* mine = wcnt + warp * E;
  for (int64_t a = a0 + lane; a < a1; a += 32) {
    const int e = idx[a];
    if (e >= 0 && e < E) atomicAdd(&mine[e], 1);
  }
  __syncthreads();
  // per expert: exclusive prefix across warps, offset by the block's base position
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = offsets[e] + blk_hist[static_cast<int64_t>(blockIdx.x) * E + e];
    for (int q = 0; q < kPermWarps; ++q) {
      const int c = wcnt[q * E + e];
      wcnt[q * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  place_assignments(idx, w, a0, a1, k, E, mine, perm, inv_perm, row_w, row_tok, perm_user);
}

// Small batches: histogram, scans, schedule and placement in one block.
template <bool kMany>
__global__ void __launch_bounds__(1024) dispatch_small_kernel(
    ScheduleArgs sa, const int32_t* __restrict__ idx, const float* __restrict__ w, int k,
    int32_t* __restrict__ counts, int32_t* __restrict__ counts_user, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv_perm, float* __restrict__ row_w, int32_t* __restrict__ row_tok,
    int32_t* __restrict__ perm_user, Ctrl* ctrl) {
  __shared__ SmallDispatchSmem sm;
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  dispatch_small_block<kMany>(sa, idx, w, k, counts, counts_user, perm, inv_perm, row_w, row_tok, perm_user, ctrl,
                              sm);
}

// x_perm[pos, :] = x[row_tok[pos], :] for the rows of experts [e_lo, e_hi) (all experts,
// or one rank's range under expert parallelism), 16-byte vectors: one warp per row at a
// time (no per-vector index arithmetic), four vectors in flight per lane
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ x, const int32_t* __restrict__ row_tok,
                                   const int32_t* __restrict__ offsets, int e_lo, int e_hi,
                                   int64_t P, int64_t Tn, int H, T* __restrict__ x_perm,
                                   Ctrl* ctrl) {
  pdl_wait();
  pdl_trigger();  // the next kernel may launch now; it waits for this one to finish
  constexpr int V = Vec16<T>::N;
  const int vpr = H / V;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t p_lo = __ldg(offsets + e_lo), p_hi = __ldg(offsets + e_hi);
  if (p_lo < 0 || p_hi > P || p_lo > p_hi) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
    return;
  }
  for (int64_t p = p_lo + ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5); p < p_hi;
       p += warps) {
    const int64_t t = __ldg(row_tok + p);
    if (t < 0 || t >= Tn) {
      if (lane == 0) set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + p * H);
    int v = lane;
    for (; v + 96 < vpr; v += 128) {
      uint4 r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) r[u] = __ldg(src + v + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u) dst[v + 32 * u] = r[u];
    }
    for (; v < vpr; v += 32) dst[v] = __ldg(src + v);
  }
}


// assignments up to which the single-block path is used
constexpr int64_t kSmallDispatch = 4096;

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t P = a.T * a.k;
  const ScheduleArgs sa = schedule_args(a);
  cudaError_t e;
  int launches = 0;
  if (P <= kSmallDispatch) {
    // tiny batches: 16 warps (shorter block barriers; the scans hold two groups a thread)
    const unsigned nthr = (P <= 64 && a.E + 2 <= 1024) ? 512 : 1024;
    // more than 128 assignments: several placing warps, groups ranked without sorting
    e = launch_pdl(P > 128 ? dispatch_small_kernel<true> : dispatch_small_kernel<false>, dim3(1), dim3(nthr), 0, st,
                   sa, a.idx, a.w, a.k, a.counts, a.counts_user, a.perm, a.inv_perm, a.row_w, a.row_tok, a.perm_user,
                   a.ctrl);
    if (e != cudaSuccess) return e;
    launches = 1;
  } else {
    const int nblk = static_cast<int>((a.T + kTokBlock - 1) / kTokBlock);
    const size_t smem_e = sizeof(int) * static_cast<size_t>(a.E);
    e = launch_pdl(hist_kernel, dim3(nblk), dim3(256), smem_e, st, a.idx, a.T, a.k, a.E, a.blk_hist, a.ctrl);
    if (e != cudaSuccess) return e;
    e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, sa, a.k, nblk, a.blk_hist, a.counts,
                   a.counts_user);
    if (e != cudaSuccess) return e;
    const size_t smem_p = smem_e * kPermWarps + sizeof(int) * (5 * static_cast<size_t>(a.E) + 8);
    if (smem_p > 48 * 1024) {
      e = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_p));
      if (e != cudaSuccess) return e;
    }
    e = launch_pdl(permute_kernel, dim3(nblk), dim3(32 * kPermWarps), smem_p, st, a.idx, a.w, a.T, a.k,
                   a.E, static_cast<const int32_t*>(a.offsets), static_cast<const int32_t*>(a.blk_hist),
                   a.perm, a.inv_perm, a.row_w, a.row_tok, a.perm_user, sa,
                   static_cast<const int32_t*>(a.counts));
    if (e != cudaSuccess) return e;
    launches = 3;
  }
  // bf16 GEMMs gather their token rows from x themselves (16-token tiles: row-gather TMA,
  // four rows per copy; 128-token tiles: gather warps); FP8 weights with 128-token tiles and
  // the fp32 path read a permuted copy
  if (a.bf16 && !a.need_x_perm) {
    count_launches(launches);
    return cudaSuccess;
  }
  const int blocks = static_cast<int>(std::min<int64_t>((P + 7) / 8, 148 * 16));  // a warp per row
  if (a.bf16)
    e = launch_pdl(gather_rows_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                   static_cast<const __nv_bfloat16*>(a.x), static_cast<const int32_t*>(a.row_tok),
                   static_cast<const int32_t*>(a.offsets), a.e_lo, a.e_hi, P, a.T, a.H,
                   static_cast<__nv_bfloat16*>(a.x_perm), a.ctrl);
  else
    e = launch_pdl(gather_rows_kernel<float>, dim3(blocks), dim3(256), 0, st,
                   static_cast<const float*>(a.x), static_cast<const int32_t*>(a.row_tok),
                   static_cast<const int32_t*>(a.offsets), a.e_lo, a.e_hi, P, a.T, a.H,
                   static_cast<float*>(a.x_perm), a.ctrl);
  count_launches(launches + 1);
  return e;
}

}  // namespace moe
