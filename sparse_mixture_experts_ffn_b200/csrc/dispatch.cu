// dispatch.cu -- per-expert histogram, exclusive scan, stable permutation of the
// (token, slot) assignments by (expert, token), the tile schedule of the grouped expert
// GEMMs, and the gather of token rows into expert order.
//
// Definitions (the routing of llm-atlas page "Step-3.5-Flash", "Champs bruts du
// config.json": moe_num_experts, moe_top_k): counts[e] = #{(t,j): idx[t,j] = e};
// offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e]; perm[offsets[e] + r] = t*k + j for
// the r-th token (ascending t) routed to e; inv_perm is its inverse.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// block-local histogram of the assignments of kTokBlock tokens
__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int64_t T,
                                                   int k, int E, int32_t* __restrict__ blk_hist,
                                                   Ctrl* ctrl) {
  extern __shared__ int sh_hist[];
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

// exclusive scan of up to 2 * blockDim.x values held two per thread; blockDim.x = 1024
__device__ int block_scan_pair(int v0, int v1, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int v = v0 + v1;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int s = warp_tot[lane];
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    warp_tot[lane] = si - s;
    if (lane == 31) warp_tot[32] = si;
  }
  __syncthreads();
  const int excl = warp_tot[warp] + incl - v;
  total = warp_tot[32];
  __syncthreads();
  return excl;  // exclusive prefix of v0; v1's is excl + v0
}

// One block of 1024 threads: per-expert block prefixes, counts, offsets, LPT group
// order and the tile schedules of both grouped GEMMs.  Group g < E is routed expert g;
// group E (when present) is the shared expert with all T tokens.
__global__ void __launch_bounds__(1024) scan_kernel(
    int64_t T, int k, int E, int nblk, int has_shared, int mt_gu, int mt_gu_shared, int mt_dn,
    int32_t* __restrict__ blk_hist, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ group_order, int32_t* __restrict__ item_start_gu,
    int32_t* __restrict__ item_start_dn, int32_t* __restrict__ counts_user,
    int32_t* __restrict__ offsets_user) {
  __shared__ int cnt[2048];
  __shared__ int order[2048];
  __shared__ int warp_tot[33];
  const int G = E + (has_shared ? 1 : 0);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      const int64_t i = static_cast<int64_t>(b) * E + e;
      const int c = blk_hist[i];
      blk_hist[i] = run;
      run += c;
    }
    cnt[e] = run;
    counts[e] = run;
    if (counts_user) counts_user[e] = run;
  }
  if (has_shared && threadIdx.x == 0) cnt[E] = static_cast<int>(T);
  __syncthreads();
  // offsets over the routed experts
  {
    const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
    const int v0 = i0 < E ? cnt[i0] : 0, v1 = i1 < E ? cnt[i1] : 0;
    int total;
    const int ex = block_scan_pair(v0, v1, warp_tot, total);
    if (i0 < E) offsets[i0] = ex;
    if (i1 < E) offsets[i1] = ex + v0;
    if (offsets_user) {
      if (i0 < E) offsets_user[i0] = ex;
      if (i1 < E) offsets_user[i1] = ex + v0;
    }
    if (threadIdx.x == 0) {
      offsets[E] = total;
      if (offsets_user) offsets_user[E] = total;
    }
  }
  // largest group first: rank by (count desc, index asc)
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int c = cnt[g];
    int r = 0;
    for (int h = 0; h < G; ++h) {
      const int ch = cnt[h];
      r += (ch > c) || (ch == c && h < g);
    }
    order[r] = g;
  }
  __syncthreads();
  for (int r = threadIdx.x; r < G; r += blockDim.x) group_order[r] = order[r];
  // tile counts per group in that order, then their prefix sums
  {
    const int r0 = 2 * threadIdx.x, r1 = r0 + 1;
    auto tiles = [&](int r, bool gu) -> int {
      if (r >= G) return 0;
      const int g = order[r];
      const int nt = (cnt[g] + kTileN - 1) / kTileN;
      const int mt = gu ? (g < E ? mt_gu : mt_gu_shared) : mt_dn;
      return nt * mt;
    };
    int total;
    int a0 = tiles(r0, true), a1 = tiles(r1, true);
    int ex = block_scan_pair(a0, a1, warp_tot, total);
    if (r0 < G) item_start_gu[r0] = ex;
    if (r1 < G) item_start_gu[r1] = ex + a0;
    if (threadIdx.x == 0) item_start_gu[G] = total;
    a0 = tiles(r0, false);
    a1 = tiles(r1, false);
    ex = block_scan_pair(a0, a1, warp_tot, total);
    if (r0 < G) item_start_dn[r0] = ex;
    if (r1 < G) item_start_dn[r1] = ex + a0;
    if (threadIdx.x == 0) item_start_dn[G] = total;
  }
}

// Stable positions: one warp walks its block's assignments in (token, slot) order, 32 at
// a time; equal experts inside a chunk get consecutive positions in lane order.
__global__ void __launch_bounds__(256) permute_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, int64_t T, int k, int E,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ blk_hist,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm, float* __restrict__ row_w,
    int32_t* __restrict__ row_tok, int32_t* __restrict__ perm_user) {
  extern __shared__ int base[];
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    base[e] = offsets[e] + blk_hist[static_cast<int64_t>(blockIdx.x) * E + e];
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const int64_t a0 = static_cast<int64_t>(blockIdx.x) * kTokBlock * k;
  const int64_t a1 = min64(a0 + static_cast<int64_t>(kTokBlock) * k, T * k);
  for (int64_t c = a0; c < a1; c += 32) {
    const int64_t a = c + lane;
    const bool valid = a < a1;
    int e = valid ? idx[a] : -1;
    if (e >= E) e = -1;  // reported by hist_kernel
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (e >= 0) pos = base[e] + rank;
    __syncwarp();
    if (e >= 0 && rank == 0) base[e] += __popc(peers);
    __syncwarp();
    if (e >= 0) {
      perm[pos] = static_cast<int32_t>(a);
      inv_perm[a] = pos;
      row_w[pos] = w[a];
      row_tok[pos] = static_cast<int32_t>(a / k);
      if (perm_user) perm_user[pos] = static_cast<int32_t>(a);
    }
  }
}

// x_perm[pos, :] = x[row_tok[pos], :], 16-byte vectors
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ x, const int32_t* __restrict__ row_tok,
                                   int64_t P, int64_t Tn, int H, T* __restrict__ x_perm,
                                   Ctrl* ctrl) {
  constexpr int V = Vec16<T>::N;
  const int vpr = H / V;
  const int64_t total = P * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = i / vpr;
    const int v = static_cast<int>(i - p * vpr);
    const int64_t t = row_tok[p];
    if (t < 0 || t >= Tn) {
      set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(x + t * H) + v);
    reinterpret_cast<uint4*>(x_perm + p * H)[v] = val;
  }
}

cudaError_t launch_dispatch(const DispatchArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int nblk = static_cast<int>((a.T + kTokBlock - 1) / kTokBlock);
  const size_t smem_e = sizeof(int) * static_cast<size_t>(a.E);
  hist_kernel<<<nblk, 256, smem_e, st>>>(a.idx, a.T, a.k, a.E, a.blk_hist, a.ctrl);
  const int mt_gu = a.I / kTileM;
  const int mt_gu_sh = a.Is / kTileM;
  const int mt_dn = a.H / kTileM;
  scan_kernel<<<1, 1024, 0, st>>>(a.T, a.k, a.E, nblk, a.Is > 0 ? 1 : 0, mt_gu, mt_gu_sh, mt_dn,
                                  a.blk_hist, a.counts, a.offsets, a.group_order, a.item_start_gu,
                                  a.item_start_dn, a.counts_user, a.offsets_user);
  permute_kernel<<<nblk, 256, smem_e, st>>>(a.idx, a.w, a.T, a.k, a.E, a.offsets, a.blk_hist,
                                            a.perm, a.inv_perm, a.row_w, a.row_tok, a.perm_user);
  const int64_t P = a.T * a.k;
  const int64_t vec = P * (a.H / (a.bf16 ? 8 : 4));
  const int blocks = static_cast<int>(std::min<int64_t>((vec + 255) / 256, 148 * 16));
  if (a.bf16)
    gather_rows_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.x), a.row_tok, P, a.T, a.H,
        static_cast<__nv_bfloat16*>(a.x_perm), a.ctrl);
  else
    gather_rows_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(a.x), a.row_tok,
                                                      P, a.T, a.H, static_cast<float*>(a.x_perm),
                                                      a.ctrl);
  count_launches(4);
  return cudaGetLastError();
}

}  // namespace moe
