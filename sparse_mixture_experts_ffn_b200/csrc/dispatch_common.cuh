// dispatch_common.cuh -- the device code of the dispatch step shared by the dispatch
// kernels and the fused small-batch routing kernel: block scans, the tile schedule of the
// grouped expert GEMMs and the stable placement of the assignments.
//
// Definitions (the routing of llm-atlas page "Step-3.5-Flash", "Champs bruts du
// config.json": moe_num_experts, moe_top_k): counts[e] = #{(t,j): idx[t,j] = e};
// offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e]; perm[offsets[e] + r] = t*k + j for
// the r-th token (ascending t) routed to e; inv_perm is its inverse.
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// exclusive scan of up to 2 * blockDim.x values held two per thread (blockDim.x a multiple
// of 32, at most 1024)
static __device__ int block_scan_pair(int v0, int v1, int* warp_tot, int& total) {
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
    const int s = (lane < static_cast<int>(blockDim.x >> 5)) ? warp_tot[lane] : 0;  // fewer warps: zeros
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

struct ScheduleArgs {
  int64_t T;
  int E, has_shared, mt_gu, mt_gu_shared, mt_dn, bn, bn_dn, ksplit;
  int e_lo, e_hi;   // routed experts that get tiles (expert parallelism: this rank's range)
  int shared_rows;  // rows of the shared-expert group
  int32_t* offsets;
  int32_t* group_order;
  int32_t* item_start_gu;
  int32_t* item_start_dn;
  int32_t* offsets_user;
  // one descriptor per tile of each grouped GEMM, in schedule order (see write_item_tables)
  int4* info_gu;
  int4* info_dn;
  int cap_gu, cap_dn;  // their capacities (host bounds of the schedule lengths)
  Ctrl* ctrl;
};

// shared-memory scratch of build_schedule / write_item_tables (groups G <= 2048)
struct __align__(16) ScheduleSmem {
  int istart_gu[2049];  // istart_gu and istart_dn (contiguous) also hold the sort keys
  int istart_dn[2049];
  int off[2049];
};
static_assert(sizeof(int) * 2 * 2049 >= sizeof(unsigned long long) * 2048, "room for the sort keys");

// From the group sizes cnt[0..G) (routed experts, then the shared expert with all T
// tokens): offsets of the routed experts, the largest-first group order and the tile
// prefix sums of both grouped GEMMs (gate/up tiles counted ksplit times, once per slice
// of the reduction).  One block with 2 * blockDim.x >= G + 1; cnt/order in shared memory,
// and the offsets and prefixes also kept in ss for write_item_tables.
static __device__ void build_schedule(const ScheduleArgs& a, int* cnt, int* order, int* warp_tot,
                                      ScheduleSmem& ss) {
  const int E = a.E, G = E + (a.has_shared ? 1 : 0);
  {
    const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
    const int v0 = i0 < E ? cnt[i0] : 0, v1 = i1 < E ? cnt[i1] : 0;
    int total;
    const int ex = block_scan_pair(v0, v1, warp_tot, total);
    if (i0 < E) a.offsets[i0] = ss.off[i0] = ex;
    if (i1 < E) a.offsets[i1] = ss.off[i1] = ex + v0;
    if (a.offsets_user) {
      if (i0 < E) a.offsets_user[i0] = ex;
      if (i1 < E) a.offsets_user[i1] = ex + v0;
    }
    if (threadIdx.x == 0) {
      a.offsets[E] = ss.off[E] = total;
      if (a.offsets_user) a.offsets_user[E] = total;
    }
  }
  // largest group first: order by (count desc, index asc), groups without rows last in
  // index order.  The groups with rows are first compacted (in index order) into the leading
  // places of order[], the others after them.  Few groups with rows (small batches): each
  // is ranked by a count over the others; many: one ascending bitonic sort of the keys
  // (~count << 32 | index) over the next power of two >= G, padded with keys above every
  // real one, two keys a thread.
  {
    const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
    const int z0 = (i0 < G && cnt[i0] > 0) ? 1 : 0, z1 = (i1 < G && cnt[i1] > 0) ? 1 : 0;
    int nnz;
    const int nz_ex = block_scan_pair(z0, z1, warp_tot, nnz);
    if (nnz <= 64) {
      if (i0 < G) order[z0 ? nz_ex : nnz + (i0 - nz_ex)] = i0;
      if (i1 < G) order[z1 ? nz_ex + z0 : nnz + (i1 - nz_ex - z0)] = i1;
      __syncthreads();
      auto rank_of = [&](int g) {
        const int c = cnt[g];
        int r = 0;
        for (int j = 0; j < nnz; ++j) {
          const int h = order[j];
          const int ch = cnt[h];
          r += (ch > c) || (ch == c && h < g);
        }
        return r;
      };
      const int r0 = z0 ? rank_of(i0) : -1, r1 = z1 ? rank_of(i1) : -1;
      __syncthreads();
      if (r0 >= 0) order[r0] = i0;
      if (r1 >= 0) order[r1] = i1;
      __syncthreads();
    } else {
      // [n <= 2048] keys in the prefix arrays, which are written only after the sort
      unsigned long long* key = reinterpret_cast<unsigned long long*>(ss.istart_gu);
      int n = 1;
      while (n < G) n <<= 1;
      for (int i = threadIdx.x; i < n; i += blockDim.x)
        key[i] = i < G ? (static_cast<unsigned long long>(~static_cast<uint32_t>(cnt[i])) << 32) |
                             static_cast<uint32_t>(i)
                       : ~0ull;
      __syncthreads();
      for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
            // pair (i, i + stride) of the stride-sized half blocks; ascending where i & size is 0
            const int i = 2 * t - (t & (stride - 1));
            const unsigned long long x = key[i], y = key[i + stride];
            const bool up = (i & size) == 0;
            if ((x > y) == up) {
              key[i] = y;
              key[i + stride] = x;
            }
          }
          __syncthreads();
        }
      }
      for (int i = threadIdx.x; i < G; i += blockDim.x) order[i] = static_cast<int>(key[i] & 0xFFFFFFFFu);
      __syncthreads();
    }
  }
  for (int r = threadIdx.x; r < G; r += blockDim.x) a.group_order[r] = order[r];
  const int r0 = 2 * threadIdx.x, r1 = r0 + 1;
  auto tiles = [&](int r, bool gu) -> int {
    if (r >= G) return 0;
    const int g = order[r];
    const int bn = gu ? a.bn : a.bn_dn;
    if (g < E && (g < a.e_lo || g >= a.e_hi)) return 0;  // another rank's expert
    const int nt = (cnt[g] + bn - 1) / bn;
    const int mt = gu ? (g < E ? a.mt_gu : a.mt_gu_shared) * a.ksplit : a.mt_dn;
    return nt * mt;
  };
  int total;
  int a0 = tiles(r0, true), a1 = tiles(r1, true);
  int ex = block_scan_pair(a0, a1, warp_tot, total);
  if (r0 < G) a.item_start_gu[r0] = ss.istart_gu[r0] = ex;
  if (r1 < G) a.item_start_gu[r1] = ss.istart_gu[r1] = ex + a0;
  if (threadIdx.x == 0) a.item_start_gu[G] = ss.istart_gu[G] = total;
  a0 = tiles(r0, false);
  a1 = tiles(r1, false);
  ex = block_scan_pair(a0, a1, warp_tot, total);
  if (r0 < G) a.item_start_dn[r0] = ss.istart_dn[r0] = ex;
  if (r1 < G) a.item_start_dn[r1] = ss.istart_dn[r1] = ex + a0;
  if (threadIdx.x == 0) a.item_start_dn[G] = ss.istart_dn[G] = total;
}

// One descriptor per tile of a grouped GEMM, so that a GEMM role finds its tile with one
// load instead of searching the group prefixes: item `it` of group slot r (group g =
// order[r], items [istart[r], istart[r + 1])) is local tile l = it - istart[r]; slice
// ks = l % ksplit, weight tile m = (l / ksplit) / ntile, token tile n = (l / ksplit) % ntile
// with ntile = ceil(cnt[g] / bn).  Stored {g, m, first row, rows | ks << 16}; the first
// row of a shared-expert tile is relative to that group's first row.  Threads t0, t0 +
// stride, ... of the caller write the items of both GEMMs; the tables (cnt[E] = rows of the
// shared group, off = routed offsets, the prefixes) come from build_schedule.
static __device__ void write_item_tables(const ScheduleArgs& a, const int* cnt, const int* order,
                                         const int* off, const int* istart_gu, const int* istart_dn,
                                         int t0, int stride) {
  const int E = a.E, G = E + (a.has_shared ? 1 : 0);
  for (int which = 0; which < 2; ++which) {
    const int* istart = which ? istart_dn : istart_gu;
    int4* info = which ? a.info_dn : a.info_gu;
    const int cap = which ? a.cap_dn : a.cap_gu;
    const int bn = which ? a.bn_dn : a.bn;
    const int ks_n = which ? 1 : a.ksplit;
    const int total = istart[G];
    if (total > cap) {  // the GEMM reports it too and runs nothing
      if (t0 == 0) set_status(a.ctrl, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    for (int it = t0; it < total; it += stride) {
      int lo = 0, hi = G - 1;
      while (lo < hi) {  // last group slot whose first item is <= it
        const int mid = (lo + hi + 1) >> 1;
        if (istart[mid] <= it) lo = mid; else hi = mid - 1;
      }
      const int g = order[lo];
      const int rows = cnt[g];
      const int ntile = (rows + bn - 1) / bn;  // >= 1: groups without rows have no items
      if (ntile < 1) {  // inconsistent prefixes: an invalid descriptor, reported by the GEMM
        info[it] = make_int4(-1, 0, 0, 0);
        continue;
      }
      const int l = it - istart[lo];
      const int tile = l / ks_n, ks = l - tile * ks_n;
      const int m = tile / ntile, n = tile - m * ntile;
      const int row0 = (g < E ? off[g] : 0) + n * bn;
      info[it] = make_int4(g, m, row0, min(bn, rows - n * bn) | (ks << 16));
    }
  }
}

// Stable placement of the assignments [a0, a1) by one warp, 32 at a time, in (token,
// slot) order: equal experts inside a chunk get consecutive positions in lane order.
// base[e] holds the next free position of expert e and is advanced.  The indices and weights
// of four chunks are loaded before the first of them is placed.
static __device__ void place_assignments(const int32_t* __restrict__ idx, const float* __restrict__ w,
                                  int64_t a0, int64_t a1, int k, int E, int* base,
                                  int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
                                  float* __restrict__ row_w, int32_t* __restrict__ row_tok,
                                  int32_t* __restrict__ perm_user) {
  const int lane = threadIdx.x & 31;
  constexpr int kAhead = 4;
  for (int64_t c0 = a0; c0 < a1; c0 += 32 * kAhead) {
    int ev[kAhead];
    float wv[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int64_t a = c0 + 32 * u + lane;
      ev[u] = (a < a1) ? idx[a] : -1;
      wv[u] = (a < a1) ? w[a] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int64_t a = c0 + 32 * u + lane;
      int e = ev[u];
      if (e < 0 || e >= E) e = -1;  // reported by the histogram
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
        row_w[pos] = wv[u];
        row_tok[pos] = static_cast<int32_t>(a / k);
        if (perm_user) perm_user[pos] = static_cast<int32_t>(a);
      }
    }
  }
}

// shared memory of the single-block dispatch
struct SmallDispatchSmem {
  int cnt[2048];
  int order[2048];
  int base[1024];
  int warp_tot[33];
  ScheduleSmem sched;
};

// The whole dispatch of a small batch by one block (2 * blockDim.x >= G + 1): histogram,
// counts, offsets, the tile schedule and descriptors, then the stable placement (one warp).
static __device__ void dispatch_small_block(const ScheduleArgs& sa, const int32_t* __restrict__ idx,
                                            const float* __restrict__ w, int k, int32_t* __restrict__ counts,
                                            int32_t* __restrict__ counts_user, int32_t* __restrict__ perm,
                                            int32_t* __restrict__ inv_perm, float* __restrict__ row_w,
                                            int32_t* __restrict__ row_tok, int32_t* __restrict__ perm_user,
                                            Ctrl* ctrl, SmallDispatchSmem& sm) {
  const int E = sa.E;
  const int64_t P = sa.T * k;
  for (int e = threadIdx.x; e < E + 1; e += blockDim.x) sm.cnt[e] = 0;
  __syncthreads();
  for (int64_t a = threadIdx.x; a < P; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) {
      set_status(ctrl, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    atomicAdd(&sm.cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    counts[e] = sm.cnt[e];
    if (counts_user) counts_user[e] = sm.cnt[e];
  }
  if (sa.has_shared && threadIdx.x == 0) sm.cnt[E] = sa.shared_rows;
  __syncthreads();
  build_schedule(sa, sm.cnt, sm.order, sm.warp_tot, sm.sched);
  __syncthreads();
  write_item_tables(sa, sm.cnt, sm.order, sm.sched.off, sm.sched.istart_gu, sm.sched.istart_dn, threadIdx.x,
                    blockDim.x);
  for (int e = threadIdx.x; e < E; e += blockDim.x) sm.base[e] = sm.sched.off[e];
  __syncthreads();
  if (threadIdx.x < 32)
    place_assignments(idx, w, 0, P, k, E, sm.base, perm, inv_perm, row_w, row_tok, perm_user);
}

// The schedule arguments of a dispatch (tile shapes of both grouped GEMMs).
inline ScheduleArgs schedule_args(const DispatchArgs& a) {
  ScheduleArgs sa{};
  sa.T = a.T;
  sa.E = a.E;
  sa.has_shared = a.Is > 0 ? 1 : 0;
  const int tm_dn = a.pair_dn ? 2 * kTileM : kTileM;
  sa.mt_gu = a.I / kTileM;
  sa.mt_gu_shared = a.Is / kTileM;
  sa.mt_dn = a.H / tm_dn;
  sa.bn = a.bn;
  sa.bn_dn = a.pair_dn ? 256 : a.bn_dn;
  sa.ksplit = a.ksplit;
  sa.e_lo = a.e_lo;
  sa.e_hi = a.e_hi;
  sa.shared_rows = a.shared_rows;
  sa.offsets = a.offsets;
  sa.group_order = a.group_order;
  sa.item_start_gu = a.item_start_gu;
  sa.item_start_dn = a.item_start_dn;
  sa.offsets_user = a.offsets_user;
  sa.info_gu = a.info_gu;
  sa.info_dn = a.info_dn;
  sa.cap_gu = a.cap_gu;
  sa.cap_dn = a.cap_dn;
  sa.ctrl = a.ctrl;
  return sa;
}

}  // namespace moe
