// dispatch_common.cuh -- the device code of the dispatch step shared by the dispatch
// kernels: block scans, the tile schedule of the grouped expert GEMMs and the stable
// placement of the assignments.
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
// of 32, at most 1024); V = unsigned long long scans two 32-bit counts packed in one value
// (high and low halves) at once, as long as the low half's total stays below 2^32
template <typename V>
static __device__ V block_scan_pair(V v0, V v1, V* warp_tot, V& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const V v = v0 + v1;
  V incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const V y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const V s = (lane < static_cast<int>(blockDim.x >> 5)) ? warp_tot[lane] : V(0);  // fewer warps: zeros
    V si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const V y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    warp_tot[lane] = si - s;
    if (lane == 31) warp_tot[32] = si;
  }
  __syncthreads();
  const V excl = warp_tot[warp] + incl - v;
  total = warp_tot[32];
  __syncthreads();
  return excl;  // exclusive prefix of v0; v1's is excl + v0
}

// log2 of a power of two (token tile widths 16, 128, 256 and reduction splits 1, 2, 4 are),
// so that tile counts and item coordinates take shifts and masks instead of divisions
__device__ __forceinline__ int log2_pow2(int x) { return __ffs(x) - 1; }

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
// of the reduction).  One block with 2 * blockDim.x >= G + 1 and blockDim.x / 64 a power
// of two; cnt/order in shared memory, and the offsets and prefixes also kept in ss for the
// descriptor writers.  Returns the number of groups with rows (they lead the order).
template <bool kWideRank>
static __device__ int build_schedule(const ScheduleArgs& a, int* cnt, int* order, unsigned long long* warp_tot,
                                     ScheduleSmem& ss) {
  using u64 = unsigned long long;
  const int E = a.E, G = E + (a.has_shared ? 1 : 0);
  const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
  // one scan for the routed offsets (low halves: the counts, whose total T*k < 2^31) and the
  // places of the groups with rows (high halves: 1 per such group)
  const int z0 = (i0 < G && cnt[i0] > 0) ? 1 : 0, z1 = (i1 < G && cnt[i1] > 0) ? 1 : 0;
  int nz_ex, nnz;
  {
    const u64 v0 = (static_cast<u64>(z0) << 32) | static_cast<uint32_t>(i0 < E ? cnt[i0] : 0);
    const u64 v1 = (static_cast<u64>(z1) << 32) | static_cast<uint32_t>(i1 < E ? cnt[i1] : 0);
    u64 tot;
    const u64 ex64 = block_scan_pair(v0, v1, warp_tot, tot);
    const int ex = static_cast<int>(ex64 & 0xFFFFFFFFu), total = static_cast<int>(tot & 0xFFFFFFFFu);
    nz_ex = static_cast<int>(ex64 >> 32);
    nnz = static_cast<int>(tot >> 32);
    const int c0 = static_cast<int>(v0 & 0xFFFFFFFFu);
    if (i0 < E) a.offsets[i0] = ss.off[i0] = ex;
    if (i1 < E) a.offsets[i1] = ss.off[i1] = ex + c0;
    if (a.offsets_user) {
      if (i0 < E) a.offsets_user[i0] = ex;
      if (i1 < E) a.offsets_user[i1] = ex + c0;
    }
    if (threadIdx.x == 0) {
      a.offsets[E] = ss.off[E] = total;
      if (a.offsets_user) a.offsets_user[E] = total;
    }
  }
  // largest group first: order by (count desc, index asc), groups without rows last in
  // index order.  Keys ~count << 32 | index rank the groups with rows.  Up to blockDim.x of
  // them (kWideRank; else up to 64): compacted into a list, each key ranked by blockDim.x / span threads (span: the
  // next power of two >= their number, at least 64) that compare it with a share of the
  // others and add their counts; more: one ascending bitonic sort of every group's key over
  // the next power of two >= G, padded with keys above every real one.
  auto key_of = [&](int g) -> u64 {
    return (static_cast<u64>(~static_cast<uint32_t>(cnt[g])) << 32) | static_cast<uint32_t>(g);
  };
  if (nnz <= (kWideRank ? static_cast<int>(blockDim.x) : 64)) {
    u64* ckey = reinterpret_cast<u64*>(ss.istart_gu);  // written only after the ranking
    if (z0) ckey[nz_ex] = key_of(i0);
    if (z1) ckey[nz_ex + z0] = key_of(i1);
    if (i0 < G && !z0) order[nnz + (i0 - nz_ex)] = i0;
    if (i1 < G && !z1) order[nnz + (i1 - nz_ex - z0)] = i1;
    __syncthreads();
    // span: a power of two >= nnz (at least 64); parts = blockDim / span threads per key
    // (blockDim.x is a power of two), each comparing its key with ceil(nnz / parts) others
    int span = 64;
    while (span < nnz) span <<= 1;
    const int parts = static_cast<int>(blockDim.x) / span, per = (nnz + parts - 1) / parts;
    const int slot = static_cast<int>(threadIdx.x) / parts, part = static_cast<int>(threadIdx.x) - slot * parts;
    int r = 0;
    u64 kg = 0;
    if (slot < nnz) {
      kg = ckey[slot];
      if (kWideRank) {
        const int h1 = min(nnz, (part + 1) * per);
#pragma unroll 4
        for (int h = part * per; h < h1; ++h) r += (ckey[h] < kg) ? 1 : 0;
      } else {  // at most 64 keys: a fixed share of 64 / parts slots each
        const int per64 = 64 / parts;
        for (int q = 0; q < per64; ++q) {
          const int h = part * per64 + q;
          r += (h < nnz && ckey[h] < kg) ? 1 : 0;
        }
      }
    }
    for (int o = parts >> 1; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    if (slot < nnz && part == 0) order[r] = static_cast<int>(kg & 0xFFFFFFFFu);
    __syncthreads();
  } else {
    // [n <= 2048] keys in the prefix arrays, which are written only after the sort
    u64* key = reinterpret_cast<u64*>(ss.istart_gu);
    int n = 1;
    while (n < G) n <<= 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) key[i] = i < G ? key_of(i) : ~0ull;
    __syncthreads();
    for (int size = 2; size <= n; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
          // pair (i, i + stride) of the stride-sized half blocks; ascending where i & size is 0
          const int i = 2 * t - (t & (stride - 1));
          const u64 x = key[i], y = key[i + stride];
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
  for (int r = threadIdx.x; r < G; r += blockDim.x) a.group_order[r] = order[r];
  // tiles of group slot r in each GEMM; one scan for both (gate/up high, down low halves)
  auto tiles = [&](int r, bool gu) -> int {
    if (r >= G) return 0;
    const int g = order[r];
    const int bn = gu ? a.bn : a.bn_dn;
    if (g < E && (g < a.e_lo || g >= a.e_hi)) return 0;  // another rank's expert
    const int nt = (cnt[g] + bn - 1) >> log2_pow2(bn);
    const int mt = gu ? (g < E ? a.mt_gu : a.mt_gu_shared) * a.ksplit : a.mt_dn;
    return nt * mt;
  };
  const int r0 = i0, r1 = i1;
  const int gu0 = tiles(r0, true), gu1 = tiles(r1, true);
  const u64 v0 = (static_cast<u64>(gu0) << 32) | static_cast<uint32_t>(tiles(r0, false));
  const u64 v1 = (static_cast<u64>(gu1) << 32) | static_cast<uint32_t>(tiles(r1, false));
  u64 tot;
  const u64 ex64 = block_scan_pair(v0, v1, warp_tot, tot);
  const int ex_gu = static_cast<int>(ex64 >> 32), ex_dn = static_cast<int>(ex64 & 0xFFFFFFFFu);
  const int dn0 = static_cast<int>(v0 & 0xFFFFFFFFu);
  if (r0 < G) {
    a.item_start_gu[r0] = ss.istart_gu[r0] = ex_gu;
    a.item_start_dn[r0] = ss.istart_dn[r0] = ex_dn;
  }
  if (r1 < G) {
    a.item_start_gu[r1] = ss.istart_gu[r1] = ex_gu + gu0;
    a.item_start_dn[r1] = ss.istart_dn[r1] = ex_dn + dn0;
  }
  if (threadIdx.x == 0) {
    a.item_start_gu[G] = ss.istart_gu[G] = static_cast<int>(tot >> 32);
    a.item_start_dn[G] = ss.istart_dn[G] = static_cast<int>(tot & 0xFFFFFFFFu);
  }
  return nnz;
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
      const int ntile = (rows + bn - 1) >> log2_pow2(bn);  // >= 1: groups without rows have no items
      if (ntile < 1) {  // inconsistent prefixes: an invalid descriptor, reported by the GEMM
        info[it] = make_int4(-1, 0, 0, 0);
        continue;
      }
      const int l = it - istart[lo];
      const int tile = l >> log2_pow2(ks_n), ks = l & (ks_n - 1);
      const int m = ntile == 1 ? tile : tile / ntile, n = tile - m * ntile;
      const int row0 = (g < E ? off[g] : 0) + n * bn;
      info[it] = make_int4(g, m, row0, min(bn, rows - n * bn) | (ks << 16));
    }
  }
}

// The same descriptors written by one block, a warp per (GEMM, group slot) with its lanes
// over the slot's items: no search.  Only the first nslots slots of the order have items
// (the groups with rows).
static __device__ void write_item_tables_by_slot(const ScheduleArgs& a, const int* cnt, const int* order,
                                                 const int* off, const int* istart_gu, const int* istart_dn,
                                                 int nslots) {
  const int E = a.E, G = E + (a.has_shared ? 1 : 0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = static_cast<int>(blockDim.x >> 5);
  const bool ok_gu = istart_gu[G] <= a.cap_gu, ok_dn = istart_dn[G] <= a.cap_dn;
  if ((!ok_gu || !ok_dn) && threadIdx.x == 0) set_status(a.ctrl, MOE_ERR_DEVICE_BOUNDS);  // the GEMM runs nothing
  for (int job = warp; job < 2 * nslots; job += nwarps) {
    const int which = job >= nslots ? 1 : 0, r = job - which * nslots;
    if (!(which ? ok_dn : ok_gu)) continue;
    const int* istart = which ? istart_dn : istart_gu;
    int4* info = which ? a.info_dn : a.info_gu;
    const int bn = which ? a.bn_dn : a.bn;
    const int ks_n = which ? 1 : a.ksplit;
    const int i0 = istart[r], n_items = istart[r + 1] - i0;
    if (n_items <= 0) continue;
    const int g = order[r], rows = cnt[g];
    const int ntile = (rows + bn - 1) >> log2_pow2(bn);
    const int rbase = g < E ? off[g] : 0;
    const int ksh = log2_pow2(ks_n);
    for (int l = lane; l < n_items; l += 32) {
      if (ntile < 1) {  // inconsistent prefixes: an invalid descriptor, reported by the GEMM
        info[i0 + l] = make_int4(-1, 0, 0, 0);
        continue;
      }
      const int tile = l >> ksh, ks = l & (ks_n - 1);
      const int m = ntile == 1 ? tile : tile / ntile, n = tile - m * ntile;  // one token tile: no division
      info[i0 + l] = make_int4(g, m, rbase + n * bn, min(bn, rows - n * bn) | (ks << 16));
    }
  }
}

// Stable placement of the assignments [a0, a1) by one warp, 32 at a time, in (token,
// slot) order: equal experts inside a chunk get consecutive positions in lane order.
// base[e] holds the next free position of expert e and is advanced.  The indices and weights
// of four chunks are loaded before the first of them is placed; those of the lane's first
// assignment (a0 + lane) may come loaded already (e_first / w_first, when have_first).
static __device__ void place_assignments(const int32_t* __restrict__ idx, const float* __restrict__ w,
                                  int64_t a0, int64_t a1, int k, int E, int* base,
                                  int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
                                  float* __restrict__ row_w, int32_t* __restrict__ row_tok,
                                  int32_t* __restrict__ perm_user, bool have_first = false,
                                  int e_first = 0, float w_first = 0.0f) {
  const int lane = threadIdx.x & 31;
  constexpr int kAhead = 4;
  for (int64_t c0 = a0; c0 < a1; c0 += 32 * kAhead) {
    int ev[kAhead];
    float wv[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int64_t a = c0 + 32 * u + lane;
      const bool pre = have_first && c0 == a0 && u == 0;
      ev[u] = (a < a1) ? (pre ? e_first : idx[a]) : -1;
      wv[u] = (a < a1) ? (pre ? w_first : w[a]) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      if (c0 + 32 * u >= a1) break;  // no assignments left (the same for every lane)
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
  unsigned long long warp_tot[33];
  ScheduleSmem sched;
};

// The whole dispatch of a small batch by one block (2 * blockDim.x >= G + 1): histogram,
// counts, offsets, the tile schedule and descriptors, then the stable placement (one warp).
// kMany (more than 128 assignments): several warps place the assignments, and up to
// blockDim.x groups with rows are ranked without sorting.
template <bool kMany>
static __device__ void dispatch_small_block(const ScheduleArgs& sa, const int32_t* __restrict__ idx,
                                            const float* __restrict__ w, int k, int32_t* __restrict__ counts,
                                            int32_t* __restrict__ counts_user, int32_t* __restrict__ perm,
                                            int32_t* __restrict__ inv_perm, float* __restrict__ row_w,
                                            int32_t* __restrict__ row_tok, int32_t* __restrict__ perm_user,
                                            Ctrl* ctrl, SmallDispatchSmem& sm) {
  const int E = sa.E;
  const int64_t P = sa.T * k;
  // this thread's first assignment (and, for the placing warp, its weight), requested before
  // the counters are cleared
  const bool has_first = static_cast<int64_t>(threadIdx.x) < P;
  const int e_first = has_first ? idx[threadIdx.x] : 0;
  const float w_first = (has_first && threadIdx.x < 32) ? w[threadIdx.x] : 0.0f;
  for (int e = threadIdx.x; e < E + 1; e += blockDim.x) sm.cnt[e] = 0;
  __syncthreads();
  for (int64_t a = threadIdx.x; a < P; a += blockDim.x) {
    const int e = (a == threadIdx.x) ? e_first : idx[a];
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
  const int nnz = build_schedule<kMany>(sa, sm.cnt, sm.order, sm.warp_tot, sm.sched);
  __syncthreads();
  // few groups with rows: a warp per group slot; many: items spread evenly over the threads
  if (nnz <= 64)
    write_item_tables_by_slot(sa, sm.cnt, sm.order, sm.sched.off, sm.sched.istart_gu, sm.sched.istart_dn, nnz);
  else
    write_item_tables(sa, sm.cnt, sm.order, sm.sched.off, sm.sched.istart_gu, sm.sched.istart_dn, threadIdx.x,
                      blockDim.x);
  for (int e = threadIdx.x; e < E; e += blockDim.x) sm.base[e] = sm.sched.off[e];
  __syncthreads();
  if (!kMany) {
    if (threadIdx.x < 32)
      place_assignments(idx, w, 0, P, k, E, sm.base, perm, inv_perm, row_w, row_tok, perm_user, true, e_first,
                        w_first);
    return;
  }
  // larger batches: W warps place consecutive ranges of the assignments, each from its own
  // per-expert bases (the experts' offsets plus the counts of the earlier ranges), in the
  // schedule tables' shared memory, free by now
  constexpr int kScratch = static_cast<int>(sizeof(ScheduleSmem) / sizeof(int));
  const int W = min(static_cast<int>(blockDim.x >> 5), min(8, kScratch / E));
  int* wb = reinterpret_cast<int*>(&sm.sched);  // [W][E]: counts, then bases
  const int64_t per = ((P + W - 1) / W + 31) / 32 * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < W * E; i += blockDim.x) wb[i] = 0;
  __syncthreads();
  if (warp < W) {
    const int64_t a0 = min64(warp * per, P), a1 = min64(a0 + per, P);
    for (int64_t a = a0 + lane; a < a1; a += 32) {
      const int e = idx[a];
      if (e >= 0 && e < E) atomicAdd(&wb[warp * E + e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = sm.base[e];
    for (int q = 0; q < W; ++q) {
      const int c = wb[q * E + e];
      wb[q * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  if (warp < W) {
    const int64_t a0 = min64(warp * per, P), a1 = min64(a0 + per, P);
    place_assignments(idx, w, a0, a1, k, E, wb + warp * E, perm, inv_perm, row_w, row_tok, perm_user);
  }
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
