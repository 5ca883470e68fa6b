// The routing plan of A <= kSmallMaxA assignments built by one CTA of 1024
// threads in shared memory (glm5next_mlp module docs, MOE_MODULE: the token
// sort): counts, offsets, 256-row tile offsets and the active list of the
// local experts, the stable sorted order, its inverse and each active
// expert's first assignment. Used by the small-A permute and by the fused
// top-k + plan kernel of the decode path.
#pragma once

#include <climits>

#include "common.cuh"

namespace rnx {

constexpr int kSmallMaxA = 1024;   // a power of two (the bitonic sort below)
constexpr int kMaxE = 1024;
// up to this many assignments the stable rank is a count over the earlier
// ones (A steps per thread); above, a bitonic sort (log2^2 kSmallMaxA / 2 steps)
constexpr int kSmallRankA = 256;

// Block-wide exclusive scan of up to blockDim.x (multiple of 32, <= 1024)
// values, one per thread; returns the exclusive prefix, *total gets the sum.
RNX_DEVICE int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? s_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nw) s_warp[lane] = wi - w;
    if (lane == 31) s_warp[32] = wi;
  }
  __syncthreads();
  const int res = inc - v + s_warp[warp];
  if (total) *total = s_warp[32];
  __syncthreads();
  return res;
}

// counts -> offsets, tile_offsets, active (one CTA of 1024 threads, E <= 1024);
// the offsets and the active list also land in shared memory (s_off[E],
// s_act[1 + E], count first), so that later steps need no global read-back.
RNX_DEVICE void finish_plan(const int* s_cnt, int E, int lb, int le, const moe_plan_t& plan, int* s_warp, int* s_off,
                            int* s_act) {
  const int e = threadIdx.x;
  const int c = e < E ? s_cnt[e] : 0;
  const bool local = e >= lb && e < le;
  int tot;
  const int off = block_exclusive_scan(c, s_warp, &tot);
  const int tiles = (local && e < E) ? (c + kRowsPerTile - 1) / kRowsPerTile : 0;
  int ttot;
  const int toff = block_exclusive_scan(tiles, s_warp, &ttot);
  const int act = (local && e < E && c > 0) ? 1 : 0;
  int atot;
  const int aoff = block_exclusive_scan(act, s_warp, &atot);
  if (e < E) {
    plan.counts[e] = c;
    plan.offsets[e] = off;
    plan.tile_offsets[e] = toff;
    s_off[e] = off;
    if (act) {
      plan.active[1 + aoff] = e;
      s_act[1 + aoff] = e;
    }
  }
  if (e == 0) {
    plan.offsets[E] = tot;
    plan.tile_offsets[E] = ttot;
    plan.active[0] = atot;
    s_act[0] = atot;
  }
}

// first[u] = sorted[offsets[e]] for the u-th active (local, non-empty) expert
// e, from the shared copies of offsets, the active list and sorted.
RNX_DEVICE void write_first(const moe_plan_t& plan, const int* s_off, const int* s_act, const int* s_sorted) {
  const int n_active = s_act[0];
  for (int u = threadIdx.x; u < n_active; u += blockDim.x) plan.first[u] = s_sorted[s_off[s_act[1 + u]]];
}


// ids: A expert ids (global memory; written before this call by any thread of
// the CTA is fine: the first barrier below orders it). Shared scratch:
// s_ids[kSmallMaxA], s_cnt[kMaxE], s_off[kMaxE], s_warp[33], s_act[kMaxE + 1],
// s_sorted[kSmallMaxA]. Every thread of the (1024-thread) CTA calls it.
RNX_DEVICE void small_plan(const int32_t* ids, int A, int E, int lb, int le, const moe_plan_t& plan,
                           uint32_t* status, int* s_ids, int* s_cnt, int* s_off, int* s_warp, int* s_act,
                           int* s_sorted) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  for (int a = threadIdx.x; a < A; a += blockDim.x) {
    int e = ids[a];
    if (e < 0 || e >= E) {
      set_status(status, kDevErrBounds);
      e = -1;
    } else {
      atomicAdd(&s_cnt[e], 1);
    }
    s_ids[a] = e;
  }
  __syncthreads();
  finish_plan(s_cnt, E, lb, le, plan, s_warp, s_off, s_act);
  __syncthreads();
  if (A > kSmallRankA) {
    // stable order by expert: a bitonic sort of the keys e * kSmallMaxA + a
    // (ids out of range and the slots past A sort last), one key per thread
    // (the CTA has kSmallMaxA threads); the k-th key is the assignment at
    // position k, offset + rank
    for (int i = threadIdx.x; i < kSmallMaxA; i += blockDim.x) {
      const int e = i < A ? s_ids[i] : -1;
      s_sorted[i] = e >= 0 ? e * kSmallMaxA + i : INT_MAX;
    }
    for (int kk = 2; kk <= kSmallMaxA; kk <<= 1)
      for (int j = kk >> 1; j > 0; j >>= 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < kSmallMaxA; i += blockDim.x) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const int x = s_sorted[i], y = s_sorted[ixj];
            if ((x > y) == ((i & kk) == 0)) {
              s_sorted[i] = y;
              s_sorted[ixj] = x;
            }
          }
        }
      }
    __syncthreads();
    for (int pos = threadIdx.x; pos < A; pos += blockDim.x) {
      const int key = s_sorted[pos];
      if (key != INT_MAX) {
        const int a = key & (kSmallMaxA - 1);
        plan.sorted[pos] = a;
        plan.inv[a] = pos;
        s_sorted[pos] = a;
      }
    }
    for (int a = threadIdx.x; a < A; a += blockDim.x)
      if (s_ids[a] < 0) plan.inv[a] = -1;
    __syncthreads();
    write_first(plan, s_off, s_act, s_sorted);
    return;
  }
  // stable position: offset + number of earlier assignments of the same expert
  for (int a0 = 0; a0 < A; a0 += blockDim.x) {
    const int a = a0 + threadIdx.x;
    const int e = a < A ? s_ids[a] : -1;
    int rank = 0;
    const int lim = min(A, a0 + (int)blockDim.x);
    for (int b = 0; b < lim; ++b) rank += (b < a && s_ids[b] == e) ? 1 : 0;
    if (a < A) {
      if (e >= 0) {
        const int pos = s_off[e] + rank;
        plan.sorted[pos] = a;
        s_sorted[pos] = a;
        plan.inv[a] = pos;
      } else {
        plan.inv[a] = -1;
      }
    }
  }
  __syncthreads();
  write_first(plan, s_off, s_act, s_sorted);
}

}  // namespace rnx
