// Token sort (glm5next_mlp module docs, MOE_MODULE: the token sort /
// permute / unpermute family): the A = T*k assignments a = t*k + j are
// grouped by expert, stably, with counts, offsets, the inverse map, per-expert
// 128-row tile offsets (local experts only) and the list of active local
// experts.
//
// Small A (decode): one CTA does everything in shared memory.
// Large A (prefill): a three-kernel counting sort -- per-256-assignment
// histograms with warp-match ranks, one CTA that scans them, an ordered scatter.

#include "common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kSmallMaxA = 1024;
constexpr int kMaxE = 1024;
constexpr int kChunk = 256;   // assignments per histogram block

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

// counts -> offsets, tile_offsets, active (one CTA of 1024 threads, E <= 1024)
RNX_DEVICE void finish_plan(const int* s_cnt, int E, int lb, int le, const moe_plan_t& plan, int* s_warp) {
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
    if (act) plan.active[1 + aoff] = e;
  }
  if (e == 0) {
    plan.offsets[E] = tot;
    plan.tile_offsets[E] = ttot;
    plan.active[0] = atot;
  }
}

// first[u] = sorted[offsets[e]] for the u-th active (local, non-empty) expert e.
// Runs after sorted[] is complete; reads offsets/active/sorted from the plan.
RNX_DEVICE void write_first(const moe_plan_t& plan, const int* s_off, const int* s_cnt, int E, int lb, int le) {
  const int n_active = plan.active[0];
  for (int u = threadIdx.x; u < n_active; u += blockDim.x) {
    const int e = plan.active[1 + u];
    plan.first[u] = plan.sorted[plan.offsets[e]];
  }
  (void)s_off;
  (void)s_cnt;
  (void)E;
  (void)lb;
  (void)le;
}

__global__ void __launch_bounds__(1024) permute_small(const int32_t* __restrict__ ids, int A, int E, int lb, int le,
                                                      moe_plan_t plan, uint32_t* status) {
  __shared__ int s_ids[kSmallMaxA];
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_off[kMaxE];
  __shared__ int s_warp[33];
  pdl_wait();
  pdl_trigger();
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
  finish_plan(s_cnt, E, lb, le, plan, s_warp);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_off[e] = plan.offsets[e];
  __syncthreads();
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
        plan.inv[a] = pos;
      } else {
        plan.inv[a] = -1;
      }
    }
  }
  __syncthreads();
  write_first(plan, s_off, s_cnt, E, lb, le);
}

// ---- large A
// scratch layout (ints): rank[A], hist[E][nb] (expert-major)
__global__ void __launch_bounds__(kChunk) permute_hist(const int32_t* __restrict__ ids, int A, int E,
                                                       int32_t* __restrict__ rank, int32_t* __restrict__ hist,
                                                       uint32_t* status) {
  extern __shared__ int s_wcnt[];   // [8][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) s_wcnt[i] = 0;
  __syncthreads();
  const int a = blockIdx.x * kChunk + threadIdx.x;
  int e = -1;
  if (a < A) {
    e = ids[a];
    if (e < 0 || e >= E) {
      set_status(status, kDevErrBounds);
      e = -1;
    }
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rw = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rw == 0) s_wcnt[warp * E + e] = __popc(peers);
  __syncthreads();
  if (a < A) {
    int r = rw;
    if (e >= 0)
      for (int w = 0; w < warp; ++w) r += s_wcnt[w * E + e];
    rank[a] = e >= 0 ? r : -1;
  }
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += s_wcnt[w * E + x];
    hist[(size_t)x * gridDim.x + blockIdx.x] = s;
  }
}

// one CTA: per-expert exclusive prefix over blocks (in place), then the plan.
// hist is expert-major [E][nb] so each warp reads one expert's run contiguously.
__global__ void __launch_bounds__(1024) permute_scan(int nb, int E, int lb, int le, int32_t* __restrict__ hist,
                                                     moe_plan_t plan) {
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_warp[33];
  constexpr int kPer = 16;   // 512 blocks per pass
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int e = warp; e < E; e += nw) {
    int32_t* he = hist + (size_t)e * nb;
    int carry = 0;
    for (int b0 = 0; b0 < nb; b0 += 32 * kPer) {
      int v[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int b = b0 + 32 * i + lane;
        v[i] = b < nb ? he[b] : 0;
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        int inc = v[i];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += n;
        }
        const int b = b0 + 32 * i + lane;
        if (b < nb) he[b] = carry + inc - v[i];
        carry += __shfl_sync(0xffffffffu, inc, 31);
      }
    }
    if (lane == 0) s_cnt[e] = carry;
  }
  __syncthreads();
  finish_plan(s_cnt, E, lb, le, plan, s_warp);
}

__global__ void __launch_bounds__(kChunk) permute_scatter(const int32_t* __restrict__ ids, int A, int E,
                                                          const int32_t* __restrict__ rank,
                                                          const int32_t* __restrict__ hist, moe_plan_t plan) {
  const int a = blockIdx.x * kChunk + threadIdx.x;
  if (a >= A) return;
  const int r = rank[a];
  if (r < 0) {
    plan.inv[a] = -1;
    return;
  }
  const int e = ids[a];
  const int pos = plan.offsets[e] + hist[(size_t)e * gridDim.x + blockIdx.x] + r;
  plan.sorted[pos] = a;
  plan.inv[a] = pos;
}

__global__ void __launch_bounds__(256) permute_first(moe_plan_t plan) {
  const int n_active = plan.active[0];
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < n_active; u += gridDim.x * blockDim.x) {
    const int e = plan.active[1 + u];
    plan.first[u] = plan.sorted[plan.offsets[e]];
  }
}

}  // namespace

size_t permute_scratch_ints(int A, int E) {
  const size_t nb = (size_t)(A + kChunk - 1) / kChunk;
  return (size_t)A + nb * (size_t)E;
}

cudaError_t launch_permute(const int32_t* ids, int A, int E, int lb, int le, const moe_plan_t& plan,
                           int32_t* scratch, uint32_t* status, cudaStream_t st) {
  if (A <= kSmallMaxA) {
    return launch_pdl(permute_small, dim3(1), dim3(1024), 0, st, ids, A, E, lb, le, plan, status);
    return cudaGetLastError();
  }
  const int nb = (A + kChunk - 1) / kChunk;
  int32_t* rank = scratch;
  int32_t* hist = scratch + A;
  permute_hist<<<nb, kChunk, 8 * E * sizeof(int), st>>>(ids, A, E, rank, hist, status);
  permute_scan<<<1, 1024, 0, st>>>(nb, E, lb, le, hist, plan);
  permute_scatter<<<nb, kChunk, 0, st>>>(ids, A, E, rank, hist, plan);
  permute_first<<<(E + 255) / 256, 256, 0, st>>>(plan);
  return cudaGetLastError();
}

}  // namespace rnx
