// Token sort (glm5next_mlp module docs, MOE_MODULE: the token sort /
// permute / unpermute family): the A = T*k assignments a = t*k + j are
// grouped by expert, stably, with counts, offsets, the inverse map, per-expert
// 256-row tile offsets (local experts only) and the list of active local
// experts.
//
// Small A (decode): one CTA does everything in shared memory.
// Large A (prefill): a three-kernel counting sort -- per-256-assignment
// histograms with warp-match ranks, one CTA that scans them, an ordered scatter.

#include "common.cuh"
#include "kernels.h"
#include "small_plan.cuh"

namespace rnx {

namespace {

constexpr int kChunk = 256;   // assignments per histogram block

__global__ void __launch_bounds__(1024) permute_small(const int32_t* __restrict__ ids, int A, int E, int lb, int le,
                                                      moe_plan_t plan, uint32_t* status) {
  __shared__ int s_ids[kSmallMaxA];
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_off[kMaxE];
  __shared__ int s_warp[33];
  __shared__ int s_act[kMaxE + 1];
  __shared__ int s_sorted[kSmallMaxA];
  pdl_wait();
  pdl_trigger();
  small_plan(ids, A, E, lb, le, plan, status, s_ids, s_cnt, s_off, s_warp, s_act, s_sorted);
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
  __shared__ int s_off[kMaxE];
  __shared__ int s_act[kMaxE + 1];
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
        if (b0 + 32 * i >= nb) break;   // warp-uniform: the rest of the pass is past the blocks
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
  finish_plan(s_cnt, E, lb, le, plan, s_warp, s_off, s_act);   // the shared copies go unused here
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
