// Sigmoid top-k selection with a correction bias that steers selection only
// (glm5next_mlp module docs, "Traps this module exists to hold": the emitted
// weight is the unbiased sigmoid score, renormalised over the chosen experts
// and multiplied by routed_scaling_factor; at most 16 experts per token,
// Constants KERNEL_MAX_TOP_K). Shared by the top-k kernels and the
// single-token decode chain.
#pragma once

#include "common.cuh"

namespace rnx {

// Candidate order of a selection (one warp per token, lane l holds experts
// l, l + 32, ...): unused non-NaN keys first (key descending, then lower
// index), then NaN keys (lower index first), then used / padding entries.

// 8 tokens per CTA. All 256 threads first evaluate the sigmoid scores and
// selection keys of the CTA's tokens into shared memory; then one warp per
// token selects its top-k.
template <int PL>
__host__ __device__ constexpr int topk_tokens() { return PL > 16 ? 2 : 8; }

// Sigmoid scores and selection keys of ntok tokens (from token t0) into
// shared memory, by all threads of the CTA.
template <int PL, int NT>
RNX_DEVICE void topk_keys(const float* __restrict__ logits, const float* __restrict__ bias, int t0, int ntok, int E,
                          float (&s_key)[NT][32 * PL], float (&s_sig)[NT][32 * PL]) {
  for (int i = threadIdx.x; i < ntok * E; i += blockDim.x) {
    const int tt = i / E, e = i - tt * E;
    const float l = logits[(size_t)(t0 + tt) * E + e];
    // sigmoid in double, rounded once to fp32; then an fp32 add of the bias
    const float sg = (float)(1.0 / (1.0 + exp(-(double)l)));
    s_sig[tt][e] = sg;
    s_key[tt][e] = __fadd_rn(sg, bias[e]);
  }
}

// One warp selects token t's top-k from its keys and writes ids / weights
// (and the ids to s_ids[0..k) as well when given). Each candidate's 32-bit
// rank key is formed once: live keys (finite or infinite) in fp32 order
// mapped to unsigned order, all above 1; NaN keys 1; taken / padding 0. A
// selection round is one warp max of the rank keys (redux), then one warp min
// of the indices that hold it (the lower index wins a tie), and the owner
// clears the chosen key.
RNX_DEVICE uint32_t rank_key(float key) {
  if (isnan(key)) return 1u;
  const uint32_t u = key == 0.f ? 0u : __float_as_uint(key);   // -0 as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);         // >= 0x007FFFFF for every non-NaN key
}

template <int PL>
RNX_DEVICE void topk_warp(const float* s_key_row, const float* s_sig_row, int t, int E, int k, float rsf,
                          int32_t* __restrict__ ids, float* __restrict__ weights, int* s_ids = nullptr) {
  const int lane = threadIdx.x & 31;
  uint32_t rk[PL];
  float sg[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    rk[i] = e < E ? rank_key(s_key_row[e]) : 0u;
    sg[i] = e < E ? s_sig_row[e] : 0.f;
  }
  float chosen_s = 0.f;   // lane j keeps the score of rank slot j
  int chosen_id = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t m = rk[0];
#pragma unroll
    for (int i = 1; i < PL; ++i) m = max(m, rk[i]);
    const uint32_t best = __reduce_max_sync(0xffffffffu, m);
    // the lowest index holding the best key: this lane's first, then the warp's
    uint32_t mine = 0xFFFFFFFFu;
#pragma unroll
    for (int i = PL - 1; i >= 0; --i) mine = rk[i] == best ? (uint32_t)(lane + 32 * i) : mine;
    const int idx = (int)__reduce_min_sync(0xffffffffu, mine);
    // the owner clears the chosen key and hands over its score
    float s_own = 0.f;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const bool hit = lane + 32 * i == idx;
      s_own = hit ? sg[i] : s_own;
      rk[i] = hit ? 0u : rk[i];
    }
    const float s_best = __shfl_sync(0xffffffffu, s_own, idx & 31);
    if (lane == j) {
      chosen_s = s_best;
      chosen_id = idx;
    }
  }
  // renormalise the UNBIASED scores over the chosen k, rank order
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, chosen_s, j);
  if (lane < k) {
    if (s_ids) s_ids[lane] = chosen_id;
    ids[(size_t)t * k + lane] = chosen_id;
    weights[(size_t)t * k + lane] = sum > 0.f ? rsf * (chosen_s / sum) : 0.f;
  }
}

}  // namespace rnx
