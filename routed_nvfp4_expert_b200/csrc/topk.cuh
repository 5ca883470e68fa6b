// Sigmoid top-k selection with a correction bias that steers selection only
// (glm5next_mlp module docs, "Traps this module exists to hold": the emitted
// weight is the unbiased sigmoid score, renormalised over the chosen experts
// and multiplied by routed_scaling_factor; at most 16 experts per token,
// Constants KERNEL_MAX_TOP_K). Shared by the top-k kernels and the
// single-token decode chain.
#pragma once

#include "common.cuh"

namespace rnx {

// One warp per token. Lane l holds experts l, l+32, ... Candidate order:
// unused finite keys first (key descending, then lower index), then NaN keys
// (lower index first), then used / padding entries.
// That order as one 64-bit integer, larger = better (one warp max per
// selection round): bits 63..62 the class (live 2, NaN 1, taken / padding 0),
// bits 61..30 a live key's fp32 bits mapped to unsigned order (a zero key as
// +0), bits 29..0 the complement of the index (the lower index wins a tie).
RNX_DEVICE unsigned long long cand_rank(int state, float key, int idx) {
  uint32_t ok = 0;
  if (state == 0) {
    const uint32_t u = key == 0.f ? 0u : __float_as_uint(key);
    ok = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
  return ((unsigned long long)(2 - state) << 62) | ((unsigned long long)ok << 30) |
         (unsigned long long)(0x3FFFFFFF - idx);
}

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
// (and the ids to s_ids[0..k) as well when given).
template <int PL>
RNX_DEVICE void topk_warp(const float* s_key_row, const float* s_sig_row, int t, int E, int k, float rsf,
                          int32_t* __restrict__ ids, float* __restrict__ weights, int* s_ids = nullptr) {
  const int lane = threadIdx.x & 31;
  float key[PL], sg[PL];
  int st[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      key[i] = s_key_row[e];
      sg[i] = s_sig_row[e];
      st[i] = isnan(key[i]) ? 1 : 0;
    } else {
      sg[i] = 0.f;
      key[i] = 0.f;
      st[i] = 2;
    }
  }
  float chosen_s = 0.f;   // lane j keeps the score of rank slot j
  int chosen_id = 0;
  for (int j = 0; j < k; ++j) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int i = 0; i < PL; ++i) best = max(best, cand_rank(st[i], key[i], lane + 32 * i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    const int idx = 0x3FFFFFFF - (int)(best & 0x3FFFFFFFull);
    // the owner marks its entry taken and hands over its score
    float s_own = 0.f;
    if ((idx & 31) == lane) {
#pragma unroll
      for (int i = 0; i < PL; ++i)
        if (lane + 32 * i == idx) {
          st[i] = 2;
          s_own = sg[i];
        }
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
