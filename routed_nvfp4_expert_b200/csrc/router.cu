// Router: fp32 logits of gate.weight, then sigmoid top-k with a correction
// bias that steers selection only (glm5next_mlp module docs, "The stack this
// layer runs" and "Traps this module exists to hold"; TensorRT-LLM PR #19136,
// "Test Coverage": the gate is fp32).

#include "common.cuh"
#include "small_plan.cuh"
#include "topk.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kMaxTopK = 16;   // the pages' KERNEL_MAX_TOP_K


// ---------------------------------------------------------------- logits
// Small T (decode): the fp32 router matrix (E x H, 4.7 MB at E=288, H=4096)
// is the only real traffic. One 128-thread CTA owns one expert row: every
// thread issues all of its 128-bit weight loads up front (H/512 of them), then
// multiplies them against the tokens, 8 tokens per pass.
constexpr int kLogitTokens = 8;
constexpr int kLogitThreads = 128;
constexpr int kLogitMaxQ = 16;     // H <= 8192 in this form

__global__ void __launch_bounds__(kLogitThreads) router_logits_gemv(const uint16_t* __restrict__ x, int T, int H, int E,
                                                                   const float* __restrict__ wr,
                                                                   float* __restrict__ logits, uint32_t* xmax,
                                                                   uint32_t* zero, int nzero) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e = blockIdx.x;
  const int nq = H >> 2;
  __shared__ float red[4][kLogitTokens];
  // the router weight row does not depend on earlier kernels: load it first
  const float4* wrow = reinterpret_cast<const float4*>(wr + (size_t)e * H);
  float4 w[kLogitMaxQ];
#pragma unroll
  for (int i = 0; i < kLogitMaxQ; ++i) {
    const int c = tid + kLogitThreads * i;
    w[i] = c < nq ? __ldg(wrow + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  pdl_wait();
  pdl_trigger();
  if (e == 0) {
    // side jobs of CTA 0: max |x_t| per token (fp32 bits; the expert pass
    // pre-scales with it) and clearing the words asked for (the call's
    // control block)
    for (int i = tid; i < nzero; i += kLogitThreads) zero[i] = 0u;
    if (xmax) {
      for (int t = 0; t < T; ++t) {
        float m = 0.f;
        for (int g = tid; g < H / 8; g += kLogitThreads) {
          const uint4 v = reinterpret_cast<const uint4*>(x + (size_t)t * H)[g];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = bf16x2_to_f32x2(w4[j]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        }
        m = warp_max(m);
        if (lane == 0) red[warp][0] = m;
        __syncthreads();
        if (tid == 0) xmax[t] = __float_as_uint(fmaxf(fmaxf(red[0][0], red[1][0]), fmaxf(red[2][0], red[3][0])));
        __syncthreads();
      }
    }
  }
  for (int t0 = 0; t0 < T; t0 += kLogitTokens) {
    float acc[kLogitTokens];
#pragma unroll
    for (int t = 0; t < kLogitTokens; ++t) {
      acc[t] = 0.f;
      if (t0 + t < T) {
        const uint16_t* xr = x + (size_t)(t0 + t) * H;
#pragma unroll
        for (int i = 0; i < kLogitMaxQ; ++i) {
          const int c = tid + kLogitThreads * i;
          if (c < nq) {
            const uint2 xv = *reinterpret_cast<const uint2*>(xr + 4 * c);
            const float2 a = bf16x2_to_f32x2(xv.x), b = bf16x2_to_f32x2(xv.y);
            acc[t] = fmaf(w[i].x, a.x, acc[t]);
            acc[t] = fmaf(w[i].y, a.y, acc[t]);
            acc[t] = fmaf(w[i].z, b.x, acc[t]);
            acc[t] = fmaf(w[i].w, b.y, acc[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kLogitTokens; ++t) {
      const float v = warp_sum(acc[t]);
      if (lane == 0) red[warp][t] = v;
    }
    __syncthreads();
    if (tid < kLogitTokens && t0 + tid < T) {
      const float v = ((red[0][tid] + red[1][tid]) + red[2][tid]) + red[3][tid];
      logits[(size_t)(t0 + tid) * E + e] = v;
    }
    __syncthreads();
  }
}

// 2 to 64 tokens: read from L2 by every CTA, the token rows cost more than
// the router matrix once T passes a token. A 256-thread CTA owns four expert
// rows (H <= 4096, in registers), so each token row is read once per four
// experts; 8 tokens per pass, one warp sum per (expert, token), the warps'
// partials added in a fixed order. CTA t < T also leaves max |x_t| (fp32
// bits) when asked.
constexpr int kRbExperts = 4, kRbThreads = 256, kRbQ = 4, kRbTokens = 8;

__global__ void __launch_bounds__(kRbThreads) router_logits_gemv4(const uint16_t* __restrict__ x, int T, int H, int E,
                                                                  const float* __restrict__ wr,
                                                                  float* __restrict__ logits, uint32_t* xmax,
                                                                  uint32_t* zero, int nzero) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e0 = blockIdx.x * kRbExperts;
  const int nq = H >> 2;
  __shared__ float red[kRbThreads / 32][kRbExperts * kRbTokens];
  float4 w[kRbExperts][kRbQ];
#pragma unroll
  for (int j = 0; j < kRbExperts; ++j)
#pragma unroll
    for (int i = 0; i < kRbQ; ++i) {
      const int c = tid + kRbThreads * i;
      w[j][i] = (c < nq && e0 + j < E) ? __ldg(reinterpret_cast<const float4*>(wr + (size_t)(e0 + j) * H) + c)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0)
    for (int i = tid; i < nzero; i += kRbThreads) zero[i] = 0u;   // the call's control block
  if (xmax && (int)blockIdx.x < T) {
    const int t = blockIdx.x;
    float m = 0.f;
    for (int g = tid; g < H / 8; g += kRbThreads) {
      const uint4 v = reinterpret_cast<const uint4*>(x + (size_t)t * H)[g];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = bf16x2_to_f32x2(w4[j]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    m = warp_max(m);
    if (lane == 0) red[warp][0] = m;
    __syncthreads();
    if (tid == 0) {
      float a = red[0][0];
#pragma unroll
      for (int q = 1; q < kRbThreads / 32; ++q) a = fmaxf(a, red[q][0]);
      xmax[t] = __float_as_uint(a);
    }
    __syncthreads();
  }
  for (int t0 = 0; t0 < T; t0 += kRbTokens) {
    float acc[kRbExperts][kRbTokens];
#pragma unroll
    for (int t = 0; t < kRbTokens; ++t) {
      float2 xa[kRbQ], xb[kRbQ];
#pragma unroll
      for (int i = 0; i < kRbQ; ++i) {
        const int c = tid + kRbThreads * i;
        uint2 xv = make_uint2(0u, 0u);
        if (t0 + t < T && c < nq) xv = *reinterpret_cast<const uint2*>(x + (size_t)(t0 + t) * H + 4 * c);
        xa[i] = bf16x2_to_f32x2(xv.x);
        xb[i] = bf16x2_to_f32x2(xv.y);
      }
#pragma unroll
      for (int j = 0; j < kRbExperts; ++j) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < kRbQ; ++i) {
          a = fmaf(w[j][i].x, xa[i].x, a);
          a = fmaf(w[j][i].y, xa[i].y, a);
          a = fmaf(w[j][i].z, xb[i].x, a);
          a = fmaf(w[j][i].w, xb[i].y, a);
        }
        acc[j][t] = a;
      }
    }
#pragma unroll
    for (int j = 0; j < kRbExperts; ++j)
#pragma unroll
      for (int t = 0; t < kRbTokens; ++t) {
        const float v = warp_sum(acc[j][t]);
        if (lane == 0) red[warp][j * kRbTokens + t] = v;
      }
    __syncthreads();
    if (tid < kRbExperts * kRbTokens) {
      const int j = tid / kRbTokens, t = tid % kRbTokens;
      if (t0 + t < T && e0 + j < E) {
        float v = red[0][tid];
#pragma unroll
        for (int q = 1; q < kRbThreads / 32; ++q) v += red[q][tid];
        logits[(size_t)(t0 + t) * E + e0 + j] = v;
      }
    }
    __syncthreads();
  }
}

// Large T (prefill): a plain tiled fp32 GEMM on CUDA cores,
// logits[T, E] = x[T, H] * Wr[E, H]^T. 64x64 output tile, 256 threads, 4x4 each.
constexpr int kSgBM = 64, kSgBN = 64, kSgBK = 16;

__global__ void __launch_bounds__(256) router_logits_sgemm(const uint16_t* __restrict__ x, int T, int H, int E,
                                                           const float* __restrict__ wr, float* __restrict__ logits) {
  __shared__ float sx[kSgBK][kSgBM + 4];
  __shared__ float sw[kSgBK][kSgBN + 4];
  const int tm0 = blockIdx.y * kSgBM, en0 = blockIdx.x * kSgBN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < H; k0 += kSgBK) {
    // 64 rows x 16 k of each operand: 1024 elements, 4 per thread
    for (int i = threadIdx.x; i < kSgBM * kSgBK; i += 256) {
      const int r = i / kSgBK, kk = i % kSgBK;
      const int t = tm0 + r, e = en0 + r;
      sx[kk][r] = (t < T) ? bf16_bits_to_f32(x[(size_t)t * H + k0 + kk]) : 0.f;
      sw[kk][r] = (e < E) ? wr[(size_t)e * H + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSgBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sx[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sw[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = tm0 + ty * 4 + i, e = en0 + tx * 4 + j;
      if (t < T && e < E) logits[(size_t)t * E + e] = acc[i][j];
    }
}

template <int PL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                   int T, int E, int k, float rsf, int32_t* __restrict__ ids,
                                                   float* __restrict__ weights) {
  constexpr int kTopkTokens = topk_tokens<PL>();
  __shared__ float s_key[kTopkTokens][32 * PL];
  __shared__ float s_sig[kTopkTokens][32 * PL];
  const int warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int t0 = blockIdx.x * kTopkTokens;
  const int ntok = min(kTopkTokens, T - t0);
  topk_keys<PL>(logits, bias, t0, ntok, E, s_key, s_sig);
  __syncthreads();
  if (warp < ntok) topk_warp<PL>(s_key[warp], s_sig[warp], t0 + warp, E, k, rsf, ids, weights);
}

// Decode with one top-k CTA's worth of tokens: selection and the routing plan
// in one launch (1024 threads): the warps of the tokens select, then the whole
// CTA builds the plan from the ids it has just written.
template <int PL>
__global__ void __launch_bounds__(1024) topk_plan_kernel(const float* __restrict__ logits,
                                                         const float* __restrict__ bias, int T, int E, int k, float rsf,
                                                         int32_t* ids, float* __restrict__ weights, int lb, int le,
                                                         moe_plan_t plan, uint32_t* status) {
  constexpr int kTopkTokens = topk_tokens<PL>();
  __shared__ float s_key[kTopkTokens][32 * PL];
  __shared__ float s_sig[kTopkTokens][32 * PL];
  __shared__ int s_ids[kSmallMaxA];
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_off[kMaxE];
  __shared__ int s_warp[33];
  __shared__ int s_act[kMaxE + 1];
  __shared__ int s_sorted[kSmallMaxA];
  const int warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  topk_keys<PL>(logits, bias, 0, T, E, s_key, s_sig);
  __syncthreads();
  if (warp < T) topk_warp<PL>(s_key[warp], s_sig[warp], warp, E, k, rsf, ids, weights);
  __syncthreads();                       // the ids, for every thread of the CTA
  small_plan(ids, T * k, E, lb, le, plan, status, s_ids, s_cnt, s_off, s_warp, s_act, s_sorted);
}

// One token: selection and its routing plan in one CTA without block-wide
// scans: with k distinct ids every plan entry is a count over the k ids.
// counts[e] = [e chosen], offsets[e] = #chosen ids < e, tile_offsets[e] =
// #chosen local ids < e (one 256-row tile per chosen local expert), sorted /
// inv by expert order, the active list of the chosen local experts in
// expert order with first[u] = its assignment. All threads load and score the
// logits (one round of loads), warp 0 selects, all threads write the plan.
constexpr int kT1PlanThreads = 256;
template <int PL>
__global__ void __launch_bounds__(kT1PlanThreads) topk_plan_t1_kernel(const float* __restrict__ logits,
                                                                      const float* __restrict__ bias, int E, int k,
                                                                      float rsf, int32_t* ids,
                                                                      float* __restrict__ weights, int lb, int le,
                                                                      moe_plan_t plan, uint32_t* status) {
  __shared__ float s_key[1][32 * PL];
  __shared__ float s_sig[1][32 * PL];
  __shared__ int s_ids[kMaxTopK];
  // the correction bias is a weight: loaded before the wait for the logits
  constexpr int kBq = (32 * PL + kT1PlanThreads - 1) / kT1PlanThreads;
  float bq[kBq];
#pragma unroll
  for (int j = 0; j < kBq; ++j) {
    const int e = threadIdx.x + kT1PlanThreads * j;
    bq[j] = e < E ? bias[e] : 0.f;
  }
  pdl_wait();
  pdl_trigger();
#pragma unroll
  for (int j = 0; j < kBq; ++j) {
    const int e = threadIdx.x + kT1PlanThreads * j;
    if (e < E) {
      // sigmoid in double, rounded once to fp32; then an fp32 add of the bias
      const float sg = (float)(1.0 / (1.0 + exp(-(double)logits[e])));
      s_sig[0][e] = sg;
      s_key[0][e] = __fadd_rn(sg, bq[j]);
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) topk_warp<PL>(s_key[0], s_sig[0], 0, E, k, rsf, ids, weights, s_ids);
  __syncthreads();
  // every plan entry is a count over the k chosen ids (read from shared
  // memory: a per-thread copy indexed by the thread would live in local memory)
  auto id_at = [&](int j) { return s_ids[j]; };
  auto valid_at = [&](int j) { const int v = s_ids[j]; return j < k && v >= 0 && v < E; };
  for (int e = threadIdx.x; e <= E; e += kT1PlanThreads) {
    int cnt = 0, off = 0, toff = 0;
    for (int j = 0; j < k; ++j) {
      const int v = id_at(j);
      if (!valid_at(j)) continue;
      cnt += v == e;
      off += v < e;
      toff += v < e && v >= lb && v < le;
    }
    if (e < E) plan.counts[e] = cnt;
    plan.offsets[e] = off;
    plan.tile_offsets[e] = toff;
  }
  if (threadIdx.x < k) {
    const int j = threadIdx.x, idj = id_at(j);
    if (valid_at(j)) {
      int pos = 0, lpos = 0;
      for (int i = 0; i < k; ++i) {
        const int v = id_at(i);
        pos += valid_at(i) && v < idj;
        lpos += valid_at(i) && v < idj && v >= lb && v < le;
      }
      plan.sorted[pos] = j;
      plan.inv[j] = pos;
      if (idj >= lb && idj < le) {
        plan.active[1 + lpos] = idj;
        plan.first[lpos] = j;
      }
    } else {
      plan.inv[j] = -1;
      set_status(status, kDevErrBounds);
    }
  }
  if (threadIdx.x == 0) {
    int nl = 0;
    for (int j = 0; j < k; ++j) nl += valid_at(j) && id_at(j) >= lb && id_at(j) < le;
    plan.active[0] = nl;
  }
}

__global__ void __launch_bounds__(256) row_absmax_kernel(const uint16_t* __restrict__ rows, int R, int K,
                                                         uint32_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= R) return;
  float m = 0.f;
  for (int g = lane; g < K / 8; g += 32) {
    const uint4 v = reinterpret_cast<const uint4*>(rows + (size_t)r * K)[g];
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_f32x2(w4[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  m = warp_max(m);
  if (lane == 0) out[r] = __float_as_uint(m);
}

}  // namespace

cudaError_t launch_row_absmax(const uint16_t* rows, int R, int K, uint32_t* out, cudaStream_t st) {
  row_absmax_kernel<<<(R + 7) / 8, 256, 0, st>>>(rows, R, K, out);
  return cudaGetLastError();
}

bool router_gemv_form(int T, int H) { return T <= 64 && H <= 4 * kLogitThreads * kLogitMaxQ; }

cudaError_t launch_router_logits(const uint16_t* x, int T, int H, int E, const float* wr, float* logits,
                                 cudaStream_t st, uint32_t* xmax, uint32_t* zero, int nzero) {
  const int rb_ctas = (E + kRbExperts - 1) / kRbExperts;
  if (router_gemv_form(T, H) && T > 1 && H <= kRbThreads * kRbQ * 4 && (!xmax || T <= rb_ctas)) {
    return launch_pdl(router_logits_gemv4, dim3(rb_ctas), dim3(kRbThreads), 0, st, x, T, H, E, wr, logits, xmax,
                      zero, nzero);
  } else if (router_gemv_form(T, H)) {
    return launch_pdl(router_logits_gemv, dim3(E), dim3(kLogitThreads), 0, st, x, T, H, E, wr, logits, xmax, zero,
                      nzero);
  } else {
    dim3 grid((E + kSgBN - 1) / kSgBN, (T + kSgBM - 1) / kSgBM);
    router_logits_sgemm<<<grid, 256, 0, st>>>(x, T, H, E, wr, logits);
  }
  return cudaGetLastError();
}

cudaError_t launch_topk_plan(const float* logits, const float* bias, int T, int E, int k, float rsf, int32_t* ids,
                             float* weights, int lb, int le, const moe_plan_t& plan, uint32_t* status,
                             cudaStream_t st) {
  if (T < 1 || T * k > kSmallMaxA || E > kMaxE) return cudaErrorNotSupported;
  if (T == 1 && k <= kMaxTopK) {
    if (E <= 32 * 4)
      return launch_pdl(topk_plan_t1_kernel<4>, dim3(1), dim3(kT1PlanThreads), 0, st, logits, bias, E, k, rsf, ids, weights, lb, le,
                        plan, status);
    if (E <= 32 * 10)
      return launch_pdl(topk_plan_t1_kernel<10>, dim3(1), dim3(kT1PlanThreads), 0, st, logits, bias, E, k, rsf, ids, weights, lb,
                        le, plan, status);
    return launch_pdl(topk_plan_t1_kernel<32>, dim3(1), dim3(kT1PlanThreads), 0, st, logits, bias, E, k, rsf, ids, weights, lb, le,
                      plan, status);
  }
  if (E <= 32 * 4 && T <= topk_tokens<4>())
    return launch_pdl(topk_plan_kernel<4>, dim3(1), dim3(1024), 0, st, logits, bias, T, E, k, rsf, ids, weights, lb,
                      le, plan, status);
  if (E > 32 * 4 && E <= 32 * 10 && T <= topk_tokens<10>())
    return launch_pdl(topk_plan_kernel<10>, dim3(1), dim3(1024), 0, st, logits, bias, T, E, k, rsf, ids, weights, lb,
                      le, plan, status);
  return cudaErrorNotSupported;   // E > 320: the per-lane key arrays outgrow 1024-thread registers
}

cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, float rsf, int32_t* ids,
                        float* weights, cudaStream_t st) {
  auto grid = [T](int tpb) { return (T + tpb - 1) / tpb; };
  if (E <= 32 * 4)
    return launch_pdl(topk_kernel<4>, dim3(grid(topk_tokens<4>())), dim3(256), 0, st, logits, bias, T, E, k, rsf, ids,
                      weights);
  else if (E <= 32 * 10)
    return launch_pdl(topk_kernel<10>, dim3(grid(topk_tokens<10>())), dim3(256), 0, st, logits, bias, T, E, k, rsf, ids,
                      weights);
  else
    return launch_pdl(topk_kernel<32>, dim3(grid(topk_tokens<32>())), dim3(256), 0, st, logits, bias, T, E, k, rsf, ids,
                      weights);
  return cudaGetLastError();
}

namespace {

// Exact three-term bf16 split of an fp32 weight: clearing the low 16 bits of
// the encoding truncates to the leading 8 significand bits (a bf16 value);
// each remainder is exact in fp32 and has 16, then 8 significant bits left.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ w, int E, int H,
                                                           uint16_t* __restrict__ w3) {
  const long long n = (long long)E * H;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long e = i / H;
    const int c = (int)(i - e * H);
    const float v = w[i];
    const float hi = __uint_as_float(__float_as_uint(v) & 0xFFFF0000u);
    const float r1 = v - hi;
    const float mid = __uint_as_float(__float_as_uint(r1) & 0xFFFF0000u);
    const float lo = r1 - mid;
    uint16_t* row = w3 + e * 3 * H;                  // order lo | mid | hi along K
    row[c] = (uint16_t)(__float_as_uint(lo) >> 16);
    row[H + c] = (uint16_t)(__float_as_uint(mid) >> 16);
    row[2 * H + c] = (uint16_t)(__float_as_uint(hi) >> 16);
  }
}

}  // namespace

cudaError_t launch_router_split(const float* w, int E, int H, uint16_t* w3, cudaStream_t st) {
  const long long n = (long long)E * H;
  if (n <= 0) return cudaSuccess;
  const int grid = (int)std::min<long long>((n + 255) / 256, (long long)kNumSMs * 16);
  router_split_kernel<<<grid, 256, 0, st>>>(w, E, H, w3);
  return cudaGetLastError();
}

}  // namespace rnx
