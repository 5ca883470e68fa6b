// Router: fp32 logits of gate.weight, then sigmoid top-k with a correction
// bias that steers selection only (glm5next_mlp module docs, "The stack this
// layer runs" and "Traps this module exists to hold"; TensorRT-LLM PR #19136,
// "Test Coverage": the gate is fp32).

#include "common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

// ---------------------------------------------------------------- logits
// Small T (decode): the fp32 router matrix (E x H, 4.7 MB at E=288, H=4096)
// is the only real traffic. Half a CTA (128 threads) owns one expert row and
// streams it with 128-bit loads; tokens are taken 8 at a time.
constexpr int kLogitTokens = 8;

__global__ void __launch_bounds__(256) router_logits_gemv(const uint16_t* __restrict__ x, int T, int H, int E,
                                                          const float* __restrict__ wr, float* __restrict__ logits) {
  const int half = threadIdx.x >> 7, t128 = threadIdx.x & 127, warp4 = t128 >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 2 + half;
  const bool valid = e < E;
  const int nq = H >> 2;
  __shared__ float red[2][4][kLogitTokens];
  const float4* wrow = reinterpret_cast<const float4*>(wr + (size_t)(valid ? e : 0) * H);
  for (int t0 = 0; t0 < T; t0 += kLogitTokens) {
    float acc[kLogitTokens];
#pragma unroll
    for (int t = 0; t < kLogitTokens; ++t) acc[t] = 0.f;
#pragma unroll 4
    for (int c = t128; c < nq; c += 128) {
      const float4 w = valid ? __ldg(wrow + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int t = 0; t < kLogitTokens; ++t) {
        if (t0 + t < T) {
          const uint2 xv = *reinterpret_cast<const uint2*>(x + (size_t)(t0 + t) * H + 4 * c);
          const float2 a = bf16x2_to_f32x2(xv.x), b = bf16x2_to_f32x2(xv.y);
          acc[t] = fmaf(w.x, a.x, acc[t]);
          acc[t] = fmaf(w.y, a.y, acc[t]);
          acc[t] = fmaf(w.z, b.x, acc[t]);
          acc[t] = fmaf(w.w, b.y, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kLogitTokens; ++t) {
      const float v = warp_sum(acc[t]);
      if (lane == 0) red[half][warp4][t] = v;
    }
    __syncthreads();
    if (t128 < kLogitTokens && t0 + t128 < T && valid) {
      const float v = ((red[half][0][t128] + red[half][1][t128]) + red[half][2][t128]) + red[half][3][t128];
      logits[(size_t)(t0 + t128) * E + e] = v;
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

// ---------------------------------------------------------------- top-k
// One warp per token. Lane l holds experts l, l+32, ... Candidate order:
// unused finite keys first (key descending, then lower index), then NaN keys
// (lower index first), then used / padding entries.
struct Cand {
  int state;   // 0 = live key, 1 = NaN key, 2 = taken or padding
  float key;
  int idx;
  float s;
};

RNX_DEVICE bool better(const Cand& a, const Cand& b) {
  if (a.state != b.state) return a.state < b.state;
  if (a.state == 0 && a.key != b.key) return a.key > b.key;
  return a.idx < b.idx;
}

template <int PL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                   int T, int E, int k, float rsf, int32_t* __restrict__ ids,
                                                   float* __restrict__ weights) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  float key[PL], sg[PL];
  int st[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float l = logits[(size_t)t * E + e];
      // sigmoid in double, rounded once to fp32; then an fp32 add of the bias
      const float s = (float)(1.0 / (1.0 + exp(-(double)l)));
      const float kk = __fadd_rn(s, bias[e]);
      sg[i] = s;
      key[i] = kk;
      st[i] = isnan(kk) ? 1 : 0;
    } else {
      sg[i] = 0.f;
      key[i] = 0.f;
      st[i] = 2;
    }
  }
  float chosen_s = 0.f;   // lane j keeps the score of rank slot j
  int chosen_id = 0;
  for (int j = 0; j < k; ++j) {
    Cand best{2, 0.f, 0x7fffffff, 0.f};
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      Cand c{st[i], key[i], lane + 32 * i, sg[i]};
      if (better(c, best)) best = c;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Cand other;
      other.state = __shfl_xor_sync(0xffffffffu, best.state, o);
      other.key = __shfl_xor_sync(0xffffffffu, best.key, o);
      other.idx = __shfl_xor_sync(0xffffffffu, best.idx, o);
      other.s = __shfl_xor_sync(0xffffffffu, best.s, o);
      if (better(other, best)) best = other;
    }
    // the owner marks its entry taken
    if ((best.idx & 31) == lane) {
#pragma unroll
      for (int i = 0; i < PL; ++i)
        if (lane + 32 * i == best.idx) st[i] = 2;
    }
    if (lane == j) {
      chosen_s = best.s;
      chosen_id = best.idx;
    }
  }
  // renormalise the UNBIASED scores over the chosen k, rank order
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, chosen_s, j);
  if (lane < k) {
    ids[(size_t)t * k + lane] = chosen_id;
    weights[(size_t)t * k + lane] = sum > 0.f ? rsf * (chosen_s / sum) : 0.f;
  }
}

}  // namespace

cudaError_t launch_router_logits(const uint16_t* x, int T, int H, int E, const float* wr, float* logits,
                                 cudaStream_t st) {
  if (T <= 64) {
    router_logits_gemv<<<(E + 1) / 2, 256, 0, st>>>(x, T, H, E, wr, logits);
  } else {
    dim3 grid((E + kSgBN - 1) / kSgBN, (T + kSgBM - 1) / kSgBM);
    router_logits_sgemm<<<grid, 256, 0, st>>>(x, T, H, E, wr, logits);
  }
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, float rsf, int32_t* ids,
                        float* weights, cudaStream_t st) {
  const int grid = (T + 7) / 8;
  if (E <= 32 * 4) topk_kernel<4><<<grid, 256, 0, st>>>(logits, bias, T, E, k, rsf, ids, weights);
  else if (E <= 32 * 10) topk_kernel<10><<<grid, 256, 0, st>>>(logits, bias, T, E, k, rsf, ids, weights);
  else topk_kernel<32><<<grid, 256, 0, st>>>(logits, bias, T, E, k, rsf, ids, weights);
  return cudaGetLastError();
}

}  // namespace rnx
