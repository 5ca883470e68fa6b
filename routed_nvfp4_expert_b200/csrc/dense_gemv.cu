// Dense BF16 FFN at small T (decode): the dense layers' gate_proj/up_proj ->
// clamped SwiGLU -> down_proj, and the BF16 shared expert of the routed site
// (glm5next_mlp module docs, "The stack this layer runs"). Both are streams
// over the bf16 weights: each warp owns output rows, lanes read 16-byte
// chunks l, l+32, ... of each row, the activations of up to 8 tokens sit in
// shared memory (x as bf16, h as fp32), fp32 accumulation; h stays fp32
// between the two projections.

#include "common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kDgWarps = 8;
constexpr int kDgThreads = kDgWarps * kWarp;
constexpr int kSeg = 8;   // 16-byte chunks per row per lane held in registers at once

// Eight activations (elements 8c .. 8c+7) from the staged rows: bf16 or fp32.
template <bool ACT_F32>
RNX_DEVICE void act8(const uint4* s_act, int idx, float (&f)[8]) {
  if (ACT_F32) {
    const float4 a = reinterpret_cast<const float4*>(s_act)[2 * idx];
    const float4 b = reinterpret_cast<const float4*>(s_act)[2 * idx + 1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  } else {
    const uint4 v = s_act[idx];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 t = bf16x2_to_f32x2(w[q]);
      f[2 * q] = t.x;
      f[2 * q + 1] = t.y;
    }
  }
}

// GATE_UP: act = x bf16 [T, K], out = h fp32 [T, rows] (clamped SwiGLU of the
// gate and up rows). DOWN: act = h fp32 [T, K], out = y [T, rows] in bf16 or
// fp32 (OUT_F32).
template <int MT, bool GATE_UP, bool OUT_F32>
__global__ void __launch_bounds__(kDgThreads)
bf16_gemv_kernel(int K, int rows, int T, float limit, const void* __restrict__ act,
                 const uint16_t* __restrict__ w0, const uint16_t* __restrict__ w1, void* __restrict__ out) {
  extern __shared__ uint4 s_act[];   // [MT][K] activations as given (bf16 or fp32)
  constexpr bool ACT_F32 = !GATE_UP;
  constexpr int ES = ACT_F32 ? 4 : 2;
  constexpr int NB = GATE_UP ? 2 : 1;
  constexpr int RPW = GATE_UP ? 1 : 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = K >> 3;                  // 8-element chunks per row
  const int rows_per_item = kDgWarps * RPW;
  const int n_items = rows / rows_per_item;
  pdl_wait();
  pdl_trigger();
  for (int t0 = 0; t0 < T; t0 += MT) {
    const int nm = min(MT, T - t0);
    __syncthreads();
    const int u4_per_row = K * ES / 16;
    for (int i = threadIdx.x; i < nm * u4_per_row; i += blockDim.x) {
      const int m = i / u4_per_row, c = i - m * u4_per_row;
      s_act[i] = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(act) + (size_t)(t0 + m) * K * ES)[c];
    }
    __syncthreads();
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int row0 = item * rows_per_item + warp * RPW;
      float acc[RPW][NB][MT];
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[r][b][m] = 0.f;
      for (int c0 = 0; c0 < nch; c0 += 32 * kSeg) {
        uint4 wv[RPW][NB][kSeg];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const uint16_t* wrow = (b == 0 ? w0 : w1) + (size_t)(row0 + r) * K;
#pragma unroll
            for (int s = 0; s < kSeg; ++s) {
              const int c = c0 + 32 * s + lane;
              wv[r][b][s] = c < nch ? ldg_stream(wrow + 8 * c) : make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
        for (int s = 0; s < kSeg; ++s) {
          const int c = c0 + 32 * s + lane;
          if (c < nch) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              if (m < nm) {
                float xf[8];
                act8<ACT_F32>(s_act, m * nch + c, xf);
#pragma unroll
                for (int r = 0; r < RPW; ++r)
#pragma unroll
                  for (int b = 0; b < NB; ++b) {
                    const uint32_t ww[4] = {wv[r][b][s].x, wv[r][b][s].y, wv[r][b][s].z, wv[r][b][s].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                      const float2 f = bf16x2_to_f32x2(ww[q]);
                      acc[r][b][m] = fmaf(f.x, xf[2 * q], acc[r][b][m]);
                      acc[r][b][m] = fmaf(f.y, xf[2 * q + 1], acc[r][b][m]);
                    }
                  }
              }
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        float tot[NB][MT];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int m = 0; m < MT; ++m) tot[b][m] = warp_sum(acc[r][b][m]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (lane == m && m < nm) {
            const float v = GATE_UP ? clamped_swiglu(tot[0][m], tot[NB - 1][m], limit) : tot[0][m];
            const size_t o = (size_t)(t0 + m) * rows + row0 + r;
            if (GATE_UP || OUT_F32) reinterpret_cast<float*>(out)[o] = v;
            else reinterpret_cast<uint16_t*>(out)[o] = f32_to_bf16_bits(v);
          }
        }
      }
    }
  }
}

template <int MT, bool GU, bool OF>
cudaError_t launch_t(int K, int rows, int T, float limit, const void* act, const uint16_t* w0,
                     const uint16_t* w1, void* out, cudaStream_t st, bool bg) {
  const size_t smem = (size_t)MT * K * (GU ? 2 : 4);
  auto kern = bf16_gemv_kernel<MT, GU, OF>;
  static size_t cached_smem = 0;
  static int per_sm = 0;
  if (cached_smem != smem) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDgThreads, smem);
    if (err != cudaSuccess) return err;
    cached_smem = smem;
  }
  const int rows_per_item = kDgWarps * (GU ? 1 : 2);
  const int items = rows / rows_per_item;
  const int grid = std::max(1, std::min(items, kNumSMs * std::max(per_sm, 1)));
  if (bg)
    return launch_ex(kern, dim3(grid), dim3(kDgThreads), smem, st, GU, launch_priority_low(), K, rows, T, limit, act,
                     w0, w1, out);
  return launch_pdl(kern, dim3(grid), dim3(kDgThreads), smem, st, K, rows, T, limit, act, w0, w1, out);
}

template <bool GU, bool OF>
cudaError_t launch_mt(int K, int rows, int T, float limit, const void* act, const uint16_t* w0,
                      const uint16_t* w1, void* out, cudaStream_t st, bool bg = false) {
  const size_t budget = 96 * 1024;
  const size_t es = GU ? 2 : 4;
  if (T >= 8 && (size_t)8 * K * es <= budget) return launch_t<8, GU, OF>(K, rows, T, limit, act, w0, w1, out, st, bg);
  if (T >= 4 && (size_t)4 * K * es <= budget) return launch_t<4, GU, OF>(K, rows, T, limit, act, w0, w1, out, st, bg);
  if (T >= 2 && (size_t)2 * K * es <= budget) return launch_t<2, GU, OF>(K, rows, T, limit, act, w0, w1, out, st, bg);
  return launch_t<1, GU, OF>(K, rows, T, limit, act, w0, w1, out, st, bg);
}

}  // namespace

cudaError_t launch_dense_gemv(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                              const uint16_t* wu, const uint16_t* wd, void* y, bool y_f32, float* hbuf,
                              cudaStream_t st, bool background) {
  cudaError_t err = launch_mt<true, true>(H, I, T, limit, x, wg, wu, hbuf, st, background);
  if (err != cudaSuccess) return err;
  return y_f32 ? launch_mt<false, true>(I, H, T, 0.f, hbuf, wd, nullptr, y, st, background)
               : launch_mt<false, false>(I, H, T, 0.f, hbuf, wd, nullptr, y, st, background);
}

cudaError_t launch_dense_ffn(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                             const uint16_t* wu, const uint16_t* wd, void* y, bool y_f32, void* hbuf,
                             uint32_t* status, cudaStream_t st, int min_t) {
  if (T >= min_t && I % 128 == 0 && H % 256 == 0) {
    // the fp32 output (the site's shared row) carries h as two bf16 terms;
    // the bf16 output (the dense FFN entry point) rounds h to bf16
    uint16_t* hb = reinterpret_cast<uint16_t*>(hbuf);
    cudaError_t err = launch_bf16_gemm(true, x, T, H, wg, wu, I, limit, hb, status, st, nullptr, y_f32);
    if (err != cudaSuccess) return err;
    return launch_bf16_gemm(false, hb, T, y_f32 ? 2 * I : I, wd, nullptr, H, 0.f,
                            y_f32 ? nullptr : static_cast<uint16_t*>(y), status, st,
                            y_f32 ? static_cast<float*>(y) : nullptr, y_f32);
  }
  return launch_dense_gemv(H, I, limit, x, T, wg, wu, wd, y, y_f32, reinterpret_cast<float*>(hbuf), st);
}

}  // namespace rnx
