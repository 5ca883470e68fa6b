// Dense BF16 FFN at small T (decode): the dense layers' gate_proj/up_proj ->
// clamped SwiGLU -> down_proj, and the BF16 shared expert of the routed site
// (glm5next_mlp module docs, "The stack this layer runs"). Both are streams
// over the bf16 weights: each warp owns output rows, lanes read 16-byte
// chunks l, l+32, ... of each row, activations sit in shared memory (bf16),
// fp32 accumulation.

#include "common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kDgWarps = 8;
constexpr int kDgThreads = kDgWarps * kWarp;
constexpr int kSeg = 8;   // 16-byte chunks per row per lane held in registers at once

template <int MT, bool GATE_UP>
__global__ void __launch_bounds__(kDgThreads)
bf16_gemv_kernel(int K, int rows, int T, float limit, const uint16_t* __restrict__ act,
                 const uint16_t* __restrict__ w0, const uint16_t* __restrict__ w1, uint16_t* __restrict__ out) {
  extern __shared__ uint4 s_act[];   // [MT][K/8]
  constexpr int NB = GATE_UP ? 2 : 1;
  constexpr int RPW = GATE_UP ? 1 : 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = K >> 3;
  const int rows_per_item = kDgWarps * RPW;
  const int n_items = rows / rows_per_item;
  for (int t0 = 0; t0 < T; t0 += MT) {
    const int nm = min(MT, T - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < nm * nch; i += blockDim.x) {
      const int m = i / nch, c = i - m * nch;
      s_act[i] = reinterpret_cast<const uint4*>(act + (size_t)(t0 + m) * K)[c];
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
                const uint4 xv = s_act[m * nch + c];
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                float xf[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float2 f = bf16x2_to_f32x2(xw[q]);
                  xf[2 * q] = f.x;
                  xf[2 * q + 1] = f.y;
                }
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
            out[(size_t)(t0 + m) * rows + row0 + r] = f32_to_bf16_bits(v);
          }
        }
      }
    }
  }
}

template <int MT, bool GU>
cudaError_t launch_t(int K, int rows, int T, float limit, const uint16_t* act, const uint16_t* w0,
                     const uint16_t* w1, uint16_t* out, cudaStream_t st) {
  const size_t smem = (size_t)MT * K * 2;
  auto kern = bf16_gemv_kernel<MT, GU>;
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
  kern<<<grid, kDgThreads, smem, st>>>(K, rows, T, limit, act, w0, w1, out);
  return cudaGetLastError();
}

template <bool GU>
cudaError_t launch_mt(int K, int rows, int T, float limit, const uint16_t* act, const uint16_t* w0,
                      const uint16_t* w1, uint16_t* out, cudaStream_t st) {
  const size_t budget = 96 * 1024;
  if (T >= 8 && (size_t)8 * K * 2 <= budget) return launch_t<8, GU>(K, rows, T, limit, act, w0, w1, out, st);
  if (T >= 4 && (size_t)4 * K * 2 <= budget) return launch_t<4, GU>(K, rows, T, limit, act, w0, w1, out, st);
  if (T >= 2 && (size_t)2 * K * 2 <= budget) return launch_t<2, GU>(K, rows, T, limit, act, w0, w1, out, st);
  return launch_t<1, GU>(K, rows, T, limit, act, w0, w1, out, st);
}

}  // namespace

cudaError_t launch_dense_gemv(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                              const uint16_t* wu, const uint16_t* wd, uint16_t* y, uint16_t* hbuf, cudaStream_t st) {
  cudaError_t err = launch_mt<true>(H, I, T, limit, x, wg, wu, hbuf, st);
  if (err != cudaSuccess) return err;
  return launch_mt<false>(I, H, T, 0.f, hbuf, wd, nullptr, y, st);
}

cudaError_t launch_dense_ffn(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                             const uint16_t* wu, const uint16_t* wd, uint16_t* y, uint16_t* hbuf, uint32_t* status,
                             cudaStream_t st) {
  if (T >= kDenseGemmMinT && I % 128 == 0 && H % 256 == 0) {
    cudaError_t err = launch_bf16_gemm(true, x, T, H, wg, wu, I, limit, hbuf, status, st);
    if (err != cudaSuccess) return err;
    return launch_bf16_gemm(false, hbuf, T, I, wd, nullptr, H, 0.f, y, status, st);
  }
  return launch_dense_gemv(H, I, limit, x, T, wg, wu, wd, y, hbuf, st);
}

}  // namespace rnx
