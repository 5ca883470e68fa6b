// HBM-bound elementwise steps: moe_combine, standalone clamped SwiGLU, and
// the NVFP4 dequantiser used to check the format bit for bit.

#include "common.cuh"
#include "kernels.h"

namespace rnx {

constexpr int kMaxTopKRows = 16;   // k <= 16 (the pages' KERNEL_MAX_TOP_K)

namespace {

// moe_combine (glm5next_mlp, "The stack this layer runs" / "Traps"): the k
// routed rows in rank order, then the unscaled shared row, fp32 accumulation,
// one rounding to bf16. Each thread owns 8 consecutive hidden elements.
__global__ void __launch_bounds__(256) combine_kernel(int T, int k, int H, const uint16_t* __restrict__ r,
                                                      const uint16_t* __restrict__ shared, uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int per_row = H >> 3;
  const long long n = (long long)T * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_row), c = (int)(i - (long long)t * per_row);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const uint4 v = reinterpret_cast<const uint4*>(r + ((size_t)t * k + j) * H)[c];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = bf16x2_to_f32x2(w[q]);
        acc[2 * q] += f.x;
        acc[2 * q + 1] += f.y;
      }
    }
    if (shared) {
      const uint4 v = reinterpret_cast<const uint4*>(shared + (size_t)t * H)[c];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = bf16x2_to_f32x2(w[q]);
        acc[2 * q] += f.x;
        acc[2 * q + 1] += f.y;
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4*>(y + (size_t)t * H)[c] = o;
  }
}

// moe_combine over fp32 rows (the decode path keeps r and the shared row in
// fp32): the same order and one rounding. Each thread owns 4 consecutive
// hidden elements; its k + 1 loads go out together before the sum.
__global__ void __launch_bounds__(128) combine_f32_kernel(int T, int k, int H, const float* __restrict__ r,
                                                          const float* __restrict__ shared, uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int per_row = H >> 2;
  const long long n = (long long)T * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_row), c = (int)(i - (long long)t * per_row);
    float4 v[kMaxTopKRows];
#pragma unroll
    for (int j = 0; j < kMaxTopKRows; ++j)
      v[j] = j < k ? reinterpret_cast<const float4*>(r + ((size_t)t * k + j) * H)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 sv = shared ? reinterpret_cast<const float4*>(shared + (size_t)t * H)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxTopKRows; ++j) {
      if (j < k) {
        acc.x += v[j].x;
        acc.y += v[j].y;
        acc.z += v[j].z;
        acc.w += v[j].w;
      }
    }
    if (shared) {
      acc.x += sv.x;
      acc.y += sv.y;
      acc.z += sv.z;
      acc.w += sv.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    reinterpret_cast<uint2*>(y + (size_t)t * H)[c] = o;
  }
}

// Padded-layout row of assignment a (the prefill down projection writes its
// rows there), -1 when its expert is outside the local range or the id was
// dropped. tile_offsets are in kRowsPerTile-row tiles.
RNX_DEVICE long long padded_pos(const PaddedIndex& q, long long a) {
  const int e = q.ids[a];
  if (e < q.local_begin || e >= q.local_end) return -1;
  const int ia = q.inv[a];
  if (ia < 0) return -1;
  return (long long)q.tile_offsets[e] * kRowsPerTile + (ia - q.offsets[e]);
}

RNX_DEVICE void add_bf16x8(float (&acc)[8], uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = bf16x2_to_f32x2(w[q]);
    acc[2 * q] += f.x;
    acc[2 * q + 1] += f.y;
  }
}

// Unpermute fused with moe_combine: y[t] = bf16(sum_j rows[pos(t, j)] +
// shared[t]), j ascending then the shared row, fp32 accumulation; a remote
// assignment adds a zero row (the same arithmetic as moe_combine over the
// gathered rows). One CTA per token at a time; positions staged in shared.
__global__ void __launch_bounds__(256) unpermute_combine_kernel(PaddedIndex q, int T, int k, int H,
                                                                const float* __restrict__ rows,
                                                                const float* __restrict__ shared,
                                                                uint16_t* __restrict__ y) {
  __shared__ long long pos[16];
  const int per_row = H >> 2;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < k) pos[threadIdx.x] = padded_pos(q, (long long)t * k + threadIdx.x);
    __syncthreads();
    for (int c = threadIdx.x; c < per_row; c += blockDim.x) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < k; ++j) {
        const long long pr = pos[j];
        const float4 v =
            pr >= 0 ? reinterpret_cast<const float4*>(rows + (size_t)pr * H)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      if (shared) {
        const float4 v = reinterpret_cast<const float4*>(shared + (size_t)t * H)[c];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      reinterpret_cast<uint2*>(y + (size_t)t * H)[c] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
  }
}

// Unpermute alone: out[t, j] = rows[pos(t, j)] (zeros for remote assignments).
__global__ void __launch_bounds__(256) unpermute_kernel(PaddedIndex q, long long A, int H,
                                                        const float* __restrict__ rows, float* __restrict__ out) {
  const int per_row = H >> 2;
  const long long n = A * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long a = i / per_row;
    const int c = (int)(i - a * per_row);
    const long long pr = padded_pos(q, a);
    reinterpret_cast<float4*>(out + (size_t)a * H)[c] =
        pr >= 0 ? reinterpret_cast<const float4*>(rows + (size_t)pr * H)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

__global__ void __launch_bounds__(256) swiglu_kernel(const float* __restrict__ gu, int M, int I, float limit,
                                                     uint16_t* __restrict__ h) {
  const int per_row = I >> 2;
  const long long n = (long long)M * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i / per_row), c = (int)(i - (long long)m * per_row);
    const float4 g = reinterpret_cast<const float4*>(gu + (size_t)m * 2 * I)[c];
    const float4 u = reinterpret_cast<const float4*>(gu + (size_t)m * 2 * I + I)[c];
    uint2 o;
    o.x = pack_bf16x2(clamped_swiglu(g.x, u.x, limit), clamped_swiglu(g.y, u.y, limit));
    o.y = pack_bf16x2(clamped_swiglu(g.z, u.z, limit), clamped_swiglu(g.w, u.w, limit));
    reinterpret_cast<uint2*>(h + (size_t)m * I)[c] = o;
  }
}

// One thread per 16-element block: e2m1 * e4m3 (exact in fp32) * tensor scale
// (one rounding).
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ codes,
                                                      const uint8_t* __restrict__ scales,
                                                      const float* __restrict__ ts, int rows, int K,
                                                      float* __restrict__ out) {
  const int nb = K >> 4;
  const long long n = (long long)rows * nb;
  const float t = ts[0];
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const uint2 q = reinterpret_cast<const uint2*>(codes)[i];
    const float s = e4m3_to_f32(scales[i]);
    uint32_t h[8];
    e2m1x8_to_f16x2x4(q.x, h[0], h[1], h[2], h[3]);
    e2m1x8_to_f16x2x4(q.y, h[4], h[5], h[6], h[7]);
    float4* o = reinterpret_cast<float4*>(out + i * 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h[2 * j]));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h[2 * j + 1]));
      o[j] = make_float4(__fmul_rn(__fmul_rn(a.x, s), t), __fmul_rn(__fmul_rn(a.y, s), t),
                         __fmul_rn(__fmul_rn(b.x, s), t), __fmul_rn(__fmul_rn(b.y, s), t));
    }
  }
}

int grid_for(long long n, int threads) {
  const long long want = (n + threads - 1) / threads;
  return (int)std::max<long long>(1, std::min<long long>(want, (long long)kNumSMs * 16));
}

}  // namespace

cudaError_t launch_combine(int T, int k, int H, const uint16_t* r, const uint16_t* shared, uint16_t* y,
                           cudaStream_t st) {
  return launch_pdl(combine_kernel, dim3(grid_for((long long)T * (H / 8), 256)), dim3(256), 0, st, T, k, H, r, shared,
                    y);
  return cudaGetLastError();
}

cudaError_t launch_combine_f32(int T, int k, int H, const float* r, const float* shared, uint16_t* y,
                               cudaStream_t st) {
  if (k > kMaxTopKRows) return cudaErrorInvalidValue;
  return launch_pdl(combine_f32_kernel, dim3(grid_for((long long)T * (H / 4), 128)), dim3(128), 0, st, T, k, H, r,
                    shared, y);
}

cudaError_t launch_unpermute_combine(const PaddedIndex& q, int T, int k, int H, const float* rows,
                                     const float* shared, uint16_t* y, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int grid = std::min(T, kNumSMs * 8);
  unpermute_combine_kernel<<<grid, 256, 0, st>>>(q, T, k, H, rows, shared, y);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const PaddedIndex& q, long long A, int H, const float* rows, float* out,
                             cudaStream_t st) {
  if (A <= 0) return cudaSuccess;
  const long long work = A * (H >> 2);
  const int grid = (int)std::min<long long>((work + 255) / 256, (long long)kNumSMs * 16);
  unpermute_kernel<<<grid, 256, 0, st>>>(q, A, H, rows, out);
  return cudaGetLastError();
}

cudaError_t launch_swiglu(const float* gu, int M, int I, float limit, uint16_t* h, cudaStream_t st) {
  swiglu_kernel<<<grid_for((long long)M * (I / 4), 256), 256, 0, st>>>(gu, M, I, limit, h);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts, int rows, int K, float* out,
                           cudaStream_t st) {
  dequant_kernel<<<grid_for((long long)rows * (K / 16), 256), 256, 0, st>>>(codes, scales, ts, rows, K, out);
  return cudaGetLastError();
}

}  // namespace rnx
