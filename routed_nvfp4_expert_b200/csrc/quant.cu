// Prefill data movement around the FP4 grouped GEMM:
//  - the padded tile layout (tile_rows: assignment of each padded row; every
//    local expert starts on a kRowsPerTile = 256-row boundary),
//  - NVFP4 encoding of bf16 activation rows (x gathered per assignment, or h
//    in place) with one fp32 scale per row, an E4M3 scale per 16 elements and
//    E2M1 codes, the scales written straight into the 512-byte atoms the
//    tensor-core scale copy reads,
//  - the one-time re-tiling of the weights' block scales into the same atoms.
//
// Activation encoding (prefill reading of the glm5next_mlp module docs'
// forward_prefill_gemm, W4A4 with a per-row second-level scale), every step
// IEEE fp32 in this order: r = max|row|; ts = r / 2688 (2688 = 6 * 448);
// per 16-block sb = e4m3_rn_satfinite((amax_blk / 6) / ts); d = e4m3(sb) * ts;
// code = e2m1_rn_satfinite(v / d). A zero row has ts = 0 and all scales and
// codes 0; a block with d = 0 gets codes 0.

#include "common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kQuantWarps = 8;

// Byte offset, inside the atoms of a [rows/128][K/64] grid, of the scale of
// row p, 16-element block b (the 32x4x4 atom: lane p%32, 4-byte column
// (p%128)/32, byte b%4 within the 64-element K block).
__host__ __device__ inline long long sf_atom_offset(long long p, int b, int KB) {
  return ((p >> 7) * KB + (b >> 2)) * 512 + (p & 31) * 16 + ((p & 127) >> 5) * 4 + (b & 3);
}

RNX_DEVICE void load16(const uint16_t* src, float (&v)[16]) {
  const uint4 a = *reinterpret_cast<const uint4*>(src);
  const uint4 c = *reinterpret_cast<const uint4*>(src + 8);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = bf16x2_to_f32x2(w[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__global__ void __launch_bounds__(kQuantWarps * 32) quant_rows_kernel(const uint16_t* __restrict__ src, long long rows,
                                                                      long long rows_pad, int K,
                                                                      const int32_t* __restrict__ row_map, int div,
                                                                      const int32_t* __restrict__ used_tiles,
                                                                      uint8_t* __restrict__ codes,
                                                                      uint8_t* __restrict__ sf,
                                                                      float* __restrict__ row_scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long p = (long long)blockIdx.x * kQuantWarps + warp;
  if (p >= rows_pad) return;
  if (used_tiles && p >= (long long)*used_tiles * kRowsPerTile) return;   // past the last tile in use
  const int nblk = K / 16, KB = K / 64;
  long long srow = -1;
  if (p < rows) {
    if (row_map) {
      const int a = row_map[p];
      srow = a < 0 ? -1 : (div > 0 ? a / div : p);
    } else {
      srow = p;
    }
  }
  uint8_t* crow = codes + p * (K / 2);
  if (srow < 0) {
    for (int b = lane; b < nblk; b += 32) {
      if (p < rows) *reinterpret_cast<uint2*>(crow + b * 8) = make_uint2(0, 0);
      sf[sf_atom_offset(p, b, KB)] = 0;
    }
    if (lane == 0 && p < rows) row_scale[p] = 0.f;
    return;
  }
  const uint16_t* x = src + srow * K;
  float m = 0.f;
  for (int b = lane; b < nblk; b += 32) {
    float v[16];
    load16(x + b * 16, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
  }
  m = warp_max(m);
  const float ts = m / 2688.0f;
  for (int b = lane; b < nblk; b += 32) {
    float v[16];
    load16(x + b * 16, v);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const float q = ts == 0.f ? 0.f : (amax / 6.0f) / ts;
    const uint8_t sb = f32_to_e4m3_satfinite(q);
    const float d = e4m3_to_f32(sb) * ts;
    uint32_t w0 = 0, w1 = 0;
    if (d != 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        w0 |= (uint32_t)f32x2_to_e2m1x2_satfinite(v[2 * i] / d, v[2 * i + 1] / d) << (8 * i);
        w1 |= (uint32_t)f32x2_to_e2m1x2_satfinite(v[8 + 2 * i] / d, v[8 + 2 * i + 1] / d) << (8 * i);
      }
    }
    *reinterpret_cast<uint2*>(crow + b * 8) = make_uint2(w0, w1);
    sf[sf_atom_offset(p, b, KB)] = sb;
  }
  if (lane == 0) row_scale[p] = ts;
}

// The prefill's x encoding, token-major: warp t (< T) encodes token t's row
// once and writes it to the padded row of each of its local assignments
// (padded row = tile_offsets[e] * 256 + inv[a] - offsets[e], the row whose
// tile_rows entry is a); warp T + p zeroes padded row p when it is padding
// inside a tile in use. Same arithmetic, in the same order, as
// quant_rows_kernel per row; x is read (and divided) once per token instead
// of once per assignment. k <= 16.
__global__ void __launch_bounds__(kQuantWarps * 32) quant_tokens_kernel(
    const uint16_t* __restrict__ x, int T, int K, int k, const int32_t* __restrict__ ids,
    const int32_t* __restrict__ inv, const int32_t* __restrict__ offsets, const int32_t* __restrict__ tile_offsets,
    int lb, int le, const int32_t* __restrict__ tile_rows, long long P, const int32_t* __restrict__ used_tiles,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ row_scale) {
  __shared__ long long s_p[kQuantWarps][16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long wg = (long long)blockIdx.x * kQuantWarps + warp;
  const int nblk = K / 16, KB = K / 64;
  const long long used = min((long long)*used_tiles * kRowsPerTile, P);
  if (wg >= T) {
    // a padding row of a tile in use: encoded as zeros
    const long long p = wg - T;
    if (p >= used || tile_rows[p] >= 0) return;
    uint8_t* crow = codes + p * (K / 2);
    for (int b = lane; b < nblk; b += 32) {
      *reinterpret_cast<uint2*>(crow + b * 8) = make_uint2(0, 0);
      sf[sf_atom_offset(p, b, KB)] = 0;
    }
    if (lane == 0) row_scale[p] = 0.f;
    return;
  }
  const int t = (int)wg;
  if (lane < k) {
    const long long a = (long long)t * k + lane;
    const int e = ids[a], pos = inv[a];
    long long p = -1;
    if (e >= lb && e < le && pos >= 0) p = (long long)tile_offsets[e] * kRowsPerTile + (pos - offsets[e]);
    s_p[warp][lane] = (p >= 0 && p < used) ? p : -1;
  }
  __syncwarp();
  bool any = false;
  for (int j = 0; j < k; ++j) any = any || s_p[warp][j] >= 0;
  if (!any) return;
  const uint16_t* xr = x + (size_t)t * K;
  float m = 0.f;
  for (int b = lane; b < nblk; b += 32) {
    float v[16];
    load16(xr + b * 16, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
  }
  m = warp_max(m);
  const float ts = m / 2688.0f;
  for (int b = lane; b < nblk; b += 32) {
    float v[16];
    load16(xr + b * 16, v);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const float q = ts == 0.f ? 0.f : (amax / 6.0f) / ts;
    const uint8_t sb = f32_to_e4m3_satfinite(q);
    const float d = e4m3_to_f32(sb) * ts;
    uint32_t w0 = 0, w1 = 0;
    if (d != 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        w0 |= (uint32_t)f32x2_to_e2m1x2_satfinite(v[2 * i] / d, v[2 * i + 1] / d) << (8 * i);
        w1 |= (uint32_t)f32x2_to_e2m1x2_satfinite(v[8 + 2 * i] / d, v[8 + 2 * i + 1] / d) << (8 * i);
      }
    }
    for (int j = 0; j < k; ++j) {
      const long long p = s_p[warp][j];
      if (p < 0) continue;
      *reinterpret_cast<uint2*>(codes + p * (K / 2) + b * 8) = make_uint2(w0, w1);
      sf[sf_atom_offset(p, b, KB)] = sb;
    }
  }
  if (lane < k && s_p[warp][lane] >= 0) row_scale[s_p[warp][lane]] = ts;
}

// tile_rows[p] for p < P_max.
__global__ void __launch_bounds__(256) tile_rows_kernel(const int32_t* __restrict__ counts,
                                                        const int32_t* __restrict__ offsets,
                                                        const int32_t* __restrict__ sorted,
                                                        const int32_t* __restrict__ tile_offsets, int E,
                                                        long long P_max, int32_t* __restrict__ tile_rows) {
  const int ntiles = tile_offsets[E];
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < P_max;
       p += (long long)gridDim.x * blockDim.x) {
    const int mt = (int)(p / kRowsPerTile);
    int a = -1;
    if (mt < ntiles) {
      int lo = 0, hi = E;   // largest e with tile_offsets[e] <= mt
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_offsets[mid] <= mt) lo = mid; else hi = mid;
      }
      const int row = (mt - tile_offsets[lo]) * kRowsPerTile + (int)(p % kRowsPerTile);
      if (row < counts[lo]) a = sorted[offsets[lo] + row];
    }
    tile_rows[p] = a;
  }
}

__global__ void __launch_bounds__(256) sf_atoms_kernel(const uint8_t* __restrict__ scales, long long total_rows, int K,
                                                       uint8_t* __restrict__ atoms) {
  const int KB = K / 64;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total_rows * KB;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long R = idx / KB;
    const int kb = (int)(idx - R * KB);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(scales + R * (K / 16) + kb * 4);
    *reinterpret_cast<uint32_t*>(atoms + sf_atom_offset(R, kb * 4, KB)) = w;
  }
}

int grid_for(long long work, int per_block) {
  const long long g = (work + per_block - 1) / per_block;
  return (int)std::max(1LL, std::min(g, (long long)kNumSMs * 16));
}

}  // namespace

int64_t padded_rows_bound(int64_t A, int64_t E_local) {
  const int64_t n = std::min(A, E_local);
  return (A + (kRowsPerTile - 1) * n) / kRowsPerTile * kRowsPerTile;
}

cudaError_t launch_tile_rows(const moe_plan_t& plan, int E, int64_t P_max, cudaStream_t st) {
  if (P_max <= 0) return cudaSuccess;
  tile_rows_kernel<<<grid_for(P_max, 256), 256, 0, st>>>(plan.counts, plan.offsets, plan.sorted, plan.tile_offsets, E,
                                                         P_max, plan.tile_rows);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(const uint16_t* src, int64_t rows, int K, const int32_t* row_map, int div,
                              const int32_t* used_tiles, uint8_t* codes, uint8_t* sf, float* row_scale,
                              cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const long long rows_pad = (rows + 127) / 128 * 128;   // whole 128-row scale atoms
  const long long grid = (rows_pad + kQuantWarps - 1) / kQuantWarps;
  quant_rows_kernel<<<(unsigned)grid, kQuantWarps * 32, 0, st>>>(src, rows, rows_pad, K, row_map, div, used_tiles,
                                                                  codes, sf, row_scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_tokens(const uint16_t* x, int T, int K, int k, const int32_t* ids, const moe_plan_t& plan,
                                int lb, int le, int64_t P, const int32_t* used_tiles, uint8_t* codes, uint8_t* sf,
                                float* row_scale, cudaStream_t st) {
  if (k > 16) return cudaErrorNotSupported;
  const long long warps = (long long)T + P;
  if (warps <= 0) return cudaSuccess;
  const long long grid = (warps + kQuantWarps - 1) / kQuantWarps;
  quant_tokens_kernel<<<(unsigned)grid, kQuantWarps * 32, 0, st>>>(x, T, K, k, ids, plan.inv, plan.offsets,
                                                                   plan.tile_offsets, lb, le, plan.tile_rows, P,
                                                                   used_tiles, codes, sf, row_scale);
  return cudaGetLastError();
}

namespace {
// Gate and up scales of E experts ([E*I, K/16] each) as one atom grid whose
// 128-row atoms hold 64 gate rows then the same 64 up rows: interleaved row
// R = (e * I/64 + j) * 128 + m is gate row e*I + 64 j + m (m < 64) or up row
// e*I + 64 j + m - 64.
__global__ void __launch_bounds__(256) sf_atoms_gu_kernel(const uint8_t* __restrict__ gate,
                                                          const uint8_t* __restrict__ up, long long total_rows, int I,
                                                          int K, uint8_t* __restrict__ atoms) {
  const int KB = K / 64;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total_rows * KB;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long R = idx / KB;
    const int kb = (int)(idx - R * KB);
    const long long blk = R >> 7;                 // e * I/64 + j
    const int m = (int)(R & 127);
    const long long e = blk / (I / 64), j = blk - e * (I / 64);
    const long long src = e * I + 64 * j + (m & 63);
    const uint8_t* bank = m < 64 ? gate : up;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(bank + src * (K / 16) + kb * 4);
    *reinterpret_cast<uint32_t*>(atoms + sf_atom_offset(R, kb * 4, KB)) = w;
  }
}
}  // namespace

cudaError_t launch_sf_atoms_gate_up(const uint8_t* gate, const uint8_t* up, int64_t n_experts, int I, int K,
                                    uint8_t* atoms, cudaStream_t st) {
  const long long total = 2LL * n_experts * I;
  if (total <= 0) return cudaSuccess;
  sf_atoms_gu_kernel<<<grid_for(total * (K / 64), 256), 256, 0, st>>>(gate, up, total, I, K, atoms);
  return cudaGetLastError();
}

cudaError_t launch_sf_atoms(const uint8_t* scales, int64_t n_experts, int rows, int K, uint8_t* atoms,
                            cudaStream_t st) {
  const long long total = (long long)n_experts * rows;
  if (total <= 0) return cudaSuccess;
  sf_atoms_kernel<<<grid_for(total * (K / 64), 256), 256, 0, st>>>(scales, total, K, atoms);
  return cudaGetLastError();
}

}  // namespace rnx
