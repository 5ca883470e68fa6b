// Decode expert projections: bf16 x / fp32 h activations x NVFP4 weights
// (W4A16), several tokens per expert.
//
// glm5next_mlp module docs, Constants / W4A16_GEMV_MODULE: at decode every
// routed-expert projection is a GEMV over the touched experts' bytes. This
// form serves T > 1: a work-item loop over (active expert, block of rows)
// whose CTA stages the expert's token rows in shared memory once (f16, scaled
// by a power of two per row) and applies each weight row to all of them. The
// single-token step runs the streamed kernels of decode_t1.cu instead.
//
// Products code * activation are exact (E2M1 and the pre-scaled activation
// are f16 values) and accumulate in fp32 (mixed-precision fma); each
// 16-element block sum is scaled by its E4M3 scale in fp32. GATE_UP fuses the
// clamped SwiGLU and writes h (fp32) per assignment; DOWN multiplies by the
// routing weight and writes r[t, j] (fp32).

#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * kWarp;

struct GemvParams {
  int K;           // reduction length (H for GATE_UP, I for DOWN)
  int rows;        // output rows per expert (I for GATE_UP, H for DOWN)
  int k;           // top_k
  int A;           // assignments T*k
  int E;
  int local_begin, local_end;
  float limit;
  const void* act;            // GATE_UP: x bf16 [T, K]; DOWN: h fp32 [A, K]
  const int32_t* offsets;     // [E+1]
  const int32_t* sorted;      // [A]
  const int32_t* active;      // [E+1]
  const float* weights;       // [A] routing weights (DOWN)
  const uint8_t* codes0;      // gate (GATE_UP) or down (DOWN) [E, rows, K/2]
  const uint8_t* scales0;     // [E, rows, K/16]
  const float* ts0;           // [E]
  const uint8_t* codes1;      // up (GATE_UP only)
  const uint8_t* scales1;
  const float* ts1;
  float* out;                 // GATE_UP: h [A, rows]; DOWN: r [A, rows]
};

// Shared-memory activation layout: row m, 16-byte unit index
//   ((m * NI + i) * 4 + q) * 32 + lane
// holds elements [32*c + 8*q, 32*c + 8*q + 8) of chunk c = 32*i + lane, so
// the 32 lanes of a warp read 512 contiguous bytes (conflict-free).
RNX_DEVICE int act_unit(int m, int NI, int c, int q) {
  return ((m * NI + (c >> 5)) * 4 + q) * 32 + (c & 31);
}

// Eight activations of a row (bf16 x or fp32 h) as fp32.
template <bool GATE_UP>
RNX_DEVICE void load8(const void* row, int g, float (&f)[8]) {
  if (GATE_UP) {
    const uint4 v = reinterpret_cast<const uint4*>(row)[g];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 t = bf16x2_to_f32x2(w[j]);
      f[2 * j] = t.x;
      f[2 * j + 1] = t.y;
    }
  } else {
    const float4 a = reinterpret_cast<const float4*>(row)[2 * g], b = reinterpret_cast<const float4*>(row)[2 * g + 1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}

// Stage the activation rows of one token pass into shared memory: f16 scaled
// by the power of two that brings the row's max |a| into [2^14, 2^15).
template <bool GATE_UP>
RNX_DEVICE void stage_rows(const GemvParams& p, int seg0, int nm, uint4* s_act, float* s_unscale, int NI) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ngroups = p.K >> 3;   // groups of 8 elements
  for (int m = warp; m < nm; m += kGemvWarps) {
    const int a = p.sorted[seg0 + m];
    // GATE_UP reads the token's x row, DOWN the assignment's h row
    const void* row = GATE_UP ? (const void*)((const uint16_t*)p.act + (size_t)(a / p.k) * p.K)
                              : (const void*)((const float*)p.act + (size_t)a * p.K);
    float mx = 0.f;
    for (int g = lane; g < ngroups; g += 32) {
      float f[8];
      load8<GATE_UP>(row, g, f);
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(f[j]));
    }
    mx = warp_max(mx);
    float up, unscale;
    prescale15(mx, up, unscale);
    if (lane == 0) s_unscale[m] = unscale;
    for (int g = lane; g < ngroups; g += 32) {
      float f[8];
      load8<GATE_UP>(row, g, f);
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __half2 h = __floats2half2_rn(f[2 * j] * up, f[2 * j + 1] * up);
        o[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      const int c = g >> 2, q = g & 3;
      s_act[act_unit(m, NI, c, q)] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Accumulate one 32-element chunk of one weight row against nm staged rows.
template <int MT>
RNX_DEVICE void chunk_dot_rows(uint4 q, uint16_t sc, const uint4* s_act, int NI, int c, int nm, float (&acc)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m < nm) {
      const uint4 x0 = s_act[act_unit(m, NI, c, 0)];
      const uint4 x1 = s_act[act_unit(m, NI, c, 1)];
      const uint4 x2 = s_act[act_unit(m, NI, c, 2)];
      const uint4 x3 = s_act[act_unit(m, NI, c, 3)];
      const uint32_t xa[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                               x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
      acc[m] = chunk_dot_f32(q, sc, xa, acc[m]);
    }
  }
}

template <int MT, int RPW, bool GATE_UP>
__global__ void __launch_bounds__(kGemvThreads)
nvfp4_gemv_kernel(GemvParams p) {
  extern __shared__ uint4 smem_u4[];
  __shared__ float s_unscale[MT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NI = (p.K / 32 + 31) / 32;            // chunks per lane
  const int nchunks = p.K / 32;
  const int rows_per_item = kGemvWarps * RPW;
  const int ipe = p.rows / rows_per_item;
  pdl_wait();
  pdl_trigger();
  const int n_active = p.active[0];
  const int n_items = n_active * ipe;
  constexpr int NB = GATE_UP ? 2 : 1;             // weight banks per row
  constexpr int MAXNI = 4;                        // K <= 4096 held in registers at once

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int u = item / ipe, rb = item - u * ipe;
    const int e = p.active[1 + u];
    const int seg0 = p.offsets[e], seg1 = p.offsets[e + 1];
    const int row0 = rb * rows_per_item + warp * RPW;

    for (int t0 = seg0; t0 < seg1; t0 += MT) {
      const int nm = min(MT, seg1 - t0);
      __syncthreads();                              // previous pass done with smem
      stage_rows<GATE_UP>(p, t0, nm, smem_u4, s_unscale, NI);
      __syncthreads();

      float acc[RPW][NB][MT];
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[r][b][m] = 0.f;

      for (int i0 = 0; i0 < NI; i0 += MAXNI) {
        // issue every weight load of this warp's rows first
        uint4 q[RPW][NB][MAXNI];
        uint16_t sc[RPW][NB][MAXNI];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const uint8_t* cb = (b == 0 ? p.codes0 : p.codes1) + ((size_t)e * p.rows + row0 + r) * (p.K / 2);
            const uint8_t* sb = (b == 0 ? p.scales0 : p.scales1) + ((size_t)e * p.rows + row0 + r) * (p.K / 16);
#pragma unroll
            for (int ii = 0; ii < MAXNI; ++ii) {
              const int c = (i0 + ii) * 32 + lane;
              if (i0 + ii < NI && c < nchunks) {
                q[r][b][ii] = ldg_stream(cb + 16 * c);
                sc[r][b][ii] = ldg_u16(sb + 2 * c);
              } else {
                q[r][b][ii] = make_uint4(0, 0, 0, 0);
                sc[r][b][ii] = 0;
              }
            }
          }
        }
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
          for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int ii = 0; ii < MAXNI; ++ii) {
              const int c = (i0 + ii) * 32 + lane;
              if (i0 + ii < NI && c < nchunks)
                chunk_dot_rows<MT>(q[r][b][ii], sc[r][b][ii], smem_u4, NI, c, nm, acc[r][b]);
            }
      }

      // reduce over lanes, then lane m stores token m
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const int row = row0 + r;
        float tot[NB][MT];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int m = 0; m < MT; ++m) tot[b][m] = warp_sum(acc[r][b][m]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (lane == m && m < nm) {
            const int a = p.sorted[t0 + m];
            const float us = s_unscale[m];
            if (GATE_UP) {
              const float g = tot[0][m] * us * p.ts0[e];
              const float uu = tot[NB - 1][m] * us * p.ts1[e];
              p.out[(size_t)a * p.rows + row] = clamped_swiglu(g, uu, p.limit);
            } else {
              const float o = tot[0][m] * us * p.ts0[e];
              p.out[(size_t)a * p.rows + row] = o * p.weights[a];
            }
          }
        }
      }
    }
  }

  if (!GATE_UP) {
    // remote assignments contribute zero rows
    // (positions past offsets[E] hold no assignment: ids dropped by the plan)
    const int rb0 = p.offsets[p.local_begin], re0 = p.offsets[p.local_end], rend = p.offsets[p.E];
    const int nremote = rb0 + (rend - re0);
    const int rows4 = p.rows / 4;  // 16-byte units per row
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long long)nremote * rows4;
         idx += (long long)gridDim.x * blockDim.x) {
      const int rp = (int)(idx / rows4), col = (int)(idx - (long long)rp * rows4);
      const int pos = rp < rb0 ? rp : re0 + (rp - rb0);
      const int a = p.sorted[pos];
      reinterpret_cast<float4*>(p.out + (size_t)a * p.rows)[col] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

template <int MT, int RPW, bool GU>
cudaError_t launch_t(const GemvParams& p, int max_items, cudaStream_t st) {
  const int NI = (p.K / 32 + 31) / 32;
  const size_t smem = (size_t)MT * NI * 4 * 32 * 16;
  auto kern = nvfp4_gemv_kernel<MT, RPW, GU>;
  // attribute + occupancy once per (instantiation, smem size): keeps these
  // calls out of any later stream capture
  static size_t cached_smem = 0;
  static int per_sm = 0;
  if (cached_smem != smem) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
    if (err != cudaSuccess) return err;
    cached_smem = smem;
  }
  int grid = std::max(1, std::min(max_items, kNumSMs * std::max(per_sm, 1)));
  return launch_pdl(kern, dim3(grid), dim3(kGemvThreads), smem, st, p);
}

GemvParams gemv_params(const ExpertGemvArgs& a, bool gu) {
  GemvParams p{};
  p.K = gu ? a.H : a.I;
  p.rows = gu ? a.I : a.H;
  p.k = a.k;
  p.A = a.T * a.k;
  p.E = a.E;
  p.local_begin = a.local_begin;
  p.local_end = a.local_end;
  p.limit = a.limit;
  p.act = a.act;
  p.offsets = a.offsets;
  p.sorted = a.sorted;
  p.active = a.active;
  p.weights = a.weights;
  if (gu) {
    p.codes0 = a.gate.codes; p.scales0 = a.gate.scales; p.ts0 = a.gate.tensor_scale;
    p.codes1 = a.up.codes;   p.scales1 = a.up.scales;   p.ts1 = a.up.tensor_scale;
  } else {
    p.codes0 = a.down.codes; p.scales0 = a.down.scales; p.ts0 = a.down.tensor_scale;
    p.codes1 = nullptr;      p.scales1 = nullptr;       p.ts1 = nullptr;
  }
  p.out = a.out;
  return p;
}

}  // namespace


cudaError_t launch_nvfp4_gemv(const ExpertGemvArgs& a, cudaStream_t st) {
  const bool gu = a.proj == MOE_PROJ_GATE_UP;
  const GemvParams p = gemv_params(a, gu);
  const int max_active = std::min(a.local_end - a.local_begin, p.A);
  const int max_tok = a.T;   // tokens per expert never exceed T (ids in a row are distinct)
  if (gu) {
    const int ipe = p.rows / (kGemvWarps * 1);
    const int items = max_active * ipe;
    if (max_tok <= 1) return launch_t<1, 1, true>(p, items, st);
    if (max_tok <= 2) return launch_t<2, 1, true>(p, items, st);
    if (max_tok <= 4) return launch_t<4, 1, true>(p, items, st);
    return launch_t<8, 1, true>(p, items, st);
  } else {
    const int rpw = 2;
    const int ipe = p.rows / (kGemvWarps * rpw);
    const int items = std::max(1, max_active * ipe);
    if (max_tok <= 1) return launch_t<1, 2, false>(p, items, st);
    if (max_tok <= 2) return launch_t<2, 2, false>(p, items, st);
    if (max_tok <= 4) return launch_t<4, 2, false>(p, items, st);
    return launch_t<8, 2, false>(p, items, st);
  }
}

}  // namespace rnx
