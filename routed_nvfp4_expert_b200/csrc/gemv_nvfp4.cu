// Decode expert projections: bf16 activations x NVFP4 weights (W4A16).
//
// glm5next_mlp module docs, Constants / W4A16_GEMV_MODULE: at decode every
// routed-expert projection is M=1, and a tile GEMM measured far below the
// memory roofline there; the decode weight kernel must stream each touched
// expert's bytes once at HBM speed. This kernel does exactly that:
//
//  * work item = (active local expert, block of 8*RPW output rows); a
//    persistent grid loops over items;
//  * each warp streams RPW weight rows with 128-bit non-allocating loads
//    (lane l reads the 16-byte chunks l, l+32, ... of a row: 32 E2M1 codes,
//    two 16-element scale blocks);
//  * E2M1 pairs become f16x2 with the hardware cvt, and multiply-add into a
//    per-16-block f16x2 partial against the activations (staged once per
//    item in shared memory as f16, pre-scaled per row by a power of two so
//    that |a| < 256: products are exact in f16, an 8-term half-block sum
//    stays far inside the f16 range); each block partial is widened to fp32
//    and scaled by its E4M3 block scale into an fp32 accumulator;
//  * all tokens routed to the expert reuse the same weight registers.
//
// GATE_UP fuses the clamped SwiGLU and writes h (bf16) per assignment;
// DOWN multiplies by the routing weight and writes r[t, j] (bf16).

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

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
  const uint16_t* act;        // GATE_UP: x [T, K]; DOWN: h [A, K]
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
  uint16_t* out;              // GATE_UP: h [A, rows]; DOWN: r [A, rows]
};

// Shared-memory activation layout: row m, 16-byte unit index
//   ((m * NI + i) * 4 + q) * 32 + lane
// holds elements [32*c + 8*q, 32*c + 8*q + 8) of chunk c = 32*i + lane, so
// the 32 lanes of a warp read 512 contiguous bytes (conflict-free).
RNX_DEVICE int act_unit(int m, int NI, int c, int q) {
  return ((m * NI + (c >> 5)) * 4 + q) * 32 + (c & 31);
}

// Stage activation rows of one token pass into shared memory (f16, pre-scaled).
template <bool GATE_UP>
RNX_DEVICE void stage_rows(const GemvParams& p, int seg0, int nm, uint4* s_act, float* s_unscale, int NI) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ngroups = p.K >> 3;   // 8 bf16 per 16-byte group
  for (int m = warp; m < nm; m += kGemvWarps) {
    const int a = p.sorted[seg0 + m];
    // GATE_UP reads the token's x row, DOWN the assignment's h row
    const uint16_t* row = p.act + (size_t)(GATE_UP ? a / p.k : a) * p.K;
    float mx = 0.f;
    for (int g = lane; g < ngroups; g += 32) {
      uint4 v = *reinterpret_cast<const uint4*>(row + 8 * g);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = bf16x2_to_f32x2(w[j]);
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    mx = warp_max(mx);
    int ex = 0;
    if (mx > 0.f && mx <= 3.0e38f) frexpf(mx, &ex);   // mx = f * 2^ex, f in [0.5, 1)
    const float up = ldexpf(1.0f, 8 - ex);             // pre-scaled max in [128, 256)
    if (lane == 0) s_unscale[m] = ldexpf(1.0f, ex - 8);
    for (int g = lane; g < ngroups; g += 32) {
      uint4 v = *reinterpret_cast<const uint4*>(row + 8 * g);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = bf16x2_to_f32x2(w[j]);
        __half2 h = __floats2half2_rn(f.x * up, f.y * up);
        o[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      const int c = g >> 2, q = g & 3;
      s_act[act_unit(m, NI, c, q)] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Accumulate one 32-element chunk of one weight row against nm activation rows.
template <int MT>
RNX_DEVICE void chunk_dot(uint4 q, uint16_t sc, const uint4* s_act, int NI, int c, int nm, float (&acc)[MT]) {
  uint32_t w[16];
  e2m1x8_to_f16x2x4(q.x, w[0], w[1], w[2], w[3]);
  e2m1x8_to_f16x2x4(q.y, w[4], w[5], w[6], w[7]);
  e2m1x8_to_f16x2x4(q.z, w[8], w[9], w[10], w[11]);
  e2m1x8_to_f16x2x4(q.w, w[12], w[13], w[14], w[15]);
  const float2 s = e4m3x2_to_f32x2(sc);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m < nm) {
      uint4 x0 = s_act[act_unit(m, NI, c, 0)];
      uint4 x1 = s_act[act_unit(m, NI, c, 1)];
      uint4 x2 = s_act[act_unit(m, NI, c, 2)];
      uint4 x3 = s_act[act_unit(m, NI, c, 3)];
      const uint32_t xa[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                               x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
      __half2 p0 = __float2half2_rn(0.f), p1 = __float2half2_rn(0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        p0 = __hfma2(*reinterpret_cast<const __half2*>(&w[j]), *reinterpret_cast<const __half2*>(&xa[j]), p0);
#pragma unroll
      for (int j = 8; j < 16; ++j)
        p1 = __hfma2(*reinterpret_cast<const __half2*>(&w[j]), *reinterpret_cast<const __half2*>(&xa[j]), p1);
      const float2 f0 = __half22float2(p0), f1 = __half22float2(p1);
      acc[m] = fmaf(s.x, f0.x + f0.y, acc[m]);
      acc[m] = fmaf(s.y, f1.x + f1.y, acc[m]);
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
              if (i0 + ii < NI && c < nchunks) chunk_dot<MT>(q[r][b][ii], sc[r][b][ii], smem_u4, NI, c, nm, acc[r][b]);
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
              p.out[(size_t)a * p.rows + row] = f32_to_bf16_bits(clamped_swiglu(g, uu, p.limit));
            } else {
              const float o = tot[0][m] * us * p.ts0[e];
              p.out[(size_t)a * p.rows + row] = f32_to_bf16_bits(o * p.weights[a]);
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
    const int rows16 = p.rows / 8;  // 16-byte units per row
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long long)nremote * rows16;
         idx += (long long)gridDim.x * blockDim.x) {
      const int rp = (int)(idx / rows16), col = (int)(idx - (long long)rp * rows16);
      const int pos = rp < rb0 ? rp : re0 + (rp - rb0);
      const int a = p.sorted[pos];
      reinterpret_cast<uint4*>(p.out + (size_t)a * p.rows)[col] = make_uint4(0, 0, 0, 0);
    }
  }
}

// ---------------------------------------------------------------------------
// Streaming form (few tokens per expert, the decode case): a producer warp
// moves each work item -- S consecutive rows of one expert, which are
// contiguous in HBM -- into a ring of shared-memory stages with bulk copies on
// the TMA engine (cp.async.bulk, evict-first L2 policy), completion tracked by
// mbarriers; 8 consumer warps compute from shared memory. A consumer lane
// always owns the same 32-element K chunks (c = lane + 32 i), so the token's
// activations stay in its registers as pre-scaled f16 for the whole kernel and
// are reloaded only when the item's token set changes.
constexpr int kStreamConsumers = 8;
constexpr int kStreamThreads = (kStreamConsumers + 1) * kWarp;

struct StreamShape {
  int S;            // rows per stage (row pairs for GATE_UP)
  int NS;           // stages in the ring
  uint32_t stage_bytes;
};

template <int MT, int NI, bool GATE_UP>
__global__ void __launch_bounds__(kStreamThreads, 1)
nvfp4_gemv_stream_kernel(GemvParams p, StreamShape sh, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[16];
  __shared__ __align__(8) uint64_t empty_bar[16];
  __shared__ volatile int abort_flag;
  constexpr int NB = GATE_UP ? 2 : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = sh.S, NS = sh.NS;
  const int RW = S / kStreamConsumers;          // rows per consumer warp per stage
  const int codes_row = p.K / 2, scales_row = p.K / 16;
  const int nchunks = p.K / 32;
  const int ipe = p.rows / S;
  const int n_items = p.active[0] * ipe;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kStreamConsumers);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // stage layout: [bank0 codes S rows][bank1 codes][bank0 scales][bank1 scales]
  auto stage_ptr = [&](int s) { return smem + (size_t)s * sh.stage_bytes; };

  if (warp == kStreamConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
        const int s = it % NS;
        const uint32_t ph = (uint32_t)(it / NS) & 1u;
        if (!mbar_wait(&empty_bar[s], ph ^ 1u) || abort_flag) {
          set_status(status, kDevErrTimeout);
          abort_flag = 1;
          break;
        }
        const int u = item / ipe, rb = item - u * ipe;
        const int e = p.active[1 + u];
        const size_t row0 = (size_t)e * p.rows + (size_t)rb * S;
        uint8_t* st = stage_ptr(s);
        mbar_arrive_expect_tx(&full_bar[s], sh.stage_bytes);
        bulk_g2s(st, p.codes0 + row0 * codes_row, S * codes_row, &full_bar[s], pol);
        if (GATE_UP) bulk_g2s(st + S * codes_row, p.codes1 + row0 * codes_row, S * codes_row, &full_bar[s], pol);
        uint8_t* sc = st + NB * S * codes_row;
        bulk_g2s(sc, p.scales0 + row0 * scales_row, S * scales_row, &full_bar[s], pol);
        if (GATE_UP) bulk_g2s(sc + S * scales_row, p.scales1 + row0 * scales_row, S * scales_row, &full_bar[s], pol);
      }
      // drain: never leave the CTA with copies still writing its shared memory
      const int issued = it;
      for (int j = max(0, issued - NS); j < issued; ++j) {
        if (!mbar_wait(&full_bar[j % NS], (uint32_t)(j / NS) & 1u)) set_status(status, kDevErrTimeout);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  uint32_t xr[MT][NI][16];        // activations, f16x2, pre-scaled
  float unscale[MT];
  int key[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) key[m] = -1;

  int it = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
    const int s = it % NS;
    const uint32_t ph = (uint32_t)(it / NS) & 1u;
    const int u = item / ipe, rb = item - u * ipe;
    const int e = p.active[1 + u];
    const int seg0 = p.offsets[e];
    const int nm = min(MT, p.offsets[e + 1] - seg0);

    // (re)load this expert's activation rows into registers while the stage lands
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < nm) {
        const int a = p.sorted[seg0 + m];
        const int src = GATE_UP ? a / p.k : a;
        if (src != key[m]) {
          key[m] = src;
          const uint16_t* row = p.act + (size_t)src * p.K;
          uint4 raw[NI][4];
          float mx = 0.f;
#pragma unroll
          for (int i = 0; i < NI; ++i) {
            const int c = i * 32 + lane;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              raw[i][q] = c < nchunks ? *reinterpret_cast<const uint4*>(row + 32 * c + 8 * q) : make_uint4(0, 0, 0, 0);
              const uint32_t w4[4] = {raw[i][q].x, raw[i][q].y, raw[i][q].z, raw[i][q].w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f = bf16x2_to_f32x2(w4[j]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
              }
            }
          }
          mx = warp_max(mx);
          int ex = 0;
          if (mx > 0.f && mx <= 3.0e38f) frexpf(mx, &ex);
          const float upv = ldexpf(1.0f, 8 - ex);
          unscale[m] = ldexpf(1.0f, ex - 8);
#pragma unroll
          for (int i = 0; i < NI; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t w4[4] = {raw[i][q].x, raw[i][q].y, raw[i][q].z, raw[i][q].w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f = bf16x2_to_f32x2(w4[j]);
                __half2 h = __floats2half2_rn(f.x * upv, f.y * upv);
                xr[m][i][4 * q + j] = *reinterpret_cast<uint32_t*>(&h);
              }
            }
        }
      }
    }

    if (!mbar_wait(&full_bar[s], ph) || abort_flag) {
      set_status(status, kDevErrTimeout);
      abort_flag = 1;
      break;
    }
    const uint8_t* st = stage_ptr(s);
    const uint8_t* sc = st + NB * S * codes_row;
    for (int r = 0; r < RW; ++r) {
      const int lr = warp * RW + r;                       // row within the stage
      float acc[NB][MT];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[b][m] = 0.f;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const uint8_t* crow = st + (size_t)(b * S + lr) * codes_row;
        const uint8_t* srow = sc + (size_t)(b * S + lr) * scales_row;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          const int c = i * 32 + lane;
          if (c < nchunks) {
            const uint4 q = *reinterpret_cast<const uint4*>(crow + 16 * c);
            const uint16_t sv = *reinterpret_cast<const uint16_t*>(srow + 2 * c);
            uint32_t w[16];
            e2m1x8_to_f16x2x4(q.x, w[0], w[1], w[2], w[3]);
            e2m1x8_to_f16x2x4(q.y, w[4], w[5], w[6], w[7]);
            e2m1x8_to_f16x2x4(q.z, w[8], w[9], w[10], w[11]);
            e2m1x8_to_f16x2x4(q.w, w[12], w[13], w[14], w[15]);
            const float2 scl = e4m3x2_to_f32x2(sv);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              __half2 p0 = __float2half2_rn(0.f), p1 = __float2half2_rn(0.f);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                p0 = __hfma2(*reinterpret_cast<const __half2*>(&w[j]), *reinterpret_cast<const __half2*>(&xr[m][i][j]), p0);
#pragma unroll
              for (int j = 8; j < 16; ++j)
                p1 = __hfma2(*reinterpret_cast<const __half2*>(&w[j]), *reinterpret_cast<const __half2*>(&xr[m][i][j]), p1);
              const float2 f0 = __half22float2(p0), f1 = __half22float2(p1);
              acc[b][m] = fmaf(scl.x, f0.x + f0.y, acc[b][m]);
              acc[b][m] = fmaf(scl.y, f1.x + f1.y, acc[b][m]);
            }
          }
        }
      }
      const int row = rb * S + lr;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float tot[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) tot[b] = warp_sum(acc[b][m]);
        if (lane == 0 && m < nm) {
          const int a = p.sorted[seg0 + m];
          if (GATE_UP) {
            const float g = tot[0] * unscale[m] * p.ts0[e];
            const float uu = tot[NB - 1] * unscale[m] * p.ts1[e];
            p.out[(size_t)a * p.rows + row] = f32_to_bf16_bits(clamped_swiglu(g, uu, p.limit));
          } else {
            p.out[(size_t)a * p.rows + row] = f32_to_bf16_bits(tot[0] * unscale[m] * p.ts0[e] * p.weights[a]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }

  if (!GATE_UP) {
    // remote assignments contribute zero rows
    const int rb0 = p.offsets[p.local_begin], re0 = p.offsets[p.local_end], rend = p.offsets[p.E];
    const int nremote = rb0 + (rend - re0);
    const int rows16 = p.rows / 8;
    const int tid = threadIdx.x;   // consumers only: 256 threads
    for (long long idx = (long long)blockIdx.x * (kStreamConsumers * kWarp) + tid; idx < (long long)nremote * rows16;
         idx += (long long)gridDim.x * (kStreamConsumers * kWarp)) {
      const int rp = (int)(idx / rows16), col = (int)(idx - (long long)rp * rows16);
      const int pos = rp < rb0 ? rp : re0 + (rp - rb0);
      const int a = p.sorted[pos];
      reinterpret_cast<uint4*>(p.out + (size_t)a * p.rows)[col] = make_uint4(0, 0, 0, 0);
    }
  }
}

template <int MT, int NI, bool GU>
cudaError_t launch_stream(const GemvParams& p, int max_items, uint32_t* status, cudaStream_t st) {
  StreamShape sh;
  const int codes_row = p.K / 2, scales_row = p.K / 16;
  const int nb = GU ? 2 : 1;
  sh.S = GU ? kStreamConsumers : 4 * kStreamConsumers;
  sh.stage_bytes = (uint32_t)(nb * sh.S * (codes_row + scales_row));
  const size_t budget = 200 * 1024;
  sh.NS = (int)std::min<size_t>(16, budget / sh.stage_bytes);
  const size_t smem = (size_t)sh.NS * sh.stage_bytes;
  auto kern = nvfp4_gemv_stream_kernel<MT, NI, GU>;
  static size_t cached = 0;
  if (cached != smem) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cached = smem;
  }
  const int grid = std::max(1, std::min(max_items, kNumSMs));
  kern<<<grid, kStreamThreads, smem, st>>>(p, sh, status);
  return cudaGetLastError();
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
  kern<<<grid, kGemvThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_nvfp4_gemv(const ExpertGemvArgs& a, cudaStream_t st) {
  GemvParams p{};
  const bool gu = a.proj == MOE_PROJ_GATE_UP;
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
  const int max_active = std::min(a.local_end - a.local_begin, p.A);
  const int max_tok = a.T;   // tokens per expert never exceed T (ids in a row are distinct)
  const int NI = (p.K / 32 + 31) / 32;
  const int S = gu ? kStreamConsumers : 4 * kStreamConsumers;
  const bool stream_ok = (p.rows % S) == 0 && (size_t)(gu ? 2 : 1) * S * (p.K / 2 + p.K / 16) * 2 <= 200 * 1024;
  if (stream_ok && max_tok * NI <= 4) {
    const int items = std::max(1, max_active * (p.rows / S));
    if (gu) {
      if (max_tok == 1 && NI == 4) return launch_stream<1, 4, true>(p, items, a.status, st);
      if (max_tok == 1 && NI <= 2) return launch_stream<1, 2, true>(p, items, a.status, st);
      if (max_tok == 1) return launch_stream<1, 1, true>(p, items, a.status, st);
      if (max_tok == 2 && NI <= 2) return launch_stream<2, 2, true>(p, items, a.status, st);
    } else {
      if (NI == 1 && max_tok == 1) return launch_stream<1, 1, false>(p, items, a.status, st);
      if (NI == 1 && max_tok == 2) return launch_stream<2, 1, false>(p, items, a.status, st);
      if (NI == 1) return launch_stream<4, 1, false>(p, items, a.status, st);
      if (NI == 2 && max_tok <= 2) return launch_stream<2, 2, false>(p, items, a.status, st);
      if (NI <= 4 && max_tok == 1) return launch_stream<1, 4, false>(p, items, a.status, st);
    }
  }
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
