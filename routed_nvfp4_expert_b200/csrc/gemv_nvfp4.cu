// Decode expert projections: bf16 activations x NVFP4 weights (W4A16).
//
// glm5next_mlp module docs, Constants / W4A16_GEMV_MODULE: at decode every
// routed-expert projection is M=1, and a tile GEMM measured far below the
// memory roofline there; the decode weight kernel must stream each touched
// expert's bytes once at HBM speed. Two forms:
//
//  * one token per expert (T = 1, the decode step): the "direct" form below
//    -- K split across warps, 8 weight rows in flight per warp, activations
//    pre-scaled from a row max computed upstream;
//  * several tokens per expert: a work-item loop over (active expert, block
//    of rows) whose CTA stages the expert's token rows in shared memory once
//    and applies each weight row to all of them.
//
// Both decode E2M1 pairs to f16x2 with the hardware cvt and multiply-add into
// a per-16-element f16x2 partial against the activations (pre-scaled per row
// by a power of two so that |a| < 256: products are exact in f16, an 8-term
// half-block sum stays far inside the f16 range); each block partial is
// widened to fp32 and scaled by its E4M3 block scale into an fp32 accumulator.
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
  const int32_t* first;       // [E] first assignment of each active expert
  const float* weights;       // [A] routing weights (DOWN)
  const uint8_t* codes0;      // gate (GATE_UP) or down (DOWN) [E, rows, K/2]
  const uint8_t* scales0;     // [E, rows, K/16]
  const float* ts0;           // [E]
  const uint8_t* codes1;      // up (GATE_UP only)
  const uint8_t* scales1;
  const float* ts1;
  uint16_t* out;              // GATE_UP: h [A, rows]; DOWN: r [A, rows]
  const uint32_t* act_max;    // direct form: max |activation row| (fp32 bits), by act row
  uint32_t* out_max;          // direct GATE_UP: atomicMax of |h| per assignment (nullable)
  uint32_t* status;           // device status word (bounded waits)
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
// Shared pieces of the one-token forms.

// 16 E2M1 code bytes (32 codes) -> 16 f16x2 words.
RNX_DEVICE void decode_chunk(const uint4& q, uint32_t (&w)[16]) {
  e2m1x8_to_f16x2x4(q.x, w[0], w[1], w[2], w[3]);
  e2m1x8_to_f16x2x4(q.y, w[4], w[5], w[6], w[7]);
  e2m1x8_to_f16x2x4(q.z, w[8], w[9], w[10], w[11]);
  e2m1x8_to_f16x2x4(q.w, w[12], w[13], w[14], w[15]);
}

// acc += s.x * (sum of the first 16 products) + s.y * (sum of the last 16)
RNX_DEVICE void chunk_fma(const uint32_t (&w)[16], const uint32_t (&x)[16], float2 s, float& acc) {
  // two independent 4-step chains per 16-element block (shorter dependency
  // chains; the f16 partials of a block are added before widening)
  __half2 p0 = __float2half2_rn(0.f), p1 = __float2half2_rn(0.f), p2 = p0, p3 = p0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    p0 = __hfma2(*reinterpret_cast<const __half2*>(&w[j]), *reinterpret_cast<const __half2*>(&x[j]), p0);
    p1 = __hfma2(*reinterpret_cast<const __half2*>(&w[j + 4]), *reinterpret_cast<const __half2*>(&x[j + 4]), p1);
    p2 = __hfma2(*reinterpret_cast<const __half2*>(&w[j + 8]), *reinterpret_cast<const __half2*>(&x[j + 8]), p2);
    p3 = __hfma2(*reinterpret_cast<const __half2*>(&w[j + 12]), *reinterpret_cast<const __half2*>(&x[j + 12]), p3);
  }
  const float2 f0 = __half22float2(__hadd2(p0, p1)), f1 = __half22float2(__hadd2(p2, p3));
  acc = fmaf(s.x, f0.x + f0.y, acc);
  acc = fmaf(s.y, f1.x + f1.y, acc);
}

// Power-of-two pre-scale from a row's max |a|: max lands in [128, 256).
RNX_DEVICE void prescale_from_max(float mx, float& up, float& unscale) {
  int ex = 0;
  if (mx > 0.f && mx <= 3.0e38f) frexpf(mx, &ex);
  up = ldexpf(1.0f, 8 - ex);
  unscale = ldexpf(1.0f, ex - 8);
}

// This lane's 32-element chunk c of an activation row, pre-scaled, as f16x2.
RNX_DEVICE void load_act_chunk(const uint16_t* row, int c, bool on, float up, uint32_t (&xr)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = on ? *reinterpret_cast<const uint4*>(row + 32 * c + 8 * q) : make_uint4(0, 0, 0, 0);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_f32x2(w4[j]);
      __half2 h = __floats2half2_rn(f.x * up, f.y * up);
      xr[4 * q + j] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

// Sum N per-lane values over the warp (N a power of two <= 32): afterwards
// lane l holds the total of value l / (32 / N); lanes that are multiples of
// 32 / N hold values 0, 1, ..., N-1. log2(N) exchange steps at distances
// 16, 8, ... each halve the values a lane holds; plain butterflies finish.
template <int N>
RNX_DEVICE float warp_reduce_rows(float (&v)[N]) {
  const int lane = threadIdx.x & 31;
  int cnt = N;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) {
    if (cnt > 1) {
      const int h = cnt >> 1;
      const bool hi = lane & d;
#pragma unroll
      for (int i = 0; i < (N > 1 ? N / 2 : 1); ++i) {
        if (i < h) {
          const float send = hi ? v[i] : v[i + h];
          const float keep = hi ? v[i + h] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, d);
        }
      }
      cnt = h;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], d);
    }
  }
  return v[0];
}

// ---------------------------------------------------------------------------
// Direct form for one token per expert (T = 1 decode). One CTA owns a block
// of consecutive rows of one expert. K is split across warps: warp w works on
// chunk group kg = w % NI (lanes own chunks c = 32 kg + lane), so it needs only
// 16 registers of activations, and keeps 8 weight rows in flight: all of its
// 128-bit weight loads are issued first, then its activation chunk is fetched
// and pre-scaled from the row's max |a| (computed upstream: by the router for
// x, by the gate/up pass for h). Row sums are reduced across each warp
// together (9 shuffles for 8 rows); the NI partial sums of a row are combined
// in shared memory in fixed order (deterministic). GATE_UP publishes the max
// |h| of its assignment (atomicMax on the bit patterns of non-negative floats,
// exact and order-independent) for the DOWN pass.
constexpr int kDirectWarps = 8;
constexpr int kDirectRows = 8;        // weight rows per warp
// 64 registers a thread (no spills): 4 CTAs (32 warps) per SM keep more weight
// loads in flight, and the down pass (512 CTAs for 8 experts at H = 4096)
// fits one wave of 4 x 148 CTAs instead of leaving a second, almost empty one
constexpr int kDirectCtasPerSm = 4;

// One work item of the direct form: CTA_ROWS output rows (row block blk) of
// expert e for its single assignment a, in two phases: item_loads() issues
// the 128-bit weight loads (8 rows per warp: GATE_UP 4 gate then 4 up rows)
// into a register set, item_finish() fetches the activation chunk,
// multiplies, reduces and stores.
struct ItemLoads {
  uint4 q[kDirectRows];
  uint16_t sv[kDirectRows];
};

template <int NI, bool GATE_UP>
__host__ __device__ constexpr int direct_cta_rows() {
  return GATE_UP ? (kDirectWarps / NI) * (kDirectRows / 2) : (kDirectWarps / NI) * kDirectRows;
}

template <int NI, bool GATE_UP>
RNX_DEVICE void item_loads(const GemvParams& p, int e, int blk, ItemLoads& L) {
  constexpr int RG = kDirectWarps / NI;
  constexpr int PAIRS = GATE_UP ? kDirectRows / 2 : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = warp % NI, rg = warp / NI;
  const int c = kg * 32 + lane;
  const bool lane_on = c < p.K / 32;
  const int row0 = blk * direct_cta_rows<NI, GATE_UP>();
#pragma unroll
  for (int r = 0; r < kDirectRows; ++r) {
    int row;
    const uint8_t *cb, *sb;
    if (GATE_UP) {
      row = row0 + rg * PAIRS + (r % PAIRS);
      cb = r < PAIRS ? p.codes0 : p.codes1;
      sb = r < PAIRS ? p.scales0 : p.scales1;
    } else {
      row = row0 + rg * kDirectRows + r;
      cb = p.codes0;
      sb = p.scales0;
    }
    const bool on = lane_on && row < p.rows;
    const size_t gr = (size_t)e * p.rows + row;
    L.q[r] = on ? ldg_stream(cb + gr * (p.K / 2) + 16 * c) : make_uint4(0, 0, 0, 0);
    L.sv[r] = on ? ldg_u16(sb + gr * (p.K / 16) + 2 * c) : (uint16_t)0;
  }
}

template <int NI, bool GATE_UP>
RNX_DEVICE void item_finish(const GemvParams& p, int e, int a, int blk, const ItemLoads& L, float* s_part) {
  constexpr int RG = kDirectWarps / NI;                  // row groups per CTA
  constexpr int PAIRS = GATE_UP ? kDirectRows / 2 : 0;   // gate/up pairs per row group
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = warp % NI, rg = warp / NI;
  const int row0 = blk * direct_cta_rows<NI, GATE_UP>();
  const int c = kg * 32 + lane;
  const bool lane_on = c < p.K / 32;
  const float ts0 = p.ts0[e], ts1 = GATE_UP ? p.ts1[e] : 0.f;
  const float wt = GATE_UP ? 0.f : p.weights[a];

  // this lane's 32-element activation chunk (x token for GATE_UP, h row for
  // DOWN) pre-scaled by the power of two that brings the row's max |a|
  // (supplied) into [128, 256)
  const uint16_t* arow = p.act + (size_t)(GATE_UP ? a / p.k : a) * p.K;
  float up, unscale;
  prescale_from_max(__uint_as_float(p.act_max[GATE_UP ? a / p.k : a]), up, unscale);
  uint32_t xr[16];
  load_act_chunk(arow, c, lane_on, up, xr);

  float acc[kDirectRows];
#pragma unroll
  for (int r = 0; r < kDirectRows; ++r) {
    acc[r] = 0.f;
    uint32_t w[16];
    decode_chunk(L.q[r], w);
    chunk_fma(w, xr, e4m3x2_to_f32x2(L.sv[r]), acc[r]);
  }
  const float tot = warp_reduce_rows<kDirectRows>(acc);   // lane 4r holds row slot r
  const int r = lane >> 2;

  if (GATE_UP) {
    if ((lane & 3) == 0) s_part[kg * RG * kDirectRows + rg * kDirectRows + r] = tot;
    __syncthreads();
    if (threadIdx.x < RG * PAIRS) {
      const int gq = threadIdx.x / PAIRS, pr = threadIdx.x % PAIRS;
      const int row = row0 + gq * PAIRS + pr;
      if (row < p.rows) {
        float g = 0.f, uu = 0.f;
#pragma unroll
        for (int k = 0; k < NI; ++k) {
          g += s_part[k * RG * kDirectRows + gq * kDirectRows + pr];
          uu += s_part[k * RG * kDirectRows + gq * kDirectRows + PAIRS + pr];
        }
        g *= unscale * ts0;
        uu *= unscale * ts1;
        const uint16_t hb = f32_to_bf16_bits(clamped_swiglu(g, uu, p.limit));
        p.out[(size_t)a * p.rows + row] = hb;
        if (p.out_max) atomicMax(p.out_max + a, __float_as_uint(fabsf(bf16_bits_to_f32(hb))));
      }
    }
  } else if (NI == 1) {
    const int row = row0 + rg * kDirectRows + r;
    if ((lane & 3) == 0 && row < p.rows)
      p.out[(size_t)a * p.rows + row] = f32_to_bf16_bits(tot * unscale * ts0 * wt);
  } else {
    if ((lane & 3) == 0) s_part[kg * RG * kDirectRows + rg * kDirectRows + r] = tot;
    __syncthreads();
    if (threadIdx.x < RG * kDirectRows) {
      const int row = row0 + threadIdx.x;
      if (row < p.rows) {
        float o = 0.f;
#pragma unroll
        for (int k = 0; k < NI; ++k) o += s_part[k * RG * kDirectRows + threadIdx.x];
        p.out[(size_t)a * p.rows + row] = f32_to_bf16_bits(o * unscale * ts0 * wt);
      }
    }
  }
}

template <int NI, bool GATE_UP>
__global__ void __launch_bounds__(kDirectWarps * kWarp, kDirectCtasPerSm)
nvfp4_gemv_direct_kernel(GemvParams p) {
  __shared__ float s_part[kDirectWarps * kDirectRows];
  const int bpe = (p.rows + direct_cta_rows<NI, GATE_UP>() - 1) / direct_cta_rows<NI, GATE_UP>();
  const int u = blockIdx.x / bpe, blk = blockIdx.x - u * bpe;
  pdl_wait();       // follows the routing plan (GATE_UP) or the h producer (DOWN)
  pdl_trigger();
  if (u >= p.active[0]) return;
  const int e = p.active[1 + u];
  ItemLoads L;
  item_loads<NI, GATE_UP>(p, e, blk, L);
  item_finish<NI, GATE_UP>(p, e, p.first[u], blk, L, s_part);
}

// remote assignments of the DOWN projection contribute zero rows
__global__ void __launch_bounds__(256) zero_remote_rows(GemvParams p) {
  const int rb0 = p.offsets[p.local_begin], re0 = p.offsets[p.local_end], rend = p.offsets[p.E];
  const int nremote = rb0 + (rend - re0);
  const int rows16 = p.rows / 8;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long long)nremote * rows16;
       idx += (long long)gridDim.x * blockDim.x) {
    const int rp = (int)(idx / rows16), col = (int)(idx - (long long)rp * rows16);
    const int pos = rp < rb0 ? rp : re0 + (rp - rb0);
    const int as = p.sorted[pos];
    reinterpret_cast<uint4*>(p.out + (size_t)as * p.rows)[col] = make_uint4(0, 0, 0, 0);
  }
}

template <int NI, bool GU>
cudaError_t launch_direct(const GemvParams& p, int max_active, bool has_remote, cudaStream_t st) {
  constexpr int RG = kDirectWarps / NI;
  constexpr int CTA_ROWS = GU ? RG * (kDirectRows / 2) : RG * kDirectRows;
  const int bpe = (p.rows + CTA_ROWS - 1) / CTA_ROWS;
  const int grid = std::max(1, max_active * bpe);
  cudaError_t err = launch_pdl(nvfp4_gemv_direct_kernel<NI, GU>, dim3(grid), dim3(kDirectWarps * kWarp), 0, st, p);
  if (err != cudaSuccess || GU || !has_remote) return err;
  zero_remote_rows<<<kNumSMs, 256, 0, st>>>(p);
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
  p.first = a.first;
  p.weights = a.weights;
  if (gu) {
    p.codes0 = a.gate.codes; p.scales0 = a.gate.scales; p.ts0 = a.gate.tensor_scale;
    p.codes1 = a.up.codes;   p.scales1 = a.up.scales;   p.ts1 = a.up.tensor_scale;
  } else {
    p.codes0 = a.down.codes; p.scales0 = a.down.scales; p.ts0 = a.down.tensor_scale;
    p.codes1 = nullptr;      p.scales1 = nullptr;       p.ts1 = nullptr;
  }
  p.out = a.out;
  p.act_max = a.act_max;
  p.out_max = a.out_max;
  p.status = a.status;
  return p;
}

}  // namespace


cudaError_t launch_nvfp4_gemv(const ExpertGemvArgs& a, cudaStream_t st) {
  const bool gu = a.proj == MOE_PROJ_GATE_UP;
  const GemvParams p = gemv_params(a, gu);
  const int max_active = std::min(a.local_end - a.local_begin, p.A);
  const int max_tok = a.T;   // tokens per expert never exceed T (ids in a row are distinct)
  const int NI = (p.K / 32 + 31) / 32;
  if (max_tok == 1 && a.act_max && p.K <= 8192) {
    const bool remote = a.local_begin > 0 || a.local_end < a.E;
    if (NI == 1) return gu ? launch_direct<1, true>(p, max_active, remote, st) : launch_direct<1, false>(p, max_active, remote, st);
    if (NI == 2) return gu ? launch_direct<2, true>(p, max_active, remote, st) : launch_direct<2, false>(p, max_active, remote, st);
    if (NI <= 4) return gu ? launch_direct<4, true>(p, max_active, remote, st) : launch_direct<4, false>(p, max_active, remote, st);
    return gu ? launch_direct<8, true>(p, max_active, remote, st) : launch_direct<8, false>(p, max_active, remote, st);
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
