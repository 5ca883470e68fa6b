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

// Bounded wait (2 s) until *c >= need, acquire at gpu scope.
RNX_DEVICE bool wait_counter(const int* c, int need) {
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    if (v >= need) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(256);
  }
}

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
  const uint8_t* pf_codes;    // direct GATE_UP: down bank to prefetch into L2 (nullable)
  const uint8_t* pf_scales;
  long long pf_codes_per_expert, pf_scales_per_expert;
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

// One work item of the direct form: CTA_ROWS output rows (row block blk) of
// expert e for its single assignment a. An item runs in two phases so that a
// persistent CTA can issue the next item's weight loads before it finishes
// the current one: item_loads() issues the 128-bit weight loads (8 rows per
// warp: GATE_UP 4 gate then 4 up rows) into a register set, item_finish()
// fetches the activation chunk, multiplies, reduces and stores. With `ready`
// non-null (fused DOWN), item_finish first waits until *ready reaches `need`
// (the expert's gate/up items are all done); a wait that runs out sets the
// status word and the item is skipped.
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
RNX_DEVICE bool item_finish(const GemvParams& p, int e, int a, int blk, const ItemLoads& L, float* s_part,
                            const int* ready, int need) {
  constexpr int RG = kDirectWarps / NI;                  // row groups per CTA
  constexpr int PAIRS = GATE_UP ? kDirectRows / 2 : 0;   // gate/up pairs per row group
  __shared__ int s_ok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = warp % NI, rg = warp / NI;
  const int row0 = blk * direct_cta_rows<NI, GATE_UP>();
  const int c = kg * 32 + lane;
  const bool lane_on = c < p.K / 32;
  const float ts0 = p.ts0[e], ts1 = GATE_UP ? p.ts1[e] : 0.f;
  const float wt = GATE_UP ? 0.f : p.weights[a];

  if (ready) {
    if (threadIdx.x == 0) {
      const bool okw = wait_counter(ready, need);
      if (!okw) set_status(p.status, kDevErrTimeout);
      s_ok = okw ? 1 : 0;
    }
    __syncthreads();
    if (!s_ok) return false;
  }

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
  return true;
}

template <int NI, bool GATE_UP>
__global__ void __launch_bounds__(kDirectWarps * kWarp, 3)
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
  item_finish<NI, GATE_UP>(p, e, p.first[u], blk, L, s_part, nullptr, 0);
}

// Gate/up and down of every active expert in one persistent kernel (one
// token per expert), streaming the weights through shared memory.
//
// Work items: the gate/up blocks of each active expert (8 output features =
// 8 gate + 8 up rows each) and its down blocks (64 output rows each); one
// item is 36 KB of codes and scales at H = 4096, I = 1024. Items are numbered
// in the order
//   gu(0), gu(1), gu(2), gu(3), dn(0), gu(4), dn(1), ..., gu(n-1), dn(n-4), ..., dn(n-1)
// (the down blocks of expert u follow the gate/up blocks of expert u + 3, so
// that by the time they are taken their h is usually complete). CTA b owns
// items b, b + G, b + 2G, ... (G = grid size) and deals them alternately to
// its two pipelines.
//
// A pipeline is a producer warp, a 3-stage ring of shared memory and 8
// compute warps. Two independent rings per SM keep HBM busier than one deeper
// ring: a single producer that must wait for its oldest stage before reusing
// it leaves the memory system idle whenever that stage is the slow one.
//  * producer (one lane): copies each item's weight rows and block scales
//    with bulk copies (TMA engine) into its ring.
//  * compute warps: gate/up -- warp w owns feature w of the item (its gate and
//    its up row over the whole K) and writes h = clamped SwiGLU itself; down
//    -- warp w owns rows 8w .. 8w + 7 and writes r. A stage is released as
//    soon as its bytes have been read.
// h is the hand-off between the two projections. It is filled with an all-ones
// pattern (a NaN that the gate/up writers never produce: they store a NaN as
// the canonical one) before this kernel runs; a down warp reads its lane's
// 32-element chunk of the assignment's h row from L2 until no element holds
// the pattern. Every element is stored once, so an element read without the
// pattern is final: no fence, counter or flag is needed. The warp then takes
// the row's max |h| over its 32 lanes (the whole row when I <= 1024) for the
// f16 pre-scale.
// Every down item has a higher number than every gate/up item of its expert,
// and each pipeline takes its items in increasing order, so every awaited
// gate/up item is held by a pipeline that reaches it without waiting on the
// awaiting one. All waits are bounded; a timeout sets the status word and
// winds the CTA down.
constexpr int kRings = 2;
constexpr int kRingStages = 3;
constexpr int kDownLag = 3;                              // dn(u) follows gu(u + kDownLag)
constexpr int kStreamStageBytes = 36864;                 // codes + scales of one item
constexpr int kStreamGroupWarps = 8;                     // compute warps per pipeline
constexpr int kStreamCompute = kRings * kStreamGroupWarps;
constexpr int kStreamProducer = kStreamCompute;          // + ring
constexpr int kStreamThreads = (kStreamCompute + kRings) * 32;
constexpr int kStreamSmem = kRings * kRingStages * kStreamStageBytes;   // + x (H f16)
constexpr int kGuRowsItem = kStreamGroupWarps;           // output features per gate/up item
constexpr int kDnRowsWarp = 8;                           // down rows per compute warp
constexpr int kDnRowsItem = kDnRowsWarp * kStreamGroupWarps;   // output rows per down item
constexpr int kStreamMaxH = 4096;
constexpr int kStreamMaxI = 1024;
constexpr int kMaxStreamExperts = 16;                    // one token: at most top_k active experts
constexpr int kItemEnd = -1;
constexpr uint32_t kHUnset = 0xFFFFFFFFu;                // two bf16 elements not yet written
constexpr bool kStreamDisabled = true;

// Item number -> packed (down << 30 | u << 16 | block) in the order above.
// bpe_g / bpe_d: gate/up and down blocks per expert.
RNX_DEVICE int stream_item(int item, int n_act, int bpe_g, int bpe_d) {
  const int lead = min(kDownLag, n_act);                 // gate/up-only steps
  const int both = n_act - lead;                         // steps with gu(j + lag) then dn(j)
  if (item < lead * bpe_g) return ((item / bpe_g) << 16) | (item % bpe_g);
  item -= lead * bpe_g;
  const int step = bpe_g + bpe_d;
  if (item < both * step) {
    const int j = item / step, r = item - j * step;
    return r < bpe_g ? (((lead + j) << 16) | r) : ((1 << 30) | (j << 16) | (r - bpe_g));
  }
  item -= both * step;                                   // trailing down blocks
  const int j = both + item / bpe_d;
  return (1 << 30) | (j << 16) | (item % bpe_d);
}

// The lane's 32-element h chunk (16 bf16 pairs) read from L2; with `wait`, a
// bounded wait until no element of the warp's chunks is unset (polling with
// a growing pause, so that waiting warps do not crowd the memory pipeline of
// the SM). Lanes past the row read nothing.
RNX_DEVICE bool load_h_chunk(const uint16_t* hrow, int c, bool on, bool wait, uint32_t (&hv)[16]) {
  const uint4* p = reinterpret_cast<const uint4*>(hrow + 32 * c);
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t pause = 128;; pause = min(2u * pause, 1024u)) {
    bool ready = true;
    if (on) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "l"(p + q)
                     : "memory");
        hv[4 * q] = v.x; hv[4 * q + 1] = v.y; hv[4 * q + 2] = v.z; hv[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        // an element is unset iff its 16 bits are all ones
        ready = ready && (hv[j] & 0xFFFFu) != 0xFFFFu && (hv[j] >> 16) != 0xFFFFu;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) hv[j] = 0u;
    }
    if (!wait || __all_sync(0xffffffffu, ready)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(pause);
  }
}

// Bounded wait (2 s) until the shared int *v >= need (acquire at CTA scope).
RNX_DEVICE bool wait_shared_at_least(const int* v, int need) {
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    int x;
    asm volatile("ld.acquire.cta.shared.b32 %0, [%1];" : "=r"(x) : "r"(smem_u32(v)) : "memory");
    if (x >= need) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(32);
  }
}

__global__ void __launch_bounds__(kStreamThreads, 1)
nvfp4_experts_stream_kernel(GemvParams gu, GemvParams dn) {
  extern __shared__ __align__(128) uint8_t s_dyn[];
  uint4* s_x = reinterpret_cast<uint4*>(s_dyn + kStreamSmem);            // x as f16, [4][H/32]
  __shared__ __align__(8) uint64_t full_bar[kRings][kRingStages], empty_bar[kRings][kRingStages];
  __shared__ int s_item[kRings][kRingStages];            // packed item of each stage, kItemEnd = end
  __shared__ int s_hseen[kRings];                        // down items whose h row warp 0 found complete
  __shared__ int s_e[kMaxStreamExperts], s_a[kMaxStreamExperts], s_n;
  __shared__ float s_tg[kMaxStreamExperts], s_tu[kMaxStreamExperts], s_td[kMaxStreamExperts],
      s_wt[kMaxStreamExperts];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = gu.K, I = gu.rows;
  const int nchG = H / 32, nchD = I / 32;
  const int gu_row_bytes = H / 2, gu_sc_bytes = H / 16, dn_row_bytes = I / 2, dn_sc_bytes = I / 16;

  if (tid == 0) {
    for (int g = 0; g < kRings; ++g) s_hseen[g] = 0;
    for (int g = 0; g < kRings; ++g)
      for (int i = 0; i < kRingStages; ++i) {
        mbar_init(&full_bar[g][i], 1);
        mbar_init(&empty_bar[g][i], kStreamGroupWarps);    // the compute warps, after reading
      }
    fence_barrier_init();
  }
  pdl_wait();       // follows the routing plan
  pdl_trigger();
  // the active experts, their assignment, tensor scales and routing weight
  if (tid == 0) s_n = min(gu.active[0], kMaxStreamExperts);
  __syncthreads();
  const int n_act = s_n;
  for (int u = tid; u < n_act; u += blockDim.x) {
    const int e = gu.active[1 + u], a = gu.first[u];
    s_e[u] = e;
    s_a[u] = a;
    s_tg[u] = gu.ts0[e];
    s_tu[u] = gu.ts1[e];
    s_td[u] = dn.ts0[e];
    s_wt[u] = dn.weights[a];
  }
  __syncthreads();
  const int bpe_g = I / kGuRowsItem, bpe_d = H / kDnRowsItem;
  const int n_all = n_act * (bpe_g + bpe_d);
  const uint32_t gcb = kGuRowsItem * gu_row_bytes, gsb = kGuRowsItem * gu_sc_bytes;
  const uint32_t dcb = kDnRowsItem * dn_row_bytes, dsb = kDnRowsItem * dn_sc_bytes;
  // this CTA's items for pipeline g: blockIdx.x + (2j + g) * G, j = 0, 1, ...
  const int item_step = kRings * gridDim.x;

  if (warp >= kStreamProducer) {
    // ------------------------------------------------------------ producer
    const int g = warp - kStreamProducer;
    uint8_t* ring = s_dyn + (size_t)g * kRingStages * kStreamStageBytes;
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (int item = blockIdx.x + g * gridDim.x;; item += item_step, ++it) {
        const int s = it % kRingStages;
        const uint32_t ph = (uint32_t)(it / kRingStages) & 1u;
        const bool free_ok = mbar_wait(&empty_bar[g][s], ph ^ 1u);
        if (!free_ok) set_status(gu.status, kDevErrTimeout);
        if (!free_ok || item >= n_all) {
          s_item[g][s] = kItemEnd;         // end of work (or abort) for the compute warps
          mbar_arrive(&full_bar[g][s]);
          ++it;
          break;
        }
        const int pk = stream_item(item, n_act, bpe_g, bpe_d);
        const int u = (pk >> 16) & 0x3FFF, blk = pk & 0xFFFF;
        s_item[g][s] = pk;
        uint8_t* st = ring + (size_t)s * kStreamStageBytes;
        if (!(pk >> 30)) {
          const size_t gr = (size_t)s_e[u] * I + blk * kGuRowsItem;
          mbar_arrive_expect_tx(&full_bar[g][s], 2 * (gcb + gsb));
          bulk_g2s(st, gu.codes0 + gr * gu_row_bytes, gcb, &full_bar[g][s], pol);
          bulk_g2s(st + gcb, gu.codes1 + gr * gu_row_bytes, gcb, &full_bar[g][s], pol);
          bulk_g2s(st + 2 * gcb, gu.scales0 + gr * gu_sc_bytes, gsb, &full_bar[g][s], pol);
          bulk_g2s(st + 2 * gcb + gsb, gu.scales1 + gr * gu_sc_bytes, gsb, &full_bar[g][s], pol);
        } else {
          const size_t gr = (size_t)s_e[u] * H + blk * kDnRowsItem;
          mbar_arrive_expect_tx(&full_bar[g][s], dcb + dsb);
          bulk_g2s(st, dn.codes0 + gr * dn_row_bytes, dcb, &full_bar[g][s], pol);
          bulk_g2s(st + dcb, dn.scales0 + gr * dn_sc_bytes, dsb, &full_bar[g][s], pol);
        }
      }
      // copies in flight must land before the CTA may exit
      for (int j = max(0, it - kRingStages); j < it; ++j)
        if (!mbar_wait(&full_bar[g][j % kRingStages], (uint32_t)(j / kRingStages) & 1u))
          set_status(gu.status, kDevErrTimeout);
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  // the token's x (one token: every gate/up item uses it), pre-scaled to f16
  float x_up, x_unscale;
  prescale_from_max(__uint_as_float(gu.act_max[0]), x_up, x_unscale);
  for (int cq = tid; cq < nchG * 4; cq += kStreamCompute * 32) {
    const int c = cq >> 2, q = cq & 3;
    const uint4 v = *reinterpret_cast<const uint4*>(gu.act + 32 * c + 8 * q);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_f32x2(w4[j]);
      __half2 h2 = __floats2half2_rn(f.x * x_up, f.y * x_up);
      o[j] = *reinterpret_cast<uint32_t*>(&h2);
    }
    s_x[q * nchG + c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kStreamCompute * 32) : "memory");

  const int g = warp / kStreamGroupWarps, gw = warp % kStreamGroupWarps;
  const uint8_t* ring = s_dyn + (size_t)g * kRingStages * kStreamStageBytes;
  int ndn = 0;                              // down items taken by this pipeline
  for (int it = 0;; ++it) {
    const int s = it % kRingStages;
    const uint32_t ph = (uint32_t)(it / kRingStages) & 1u;
    if (__any_sync(0xffffffffu, !mbar_wait(&full_bar[g][s], ph))) {
      if (lane == 0) set_status(gu.status, kDevErrTimeout);
      break;
    }
    const int pk = s_item[g][s];
    if (pk == kItemEnd) break;
    const int u = (pk >> 16) & 0x3FFF, blk = pk & 0xFFFF, a = s_a[u];
    const uint8_t* st = ring + (size_t)s * kStreamStageBytes;
    if (!(pk >> 30)) {
      // gate/up: this warp's feature, gate row gw and up row gw of the item
      const int f = blk * kGuRowsItem + gw;
      const uint8_t* cg = st + gw * gu_row_bytes;
      const uint8_t* cu = st + gcb + gw * gu_row_bytes;
      const uint8_t* sg = st + 2 * gcb + gw * gu_sc_bytes;
      const uint8_t* su = sg + gsb;
      float acc[2] = {0.f, 0.f};
      for (int c = lane; c < nchG; c += 32) {
        uint32_t xr[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = s_x[q * nchG + c];
          xr[4 * q] = v.x; xr[4 * q + 1] = v.y; xr[4 * q + 2] = v.z; xr[4 * q + 3] = v.w;
        }
        uint32_t w[16];
        decode_chunk(*reinterpret_cast<const uint4*>(cg + 16 * c), w);
        chunk_fma(w, xr, e4m3x2_to_f32x2(*reinterpret_cast<const uint16_t*>(sg + 2 * c)), acc[0]);
        decode_chunk(*reinterpret_cast<const uint4*>(cu + 16 * c), w);
        chunk_fma(w, xr, e4m3x2_to_f32x2(*reinterpret_cast<const uint16_t*>(su + 2 * c)), acc[1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[g][s]);   // stage read
      const float tot = warp_reduce_rows<2>(acc);      // lanes 0-15: gate, 16-31: up
      const float upv = __shfl_sync(0xffffffffu, tot, 16);
      if (lane == 0) {
        const float gt = tot * x_unscale * s_tg[u], uu = upv * x_unscale * s_tu[u];
        uint16_t hb = f32_to_bf16_bits(clamped_swiglu(gt, uu, gu.limit));
        if ((hb & 0x7FFFu) > 0x7F80u) hb = 0x7FC0u;     // any NaN as the canonical one
        asm volatile("st.relaxed.gpu.global.b16 [%0], %1;" ::"l"(gu.out + (size_t)a * I + f), "h"(hb) : "memory");
      }
    } else {
      // down: rows 8 gw .. 8 gw + 7 of the item, lane c chunk c of h. Warp 0
      // of the pipeline waits until the row is complete; the others then read
      // it once (each element is stored once, so what warp 0 saw is final)
      const int row0 = blk * kDnRowsItem + gw * kDnRowsWarp;
      uint32_t hv[16];
      const bool lane_on = lane < nchD;
      const uint16_t* hrow = dn.act + (size_t)a * I;
      if (gw == 0) {
        if (!load_h_chunk(hrow, lane, lane_on, true, hv) && lane == 0) set_status(gu.status, kDevErrTimeout);
        __syncwarp();
        if (lane == 0) asm volatile("st.release.cta.shared.b32 [%0], %1;" ::"r"(smem_u32(&s_hseen[g])), "r"(ndn + 1) : "memory");
      } else {
        if (lane == 0 && !wait_shared_at_least(&s_hseen[g], ndn + 1)) set_status(gu.status, kDevErrTimeout);
        __syncwarp();
        load_h_chunk(hrow, lane, lane_on, false, hv);
      }
      ++ndn;
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 f = bf16x2_to_f32x2(hv[j]);
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
      mx = warp_max(mx);
      float up, unscale;
      prescale_from_max(mx, up, unscale);
      uint32_t xr[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 f = bf16x2_to_f32x2(hv[j]);
        __half2 h2 = __floats2half2_rn(f.x * up, f.y * up);
        xr[j] = *reinterpret_cast<uint32_t*>(&h2);
      }
      const uint8_t* cb = st + gw * kDnRowsWarp * dn_row_bytes;
      const uint8_t* sb = st + dcb + gw * kDnRowsWarp * dn_sc_bytes;
      float acc[kDnRowsWarp];
#pragma unroll
      for (int r = 0; r < kDnRowsWarp; ++r) acc[r] = 0.f;
      if (lane_on) {
#pragma unroll
        for (int r = 0; r < kDnRowsWarp; ++r) {
          const uint4 qv = *reinterpret_cast<const uint4*>(cb + r * dn_row_bytes + 16 * lane);
          const uint16_t sv = *reinterpret_cast<const uint16_t*>(sb + r * dn_sc_bytes + 2 * lane);
          uint32_t w[16];
          decode_chunk(qv, w);
          chunk_fma(w, xr, e4m3x2_to_f32x2(sv), acc[r]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[g][s]);   // stage read
      const float tot = warp_reduce_rows<kDnRowsWarp>(acc);   // lane 4r holds row r
      if ((lane & 3) == 0)
        dn.out[(size_t)a * H + row0 + (lane >> 2)] = f32_to_bf16_bits(tot * unscale * s_td[u] * s_wt[u]);
    }
  }
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
  if (gu && a.prefetch_down && a.down.codes) {
    p.pf_codes = a.down.codes;
    p.pf_scales = a.down.scales;
    p.pf_codes_per_expert = (long long)a.H * a.I / 2;
    p.pf_scales_per_expert = (long long)a.H * a.I / 16;
  }
  return p;
}

}  // namespace

cudaError_t launch_decode_experts(const ExpertGemvArgs& a, uint16_t* h, uint16_t* r, cudaStream_t st) {
  // one token; an item's rows (16 x H/2 + 16 x H/16 and 64 x I/2 + 64 x I/16
  // bytes) fit one 36 KB stage, and one warp's lanes cover an h row (I <= 1024)
  // measured slower than the two direct GEMV launches on B200 (the down
  // blocks wait several microseconds for h under full HBM load): not taken
  if (kStreamDisabled || a.T != 1 || !a.act_max || a.H > kStreamMaxH || a.I > kStreamMaxI || a.H % kDnRowsItem ||
      a.I % kGuRowsItem || a.I % 32)
    return cudaErrorNotSupported;
  ExpertGemvArgs g = a, d = a;
  g.proj = MOE_PROJ_GATE_UP; g.act = a.act; g.out = h; g.out_max = nullptr;
  d.proj = MOE_PROJ_DOWN; d.act = h; d.out = r; d.act_max = nullptr; d.out_max = nullptr;
  const GemvParams pg = gemv_params(g, true), pd = gemv_params(d, false);
  const int max_active = std::min(a.local_end - a.local_begin, a.T * a.k);
  const bool remote = a.local_begin > 0 || a.local_end < a.E;
  const size_t smem = (size_t)kStreamSmem + (size_t)a.H * 2;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t err = cudaFuncSetAttribute(nvfp4_experts_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)((size_t)kStreamSmem + kStreamMaxH * 2));
    if (err != cudaSuccess) return err;
    attr_done = true;
  }
  const int items = max_active * (a.I / kGuRowsItem + a.H / kDnRowsItem);
  const int grid = std::max(1, std::min((items + kRings - 1) / kRings, kNumSMs));
  cudaError_t err = launch_pdl(nvfp4_experts_stream_kernel, dim3(grid), dim3(kStreamThreads), smem, st, pg, pd);
  if (err != cudaSuccess || !remote) return err;
  zero_remote_rows<<<kNumSMs, 256, 0, st>>>(pd);
  return cudaGetLastError();
}

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
