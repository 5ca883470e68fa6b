// Single-token decode of the routed experts on the tensor cores
// (glm5next_mlp module docs, Constants / W4A16_GEMV_MODULE: at decode every
// routed-expert projection is M = 1, so the step is a stream over the touched
// experts' bytes). Two launches chained by programmatic dependent launch:
//
//   gate/up  every pair of rows of the live experts' NVFP4 gate and up
//            matrices against x, then the clamped SwiGLU: h fp32 [k, I];
//   down     every 16-row tile of the live experts' NVFP4 down matrices
//            against h, times the routing weight: r fp32 [k, H] (rows of
//            assignments that are not live are zero). moe_combine then sums
//            r and the shared row.
//
// One CTA of 16 warps per SM. Each warp streams its weight rows straight into
// registers with coalesced 128-bit loads (a warp reads 512 contiguous bytes of
// a row per load; about 8 KB per warp in flight), no shared-memory staging of
// weights, and multiplies them on the tensor cores with mma.sync m16n8k16
// (f16 operands, fp32 accumulators). Gate/up also asks L2 for the down
// kernel's tiles; the down kernel loads its first tile before it waits for h.
//
// Arithmetic. Weights are the A operand: each E2M1 code is decoded to f16 by
// the hardware cvt and multiplied (f16) by its block's E4M3 scale; the product
// has at most 6 significant bits and lies in [2^-10, 2688], so it is exact in
// f16. The activation (x, or h) times a per-row power of two (max |a| in
// [2^14, 2^15)) in f16 is the B operand. Every product is exact in the tensor
// core's fp32 accumulation, so only the fp32 sums round; the power of two and
// the tensor scale are applied to the fp32 totals.
//
// Layout. A dot product does not depend on the order of its terms; the
// kernels only choose which weights meet which activations in one mma. Both
// work on pairs of weight rows: an mma's 16 A rows are (row 0 of the pair,
// octant g) and (row 1, octant g) for g = 0..7, where octant g of a row is
// its 128-code chunks g, g + 8, g + 16, ...; B column n holds the activation's
// octant n. The diagonal D[g][g] (and D[g + 8][g]) is then octant g's partial
// dot product of each row, and the sum over the eight octants finishes it.
// Lane (g, t) holds, per step, the 16 bytes of chunk 8 c + g at 16 t of each
// row, so a warp load covers 512 contiguous bytes; its 16 k-slots per mma
// hold four consecutive codes of those 32, and B holds the activation at the
// same positions.

#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kMaxLive = 16;               // top-k <= 16
constexpr int kWarps = 16;                 // warps per CTA, one CTA per SM
constexpr int kThreads = kWarps * kWarp;

RNX_DEVICE uint32_t e4m3x2_to_f16x2(uint16_t s) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
  return h;
}
RNX_DEVICE uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
RNX_DEVICE uint32_t lo_lo(uint32_t v) { return __byte_perm(v, 0u, 0x1010); }
RNX_DEVICE uint32_t hi_hi(uint32_t v) { return __byte_perm(v, 0u, 0x3232); }

RNX_DEVICE void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                          uint32_t b1);

// Two E2M1 bytes of w (bytes 0, 1, or 2, 3 when HI) -> two f16x2 words.
template <bool HI>
RNX_DEVICE void e2m1_pair(uint32_t w, uint32_t& a, uint32_t& b) {
  if (HI)
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b2;\n\tcvt.rn.f16x2.e2m1x2 %1, b3;\n\t}"
        : "=r"(a), "=r"(b)
        : "r"(w));
  else
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t}"
        : "=r"(a), "=r"(b)
        : "r"(w));
}
RNX_DEVICE uint32_t word_of(const uint4& q, int i) { return i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w; }

// One mma step ii (0..7) of a 16-code chunk pair: A rows from the lane's 16
// bytes of its two rows (bytes 2 ii, 2 ii + 1, each code times its block
// scale z), B = b.
template <int II>
RNX_DEVICE void mma_step(float (&acc)[4], const uint4& q0, const uint4& q1, uint32_t z0, uint32_t z1, uint2 b) {
  uint32_t a0, a2, a1, a3;
  e2m1_pair<(II & 1) != 0>(word_of(q0, II >> 1), a0, a2);
  e2m1_pair<(II & 1) != 0>(word_of(q1, II >> 1), a1, a3);
  mma_16816(acc, hmul2(a0, z0), hmul2(a1, z1), hmul2(a2, z0), hmul2(a3, z1), b.x, b.y);
}

RNX_DEVICE void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The token's live experts from the routing plan (active list, expert order;
// first[u] = the assignment), kept only when the id and assignment are in
// range: s_live[0] = count, s_live[1 + u] = expert, s_live[1 + kMaxLive + u] =
// assignment, s_ts[u] / s_ts[kMaxLive + u] = the two tensor scales asked for
// (bank0, bank1; bank1 may be null). All threads call it (two barriers).
RNX_DEVICE void load_live(const DecodeT1Args& p, const float* ts0, const float* ts1, int* s_tmp, int* s_live,
                          float* s_ts) {
  const int u = threadIdx.x;
  if (u < kMaxLive) {
    // one round for the count, the ids and the assignments (entries past the
    // count are read but not used; the arrays hold at least E entries), one
    // for the tensor scales
    const int n = min(p.active[0], kMaxLive);
    int e = -1, a = -1;
    if (u < p.E) {
      e = p.active[1 + u];
      a = p.first[u];
    }
    const bool ok = u < n && e >= 0 && e < p.E && e >= p.lb && e < p.le && a >= 0 && a < p.k;
    if (u < n && !ok && blockIdx.x == 0) set_status(p.status, kDevErrBounds);
    float t0 = 0.f, t1 = 0.f;
    if (ok) {
      t0 = ts0[e];
      if (ts1) t1 = ts1[e];
    }
    s_tmp[u] = ok ? e : -1;
    s_tmp[kMaxLive + u] = a;
    reinterpret_cast<float*>(s_tmp)[2 * kMaxLive + u] = t0;
    reinterpret_cast<float*>(s_tmp)[3 * kMaxLive + u] = t1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int v = 0; v < kMaxLive; ++v) {
      if (s_tmp[v] < 0) continue;
      s_live[1 + n] = s_tmp[v];
      s_live[1 + kMaxLive + n] = s_tmp[kMaxLive + v];
      s_ts[n] = reinterpret_cast<float*>(s_tmp)[2 * kMaxLive + v];
      s_ts[kMaxLive + n] = reinterpret_cast<float*>(s_tmp)[3 * kMaxLive + v];
      ++n;
    }
    s_live[0] = n;
  }
  __syncthreads();
}

// Row-pair loads and products (both kernels). Rows r and r + 1 of a bank
// with K codes per row; octant g of a row = its 128-code chunks g, g + 8,
// g + 16, ...; step c covers chunks 8 c .. 8 c + 7, so lane (g, t) reads the
// 16 bytes at 64 (8 c + g) + 16 t and a warp reads 512 contiguous bytes of a
// row per step (its scales: 64 contiguous bytes). Chunks past K / 128 read
// as zero.
RNX_DEVICE void pair_load(const nvfp4_bank_t& bk, size_t r, int K, int c, int g, int t, uint4 (&q)[2], uint32_t& sc) {
  const bool on = 8 * c + g < K / 128;
  const uint8_t* cp = bk.codes + r * (K / 2) + 64 * (8 * c + g) + 16 * t;
  q[0] = on ? ldg_stream(cp) : make_uint4(0u, 0u, 0u, 0u);
  q[1] = on ? ldg_stream(cp + K / 2) : make_uint4(0u, 0u, 0u, 0u);
  const uint8_t* sp = bk.scales + r * (K / 16) + 8 * (8 * c + g) + 2 * t;
  sc = on ? (uint32_t)ldg_u16(sp) | ((uint32_t)ldg_u16(sp + K / 16) << 16) : 0u;
}

// The 8 mma of one step: A rows g = (row 0, octant g), g + 8 = (row 1,
// octant g); bj = the step's B fragments at this lane (entry 32 i).
RNX_DEVICE void pair_mma(const uint4 (&q)[2], uint32_t sc, const uint2* bj, float (&acc)[2][4]) {
  const uint32_t s0 = e4m3x2_to_f16x2((uint16_t)(sc & 0xFFFFu)), s1 = e4m3x2_to_f16x2((uint16_t)(sc >> 16));
  const uint32_t s0a = lo_lo(s0), s0b = hi_hi(s0), s1a = lo_lo(s1), s1b = hi_hi(s1);
#define RNX_PAIR_STEP(II) \
  mma_step<II>(acc[(II) & 1], q[0], q[1], (II) < 4 ? s0a : s0b, (II) < 4 ? s1a : s1b, bj[(II) * 32]);
  RNX_PAIR_STEP(0) RNX_PAIR_STEP(1) RNX_PAIR_STEP(2) RNX_PAIR_STEP(3)
  RNX_PAIR_STEP(4) RNX_PAIR_STEP(5) RNX_PAIR_STEP(6) RNX_PAIR_STEP(7)
#undef RNX_PAIR_STEP
}

// The same with one accumulation chain.
RNX_DEVICE void pair_mma1(const uint4 (&q)[2], uint32_t sc, const uint2* bj, float (&acc)[4]) {
  const uint32_t s0 = e4m3x2_to_f16x2((uint16_t)(sc & 0xFFFFu)), s1 = e4m3x2_to_f16x2((uint16_t)(sc >> 16));
  const uint32_t s0a = lo_lo(s0), s0b = hi_hi(s0), s1a = lo_lo(s1), s1b = hi_hi(s1);
#define RNX_PAIR_STEP(II) mma_step<II>(acc, q[0], q[1], (II) < 4 ? s0a : s0b, (II) < 4 ? s1a : s1b, bj[(II) * 32]);
  RNX_PAIR_STEP(0) RNX_PAIR_STEP(1) RNX_PAIR_STEP(2) RNX_PAIR_STEP(3)
  RNX_PAIR_STEP(4) RNX_PAIR_STEP(5) RNX_PAIR_STEP(6) RNX_PAIR_STEP(7)
#undef RNX_PAIR_STEP
}
RNX_DEVICE void pair_diag1(const float (&acc)[4], int g, int t, float* red) {
  if (t == (g >> 1)) {
    red[g] = (g & 1) ? acc[1] : acc[0];
    red[8 + g] = (g & 1) ? acc[3] : acc[2];
  }
}

// The diagonal of a pair's accumulator: octant g of row 0 is D[g][g], of row
// 1 D[g + 8][g], in lane (g, g / 2), element g % 2. Writes them to red[0..8)
// (row 0) and red[8..16) (row 1), indexed by octant.
RNX_DEVICE void pair_diag(const float (&acc)[2][4], int g, int t, float* red) {
  if (t == (g >> 1)) {
    red[g] = (g & 1) ? acc[0][1] + acc[1][1] : acc[0][0] + acc[1][0];
    red[8 + g] = (g & 1) ? acc[0][3] + acc[1][3] : acc[0][2] + acc[1][2];
  }
}
RNX_DEVICE float octant_sum(const float* v) {
  return ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
}

// B fragments of a K-element activation row a (scaled by up, rounded to f16)
// in the order of pair_mma: entry (c * 8 + i) * 32 + lane =
// a[128 (8 c + n) + 32 t + 4 i + 0..3] with n = lane / 4, t = lane % 4 (zeros
// past K).
RNX_DEVICE uint2 b_frag_f16(float4 v, float up) {
  __half2 h0 = __floats2half2_rn(v.x * up, v.y * up), h1 = __floats2half2_rn(v.z * up, v.w * up);
  return make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
}
RNX_DEVICE int b_frag_pos(int f) {    // element index of entry f (4 consecutive elements)
  const int ln = f & 31, i = (f >> 5) & 7, c = f >> 8;
  return 128 * (8 * c + (ln >> 2)) + 32 * (ln & 3) + 4 * i;
}

// ============================================================== gate/up
//
// Item = a pair of rows (2 rp, 2 rp + 1) of one live expert's gate and up
// matrices, full K; one warp per item at a time. NCH = H / 1024 steps, taken
// 4 at a time into registers.

__global__ void __launch_bounds__(kThreads, 1) t1_gate_up_kernel(const DecodeT1Args p) {
  __shared__ __align__(16) uint2 xs[8192 / 4];      // x as B fragments, H <= 8192
  __shared__ float s_red[kWarps][2][16];
  __shared__ int s_live[1 + 2 * kMaxLive];
  __shared__ int s_tmp[4 * kMaxLive];
  __shared__ float s_ts[2 * kMaxLive];
  const int H = p.H, I = p.I, NCH = H / 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  pdl_wait();              // the plan and max |x| come from earlier launches
  pdl_trigger();
  load_live(p, p.gate.tensor_scale, p.up.tensor_scale, s_tmp, s_live, s_ts);
  const int n_live = s_live[0];
  const int N = n_live * (I / 2), GW = gridDim.x * kWarps;
  const int first = blockIdx.x * kWarps + warp;
  auto rows = [&](int i, int& u) {
    u = i / (I / 2);
    return (size_t)s_live[1 + u] * I + 2 * (size_t)(i - u * (I / 2));
  };
  if (first < N) {            // the first item into L2 while x is staged
    int u;
    const size_t r0 = rows(first, u);
    for (int o = lane * 128; o < H; o += 32 * 128) {
      prefetch_l2(p.gate.codes + r0 * (H / 2) + o);
      prefetch_l2(p.up.codes + r0 * (H / 2) + o);
    }
    if (lane * 128 < H / 8) {
      prefetch_l2(p.gate.scales + r0 * (H / 16) + lane * 128);
      prefetch_l2(p.up.scales + r0 * (H / 16) + lane * 128);
    }
  }
  float up, unscale;
  prescale15(__uint_as_float(*p.xmax), up, unscale);
  for (int f = threadIdx.x; f < H / 4; f += kThreads) {
    const uint2 v = *reinterpret_cast<const uint2*>(p.x + b_frag_pos(f));
    const float2 a = bf16x2_to_f32x2(v.x), b = bf16x2_to_f32x2(v.y);
    xs[f] = b_frag_f16(make_float4(a.x, a.y, b.x, b.y), up);
  }
  __syncthreads();

  uint4 qg[4][2], qu[4][2];  // [step][row] of the gate and up rows
  uint32_t sg[4], su[4];
  auto load4 = [&](size_t r0, int c0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (c0 + j < NCH) {
        pair_load(p.gate, r0, H, c0 + j, g, t, qg[j], sg[j]);
        pair_load(p.up, r0, H, c0 + j, g, t, qu[j], su[j]);
      }
    }
  };
  if (first < N) {
    int u;
    load4(rows(first, u), 0);
  }
  // Ask L2 for this warp's later items and for a share of the down kernel's
  // tiles (all of the step's expert bytes fit in L2), after the first item's
  // own loads went out.
  for (int i = first + GW; i < N; i += GW) {
    int u;
    const size_t r0 = rows(i, u);
    for (int o = lane * 128; o < H; o += 32 * 128) {          // 2 rows x H/2 code bytes per matrix
      prefetch_l2(p.gate.codes + r0 * (H / 2) + o);
      prefetch_l2(p.up.codes + r0 * (H / 2) + o);
    }
    if (lane * 128 < H / 8) {                                  // 2 rows x H/16 scale bytes
      prefetch_l2(p.gate.scales + r0 * (H / 16) + lane * 128);
      prefetch_l2(p.up.scales + r0 * (H / 16) + lane * 128);
    }
  }
  if (p.l2_down) {
    const int TPE = p.H / 16, ND = n_live * TPE;
    for (int i = first; i < ND; i += GW) {                     // 16-row down tiles: I/2 + I/16 bytes a row
      const int u = i / TPE;
      const size_t row0 = (size_t)s_live[1 + u] * H + 16 * (size_t)(i - u * TPE);
      for (int o = lane * 128; o < 8 * I; o += 32 * 128) prefetch_l2(p.down.codes + row0 * (I / 2) + o);
      if (lane * 128 < I) prefetch_l2(p.down.scales + row0 * (I / 16) + lane * 128);
    }
  }

  for (int i = first; i < N; i += GW) {
    int u;
    const size_t r0 = rows(i, u);
    float ag[2][4], au[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) ag[j][q] = au[j][q] = 0.f;
    for (int c0 = 0; c0 < NCH; c0 += 4) {
      if (c0 > 0) load4(r0, c0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (c0 + j < NCH) {
          const uint2* bj = xs + (c0 + j) * 256 + lane;
          pair_mma(qg[j], sg[j], bj, ag);
          pair_mma(qu[j], su[j], bj, au);
        }
      }
    }
    if (i + GW < N) {
      int u2;
      load4(rows(i + GW, u2), 0);        // the next item's first steps (L2) while this one finishes
    }
    float* red = &s_red[warp][0][0];
    pair_diag(ag, g, t, red);
    pair_diag(au, g, t, red + 16);
    __syncwarp();
    if (lane < 2) {
      const float gs = octant_sum(red + 8 * lane) * unscale * s_ts[u];
      const float us = octant_sum(red + 16 + 8 * lane) * unscale * s_ts[kMaxLive + u];
      const size_t a = (size_t)s_live[1 + kMaxLive + u];
      p.h[a * I + (r0 - (size_t)s_live[1 + u] * I) + lane] = clamped_swiglu(gs, us, p.limit);
    }
    __syncwarp();
  }

  // h rows of assignments that are not live (remote experts, dropped ids)
  // are zero: this CTA's slice of each
  const int n0 = (int)((long long)blockIdx.x * I / gridDim.x), n1 = (int)((long long)(blockIdx.x + 1) * I / gridDim.x);
  for (int a = 0; a < p.k; ++a) {
    bool live = false;
    for (int uu = 0; uu < n_live; ++uu) live |= s_live[1 + kMaxLive + uu] == a;
    if (!live)
      for (int x = n0 + (int)threadIdx.x; x < n1; x += kThreads) p.h[(size_t)a * I + x] = 0.f;
  }
}

// ============================================================== down
//
// Item = a 16-row tile (8 row pairs) of one live expert's down matrix, full
// K = I in NCD = ceil(I / 1024) steps, one step of all 8 pairs in
// registers at a time; one warp per item at a time.

constexpr int kHq = 4;           // B-fragment entries of h per thread held in registers while staging

// ONE_STEP: I <= 1024, every pair's K in one step (its diagonal taken right
// after its 8 mma); else I = 2048, two steps, the tile in two halves of four
// pairs.
template <bool ONE_STEP>
__global__ void __launch_bounds__(kThreads, 1) t1_down_kernel(const DecodeT1Args p) {
  extern __shared__ __align__(16) uint2 hs[];               // h as B fragments: k x NCD x 256
  __shared__ float s_red[kWarps][8][16];
  __shared__ float s_up[kMaxLive], s_sc[kMaxLive];
  __shared__ uint32_t s_max[kMaxLive];
  __shared__ int s_live[1 + 2 * kMaxLive];
  __shared__ int s_tmp[4 * kMaxLive];
  __shared__ float s_ts[2 * kMaxLive];
  const int H = p.H, I = p.I, k = p.k, NCD = (I + 1023) / 1024, FPE = NCD * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  // The plan comes from two launches back, complete when this grid starts.
  // The weights were requested into L2 by the gate/up launch: h is staged
  // first (its loads would otherwise queue behind the weight loads).
  load_live(p, p.down.tensor_scale, nullptr, s_tmp, s_live, s_ts);
  const int n_live = s_live[0];
  const int TPE = H / 16, N = n_live * TPE, GW = gridDim.x * kWarps;
  int i = blockIdx.x * kWarps + warp;
  uint4 q[8][2];
  uint32_t sc[8];
  auto row_of = [&](int it, int& u) {
    u = it / TPE;
    return (size_t)s_live[1 + u] * H + 16 * (size_t)(it - u * TPE);
  };
  if (threadIdx.x < kMaxLive) s_max[threadIdx.x] = 0u;
  pdl_wait();                // h comes from the previous launch
  pdl_trigger();

  // h rows of the live experts as B fragments (b_frag_pos order) times the
  // row's power of two: the row maxima first (one shared atomic per warp: a
  // warp's 32 consecutive entries lie in one row), then the conversion.
  {
    const int nq = n_live * FPE;
    const bool in_regs = nq <= kHq * kThreads;
    float4 v[kHq];
    auto load_h = [&](int f) {
      const int u = f / FPE, pos = b_frag_pos(f - u * FPE);
      if (pos >= I) return make_float4(0.f, 0.f, 0.f, 0.f);
      return *reinterpret_cast<const float4*>(p.h + (size_t)s_live[1 + kMaxLive + u] * I + pos);
    };
    auto amax4 = [](float4 a) { return fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))); };
    __syncthreads();
    if (in_regs) {
#pragma unroll
      for (int qq = 0; qq < kHq; ++qq) {
        const int f = threadIdx.x + qq * kThreads;
        v[qq] = f < nq ? load_h(f) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    for (int qn = 0; qn * kThreads < nq; ++qn) {
      const int f = threadIdx.x + qn * kThreads;            // warp-uniform: f < nq for all lanes or none
      if (f - lane < nq) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (in_regs) {
#pragma unroll
          for (int qq = 0; qq < kHq; ++qq)
            if (qq == qn) a = v[qq];
        } else {
          a = load_h(f);
        }
        const float m = warp_max(amax4(a));
        if (lane == 0) atomicMax(&s_max[f / FPE], __float_as_uint(m));   // non-negative floats order as integers
      }
    }
    __syncthreads();
    if (threadIdx.x < n_live) {
      float upx, us;
      prescale15(__uint_as_float(s_max[threadIdx.x]), upx, us);
      s_up[threadIdx.x] = upx;
      s_sc[threadIdx.x] = us * s_ts[threadIdx.x] * p.weights[s_live[1 + kMaxLive + threadIdx.x]];
    }
    __syncthreads();
    for (int qn = 0; qn * kThreads < nq; ++qn) {
      const int f = threadIdx.x + qn * kThreads;
      if (f < nq) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (in_regs) {
#pragma unroll
          for (int qq = 0; qq < kHq; ++qq)
            if (qq == qn) a = v[qq];
        } else {
          a = load_h(f);
        }
        hs[f] = b_frag_f16(a, s_up[f / FPE]);
      }
    }
    __syncthreads();
  }

  if (i < N) {
    int u;
    const size_t r0 = row_of(i, u);
#pragma unroll
    for (int pr = 0; pr < (ONE_STEP ? 8 : 4); ++pr) pair_load(p.down, r0 + 2 * pr, I, 0, g, t, q[pr], sc[pr]);
  }
  for (; i < N; i += GW) {
    int u;
    const size_t row0 = row_of(i, u);
    const uint2* bf = hs + (size_t)u * FPE + lane;
    float* red = &s_red[warp][0][0];
    if (ONE_STEP) {
#pragma unroll
      for (int pr = 0; pr < 8; ++pr) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        pair_mma1(q[pr], sc[pr], bf, acc);
        pair_diag1(acc, g, t, red + 16 * pr);
      }
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float acc[4][4];
#pragma unroll
        for (int pr = 0; pr < 4; ++pr)
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) acc[pr][qq] = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (half > 0 || c > 0) {
#pragma unroll
            for (int pr = 0; pr < 4; ++pr) pair_load(p.down, row0 + 2 * (4 * half + pr), I, c, g, t, q[pr], sc[pr]);
          }
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) pair_mma1(q[pr], sc[pr], bf + c * 256, acc[pr]);
        }
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) pair_diag1(acc[pr], g, t, red + 16 * (4 * half + pr));
      }
    }
    if (i + GW < N) {
      int u2;
      const size_t rn = row_of(i + GW, u2);
#pragma unroll
      for (int pr = 0; pr < (ONE_STEP ? 8 : 4); ++pr) pair_load(p.down, rn + 2 * pr, I, 0, g, t, q[pr], sc[pr]);
    }
    __syncwarp();
    if (lane < 16) {
      // lane = 2 pair + row: output row row0 + lane; rows 0, 1 of pair pr at red[16 pr + 8 row]
      const int pr = lane >> 1, rr = lane & 1;
      const size_t a = (size_t)s_live[1 + kMaxLive + u];
      p.r[a * H + (row0 - (size_t)s_live[1 + u] * H) + lane] = octant_sum(red + 16 * pr + 8 * rr) * s_sc[u];
    }
    __syncwarp();
  }

  // rows of assignments that are not live (remote experts, dropped ids) are
  // zero: this CTA's slice of each
  const int n0 = (int)((long long)blockIdx.x * H / gridDim.x), n1 = (int)((long long)(blockIdx.x + 1) * H / gridDim.x);
  for (int a = 0; a < k; ++a) {
    bool live = false;
    for (int uu = 0; uu < n_live; ++uu) live |= s_live[1 + kMaxLive + uu] == a;
    if (!live)
      for (int r = n0 + (int)threadIdx.x; r < n1; r += kThreads) p.r[(size_t)a * H + r] = 0.f;
  }
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kNumSMs;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = kNumSMs;
    cached[dev] = n;
  }
  return cached[dev];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

bool decode_t1_supported(int H, int I, int E, int k) {
  if (H % 1024 || H > 8192 || I % 128 || I > 2048 || k < 1 || k > kMaxLive || E < 1 || E > 1024) return false;
  return (long long)E * (H > I ? H : I) < (1ll << 31);
}

cudaError_t launch_decode_t1_gate_up(const DecodeT1Args& a, cudaStream_t st) {
  if (!decode_t1_supported(a.H, a.I, a.E, a.k)) return cudaErrorInvalidValue;
  if (!aligned16(a.gate.codes) || !aligned16(a.up.codes) || ((uintptr_t)a.gate.scales & 1u) ||
      ((uintptr_t)a.up.scales & 1u) || ((uintptr_t)a.x & 7u) || ((uintptr_t)a.h & 7u))
    return cudaErrorInvalidValue;
  return launch_pdl(t1_gate_up_kernel, dim3(sm_count()), dim3(kThreads), 0, st, a);
}

cudaError_t launch_decode_t1_down(const DecodeT1Args& a, cudaStream_t st) {
  if (!decode_t1_supported(a.H, a.I, a.E, a.k)) return cudaErrorInvalidValue;
  if (!aligned16(a.down.codes) || ((uintptr_t)a.down.scales & 1u) || !aligned16(a.h)) return cudaErrorInvalidValue;
  const int smem = a.k * ((a.I + 1023) / 1024) * 256 * 8;
  auto kern = a.I <= 1024 ? t1_down_kernel<true> : t1_down_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(sm_count()), dim3(kThreads), (size_t)smem, st, a);
}

}  // namespace rnx
