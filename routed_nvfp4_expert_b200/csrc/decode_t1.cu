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
// registers with coalesced 128-bit loads (about 9 KB per warp in flight, 144
// KB per SM), no shared-memory staging of weights, and multiplies them on the
// tensor cores with mma.sync m16n8k16 (f16 operands, fp32 accumulators). The
// down kernel issues the loads of its first tile before it waits for h.
//
// Arithmetic. Weights are the A operand: each E2M1 code is decoded to f16 by
// the hardware cvt and multiplied (f16) by its block's E4M3 scale; the product
// has at most 6 significant bits and lies in [2^-10, 2688], so it is exact in
// f16. The activation (x, or h) times a per-row power of two (max |a| in
// [2^14, 2^15)) in f16 is the B operand. Every product is exact in the tensor
// core's fp32 accumulation, so only the fp32 sums round; the power of two and
// the tensor scale are applied to the fp32 totals.
//
// Layouts. A dot product does not depend on the order of its terms; the
// kernels only choose which weights meet which activations in one mma.
//   gate/up: an mma's 16 A rows are (row 0 of the pair, K octant g) and
//     (row 1, octant g) for g = 0..7, and B column n holds x's octant n, so
//     the diagonal D[g][g] (and D[g + 8][g]) is octant g's partial dot
//     product of each row; a warp sum over the eight octants finishes it. Lane
//     (g, t) reads 16 contiguous bytes of each row per step.
//   down: an mma's 16 A rows are 16 consecutive weight rows over the same 16
//     k positions and B column 0 holds h (the other columns are zero); lane
//     (g, t) holds rows g and g + 8.
// In both, the 16 k-slots of lane (g, t) hold four consecutive codes of the
// 32 it loaded, and B holds the activation at the same positions.

#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"

namespace rnx {

namespace {

constexpr int kMaxLive = 16;               // top-k <= 16
constexpr int kWarps = 16;                 // warps per CTA, one CTA per SM
constexpr int kThreads = kWarps * kWarp;
constexpr int kDnBatch = 8;                // down: 128-code chunks held in registers at a time

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

// ============================================================== gate/up
//
// Item = a pair of rows (2 rp, 2 rp + 1) of one live expert's gate and up
// matrices, full K; one warp per item at a time. NCH = H / 1024 steps of
// 128 codes per octant, taken 4 at a time into registers.

__global__ void __launch_bounds__(kThreads, 1) t1_gate_up_kernel(const DecodeT1Args p) {
  __shared__ __align__(16) uint2 xs[8192 / 4];      // x as B fragments, H <= 8192
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
  auto rows = [&](int i, int& u, size_t& r0) {
    u = i / (I / 2);
    r0 = (size_t)s_live[1 + u] * I + 2 * (size_t)(i - u * (I / 2));
  };
  // x as B fragments: entry ((c * 8 + i) * 32 + lane') = x[n H/8 + 128 c + 32 t' + 4 i + 0..3],
  // n = lane' / 4 (octant), t' = lane' % 4
  float up, unscale;
  prescale15(__uint_as_float(*p.xmax), up, unscale);
  for (int f = threadIdx.x; f < H / 4; f += kThreads) {
    const int ln = f & 31, i = (f >> 5) & 7, c = f >> 8;
    const uint2 v = *reinterpret_cast<const uint2*>(p.x + (ln >> 2) * (H / 8) + 128 * c + 32 * (ln & 3) + 4 * i);
    const float2 a = bf16x2_to_f32x2(v.x), b = bf16x2_to_f32x2(v.y);
    __half2 h0 = __floats2half2_rn(a.x * up, a.y * up), h1 = __floats2half2_rn(b.x * up, b.y * up);
    xs[f] = make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
  }
  __syncthreads();

  // Ask L2 for every weight byte this CTA's warps will read, then for a share
  // of the down kernel's tiles (all of the step's expert bytes fit in L2): the
  // memory system streams from DRAM without gaps while the warps compute from
  // L2. x was staged first so that its loads did not queue behind these.
  for (int i = first; i < N; i += GW) {
    int u;
    size_t r0;
    rows(i, u, r0);
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
    size_t r0;
    rows(i, u, r0);
    float acc[2][2][4];      // [matrix][chain][fragment]
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[m][j][q] = 0.f;
    for (int c0 = 0; c0 < NCH; c0 += 4) {
      // this lane's 16 bytes of each row at octant g, steps c0 .. c0 + 3
      uint4 q[2][2][4];        // [matrix][row][step]
      uint32_t sc[2][4];       // [matrix][step]: row 0's scale pair, row 1's in the high half
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const nvfp4_bank_t& bk = m ? p.up : p.gate;
        const uint8_t* sp = bk.scales + r0 * (H / 16) + g * (H / 128) + 2 * t;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const uint8_t* cp = bk.codes + (r0 + rr) * (H / 2) + g * (H / 16) + 16 * t;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            q[m][rr][j] = c0 + j < NCH ? ldg_stream(cp + 64 * (c0 + j)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          sc[m][j] = c0 + j < NCH ? (uint32_t)ldg_u16(sp + 8 * (c0 + j)) |
                                        ((uint32_t)ldg_u16(sp + H / 16 + 8 * (c0 + j)) << 16)
                                  : 0u;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (c0 + j < NCH) {
          uint32_t z[2][4];      // per matrix: row 0 block 2t, 2t + 1, row 1 block 2t, 2t + 1 (f16x2 broadcast)
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const uint32_t s0 = e4m3x2_to_f16x2((uint16_t)(sc[m][j] & 0xFFFFu)),
                           s1 = e4m3x2_to_f16x2((uint16_t)(sc[m][j] >> 16));
            z[m][0] = lo_lo(s0);
            z[m][1] = hi_hi(s0);
            z[m][2] = lo_lo(s1);
            z[m][3] = hi_hi(s1);
          }
          const uint2* bj = xs + (c0 + j) * 8 * 32 + lane;
#define RNX_GU_STEP(II)                                                                                    \
  {                                                                                                         \
    const uint2 b = bj[(II) * 32];                                                                          \
    mma_step<II>(acc[0][(II) & 1], q[0][0][j], q[0][1][j], z[0][(II) < 4 ? 0 : 1], z[0][(II) < 4 ? 2 : 3], b); \
    mma_step<II>(acc[1][(II) & 1], q[1][0][j], q[1][1][j], z[1][(II) < 4 ? 0 : 1], z[1][(II) < 4 ? 2 : 3], b); \
  }
          RNX_GU_STEP(0) RNX_GU_STEP(1) RNX_GU_STEP(2) RNX_GU_STEP(3)
          RNX_GU_STEP(4) RNX_GU_STEP(5) RNX_GU_STEP(6) RNX_GU_STEP(7)
#undef RNX_GU_STEP
        }
      }
    }
    // the diagonal: octant g of row 0 is D[g][g], of row 1 D[g + 8][g], in
    // lane (g, g / 2), element g % 2; then the sum over the eight octants
    float v[2][2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      float d[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) d[q] = acc[m][0][q] + acc[m][1][q];
      const bool mine = t == (g >> 1);
      v[m][0] = warp_sum(mine ? ((g & 1) ? d[1] : d[0]) : 0.f);
      v[m][1] = warp_sum(mine ? ((g & 1) ? d[3] : d[2]) : 0.f);
    }
    if (lane == 0) {
      const float sg = unscale * s_ts[u], su = unscale * s_ts[kMaxLive + u];
      const float2 hv = make_float2(clamped_swiglu(v[0][0] * sg, v[1][0] * su, p.limit),
                                    clamped_swiglu(v[0][1] * sg, v[1][1] * su, p.limit));
      const size_t a = (size_t)s_live[1 + kMaxLive + u];
      *reinterpret_cast<float2*>(p.h + a * I + (r0 - (size_t)s_live[1 + u] * I)) = hv;
    }
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
// Item = a 16-row tile of one live expert's down matrix, full K (I / 128
// chunks, kDnBatch at a time in registers); one warp per item at a time.

struct DnTile {
  uint4 q[2][kDnBatch];      // rows g and g + 8, chunk c0 + j, this lane's 16 bytes
  uint32_t sc[kDnBatch];     // their E4M3 scale pairs: row g's, row g + 8's in the high half
};

RNX_DEVICE void dn_load(const DecodeT1Args& p, size_t row0, int c0, int nch, int g, int t, DnTile& T) {
  const int I = p.I;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const uint8_t* cp = p.down.codes + (row0 + g + 8 * rr) * (I / 2) + 16 * t;
#pragma unroll
    for (int j = 0; j < kDnBatch; ++j) T.q[rr][j] = c0 + j < nch ? ldg_stream(cp + 64 * (c0 + j)) : make_uint4(0u, 0u, 0u, 0u);
  }
  const uint8_t* sp = p.down.scales + (row0 + g) * (I / 16) + 2 * t;
#pragma unroll
  for (int j = 0; j < kDnBatch; ++j)
    T.sc[j] = c0 + j < nch ? (uint32_t)ldg_u16(sp + 8 * (c0 + j)) | ((uint32_t)ldg_u16(sp + 8 * (I / 16) + 8 * (c0 + j)) << 16)
                           : 0u;
}

RNX_DEVICE void dn_mma(const DnTile& T, int c0, int nch, const uint2* bf, bool b_on, int t, float (&acc)[4][4]) {
#pragma unroll
  for (int j = 0; j < kDnBatch; ++j) {
    if (c0 + j < nch) {
      const uint32_t s0 = e4m3x2_to_f16x2((uint16_t)(T.sc[j] & 0xFFFFu)), s1 = e4m3x2_to_f16x2((uint16_t)(T.sc[j] >> 16));
      const uint32_t s0a = lo_lo(s0), s0b = hi_hi(s0), s1a = lo_lo(s1), s1b = hi_hi(s1);
      const uint2* bj = bf + (c0 + j) * 8 * 4 + t;
#define RNX_DN_STEP(II)                                                                                        \
  mma_step<II>(acc[(II) & 3], T.q[0][j], T.q[1][j], (II) < 4 ? s0a : s0b, (II) < 4 ? s1a : s1b,                \
               b_on ? bj[(II) * 4] : make_uint2(0u, 0u));
      RNX_DN_STEP(0) RNX_DN_STEP(1) RNX_DN_STEP(2) RNX_DN_STEP(3)
      RNX_DN_STEP(4) RNX_DN_STEP(5) RNX_DN_STEP(6) RNX_DN_STEP(7)
#undef RNX_DN_STEP
    }
  }
}

constexpr int kHq = 8;           // float4 of h per thread held in registers while staging

__global__ void __launch_bounds__(kThreads, 1) t1_down_kernel(const DecodeT1Args p) {
  extern __shared__ __align__(16) uint2 hs[];               // h as B fragments: k x I f16
  __shared__ float s_up[kMaxLive], s_sc[kMaxLive];
  __shared__ uint32_t s_max[kMaxLive];
  __shared__ int s_live[1 + 2 * kMaxLive];
  __shared__ int s_tmp[4 * kMaxLive];
  __shared__ float s_ts[2 * kMaxLive];
  const int H = p.H, I = p.I, k = p.k, NCH = I / 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  // The plan comes from two launches back, complete when this grid starts:
  // the first tile's weights are loaded before the wait for h.
  load_live(p, p.down.tensor_scale, nullptr, s_tmp, s_live, s_ts);
  const int n_live = s_live[0];
  const int TPE = H / 16, N = n_live * TPE, GW = gridDim.x * kWarps;
  int i = blockIdx.x * kWarps + warp;
  DnTile T;
  auto row_of = [&](int it, int& u) {
    u = it / TPE;
    return (size_t)s_live[1 + u] * H + 16 * (size_t)(it - u * TPE);
  };
  if (i < N) {
    int u;
    dn_load(p, row_of(i, u), 0, NCH, g, t, T);
  }
  if (threadIdx.x < kMaxLive) s_max[threadIdx.x] = 0u;
  pdl_wait();                // h comes from the previous launch
  pdl_trigger();

  // h rows of the live experts as B fragments: entry ((c * 8 + i) * 4 + t) =
  // h[128 c + 32 t + 4 i + 0..3] times the row's power of two. The row maxima
  // first (one shared atomic per warp and row: a warp's 32 consecutive float4
  // lie in one row), then the conversion.
  {
    const int nq = n_live * (I / 4);
    const bool in_regs = nq <= kHq * kThreads;
    float4 v[kHq];
    auto load_h = [&](int f) {
      const int u = f / (I / 4);
      return *reinterpret_cast<const float4*>(p.h + (size_t)s_live[1 + kMaxLive + u] * I + 4 * (f - u * (I / 4)));
    };
    auto amax4 = [](float4 a) { return fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))); };
    __syncthreads();
    if (in_regs) {
#pragma unroll
      for (int q = 0; q < kHq; ++q) {
        const int f = threadIdx.x + q * kThreads;
        v[q] = f < nq ? load_h(f) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    for (int q = 0; q * kThreads < nq; ++q) {
      const int f = threadIdx.x + q * kThreads;             // warp-uniform: f < nq for all lanes or none
      if (f - lane < nq) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (in_regs) {
#pragma unroll
          for (int qq = 0; qq < kHq; ++qq)
            if (qq == q) a = v[qq];
        } else {
          a = load_h(f);
        }
        const float m = warp_max(amax4(a));
        if (lane == 0) atomicMax(&s_max[f / (I / 4)], __float_as_uint(m));   // non-negative floats order as integers
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
    for (int q = 0; q * kThreads < nq; ++q) {
      const int f = threadIdx.x + q * kThreads;
      if (f < nq) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (in_regs) {
#pragma unroll
          for (int qq = 0; qq < kHq; ++qq)
            if (qq == q) a = v[qq];
        } else {
          a = load_h(f);
        }
        const int u = f / (I / 4), pos = 4 * (f - u * (I / 4));
        const float upx = s_up[u];
        __half2 h0 = __floats2half2_rn(a.x * upx, a.y * upx), h1 = __floats2half2_rn(a.z * upx, a.w * upx);
        hs[(size_t)u * (I / 4) + ((pos >> 7) * 8 + ((pos >> 2) & 7)) * 4 + ((pos >> 5) & 3)] =
            make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
      }
    }
    __syncthreads();
  }

  for (; i < N; i += GW) {
    int u;
    const size_t row0 = row_of(i, u);
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
    const uint2* bf = hs + (size_t)u * (I / 4);
    for (int c0 = 0; c0 < NCH; c0 += kDnBatch) {
      if (c0 > 0) dn_load(p, row0, c0, NCH, g, t, T);
      dn_mma(T, c0, NCH, bf, lane < 4, t, acc);
    }
    if (t == 0) {
      const float sc = s_sc[u];
      const size_t a = (size_t)s_live[1 + kMaxLive + u];
      float* rr = p.r + a * H + (row0 - (size_t)s_live[1 + u] * H);
      rr[g] = ((acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0])) * sc;
      rr[g + 8] = ((acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2])) * sc;
    }
    if (i + GW < N) {
      int u2;
      dn_load(p, row_of(i + GW, u2), 0, NCH, g, t, T);
    }
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
  const int smem = a.k * a.I * 2;
  cudaError_t e = cudaFuncSetAttribute(t1_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(t1_down_kernel, dim3(sm_count()), dim3(kThreads), (size_t)smem, st, a);
}

}  // namespace rnx
