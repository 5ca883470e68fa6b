// Single-token decode of the routed experts on the tensor cores
// (glm5next_mlp module docs, Constants / W4A16_GEMV_MODULE: at decode every
// routed-expert projection is M = 1, so the step is a stream over the touched
// experts' bytes). Two launches chained by programmatic dependent launch:
//
//   gate/up  the live experts' NVFP4 gate and up rows against x, with the
//            clamped SwiGLU (h, fp32 [k, I]);
//   down     the live experts' NVFP4 down rows against h, times the routing
//            weight (r, fp32 [k, H]; rows of assignments that are not live are
//            zero). moe_combine then sums r and the shared row.
//
// Both kernels run one CTA per SM: a producer warp streams 16-row tiles of
// codes and E4M3 scales into a ring of shared-memory stages with TMA (128-byte
// swizzle for the codes), sixteen consumer warps multiply them on the tensor
// cores with mma.sync m16n8k16 (f16 operands, fp32 accumulators).
//
// Arithmetic. A 16-row weight tile is the A operand: each E2M1 code is decoded
// to f16 by the hardware cvt and multiplied (f16) by its block's E4M3 scale;
// the product has at most 6 significant bits and lies in [2^-10, 2688], so it
// is exact in f16. The activation (x, or h) times a per-row power of two
// (max |a| in [2^14, 2^15)) in f16 is the B operand, column 0 (the other seven
// columns are zero). Every product is exact in the tensor core's fp32
// accumulation, so only the fp32 sums round; the power of two and the tensor
// scale are applied to the fp32 totals.
//
// K order. The 16 k-slots of one mma hold, in the A fragment of lane (g, t),
// four consecutive codes of the 32 that lane loaded (one 16-byte word of its
// row); B holds the activation at the same positions. A dot product does not
// depend on the order of its terms, so this is the plain row . activation.

#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tensor_map.h"
#include "tma.cuh"

namespace rnx {

namespace {

constexpr int kMaxLive = 16;               // top-k <= 16
// Consumer warps per CTA. A gate/up consumer holds its ring stage while it
// computes, so the ring keeps NS - kGuConsumers stages of copies in flight;
// the down kernel has its whole share of tiles in flight before it starts.
constexpr int kGuConsumers = 8;
constexpr int kDnConsumers = 16;
constexpr int kGuThreads = (kGuConsumers + 1) * kWarp;
constexpr int kDnThreads = (kDnConsumers + 1) * kWarp;
// Status bits 8..13 name the bounded wait that ran out.
enum : uint32_t {
  kWaitGuEmpty = 1u << 8,
  kWaitGuFull = 1u << 9,
  kWaitGuDrain = 1u << 10,
  kWaitDnEmpty = 1u << 11,
  kWaitDnFull = 1u << 12,
  kWaitDnDrain = 1u << 13,
};
constexpr int kSmemBudget = 200 * 1024;
constexpr int kBox = 2048;                 // one code box: 16 rows x 128 bytes (256 codes)
constexpr int kGuCodes = 512;              // codes per row in one gate/up stage
constexpr int kGuStage = 4 * kBox + 2 * 16 * (kGuCodes / 16);   // gate, up boxes + their scales: 9216
constexpr int kMaxStages = 24;

RNX_DEVICE void named_bar_sync(int id, int nthreads) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory"); }

// mma tile row of fragment row g (0..7): rows g and g + 1 (the two row
// groups one shared-memory wavefront serves) sit 4 apart in the tile, so their
// swizzled 16-byte words fall in opposite halves of the 128-byte line.
RNX_DEVICE int tile_row(int g) { return ((g & 1) << 2) | (g >> 1); }

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
                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp's share of a stage: NM matrices (mat_stride bytes apart; scales
// sf_stride apart, sp bytes per scale row) of 16 rows x (2 npair) chunks of
// 128 codes, against the B fragments bf of those chunks (8 per chunk, one
// uint2 per lane t). Codes sit in boxes of 16 rows x 128 bytes written by TMA
// with the 128-byte swizzle (16-byte word w of row r at w ^ (r & 7)).
// acc[m][c & 1] accumulates chunk c (two chains per matrix).
template <int NM>
RNX_DEVICE void stage_mma(const uint8_t* st, int mat_stride, const uint8_t* sf, int sf_stride, int sp, int npair,
                          const uint2* bf, bool b_on, int g, int t, float (&acc)[NM][2][4]) {
  const int r0 = tile_row(g);
  for (int cp = 0; cp < npair; ++cp) {
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
      const int c = 2 * cp + hc;
      const int o0 = cp * kBox + r0 * 128 + ((((hc << 2) | t) ^ r0) << 4);   // row r0 + 8: o0 + 1024
      uint2 b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) b[i] = b_on ? bf[(c * 8 + i) * 4 + t] : make_uint2(0u, 0u);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint8_t* cm = st + m * mat_stride;
        const uint4 q0 = *reinterpret_cast<const uint4*>(cm + o0);
        const uint4 q1 = *reinterpret_cast<const uint4*>(cm + o0 + 1024);
        const uint8_t* sm = sf + m * sf_stride + 8 * c + 2 * t;
        const uint32_t s0 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(sm + r0 * sp));
        const uint32_t s1 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(sm + (r0 + 8) * sp));
        uint32_t w0[16], w1[16];
        e2m1x8_to_f16x2x4(q0.x, w0[0], w0[1], w0[2], w0[3]);
        e2m1x8_to_f16x2x4(q0.y, w0[4], w0[5], w0[6], w0[7]);
        e2m1x8_to_f16x2x4(q0.z, w0[8], w0[9], w0[10], w0[11]);
        e2m1x8_to_f16x2x4(q0.w, w0[12], w0[13], w0[14], w0[15]);
        e2m1x8_to_f16x2x4(q1.x, w1[0], w1[1], w1[2], w1[3]);
        e2m1x8_to_f16x2x4(q1.y, w1[4], w1[5], w1[6], w1[7]);
        e2m1x8_to_f16x2x4(q1.z, w1[8], w1[9], w1[10], w1[11]);
        e2m1x8_to_f16x2x4(q1.w, w1[12], w1[13], w1[14], w1[15]);
        // the lane's 32 codes are two 16-code blocks: words 0..7, 8..15
        const uint32_t s0a = lo_lo(s0), s0b = hi_hi(s0), s1a = lo_lo(s1), s1b = hi_hi(s1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t sc0 = i < 4 ? s0a : s0b, sc1 = i < 4 ? s1a : s1b;
          mma_16816(acc[m][hc], hmul2(w0[2 * i], sc0), hmul2(w1[2 * i], sc1), hmul2(w0[2 * i + 1], sc0),
                    hmul2(w1[2 * i + 1], sc1), b[i].x, b[i].y);
        }
      }
    }
  }
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

struct GuParams {
  CUtensorMap gc, uc;      // gate / up codes [E I, H/2] bytes, box 128 B x 16 rows, SW128
  CUtensorMap gs, us;      // gate / up scales [E I, H/16] bytes, box 32 B x 16 rows
  DecodeT1Args a;
};

// Shared memory of one gate/up CTA (offsets from the 1024-aligned base):
// NS ring stages, x as B fragments (H f16), NB item slots of P partial tiles
// (gate 16 + up 16 fp32 each) with their arrival counters, barriers, the live
// list.
struct GuLayout {
  int P, NS, NB, xs, part, cnt, bar, live, tmp, ts, flag, total;
};
__host__ __device__ inline GuLayout gu_layout(int H) {
  GuLayout L{};
  L.P = H / kGuCodes;
  for (int ns = kMaxStages; ns >= 2; --ns) {
    L.NS = ns;
    // an item slot is reused kGuConsumers + ns stages later at the earliest:
    // by then the warp that summed the item has released its next stage
    L.NB = 1 + (ns + kGuConsumers - 1 + L.P - 1) / L.P;
    L.xs = ns * kGuStage;
    L.part = L.xs + H * 2;
    L.cnt = L.part + L.NB * L.P * 32 * 4;
    L.bar = (L.cnt + L.NB * 4 + 7) / 8 * 8;
    L.live = L.bar + 2 * ns * 8;
    L.tmp = L.live + (1 + 2 * kMaxLive) * 4;
    L.ts = L.tmp + 4 * kMaxLive * 4;
    L.flag = L.ts + 2 * kMaxLive * 4;
    L.total = L.flag + 16 + 1024;     // + alignment slack of the dynamic base
    if (L.total <= kSmemBudget) break;
  }
  return L;
}

__global__ void __launch_bounds__(kGuThreads, 1) t1_gate_up_kernel(const __grid_constant__ GuParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const DecodeT1Args& p = prm.a;
  const int H = p.H, I = p.I;
  const GuLayout L = gu_layout(H);
  const int P = L.P, NS = L.NS, NB = L.NB;
  uint2* xs = reinterpret_cast<uint2*>(smem + L.xs);
  float* part = reinterpret_cast<float*>(smem + L.part);
  int* cnt = reinterpret_cast<int*>(smem + L.cnt);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + NS;
  int* s_live = reinterpret_cast<int*>(smem + L.live);
  float* s_ts = reinterpret_cast<float*>(smem + L.ts);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L.flag);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) cnt[b] = 0;
    *s_abort = 0;
    fence_barrier_init();
  }
  pdl_wait();              // the plan and max |x| come from earlier launches
  pdl_trigger();
  load_live(p, p.gate.tensor_scale, p.up.tensor_scale, reinterpret_cast<int*>(smem + L.tmp), s_live, s_ts);
  const int n_live = s_live[0];
  const int TPE = I / 16;                    // 16-row tiles per expert
  const int N = n_live * TPE, G = gridDim.x, c0 = blockIdx.x;
  const int n_items = c0 < N ? (N - 1 - c0) / G + 1 : 0;
  const int n_stages = n_items * P;

  if (warp == kGuConsumers) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int m = 0; m < n_stages; ++m) {
        if (*s_abort) break;
        const int s = m % NS;
        if (m >= NS && !mbar_wait(&empty[s], ((uint32_t)(m / NS) & 1u) ^ 1u)) {
          set_status(p.status, kDevErrTimeout | kWaitGuEmpty);
          *s_abort = 1;
          break;
        }
        const int j = m / P, pt = m - j * P;
        const int i = c0 + j * G, u = i / TPE, tile = i - u * TPE;
        const int row0 = s_live[1 + u] * I + tile * 16;
        uint8_t* st = smem + (size_t)s * kGuStage;
        const int x0 = pt * (kGuCodes / 2);
        mbar_arrive_expect_tx(&full[s], (uint32_t)kGuStage);
        tma_load_2d(st, &prm.gc, x0, row0, &full[s]);
        tma_load_2d(st + kBox, &prm.gc, x0 + 128, row0, &full[s]);
        tma_load_2d(st + 2 * kBox, &prm.uc, x0, row0, &full[s]);
        tma_load_2d(st + 3 * kBox, &prm.uc, x0 + 128, row0, &full[s]);
        tma_load_2d(st + 4 * kBox, &prm.gs, pt * (kGuCodes / 16), row0, &full[s]);
        tma_load_2d(st + 4 * kBox + 512, &prm.us, pt * (kGuCodes / 16), row0, &full[s]);
        issued = m + 1;
      }
      // no copy may still be landing when the CTA exits
      for (int m = max(0, issued - NS); m < issued; ++m)
        if (!mbar_wait(&full[m % NS], (uint32_t)(m / NS) & 1u)) set_status(p.status, kDevErrTimeout | kWaitGuDrain);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  float up, unscale;
  prescale15(__uint_as_float(*p.xmax), up, unscale);
  // x as B fragments: entry (chunk cg, step i, lane t) = x[128 cg + 32 t + 4 i + 0..3]
  for (int f = threadIdx.x; f < H / 4; f += kGuConsumers * kWarp) {
    const int t = f & 3, i = (f >> 2) & 7, cg = f >> 5;
    const uint2 v = *reinterpret_cast<const uint2*>(p.x + 128 * cg + 32 * t + 4 * i);
    const float2 a = bf16x2_to_f32x2(v.x), b = bf16x2_to_f32x2(v.y);
    __half2 h0 = __floats2half2_rn(a.x * up, a.y * up), h1 = __floats2half2_rn(b.x * up, b.y * up);
    xs[f] = make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
  }
  named_bar_sync(1, kGuConsumers * kWarp);

  const int g = lane >> 2, t = lane & 3;
  for (int m = warp; m < n_stages; m += kGuConsumers) {
    if (*s_abort) break;
    const int s = m % NS;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(m / NS) & 1u));
    if (!ok) {
      if (lane == 0) {
        set_status(p.status, kDevErrTimeout | kWaitGuFull);
        *s_abort = 1;
      }
      break;
    }
    const int j = m / P, pt = m - j * P;
    const int i = c0 + j * G, u = i / TPE, tile = i - u * TPE;
    float acc[2][2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][b][q] = 0.f;
    const uint8_t* st = smem + (size_t)s * kGuStage;
    stage_mma<2>(st, 2 * kBox, st + 4 * kBox, 512, kGuCodes / 16, kGuCodes / 256, xs + pt * (kGuCodes / 128) * 32,
                 lane < 4, g, t, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    // column 0 of the tile lives in lanes t == 0: rows tile_row(g), + 8
    const int slot = j % NB;
    float* pb = part + (slot * P + pt) * 32;
    if (t == 0) {
      const int r0 = tile_row(g);
      pb[r0] = acc[0][0][0] + acc[0][1][0];
      pb[r0 + 8] = acc[0][0][2] + acc[0][1][2];
      pb[16 + r0] = acc[1][0][0] + acc[1][1][0];
      pb[16 + r0 + 8] = acc[1][0][2] + acc[1][1][2];
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&cnt[slot], 1) == P - 1;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      // the tile's P partial sums in part order, then the SwiGLU
      __threadfence_block();
      if (lane < 16) {
        const float* pj = part + slot * P * 32;
        float gs = 0.f, us = 0.f;
        for (int q = 0; q < P; ++q) {
          gs += pj[q * 32 + lane];
          us += pj[q * 32 + 16 + lane];
        }
        gs *= unscale * s_ts[u];
        us *= unscale * s_ts[kMaxLive + u];
        const int a = s_live[1 + kMaxLive + u];
        p.h[(size_t)a * I + tile * 16 + lane] = clamped_swiglu(gs, us, p.limit);
      }
      __syncwarp();
      if (lane == 0) cnt[slot] = 0;
    }
  }
}

// ============================================================== down

struct DnParams {
  CUtensorMap dc;          // down codes [E H, I/2] bytes, box 128 B x 16 rows, SW128
  CUtensorMap ds;          // down scales [E H, I/16] bytes, box I/16 B x 16 rows
  DecodeT1Args a;
};

struct DnLayout {
  int stage, NS, hs, hsc, hmax, bar, live, tmp, ts, flag, total;
};
constexpr int kHq = 16;          // float4 of h per consumer thread: k I / 4 <= kHq * 512 (k <= 16, I <= 2048)
__host__ __device__ inline int dn_stage_bytes(int I) { return (9 * I + 1023) / 1024 * 1024; }
__host__ __device__ inline DnLayout dn_layout(int I, int k) {
  DnLayout L{};
  L.stage = dn_stage_bytes(I);
  for (int ns = kMaxStages; ns >= 1; --ns) {
    L.NS = ns;
    L.hs = ns * L.stage;
    L.hsc = L.hs + k * I * 2;
    L.hmax = L.hsc + kMaxLive * 4;
    L.bar = (L.hmax + kMaxLive * 4 + 7) / 8 * 8;
    L.live = L.bar + 2 * ns * 8;
    L.tmp = L.live + (1 + 2 * kMaxLive) * 4;
    L.ts = L.tmp + 4 * kMaxLive * 4;
    L.flag = L.ts + 2 * kMaxLive * 4;
    L.total = L.flag + 16 + 1024;
    if (L.total <= kSmemBudget) break;
  }
  return L;
}

__global__ void __launch_bounds__(kDnThreads, 1) t1_down_kernel(const __grid_constant__ DnParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const DecodeT1Args& p = prm.a;
  const int H = p.H, I = p.I, k = p.k;
  const DnLayout L = dn_layout(I, k);
  const int NS = L.NS;
  // Each consumer warp owns D ring slots and consumes their phases in order
  // (item m: warp m % WE, its (m / WE)-th item), so no wait can target a
  // phase two ahead of its barrier.
  const int WE = min(kDnConsumers, NS), D = NS / WE;
  uint2* hs = reinterpret_cast<uint2*>(smem + L.hs);
  float* hsc = reinterpret_cast<float*>(smem + L.hsc);
  uint32_t* hmax = reinterpret_cast<uint32_t*>(smem + L.hmax);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + NS;
  int* s_live = reinterpret_cast<int*>(smem + L.live);
  float* s_ts = reinterpret_cast<float*>(smem + L.ts);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L.flag);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  // The plan comes from two launches back, complete when this grid starts:
  // the weight stream starts before the wait for h.
  load_live(p, p.down.tensor_scale, nullptr, reinterpret_cast<int*>(smem + L.tmp), s_live, s_ts);
  const int n_live = s_live[0];
  const int TPE = H / 16;
  const int N = n_live * TPE, G = gridDim.x, c0 = blockIdx.x;
  const int n_items = c0 < N ? (N - 1 - c0) / G + 1 : 0;
  const int nbox = I / 256;

  if (warp == kDnConsumers) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int m = 0; m < n_items; ++m) {
        if (*s_abort) break;
        const int w = m % WE, l = m / WE, s = w * D + l % D;
        if (l >= D && !mbar_wait(&empty[s], ((uint32_t)(l / D) & 1u) ^ 1u)) {
          set_status(p.status, kDevErrTimeout | kWaitDnEmpty);
          *s_abort = 1;
          break;
        }
        const int i = c0 + m * G, u = i / TPE, tile = i - u * TPE;
        const int row0 = s_live[1 + u] * H + tile * 16;
        uint8_t* st = smem + (size_t)s * L.stage;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(9 * I));
        for (int b = 0; b < nbox; ++b) tma_load_2d(st + b * kBox, &prm.dc, b * 128, row0, &full[s]);
        tma_load_2d(st + 8 * I, &prm.ds, 0, row0, &full[s]);
        issued = m + 1;
      }
      for (int m = max(0, issued - WE * D); m < issued; ++m) {
        const int w = m % WE, l = m / WE;
        if (!mbar_wait(&full[w * D + l % D], (uint32_t)(l / D) & 1u)) set_status(p.status, kDevErrTimeout | kWaitDnDrain);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  pdl_wait();                // h comes from the previous launch
  pdl_trigger();
  // h rows of the live experts as B fragments (f16, a power of two per row
  // from the row's max |h|), and each row's output factor. All consumer
  // threads: one round of loads (kHq float4 per thread, issued together), the
  // row maxima through shared memory, then the conversion.
  {
    const int tid = threadIdx.x, nq = n_live * (I / 4);
    float4 v[kHq];
#pragma unroll
    for (int q = 0; q < kHq; ++q) {
      const int f = tid + q * kDnConsumers * kWarp;
      if (f < nq) {
        const int u = f / (I / 4), c = f - u * (I / 4);
        v[q] = *reinterpret_cast<const float4*>(p.h + (size_t)s_live[1 + kMaxLive + u] * I + 4 * c);
      } else {
        v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (tid < kMaxLive) hmax[tid] = 0u;
    named_bar_sync(1, kDnConsumers * kWarp);
#pragma unroll
    for (int q = 0; q < kHq; ++q) {
      const int f = tid + q * kDnConsumers * kWarp;
      if (f < nq) {
        const float m = fmaxf(fmaxf(fabsf(v[q].x), fabsf(v[q].y)), fmaxf(fabsf(v[q].z), fabsf(v[q].w)));
        atomicMax(&hmax[f / (I / 4)], __float_as_uint(m));       // non-negative floats order as integers
      }
    }
    named_bar_sync(1, kDnConsumers * kWarp);
#pragma unroll
    for (int q = 0; q < kHq; ++q) {
      const int f = tid + q * kDnConsumers * kWarp;
      if (f < nq) {
        const int u = f / (I / 4), c = f - u * (I / 4), pos = 4 * c;
        float upx, unscale;
        prescale15(__uint_as_float(hmax[u]), upx, unscale);
        __half2 h0 = __floats2half2_rn(v[q].x * upx, v[q].y * upx);
        __half2 h1 = __floats2half2_rn(v[q].z * upx, v[q].w * upx);
        hs[(size_t)u * (I / 4) + ((pos >> 7) * 8 + ((pos >> 2) & 7)) * 4 + ((pos >> 5) & 3)] =
            make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
      }
    }
    if (tid < n_live) {
      float upx, unscale;
      prescale15(__uint_as_float(hmax[tid]), upx, unscale);
      hsc[tid] = unscale * s_ts[tid] * p.weights[s_live[1 + kMaxLive + tid]];
    }
  }
  named_bar_sync(1, kDnConsumers * kWarp);

  const int g = lane >> 2, t = lane & 3;
  for (int m = warp; m < n_items && warp < WE; m += WE) {
    if (*s_abort) break;
    const int l = m / WE, s = warp * D + l % D;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(l / D) & 1u));
    if (!ok) {
      if (lane == 0) {
        set_status(p.status, kDevErrTimeout | kWaitDnFull);
        *s_abort = 1;
      }
      break;
    }
    const int i = c0 + m * G, u = i / TPE, tile = i - u * TPE;
    float acc[1][2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[0][b][q] = 0.f;
    const uint8_t* st = smem + (size_t)s * L.stage;
    stage_mma<1>(st, 0, st + 8 * I, 0, I / 16, I / 256, hs + (size_t)u * (I / 4), lane < 4, g, t, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (t == 0) {
      const int a = s_live[1 + kMaxLive + u];
      const float sc = hsc[u];
      const int r0 = tile_row(g);
      float* rr = p.r + (size_t)a * H + tile * 16;
      rr[r0] = (acc[0][0][0] + acc[0][1][0]) * sc;
      rr[r0 + 8] = (acc[0][0][2] + acc[0][1][2]) * sc;
    }
  }

  // rows of assignments that are not live (remote experts, dropped ids) are
  // zero: this CTA's slice of each
  const int n0 = (int)((long long)c0 * H / G), n1 = (int)((long long)(c0 + 1) * H / G);
  for (int a = 0; a < k; ++a) {
    bool live = false;
    for (int u = 0; u < n_live; ++u) live |= s_live[1 + kMaxLive + u] == a;
    if (!live)
      for (int r = n0 + (int)threadIdx.x; r < n1; r += kDnConsumers * kWarp) p.r[(size_t)a * H + r] = 0.f;
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
  if (H % kGuCodes || H > 8192 || I % 256 || I > 2048 || k < 1 || k > kMaxLive || E < 1 || E > 1024) return false;
  if ((long long)E * (H > I ? H : I) >= (1ll << 31)) return false;
  const GuLayout g = gu_layout(H);
  if (g.total > kSmemBudget || g.NS < 2) return false;
  const DnLayout d = dn_layout(I, k);
  if (d.total > kSmemBudget || d.NS < 2) return false;
  return true;
}

cudaError_t launch_decode_t1_gate_up(const DecodeT1Args& a, cudaStream_t st) {
  if (!decode_t1_supported(a.H, a.I, a.E, a.k)) return cudaErrorInvalidValue;
  if (!aligned16(a.gate.codes) || !aligned16(a.up.codes) || !aligned16(a.gate.scales) || !aligned16(a.up.scales) ||
      ((uintptr_t)a.x & 7u))
    return cudaErrorInvalidValue;
  GuParams p;
  memset(&p, 0, sizeof p);
  const uint64_t rows = (uint64_t)a.E * a.I;
  if (!make_tensor_map_2d(&p.gc, a.gate.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.H / 2, rows, 128, 16,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&p.uc, a.up.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.H / 2, rows, 128, 16,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&p.gs, a.gate.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.H / 16, rows, kGuCodes / 16, 16,
                          CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&p.us, a.up.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.H / 16, rows, kGuCodes / 16, 16,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  p.a = a;
  const GuLayout L = gu_layout(a.H);
  cudaError_t e = cudaFuncSetAttribute(t1_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(t1_gate_up_kernel, dim3(sm_count()), dim3(kGuThreads), (size_t)L.total, st, p);
}

cudaError_t launch_decode_t1_down(const DecodeT1Args& a, cudaStream_t st) {
  if (!decode_t1_supported(a.H, a.I, a.E, a.k)) return cudaErrorInvalidValue;
  if (!aligned16(a.down.codes) || !aligned16(a.down.scales) || !aligned16(a.h)) return cudaErrorInvalidValue;
  DnParams p;
  memset(&p, 0, sizeof p);
  const uint64_t rows = (uint64_t)a.E * a.H;
  if (!make_tensor_map_2d(&p.dc, a.down.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.I / 2, rows, 128, 16,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&p.ds, a.down.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.I / 16, rows, a.I / 16, 16,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  p.a = a;
  const DnLayout L = dn_layout(a.I, a.k);
  cudaError_t e = cudaFuncSetAttribute(t1_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(t1_down_kernel, dim3(sm_count()), dim3(kDnThreads), (size_t)L.total, st, p);
}

}  // namespace rnx
