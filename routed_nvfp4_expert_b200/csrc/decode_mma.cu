// Decode with a handful of tokens (T <= 8) on the tensor cores
// (glm5next_mlp module docs, Constants / W4A16_GEMV_MODULE: at decode every
// routed-expert projection is a GEMV with M = 1 per token, so the step is a
// stream over the touched experts' bytes). Two launches chained by
// programmatic dependent launch:
//
//   gate/up  16-row tiles of the live experts' NVFP4 gate and up matrices
//            against the expert's tokens, then the clamped SwiGLU:
//            h fp32 [T*k, I] (rows of assignments that are not live are zero);
//   down     16-row tiles of the live experts' NVFP4 down matrices against
//            the expert's h rows, times the routing weight: r fp32 [T*k, H]
//            (zero rows for assignments that are not live). moe_combine then
//            sums r and the shared row.
//
// One CTA of 16 warps per SM. A warp streams its weight rows straight into
// registers with coalesced 128-bit loads and keeps the next steps' loads in
// flight while it multiplies the current one (a ring of register slots: each
// step's slot is refilled, for the step DEPTH ahead, as soon as it is used),
// so the loads of one warp span its item boundaries and no warp waits for a
// whole item before it computes.
//
// Arithmetic. Weights are the A operand of mma.sync m16n8k16 (f16 operands,
// fp32 accumulators): each E2M1 code is decoded to f16 by the hardware cvt
// and multiplied (f16) by its block's E4M3 scale; the product has at most 6
// significant bits and lies in [2^-10, 2688], so it is exact in f16. The B
// operand holds the activations of up to 8 tokens (one per column), each
// times a power of two that brings the row's max |a| into [2^14, 2^15) (exact
// for bf16 x; h is rounded to 11 significant bits). Every product is exact in
// the fp32 accumulation, so only the fp32 sums round; the power of two and
// the tensor scale are applied to the fp32 totals.
//
// Layout. A dot product does not depend on the order of its terms, so the
// kernels choose which codes meet which mma k-slots. Lane (g, t) of a warp
// loads, per step, 16 contiguous bytes (32 codes) of tile rows g and g + 8 at
// byte 16 t + 64 s of the step's 64-byte window, so one warp load covers 64
// contiguous bytes of each of 8 rows; its 8 mma per step each take four
// consecutive codes of those 32 (k-slots 2t, 2t+1, 2t+8, 2t+9), and B holds
// each token's activations at the same four positions.

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "gemv_common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace rnx {

namespace {

constexpr int kWarps = 16;                 // warps per CTA, one CTA per SM
constexpr int kThreads = kWarps * kWarp;
constexpr int kMaxCols = 8;                // tokens per expert (mma N)
constexpr int kMaxAsg = 128;               // T * k
constexpr int kMaxLive = 128;              // live experts <= T * k
constexpr int kDepthGU = 4;                // gate/up steps in flight per warp
constexpr int kDepthD = 6;                 // down steps in flight per warp
constexpr int kPad = 8;                    // f16 elements of padding per staged activation row

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

// Two E2M1 bytes of w (bytes 0, 1, or 2, 3 when HI) -> two f16x2 words (the
// low nibble, the even element, in the low half).
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

// Loads that the compiler keeps in program order with each other: the
// activation loads of a launch's prologue go out ahead of its first weight
// loads (the weight ring: streaming, no L1 allocation).
RNX_DEVICE uint4 ldg_ordered(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
RNX_DEVICE uint4 ldg_ring(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
RNX_DEVICE uint32_t ldg_ring_u16(const void* p) {
  uint16_t r;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}
RNX_DEVICE float4 ldg_f4_ordered(const float* p) {
  float4 r;
  asm volatile("ld.global.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
  return r;
}

RNX_DEVICE void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The 8 mma of one step of one matrix: q0 / q1 = the lane's 16 bytes of tile
// rows g / g + 8, sc = their two scale bytes each (row g in the low half),
// b[j] = the lane's B words for mma 2j (x, y) and 2j + 1 (z, w).
RNX_DEVICE void step_mma(float (&acc)[4], const uint4& q0, const uint4& q1, uint32_t sc, const uint4 (&b)[4]) {
  const uint32_t s0 = e4m3x2_to_f16x2((uint16_t)(sc & 0xFFFFu)), s1 = e4m3x2_to_f16x2((uint16_t)(sc >> 16));
  const uint32_t z0a = lo_lo(s0), z0b = hi_hi(s0), z1a = lo_lo(s1), z1b = hi_hi(s1);
#pragma unroll
  for (int ii = 0; ii < 8; ++ii) {
    uint32_t a0, a1, a2, a3;
    if (ii & 1) {
      e2m1_pair<true>(word_of(q0, ii >> 1), a0, a2);
      e2m1_pair<true>(word_of(q1, ii >> 1), a1, a3);
    } else {
      e2m1_pair<false>(word_of(q0, ii >> 1), a0, a2);
      e2m1_pair<false>(word_of(q1, ii >> 1), a1, a3);
    }
    const uint32_t z0 = ii < 4 ? z0a : z0b, z1 = ii < 4 ? z1a : z1b;
    const uint4& bb = b[ii >> 1];
    mma_16816(acc, hmul2(a0, z0), hmul2(a1, z1), hmul2(a2, z0), hmul2(a3, z1), (ii & 1) ? bb.z : bb.x,
              (ii & 1) ? bb.w : bb.y);
  }
}

// The routing plan's live experts in shared memory: e[u], the expert of live
// slot u (expert order), n[u] its token count (0 when its plan entry is out of
// range: its tiles then read expert 0's bytes and write nothing), off[u] its
// first entry in sorted[]; tsa / tsb the tensor scales asked for (filled by
// load_scales, after the plan).
struct PlanS {
  int n_live;
  int e[kMaxLive], n[kMaxLive], off[kMaxLive];
  int sorted[kMaxAsg];
  uint8_t live_asg[kMaxAsg];
  float tsa[kMaxLive], tsb[kMaxLive];
};
constexpr int kMaxE = 1024;

// One round of global loads (the active list, every expert's count and
// offset, the sorted assignments), then the live slots from shared memory.
// All threads call it (three barriers).
RNX_DEVICE void load_plan(const DecodeMmaArgs& p, PlanS& S, int* s_cnt, int* s_off) {
  const int TK = p.T * p.k, E = p.E, i = threadIdx.x;
  const int n_raw = min(min(max(p.active[0], 0), E), kMaxLive);   // active holds E + 1 entries
  for (int e = i; e < E; e += blockDim.x) {
    s_cnt[e] = p.counts[e];
    s_off[e] = p.offsets[e];
  }
  int act = 0;
  if (i < min(E, kMaxLive)) act = p.active[1 + i];
  if (i < kMaxAsg) {
    int v = 0;
    if (i < TK) {
      v = p.sorted[i];
      if (v < 0 || v >= TK) {
        set_status(p.status, kDevErrBounds);
        v = 0;
      }
    }
    S.sorted[i] = v;
    S.live_asg[i] = 0;
  }
  if (i == 0) S.n_live = n_raw;
  __syncthreads();
  if (i < n_raw) {
    int e = act, off = 0, cnt = 0;
    bool ok = e >= 0 && e < E && e >= p.lb && e < p.le;
    if (ok) {
      off = s_off[e];
      cnt = s_cnt[e];
      ok = off >= 0 && cnt >= 1 && cnt <= min(p.T, kMaxCols) && off + cnt <= TK;
    }
    if (!ok) {
      if (blockIdx.x == 0) set_status(p.status, kDevErrBounds);
      e = 0;
      off = 0;
      cnt = 0;
    }
    S.e[i] = e;
    S.n[i] = cnt;
    S.off[i] = off;
  }
  __syncthreads();
  if (i < n_raw)
    for (int c = 0; c < S.n[i]; ++c) S.live_asg[S.sorted[S.off[i] + c]] = 1;
  __syncthreads();
}

// The live experts' tensor scales (visible after the caller's next barrier).
RNX_DEVICE void load_scales(const PlanS& S, const float* ts0, const float* ts1, PlanS& W) {
  const int i = threadIdx.x;
  if (i < S.n_live) {
    const bool ok = S.n[i] > 0;
    W.tsa[i] = ok ? ts0[S.e[i]] : 0.f;
    W.tsb[i] = (ok && ts1) ? ts1[S.e[i]] : 0.f;
  }
}

// Zero rows (of `width` floats) of the assignments that are not live: this
// CTA's slice of each.
RNX_DEVICE void zero_dead_rows(const PlanS& S, int TK, int width, float* out) {
  const int n0 = (int)((long long)blockIdx.x * width / gridDim.x);
  const int n1 = (int)((long long)(blockIdx.x + 1) * width / gridDim.x);
  for (int a = 0; a < TK; ++a)
    if (!S.live_asg[a])
      for (int c = n0 + (int)threadIdx.x; c < n1; c += blockDim.x) out[(size_t)a * width + c] = 0.f;
}


// ============================================================== gate/up
//
// Work unit = two 8-row blocks of the live experts' gate and up matrices
// (mma rows g and g + 8), full K = H split over the 4 warps of a CTA slot
// (NS = H / 512 steps of 128 codes each); the slot's warps meet at a named
// barrier and the slot sums the quarters in a fixed order and applies the
// SwiGLU. Blocks go round-robin over the CTAs (block b to CTA b mod G), so
// every SM streams the same bytes to within one 8-row block; with one token
// any two of a CTA's blocks form a unit, with several tokens a unit is the
// two halves of one 16-row tile (one expert: one set of token columns).

struct GuRegs {
  uint4 g0, g1, u0, u1;
  uint32_t sg, su;
};

constexpr int kSeg = 4;                    // K split across the warps of a slot
constexpr int kSlots = kWarps / kSeg;      // units per CTA round

RNX_DEVICE void bar_named(int id, int count) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1) mma_gate_up_kernel(const DecodeMmaArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ PlanS S;
  __shared__ int s_cnt[kMaxE], s_off[kMaxE];
  __shared__ float s_unscale[kMaxCols];
  const int H = p.H, I = p.I, T = p.T, k = p.k, TK = T * k;
  const int XR = H + kPad;                                   // staged row length (f16)
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);          // [T][XR] f16 bits
  float* red = reinterpret_cast<float*>(smem + (((size_t)T * XR * 2 + 15) & ~(size_t)15));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int slot = warp / kSeg, seg = warp % kSeg;
  const int NS = H / 512;

  // x first (the tokens as B columns: f16 of x times the token's power of
  // two, in passes of kXq 16-byte chunks per thread), before the wait: x is
  // the call's input, and max |x_t| comes from the launch two back (the
  // router), which had completed when the previous launch passed its own
  // wait, before this one could start. The plan, from the previous launch,
  // is read after the wait.
  constexpr int kXq = 4;
  const int NXC = T * (H / 8);
  float xup[kMaxCols];
#pragma unroll
  for (int tk = 0; tk < kMaxCols; ++tk) {
    float un = 1.f;
    xup[tk] = 1.f;
    if (tk < T) prescale15(__uint_as_float(p.xmax[tk]), xup[tk], un);
    if (threadIdx.x == 0 && tk < T) s_unscale[tk] = un;
  }
  for (int c0 = 0; c0 < NXC; c0 += kThreads * kXq) {
    uint4 xv[kXq];
#pragma unroll
    for (int j = 0; j < kXq; ++j) {
      const int cc = c0 + threadIdx.x + kThreads * j;
      if (cc < NXC) xv[j] = ldg_ordered(p.x + (size_t)(cc / (H / 8)) * H + 8 * (cc % (H / 8)));
    }
#pragma unroll
    for (int j = 0; j < kXq; ++j) {
      const int cc = c0 + threadIdx.x + kThreads * j;
      if (cc < NXC) {
        const int tk = cc / (H / 8), q = cc - tk * (H / 8);
        float up = xup[0];
#pragma unroll
        for (int z = 1; z < kMaxCols; ++z)
          if (z == tk) up = xup[z];
        const uint32_t w4[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
        uint32_t o[4];
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const float2 f = bf16x2_to_f32x2(w4[z]);
          __half2 h2 = __floats2half2_rn(f.x * up, f.y * up);
          o[z] = *reinterpret_cast<uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(xs + (size_t)tk * XR + 8 * q) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  pdl_wait();
  pdl_trigger();
  load_plan(p, S, s_cnt, s_off);
  load_scales(S, p.gate.tensor_scale, p.up.tensor_scale, S);
  const int BPE = I / 8, NB = S.n_live * BPE, G = gridDim.x;
  // this CTA's blocks: blockIdx + G j for j < nb; unit i = blocks (2i, 2i + 1)
  // of that list (one token), or tile blockIdx + G i = blocks (2 tile, 2 tile
  // + 1) (several tokens)
  const bool one = T == 1;
  const int c = blockIdx.x;
  const int nb = c < NB ? (NB - 1 - c) / G + 1 : 0;
  const int NTl = NB / 2, ntl = c < NTl ? (NTl - 1 - c) / G + 1 : 0;
  const int NU = one ? (nb + 1) / 2 : ntl;
  // this slot's units: slot + kSlots rho
  const int R = slot < NU ? (NU - 1 - slot) / kSlots + 1 : 0;
  const int Q = R * NS;
  auto unit_blocks = [&](int rho, int& ba, int& bb) {
    const int i = slot + kSlots * rho;
    if (one) {
      ba = c + G * (2 * i);
      bb = 2 * i + 1 < nb ? c + G * (2 * i + 1) : -1;
    } else {
      ba = 2 * (c + G * i);
      bb = ba + 1;
    }
  };

  // Weight ring load cursor: round lr, step ls, lane byte offsets of its two rows
  // (32-bit: a bank's codes are below 4 GB).
  int lr = 0, ls = 0;
  uint32_t oca = 0, ocb = 0, osa = 0, osb = 0;
  auto unit_offsets = [&](int rho) {
    int ba, bb;
    unit_blocks(rho, ba, bb);
    if (bb < 0) bb = ba;                   // a lone block: its twin rows read again, not written
    const int ua = ba / BPE, ub = bb / BPE;
    const uint32_t ra = (uint32_t)S.e[ua] * (uint32_t)I + 8 * (ba - ua * BPE) + g;
    const uint32_t rb = (uint32_t)S.e[ub] * (uint32_t)I + 8 * (bb - ub * BPE) + g;
    oca = ra * (uint32_t)(H / 2) + seg * (H / 8) + 16 * t;
    ocb = rb * (uint32_t)(H / 2) + seg * (H / 8) + 16 * t;
    osa = ra * (uint32_t)(H / 16) + seg * (H / 64) + 2 * t;
    osb = rb * (uint32_t)(H / 16) + seg * (H / 64) + 2 * t;
  };
  auto load = [&](GuRegs& r) {
    const uint32_t d = 64 * ls, e8 = 8 * ls;
    r.g0 = ldg_ring(p.gate.codes + (oca + d));
    r.g1 = ldg_ring(p.gate.codes + (ocb + d));
    r.u0 = ldg_ring(p.up.codes + (oca + d));
    r.u1 = ldg_ring(p.up.codes + (ocb + d));
    r.sg = ldg_ring_u16(p.gate.scales + (osa + e8)) | (ldg_ring_u16(p.gate.scales + (osb + e8)) << 16);
    r.su = ldg_ring_u16(p.up.scales + (osa + e8)) | (ldg_ring_u16(p.up.scales + (osb + e8)) << 16);
    if (++ls == NS) {
      ls = 0;
      if (++lr < R) unit_offsets(lr);
    }
  };
  GuRegs ring[kDepthGU];

  // the weight ring goes out once x is staged (issued earlier, its requests
  // would hold up the staging's own loads in the memory queues), and after
  // the barrier: a warp whose ring loads stall on a full memory queue holds
  // up no other warp
  __syncthreads();
  if (R > 0) unit_offsets(0);
#pragma unroll
  for (int j = 0; j < kDepthGU; ++j)
    if (j < Q) load(ring[j]);

  // compute cursor: round cr, step cs
  int cr = 0, cs = 0, cba = 0, cbb = -1;
  const uint16_t* brow = xs;
  auto unit_setup = [&](int rho) {
    unit_blocks(rho, cba, cbb);
    const int u = cba / BPE;                // several tokens: both blocks belong to expert u
    const int n = max(S.n[u], 1), col = g < n ? g : 0;
    const int tok = S.sorted[S.off[u] + col] / k;
    brow = xs + (size_t)tok * XR + seg * (H / 4) + 32 * t;
  };
  if (R > 0) unit_setup(0);
  float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
  int buf = 0;

  auto finish_unit = [&]() {
    // the slot's partial sums: red[buf][slot][seg][gate/up][16 rows][8 cols]
    float* rs = red + ((size_t)(buf * kSlots + slot) * kSeg + seg) * 256;
    *reinterpret_cast<float2*>(rs + 8 * g + 2 * t) = make_float2(ag[0], ag[1]);
    *reinterpret_cast<float2*>(rs + 8 * (g + 8) + 2 * t) = make_float2(ag[2], ag[3]);
    *reinterpret_cast<float2*>(rs + 128 + 8 * g + 2 * t) = make_float2(au[0], au[1]);
    *reinterpret_cast<float2*>(rs + 128 + 8 * (g + 8) + 2 * t) = make_float2(au[2], au[3]);
    bar_named(1 + slot, kSeg * kWarp);
    const int i = seg * kWarp + lane, row = i >> 3, col = i & 7;     // 16 rows x 8 columns
    const int blk = row < 8 ? cba : cbb;
    if (blk >= 0) {
      const int u = blk / BPE;
      if (col < S.n[u]) {
        const float* r0 = red + (size_t)(buf * kSlots + slot) * kSeg * 256;
        float gs = 0.f, us = 0.f;
#pragma unroll
        for (int q = 0; q < kSeg; ++q) {
          gs += r0[q * 256 + 8 * row + col];
          us += r0[q * 256 + 128 + 8 * row + col];
        }
        const int a = S.sorted[S.off[u] + col];
        const float un = s_unscale[a / k];
        p.h[(size_t)a * I + 8 * (blk - u * BPE) + (row & 7)] =
            clamped_swiglu(gs * un * S.tsa[u], us * un * S.tsb[u], p.limit);
      }
    }
    buf ^= 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) ag[q] = au[q] = 0.f;
  };

  for (int q0 = 0; q0 < Q; q0 += kDepthGU) {
#pragma unroll
    for (int j = 0; j < kDepthGU; ++j) {
      if (q0 + j < Q) {
        const uint4* bp = reinterpret_cast<const uint4*>(brow + 128 * cs);
        const uint4 b[4] = {bp[0], bp[1], bp[2], bp[3]};
        step_mma(ag, ring[j].g0, ring[j].g1, ring[j].sg, b);
        step_mma(au, ring[j].u0, ring[j].u1, ring[j].su, b);
        if (q0 + j + kDepthGU < Q) load(ring[j]);
        if (++cs == NS) {
          cs = 0;
          finish_unit();
          if (++cr < R) unit_setup(cr);
        }
      }
    }
  }
  zero_dead_rows(S, TK, I, p.h);
}

// h rows of the live assignments as B columns, f16 of h times the row's
// power of two: a fixed one from the clamp's bound on |h| when the limit is
// finite (s_up / s_sc set by the caller), else from each row's maximum (a
// first pass; one shared atomic per warp and row: with I a multiple of 128 a
// warp's 32 float4 lie in one row). Loads go out kHq at a time per thread.
// All threads call it; a barrier of the caller's then publishes hs.
RNX_DEVICE void stage_h(const DecodeMmaArgs& p, const PlanS& S, uint16_t* hs, uint32_t* s_max, float* s_up,
                        float* s_sc, float wa, bool fixed) {
  const int I = p.I, TK = p.T * p.k, HR = I + kPad, lane = threadIdx.x & 31;
  constexpr int kHq = 4;
  const int Q4 = I / 4, NH = TK * Q4;                      // NH % 32 == 0: warp-uniform bounds
  __syncthreads();
  if (!fixed) {
    for (int c0 = 0; c0 < NH; c0 += kThreads * kHq) {
      float4 v[kHq];
#pragma unroll
      for (int j = 0; j < kHq; ++j) {
        const int c = c0 + threadIdx.x + kThreads * j, a = c / Q4;
        v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c < NH && S.live_asg[a]) v[j] = ldg_f4_ordered(p.h + (size_t)a * I + 4 * (c - a * Q4));
      }
#pragma unroll
      for (int j = 0; j < kHq; ++j) {
        const int c = c0 + threadIdx.x + kThreads * j;
        if (c < NH) {
          const float m = warp_max(fmaxf(fmaxf(fabsf(v[j].x), fabsf(v[j].y)), fmaxf(fabsf(v[j].z), fabsf(v[j].w))));
          if (lane == 0) atomicMax(&s_max[c / Q4], __float_as_uint(m));   // non-negative floats order as integers
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < TK) {
      float upx, us;
      prescale15(__uint_as_float(s_max[threadIdx.x]), upx, us);
      s_up[threadIdx.x] = upx;
      s_sc[threadIdx.x] = us * wa;
    }
    __syncthreads();
  }
  for (int c0 = 0; c0 < NH; c0 += kThreads * kHq) {
    float4 v[kHq];
#pragma unroll
    for (int j = 0; j < kHq; ++j) {
      const int c = c0 + threadIdx.x + kThreads * j, a = c / Q4;
      v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < NH && S.live_asg[a]) v[j] = ldg_f4_ordered(p.h + (size_t)a * I + 4 * (c - a * Q4));
    }
#pragma unroll
    for (int j = 0; j < kHq; ++j) {
      const int c = c0 + threadIdx.x + kThreads * j;
      if (c < NH) {
        const int a = c / Q4, q = c - a * Q4;
        const float upx = s_up[a];
        __half2 h0 = __floats2half2_rn(v[j].x * upx, v[j].y * upx), h1 = __floats2half2_rn(v[j].z * upx, v[j].w * upx);
        *reinterpret_cast<uint2*>(hs + (size_t)a * HR + 4 * q) =
            make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
      }
    }
  }
}

// ============================================================== down
//
// Item = a 16-row tile of one live expert's down matrix against the expert's
// h rows, full K = I in NSD = I / 128 steps; tile tau goes to warp
// blockIdx + G w of round tau / (G * 16), so consecutive tiles land on
// different SMs.

struct DnRegs {
  uint4 c0, c1;
  uint32_t sc;
};

__global__ void __launch_bounds__(kThreads, 1) mma_down_kernel(const DecodeMmaArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ PlanS S;
  __shared__ int s_cnt[kMaxE], s_off[kMaxE];
  __shared__ float s_sc[kMaxAsg], s_up[kMaxAsg];
  __shared__ uint32_t s_max[kMaxAsg];
  const int H = p.H, I = p.I, T = p.T, k = p.k, TK = T * k;
  const int HR = I + kPad;
  uint16_t* hs = reinterpret_cast<uint16_t*>(smem);           // [TK][HR] f16 bits
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int NSD = I / 128;

  // The plan and the routing weights come from two launches back, complete
  // when this grid starts: the plan and the tensor scales before the wait for
  // h; after it h is staged, then the weight ring goes out (issued earlier,
  // its requests would hold up the staging's own loads in the memory queues).
  load_plan(p, S, s_cnt, s_off);
  load_scales(S, p.down.tensor_scale, nullptr, S);
  const int TPE = H / 16, NT = S.n_live * TPE, G = gridDim.x, GW = G * kWarps;
  const int tile0 = blockIdx.x + G * warp;
  const int R = tile0 < NT ? (NT - 1 - tile0) / GW + 1 : 0;
  const int Q = R * NSD;
  float wa = 0.f;
  if (threadIdx.x < TK) wa = p.weights[threadIdx.x];
  if (threadIdx.x < kMaxAsg) s_max[threadIdx.x] = 0u;
  const bool fixed = p.h_up > 0.f;
  if (fixed && threadIdx.x < TK) {
    s_up[threadIdx.x] = p.h_up;
    s_sc[threadIdx.x] = p.h_unscale * wa;
  }

  int lr = 0, ls = 0;
  uint32_t oc = 0, os = 0;
  auto tile_offsets = [&](int rho) {
    const int tau = tile0 + GW * rho;
    const int u = tau / TPE, rb = tau - u * TPE;
    const uint32_t row = (uint32_t)S.e[u] * (uint32_t)H + 16 * rb + g;
    oc = row * (uint32_t)(I / 2) + 16 * t;
    os = row * (uint32_t)(I / 16) + 2 * t;
  };
  auto load = [&](DnRegs& r) {
    const uint32_t c = oc + 64 * ls, sofs = os + 8 * ls;
    r.c0 = ldg_ring(p.down.codes + c);
    r.c1 = ldg_ring(p.down.codes + (c + 4 * I));
    r.sc = ldg_ring_u16(p.down.scales + sofs) | (ldg_ring_u16(p.down.scales + (sofs + I / 2)) << 16);
    if (++ls == NSD) {
      ls = 0;
      if (++lr < R) tile_offsets(lr);
    }
  };
  DnRegs ring[kDepthD];
  pdl_wait();                // h comes from the previous launch
  pdl_trigger();

  stage_h(p, S, hs, s_max, s_up, s_sc, wa, fixed);
  __syncthreads();
  if (R > 0) tile_offsets(0);
#pragma unroll
  for (int j = 0; j < kDepthD; ++j)
    if (j < Q) load(ring[j]);

  int cr = 0, cs = 0, cu = 0, crb = 0;
  const uint16_t* brow = hs;
  auto tile_setup = [&](int rho) {
    const int tau = tile0 + GW * rho;
    cu = tau / TPE;
    crb = tau - cu * TPE;
    const int n = max(S.n[cu], 1), col = g < n ? g : 0;
    brow = hs + (size_t)S.sorted[S.off[cu] + col] * HR + 32 * t;
  };
  if (R > 0) tile_setup(0);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  auto finish_item = [&]() {
    // lane (g, t) holds columns 2t, 2t + 1 of rows g, g + 8
    const int n = S.n[cu];
    const size_t row = 16 * (size_t)crb;
    const float ts = S.tsa[cu];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int col = 2 * t + h2;
      if (col < n) {
        const int a = S.sorted[S.off[cu] + col];
        const float sc = s_sc[a] * ts;
        p.r[(size_t)a * H + row + g] = acc[h2] * sc;
        p.r[(size_t)a * H + row + g + 8] = acc[2 + h2] * sc;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = 0.f;
  };

  for (int q0 = 0; q0 < Q; q0 += kDepthD) {
#pragma unroll
    for (int j = 0; j < kDepthD; ++j) {
      if (q0 + j < Q) {
        const uint4* bp = reinterpret_cast<const uint4*>(brow + 128 * cs);
        const uint4 b[4] = {bp[0], bp[1], bp[2], bp[3]};
        step_mma(acc, ring[j].c0, ring[j].c1, ring[j].sc, b);
        if (q0 + j + kDepthD < Q) load(ring[j]);
        if (++cs == NSD) {
          cs = 0;
          finish_item();
          if (++cr < R) tile_setup(cr);
        }
      }
    }
  }
  zero_dead_rows(S, TK, H, p.r);
}

// Down with bulk copies (one token's worth of assignments, I up to 1024):
// a tile's 16 rows of codes are contiguous in the bank (8 I bytes), and so
// are their scales (I bytes), so each warp pulls its tile into its own
// shared-memory stage with two bulk copies (the TMA engine, no load slots of
// the SM held) issued before the wait for h, and multiplies from there.
// Every wait on a copy is bounded: when it runs out the status word gets the
// timeout bit and the warp waits (bounded again) for the copy before it
// leaves.

__global__ void __launch_bounds__(kThreads, 1) mma_down_bulk_kernel(const DecodeMmaArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ PlanS S;
  __shared__ int s_cnt[kMaxE], s_off[kMaxE];
  __shared__ float s_sc[kMaxAsg], s_up[kMaxAsg];
  __shared__ uint32_t s_max[kMaxAsg];
  __shared__ __align__(8) uint64_t s_bar[kWarps];
  const int H = p.H, I = p.I, T = p.T, k = p.k, TK = T * k;
  const int HR = I + kPad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int NSD = I / 128;
  const uint32_t SB = 9u * (uint32_t)I;                       // stage bytes: 8 I of codes, I of scales
  uint8_t* stage = smem + (size_t)warp * SB;
  uint16_t* hs = reinterpret_cast<uint16_t*>(smem + (size_t)kWarps * SB);   // [TK][HR] f16 bits
  uint64_t* bar = &s_bar[warp];
  if (lane == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncwarp();

  // The plan and the routing weights come from two launches back, complete
  // when this grid starts: the plan, the tensor scales and this warp's first
  // tile before the wait for h.
  load_plan(p, S, s_cnt, s_off);
  load_scales(S, p.down.tensor_scale, nullptr, S);
  const int TPE = H / 16, NT = S.n_live * TPE, G = gridDim.x, GW = G * kWarps;
  const int tile0 = blockIdx.x + G * warp;
  const int R = tile0 < NT ? (NT - 1 - tile0) / GW + 1 : 0;
  auto issue = [&](int rho) {                 // lane 0: tile rho of this warp into the stage
    const int tau = tile0 + GW * rho;
    const int u = tau / TPE, rb = tau - u * TPE;
    const size_t row0 = (size_t)S.e[u] * H + 16 * rb;
    mbar_arrive_expect_tx(bar, SB);
    bulk_g2s(stage, p.down.codes + row0 * (I / 2), 8u * (uint32_t)I, bar);
    bulk_g2s(stage + 8 * I, p.down.scales + row0 * (I / 16), (uint32_t)I, bar);
  };
  if (R > 0 && lane == 0) issue(0);
  float wa = 0.f;
  if (threadIdx.x < TK) wa = p.weights[threadIdx.x];
  if (threadIdx.x < kMaxAsg) s_max[threadIdx.x] = 0u;
  const bool fixed = p.h_up > 0.f;
  if (fixed && threadIdx.x < TK) {
    s_up[threadIdx.x] = p.h_up;
    s_sc[threadIdx.x] = p.h_unscale * wa;
  }

  pdl_wait();                // h comes from the previous launch
  pdl_trigger();
  __syncthreads();
  stage_h(p, S, hs, s_max, s_up, s_sc, wa, fixed);
  __syncthreads();

  for (int rho = 0; rho < R; ++rho) {
    if (!mbar_wait(bar, (uint32_t)(rho & 1), p.wait_limit_ns)) {
      if (lane == 0) set_status(p.status, kDevErrTimeout);
      mbar_wait(bar, (uint32_t)(rho & 1), p.wait_limit_ns);   // the copy's own end, bounded again
      break;
    }
    const int tau = tile0 + GW * rho;
    const int cu = tau / TPE, crb = tau - cu * TPE;
    const int n = S.n[cu], col0 = g < max(n, 1) ? g : 0;
    const uint16_t* brow = hs + (size_t)S.sorted[S.off[cu] + col0] * HR + 32 * t;
    const uint8_t* r0 = stage + g * (I / 2) + 16 * t;
    const uint8_t* r1 = r0 + 8 * (I / 2);
    const uint8_t* s0 = stage + 8 * I + g * (I / 16) + 2 * t;
    const uint8_t* s1 = s0 + 8 * (I / 16);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int st = 0; st < NSD; ++st) {
      const uint4 q0 = *reinterpret_cast<const uint4*>(r0 + 64 * st);
      const uint4 q1 = *reinterpret_cast<const uint4*>(r1 + 64 * st);
      const uint32_t sc = (uint32_t)*reinterpret_cast<const uint16_t*>(s0 + 8 * st) |
                          ((uint32_t)*reinterpret_cast<const uint16_t*>(s1 + 8 * st) << 16);
      const uint4* bp = reinterpret_cast<const uint4*>(brow + 128 * st);
      const uint4 b[4] = {bp[0], bp[1], bp[2], bp[3]};
      step_mma(acc, q0, q1, sc, b);
    }
    // lane (g, t) holds columns 2t, 2t + 1 of rows g, g + 8
    const size_t row = 16 * (size_t)crb;
    const float ts = S.tsa[cu];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int col = 2 * t + h2;
      if (col < n) {
        const int a = S.sorted[S.off[cu] + col];
        const float sc = s_sc[a] * ts;
        p.r[(size_t)a * H + row + g] = acc[h2] * sc;
        p.r[(size_t)a * H + row + g + 8] = acc[2 + h2] * sc;
      }
    }
    if (rho + 1 < R) {
      __syncwarp();                          // every lane done with the stage
      fence_proxy_async_smem();
      if (lane == 0) issue(rho + 1);
    }
  }
  zero_dead_rows(S, TK, H, p.r);
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

size_t gate_up_smem(int T, int H) {
  return (((size_t)T * (H + kPad) * 2 + 15) & ~(size_t)15) + (size_t)2 * kSlots * kSeg * 256 * sizeof(float);
}
size_t down_smem(int T, int k, int I) { return (size_t)T * k * (I + kPad) * 2; }
size_t down_bulk_smem(int T, int k, int I) { return (size_t)kWarps * 9 * I + down_smem(T, k, I); }
constexpr size_t kBulkSmemBudget = 200 * 1024;   // with the static shared memory, under 227 KB

constexpr size_t kSmemBudget = 200 * 1024;

}  // namespace


bool decode_mma_supported(int T, int H, int I, int E, int k) {
  if (T < 1 || T > kMaxCols || H % 1024 || H > 8192 || I % 128 || I > 2048 || k < 1 || k > 16 || E < 1 ||
      E > kMaxE || T * k > kMaxAsg)
    return false;
  if (gate_up_smem(T, H) > kSmemBudget || down_smem(T, k, I) > kSmemBudget) return false;
  return (long long)E * H * I / 2 < (1ll << 32);               // 32-bit byte offsets into a bank
}

cudaError_t launch_decode_mma_gate_up(const DecodeMmaArgs& a, cudaStream_t st) {
  if (!decode_mma_supported(a.T, a.H, a.I, a.E, a.k)) return cudaErrorInvalidValue;
  if (!aligned16(a.gate.codes) || !aligned16(a.up.codes) || ((uintptr_t)a.gate.scales & 1u) ||
      ((uintptr_t)a.up.scales & 1u) || !aligned16(a.x) || ((uintptr_t)a.h & 3u))
    return cudaErrorInvalidValue;
  const size_t smem = gate_up_smem(a.T, a.H);
  cudaError_t e = cudaFuncSetAttribute(mma_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(mma_gate_up_kernel, dim3(sm_count()), dim3(kThreads), smem, st, a);
}

cudaError_t launch_decode_mma_down(const DecodeMmaArgs& a, cudaStream_t st) {
  if (!decode_mma_supported(a.T, a.H, a.I, a.E, a.k)) return cudaErrorInvalidValue;
  if (!aligned16(a.down.codes) || ((uintptr_t)a.down.scales & 1u) || !aligned16(a.h) || ((uintptr_t)a.r & 3u))
    return cudaErrorInvalidValue;
  const size_t smem = down_smem(a.T, a.k, a.I);
  cudaError_t e = cudaFuncSetAttribute(mma_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // |h| = |silu(min(g, L))| |clamp(u, -L, L)| <= max(L, 0.28) L (silu(z) <= z
  // for z >= 0 and |silu(z)| < 0.279 for z < 0): with a finite limit one power
  // of two puts every h row under 2^15 in f16
  DecodeMmaArgs b = a;
  b.h_up = 0.f;
  b.h_unscale = 0.f;
  const double bound = std::max((double)a.limit, 0.28) * (double)a.limit;
  if (std::isfinite(bound) && bound > 0.0 && bound < 1e30) {
    int ex = 0;
    std::frexp(bound, &ex);
    b.h_up = (float)std::ldexp(1.0, 15 - ex);
    b.h_unscale = (float)std::ldexp(1.0, ex - 15);
  }
  b.wait_limit_ns = b.wait_limit_ns ? b.wait_limit_ns : kWaitLimitNs;
  if (down_bulk_smem(a.T, a.k, a.I) <= kBulkSmemBudget && aligned16(a.down.scales)) {
    const size_t bs = down_bulk_smem(a.T, a.k, a.I);
    e = cudaFuncSetAttribute(mma_down_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bs);
    if (e != cudaSuccess) return e;
    return launch_pdl(mma_down_bulk_kernel, dim3(sm_count()), dim3(kThreads), bs, st, b);
  }
  return launch_pdl(mma_down_kernel, dim3(sm_count()), dim3(kThreads), smem, st, b);
}

}  // namespace rnx
