// Single-token decode of the routed MoE site in three launches chained by
// programmatic dependent launch (glm5next_mlp module docs, "The stack this
// layer runs"; Constants / W4A16_GEMV_MODULE: at decode every routed-expert
// projection is M = 1, so the step is a stream over the touched experts'
// bytes):
//
//   K1  router logits (fp32 gate.weight . x) + sigmoid top-k by the last
//       router CTA to finish, and, in the same grid, the BF16 shared expert's
//       gate/up with its clamped SwiGLU (h_shared, fp32);
//   K2  the routed experts' NVFP4 gate/up with the clamped SwiGLU (h, fp32),
//       streamed through a ring of bulk copies (TMA engine) in shared memory
//       by one producer warp per CTA, one CTA per SM; the producer warp
//       finally asks L2 for the slice of down weights that K3's CTA of the
//       same index will read;
//   K3  each CTA owns a block of output rows: the routed NVFP4 down rows of
//       every chosen expert and the shared expert's BF16 down rows for that
//       block, all loaded at once by bulk copies issued before it waits for
//       K2, then moe_combine on the spot: y = bf16(sum_j w_j o_j + shared),
//       j in rank order, fp32 throughout (the combine happens before any
//       reduce: section "Why one all-reduce covers BOTH EP and TP").
//
// Arithmetic: NVFP4 codes are decoded to f16 with the hardware cvt; the
// activation (x, or h) is scaled by a power of two per row into f16 (a bf16
// x is exact there, an fp32 h keeps 11 significant bits); every
// product code * activation is exact and accumulated in fp32 by the
// mixed-precision fma (f16 inputs, fp32 accumulator); each 16-element block
// sum is scaled by its E4M3 scale in fp32.

#include "common.cuh"
#include "kernels.h"
#include "gemv_common.cuh"
#include "tma.cuh"
#include "topk.cuh"

namespace rnx {

namespace {

// Self-checks of the data-dependent accesses (built with -DRNX_DEVICE_CHECKS):
// a failed check ORs the bounds bit and the check's id (bits 8..15) into the
// status word and skips the access.
#ifdef RNX_DEVICE_CHECKS
#define RNX_DCHECK(cond, id, status) (((cond)) ? true : (set_status((status), kDevErrBounds | ((uint32_t)(id) << 8)), false))
#else
#define RNX_DCHECK(cond, id, status) true
#endif
RNX_DEVICE bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

RNX_DEVICE void named_bar_sync(int id, int nthreads) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory"); }

// The token's live assignments (expert inside the local range, id valid), in
// assignment order: from ids[0..k) (slot j = assignment j), or from a routing
// plan's active list (expert order; first[u] = the assignment). One thread.
// s_live[0] = count, s_live[1 + u] = expert, s_live[1 + kMaxK + u] = assignment.
constexpr int kMaxK = 16;
RNX_DEVICE void build_live(const int32_t* ids, const int32_t* active, const int32_t* first, int k, int E, int lb,
                           int le, uint32_t* status, bool report, int* s_live) {
  int n = 0;
  if (ids) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[j];
      if (e < 0 || e >= E) {
        if (report) set_status(status, kDevErrBounds);
        continue;
      }
      if (e < lb || e >= le) continue;
      s_live[1 + n] = e;
      s_live[1 + kMaxK + n] = j;
      ++n;
    }
  } else {
    n = min(active[0], kMaxK);
    for (int u = 0; u < n; ++u) {
      s_live[1 + u] = active[1 + u];
      s_live[1 + kMaxK + u] = first[u];
    }
  }
  s_live[0] = n;
}

// Balanced split of H output rows over G CTAs: CTA c owns [row_begin(c), row_begin(c + 1)).
RNX_DEVICE __host__ int row_begin(int c, int H, int G) { return (int)(((long long)c * H) / G); }

// ============================================================== K1
constexpr int kK1Threads = 256;
constexpr int kK1MaxQ = 16;        // router: H / 512 float4 per thread (H <= 8192)
constexpr int kK1SharedRound = 8;  // shared gate/up: uint4 of each row per lane per round

template <int PL>
__global__ void __launch_bounds__(kK1Threads, 2) k1_router_topk_shared(DecodeT1Args p) {
  __shared__ float red[8];
  __shared__ int s_last;
  __shared__ float s_key[1][32 * PL];
  __shared__ float s_sig[1][32 * PL];
  __shared__ __align__(16) uint16_t s_x[8192];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_router = (p.E + 1) / 2;
  const int H = p.H;

  if ((int)blockIdx.x < n_router) {
    // ---------------------------------------------------------- router
    const int half = warp >> 2, th = tid & 127;
    const int e = 2 * blockIdx.x + half;
    const bool e_on = e < p.E;
    const int nq = H >> 2;
    const float4* wrow = reinterpret_cast<const float4*>(p.router_w + (size_t)(e_on ? e : 0) * H);
    float4 w[kK1MaxQ];
#pragma unroll
    for (int i = 0; i < kK1MaxQ; ++i) {
      const int c = th + 128 * i;
      w[i] = (e_on && c < nq) ? __ldg(wrow + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    pdl_wait();
    pdl_trigger();
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kK1MaxQ; ++i) {
      const int c = th + 128 * i;
      if (c < nq) {
        const uint2 xv = *reinterpret_cast<const uint2*>(p.x + 4 * c);
        const float2 a = bf16x2_to_f32x2(xv.x), b = bf16x2_to_f32x2(xv.y);
        acc = fmaf(w[i].x, a.x, acc);
        acc = fmaf(w[i].y, a.y, acc);
        acc = fmaf(w[i].z, b.x, acc);
        acc = fmaf(w[i].w, b.y, acc);
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) red[warp] = acc;
    if (blockIdx.x == 0) {
      // max |x| for the gate/up pass's f16 pre-scale
      float m = 0.f;
      for (int g = tid; g < H / 8; g += kK1Threads) {
        const uint4 v = reinterpret_cast<const uint4*>(p.x)[g];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = bf16x2_to_f32x2(w4[j]);
          m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      m = warp_max(m);
      __syncthreads();
      if (lane == 0) s_key[0][warp] = m;
      __syncthreads();
      if (tid == 0) {
        float mm = 0.f;
        for (int i = 0; i < 8; ++i) mm = fmaxf(mm, s_key[0][i]);
        *p.xmax = __float_as_uint(mm);
      }
    }
    __syncthreads();
    if (tid < 2 && 2 * (int)blockIdx.x + tid < p.E) {
      const float v = ((red[4 * tid] + red[4 * tid + 1]) + red[4 * tid + 2]) + red[4 * tid + 3];
      p.logits[2 * blockIdx.x + tid] = v;
    }
    // the last router CTA to finish runs the selection
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(p.ticket, 1u);
      s_last = prev == (unsigned)(n_router - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // selection keys from the (now complete) logits, then one warp selects
    for (int i = tid; i < p.E; i += kK1Threads) {
      const float l = __ldcg(p.logits + i);
      const float sg = (float)(1.0 / (1.0 + exp(-(double)l)));
      s_sig[0][i] = sg;
      s_key[0][i] = __fadd_rn(sg, p.router_bias[i]);
    }
    __syncthreads();
    if (warp == 0) topk_warp<PL>(s_key[0], s_sig[0], 0, p.E, p.k, p.rsf, p.ids, p.weights);
    __syncthreads();                       // ids visible to the whole CTA
    if (p.plan.counts) {
      // the routing plan of one token (counts, offsets, sorted, inv, tile
      // offsets, active list, first): k distinct ids, O(E k) per CTA
      int id[kMaxK];
      bool valid[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        id[j] = j < p.k ? p.ids[j] : -1;
        valid[j] = j < p.k && id[j] >= 0 && id[j] < p.E;
      }
      for (int e = tid; e <= p.E; e += kK1Threads) {
        int cnt = 0, off = 0, toff = 0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
          if (!valid[j]) continue;
          cnt += id[j] == e;
          off += id[j] < e;
          toff += (id[j] < e && id[j] >= p.lb && id[j] < p.le);
        }
        if (e < p.E) p.plan.counts[e] = cnt;
        p.plan.offsets[e] = off;
        p.plan.tile_offsets[e] = toff;
      }
      if (tid < p.k) {
        const int j = tid;
        if (valid[j]) {
          int pos = 0, lpos = 0;
#pragma unroll
          for (int i = 0; i < kMaxK; ++i) {
            pos += valid[i] && id[i] < id[j];
            lpos += valid[i] && id[i] < id[j] && id[i] >= p.lb && id[i] < p.le;
          }
          p.plan.sorted[pos] = j;
          p.plan.inv[j] = pos;
          if (id[j] >= p.lb && id[j] < p.le) {
            p.plan.active[1 + lpos] = id[j];
            p.plan.first[lpos] = j;
          }
        } else {
          p.plan.inv[j] = -1;
          set_status(p.status, kDevErrBounds);
        }
      }
      if (tid == 0) {
        int nl = 0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) nl += valid[j] && id[j] >= p.lb && id[j] < p.le;
        p.plan.active[0] = nl;
      }
    }
    return;
  }

  // ------------------------------------------------------------ shared gate/up
  // one row pair (gate row, up row) per warp; weights stream in rounds of
  // 8 uint4 per row per lane, the first round issued before the wait
  const int row = ((int)blockIdx.x - n_router) * 8 + warp;
  const bool row_on = row < p.Is;
  const int nu4 = H >> 3;                       // uint4 per row
  const uint4* grow = reinterpret_cast<const uint4*>(p.sh_gate + (size_t)(row_on ? row : 0) * H);
  const uint4* urow = reinterpret_cast<const uint4*>(p.sh_up + (size_t)(row_on ? row : 0) * H);
  uint4 wg[kK1SharedRound], wu[kK1SharedRound];
#pragma unroll
  for (int i = 0; i < kK1SharedRound; ++i) {
    const int c = lane + 32 * i;
    wg[i] = (row_on && c < nu4) ? ldg_stream(grow + c) : make_uint4(0, 0, 0, 0);
    wu[i] = (row_on && c < nu4) ? ldg_stream(urow + c) : make_uint4(0, 0, 0, 0);
  }
  pdl_wait();
  pdl_trigger();
  for (int g = tid; g < nu4; g += kK1Threads) reinterpret_cast<uint4*>(s_x)[g] = reinterpret_cast<const uint4*>(p.x)[g];
  __syncthreads();
  float ag = 0.f, au = 0.f;
  const int rounds = (nu4 + 32 * kK1SharedRound - 1) / (32 * kK1SharedRound);
  for (int rd = 0; rd < rounds; ++rd) {
    if (rd > 0) {
#pragma unroll
      for (int i = 0; i < kK1SharedRound; ++i) {
        const int c = rd * 32 * kK1SharedRound + lane + 32 * i;
        wg[i] = (row_on && c < nu4) ? ldg_stream(grow + c) : make_uint4(0, 0, 0, 0);
        wu[i] = (row_on && c < nu4) ? ldg_stream(urow + c) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int i = 0; i < kK1SharedRound; ++i) {
      const int c = rd * 32 * kK1SharedRound + lane + 32 * i;
      if (c < nu4) {
        const uint4 xv = reinterpret_cast<const uint4*>(s_x)[c];
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const uint32_t gw[4] = {wg[i].x, wg[i].y, wg[i].z, wg[i].w};
        const uint32_t uw[4] = {wu[i].x, wu[i].y, wu[i].z, wu[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 xf = bf16x2_to_f32x2(xw[q]);
          const float2 gf = bf16x2_to_f32x2(gw[q]);
          const float2 uf = bf16x2_to_f32x2(uw[q]);
          ag = fmaf(gf.x, xf.x, ag);
          ag = fmaf(gf.y, xf.y, ag);
          au = fmaf(uf.x, xf.x, au);
          au = fmaf(uf.y, xf.y, au);
        }
      }
    }
  }
  ag = warp_sum(ag);
  au = warp_sum(au);
  if (lane == 0 && row_on) {
    const float hv = clamped_swiglu(ag, au, p.limit);
    p.h_shared[row] = hv;
  }
}

// ============================================================== K2
constexpr int kGuR = 4;                 // row pairs (gate row + up row) per stage
constexpr int kGuKS = 4;                // K slices
constexpr int kGuRG = 2;                // row groups (kGuR / kGuRG row pairs each)
constexpr int kGuConsumers = kGuKS * kGuRG;
constexpr int kGuThreads = (kGuConsumers + 1) * kWarp;
constexpr int kGuMaxStages = 16;
constexpr int kGuSmemBudget = 200 * 1024;

__host__ __device__ inline int gu_stage_bytes(int K) { return kGuR * K + kGuR * K / 8; }

struct GuSmem {
  int stage_bytes, nstages, bar_off, red_off, live_off, ts_off, flag_off, total;
};
__host__ __device__ inline GuSmem gu_smem(int K) {
  GuSmem s;
  s.stage_bytes = gu_stage_bytes(K);
  s.nstages = kGuSmemBudget / s.stage_bytes;
  if (s.nstages > kGuMaxStages) s.nstages = kGuMaxStages;
  s.bar_off = s.nstages * s.stage_bytes;
  s.red_off = s.bar_off + 2 * s.nstages * 8;
  s.live_off = s.red_off + 2 * kGuKS * 2 * kGuR * 4;
  s.ts_off = s.live_off + (1 + 2 * kMaxK) * 4;
  s.flag_off = s.ts_off + 2 * kMaxK * 4;
  s.total = s.flag_off + 16;
  return s;
}

template <int CPL>
__global__ void __launch_bounds__(kGuThreads, 1) k2_gate_up(DecodeT1Args p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const GuSmem L = gu_smem(p.H);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + L.nstages;
  float* red = reinterpret_cast<float*>(smem + L.red_off);          // [2][KS][2R]
  int* s_live = reinterpret_cast<int*>(smem + L.live_off);
  float* s_ts = reinterpret_cast<float*>(smem + L.ts_off);           // [2][kMaxK] gate, up tensor scales
  // iteration at which the consumers stop (set by a consumer whose wait ran
  // out before it reaches that iteration's barrier; read after the barrier,
  // so every consumer breaks at the same iteration)
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L.flag_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.H, I = p.I, NS = L.nstages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGuConsumers);
    }
    fence_barrier_init();
    *s_abort = 0x7fffffff;
  }
  pdl_wait();              // ids (or the plan) and the x max come from earlier launches
  pdl_trigger();
  if (threadIdx.x == 0)
    build_live(p.ids, p.active, p.first, p.k, p.E, p.lb, p.le, p.status, blockIdx.x == 0, s_live);
  __syncthreads();
  const int n_live = s_live[0];
  // the live experts' tensor scales, read once (the per-item epilogue would
  // otherwise wait on a global load every item)
  if (threadIdx.x < n_live) {
    s_ts[threadIdx.x] = p.gate.tensor_scale[s_live[1 + threadIdx.x]];
    s_ts[kMaxK + threadIdx.x] = p.up.tensor_scale[s_live[1 + threadIdx.x]];
  }
  __syncthreads();
  const int NB = I / kGuR;
  const int N = n_live * NB;
  const int G = gridDim.x, c0 = blockIdx.x;
  const int n_mine = c0 < N ? (N - 1 - c0) / G + 1 : 0;
  const int half_codes = kGuR * K / 2, scales_bytes = kGuR * K / 16;

  if (warp == kGuConsumers) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      for (int m = 0; m < n_mine; ++m) {
        const int i = c0 + m * G;
        const int u = i / NB, rb = i - u * NB;
        const int e = s_live[1 + u];
        const int s = m % NS;
        if (m >= NS && !mbar_wait(&empty[s], ((uint32_t)(m / NS) & 1u) ^ 1u)) {
          set_status(p.status, kDevErrTimeout);   // consumers then run out on the stage it never fills
          break;
        }
        uint8_t* st = smem + (size_t)s * L.stage_bytes;
        const size_t row0 = (size_t)e * I + (size_t)rb * kGuR;
        if (!RNX_DCHECK(e >= 0 && e < p.E && row0 + kGuR <= (size_t)p.E * I, 10, p.status)) break;
        if (!RNX_DCHECK(al16(st) && al16(p.gate.codes + row0 * (K / 2)) && al16(p.gate.scales + row0 * (K / 16)) &&
                            half_codes % 16 == 0 && scales_bytes % 16 == 0 &&
                            (size_t)(s + 1) * L.stage_bytes <= (size_t)L.bar_off,
                        11, p.status))
          break;
        mbar_arrive_expect_tx(&full[s], (uint32_t)L.stage_bytes);
        bulk_g2s(st, p.gate.codes + row0 * (K / 2), half_codes, &full[s]);
        bulk_g2s(st + half_codes, p.up.codes + row0 * (K / 2), half_codes, &full[s]);
        bulk_g2s(st + 2 * half_codes, p.gate.scales + row0 * (K / 16), scales_bytes, &full[s]);
        bulk_g2s(st + 2 * half_codes + scales_bytes, p.up.scales + row0 * (K / 16), scales_bytes, &full[s]);
      }
    }
    __syncwarp();
    // the down pass's CTA of this index reads these rows next: the producer
    // warp asks L2 for them (plain prefetches, one per 128-byte line) while
    // the consumers compute the last stages
    if (p.l2_prefetch) {
      const int n0 = row_begin(c0, p.H, G), n1 = row_begin(c0 + 1, p.H, G);
      const size_t cb = (size_t)(n1 - n0) * (I / 2), sb = (size_t)(n1 - n0) * (I / 16);
      for (int u = 0; u < n_live; ++u) {
        const size_t e = (size_t)s_live[1 + u];
        const uint8_t* c = p.down.codes + (e * p.H + n0) * (I / 2);
        const uint8_t* sc = p.down.scales + (e * p.H + n0) * (I / 16);
        for (size_t o = 128 * (size_t)lane; o < cb; o += 128 * 32) prefetch_l2(c + o);
        for (size_t o = 128 * (size_t)lane; o < sb; o += 128 * 32) prefetch_l2(sc + o);
      }
      if (p.sh_down) {
        const uint8_t* sd = reinterpret_cast<const uint8_t*>(p.sh_down + (size_t)n0 * p.Is);
        const size_t db = (size_t)(n1 - n0) * p.Is * 2;
        for (size_t o = 128 * (size_t)lane; o < db; o += 128 * 32) prefetch_l2(sd + o);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int ks = warp % kGuKS, rg = warp / kGuKS;
  const int CS = (K / 32) / kGuKS;         // chunks per K slice
  float up, unscale;
  prescale15(__uint_as_float(*p.xmax), up, unscale);
  uint32_t xr[CPL][16];
#pragma unroll
  for (int i = 0; i < CPL; ++i) act_chunk_bf16(p.x, ks * CS + lane + 32 * i, lane + 32 * i < CS, up, xr[i]);
  constexpr int RPW = kGuR / kGuRG;        // row pairs per warp

  for (int m = 0; m < n_mine; ++m) {
    const int i = c0 + m * G;
    const int u = i / NB, rb = i - u * NB;
    const int s = m % NS;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(m / NS) & 1u));
    float acc[2 * RPW];
#pragma unroll
    for (int r = 0; r < 2 * RPW; ++r) acc[r] = 0.f;
    if (ok) {
      const uint8_t* st = smem + (size_t)s * L.stage_bytes;
#pragma unroll
      for (int ci = 0; ci < CPL; ++ci) {
        const int cl = lane + 32 * ci;
        if (cl < CS) {
          const int c = ks * CS + cl;
#pragma unroll
          for (int r = 0; r < 2 * RPW; ++r) {
            const int bank = r / RPW, rr = rg * RPW + (r % RPW);
            const uint4 q = *reinterpret_cast<const uint4*>(st + bank * half_codes + rr * (K / 2) + 16 * c);
            const uint16_t sc =
                *reinterpret_cast<const uint16_t*>(st + 2 * half_codes + bank * scales_bytes + rr * (K / 16) + 2 * c);
            acc[r] = chunk_dot_f32(q, sc, xr[ci], acc[r]);
          }
        }
      }
    } else if (lane == 0) {
      set_status(p.status, kDevErrTimeout);
      atomicMin(const_cast<int*>(s_abort), m);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    const float tot = warp_reduce_rows<2 * RPW>(acc);       // lane 8 r holds slot r
    float* rb_red = red + (m & 1) * (kGuKS * 2 * kGuR);
    if ((lane & (32 / (2 * RPW) - 1)) == 0) {
      const int r = lane / (32 / (2 * RPW));
      const int bank = r / RPW, rr = rg * RPW + (r % RPW);
      rb_red[ks * 2 * kGuR + bank * kGuR + rr] = tot;
    }
    named_bar_sync(1, kGuConsumers * kWarp);
    if (*s_abort <= m) break;
    if (threadIdx.x < kGuR) {
      const int rr = threadIdx.x;
      const int e = s_live[1 + u], a = s_live[1 + kMaxK + u];
      float g = 0.f, uu = 0.f;
#pragma unroll
      for (int k2 = 0; k2 < kGuKS; ++k2) {
        g += rb_red[k2 * 2 * kGuR + rr];
        uu += rb_red[k2 * 2 * kGuR + kGuR + rr];
      }
      g *= unscale * s_ts[u];
      uu *= unscale * s_ts[kMaxK + u];
      const float hv = clamped_swiglu(g, uu, p.limit);
      if (RNX_DCHECK(a >= 0 && a < p.k && rb * kGuR + rr < I && e >= 0 && e < p.E, 13, p.status))
        p.h[(size_t)a * I + rb * kGuR + rr] = hv;
    }
  }
}

// ============================================================== K3
constexpr int kDnWarps = 16;
constexpr int kDnThreads = kDnWarps * kWarp;
constexpr int kDnRowBatch = 8;

struct DnSmem {
  int nr, seg_codes, seg_scales, codes_off, scales_off, shared_off, bar_off, rs_off, sh_off, live_off, flag_off, total;
};
// Shared-memory plan of one K3 CTA: nr rows of k routed segments (codes,
// scales) and of the shared expert's down rows, one mbarrier per segment.
__host__ __device__ inline DnSmem dn_smem(int H, int I, int Is, int k, int G) {
  DnSmem s;
  s.nr = (H + G - 1) / G;
  s.seg_codes = (s.nr * (I / 2) + 15) / 16 * 16;
  s.seg_scales = (s.nr * (I / 16) + 15) / 16 * 16;
  s.codes_off = 0;
  s.scales_off = s.codes_off + k * s.seg_codes;
  s.shared_off = s.scales_off + k * s.seg_scales;
  s.bar_off = (s.shared_off + s.nr * Is * 2 + 15) / 16 * 16;
  s.rs_off = s.bar_off + (k + 1) * 8;
  s.sh_off = s.rs_off + k * s.nr * 4;
  s.live_off = s.sh_off + s.nr * 4;
  s.flag_off = s.live_off + (1 + 2 * kMaxK) * 4;
  s.total = s.flag_off + 16;
  return s;
}

template <int CPL>
__global__ void __launch_bounds__(kDnThreads, 1) k3_down_combine(DecodeT1Args p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int G = gridDim.x, c0 = blockIdx.x;
  const int H = p.H, I = p.I, k = p.k;
  const bool with_shared = p.sh_down != nullptr;
  const int Is = with_shared ? p.Is : 0;
  const DnSmem L = dn_smem(H, I, Is, k, G);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  float* rs = reinterpret_cast<float*>(smem + L.rs_off);         // [k][nr] weighted routed rows
  float* sh = reinterpret_cast<float*>(smem + L.sh_off);         // [nr] shared rows
  int* s_live = reinterpret_cast<int*>(smem + L.live_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = row_begin(c0, H, G), n1 = row_begin(c0 + 1, H, G), nrows = n1 - n0;

  // The ids come from two launches back, complete when this grid starts: the
  // weight loads go out before the wait for h. Codes and the shared rows by
  // bulk copies (one mbarrier per segment); the E4M3 scales (a ninth of the
  // bytes, rows of I/16 bytes that need not be 16-byte aligned) by plain
  // 4-byte loads of all threads.
  if (threadIdx.x == 0) {
    build_live(p.ids, p.active, p.first, k, p.E, p.lb, p.le, p.status, false, s_live);
    for (int s = 0; s <= k; ++s) mbar_init(&bar[s], 1);
    fence_barrier_init();
    const int n_live = s_live[0];
    if (nrows > 0) {
      for (int u = 0; u < n_live; ++u) {
        const size_t e = (size_t)s_live[1 + u];
        const uint32_t cb = (uint32_t)(nrows * (I / 2));
        if (!RNX_DCHECK(e < (size_t)p.E && nrows <= L.nr && cb <= (uint32_t)L.seg_codes && cb % 16 == 0 &&
                            al16(smem + L.codes_off + u * L.seg_codes) && al16(p.down.codes + (e * H + n0) * (I / 2)),
                        20, p.status))
          continue;
        mbar_arrive_expect_tx(&bar[u], cb);
        bulk_g2s(smem + L.codes_off + u * L.seg_codes, p.down.codes + (e * H + n0) * (I / 2), cb, &bar[u]);
      }
      if (with_shared && RNX_DCHECK(al16(smem + L.shared_off) && al16(p.sh_down + (size_t)n0 * Is) &&
                                        (L.shared_off + nrows * Is * 2) <= L.bar_off,
                                    21, p.status)) {
        const uint32_t b = (uint32_t)(nrows * Is * 2);
        mbar_arrive_expect_tx(&bar[k], b);
        bulk_g2s(smem + L.shared_off, p.sh_down + (size_t)n0 * Is, b, &bar[k]);
      }
    }
  }
  for (int i = threadIdx.x; i < k * L.nr; i += kDnThreads) rs[i] = 0.f;
  __syncthreads();
  {
    const int n_live = s_live[0];
    const int words = nrows * (I / 16) / 4;          // 4-byte words of one segment's scales
    for (int i = threadIdx.x; i < n_live * words; i += kDnThreads) {
      const int u = i / words, wd = i - u * words;
      const size_t e = (size_t)s_live[1 + u];
      const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p.down.scales + (e * H + n0) * (I / 16)) + wd);
      reinterpret_cast<uint32_t*>(smem + L.scales_off + u * L.seg_scales)[wd] = v;
    }
  }
  __syncthreads();
  pdl_wait();                // h comes from the previous launch
  pdl_trigger();
  const int n_live = s_live[0];

  // routed rows: task t = (live assignment u, part of the row block); the
  // parts split each assignment's rows so that every warp has a task
  const int parts = n_live > 0 ? max(1, kDnWarps / n_live) : 1;
  for (int task = warp; task < n_live * parts; task += kDnWarps) {
    const int u = task / parts, part = task - u * parts;
    const int ra = part * nrows / parts, rz = (part + 1) * nrows / parts;
    const bool ok = nrows == 0 || __all_sync(0xffffffffu, mbar_wait(&bar[u], 0));
    if (!ok) {
      if (lane == 0) set_status(p.status, kDevErrTimeout);
      continue;
    }
    const int e = s_live[1 + u], a = s_live[1 + kMaxK + u];
    if (!RNX_DCHECK(e >= 0 && e < p.E && a >= 0 && a < k && rz <= L.nr, 22, p.status)) continue;
    // the warp holds the whole h row (chunk lane + 32 i per lane): its max
    // |h| sets the f16 pre-scale
    const float* hrow = p.h + (size_t)a * I;
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int c = lane + 32 * i;
      if (c < I / 32) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(hrow + 32 * c + 4 * q);
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
      }
    }
    mx = warp_max(mx);
    float upx, unscale;
    prescale15(mx, upx, unscale);
    uint32_t xr[CPL][16];
#pragma unroll
    for (int i = 0; i < CPL; ++i) act_chunk_f32(hrow, lane + 32 * i, lane + 32 * i < I / 32, upx, xr[i]);
    const float scale = unscale * p.down.tensor_scale[e] * p.weights[a];
    const uint8_t* codes = smem + L.codes_off + u * L.seg_codes;
    const uint8_t* scales = smem + L.scales_off + u * L.seg_scales;
    for (int r0 = ra; r0 < rz; r0 += kDnRowBatch) {
      float acc[kDnRowBatch];
#pragma unroll
      for (int rr = 0; rr < kDnRowBatch; ++rr) {
        acc[rr] = 0.f;
        const int r = r0 + rr;
        if (r < rz) {
#pragma unroll
          for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < I / 32) {
              const uint4 q = *reinterpret_cast<const uint4*>(codes + r * (I / 2) + 16 * c);
              const uint16_t sc = *reinterpret_cast<const uint16_t*>(scales + r * (I / 16) + 2 * c);
              acc[rr] = chunk_dot_f32(q, sc, xr[i], acc[rr]);
            }
          }
        }
      }
      const float tot = warp_reduce_rows<kDnRowBatch>(acc);   // lane 4 r holds row r0 + r
      const int r = r0 + (lane >> 2);
      if ((lane & 3) == 0 && r < rz) {
        const float v = tot * scale;
        rs[a * L.nr + r] = v;
        if (p.r) p.r[(size_t)a * H + n0 + r] = v;
      }
    }
  }

  // shared expert's down rows: fp32 FMAs of the bf16 weights and h_shared
  if (with_shared && nrows > 0) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar[k], 0));
    if (!ok) {
      if (lane == 0) set_status(p.status, kDevErrTimeout);
    } else {
      const int nu4 = Is / 8;
      for (int r = warp; r < nrows; r += kDnWarps) {
        const uint4* wrow = reinterpret_cast<const uint4*>(smem + L.shared_off + (size_t)r * Is * 2);
        float acc = 0.f;
        for (int c = lane; c < nu4; c += 32) {
          const uint4 wv = wrow[c];
          const float4 h0 = *reinterpret_cast<const float4*>(p.h_shared + 8 * c);
          const float4 h1 = *reinterpret_cast<const float4*>(p.h_shared + 8 * c + 4);
          const float2 w0 = bf16x2_to_f32x2(wv.x), w1 = bf16x2_to_f32x2(wv.y);
          const float2 w2 = bf16x2_to_f32x2(wv.z), w3 = bf16x2_to_f32x2(wv.w);
          acc = fmaf(w0.x, h0.x, acc);
          acc = fmaf(w0.y, h0.y, acc);
          acc = fmaf(w1.x, h0.z, acc);
          acc = fmaf(w1.y, h0.w, acc);
          acc = fmaf(w2.x, h1.x, acc);
          acc = fmaf(w2.y, h1.y, acc);
          acc = fmaf(w3.x, h1.z, acc);
          acc = fmaf(w3.y, h1.w, acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) sh[r] = acc;
      }
    }
  }
  __syncthreads();

  // rows of assignments that are not live (remote experts, dropped ids) are zero
  if (p.r) {
    for (int a = 0; a < k; ++a) {
      bool live = false;
      for (int u = 0; u < n_live; ++u) live |= s_live[1 + kMaxK + u] == a;
      if (!live)
        for (int r = threadIdx.x; r < nrows; r += kDnThreads) p.r[(size_t)a * H + n0 + r] = 0.f;
    }
  }
  // moe_combine: the k routed rows in rank order, then the shared row, fp32,
  // one rounding to bf16
  if (p.y) {
    for (int r = threadIdx.x; r < nrows; r += kDnThreads) {
      float acc = 0.f;
      for (int j = 0; j < k; ++j) acc += rs[j * L.nr + r];
      if (with_shared) {
        acc += sh[r];
        if (p.shared_out) p.shared_out[n0 + r] = sh[r];
      }
      p.y[n0 + r] = f32_to_bf16_bits(acc);
    }
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

template <typename Kern>
cudaError_t set_smem(Kern kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

bool decode_t1_supported(int H, int I, int Is, int E, int k) {
  const int G = sm_count();
  if (H % 256 || H > 8192 || I % 64 || I > 2048 || k < 1 || k > kMaxK || E < 1 || E > 1024) return false;
  if (Is < 0 || Is % 8 || Is > 8192) return false;
  if (I % kGuR) return false;
  if (gu_smem(H).nstages < 2 || gu_smem(H).total > 227 * 1024) return false;
  if (dn_smem(H, I, Is, k, G).total > 227 * 1024) return false;
  return true;
}

cudaError_t launch_decode_t1_gate_up(const DecodeT1Args& p, cudaStream_t st) {
  const GuSmem L = gu_smem(p.H);
  const int CPL = ((p.H / 32) / kGuKS + 31) / 32;
  auto kern = CPL <= 1 ? k2_gate_up<1> : k2_gate_up<2>;
  cudaError_t e = set_smem(kern, L.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(sm_count()), dim3(kGuThreads), (size_t)L.total, st, p);
}

cudaError_t launch_decode_t1_down(const DecodeT1Args& p, cudaStream_t st) {
  const int G = sm_count();
  const DnSmem L = dn_smem(p.H, p.I, p.sh_down ? p.Is : 0, p.k, G);
  const int CPL = (p.I / 32 + 31) / 32;
  auto kern = CPL <= 1 ? k3_down_combine<1> : k3_down_combine<2>;
  cudaError_t e = set_smem(kern, L.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(G), dim3(kDnThreads), (size_t)L.total, st, p);
}

cudaError_t launch_decode_t1_router(const DecodeT1Args& p, cudaStream_t st) {
  const int grid = (p.E + 1) / 2 + (p.Is + 7) / 8;
  if (p.E <= 32 * 4) return launch_pdl(k1_router_topk_shared<4>, dim3(grid), dim3(kK1Threads), 0, st, p);
  if (p.E <= 32 * 10) return launch_pdl(k1_router_topk_shared<10>, dim3(grid), dim3(kK1Threads), 0, st, p);
  return launch_pdl(k1_router_topk_shared<32>, dim3(grid), dim3(kK1Threads), 0, st, p);
}

}  // namespace rnx
