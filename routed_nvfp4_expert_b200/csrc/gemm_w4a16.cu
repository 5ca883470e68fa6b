// Prefill expert projections in the pages' own numerics: a grouped W4A16 GEMM
// (glm5next_mlp module docs, forward_prefill_gemm: the routed experts'
// prefill runs "through the shared tensor-core grouped W4A16 GEMM"): NVFP4
// weights, 16-bit activations, on tcgen05 kind::f16 with fp32 accumulators in
// TMEM.
//
// The weights stay NVFP4 in HBM. Per K slice of 64 elements the producer warp
// brings the tile's packed codes (32 bytes per weight row) and its scale atoms
// into a raw ring by TMA; four dequantisation warps turn them into the f16
// B tile of the MMA ring, each element = E2M1 code x E4M3 block scale, which is
// exact in f16 (6 significant bits, magnitudes 2^-10 .. 2688), written in the
// 128-byte swizzled K-major layout the MMA reads. The tensor scale is applied
// in the epilogue. Activations are f16 too (kind::f16 takes one type for both
// operands): x rows scaled by a power of two per row into [2^14, 2^15) by the
// gather that builds the padded tile order (exact for bf16 x), h as the
// gate/up epilogue's f16 output (11 significant bits, saturating).
//
// Tile = 128 padded rows x 256 weight rows (GATE_UP: 128 gate + the same 128
// up rows; DOWN: 256 output features), one CTA per tile, persistent CTAs over
// the (m-tile, n-tile) list with the n-tiles innermost, two 256-column
// accumulators alternating between tiles.
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer, warp 2 = TMEM
// allocator, warps 4-7 = epilogue (one per TMEM lane quadrant), warps 8-15 =
// dequantisation (the part that bounds a tile's time). Every wait
// is bounded; a timeout sets the device status word and winds the CTA down.
// No TMA load uses cluster multicast.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tensor_map.h"

namespace rnx {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kStepK = 64;                      // f16 elements per stage: 128 bytes per row
constexpr int kStages = 3;                      // MMA ring (A + dequantised B)
constexpr int kRawStages = 4;                   // raw ring (codes + scale atoms)
constexpr int kABytes = kTileM * 128;           // 16 KB
constexpr int kBBytes = kTileN * 128;           // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;  // 48 KB
constexpr int kRawCodeBytes = kTileN * 32;      // 256 rows x 64 codes
constexpr int kRawSfBytes = 1024;               // 2 scale atoms (256 rows x 4 blocks)
constexpr int kRawBytes = kRawCodeBytes + kRawSfBytes;
constexpr int kSmemBytes = kStages * kStageBytes + kRawStages * kRawBytes + 1024;
constexpr int kFirstEpiWarp = 4;
constexpr int kEpiWarps = 4;                    // one per TMEM lane quadrant, both column halves
constexpr int kFirstDqWarp = 8;
constexpr int kDqWarps = 8;                     // the dequantisation bounds the launch: most warps go there
constexpr int kThreads = (kFirstDqWarp + kDqWarps) * 32;   // 512
constexpr uint32_t kTmemCols = 512;                        // two 256-column accumulators
constexpr int kMaxExperts = 1024;

// Instruction descriptor of kind::f16 with f16 A/B, fp32 accumulate, K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct W4Params {
  CUtensorMap tma_a;       // A f16 [P, K]; box 64 x 128 rows, SW128
  CUtensorMap tma_c0;      // gate (or down) codes [E*rows, K/2] bytes; box 32 B x 128 rows
  CUtensorMap tma_c1;      // up codes (GATE_UP)
  CUtensorMap tma_sf;      // scale atoms as [2 n_atoms, 256]; box 256 x 4 (2 atoms)
  void* out;               // GATE_UP: h f16 [P, I]; DOWN: rows fp32 [P, H]
  const float* row_scale;  // [P] A row unscale (nullable: 1)
  const float* ts0;        // [E]
  const float* ts1;        // [E]
  const int32_t* tile_offsets;   // [E+1], 256-row tiles
  const int32_t* tile_rows;      // [P]
  const float* weights;          // [A]
  uint32_t* status;
  int E, K, out_cols, bank_rows;
  float limit;
  int sparse;                    // see W4a16GemmArgs::sparse
};

// Sparse mode (a decode batch: a few tokens per expert): a 128-row half tile
// whose first row is padding holds nothing but padding, since an expert's
// real rows come first in its 256-row tiles. Every role skips such tiles
// alike, before touching any ring or accumulator counter.
RNX_DEVICE bool skip_half(const W4Params& p, int mt) {
  return p.sparse && __ldg(p.tile_rows + (size_t)mt * kTileM) < 0;
}

RNX_DEVICE int find_expert(const int32_t* s_toff, int E, int t256) {
  int lo = 0, hi = E;                 // largest e with s_toff[e] <= t256
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_toff[mid] <= t256) lo = mid; else hi = mid;
  }
  return lo;
}

// Byte offset of scale block b (0..3) of atom row m inside a 512-byte atom.
RNX_DEVICE int atom_byte(int m, int b) { return (m & 31) * 16 + ((m & 127) >> 5) * 4 + b; }

RNX_DEVICE uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

RNX_DEVICE uint32_t pack_f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1) w4a16_gemm_kernel(const __grid_constant__ W4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* raw = smem + (size_t)kStages * kStageBytes;
  __shared__ __align__(8) uint64_t a_full[kStages], b_full[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t raw_full[kRawStages], raw_empty[kRawStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int abort_flag;
  __shared__ int s_toff[kMaxExperts + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int n_ksteps = p.K / kStepK;
  const int n_ntiles = GATE_UP ? p.out_cols / 128 : p.out_cols / kTileN;

  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_toff[i] = p.tile_offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&b_full[s], kDqWarps);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kDqWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_mtiles = 2 * s_toff[E];
  const int n_tiles = n_mtiles * n_ntiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // it_r / it_a count the raw and A stages issued so far
    int it_r = 0, it_a = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;   // n-tiles innermost
      if (skip_half(p, mt)) continue;
      const int e = find_expert(s_toff, E, mt >> 1);
      // the tile's scale atoms: GATE_UP interleaved atoms 2 nt, 2 nt + 1 (64
      // gate + 64 up rows each); DOWN atoms 2 nt, 2 nt + 1 of 128 rows
      const int atom0 = GATE_UP ? e * (p.bank_rows / 64) + 2 * nt : e * (p.bank_rows / 128) + 2 * nt;
      const int KB = p.K / 64;
      for (int ks = 0; ks < n_ksteps; ++ks) {
        const int rs = it_r % kRawStages;
        if (__any_sync(0xffffffffu, !mbar_wait_poll(&raw_empty[rs], ((uint32_t)(it_r / kRawStages) & 1u) ^ 1u) ||
                                        abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* r = raw + (size_t)rs * kRawBytes;
          mbar_arrive_expect_tx(&raw_full[rs], (uint32_t)kRawBytes);
          if (GATE_UP) {
            tma_load_2d(r, &p.tma_c0, ks * 32, e * p.bank_rows + nt * 128, &raw_full[rs]);
            tma_load_2d(r + kRawCodeBytes / 2, &p.tma_c1, ks * 32, e * p.bank_rows + nt * 128, &raw_full[rs]);
          } else {
            tma_load_2d(r, &p.tma_c0, ks * 32, e * p.bank_rows + nt * kTileN, &raw_full[rs]);
            tma_load_2d(r + kRawCodeBytes / 2, &p.tma_c0, ks * 32, e * p.bank_rows + nt * kTileN + 128, &raw_full[rs]);
          }
          // atoms atom0, atom0 + 1 of K block ks: rows 2 (j KB + ks), +1 of the [2 n_atoms, 256] view
          tma_load_2d(r + kRawCodeBytes, &p.tma_sf, 0, 2 * (atom0 * KB + ks), &raw_full[rs]);
          tma_load_2d(r + kRawCodeBytes + 512, &p.tma_sf, 0, 2 * ((atom0 + 1) * KB + ks), &raw_full[rs]);
        }
        __syncwarp();
        ++it_r;
        const int s = it_a % kStages;
        if (__any_sync(0xffffffffu, !mbar_wait_poll(&empty_bar[s], ((uint32_t)(it_a / kStages) & 1u) ^ 1u) ||
                                        abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&a_full[s], (uint32_t)kABytes);
          tma_load_2d(smem + (size_t)s * kStageBytes, &p.tma_a, ks * kStepK, mt * kTileM, &a_full[s]);
        }
        __syncwarp();
        ++it_a;
      }
    }
    if (!ok && lane == 0) {
      set_status(p.status, kDevErrTimeout);
      abort_flag = 1;
    }
    // drain: every copy issued must have landed before the CTA may exit (a
    // stage reused later had landed before its reuse)
    for (int j = max(0, it_r - kRawStages); j < it_r; ++j)
      if (!mbar_wait(&raw_full[j % kRawStages], (uint32_t)(j / kRawStages) & 1u) && lane == 0)
        set_status(p.status, kDevErrTimeout);
    for (int j = max(0, it_a - kStages); j < it_a; ++j)
      if (!mbar_wait(&a_full[j % kStages], (uint32_t)(j / kStages) & 1u) && lane == 0)
        set_status(p.status, kDevErrTimeout);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_f16(kTileM, kTileN);
    const uint32_t s0 = smem_u32(smem);
    const uint64_t dA0 = sdesc_k_sw128(s0), dB0 = sdesc_k_sw128(s0 + kABytes);
    int it = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc) {
      if (skip_half(p, tile / n_ntiles)) {
        --tc;   // skipped tiles take no accumulator turn
        continue;
      }
      const int b = tc & 1;
      const uint32_t use = (uint32_t)(tc >> 1);
      if (__any_sync(0xffffffffu, !mbar_wait_poll(&acc_empty[b], (use & 1u) ^ 1u))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + 256u * b;
      for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (__any_sync(0xffffffffu, !mbar_wait_poll(&a_full[s], ph) || !mbar_wait_poll(&b_full[s], ph) || abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t so = (uint64_t)((s * kStageBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)   // K = 16 per MMA: 32 bytes of each row
            mma_bf16(acc, dA0 + so + 2 * kb, dB0 + so + 2 * kb, idesc, (ks > 0 || kb > 0) ? 1u : 0u);
          mma_commit(&empty_bar[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&acc_full[b]);
      __syncwarp();
    }
    if (!ok && lane == 0) {
      set_status(p.status, kDevErrTimeout);
      abort_flag = 1;
    }
    if (elect_one()) mma_commit(&mma_done);
    __syncwarp();
    if (!mbar_wait(&mma_done, 0) && lane == 0) set_status(p.status, kDevErrTimeout);
  } else if (warp >= kFirstDqWarp) {
    // ------------------------------------------------------------ dequantisation
    // Thread t of the dequantisation warps owns B rows t, t + 32 kDqWarps, ...
    // of every stage.
    const int t = threadIdx.x - kFirstDqWarp * 32;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      if (skip_half(p, tile / n_ntiles)) continue;
      for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
        const int s = it % kStages, rs = it % kRawStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u, rph = (uint32_t)(it / kRawStages) & 1u;
        if (__any_sync(0xffffffffu, !mbar_wait_poll(&raw_full[rs], rph) || !mbar_wait_poll(&empty_bar[s], ph ^ 1u) ||
                                        abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* r = raw + (size_t)rs * kRawBytes;
        uint8_t* sB = smem + (size_t)s * kStageBytes + kABytes;
#pragma unroll
        for (int row = t; row < kTileN; row += kDqWarps * 32) {
          // scale atom of this B row (see the producer): GATE_UP rows 0..127
          // gate, 128..255 up, 64 of each per interleaved atom
          int j, m;
          if (GATE_UP) {
            const int g = row & 127;
            j = g >> 6;
            m = (row < 128 ? 0 : 64) + (g & 63);
          } else {
            j = row >> 7;
            m = row & 127;
          }
          const uint32_t sc4 = *reinterpret_cast<const uint32_t*>(r + kRawCodeBytes + j * 512 + atom_byte(m, 0));
          uint32_t s01, s23;   // block scales as f16x2 pairs
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s01) : "h"((uint16_t)(sc4 & 0xFFFF)));
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s23) : "h"((uint16_t)(sc4 >> 16)));
          const uint32_t sb[4] = {(s01 & 0xFFFFu) * 0x10001u, (s01 >> 16) * 0x10001u, (s23 & 0xFFFFu) * 0x10001u,
                                  (s23 >> 16) * 0x10001u};
          const uint4 q0 = *reinterpret_cast<const uint4*>(r + row * 32);
          const uint4 q1 = *reinterpret_cast<const uint4*>(r + row * 32 + 16);
          const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {      // 16-byte output chunk c = 8 elements, block c / 2
            uint32_t w0, w1, w2, w3;
            e2m1x8_to_f16x2x4(qw[c], w0, w1, w2, w3);
            const uint32_t sv = sb[c >> 1];
            const uint4 o = make_uint4(hmul2_u32(w0, sv), hmul2_u32(w1, sv), hmul2_u32(w2, sv), hmul2_u32(w3, sv));
            *reinterpret_cast<uint4*>(sB + row * 128 + ((c ^ (row & 7)) << 4)) = o;
          }
        }
        fence_proxy_async_smem();          // generic writes visible to the tensor core's reads
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&b_full[s]);
          mbar_arrive(&raw_empty[rs]);
        }
      }
    }
    if (!ok && lane == 0) {
      set_status(p.status, kDevErrTimeout);
      abort_flag = 1;
    }
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      if (skip_half(p, tile / n_ntiles)) {
        --tc;
        continue;
      }
      const int b = tc & 1;
      const uint32_t use = (uint32_t)(tc >> 1);
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
      const int e = find_expert(s_toff, E, mt >> 1);
      const int row = mt * kTileM + q * 32 + lane;
      const float rs = p.row_scale ? p.row_scale[row] : 1.f;
      if (__any_sync(0xffffffffu, !mbar_wait_poll(&acc_full[b], use & 1u) || abort_flag)) {
        if (lane == 0) {
          set_status(p.status, kDevErrTimeout);
          abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t tq = tmem + 256u * b + ((uint32_t)(q * 32) << 16);
      // the accumulator in column halves ch and, within each, two passes
      // (fewer live registers); the buffer is released after all of them,
      // the MMAs meanwhile fill the other one
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        if (GATE_UP) {
          const float sg = rs * p.ts0[e], su = rs * p.ts1[e];
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + (size_t)row * p.out_cols +
                                                nt * 128 + 64 * ch);
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t g[32], u[32];
            tmem_ld32(tq + 64 * ch + 32 * hh, g);
            tmem_ld32(tq + 128 + 64 * ch + 32 * hh, u);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int k0 = 8 * c + 2 * i;
                w[i] = pack_f16x2_sat(
                    clamped_swiglu_fast(__uint_as_float(g[k0]) * sg, __uint_as_float(u[k0]) * su, p.limit),
                    clamped_swiglu_fast(__uint_as_float(g[k0 + 1]) * sg, __uint_as_float(u[k0 + 1]) * su, p.limit));
              }
              dst[4 * hh + c] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        } else {
          const int asg = p.tile_rows[row];
          const float sc = asg >= 0 ? rs * p.ts0[e] * p.weights[asg] : 0.f;
          // sparse: row p goes to assignment row tile_rows[p]; padding rows are
          // not written
          const bool keep = !p.sparse || asg >= 0;
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) +
                                                  (size_t)(p.sparse ? max(asg, 0) : row) * p.out_cols +
                                                  nt * kTileN + 128 * ch);
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[64];
            tmem_ld32(tq + 128 * ch + 64 * hh, v);
            tmem_ld32(tq + 128 * ch + 64 * hh + 32, v + 32);
            tmem_ld_wait();
            if (keep) {
#pragma unroll
              for (int c = 0; c < 16; ++c)
                dst[16 * hh + c] = make_float4(__uint_as_float(v[4 * c]) * sc, __uint_as_float(v[4 * c + 1]) * sc,
                                               __uint_as_float(v[4 * c + 2]) * sc, __uint_as_float(v[4 * c + 3]) * sc);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Padded tile rows of x as f16: row p holds token tile_rows[p] / k scaled by
// the power of two that brings its max |x| into [2^14, 2^15) (exact for bf16),
// unscale[p] the inverse; padding rows (and rows past the used tiles) zero.
RNX_DEVICE void gather_row_f16(long long row, const uint16_t* __restrict__ x, int H, int k,
                               const int32_t* __restrict__ tile_rows, uint16_t* __restrict__ xa,
                               float* __restrict__ unscale, int sparse) {
  const int lane = threadIdx.x & 31;
  const int a = tile_rows[row];
  uint4* dst = reinterpret_cast<uint4*>(xa + row * H);
  // sparse: halves holding only padding are skipped by the GEMMs, never read
  if (a < 0 && sparse && tile_rows[row & ~(long long)(kTileM - 1)] < 0) return;
  if (a < 0) {
    for (int g = lane; g < H / 8; g += 32) dst[g] = make_uint4(0, 0, 0, 0);
    if (lane == 0) unscale[row] = 0.f;
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(a / k) * H);
  float m = 0.f;
  for (int g = lane; g < H / 8; g += 32) {
    const uint4 v = src[g];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_f32x2(w[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  m = warp_max(m);
  int ex = 0;
  if (m > 0.f && m <= 3.0e38f) frexpf(m, &ex);
  const float up = ldexpf(1.0f, 15 - ex);
  for (int g = lane; g < H / 8; g += 32) {
    const uint4 v = src[g];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_f32x2(w[j]);
      __half2 h = __floats2half2_rn(f.x * up, f.y * up);
      o[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    dst[g] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (lane == 0) unscale[row] = ldexpf(1.0f, ex - 15);
}

// Warps stride over the rows of the tiles in use (rows past them are never
// read); the grid is bounded by the SM count, as the row bound P covers the
// worst routing.
__global__ void __launch_bounds__(256) gather_x_f16_kernel(const uint16_t* __restrict__ x, int H, int k,
                                                           const int32_t* __restrict__ tile_rows,
                                                           const int32_t* __restrict__ used_tiles, long long P,
                                                           uint16_t* __restrict__ xa, float* __restrict__ unscale,
                                                           int sparse) {
  const long long lim = min(P, (long long)*used_tiles * kRowsPerTile);
  for (long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); row < lim; row += (long long)gridDim.x * 8)
    gather_row_f16(row, x, H, k, tile_rows, xa, unscale, sparse);
}

bool f16_map(CUtensorMap* m, const void* base, int K, int64_t rows) {
  return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)rows, kStepK, kTileM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
}

bool code_map32(CUtensorMap* m, const uint8_t* base, int K, int64_t rows) {
  return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)rows, 32, 128,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool atom_map2(CUtensorMap* m, const uint8_t* base, int64_t n_atoms) {
  return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, (uint64_t)(2 * n_atoms), 256, 2,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace

cudaError_t launch_gather_x_f16(const uint16_t* x, int H, int k, const int32_t* tile_rows, const int32_t* used_tiles,
                                int64_t P, uint16_t* xa, float* unscale, cudaStream_t st, bool sparse) {
  if (P <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<int64_t>((P + 7) / 8, 8 * kNumSMs);
  gather_x_f16_kernel<<<grid, 256, 0, st>>>(x, H, k, tile_rows, used_tiles, P, xa, unscale, sparse ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_w4a16_grouped_gemm(const W4a16GemmArgs& a, cudaStream_t st) {
  if (a.E > kMaxExperts || a.P_max % kRowsPerTile || a.K % kStepK) return cudaErrorInvalidValue;
  if (a.P_max == 0) return cudaSuccess;   // no local expert: no rows, no tiles
  if (a.gate_up ? (a.out_cols % 128) : (a.out_cols % kTileN)) return cudaErrorInvalidValue;
  W4Params p;
  memset(&p, 0, sizeof p);
  const bool gu = a.gate_up;
  const int KB = a.K / 64;
  const int64_t brows = (int64_t)a.E * a.bank_rows;
  if (!f16_map(&p.tma_a, a.act, a.K, a.P_max)) return cudaErrorInvalidValue;
  if (!code_map32(&p.tma_c0, a.b0_codes, a.K, brows)) return cudaErrorInvalidValue;
  if (gu && !code_map32(&p.tma_c1, a.b1_codes, a.K, brows)) return cudaErrorInvalidValue;
  if (!atom_map2(&p.tma_sf, a.b_sf, (gu ? 2 * brows : brows) / 128 * KB)) return cudaErrorInvalidValue;
  p.out = a.out;
  p.row_scale = a.row_scale;
  p.ts0 = a.ts0;
  p.ts1 = a.ts1;
  p.tile_offsets = a.tile_offsets;
  p.tile_rows = a.tile_rows;
  p.weights = a.weights;
  p.status = a.status;
  p.E = a.E;
  p.K = a.K;
  p.out_cols = a.out_cols;
  p.bank_rows = a.bank_rows;
  p.limit = a.limit;
  p.sparse = a.sparse ? 1 : 0;
  auto kern = gu ? w4a16_gemm_kernel<true> : w4a16_gemm_kernel<false>;
  static bool attr_done[2] = {false, false};
  if (!attr_done[gu]) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done[gu] = true;
  }
  kern<<<kNumSMs, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace rnx
