// GEMMs on the 5th-generation tensor cores (tcgen05, accumulators in tensor
// memory), one persistent warp-specialised kernel in two flavours:
//
//  FP4: the prefill expert projections, a grouped GEMM with block-scaled FP4
//       (kind::mxf4nvf4, one E4M3 scale per 16 elements on both operands).
//       glm5next_mlp module docs, forward_prefill_gemm: the routed experts'
//       prefill runs as a grouped GEMM over the tokens sorted by expert. Here
//       the activations are NVFP4 as well (W4A4, one fp32 scale per token
//       row), so the whole contraction runs on the block-scaled FP4 path.
//         A: activation rows in the padded tile layout (every expert starts on
//            a 128-row tile): codes [P, K/2], scale atoms, a scale per row
//         B: the expert's weight rows: codes [rows, K/2] canonical, scale
//            atoms prepared once by moe_prepare_weights
//  BF16: the dense FFN and the shared expert at large T (kind::f16 with bf16
//        operands): A = x [M, K], B = weight rows [N, K].
//
//  GATE_UP: tile = 128 rows x (128 gate + 128 up weight rows); the epilogue
//           applies the scales, the clamped SwiGLU, rounds h to bf16 and
//           stores it (FP4: padded row p; BF16: row m).
//  DOWN:    tile = 128 rows x 256 output features; FP4: times the scales and
//           the routing weight, scattered to r[a] of the row's assignment;
//           BF16: stored to y[m].
//
// One persistent CTA per SM walks the (m-tile, n-tile) list. Warp roles:
// warp 0 = TMA producer (4-stage ring of 128-byte K slices: 256 FP4 or 64
// bf16 elements per row), warp 1 = MMA issuer (one thread; FP4 scale atoms go
// to TMEM with tcgen05.cp right before their MMAs), warp 2 = TMEM allocator,
// warps 4-11 = epilogue (warp w owns TMEM lane quadrant w % 4 and one half of
// the accumulator columns; it copies its part to registers and releases the
// accumulator before the SwiGLU / scaling and the stores). BF16 double-buffers
// the accumulator in TMEM; FP4 needs the other half of TMEM for the scales.
// Every wait is bounded: a timeout sets the device status word, every role
// winds down, in-flight copies and MMAs are drained and TMEM is freed before
// the CTA exits. No TMA load uses cluster multicast.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rnx {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 256;          // MMA N (GATE_UP: 128 gate + 128 up)
constexpr int kRowBytes = 128;       // K slice per stage and row: one 128-byte swizzle span
constexpr int kStages = 4;
constexpr int kABytes = kTileM * kRowBytes;          // 16 KB
constexpr int kBBytes = kTileN * kRowBytes;          // 32 KB
constexpr int kSfaBytes = 2048;                      // FP4: 4 scale atoms of A (one per 64-element K block)
constexpr int kSfbBytes = 4096;                      // FP4: 8 scale atoms of B
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 54 KB
constexpr int kSmemBytes = kStages * kStageBytes + 1024;                  // + alignment slack
constexpr int kFirstEpiWarp = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kFirstEpiWarp + kEpiWarps) * 32;   // 384
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxExpertsSmem = 1024;
// TMEM columns. FP4: accumulator [0, 256); per pipeline stage s, 48 scale
// columns at 256 + 48 s (SFA 4 per K block, SFB 8 per K block). A stage's
// scale columns are rewritten only after the MMAs that read them completed
// (the same commit that frees the stage's shared memory). BF16: accumulator
// buffers at columns 0 and 256.
constexpr uint32_t kColSf = 256, kSfColsPerStage = 48;
static_assert(kColSf + kStages * kSfColsPerStage <= kTmemCols, "TMEM columns");

struct GemmParams {
  CUtensorMap tma_a;       // A [rows, K]; box 128 B x 128 rows, SW128
  CUtensorMap tma_b0;      // GATE_UP: gate rows (box 128 rows); DOWN: weight rows (box 256 rows)
  CUtensorMap tma_b1;      // GATE_UP: up rows
  // FP4 only
  const uint8_t* sfa;      // [P/128][K/64][512]
  const uint8_t* sfb0;     // [E][rows/128][K/64][512]
  const uint8_t* sfb1;
  const float* row_scale;  // [P] second-level scale of each A row
  const float* ts0;        // [E]
  const float* ts1;        // [E] (GATE_UP)
  const int32_t* tile_offsets;   // [E+1]
  const int32_t* tile_rows;      // [P]: assignment of each padded row, -1 = padding
  const float* weights;          // [A] (DOWN)
  // both
  uint16_t* out;                 // FP4 GATE_UP: h [P, out_cols]; FP4 DOWN: r [A, out_cols]; BF16: [M, out_cols]
  uint32_t* status;
  int E, K, out_cols, bank_rows;   // bank_rows: rows of one expert in the B bank (FP4)
  int M;                           // BF16: rows of A
  int m_fastest;                   // tile order: 1 = m-tiles innermost (weights stay in L2 across m)
  float limit;
};

RNX_DEVICE int find_expert(const int32_t* s_toff, int E, int mt) {
  int lo = 0, hi = E;                 // largest e with s_toff[e] <= mt
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_toff[mid] <= mt) lo = mid; else hi = mid;
  }
  return lo;
}

template <bool FP4, bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr int kAccBufs = FP4 ? 1 : 2;
  constexpr int kElemsPerStage = FP4 ? 256 : 64;   // K elements in one 128-byte row slice
  constexpr int kElemsPerMma = FP4 ? 64 : 16;      // K of one MMA (32 bytes of each row)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int abort_flag;
  __shared__ int s_toff[FP4 ? kMaxExpertsSmem + 1 : 2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = FP4 ? p.E : 1;
  const int KB = p.K / 64;                          // FP4: 64-element scale blocks (one MMA each)
  const int n_ksteps = (p.K + kElemsPerStage - 1) / kElemsPerStage;
  const int n_ntiles = GATE_UP ? p.out_cols / 128 : p.out_cols / kTileN;

  if (FP4) {
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_toff[i] = p.tile_offsets[i];
  } else if (threadIdx.x == 0) {
    s_toff[0] = 0;
    s_toff[1] = (p.M + kTileM - 1) / kTileM;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
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
  const int n_mtiles = s_toff[E];
  const int n_tiles = n_mtiles * n_ntiles;
  auto tile_coords = [&](int tile, int& mt, int& nt) {
    if (p.m_fastest) {
      nt = tile / n_mtiles;
      mt = tile - nt * n_mtiles;
    } else {
      mt = tile / n_ntiles;
      nt = tile - mt * n_ntiles;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, mt, nt);
        const int e = FP4 ? find_expert(s_toff, E, mt) : 0;
        for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(&empty_bar[s], ph ^ 1u) || abort_flag) {
            set_status(p.status, kDevErrTimeout);
            abort_flag = 1;
            break;
          }
          uint8_t* st = smem + (size_t)s * kStageBytes;
          uint8_t* sA = st;
          uint8_t* sB = st + kABytes;
          const int x = FP4 ? ks * kRowBytes : ks * kElemsPerStage;   // innermost TMA coordinate (elements)
          const int kb0 = ks * 4, kbn = FP4 ? min(4, KB - kb0) : 0;
          mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(kABytes + kBBytes + 3 * kbn * 512));
          tma_load_2d(sA, &p.tma_a, x, mt * kTileM, &full_bar[s]);
          const int brow = e * p.bank_rows + nt * (GATE_UP ? 128 : kTileN);
          if (GATE_UP) {
            tma_load_2d(sB, &p.tma_b0, x, brow, &full_bar[s]);
            tma_load_2d(sB + kBBytes / 2, &p.tma_b1, x, brow, &full_bar[s]);
          } else {
            tma_load_2d(sB, &p.tma_b0, x, brow, &full_bar[s]);
          }
          if (FP4) {
            uint8_t* sSFA = sB + kBBytes;
            uint8_t* sSFB = sSFA + kSfaBytes;
            bulk_g2s_plain(sSFA, p.sfa + ((size_t)mt * KB + kb0) * 512, kbn * 512, &full_bar[s]);
            const size_t rb = (size_t)e * (p.bank_rows / 128);
            if (GATE_UP) {
              bulk_g2s_plain(sSFB, p.sfb0 + ((rb + nt) * KB + kb0) * 512, kbn * 512, &full_bar[s]);
              bulk_g2s_plain(sSFB + 2048, p.sfb1 + ((rb + nt) * KB + kb0) * 512, kbn * 512, &full_bar[s]);
            } else {
              bulk_g2s_plain(sSFB, p.sfb0 + ((rb + 2 * nt) * KB + kb0) * 512, kbn * 512, &full_bar[s]);
              bulk_g2s_plain(sSFB + 2048, p.sfb0 + ((rb + 2 * nt + 1) * KB + kb0) * 512, kbn * 512, &full_bar[s]);
            }
          }
        }
      }
      // drain: every copy issued must have landed before the CTA may exit
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!mbar_wait(&full_bar[j % kStages], (uint32_t)(j / kStages) & 1u)) set_status(p.status, kDevErrTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = FP4 ? idesc_mxf4nvf4(kTileM, kTileN) : idesc_bf16(kTileM, kTileN);
      int it = 0, tc = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x, ++tc) {
        const int b = tc % kAccBufs;
        const uint32_t use = (uint32_t)(tc / kAccBufs);
        // the epilogue must have drained this accumulator buffer's previous tile
        if (!mbar_wait(&acc_empty[b], (use & 1u) ^ 1u)) {
          set_status(p.status, kDevErrTimeout);
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + 256u * b;
        for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(&full_bar[s], ph) || abort_flag) {
            set_status(p.status, kDevErrTimeout);
            abort_flag = 1;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + (size_t)s * kStageBytes;
          const uint32_t aA = smem_u32(st), aB = aA + kABytes;
          const int nmma = min(4, (p.K - ks * kElemsPerStage) / kElemsPerMma);
          if (FP4) {
            const uint32_t aSFA = aB + kBBytes, aSFB = aSFA + kSfaBytes;
            const uint32_t sfa_col = tmem + kColSf + kSfColsPerStage * s, sfb_col = sfa_col + 16;
            for (int kb = 0; kb < nmma; ++kb) {
              tmem_cp_sf(sfa_col + 4 * kb, sdesc_sf_atom(aSFA + kb * 512));
              tmem_cp_sf(sfb_col + 8 * kb, sdesc_sf_atom(aSFB + kb * 512));
              tmem_cp_sf(sfb_col + 8 * kb + 4, sdesc_sf_atom(aSFB + 2048 + kb * 512));
            }
            for (int kb = 0; kb < nmma; ++kb)
              mma_mxf4nvf4(acc, sdesc_k_sw128(aA + 32 * kb), sdesc_k_sw128(aB + 32 * kb), idesc, sfa_col + 4 * kb,
                           sfb_col + 8 * kb, (ks > 0 || kb > 0) ? 1u : 0u);
          } else {
            for (int kb = 0; kb < nmma; ++kb)
              mma_bf16(acc, sdesc_k_sw128(aA + 32 * kb), sdesc_k_sw128(aB + 32 * kb), idesc,
                       (ks > 0 || kb > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[s]);          // the stage is free once these MMAs have read it
        }
        if (abort_flag) break;
        mma_commit(&acc_full[b]);             // the accumulator is final once every MMA is done
      }
      mma_commit(&mma_done);
      if (!mbar_wait(&mma_done, 0)) set_status(p.status, kDevErrTimeout);
    }
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                          // TMEM lane quadrant this warp may access
    const int ch = (warp - kFirstEpiWarp) >> 2;     // column half
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      const int b = tc % kAccBufs;
      const uint32_t use = (uint32_t)(tc / kAccBufs);
      int mt, nt;
      tile_coords(tile, mt, nt);
      const int e = FP4 ? find_expert(s_toff, E, mt) : 0;
      const int prow = mt * kTileM + q * 32 + lane;   // A row = TMEM lane of this thread
      int asg = prow;
      bool valid;
      float rs = 1.f;
      if (FP4) {
        asg = p.tile_rows[prow];
        valid = asg >= 0;
        rs = p.row_scale[prow];
      } else {
        valid = prow < p.M;
      }
      if (!mbar_wait(&acc_full[b], use & 1u) || abort_flag) {
        set_status(p.status, kDevErrTimeout);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tq = tmem + 256u * b + ((uint32_t)(q * 32) << 16);
      if (GATE_UP) {
        const float sg = FP4 ? rs * p.ts0[e] : 1.f, su = FP4 ? rs * p.ts1[e] : 1.f;
        uint32_t g[64], u[64];
        tmem_ld32(tq + 64 * ch, g);
        tmem_ld32(tq + 64 * ch + 32, g + 32);
        tmem_ld32(tq + 128 + 64 * ch, u);
        tmem_ld32(tq + 128 + 64 * ch + 32, u + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        if (FP4 || valid) {   // FP4 padding rows are written too (as zeros)
          uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)prow * p.out_cols + nt * 128 + 64 * ch);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k0 = 8 * c + 2 * i;
              w[i] = pack_bf16x2(
                  clamped_swiglu_fast(__uint_as_float(g[k0]) * sg, __uint_as_float(u[k0]) * su, p.limit),
                  clamped_swiglu_fast(__uint_as_float(g[k0 + 1]) * sg, __uint_as_float(u[k0 + 1]) * su, p.limit));
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      } else {
        const int a = valid ? asg : 0;
        const float sc = FP4 ? (valid ? rs * p.ts0[e] * p.weights[a] : 0.f) : 1.f;
        uint32_t v[128];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld32(tq + 128 * ch + 32 * j, v + 32 * j);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)a * p.out_cols + nt * kTileN + 128 * ch);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = pack_bf16x2(__uint_as_float(v[8 * c + 2 * i]) * sc, __uint_as_float(v[8 * c + 2 * i + 1]) * sc);
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2D tensor [rows, cols] (cols contiguous) of 1-byte (FP4 pairs) or 2-byte
// (bf16) elements; box = 128 bytes x box_rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, bool bf16, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = bf16 ? 2 : 1;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {(cuuint32_t)(kRowBytes / esz), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool FP4, bool GU>
cudaError_t launch(const GemmParams& p, cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t err = cudaFuncSetAttribute(tc_gemm_kernel<FP4, GU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done = true;
  }
  tc_gemm_kernel<FP4, GU><<<kNumSMs, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fp4_grouped_gemm(const Fp4GemmArgs& a, cudaStream_t st) {
  if (a.E > kMaxExpertsSmem) return cudaErrorInvalidValue;
  GemmParams p;
  memset(&p, 0, sizeof p);
  const bool gu = a.gate_up;
  const uint64_t row_bytes = (uint64_t)a.K / 2;
  if (!make_map(&p.tma_a, a.a_codes, false, row_bytes, (uint64_t)a.P_max, 128)) return cudaErrorInvalidValue;
  if (!make_map(&p.tma_b0, a.b0_codes, false, row_bytes, (uint64_t)a.E * a.bank_rows, gu ? 128 : 256))
    return cudaErrorInvalidValue;
  if (gu && !make_map(&p.tma_b1, a.b1_codes, false, row_bytes, (uint64_t)a.E * a.bank_rows, 128))
    return cudaErrorInvalidValue;
  p.sfa = a.a_sf;
  p.sfb0 = a.b0_sf;
  p.sfb1 = a.b1_sf;
  p.row_scale = a.row_scale;
  p.ts0 = a.ts0;
  p.ts1 = a.ts1;
  p.tile_offsets = a.tile_offsets;
  p.tile_rows = a.tile_rows;
  p.weights = a.weights;
  p.out = a.out;
  p.status = a.status;
  p.E = a.E;
  p.K = a.K;
  p.out_cols = a.out_cols;
  p.bank_rows = a.bank_rows;
  p.m_fastest = 0;   // m-tiles of one expert are adjacent: a wave shares few experts' weights
  p.limit = a.limit;
  return gu ? launch<true, true>(p, st) : launch<true, false>(p, st);
}

cudaError_t launch_bf16_gemm(bool gate_up, const uint16_t* a, int M, int K, const uint16_t* b0, const uint16_t* b1,
                             int N, float limit, uint16_t* out, uint32_t* status, cudaStream_t st) {
  GemmParams p;
  memset(&p, 0, sizeof p);
  if (!make_map(&p.tma_a, a, true, (uint64_t)K, (uint64_t)M, 128)) return cudaErrorInvalidValue;
  if (!make_map(&p.tma_b0, b0, true, (uint64_t)K, (uint64_t)N, gate_up ? 128 : 256)) return cudaErrorInvalidValue;
  if (gate_up && !make_map(&p.tma_b1, b1, true, (uint64_t)K, (uint64_t)N, 128)) return cudaErrorInvalidValue;
  p.out = out;
  p.status = status;
  p.E = 1;
  p.K = K;
  p.out_cols = N;
  p.bank_rows = 0;
  p.M = M;
  p.m_fastest = 1;   // weights larger than L2: every weight tile is read once, x stays in L2
  p.limit = limit;
  return gate_up ? launch<false, true>(p, st) : launch<false, false>(p, st);
}

}  // namespace rnx
