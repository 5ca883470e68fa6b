// Prefill expert projections: grouped GEMM on the 5th-generation tensor cores
// with block-scaled FP4 (tcgen05.mma kind::mxf4nvf4, one E4M3 scale per 16
// elements on both operands, fp32 accumulation in tensor memory).
//
// glm5next_mlp module docs, forward_prefill_gemm: the routed experts' prefill
// runs as a grouped GEMM over the tokens sorted by expert. Here the
// activations are NVFP4 as well (W4A4, one fp32 scale per token row), so the
// whole contraction runs on the block-scaled FP4 tensor-core path.
//
//   A: activation rows in expert order, padded so that every expert starts on
//      a 128-row tile (codes [P, K/2], scale atoms, one fp32 scale per row)
//   B: the expert's weight rows (codes [rows, K/2] in canonical layout, scale
//      atoms prepared once by moe_prepare_weights)
//   GATE_UP: tile = 128 rows x (128 gate + 128 up rows); the epilogue applies
//            the two second-level scales, the clamped SwiGLU, rounds h to
//            bf16, stores it [P, I] and publishes max |h| per row
//   DOWN:    tile = 128 rows x 256 output features; the epilogue applies the
//            scales and the routing weight and scatters bf16 rows to r[t, j]
//
// One persistent CTA per SM walks the (m-tile, n-tile) list. Warp roles:
// warp 0 = TMA producer (4-stage ring, 54 KB per stage), warp 1 = MMA issuer
// (one thread; scale atoms go to TMEM with tcgen05.cp right before their
// MMAs), warp 2 = TMEM allocator, warps 4-7 = epilogue (each owns one 32-lane
// quadrant of the accumulator). Every wait is bounded; a timeout sets the
// device status word, every role winds down, in-flight copies and MMAs are
// drained and TMEM is freed before the CTA exits.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rnx {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 256;          // MMA N (GATE_UP: 128 gate + 128 up)
constexpr int kStepK = 256;          // FP4 elements per stage (128 bytes per row)
constexpr int kStages = 4;
constexpr int kABytes = kTileM * kStepK / 2;         // 16 KB
constexpr int kBBytes = kTileN * kStepK / 2;         // 32 KB
constexpr int kSfaBytes = kTileM * kStepK / 16;      // 2 KB: 4 atoms
constexpr int kSfbBytes = kTileN * kStepK / 16;      // 4 KB: 8 atoms
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 54 KB
constexpr int kSmemBytes = kStages * kStageBytes + 1024;                  // + alignment slack
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: accumulator [0, 256); per pipeline stage s, 48 scale columns
// at 256 + 48 s: SFA 4 per K block (16), SFB 8 per K block (32). A stage's
// scale columns are rewritten only after the MMAs that read them completed
// (the same commit that frees the stage's shared memory).
constexpr uint32_t kColAcc = 0, kColSf = 256, kSfColsPerStage = 48;
static_assert(kColSf + kStages * kSfColsPerStage <= kTmemCols, "TMEM columns");

struct Fp4GemmParams {
  CUtensorMap tma_a;       // A codes [P, K/2] bytes, box 128 B x 128 rows, SW128
  CUtensorMap tma_b0;      // GATE_UP: gate codes [E*I, K/2], box 128 rows; DOWN: down [E*H, K/2], box 256 rows
  CUtensorMap tma_b1;      // GATE_UP: up codes
  const uint8_t* sfa;      // [P/128][K/64][512]
  const uint8_t* sfb0;     // [E][rows/128][K/64][512]
  const uint8_t* sfb1;
  const float* row_scale;  // [P] second-level scale of each A row
  const float* ts0;        // [E]
  const float* ts1;        // [E] (GATE_UP)
  const int32_t* tile_offsets;   // [E+1]
  const int32_t* tile_rows;      // [P]: assignment of each padded row, -1 = padding
  const float* weights;          // [A] (DOWN)
  uint16_t* out;                 // GATE_UP: h [P, out_cols]; DOWN: r [A, out_cols]
  uint32_t* status;
  int E, K, out_cols, bank_rows;   // bank_rows: rows of one expert in the B bank (I or H)
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

template <bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1) fp4_grouped_gemm_kernel(const __grid_constant__ Fp4GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int abort_flag;
  __shared__ int s_toff[1025];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int KB = p.K / 64;                          // 64-element K blocks (one MMA each)
  const int n_ksteps = (p.K + kStepK - 1) / kStepK;
  const int n_ntiles = GATE_UP ? p.out_cols / 128 : p.out_cols / kTileN;

  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_toff[i] = p.tile_offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 4);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
        const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
        const int e = find_expert(s_toff, E, mt);
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
          uint8_t* sSFA = sB + kBBytes;
          uint8_t* sSFB = sSFA + kSfaBytes;
          const int kb0 = ks * 4, kbn = min(4, KB - kb0);
          mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(kABytes + kBBytes + 3 * kbn * 512));
          tma_load_2d(sA, &p.tma_a, ks * 128, mt * kTileM, &full_bar[s]);
          if (GATE_UP) {
            tma_load_2d(sB, &p.tma_b0, ks * 128, e * p.bank_rows + nt * 128, &full_bar[s]);
            tma_load_2d(sB + kBBytes / 2, &p.tma_b1, ks * 128, e * p.bank_rows + nt * 128, &full_bar[s]);
          } else {
            tma_load_2d(sB, &p.tma_b0, ks * 128, e * p.bank_rows + nt * kTileN, &full_bar[s]);
          }
          bulk_g2s_plain(sSFA, p.sfa + ((size_t)mt * KB + kb0) * 512, kbn * 512, &full_bar[s]);
          const int rb_per_e = p.bank_rows / 128;
          if (GATE_UP) {
            bulk_g2s_plain(sSFB, p.sfb0 + (((size_t)e * rb_per_e + nt) * KB + kb0) * 512, kbn * 512, &full_bar[s]);
            bulk_g2s_plain(sSFB + 2048, p.sfb1 + (((size_t)e * rb_per_e + nt) * KB + kb0) * 512, kbn * 512,
                           &full_bar[s]);
          } else {
            bulk_g2s_plain(sSFB, p.sfb0 + (((size_t)e * rb_per_e + 2 * nt) * KB + kb0) * 512, kbn * 512, &full_bar[s]);
            bulk_g2s_plain(sSFB + 2048, p.sfb0 + (((size_t)e * rb_per_e + 2 * nt + 1) * KB + kb0) * 512, kbn * 512,
                           &full_bar[s]);
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
      const uint32_t idesc = idesc_mxf4nvf4(kTileM, kTileN);
      int it = 0, tc = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x, ++tc) {
        // the epilogue must have drained the accumulator of the previous tile
        if (!mbar_wait(&acc_empty, ((uint32_t)tc & 1u) ^ 1u)) {
          set_status(p.status, kDevErrTimeout);
          abort_flag = 1;
          break;
        }
        tc_fence_after();
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
          const uint32_t aA = smem_u32(st), aB = aA + kABytes, aSFA = aB + kBBytes, aSFB = aSFA + kSfaBytes;
          const int kbn = min(4, KB - ks * 4);
          const uint32_t sfa_col = tmem + kColSf + kSfColsPerStage * s, sfb_col = sfa_col + 16;
          for (int kb = 0; kb < kbn; ++kb) {
            tmem_cp_sf(sfa_col + 4 * kb, sdesc_sf_atom(aSFA + kb * 512));
            tmem_cp_sf(sfb_col + 8 * kb, sdesc_sf_atom(aSFB + kb * 512));
            tmem_cp_sf(sfb_col + 8 * kb + 4, sdesc_sf_atom(aSFB + 2048 + kb * 512));
          }
          for (int kb = 0; kb < kbn; ++kb) {
            mma_mxf4nvf4(tmem + kColAcc, sdesc_k_sw128(aA + 32 * kb), sdesc_k_sw128(aB + 32 * kb), idesc,
                         sfa_col + 4 * kb, sfb_col + 8 * kb, (ks > 0 || kb > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[s]);          // the stage is free once these MMAs have read it
        }
        if (abort_flag) break;
        mma_commit(&acc_full);                // the accumulator is final once every MMA is done
      }
      mma_commit(&mma_done);
      if (!mbar_wait(&mma_done, 0)) set_status(p.status, kDevErrTimeout);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quadrant
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      if (!mbar_wait(&acc_full, (uint32_t)tc & 1u) || abort_flag) {
        set_status(p.status, kDevErrTimeout);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
      const int e = find_expert(s_toff, E, mt);
      const int prow = mt * kTileM + q * 32 + lane;   // padded A row = TMEM lane of this thread
      const int asg = p.tile_rows[prow];
      const bool valid = asg >= 0;
      const float rs = p.row_scale[prow];
      const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
      if (GATE_UP) {
        const float sg = rs * p.ts0[e], su = rs * p.ts1[e];
        uint16_t* orow = p.out + (size_t)prow * p.out_cols + nt * 128;
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
          uint32_t g[32], u[32];
          tmem_ld32(tq + kColAcc + 32 * j, g);
          tmem_ld32(tq + kColAcc + 128 + 32 * j, u);
          tmem_ld_wait();
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = clamped_swiglu(__uint_as_float(g[2 * i]) * sg, __uint_as_float(u[2 * i]) * su, p.limit);
            const float h1 =
                clamped_swiglu(__uint_as_float(g[2 * i + 1]) * sg, __uint_as_float(u[2 * i + 1]) * su, p.limit);
            packed[i] = pack_bf16x2(h0, h1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * j);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      } else {
        const int a = valid ? asg : 0;
        const float sc = valid ? rs * p.ts0[e] * p.weights[a] : 0.f;
        uint16_t* orow = p.out + (size_t)a * p.out_cols + nt * kTileN;
#pragma unroll 1
        for (int j = 0; j < kTileN / 32; ++j) {
          uint32_t v[32];
          tmem_ld32(tq + kColAcc + 32 * j, v);
          tmem_ld_wait();
          if (valid) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * sc, __uint_as_float(v[2 * i + 1]) * sc);
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * j);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty);
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

// 2D byte tensor [rows, row_bytes] (row_bytes contiguous), box 128 B x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_fp4_grouped_gemm(const Fp4GemmArgs& a, cudaStream_t st) {
  Fp4GemmParams p;
  memset(&p, 0, sizeof p);
  const bool gu = a.gate_up;
  const uint64_t row_bytes = (uint64_t)a.K / 2;
  if (!make_map(&p.tma_a, a.a_codes, row_bytes, (uint64_t)a.P_max, 128)) return cudaErrorInvalidValue;
  if (!make_map(&p.tma_b0, a.b0_codes, row_bytes, (uint64_t)a.E * a.bank_rows, gu ? 128 : 256)) return cudaErrorInvalidValue;
  if (gu && !make_map(&p.tma_b1, a.b1_codes, row_bytes, (uint64_t)a.E * a.bank_rows, 128)) return cudaErrorInvalidValue;
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
  p.limit = a.limit;
  auto kern = gu ? fp4_grouped_gemm_kernel<true> : fp4_grouped_gemm_kernel<false>;
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
