// Prefill expert projections: grouped GEMM with block-scaled FP4 on CTA pairs
// (tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16: one E4M3
// scale per 16 elements on both operands, fp32 accumulation in TMEM).
//
// glm5next_mlp module docs, forward_prefill_gemm: the routed experts' prefill
// runs as a grouped GEMM over the tokens sorted by expert. Here the
// activations are NVFP4 as well (W4A4, one fp32 scale per token row), so the
// whole contraction runs on the block-scaled FP4 tensor-core path.
//
// Tile = 256 rows (one expert segment slice of the padded tile layout, whose
// experts start on 256-row boundaries) x 256 weight rows, K in slices of 256
// FP4 elements (128 bytes per row). A cluster of two CTAs computes it: CTA r
// holds A rows [128 r, 128 r + 128) and B rows [128 r, 128 r + 128) of the
// tile, its own scale atoms of A and all scale atoms of B; the even CTA
// issues the MMAs (M = 256, N = 256, K = 64) and the scale copies for both, so
// every CTA streams half the B bytes a single-CTA 128 x 256 tile would.
//   GATE_UP: 128 intermediate features per tile, their gate and up rows in
//            the order of moe_prepare_weights' interleaved scale atoms: CTA r
//            holds gate rows 64 r .. 64 r + 63 then the same up rows, so the
//            accumulator's columns 128 r .. +63 are gate and +64 .. +127 up
//            of features 64 r .. 64 r + 63; the epilogue applies the scales
//            and the clamped SwiGLU, rounds h to bf16, stores [P, I].
//   DOWN:    256 output features; the epilogue applies the scales and the
//            routing weight and writes fp32 rows [P, H] in the padded tile
//            order (the unpermute is fused into the combine that follows,
//            which sums them in fp32).
//
// Warp roles per CTA: warp 0 = TMA producer (5-stage ring, 38 KB per stage,
// completions counted on the even CTA's barrier), warp 1 = MMA issuer (even
// CTA only, one thread), warp 2 = TMEM allocator (both CTAs), warps 4-11 =
// epilogue (warp w reads TMEM lane quadrant w % 4 and one half of the 256
// accumulator columns, copies them to registers and releases the accumulator
// before the SwiGLU / scaling and the stores). Every wait is bounded; a
// timeout sets the device status word and winds the pair down. No TMA load
// uses cluster multicast (only the MMA completion commit is multicast).

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tensor_map.h"

namespace rnx {

namespace {

constexpr int kPairM = 256;          // rows of one pair tile (128 per CTA)
constexpr int kTileN = 256;          // MMA N
constexpr int kStepK = 256;          // FP4 elements per stage (128 bytes per row)
constexpr int kStages = 4;
constexpr int kABytes = 128 * 128;   // this CTA's A rows x 128 bytes
constexpr int kBBytes = 128 * 128;   // this CTA's half of B
constexpr int kSfaBytes = 2048;      // 4 atoms: this CTA's 128 rows, 4 K blocks
constexpr int kSfbBytes = 4096;      // 8 atoms: all 256 B rows, 4 K blocks
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 38 KB
// epilogue staging: each epilogue warp owns two 32-row x 128-byte boxes in
// the 128-byte swizzled layout of the output tensor map (TMA tensor stores)
constexpr int kEpiBoxBytes = 32 * 128;
constexpr int kEpiStageBytes = 2 * kEpiBoxBytes;                           // per warp
constexpr int kSmemBytes = kStages * kStageBytes + 8 * kEpiStageBytes + 1024;
constexpr uint32_t kTxBytesPair = 2u * kStageBytes;                      // both CTAs' bytes of one stage
constexpr int kFirstEpiWarp = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kFirstEpiWarp + kEpiWarps) * 32;   // 384
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxExperts = 1024;
// TMEM columns: accumulator [0, 256); per stage s, scales at 256 + 48 s (SFA
// 4 columns per K block, SFB 8). A stage's scale columns are rewritten only
// after the MMAs that read them completed (the commit that frees the stage).
constexpr uint32_t kColSf = 256, kSfColsPerStage = 48;
static_assert(kColSf + kStages * kSfColsPerStage <= kTmemCols, "TMEM columns");

struct PairParams {
  CUtensorMap tma_a;       // A codes [P, K/2] bytes, box 128 B x 128 rows, SW128
  CUtensorMap tma_b0;      // gate (or down) codes [E*rows, K/2]; box 128 B x 64 (GATE_UP) or 128 rows
  CUtensorMap tma_b1;      // up codes (GATE_UP), box 128 B x 64 rows
  CUtensorMap tma_sfa;     // A scale atoms viewed as [bytes/256, 256], box 256 x 8 (4 atoms)
  CUtensorMap tma_sfb0;    // GATE_UP: interleaved gate/up atoms; DOWN: down atoms; same view
  CUtensorMap tma_out;     // output [P, out_cols]: GATE_UP bf16, box 64 x 32; DOWN fp32, box 32 x 32; SW128
  const float* row_scale;  // [P]
  const float* ts0;        // [E]
  const float* ts1;        // [E]
  const int32_t* tile_offsets;   // [E+1], 256-row tiles
  const int32_t* tile_rows;      // [P]
  const float* weights;          // [A]
  uint32_t* status;
  int E, K, out_cols, bank_rows;
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fp4_pair_gemm_kernel(const __grid_constant__ PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int abort_flag;
  __shared__ int s_toff[kMaxExperts + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = even CTA (issues the MMAs)
  const int E = p.E;
  const int KB = p.K / 64;
  const int n_ksteps = (p.K + kStepK - 1) / kStepK;
  const int n_ntiles = GATE_UP ? p.out_cols / 128 : p.out_cols / kTileN;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_toff[i] = p.tile_offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 2 * kEpiWarps);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(&s_tmem, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();          // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_mtiles = s_toff[E];
  const int n_tiles = n_mtiles * n_ntiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // The whole warp runs the loop (warp-uniform state); one elected lane issues.
    int it = 0;
    bool ok = true;
    for (int tile = pair; tile < n_tiles && ok; tile += n_pairs) {
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
      const int e = find_expert(s_toff, E, mt);
      const int arow = mt * kPairM + 128 * (int)rank;   // this CTA's A rows
      const int rb = e * (p.bank_rows / 128);
      for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (__any_sync(0xffffffffu, !mbar_wait(&empty_bar[s], ph ^ 1u) || abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* st = smem + (size_t)s * kStageBytes;
          uint8_t* sA = st;
          uint8_t* sB = st + kABytes;
          uint8_t* sSFA = sB + kBBytes;
          uint8_t* sSFB = sSFA + kSfaBytes;
          const uint32_t bar = mapa_shared(smem_u32(&full_bar[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], kTxBytesPair);
          const int kb0 = ks * 4;
          tma_load_2d_pair(sA, &p.tma_a, ks * 128, arow, bar);
          if (GATE_UP) {
            // gate rows then up rows of features nt * 128 + 64 r .. + 63
            const int g0 = e * p.bank_rows + nt * 128 + 64 * (int)rank;
            tma_load_2d_pair(sB, &p.tma_b0, ks * 128, g0, bar);
            tma_load_2d_pair(sB + kBBytes / 2, &p.tma_b1, ks * 128, g0, bar);
          } else {
            tma_load_2d_pair(sB, &p.tma_b0, ks * 128, e * p.bank_rows + nt * kTileN + 128 * (int)rank, bar);
          }
          // scale atoms, 256-byte rows: atom j of a [..][KB][512] array spans rows 2j, 2j+1
          tma_load_2d_pair(sSFA, &p.tma_sfa, 0, 2 * ((mt * 2 + (int)rank) * KB + kb0), bar);
          if (GATE_UP) {
            // interleaved atoms 2 nt and 2 nt + 1 of this expert: B rows 0..127 and 128..255
            const int ia = e * (p.bank_rows / 64) + 2 * nt;
            tma_load_2d_pair(sSFB, &p.tma_sfb0, 0, 2 * (ia * KB + kb0), bar);
            tma_load_2d_pair(sSFB + 2048, &p.tma_sfb0, 0, 2 * ((ia + 1) * KB + kb0), bar);
          } else {
            tma_load_2d_pair(sSFB, &p.tma_sfb0, 0, 2 * ((rb + 2 * nt) * KB + kb0), bar);
            tma_load_2d_pair(sSFB + 2048, &p.tma_sfb0, 0, 2 * ((rb + 2 * nt + 1) * KB + kb0), bar);
          }
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      set_status(p.status, kDevErrTimeout);
      abort_flag = 1;
    }
    // drain (even CTA: its full barriers count both CTAs' bytes)
    if (rank == 0)
      for (int j = max(0, it - kStages); j < it; ++j)
        if (!mbar_wait(&full_bar[j % kStages], (uint32_t)(j / kStages) & 1u) && lane == 0)
          set_status(p.status, kDevErrTimeout);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    // Whole warp in the loop, one elected lane issues; the descriptors of
    // stage 0 are built once and advanced by constant offsets (16-byte units).
    if (rank == 0) {
      const uint32_t idesc = idesc_mxf4nvf4(kPairM, kTileN);
      const uint32_t s0 = smem_u32(smem);
      const uint64_t dA0 = sdesc_k_sw128(s0), dB0 = sdesc_k_sw128(s0 + kABytes);
      const uint64_t dSA0 = sdesc_sf_atom(s0 + kABytes + kBBytes);
      const uint64_t dSB0 = sdesc_sf_atom(s0 + kABytes + kBBytes + kSfaBytes);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = pair; tile < n_tiles && ok; tile += n_pairs, ++tc) {
        // both CTAs' epilogues must have drained the accumulator of the previous tile
        if (__any_sync(0xffffffffu, !mbar_wait_cluster(&acc_empty, ((uint32_t)tc & 1u) ^ 1u))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (__any_sync(0xffffffffu, !mbar_wait(&full_bar[s], ph) || abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t so = (uint64_t)((s * kStageBytes) >> 4);
          const uint32_t sfa_col = tmem + kColSf + kSfColsPerStage * s, sfb_col = sfa_col + 16;
          const int nmma = min(4, KB - ks * 4);
          if (elect_one()) {
            if (nmma == 4) {
#pragma unroll
              for (int kb = 0; kb < 4; ++kb) {
                tmem_cp_sf_pair(sfa_col + 4 * kb, dSA0 + so + 32 * kb);          // 512-byte atoms
                tmem_cp_sf_pair(sfb_col + 8 * kb, dSB0 + so + 32 * kb);
                tmem_cp_sf_pair(sfb_col + 8 * kb + 4, dSB0 + so + 128 + 32 * kb);
              }
#pragma unroll
              for (int kb = 0; kb < 4; ++kb)   // K = 64 per MMA: 32 bytes of each row
                mma_mxf4nvf4_pair(tmem, dA0 + so + 2 * kb, dB0 + so + 2 * kb, idesc, sfa_col + 4 * kb, sfb_col + 8 * kb,
                                  (ks > 0 || kb > 0) ? 1u : 0u);
            } else {
              for (int kb = 0; kb < nmma; ++kb) {
                tmem_cp_sf_pair(sfa_col + 4 * kb, dSA0 + so + 32 * kb);
                tmem_cp_sf_pair(sfb_col + 8 * kb, dSB0 + so + 32 * kb);
                tmem_cp_sf_pair(sfb_col + 8 * kb + 4, dSB0 + so + 128 + 32 * kb);
              }
              for (int kb = 0; kb < nmma; ++kb)
                mma_mxf4nvf4_pair(tmem, dA0 + so + 2 * kb, dB0 + so + 2 * kb, idesc, sfa_col + 4 * kb, sfb_col + 8 * kb,
                                  (ks > 0 || kb > 0) ? 1u : 0u);
            }
            mma_commit_pair_mc(&empty_bar[s], 0x3);   // frees the stage in both CTAs
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit_pair_mc(&acc_full, 0x3);   // accumulator final in both CTAs
        __syncwarp();
      }
      if (!ok && lane == 0) {
        set_status(p.status, kDevErrTimeout);
        abort_flag = 1;
      }
      if (elect_one()) mma_commit_pair_mc(&mma_done, 0x1);
      __syncwarp();
      if (!mbar_wait(&mma_done, 0) && lane == 0) set_status(p.status, kDevErrTimeout);
    }
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Each thread owns one accumulator row (its TMEM lane) and one column half.
    // The finished values go to this warp's swizzled staging boxes (GATE_UP:
    // one 32-row x 64-column bf16 box; DOWN: fp32, two passes of two 32-row x
    // 32-column boxes); lane 0 writes each box with one TMA tensor store.
    // Output rows are in the padded tile order (padding rows hold zeros).
    const int q = warp & 3;
    const int ch = (warp - kFirstEpiWarp) >> 2;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t acc_empty_even = mapa_shared(smem_u32(&acc_empty), 0);
    uint8_t* boxes = smem + (size_t)kStages * kStageBytes + (size_t)(warp - kFirstEpiWarp) * kEpiStageBytes;
    int tc = 0;
    for (int tile = pair; tile < n_tiles; tile += n_pairs, ++tc) {
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
      const int e = find_expert(s_toff, E, mt);
      const int row0 = mt * kPairM + 128 * (int)rank + q * 32;   // first padded row of this warp
      const int asg = p.tile_rows[row0 + lane];
      const float rs = p.row_scale[row0 + lane];
      if (__any_sync(0xffffffffu, !mbar_wait(&acc_full, (uint32_t)tc & 1u) || abort_flag)) {
        if (lane == 0) {
          set_status(p.status, kDevErrTimeout);
          abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      if (GATE_UP) {
        // columns 128 ch .. +63 gate, +64 .. +127 up of features 64 ch .. +63
        const float sg = rs * p.ts0[e], su = rs * p.ts1[e];
        uint32_t g[64], u[64];
        tmem_ld32(tq + 128 * ch, g);
        tmem_ld32(tq + 128 * ch + 32, g + 32);
        tmem_ld32(tq + 128 * ch + 64, u);
        tmem_ld32(tq + 128 * ch + 96, u + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_even);
        const int col0 = nt * 128 + 64 * ch;         // first output column of this warp's box
        uint4 w4[8];
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
          w4[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // the previous tile's stores must have read the staging box
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)                  // 16-byte chunk c of this row, 128-byte swizzle
          *reinterpret_cast<uint4*>(boxes + lane * 128 + ((c ^ (lane & 7)) << 4)) = w4[c];
        fence_proxy_async_smem();                    // generic-proxy writes visible to the tensor store
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tma_out, col0, row0, boxes);
          bulk_commit_group();
        }
        __syncwarp();
      } else {
        // fp32 rows: 128 columns per thread, two passes of two 32-column boxes
        const float sc = asg >= 0 ? rs * p.ts0[e] * p.weights[asg] : 0.f;
        uint32_t v[128];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld32(tq + 128 * ch + 32 * j, v + 32 * j);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_even);
        const int col0 = nt * kTileN + 128 * ch;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          if (lane == 0) bulk_wait_read_all();      // the boxes' previous stores have read them
          __syncwarp();
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int x = 64 * pass + 32 * b + 4 * c;
              *reinterpret_cast<float4*>(boxes + b * kEpiBoxBytes + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_float4(__uint_as_float(v[x]) * sc, __uint_as_float(v[x + 1]) * sc,
                              __uint_as_float(v[x + 2]) * sc, __uint_as_float(v[x + 3]) * sc);
            }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int b = 0; b < 2; ++b) tma_store_2d(&p.tma_out, col0 + 64 * pass + 32 * b, row0, boxes + b * kEpiBoxBytes);
            bulk_commit_group();
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  // no CTA leaves (or frees TMEM) while the pair's MMAs or copies may still
  // touch its shared or tensor memory
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

bool code_map(CUtensorMap* m, const uint8_t* base, int K, int64_t rows, uint32_t box_rows) {
  return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)rows, 128, box_rows,
                            CU_TENSOR_MAP_SWIZZLE_128B);
}

// scale atoms [n_atoms][512] viewed as [2 n_atoms, 256]; box = 4 atoms
bool atom_map(CUtensorMap* m, const uint8_t* base, int64_t n_atoms) {
  return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, (uint64_t)(2 * n_atoms), 256, 8,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace

cudaError_t launch_fp4_grouped_gemm(const Fp4GemmArgs& a, cudaStream_t st) {
  if (a.E > kMaxExperts || a.P_max % kPairM) return cudaErrorInvalidValue;
  PairParams p;
  memset(&p, 0, sizeof p);
  const bool gu = a.gate_up;
  const int KB = a.K / 64;
  const int64_t brows = (int64_t)a.E * a.bank_rows;
  if (!code_map(&p.tma_a, a.a_codes, a.K, a.P_max, 128)) return cudaErrorInvalidValue;
  if (!code_map(&p.tma_b0, a.b0_codes, a.K, brows, gu ? 64 : 128)) return cudaErrorInvalidValue;
  if (gu && !code_map(&p.tma_b1, a.b1_codes, a.K, brows, 64)) return cudaErrorInvalidValue;
  if (!atom_map(&p.tma_sfa, a.a_sf, a.P_max / 128 * KB)) return cudaErrorInvalidValue;
  // GATE_UP: interleaved gate/up atoms, 2 E I / 128 row blocks
  if (!atom_map(&p.tma_sfb0, a.b0_sf, (gu ? 2 * brows : brows) / 128 * KB)) return cudaErrorInvalidValue;
  // output boxes: GATE_UP bf16 h, 64 columns x 32 rows; DOWN fp32 rows, 32 x 32
  const bool out_ok =
      gu ? make_tensor_map_2d(&p.tma_out, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.out_cols,
                              (uint64_t)a.P_max, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B)
         : make_tensor_map_2d(&p.tma_out, a.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)a.out_cols,
                              (uint64_t)a.P_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!out_ok) return cudaErrorInvalidValue;
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
  auto kern = gu ? fp4_pair_gemm_kernel<true> : fp4_pair_gemm_kernel<false>;
  static bool attr_done[2] = {false, false};
  if (!attr_done[gu]) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done[gu] = true;
  }
  kern<<<kNumSMs, kThreads, kSmemBytes, st>>>(p);   // 74 clusters of 2 (compile-time cluster shape)
  return cudaGetLastError();
}

}  // namespace rnx
