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
//            order with plain coalesced stores after a transpose through
//            shared memory (the unpermute is fused into the combine that
//            follows, which sums them in fp32).
//
// Warp roles per CTA: warp 0 = TMA producer (ring of 38 KB stages, 5 deep
// for GATE_UP and 4 for DOWN; completions counted on the even CTA's
// barrier), warp 1 = MMA issuer (even CTA only, one thread), warp 2 = TMEM
// allocator (both CTAs), warps 4-11 = epilogue (warp w reads TMEM lane
// quadrant w % 4 and one half of the 256 accumulator columns, copies them to
// registers and releases the accumulator with a CTA-scope arrive before the
// SwiGLU / scaling and the stores). Every wait is bounded; a
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
constexpr int kStages = 5;           // GATE_UP ring depth (DOWN: 4, its larger staging takes the fifth)
constexpr int kABytes = 128 * 128;   // this CTA's A rows x 128 bytes
constexpr int kBBytes = 128 * 128;   // this CTA's half of B
constexpr int kSfaBytes = 2048;      // 4 atoms: this CTA's 128 rows, 4 K blocks
constexpr int kSfbBytes = 4096;      // 8 atoms: all 256 B rows, 4 K blocks
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 38 KB
// epilogue staging per epilogue warp: GATE_UP, one 32-row x 128-byte box in
// the 128-byte swizzled layout of the output tensor map (TMA tensor stores);
// DOWN, 32 rows x 256 bytes through which its fp32 rows are transposed
constexpr int kEpiBoxBytes = 32 * 128;
template <bool GATE_UP>
__host__ __device__ constexpr int stages_of() { return GATE_UP ? kStages : kStages - 1; }
template <bool GATE_UP>
__host__ __device__ constexpr int epi_stage_bytes_of() { return GATE_UP ? kEpiBoxBytes : 2 * kEpiBoxBytes; }
template <bool GATE_UP>
__host__ __device__ constexpr int smem_bytes_of() {
  return stages_of<GATE_UP>() * kStageBytes + 8 * epi_stage_bytes_of<GATE_UP>() + 1024;
}
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
  CUtensorMap tma_out;     // GATE_UP output h [P, out_cols] bf16, box 64 x 32, SW128
  float* out_f32;          // DOWN output [P, out_cols] fp32
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

// largest e with tile_offsets[e] <= mt. SMEM: the table was copied to shared
// memory (DOWN); else it is read through the read-only cache (GATE_UP, whose
// 5-stage ring and staging leave no room for it).
template <bool SMEM>
RNX_DEVICE int find_expert(const int32_t* __restrict__ toff, int E, int mt) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((SMEM ? toff[mid] : __ldg(toff + mid)) <= mt) lo = mid; else hi = mid;
  }
  return lo;
}

// DOWN epilogue transpose: lane r writes its row's 64 scaled fp32 values
// into row r of a 32-row x 256-byte area (16-byte chunk c at position
// c ^ (r & 15)) ...
__device__ __forceinline__ void stage_rows_256(uint8_t* area, const uint32_t (&v)[64], float sc, int lane) {
#pragma unroll
  for (int c = 0; c < 16; ++c)
    *reinterpret_cast<float4*>(area + lane * 256 + ((c ^ (lane & 15)) << 4)) =
        make_float4(__uint_as_float(v[4 * c]) * sc, __uint_as_float(v[4 * c + 1]) * sc,
                    __uint_as_float(v[4 * c + 2]) * sc, __uint_as_float(v[4 * c + 3]) * sc);
  __syncwarp();
}
// ... and the warp stores the area row by row, 16 lanes per 256-byte row
// segment (row r at dst + r * ld floats).
__device__ __forceinline__ void store_rows_256(const uint8_t* area, float* dst, int ld, int c16, int rsub) {
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const int r = 2 * i + rsub;
    const float4 x4 = *reinterpret_cast<const float4*>(area + r * 256 + ((c16 ^ (r & 15)) << 4));
    *reinterpret_cast<float4*>(dst + (size_t)r * ld) = x4;
  }
  __syncwarp();
}

template <bool GATE_UP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fp4_pair_gemm_kernel(const __grid_constant__ PairParams p) {
  constexpr int kS = stages_of<GATE_UP>();
  constexpr int kEpiStage = epi_stage_bytes_of<GATE_UP>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kS], empty_bar[kS];
  __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int abort_flag;
  __shared__ int s_toff[GATE_UP ? 1 : kMaxExperts + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = even CTA (issues the MMAs)
  const int E = p.E;
  const int KB = p.K / 64;
  const int n_ksteps = (p.K + kStepK - 1) / kStepK;
  const int n_ntiles = GATE_UP ? p.out_cols / 128 : p.out_cols / kTileN;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (!GATE_UP)   // published by the cluster barrier below
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_toff[i] = p.tile_offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kS; ++s) {
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
  const int n_mtiles = __ldg(p.tile_offsets + E);
  const int32_t* toff = GATE_UP ? p.tile_offsets : s_toff;
  const int n_tiles = n_mtiles * n_ntiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // The whole warp runs the loop (warp-uniform state); one elected lane issues.
    int it = 0;
    bool ok = true;
    for (int tile = pair; tile < n_tiles && ok; tile += n_pairs) {
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
      const int e = find_expert<!GATE_UP>(toff, E, mt);
      const int arow = mt * kPairM + 128 * (int)rank;   // this CTA's A rows
      const int rb = e * (p.bank_rows / 128);
      for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
        const int s = it % kS;
        const uint32_t ph = (uint32_t)(it / kS) & 1u;
        if (__any_sync(0xffffffffu, !mbar_wait_poll(&empty_bar[s], ph ^ 1u) || abort_flag)) {
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
      for (int j = max(0, it - kS); j < it; ++j)
        if (!mbar_wait(&full_bar[j % kS], (uint32_t)(j / kS) & 1u) && lane == 0)
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
          const int s = it % kS;
          const uint32_t ph = (uint32_t)(it / kS) & 1u;
          if (__any_sync(0xffffffffu, !mbar_wait_poll(&full_bar[s], ph) || abort_flag)) {
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
    // The finished values go through this warp's swizzled staging box
    // (GATE_UP: one 32-row x 64-column bf16 box, written by lane 0 with one
    // TMA tensor store; DOWN: two 32-row x 64-column fp32 halves, read back
    // row-contiguous and stored by all lanes).
    // Output rows are in the padded tile order (padding rows hold zeros).
    const int q = warp & 3;
    const int ch = (warp - kFirstEpiWarp) >> 2;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t acc_empty_even = mapa_shared(smem_u32(&acc_empty), 0);
    uint8_t* boxes = smem + (size_t)kS * kStageBytes + (size_t)(warp - kFirstEpiWarp) * kEpiStage;
    // This lane's row metadata is read ahead so that no global load latency
    // sits between an accumulator's completion and its release: two tiles
    // ahead the expert, the row's assignment, its A unscale and the expert's
    // tensor scales; one tile ahead the routing weight of that assignment.
    struct RowMeta {
      int asg;
      float rs, t0, t1;
    };
    auto meta_of = [&](int tile) {
      RowMeta m{-1, 0.f, 0.f, 0.f};
      if (tile < n_tiles) {
        const int mt = tile / n_ntiles;
        const int e = find_expert<!GATE_UP>(toff, E, mt);
        const int row = mt * kPairM + 128 * (int)rank + q * 32 + lane;
        m.asg = __ldg(p.tile_rows + row);
        m.rs = __ldg(p.row_scale + row);
        m.t0 = __ldg(p.ts0 + e);
        if (GATE_UP) m.t1 = __ldg(p.ts1 + e);
      }
      return m;
    };
    auto weight_of = [&](const RowMeta& m) { return !GATE_UP && m.asg >= 0 ? __ldg(p.weights + m.asg) : 0.f; };
    RowMeta m_cur = meta_of(pair), m_next = meta_of(pair + n_pairs);
    float w_cur = weight_of(m_cur);
    int tc = 0;
    for (int tile = pair; tile < n_tiles; tile += n_pairs, ++tc) {
      const int mt = tile / n_ntiles, nt = tile - mt * n_ntiles;
      const int row0 = mt * kPairM + 128 * (int)rank + q * 32;   // first padded row of this warp
      const RowMeta m = m_cur;
      const float w = w_cur;
      // issued right after the release, ahead of this tile's stores, so that
      // they do not queue behind them
      auto advance_meta = [&]() {
        m_cur = m_next;
        w_cur = weight_of(m_next);
        m_next = meta_of(tile + 2 * n_pairs);
      };
      if (__any_sync(0xffffffffu, !mbar_wait_poll(&acc_full, (uint32_t)tc & 1u) || abort_flag)) {
        if (lane == 0) {
          set_status(p.status, kDevErrTimeout);
          abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      if (GATE_UP) {
        // columns 128 ch .. +63 gate, +64 .. +127 up of features 64 ch .. +63
        const float sg = m.rs * m.t0, su = m.rs * m.t1;
        uint32_t g[64], u[64];
        tmem_ld32(tq + 128 * ch, g);
        tmem_ld32(tq + 128 * ch + 32, g + 32);
        tmem_ld32(tq + 128 * ch + 64, u);
        tmem_ld32(tq + 128 * ch + 96, u + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_even);
        advance_meta();
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
        // fp32 rows: 128 columns per thread in two halves of 64, transposed
        // through the warp's staging area (32 rows x 256 B, 16-byte chunks
        // XOR-swizzled by the row, so both the row-per-lane writes and the
        // row-contiguous reads take the minimum 4 wavefronts) and stored with
        // plain 16-byte stores, 16 lanes per 256-byte row segment: each store
        // instruction writes four whole 128-byte lines. The first half goes
        // to shared memory and the second to registers before the
        // accumulator is released, so no global store precedes the release.
        const float sc = m.asg >= 0 ? m.rs * m.t0 * w : 0.f;
        const int c16 = lane & 15, rsub = lane >> 4;
        float* out_base = p.out_f32 + (size_t)row0 * p.out_cols + nt * kTileN + 128 * ch + 4 * c16;
        uint32_t v[64];
        tmem_ld32(tq + 128 * ch, v);
        tmem_ld32(tq + 128 * ch + 32, v + 32);
        tmem_ld_wait();
        __syncwarp();                                  // the previous tile's reads of the area are done
        stage_rows_256(boxes, v, sc, lane);
        tmem_ld32(tq + 128 * ch + 64, v);
        tmem_ld32(tq + 128 * ch + 96, v + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_even);
        advance_meta();
        store_rows_256(boxes, out_base, p.out_cols, c16, rsub);
        stage_rows_256(boxes, v, sc, lane);
        store_rows_256(boxes, out_base + 64, p.out_cols, c16, rsub);
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
  if (a.P_max == 0) return cudaSuccess;   // no local expert: no rows, no tiles
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
  // output boxes (GATE_UP only): bf16 h, 64 columns x 32 rows
  if (gu && !make_tensor_map_2d(&p.tma_out, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.out_cols,
                                (uint64_t)a.P_max, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // DOWN rows are stored 16 bytes at a time (whole 128-byte lines when the
  // output is 256-byte aligned, as the workspace is)
  if (!gu && (reinterpret_cast<uintptr_t>(a.out) % 16 || a.out_cols % kTileN)) return cudaErrorInvalidValue;
  p.out_f32 = gu ? nullptr : static_cast<float*>(a.out);
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
  const int smem_bytes = gu ? smem_bytes_of<true>() : smem_bytes_of<false>();
  static bool attr_done[2] = {false, false};
  if (!attr_done[gu]) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (err != cudaSuccess) return err;
    attr_done[gu] = true;
  }
  kern<<<kNumSMs, kThreads, smem_bytes, st>>>(p);   // 74 clusters of 2 (compile-time cluster shape)
  return cudaGetLastError();
}

}  // namespace rnx
