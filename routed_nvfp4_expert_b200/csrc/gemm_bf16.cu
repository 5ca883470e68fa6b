// Dense BF16 GEMMs on the 5th-generation tensor cores (tcgen05.mma
// kind::f16 with bf16 operands, fp32 accumulators in tensor memory): the dense
// FFN and the shared expert at large T (glm5next_mlp module docs, "The stack
// this layer runs": DENSE gate_proj/up_proj -> clamped SwiGLU -> down_proj;
// shared_experts BF16 gate/up -> clamped SwiGLU -> BF16 down).
//   A = x [M, K] (or h), B = weight rows [N, K], both K-major bf16.
//   GATE_UP: tile = 128 rows x (128 gate + 128 up weight rows); the epilogue
//            applies the clamped SwiGLU and stores h bf16 [M, N].
//   DOWN:    tile = 128 rows x 256 output features, stored bf16 [M, N].
//   LOGITS:  the router logits at large T (the glm5next_mlp stack's
//            gate.weight -> fp32 logits) as one bf16 GEMM over K = 3H: the fp32
//            router weight is split exactly into three bf16 terms w = lo + mid
//            + hi ([E, 3H] in that order, built by moe_prepare_weights), x is
//            read three times along K, products of bf16 are exact in fp32.
//            The tensor core's accumulation does not round to nearest, so the
//            small lo and mid terms go first into an empty accumulator and the
//            hi terms are spread over four accumulators (N = 128 tiles), whose
//            partial sums the epilogue adds in fp32; fp32 logits [M, E].
//
// One persistent CTA per SM walks the (m-tile, n-tile) list with the m-tiles
// innermost, so each weight tile is read from HBM once while x stays in L2.
// Warp roles: warp 0 = TMA producer (4-stage ring of 64-element K slices, 128
// bytes per row, 128-byte swizzle), warp 1 = MMA issuer (one thread, four
// M=128 N=256 K=16 MMAs per stage), warp 2 = TMEM allocator (two 256-column
// accumulators), warps 4-11 = epilogue (warp w reads TMEM lane quadrant w % 4
// and one half of the accumulator columns, copies them to registers and
// releases the buffer before the SwiGLU and the stores). Every wait is
// bounded; a timeout sets the device status word and winds the CTA down
// (copies and MMAs in flight drained, TMEM freed). No TMA load uses cluster
// multicast.

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tensor_map.h"

namespace rnx {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 256;          // MMA N (GATE_UP: 128 gate + 128 up)
constexpr int kStepK = 64;           // bf16 elements per stage: 128 bytes per row (one swizzle span)
constexpr int kStages = 4;
constexpr int kABytes = kTileM * 128;                // 16 KB
constexpr int kBBytes = kTileN * 128;                // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;       // 48 KB
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kFirstEpiWarp = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kFirstEpiWarp + kEpiWarps) * 32;   // 384
constexpr uint32_t kTmemCols = 512;                          // two 256-column accumulators

enum { kModeGateUp = 0, kModeDown = 1, kModeLogits = 2 };

struct GemmParams {
  CUtensorMap tma_a;       // A [M, a_period] bf16; box 64 x 128 rows, SW128
  CUtensorMap tma_b0;      // GATE_UP: gate rows (box 128 rows); DOWN / LOGITS: weight rows (box 256 rows)
  CUtensorMap tma_b1;      // GATE_UP: up rows
  uint16_t* out;           // GATE_UP / DOWN: bf16 [M, out_cols]
  float* out_f32;          // LOGITS, and DOWN when set: fp32 [M, out_cols], columns < out_cols written
  uint32_t* status;
  int M, K, out_cols;
  int a_period;            // A's K extent; the K loop reads A at k mod a_period (LOGITS: K = 3 a_period)
  int b_period;            // DOWN: B's K extent; the K loop reads B at k mod b_period (0: K). With
                           // A = [h_hi | h_lo] and b_period = K / 2 the product is (h_hi + h_lo) . b
  int split_h;             // GATE_UP: h written as two bf16 terms per element, h_hi at column c and
                           // h_lo = bf16(h - h_hi) at column out_cols + c (row pitch 2 out_cols)
  float limit;
  unsigned long long wait_ns;   // limit of the main-loop waits (the drain waits keep the default)
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) bf16_gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool GATE_UP = MODE == kModeGateUp;
  constexpr bool LOGITS = MODE == kModeLogits;
  // LOGITS: N = 128 tiles and four 128-column accumulators in one buffer (the
  // K segments lo | mid | hi of the split weight go to accumulator 0, the
  // hi segment's later three quarters to 1..3; partial sums added in fp32)
  constexpr int kTN = LOGITS ? 128 : kTileN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_ksteps = p.K / kStepK;
  const int n_ntiles = GATE_UP ? p.out_cols / 128 : (p.out_cols + kTN - 1) / kTN;
  const int seg = p.a_period / kStepK, q4 = seg / 4;     // LOGITS: k-steps per segment / per hi quarter
  const int n_mtiles = (p.M + kTileM - 1) / kTileM;
  const int n_tiles = n_mtiles * n_ntiles;

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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (warp-uniform state); one elected lane issues.
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int nt = tile / n_mtiles, mt = tile - nt * n_mtiles;   // m-tiles innermost
      for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (__any_sync(0xffffffffu, !mbar_wait(&empty_bar[s], ph ^ 1u, p.wait_ns) || abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* sA = smem + (size_t)s * kStageBytes;
          uint8_t* sB = sA + kABytes;
          mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(kABytes + (LOGITS ? kBBytes / 2 : kBBytes)));
          tma_load_2d(sA, &p.tma_a, LOGITS ? (ks * kStepK) % p.a_period : ks * kStepK, mt * kTileM, &full_bar[s]);
          if (GATE_UP) {
            tma_load_2d(sB, &p.tma_b0, ks * kStepK, nt * 128, &full_bar[s]);
            tma_load_2d(sB + kBBytes / 2, &p.tma_b1, ks * kStepK, nt * 128, &full_bar[s]);
          } else {
            tma_load_2d(sB, &p.tma_b0, p.b_period ? (ks * kStepK) % p.b_period : ks * kStepK, nt * kTN,
                        &full_bar[s]);
          }
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      set_status(p.status, kDevErrTimeout);
      abort_flag = 1;
    }
    // drain: every copy issued must have landed before the CTA may exit
    for (int j = max(0, it - kStages); j < it; ++j)
      if (!mbar_wait(&full_bar[j % kStages], (uint32_t)(j / kStages) & 1u) && lane == 0)
        set_status(p.status, kDevErrTimeout);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Whole warp in the loop, one elected lane issues; stage-0 descriptors are
    // built once and advanced by constant offsets (16-byte units).
    const uint32_t idesc = idesc_bf16(kTileM, kTN);
    const uint32_t s0 = smem_u32(smem);
    const uint64_t dA0 = sdesc_k_sw128(s0), dB0 = sdesc_k_sw128(s0 + kABytes);
    int it = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc) {
      const int b = LOGITS ? 0 : (tc & 1);
      const uint32_t use = LOGITS ? (uint32_t)tc : (uint32_t)(tc >> 1);
      // the epilogue must have drained this accumulator buffer's previous tile
      if (__any_sync(0xffffffffu, !mbar_wait(&acc_empty[b], (use & 1u) ^ 1u, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + 256u * b;
      for (int ks = 0; ks < n_ksteps; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (__any_sync(0xffffffffu, !mbar_wait(&full_bar[s], ph, p.wait_ns) || abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t so = (uint64_t)((s * kStageBytes) >> 4);
        if (elect_one()) {
          if (LOGITS) {
            const int ai = ks < 2 * seg + q4 ? 0 : min(3, (ks - 2 * seg) / q4);
            const int first = ai == 0 ? 0 : 2 * seg + ai * q4;   // first k-step into this accumulator
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              mma_bf16(acc + 128u * ai, dA0 + so + 2 * kb, dB0 + so + 2 * kb, idesc,
                       (ks > first || kb > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)   // K = 16 per MMA: 32 bytes of each row
              mma_bf16(acc, dA0 + so + 2 * kb, dB0 + so + 2 * kb, idesc, (ks > 0 || kb > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[s]);          // the stage is free once these MMAs have read it
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&acc_full[b]);   // the accumulator is final once every MMA is done
      __syncwarp();
    }
    if (!ok && lane == 0) {
      set_status(p.status, kDevErrTimeout);
      abort_flag = 1;
    }
    if (elect_one()) mma_commit(&mma_done);
    __syncwarp();
    if (!mbar_wait(&mma_done, 0) && lane == 0) set_status(p.status, kDevErrTimeout);
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                          // TMEM lane quadrant this warp may access
    const int ch = (warp - kFirstEpiWarp) >> 2;     // column half
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      const int b = LOGITS ? 0 : (tc & 1);
      const uint32_t use = LOGITS ? (uint32_t)tc : (uint32_t)(tc >> 1);
      const int nt = tile / n_mtiles, mt = tile - nt * n_mtiles;
      const int row = mt * kTileM + q * 32 + lane;   // A row = TMEM lane of this thread
      const bool valid = row < p.M;
      // warp-uniform decision: the tcgen05.ld below is a whole-warp instruction
      if (__any_sync(0xffffffffu, !mbar_wait(&acc_full[b], use & 1u, p.wait_ns) || abort_flag)) {
        if (lane == 0) {
          set_status(p.status, kDevErrTimeout);
          abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t tq = tmem + 256u * b + ((uint32_t)(q * 32) << 16);
      if (GATE_UP) {
        uint32_t g[64], u[64];
        tmem_ld32(tq + 64 * ch, g);
        tmem_ld32(tq + 64 * ch + 32, g + 32);
        tmem_ld32(tq + 128 + 64 * ch, u);
        tmem_ld32(tq + 128 + 64 * ch + 32, u + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        if (valid) {
          const size_t pitch = p.split_h ? 2 * (size_t)p.out_cols : (size_t)p.out_cols;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * pitch + nt * 128 + 64 * ch);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t w[4], wl[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k0 = 8 * c + 2 * i;
              const float h0 = clamped_swiglu_fast(__uint_as_float(g[k0]), __uint_as_float(u[k0]), p.limit);
              const float h1 = clamped_swiglu_fast(__uint_as_float(g[k0 + 1]), __uint_as_float(u[k0 + 1]), p.limit);
              w[i] = pack_bf16x2(h0, h1);
              // the rounding error of the bf16 term, itself in bf16 (exact difference in fp32)
              wl[i] = pack_bf16x2(h0 - __uint_as_float(w[i] << 16), h1 - __uint_as_float(w[i] & 0xFFFF0000u));
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
            if (p.split_h) dst[c + p.out_cols / 8] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          }
        }
      } else if (LOGITS) {
        // this warp's 64 columns, 32 at a time: the four accumulators summed in fp32
#pragma unroll 1
        for (int sub = 0; sub < 2; ++sub) {
          const int cl = 64 * ch + 32 * sub;         // column within the tile
          uint32_t a[4][32];
#pragma unroll
          for (int i = 0; i < 4; ++i) tmem_ld32(tq + 128 * i + cl, a[i]);
          tmem_ld_wait();
          if (valid) {
            float* dst = p.out_f32 + (size_t)row * p.out_cols + nt * kTN + cl;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float o[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int x = 4 * c + j;
                o[j] = ((__uint_as_float(a[0][x]) + __uint_as_float(a[1][x])) + __uint_as_float(a[2][x])) +
                       __uint_as_float(a[3][x]);
              }
              if (nt * kTN + cl + 4 * c < p.out_cols) *reinterpret_cast<float4*>(dst + 4 * c) = make_float4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
      } else {
        uint32_t v[128];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld32(tq + 128 * ch + 32 * j, v + 32 * j);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
        if (valid && p.out_f32) {
          // fp32 rows (the site's shared expert, summed in fp32 by the combine)
          float4* dst = reinterpret_cast<float4*>(p.out_f32 + (size_t)row * p.out_cols + nt * kTileN + 128 * ch);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            dst[c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                 __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * p.out_cols + nt * kTileN + 128 * ch);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = pack_bf16x2(__uint_as_float(v[8 * c + 2 * i]), __uint_as_float(v[8 * c + 2 * i + 1]));
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

bool bf16_map(CUtensorMap* m, const uint16_t* base, int K, int rows, uint32_t box_rows) {
  return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)K, (uint64_t)rows, kStepK,
                            box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int MODE>
cudaError_t launch(const GemmParams& p, cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t err = cudaFuncSetAttribute(bf16_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done = true;
  }
  bf16_gemm_kernel<MODE><<<kNumSMs, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Main-loop wait limit of the BF16 GEMM launches (the drain waits keep the
// default): kWaitLimitNs unless a test lowered it.
static unsigned long long g_gemm_wait_ns = kWaitLimitNs;
void set_test_wait_limit_ns(unsigned long long ns) { g_gemm_wait_ns = ns; }

cudaError_t launch_bf16_gemm(bool gate_up, const uint16_t* a, int M, int K, const uint16_t* b0, const uint16_t* b1,
                             int N, float limit, uint16_t* out, uint32_t* status, cudaStream_t st, float* out_f32,
                             bool split) {
  if (M <= 0 || K % kStepK || N % (gate_up ? 128 : kTileN)) return cudaErrorInvalidValue;
  const bool split_down = split && !gate_up;
  if (split_down && (K / 2) % kStepK) return cudaErrorInvalidValue;
  GemmParams p;
  memset(&p, 0, sizeof p);
  if (!bf16_map(&p.tma_a, a, K, M, kTileM)) return cudaErrorInvalidValue;
  if (!bf16_map(&p.tma_b0, b0, split_down ? K / 2 : K, N, gate_up ? 128 : kTileN)) return cudaErrorInvalidValue;
  p.b_period = split_down ? K / 2 : 0;
  p.split_h = split && gate_up;
  if (gate_up && !bf16_map(&p.tma_b1, b1, K, N, 128)) return cudaErrorInvalidValue;
  p.out = out;
  p.out_f32 = gate_up ? nullptr : out_f32;
  p.status = status;
  p.M = M;
  p.K = K;
  p.out_cols = N;
  p.a_period = K;
  p.limit = limit;
  p.wait_ns = g_gemm_wait_ns;
  return gate_up ? launch<kModeGateUp>(p, st) : launch<kModeDown>(p, st);
}

cudaError_t launch_router_logits_tc(const uint16_t* x, int T, int H, int E, const uint16_t* w3, float* logits,
                                    uint32_t* status, cudaStream_t st) {
  if (T <= 0 || H % kStepK || E % 4) return cudaErrorInvalidValue;
  GemmParams p;
  memset(&p, 0, sizeof p);
  if (!bf16_map(&p.tma_a, x, H, T, kTileM)) return cudaErrorInvalidValue;
  if (H % 256) return cudaErrorInvalidValue;   // four hi quarters of whole 64-element k-steps
  if (!bf16_map(&p.tma_b0, w3, 3 * H, E, 128)) return cudaErrorInvalidValue;
  p.out_f32 = logits;
  p.status = status;
  p.M = T;
  p.K = 3 * H;
  p.out_cols = E;
  p.a_period = H;
  p.wait_ns = g_gemm_wait_ns;
  return launch<kModeLogits>(p, st);
}

}  // namespace rnx
