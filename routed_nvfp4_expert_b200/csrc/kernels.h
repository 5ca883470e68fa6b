// Internal launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <utility>

#include "../../include/routed_nvfp4.h"

namespace rnx {

// Launch priorities (cudaLaunchAttributePriority): the library's kernels go
// at the device's greatest priority, except the decode shared expert's on the
// auxiliary stream, which runs at the least one, so that when SMs free up the
// routed chain's CTAs are placed first.
inline int launch_priority_high() {
  static int prio = 1;                       // 1: not asked yet
  if (prio == 1) {
    int least = 0, greatest = 0;
    prio = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess ? greatest : 0;
  }
  return prio;
}
inline int launch_priority_low() {
  static int prio = 1;
  if (prio == 1) {
    int least = 0, greatest = 0;
    prio = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess ? least : 0;
  }
  return prio;
}

// Launch with a priority and, when pdl is set, programmatic stream
// serialization (see pdl_wait / pdl_trigger).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      int prio, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  attr[n].id = cudaLaunchAttributePriority;
  attr[n].val.priority = prio;
  ++n;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  return launch_ex(kern, grid, block, smem, st, true, launch_priority_high(), std::forward<Args>(args)...);
}

struct ExpertGemvArgs {
  int proj;                 // MOE_PROJ_GATE_UP / MOE_PROJ_DOWN
  int T, H, I, E, k;
  int local_begin, local_end;
  float limit;
  const void* act;          // GATE_UP: x bf16 [T, H]; DOWN: h fp32 [T*k, I]
  const int32_t* offsets;
  const int32_t* sorted;
  const int32_t* active;
  const int32_t* first;     // plan.first: first assignment of each active expert
  const float* weights;
  nvfp4_bank_t gate, up, down;
  float* out;               // GATE_UP: h fp32 [T*k, I]; DOWN: r fp32 [T*k, H]
  uint32_t* status;         // device status word (bounded-wait timeouts)
};

cudaError_t launch_nvfp4_gemv(const ExpertGemvArgs& a, cudaStream_t st);

// Decode expert projections for a handful of tokens on the tensor cores
// (decode_mma.cu), from the routing plan: gate/up writes h (clamped SwiGLU of
// the live experts' gate and up projections; zero rows for the other
// assignments), down writes the weighted rows r (zero rows likewise).
struct DecodeMmaArgs {
  int T, H, I, E, k, lb, le;
  float limit;
  const uint16_t* x;                 // bf16 [T, H], 16-byte aligned
  nvfp4_bank_t gate, up, down;
  const int32_t* active;             // routing plan: active local experts (count first)
  const int32_t* counts;             // routing plan: assignments per expert
  const int32_t* offsets;            // routing plan: first entry of each expert in sorted
  const int32_t* sorted;             // routing plan: assignments grouped by expert
  const float* weights;              // [T*k] routing weights
  const uint32_t* xmax;              // [T] max |x_t| (fp32 bits)
  float* h;                          // fp32 [T*k, I]
  float* r;                          // fp32 [T*k, H] weighted routed rows
  uint32_t* status;
  float h_up, h_unscale;             // set by the down launcher: fixed power of two for h (0: per-row maxima)
  unsigned long long wait_limit_ns;  // bound on each wait for a bulk copy (0: the library default)
};
// 1 <= T <= 8, H a multiple of 1024 up to 8192, I a multiple of 128 up to
// 2048, k <= 16, T*k <= 128, E <= 1024, a bank below 4 GB, and the staged
// activations fit in shared memory (T*(H+8)*2 and T*k*(I+8)*2 bytes, 200 KB
// each).
bool decode_mma_supported(int T, int H, int I, int E, int k);
cudaError_t launch_decode_mma_gate_up(const DecodeMmaArgs& p, cudaStream_t st);
cudaError_t launch_decode_mma_down(const DecodeMmaArgs& p, cudaStream_t st);

// router
// xmax (nullable): receives max |x_t| per token as fp32 bits; zero (nullable):
// nzero uint32 words set to 0 (the h-max array of the next expert pass). The
// side jobs run only in the GEMV form (T <= 64).
cudaError_t launch_router_logits(const uint16_t* x, int T, int H, int E, const float* wr, float* logits,
                                 cudaStream_t st, uint32_t* xmax = nullptr, uint32_t* zero = nullptr, int nzero = 0);
// The GEMV form (the one with the side jobs above) serves these shapes.
bool router_gemv_form(int T, int H);
// max |row| as fp32 bits for R rows of K bf16 elements
cudaError_t launch_row_absmax(const uint16_t* rows, int R, int K, uint32_t* out, cudaStream_t st);
cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, float rsf, int32_t* ids,
                        float* weights, cudaStream_t st);
// Top-k and the routing plan in one launch when the tokens fit one top-k CTA
// (T <= 8) and E <= 320, T*k <= 1024; else cudaErrorNotSupported.
cudaError_t launch_topk_plan(const float* logits, const float* bias, int T, int E, int k, float rsf, int32_t* ids,
                             float* weights, int lb, int le, const moe_plan_t& plan, uint32_t* status,
                             cudaStream_t st);

// permutation; scratch is int32 workspace of permute_scratch_ints(T*k, E) entries
size_t permute_scratch_ints(int A, int E);
cudaError_t launch_permute(const int32_t* ids, int A, int E, int local_begin, int local_end, const moe_plan_t& plan,
                           int32_t* scratch, uint32_t* status, cudaStream_t st);

// elementwise
// Where the prefill down projection left assignment a's row: padded row
// tile_offsets[e] * kRowsPerTile + inv[a] - offsets[e] for a local expert e = ids[a].
struct PaddedIndex {
  const int32_t* ids;
  const int32_t* inv;
  const int32_t* offsets;
  const int32_t* tile_offsets;
  int local_begin, local_end;
};
// rows: fp32 [P, H] weighted down rows in the padded tile order; shared:
// fp32 [T, H] (nullable).
cudaError_t launch_unpermute_combine(const PaddedIndex& q, int T, int k, int H, const float* rows,
                                     const float* shared, uint16_t* y, cudaStream_t st);
cudaError_t launch_unpermute(const PaddedIndex& q, long long A, int H, const float* rows, float* out,
                             cudaStream_t st);
cudaError_t launch_combine(int T, int k, int H, const uint16_t* r, const uint16_t* shared, uint16_t* y,
                           cudaStream_t st);
// the same over fp32 rows and an fp32 shared row (the decode path)
cudaError_t launch_combine_f32(int T, int k, int H, const float* r, const float* shared, uint16_t* y,
                               cudaStream_t st);
cudaError_t launch_swiglu(const float* gu, int M, int I, float limit, uint16_t* h, cudaStream_t st);

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts, int rows, int K, float* out,
                           cudaStream_t st);

// dense BF16 FFN (decode GEMV form): hbuf fp32 [T, I] scratch; y bf16 or
// fp32 (y_f32) [T, H]
// background: the decode site's shared expert on its auxiliary stream (least
// priority; the down GEMV launched only once the gate/up one is done, so that
// it holds no SM while it waits).
cudaError_t launch_dense_gemv(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                              const uint16_t* wu, const uint16_t* wd, void* y, bool y_f32, float* hbuf,
                              cudaStream_t st, bool background = false);

// BF16 GEMM on tcgen05 (kind::f16): out [M, N] = a [M, K] . b^T with b [N, K].
// gate_up: b0 = gate rows, b1 = up rows; out = clamped_swiglu(a.b0^T, a.b1^T).
// N a multiple of 128 (gate_up) or 256, K a multiple of 64. status: device
// word for bounded-wait timeouts (nullable). out_f32 (not gate_up): fp32
// output [M, N] in place of out. split: gate_up writes h as two bf16 terms
// (hi at column c, lo = bf16(h - hi) at N + c; out [M, 2N]); the down
// product then takes a = [hi | lo] with K = 2 x the weight's K, reading b0
// twice, so h enters with 16 significant bits.
cudaError_t launch_bf16_gemm(bool gate_up, const uint16_t* a, int M, int K, const uint16_t* b0, const uint16_t* b1,
                             int N, float limit, uint16_t* out, uint32_t* status, cudaStream_t st,
                             float* out_f32 = nullptr, bool split = false);
// Limit of the BF16 GEMM's main-loop waits for later launches (host setting;
// 0 = give up at the first incomplete poll). Test hook for the timeout path.
void set_test_wait_limit_ns(unsigned long long ns);

// Router logits on the tensor cores: logits [T, E] fp32 = x [T, H] . w^T with
// w given exactly as w3 [E, 3H] bf16 = (lo | mid | hi) per row. E % 4 == 0,
// H % 256 == 0.
cudaError_t launch_router_logits_tc(const uint16_t* x, int T, int H, int E, const uint16_t* w3, float* logits,
                                    uint32_t* status, cudaStream_t st);
// w3 [E, 3H] bf16 (lo | mid | hi) from the fp32 router weight [E, H]: hi = w
// with the low 16 bits cleared, mid likewise from w - hi, lo = w - hi - mid
// (all exact).
cudaError_t launch_router_split(const float* w, int E, int H, uint16_t* w3, cudaStream_t st);

// Dense BF16 FFN, picking the GEMV form for small T and the tcgen05 GEMM for
// T >= min_t (default kDenseGemmMinT; when the shapes allow it).
constexpr int kDenseGemmMinT = 128;
// hbuf: T*I*4 bytes (fp32 h in the GEMV form; in the GEMM form bf16 h, or,
// when y_f32, h as two bf16 terms hi + lo).
// y: bf16 [T, H], or fp32 when y_f32.
cudaError_t launch_dense_ffn(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                             const uint16_t* wu, const uint16_t* wd, void* y, bool y_f32, void* hbuf,
                             uint32_t* status, cudaStream_t st, int min_t = kDenseGemmMinT);

// ---------------------------------------------------------------- prefill (W4A4, tcgen05)

// Padded tile layout of the prefill: every local expert's rows start on a
// 256-row tile (kRowsPerTile). tile_rows[p] = assignment at padded row p, -1 for padding.
// P_max = padded_rows_bound(A, E_local) rows are written (rows past the last
// used tile get -1 too).
int64_t padded_rows_bound(int64_t A, int64_t E_local);
cudaError_t launch_tile_rows(const moe_plan_t& plan, int E, int64_t P_max, cudaStream_t st);

// NVFP4 encoding of bf16 rows (per-row fp32 scale r/2688, E4M3 per 16, E2M1).
// Output row p reads source row: row_map ? (row_map[p] < 0 ? none : div > 0 ? row_map[p] / div : p) : p
// ("none" = a zero row).
// codes [rows, K/2]; sf atoms [ceil(rows/128)][K/64][512]; row_scale [rows].
// Rows in [rows, ceil128(rows)) get zero scale bytes. used_tiles (nullable,
// device int): rows at or past used_tiles*128 are left untouched.
cudaError_t launch_quant_rows(const uint16_t* src, int64_t rows, int K, const int32_t* row_map, int div,
                              const int32_t* used_tiles, uint8_t* codes, uint8_t* sf, float* row_scale,
                              cudaStream_t st);
// The prefill's x encoding token-major (each token encoded once, written to
// the padded rows of its local assignments; padding rows of used tiles
// zeroed): the same bytes as launch_quant_rows(x, P, K, tile_rows, k, ...).
// k <= 16, else cudaErrorNotSupported.
cudaError_t launch_quant_tokens(const uint16_t* x, int T, int K, int k, const int32_t* ids, const moe_plan_t& plan,
                                int lb, int le, int64_t P, const int32_t* used_tiles, uint8_t* codes, uint8_t* sf,
                                float* row_scale, cudaStream_t st);

// Canonical block scales [n_experts * rows, K/16] -> atoms [n_experts][rows/128][K/64][512].
cudaError_t launch_sf_atoms(const uint8_t* scales, int64_t n_experts, int rows, int K, uint8_t* atoms, cudaStream_t st);
// Gate and up block scales ([E*I, K/16] each) -> atoms [E][I/64][K/64][512]
// whose 128 rows are 64 gate rows then the same 64 up rows (I % 64 == 0).
cudaError_t launch_sf_atoms_gate_up(const uint8_t* gate, const uint8_t* up, int64_t n_experts, int I, int K,
                                    uint8_t* atoms, cudaStream_t st);

struct Fp4GemmArgs {
  bool gate_up;
  int E, K, out_cols, bank_rows;   // bank_rows: rows of one expert in the weight bank (I for gate/up, H for down)
  int64_t P_max;                   // rows of the A operand buffers
  float limit;
  const uint8_t* a_codes;          // [P_max, K/2]
  const uint8_t* a_sf;             // atoms [P_max/128][K/64][512]
  const float* row_scale;          // [P_max]
  const uint8_t* b0_codes;         // gate (or down) codes [E*bank_rows, K/2]
  const uint8_t* b1_codes;         // up codes (gate_up)
  const uint8_t* b0_sf;            // GATE_UP: interleaved gate/up atoms [E][I/64][K/64][512];
                                   // DOWN: atoms [E][H/128][K/64][512]
  const uint8_t* b1_sf;            // unused
  const float* ts0;
  const float* ts1;
  const int32_t* tile_offsets;     // [E+1]
  const int32_t* tile_rows;        // [P_max]
  const float* weights;            // [A] routing weights (down)
  void* out;                       // [P_max, out_cols] in the padded tile order: GATE_UP h bf16,
                                   // DOWN weighted rows fp32
  uint32_t* status;
};
cudaError_t launch_fp4_grouped_gemm(const Fp4GemmArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- prefill (W4A16, tcgen05 kind::f16)

// x rows in the padded tile order as f16, each scaled by the power of two that
// brings its max |x| into [2^14, 2^15); unscale[p] the inverse (0 on padding
// rows). Rows at or past used_tiles * 256 are not written, nor (sparse) the
// rows of 128-row halves that hold only padding.
cudaError_t launch_gather_x_f16(const uint16_t* x, int H, int k, const int32_t* tile_rows, const int32_t* used_tiles,
                                int64_t P, uint16_t* xa, float* unscale, cudaStream_t st, bool sparse = false);

struct W4a16GemmArgs {
  bool gate_up;
  int E, K, out_cols, bank_rows;   // bank_rows: rows of one expert (I for gate/up, H for down)
  int64_t P_max;
  float limit;
  const uint16_t* act;             // f16 [P_max, K] (GATE_UP: gathered x; DOWN: h)
  const float* row_scale;          // [P_max] A row unscale (nullable: 1)
  const uint8_t* b0_codes;         // gate (or down) codes [E*bank_rows, K/2]
  const uint8_t* b1_codes;         // up codes (GATE_UP)
  const uint8_t* b_sf;             // GATE_UP: interleaved gate/up atoms; DOWN: down atoms
  const float* ts0;
  const float* ts1;
  const int32_t* tile_offsets;     // [E+1]
  const int32_t* tile_rows;        // [P_max]
  const float* weights;            // [A] routing weights (DOWN)
  void* out;                       // GATE_UP: h f16 [P_max, I]; DOWN: rows fp32 [P_max, H]
  uint32_t* status;
  bool sparse = false;             // decode batches: 128-row halves holding only padding are skipped, and
                                   // DOWN writes row p to out row tile_rows[p] (rows fp32 [A, H] in
                                   // assignment order; padding rows not written)
};
cudaError_t launch_w4a16_grouped_gemm(const W4a16GemmArgs& a, cudaStream_t st);

}  // namespace rnx
