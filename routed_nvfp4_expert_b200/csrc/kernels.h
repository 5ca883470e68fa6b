// Internal launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <utility>

#include "../../include/routed_nvfp4.h"

namespace rnx {

// Launch with programmatic stream serialization (see pdl_wait / pdl_trigger).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct ExpertGemvArgs {
  int proj;                 // MOE_PROJ_GATE_UP / MOE_PROJ_DOWN
  int T, H, I, E, k;
  int local_begin, local_end;
  float limit;
  const uint16_t* act;
  const int32_t* offsets;
  const int32_t* sorted;
  const int32_t* active;
  const int32_t* first;     // plan.first: first assignment of each active expert
  const float* weights;
  nvfp4_bank_t gate, up, down;
  uint16_t* out;
  uint32_t* status;         // device status word (bounded-wait timeouts)
  const uint32_t* act_max;  // optional: max |activation row| as fp32 bits (x rows by token / h rows by assignment)
  uint32_t* out_max;        // optional (GATE_UP): receives max |h| per assignment; must start at 0
};

cudaError_t launch_nvfp4_gemv(const ExpertGemvArgs& a, cudaStream_t st);

// router
// xmax (nullable): receives max |x_t| per token as fp32 bits; zero (nullable):
// nzero uint32 words set to 0 (the h-max array of the next expert pass). The
// side jobs run only in the GEMV form (T <= 64).
cudaError_t launch_router_logits(const uint16_t* x, int T, int H, int E, const float* wr, float* logits,
                                 cudaStream_t st, uint32_t* xmax = nullptr, uint32_t* zero = nullptr, int nzero = 0);
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
cudaError_t launch_unpermute_combine(const PaddedIndex& q, int T, int k, int H, const uint16_t* rows,
                                     const uint16_t* shared, uint16_t* y, cudaStream_t st);
cudaError_t launch_unpermute(const PaddedIndex& q, long long A, int H, const uint16_t* rows, uint16_t* out,
                             cudaStream_t st);
cudaError_t launch_combine(int T, int k, int H, const uint16_t* r, const uint16_t* shared, uint16_t* y,
                           cudaStream_t st);
cudaError_t launch_swiglu(const float* gu, int M, int I, float limit, uint16_t* h, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts, int rows, int K, float* out,
                           cudaStream_t st);

// dense BF16 FFN (decode GEMV form): hbuf bf16 [T, I] scratch
cudaError_t launch_dense_gemv(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                              const uint16_t* wu, const uint16_t* wd, uint16_t* y, uint16_t* hbuf, cudaStream_t st);

// BF16 GEMM on tcgen05 (kind::f16): out [M, N] = a [M, K] . b^T with b [N, K].
// gate_up: b0 = gate rows, b1 = up rows; out = clamped_swiglu(a.b0^T, a.b1^T).
// N a multiple of 128 (gate_up) or 256, K a multiple of 64. status: device
// word for bounded-wait timeouts (nullable).
cudaError_t launch_bf16_gemm(bool gate_up, const uint16_t* a, int M, int K, const uint16_t* b0, const uint16_t* b1,
                             int N, float limit, uint16_t* out, uint32_t* status, cudaStream_t st);

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
// T >= kDenseGemmMinT (when the shapes allow it).
constexpr int kDenseGemmMinT = 128;
cudaError_t launch_dense_ffn(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                             const uint16_t* wu, const uint16_t* wd, uint16_t* y, uint16_t* hbuf, uint32_t* status,
                             cudaStream_t st);

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
  const uint8_t* b0_sf;            // atoms [E][bank_rows/128][K/64][512]
  const uint8_t* b1_sf;
  const float* ts0;
  const float* ts1;
  const int32_t* tile_offsets;     // [E+1]
  const int32_t* tile_rows;        // [P_max]
  const float* weights;            // [A] routing weights (down)
  uint16_t* out;                   // [P_max, out_cols] in the padded tile order (h, or weighted down rows)
  uint32_t* status;
};
cudaError_t launch_fp4_grouped_gemm(const Fp4GemmArgs& a, cudaStream_t st);

}  // namespace rnx
