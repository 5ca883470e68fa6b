// Internal launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/routed_nvfp4.h"

namespace rnx {

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
  bool prefetch_down;       // GATE_UP (one token per expert): pull the experts' down weights into L2
};

cudaError_t launch_nvfp4_gemv(const ExpertGemvArgs& a, cudaStream_t st);

// router
// xmax (nullable): receives max |x_t| per token as fp32 bits; zero (nullable):
// nzero uint32 words set to 0 (the h-max array of the next expert pass).
cudaError_t launch_router_logits(const uint16_t* x, int T, int H, int E, const float* wr, float* logits,
                                 cudaStream_t st, uint32_t* xmax = nullptr, uint32_t* zero = nullptr, int nzero = 0);
// max |row| as fp32 bits for R rows of K bf16 elements
cudaError_t launch_row_absmax(const uint16_t* rows, int R, int K, uint32_t* out, cudaStream_t st);
cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, float rsf, int32_t* ids,
                        float* weights, cudaStream_t st);

// permutation; scratch is int32 workspace of permute_scratch_ints(T*k, E) entries
size_t permute_scratch_ints(int A, int E);
cudaError_t launch_permute(const int32_t* ids, int A, int E, int local_begin, int local_end, const moe_plan_t& plan,
                           int32_t* scratch, uint32_t* status, cudaStream_t st);

// elementwise
cudaError_t launch_combine(int T, int k, int H, const uint16_t* r, const uint16_t* shared, uint16_t* y,
                           cudaStream_t st);
cudaError_t launch_swiglu(const float* gu, int M, int I, float limit, uint16_t* h, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts, int rows, int K, float* out,
                           cudaStream_t st);

// dense BF16 FFN (decode GEMV form): hbuf bf16 [T, I] scratch
cudaError_t launch_dense_gemv(int H, int I, float limit, const uint16_t* x, int T, const uint16_t* wg,
                              const uint16_t* wu, const uint16_t* wd, uint16_t* y, uint16_t* hbuf, cudaStream_t st);

}  // namespace rnx
