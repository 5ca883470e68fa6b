/*
 * routed_nvfp4.h -- C ABI of the B200 (sm_100a) routed NVFP4 MoE MLP site.
 *
 * The operation is the GLM-5.3-Flash MLP site described by the glm5next_mlp
 * module docs ("GLM-5.3-Flash MLP production surface"), section "The stack
 * this layer runs":
 *
 *   DENSE  (layers 0..first_k_dense_replace): x -> gate_proj/up_proj ->
 *          clamped SwiGLU -> down_proj                       (dense_ffn_bf16)
 *   ROUTED (every later layer):
 *     x -> gate.weight -> fp32 logits -> router_topk -> ids[K], weights[K]
 *                                                       (moe_router_topk)
 *     experts[id] (LOCAL ids only): NVFP4 gate/up -> clamped SwiGLU ->
 *          NVFP4 down           (nvfp4_expert_gemv / nvfp4_grouped_gemm)
 *     shared expert: BF16 gate/up -> clamped SwiGLU -> BF16 down
 *     moe_combine -> partial                             (moe_combine)
 *
 * and the rules of its section "Traps this module exists to hold": the
 * SwiGLU clamp is asymmetric (gate bounded above only, up bounded on both
 * sides) with a limit that is never defaulted; the router's correction bias
 * steers selection only and each emitted weight is the unbiased sigmoid
 * score, renormalised over the chosen k and multiplied by
 * routed_scaling_factor; the shared expert is never scaled; num_experts is
 * the FULL expert count and the local range is a separate field. The
 * Constants section's KERNEL_MAX_TOP_K caps k at 16.
 *
 * NVFP4 (the experts' format): E2M1 values (OCP MX v1.0), one E4M3 scale per
 * 16 consecutive elements along K (OCP OFP8), one fp32 scale per tensor;
 * value = e2m1 * e4m3 * tensor_scale. Canonical layout: row-major [rows, K],
 * two codes per byte with the even element in the low nibble; scales
 * row-major [rows, K/16].
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers unless a comment says otherwise,
 *    16-byte aligned. The caller owns every buffer; the library allocates and
 *    frees no device memory and keeps no state besides a thread-local error
 *    message, the thread-local stage-timing events of moe_set_stage_events()
 *    and, per host thread and device, the auxiliary stream and event pair on
 *    which the decode forward runs the shared expert concurrently
 *    (created by the first such call on that thread and device: make it before
 *    any stream capture on that thread).
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Every call is
 *    stream-ordered and asynchronous; nothing synchronises except
 *    moe_read_device_status().
 *  - A call validates its arguments first. On failure it returns a non-zero
 *    moe_status_t, launches nothing, and moe_last_error() describes why.
 *  - T = 0 (no tokens) is a no-op that returns MOE_OK.
 *  - Errors found on the device (an index out of range, a bounded wait that
 *    ran out) are OR-ed into the status word at the start of the workspace
 *    and reported by moe_read_device_status(); the affected outputs are then
 *    unspecified but every access stays in bounds.
 */
#ifndef ROUTED_NVFP4_H
#define ROUTED_NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* bad pointer, size, alignment or config field */
  MOE_ERR_UNSUPPORTED = 2,    /* valid request outside what the kernels cover */
  MOE_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required */
  MOE_ERR_CUDA = 4,           /* a CUDA launch or runtime call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait ran out */
  MOE_ERR_DEVICE_BOUNDS = 6   /* a device-side index check failed */
} moe_status_t;

/* Which implementation of the routed experts moe_forward runs. */
typedef enum {
  MOE_PATH_DECODE = 0,         /* W4A16 GEMV: bf16 activations x NVFP4 weights */
  MOE_PATH_PREFILL = 1,        /* W4A4 grouped GEMM on tcgen05 block-scaled FP4 */
  MOE_PATH_PREFILL_W4A16 = 2   /* W4A16 grouped GEMM on tcgen05 kind::f16 (the pages' prefill) */
} moe_path_t;

/* Projection selector of the expert kernels. */
typedef enum {
  MOE_PROJ_GATE_UP = 0, /* gate and up, fused clamped SwiGLU -> h */
  MOE_PROJ_DOWN = 1     /* down, times the routing weight -> r[t, j] */
} moe_proj_t;

/*
 * Site geometry for one rank (Glm5NextMlpConfig: "read from the checkpoint
 * config -- never defaulted"). Every field is required and validated.
 *   hidden               H, multiple of 64
 *   intermediate         I of each routed expert, multiple of 64
 *   shared_intermediate  Is of the BF16 shared expert, multiple of 64; 0 = none
 *   num_experts          E, the FULL expert count the router ranks
 *   local_begin/end      [begin, end) experts this rank computes; ids outside
 *                        contribute zero (masked-local expert parallelism);
 *                        [0, E) on one GPU
 *   top_k                1 .. min(16, E)
 *   routed_scaling_factor  finite
 *   swiglu_limit         > 0; +inf allowed (no clamp); NaN rejected
 */
typedef struct {
  int32_t hidden;
  int32_t intermediate;
  int32_t shared_intermediate;
  int32_t num_experts;
  int32_t local_begin;
  int32_t local_end;
  int32_t top_k;
  float routed_scaling_factor;
  float swiglu_limit;
} moe_config_t;

/* One projection of all E experts in canonical NVFP4 layout, contiguous per
 * expert: codes [E, rows, cols/2], scales [E, rows, cols/16], tensor_scale [E]
 * (device fp32). gate/up: rows = I, cols = H. down: rows = H, cols = I. */
typedef struct {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* tensor_scale;
} nvfp4_bank_t;

/* Weights of one routed site (Glm5NextMoeWeights), already sharded for this
 * rank. router_w fp32 [E, H] row-major; router_bias fp32 [E]; shared_* bf16
 * row-major: gate and up [Is, H], down [H, Is] (NULL when Is == 0).
 * prepared: the experts' block scales re-tiled by moe_prepare_weights()
 * (moe_prepared_size() bytes) for the tensor-core prefill path; NULL is
 * allowed when only MOE_PATH_DECODE runs. */
typedef struct {
  const float* router_w;
  const float* router_bias;
  nvfp4_bank_t gate;
  nvfp4_bank_t up;
  nvfp4_bank_t down;
  const uint16_t* shared_gate;
  const uint16_t* shared_up;
  const uint16_t* shared_down;
  const uint8_t* prepared;
} moe_weights_t;

/*
 * Routing plan: the A = T*k assignments (a = t*k + j, j = rank slot) grouped
 * by expert, stably (token order inside each expert). Device int32 arrays:
 *   counts       [E]    assignments per expert
 *   offsets      [E+1]  segment starts, offsets[E] = A
 *   sorted       [A]    assignment at sorted position p
 *   inv          [A]    sorted position of assignment a
 *   tile_offsets [E+1]  prefix sum over experts of ceil(counts/256) for LOCAL
 *                       experts (0 tiles for remote ones): 256-row tiles
 *   active       [E+1]  active[0] = number of LOCAL experts with counts > 0,
 *                       active[1..] = their ids in ascending order
 *   first        [E]    first[u] = sorted[offsets[active[1+u]]], the first
 *                       assignment of the u-th active expert
 *   tile_rows    [P]    P = moe_padded_rows(cfg, T): the padded tile layout
 *                       of the prefill, in which every LOCAL expert's rows
 *                       start on a 256-row tile (tile_offsets); tile_rows[p]
 *                       is the assignment at padded row p, -1 for padding and
 *                       for rows past the last tile. Filled by moe_permute
 *                       and by the prefill path of moe_forward.
 */
typedef struct {
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted;
  int32_t* inv;
  int32_t* tile_offsets;
  int32_t* active;
  int32_t* first;
  int32_t* tile_rows;
} moe_plan_t;

/* ------------------------------------------------------------------ sizes */

/* Bytes of workspace moe_forward needs for T tokens on `path` (0 on invalid
 * arguments; moe_last_error() says why). The same workspace also serves every
 * single-step entry point that takes one. Contents need no initialisation.
 * MOE_PATH_DECODE with T >= 9 (I % 128 == 0, H % 256 == 0) includes the
 * grouped W4A16 GEMM's buffers in the padded tile layout (x as f16 [P, H],
 * h as f16 [P, I], P = moe_padded_rows(cfg, T)): about 0.68 GB at T = 32 and
 * 0.77 GB at T = 64 for H = 4096, I = 1024, E = 288, k = 8. A decode
 * workspace smaller than that but large enough for the plain decode layout
 * is accepted, and the forward then runs the GEMV form (nvfp4_expert_gemv). */
size_t moe_workspace_size(const moe_config_t* cfg, int32_t T, int32_t path);

/* Bytes of the routing plan arrays for T tokens (one buffer, carved by
 * moe_plan_carve). */
size_t moe_plan_size(const moe_config_t* cfg, int32_t T);

/* Carve a plan out of one device buffer of moe_plan_size() bytes. Host-only
 * pointer arithmetic; launches nothing. */
moe_status_t moe_plan_carve(const moe_config_t* cfg, int32_t T, void* buf, size_t bytes, moe_plan_t* plan);

/* Rows P of the prefill's padded tile layout for T tokens: an upper bound on
 * sum over local experts of ceil(counts/256) * 256, namely
 * floor((A + 255 * min(A, E_local)) / 256) * 256 with A = T*k (0 on invalid
 * arguments). Sizes tile_rows and the quantised activation buffers. */
int64_t moe_padded_rows(const moe_config_t* cfg, int32_t T);

/* Bytes of the prepared weights: the block scales of gate, up and down
 * re-tiled into the 512-byte scale atoms of the tensor-core path
 * (3 * E * I * H / 16 bytes), then the router weight split into three bf16
 * terms (E * 3H * 2 bytes), each part starting on a 256-byte boundary. */
size_t moe_prepared_size(const moe_config_t* cfg);

/*
 * Re-tile the experts' block scales for the prefill path. dst (device,
 * 256-byte aligned, moe_prepared_size() bytes) receives 512-byte scale atoms
 * of 128 rows x 4 K blocks of 16: the scale of atom row m, 16-element block b
 * sits at byte (m%32)*16 + ((m%128)/32)*4 + b%4 of atom (m/128, b/4) (32 lanes
 * x 4 columns x 4 blocks, the layout the 32x128b tensor-memory copy spreads
 * over the four lane quadrants). First gate and up interleaved, atoms
 * [E][I/64][H/64][512] whose 128 rows are gate rows 64 j .. 64 j + 63 then up
 * rows 64 j .. 64 j + 63 of the expert (one N = 128 tile of the gate/up
 * GEMM); then down, atoms [E][H/128][I/64][512]. Requires I % 128 == 0 and
 * H % 256 == 0. Codes are used in place. Then the router weight w fp32 [E, H]
 * as w3 bf16 [E, 3H] = (lo | mid | hi) per row with w = hi + mid + lo exactly
 * (hi: w with the low 16 bits of its encoding cleared; mid: the same applied
 * to w - hi; lo = w - hi - mid), so the prefill's router logits run as one
 * bf16 tensor-core GEMM over K = 3H whose products are exact in the fp32
 * accumulator. Run once per weight set; stream-ordered.
 */
moe_status_t moe_prepare_weights(const moe_config_t* cfg, const moe_weights_t* w, void* dst, size_t dst_bytes,
                                 void* stream);

/* ------------------------------------------------------------ the steps */

/*
 * Router (glm5next_mlp, "The stack this layer runs": gate.weight -> fp32
 * logits -> router_topk; "Traps": the bias steers selection only).
 *   x       bf16 [T, H]
 *   logits  out fp32 [T, E]: l[t,e] = sum_i Wr[e,i] * x[t,i], fp32 accumulate
 *   ids     out int32 [T, k]: top-k of key = fl32(fl32(sigmoid(l)) + bias) in
 *           rank order; equal keys go to the lower expert index. The sigmoid
 *           is evaluated in double and rounded once to fp32.
 *   weights out fp32 [T, k]: rsf * s_j / sum_chosen s with s = fl32 sigmoid
 *           of the chosen experts' logits (unbiased); 0 if the sum is 0.
 * All of the FULL expert count are ranked (local range ignored here).
 */
moe_status_t moe_router_topk(const moe_config_t* cfg, const uint16_t* x, int32_t T,
                             const float* router_w, const float* router_bias,
                             float* logits, int32_t* ids, float* weights, void* stream);

/*
 * Token sort (the module list's moe_permute family): builds `plan` from ids
 * int32 [T, k], including plan.tile_rows. ids outside [0, E) set
 * MOE_ERR_DEVICE_BOUNDS in the workspace status word and are dropped.
 * ws: workspace of at least moe_workspace_size(cfg, T, MOE_PATH_DECODE)
 * bytes (status word and sort scratch).
 */
moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* ids, int32_t T,
                         const moe_plan_t* plan, void* ws, size_t ws_bytes, void* stream);

/*
 * Decode expert projections (the module list's W4A16 GEMV: "Every
 * routed-expert projection here is M=1"): bf16 activations times NVFP4
 * weights, one pass over each touched expert's bytes for all of that expert's
 * tokens. Every product code * activation is exact (the code as f16, the
 * activation scaled by a power of two per row into f16) and accumulates in
 * fp32; each 16-element block sum is scaled by its E4M3 scale in fp32.
 *   MOE_PROJ_GATE_UP: act = x bf16 [T, H]; out = h fp32 [T*k, I] with
 *       h[a] = clamped_swiglu(gate_e . x_t, up_e . x_t) for assignment
 *       a = t*k + j of LOCAL expert e = ids[t, j]; rows of remote
 *       assignments are not written. `weights` is ignored (may be NULL).
 *   MOE_PROJ_DOWN: act = h fp32 [T*k, I] (h enters the products rounded to
 *       11 significant bits); out = r fp32 [T*k, H] with
 *       r[a] = weights[a] * (down_e . h[a]); rows of remote assignments are
 *       written as zeros.
 *   plan: from moe_permute (or moe_forward) for the same ids.
 *   ws:   workspace of at least moe_workspace_size(cfg, T, MOE_PATH_DECODE)
 *         bytes (status word, activation maximum).
 * T = 1 runs the streamed single-token kernels (one CTA per SM, weights
 * through a ring of bulk copies in shared memory); larger T a work-item loop
 * over (active expert, block of rows) that applies each weight row to up to 8
 * of the expert's tokens at once.
 */
moe_status_t nvfp4_expert_gemv(const moe_config_t* cfg, int32_t proj, const void* act, int32_t T,
                               const moe_plan_t* plan, const float* weights,
                               const moe_weights_t* w, float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * NVFP4 encoding of activation rows for the prefill (the reading of the
 * glm5next_mlp module docs' forward_prefill_gemm as W4A4 on block-scaled FP4
 * tensor cores; the pages' own prefill keeps activations in bf16). Every step
 * in IEEE fp32, per row: r = max|row|, row_scale = r / 2688 (2688 = 6 * 448);
 * per block of 16: sb = e4m3_rn_satfinite((amax_block / 6) / row_scale),
 * d = e4m3(sb) * row_scale, code = e2m1_rn_satfinite(v / d). A zero row has
 * row_scale 0 and all scales and codes 0; a block with d = 0 gets codes 0.
 *   src       bf16 [rows, K], K a multiple of 64
 *   codes     out [rows, K/2] (even element in the low nibble)
 *   sf_atoms  out [ceil(rows/128)][K/64][512] in the atom layout of
 *             moe_prepare_weights; rows past `rows` in the last tile get 0
 *   row_scale out fp32 [rows]
 */
moe_status_t nvfp4_quantize_rows(const uint16_t* src, int32_t rows, int32_t K, uint8_t* codes, uint8_t* sf_atoms,
                                 float* row_scale, void* stream);

/*
 * Prefill expert projections (the glm5next_mlp module docs'
 * forward_prefill_gemm: the routed experts as one grouped GEMM over the
 * tokens sorted by expert), here as W4A4 on tcgen05 block-scaled FP4
 * (kind::mxf4nvf4, E4M3 scale per 16 on both operands, fp32 accumulation).
 * The A operand is in the padded tile layout of plan.tile_rows, P =
 * moe_padded_rows(cfg, T) rows: act_codes [P, K/2], act_sf atoms
 * [P/128][K/64][512], act_scale fp32 [P] (from nvfp4_quantize_rows or the
 * prefill of moe_forward); padding rows must be zero (codes, scales, scale).
 *   MOE_PROJ_GATE_UP (K = H): out = h bf16 [P, I], h[p] = clamped_swiglu(
 *       g, u) of padded row p (0 on padding rows); `weights` unused.
 *   MOE_PROJ_DOWN (K = I): out = rows fp32 [P, H] in the padded tile order,
 *       rows[p] = weights[a] * (down_e . hdeq[p]) for the assignment a at
 *       padded row p (0 on padding rows); moe_unpermute /
 *       moe_unpermute_combine bring them back to token order.
 *   Requires w->prepared, I % 128 == 0, H % 256 == 0.
 *   ws: at least moe_workspace_size(cfg, T, MOE_PATH_PREFILL) bytes (status).
 * The kernel runs on clusters of two CTAs (tcgen05.mma.cta_group::2, tiles of
 * 256 rows x 256 weight rows, M split across the pair, each CTA loading half
 * of the weight tile, one TMEM accumulator); no TMA load uses cluster
 * multicast.
 */
moe_status_t nvfp4_grouped_gemm(const moe_config_t* cfg, int32_t proj, const uint8_t* act_codes,
                                const uint8_t* act_sf, const float* act_scale, int32_t T, const moe_plan_t* plan,
                                const float* weights, const moe_weights_t* w, void* out, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * Prefill expert projections in the pages' own numerics (the glm5next_mlp
 * module docs' forward_prefill_gemm: "the shared tensor-core grouped W4A16
 * GEMM"): NVFP4 weights x 16-bit activations on tcgen05 kind::f16, fp32
 * accumulation. The weights are dequantised in shared memory, each element
 * e2m1 x e4m3 exact in f16; the tensor scale is applied in the epilogue. The
 * A operand is f16 in the padded tile layout of plan.tile_rows, P =
 * moe_padded_rows(cfg, T) rows, padding rows zero:
 *   MOE_PROJ_GATE_UP (K = H): act = x rows, each scaled by a power of two
 *       (moe_forward's gather: max |x| into [2^14, 2^15), exact for bf16 x),
 *       act_scale fp32 [P] the inverse; out = h f16 [P, I] =
 *       clamped_swiglu(g, u) (saturating to the f16 range; 0 on padding rows);
 *       `weights` unused.
 *   MOE_PROJ_DOWN (K = I): act = h f16 [P, I]; act_scale NULL (1); out = rows
 *       fp32 [P, H] in the padded tile order, rows[p] = weights[a] *
 *       (down_e . h[p]) (0 on padding rows); moe_unpermute(_combine) brings
 *       them back to token order.
 *   Requires w->prepared (the interleaved gate/up and the down scale atoms),
 *   I % 128 == 0, H % 256 == 0. ws: at least moe_workspace_size(cfg, T,
 *   MOE_PATH_PREFILL_W4A16) bytes (status word).
 * One CTA per 128-row x 256-weight-row tile, 148 persistent CTAs, two TMEM
 * accumulators; no TMA load uses cluster multicast.
 */
moe_status_t nvfp4_grouped_gemm_w4a16(const moe_config_t* cfg, int32_t proj, const uint16_t* act,
                                      const float* act_scale, int32_t T, const moe_plan_t* plan, const float* weights,
                                      const moe_weights_t* w, void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Unpermute (the module list's moe_permute family: token sort / permute /
 * unpermute): rows of the padded tile order back to token order.
 *   rows fp32 [P, H] (nvfp4_grouped_gemm DOWN); ids int32 [T, k] and plan from
 *   the same routing; out fp32 [T, k, H]: out[t, j] = rows[p] with p =
 *   tile_offsets[e] * 256 + inv[a] - offsets[e] for a = t*k + j, e = ids[a]
 *   local; zeros for remote assignments.
 */
moe_status_t moe_unpermute(const moe_config_t* cfg, const float* rows, int32_t T, const moe_plan_t* plan,
                           const int32_t* ids, float* out, void* stream);

/*
 * Unpermute fused with moe_combine (the prefill's last step): y[t] =
 * bf16( sum_{j=0}^{k-1} rows[p(t, j)] + shared[t] ), j ascending, then the
 * unscaled shared row (fp32 [T, H], NULL = none), fp32 accumulation, one
 * rounding; rows fp32 [P, H]; a remote assignment adds a zero row. Same
 * result as moe_unpermute then moe_combine_f32.
 */
moe_status_t moe_unpermute_combine(const moe_config_t* cfg, const float* rows, int32_t T, const moe_plan_t* plan,
                                   const int32_t* ids, const float* shared, uint16_t* y, void* stream);

/*
 * Clamped SwiGLU (glm5next_mlp "Traps": the clamp is asymmetric):
 *   h[m, i] = silu(min(g, L)) * min(max(u, -L), L),  silu(z) = z / (1 + e^-z)
 *   gu fp32 [M, 2*I]: gate in columns [0, I), up in [I, 2I); h bf16 [M, I].
 */
moe_status_t clamped_swiglu(const float* gu, int32_t M, int32_t I, float limit, uint16_t* h, void* stream);

/*
 * moe_combine (glm5next_mlp, "The stack this layer runs" and "Traps"):
 *   y[t] = bf16( (sum_{j=0}^{k-1} r[t, j]) + shared[t] ), fp32 accumulation in
 *   that order; the shared row is added unscaled.
 *   r bf16 [T, k, H]; shared bf16 [T, H] or NULL; y bf16 [T, H].
 */
moe_status_t moe_combine(int32_t T, int32_t k, int32_t H, const uint16_t* r, const uint16_t* shared,
                         uint16_t* y, void* stream);

/*
 * moe_combine over fp32 partials (the decode path keeps the routed rows and
 * the shared row in fp32 until this one rounding): the same order and
 * arithmetic as moe_combine. r fp32 [T, k, H]; shared fp32 [T, H] or NULL;
 * y bf16 [T, H]; H a multiple of 4.
 */
moe_status_t moe_combine_f32(int32_t T, int32_t k, int32_t H, const float* r, const float* shared,
                             uint16_t* y, void* stream);

/*
 * Dense BF16 FFN (glm5next_mlp, DENSE layers; also the shared expert):
 *   y = down_proj( clamped_swiglu(gate_proj x, up_proj x) )
 *   x bf16 [T, H]; wg, wu bf16 [I, H]; wd bf16 [H, I]; y bf16 [T, H].
 *   fp32 accumulation. T >= 128 with I % 128 == 0 and H % 256 == 0 runs as
 *   two tcgen05 BF16 GEMMs (kind::f16; h is rounded to bf16, the second
 *   GEMM's operand type); smaller T as a GEMV that streams the weights once
 *   per group of up to 8 tokens and keeps h in fp32. H and I multiples of 64.
 *   ws: at least dense_ffn_workspace_size(H, I, T); its first 4 bytes are a
 *   device status word (moe_read_device_status).
 */
size_t dense_ffn_workspace_size(int32_t H, int32_t I, int32_t T);
moe_status_t dense_ffn_bf16(int32_t H, int32_t I, float limit, const uint16_t* x, int32_t T,
                            const uint16_t* wg, const uint16_t* wu, const uint16_t* wd, uint16_t* y,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * NVFP4 dequantisation (debug / bit-exact check of the format):
 *   out fp32 [rows, K] = e2m1(code) * e4m3(scale) * tensor_scale[0]
 *   codes [rows, K/2], scales [rows, K/16] canonical; K multiple of 16.
 *   The fp32 product is exact whenever it is a normal fp32 number.
 */
moe_status_t nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                           int32_t rows, int32_t K, float* out, void* stream);

/* ------------------------------------------------------------ whole site */

/*
 * One routed site forward: router, top-k, experts (path), shared expert,
 * combine. x bf16 [T, H] -> y bf16 [T, H]. ws: moe_workspace_size(cfg, T,
 * path) bytes. The routing plan, logits, ids and weights of the call stay in
 * the workspace until the next call (see moe_workspace_views).
 *   MOE_PATH_DECODE: W4A16 GEMV experts (nvfp4_expert_gemv) with h, the
 *     routed rows r and the shared row kept in fp32 up to the combine's one
 *     bf16 rounding.
 *     Launches, chained by programmatic dependent launch: router logits
 *     (with max |x| per token); top-k with the routing plan (one launch up to
 *     8 tokens, E <= 320, else top-k and the permute); the routed experts'
 *     gate/up and down; moe_combine_f32. The shared expert runs on the
 *     library's auxiliary stream of this host thread and device, forked from
 *     and joined back into `stream` with events.
 *     T <= 8 with H % 1024 == 0, H <= 8192, I % 128 == 0, I <= 2048, k <= 16,
 *     E <= 1024: the expert projections run on the tensor cores, each warp
 *     loading its weight rows straight into registers with 128-bit loads and
 *     multiplying them with mma.sync (each E2M1 code times its E4M3 scale
 *     exact in f16, x or h scaled by a power of two into f16, fp32
 *     accumulation). T >= 9 with I % 128 == 0, H % 256 == 0, w->prepared set
 *     and ws of at least moe_workspace_size(cfg, T, MOE_PATH_DECODE) bytes:
 *     the grouped W4A16 GEMM of MOE_PATH_PREFILL_W4A16 (x gathered to f16
 *     rows, h in f16, the same exact-product numerics), skipping the 128-row
 *     halves of the padded tile layout that hold only padding, with the down
 *     GEMM writing r in assignment order. Otherwise the GEMV kernels of
 *     nvfp4_expert_gemv.
 *   MOE_PATH_PREFILL_W4A16: the pages' prefill numerics: permute with the
 *     padded tile layout, x gathered to f16 rows (per-row power-of-two scale),
 *     grouped W4A16 GEMM gate/up (nvfp4_grouped_gemm_w4a16) with the clamped
 *     SwiGLU, h in f16, grouped W4A16 GEMM down with the routing weight,
 *     unpermute fused with the combine; needs w->prepared, I % 128 == 0,
 *     H % 256 == 0.
 *   MOE_PATH_PREFILL: permute with the padded tile layout, x encoded to
 *     NVFP4 per token row and written to its assignments' padded rows (the
 *     bytes nvfp4_quantize_rows gives per assignment row), grouped GEMM
 *     gate/up with the clamped SwiGLU, h rounded to bf16 and encoded to NVFP4
 *     per row, grouped GEMM down with the routing weight, unpermute fused with
 *     the combine; needs w->prepared, I % 128 == 0, H % 256 == 0.
 */
moe_status_t moe_forward(const moe_config_t* cfg, const moe_weights_t* w, const uint16_t* x, int32_t T,
                         int32_t path, uint16_t* y, void* ws, size_t ws_bytes, void* stream);

/* Device pointers (inside ws) of the intermediates moe_forward leaves behind:
 * logits fp32 [T,E], ids int32 [T,k], weights fp32 [T,k], the plan; h (decode:
 * fp32 [T*k, I], or f16 [P, I] in padded tile rows when the decode ran on the
 * grouped W4A16 GEMM; prefill: [P, I] in padded tile rows, bf16 on
 * MOE_PATH_PREFILL, f16 on MOE_PATH_PREFILL_W4A16); r (fp32; decode: [T*k, H] in token order;
 * prefill: [P, H] in the padded tile order); shared (fp32 [T, H]; NULL when
 * Is == 0); and on MOE_PATH_PREFILL the NVFP4-encoded x and h in padded tile
 * rows (codes, scale atoms, row scales; NULL otherwise). Host-only pointer
 * arithmetic. */
typedef struct {
  float* logits;
  int32_t* ids;
  float* weights;
  moe_plan_t plan;
  void* h;
  void* r;
  void* shared;
  uint8_t* xq_codes;
  uint8_t* xq_sf;
  float* xq_scale;
  uint8_t* hq_codes;
  uint8_t* hq_sf;
  float* hq_scale;
} moe_views_t;
moe_status_t moe_workspace_views(const moe_config_t* cfg, int32_t T, int32_t path, void* ws, size_t ws_bytes,
                                 moe_views_t* views);

/*
 * Optional stage timing of moe_forward (profiling hook; thread-local state).
 * `events` holds n cudaEvent_t handles the caller created (timing enabled);
 * while set, moe_forward records events[s] on its stream before stage s, for
 * every s < n - 1 up to the last stage, and events[n-1] after the last stage.
 * Stages are numbered by moe_stage_t whichever path runs; a stage the path
 * does not have is recorded with zero length; a NULL entry is not recorded.
 * Under stream capture the records become graph event nodes
 * (cudaEventRecordExternal). n must be 0 (off, events may be NULL) or
 * MOE_STAGE_COUNT + 1.
 */
typedef enum {
  MOE_STAGE_ROUTER_LOGITS = 0,
  MOE_STAGE_TOPK = 1,
  MOE_STAGE_PERMUTE = 2,
  MOE_STAGE_ACT_QUANT = 3,
  MOE_STAGE_EXPERT_GATE_UP = 4,
  MOE_STAGE_H_QUANT = 5,
  MOE_STAGE_EXPERT_DOWN = 6,
  MOE_STAGE_SHARED = 7,
  MOE_STAGE_COMBINE = 8,
  MOE_STAGE_COUNT = 9
} moe_stage_t;
moe_status_t moe_set_stage_events(void* const* events, int32_t n);

/*
 * Test hook of the failure path (not for production use; process-wide host
 * setting read at launch): the limit of the main-loop waits of the BF16
 * tensor-core GEMM (dense_ffn_bf16 / the shared expert at T >= 128, the
 * prefill router). ns >= 0 sets it (0 = a wait gives up as soon as it finds
 * the awaited copy or MMA still in flight); ns < 0 restores the default 2 s.
 * A wait that runs out sets MOE_ERR_DEVICE_TIMEOUT in the status word; the
 * kernel then issues nothing more, waits with the default limit for every copy
 * and MMA it already issued, frees its tensor memory and returns, so later
 * calls on the device run normally. The outputs of the failed call are
 * unspecified.
 */
moe_status_t moe_set_wait_limit(int64_t ns);

/* Synchronises `stream`, reads the workspace status word, clears it, and
 * returns MOE_ERR_DEVICE_TIMEOUT / MOE_ERR_DEVICE_BOUNDS / MOE_OK. */
moe_status_t moe_read_device_status(void* ws, void* stream);

/* Thread-local description of the last failed call on this thread ("" if none). */
const char* moe_last_error(void);

/*
 * Decode forward without a caller workspace -- no counterpart in the pages:
 * it exists for callers that cannot allocate device memory (a memory pool or
 * custom allocator that forbids cudaMalloc, a framework callback that may not
 * allocate, a C host program holding only the device pointers of its tensors).
 * Same computation and arguments as moe_forward(cfg, w, x, T,
 * MOE_PATH_DECODE, y, ws, ws_bytes, stream), minus the workspace: the scratch
 * is a library-owned 8 MiB device buffer that every GPU loading the library
 * keeps until the process exits. Calls needing more than that
 * (moe_workspace_size(cfg, T, MOE_PATH_DECODE) > 8 MiB) fail with
 * MOE_ERR_WORKSPACE before touching the device. The first call on each device
 * looks up the buffer's device address (cudaGetSymbolAddress, with that device
 * current) and caches it for the life of the process: make that first call
 * before any stream capture on the device, and make no call on a device after
 * cudaDeviceReset() of it (the cached address would be stale). All calls on a
 * device share the buffer, which keeps the previous call's contents; calls
 * whose GPU work overlaps in time (two streams, two host threads) race on it
 * and must be serialised by the caller. Allocates nothing (no cudaMalloc /
 * cudaFree). The routing intermediates are not exposed.
 */
moe_status_t moe_forward_decode_noalloc(const moe_config_t* cfg, const moe_weights_t* w, const uint16_t* x,
                                        int32_t T, uint16_t* y, void* stream);

/*
 * Device-side errors of the last moe_forward_decode_noalloc call on the
 * current device (an id out of range, a bounded wait that ran out): the status
 * word sits at the start of the library's scratch buffer, where a caller has no
 * pointer to it. Synchronises `stream`, reads and clears the word, and returns
 * MOE_ERR_DEVICE_TIMEOUT / MOE_ERR_DEVICE_BOUNDS / MOE_OK, as
 * moe_read_device_status does for a caller's workspace. The next
 * moe_forward_decode_noalloc call clears the word as well.
 */
moe_status_t moe_noalloc_read_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROUTED_NVFP4_H */
