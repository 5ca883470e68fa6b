// C ABI of the routed NVFP4 MoE site: argument validation, workspace layout,
// and the order of launches. Every device step runs in the kernels of this
// library; nothing here computes on the host.

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace {

thread_local char g_err[512] = "";

// Decode runs the shared expert on an auxiliary stream, concurrently with the
// router, the routing plan and the routed experts (it only needs x): per host
// thread and device, one non-blocking stream and a fork / join event pair,
// created on first use (before any stream capture) and kept for the process.
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
thread_local SideStream g_side[kMaxDevices];

cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  SideStream& s = g_side[dev];
  if (!s.st || !s.fork || !s.join) {
    // all three handles or none: a partial creation is undone and reported
    SideStream n;
    e = cudaStreamCreateWithFlags(&n.st, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (n.join) cudaEventDestroy(n.join);
      if (n.fork) cudaEventDestroy(n.fork);
      if (n.st) cudaStreamDestroy(n.st);
      return e;
    }
    s = n;
  }
  *out = &s;
  return cudaSuccess;
}
thread_local cudaEvent_t g_stage_ev[MOE_STAGE_COUNT + 1];
thread_local int g_n_stage_ev = 0;

// Record the stage-timing event before `stage` (or after the last stage when
// stage == MOE_STAGE_COUNT), if the caller registered events.
cudaError_t mark(int stage, cudaStream_t st) {
  if (g_n_stage_ev <= stage || !g_stage_ev[stage]) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(g_stage_ev[stage], st, cudaEventRecordExternal);
  return cudaEventRecord(g_stage_ev[stage], st);
}

moe_status_t fail(moe_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

moe_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define RNX_CUDA(call, where)                      \
  do {                                             \
    cudaError_t e_ = (call);                       \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

#define RNX_PTR(p, name)                                                              \
  do {                                                                                \
    if (!(p)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);                   \
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 16;            // KERNEL_MAX_TOP_K
constexpr size_t kAlign = 256;

size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

moe_status_t check_cfg(const moe_config_t* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
  if (c->hidden <= 0 || c->hidden % 64) return fail(MOE_ERR_INVALID_ARG, "hidden=%d must be a positive multiple of 64", c->hidden);
  if (c->intermediate <= 0 || c->intermediate % 64)
    return fail(MOE_ERR_INVALID_ARG, "intermediate=%d must be a positive multiple of 64", c->intermediate);
  if (c->shared_intermediate < 0 || c->shared_intermediate % 64)
    return fail(MOE_ERR_INVALID_ARG, "shared_intermediate=%d must be 0 or a multiple of 64", c->shared_intermediate);
  if (c->num_experts <= 0) return fail(MOE_ERR_INVALID_ARG, "num_experts=%d must be positive", c->num_experts);
  if (c->num_experts > kMaxExperts)
    return fail(MOE_ERR_UNSUPPORTED, "num_experts=%d above the supported %d", c->num_experts, kMaxExperts);
  if (c->local_begin < 0 || c->local_begin > c->local_end || c->local_end > c->num_experts)
    return fail(MOE_ERR_INVALID_ARG, "local range [%d,%d) not inside [0,%d)", c->local_begin, c->local_end, c->num_experts);
  if (c->top_k < 1 || c->top_k > kMaxTopK || c->top_k > c->num_experts)
    return fail(MOE_ERR_INVALID_ARG, "top_k=%d must be in 1..min(16, num_experts)", c->top_k);
  if (!std::isfinite(c->routed_scaling_factor)) return fail(MOE_ERR_INVALID_ARG, "routed_scaling_factor is not finite");
  if (std::isnan(c->swiglu_limit) || !(c->swiglu_limit > 0.f))
    return fail(MOE_ERR_INVALID_ARG, "swiglu_limit must be > 0 (inf allowed, NaN rejected)");
  return MOE_OK;
}

moe_status_t check_T(int32_t T) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d is negative", T);
  if ((int64_t)T * kMaxTopK > (1LL << 30)) return fail(MOE_ERR_UNSUPPORTED, "T=%d too large", T);
  return MOE_OK;
}

moe_status_t check_bank(const nvfp4_bank_t& b, const char* name) {
  char buf[64];
  snprintf(buf, sizeof buf, "%s.codes", name);
  RNX_PTR(b.codes, buf);
  snprintf(buf, sizeof buf, "%s.scales", name);
  RNX_PTR(b.scales, buf);
  snprintf(buf, sizeof buf, "%s.tensor_scale", name);
  if (!b.tensor_scale) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", buf);
  return MOE_OK;
}

// ------------------------------------------------------------ layouts

struct PlanLayout {
  size_t counts, offsets, sorted, inv, tile_offsets, active, first, tile_rows, bytes;
  int64_t P;   // rows of the padded tile layout
};

int64_t padded_rows(const moe_config_t* c, int64_t A) {
  return rnx::padded_rows_bound(A, (int64_t)c->local_end - c->local_begin);
}

PlanLayout plan_layout(const moe_config_t* c, int A) {
  const int E = c->num_experts;
  PlanLayout L{};
  L.P = padded_rows(c, A);
  size_t o = 0;
  L.counts = o; o = up(o + 4 * (size_t)E);
  L.offsets = o; o = up(o + 4 * (size_t)(E + 1));
  L.sorted = o; o = up(o + 4 * (size_t)A);
  L.inv = o; o = up(o + 4 * (size_t)A);
  L.tile_offsets = o; o = up(o + 4 * (size_t)(E + 1));
  L.active = o; o = up(o + 4 * (size_t)(E + 1));
  L.first = o; o = up(o + 4 * (size_t)E);
  L.tile_rows = o; o = up(o + 4 * (size_t)L.P);
  L.bytes = o;
  return L;
}

moe_plan_t plan_at(char* base, const PlanLayout& L) {
  moe_plan_t p;
  p.counts = (int32_t*)(base + L.counts);
  p.offsets = (int32_t*)(base + L.offsets);
  p.sorted = (int32_t*)(base + L.sorted);
  p.inv = (int32_t*)(base + L.inv);
  p.tile_offsets = (int32_t*)(base + L.tile_offsets);
  p.active = (int32_t*)(base + L.active);
  p.first = (int32_t*)(base + L.first);
  p.tile_rows = (int32_t*)(base + L.tile_rows);
  return p;
}

struct WsLayout {
  size_t status, logits, ids, weights, plan, scratch, h, r, shared_h, shared, xmax;
  size_t xq, xsf, xts, hq, hsf, hts;   // prefill: NVFP4 x and h in padded tile rows
  size_t bytes;
  PlanLayout pl;
  bool grouped;   // decode layout with the grouped W4A16 GEMM's buffers
};

// Control block at the start of every workspace, cleared at the start of each
// call that uses it: the device status word, then the single-token router's
// arrival counter.
constexpr size_t kCtrlBytes = 16;

// Decode batches of more tokens than the tensor-core GEMV takes run their
// experts on the grouped W4A16 GEMM (same numerics: 16-bit activations, each
// weight exact in f16, fp32 accumulation) when the shapes fit it, the
// prepared scale atoms exist and the workspace holds its buffers.
constexpr int kDecodeGroupedMinT = 9;
bool decode_grouped_shape(const moe_config_t* c, int T) {
  return T >= kDecodeGroupedMinT && c->intermediate % 128 == 0 && c->hidden % 256 == 0;
}

// grouped: decode layout with the grouped GEMM's buffers (-1: whenever the
// shapes allow it, as moe_workspace_size sizes it)
WsLayout ws_layout(const moe_config_t* c, int T, int path, int grouped = -1) {
  WsLayout L{};
  const int E = c->num_experts, k = c->top_k, H = c->hidden, I = c->intermediate, Is = c->shared_intermediate;
  const size_t A = (size_t)T * k;
  size_t o = 0;
  L.status = o; o = up(o + kCtrlBytes);
  L.logits = o; o = up(o + 4 * (size_t)T * E);
  L.ids = o; o = up(o + 4 * A);
  L.weights = o; o = up(o + 4 * A);
  L.pl = plan_layout(c, (int)A);
  L.plan = o; o = up(o + L.pl.bytes);
  L.scratch = o; o = up(o + 4 * rnx::permute_scratch_ints((int)A, E));
  const bool w4 = path == MOE_PATH_PREFILL_W4A16;
  const bool pre = path == MOE_PATH_PREFILL || w4;
  const bool grp = path == MOE_PATH_DECODE && (grouped < 0 ? decode_grouped_shape(c, T) : grouped != 0);
  const size_t P = (size_t)L.pl.P;
  L.grouped = grp;
  // the routed rows r and the shared row are fp32 on every path (the combine
  // sums them in fp32 and rounds y once); h is fp32 at decode, 16-bit in the
  // prefill's padded tile rows (and in the decode's, on the grouped GEMM,
  // whose down GEMM writes r in assignment order)
  L.h = o; o = up(o + (pre ? 2 * P : grp ? std::max(2 * P, 4 * A) : 4 * A) * I);
  L.r = o; o = up(o + 4 * (pre ? P : A) * H);   // prefill: down rows in the padded tile order
  L.shared_h = o; o = up(o + 4 * (size_t)T * Is);
  L.shared = o; o = up(o + 4 * (size_t)T * H);
  L.xmax = o; o = up(o + 4 * (size_t)T);
  if (w4 || grp) {                            // x as f16 rows in the padded tile order, their unscales
    L.xq = o; o = up(o + P * H * 2);
    L.xts = o; o = up(o + 4 * P);
  } else if (pre) {
    L.xq = o; o = up(o + P * H / 2);
    L.xsf = o; o = up(o + P * H / 16);
    L.xts = o; o = up(o + 4 * P);
    L.hq = o; o = up(o + P * I / 2);
    L.hsf = o; o = up(o + P * I / 16);
    L.hts = o; o = up(o + 4 * P);
  }
  L.bytes = o;
  return L;
}

// Shapes the tensor-core prefill path covers.
moe_status_t check_prefill_shape(const moe_config_t* c) {
  if (c->intermediate % 128) return fail(MOE_ERR_UNSUPPORTED, "prefill needs intermediate %% 128 == 0 (got %d)", c->intermediate);
  if (c->hidden % 256) return fail(MOE_ERR_UNSUPPORTED, "prefill needs hidden %% 256 == 0 (got %d)", c->hidden);
  return MOE_OK;
}

// Prepared weights: the experts' block scales as 512-byte atoms -- gate and
// up interleaved (each 128-row atom = 64 gate rows, then the same 64 up rows),
// then down -- and the router weight split exactly into three bf16 terms
// [E, 3H].
struct PreparedLayout {
  size_t gate_up, down, router3, bytes;
};
PreparedLayout prepared_layout(const moe_config_t* c) {
  const size_t per = (size_t)c->num_experts * c->intermediate * c->hidden / 16;
  const size_t r3 = up(3 * per);
  return PreparedLayout{0, 2 * per, r3, r3 + up((size_t)c->num_experts * 3 * c->hidden * 2)};
}

// Prefill router on the tensor cores (needs the prepared split and E % 4 == 0).
bool router_on_tensor_cores(const moe_config_t* c, int T, const moe_weights_t* w) {
  return w->prepared && T >= rnx::kDenseGemmMinT && c->num_experts % 4 == 0;
}

rnx::Fp4GemmArgs gemm_args(const moe_config_t* c, int proj, const uint8_t* codes, const uint8_t* sf,
                           const float* scale, int64_t P, const moe_plan_t& plan, const float* weights,
                           const moe_weights_t* w, void* out, uint32_t* status) {
  const PreparedLayout PL = prepared_layout(c);
  rnx::Fp4GemmArgs g{};
  g.gate_up = proj == MOE_PROJ_GATE_UP;
  g.E = c->num_experts;
  g.K = g.gate_up ? c->hidden : c->intermediate;
  g.out_cols = g.gate_up ? c->intermediate : c->hidden;
  g.bank_rows = g.gate_up ? c->intermediate : c->hidden;
  g.P_max = P;
  g.limit = c->swiglu_limit;
  g.a_codes = codes;
  g.a_sf = sf;
  g.row_scale = scale;
  if (g.gate_up) {
    g.b0_codes = w->gate.codes; g.b0_sf = w->prepared + PL.gate_up; g.ts0 = w->gate.tensor_scale;
    g.b1_codes = w->up.codes;   g.b1_sf = nullptr;                   g.ts1 = w->up.tensor_scale;
  } else {
    g.b0_codes = w->down.codes; g.b0_sf = w->prepared + PL.down; g.ts0 = w->down.tensor_scale;
  }
  g.tile_offsets = plan.tile_offsets;
  g.tile_rows = plan.tile_rows;
  g.weights = weights;
  g.out = out;
  g.status = status;
  return g;
}

rnx::W4a16GemmArgs w4a16_args(const moe_config_t* c, int proj, const uint16_t* act, const float* act_scale,
                              int64_t P, const moe_plan_t& plan, const float* weights, const moe_weights_t* w,
                              void* out, uint32_t* status) {
  const PreparedLayout PL = prepared_layout(c);
  rnx::W4a16GemmArgs g{};
  g.gate_up = proj == MOE_PROJ_GATE_UP;
  g.E = c->num_experts;
  g.K = g.gate_up ? c->hidden : c->intermediate;
  g.out_cols = g.gate_up ? c->intermediate : c->hidden;
  g.bank_rows = g.gate_up ? c->intermediate : c->hidden;
  g.P_max = P;
  g.limit = c->swiglu_limit;
  g.act = act;
  g.row_scale = act_scale;
  if (g.gate_up) {
    g.b0_codes = w->gate.codes; g.b1_codes = w->up.codes; g.b_sf = w->prepared + PL.gate_up;
    g.ts0 = w->gate.tensor_scale; g.ts1 = w->up.tensor_scale;
  } else {
    g.b0_codes = w->down.codes; g.b_sf = w->prepared + PL.down; g.ts0 = w->down.tensor_scale;
  }
  g.tile_offsets = plan.tile_offsets;
  g.tile_rows = plan.tile_rows;
  g.weights = weights;
  g.out = out;
  g.status = status;
  return g;
}

// The layout a call uses: the decode's grouped-GEMM layout whenever the
// shapes allow it and the workspace holds it (moe_forward and
// moe_workspace_views apply the same rule), else the plain one.
moe_status_t check_ws(const moe_config_t* c, int T, int path, void* ws, size_t ws_bytes, WsLayout* L) {
  const bool grp = path == MOE_PATH_DECODE && decode_grouped_shape(c, T) && ws_bytes >= ws_layout(c, T, path, 1).bytes;
  *L = ws_layout(c, T, path, grp ? 1 : 0);
  if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if (((uintptr_t)ws % kAlign) != 0) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < L->bytes) return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L->bytes);
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_last_error(void) { return g_err; }

moe_status_t moe_set_stage_events(void* const* events, int32_t n) {
  if (n == 0) {
    g_n_stage_ev = 0;
    return MOE_OK;
  }
  if (n != MOE_STAGE_COUNT + 1 || !events) return fail(MOE_ERR_INVALID_ARG, "need %d stage events", MOE_STAGE_COUNT + 1);
  for (int i = 0; i < n; ++i) g_stage_ev[i] = (cudaEvent_t)events[i];   // NULL entries are skipped
  g_n_stage_ev = n;
  return MOE_OK;
}

size_t moe_workspace_size(const moe_config_t* cfg, int32_t T, int32_t path) {
  if (check_cfg(cfg) != MOE_OK || check_T(T) != MOE_OK) return 0;
  if (path != MOE_PATH_DECODE && path != MOE_PATH_PREFILL && path != MOE_PATH_PREFILL_W4A16) {
    fail(MOE_ERR_INVALID_ARG, "unknown path %d", path);
    return 0;
  }
  return ws_layout(cfg, T, path).bytes;
}

size_t moe_plan_size(const moe_config_t* cfg, int32_t T) {
  if (check_cfg(cfg) != MOE_OK || check_T(T) != MOE_OK) return 0;
  return plan_layout(cfg, T * cfg->top_k).bytes;
}

moe_status_t moe_plan_carve(const moe_config_t* cfg, int32_t T, void* buf, size_t bytes, moe_plan_t* plan) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  const PlanLayout L = plan_layout(cfg, T * cfg->top_k);
  if (!buf || ((uintptr_t)buf % kAlign)) return fail(MOE_ERR_INVALID_ARG, "plan buffer NULL or not 256-byte aligned");
  if (bytes < L.bytes) return fail(MOE_ERR_WORKSPACE, "plan buffer has %zu bytes, needs %zu", bytes, L.bytes);
  *plan = plan_at((char*)buf, L);
  return MOE_OK;
}

moe_status_t moe_workspace_views(const moe_config_t* cfg, int32_t T, int32_t path, void* ws, size_t ws_bytes,
                                 moe_views_t* v) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (!v) return fail(MOE_ERR_INVALID_ARG, "views is NULL");
  WsLayout L;
  if ((s = check_ws(cfg, T, path, ws, ws_bytes, &L)) != MOE_OK) return s;
  char* b = (char*)ws;
  v->logits = (float*)(b + L.logits);
  v->ids = (int32_t*)(b + L.ids);
  v->weights = (float*)(b + L.weights);
  v->plan = plan_at(b + L.plan, L.pl);
  v->h = b + L.h;
  v->r = b + L.r;
  v->shared = cfg->shared_intermediate > 0 ? b + L.shared : nullptr;
  const bool pre = path == MOE_PATH_PREFILL, w4 = path == MOE_PATH_PREFILL_W4A16;
  v->xq_codes = pre || w4 ? (uint8_t*)(b + L.xq) : nullptr;   // W4A16: the f16 x rows
  v->xq_sf = pre ? (uint8_t*)(b + L.xsf) : nullptr;
  v->xq_scale = pre || w4 ? (float*)(b + L.xts) : nullptr;
  v->hq_codes = pre ? (uint8_t*)(b + L.hq) : nullptr;
  v->hq_sf = pre ? (uint8_t*)(b + L.hsf) : nullptr;
  v->hq_scale = pre ? (float*)(b + L.hts) : nullptr;
  return MOE_OK;
}

int64_t moe_padded_rows(const moe_config_t* cfg, int32_t T) {
  if (check_cfg(cfg) != MOE_OK || check_T(T) != MOE_OK) return 0;
  return padded_rows(cfg, (int64_t)T * cfg->top_k);
}

size_t moe_prepared_size(const moe_config_t* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return prepared_layout(cfg).bytes;
}

moe_status_t moe_prepare_weights(const moe_config_t* cfg, const moe_weights_t* w, void* dst, size_t dst_bytes,
                                 void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_prefill_shape(cfg)) != MOE_OK) return s;
  if (!w) return fail(MOE_ERR_INVALID_ARG, "weights struct is NULL");
  if ((s = check_bank(w->gate, "gate")) != MOE_OK || (s = check_bank(w->up, "up")) != MOE_OK ||
      (s = check_bank(w->down, "down")) != MOE_OK)
    return s;
  RNX_PTR(w->router_w, "router_w");
  const PreparedLayout PL = prepared_layout(cfg);
  if (!dst || ((uintptr_t)dst % kAlign)) return fail(MOE_ERR_INVALID_ARG, "dst NULL or not 256-byte aligned");
  if (dst_bytes < PL.bytes) return fail(MOE_ERR_WORKSPACE, "dst has %zu bytes, needs %zu", dst_bytes, PL.bytes);
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* d = (uint8_t*)dst;
  const int E = cfg->num_experts, H = cfg->hidden, I = cfg->intermediate;
  RNX_CUDA(rnx::launch_sf_atoms_gate_up(w->gate.scales, w->up.scales, E, I, H, d + PL.gate_up, st),
           "prepare gate/up scales");
  RNX_CUDA(rnx::launch_sf_atoms(w->down.scales, E, H, I, d + PL.down, st), "prepare down scales");
  RNX_CUDA(rnx::launch_router_split(w->router_w, E, H, (uint16_t*)(d + PL.router3), st), "prepare router split");
  return MOE_OK;
}

moe_status_t nvfp4_quantize_rows(const uint16_t* src, int32_t rows, int32_t K, uint8_t* codes, uint8_t* sf_atoms,
                                 float* row_scale, void* stream) {
  if (rows < 0 || K <= 0 || K % 64) return fail(MOE_ERR_INVALID_ARG, "rows=%d K=%d: K must be a positive multiple of 64", rows, K);
  if (rows == 0) return MOE_OK;
  RNX_PTR(src, "src");
  RNX_PTR(codes, "codes");
  RNX_PTR(sf_atoms, "sf_atoms");
  RNX_PTR(row_scale, "row_scale");
  RNX_CUDA(rnx::launch_quant_rows(src, rows, K, nullptr, 0, nullptr, codes, sf_atoms, row_scale, (cudaStream_t)stream),
           "nvfp4_quantize_rows");
  return MOE_OK;
}

moe_status_t nvfp4_grouped_gemm(const moe_config_t* cfg, int32_t proj, const uint8_t* act_codes,
                                const uint8_t* act_sf, const float* act_scale, int32_t T, const moe_plan_t* plan,
                                const float* weights, const moe_weights_t* w, void* out, void* ws,
                                size_t ws_bytes, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK || (s = check_prefill_shape(cfg)) != MOE_OK)
    return s;
  if (proj != MOE_PROJ_GATE_UP && proj != MOE_PROJ_DOWN) return fail(MOE_ERR_INVALID_ARG, "unknown proj %d", proj);
  if (T == 0) return MOE_OK;
  RNX_PTR(act_codes, "act_codes");
  RNX_PTR(act_sf, "act_sf");
  RNX_PTR(act_scale, "act_scale");
  RNX_PTR(out, "out");
  if (!plan || !w) return fail(MOE_ERR_INVALID_ARG, "plan / weights struct is NULL");
  RNX_PTR(plan->tile_offsets, "plan.tile_offsets");
  RNX_PTR(plan->tile_rows, "plan.tile_rows");
  RNX_PTR(w->prepared, "prepared");
  if (proj == MOE_PROJ_GATE_UP) {
    if ((s = check_bank(w->gate, "gate")) != MOE_OK || (s = check_bank(w->up, "up")) != MOE_OK) return s;
  } else {
    if ((s = check_bank(w->down, "down")) != MOE_OK) return s;
    RNX_PTR(weights, "weights");
    RNX_PTR(plan->offsets, "plan.offsets");
    RNX_PTR(plan->sorted, "plan.sorted");
  }
  WsLayout L;
  if ((s = check_ws(cfg, T, MOE_PATH_PREFILL, ws, ws_bytes, &L)) != MOE_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* b = (char*)ws;
  uint32_t* status = (uint32_t*)(b + L.status);
  RNX_CUDA(cudaMemsetAsync(status, 0, 4, st), "clear status");
  const rnx::Fp4GemmArgs g = gemm_args(cfg, proj, act_codes, act_sf, act_scale, L.pl.P, *plan, weights, w, out, status);
  RNX_CUDA(rnx::launch_fp4_grouped_gemm(g, st), "nvfp4_grouped_gemm");
  return MOE_OK;
}

moe_status_t nvfp4_grouped_gemm_w4a16(const moe_config_t* cfg, int32_t proj, const uint16_t* act,
                                      const float* act_scale, int32_t T, const moe_plan_t* plan, const float* weights,
                                      const moe_weights_t* w, void* out, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK || (s = check_prefill_shape(cfg)) != MOE_OK)
    return s;
  if (proj != MOE_PROJ_GATE_UP && proj != MOE_PROJ_DOWN) return fail(MOE_ERR_INVALID_ARG, "unknown proj %d", proj);
  if (T == 0) return MOE_OK;
  RNX_PTR(act, "act");
  RNX_PTR(out, "out");
  if (act_scale && !aligned16(act_scale)) return fail(MOE_ERR_INVALID_ARG, "act_scale is not 16-byte aligned");
  if (!plan || !w) return fail(MOE_ERR_INVALID_ARG, "plan / weights struct is NULL");
  RNX_PTR(plan->tile_offsets, "plan.tile_offsets");
  RNX_PTR(plan->tile_rows, "plan.tile_rows");
  RNX_PTR(w->prepared, "prepared");
  if (proj == MOE_PROJ_GATE_UP) {
    if ((s = check_bank(w->gate, "gate")) != MOE_OK || (s = check_bank(w->up, "up")) != MOE_OK) return s;
  } else {
    if ((s = check_bank(w->down, "down")) != MOE_OK) return s;
    RNX_PTR(weights, "weights");
  }
  WsLayout L;
  if ((s = check_ws(cfg, T, MOE_PATH_PREFILL_W4A16, ws, ws_bytes, &L)) != MOE_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* status = (uint32_t*)((char*)ws + L.status);
  RNX_CUDA(cudaMemsetAsync(status, 0, 4, st), "clear status");
  const rnx::W4a16GemmArgs g = w4a16_args(cfg, proj, act, act_scale, L.pl.P, *plan, weights, w, out, status);
  RNX_CUDA(rnx::launch_w4a16_grouped_gemm(g, st), "nvfp4_grouped_gemm_w4a16");
  return MOE_OK;
}

moe_status_t moe_unpermute(const moe_config_t* cfg, const float* rows, int32_t T, const moe_plan_t* plan,
                           const int32_t* ids, float* out, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  RNX_PTR(rows, "rows");
  RNX_PTR(ids, "ids");
  RNX_PTR(out, "out");
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  RNX_PTR(plan->offsets, "plan.offsets");
  RNX_PTR(plan->inv, "plan.inv");
  RNX_PTR(plan->tile_offsets, "plan.tile_offsets");
  const rnx::PaddedIndex q{ids, plan->inv, plan->offsets, plan->tile_offsets, cfg->local_begin, cfg->local_end};
  RNX_CUDA(rnx::launch_unpermute(q, (long long)T * cfg->top_k, cfg->hidden, rows, out, (cudaStream_t)stream),
           "moe_unpermute");
  return MOE_OK;
}

moe_status_t moe_unpermute_combine(const moe_config_t* cfg, const float* rows, int32_t T, const moe_plan_t* plan,
                                   const int32_t* ids, const float* shared, uint16_t* y, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  RNX_PTR(rows, "rows");
  RNX_PTR(ids, "ids");
  RNX_PTR(y, "y");
  if (shared && !aligned16(shared)) return fail(MOE_ERR_INVALID_ARG, "shared is not 16-byte aligned");
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  RNX_PTR(plan->offsets, "plan.offsets");
  RNX_PTR(plan->inv, "plan.inv");
  RNX_PTR(plan->tile_offsets, "plan.tile_offsets");
  const rnx::PaddedIndex q{ids, plan->inv, plan->offsets, plan->tile_offsets, cfg->local_begin, cfg->local_end};
  RNX_CUDA(rnx::launch_unpermute_combine(q, T, cfg->top_k, cfg->hidden, rows, shared, y, (cudaStream_t)stream),
           "moe_unpermute_combine");
  return MOE_OK;
}

moe_status_t moe_set_wait_limit(int64_t ns) {
  if (ns < 0) {
    rnx::set_test_wait_limit_ns(rnx::kWaitLimitNs);
    return MOE_OK;
  }
  rnx::set_test_wait_limit_ns((unsigned long long)ns);
  return MOE_OK;
}

moe_status_t moe_read_device_status(void* ws, void* stream) {
  if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  RNX_CUDA(cudaStreamSynchronize(st), "cudaStreamSynchronize");
  uint32_t word = 0;
  RNX_CUDA(cudaMemcpy(&word, ws, sizeof word, cudaMemcpyDeviceToHost), "cudaMemcpy(status)");
  RNX_CUDA(cudaMemsetAsync(ws, 0, sizeof word, st), "cudaMemsetAsync(status)");
  RNX_CUDA(cudaStreamSynchronize(st), "cudaStreamSynchronize");
  if (word & rnx::kDevErrTimeout) return fail(MOE_ERR_DEVICE_TIMEOUT, "a device-side bounded wait ran out (status 0x%x)", word);
  if (word & rnx::kDevErrBounds) return fail(MOE_ERR_DEVICE_BOUNDS, "a device-side index check failed (status 0x%x)", word);
  return MOE_OK;
}

moe_status_t moe_router_topk(const moe_config_t* cfg, const uint16_t* x, int32_t T, const float* router_w,
                             const float* router_bias, float* logits, int32_t* ids, float* weights, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  RNX_PTR(x, "x");
  RNX_PTR(router_w, "router_w");
  RNX_PTR(router_bias, "router_bias");
  RNX_PTR(logits, "logits");
  RNX_PTR(ids, "ids");
  RNX_PTR(weights, "weights");
  cudaStream_t st = (cudaStream_t)stream;
  const int E = cfg->num_experts;
  RNX_CUDA(rnx::launch_router_logits(x, T, cfg->hidden, E, router_w, logits, st), "router logits");
  RNX_CUDA(rnx::launch_topk(logits, router_bias, T, E, cfg->top_k, cfg->routed_scaling_factor, ids, weights, st),
           "router top-k");
  return MOE_OK;
}

moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* ids, int32_t T, const moe_plan_t* plan, void* ws,
                         size_t ws_bytes, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  RNX_PTR(ids, "ids");
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  RNX_PTR(plan->counts, "plan.counts");
  RNX_PTR(plan->offsets, "plan.offsets");
  RNX_PTR(plan->sorted, "plan.sorted");
  RNX_PTR(plan->inv, "plan.inv");
  RNX_PTR(plan->tile_offsets, "plan.tile_offsets");
  RNX_PTR(plan->active, "plan.active");
  RNX_PTR(plan->first, "plan.first");
  RNX_PTR(plan->tile_rows, "plan.tile_rows");
  // only the status word and the sort scratch are used: they sit at the same
  // offsets on both paths, so either path's workspace serves
  const WsLayout L = ws_layout(cfg, T, MOE_PATH_DECODE);
  const size_t need = L.scratch + 4 * rnx::permute_scratch_ints(T * cfg->top_k, cfg->num_experts);
  if (!ws || ((uintptr_t)ws % kAlign) != 0) return fail(MOE_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  char* b = (char*)ws;
  RNX_CUDA(cudaMemsetAsync(b + L.status, 0, 4, st), "clear status");
  RNX_CUDA(rnx::launch_permute(ids, T * cfg->top_k, cfg->num_experts, cfg->local_begin, cfg->local_end, *plan,
                               (int32_t*)(b + L.scratch), (uint32_t*)(b + L.status), st),
           "permute");
  RNX_CUDA(rnx::launch_tile_rows(*plan, cfg->num_experts, L.pl.P, st), "tile rows");
  return MOE_OK;
}

moe_status_t nvfp4_expert_gemv(const moe_config_t* cfg, int32_t proj, const void* act, int32_t T,
                               const moe_plan_t* plan, const float* weights, const moe_weights_t* w, float* out,
                               void* ws, size_t ws_bytes, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (proj != MOE_PROJ_GATE_UP && proj != MOE_PROJ_DOWN) return fail(MOE_ERR_INVALID_ARG, "unknown proj %d", proj);
  if (T == 0) return MOE_OK;
  RNX_PTR(act, "act");
  RNX_PTR(out, "out");
  if (!plan || !w) return fail(MOE_ERR_INVALID_ARG, "plan / weights struct is NULL");
  RNX_PTR(plan->offsets, "plan.offsets");
  RNX_PTR(plan->sorted, "plan.sorted");
  RNX_PTR(plan->active, "plan.active");
  RNX_PTR(plan->first, "plan.first");
  if (proj == MOE_PROJ_GATE_UP) {
    if ((s = check_bank(w->gate, "gate")) != MOE_OK || (s = check_bank(w->up, "up")) != MOE_OK) return s;
  } else {
    if ((s = check_bank(w->down, "down")) != MOE_OK) return s;
    RNX_PTR(weights, "weights");
  }
  WsLayout L;
  if ((s = check_ws(cfg, T, MOE_PATH_DECODE, ws, ws_bytes, &L)) != MOE_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* b = (char*)ws;
  uint32_t* status = (uint32_t*)(b + L.status);
  RNX_CUDA(cudaMemsetAsync(status, 0, kCtrlBytes, st), "clear status");
  const int H = cfg->hidden, I = cfg->intermediate, k = cfg->top_k;
  if (rnx::decode_mma_supported(T, H, I, cfg->num_experts, k) && aligned16(act)) {
    // a handful of tokens: the tensor-core decode kernels, fed from the plan
    RNX_PTR(plan->counts, "plan.counts");
    rnx::DecodeMmaArgs a{};
    a.T = T; a.H = H; a.I = I; a.E = cfg->num_experts; a.k = k;
    a.lb = cfg->local_begin; a.le = cfg->local_end;
    a.limit = cfg->swiglu_limit;
    a.gate = w->gate; a.up = w->up; a.down = w->down;
    a.active = plan->active; a.counts = plan->counts; a.offsets = plan->offsets; a.sorted = plan->sorted;
    a.status = status;
    if (proj == MOE_PROJ_GATE_UP) {
      uint32_t* xmax = (uint32_t*)(b + L.xmax);
      RNX_CUDA(rnx::launch_row_absmax((const uint16_t*)act, T, H, xmax, st), "activation row max");
      a.x = (const uint16_t*)act; a.xmax = xmax; a.h = out;
      RNX_CUDA(rnx::launch_decode_mma_gate_up(a, st), "nvfp4_expert_gemv (gate/up)");
    } else {
      a.h = (float*)act; a.weights = weights; a.r = out;
      RNX_CUDA(rnx::launch_decode_mma_down(a, st), "nvfp4_expert_gemv (down)");
    }
    return MOE_OK;
  }
  rnx::ExpertGemvArgs a{};
  a.proj = proj;
  a.T = T; a.H = H; a.I = I; a.E = cfg->num_experts; a.k = k;
  a.local_begin = cfg->local_begin; a.local_end = cfg->local_end;
  a.limit = cfg->swiglu_limit;
  a.act = act;
  a.offsets = plan->offsets; a.sorted = plan->sorted; a.active = plan->active; a.first = plan->first;
  a.weights = weights;
  a.gate = w->gate; a.up = w->up; a.down = w->down;
  a.out = out;
  a.status = status;
  RNX_CUDA(rnx::launch_nvfp4_gemv(a, st), "nvfp4_expert_gemv");
  return MOE_OK;
}

moe_status_t clamped_swiglu(const float* gu, int32_t M, int32_t I, float limit, uint16_t* h, void* stream) {
  if (M < 0 || I <= 0 || I % 4) return fail(MOE_ERR_INVALID_ARG, "M=%d, I=%d: need M >= 0, I a positive multiple of 4", M, I);
  if (std::isnan(limit) || !(limit > 0.f)) return fail(MOE_ERR_INVALID_ARG, "limit must be > 0");
  if (M == 0) return MOE_OK;
  RNX_PTR(gu, "gu");
  RNX_PTR(h, "h");
  RNX_CUDA(rnx::launch_swiglu(gu, M, I, limit, h, (cudaStream_t)stream), "clamped_swiglu");
  return MOE_OK;
}

moe_status_t moe_combine(int32_t T, int32_t k, int32_t H, const uint16_t* r, const uint16_t* shared, uint16_t* y,
                         void* stream) {
  if (T < 0 || k < 1 || k > kMaxTopK || H <= 0 || H % 8)
    return fail(MOE_ERR_INVALID_ARG, "T=%d k=%d H=%d: need T >= 0, 1 <= k <= 16, H a positive multiple of 8", T, k, H);
  if (T == 0) return MOE_OK;
  RNX_PTR(r, "r");
  RNX_PTR(y, "y");
  if (shared && !aligned16(shared)) return fail(MOE_ERR_INVALID_ARG, "shared is not 16-byte aligned");
  RNX_CUDA(rnx::launch_combine(T, k, H, r, shared, y, (cudaStream_t)stream), "moe_combine");
  return MOE_OK;
}

moe_status_t moe_combine_f32(int32_t T, int32_t k, int32_t H, const float* r, const float* shared, uint16_t* y,
                             void* stream) {
  if (T < 0 || k < 1 || k > kMaxTopK || H <= 0 || H % 4)
    return fail(MOE_ERR_INVALID_ARG, "T=%d k=%d H=%d: need T >= 0, 1 <= k <= 16, H a positive multiple of 4", T, k, H);
  if (T == 0) return MOE_OK;
  RNX_PTR(r, "r");
  RNX_PTR(y, "y");
  if (shared && !aligned16(shared)) return fail(MOE_ERR_INVALID_ARG, "shared is not 16-byte aligned");
  RNX_CUDA(rnx::launch_combine_f32(T, k, H, r, shared, y, (cudaStream_t)stream), "moe_combine_f32");
  return MOE_OK;
}

size_t dense_ffn_workspace_size(int32_t H, int32_t I, int32_t T) {
  if (H <= 0 || I <= 0 || T < 0) return 0;
  return up(4) + up(4 * (size_t)T * I);
}

moe_status_t dense_ffn_bf16(int32_t H, int32_t I, float limit, const uint16_t* x, int32_t T, const uint16_t* wg,
                            const uint16_t* wu, const uint16_t* wd, uint16_t* y, void* ws, size_t ws_bytes,
                            void* stream) {
  if (H <= 0 || H % 64 || I <= 0 || I % 64 || T < 0)
    return fail(MOE_ERR_INVALID_ARG, "H=%d I=%d T=%d: need H, I positive multiples of 64, T >= 0", H, I, T);
  if (std::isnan(limit) || !(limit > 0.f)) return fail(MOE_ERR_INVALID_ARG, "limit must be > 0");
  if (T == 0) return MOE_OK;
  RNX_PTR(x, "x");
  RNX_PTR(wg, "wg");
  RNX_PTR(wu, "wu");
  RNX_PTR(wd, "wd");
  RNX_PTR(y, "y");
  if (!ws || ((uintptr_t)ws % kAlign)) return fail(MOE_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < dense_ffn_workspace_size(H, I, T))
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, dense_ffn_workspace_size(H, I, T));
  void* hbuf = (char*)ws + up(4);
  cudaStream_t st = (cudaStream_t)stream;
  RNX_CUDA(cudaMemsetAsync(ws, 0, 4, st), "clear status");
  RNX_CUDA(rnx::launch_dense_ffn(H, I, limit, x, T, wg, wu, wd, y, false, hbuf, (uint32_t*)ws, st), "dense_ffn_bf16");
  return MOE_OK;
}

moe_status_t nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int32_t rows,
                           int32_t K, float* out, void* stream) {
  if (rows < 0 || K <= 0 || K % 16) return fail(MOE_ERR_INVALID_ARG, "rows=%d K=%d: K must be a positive multiple of 16", rows, K);
  if (rows == 0) return MOE_OK;
  if (!codes || ((uintptr_t)codes & 7)) return fail(MOE_ERR_INVALID_ARG, "codes NULL or not 8-byte aligned");
  if (!scales || !tensor_scale) return fail(MOE_ERR_INVALID_ARG, "scales / tensor_scale is NULL");
  RNX_PTR(out, "out");
  RNX_CUDA(rnx::launch_dequant(codes, scales, tensor_scale, rows, K, out, (cudaStream_t)stream), "nvfp4_dequant");
  return MOE_OK;
}

moe_status_t moe_forward(const moe_config_t* cfg, const moe_weights_t* w, const uint16_t* x, int32_t T, int32_t path,
                         uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  if (path != MOE_PATH_DECODE && path != MOE_PATH_PREFILL && path != MOE_PATH_PREFILL_W4A16)
    return fail(MOE_ERR_INVALID_ARG, "unknown path %d", path);
  if (T == 0) return MOE_OK;
  if (!w) return fail(MOE_ERR_INVALID_ARG, "weights struct is NULL");
  RNX_PTR(x, "x");
  RNX_PTR(y, "y");
  RNX_PTR(w->router_w, "router_w");
  RNX_PTR(w->router_bias, "router_bias");
  if ((s = check_bank(w->gate, "gate")) != MOE_OK || (s = check_bank(w->up, "up")) != MOE_OK ||
      (s = check_bank(w->down, "down")) != MOE_OK)
    return s;
  const int Is = cfg->shared_intermediate;
  if (Is > 0) {
    RNX_PTR(w->shared_gate, "shared_gate");
    RNX_PTR(w->shared_up, "shared_up");
    RNX_PTR(w->shared_down, "shared_down");
  }
  if (path != MOE_PATH_DECODE) {
    if ((s = check_prefill_shape(cfg)) != MOE_OK) return s;
    RNX_PTR(w->prepared, "prepared");
  }
  WsLayout L;
  if ((s = check_ws(cfg, T, path, ws, ws_bytes, &L)) != MOE_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  char* b = (char*)ws;
  const int E = cfg->num_experts, k = cfg->top_k, H = cfg->hidden, I = cfg->intermediate;
  float* logits = (float*)(b + L.logits);
  int32_t* ids = (int32_t*)(b + L.ids);
  float* wts = (float*)(b + L.weights);
  moe_plan_t plan = plan_at(b + L.plan, L.pl);
  uint32_t* status = (uint32_t*)(b + L.status);
  const bool decode = path == MOE_PATH_DECODE;
  const bool t1 = decode && rnx::decode_mma_supported(T, H, I, E, k) && aligned16(x);
  const bool grouped = decode && !t1 && L.grouped && w->prepared;
  // the control block starts at zero: cleared by the router's GEMV (its first
  // CTA, before any later kernel of the call can set a bit; no memset node
  // in front of the router), else by a memset (also when the shared expert's
  // GEMMs, which can set a bit, run beside the router)
  const bool router_clears = decode && rnx::router_gemv_form(T, H) && !grouped;
  if (!router_clears) RNX_CUDA(cudaMemsetAsync(status, 0, kCtrlBytes, st), "clear status");

  // decode: the shared expert forks off to the auxiliary stream right away.
  // With one token its launches follow the router's (the router then does
  // not wait behind them to start); with several tokens they are longer and
  // run ahead of the router, clear of the top-k that follows it. Up to 8
  // tokens the routed experts run on the tensor-core expert kernels (one CTA
  // per SM, weight rows streamed into registers, fed from the routing plan;
  // the router's GEMV also leaves max |x_t| for their f16 pre-scale). A
  // larger batch takes the grouped W4A16 GEMM, and its shared expert the
  // tcgen05 GEMMs (the GEMV form would stream the weights once per 8
  // tokens), done beside the router, top-k and permute, before the grouped
  // GEMM's persistent CTAs take every SM.
  SideStream* side = nullptr;
  const bool shared_aside = Is > 0 && decode;
  void* shared = Is > 0 ? (void*)(b + L.shared) : nullptr;
  auto launch_shared = [&]() -> moe_status_t {
    if (grouped)
      RNX_CUDA(rnx::launch_dense_ffn(H, Is, cfg->swiglu_limit, x, T, w->shared_gate, w->shared_up, w->shared_down,
                                     shared, true, b + L.shared_h, status, side->st, 1),
               "shared expert");
    else
      RNX_CUDA(rnx::launch_dense_gemv(H, Is, cfg->swiglu_limit, x, T, w->shared_gate, w->shared_up, w->shared_down,
                                      shared, true, (float*)(b + L.shared_h), side->st, true),
               "shared expert");
    RNX_CUDA(cudaEventRecord(side->join, side->st), "join event");
    return MOE_OK;
  };
  if (shared_aside) {
    RNX_CUDA(side_stream(&side), "auxiliary stream");
    RNX_CUDA(cudaEventRecord(side->fork, st), "fork event");
    RNX_CUDA(cudaStreamWaitEvent(side->st, side->fork, 0), "fork wait");
    if (T > 1 && (s = launch_shared()) != MOE_OK) return s;
  }
  uint32_t* xmax = (uint32_t*)(b + L.xmax);
  RNX_CUDA(mark(MOE_STAGE_ROUTER_LOGITS, st), "stage event");
  if (!decode && router_on_tensor_cores(cfg, T, w)) {
    const uint16_t* w3 = (const uint16_t*)(w->prepared + prepared_layout(cfg).router3);
    RNX_CUDA(rnx::launch_router_logits_tc(x, T, H, E, w3, logits, status, st), "router logits (tensor cores)");
  } else {
    RNX_CUDA(rnx::launch_router_logits(x, T, H, E, w->router_w, logits, st, t1 ? xmax : nullptr,
                                       router_clears ? status : nullptr, router_clears ? (int)(kCtrlBytes / 4) : 0),
             "router logits");
  }
  if (shared_aside && T == 1 && (s = launch_shared()) != MOE_OK) return s;
  RNX_CUDA(mark(MOE_STAGE_TOPK, st), "stage event");
  // decode with a handful of tokens: selection and plan in one launch (the
  // permute stage then has zero length)
  cudaError_t fp = cudaErrorNotSupported;
  if (decode)
    fp = rnx::launch_topk_plan(logits, w->router_bias, T, E, k, cfg->routed_scaling_factor, ids, wts,
                               cfg->local_begin, cfg->local_end, plan, status, st);
  if (fp == cudaErrorNotSupported) {
    RNX_CUDA(rnx::launch_topk(logits, w->router_bias, T, E, k, cfg->routed_scaling_factor, ids, wts, st), "top-k");
    RNX_CUDA(mark(MOE_STAGE_PERMUTE, st), "stage event");
    RNX_CUDA(rnx::launch_permute(ids, T * k, E, cfg->local_begin, cfg->local_end, plan, (int32_t*)(b + L.scratch),
                                 status, st),
             "permute");
  } else {
    RNX_CUDA(fp, "top-k + plan");
    RNX_CUDA(mark(MOE_STAGE_PERMUTE, st), "stage event");
  }
  RNX_CUDA(mark(MOE_STAGE_ACT_QUANT, st), "stage event");
  if (path == MOE_PATH_PREFILL_W4A16) {
    // the pages' prefill numerics: NVFP4 weights x 16-bit activations on the
    // tensor cores (kind::f16), x gathered into the padded tile order as f16
    const int64_t P = L.pl.P;
    uint16_t* h = (uint16_t*)(b + L.h);
    float* r = (float*)(b + L.r);
    uint16_t* xa = (uint16_t*)(b + L.xq);
    float* xs = (float*)(b + L.xts);
    const int32_t* used_tiles = plan.tile_offsets + E;
    RNX_CUDA(rnx::launch_tile_rows(plan, E, P, st), "tile rows");
    RNX_CUDA(rnx::launch_gather_x_f16(x, H, k, plan.tile_rows, used_tiles, P, xa, xs, st), "x gather (f16)");
    RNX_CUDA(mark(MOE_STAGE_EXPERT_GATE_UP, st), "stage event");
    rnx::W4a16GemmArgs g = w4a16_args(cfg, MOE_PROJ_GATE_UP, xa, xs, P, plan, wts, w, h, status);
    RNX_CUDA(rnx::launch_w4a16_grouped_gemm(g, st), "expert gate/up (W4A16)");
    RNX_CUDA(mark(MOE_STAGE_H_QUANT, st), "stage event");
    RNX_CUDA(mark(MOE_STAGE_EXPERT_DOWN, st), "stage event");
    g = w4a16_args(cfg, MOE_PROJ_DOWN, h, nullptr, P, plan, wts, w, r, status);
    RNX_CUDA(rnx::launch_w4a16_grouped_gemm(g, st), "expert down (W4A16)");
    RNX_CUDA(mark(MOE_STAGE_SHARED, st), "stage event");
    if (Is > 0)
      RNX_CUDA(rnx::launch_dense_ffn(H, Is, cfg->swiglu_limit, x, T, w->shared_gate, w->shared_up, w->shared_down,
                                     shared, true, b + L.shared_h, status, st),
               "shared expert");
    RNX_CUDA(mark(MOE_STAGE_COMBINE, st), "stage event");
    const rnx::PaddedIndex q{ids, plan.inv, plan.offsets, plan.tile_offsets, cfg->local_begin, cfg->local_end};
    RNX_CUDA(rnx::launch_unpermute_combine(q, T, k, H, r, (const float*)shared, y, st), "unpermute + combine");
  } else if (!decode) {
    const int64_t P = L.pl.P;
    uint16_t* h = (uint16_t*)(b + L.h);
    float* r = (float*)(b + L.r);
    uint8_t* xq = (uint8_t*)(b + L.xq);
    uint8_t* xsf = (uint8_t*)(b + L.xsf);
    float* xts = (float*)(b + L.xts);
    uint8_t* hq = (uint8_t*)(b + L.hq);
    uint8_t* hsf = (uint8_t*)(b + L.hsf);
    float* hts = (float*)(b + L.hts);
    const int32_t* used_tiles = plan.tile_offsets + E;
    RNX_CUDA(rnx::launch_tile_rows(plan, E, P, st), "tile rows");
    RNX_CUDA(rnx::launch_quant_tokens(x, T, H, k, ids, plan, cfg->local_begin, cfg->local_end, P, used_tiles, xq, xsf,
                                      xts, st),
             "x quant");
    RNX_CUDA(mark(MOE_STAGE_EXPERT_GATE_UP, st), "stage event");
    rnx::Fp4GemmArgs g = gemm_args(cfg, MOE_PROJ_GATE_UP, xq, xsf, xts, P, plan, wts, w, h, status);
    RNX_CUDA(rnx::launch_fp4_grouped_gemm(g, st), "expert gate/up (tcgen05)");
    RNX_CUDA(mark(MOE_STAGE_H_QUANT, st), "stage event");
    RNX_CUDA(rnx::launch_quant_rows(h, P, I, plan.tile_rows, 0, used_tiles, hq, hsf, hts, st), "h quant");
    RNX_CUDA(mark(MOE_STAGE_EXPERT_DOWN, st), "stage event");
    g = gemm_args(cfg, MOE_PROJ_DOWN, hq, hsf, hts, P, plan, wts, w, r, status);
    RNX_CUDA(rnx::launch_fp4_grouped_gemm(g, st), "expert down (tcgen05)");
    RNX_CUDA(mark(MOE_STAGE_SHARED, st), "stage event");
    if (Is > 0)
      RNX_CUDA(rnx::launch_dense_ffn(H, Is, cfg->swiglu_limit, x, T, w->shared_gate, w->shared_up, w->shared_down,
                                     shared, true, b + L.shared_h, status, st),
               "shared expert");
    RNX_CUDA(mark(MOE_STAGE_COMBINE, st), "stage event");
    const rnx::PaddedIndex q{ids, plan.inv, plan.offsets, plan.tile_offsets, cfg->local_begin, cfg->local_end};
    RNX_CUDA(rnx::launch_unpermute_combine(q, T, k, H, r, (const float*)shared, y, st), "unpermute + combine");
  } else {
    float* h = (float*)(b + L.h);
    float* r = (float*)(b + L.r);
    rnx::ExpertGemvArgs a{};
    a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
    a.local_begin = cfg->local_begin; a.local_end = cfg->local_end;
    a.limit = cfg->swiglu_limit;
    a.offsets = plan.offsets; a.sorted = plan.sorted; a.active = plan.active; a.first = plan.first;
    a.weights = wts;
    a.gate = w->gate; a.up = w->up; a.down = w->down;
    a.status = status;
    if (grouped) {
      // a decode batch on the grouped W4A16 GEMM: x gathered to f16 rows of
      // the padded tile order, 128-row halves of padding skipped; the down
      // GEMM writes r [T*k, H] in assignment order (rows of assignments
      // outside the local range are zeroed first, as no tile writes them)
      const int64_t P = L.pl.P;
      uint16_t* hh = (uint16_t*)(b + L.h);
      uint16_t* xa = (uint16_t*)(b + L.xq);
      float* xs = (float*)(b + L.xts);
      const int32_t* used_tiles = plan.tile_offsets + E;
      RNX_CUDA(rnx::launch_tile_rows(plan, E, P, st), "tile rows");
      RNX_CUDA(rnx::launch_gather_x_f16(x, H, k, plan.tile_rows, used_tiles, P, xa, xs, st, true), "x gather (f16)");
      if (cfg->local_begin > 0 || cfg->local_end < E)
        RNX_CUDA(cudaMemsetAsync(r, 0, sizeof(float) * (size_t)T * k * H, st), "clear remote rows");
      RNX_CUDA(mark(MOE_STAGE_EXPERT_GATE_UP, st), "stage event");
      rnx::W4a16GemmArgs g = w4a16_args(cfg, MOE_PROJ_GATE_UP, xa, xs, P, plan, wts, w, hh, status);
      g.sparse = true;
      RNX_CUDA(rnx::launch_w4a16_grouped_gemm(g, st), "expert gate/up (grouped W4A16)");
      RNX_CUDA(mark(MOE_STAGE_H_QUANT, st), "stage event");
      RNX_CUDA(mark(MOE_STAGE_EXPERT_DOWN, st), "stage event");
      g = w4a16_args(cfg, MOE_PROJ_DOWN, hh, nullptr, P, plan, wts, w, r, status);
      g.sparse = true;
      RNX_CUDA(rnx::launch_w4a16_grouped_gemm(g, st), "expert down (grouped W4A16)");
    } else if (t1) {
      rnx::DecodeMmaArgs d{};
      d.T = T; d.H = H; d.I = I; d.E = E; d.k = k;
      d.lb = cfg->local_begin; d.le = cfg->local_end;
      d.limit = cfg->swiglu_limit;
      d.x = x;
      d.gate = w->gate; d.up = w->up; d.down = w->down;
      d.active = plan.active; d.counts = plan.counts; d.offsets = plan.offsets; d.sorted = plan.sorted;
      d.weights = wts; d.xmax = xmax; d.h = h; d.r = r;
      d.status = status;
      RNX_CUDA(mark(MOE_STAGE_EXPERT_GATE_UP, st), "stage event");
      RNX_CUDA(rnx::launch_decode_mma_gate_up(d, st), "expert gate/up");
      RNX_CUDA(mark(MOE_STAGE_H_QUANT, st), "stage event");
      RNX_CUDA(mark(MOE_STAGE_EXPERT_DOWN, st), "stage event");
      RNX_CUDA(rnx::launch_decode_mma_down(d, st), "expert down");
    } else {
      a.proj = MOE_PROJ_GATE_UP; a.act = x; a.out = h;
      RNX_CUDA(mark(MOE_STAGE_EXPERT_GATE_UP, st), "stage event");
      RNX_CUDA(rnx::launch_nvfp4_gemv(a, st), "expert gate/up");
      RNX_CUDA(mark(MOE_STAGE_H_QUANT, st), "stage event");
      a.proj = MOE_PROJ_DOWN; a.act = h; a.out = r;
      RNX_CUDA(mark(MOE_STAGE_EXPERT_DOWN, st), "stage event");
      RNX_CUDA(rnx::launch_nvfp4_gemv(a, st), "expert down");
    }
    RNX_CUDA(mark(MOE_STAGE_SHARED, st), "stage event");
    if (shared_aside) RNX_CUDA(cudaStreamWaitEvent(st, side->join, 0), "join wait");
    RNX_CUDA(mark(MOE_STAGE_COMBINE, st), "stage event");
    RNX_CUDA(rnx::launch_combine_f32(T, k, H, r, (const float*)shared, y, st), "combine");
  }
  RNX_CUDA(mark(MOE_STAGE_COUNT, st), "stage event");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Decode forward for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: code running
// where the CUDA allocator must not be touched (a memory pool or custom
// allocator owns every byte and forbids cudaMalloc, or a framework callback
// that may not allocate), or a plain C host program that holds only the device
// pointers of its tensors. moe_forward_decode_noalloc runs the same decode
// forward as moe_forward(..., MOE_PATH_DECODE, ...) but takes its scratch from
// one buffer that lives in this library: g_noalloc_scratch below, 8 MiB, which
// every GPU that loads the library keeps until the process exits.
//
// On the host the array's name denotes a host-side stand-in, not a device
// address, so the first call on each device asks the runtime for the device
// address with cudaGetSymbolAddress (that device current) and caches it; that
// first call should come before any stream capture on the device. All calls
// on a device share the buffer and it keeps what the last call left in it; the
// forward clears what must start at zero (the status word, the h-max array)
// itself. Calls whose GPU work overlaps in time -- on two streams or from two
// host threads -- race on the buffer: serialise them on one stream.

static __device__ __align__(256) unsigned char g_noalloc_scratch[8u << 20];

namespace {
constexpr size_t kNoAllocBytes = sizeof(g_noalloc_scratch);
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_dev[kNoAllocMaxDevices] = {};
}  // namespace

// Device address of this library's scratch buffer on the current device,
// looked up once per device (that device current) and cached.
moe_status_t noalloc_scratch(void** out) {
  int dev = 0;
  RNX_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_dev[dev]) {
    void* p = nullptr;
    RNX_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(noalloc scratch)");
    if (!p) return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress returned NULL");
    g_noalloc_dev[dev] = p;
  }
  *out = g_noalloc_dev[dev];
  return MOE_OK;
}

moe_status_t moe_forward_decode_noalloc(const moe_config_t* cfg, const moe_weights_t* w, const uint16_t* x,
                                        int32_t T, uint16_t* y, void* stream) {
  moe_status_t s;
  if ((s = check_cfg(cfg)) != MOE_OK || (s = check_T(T)) != MOE_OK) return s;
  const size_t need = ws_layout(cfg, T, MOE_PATH_DECODE, 0).bytes;
  if (need > kNoAllocBytes)
    return fail(MOE_ERR_WORKSPACE, "moe_forward_decode_noalloc: T=%d needs %zu bytes of scratch, the built-in buffer "
                "holds %zu", T, need, kNoAllocBytes);
  if (T == 0) return MOE_OK;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != MOE_OK) return s;
  return moe_forward(cfg, w, x, T, MOE_PATH_DECODE, y, scratch, kNoAllocBytes, stream);
}

// The device status word of the last moe_forward_decode_noalloc call on the
// current device (it lives at the start of the library's scratch buffer):
// synchronises `stream`, reads and clears the word, like moe_read_device_status.
moe_status_t moe_noalloc_read_device_status(void* stream) {
  void* scratch = nullptr;
  moe_status_t s;
  if ((s = noalloc_scratch(&scratch)) != MOE_OK) return s;
  return moe_read_device_status(scratch, stream);
}

}  // extern "C"
