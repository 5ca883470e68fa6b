// Shared device helpers for the routed NVFP4 MoE kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/routed_nvfp4.h"

#define RNX_DEVICE __device__ __forceinline__

namespace rnx {

constexpr int kWarp = 32;
constexpr int kNumSMs = 148;          // B200
constexpr int kRowsPerTile = 256;     // expert segments of the padded prefill layout start on these
                                      // boundaries (M of one CTA-pair tile of the FP4 grouped GEMM)

// Device status word (first 4 bytes of every workspace). Kernels OR error
// bits in; moe_read_device_status() reads and clears it.
enum : uint32_t {
  kDevErrTimeout = 1u << 0,
  kDevErrBounds = 1u << 1,
};

RNX_DEVICE void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

RNX_DEVICE float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

RNX_DEVICE uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Two bf16 in one 32-bit word -> two fp32 (element 0 in the low half).
RNX_DEVICE float2 bf16x2_to_f32x2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

RNX_DEVICE uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

// Four bytes of packed E2M1 (8 codes, even element in each byte's low nibble)
// -> four f16x2 words (hardware cvt, exact: every E2M1 value is an f16).
RNX_DEVICE void e2m1x8_to_f16x2x4(uint32_t q, uint32_t& h0, uint32_t& h1, uint32_t& h2, uint32_t& h3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(q));
}

// Two E4M3 bytes (low byte = element 0) -> two fp32 (exact via f16).
RNX_DEVICE float2 e4m3x2_to_f32x2(uint16_t s) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

RNX_DEVICE float e4m3_to_f32(uint8_t s) { return e4m3x2_to_f32x2((uint16_t)s).x; }

// fp32 -> E4M3 byte, round to nearest even, satfinite.
RNX_DEVICE uint8_t f32_to_e4m3_satfinite(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return (uint8_t)(r & 0xFF);
}

// Two fp32 -> one byte of two E2M1 codes (lo in the low nibble), RNE, satfinite.
RNX_DEVICE uint8_t f32x2_to_e2m1x2_satfinite(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "mov.b16 %0, {t, 0};\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return (uint8_t)(r & 0xFF);
}

RNX_DEVICE float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

RNX_DEVICE float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Clamped SwiGLU: silu(min(g, L)) * clamp(u, -L, L). Asymmetric: the gate is
// bounded above only, the up projection on both sides.
RNX_DEVICE float clamped_swiglu(float g, float u, float limit) {
  float gc = fminf(g, limit);
  float uc = fminf(fmaxf(u, -limit), limit);
  return gc / (1.0f + expf(-gc)) * uc;
}

// The same with the fast exponential and division intrinsics (__expf,
// __fdividef): a few fp32 ulps from clamped_swiglu, far inside the bf16
// rounding that follows; used where the epilogue's issue rate matters.
RNX_DEVICE float clamped_swiglu_fast(float g, float u, float limit) {
  const float gc = fminf(g, limit);
  const float uc = fminf(fmaxf(u, -limit), limit);
  return __fdividef(gc, 1.0f + __expf(-gc)) * uc;
}

// Programmatic dependent launch. A kernel launched with the programmatic
// stream-serialization attribute may start before the previous kernel of the
// stream finished; pdl_wait() blocks until that kernel completed and its
// writes are visible (a no-op without a programmatic dependency). Every kernel
// of the chain calls pdl_trigger() only after its own pdl_wait(), so when a
// kernel starts, the kernel two steps earlier has completed: work before
// pdl_wait() may read what that one (and anything earlier) wrote, but nothing
// the immediately preceding kernel writes.
RNX_DEVICE void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
RNX_DEVICE void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Read-only, no-L1-allocate 128-bit global load for streamed weights.
RNX_DEVICE uint4 ldg_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Ask L2 to fetch the 128-byte line holding p (no register result).
RNX_DEVICE void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

RNX_DEVICE uint16_t ldg_u16(const void* p) {
  uint16_t r;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

}  // namespace rnx
