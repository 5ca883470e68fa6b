// Device pieces shared by the decode GEMV kernels: NVFP4 chunk dot products
// with exact products and fp32 accumulation, activation pre-scaling into f16,
// and warp reductions of several rows at once.
//
// A 32-element chunk of a weight row is 16 code bytes (two E2M1 codes per
// byte, the even element in the low nibble) plus the two E4M3 scales of its
// 16-element blocks. Codes are decoded to f16 with the hardware cvt (every
// E2M1 value is an f16); the activation chunk is held as f16 scaled by a power
// of two per row, so each product code * activation is exact in fp32 and only
// the fp32 accumulation rounds (mixed-precision fma: f16 inputs, fp32
// accumulator).
#pragma once

#include "common.cuh"

namespace rnx {

// fp32 acc + (a * b) with a, b one f16 half of two f16x2 words: the product
// of two f16 values is exact in fp32, so only the accumulation rounds.
RNX_DEVICE float fma_f16lo(uint32_t a2, uint32_t b2, float acc) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t}"
      : "+f"(acc)
      : "r"(a2), "r"(b2));
  return acc;
}
RNX_DEVICE float fma_f16hi(uint32_t a2, uint32_t b2, float acc) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a2), "r"(b2));
  return acc;
}

// acc + s0 * <codes 0..15, x 0..15> + s1 * <codes 16..31, x 16..31> for one
// 32-element chunk: q = 16 code bytes (even element in the low nibble), sc =
// the chunk's two E4M3 block scales (low byte first), x = the activation chunk
// as 16 f16x2 words (element 2i in the low half of word i).
RNX_DEVICE float chunk_dot_f32(const uint4& q, uint16_t sc, const uint32_t (&x)[16], float acc) {
  uint32_t w[16];
  e2m1x8_to_f16x2x4(q.x, w[0], w[1], w[2], w[3]);
  e2m1x8_to_f16x2x4(q.y, w[4], w[5], w[6], w[7]);
  e2m1x8_to_f16x2x4(q.z, w[8], w[9], w[10], w[11]);
  e2m1x8_to_f16x2x4(q.w, w[12], w[13], w[14], w[15]);
  float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    b0 = fma_f16lo(w[j], x[j], b0);
    b1 = fma_f16hi(w[j], x[j], b1);
    b2 = fma_f16lo(w[j + 8], x[j + 8], b2);
    b3 = fma_f16hi(w[j + 8], x[j + 8], b3);
  }
  const float2 s = e4m3x2_to_f32x2(sc);
  acc = fmaf(s.x, b0 + b1, acc);
  return fmaf(s.y, b2 + b3, acc);
}

// Power of two that brings a row's max |a| into [2^14, 2^15) (f16 keeps 11
// significant bits down to 2^-14); up = 2^(15 - ex), unscale = 2^(ex - 15).
RNX_DEVICE void prescale15(float mx, float& up, float& unscale) {
  int ex = 0;
  if (mx > 0.f && mx <= 3.0e38f) frexpf(mx, &ex);
  up = ldexpf(1.0f, 15 - ex);
  unscale = ldexpf(1.0f, ex - 15);
}

// 32 bf16 activations (chunk c of a row) -> 16 f16x2 words scaled by up.
RNX_DEVICE void act_chunk_bf16(const uint16_t* row, int c, bool on, float up, uint32_t (&xr)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = on ? *reinterpret_cast<const uint4*>(row + 32 * c + 8 * q) : make_uint4(0, 0, 0, 0);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = bf16x2_to_f32x2(w4[j]);
      __half2 h = __floats2half2_rn(f.x * up, f.y * up);
      xr[4 * q + j] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

// 32 fp32 activations (chunk c of a row) -> 16 f16x2 words scaled by up.
RNX_DEVICE void act_chunk_f32(const float* row, int c, bool on, float up, uint32_t (&xr)[16]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = on ? *reinterpret_cast<const float4*>(row + 32 * c + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
    __half2 h0 = __floats2half2_rn(v.x * up, v.y * up);
    __half2 h1 = __floats2half2_rn(v.z * up, v.w * up);
    xr[2 * q] = *reinterpret_cast<uint32_t*>(&h0);
    xr[2 * q + 1] = *reinterpret_cast<uint32_t*>(&h1);
  }
}

// Sum N per-lane values over the warp (N a power of two <= 32): afterwards
// lane l holds the total of value l / (32 / N). log2(N) exchange steps at
// distances 16, 8, ... each halve the values a lane holds; plain butterflies
// finish.
template <int N>
RNX_DEVICE float warp_reduce_rows(float (&v)[N]) {
  const int lane = threadIdx.x & 31;
  int cnt = N;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) {
    if (cnt > 1) {
      const int h = cnt >> 1;
      const bool hi = lane & d;
#pragma unroll
      for (int i = 0; i < (N > 1 ? N / 2 : 1); ++i) {
        if (i < h) {
          const float send = hi ? v[i] : v[i + h];
          const float keep = hi ? v[i + h] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, d);
        }
      }
      cnt = h;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], d);
    }
  }
  return v[0];
}

}  // namespace rnx
