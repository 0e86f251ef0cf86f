// Shared device helpers of libmoe: bf16/fp16 bits, the packed-nibble dot
// product and warp reductions.
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Device-side check word: a kernel that meets an out-of-range index skips the
// access and sets a bit here; moe_sync() reads and clears it.
__device__ unsigned int g_check_word = 0;  // defined once: libmoe is one CUDA translation unit

enum : unsigned { CHECK_EXPERT_ID = 1u, CHECK_PAIR_ID = 2u, CHECK_WAIT = 4u, CHECK_EP_ROW = 8u };

__device__ __forceinline__ void flag_check(unsigned bit) { atomicOr(&g_check_word, bit); }

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) {
  uint16_t r;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

// acc += lo(h)*lo(x) + hi(h)*hi(x): fp16 operands, exact fp16 x fp16 product,
// fp32 accumulate (mixed-precision fma of PTX ISA 8.6, sm_100+).
__device__ __forceinline__ float fma2_f16_f32(uint32_t h, uint32_t x, float acc) {
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
      "fma.rn.f32.f16 %0, a1, b1, %0;\n\t}"
      : "+f"(acc)
      : "r"(h), "r"(x));
  return acc;
}

// ---------------------------------------------------------------- 4-bit dot
// Activation layout for the 4-bit dot ("nibble-paired"): for every 32-bit
// weight word (elements 8m .. 8m+7) the activation is stored as four half2
//   P0 = (v0, v4)  P1 = (v1/16, v5/16)  P2 = (v2, v6)  P3 = (v3/16, v7/16)
// matching the half2 that one LOP3 makes from the word: (w & 0x000F000F) |
// 0x64006400 is (1024 + q0, 1024 + q4); the 0x00F000F0 mask gives
// (1024 + 16 q1, 1024 + 16 q5); the same on w >> 8 gives nibbles 2, 6 and 3, 7.
// Each product (1024 + s q) * (v / s) = 1024 v / s + q v is exact in fp32, so
//   sum_c q_c v_c = acc - 1024 * (sum of the stored halves)
// The correction ("off") and the plain sum of v per 32-element chunk are
// precomputed once per activation vector.

// One 32-bit weight word against its four activation half2.
__device__ __forceinline__ void dot_word4(uint32_t w, const uint32_t* p, float& a0, float& a1) {
  const uint32_t w8 = w >> 8;
  const uint32_t h0 = (w & 0x000F000Fu) | 0x64006400u;
  const uint32_t h1 = (w & 0x00F000F0u) | 0x64006400u;
  const uint32_t h2 = (w8 & 0x000F000Fu) | 0x64006400u;
  const uint32_t h3 = (w8 & 0x00F000F0u) | 0x64006400u;
  a0 = fma2_f16_f32(h0, p[0], a0);
  a1 = fma2_f16_f32(h1, p[1], a1);
  a0 = fma2_f16_f32(h2, p[2], a0);
  a1 = fma2_f16_f32(h3, p[3], a1);
}

// 32 elements (one uint4 of weights, half a quantisation group).
__device__ __forceinline__ float dot_chunk4(const uint4& q, const uint32_t* p16) {
  float a0 = 0.f, a1 = 0.f;
  dot_word4(q.x, p16 + 0, a0, a1);
  dot_word4(q.y, p16 + 4, a0, a1);
  dot_word4(q.z, p16 + 8, a0, a1);
  dot_word4(q.w, p16 + 12, a0, a1);
  return a0 + a1;
}

// Build the nibble-paired half2 of one 8-element word from fp32 values.
__device__ __forceinline__ void pair_word4(const float v[8], uint32_t p[4]) {
  // round to fp16 first, then divide by 16 (exact) so both halves share the rounding
  const __half h1 = __float2half_rn(v[1]), h3 = __float2half_rn(v[3]);
  const __half h5 = __float2half_rn(v[5]), h7 = __float2half_rn(v[7]);
  p[0] = pack_half2(v[0], v[4]);
  p[1] = pack_half2(__half2float(h1) * 0.0625f, __half2float(h5) * 0.0625f);
  p[2] = pack_half2(v[2], v[6]);
  p[3] = pack_half2(__half2float(h3) * 0.0625f, __half2float(h7) * 0.0625f);
}

// ---------------------------------------------------------------- 8-bit dot
// Router layout ("byte-paired"): for every weight word (elements 4m .. 4m+3)
//   P0 = (v0, v2)  P1 = (v1, v3)
// (w & 0x00FF00FF) | 0x64006400 is (1024 + b0, 1024 + b2); the same on w >> 8
// gives bytes 1 and 3.  sum_c b_c v_c = acc - 1024 * (sum of stored halves).
__device__ __forceinline__ void dot_word8(uint32_t w, const uint32_t* p, float& a0, float& a1) {
  const uint32_t h0 = (w & 0x00FF00FFu) | 0x64006400u;
  const uint32_t h1 = ((w >> 8) & 0x00FF00FFu) | 0x64006400u;
  a0 = fma2_f16_f32(h0, p[0], a0);
  a1 = fma2_f16_f32(h1, p[1], a1);
}

__device__ __forceinline__ float gelu_tanh(float z) {
  const float k0 = 0.7978845608028654f;   // sqrt(2/pi)
  const float inner = k0 * (z + 0.044715f * z * z * z);
  return 0.5f * z * (1.f + tanhf(inner));
}

}  // namespace moe
