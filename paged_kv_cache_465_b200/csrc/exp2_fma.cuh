// 2^x on the FMA pipe: a polynomial stand-in for the special-function unit's ex2. The
// prefill softmax computes a share of its exponentials this way, so that the FMA pipe and
// the special-function unit split the work. Masked scores (-inf) come out as about 2^-125
// instead of 0: next to a row sum of at least 1 that weight is far below float32 rounding.
//
// Method: range reduction x = j + f with j = rint(x) and |f| <= 1/2, a polynomial for 2^f,
// and 2^j applied by an integer add into the exponent field. The polynomial is the degree-3
// one closest to 2^f on [-1/2, 1/2] in relative error, found by the Remez exchange
// algorithm and rounded to float32; its largest relative error there is 7.5e-5 (2^-13.7),
// well under the 2^-9 rounding step of the bf16 probabilities it feeds.
//
// The scalar form compiles for the host as well, so the same source can be checked on a CPU.
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

#if !defined(__CUDACC__)
#define __host__
#define __device__
#define __forceinline__ inline
#endif

namespace pa {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kRint = 12582912.f;  // 1.5 * 2^23: x + kRint holds rint(x) in its low bits
constexpr float kExp2Min = -125.f;   // smaller arguments (and -inf) give about 2^-125

__host__ __device__ __forceinline__ uint32_t f32_bits(float x) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(x);
#else
  uint32_t u;
  memcpy(&u, &x, 4);
  return u;
#endif
}

__host__ __device__ __forceinline__ float bits_f32(uint32_t u) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  float x;
  memcpy(&x, &u, 4);
  return x;
#endif
}

// 2^x for x < 128. x + 1.5 * 2^23 rounds x to the nearest integer j (ties to even) and
// holds j in the low bits of its mantissa, so (bits of that sum) << 23 is exactly j << 23
// modulo 2^32; adding it to the bits of p = 2^f in [2^-1/2, 2^1/2] scales p by 2^j.
// Results stay normal for x >= -125.
__host__ __device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, kExp2Min);
  const float t = x + kRint;
  const float f = x - (t - kRint);
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return bits_f32(f32_bits(p) + (f32_bits(t) << 23));
}

#if defined(__CUDACC__)
// Packed two-lane float32 fused multiply-add (sm_100): each lane rounds exactly as the
// scalar instruction would, so packed and scalar code give identical bits.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// max of three floats in one instruction (sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

#endif

}  // namespace pa
