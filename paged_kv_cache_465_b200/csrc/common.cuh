// Shared device helpers of libpagedattn: dtype traits, conversions written as single PTX
// instructions, the device error word, and launch-check macros.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pagedattn.h"

namespace pa {

// ---------------------------------------------------------------------------------------
// Device error word: kernels OR PA_DEVERR_* bits into it instead of faulting; the host
// reads and clears it with pa_device_error(). One word per device (file-scope __device__).
// ---------------------------------------------------------------------------------------
__device__ unsigned int g_error_word;

__device__ __forceinline__ void flag_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

// int8 zero points must lie in the byte's range: only there is code - zero exact in every
// kernel's arithmetic (f16 and bf16 operands of the tensor-core paths). A block whose
// zero point is outside is skipped like a bad block id and PA_DEVERR_ZERO recorded.
__device__ __forceinline__ bool zero_in_range(int z) { return z >= -128 && z <= 127; }

// ---------------------------------------------------------------------------------------
// Conversions. Each is one documented PTX conversion instruction.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two floats -> packed bf16x2 (a in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two floats -> packed f16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two floats -> two E4M3 bytes (lo in byte 0), round to nearest even, saturate to +-448.
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 bytes (byte 0 -> low half) -> f16x2. Exact: every E4M3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t x) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(x));
  return r;
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi) : "r"(h));
  return make_float2(lo, hi);
}

// 1/x on the special-function unit (PTX rcp.approx, subnormals kept; about one ulp).
__device__ __forceinline__ float fast_rcp(float x) {
  float y;
  asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the special-function unit (PTX ex2.approx; relative error ~2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start before its predecessor in the stream finishes; it must wait here before it
// reads anything the predecessor (or earlier work) wrote. No-op for ordinary launches.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel in the stream (launched with programmatic serialization) be
// scheduled; it still waits for this grid's completion in its own pdl_wait().
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Element size in bytes of a pa_dtype.
inline int dtype_bytes(pa_dtype t) { return t == PA_F32 ? 4 : (t == PA_BF16 ? 2 : 1); }

}  // namespace pa

// Launch with programmatic stream serialization (the kernel must call pdl_wait() first).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define PA_CHECK_LAUNCH()                                  \
  do {                                                     \
    cudaError_t e_ = cudaGetLastError();                   \
    if (e_ != cudaSuccess) return PA_ERR_CUDA;             \
  } while (0)
