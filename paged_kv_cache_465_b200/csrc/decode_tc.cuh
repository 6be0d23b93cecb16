// Tensor-core paged decode attention (bf16 / fp8 caches). Filled in by the TC kernel.
#pragma once

#include "decode_simt.cuh"

namespace pa {

// 0 = automatic, 1 = CUDA-core path only, 2 = tensor-core path where supported.
static int g_decode_impl = 0;

inline bool tc_supported(const pa_decode_desc*) { return false; }

inline cudaError_t launch_tc(const DecodeArgs&, const pa_decode_desc*, dim3, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pa
