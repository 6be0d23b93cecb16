// Slot-mapped cache write (reshape_and_cache) and copy-on-write block copy (copy_blocks).
//
// [KVPaged] "PagedAttention: OS virtual-memory style management": new tokens land in the
// block the block table maps their logical position to. [KVPaged] "Prefix sharing and
// copy-on-write": a shared block is copied before a sharer writes into it. [KVPaged] "KV
// quantization: FP8 and INT8": fp8 stores E4M3(x / scale), int8 an affine code with a scale
// and a zero point, per (block, kv head).
//
// Both are pure HBM streams: one CTA per token (write) or per (pair, K|V) (copy), 16-byte
// vector accesses, no shared memory.
#pragma once

#include "common.cuh"

namespace pa {

// 8 consecutive elements of one token row, loaded as float.
template <pa_dtype IN>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&x)[8]) {
  if constexpr (IN == PA_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx));
    x[0] = bf16_lo(a.x); x[1] = bf16_hi(a.x); x[2] = bf16_lo(a.y); x[3] = bf16_hi(a.y);
    x[4] = bf16_lo(a.z); x[5] = bf16_hi(a.z); x[6] = bf16_lo(a.w); x[7] = bf16_hi(a.w);
  }
}

// One CTA per token; threads stride over the token's (kv head, 8-element chunk) pairs of K
// then V. head_dim is a multiple of 8, so a chunk never straddles two heads.
template <pa_dtype IN, pa_dtype CACHE>
__global__ void reshape_and_cache_kernel(const void* __restrict__ k, const void* __restrict__ v,
                                         void* __restrict__ k_cache, void* __restrict__ v_cache,
                                         const int64_t* __restrict__ slot_mapping,
                                         int64_t k_stride, int64_t v_stride, int num_kv_heads,
                                         int head_dim, int block_size, int num_blocks,
                                         const float* __restrict__ k_scales,
                                         const float* __restrict__ v_scales,
                                         const int32_t* __restrict__ k_zeros,
                                         const int32_t* __restrict__ v_zeros) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;  // padding token
  if (slot >= (int64_t)num_blocks * block_size) {
    if (threadIdx.x == 0) flag_error(PA_DEVERR_SLOT);
    return;
  }
  const int64_t blk = slot / block_size;
  const int off = (int)(slot % block_size);
  const int chunks_per_head = head_dim / 8;
  const int chunks = num_kv_heads * chunks_per_head;
  for (int i = threadIdx.x; i < 2 * chunks; i += blockDim.x) {
    const bool is_v = i >= chunks;
    const int c = is_v ? i - chunks : i;
    const int h = c / chunks_per_head;
    const int d0 = (c % chunks_per_head) * 8;
    float x[8];
    load8<IN>(is_v ? v : k, (int64_t)t * (is_v ? v_stride : k_stride) + (int64_t)h * head_dim + d0, x);
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim + d0;
    void* cache = is_v ? v_cache : k_cache;
    if constexpr (CACHE == PA_F32) {
      float4* p = reinterpret_cast<float4*>(static_cast<float*>(cache) + dst);
      p[0] = make_float4(x[0], x[1], x[2], x[3]);
      p[1] = make_float4(x[4], x[5], x[6], x[7]);
    } else if constexpr (CACHE == PA_BF16) {
      uint4 w;
      w.x = pack_bf16x2(x[0], x[1]); w.y = pack_bf16x2(x[2], x[3]);
      w.z = pack_bf16x2(x[4], x[5]); w.w = pack_bf16x2(x[6], x[7]);
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(cache) + dst) = w;
    } else if constexpr (CACHE == PA_INT8) {
      const int64_t sh = blk * num_kv_heads + h;
      const float s = (is_v ? v_scales : k_scales)[sh];
      const int z = (is_v ? v_zeros : k_zeros)[sh];
      if (!zero_in_range(z)) {  // the row is not written
        flag_error(PA_DEVERR_ZERO);
        continue;
      }
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // round half to even; |y| is clamped first so the sum cannot overflow (the result
        // is clamped to the int8 range anyway)
        const float y = fminf(fmaxf(__fdiv_rn(x[j], s), -1024.f), 1024.f);
        const int c = min(127, max(-128, __float2int_rn(y) + z));
        w[j >> 2] |= ((uint32_t)c & 0xffu) << (8 * (j & 3));
      }
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(cache) + dst) = make_uint2(w[0], w[1]);
    } else {
      const float s = (is_v ? v_scales : k_scales)[blk * num_kv_heads + h];
      uint16_t b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        b[j] = pack_e4m3x2(__fdiv_rn(x[2 * j], s), __fdiv_rn(x[2 * j + 1], s));
      uint2 w;
      w.x = (uint32_t)b[0] | ((uint32_t)b[1] << 16);
      w.y = (uint32_t)b[2] | ((uint32_t)b[3] << 16);
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(cache) + dst) = w;
    }
  }
}

// One CTA per (pair, K|V): copies the whole block (all kv heads) with 16-byte accesses.
__global__ void copy_blocks_kernel(uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                                   float* __restrict__ k_scales, float* __restrict__ v_scales,
                                   int32_t* __restrict__ k_zeros, int32_t* __restrict__ v_zeros,
                                   const int32_t* __restrict__ pairs, int64_t block_bytes,
                                   int num_kv_heads, int num_blocks) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  const bool is_v = blockIdx.y == 1;
  const int src = pairs[2 * i], dst = pairs[2 * i + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && !is_v) flag_error(PA_DEVERR_PAIR);
    return;
  }
  uint8_t* cache = is_v ? v_cache : k_cache;
  const uint4* s = reinterpret_cast<const uint4*>(cache + (int64_t)src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>(cache + (int64_t)dst * block_bytes);
  const int n = (int)(block_bytes / 16);
  for (int j = threadIdx.x; j < n; j += blockDim.x) d[j] = s[j];
  float* sc = is_v ? v_scales : k_scales;
  if (sc != nullptr)
    for (int h = threadIdx.x; h < num_kv_heads; h += blockDim.x)
      sc[(int64_t)dst * num_kv_heads + h] = sc[(int64_t)src * num_kv_heads + h];
  int32_t* zp = is_v ? v_zeros : k_zeros;
  if (zp != nullptr)
    for (int h = threadIdx.x; h < num_kv_heads; h += blockDim.x)
      zp[(int64_t)dst * num_kv_heads + h] = zp[(int64_t)src * num_kv_heads + h];
}

}  // namespace pa
