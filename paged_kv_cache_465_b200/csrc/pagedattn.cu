// C-ABI entry points of libpagedattn.so: argument validation and kernel dispatch.
// Declarations and contracts: include/pagedattn.h.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "cache_ops.cuh"
#include "decode_simt.cuh"
#include "decode_tc.cuh"
#include "prefill_tc.cuh"

namespace pa {
namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split-path workspace: plan area (counters, item list) followed by the partials
// (m, l, acc) of every (seq, q head, partition).
struct WorkspaceLayout {
  size_t cnt_off, list_off, m_off, l_off, acc_off, total;
  int parts;
};

bool desc_ok(const pa_decode_desc* d) {
  if (d == nullptr) return false;
  if (d->num_seqs < 0 || d->num_seqs > 65535) return false;
  if (d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->num_kv_heads > 65535) return false;
  if (d->num_q_heads % d->num_kv_heads != 0) return false;
  if (d->head_dim <= 0 || d->block_size <= 0 || d->num_blocks <= 0) return false;
  if (d->max_blocks_per_seq <= 0) return false;
  if (d->partition_size == PA_PARTITION_AUTO) return true;
  if (d->partition_size < 0 || d->partition_size % d->block_size != 0) return false;
  return true;
}

// The partition the library takes for PA_PARTITION_AUTO: one pass (0) when no context can
// exceed 512 tokens; else 512 tokens when there are at least 1024 (sequence, kv head)
// pairs, else 1024. Measured on a B200 (decode call, fraction of the measured copy
// bandwidth): 256 sequences x 8 kv heads up to 8192 tokens, fp8: 0.77 at 512 (warp
// workers) against 0.73 at 1024 (one CTA per item); 32 x 8 up to 4096 tokens, bf16: 0.63
// at 1024 against 0.59 at 512 and 0.49 in one pass; 8 x 8 at 131072 tokens, bf16: 1.00 at
// 1024 against 0.95 at 512; 100 x 8 at 250 tokens: one pass fastest. With few pairs,
// longer items split over a CTA's four warps finish sooner. It depends on the shape only,
// never on the context lengths themselves (device data) or on where blocks sit, so
// results stay independent of the physical placement.
int auto_partition(const pa_decode_desc* d, int max_context_len) {
  if (max_context_len <= 512) return 0;
  return (int64_t)d->num_seqs * d->num_kv_heads >= 1024 ? 512 : 1024;
}

// desc with PA_PARTITION_AUTO replaced by the partition the library takes.
pa_decode_desc resolved(const pa_decode_desc* d, int max_context_len) {
  pa_decode_desc r = *d;
  if (r.partition_size == PA_PARTITION_AUTO) r.partition_size = auto_partition(d, max_context_len);
  return r;
}

bool desc_supported(const pa_decode_desc* d) {
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->block_size != 8 && d->block_size != 16 && d->block_size != 32) return false;
  if (d->partition_size % kSub != 0) return false;  // partitions start on 16-token sub-tiles
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256) return false;
  if (G > 16 || G * d->head_dim > 2048) return false;
  if (d->kv_dtype == PA_F32) return d->q_dtype == PA_F32 && d->out_dtype == PA_F32;
  if (d->kv_dtype == PA_BF16 || d->kv_dtype == PA_FP8_E4M3 || d->kv_dtype == PA_INT8)
    return d->q_dtype == PA_BF16 && d->out_dtype == PA_BF16;
  return false;
}

WorkspaceLayout layout_for(const pa_decode_desc* d, int max_context_len) {
  WorkspaceLayout w{0, 0, 0, 0, 0, 0, 0};
  if (d->partition_size == 0 || max_context_len <= 0) return w;
  w.parts = (max_context_len + d->partition_size - 1) / d->partition_size;
  const size_t rows = (size_t)d->num_seqs * d->num_q_heads * w.parts;
  w.cnt_off = 0;
  w.list_off = 256;
  w.m_off = w.list_off + round_up((size_t)d->num_seqs * w.parts * 16, 256);
  w.l_off = w.m_off + round_up(rows * sizeof(float), 256);
  w.acc_off = w.l_off + round_up(rows * sizeof(float), 256);
  w.total = w.acc_off + round_up(rows * (size_t)d->head_dim * sizeof(float), 256);
  return w;
}

int pad_group(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : G <= 8 ? 8 : 16; }

// Which kernels a decode call runs: the tensor-core family (and which of its kernels, the
// persistent ones after a plan kernel) or the CUDA-core path; a split call ends with the
// log-sum-exp reduce.
struct DecodeRoute {
  bool split, tc;
  tc::TcKind kind;
  int launches;  // kernel launches of the call
};

DecodeRoute route_for(const pa_decode_desc* d, const WorkspaceLayout& wl, int impl) {
  DecodeRoute r{wl.total > 0, false, tc::kTcGrid, 1};
  if (impl != 1 && tc_supported(d)) {
    r.tc = true;
    r.kind = tc_kind(d, r.split, impl);
    r.launches = (r.kind != tc::kTcGrid ? 2 : 1) + (r.split ? 1 : 0);
  } else {
    r.launches = r.split ? 2 : 1;
  }
  return r;
}

template <pa_dtype KV, int D, int GP>
cudaError_t launch_simt(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  if constexpr (GP * D <= 2048) {
    decode_simt_kernel<KV, D, GP><<<grid, kSimtWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
  } else {
    return cudaErrorInvalidValue;
  }
}

template <pa_dtype KV, int D>
cudaError_t launch_simt_g(const DecodeArgs& a, int gp, dim3 grid, cudaStream_t st) {
  switch (gp) {
    case 1: return launch_simt<KV, D, 1>(a, grid, st);
    case 2: return launch_simt<KV, D, 2>(a, grid, st);
    case 4: return launch_simt<KV, D, 4>(a, grid, st);
    case 8: return launch_simt<KV, D, 8>(a, grid, st);
    default: return launch_simt<KV, D, 16>(a, grid, st);
  }
}

template <pa_dtype KV>
cudaError_t launch_simt_d(const DecodeArgs& a, int D, int gp, dim3 grid, cudaStream_t st) {
  switch (D) {
    case 64: return launch_simt_g<KV, 64>(a, gp, grid, st);
    case 128: return launch_simt_g<KV, 128>(a, gp, grid, st);
    default: return launch_simt_g<KV, 256>(a, gp, grid, st);
  }
}

// Rows with up to 32 partitions: one warp per row; more: one CTA of 4 warps per row.
cudaError_t launch_reduce(const DecodeArgs& a, int D, cudaStream_t st) {
  const dim3 block(128);
  if (a.max_parts > 32) {
    const dim3 grid(a.num_q_heads, a.num_seqs);
    switch (D) {
      case 64: return launch_pdl(lse_reduce_block_kernel<64>, grid, block, 0, st, a);
      case 128: return launch_pdl(lse_reduce_block_kernel<128>, grid, block, 0, st, a);
      default: return launch_pdl(lse_reduce_block_kernel<256>, grid, block, 0, st, a);
    }
  }
  const int64_t rows = (int64_t)a.num_seqs * a.num_q_heads;
  const dim3 grid((unsigned)((rows + 3) / 4));
  switch (D) {
    case 64: return launch_pdl(lse_reduce_kernel<64>, grid, block, 0, st, a);
    case 128: return launch_pdl(lse_reduce_kernel<128>, grid, block, 0, st, a);
    default: return launch_pdl(lse_reduce_kernel<256>, grid, block, 0, st, a);
  }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_version(void) { return "pagedattn 0.4 sm_100a"; }

pa_status pa_set_decode_impl(int impl) {
  if (impl < 0 || impl > 5) return PA_ERR_INVALID;
  g_decode_impl.store(impl, std::memory_order_relaxed);
  return PA_OK;
}

size_t paged_attn_workspace_size(const pa_decode_desc* desc, int max_context_len) {
  if (!desc_ok(desc) || max_context_len < 0) return 0;
  const pa_decode_desc d = resolved(desc, max_context_len);
  return layout_for(&d, max_context_len).total;
}

int paged_attn_partition_size(const pa_decode_desc* desc, int max_context_len) {
  if (!desc_ok(desc) || max_context_len < 0) return -1;
  return resolved(desc, max_context_len).partition_size;
}

int paged_attn_decode_launches(const pa_decode_desc* desc, int max_context_len) {
  if (!desc_ok(desc) || max_context_len < 0) return 0;
  const pa_decode_desc d = resolved(desc, max_context_len);
  if (!desc_supported(&d) || d.num_seqs == 0) return 0;
  return route_for(&d, layout_for(&d, max_context_len),
                   g_decode_impl.load(std::memory_order_relaxed)).launches;
}

pa_status paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            float scale, void* out, const pa_decode_desc* desc,
                            int max_context_len, const float* k_scales, const float* v_scales,
                            const int32_t* k_zeros, const int32_t* v_zeros, float* lse_out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!desc_ok(desc) || max_context_len < 0 || !std::isfinite(scale)) return PA_ERR_INVALID;
  const pa_decode_desc rdesc = resolved(desc, max_context_len);
  desc = &rdesc;
  if (!desc_supported(desc)) return PA_ERR_UNSUPPORTED;
  if (desc->num_seqs == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(out))
    return PA_ERR_INVALID;
  if ((int64_t)desc->max_blocks_per_seq * desc->block_size < (int64_t)max_context_len)
    return PA_ERR_INVALID;
  const bool quant = desc->kv_dtype == PA_FP8_E4M3 || desc->kv_dtype == PA_INT8;
  if (quant && (!k_scales || !v_scales)) return PA_ERR_INVALID;
  if (desc->kv_dtype == PA_INT8 && (!k_zeros || !v_zeros)) return PA_ERR_INVALID;
  const WorkspaceLayout wl = layout_for(desc, max_context_len);
  if (wl.total > 0 && (workspace == nullptr || workspace_bytes < wl.total || !aligned16(workspace)))
    return PA_ERR_WORKSPACE;

  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
  a.block_tables = block_tables; a.context_lens = context_lens;
  a.out = out; a.lse_out = lse_out; a.k_scales = k_scales; a.v_scales = v_scales;
  a.k_zeros = k_zeros; a.v_zeros = v_zeros;
  a.scale_log2 = scale * kLog2e;
  a.num_seqs = desc->num_seqs; a.num_q_heads = desc->num_q_heads;
  a.num_kv_heads = desc->num_kv_heads; a.group = desc->num_q_heads / desc->num_kv_heads;
  a.max_blocks_per_seq = desc->max_blocks_per_seq; a.num_blocks = desc->num_blocks;
  a.block_size = desc->block_size;
  a.max_context_len = max_context_len;
  a.q_dtype = desc->q_dtype; a.out_dtype = desc->out_dtype;
  const bool split = wl.total > 0;
  if (split) {
    char* ws = static_cast<char*>(workspace);
    a.part_m = reinterpret_cast<float*>(ws + wl.m_off);
    a.part_l = reinterpret_cast<float*>(ws + wl.l_off);
    a.part_acc = reinterpret_cast<float*>(ws + wl.acc_off);
    a.part_tokens = desc->partition_size;
    a.max_parts = wl.parts;
    a.final_pass = 0;
  } else {
    a.part_tokens = (int)round_up((size_t)(max_context_len > 0 ? max_context_len : 1), kSub);
    a.max_parts = 1;
    a.final_pass = 1;
  }
  const cudaStream_t st = as_stream(stream);
  const dim3 grid(split ? wl.parts : 1, desc->num_kv_heads, desc->num_seqs);
  const int D = desc->head_dim;
  const int gp = pad_group(a.group);
  cudaError_t e;
  const DecodeRoute r = route_for(desc, wl, g_decode_impl.load(std::memory_order_relaxed));
  if (r.tc) {
    tc::PlanView pl;
    if (r.kind != tc::kTcGrid) {
      char* ws = static_cast<char*>(workspace);
      pl.counters = reinterpret_cast<uint32_t*>(ws + wl.cnt_off);
      pl.list = reinterpret_cast<int4*>(ws + wl.list_off);
      a.skip_single = 1;  // single-partition sequences are written by the kernel itself
    }
    e = launch_tc(a, desc, grid, r.kind == tc::kTcGrid ? nullptr : &pl, r.kind, st);
  } else {
    switch (desc->kv_dtype) {
      case PA_F32: e = launch_simt_d<PA_F32>(a, D, gp, grid, st); break;
      case PA_BF16: e = launch_simt_d<PA_BF16>(a, D, gp, grid, st); break;
      case PA_INT8: e = launch_simt_d<PA_INT8>(a, D, gp, grid, st); break;
      default: e = launch_simt_d<PA_FP8_E4M3>(a, D, gp, grid, st); break;
    }
  }
  if (e != cudaSuccess) return PA_ERR_CUDA;
  if (split && launch_reduce(a, D, st) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

pa_status paged_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             const int32_t* query_start, int num_tokens, int max_query_len,
                             float scale, void* out, const pa_decode_desc* desc,
                             int max_context_len, const float* k_scales, const float* v_scales,
                             const int32_t* k_zeros, const int32_t* v_zeros, float* lse_out,
                             void* stream) {
  if (!desc_ok(desc) || desc->partition_size != 0 || num_tokens < 0 || max_query_len < 0 ||
      max_context_len < max_query_len || !std::isfinite(scale))
    return PA_ERR_INVALID;
  if (!desc_supported(desc)) return PA_ERR_UNSUPPORTED;
  if (desc->num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start || !out)
    return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(out))
    return PA_ERR_INVALID;
  if ((int64_t)desc->max_blocks_per_seq * desc->block_size < (int64_t)max_context_len)
    return PA_ERR_INVALID;
  const bool quant = desc->kv_dtype == PA_FP8_E4M3 || desc->kv_dtype == PA_INT8;
  if (quant && (!k_scales || !v_scales)) return PA_ERR_INVALID;
  if (desc->kv_dtype == PA_INT8 && (!k_zeros || !v_zeros)) return PA_ERR_INVALID;
  const cudaStream_t st = as_stream(stream);
  if (max_query_len == 0) return PA_OK;
  cudaError_t e;
  if (g_decode_impl.load(std::memory_order_relaxed) != 1 && prefill_tc_supported(desc)) {
    pf::PrefillArgs a;
    a.block_tables = block_tables; a.context_lens = context_lens; a.query_start = query_start;
    a.out = out; a.lse_out = lse_out;
    a.k_scales = k_scales; a.v_scales = v_scales; a.k_zeros = k_zeros; a.v_zeros = v_zeros;
    a.scale_log2 = scale * kLog2e;
    a.num_seqs = desc->num_seqs; a.num_tokens = num_tokens;
    a.num_q_heads = desc->num_q_heads; a.num_kv_heads = desc->num_kv_heads;
    a.group = desc->num_q_heads / desc->num_kv_heads;
    a.max_blocks_per_seq = desc->max_blocks_per_seq; a.num_blocks = desc->num_blocks;
    a.max_context_len = max_context_len; a.max_query_len = max_query_len;
    e = launch_prefill_tc(a, desc->block_size, desc->kv_dtype, q, k_cache, v_cache, st);
  } else {
    // CUDA-core path: every new token is one work row of the single-pass decode kernel
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
    a.block_tables = block_tables; a.context_lens = context_lens;
    a.out = out; a.lse_out = lse_out; a.k_scales = k_scales; a.v_scales = v_scales;
    a.k_zeros = k_zeros; a.v_zeros = v_zeros;
    a.scale_log2 = scale * kLog2e;
    a.num_seqs = desc->num_seqs; a.num_q_heads = desc->num_q_heads;
    a.num_kv_heads = desc->num_kv_heads; a.group = desc->num_q_heads / desc->num_kv_heads;
    a.max_blocks_per_seq = desc->max_blocks_per_seq; a.num_blocks = desc->num_blocks;
    a.block_size = desc->block_size;
    a.max_context_len = max_context_len;
    a.q_dtype = desc->q_dtype; a.out_dtype = desc->out_dtype;
    a.part_tokens = (int)round_up((size_t)(max_context_len > 0 ? max_context_len : 1), kSub);
    a.max_parts = 1;
    a.final_pass = 1;
    a.query_start = query_start;
    a.num_tokens = num_tokens;
    const dim3 grid(num_tokens, desc->num_kv_heads, 1);
    const int gp = pad_group(a.group);
    switch (desc->kv_dtype) {
      case PA_F32: e = launch_simt_d<PA_F32>(a, desc->head_dim, gp, grid, st); break;
      case PA_BF16: e = launch_simt_d<PA_BF16>(a, desc->head_dim, gp, grid, st); break;
      case PA_INT8: e = launch_simt_d<PA_INT8>(a, desc->head_dim, gp, grid, st); break;
      default: e = launch_simt_d<PA_FP8_E4M3>(a, desc->head_dim, gp, grid, st); break;
    }
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                            const int64_t* slot_mapping, int num_tokens, int64_t k_stride,
                            int64_t v_stride, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, pa_dtype in_dtype, pa_dtype cache_dtype,
                            const float* k_scales, const float* v_scales,
                            const int32_t* k_zeros, const int32_t* v_zeros, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 != 0 ||
      block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID;
  if (in_dtype != PA_F32 && in_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (cache_dtype == PA_F32 && in_dtype != PA_F32) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  if (k_stride < row || v_stride < row) return PA_ERR_INVALID;
  // 16-byte vector loads of 8 input elements
  const int64_t align_elems = in_dtype == PA_F32 ? 4 : 8;
  if (k_stride % align_elems || v_stride % align_elems || !aligned16(k) || !aligned16(v) ||
      !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  if ((cache_dtype == PA_FP8_E4M3 || cache_dtype == PA_INT8) && (!k_scales || !v_scales))
    return PA_ERR_INVALID;
  if (cache_dtype == PA_INT8 && (!k_zeros || !v_zeros)) return PA_ERR_INVALID;
  const cudaStream_t st = as_stream(stream);
  const dim3 grid(num_tokens);
  const int threads = 128;
  cudaError_t e = cudaSuccess;
#define PA_RC(IN, C)                                                                          \
  e = launch_pdl(reshape_and_cache_kernel<IN, C>, grid, dim3(threads), 0, st, k, v, k_cache,  \
                 v_cache, slot_mapping, k_stride, v_stride, num_kv_heads, head_dim,          \
                 block_size, num_blocks, k_scales, v_scales, k_zeros, v_zeros)
  if (in_dtype == PA_F32) {
    if (cache_dtype == PA_F32) PA_RC(PA_F32, PA_F32);
    else if (cache_dtype == PA_BF16) PA_RC(PA_F32, PA_BF16);
    else if (cache_dtype == PA_FP8_E4M3) PA_RC(PA_F32, PA_FP8_E4M3);
    else if (cache_dtype == PA_INT8) PA_RC(PA_F32, PA_INT8);
    else return PA_ERR_UNSUPPORTED;
  } else {
    if (cache_dtype == PA_BF16) PA_RC(PA_BF16, PA_BF16);
    else if (cache_dtype == PA_FP8_E4M3) PA_RC(PA_BF16, PA_FP8_E4M3);
    else if (cache_dtype == PA_INT8) PA_RC(PA_BF16, PA_INT8);
    else return PA_ERR_UNSUPPORTED;
  }
#undef PA_RC
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status copy_blocks(void* k_cache, void* v_cache, float* k_scales, float* v_scales,
                      int32_t* k_zeros, int32_t* v_zeros, const int32_t* pairs, int num_pairs,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      pa_dtype cache_dtype, void* stream) {
  if (num_pairs < 0 || num_pairs > 65535 * 1024 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID;
  if (cache_dtype != PA_F32 && cache_dtype != PA_BF16 && cache_dtype != PA_FP8_E4M3 &&
      cache_dtype != PA_INT8)
    return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !pairs || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * dtype_bytes(cache_dtype);
  if (block_bytes % 16 != 0) return PA_ERR_INVALID;
  const bool quant = cache_dtype == PA_FP8_E4M3 || cache_dtype == PA_INT8;
  if (quant && (!k_scales || !v_scales)) return PA_ERR_INVALID;
  if (cache_dtype == PA_INT8 && (!k_zeros || !v_zeros)) return PA_ERR_INVALID;
  const bool i8 = cache_dtype == PA_INT8;
  const cudaError_t e = launch_pdl(
      copy_blocks_kernel, dim3(num_pairs, 2), dim3(256), 0, as_stream(stream),
      static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache),
      quant ? k_scales : nullptr, quant ? v_scales : nullptr, i8 ? k_zeros : nullptr,
      i8 ? v_zeros : nullptr, pairs, block_bytes, num_kv_heads, num_blocks);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Allocation-free decode: the split-KV scratch lives in one fixed array of this library's
// device image. In host code `g_noalloc_scratch` names a host-side stand-in, not device
// memory, so it is never passed to a kernel: the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::atomic<void*> g_noalloc_ptr[kMaxDevices];  // static storage: zero-initialised
std::mutex g_noalloc_mu;

// Device address of the fixed array on the current device, looked up on the first call
// there (with that device current) and cached.
pa_status noalloc_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return PA_ERR_CUDA;
      g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *ptr = p;
  return PA_OK;
}
}  // namespace

pa_status paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, const int32_t* context_lens,
                                    float scale, void* out, const pa_decode_desc* desc,
                                    int max_context_len, const float* k_scales,
                                    const float* v_scales, const int32_t* k_zeros,
                                    const int32_t* v_zeros, float* lse_out, void* stream) {
  if (!desc_ok(desc) || max_context_len < 0) return PA_ERR_INVALID;
  if (paged_attn_workspace_size(desc, max_context_len) > PA_NOALLOC_SCRATCH_BYTES)
    return PA_ERR_WORKSPACE;
  // the look-up runs on every call, needed or not, so that the first call on a device does
  // it whatever its shape
  void* ws = nullptr;
  const pa_status st = noalloc_scratch(&ws);
  if (st != PA_OK) return st;
  return paged_attn_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, desc,
                           max_context_len, k_scales, v_scales, k_zeros, v_zeros, lse_out, ws,
                           (size_t)PA_NOALLOC_SCRATCH_BYTES, stream);
}

pa_status pa_device_error(int* bits_out, void* stream) {
  if (bits_out == nullptr) return PA_ERR_INVALID;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return PA_ERR_CUDA;
  unsigned int w = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
  *bits_out = (int)w;
  return w == 0 ? PA_OK : PA_ERR_DEVICE;
}

}  // extern "C"
