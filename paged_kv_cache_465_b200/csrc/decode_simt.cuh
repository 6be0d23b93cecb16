// Paged decode attention on the CUDA cores (fp32 FMA), the reference-precision path.
//
// [KVPaged] "Core principle: what is the KV cache": softmax(q K^T / sqrt(d)) V for one new
// query per sequence; [Ch4PA] "PagedAttention algorithm": each logical block is looked up
// in the block table and its K/V tile gathered; [KVPaged] "GQA and MQA": the G query heads
// of a group share one kv head, so one CTA serves the whole group and reads each K/V tile
// once for all G heads.
//
// Work item = (sequence, kv head, partition of `part_tokens` logical tokens). A CTA of 4
// warps takes one item; warp w walks the item's blocks w, w+4, ... so the reduction order
// depends only on logical positions (results are independent of physical placement).
// Per block of 16 tokens a warp computes the 16 x G scores with lane = (token, half of d),
// keeps a running max / sum per query head (online softmax in the log2 domain), and
// accumulates P V with lane = 4-channel slice of d. Warps are merged through shared memory
// at the end; the item either writes the normalised output (single pass) or its
// (max, sum, unnormalised output) partial for the log-sum-exp reduction.
//
// This path issues roughly (G + 1) fp32 instructions per KV element and is therefore
// ALU-bound on B200 for G >= 4 at full HBM bandwidth; the tensor-core path replaces it for
// bf16 / fp8 caches and it stays the path for fp32 caches and unusual shapes.
#pragma once

#include "common.cuh"

namespace pa {

constexpr int kSimtWarps = 4;
// Tokens per sub-tile: the unit every decode kernel steps through. A block of 32 tokens is
// two sub-tiles, a block of 8 tokens half of one.
constexpr int kSub = 16;

template <pa_dtype KV>
struct KvTraits;
template <>
struct KvTraits<PA_F32> { static constexpr int bytes = 4; };
template <>
struct KvTraits<PA_BF16> { static constexpr int bytes = 2; };
template <>
struct KvTraits<PA_FP8_E4M3> { static constexpr int bytes = 1; };
template <>
struct KvTraits<PA_INT8> { static constexpr int bytes = 1; };

// 16 bytes of KV -> 16/bytes floats (raw stored value: no scale applied; int8 gives the
// signed code, the zero point is subtracted by the caller).
template <pa_dtype KV>
__device__ __forceinline__ void unpack16(uint4 w, float* x) {
  if constexpr (KV == PA_INT8) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) x[j] = (float)(int8_t)((ws[j >> 2] >> (8 * (j & 3))) & 0xff);
  } else if constexpr (KV == PA_F32) {
    x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
  } else if constexpr (KV == PA_BF16) {
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
  } else {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 a = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(ws[j] & 0xffff)));
      float2 b = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(ws[j] >> 16)));
      x[4 * j + 0] = a.x; x[4 * j + 1] = a.y; x[4 * j + 2] = b.x; x[4 * j + 3] = b.y;
    }
  }
}

// D/32 consecutive channels of one token row (the lane's P.V slice), as floats.
template <pa_dtype KV, int D>
__device__ __forceinline__ void load_vslice(const uint8_t* row, int lane, float* x) {
  constexpr int N = D / 32;                     // channels per lane: 2, 4 or 8
  constexpr int BYTES = N * KvTraits<KV>::bytes;  // 2..32
  const uint8_t* p = row + lane * BYTES;
  if constexpr (KV == PA_F32) {
#pragma unroll
    for (int j = 0; j < N; j += 2) {
      float2 a = __ldg(reinterpret_cast<const float2*>(p) + j / 2);
      x[j] = a.x; x[j + 1] = a.y;
    }
  } else if constexpr (KV == PA_BF16) {
#pragma unroll
    for (int j = 0; j < N; j += 2) {
      uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(p) + j / 2);
      x[j] = bf16_lo(w); x[j + 1] = bf16_hi(w);
    }
  } else if constexpr (KV == PA_INT8) {
#pragma unroll
    for (int j = 0; j < N; j += 2) {
      uint16_t w = __ldg(reinterpret_cast<const uint16_t*>(p) + j / 2);
      x[j] = (float)(int8_t)(w & 0xff); x[j + 1] = (float)(int8_t)(w >> 8);
    }
  } else {
#pragma unroll
    for (int j = 0; j < N; j += 2) {
      uint16_t w = __ldg(reinterpret_cast<const uint16_t*>(p) + j / 2);
      float2 a = f16x2_to_float2(e4m3x2_to_f16x2(w));
      x[j] = a.x; x[j + 1] = a.y;
    }
  }
}

struct DecodeArgs {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  void* out;
  float* lse_out;
  const float* k_scales;
  const float* v_scales;
  const int32_t* k_zeros;  // int8 caches
  const int32_t* v_zeros;
  float* part_m;    // [S][Hq][P]   log2-domain running max of each partition
  float* part_l;    // [S][Hq][P]   sum of exp2(z - m)
  float* part_acc;  // [S][Hq][P][D] unnormalised sum of exp2(z - m) V
  float scale_log2;  // scale * log2(e)
  int num_seqs, num_q_heads, num_kv_heads, group;
  int max_blocks_per_seq, num_blocks;
  int block_size;    // tokens per physical block: 8, 16 or 32
  int part_tokens;   // tokens per work item (a multiple of 16 and of the block size)
  int max_parts;     // P: partitions per sequence in the workspace
  int max_context_len;
  int final_pass;    // 1: one item covers the whole context, write out directly
  int skip_single;   // split path: single-partition sequences were written directly
  // split path, warp workers: warp w < static_seqs * Hkv takes partition 0 of (sequence
  // w / Hkv, kv head w % Hkv) as its first item, without the plan; the plan lists the rest
  int static_seqs;
  pa_dtype q_dtype, out_dtype;
  // prefill rows (CUDA-core kernel only): work row s is new token s; the tokens of
  // sequence q are rows query_start[q] .. query_start[q+1]-1, the last ones of its context
  const int32_t* query_start;  // [num_seqs + 1], or null for decode rows
  int num_tokens;
};

__device__ __forceinline__ float load_q(const void* q, pa_dtype t, int64_t i) {
  return t == PA_F32 ? static_cast<const float*>(q)[i]
                     : __uint_as_float((uint32_t) static_cast<const uint16_t*>(q)[i] << 16);
}

__device__ __forceinline__ void store_out(void* out, pa_dtype t, int64_t i, float x) {
  if (t == PA_F32) static_cast<float*>(out)[i] = x;
  else static_cast<uint16_t*>(out)[i] = (uint16_t)(pack_bf16x2(x, 0.f) & 0xffff);
}

// Clamp a device-side context length into [0, max_context_len]; flag anything outside.
__device__ __forceinline__ int checked_ctx(const DecodeArgs& a, int s) {
  int c = a.context_lens[s];
  if (c < 0 || c > a.max_context_len) {
    if (threadIdx.x == 0) flag_error(PA_DEVERR_CONTEXT);
    c = c < 0 ? 0 : a.max_context_len;
  }
  return c;
}

// Work row s of a prefill call: its sequence (block-table row) and the number of keys it
// sees (its position + 1). A row whose sequence has an inconsistent query range (not
// ascending, past num_tokens, more new tokens than context) sees no key and is flagged.
struct RowView {
  int ctx, seq;
};
__device__ __forceinline__ RowView prefill_row(const DecodeArgs& a, int t) {
  int lo = 0, hi = a.num_seqs;  // largest q with query_start[q] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.query_start[mid] <= t) lo = mid;
    else hi = mid;
  }
  const int q0 = a.query_start[lo], q1 = a.query_start[lo + 1];
  const int c = a.context_lens[lo];
  if (q0 < 0 || q0 > t || t >= q1 || q1 > a.num_tokens || c < q1 - q0 || c > a.max_context_len) {
    if (threadIdx.x == 0) flag_error(PA_DEVERR_QUERY);
    return RowView{0, lo};
  }
  return RowView{c - (q1 - t) + 1, lo};
}

// Writes the merged state of a work item: either out/lse (final) or the partial.
// m2 is the log2-domain max, l the sum, acc[d] the unnormalised output of head h.
__device__ __forceinline__ void emit(const DecodeArgs& a, int s, int h, int part, int D, int d,
                                     float m2, float l, float acc) {
  const int64_t row = (int64_t)s * a.num_q_heads + h;
  if (a.final_pass) {
    const float o = l > 0.f ? acc / l : 0.f;
    store_out(a.out, a.out_dtype, row * D + d, o);
    if (d == 0 && a.lse_out != nullptr)
      a.lse_out[row] = l > 0.f ? (m2 + __log2f(l)) * kLn2 : -INFINITY;
  } else {
    const int64_t pr = row * a.max_parts + part;
    a.part_acc[pr * D + d] = acc;
    if (d == 0) { a.part_m[pr] = m2; a.part_l[pr] = l; }
  }
}

template <pa_dtype KV, int D, int GP>
__global__ void __launch_bounds__(kSimtWarps * 32)
decode_simt_kernel(const DecodeArgs a) {
  constexpr int ES = KvTraits<KV>::bytes;
  constexpr int HALF = D / 2;               // channels per lane in the score phase
  constexpr int EPC = 16 / ES;              // elements per 16-byte chunk
  constexpr int CH = HALF / EPC;            // chunks per lane per token row
  constexpr int NV = D / 32;                // channels per lane in the P.V phase
  constexpr int QROW = D + 4;               // padded q row (floats); halves in different banks

  __shared__ __align__(16) float sq[GP * QROW];
  __shared__ __align__(16) float sp[kSimtWarps][kSub][GP];
  __shared__ float sm[kSimtWarps][GP], sl[kSimtWarps][GP];
  __shared__ __align__(16) float sacc[kSimtWarps][GP][D];

  // decode: grid (partitions, Hkv, S); prefill: grid (new tokens, Hkv, 1), one pass
  const bool pre = a.query_start != nullptr;
  const int part = pre ? 0 : blockIdx.x, kvh = blockIdx.y, s = pre ? blockIdx.x : blockIdx.z;
  const RowView rv = pre ? prefill_row(a, s) : RowView{checked_ctx(a, s), s};
  const int ctx = rv.ctx;
  const int t0 = part * a.part_tokens;
  if (!a.final_pass && t0 >= ctx) return;  // empty partition: nothing to write
  const int t1 = min(ctx, t0 + a.part_tokens);
  const int G = a.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // q of the group, pre-multiplied by scale*log2(e); rows >= G are zero.
  for (int i = threadIdx.x; i < GP * D; i += blockDim.x) {
    const int g = i / D, d = i % D;
    float x = 0.f;
    if (g < G) x = load_q(a.q, a.q_dtype, ((int64_t)s * a.num_q_heads + kvh * G + g) * D + d) *
                   a.scale_log2;
    sq[g * QROW + d + (d >= HALF ? 4 : 0)] = x;
  }
  __syncthreads();

  float m[GP], lsum[GP], acc[GP][NV];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m[g] = -INFINITY; lsum[g] = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) acc[g][j] = 0.f;
  }

  // Tokens are taken in 16-token chunks of logical positions (any block size): lane
  // (tok, half) owns token 16c + tok of chunk c, looks its block up in the table and reads
  // its row at ((block * Hkv + kvh) * block_size + offset) * D elements.
  const int tok = lane & 15, half = lane >> 4;
  const int BS = a.block_size;
  const int c_begin = t0 / kSub, c_end = (t1 + kSub - 1) / kSub;
  const int32_t* bt = a.block_tables + (int64_t)rv.seq * a.max_blocks_per_seq;
  const uint8_t* kbase = static_cast<const uint8_t*>(a.k_cache);
  const uint8_t* vbase = static_cast<const uint8_t*>(a.v_cache);

  for (int c = c_begin + warp; c < c_end; c += kSimtWarps) {
    const int t = c * kSub + tok;
    bool valid = t >= t0 && t < t1;
    int64_t row = -1;  // byte offset of the token's K / V row, -1 when not read
    float ks = 1.f, vs = 1.f, kz = 0.f, vz = 0.f;
    if (valid) {
      const int phys = bt[t / BS];
      if (phys < 0 || phys >= a.num_blocks) {
        if (half == 0) flag_error(PA_DEVERR_BLOCK_ID);
        valid = false;
      } else {
        const int64_t bh = (int64_t)phys * a.num_kv_heads + kvh;
        row = (bh * BS + t % BS) * D * ES;
        if constexpr (KV == PA_FP8_E4M3 || KV == PA_INT8) {
          ks = a.k_scales[bh];
          vs = a.v_scales[bh];
        }
        if constexpr (KV == PA_INT8) {
          const int kzi = a.k_zeros[bh], vzi = a.v_zeros[bh];
          if (!zero_in_range(kzi) || !zero_in_range(vzi)) {  // the block is skipped
            if (half == 0) flag_error(PA_DEVERR_ZERO);
            valid = false;
            row = -1;
          }
          kz = (float)kzi;
          vz = (float)vzi;
        }
      }
    }
    if (!__any_sync(0xffffffffu, valid)) continue;
    // ---- scores: lane (tok, half) -> partial dot over its half of d ----
    float sc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) sc[g] = 0.f;
    if (valid) {
      const uint4* krow = reinterpret_cast<const uint4*>(kbase + row + half * HALF * ES);
#pragma unroll
      for (int cc = 0; cc < CH; ++cc) {
        float kx[EPC];
        unpack16<KV>(__ldg(krow + cc), kx);
        if constexpr (KV == PA_INT8) {
#pragma unroll
          for (int e = 0; e < EPC; ++e) kx[e] -= kz;  // exact: small integers
        }
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float* qr = sq + g * QROW + half * (HALF + 4) + cc * EPC;
#pragma unroll
          for (int e = 0; e < EPC; e += 4) {
            float4 qv = *reinterpret_cast<const float4*>(qr + e);
            sc[g] = fmaf(qv.x, kx[e], sc[g]);
            sc[g] = fmaf(qv.y, kx[e + 1], sc[g]);
            sc[g] = fmaf(qv.z, kx[e + 2], sc[g]);
            sc[g] = fmaf(qv.w, kx[e + 3], sc[g]);
          }
        }
      }
    }
    float p[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float z = sc[g] + __shfl_xor_sync(0xffffffffu, sc[g], 16);
      z = valid ? z * ks : -INFINITY;
      float bm = z;
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
      const float mn = fmaxf(m[g], bm);   // finite: the chunk holds a valid token
      const float alpha = fast_exp2(m[g] - mn);
      m[g] = mn;
      p[g] = valid ? fast_exp2(z - mn) : 0.f;
      lsum[g] = lsum[g] * alpha + (half == 0 ? p[g] : 0.f);
#pragma unroll
      for (int j = 0; j < NV; ++j) acc[g][j] *= alpha;
    }
    if (half == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g) sp[warp][tok][g] = p[g] * vs;
    }
    __syncwarp();
    // ---- P.V: lane -> channels [lane*NV, lane*NV + NV) ----
    // tokens past the item or in an unreadable block are skipped (their rows may hold
    // anything, even NaN)
    const int nv = min(kSub, t1 - c * kSub);
#pragma unroll 4
    for (int tt = 0; tt < nv; ++tt) {
      const int64_t r = __shfl_sync(0xffffffffu, row, tt);
      if (r < 0) continue;
      float vx[NV];
      load_vslice<KV, D>(vbase + r, lane, vx);
      if constexpr (KV == PA_INT8) {
        const float z = __shfl_sync(0xffffffffu, vz, tt);
#pragma unroll
        for (int j = 0; j < NV; ++j) vx[j] -= z;
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pg = sp[warp][tt][g];
#pragma unroll
        for (int j = 0; j < NV; ++j) acc[g][j] = fmaf(pg, vx[j], acc[g][j]);
      }
    }
    __syncwarp();
  }

  // ---- merge the warps ----
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    float l = lsum[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) { sm[warp][g] = m[g]; sl[warp][g] = l; }
#pragma unroll
    for (int j = 0; j < NV; ++j) sacc[warp][g][lane * NV + j] = acc[g][j];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int g = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kSimtWarps; ++w) M = fmaxf(M, sm[w][g]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kSimtWarps; ++w) {
        const float f = fast_exp2(sm[w][g] - M);
        L = fmaf(f, sl[w][g], L);
        A = fmaf(f, sacc[w][g][d], A);
      }
    }
    emit(a, s, kvh * G + g, part, D, d, M, L, A);
  }
}

// Log-sum-exp merge of the partitions of each (sequence, query head), one warp per row:
// 4 rows per CTA of 128 threads, grid ceil(S * Hq / 4). Lane p holds partition p's max and
// sum (32 partitions at a time): M = max_p m_p and L = sum_p 2^(m_p - M) l_p by shuffles;
// every lane owns float4 channel quads and accumulates sum_p 2^(m_p - M) acc_p in partition
// order. The order depends only on partition indices, so the result is deterministic and
// independent of physical block placement.
template <int D>
__global__ void __launch_bounds__(128) lse_reduce_kernel(const DecodeArgs a) {
  constexpr int QUADS = D / 4;
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t rowid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (rowid >= (int64_t)a.num_seqs * a.num_q_heads) return;
  const int s = (int)(rowid / a.num_q_heads);
  const int ctx = checked_ctx(a, s);
  const int np = (ctx + a.part_tokens - 1) / a.part_tokens;
  if (a.skip_single && np <= 1) return;
  const int64_t row = rowid;
  const float* pm = a.part_m + row * a.max_parts;
  const float* pl = a.part_l + row * a.max_parts;
  const float4* pacc = reinterpret_cast<const float4*>(a.part_acc + row * a.max_parts * D);

  // the first 32 partitions' maxima and sums are read together (one round trip)
  const float m0 = lane < np ? pm[lane] : -INFINITY;
  const float l0 = lane < np ? pl[lane] : 0.f;
  float M = m0;
  for (int p = lane + 32; p < np; p += 32) M = fmaxf(M, pm[p]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  constexpr int NQ = (QUADS + 31) / 32;  // quads per lane
  float4 acc[NQ];
#pragma unroll
  for (int j = 0; j < NQ; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int c0 = 0; c0 < np; c0 += 32) {
    const int p = c0 + lane;
    const float mp = c0 == 0 ? m0 : (p < np ? pm[p] : -INFINITY);
    const float lp = c0 == 0 ? l0 : (p < np ? pl[p] : 0.f);
    const float w = (p < np && M != -INFINITY) ? fast_exp2(mp - M) : 0.f;
    if (p < np) lsum = fmaf(w, lp, lsum);
    const int n = min(32, np - c0);
#pragma unroll 8
    for (int k = 0; k < n; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float4* src = pacc + (int64_t)(c0 + k) * QUADS;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const int q = lane + 32 * j;
        if (q < QUADS) {
          const float4 v = __ldg(src + q);
          acc[j].x = fmaf(wk, v.x, acc[j].x); acc[j].y = fmaf(wk, v.y, acc[j].y);
          acc[j].z = fmaf(wk, v.z, acc[j].z); acc[j].w = fmaf(wk, v.w, acc[j].w);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    const int q = lane + 32 * j;
    if (q < QUADS) {
      const int64_t o = row * D + 4 * q;
      store_out(a.out, a.out_dtype, o, acc[j].x * inv);
      store_out(a.out, a.out_dtype, o + 1, acc[j].y * inv);
      store_out(a.out, a.out_dtype, o + 2, acc[j].z * inv);
      store_out(a.out, a.out_dtype, o + 3, acc[j].w * inv);
    }
  }
  if (lane == 0 && a.lse_out != nullptr)
    a.lse_out[row] = lsum > 0.f ? (M + __log2f(lsum)) * kLn2 : -INFINITY;
}

// Same merge for rows with many partitions: one CTA of 4 warps per (sequence, query head),
// grid (Hq, S). Warp w takes the 32-partition chunks c with c % 4 == w (in order); the
// four warps' sums are added in warp order, so the order again depends only on partition
// indices.
template <int D>
__global__ void __launch_bounds__(128) lse_reduce_block_kernel(const DecodeArgs a) {
  constexpr int QUADS = D / 4;
  constexpr int NQ = (QUADS + 31) / 32;
  __shared__ float sm_max[4], sm_l[4];
  __shared__ __align__(16) float sm_acc[4][D];
  pdl_wait();
  const int h = blockIdx.x, s = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ctx = checked_ctx(a, s);
  const int np = (ctx + a.part_tokens - 1) / a.part_tokens;
  if (a.skip_single && np <= 1) return;
  const int64_t row = (int64_t)s * a.num_q_heads + h;
  const float* pm = a.part_m + row * a.max_parts;
  const float* pl = a.part_l + row * a.max_parts;
  const float4* pacc = reinterpret_cast<const float4*>(a.part_acc + row * a.max_parts * D);

  float M = -INFINITY;
  for (int p = threadIdx.x; p < np; p += 128) M = fmaxf(M, pm[p]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) sm_max[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(sm_max[0], sm_max[1]), fmaxf(sm_max[2], sm_max[3]));

  float4 acc[NQ];
#pragma unroll
  for (int j = 0; j < NQ; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int c0 = 32 * warp; c0 < np; c0 += 128) {
    const int p = c0 + lane;
    const float w = (p < np && M != -INFINITY) ? fast_exp2(pm[p] - M) : 0.f;
    if (p < np) lsum = fmaf(w, pl[p], lsum);
    const int n = min(32, np - c0);
#pragma unroll 4
    for (int k = 0; k < n; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float4* src = pacc + (int64_t)(c0 + k) * QUADS;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const int q = lane + 32 * j;
        if (q < QUADS) {
          const float4 v = __ldg(src + q);
          acc[j].x = fmaf(wk, v.x, acc[j].x); acc[j].y = fmaf(wk, v.y, acc[j].y);
          acc[j].z = fmaf(wk, v.z, acc[j].z); acc[j].w = fmaf(wk, v.w, acc[j].w);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if (lane == 0) sm_l[warp] = lsum;
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    const int q = lane + 32 * j;
    if (q < QUADS) reinterpret_cast<float4*>(sm_acc[warp])[q] = acc[j];
  }
  __syncthreads();
  const float L = ((sm_l[0] + sm_l[1]) + sm_l[2]) + sm_l[3];
  for (int d = threadIdx.x; d < D; d += 128) {
    const float A = ((sm_acc[0][d] + sm_acc[1][d]) + sm_acc[2][d]) + sm_acc[3][d];
    store_out(a.out, a.out_dtype, row * D + d, L > 0.f ? A / L : 0.f);
  }
  if (threadIdx.x == 0 && a.lse_out != nullptr)
    a.lse_out[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace pa
