// Prefill attention on the fifth-generation tensor cores: the new tokens of a step attend
// causally to their sequence's cached keys through the block table.
//
// [KVPaged] "Core principle: what is the KV cache" (each token attends to itself and every
// earlier token; the prompt's K/V is computed once and cached) and "Prefix sharing and
// copy-on-write" (a cached prefix's K/V is computed once, so a step may bring only the
// tokens after it); [Ch4PA] "PagedAttention algorithm" (keys and values are gathered from
// non-contiguous blocks through the block table).
//
// One CTA per (pair of 128-row query tiles, kv head, sequence), one CTA per SM. A tile row
// is a (new token, query head of the kv head's group) pair, so one key/value tile serves
// the whole group, and both query tiles of the CTA share it: each K/V tile crosses L2 once
// per 256 rows. Keys are taken 128 at a time:
//   warp 9              TMA: both Q tiles once; K and V of key tile j into their own rings,
//                       one (block, 64-channel half) box per lane straight from the paged
//                       pool, block ids read one tile ahead; a K stage is refilled once its
//                       S products are done, a V stage once its P V products are done;
//   warp 8 (one lane)   tcgen05.mma, ping-pong over the two query tiles: O_0 += P_0(j) V_j,
//                       S_0(j+1) = Q_0 K_{j+1}^T, then the same for tile 1. Each query tile
//                       has one S buffer in tensor memory; P_x(j) is written over S_x(j) and
//                       read by the P V product before S_x(j+1) overwrites it (products run
//                       in issue order). While one tile is in softmax, the tensor core runs
//                       the other tile's products;
//   warps 0-3 / 4-7     softmax of query tile 0 / 1, one thread per row (= tensor-memory
//                       lane): causal mask, running max (rescaling O in tensor memory only
//                       when the max grows by more than 2^8), P as bf16 pairs written over
//                       S; finally O / l to `out` and the log-sum-exp to `lse_out`.
// Operands in shared memory use the 128-byte-swizzled layouts the tensor core reads: Q and
// K K-major (rows of 64 channels, 128 B), V MN-major (rows of keys).
// Every wait is bounded; a CTA that gives up flags PA_DEVERR_TIMEOUT, lets its issued
// copies and products finish, and releases its tensor memory.
#pragma once

#include "decode_tc.cuh"

namespace pa {
namespace pf {

using tc::evict_first_policy;
using tc::mbar_arrive;
using tc::mbar_arrive_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::smem_u32;

constexpr int kBM = 128;                  // rows of a query tile: (new token, head) pairs
constexpr int kQT = 2;                    // query tiles per CTA, sharing every key tile
constexpr int kBN = 128;                  // keys per key tile
constexpr int kD = 128;                   // head dimension
constexpr int kMmaWarp = 8, kTmaWarp = 9;  // warps 0-7 softmax (two warpgroups)
constexpr int kConvWarp0 = 10;            // fp8 / int8 caches: warps 10-11 dequantise
constexpr int kConvThreads = 64;
constexpr int kQSlab = kBM * 128;         // 64 channels (128 B) x 128 rows
constexpr int kQBytes = 2 * kQSlab;       // one query tile
constexpr int kKVSlab = kBN * 128;        // 64 channels x 128 keys
constexpr int kKVBytes = 2 * kKVSlab;
#ifndef PA_PF_KSTAGES
#define PA_PF_KSTAGES 2
#endif
#ifndef PA_PF_VSTAGES
#define PA_PF_VSTAGES 2
#endif
constexpr int kKSt = PA_PF_KSTAGES, kVSt = PA_PF_VSTAGES;  // ring depths
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQT * kQBytes;
constexpr int kOffV = kOffK + kKSt * kKVBytes;
// Shared-memory map per cache type: a quantised cache adds a staging buffer for the codes
// of one K tile and one V tile (TMA lands them there, the converter warps write the bf16
// stages from them) and the tile's per-block scales and zero points.
template <bool QUANT>
struct PfLayout {
  static constexpr int kThreads = QUANT ? 384 : 320;
  static constexpr int kStage8 = QUANT ? kBN * 128 : 0;         // 128 keys x 128 one-byte codes
  static constexpr int kOffK8 = kOffV + kVSt * kKVBytes;
  static constexpr int kOffV8 = kOffK8 + kStage8;
  static constexpr int kOffScale = kOffV8 + kStage8;            // float [2][32], int [2][32]
  static constexpr int kOffSide = kOffScale + (QUANT ? 512 : 0);  // float [4][2][32]
  static constexpr int kOffBar = kOffSide + (QUANT ? 1024 : 0);
  static constexpr int kSmem = kOffBar + 256 + 1024;            // + barriers, + alignment slack
};
constexpr uint32_t kTileCols = 256;       // tensor memory of a query tile: S (P over its
constexpr uint32_t kOCol = 128;           // first 64 columns) at column 0, O at 128
constexpr uint32_t kTmemCols = kQT * kTileCols;

// barrier indices; the P V products of a query tile complete on a ring of four barriers,
// so its softmax waits for one only when it rescales O (no phase of a barrier is ever two
// ahead of its waiter)
constexpr int kORing = 4;
constexpr int kBarQ = 0;
constexpr int kBarKF = 1;
constexpr int kBarKE = kBarKF + kKSt;
constexpr int kBarVF = kBarKE + kKSt;
constexpr int kBarVE = kBarVF + kVSt;
constexpr int kBarSF = kBarVE + kVSt;      // [query tile]
constexpr int kBarP = kBarSF + kQT;        // [query tile], kBM arrivals
constexpr int kBarO = kBarP + kQT;         // [query tile][ring]
constexpr int kBarFin = kBarO + kQT * kORing;
constexpr int kBarK8F = kBarFin + 1;       // quantised: codes of the tile staged (TMA)
constexpr int kBarK8E = kBarK8F + 1;       // quantised: staging read by the converters
constexpr int kBarV8F = kBarK8E + 1;
constexpr int kBarV8E = kBarV8F + 1;
constexpr int kBarSC = kBarV8E + 1;        // quantised: [4] a tile's K / V scales for the softmax
constexpr int kSideRing = 4;
constexpr int kNumBars = kBarSC + kSideRing;
static_assert(kNumBars * 8 + 8 <= 256, "barrier area");

// Instruction descriptors (kind::f16): f32 accumulator, bf16 A and B, M = 128.
// S = Q K^T: A and B K-major, N = 128 keys. O += P V: A (P) from tensor memory, B (V)
// MN-major, N = 128 channels.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                             ((uint32_t)(kBM >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(kD >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading and stride
// byte offsets (16-byte units), descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
// Two f16 (low half first) -> f32.
__device__ __forceinline__ void f16x2_to_f32(uint32_t h, float& lo, float& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\t"
      "cvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi) : "r"(h));
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, int w, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w),
        "r"(bar), "l"(policy)
      : "memory");
}

// ---- tensor memory and tcgen05 ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}
// D (tensor memory) = A B (+ D when acc != 0), A from tensor memory (K-major: a row per
// lane, two bf16 per column), B from a shared-memory descriptor.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
// D (tensor memory) = A B (+ D when acc != 0), A and B from shared-memory descriptors.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {"
               "%0, %1, %2, %3, %4, %5, %6, %7,"
               "%8, %9, %10, %11, %12, %13, %14, %15,"
               "%16, %17, %18, %19, %20, %21, %22, %23,"
               "%24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]),
                 "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                 "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                 "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
                 "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                 "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                 "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {"
               "%1, %2, %3, %4, %5, %6, %7, %8,"
               "%9, %10, %11, %12, %13, %14, %15, %16,"
               "%17, %18, %19, %20, %21, %22, %23, %24,"
               "%25, %26, %27, %28, %29, %30, %31, %32};"
               :: "r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]),
                 "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
                 "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]),
                 "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
                 "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
                 "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
                 "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
                 "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {"
               "%1, %2, %3, %4, %5, %6, %7, %8,"
               "%9, %10, %11, %12, %13, %14, %15, %16};"
               :: "r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]),
                 "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
                 "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]),
                 "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}
// tcgen05.wait::ld that also "rewrites" the loaded registers, so no use of them can be
// scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]),
                 "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                 "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct PrefillArgs {
  const int32_t* block_tables;  // [S][max_blocks_per_seq]
  const int32_t* context_lens;  // [S]
  const int32_t* query_start;   // [S + 1]
  void* out;                    // [T][Hq][128] bf16
  float* lse_out;               // [T][Hq] or null
  const float* k_scales;        // fp8 / int8: [num_blocks][Hkv]
  const float* v_scales;
  const int32_t* k_zeros;       // int8: [num_blocks][Hkv]
  const int32_t* v_zeros;
  float scale_log2;             // scale * log2(e)
  int num_seqs, num_tokens, num_q_heads, num_kv_heads, group;
  int max_blocks_per_seq, num_blocks, max_context_len, max_query_len;
};

// The new tokens of sequence s: rows [q0, q0 + n) of q, positions ctx - n .. ctx - 1.
// False (and flagged by thread 0) when the ranges are inconsistent.
__device__ __forceinline__ bool seq_rows(const PrefillArgs& a, int s, int& q0, int& n,
                                         int& ctx) {
  q0 = a.query_start[s];
  const int q1 = a.query_start[s + 1];
  n = q1 - q0;
  ctx = a.context_lens[s];
  const bool ok = q0 >= 0 && n >= 0 && q1 <= a.num_tokens && n <= ctx &&
                  ctx <= a.max_context_len && n <= a.max_query_len;
  if (!ok && threadIdx.x == 0) flag_error(PA_DEVERR_QUERY);
  return ok;
}

template <int BS, pa_dtype KV>
__global__ void __launch_bounds__(PfLayout<KV != PA_BF16>::kThreads, 1)
prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap qmap,
                  const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap) {
  static_assert(kBN % BS == 0 && kBN / BS <= 32, "block size");
  constexpr bool QUANT = KV != PA_BF16;  // fp8 / int8 codes, dequantised to bf16 in smem
  using L = PfLayout<QUANT>;
  constexpr int kThreads = L::kThreads, kOffBar = L::kOffBar;
  constexpr int NB_T = kBN / BS;  // blocks per key tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.group, TM = kBM / G;  // new tokens per query tile
  const int s = blockIdx.z, kvh = blockIdx.y;
  const int qp = (int)gridDim.x - 1 - (int)blockIdx.x;  // longest pairs (most keys) first

  int q0, n, ctx;
  if (!seq_rows(a, s, q0, n, ctx) || 2 * qp * TM >= n) return;  // before any set-up
  const int pos0 = ctx - n;                     // position of the sequence's first new token
  // query tiles 2qp and 2qp+1 of the sequence's new tokens; the second may be empty
  int tok0[kQT], ntok[kQT], pos_min[kQT], ntl[kQT];
#pragma unroll
  for (int x = 0; x < kQT; ++x) {
    tok0[x] = (2 * qp + x) * TM;
    ntok[x] = max(0, min(TM, n - tok0[x]));
    pos_min[x] = pos0 + tok0[x];
    ntl[x] = ntok[x] > 0 ? (pos_min[x] + ntok[x] + kBN - 1) / kBN : 0;  // key tiles it needs
  }
  const int kv_end = ntok[1] > 0 ? pos_min[1] + ntok[1] : pos_min[0] + ntok[0];
  const int ntiles = max(ntl[0], ntl[1]);

  const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK);
  const uint32_t sV = smem_u32(smem + kOffV);
  const uint32_t bar0 = smem_u32(smem + kOffBar);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * kNumBars);
  volatile int* dead = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int32_t* bt = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
  // a block the kernel cannot use: id out of range, or (int8) a zero point outside the
  // byte's range; such blocks are skipped (not loaded, their keys masked)
  auto block_bad = [&](int p) {
    if (p < 0 || p >= a.num_blocks) return true;
    if constexpr (KV == PA_INT8) {
      const int64_t bh = (int64_t)p * a.num_kv_heads + kvh;
      return !zero_in_range(a.k_zeros[bh]) || !zero_in_range(a.v_zeros[bh]);
    }
    return false;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if (i >= kBarP && i < kBarP + kQT) count = kBM;
      // quantised: the bf16 stages are filled, and the staging read, by the converters
      if (QUANT && ((i >= kBarKF && i < kBarKF + kKSt) || (i >= kBarVF && i < kBarVF + kVSt) ||
                    i == kBarK8E || i == kBarV8E || (i >= kBarSC && i < kBarSC + kSideRing)))
        count = kConvThreads;
      mbar_init(bar(i), count);
    }
    *dead = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  // any block id out of range among the keys the CTA sees? (then tiles are checked one by
  // one; otherwise no per-tile checks)
  int bad = 0;
  for (int b = threadIdx.x; b < (kv_end + BS - 1) / BS; b += kThreads) bad |= block_bad(bt[b]);
  tc_fence_before();
  const bool any_bad = __syncthreads_or(bad) != 0;
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ---------------- producer (whole warp): both Q tiles once, then K and V tiles through
    // their rings; lane b < NB_T holds block b of a key tile (read one tile ahead), each
    // lane issues one (block, half) box.
    if (lane == 0) {
      mbar_arrive_tx(bar(kBarQ), kQT * kQBytes);
      const uint64_t pol = evict_first_policy();
#pragma unroll
      for (int x = 0; x < kQT; ++x)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tma_load_4d(sQ + x * kQBytes + h * kQSlab, &qmap, 0, h, kvh * G, q0 + tok0[x],
                      bar(kBarQ), pol);
    }
    auto fetch = [&](int j) {
      int p = -1;
      if (j < ntiles && lane < NB_T && j * kBN + lane * BS < kv_end) {
        p = bt[j * NB_T + lane];
        if (p < 0 || p >= a.num_blocks) {
          flag_error(PA_DEVERR_BLOCK_ID);
          p = -1;
        } else if (block_bad(p)) {
          flag_error(PA_DEVERR_ZERO);
          p = -1;
        }
      }
      return p;
    };
    int last_k[kKSt], last_v[kVSt];
    for (int i = 0; i < kKSt; ++i) last_k[i] = -1;
    for (int i = 0; i < kVSt; ++i) last_v[i] = -1;
    int p_cur = fetch(0);
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (__shfl_sync(0xffffffffu, *dead ? 1 : 0, 0)) break;
      const int p_next = fetch(j + 1);
      const uint32_t bytes =
          (uint32_t)__popc(__ballot_sync(0xffffffffu, p_cur >= 0)) * 2u * BS * 128u;
      const int pb = __shfl_sync(0xffffffffu, p_cur, (lane >> 1) & 31);
#pragma unroll
      for (int kv = 0; kv < 2 && QUANT; ++kv) {
        // quantised: the tile's codes go to the staging buffer once the converters have
        // read the previous tile, with the blocks' scales (and zero points) beside them
        bool w = true;
        if (lane == 0 && j >= 1) w = mbar_wait(bar(kv ? kBarV8E : kBarK8E), (j - 1) & 1);
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
        if (lane < NB_T) {
          float* sc = reinterpret_cast<float*>(smem + L::kOffScale) + kv * 32;
          int* zp = reinterpret_cast<int*>(smem + L::kOffScale + 256) + kv * 32;
          const int64_t bh = (int64_t)(p_cur >= 0 ? p_cur : 0) * a.num_kv_heads + kvh;
          sc[lane] = p_cur >= 0 ? (kv ? a.v_scales : a.k_scales)[bh] : 1.f;  // absent: masked
          zp[lane] = (KV == PA_INT8 && p_cur >= 0) ? (kv ? a.v_zeros : a.k_zeros)[bh] : 0;
        }
        __syncwarp();
        const uint32_t fb = bar(kv ? kBarV8F : kBarK8F);
        if (lane == 0) mbar_arrive_tx(fb, bytes / 2);  // one byte per element
        __syncwarp();
        if (lane < NB_T && p_cur >= 0)
          tma_load_2d(smem_u32(smem + (kv ? L::kOffV8 : L::kOffK8)) + lane * BS * 128,
                      kv ? &vmap : &kmap, 0, (p_cur * a.num_kv_heads + kvh) * BS, fb);
        if (kv) last_v[0] = j;
        else last_k[0] = j;
      }
#pragma unroll
      for (int kv = 0; kv < 2 && !QUANT; ++kv) {
        const int nst = kv ? kVSt : kKSt;
        const int st = j % nst;
        bool w = true;
        if (lane == 0 && j >= nst)
          w = mbar_wait(bar((kv ? kBarVE : kBarKE) + st), ((j / nst) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
        const uint32_t fb = bar((kv ? kBarVF : kBarKF) + st);
        if (lane == 0) mbar_arrive_tx(fb, bytes);
        __syncwarp();
        if (lane < 2 * NB_T && pb >= 0) {
          const int b = lane >> 1, h = lane & 1;
          const uint32_t dst = (kv ? sV : sK) + st * kKVBytes + h * kKVSlab + b * BS * 128;
          tma_load_3d(dst, kv ? &vmap : &kmap, 0, h, (pb * a.num_kv_heads + kvh) * BS, fb);
        }
        if (kv) last_v[st] = j;
        else last_k[st] = j;
      }
      if (!ok) {
        if (lane == 0) {
          flag_error(PA_DEVERR_TIMEOUT);
          *dead = 1;
        }
        break;
      }
      p_cur = p_next;
    }
    if (lane == 0 && *dead) {
      // copies still in flight complete before the CTA's shared memory is released
      if (QUANT) {
        if (last_k[0] >= 0) mbar_wait(bar(kBarK8F), last_k[0] & 1);
        if (last_v[0] >= 0) mbar_wait(bar(kBarV8F), last_v[0] & 1);
      } else {
        for (int i = 0; i < kKSt; ++i)
          if (last_k[i] >= 0) mbar_wait(bar(kBarKF + i), (last_k[i] / kKSt) & 1);
        for (int i = 0; i < kVSt; ++i)
          if (last_v[i] >= 0) mbar_wait(bar(kBarVF + i), (last_v[i] / kVSt) & 1);
      }
      mbar_wait(bar(kBarQ), 0);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // S_x(j) = Q_x K_j^T into S buffer j % 2 of query tile x
      auto issue_s = [&](int x, int j) {
        const uint32_t kst = sK + (j % kKSt) * kKVBytes;
        const uint32_t qx = sQ + x * kQBytes;
        const uint32_t d = tmem + x * kTileCols;  // one S buffer per query tile
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t oq = (kk >> 2) * kQSlab + (kk & 3) * 32;
          const uint32_t ok_ = (kk >> 2) * kKVSlab + (kk & 3) * 32;
          umma_bf16(d, sdesc(qx + oq, 16, 1024), sdesc(kst + ok_, 16, 1024), kIdescS, kk > 0);
        }
        umma_commit(bar(kBarSF + x));
      };
      // O_x += P_x(j) V_j, P_x(j) over S_x(j) in tensor memory
      auto issue_pv = [&](int x, int j) {
        const uint32_t vst = sV + (j % kVSt) * kKVBytes;
        const uint32_t px = tmem + x * kTileCols;  // P_x(j) over S_x(j)
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_bf16_ts(tmem + x * kTileCols + kOCol, px + kk * 8,
                       sdesc(vst + kk * 16 * 128, kKVSlab, 1024), kIdescPV, (j > 0 || kk > 0));
        umma_commit(bar(kBarO + x * kORing + j % kORing));
      };
      bool live = mbar_wait(bar(kBarQ), 0) && mbar_wait(bar(kBarKF), 0);
      if (live) {
        tc_fence_after();
        for (int x = 0; x < kQT; ++x)
          if (ntl[x] > 0) issue_s(x, 0);
        umma_commit(bar(kBarKE));  // the K stage is free once the S products are done
      }
      // per key tile: P V of query tile 0, then its next S (the S buffer holds P until the
      // P V product has read it: products run in issue order), then the same for tile 1
      for (int j = 0; live && j < ntiles; ++j) {
        if (!mbar_wait(bar(kBarVF + (j % kVSt)), (j / kVSt) & 1)) {
          live = false;
          break;
        }
        bool kready = false;
        for (int x = 0; x < kQT && live; ++x) {
          if (j >= ntl[x]) continue;
          if (!mbar_wait(bar(kBarP + x), j & 1)) {
            live = false;
            break;
          }
          tc_fence_after();
          issue_pv(x, j);
          if (j + 1 < ntl[x]) {
            if (!kready && !mbar_wait(bar(kBarKF + ((j + 1) % kKSt)), ((j + 1) / kKSt) & 1)) {
              live = false;
              break;
            }
            kready = true;
            issue_s(x, j + 1);
          }
        }
        if (kready) umma_commit(bar(kBarKE + ((j + 1) % kKSt)));
        umma_commit(bar(kBarVE + (j % kVSt)));
        if (*dead) live = false;
      }
      if (!live) {
        flag_error(PA_DEVERR_TIMEOUT);
        *dead = 1;
      }
      // every product of the CTA completes before tensor memory is released
      umma_commit(bar(kBarFin));
      mbar_wait(bar(kBarFin), 0);
    }
    __syncwarp();
  } else if (QUANT && warp >= kConvWarp0) {
    // ---------------- converters (quantised caches): staged codes -> bf16 stages ----------------
    // Thread ct takes 16 chunks of 16 codes: chunk = ct + 64 it, key row t = chunk / 8,
    // channels 16 (chunk % 8) ..; value = the E4M3 code's value (fp8) or code - zero (int8)
    // of the key's block, exact in bf16, stored in the 128-byte-swizzled K-major (K) /
    // MN-major (V) layout the products read, exactly where TMA would put bf16. The blocks'
    // scales go to the softmax through a ring of four slots (K scale on the scores, V
    // scale on P), so the dequantisation adds no rounding.
    const int ct = threadIdx.x - kConvWarp0 * 32;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
#pragma unroll 1
      for (int kv = 0; kv < 2; ++kv) {
        const int nst = kv ? kVSt : kKSt;
        const int st = j % nst;
        bool w = !*dead && mbar_wait(bar(kv ? kBarV8F : kBarK8F), j & 1);
        if (w && j >= nst) w = mbar_wait(bar((kv ? kBarVE : kBarKE) + st), ((j / nst) - 1) & 1);
        if (!w) {
          ok = false;
          break;
        }
        const uint8_t* src = smem + (kv ? L::kOffV8 : L::kOffK8);
        const float* sc = reinterpret_cast<const float*>(smem + L::kOffScale) + kv * 32;
        const int* zp = reinterpret_cast<const int*>(smem + L::kOffScale + 256) + kv * 32;
        const uint32_t dst = (kv ? sV : sK) + st * kKVBytes;
#pragma unroll 4
        for (int it = 0; it < kBN * 8 / kConvThreads; ++it) {
          const int chunk = ct + kConvThreads * it;
          const int t = chunk >> 3, q8 = chunk & 7;
          const uint4 raw = *reinterpret_cast<const uint4*>(src + t * 128 + q8 * 16);
          const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t o[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float f[4];
            if constexpr (KV == PA_INT8) {
              const float z = (float)zp[t / BS];
#pragma unroll
              for (int e = 0; e < 4; ++e) f[e] = (float)(int8_t)(wd[k] >> (8 * e)) - z;
            } else {  // E4M3 -> f16 -> f32, both exact
              f16x2_to_f32(e4m3x2_to_f16x2((uint16_t)(wd[k] & 0xffffu)), f[0], f[1]);
              f16x2_to_f32(e4m3x2_to_f16x2((uint16_t)(wd[k] >> 16)), f[2], f[3]);
            }
            o[2 * k] = pack_bf16x2(f[0], f[1]);
            o[2 * k + 1] = pack_bf16x2(f[2], f[3]);
          }
          // channels 16 q8 .. 16 q8 + 15: half q8 / 4 of the channels, 16-byte chunks
          // 2 (q8 % 4) and 2 (q8 % 4) + 1 of the key's 128-byte row, swizzled by row % 8
          const uint32_t row = dst + (q8 >> 2) * kKVSlab + t * 128;
          const int c0 = 2 * (q8 & 3);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       ::"r"(row + ((c0 ^ (t & 7)) << 4)), "r"(o[0]), "r"(o[1]), "r"(o[2]),
                         "r"(o[3]) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       ::"r"(row + (((c0 + 1) ^ (t & 7)) << 4)), "r"(o[4]), "r"(o[5]), "r"(o[6]),
                         "r"(o[7]) : "memory");
        }
        // the tile's block scales for the softmax (slot j % 4 is free: the softmax of tile
        // j - 4 finished before the S products of tile j - 2, which freed this stage)
        if (ct < NB_T)
          reinterpret_cast<float*>(smem + L::kOffSide)[((j % kSideRing) * 2 + kv) * 32 + ct] =
              sc[ct];
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(bar(kv ? kBarV8E : kBarK8E));           // staging read
        mbar_arrive(bar((kv ? kBarVF : kBarKF) + st));       // bf16 stage written
      }
      if (ok) mbar_arrive(bar(kBarSC + j % kSideRing));     // K and V scales of tile j
    }
    if (!ok) {
      flag_error(PA_DEVERR_TIMEOUT);
      *dead = 1;
    }
  } else {
    // ------- softmax: warpgroup x owns query tile x, thread r its row r (tensor-memory lane r) -------
    const int x = warp >> 2;
    const int r = threadIdx.x & (kBM - 1);
    const int tr = r / G, g = r - tr * G;
    const int nt = ntl[x];
    const int pmin = pos_min[x];
    const bool row_valid = tr < ntok[x];
    const int prow = pmin + min(tr, max(ntok[x], 1) - 1);   // this row's position
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + x * kTileCols;
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;                  // log2-domain reference max, sum
    bool ok = true;
    // waits are made warp-uniform: the tcgen05.ld / st below are warp-collective
    auto wait_all = [&](uint32_t b, uint32_t parity) {
      const bool w = !*dead && mbar_wait(b, parity);
      return __all_sync(0xffffffffu, w);
    };
    for (int j = 0; j < nt; ++j) {
      if (!wait_all(bar(kBarSF + x), j & 1)) { ok = false; break; }
      if (QUANT && !wait_all(bar(kBarSC + j % kSideRing), (j / kSideRing) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int t0 = j * kBN;
      const int vlim = min(kBN, kv_end - t0);             // keys of the tile that were loaded
      uint32_t badm = 0;  // blocks of the tile with an out-of-range id (skipped, masked)
      if (any_bad) {
        bool b = false;
        if (lane < (vlim + BS - 1) / BS) b = block_bad(bt[t0 / BS + lane]);
        badm = __ballot_sync(0xffffffffu, b);
      }
      const uint32_t sbuf = lane_addr;  // the query tile's S buffer
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(sbuf + c * 32, sv[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_wait_ld(sv[c]);
      // quantised caches: the scores of key block b carry its K scale (the products ran on
      // the codes' exact values); scale them into the log2 domain before the mask, so that
      // masked keys are -inf whatever their block's scale
      const float* side = reinterpret_cast<const float*>(smem + L::kOffSide) +
                          (j % kSideRing) * 2 * 32;  // [K scales][V scales] of tile j
      if constexpr (QUANT) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int b = 0; b < 32 / BS; ++b) {
            const float ks = side[(c * 32) / BS + b] * sl2;
#pragma unroll
            for (int e = b * BS; e < (b + 1) * BS; ++e)
              sv[c][e] = __float_as_uint(__uint_as_float(sv[c][e]) * ks);
          }
      }
      // causal / existence / bad-block mask, then the row max of the raw scores
      const bool masked = t0 + kBN - 1 > pmin || badm != 0;  // uniform in the warpgroup
      if (masked) {
        const int lim = prow - t0;                   // visible: key <= lim
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = c * 32 + e;
            if (col > lim || ((badm >> (col / BS)) & 1u)) sv[c][e] = 0xff800000u;  // -inf
          }
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(sv[c][e]));
#pragma unroll
      for (int k = 0; k < 4; ++k) mx8[k] = fmaxf(mx8[k], mx8[k + 4]);
      const float mx =
          fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])) * (QUANT ? 1.f : sl2);
      const float m_new = fmaxf(m_used, mx);
      float alpha = 1.f;
      if (m_new > m_used + 8.f) {  // lazy rescale: P stays below 2^8 otherwise
        alpha = fast_exp2(m_used - m_new);
        m_used = m_new;
      }
      const float mneg = m_used == -INFINITY ? 0.f : -m_used;
      float rs8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) rs8[k] = 0.f;
      const float xs = QUANT ? 1.f : sl2;  // quantised: scores already scaled above
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sv[c][e]), xs, mneg));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sv[c][e + 1]), xs, mneg));
          rs8[e & 7] += p0;
          rs8[(e + 1) & 7] += p1;
          if constexpr (QUANT) {  // P carries the V scale of its key's block
            const float vs = side[32 + (c * 32 + e) / BS];
            pk[e >> 1] = pack_bf16x2(p0 * vs, p1 * vs);
          } else {
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
        }
        tmem_st16(sbuf + c * 16, pk);  // P over the first 64 columns of S
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) rs8[k] += rs8[k + 4];
      l = l * alpha + ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3]));
      tmem_wait_st();
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O holds P(j-1) V(j-1) once the previous product is done: rescale it
        if (!wait_all(bar(kBarO + x * kORing + (j - 1) % kORing), ((j - 1) / kORing) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kOCol + c * 32, o);
          tmem_wait_ld(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_addr + kOCol + c * 32, o);
        }
        tmem_wait_st();
      }
      // rows of V past the keys that exist or in a skipped block may hold anything (NaN):
      // zero them before the products read them (both warpgroups zero the same rows)
      if (vlim < kBN || badm != 0) {
        if (!wait_all(bar(kBarVF + (j % kVSt)), (j / kVSt) & 1)) { ok = false; break; }
        if (r >= vlim || ((badm >> (r / BS)) & 1u)) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t vrow = sV + (j % kVSt) * kKVBytes + h * kKVSlab + r * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + k * 16), "r"(0)
                           : "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tc_fence_before();
      mbar_arrive(bar(kBarP + x));
    }
    if (ok && nt > 0)
      ok = wait_all(bar(kBarO + x * kORing + (nt - 1) % kORing), ((nt - 1) / kORing) & 1);
    if (ok && nt > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t orow = (int64_t)(q0 + tok0[x] + tr) * a.num_q_heads + kvh * G + g;
      uint16_t* op = static_cast<uint16_t*>(a.out) + orow * kD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_addr + kOCol + c * 32, o);
        tmem_wait_ld(o);
        if (row_valid) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv);
            *reinterpret_cast<uint4*>(op + c * 32 + 8 * k) = w;
          }
        }
      }
      if (row_valid && a.lse_out != nullptr)
        a.lse_out[orow] = l > 0.f ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
    } else if (!ok) {
      if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
      *dead = 1;
    }
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
// q [T][Hq][128] bf16 as (64 channels, half, head, token); a box is the tile's rows of one
// half: G heads x (128 / G) tokens, rows (token, head) of 128 B.
inline bool make_q_map(CUtensorMap* m, const void* q, int num_tokens, int hq, int group) {
  auto enc = tc::encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {64, 2, (cuuint64_t)hq, (cuuint64_t)num_tokens};
  cuuint64_t strides[3] = {128, 256, (cuuint64_t)hq * 256};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)group, (cuuint32_t)(kBM / group)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// A bf16 pool [NB][Hkv][BS][128] as (64 channels, half, token row); a box is one block's
// tokens of one half.
inline bool make_kv_map(CUtensorMap* m, const void* pool, int64_t token_rows, int bs) {
  auto enc = tc::encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {64, 2, (cuuint64_t)token_rows};
  cuuint64_t strides[2] = {128, 256};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)bs};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// A one-byte-code pool (fp8 / int8) [NB][Hkv][BS][128] as rows of 128 bytes; a box is one
// block's tokens, landing unswizzled in the staging buffer.
inline bool make_kv8_map(CUtensorMap* m, const void* pool, int64_t token_rows, int bs) {
  auto enc = tc::encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)token_rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, (cuuint32_t)bs};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(pool), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int BS, pa_dtype KV>
inline cudaError_t launch_bs(const PrefillArgs& a, const void* q, const void* kc, const void* vc,
                             cudaStream_t st) {
  using L = PfLayout<KV != PA_BF16>;
  CUtensorMap qm, km, vm;
  const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
  const bool maps = KV == PA_BF16
                        ? make_kv_map(&km, kc, rows, BS) && make_kv_map(&vm, vc, rows, BS)
                        : make_kv8_map(&km, kc, rows, BS) && make_kv8_map(&vm, vc, rows, BS);
  if (!maps || !make_q_map(&qm, q, a.num_tokens, a.num_q_heads, a.group))
    return cudaErrorInvalidValue;
  static tc::DeviceCache slots;
  int per_sm = 0;
  const cudaError_t e =
      tc::resident_per_sm(prefill_tc_kernel<BS, KV>, L::kThreads, L::kSmem, slots, &per_sm);
  if (e != cudaSuccess) return e;
  const int tiles = (a.max_query_len * a.group + kBM - 1) / kBM;
  const dim3 grid((tiles + kQT - 1) / kQT, a.num_kv_heads, a.num_seqs);
  prefill_tc_kernel<BS, KV><<<grid, L::kThreads, L::kSmem, st>>>(a, qm, km, vm);
  return cudaGetLastError();
}

}  // namespace pf

// Shapes the tensor-core prefill kernel takes: bf16 q / out, a bf16, fp8 or int8 cache,
// head_dim 128, a group that divides the 128 tile rows, blocks of 8, 16 or 32 tokens.
inline bool prefill_tc_supported(const pa_decode_desc* d) {
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->q_dtype != PA_BF16 || d->out_dtype != PA_BF16) return false;
  if (d->kv_dtype != PA_BF16 && d->kv_dtype != PA_FP8_E4M3 && d->kv_dtype != PA_INT8)
    return false;
  if (d->head_dim != pf::kD) return false;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return false;
  if (d->block_size != 8 && d->block_size != 16 && d->block_size != 32) return false;
  return (int64_t)d->num_blocks * d->num_kv_heads * d->block_size < ((int64_t)1 << 31);
}

inline cudaError_t launch_prefill_tc(const pf::PrefillArgs& a, int block_size, pa_dtype kv,
                                     const void* q, const void* kc, const void* vc,
                                     cudaStream_t st) {
  auto by_bs = [&](auto kvc) -> cudaError_t {
    constexpr pa_dtype KV = decltype(kvc)::value;
    if (block_size == 8) return pf::launch_bs<8, KV>(a, q, kc, vc, st);
    if (block_size == 32) return pf::launch_bs<32, KV>(a, q, kc, vc, st);
    return pf::launch_bs<16, KV>(a, q, kc, vc, st);
  };
  if (kv == PA_FP8_E4M3) return by_bs(std::integral_constant<pa_dtype, PA_FP8_E4M3>{});
  if (kv == PA_INT8) return by_bs(std::integral_constant<pa_dtype, PA_INT8>{});
  return by_bs(std::integral_constant<pa_dtype, PA_BF16>{});
}

}  // namespace pa
