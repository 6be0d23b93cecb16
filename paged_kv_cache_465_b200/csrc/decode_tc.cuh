// Paged decode attention on the tensor cores, for bf16 and fp8-e4m3 caches (head_dim 128,
// up to 8 query heads per kv head).
//
// Same function and work decomposition as the CUDA-core path (decode_simt.cuh): a CTA of 4
// warps takes one (sequence, kv head, partition) item, warp w walks the item's logical
// blocks w, w+4, ... and the warps are merged at the end, so results do not depend on
// where blocks sit physically ([Ch4PA] "PagedAttention algorithm": blocks are gathered
// through the block table; [KVPaged] "GQA and MQA": one K/V tile serves all G query heads
// of its group).
//
// Why tensor cores: per KV element the group needs G multiply-adds for q.K and G for P.V;
// at B200's HBM rate that is ~(G+1) fp32 issue slots per element on the CUDA cores, more
// than the SMs can issue for G >= 4. Here one 16-token block costs a warp 16 mma.sync
// (m16n8k16) instead: S^T = K . Q^T (M = 16 tokens, N = 8 query heads, K = 128 channels)
// and O^T += V^T . P^T (M = 16 channels x 8 tiles, N = 8 heads, K = 16 tokens). Both
// products are skinny (N = G <= 8), so the warp-level mma fits them; the kernel stays
// bound by HBM.
//
// Data movement: each (physical block, kv head) tile is contiguous in the pool
// ([NB][Hkv][16][128]); one TMA tensor copy (cp.async.bulk.tensor, 128-byte swizzle, L2
// evict-first) brings it into shared memory, completing on a per-stage mbarrier. Every
// warp owns a ring of NSTAGE stages and keeps NSTAGE blocks (K and V) in flight while it
// computes. ldmatrix reads the swizzled tiles without bank conflicts; .trans gives V^T.
//
// fp8: E4M3 bytes are widened exactly to f16 (cvt.rn.f16x2.e4m3x2) and multiplied in f16;
// q is scaled by a power of two into f16 range (undone exactly in the score scale). The
// per-(block, kv head) K scale folds into the score scale; the V scale folds into P as
// P * v_scale[b] / v_ref, where v_ref is the running maximum V scale of the warp (the
// accumulator is rescaled when it grows, like the running softmax maximum), so P stays
// within [0, 1].
//
// Every wait on an mbarrier is bounded (about one second of %globaltimer); on expiry the
// warp records PA_DEVERR_TIMEOUT, stops consuming, waits (bounded) for the copies it
// issued and then finishes normally.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "decode_simt.cuh"

namespace pa {

// 0 = automatic, 1 = CUDA-core path only, 2 = tensor cores where supported.
static int g_decode_impl = 0;

namespace tc {

constexpr int kD = 128;
constexpr int kNW = 4;                         // warps per CTA
constexpr uint64_t kWaitNs = 1000000000ull;    // bound of one mbarrier wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity; false after ~kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) return false;
  }
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// 2-D TMA tile load into this CTA's shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
template <bool F16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}
__device__ __forceinline__ uint32_t lo16(uint32_t x) { return x & 0xffffu; }
__device__ __forceinline__ uint32_t hi16(uint32_t x) { return x >> 16; }

// Byte address of (row r, 16-byte chunk c) in a tile of 128-byte rows written by TMA with
// the 128-byte swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz(uint32_t tile, int r, int c) {
  return tile + r * 128 + ((c ^ (r & 7)) << 4);
}

template <pa_dtype KV>
struct TcCfg {
  static constexpr bool kFp8 = KV == PA_FP8_E4M3;
  static constexpr int kTile = kFp8 ? 2048 : 4096;      // one (block, head) tile of K or V
  static constexpr int kStage = 2 * kTile;              // K + V
  static constexpr int kNStage = kFp8 ? 4 : 3;          // blocks in flight per warp
  static constexpr int kSmem = kNW * kNStage * kStage + kNW * kNStage * 8 + 1024;
};

template <pa_dtype KV>
__global__ void __launch_bounds__(kNW * 32)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap) {
  using C = TcCfg<KV>;
  constexpr bool FP8 = C::kFp8;
  constexpr int TILE = C::kTile, STAGE = C::kStage, NST = C::kNStage;
  constexpr int ROWS = TILE / 128;  // tensor-map rows per tile (32 bf16 / 16 fp8)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));

  const int part = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
  const int ctx = checked_ctx(a, s);
  const int t0 = part * a.part_tokens;
  if (!a.final_pass && t0 >= ctx) return;
  const int t1 = min(ctx, t0 + a.part_tokens);
  const int G = a.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;

  const uint32_t wtiles = smem_u32(smem + warp * NST * STAGE);
  const uint32_t bars = smem_u32(smem + kNW * NST * STAGE) + warp * NST * 8;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) mbar_init(bars + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncwarp();

  // ---- q of the group as mma B fragments (rows g >= G are zero) ----
  uint32_t qf[8][2];
  float zscale = a.scale_log2;
  {
    const uint16_t* qp = static_cast<const uint16_t*>(a.q) +
                         ((int64_t)s * a.num_q_heads + kvh * G + gq) * kD;
    const bool live = gq < G;
    if constexpr (!FP8) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        qf[j][0] = live ? *reinterpret_cast<const uint32_t*>(qp + 16 * j + 2 * tq) : 0u;
        qf[j][1] = live ? *reinterpret_cast<const uint32_t*>(qp + 16 * j + 8 + 2 * tq) : 0u;
      }
    } else {
      // k-step c uses channels 16c + 4tq + {0,1} (low pair) and + {2,3} (high pair)
      float qv[8][4];
      float amax = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint2 w = live ? *reinterpret_cast<const uint2*>(qp + 16 * c + 4 * tq) : make_uint2(0, 0);
        qv[c][0] = bf16_lo(w.x); qv[c][1] = bf16_hi(w.x);
        qv[c][2] = bf16_lo(w.y); qv[c][3] = bf16_hi(w.y);
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(qv[c][e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      // power of two putting max|q| in [2^14, 2^15): exact scaling into f16 range
      int e = 0;
      const uint32_t ebits = (__float_as_uint(amax) >> 23) & 0xff;
      if (ebits != 0 && ebits != 0xff) e = 15 - ((int)ebits - 126);
      e = max(-100, min(100, e));
      const float up = __uint_as_float((uint32_t)(127 + e) << 23);
      const float down = __uint_as_float((uint32_t)(127 - e) << 23);
      zscale *= down;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        qf[c][0] = pack_f16x2(qv[c][0] * up, qv[c][1] * up);
        qf[c][1] = pack_f16x2(qv[c][2] * up, qv[c][3] * up);
      }
    }
  }

  // ---- this warp's blocks and its block-table windows (32 entries per register) ----
  const int b_begin = t0 / kBS, b_end = (t1 + kBS - 1) / kBS;
  const int nblk = b_end - b_begin;
  const int nmine = nblk > warp ? (nblk - warp + kNW - 1) / kNW : 0;
  const int32_t* bt = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
  auto load_window = [&](int base, int& p, float& ks, float& vs) {
    const int k = base + lane;
    p = -2;
    ks = 1.f;
    vs = 1.f;
    if (k < nmine) {
      p = bt[b_begin + warp + k * kNW];
      if (p < 0 || p >= a.num_blocks) {
        flag_error(PA_DEVERR_BLOCK_ID);
        p = -1;
      } else if constexpr (FP8) {
        ks = a.k_scales[(int64_t)p * a.num_kv_heads + kvh];
        vs = a.v_scales[(int64_t)p * a.num_kv_heads + kvh];
      }
    }
  };
  int cur_p, nxt_p;
  float cur_ks, cur_vs, nxt_ks, nxt_vs;
  load_window(0, cur_p, cur_ks, cur_vs);
  load_window(32, nxt_p, nxt_ks, nxt_vs);
  const uint64_t policy = evict_first_policy();
  const int kvrow_stride = ROWS;  // tensor-map rows per (block, head) tile
  auto issue = [&](int k, int wbase, int stage) {
    const int rel = k - wbase;
    const int p = rel < 32 ? __shfl_sync(0xffffffffu, cur_p, rel)
                           : __shfl_sync(0xffffffffu, nxt_p, rel - 32);
    if (lane == 0) {
      const uint32_t bar = bars + 8 * stage;
      if (p >= 0) {
        const int row = (p * a.num_kv_heads + kvh) * kvrow_stride;
        const uint32_t dst = wtiles + stage * STAGE;
        mbar_arrive_tx(bar, STAGE);
        tma_load_2d(dst, &kmap, 0, row, bar, policy);
        tma_load_2d(dst + TILE, &vmap, 0, row, bar, policy);
      } else {
        mbar_arrive(bar);  // completes the phase; the consumer skips the block
      }
    }
  };
  for (int k = 0; k < NST && k < nmine; ++k) issue(k, 0, k);

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float vref = 0.f;  // fp8: running max of the V scales seen (acc is in units of vref)
  bool timed_out = false;
  int consumed = 0;

  for (int i = 0; i < nmine; ++i) {
    const int wbase = i & ~31;
    if ((i & 31) == 0 && i > 0) {
      cur_p = nxt_p; cur_ks = nxt_ks; cur_vs = nxt_vs;
      load_window(i + 32, nxt_p, nxt_ks, nxt_vs);
    }
    const int stage = i % NST;
    const uint32_t par = (uint32_t)((i / NST) & 1);
    const int p = __shfl_sync(0xffffffffu, cur_p, i & 31);
    if (!mbar_wait(bars + 8 * stage, par)) {
      if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
      timed_out = true;
      break;
    }
    consumed = i + 1;
    if (p >= 0) {
      const int b = b_begin + warp + i * kNW;
      const int nvalid = min(kBS, t1 - b * kBS);
      const uint32_t kt = wtiles + stage * STAGE, vt = kt + TILE;
      float zs = zscale;
      float pv = 1.f, beta = 1.f;
      if constexpr (FP8) {
        const float ks = __shfl_sync(0xffffffffu, cur_ks, i & 31);
        const float vs = __shfl_sync(0xffffffffu, cur_vs, i & 31);
        zs *= ks;
        const float vnew = fmaxf(vref, vs);
        beta = vref > 0.f ? vref / vnew : 1.f;
        pv = vnew > 0.f ? vs / vnew : 0.f;
        vref = vnew;
      }
      // ---- S^T = K Q^T : 16 tokens x 8 heads ----
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (!FP8) {
        // rows of the tile: 2*token + (channel >= 64); chunk = (channel % 64) / 8
        const int mi = lane >> 3;
        const int tok = (lane & 7) + 8 * (mi & 1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int d0 = 16 * j + 8 * (mi >> 1);
          uint32_t r[4];
          ldsm_x4(swz(kt, 2 * tok + (d0 >> 6), (d0 & 63) >> 3), r);
          mma16816<false>(sc, r, qf[j][0], qf[j][1]);
        }
      } else {
        const int mi = lane >> 3;
        const int tok = (lane & 7) + 8 * (mi & 1);
#pragma unroll
        for (int cp = 0; cp < 4; ++cp) {
          uint32_t r[4];
          ldsm_x4(swz(kt, tok, 2 * cp + (mi >> 1)), r);
          uint32_t x0[4] = {e4m3x2_to_f16x2((uint16_t)lo16(r[0])), e4m3x2_to_f16x2((uint16_t)lo16(r[1])),
                            e4m3x2_to_f16x2((uint16_t)hi16(r[0])), e4m3x2_to_f16x2((uint16_t)hi16(r[1]))};
          mma16816<true>(sc, x0, qf[2 * cp][0], qf[2 * cp][1]);
          uint32_t x1[4] = {e4m3x2_to_f16x2((uint16_t)lo16(r[2])), e4m3x2_to_f16x2((uint16_t)lo16(r[3])),
                            e4m3x2_to_f16x2((uint16_t)hi16(r[2])), e4m3x2_to_f16x2((uint16_t)hi16(r[3]))};
          mma16816<true>(sc, x1, qf[2 * cp + 1][0], qf[2 * cp + 1][1]);
        }
      }
      // ---- online softmax (log2 domain); thread holds tokens gq, gq+8 x heads 2tq, 2tq+1 ----
      const bool va = gq < nvalid, vb = gq + 8 < nvalid;
      const float z0 = va ? sc[0] * zs : -INFINITY, z1 = va ? sc[1] * zs : -INFINITY;
      const float z2 = vb ? sc[2] * zs : -INFINITY, z3 = vb ? sc[3] * zs : -INFINITY;
      float bm0 = fmaxf(z0, z2), bm1 = fmaxf(z1, z3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, o));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, o));
      }
      const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
      const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      const float p0 = fast_exp2(z0 - mn0), p1 = fast_exp2(z1 - mn1);
      const float p2 = fast_exp2(z2 - mn0), p3 = fast_exp2(z3 - mn1);
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
      if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f || beta != 1.f)) {
        const float f0 = al0 * beta, f1 = al1 * beta;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          acc[t][0] *= f0; acc[t][1] *= f1; acc[t][2] *= f0; acc[t][3] *= f1;
        }
      }
      // P^T as B fragments: pack [token][head] pairs, transpose 8x8 in registers
      uint32_t pb0, pb1;
      if constexpr (FP8) {
        pb0 = movm_t(pack_f16x2(p0 * pv, p1 * pv));
        pb1 = movm_t(pack_f16x2(p2 * pv, p3 * pv));
      } else {
        pb0 = movm_t(pack_bf16x2(p0, p1));
        pb1 = movm_t(pack_bf16x2(p2, p3));
      }
      // rows of tokens past the context may hold anything: zero them before P.V
      if (nvalid < kBS) {
        const int bytes_per_tok = TILE / kBS;
        for (int o = nvalid * bytes_per_tok + lane * 16; o < TILE; o += 32 * 16)
          asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(vt + o), "r"(0) : "memory");
        __syncwarp();
      }
      // ---- O^T += V^T P^T ----
      if constexpr (!FP8) {
        const int mi = lane >> 3;
        const int tok = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int d0 = 16 * t + 8 * (mi & 1);
          uint32_t r[4];
          ldsm_x4_t(swz(vt, 2 * tok + (d0 >> 6), (d0 & 63) >> 3), r);
          mma16816<false>(acc[t], r, pb0, pb1);
        }
      } else {
        const int mi = lane >> 3;
        const int tok = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
        for (int cp = 0; cp < 4; ++cp) {
          uint32_t r[4];
          ldsm_x4_t(swz(vt, tok, 2 * cp + (mi & 1)), r);
          uint32_t y[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) y[u] = __byte_perm(r[u], 0, 0x3120);
          uint32_t ev[4] = {e4m3x2_to_f16x2((uint16_t)lo16(y[0])), e4m3x2_to_f16x2((uint16_t)lo16(y[1])),
                            e4m3x2_to_f16x2((uint16_t)lo16(y[2])), e4m3x2_to_f16x2((uint16_t)lo16(y[3]))};
          mma16816<true>(acc[2 * cp], ev, pb0, pb1);
          uint32_t od[4] = {e4m3x2_to_f16x2((uint16_t)hi16(y[0])), e4m3x2_to_f16x2((uint16_t)hi16(y[1])),
                            e4m3x2_to_f16x2((uint16_t)hi16(y[2])), e4m3x2_to_f16x2((uint16_t)hi16(y[3]))};
          mma16816<true>(acc[2 * cp + 1], od, pb0, pb1);
        }
      }
    }
    __syncwarp();
    if (i + NST < nmine) issue(i + NST, wbase, stage);
  }
  if (timed_out) {
    // wait (bounded) for every copy this warp issued and did not consume
    const int issued = min(nmine, consumed + NST);
    for (int k = consumed; k < issued; ++k) {
      if (!mbar_wait(bars + 8 * (k % NST), (uint32_t)((k / NST) & 1))) break;
    }
  }

  // ---- merge the warps through shared memory (stage buffers are free now) ----
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();
  float* sacc = reinterpret_cast<float*>(smem);             // [kNW][8][kD]
  float* smx = sacc + kNW * 8 * kD;                          // [kNW][8]
  float* slx = smx + kNW * 8;                                // [kNW][8]
  if (gq == 0) {
    smx[warp * 8 + 2 * tq] = m0; smx[warp * 8 + 2 * tq + 1] = m1;
    slx[warp * 8 + 2 * tq] = l0; slx[warp * 8 + 2 * tq + 1] = l1;
  }
  const float unit = FP8 ? vref : 1.f;
  float* wacc = sacc + warp * 8 * kD;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    int dA, dB;
    if constexpr (FP8) {
      const int cp = t >> 1, par = t & 1;
      dA = 32 * cp + 2 * gq + par;
      dB = 32 * cp + 16 + 2 * gq + par;
    } else {
      dA = 16 * t + gq;
      dB = 16 * t + 8 + gq;
    }
    wacc[(2 * tq) * kD + dA] = acc[t][0] * unit;
    wacc[(2 * tq + 1) * kD + dA] = acc[t][1] * unit;
    wacc[(2 * tq) * kD + dB] = acc[t][2] * unit;
    wacc[(2 * tq + 1) * kD + dB] = acc[t][3] * unit;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
    const int g = idx / kD, d = idx % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, smx[w * 8 + g]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float f = fast_exp2(smx[w * 8 + g] - M);
        L = fmaf(f, slx[w * 8 + g], L);
        A = fmaf(f, sacc[(w * 8 + g) * kD + d], A);
      }
    }
    emit(a, s, kvh * G + g, part, kD, d, M, L, A);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// The pool seen as rows of 128 bytes: a (block, head) tile is `rows` consecutive rows.
inline bool make_map(CUtensorMap* m, const void* base, int64_t total_rows, pa_dtype kv) {
  auto enc = encoder();
  if (enc == nullptr) return false;
  const bool fp8 = kv == PA_FP8_E4M3;
  cuuint64_t dims[2] = {(cuuint64_t)(fp8 ? 128 : 64), (cuuint64_t)total_rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {(cuuint32_t)(fp8 ? 128 : 64), (cuuint32_t)(fp8 ? 16 : 32)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <pa_dtype KV>
inline cudaError_t launch_tc_kv(const DecodeArgs& a, const pa_decode_desc* d, dim3 grid,
                                cudaStream_t st) {
  using C = TcCfg<KV>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<KV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int64_t rows = (int64_t)d->num_blocks * d->num_kv_heads * (C::kTile / 128);
  CUtensorMap km, vm;
  if (!make_map(&km, a.k_cache, rows, KV) || !make_map(&vm, a.v_cache, rows, KV))
    return cudaErrorInvalidValue;
  decode_tc_kernel<KV><<<grid, kNW * 32, C::kSmem, st>>>(a, km, vm);
  return cudaGetLastError();
}

}  // namespace tc

inline bool tc_supported(const pa_decode_desc* d) {
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->kv_dtype != PA_BF16 && d->kv_dtype != PA_FP8_E4M3) return false;
  if (d->q_dtype != PA_BF16 || d->out_dtype != PA_BF16) return false;
  if (d->head_dim != tc::kD || d->block_size != kBS || G > 8) return false;
  const int64_t rows = (int64_t)d->num_blocks * d->num_kv_heads * 32;
  return rows < (int64_t)1 << 31;
}

inline cudaError_t launch_tc(const DecodeArgs& a, const pa_decode_desc* d, dim3 grid,
                             cudaStream_t st) {
  if (d->kv_dtype == PA_BF16) return tc::launch_tc_kv<PA_BF16>(a, d, grid, st);
  return tc::launch_tc_kv<PA_FP8_E4M3>(a, d, grid, st);
}

}  // namespace pa
