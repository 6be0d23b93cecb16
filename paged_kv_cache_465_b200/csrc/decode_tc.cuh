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
// than the SMs can issue for G >= 4. Here one 16-token sub-tile costs a warp 16 mma.sync
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
// accumulator is rescaled when it grows, like the running softmax maximum), so the weight
// never exceeds P itself (at most 2^8 with the lazy softmax maximum of tc_block).
//
// Every wait on an mbarrier is bounded (about one second of %globaltimer); on expiry the
// warp records PA_DEVERR_TIMEOUT, stops consuming, waits (bounded) for the copies it
// issued and then finishes normally.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>

#include "decode_simt.cuh"

namespace pa {

// 0 = automatic, 1 = CUDA-core path only, 2 = tensor cores where supported (automatic
// kernel choice), 3 / 4 / 5 = tensor cores with the grid / persistent-CTA / warp-worker
// kernel where the shape allows it (see tc_kind). Atomic: calls on other host threads read
// it while pa_set_decode_impl writes it.
static std::atomic<int> g_decode_impl{0};

// Stage depth of the persistent kernel's per-warp rings (blocks in flight per warp).
#ifndef PA_TC_PSTAGE_BF16
#define PA_TC_PSTAGE_BF16 2
#endif
#ifndef PA_TC_PSTAGE_FP8
#define PA_TC_PSTAGE_FP8 3
#endif

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
// Store with an L2 eviction-priority policy (the split partials: kept in L2 for the reduce
// launch that reads them right after, while the K/V stream passes through evict-first).
__device__ __forceinline__ void st_hint(float* p, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(policy)
               : "memory");
}
__device__ __forceinline__ uint64_t evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
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
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// int8 codes -> exact f16 (code - zero). The byte is made offset-binary (u = code + 128),
// placed under an f16 exponent of 2^10 (0x64uu = 1024 + u) and (1152 + zero) subtracted:
// all values are integers below 2048, so every step is exact. `sel` picks the two bytes
// of `x_ob` (already XORed with 0x80808080); zc = f16x2(1152 + zero, 1152 + zero).
__device__ __forceinline__ uint32_t i8x2_to_f16x2(uint32_t x_ob, uint32_t sel, uint32_t zc) {
  return hsub2(__byte_perm(x_ob, 0x64646464u, sel), zc);
}
// (K, V) zero points of one block packed as two int16 -> the two subtraction constants.
__device__ __forceinline__ void zero_consts(uint32_t packed, uint32_t& kzc, uint32_t& vzc) {
  const float kz = (float)(int16_t)(packed & 0xffffu), vz = (float)(int16_t)(packed >> 16);
  kzc = pack_f16x2(1152.f + kz, 1152.f + kz);
  vzc = pack_f16x2(1152.f + vz, 1152.f + vz);
}
__device__ __forceinline__ uint32_t pack_zeros(int kz, int vz) {
  return ((uint32_t)kz & 0xffffu) | ((uint32_t)vz << 16);
}
__device__ __forceinline__ uint32_t hi16(uint32_t x) { return x >> 16; }

// Byte address of (row r, 16-byte chunk c) in a tile of 128-byte rows written by TMA with
// the 128-byte swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz(uint32_t tile, int r, int c) {
  return tile + r * 128 + ((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <pa_dtype KV>
struct TcCfg {
  static constexpr bool kFp8 = KV != PA_BF16;  // one-byte codes (fp8 or int8) -> f16 mma
  static constexpr int kTile = kFp8 ? 2048 : 4096;      // one (block, head) tile of K or V
  static constexpr int kStage = 2 * kTile;              // K + V
  static constexpr int kRows = kTile / 128;             // tensor-map rows per tile
  // CTA-per-item kernel (single pass): stages only
  static constexpr int kNStage = kFp8 ? 4 : 3;
  static constexpr int kSmem = kNW * kNStage * kStage + kNW * kNStage * 8 + 1024;
  // persistent kernel (split path): blocks in flight per warp
  static constexpr int kPStage = kFp8 ? PA_TC_PSTAGE_FP8 : PA_TC_PSTAGE_BF16;
  static constexpr int kPStageBytes = kNW * kPStage * kStage;
  static constexpr int kQBytes = 8 * kD * 2;            // one group's q (<= 8 heads, bf16)
  static constexpr int kMergeBytes = kNW * 8 * kD * 4 + 2 * kNW * 8 * 4;
  static constexpr int kPSmem = kPStageBytes + 2 * kQBytes + kMergeBytes + 256 + 1024;
};

// Per-warp running state of one work item: O^T fragments (8 tiles of 16 channels x 8
// heads), running max / sum of the two heads this thread holds, fp8 V-scale reference.
struct WarpAcc {
  float acc[8][4];
  float m0, m1, l0, l1, vref;
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
    vref = 0.f;
  }
};

// q of one group in the registers of the mma B fragments (rows g >= G zero), raw bf16
// words: bf16 path word (j, 0/1) = channels 16j + 2tq + {0,1} / 16j + 8 + 2tq + {0,1};
// fp8 path words (c, 0/1) = channels 16c + 4tq + {0,1} / {2,3}. `qp` points at the group's
// first row (global or shared memory, rows of kD).
template <bool FP8>
__device__ __forceinline__ void load_q_raw(const uint16_t* qp, int G, int lane,
                                           uint32_t (&raw)[8][2]) {
  const int gq = lane >> 2, tq = lane & 3;
  const bool live = gq < G;
  const uint16_t* r = qp + gq * kD;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if constexpr (!FP8) {
      raw[j][0] = live ? *reinterpret_cast<const uint32_t*>(r + 16 * j + 2 * tq) : 0u;
      raw[j][1] = live ? *reinterpret_cast<const uint32_t*>(r + 16 * j + 8 + 2 * tq) : 0u;
    } else {
      const uint2 w = live ? *reinterpret_cast<const uint2*>(r + 16 * j + 4 * tq) : make_uint2(0, 0);
      raw[j][0] = w.x;
      raw[j][1] = w.y;
    }
  }
}

// B fragments from the raw words; returns the log2-domain score scale. fp8: q is scaled by
// the power of two putting max|q| of the group in [2^14, 2^15) and converted to f16 (exact
// for bf16 inputs in that range); the scale is undone in the returned factor.
template <bool FP8>
__device__ __forceinline__ float q_frags(const uint32_t (&raw)[8][2], float scale_log2,
                                         uint32_t (&qf)[8][2]) {
  if constexpr (!FP8) {
#pragma unroll
    for (int j = 0; j < 8; ++j) { qf[j][0] = raw[j][0]; qf[j][1] = raw[j][1]; }
    return scale_log2;
  } else {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(raw[j][h])), fabsf(bf16_hi(raw[j][h]))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = 0;
    const uint32_t ebits = (__float_as_uint(amax) >> 23) & 0xff;
    if (ebits != 0 && ebits != 0xff) e = 15 - ((int)ebits - 126);
    e = max(-100, min(100, e));
    const float up = __uint_as_float((uint32_t)(127 + e) << 23);
    const float down = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        qf[j][h] = pack_f16x2(bf16_lo(raw[j][h]) * up, bf16_hi(raw[j][h]) * up);
    return scale_log2 * down;
  }
}

template <bool FP8>
__device__ __forceinline__ float load_q_frags(const uint16_t* qp, int G, int lane,
                                              float scale_log2, uint32_t (&qf)[8][2]) {
  uint32_t raw[8][2];
  load_q_raw<FP8>(qp, G, lane, raw);
  return q_frags<FP8>(raw, scale_log2, qf);
}

// One 16-token sub-tile: S^T = K Q^T on the tensor cores, online softmax, O^T += V^T P^T.
// kt / vt: shared addresses of the sub-tile's swizzled K and V tiles; nvalid: its tokens
// inside the work item; hp: per-half score scale (log2 domain x K scale), V scale and int8
// zero-point constants.
// The K products run as two independent accumulation chains and the V fragments are read
// before the softmax, so a warp has independent work in flight at every step.
// Per-half dequantisation parameters of a 16-token sub-tile: tokens 0-7 come from one
// block and 8-15 from another when blocks hold 8 tokens; otherwise both halves are equal.
// Growth of a score over its head's reference maximum (log2 units) that P may absorb
// before the reference is raised (P <= 2^kSlack).
constexpr float kSlack = 8.f;

struct HalfParams {
  float zs0, zs1;              // log2-domain score scale (x K scale) of each half
  float vs0, vs1;              // V scale of each half
  uint32_t kzc0, kzc1;         // int8: f16x2 (1152 + K zero point) of each half
  uint32_t vzc0, vzc1;         // int8: f16x2 (1152 + V zero point) of each half
};

template <pa_dtype KV>
__device__ __forceinline__ void tc_block(uint32_t kt, uint32_t vt, int nvalid,
                                         const HalfParams& hp, const uint32_t (&qf)[8][2],
                                         WarpAcc& w, int lane) {
  constexpr bool FP8 = KV != PA_BF16;  // one-byte codes, f16 products
  constexpr bool I8 = KV == PA_INT8;
  constexpr int TILE = FP8 ? 2048 : 4096;
  const int gq = lane >> 2;
  float pv0 = 1.f, pv1 = 1.f, beta = 1.f;
  if constexpr (FP8) {
    const float vnew = fmaxf(w.vref, fmaxf(hp.vs0, hp.vs1));
    // one approximate reciprocal rather than three divisions (P is rounded to f16 next);
    // beta stays exactly 1 while the reference does not grow
    const float rv = vnew > 0.f ? fast_rcp(vnew) : 0.f;
    beta = (w.vref > 0.f && vnew != w.vref) ? w.vref * rv : 1.f;
    pv0 = hp.vs0 * rv;
    pv1 = hp.vs1 * rv;
    w.vref = vnew;
  }
  // rows of tokens past the item may hold anything (even NaN): zero them before P.V reads
  if (nvalid < kSub) {
    const int bytes_per_tok = TILE / kSub;
    for (int o = nvalid * bytes_per_tok + lane * 16; o < TILE; o += 32 * 16)
      asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(vt + o), "r"(0) : "memory");
    __syncwarp();
  }
  const int mi = lane >> 3;
  // ---- S^T = K Q^T : 16 tokens x 8 heads, two independent chains ----
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const int tok = (lane & 7) + 8 * (mi & 1);
    if constexpr (!FP8) {
      // rows of the tile: 2*token + (channel >= 64); chunk = (channel % 64) / 8
      uint32_t r[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int d0 = 16 * j + 8 * (mi >> 1);
        ldsm_x4(swz(kt, 2 * tok + (d0 >> 6), (d0 & 63) >> 3), r[j]);
      }
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        mma16816<false>(sa, r[j], qf[j][0], qf[j][1]);
        mma16816<false>(sb, r[j + 1], qf[j + 1][0], qf[j + 1][1]);
      }
    } else {
      uint32_t r[4][4];
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) ldsm_x4(swz(kt, tok, 2 * cp + (mi >> 1)), r[cp]);
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) {
        // a register holds 4 consecutive channels of one token: pairs (0,1) and (2,3)
        uint32_t x0[4], x1[4];
        if constexpr (I8) {
          // registers 0 and 2 hold tokens 0-7, registers 1 and 3 tokens 8-15
          uint32_t u[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) u[e] = r[cp][e] ^ 0x80808080u;
          x0[0] = i8x2_to_f16x2(u[0], 0x4140, hp.kzc0); x0[1] = i8x2_to_f16x2(u[1], 0x4140, hp.kzc1);
          x0[2] = i8x2_to_f16x2(u[0], 0x4342, hp.kzc0); x0[3] = i8x2_to_f16x2(u[1], 0x4342, hp.kzc1);
          x1[0] = i8x2_to_f16x2(u[2], 0x4140, hp.kzc0); x1[1] = i8x2_to_f16x2(u[3], 0x4140, hp.kzc1);
          x1[2] = i8x2_to_f16x2(u[2], 0x4342, hp.kzc0); x1[3] = i8x2_to_f16x2(u[3], 0x4342, hp.kzc1);
        } else {
          x0[0] = e4m3x2_to_f16x2((uint16_t)lo16(r[cp][0])); x0[1] = e4m3x2_to_f16x2((uint16_t)lo16(r[cp][1]));
          x0[2] = e4m3x2_to_f16x2((uint16_t)hi16(r[cp][0])); x0[3] = e4m3x2_to_f16x2((uint16_t)hi16(r[cp][1]));
          x1[0] = e4m3x2_to_f16x2((uint16_t)lo16(r[cp][2])); x1[1] = e4m3x2_to_f16x2((uint16_t)lo16(r[cp][3]));
          x1[2] = e4m3x2_to_f16x2((uint16_t)hi16(r[cp][2])); x1[3] = e4m3x2_to_f16x2((uint16_t)hi16(r[cp][3]));
        }
        mma16816<true>(sa, x0, qf[2 * cp][0], qf[2 * cp][1]);
        mma16816<true>(sb, x1, qf[2 * cp + 1][0], qf[2 * cp + 1][1]);
      }
    }
  }
  // ---- V fragments (independent of the softmax) ----
  uint32_t vr[8][4];
  {
    const int tok = (lane & 7) + 8 * (mi >> 1);
    if constexpr (!FP8) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int d0 = 16 * t + 8 * (mi & 1);
        ldsm_x4_t(swz(vt, 2 * tok + (d0 >> 6), (d0 & 63) >> 3), vr[t]);
      }
    } else {
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) ldsm_x4_t(swz(vt, tok, 2 * cp + (mi & 1)), vr[cp]);
    }
  }
  // ---- online softmax (log2 domain); thread holds tokens gq, gq+8 x heads 2tq, 2tq+1 ----
  const bool va = gq < nvalid, vb = gq + 8 < nvalid;
  const float z0 = va ? (sa[0] + sb[0]) * hp.zs0 : -INFINITY;
  const float z1 = va ? (sa[1] + sb[1]) * hp.zs0 : -INFINITY;
  const float z2 = vb ? (sa[2] + sb[2]) * hp.zs1 : -INFINITY;
  const float z3 = vb ? (sa[3] + sb[3]) * hp.zs1 : -INFINITY;
  // The reference m of a head is raised (to the running maximum, found across the 8 lanes
  // of the head) only when a score exceeds it by more than kSlack; otherwise P is taken
  // against the stale m and may reach 2^kSlack (f16 holds it exactly as well as a value
  // below 1), so most sub-tiles skip the cross-lane maximum and the rescale. The outcome
  // depends only on the scores, never on where the blocks sit.
  float bm0 = fmaxf(z0, z2), bm1 = fmaxf(z1, z3);
  float al0 = 1.f, al1 = 1.f;
  if (__any_sync(0xffffffffu, bm0 > w.m0 + kSlack || bm1 > w.m1 + kSlack)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, o));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, o));
    }
    const float mn0 = fmaxf(w.m0, bm0), mn1 = fmaxf(w.m1, bm1);
    al0 = fast_exp2(w.m0 - mn0);
    al1 = fast_exp2(w.m1 - mn1);
    w.m0 = mn0;
    w.m1 = mn1;
  }
  const float p0 = fast_exp2(z0 - w.m0), p1 = fast_exp2(z1 - w.m1);
  const float p2 = fast_exp2(z2 - w.m0), p3 = fast_exp2(z3 - w.m1);
  w.l0 = w.l0 * al0 + (p0 + p2);
  w.l1 = w.l1 * al1 + (p1 + p3);
  if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f || beta != 1.f)) {
    const float f0 = al0 * beta, f1 = al1 * beta;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      w.acc[t][0] *= f0; w.acc[t][1] *= f1; w.acc[t][2] *= f0; w.acc[t][3] *= f1;
    }
  }
  // P^T as B fragments: pack [token][head] pairs, transpose 8x8 in registers
  uint32_t pb0, pb1;
  if constexpr (FP8) {
    pb0 = movm_t(pack_f16x2(p0 * pv0, p1 * pv0));
    pb1 = movm_t(pack_f16x2(p2 * pv1, p3 * pv1));
  } else {
    pb0 = movm_t(pack_bf16x2(p0, p1));
    pb1 = movm_t(pack_bf16x2(p2, p3));
  }
  // ---- O^T += V^T P^T ----
  if constexpr (!FP8) {
#pragma unroll
    for (int t = 0; t < 8; ++t) mma16816<false>(w.acc[t], vr[t], pb0, pb1);
  } else {
#pragma unroll
    for (int cp = 0; cp < 4; ++cp) {
      // a register holds channels (2j, 2j+1) of tokens t0 (low half) and t1 (high half):
      // pairs (t0, t1) at channel 2j are bytes (0, 2), at channel 2j+1 bytes (1, 3)
      uint32_t ev[4], od[4];
      if constexpr (I8) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // registers 0, 1: tokens 0-7; 2, 3: tokens 8-15
          const uint32_t u = vr[cp][e] ^ 0x80808080u;
          ev[e] = i8x2_to_f16x2(u, 0x4240, e < 2 ? hp.vzc0 : hp.vzc1);
          od[e] = i8x2_to_f16x2(u, 0x4341, e < 2 ? hp.vzc0 : hp.vzc1);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t y = __byte_perm(vr[cp][e], 0, 0x3120);
          ev[e] = e4m3x2_to_f16x2((uint16_t)lo16(y));
          od[e] = e4m3x2_to_f16x2((uint16_t)hi16(y));
        }
      }
      mma16816<true>(w.acc[2 * cp], ev, pb0, pb1);
      mma16816<true>(w.acc[2 * cp + 1], od, pb0, pb1);
    }
  }
}

// Writes a warp's finished state into the merge area: m/l per head and the unnormalised
// output [8][kD] (true units: fp8 accumulators are scaled back by vref).
template <bool FP8>
__device__ __forceinline__ void stash_warp(WarpAcc& w, float* sacc, float* smx, float* slx,
                                           int warp, int lane) {
  const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, o);
    w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, o);
  }
  if (gq == 0) {
    smx[warp * 8 + 2 * tq] = w.m0; smx[warp * 8 + 2 * tq + 1] = w.m1;
    slx[warp * 8 + 2 * tq] = w.l0; slx[warp * 8 + 2 * tq + 1] = w.l1;
  }
  const float unit = FP8 ? w.vref : 1.f;
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
    wacc[(2 * tq) * kD + dA] = w.acc[t][0] * unit;
    wacc[(2 * tq + 1) * kD + dA] = w.acc[t][1] * unit;
    wacc[(2 * tq) * kD + dB] = w.acc[t][2] * unit;
    wacc[(2 * tq + 1) * kD + dB] = w.acc[t][3] * unit;
  }
}

// Combines the kNW warps' states of head g, channel d (after stash_warp + __syncthreads).
__device__ __forceinline__ void combine_warps(const float* sacc, const float* smx,
                                              const float* slx, int g, int d, float& M, float& L,
                                              float& A) {
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kNW; ++w) M = fmaxf(M, smx[w * 8 + g]);
  L = 0.f;
  A = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kNW; ++w) {
      const float f = fast_exp2(smx[w * 8 + g] - M);
      L = fmaf(f, slx[w * 8 + g], L);
      A = fmaf(f, sacc[(w * 8 + g) * kD + d], A);
    }
  }
}

// =======================================================================================
// Block-table view of 16-token sub-tiles (any block size: 8, 16 or 32 tokens)
// =======================================================================================
// Sub-tile c covers logical tokens [16c, 16c + 16). Blocks of 16 or 32 tokens hold one or
// two whole sub-tiles (contiguous in the (block, kv head) region); with 8-token blocks a
// sub-tile has two halves from two blocks, each with its own scales.
struct SubWin {
  int p0, p1;          // physical blocks of the halves; p1 = -3: second half absent
  float ks0, vs0, ks1, vs1;
  uint32_t z0, z1;     // int8: packed (K, V) zero points
};

// Block ids, scales and zero points are read through L2 (ld.global.cg): each is read once
// per item, and a warp worker reads its first item's before the plan kernel has finished.
template <pa_dtype KV, int BS>
__device__ __forceinline__ void load_sub(const DecodeArgs& a, const int32_t* btrow, int c,
                                         int t1, int kvh, SubWin& w) {
  auto one = [&](int blk, int& p, float& ks, float& vs, uint32_t& z) {
    p = __ldcg(btrow + blk);
    ks = 1.f;
    vs = 1.f;
    z = 0;
    if (p < 0 || p >= a.num_blocks) {
      flag_error(PA_DEVERR_BLOCK_ID);
      p = -1;
      return;
    }
    if constexpr (KV != PA_BF16) {
      const int64_t bh = (int64_t)p * a.num_kv_heads + kvh;
      ks = __ldcg(a.k_scales + bh);
      vs = __ldcg(a.v_scales + bh);
      if constexpr (KV == PA_INT8) {
        const int kz = __ldcg(a.k_zeros + bh), vz = __ldcg(a.v_zeros + bh);
        if (!zero_in_range(kz) || !zero_in_range(vz)) {
          flag_error(PA_DEVERR_ZERO);
          p = -1;
          return;
        }
        z = pack_zeros(kz, vz);
      }
    }
  };
  if constexpr (BS == 8) {
    one(2 * c, w.p0, w.ks0, w.vs0, w.z0);
    if (c * kSub + 8 < t1) {
      one(2 * c + 1, w.p1, w.ks1, w.vs1, w.z1);
    } else {
      w.p1 = -3; w.ks1 = w.ks0; w.vs1 = w.vs0; w.z1 = w.z0;
    }
  } else {
    one(c * kSub / BS, w.p0, w.ks0, w.vs0, w.z0);
    w.p1 = w.p0; w.ks1 = w.ks0; w.vs1 = w.vs0; w.z1 = w.z0;
  }
}

__device__ __forceinline__ void empty_sub(SubWin& w) {
  w.p0 = -2; w.p1 = -3; w.ks0 = w.vs0 = w.ks1 = w.vs1 = 1.f; w.z0 = w.z1 = 0;
}

// Lane k's window entry, broadcast to the warp.
template <int BS>
__device__ __forceinline__ SubWin shfl_sub(const SubWin& w, int k) {
  SubWin r;
  r.p0 = __shfl_sync(0xffffffffu, w.p0, k);
  r.ks0 = __shfl_sync(0xffffffffu, w.ks0, k);
  r.vs0 = __shfl_sync(0xffffffffu, w.vs0, k);
  r.z0 = __shfl_sync(0xffffffffu, w.z0, k);
  if constexpr (BS == 8) {
    r.p1 = __shfl_sync(0xffffffffu, w.p1, k);
    r.ks1 = __shfl_sync(0xffffffffu, w.ks1, k);
    r.vs1 = __shfl_sync(0xffffffffu, w.vs1, k);
    r.z1 = __shfl_sync(0xffffffffu, w.z1, k);
  } else {
    r.p1 = r.p0; r.ks1 = r.ks0; r.vs1 = r.vs0; r.z1 = r.z0;
  }
  return r;
}

__device__ __forceinline__ SubWin select_sub(bool first, const SubWin& a, const SubWin& b) {
  SubWin r;
  r.p0 = first ? a.p0 : b.p0;
  r.p1 = first ? a.p1 : b.p1;
  r.ks0 = first ? a.ks0 : b.ks0;
  r.vs0 = first ? a.vs0 : b.vs0;
  r.ks1 = first ? a.ks1 : b.ks1;
  r.vs1 = first ? a.vs1 : b.vs1;
  r.z0 = first ? a.z0 : b.z0;
  r.z1 = first ? a.z1 : b.z1;
  return r;
}

// A sub-tile the consumer can use: its blocks exist and are in range.
__device__ __forceinline__ bool sub_ok(const SubWin& w) { return w.p0 >= 0 && w.p1 != -1; }

// Lane 0: TMA copies of sub-tile c's K and V tiles into the stage at dst (V at dst + TILE),
// completing on bar; a plain arrive when the sub-tile is skipped.
template <pa_dtype KV, int BS>
__device__ __forceinline__ void issue_sub(uint32_t dst, const CUtensorMap* kmap,
                                          const CUtensorMap* vmap, uint32_t bar,
                                          uint64_t policy, const SubWin& w, int c, int kvh,
                                          int Hkv) {
  constexpr int TILE = TcCfg<KV>::kTile, R16 = TcCfg<KV>::kRows;
  // the stage was last read (and maybe written) through the generic proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (!sub_ok(w)) {
    mbar_arrive(bar);  // completes the phase; the consumer skips the sub-tile
    return;
  }
  if constexpr (BS == 8) {
    constexpr int HALF = TILE / 2, R8 = R16 / 2;
    const bool two = w.p1 >= 0;
    mbar_arrive_tx(bar, (two ? 4u : 2u) * HALF);
    const int r0 = (w.p0 * Hkv + kvh) * R8;
    tma_load_2d(dst, kmap, 0, r0, bar, policy);
    tma_load_2d(dst + TILE, vmap, 0, r0, bar, policy);
    if (two) {
      const int r1 = (w.p1 * Hkv + kvh) * R8;
      tma_load_2d(dst + HALF, kmap, 0, r1, bar, policy);
      tma_load_2d(dst + TILE + HALF, vmap, 0, r1, bar, policy);
    }
  } else {
    constexpr int PER = BS / kSub;  // sub-tiles per block
    const int row = ((w.p0 * Hkv + kvh) * PER + c % PER) * R16;
    mbar_arrive_tx(bar, 2 * TILE);
    tma_load_2d(dst, kmap, 0, row, bar, policy);
    tma_load_2d(dst + TILE, vmap, 0, row, bar, policy);
  }
}

template <pa_dtype KV>
__device__ __forceinline__ HalfParams half_params(const SubWin& w, float zscale) {
  HalfParams h;
  h.zs0 = zscale * w.ks0;
  h.zs1 = zscale * w.ks1;
  h.vs0 = w.vs0;
  h.vs1 = w.vs1;
  h.kzc0 = h.kzc1 = h.vzc0 = h.vzc1 = 0;
  if constexpr (KV == PA_INT8) {
    zero_consts(w.z0, h.kzc0, h.vzc0);
    zero_consts(w.z1, h.kzc1, h.vzc1);
  }
  return h;
}

// =======================================================================================
// One CTA per work item, grid (partitions, Hkv, S): warp w takes the item's sub-tiles
// w, w+4, ... through its own TMA ring; warps merge through shared memory at the end.
// =======================================================================================
template <pa_dtype KV, int BS>
__global__ void __launch_bounds__(kNW * 32)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap) {
  using C = TcCfg<KV>;
  constexpr bool FP8 = C::kFp8;
  constexpr int TILE = C::kTile, STAGE = C::kStage, NST = C::kNStage;
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

  const uint32_t wtiles = smem_u32(smem + warp * NST * STAGE);
  const uint32_t bars = smem_u32(smem + kNW * NST * STAGE) + warp * NST * 8;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) mbar_init(bars + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncwarp();

  uint32_t qf[8][2];
  const float zscale = load_q_frags<FP8>(
      static_cast<const uint16_t*>(a.q) + ((int64_t)s * a.num_q_heads + kvh * G) * kD, G, lane,
      a.scale_log2, qf);

  // ---- this warp's sub-tiles and their block-table windows (32 per register set) ----
  const int c_begin = t0 / kSub, c_end = (t1 + kSub - 1) / kSub;
  const int nsub = c_end - c_begin;
  const int nmine = nsub > warp ? (nsub - warp + kNW - 1) / kNW : 0;
  const int32_t* bt = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
  auto sub_of = [&](int k) { return c_begin + warp + k * kNW; };
  auto load_window = [&](int base, SubWin& w) {
    const int k = base + lane;
    if (k < nmine) load_sub<KV, BS>(a, bt, sub_of(k), t1, kvh, w);
    else empty_sub(w);
  };
  SubWin cur, nxt;
  load_window(0, cur);
  load_window(32, nxt);
  const uint64_t policy = evict_first_policy();
  auto issue = [&](int k, int wbase, int stage) {
    const int rel = k - wbase;
    const SubWin w = rel < 32 ? shfl_sub<BS>(cur, rel) : shfl_sub<BS>(nxt, rel - 32);
    if (lane == 0)
      issue_sub<KV, BS>(wtiles + stage * STAGE, &kmap, &vmap, bars + 8 * stage, policy, w,
                        sub_of(k), kvh, a.num_kv_heads);
  };
  for (int k = 0; k < NST && k < nmine; ++k) issue(k, 0, k);

  WarpAcc w;
  w.reset();
  bool timed_out = false;
  int consumed = 0;
  for (int i = 0; i < nmine; ++i) {
    const int wbase = i & ~31;
    if ((i & 31) == 0 && i > 0) {
      cur = nxt;
      load_window(i + 32, nxt);
    }
    const int stage = i % NST;
    const SubWin sw = shfl_sub<BS>(cur, i & 31);
    if (!mbar_wait(bars + 8 * stage, (uint32_t)((i / NST) & 1))) {
      if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
      timed_out = true;
      break;
    }
    consumed = i + 1;
    if (sub_ok(sw)) {
      const int c = sub_of(i);
      const uint32_t kt = wtiles + stage * STAGE;
      tc_block<KV>(kt, kt + TILE, min(kSub, t1 - c * kSub), half_params<KV>(sw, zscale), qf, w,
                   lane);
    }
    __syncwarp();
    if (i + NST < nmine) issue(i + NST, wbase, stage);
  }
  if (timed_out) {
    // wait (bounded) for every copy this warp issued and did not consume
    const int issued = min(nmine, consumed + NST);
    for (int k = consumed; k < issued; ++k)
      if (!mbar_wait(bars + 8 * (k % NST), (uint32_t)((k / NST) & 1))) break;
  }

  // ---- merge the warps through shared memory (stage buffers are free now) ----
  __syncthreads();
  float* sacc = reinterpret_cast<float*>(smem);  // [kNW][8][kD]
  float* smx = sacc + kNW * 8 * kD;               // [kNW][8]
  float* slx = smx + kNW * 8;                     // [kNW][8]
  stash_warp<FP8>(w, sacc, smx, slx, warp, lane);
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
    const int g = idx / kD, d = idx % kD;
    float M, L, A;
    combine_warps(sacc, smx, slx, g, d, M, L, A);
    emit(a, s, kvh * G + g, part, kD, d, M, L, A);
  }
}

// =======================================================================================
// Split path: plan kernel + persistent kernels; lse_reduce_kernel merges the partitions.
// =======================================================================================
// Workspace of the split path (offsets in bytes, each region 256-aligned):
//   [0]     uint32 fetch counter, uint32 total items
//   list    int4 (seq, partition, context length, 0) per partition item, largest first
//           (the context length rides along so that a worker's fetch needs one read less)
//   m, l    float [S][Hq][P];  acc float [S][Hq][P][kD]   (partials, as the CUDA-core path)
// Sequences with a single partition are written to `out` directly; the others are merged
// by lse_reduce_kernel afterwards (spread over every (seq, q head)).
struct PlanView {
  uint32_t* counters;  // [0] fetch, [1] total
  int4* list;
};

// One CTA of 1024 threads: counts partitions per size (sub-tiles per item), orders them
// largest first (full partitions, then partial ones by size; a counting sort), writes the
// list, zeroes the fetch counter, and writes out = 0 / lse = -inf for empty sequences.
// Largest first keeps the launch's tail short: the last items taken are the smallest.
// The order affects scheduling only: every item's result depends on logical positions.
__global__ void __launch_bounds__(1024) plan_kernel(const DecodeArgs a, const PlanView pl) {
  __shared__ int cnt[130], off[130];
  pdl_wait();
  pdl_trigger();
  const int P = a.part_tokens;
  const int nbk = P / kSub;  // sub-tiles of a full partition (<= 128)
  for (int i = threadIdx.x; i < 130; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int ctx = checked_ctx(a, s);
    if (ctx == 0) {
      for (int h = 0; h < a.num_q_heads; ++h) {
        const int64_t row = (int64_t)s * a.num_q_heads + h;
        for (int d = 0; d < kD; ++d) store_out(a.out, a.out_dtype, row * kD + d, 0.f);
        if (a.lse_out != nullptr) a.lse_out[row] = -INFINITY;
      }
      continue;
    }
    // partition 0 of the first static_seqs sequences is a warp's first item already
    const int skip = s < a.static_seqs ? 1 : 0;
    const int full = ctx / P, rem = ctx % P;
    if (full > skip) atomicAdd(&cnt[nbk], full - skip);
    if (rem && (full > 0 || !skip)) atomicAdd(&cnt[(rem + kSub - 1) / kSub], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int b = nbk; b >= 1; --b) {
      off[b] = acc;
      acc += cnt[b];
    }
    pl.counters[0] = 0;
    pl.counters[1] = (uint32_t)acc * (uint32_t)a.num_kv_heads;
  }
  __syncthreads();
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int ctx = checked_ctx(a, s);
    const int skip = s < a.static_seqs ? 1 : 0;
    const int full = ctx / P, rem = ctx % P;
    if (full > skip) {
      const int base = atomicAdd(&off[nbk], full - skip);
      for (int j = skip; j < full; ++j) pl.list[base + j - skip] = make_int4(s, j, ctx, 0);
    }
    if (rem && (full > 0 || !skip))
      pl.list[atomicAdd(&off[(rem + kSub - 1) / kSub], 1)] = make_int4(s, full, ctx, 0);
  }
}

// Work item slot shared by the CTA (written by thread 0 between barriers).
struct ItemSlot {
  int valid, s, part, kvh, ctx;
};

// Persistent CTAs: 16-token blocks only (a block is one sub-tile).
template <pa_dtype KV>
__global__ void __launch_bounds__(kNW * 32)
decode_tc_persistent(const DecodeArgs a, const PlanView pl,
                     const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap) {
  using C = TcCfg<KV>;
  constexpr bool FP8 = C::kFp8;
  constexpr int TILE = C::kTile, STAGE = C::kStage, NST = C::kPStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qbuf = smem + C::kPStageBytes;                        // [2][8][kD] bf16
  float* sacc = reinterpret_cast<float*>(qbuf + 2 * C::kQBytes);  // [kNW][8][kD]
  float* smx = sacc + kNW * 8 * kD;
  float* slx = smx + kNW * 8;
  uint64_t* barmem = reinterpret_cast<uint64_t*>(slx + kNW * 8);  // [kNW*NST] + [2] q
  ItemSlot* slots = reinterpret_cast<ItemSlot*>(barmem + kNW * NST + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.group, Hkv = a.num_kv_heads, P = a.part_tokens;
  const uint32_t wtiles = smem_u32(smem + warp * NST * STAGE);
  const uint32_t bars = smem_u32(barmem) + warp * NST * 8;
  const uint32_t qbars = smem_u32(barmem + kNW * NST);
  pdl_wait();  // the plan kernel's list and counters
  const uint32_t total = pl.counters[1];
  const uint64_t policy = evict_first_policy();

  // thread 0: take the next item from the shared counter into slot `sl`, start its q copy
  auto fetch = [&](int sl) {
    const uint32_t it = atomicAdd(&pl.counters[0], 1u);
    ItemSlot x{0, 0, 0, 0, 0};
    if (it < total) {
      const int4 sp = pl.list[it / Hkv];
      x = ItemSlot{1, sp.x, sp.y, (int)(it % Hkv), sp.z};
      const uint32_t qb = qbars + 8 * sl;
      mbar_arrive_tx(qb, (uint32_t)(G * kD * 2));
      bulk_load_1d(smem_u32(qbuf + sl * C::kQBytes),
                   static_cast<const uint16_t*>(a.q) + ((int64_t)x.s * a.num_q_heads + x.kvh * G) * kD,
                   (uint32_t)(G * kD * 2), qb);
    }
    slots[sl] = x;
  };

  if (tid == 0) {
    for (int i = 0; i < kNW * NST + 2; ++i) mbar_init(smem_u32(barmem + i), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    fetch(0);
    fetch(1);
  }
  __syncthreads();

  // Per-warp view of an item: its blocks are b_begin + warp + k*kNW, k < nmine (<= 32).
  struct WarpItem {
    int valid, s, kvh, part, t1, b_begin, nmine, np;
  };
  auto item_view = [&](int sl) {
    const ItemSlot x = slots[sl];
    WarpItem v{x.valid, x.s, x.kvh, x.part, 0, 0, 0, 0};
    if (x.valid) {
      const int ctx = x.ctx;  // checked by the plan kernel
      const int t0 = x.part * P;
      v.t1 = min(ctx, t0 + P);
      v.b_begin = t0 / kSub;
      const int nblk = (v.t1 + kSub - 1) / kSub - v.b_begin;
      v.nmine = nblk > warp ? (nblk - warp + kNW - 1) / kNW : 0;
      v.np = (ctx + P - 1) / P;
    }
    return v;
  };
  // block-table window of an item for this warp: lane k holds block k's (phys, ks, vs, z)
  auto load_window = [&](const WarpItem& v, int& p, float& ks, float& vs, uint32_t& z) {
    p = -2;
    ks = 1.f;
    vs = 1.f;
    z = 0;
    if (v.valid && lane < v.nmine) {
      p = a.block_tables[(int64_t)v.s * a.max_blocks_per_seq + v.b_begin + warp + lane * kNW];
      if (p < 0 || p >= a.num_blocks) {
        flag_error(PA_DEVERR_BLOCK_ID);
        p = -1;
      } else if constexpr (FP8) {
        ks = a.k_scales[(int64_t)p * Hkv + v.kvh];
        vs = a.v_scales[(int64_t)p * Hkv + v.kvh];
        if constexpr (KV == PA_INT8) {
          const int kz = a.k_zeros[(int64_t)p * Hkv + v.kvh];
          const int vz = a.v_zeros[(int64_t)p * Hkv + v.kvh];
          if (!zero_in_range(kz) || !zero_in_range(vz)) {
            flag_error(PA_DEVERR_ZERO);
            p = -1;
          }
          z = pack_zeros(kz, vz);
        }
      }
    }
  };

  int k = 0;  // CTA-local item counter: item k lives in slot k & 1
  WarpItem cur = item_view(0), nxt = item_view(1);
  int cur_p, nxt_p;
  float cur_ks, cur_vs, nxt_ks, nxt_vs;
  uint32_t cur_z, nxt_z;
  load_window(cur, cur_p, cur_ks, cur_vs, cur_z);
  load_window(nxt, nxt_p, nxt_ks, nxt_vs, nxt_z);

  // producer position in this warp's block stream: (pslot 0 = cur / 1 = nxt, pk)
  int pslot = 0, pk = 0;
  uint32_t g_iss = 0, g_cons = 0;
  bool dead = false;
  auto produce = [&]() {
    while (!dead && g_iss - g_cons < (uint32_t)NST) {
      if (pslot == 0 && pk >= cur.nmine) { pslot = 1; pk = 0; }
      if (pslot == 1 && (!nxt.valid || pk >= nxt.nmine)) break;
      const WarpItem& v = pslot == 0 ? cur : nxt;
      const int p = __shfl_sync(0xffffffffu, pslot == 0 ? cur_p : nxt_p, pk);
      const int stage = g_iss % NST;
      if (lane == 0) {
        const uint32_t bar = bars + 8 * stage;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (p >= 0) {
          const int row = (p * Hkv + v.kvh) * C::kRows;
          const uint32_t dst = wtiles + stage * STAGE;
          mbar_arrive_tx(bar, STAGE);
          tma_load_2d(dst, &kmap, 0, row, bar, policy);
          tma_load_2d(dst + TILE, &vmap, 0, row, bar, policy);
        } else {
          mbar_arrive(bar);
        }
      }
      ++g_iss;
      ++pk;
    }
  };
  produce();

  uint32_t qf[8][2];
  WarpAcc w;
  while (cur.valid) {
    // q of the item (bulk copy completes on its slot's barrier)
    const int sl = k & 1;
    if (!dead && !mbar_wait(qbars + 8 * sl, (uint32_t)((k >> 1) & 1))) {
      if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
      dead = true;
    }
    const float zscale = load_q_frags<FP8>(reinterpret_cast<const uint16_t*>(qbuf + sl * C::kQBytes),
                                           G, lane, a.scale_log2, qf);
    w.reset();
    for (int i = 0; i < cur.nmine; ++i) {
      const int p = __shfl_sync(0xffffffffu, cur_p, i);
      const float ks = __shfl_sync(0xffffffffu, cur_ks, i);
      const float vs = __shfl_sync(0xffffffffu, cur_vs, i);
      uint32_t kzc = 0, vzc = 0;
      if constexpr (KV == PA_INT8) zero_consts(__shfl_sync(0xffffffffu, cur_z, i), kzc, vzc);
      const int stage = g_cons % NST;
      if (!dead && !mbar_wait(bars + 8 * stage, (g_cons / NST) & 1)) {
        if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
        dead = true;
      }
      if (!dead && p >= 0) {
        const int b = cur.b_begin + warp + i * kNW;
        const uint32_t kt = wtiles + stage * STAGE;
        const HalfParams hp{zscale * ks, zscale * ks, vs, vs, kzc, kzc, vzc, vzc};
        tc_block<KV>(kt, kt + TILE, min(kSub, cur.t1 - b * kSub), hp, qf, w, lane);
      }
      __syncwarp();
      ++g_cons;
      produce();
    }
    // ---- item finished by this warp: merge the warps ----
    stash_warp<FP8>(w, sacc, smx, slx, warp, lane);
    __syncthreads();  // [A] merge area complete; slot k&1 and its q buffer are free
    if (tid == 0) fetch(sl);  // item k+2 into the slot item k used
    const int s = cur.s, kvh = cur.kvh, part = cur.part, np = cur.np;
    for (int idx = tid; idx < G * kD; idx += blockDim.x) {
      const int g = idx / kD, d = idx % kD;
      float M, L, A;
      combine_warps(sacc, smx, slx, g, d, M, L, A);
      const int64_t row = (int64_t)s * a.num_q_heads + kvh * G + g;
      if (np == 1) {
        store_out(a.out, a.out_dtype, row * kD + d, L > 0.f ? A / L : 0.f);
        if (d == 0 && a.lse_out != nullptr)
          a.lse_out[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
      } else {
        const int64_t pr = row * a.max_parts + part;
        a.part_acc[pr * kD + d] = A;
        if (d == 0) { a.part_m[pr] = M; a.part_l[pr] = L; }
      }
    }
    __syncthreads();  // [A2] merge area read by every thread; slot k&1 holds item k+2
    // ---- advance: item k+1 becomes current, item k+2 (just fetched) the next ----
    ++k;
    cur = nxt;
    cur_p = nxt_p; cur_ks = nxt_ks; cur_vs = nxt_vs; cur_z = nxt_z;
    nxt = item_view((k + 1) & 1);
    load_window(nxt, nxt_p, nxt_ks, nxt_vs, nxt_z);
    pslot = 0;  // the producer finished item k, so it was positioned in item k+1
    produce();
  }
  if (dead) {
    // wait (bounded) for the copies this warp issued and did not consume
    for (uint32_t j = g_cons; j < g_iss; ++j)
      if (!mbar_wait(bars + 8 * (j % NST), (j / NST) & 1)) break;
  }
}

// =======================================================================================
// Split path, warp workers: every warp of the grid is an independent worker that takes
// (sequence, partition, kv head) items from the shared counter and streams all blocks of
// the item through its own TMA ring; no shared merge area and no CTA barrier after set-up.
// q of the next item and its block-table window are fetched while the current one runs.
// Partitions of at most 512 tokens (32 blocks: one register window per item).
// =======================================================================================
#ifndef PA_TCW_WARPS
#define PA_TCW_WARPS 1
#endif
#ifndef PA_TCW_STAGE_BF16
#define PA_TCW_STAGE_BF16 3
#endif
#ifndef PA_TCW_STAGE_FP8
#define PA_TCW_STAGE_FP8 3
#endif
constexpr int kWW = PA_TCW_WARPS;

#ifndef PA_TCW_MIN_WARPS
#define PA_TCW_MIN_WARPS 16  // resident warps per SM the register budget is sized for
#endif

// Shared memory of one CTA of kWW warp workers: their TMA rings (1024-byte aligned, the
// 128-byte swizzle's period), then one q buffer per warp sized for the call's group (G
// heads of kD bf16), then each warp's barriers, plus alignment slack. Sizing the q buffers
// by G lets more workers, hence more bytes in flight, fit in an SM's shared memory (fp8
// with four query heads per kv head: 15 warps per SM instead of 14). (Two workers per CTA
// sharing the slack would fit 16, but made ptxas spill.)
template <pa_dtype KV>
struct TcwCfg {
  static constexpr int kNStage = KV == PA_FP8_E4M3 ? PA_TCW_STAGE_FP8 : PA_TCW_STAGE_BF16;
  __host__ __device__ static constexpr int qbytes(int G) { return G * kD * 2; }
  __host__ __device__ static constexpr int smem(int G) {
    return kWW * kNStage * TcCfg<KV>::kStage + kWW * qbytes(G) + kWW * (kNStage + 1) * 8 + 1024;
  }
  static constexpr int kMaxSmem = smem(8);
};


template <pa_dtype KV, int BS>
__global__ void __launch_bounds__(kWW * 32, PA_TCW_MIN_WARPS / kWW)
decode_tc_warps(const DecodeArgs a, const PlanView pl, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap) {
  using C = TcCfg<KV>;
  constexpr bool FP8 = C::kFp8;
  constexpr int TILE = C::kTile, STAGE = C::kStage, NST = TcwCfg<KV>::kNStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int G = a.group, Hkv = a.num_kv_heads, P = a.part_tokens;
  const uint32_t wtiles = smem_u32(smem + warp * NST * STAGE);
  const int qbytes = TcwCfg<KV>::qbytes(a.group);
  uint8_t* qbuf = smem + kWW * NST * STAGE + warp * qbytes;
  const uint32_t bars = smem_u32(smem + kWW * NST * STAGE + kWW * qbytes) +
                        warp * (NST + 1) * 8;
  const uint32_t qbar = bars + NST * 8;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i <= NST; ++i) mbar_init(bars + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncwarp();
  uint32_t total = 0;  // items in the plan's list, read once the plan has finished
  const uint64_t policy = evict_first_policy();

  // an item's sub-tiles are c_begin + k, k < nsub (<= 32)
  struct Item {
    int valid, s, kvh, part, t1, c_begin, nsub, np;
  };
  // This warp's first item: partition 0 of (sequence gw / Hkv, kv head gw % Hkv) for
  // gw < static_seqs * Hkv. It needs no plan, so it is read and starts streaming before the
  // plan kernel has finished; its inputs were written before the plan kernel started (that
  // kernel waits for its predecessors before it lets this one launch), and they are read
  // through L2.
  auto static_item = [&]() {
    Item v{0, 0, 0, 0, 0, 0, 0, 0};
    const int gw = blockIdx.x * kWW + warp;
    if (gw < a.static_seqs * Hkv) {
      const int s = gw / Hkv;
      int ctx = __ldcg(a.context_lens + s);  // clamped and flagged as checked_ctx does
      if (ctx < 0 || ctx > a.max_context_len) {
        if (lane == 0) flag_error(PA_DEVERR_CONTEXT);
        ctx = ctx < 0 ? 0 : a.max_context_len;
      }
      if (ctx > 0) {
        v.valid = 1;
        v.s = s;
        v.kvh = gw % Hkv;
        v.t1 = min(ctx, P);
        v.nsub = (v.t1 + kSub - 1) / kSub;
        v.np = (ctx + P - 1) / P;
      }
    }
    return v;
  };
  auto fetch = [&]() {
    uint32_t it = 0;
    if (lane == 0) it = atomicAdd(&pl.counters[0], 1u);
    it = __shfl_sync(0xffffffffu, it, 0);
    Item v{0, 0, 0, 0, 0, 0, 0, 0};
    if (it < total) {
      const int4 sp = pl.list[it / Hkv];
      const int ctx = sp.z;  // checked by the plan kernel
      const int t0 = sp.y * P;
      v.valid = 1;
      v.s = sp.x;
      v.kvh = (int)(it % Hkv);
      v.part = sp.y;
      v.t1 = min(ctx, t0 + P);
      v.c_begin = t0 / kSub;
      v.nsub = (v.t1 + kSub - 1) / kSub - v.c_begin;
      v.np = (ctx + P - 1) / P;
    }
    return v;
  };
  // lane k holds sub-tile k's blocks, scales and zero points of an item
  auto load_window = [&](const Item& v, SubWin& w) {
    if (v.valid && lane < v.nsub)
      load_sub<KV, BS>(a, a.block_tables + (int64_t)v.s * a.max_blocks_per_seq, v.c_begin + lane,
                       v.t1, v.kvh, w);
    else
      empty_sub(w);
  };
  // lane 0: copy an item's q group (G rows, contiguous) into this warp's q buffer
  uint32_t qwaits = 0;  // q copies waited for (barrier phase)
  bool qpend = false;   // a q copy is in flight
  auto copy_q = [&](const Item& v) {
    qpend = v.valid;
    if (lane == 0 && v.valid) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_tx(qbar, (uint32_t)(G * kD * 2));
      bulk_load_1d(smem_u32(qbuf),
                   static_cast<const uint16_t*>(a.q) + ((int64_t)v.s * a.num_q_heads + v.kvh * G) * kD,
                   (uint32_t)(G * kD * 2), qbar);
    }
  };

  int pslot = 0, pk = 0;
  uint32_t g_iss = 0, g_cons = 0;
  bool dead = false;
  // The first item streams, and is consumed, before the plan has finished: the second is
  // fetched (which waits for the plan kernel) only NST + 1 sub-tiles before the end of the
  // first, and the producer stops at the end of an item whose successor is not resolved
  // yet. Not with 8-token blocks, where the extra live state would spill: there both items
  // are resolved first.
  constexpr bool kRamp = BS != 8;
  bool listed = false;  // the plan has finished and the second item is resolved
  Item cur = static_item(), nxt{0, 0, 0, 0, 0, 0, 0, 0};
  SubWin cur_w, nxt_w;
  empty_sub(nxt_w);
  auto produce = [&]() {
    while (!dead && g_iss - g_cons < (uint32_t)NST) {
      if (pslot == 0 && pk >= cur.nsub) { pslot = 1; pk = 0; }
      if (pslot == 1 && (!nxt.valid || pk >= nxt.nsub)) break;
      // field-wise selects: a reference to one of the two items would put both in local
      // memory
      const bool first = pslot == 0;
      const int c_begin = first ? cur.c_begin : nxt.c_begin, kvh = first ? cur.kvh : nxt.kvh;
      const SubWin sw = shfl_sub<BS>(select_sub(first, cur_w, nxt_w), pk);
      const int stage = g_iss % NST;
      if (lane == 0)
        issue_sub<KV, BS>(wtiles + stage * STAGE, &kmap, &vmap, bars + 8 * stage, policy, sw,
                          c_begin + pk, kvh, Hkv);
      ++g_iss;
      ++pk;
    }
  };
  auto start = [&]() {
    load_window(cur, cur_w);
    copy_q(cur);
    produce();
  };
  auto take_list = [&]() {
    pdl_wait();  // the plan kernel's list and counters
    total = pl.counters[1];
    listed = true;
  };
  if constexpr (kRamp) {
    if (cur.valid) start();
    if (!cur.valid || cur.nsub <= NST + 1) {
      take_list();
      if (!cur.valid) {  // no static item: the first comes from the list
        cur = fetch();
        if (cur.valid) start();
      }
      nxt = fetch();
      load_window(nxt, nxt_w);
      produce();
    }
  } else {
    take_list();
    if (!cur.valid) cur = fetch();
    nxt = fetch();
    load_window(nxt, nxt_w);
    start();
  }

  uint32_t qf[8][2];
  WarpAcc w;
  while (cur.valid) {
    if (!dead) {
      if (mbar_wait(qbar, qwaits & 1)) {
        ++qwaits;
        qpend = false;
      } else {
        if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
        dead = true;
      }
    }
    const float zscale = load_q_frags<FP8>(reinterpret_cast<const uint16_t*>(qbuf), G, lane,
                                           a.scale_log2, qf);
    __syncwarp();
    if (!dead && listed) copy_q(nxt);  // the buffer is free once every lane holds its fragments
    w.reset();
    for (int i = 0; i < cur.nsub; ++i) {
      const SubWin sw = shfl_sub<BS>(cur_w, i);
      const int stage = g_cons % NST;
      if (!dead && !mbar_wait(bars + 8 * stage, (g_cons / NST) & 1)) {
        if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
        dead = true;
      }
      if (!dead && sub_ok(sw)) {
        const uint32_t kt = wtiles + stage * STAGE;
        tc_block<KV>(kt, kt + TILE, min(kSub, cur.t1 - (cur.c_begin + i) * kSub),
                     half_params<KV>(sw, zscale), qf, w, lane);
      }
      __syncwarp();
      ++g_cons;
      if (kRamp && !listed && i + 1 >= cur.nsub - NST - 1) {  // the first item's successor
        take_list();
        nxt = fetch();
        load_window(nxt, nxt_w);
        if (!dead) copy_q(nxt);
      }
      produce();
    }
    // ---- item done: its output (single partition) or its partial ----
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, o);
      w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, o);
    }
    const float unit = FP8 ? w.vref : 1.f;
    const int64_t row0 = (int64_t)cur.s * a.num_q_heads + cur.kvh * G;
    const int g0 = 2 * tq, g1 = 2 * tq + 1;
    const bool live0 = g0 < G, live1 = g1 < G;
    const float ms[2] = {w.m0, w.m1}, ls[2] = {w.l0, w.l1};
    const uint64_t keep = evict_last_policy();
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      int dA, dB;
      if constexpr (FP8) {
        dA = 32 * (t >> 1) + 2 * gq + (t & 1);
        dB = dA + 16;
      } else {
        dA = 16 * t + gq;
        dB = dA + 8;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!(h == 0 ? live0 : live1)) continue;
        const int64_t row = row0 + 2 * tq + h;
        const float x0 = w.acc[t][h] * unit, x1 = w.acc[t][2 + h] * unit;
        if (cur.np == 1) {
          const float inv = ls[h] > 0.f ? 1.f / ls[h] : 0.f;
          store_out(a.out, a.out_dtype, row * kD + dA, x0 * inv);
          store_out(a.out, a.out_dtype, row * kD + dB, x1 * inv);
        } else {
          const int64_t pr = (row * a.max_parts + cur.part) * kD;
          st_hint(a.part_acc + pr + dA, x0, keep);
          st_hint(a.part_acc + pr + dB, x1, keep);
        }
      }
    }
    if (gq == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!(h == 0 ? live0 : live1)) continue;
        const int64_t row = row0 + 2 * tq + h;
        if (cur.np == 1) {
          if (a.lse_out != nullptr)
            a.lse_out[row] = ls[h] > 0.f ? (ms[h] + __log2f(ls[h])) * kLn2 : -INFINITY;
        } else {
          const int64_t pr = row * a.max_parts + cur.part;
          st_hint(a.part_m + pr, ms[h], keep);
          st_hint(a.part_l + pr, ls[h], keep);
        }
      }
    }
    // ---- advance ----
    cur = nxt;
    cur_w = nxt_w;
    nxt = fetch();
    load_window(nxt, nxt_w);
    pslot = 0;
    produce();
  }
  pdl_trigger();  // no more items: the reduce may be scheduled (it waits for this grid)
  if (dead) {
    // wait (bounded) for the copies this warp issued and did not consume
    for (uint32_t j = g_cons; j < g_iss; ++j)
      if (!mbar_wait(bars + 8 * (j % NST), (j / NST) & 1)) break;
    if (qpend) mbar_wait(qbar, qwaits & 1);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
// The driver's tensor-map encoder, looked up once (a function-local static is initialised
// once even when several host threads make their first call together).
inline PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

// The pool seen as rows of 128 bytes: a token's K (or V) is one row (one-byte codes) or
// two (bf16); a box is one 16-token sub-tile, or half of one for 8-token blocks.
inline bool make_map(CUtensorMap* m, const void* base, int64_t total_rows, pa_dtype kv,
                     int block_size) {
  auto enc = encoder();
  if (enc == nullptr) return false;
  const bool fp8 = kv != PA_BF16;  // one-byte codes (fp8 or int8), copied as raw bytes
  const int box_tokens = block_size < kSub ? block_size : kSub;
  cuuint64_t dims[2] = {(cuuint64_t)(fp8 ? 128 : 64), (cuuint64_t)total_rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {(cuuint32_t)(fp8 ? 128 : 64), (cuuint32_t)(box_tokens * (fp8 ? 1 : 2))};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;  // per-device caches of the launch set-up

// Per-device cache entries are atomics: first calls on several host threads may fill the
// same entry at once (with the same value), and later calls read it without a lock.
using DeviceCache = std::atomic<int>[kMaxDevices];

inline int sm_count() {
  static DeviceCache cache;  // static storage: zero-initialised
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Tensor-core kernel families: grid of one CTA per item, persistent CTAs sharing an item,
// persistent warp workers.
enum TcKind { kTcGrid = 0, kTcCta = 1, kTcWarps = 2 };

// `smem_limit`: the kernel's dynamic shared-memory limit (the largest any launch uses);
// `smem`: this launch's size, for the occupancy.
template <typename K>
inline cudaError_t occupancy(K kernel, int threads, int smem, int* per_sm, int smem_limit = 0) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_limit > smem ? smem_limit : smem);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, kernel, threads, smem);
  if (e == cudaSuccess && *per_sm <= 0) e = cudaErrorInvalidConfiguration;
  return e;
}

// Launch set-up of one kernel on the current device: its dynamic shared-memory limit is
// raised and its resident CTAs per SM measured once per device the process uses (`slots`
// is the kernel's per-device cache; concurrent first calls store the same values).
template <typename K>
inline cudaError_t resident_per_sm(K kernel, int threads, int smem, DeviceCache& slots,
                                   int* per_sm, int smem_limit = 0) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int n = slots[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    e = occupancy(kernel, threads, smem, &n, smem_limit);
    if (e != cudaSuccess) return e;
    slots[dev].store(n, std::memory_order_relaxed);
  }
  *per_sm = n;
  return cudaSuccess;
}

template <pa_dtype KV, int BS>
inline cudaError_t launch_tc_kv(const DecodeArgs& a, const pa_decode_desc* d, dim3 grid,
                                const PlanView* pl, TcKind kind, cudaStream_t st) {
  using C = TcCfg<KV>;
  const int64_t rows = (int64_t)d->num_blocks * d->num_kv_heads * BS * (C::kFp8 ? 1 : 2);
  CUtensorMap km, vm;
  if (!make_map(&km, a.k_cache, rows, KV, BS) || !make_map(&vm, a.v_cache, rows, KV, BS))
    return cudaErrorInvalidValue;
  if (kind == kTcGrid) {
    static DeviceCache slots;
    int per_sm = 0;
    cudaError_t e = resident_per_sm(decode_tc_kernel<KV, BS>, kNW * 32, C::kSmem, slots, &per_sm);
    if (e != cudaSuccess) return e;
    decode_tc_kernel<KV, BS><<<grid, kNW * 32, C::kSmem, st>>>(a, km, vm);
    return cudaGetLastError();
  }
  const int sms = sm_count();
  if (sms <= 0 || pl == nullptr) return cudaErrorInvalidValue;
  cudaError_t e;
  if (kind == kTcWarps) {
    // occupancy depends on the group's q buffers: measured (and cached) per group size; the
    // kernel's shared-memory limit is set for the largest group
    static DeviceCache slots_g[8];
    int per_sm = 0;
    const int gsz = TcwCfg<KV>::smem(a.group);
    e = resident_per_sm(decode_tc_warps<KV, BS>, kWW * 32, gsz, slots_g[a.group - 1], &per_sm,
                        TcwCfg<KV>::kMaxSmem);
    if (e != cudaSuccess) return e;
    const int warps = sms * per_sm * kWW;
    DecodeArgs w = a;
    w.static_seqs = min(warps / a.num_kv_heads, a.num_seqs);  // whole sequences only
    e = launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, st, w, *pl);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_tc_warps<KV, BS>, dim3(sms * per_sm), dim3(kWW * 32), gsz, st, w,
                   *pl, km, vm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  e = launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, st, a, *pl);
  if (e != cudaSuccess) return e;
  if (kind == kTcCta) {
    if constexpr (BS != kSub) return cudaErrorInvalidValue;
    static DeviceCache slots;
    int per_sm = 0;
    e = resident_per_sm(decode_tc_persistent<KV>, kNW * 32, C::kPSmem, slots, &per_sm);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_tc_persistent<KV>, dim3(sms * per_sm), dim3(kNW * 32), C::kPSmem, st,
                   a, *pl, km, vm);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace tc

inline bool tc_supported(const pa_decode_desc* d) {
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->kv_dtype != PA_BF16 && d->kv_dtype != PA_FP8_E4M3 && d->kv_dtype != PA_INT8)
    return false;
  if (d->q_dtype != PA_BF16 || d->out_dtype != PA_BF16) return false;
  if (d->head_dim != tc::kD || G > 8) return false;
  if (d->block_size != 8 && d->block_size != 16 && d->block_size != 32) return false;
  const int64_t rows = (int64_t)d->num_blocks * d->num_kv_heads * d->block_size * 2;
  return rows < (int64_t)1 << 31;
}

// Which tensor-core kernel runs a call. impl: 2 = automatic, 3 = grid, 4 = persistent
// CTAs, 5 = persistent warps. The persistent kernels need the split path (a workspace for
// the plan) and keep one partition's 16-token sub-tiles per warp in 32-entry register
// windows: persistent CTAs (16-token blocks only) up to 32 * 4 sub-tiles (2048 tokens),
// warp workers up to 32 sub-tiles (512 tokens). Automatic: warp workers where they fit,
// else one CTA per item (faster than the persistent CTAs wherever both were measured on
// a B200: 1024-token partitions of 32 sequences, 512-token ones of 8 x 131072 tokens).
inline tc::TcKind tc_kind(const pa_decode_desc* d, bool split, int impl) {
  const int P = d->partition_size;
  const bool cta_ok = split && d->block_size == kSub && P <= 32 * tc::kNW * kSub;
  const bool warps_ok = split && P <= 32 * kSub;
  if (impl == 3) return tc::kTcGrid;
  if (impl == 4) return cta_ok ? tc::kTcCta : tc::kTcGrid;
  if (impl == 5) return warps_ok ? tc::kTcWarps : (cta_ok ? tc::kTcCta : tc::kTcGrid);
  return warps_ok ? tc::kTcWarps : tc::kTcGrid;
}

inline cudaError_t launch_tc(const DecodeArgs& a, const pa_decode_desc* d, dim3 grid,
                             const tc::PlanView* pl, tc::TcKind kind, cudaStream_t st) {
  auto by_bs = [&](auto kv) -> cudaError_t {
    constexpr pa_dtype KV = decltype(kv)::value;
    if (d->block_size == 8) return tc::launch_tc_kv<KV, 8>(a, d, grid, pl, kind, st);
    if (d->block_size == 32) return tc::launch_tc_kv<KV, 32>(a, d, grid, pl, kind, st);
    return tc::launch_tc_kv<KV, 16>(a, d, grid, pl, kind, st);
  };
  if (d->kv_dtype == PA_BF16) return by_bs(std::integral_constant<pa_dtype, PA_BF16>{});
  if (d->kv_dtype == PA_INT8) return by_bs(std::integral_constant<pa_dtype, PA_INT8>{});
  return by_bs(std::integral_constant<pa_dtype, PA_FP8_E4M3>{});
}

}  // namespace pa
