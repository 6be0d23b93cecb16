/*
 * pagedattn.h — C ABI of libpagedattn.so, paged decode attention for NVIDIA B200 (sm_100a).
 *
 * Scope: the decode-step hot path of PagedAttention. The KV cache is cut into fixed-size
 * blocks (8, 16 or 32 tokens; 16 by default) scattered through a physical block pool; a per-sequence block table maps
 * logical blocks to physical ones; sequences with a common prefix share physical blocks,
 * counted by ref_count, and a shared block is copied before it is written (copy-on-write).
 * Sources (page title, section):
 *   [KVPaged] "KV cache and paged attention" (youngju.dev)
 *   [Ch4PA]   "Why PagedAttention cuts GPU memory waste by up to 95%" (iq-universe.github.io,
 *             ch4-paged-attention)
 *   [OpsVLLM] "How does vLLM PagedAttention manage the KV cache" (opsoai.com)
 *   [KVFail]  "Transformer inference KV-cache memory-management failure modes"
 *             (knowledge.openakashic.com)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named *_cache, q, out, k, v, block_tables, context_lens, query_start,
 *   slot_mapping, pairs, *_scales, *_zeros, lse_out and workspace are DEVICE pointers; the
 *   caller owns them. The library allocates no device memory (paged_attn_decode_noalloc's
 *   fixed array is compiled into the library, below).
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Device
 *   work is enqueued asynchronously on it; a PA_OK return means "enqueued".
 * - Every call validates its host-side arguments first and returns an error without
 *   enqueuing anything when they are wrong. Faults of asynchronous work show up at the next
 *   synchronisation, as with any CUDA launch.
 * - Data that lives on the device cannot be validated by the host. Kernels bounds-check
 *   every block id, slot and copy pair they read; an out-of-range value is skipped (the
 *   access is not made) and recorded in a device error word, see pa_device_error().
 * - Cache layout: cache[num_blocks][num_kv_heads][block_size][head_dim], row-major, so each
 *   (physical block, kv head) tile is contiguous (the pages give no layout; this is the
 *   library's choice). fp8 caches carry float32 scales[num_blocks][num_kv_heads], one per
 *   (block, kv head), separately for K and V: stored value = E4M3(x / scale). int8 caches
 *   ([KVPaged] "KV quantization: FP8 and INT8": one byte per element with a scale and a
 *   zero point) carry the same scales plus int32 zero points[num_blocks][num_kv_heads]:
 *   stored code = clamp(round_half_even(x / scale) + zero, -128, 127), value =
 *   (code - zero) * scale. Zero points must lie in [-128, 127], the byte's own range
 *   (an affine int8 code needs no other); there code - zero is exact in every kernel. A
 *   block whose K or V zero point lies outside is treated like a bad block id: attention
 *   skips it and the cache write skips its rows, and PA_DEVERR_ZERO is recorded.
 * - q and out: [num_seqs][num_q_heads][head_dim] row-major. Query head h reads kv head
 *   h / (num_q_heads / num_kv_heads) ([KVPaged] "GQA and MQA": query heads are grouped and
 *   each group shares one KV head).
 * - block_tables: int32 [num_seqs][max_blocks_per_seq]; entry b of row s is the physical
 *   block holding logical tokens [B*b, B*b+B) of sequence s (B = block_size); entries at or beyond
 *   ceil(context_lens[s] / block_size) are never read ([Ch4PA] "PagedAttention algorithm":
 *   the block table maps logical block ids to physical blocks that need not be contiguous).
 * - context_lens[s] counts every cached token of sequence s, including the token being
 *   decoded (whose K/V must have been written by reshape_and_cache first).
 *
 * Supported today: block_size 8, 16 or 32 ([KVPaged] "the block-size knob" and [Ch4PA]
 * "Theorem 1, fragmentation bound": smaller blocks waste less of the last block, larger
 * ones need shorter tables; 16 is the usual default); head_dim 64, 128 or 256; num_q_heads a multiple of
 * num_kv_heads with a group of at most 16; (q, kv, out) dtypes (f32, f32, f32),
 * (bf16, bf16, bf16), (bf16, fp8_e4m3, bf16) and (bf16, int8, bf16). Anything else returns
 * PA_ERR_UNSUPPORTED.
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2, PA_INT8 = 3 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = -1,      /* bad argument: null pointer, size out of range, bad id      */
  PA_ERR_UNSUPPORTED = -2,  /* valid but not implemented (dtype combination, head_dim...) */
  PA_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed                       */
  PA_ERR_NO_BLOCKS = -4,    /* allocator: not enough free blocks; nothing was changed     */
  PA_ERR_WORKSPACE = -5,    /* workspace missing or smaller than paged_attn_workspace_size */
  PA_ERR_DEVICE = -6        /* a kernel recorded a bad block id / slot / pair, see below  */
} pa_status;

/* Bits of the device error word (pa_device_error). */
#define PA_DEVERR_BLOCK_ID 0x1   /* block table entry outside [0, num_blocks)          */
#define PA_DEVERR_SLOT 0x2       /* slot_mapping entry outside [-inf, num_blocks*bs)    */
#define PA_DEVERR_PAIR 0x4       /* copy_blocks pair outside [0, num_blocks)            */
#define PA_DEVERR_CONTEXT 0x8    /* context_lens entry < 0 or > max_context_len         */
#define PA_DEVERR_TIMEOUT 0x10   /* a bounded wait on an asynchronous copy gave up      */
#define PA_DEVERR_QUERY 0x20     /* prefill query_start not ascending, past num_tokens, */
                                 /* or more new tokens than context (or max_query_len)  */
#define PA_DEVERR_ZERO 0x40      /* int8 zero point outside [-128, 127]                 */

/*
 * partition_size value that lets the library choose the split for a decode call: one
 * pass (0) when max_context_len <= 512; else 512 tokens when num_seqs * num_kv_heads >=
 * 1024, else 1024. The choice depends only on the descriptor and max_context_len, so
 * results stay independent of where blocks sit; paged_attn_partition_size() reports it.
 */
#define PA_PARTITION_AUTO (-1)

/* Shape and dtypes of one paged decode-attention call. */
typedef struct {
  int num_seqs;            /* S >= 0                                                   */
  int num_q_heads;         /* Hq                                                       */
  int num_kv_heads;        /* Hkv; Hq % Hkv == 0                                       */
  int head_dim;            /* d                                                        */
  int block_size;          /* tokens per block: 8, 16 or 32                            */
  int max_blocks_per_seq;  /* row stride of block_tables                               */
  int num_blocks;          /* physical blocks in the pool (bounds check)               */
  int partition_size;      /* split-KV partition in tokens, a multiple of block_size   */
                           /* and of 16;                                               */
                           /* 0 = one pass over the whole context per (seq, kv head);  */
                           /* PA_PARTITION_AUTO = the library's choice (below)         */
  pa_dtype q_dtype, kv_dtype, out_dtype;
} pa_decode_desc;

/*
 * Bytes of device workspace paged_attn_decode needs for this shape when no context is
 * longer than max_context_len (0 when partition_size == 0). Returns 0 for an invalid
 * descriptor as well; paged_attn_decode then reports the error.
 */
size_t paged_attn_workspace_size(const pa_decode_desc* desc, int max_context_len);

/*
 * The partition (tokens; 0 = one pass) a paged_attn_decode call with this descriptor uses:
 * desc->partition_size itself, or the library's choice for PA_PARTITION_AUTO. -1 for an
 * invalid descriptor.
 */
int paged_attn_partition_size(const pa_decode_desc* desc, int max_context_len);

/*
 * Number of kernel launches one paged_attn_decode call with this descriptor makes under
 * the current pa_set_decode_impl choice (0 for an invalid, unsupported or empty call):
 * the plan kernel of the persistent tensor-core kernels, the attention kernel, and the
 * log-sum-exp reduce when the split path's partitions are not merged in place. For
 * callers that count launches (profiling, launch budgets).
 */
int paged_attn_decode_launches(const pa_decode_desc* desc, int max_context_len);

/*
 * Decode attention over the paged cache ([KVPaged] "Core principle: what is the KV cache":
 * attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V, one new query per sequence; [Ch4PA]
 * "PagedAttention algorithm": the kernel looks every logical block up in the block table
 * and gathers the non-contiguous K and V blocks). For every sequence s and query head h,
 * with g = h / (Hq/Hkv) and the cached tokens t < context_lens[s]:
 *     z_t = scale * q[s][h] . K_t,   out[s][h] = sum_t softmax(z)_t V_t,
 *     lse_out[s][h] = log sum_t exp(z_t)                    (natural log, float32)
 * fp8 caches are dequantised as E4M3 value * scales[block][g], int8 caches as
 * (code - zeros[block][g]) * scales[block][g]. Accumulation is float32.
 * With partition_size > 0 the context is cut into partitions of that many logical tokens,
 * each reduced to (max, sum, unnormalised output) in `workspace`, then combined by a
 * log-sum-exp reduction; the result does not depend on where blocks sit physically.
 *   q, out         [S][Hq][d] in desc->q_dtype / desc->out_dtype
 *   k_cache/v_cache pool in desc->kv_dtype (layout above)
 *   block_tables   int32 [S][max_blocks_per_seq];  context_lens int32 [S]
 *   max_context_len  host int >= every context_lens entry (sizes the grid)
 *   k_scales/v_scales float32 [num_blocks][Hkv], required for fp8 and int8, else ignored
 *   k_zeros/v_zeros  int32 [num_blocks][Hkv], required for int8, ignored otherwise
 *   lse_out        float32 [S][Hq] or NULL
 *   workspace      device bytes, >= paged_attn_workspace_size(desc, max_context_len),
 *                  16-byte aligned; may be NULL when that size is 0
 * A sequence with context length 0 gets out = 0 and lse = -inf.
 */
pa_status paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            float scale, void* out, const pa_decode_desc* desc,
                            int max_context_len, const float* k_scales, const float* v_scales,
                            const int32_t* k_zeros, const int32_t* v_zeros, float* lse_out,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Prefill attention over the paged cache: the new tokens of a step attend causally to
 * their sequence's cached tokens ([KVPaged] "Core principle: what is the KV cache": the
 * prompt's K/V is computed once and cached, each token attending to itself and all earlier
 * tokens; "Prefix sharing and copy-on-write": a cached prefix's K/V is computed once, so
 * a step may bring only the tokens after it, as may a prompt cut into chunks). Sequence s
 * brings n_s = query_start[s+1] - query_start[s] new tokens, rows query_start[s] .. of q,
 * whose K/V were written by reshape_and_cache first as the last n_s of its
 * context_lens[s] positions. Row i of sequence s sits at position p = context_lens[s] -
 * n_s + i; for query head h (kv head g = h / (Hq/Hkv)):
 *     z_t = scale * q[row][h] . K_t (t <= p),  out[row][h] = sum_t softmax(z)_t V_t,
 *     lse_out[row][h] = log sum_t exp(z_t)              (natural log, float32)
 * with fp8 / int8 dequantisation as in paged_attn_decode. Accumulation is float32.
 *   q, out        [num_tokens][Hq][d] in desc->q_dtype / desc->out_dtype
 *   query_start   int32 [num_seqs + 1], ascending, query_start[0] = 0,
 *                 query_start[num_seqs] = num_tokens
 *   max_query_len host int >= every n_s (sizes the grid); max_context_len >= every
 *                 context_lens entry and >= max_query_len
 *   block_tables, context_lens, k/v scales and zeros, lse_out: as in paged_attn_decode
 *   desc          as in paged_attn_decode with partition_size 0
 * bf16 q / out with a bf16, fp8 or int8 cache, head_dim 128 and a group of 1, 2, 4, 8 or
 * 16 run on the tensor cores (tcgen05, accumulators in tensor memory; fp8 / int8 codes are
 * converted exactly to bf16 in shared memory and their scales applied to the scores and
 * to P); every other supported shape, or pa_set_decode_impl(1), runs one CUDA-core pass
 * per new token. No workspace.
 * A sequence whose query range is inconsistent (descending, past num_tokens, more new
 * tokens than context or than max_query_len) is skipped and PA_DEVERR_QUERY recorded.
 */
pa_status paged_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             const int32_t* query_start, int num_tokens, int max_query_len,
                             float scale, void* out, const pa_decode_desc* desc,
                             int max_context_len, const float* k_scales, const float* v_scales,
                             const int32_t* k_zeros, const int32_t* v_zeros, float* lse_out,
                             void* stream);

/*
 * Largest workspace (bytes) that paged_attn_decode_noalloc can serve from its fixed device
 * array: 32 MiB.
 */
#define PA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * paged_attn_decode for callers that cannot allocate device memory. Some callers may not
 * call cudaMalloc at all: a plugin inside a host runtime that owns every device allocation
 * through its own allocator, a caller with no workspace argument to forward, a latency-
 * bound loop that must not risk cudaMalloc's implicit device synchronisation. This entry
 * point takes the same arguments as paged_attn_decode minus the workspace and computes the
 * same result, bit for bit; the split-KV scratch comes from one fixed array compiled into
 * this library (PA_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that loads the library
 * until the process exits). The pages have no counterpart of this call; it exists only for
 * such callers.
 * - Calls that need more scratch than PA_NOALLOC_SCRATCH_BYTES
 *   (paged_attn_workspace_size(desc, max_context_len) larger than it) return
 *   PA_ERR_WORKSPACE and enqueue nothing.
 * - The first call on a device, whatever its shape, looks the array's device address up
 *   (once per device, with that device current); make that first call before any stream
 *   capture.
 * - It calls no cudaMalloc, cudaFree or other allocating routine.
 * - Every call on a device shares the one array, which keeps the last call's contents. The
 *   kernels re-initialise what they read (work counter, partials) on every call, so stale
 *   contents never matter; but calls that overlap on the GPU (different streams, or
 *   different host threads) race on the array: serialise them.
 */
pa_status paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, const int32_t* context_lens,
                                    float scale, void* out, const pa_decode_desc* desc,
                                    int max_context_len, const float* k_scales,
                                    const float* v_scales, const int32_t* k_zeros,
                                    const int32_t* v_zeros, float* lse_out, void* stream);

/*
 * Slot-mapped write of new tokens' K and V into the pool ([KVPaged] "PagedAttention: OS
 * virtual-memory style management": one block is allocated as tokens accumulate and the
 * block table maps logical positions to physical blocks). For token t with
 * slot = slot_mapping[t] >= 0, block = slot / block_size, offset = slot % block_size:
 *     k_cache[block][h][offset][:] = convert(k[t][h][:])   for every kv head h (same for v)
 * convert: f32->f32 and bf16->bf16 copy bits; f32->bf16 rounds to nearest even; f32 or
 * bf16 -> fp8 stores E4M3(x / scale[block][h]) with an IEEE float32 division, round to
 * nearest even, saturating to +-448; f32 or bf16 -> int8 stores
 * clamp(round_half_even(x / scale[block][h]) + zero[block][h], -128, 127), same division.
 * A negative slot is a padding token and is skipped.
 *   k, v             device [num_tokens][Hkv][head_dim] rows, token stride k_stride /
 *                    v_stride elements (>= Hkv*head_dim), in in_dtype
 *   slot_mapping     int64 [num_tokens]
 *   k_scales/v_scales float32 [num_blocks][Hkv], fp8 and int8 caches (read, not written)
 *   k_zeros/v_zeros  int32 [num_blocks][Hkv], int8 caches only (read, not written)
 * Tokens must map to distinct slots (two writes to one slot race).
 */
pa_status reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                            const int64_t* slot_mapping, int num_tokens, int64_t k_stride,
                            int64_t v_stride, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, pa_dtype in_dtype, pa_dtype cache_dtype,
                            const float* k_scales, const float* v_scales,
                            const int32_t* k_zeros, const int32_t* v_zeros, void* stream);

/*
 * Copy-on-write block copy ([KVPaged] "Prefix sharing and copy-on-write": a shared block is
 * copied before one sharer modifies it; [Ch4PA] "Prefix Caching": copies happen only on
 * write). For each pair i, (src, dst) = (pairs[2i], pairs[2i+1]) (device int32 [n][2]):
 * the K and V tiles of every kv head of block src are copied to block dst, and for fp8
 * and int8 caches the scales too (k_scales/v_scales may be NULL otherwise), for int8 also
 * the zero points (k_zeros/v_zeros may be NULL otherwise). No dst may appear twice
 * or also be a src: such copies race. Enqueue it before the reshape_and_cache that writes
 * into the destination blocks.
 */
pa_status copy_blocks(void* k_cache, void* v_cache, float* k_scales, float* v_scales,
                      int32_t* k_zeros, int32_t* v_zeros, const int32_t* pairs, int num_pairs,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      pa_dtype cache_dtype, void* stream);

/*
 * Reads and clears the device error word of the current device (a bitwise OR of
 * PA_DEVERR_* recorded by kernels since the last call). Synchronises `stream` first.
 * Returns PA_OK when the word was 0, PA_ERR_DEVICE otherwise (bits in *bits_out).
 */
pa_status pa_device_error(int* bits_out, void* stream);

/*
 * Selects the decode kernels used by later paged_attn_decode calls in this process:
 * 0 = automatic (tensor cores for bf16 / fp8 / int8 caches where the shape is supported:
 * persistent warp workers for partitions <= 512 tokens, else one CTA per work item; else
 * the CUDA-core fp32 path), 1 = CUDA-core path only, 2 = same as 0, 3 / 4 / 5 = tensor
 * cores with a fixed kernel where the call allows it: 3 one CTA per work item, 4
 * persistent CTAs that share each work item (split path, partitions <= 2048 tokens), 5
 * persistent warp workers, one work item per warp (split path, partitions <= 512 tokens). All compute the
 * same function; they differ in how work is scheduled and how q.K and P.V are multiplied.
 * Returns PA_ERR_INVALID for any other value. Not thread-safe.
 */
pa_status pa_set_decode_impl(int impl);

/* Library version string, e.g. "pagedattn 0.1 sm_100a". */
const char* pa_version(void);

/* ------------------------------------------------------------------------------------- */
/* Host block allocator ([Ch4PA] "Borrowing the fix from OS paging": a free list of       */
/* fixed-size units; [KVFail] Key Points: blocks come from a free queue and an allocation */
/* fails when too few are free; [KVPaged] "Prefix sharing and copy-on-write" and [Ch4PA]  */
/* "Prefix Caching": ref_count per block, copy only on write).                            */
/*                                                                                       */
/* Policy: FIFO free queue (initial order given or 0..N-1); allocation pops the front; a */
/* block whose ref_count reaches 0 is pushed to the back. add_seq allocates              */
/* ceil(n/block_size) blocks; fork copies the parent's table and length and increments  */
/* every block's ref_count; append first copies the last block if it is partially filled */
/* AND shared (one new block, the pair (old, new) reported, old loses one reference),    */
/* then pops one block per new block boundary crossed. Every call either succeeds fully  */
/* or returns an error and changes nothing. Host only; not thread-safe; the caller owns   */
/* the object. Sequence ids are any non-negative int.                                    */
/* ------------------------------------------------------------------------------------- */
typedef struct pa_allocator pa_allocator;

/* NULL on bad sizes / allocation failure. */
pa_allocator* pa_alloc_create(int num_blocks, int block_size);
/* `order`: host int32[num_blocks], a permutation of 0..num_blocks-1 giving the initial
 * free-queue order. NULL when it is not a permutation. */
pa_allocator* pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t* order);
void pa_alloc_destroy(pa_allocator* a);
int pa_alloc_num_free(const pa_allocator* a);
/* -1 for a block id out of range. */
int pa_alloc_ref_count(const pa_allocator* a, int block);
/* New sequence of num_tokens tokens; host int64 slots_out[num_tokens] (may be NULL)
 * receives slot = block*block_size + offset of every token. */
pa_status pa_alloc_add_seq(pa_allocator* a, int seq_id, int num_tokens, int64_t* slots_out);
pa_status pa_alloc_fork(pa_allocator* a, int parent_id, int child_id);
/* Appends num_tokens tokens; slots_out[num_tokens] receives their slots; cow_pairs_out
 * (host int32[2], may be NULL only if no copy can occur) receives (src, dst) of the
 * copy-on-write copy and *num_cow_out is 0 or 1. */
pa_status pa_alloc_append(pa_allocator* a, int seq_id, int num_tokens, int64_t* slots_out,
                          int32_t* cow_pairs_out, int* num_cow_out);
/*
 * One decode step's appends in one call: num_tokens[i] tokens to sequence seq_ids[i] for
 * i = 0 .. n-1, in that order, with the same results as n pa_alloc_append calls, except
 * that the batch is all-or-nothing: when the free queue cannot serve the whole batch (the
 * copies included), PA_ERR_NO_BLOCKS is returned and nothing changes. Sequence ids must be
 * distinct and known (else PA_ERR_INVALID, nothing changed).
 *   seq_ids, num_tokens  host int32 [n]
 *   slots_out            host int64 [sum of num_tokens] or NULL: sequence i's slots follow
 *                        sequence i-1's
 *   cow_pairs_out        host int32 [n][2], NULL only if no copy can occur: the (src, dst)
 *                        copy-on-write pairs in batch order; *num_cow_out (may be NULL)
 *                        receives their number
 * One call per step instead of one per sequence keeps the host's share of a decode step
 * small for large batches.
 */
pa_status pa_alloc_append_batch(pa_allocator* a, int n, const int32_t* seq_ids,
                                const int32_t* num_tokens, int64_t* slots_out,
                                int32_t* cow_pairs_out, int* num_cow_out);
pa_status pa_alloc_free_seq(pa_allocator* a, int seq_id);
/* Copies at most `cap` entries of the sequence's block table into out (host int32) and
 * returns the table's length, or -1 for an unknown sequence. */
int pa_alloc_block_table(const pa_allocator* a, int seq_id, int32_t* out, int cap);
/* Tokens held by the sequence, -1 if unknown. */
int pa_alloc_seq_len(const pa_allocator* a, int seq_id);
/* Writes the free queue front-to-back into out (at most cap entries); returns its size. */
int pa_alloc_free_queue(const pa_allocator* a, int32_t* out, int cap);

/* ------------------------------------------------------------------------------------- */
/* Automatic prefix caching ([Ch4PA] "Prefix Caching": a SHA-256 hash of the prefix       */
/* identifies identical blocks and hits raise ref_count; [KVPaged] "Prefix cache lifetime */
/* and invalidation": a hit skips recomputing the prefix KV, eviction is least recently   */
/* used; [KVFail] Key Points: a cached block is evicted when the free queue hands it out). */
/* Every full block i of a sequence added with its tokens gets the chained hash           */
/*   h_i = SHA-256(h_{i-1} || tokens of block i as little-endian int32), h_{-1} empty.    */
/* ------------------------------------------------------------------------------------- */
/*
 * New sequence of num_tokens token ids (host int32 tokens[num_tokens]). Its longest run of
 * leading full blocks whose hashes are cached is reused (ref_count + 1; a cached block
 * waiting in the free queue is taken out of it); the remaining blocks are popped from the
 * queue front (a popped block loses any cache entry it had: eviction) and its other full
 * blocks are registered in the cache. slots_out[num_tokens] receives every token's slot;
 * *cached_tokens_out (may be NULL) the number of leading tokens whose K/V is already in
 * the cache (the caller writes only the tokens after them). A freed block keeps its entry
 * while it waits in the free queue. PA_ERR_NO_BLOCKS (nothing changed) when the free queue,
 * minus the cached blocks this call reuses, is too short.
 */
pa_status pa_alloc_add_seq_tokens(pa_allocator* a, int seq_id, const int32_t* tokens,
                                  int num_tokens, int64_t* slots_out, int* cached_tokens_out);
/* Number of blocks with a prefix-cache entry (in use or waiting in the free queue). */
int pa_alloc_num_cached(const pa_allocator* a);
/* Totals since creation: blocks reused by hits, cache entries evicted. */
pa_status pa_alloc_cache_stats(const pa_allocator* a, int64_t* hit_blocks, int64_t* evictions);
/* Copies block's chained hash (32 bytes) into out32 and returns 1, or returns 0 when the
 * block has no cache entry. */
int pa_alloc_block_hash(const pa_allocator* a, int block, uint8_t* out32);
/* SHA-256 (FIPS 180-4) of len bytes at data into out32: the hash the prefix cache uses. */
void pa_sha256(const void* data, size_t len, uint8_t* out32);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDATTN_H_ */
