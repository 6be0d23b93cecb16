// Host block allocator of the paged KV cache (C ABI in include/pagedattn.h).
//
// [Ch4PA] "Borrowing the fix from OS paging": fixed-size units kept on a free list always
// satisfy an allocation while enough units remain, so there is no external fragmentation.
// [KVFail] Key Points: blocks are handed out from a free queue and an allocation fails when
// too few free blocks remain. [KVPaged] "PagedAttention: OS virtual-memory style
// management": a block is allocated as tokens accumulate; the block table maps a
// sequence's logical positions to physical blocks. [KVPaged] "Prefix sharing and
// copy-on-write" and [Ch4PA] "Prefix Caching": forked sequences point at the same physical
// blocks, ref_count counts the sharers, and a shared block is copied only when written.
//
// Policy: FIFO free queue, pop front, push back when a block's ref_count reaches 0 (in
// block-table order). Append copies the last block first when it is partially filled and
// shared, then pops one block per block boundary crossed. Every operation checks its
// preconditions before changing anything, so a failed call leaves the state untouched.
//
// Automatic prefix caching ([Ch4PA] "Prefix Caching": a SHA-256 hash of the prefix
// identifies identical blocks, hits raise ref_count; [KVPaged] "Prefix cache lifetime and
// invalidation": a hit skips recomputing the KV, eviction is least-recently-used; [KVFail]
// Key Points: a cached block is evicted when the free queue hands it out again):
// every full block of a sequence added with its token ids gets the chained hash
// h_i = SHA-256(h_{i-1} || token ids of block i as little-endian int32), h_-1 empty. A new
// sequence reuses the cached blocks of its longest matching run of full blocks; its other
// full blocks are registered. A freed block keeps its entry while it waits in the free
// queue (so the queue order is the LRU order) and loses it when the queue hands it out.
// The free queue is an intrusive doubly linked list, so a hit can take a waiting block out
// of the middle in O(1).
#include <algorithm>
#include <array>
#include <climits>
#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"

namespace {

// ---------------------------------------------------------------------------------------
// SHA-256 (FIPS 180-4): 64 rounds over 512-bit blocks of the padded message.
// ---------------------------------------------------------------------------------------
struct Sha256 {
  uint32_t h[8] = {0x6a09e667, 0xbb67ae85, 0x3c6ef372, 0xa54ff53a,
                   0x510e527f, 0x9b05688c, 0x1f83d9ab, 0x5be0cd19};
  uint8_t buf[64];
  size_t fill = 0;
  uint64_t bits = 0;

  static uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

  void block(const uint8_t* p) {
    static const uint32_t K[64] = {
        0x428a2f98, 0x71374491, 0xb5c0fbcf, 0xe9b5dba5, 0x3956c25b, 0x59f111f1, 0x923f82a4,
        0xab1c5ed5, 0xd807aa98, 0x12835b01, 0x243185be, 0x550c7dc3, 0x72be5d74, 0x80deb1fe,
        0x9bdc06a7, 0xc19bf174, 0xe49b69c1, 0xefbe4786, 0x0fc19dc6, 0x240ca1cc, 0x2de92c6f,
        0x4a7484aa, 0x5cb0a9dc, 0x76f988da, 0x983e5152, 0xa831c66d, 0xb00327c8, 0xbf597fc7,
        0xc6e00bf3, 0xd5a79147, 0x06ca6351, 0x14292967, 0x27b70a85, 0x2e1b2138, 0x4d2c6dfc,
        0x53380d13, 0x650a7354, 0x766a0abb, 0x81c2c92e, 0x92722c85, 0xa2bfe8a1, 0xa81a664b,
        0xc24b8b70, 0xc76c51a3, 0xd192e819, 0xd6990624, 0xf40e3585, 0x106aa070, 0x19a4c116,
        0x1e376c08, 0x2748774c, 0x34b0bcb5, 0x391c0cb3, 0x4ed8aa4a, 0x5b9cca4f, 0x682e6ff3,
        0x748f82ee, 0x78a5636f, 0x84c87814, 0x8cc70208, 0x90befffa, 0xa4506ceb, 0xbef9a3f7,
        0xc67178f2};
    uint32_t w[64];
    for (int i = 0; i < 16; ++i)
      w[i] = (uint32_t)p[4 * i] << 24 | (uint32_t)p[4 * i + 1] << 16 |
             (uint32_t)p[4 * i + 2] << 8 | (uint32_t)p[4 * i + 3];
    for (int i = 16; i < 64; ++i) {
      const uint32_t s0 = rotr(w[i - 15], 7) ^ rotr(w[i - 15], 18) ^ (w[i - 15] >> 3);
      const uint32_t s1 = rotr(w[i - 2], 17) ^ rotr(w[i - 2], 19) ^ (w[i - 2] >> 10);
      w[i] = w[i - 16] + s0 + w[i - 7] + s1;
    }
    uint32_t a = h[0], b = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], k = h[7];
    for (int i = 0; i < 64; ++i) {
      const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
      const uint32_t ch = (e & f) ^ (~e & g);
      const uint32_t t1 = k + S1 + ch + K[i] + w[i];
      const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
      const uint32_t maj = (a & b) ^ (a & c) ^ (b & c);
      const uint32_t t2 = S0 + maj;
      k = g; g = f; f = e; e = d + t1; d = c; c = b; b = a; a = t1 + t2;
    }
    h[0] += a; h[1] += b; h[2] += c; h[3] += d; h[4] += e; h[5] += f; h[6] += g; h[7] += k;
  }
  void update(const void* data, size_t n) {
    const uint8_t* p = static_cast<const uint8_t*>(data);
    bits += (uint64_t)n * 8;
    while (n > 0) {
      const size_t take = (64 - fill) < n ? (64 - fill) : n;
      std::memcpy(buf + fill, p, take);
      fill += take;
      p += take;
      n -= take;
      if (fill == 64) {
        block(buf);
        fill = 0;
      }
    }
  }
  void final(uint8_t out[32]) {
    const uint64_t total = bits;
    const uint8_t one = 0x80, zero = 0;
    update(&one, 1);
    while (fill != 56) update(&zero, 1);
    uint8_t len[8];
    for (int i = 0; i < 8; ++i) len[i] = (uint8_t)(total >> (56 - 8 * i));
    update(len, 8);
    for (int i = 0; i < 8; ++i)
      for (int j = 0; j < 4; ++j) out[4 * i + j] = (uint8_t)(h[i] >> (24 - 8 * j));
  }
};

using Digest = std::array<uint8_t, 32>;

struct DigestHash {
  size_t operator()(const Digest& d) const {
    size_t x;
    std::memcpy(&x, d.data(), sizeof(x));
    return x;
  }
};

// h_i = SHA-256(h_{i-1} || block tokens as little-endian int32), h_{-1} = empty.
Digest chain_hash(const Digest* parent, const int32_t* tokens, int n) {
  Sha256 s;
  if (parent != nullptr) s.update(parent->data(), 32);
  for (int i = 0; i < n; ++i) {
    const uint32_t t = (uint32_t)tokens[i];
    const uint8_t le[4] = {(uint8_t)t, (uint8_t)(t >> 8), (uint8_t)(t >> 16), (uint8_t)(t >> 24)};
    s.update(le, 4);
  }
  Digest d;
  s.final(d.data());
  return d;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

struct pa_allocator {
  int num_blocks;
  int block_size;
  // free queue: intrusive doubly linked list over block ids
  std::vector<int32_t> prev, next;
  std::vector<char> in_free;
  int32_t head = -1, tail = -1;
  int nfree = 0;
  std::vector<int32_t> refs;
  std::unordered_map<int, std::vector<int32_t>> tables;
  std::unordered_map<int, int> lens;
  // prefix cache
  std::vector<Digest> block_hash;
  std::vector<char> has_hash;
  std::unordered_map<Digest, int32_t, DigestHash> cached;
  int64_t hit_blocks = 0, evictions = 0;

  void push_back(int32_t b) {
    prev[b] = tail;
    next[b] = -1;
    if (tail >= 0) next[tail] = b; else head = b;
    tail = b;
    in_free[b] = 1;
    ++nfree;
  }
  void unlink(int32_t b) {
    if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
    if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
    prev[b] = next[b] = -1;
    in_free[b] = 0;
    --nfree;
  }
  // Hands out the front of the queue; a block still holding a cache entry loses it.
  int32_t pop() {
    const int32_t b = head;
    unlink(b);
    if (has_hash[b]) {
      cached.erase(block_hash[b]);
      has_hash[b] = 0;
      ++evictions;
    }
    refs[b] = 1;
    return b;
  }
  void release(int32_t b) {
    refs[b] -= 1;
    if (refs[b] == 0) push_back(b);
  }
  // Appends n tokens to an existing sequence whose preconditions were checked (enough free
  // blocks; a pair buffer when a copy can occur): copies the last block first when it is
  // partially filled and shared, then pops one block per block boundary crossed. Writes
  // the tokens' slots and the copy pair; returns the number of pairs (0 or 1).
  // `row` and `len` are the sequence's block table and length.
  int append_checked(std::vector<int32_t>& row, int& len, int n, int64_t* slots_out,
                     int32_t* pair_out) {
    const int L = len;
    const bool cow = n > 0 && L % block_size != 0 && refs[row.back()] > 1;
    if (cow) {
      const int32_t old_b = row.back();
      const int32_t new_b = pop();
      refs[old_b] -= 1;
      row.back() = new_b;
      pair_out[0] = old_b;
      pair_out[1] = new_b;
    }
    const int64_t grow = ceil_div((int64_t)L + n, block_size) - ceil_div(L, block_size);
    for (int64_t i = 0; i < grow; ++i) row.push_back(pop());
    len = L + n;
    row_slots(row, L, n, slots_out);
    return cow ? 1 : 0;
  }
  void row_slots(const std::vector<int32_t>& row, int start, int n, int64_t* out) const {
    if (out == nullptr) return;
    for (int i = 0; i < n; ++i) {
      const int p = start + i;
      out[i] = (int64_t)row[p / block_size] * block_size + p % block_size;
    }
  }
  void slots(int seq, int start, int n, int64_t* out) const {
    row_slots(tables.at(seq), start, n, out);
  }
};

extern "C" {

pa_allocator* pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t* order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pa_allocator* a = new (std::nothrow) pa_allocator();
  if (a == nullptr) return nullptr;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->prev.assign(num_blocks, -1);
  a->next.assign(num_blocks, -1);
  a->in_free.assign(num_blocks, 0);
  a->refs.assign(num_blocks, 0);
  a->block_hash.resize(num_blocks);
  a->has_hash.assign(num_blocks, 0);
  if (order == nullptr) {
    for (int b = 0; b < num_blocks; ++b) a->push_back(b);
  } else {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return nullptr;
      }
      seen[b] = 1;
      a->push_back(b);
    }
  }
  return a;
}

pa_allocator* pa_alloc_create(int num_blocks, int block_size) {
  return pa_alloc_create_ordered(num_blocks, block_size, nullptr);
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

int pa_alloc_num_free(const pa_allocator* a) { return a ? a->nfree : -1; }

int pa_alloc_ref_count(const pa_allocator* a, int block) {
  if (a == nullptr || block < 0 || block >= a->num_blocks) return -1;
  return a->refs[block];
}

pa_status pa_alloc_add_seq(pa_allocator* a, int seq_id, int num_tokens, int64_t* slots_out) {
  if (a == nullptr || seq_id < 0 || num_tokens < 0) return PA_ERR_INVALID;
  if (a->tables.count(seq_id)) return PA_ERR_INVALID;
  const int64_t need = ceil_div(num_tokens, a->block_size);
  if (need > a->nfree) return PA_ERR_NO_BLOCKS;
  std::vector<int32_t> row;
  row.reserve(need);
  for (int64_t i = 0; i < need; ++i) row.push_back(a->pop());
  a->tables.emplace(seq_id, std::move(row));
  a->lens[seq_id] = num_tokens;
  a->slots(seq_id, 0, num_tokens, slots_out);
  return PA_OK;
}

pa_status pa_alloc_add_seq_tokens(pa_allocator* a, int seq_id, const int32_t* tokens,
                                  int num_tokens, int64_t* slots_out, int* cached_tokens_out) {
  if (a == nullptr || seq_id < 0 || num_tokens < 0) return PA_ERR_INVALID;
  if (num_tokens > 0 && tokens == nullptr) return PA_ERR_INVALID;
  if (a->tables.count(seq_id)) return PA_ERR_INVALID;
  const int B = a->block_size;
  const int nfull = num_tokens / B;
  const int64_t nblk = ceil_div(num_tokens, B);
  std::vector<Digest> h(nfull);
  int hits = 0;
  int hits_waiting = 0;  // hit blocks that sit in the free queue
  std::vector<int32_t> hit_blocks;
  for (int i = 0; i < nfull; ++i) {
    h[i] = chain_hash(i ? &h[i - 1] : nullptr, tokens + (int64_t)i * B, B);
    if (hits == i) {
      auto it = a->cached.find(h[i]);
      if (it != a->cached.end()) {
        hit_blocks.push_back(it->second);
        hits_waiting += a->in_free[it->second] ? 1 : 0;
        ++hits;
      }
    }
  }
  if (nblk - hits > a->nfree - hits_waiting) return PA_ERR_NO_BLOCKS;
  std::vector<int32_t> row;
  row.reserve(nblk);
  for (int32_t b : hit_blocks) {  // take hits out of the queue first: they must not be popped
    if (a->in_free[b]) a->unlink(b);
    a->refs[b] += 1;
    row.push_back(b);
  }
  for (int64_t i = hits; i < nblk; ++i) {
    const int32_t b = a->pop();
    row.push_back(b);
    if (i < nfull) {  // a full block of this prompt: register it
      a->block_hash[b] = h[i];
      a->has_hash[b] = 1;
      a->cached[h[i]] = b;
    }
  }
  a->hit_blocks += hits;
  a->tables.emplace(seq_id, std::move(row));
  a->lens[seq_id] = num_tokens;
  a->slots(seq_id, 0, num_tokens, slots_out);
  if (cached_tokens_out) *cached_tokens_out = hits * B;
  return PA_OK;
}

pa_status pa_alloc_fork(pa_allocator* a, int parent_id, int child_id) {
  if (a == nullptr || child_id < 0) return PA_ERR_INVALID;
  auto it = a->tables.find(parent_id);
  if (it == a->tables.end() || a->tables.count(child_id)) return PA_ERR_INVALID;
  std::vector<int32_t> row = it->second;
  for (int32_t b : row) a->refs[b] += 1;
  a->lens[child_id] = a->lens[parent_id];
  a->tables.emplace(child_id, std::move(row));
  return PA_OK;
}

pa_status pa_alloc_append(pa_allocator* a, int seq_id, int num_tokens, int64_t* slots_out,
                          int32_t* cow_pairs_out, int* num_cow_out) {
  if (a == nullptr || num_tokens < 0) return PA_ERR_INVALID;
  auto it = a->tables.find(seq_id);
  if (it == a->tables.end()) return PA_ERR_INVALID;
  const std::vector<int32_t>& row = it->second;
  const int B = a->block_size;
  const int L = a->lens.at(seq_id);
  if ((int64_t)L + num_tokens > INT32_MAX) return PA_ERR_INVALID;
  const bool cow = num_tokens > 0 && L % B != 0 && a->refs[row.back()] > 1;
  if (cow && cow_pairs_out == nullptr) return PA_ERR_INVALID;
  const int64_t grow = ceil_div((int64_t)L + num_tokens, B) - ceil_div(L, B);
  if ((cow ? 1 : 0) + grow > (int64_t)a->nfree) return PA_ERR_NO_BLOCKS;
  const int ncow = a->append_checked(it->second, a->lens[seq_id], num_tokens, slots_out,
                                     cow_pairs_out);
  if (num_cow_out) *num_cow_out = ncow;
  return PA_OK;
}

pa_status pa_alloc_append_batch(pa_allocator* a, int n, const int32_t* seq_ids,
                                const int32_t* num_tokens, int64_t* slots_out,
                                int32_t* cow_pairs_out, int* num_cow_out) {
  if (a == nullptr || n < 0) return PA_ERR_INVALID;
  if (n > 0 && (seq_ids == nullptr || num_tokens == nullptr)) return PA_ERR_INVALID;
  const int B = a->block_size;
  std::vector<int32_t> ids(seq_ids, seq_ids + n);  // distinct ids
  std::sort(ids.begin(), ids.end());
  if (std::adjacent_find(ids.begin(), ids.end()) != ids.end()) return PA_ERR_INVALID;
  // checks, and the blocks the whole batch pops: the appends run in batch order, and a
  // copy-on-write drops the old block's ref_count, which later sequences of the batch see
  struct Item {
    std::vector<int32_t>* row;
    int* len;
  };
  std::vector<Item> items((size_t)n);
  std::unordered_map<int32_t, int> ref_delta;
  int64_t need = 0;
  bool any_cow = false;
  for (int i = 0; i < n; ++i) {
    const int s = seq_ids[i], k = num_tokens[i];
    if (k < 0) return PA_ERR_INVALID;
    auto it = a->tables.find(s);
    if (it == a->tables.end()) return PA_ERR_INVALID;
    int& L = a->lens.find(s)->second;
    if ((int64_t)L + k > INT32_MAX) return PA_ERR_INVALID;
    items[i] = Item{&it->second, &L};
    if (k > 0 && L % B != 0) {
      const int32_t last = it->second.back();
      auto d = ref_delta.find(last);
      const int refs = a->refs[last] + (d == ref_delta.end() ? 0 : d->second);
      if (refs > 1) {
        ref_delta[last] -= 1;
        need += 1;
        any_cow = true;
      }
    }
    need += ceil_div((int64_t)L + k, B) - ceil_div(L, B);
  }
  if (any_cow && cow_pairs_out == nullptr) return PA_ERR_INVALID;
  if (need > (int64_t)a->nfree) return PA_ERR_NO_BLOCKS;
  int64_t off = 0;
  int ncow = 0;
  for (int i = 0; i < n; ++i) {
    ncow += a->append_checked(*items[i].row, *items[i].len, num_tokens[i],
                              slots_out ? slots_out + off : nullptr,
                              cow_pairs_out ? cow_pairs_out + 2 * ncow : nullptr);
    off += num_tokens[i];
  }
  if (num_cow_out) *num_cow_out = ncow;
  return PA_OK;
}

pa_status pa_alloc_free_seq(pa_allocator* a, int seq_id) {
  if (a == nullptr) return PA_ERR_INVALID;
  auto it = a->tables.find(seq_id);
  if (it == a->tables.end()) return PA_ERR_INVALID;
  for (int32_t b : it->second) a->release(b);
  a->tables.erase(it);
  a->lens.erase(seq_id);
  return PA_OK;
}

int pa_alloc_block_table(const pa_allocator* a, int seq_id, int32_t* out, int cap) {
  if (a == nullptr) return -1;
  auto it = a->tables.find(seq_id);
  if (it == a->tables.end()) return -1;
  const int n = (int)it->second.size();
  if (out != nullptr)
    for (int i = 0; i < n && i < cap; ++i) out[i] = it->second[i];
  return n;
}

int pa_alloc_seq_len(const pa_allocator* a, int seq_id) {
  if (a == nullptr) return -1;
  auto it = a->lens.find(seq_id);
  return it == a->lens.end() ? -1 : it->second;
}

int pa_alloc_free_queue(const pa_allocator* a, int32_t* out, int cap) {
  if (a == nullptr) return -1;
  if (out != nullptr) {
    int i = 0;
    for (int32_t b = a->head; b >= 0 && i < cap; b = a->next[b], ++i) out[i] = b;
  }
  return a->nfree;
}

int pa_alloc_num_cached(const pa_allocator* a) { return a ? (int)a->cached.size() : -1; }

pa_status pa_alloc_cache_stats(const pa_allocator* a, int64_t* hit_blocks,
                               int64_t* evictions) {
  if (a == nullptr) return PA_ERR_INVALID;
  if (hit_blocks) *hit_blocks = a->hit_blocks;
  if (evictions) *evictions = a->evictions;
  return PA_OK;
}

int pa_alloc_block_hash(const pa_allocator* a, int block, uint8_t* out32) {
  if (a == nullptr || block < 0 || block >= a->num_blocks || !a->has_hash[block]) return 0;
  if (out32 != nullptr) std::memcpy(out32, a->block_hash[block].data(), 32);
  return 1;
}

void pa_sha256(const void* data, size_t len, uint8_t* out32) {
  Sha256 s;
  if (len > 0) s.update(data, len);
  s.final(out32);
}

}  // extern "C"
