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
#include <climits>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"

struct pa_allocator {
  int num_blocks;
  int block_size;
  std::deque<int32_t> free_q;
  std::vector<int32_t> refs;
  std::unordered_map<int, std::vector<int32_t>> tables;
  std::unordered_map<int, int> lens;

  int32_t pop() {
    const int32_t b = free_q.front();
    free_q.pop_front();
    refs[b] = 1;
    return b;
  }
  void slots(int seq, int start, int n, int64_t* out) const {
    if (out == nullptr) return;
    const std::vector<int32_t>& row = tables.at(seq);
    for (int i = 0; i < n; ++i) {
      const int p = start + i;
      out[i] = (int64_t)row[p / block_size] * block_size + p % block_size;
    }
  }
};

namespace {
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
}  // namespace

extern "C" {

pa_allocator* pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t* order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pa_allocator* a = new (std::nothrow) pa_allocator();
  if (a == nullptr) return nullptr;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->refs.assign(num_blocks, 0);
  if (order == nullptr) {
    for (int b = 0; b < num_blocks; ++b) a->free_q.push_back(b);
  } else {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return nullptr;
      }
      seen[b] = 1;
      a->free_q.push_back(b);
    }
  }
  return a;
}

pa_allocator* pa_alloc_create(int num_blocks, int block_size) {
  return pa_alloc_create_ordered(num_blocks, block_size, nullptr);
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

int pa_alloc_num_free(const pa_allocator* a) { return a ? (int)a->free_q.size() : -1; }

int pa_alloc_ref_count(const pa_allocator* a, int block) {
  if (a == nullptr || block < 0 || block >= a->num_blocks) return -1;
  return a->refs[block];
}

pa_status pa_alloc_add_seq(pa_allocator* a, int seq_id, int num_tokens, int64_t* slots_out) {
  if (a == nullptr || seq_id < 0 || num_tokens < 0) return PA_ERR_INVALID;
  if (a->tables.count(seq_id)) return PA_ERR_INVALID;
  const int64_t need = ceil_div(num_tokens, a->block_size);
  if (need > (int64_t)a->free_q.size()) return PA_ERR_NO_BLOCKS;
  std::vector<int32_t> row;
  row.reserve(need);
  for (int64_t i = 0; i < need; ++i) row.push_back(a->pop());
  a->tables.emplace(seq_id, std::move(row));
  a->lens[seq_id] = num_tokens;
  a->slots(seq_id, 0, num_tokens, slots_out);
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
  std::vector<int32_t>& row = it->second;
  const int B = a->block_size;
  const int L = a->lens[seq_id];
  if ((int64_t)L + num_tokens > INT32_MAX) return PA_ERR_INVALID;
  const bool cow = num_tokens > 0 && L % B != 0 && a->refs[row.back()] > 1;
  if (cow && cow_pairs_out == nullptr) return PA_ERR_INVALID;
  const int64_t grow = ceil_div((int64_t)L + num_tokens, B) - ceil_div(L, B);
  if ((cow ? 1 : 0) + grow > (int64_t)a->free_q.size()) return PA_ERR_NO_BLOCKS;
  int ncow = 0;
  if (cow) {
    const int32_t old_b = row.back();
    const int32_t new_b = a->pop();
    a->refs[old_b] -= 1;
    row.back() = new_b;
    cow_pairs_out[0] = old_b;
    cow_pairs_out[1] = new_b;
    ncow = 1;
  }
  for (int64_t i = 0; i < grow; ++i) row.push_back(a->pop());
  a->lens[seq_id] = L + num_tokens;
  if (num_cow_out) *num_cow_out = ncow;
  a->slots(seq_id, L, num_tokens, slots_out);
  return PA_OK;
}

pa_status pa_alloc_free_seq(pa_allocator* a, int seq_id) {
  if (a == nullptr) return PA_ERR_INVALID;
  auto it = a->tables.find(seq_id);
  if (it == a->tables.end()) return PA_ERR_INVALID;
  for (int32_t b : it->second) {
    a->refs[b] -= 1;
    if (a->refs[b] == 0) a->free_q.push_back(b);
  }
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
  const int n = (int)a->free_q.size();
  if (out != nullptr) {
    int i = 0;
    for (auto it = a->free_q.begin(); it != a->free_q.end() && i < cap; ++it, ++i) out[i] = *it;
  }
  return n;
}

}  // extern "C"
