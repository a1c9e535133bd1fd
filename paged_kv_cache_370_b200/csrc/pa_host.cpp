// pa_host.cpp -- host-side parts of the library: the block manager (free list,
// reference counts, copy-on-write decisions), slot computation and status names.
//
// The block manager follows the pages' description of paged KV management:
// fixed-size blocks handed out from a free list on demand and returned for
// reuse when a request ends ("大语言模型推理内存管理算法 paged attention",
// sections 7 and 8; "08. PagedAttention：把 KV Cache 分页管理", section
// "借用操作系统的办法：分页"), block tables shared between sequences with a
// reference count per block (same page, section "分页还顺带解决了什么"), and
// copy-on-write when a sequence writes into a shared block ("PagedAttention
// 核心思想解析", section 2.3), and the release of blocks a sliding window has
// moved past (same page, section 5.2). Slots are block_table[logical block] *
// block_size + offset (third page, section "为什么叫 PagedAttention").
//
// The free list is a LIFO stack of block ids: a freed block is the next one
// handed out, which keeps recently used blocks warm in L2.

#include "pa.h"

#include <algorithm>
#include <new>
#include <unordered_map>
#include <vector>

namespace {

// Table entry of a block released because a sliding window moved past it.
constexpr int32_t kReleased = -1;

struct Sequence {
  std::vector<int32_t> blocks;  // logical block i -> physical block (or kReleased)
  int64_t len = 0;              // tokens stored
  bool swapped = false;         // blocks name host swap-space blocks
};

}  // namespace

struct pa_alloc {
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // back() is handed out next
  std::vector<int32_t> ref_count;   // per physical block
  std::unordered_map<int64_t, Sequence> seqs;
  std::vector<int32_t> host_free;   // host swap-space blocks, back() handed out next
  std::vector<int32_t> host_ref;    // per host block

  int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }

  int32_t pop() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    ref_count[b] = 1;
    return b;
  }
};

extern "C" {

pa_status pa_alloc_create(int num_blocks, int block_size, pa_alloc **out) {
  if (!out || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID;
  pa_alloc *a = new (std::nothrow) pa_alloc();
  if (!a) return PA_ERR_INVALID;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ref_count.assign(num_blocks, 0);
  a->free_stack.resize(num_blocks);
  for (int i = 0; i < num_blocks; ++i) a->free_stack[i] = num_blocks - 1 - i;  // block 0 first
  *out = a;
  return PA_OK;
}

void pa_alloc_destroy(pa_alloc *a) { delete a; }

pa_status pa_alloc_add_seq(pa_alloc *a, int64_t seq_id, int num_tokens) {
  if (!a || num_tokens < 0) return PA_ERR_INVALID;
  if (a->seqs.count(seq_id)) return PA_ERR_STATE;
  int64_t need = a->blocks_for(num_tokens);
  if (need > (int64_t)a->free_stack.size()) return PA_ERR_OUT_OF_BLOCKS;
  Sequence s;
  s.blocks.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->pop());
  s.len = num_tokens;
  a->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

pa_status pa_alloc_fork(pa_alloc *a, int64_t parent, int64_t child) {
  if (!a) return PA_ERR_INVALID;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child) || it->second.swapped) return PA_ERR_STATE;
  Sequence c = it->second;
  for (int32_t b : c.blocks)
    if (b != kReleased) a->ref_count[b] += 1;
  a->seqs.emplace(child, std::move(c));
  return PA_OK;
}

pa_status pa_alloc_append_slot(pa_alloc *a, int64_t seq_id, int64_t *slot, int64_t *cow_src,
                               int64_t *cow_dst) {
  if (!a || !slot) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end() || it->second.swapped) return PA_ERR_STATE;
  Sequence &s = it->second;
  const int64_t pos = s.len;
  const int64_t logical = pos / a->block_size;
  const int64_t offset = pos % a->block_size;
  int64_t src = -1, dst = -1;
  if (logical == (int64_t)s.blocks.size()) {
    // the last block is full (or there is none): take a new one
    if (a->free_stack.empty()) return PA_ERR_OUT_OF_BLOCKS;
    s.blocks.push_back(a->pop());
  } else {
    int32_t blk = s.blocks[logical];
    if (a->ref_count[blk] > 1) {
      // shared block: copy on write
      if (a->free_stack.empty()) return PA_ERR_OUT_OF_BLOCKS;
      int32_t fresh = a->pop();
      a->ref_count[blk] -= 1;
      s.blocks[logical] = fresh;
      src = blk;
      dst = fresh;
    }
  }
  s.len = pos + 1;
  *slot = (int64_t)s.blocks[logical] * a->block_size + offset;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_OK;
}

pa_status pa_alloc_seq_slots(const pa_alloc *a, int64_t seq_id, int start, int count,
                             int64_t *slots) {
  if (!a || start < 0 || count < 0 || (count && !slots)) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end() || it->second.swapped) return PA_ERR_STATE;
  const Sequence &s = it->second;
  if ((int64_t)start + count > s.len) return PA_ERR_INVALID;
  for (int i = 0; i < count; ++i)
    if (s.blocks[((int64_t)start + i) / a->block_size] == kReleased) return PA_ERR_STATE;
  for (int i = 0; i < count; ++i) {
    int64_t pos = (int64_t)start + i;
    slots[i] = (int64_t)s.blocks[pos / a->block_size] * a->block_size + pos % a->block_size;
  }
  return PA_OK;
}

pa_status pa_alloc_free_seq(pa_alloc *a, int64_t seq_id) {
  if (!a) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_STATE;
  const std::vector<int32_t> &blocks = it->second.blocks;
  std::vector<int32_t> &ref = it->second.swapped ? a->host_ref : a->ref_count;
  std::vector<int32_t> &free_list = it->second.swapped ? a->host_free : a->free_stack;
  for (int32_t b : blocks)
    if (b != kReleased && ref[b] <= 0) return PA_ERR_STATE;  // would underflow: refuse, change nothing
  for (auto r = blocks.rbegin(); r != blocks.rend(); ++r) {
    if (*r != kReleased && --ref[*r] == 0) free_list.push_back(*r);
  }
  a->seqs.erase(it);
  return PA_OK;
}

pa_status pa_alloc_slide_window(pa_alloc *a, int64_t seq_id, int window, int *freed) {
  if (!a || window <= 0) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end() || it->second.swapped) return PA_ERR_STATE;
  Sequence &s = it->second;
  // blocks wholly before the window [len - window, len) of the current length
  const int64_t lo = s.len > window ? s.len - window : 0;
  const int64_t gone = lo / a->block_size;
  int n = 0;
  for (int64_t i = 0; i < gone; ++i) {
    int32_t b = s.blocks[i];
    if (b == kReleased) continue;
    if (a->ref_count[b] <= 0) return PA_ERR_STATE;
    s.blocks[i] = kReleased;
    if (--a->ref_count[b] == 0) {
      a->free_stack.push_back(b);
      ++n;
    }
  }
  if (freed) *freed = n;
  return PA_OK;
}

pa_status pa_alloc_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int cap,
                               int *num_blocks, int *num_tokens) {
  if (!a) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_STATE;
  const Sequence &s = it->second;
  if (num_blocks) *num_blocks = (int)s.blocks.size();
  if (num_tokens) *num_tokens = (int)s.len;
  if (out) {
    if (cap < (int)s.blocks.size()) return PA_ERR_INVALID;
    std::copy(s.blocks.begin(), s.blocks.end(), out);
  }
  return PA_OK;
}

pa_status pa_alloc_fill_tables(const pa_alloc *a, const int64_t *seq_ids, int n,
                               int32_t *block_tables, int max_blocks_per_seq, int32_t pad,
                               int32_t *context_lens) {
  if (!a || n < 0 || (n && (!seq_ids || !block_tables)) || max_blocks_per_seq <= 0)
    return PA_ERR_INVALID;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end() || it->second.swapped) return PA_ERR_STATE;
    const Sequence &s = it->second;
    if ((int)s.blocks.size() > max_blocks_per_seq) return PA_ERR_INVALID;
    int32_t *row = block_tables + (size_t)i * max_blocks_per_seq;
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    std::fill(row + s.blocks.size(), row + max_blocks_per_seq, pad);
    if (context_lens) context_lens[i] = (int32_t)s.len;
  }
  return PA_OK;
}

pa_status pa_alloc_ref_count(const pa_alloc *a, int32_t block, int *ref_count) {
  if (!a || !ref_count || block < 0 || block >= a->num_blocks) return PA_ERR_INVALID;
  *ref_count = a->ref_count[block];
  return PA_OK;
}

pa_status pa_alloc_stats(const pa_alloc *a, int *free_blocks, int64_t *used_tokens,
                         int64_t *wasted_tokens) {
  if (!a) return PA_ERR_INVALID;
  // A block's fill is the most positions any sequence referencing it stores there.
  std::unordered_map<int32_t, int> fill;
  for (const auto &kv : a->seqs) {
    const Sequence &s = kv.second;
    if (s.swapped) continue;  // its blocks are in the host swap space
    for (size_t i = 0; i < s.blocks.size(); ++i) {
      if (s.blocks[i] == kReleased) continue;
      int64_t f = std::min<int64_t>(a->block_size, s.len - (int64_t)i * a->block_size);
      int &cur = fill[s.blocks[i]];
      cur = std::max<int>(cur, (int)std::max<int64_t>(f, 0));
    }
  }
  int64_t used = 0;
  for (const auto &kv : fill) used += kv.second;
  const int64_t used_blocks = a->num_blocks - (int64_t)a->free_stack.size();
  if (free_blocks) *free_blocks = (int)a->free_stack.size();
  if (used_tokens) *used_tokens = used;
  if (wasted_tokens) *wasted_tokens = used_blocks * a->block_size - used;
  return PA_OK;
}

pa_status pa_alloc_set_host_blocks(pa_alloc *a, int num_host_blocks) {
  if (!a || num_host_blocks <= 0) return PA_ERR_INVALID;
  if (!a->host_ref.empty()) return PA_ERR_STATE;
  a->host_ref.assign(num_host_blocks, 0);
  a->host_free.resize(num_host_blocks);
  for (int i = 0; i < num_host_blocks; ++i) a->host_free[i] = num_host_blocks - 1 - i;
  return PA_OK;
}

// Move a group of sequences between the device pool and the host swap space.
// Blocks the group shares move once; a block also held outside the group is
// copied and stays on its side for the others. All or nothing.
static pa_status swap_group(pa_alloc *a, const int64_t *seq_ids, int n, int64_t *pairs, int cap,
                            int *num_pairs, bool out) {
  if (!a || n < 0 || (n && !seq_ids) || !num_pairs || cap < 0 || (cap && !pairs))
    return PA_ERR_INVALID;
  if (a->host_ref.empty()) return PA_ERR_STATE;  // no swap space
  std::vector<Sequence *> group;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end() || it->second.swapped == out) return PA_ERR_STATE;
    for (Sequence *g : group)
      if (g == &it->second) return PA_ERR_INVALID;  // listed twice
    group.push_back(&it->second);
  }
  // distinct blocks in order of first use, with the group's references to each
  std::vector<int32_t> order;
  std::unordered_map<int32_t, int> refs;
  for (Sequence *g : group)
    for (int32_t b : g->blocks) {
      if (b == kReleased) continue;
      if (refs[b]++ == 0) order.push_back(b);
    }
  std::vector<int32_t> &src_ref = out ? a->ref_count : a->host_ref;
  std::vector<int32_t> &src_free = out ? a->free_stack : a->host_free;
  std::vector<int32_t> &dst_ref = out ? a->host_ref : a->ref_count;
  std::vector<int32_t> &dst_free = out ? a->host_free : a->free_stack;
  for (int32_t b : order)
    if (src_ref[b] < refs[b]) return PA_ERR_STATE;
  if (order.size() > dst_free.size()) return PA_ERR_OUT_OF_BLOCKS;
  if ((int)order.size() > cap) return PA_ERR_INVALID;
  std::unordered_map<int32_t, int32_t> moved;
  for (size_t i = 0; i < order.size(); ++i) {
    const int32_t b = order[i];
    const int32_t d = dst_free.back();
    dst_free.pop_back();
    dst_ref[d] = refs[b];
    if ((src_ref[b] -= refs[b]) == 0) src_free.push_back(b);
    moved[b] = d;
    pairs[2 * i] = b;
    pairs[2 * i + 1] = d;
  }
  for (Sequence *g : group) {
    for (int32_t &b : g->blocks)
      if (b != kReleased) b = moved[b];
    g->swapped = out;
  }
  *num_pairs = (int)order.size();
  return PA_OK;
}

pa_status pa_alloc_swap_out(pa_alloc *a, const int64_t *seq_ids, int n, int64_t *pairs, int cap,
                            int *num_pairs) {
  return swap_group(a, seq_ids, n, pairs, cap, num_pairs, true);
}

pa_status pa_alloc_swap_in(pa_alloc *a, const int64_t *seq_ids, int n, int64_t *pairs, int cap,
                           int *num_pairs) {
  return swap_group(a, seq_ids, n, pairs, cap, num_pairs, false);
}

pa_status pa_alloc_is_swapped(const pa_alloc *a, int64_t seq_id, int *swapped) {
  if (!a || !swapped) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_STATE;
  *swapped = it->second.swapped ? 1 : 0;
  return PA_OK;
}

pa_status pa_alloc_host_free(const pa_alloc *a, int *free_host_blocks) {
  if (!a || !free_host_blocks) return PA_ERR_INVALID;
  *free_host_blocks = (int)a->host_free.size();
  return PA_OK;
}

pa_status pa_slot_mapping(const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *counts, int num_seqs, int block_size, int64_t *slots) {
  if (num_seqs < 0 || block_size <= 0 || max_blocks_per_seq <= 0) return PA_ERR_INVALID;
  if (num_seqs && (!block_tables || !counts || !slots)) return PA_ERR_INVALID;
  int64_t k = 0;
  for (int b = 0; b < num_seqs; ++b) {
    const int32_t *row = block_tables + (size_t)b * max_blocks_per_seq;
    if (counts[b] < 0 || (int64_t)counts[b] > (int64_t)max_blocks_per_seq * block_size)
      return PA_ERR_INVALID;
    for (int t = 0; t < counts[b]; ++t)
      slots[k++] = (int64_t)row[t / block_size] * block_size + t % block_size;
  }
  return PA_OK;
}

const char *pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID";
    case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS";
    case PA_ERR_STATE: return "PA_ERR_STATE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
  }
  return "PA_ERR_UNKNOWN";
}

}  // extern "C"
