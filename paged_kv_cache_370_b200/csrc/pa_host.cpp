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
//
// Prefix caching ("大语言模型推理内存管理算法 paged attention", section 9;
// "08. PagedAttention：把 KV Cache 分页管理", section "分页还顺带解决了什么":
// requests whose prompts begin alike share their first, completely filled
// blocks). A cached block stands for one token prefix: every token from
// position 0 to the end of the block. The prefixes form a trie whose nodes are
// keyed by (parent node, the block's own tokens) and checked in full on every
// lookup, so a hit never rests on the hash alone; a node may have no block
// (its block was reused) while longer prefixes below it are still cached. A
// cached block whose last reference goes keeps its contents and waits,
// counted as free, in a list ordered by release time; it is reused (oldest
// first) only when no plain free block is left.

#include "pa.h"

#include <algorithm>
#include <cstring>
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
  std::vector<int32_t> free_stack;  // free blocks holding no cached prefix; back() next
  std::vector<int32_t> ref_count;   // per physical block
  std::unordered_map<int64_t, Sequence> seqs;
  std::vector<int32_t> host_free;   // host swap-space blocks, back() handed out next
  std::vector<int32_t> host_ref;    // per host block

  // ---- prefix cache: a trie of token prefixes, one node per distinct
  // prefix of whole blocks that is cached or has a cached extension
  struct Node {
    int64_t parent = -1;  // the node of the prefix one block shorter; -1 at the root
    int32_t block = -1;   // the block holding this prefix's last block_size tokens, or -1
    int32_t children = 0;
  };
  std::vector<Node> nodes;
  std::vector<int32_t> node_tokens;     // [node][block_size]: the node's own tokens
  std::vector<int64_t> spare_nodes;     // deleted node slots
  std::unordered_multimap<uint64_t, int64_t> index;  // key hash -> node
  std::vector<int64_t> node_of;         // per block: its node, or -1
  int64_t cached = 0;                   // blocks holding a cached prefix
  // free cached blocks, oldest release first: an intrusive list through lru_next/lru_prev
  std::vector<int32_t> lru_prev, lru_next;
  int32_t lru_head = -1, lru_tail = -1;
  int64_t lru_size = 0;

  int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }
  int64_t num_free() const { return (int64_t)free_stack.size() + lru_size; }
  bool cache_ready() const { return !node_of.empty(); }

  void cache_init() {
    if (cache_ready()) return;
    node_of.assign(num_blocks, -1);
    lru_prev.assign(num_blocks, -1);
    lru_next.assign(num_blocks, -1);
  }

  // FNV-1a (Fowler, Noll, Vo) over the parent node and the block's tokens.
  uint64_t key_hash(int64_t parent, const int32_t *tok) const {
    uint64_t h = 1469598103934665603ull;
    auto eat = [&h](const void *p, size_t n) {
      const unsigned char *c = static_cast<const unsigned char *>(p);
      for (size_t i = 0; i < n; ++i) {
        h ^= c[i];
        h *= 1099511628211ull;
      }
    };
    eat(&parent, sizeof parent);
    eat(tok, sizeof(int32_t) * (size_t)block_size);
    return h;
  }

  const int32_t *tokens_of(int64_t n) const { return &node_tokens[(size_t)n * block_size]; }

  // The node for (parent, tok), or -1; the key is checked in full.
  int64_t find(int64_t parent, const int32_t *tok) const {
    if (!cache_ready()) return -1;
    auto range = index.equal_range(key_hash(parent, tok));
    for (auto it = range.first; it != range.second; ++it) {
      const int64_t n = it->second;
      if (nodes[n].parent == parent &&
          std::memcmp(tokens_of(n), tok, sizeof(int32_t) * block_size) == 0)
        return n;
    }
    return -1;
  }

  int64_t find_or_add(int64_t parent, const int32_t *tok) {
    int64_t n = find(parent, tok);
    if (n >= 0) return n;
    if (!spare_nodes.empty()) {
      n = spare_nodes.back();
      spare_nodes.pop_back();
    } else {
      n = (int64_t)nodes.size();
      nodes.emplace_back();
      node_tokens.resize(node_tokens.size() + block_size);
    }
    nodes[n] = Node{parent, -1, 0};
    std::memcpy(&node_tokens[(size_t)n * block_size], tok, sizeof(int32_t) * block_size);
    index.emplace(key_hash(parent, tok), n);
    if (parent >= 0) nodes[parent].children += 1;
    return n;
  }

  // Delete nodes that hold no block and lead to none, from n towards the root.
  void prune(int64_t n) {
    while (n >= 0 && nodes[n].block < 0 && nodes[n].children == 0) {
      auto range = index.equal_range(key_hash(nodes[n].parent, tokens_of(n)));
      for (auto it = range.first; it != range.second; ++it)
        if (it->second == n) {
          index.erase(it);
          break;
        }
      const int64_t up = nodes[n].parent;
      spare_nodes.push_back(n);
      if (up >= 0) nodes[up].children -= 1;
      n = up;
    }
  }

  // Block b no longer holds its prefix (it is about to be reused).
  void uncache(int32_t b) {
    const int64_t n = node_of[b];
    nodes[n].block = -1;
    node_of[b] = -1;
    --cached;
    prune(n);
  }

  void lru_unlink(int32_t b) {
    if (lru_prev[b] >= 0) lru_next[lru_prev[b]] = lru_next[b]; else lru_head = lru_next[b];
    if (lru_next[b] >= 0) lru_prev[lru_next[b]] = lru_prev[b]; else lru_tail = lru_prev[b];
    lru_prev[b] = lru_next[b] = -1;
    --lru_size;
  }

  void lru_append(int32_t b) {
    lru_prev[b] = lru_tail;
    lru_next[b] = -1;
    if (lru_tail >= 0) lru_next[lru_tail] = b; else lru_head = b;
    lru_tail = b;
    ++lru_size;
  }

  // A free block with reference count 1. The caller checked num_free() > 0.
  int32_t take() {
    int32_t b;
    if (!free_stack.empty()) {
      b = free_stack.back();
      free_stack.pop_back();
    } else {
      b = lru_head;  // the cached block released longest ago
      lru_unlink(b);
      uncache(b);
    }
    ref_count[b] = 1;
    return b;
  }

  // Block b's count has just reached zero.
  void release(int32_t b) {
    if (cache_ready() && node_of[b] >= 0)
      lru_append(b);
    else
      free_stack.push_back(b);
  }

  // A cached block gains a reference (leaving the free list if it was there).
  void reuse(int32_t b) {
    if (ref_count[b] == 0) lru_unlink(b);
    ref_count[b] += 1;
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
  if (need > a->num_free()) return PA_ERR_OUT_OF_BLOCKS;
  Sequence s;
  s.blocks.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->take());
  s.len = num_tokens;
  a->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

pa_status pa_alloc_add_seq_cached(pa_alloc *a, int64_t seq_id, const int32_t *tokens,
                                  int num_tokens, int *num_cached_tokens) {
  if (!a || num_tokens < 0 || (num_tokens && !tokens)) return PA_ERR_INVALID;
  if (a->seqs.count(seq_id)) return PA_ERR_STATE;
  a->cache_init();
  const int bs = a->block_size;
  const int64_t need = a->blocks_for(num_tokens);
  // the cached prefix: full blocks within the first num_tokens - 1 tokens, from the start
  const int64_t lookable = num_tokens > 0 ? (int64_t)(num_tokens - 1) / bs : 0;
  std::vector<int32_t> hits;
  int64_t node = -1, idle_hits = 0;
  for (int64_t i = 0; i < lookable; ++i) {
    const int64_t n = a->find(node, tokens + i * bs);
    if (n < 0 || a->nodes[n].block < 0) break;
    const int32_t b = a->nodes[n].block;
    hits.push_back(b);
    if (a->ref_count[b] == 0) ++idle_hits;  // counted as free now, not after the reuse
    node = n;
  }
  if (need - (int64_t)hits.size() > a->num_free() - idle_hits) return PA_ERR_OUT_OF_BLOCKS;
  Sequence s;
  s.blocks.reserve(need);
  for (int32_t b : hits) {  // before any take(), so no eviction can reach them
    a->reuse(b);
    s.blocks.push_back(b);
  }
  for (int64_t i = (int64_t)hits.size(); i < need; ++i) s.blocks.push_back(a->take());
  // cache the full blocks this prompt fills whose prefix no block holds yet
  const int64_t full = num_tokens / bs;
  for (int64_t i = (int64_t)hits.size(); i < full; ++i) {
    node = a->find_or_add(node, tokens + i * bs);
    if (a->nodes[node].block >= 0) continue;  // held by another block already
    a->nodes[node].block = s.blocks[i];
    a->node_of[s.blocks[i]] = node;
    ++a->cached;
  }
  s.len = num_tokens;
  a->seqs.emplace(seq_id, std::move(s));
  if (num_cached_tokens) *num_cached_tokens = (int)((int64_t)hits.size() * bs);
  return PA_OK;
}

pa_status pa_alloc_cached_blocks(const pa_alloc *a, int *cached_blocks, int *cached_free_blocks) {
  if (!a) return PA_ERR_INVALID;
  if (cached_blocks) *cached_blocks = (int)a->cached;
  if (cached_free_blocks) *cached_free_blocks = (int)a->lru_size;
  return PA_OK;
}

pa_status pa_alloc_reset_prefix_cache(pa_alloc *a) {
  if (!a) return PA_ERR_INVALID;
  if (!a->cache_ready()) return PA_OK;
  for (int32_t b = a->lru_head; b >= 0;) {  // free cached blocks become plain free blocks
    const int32_t next = a->lru_next[b];
    a->lru_prev[b] = a->lru_next[b] = -1;
    a->free_stack.push_back(b);
    b = next;
  }
  a->lru_head = a->lru_tail = -1;
  a->lru_size = 0;
  std::fill(a->node_of.begin(), a->node_of.end(), -1);
  a->nodes.clear();
  a->node_tokens.clear();
  a->spare_nodes.clear();
  a->index.clear();
  a->cached = 0;
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
    if (a->num_free() == 0) return PA_ERR_OUT_OF_BLOCKS;
    s.blocks.push_back(a->take());
  } else {
    int32_t blk = s.blocks[logical];
    if (a->ref_count[blk] > 1) {
      // shared block: copy on write
      if (a->num_free() == 0) return PA_ERR_OUT_OF_BLOCKS;
      int32_t fresh = a->take();
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
  const bool host = it->second.swapped;
  std::vector<int32_t> &ref = host ? a->host_ref : a->ref_count;
  for (int32_t b : blocks)
    if (b != kReleased && ref[b] <= 0) return PA_ERR_STATE;  // would underflow: refuse, change nothing
  for (auto r = blocks.rbegin(); r != blocks.rend(); ++r) {
    if (*r == kReleased || --ref[*r] != 0) continue;
    if (host)
      a->host_free.push_back(*r);
    else
      a->release(*r);
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
      a->release(b);
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
  const int64_t used_blocks = a->num_blocks - a->num_free();
  if (free_blocks) *free_blocks = (int)a->num_free();
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
  std::vector<int32_t> &dst_ref = out ? a->host_ref : a->ref_count;
  for (int32_t b : order)
    if (src_ref[b] < refs[b]) return PA_ERR_STATE;
  const int64_t dst_free = out ? (int64_t)a->host_free.size() : a->num_free();
  if ((int64_t)order.size() > dst_free) return PA_ERR_OUT_OF_BLOCKS;
  if ((int)order.size() > cap) return PA_ERR_INVALID;
  std::unordered_map<int32_t, int32_t> moved;
  for (size_t i = 0; i < order.size(); ++i) {
    const int32_t b = order[i];
    int32_t d;
    if (out) {
      d = a->host_free.back();
      a->host_free.pop_back();
    } else {
      d = a->take();
    }
    dst_ref[d] = refs[b];
    if ((src_ref[b] -= refs[b]) == 0) {
      if (out)
        a->release(b);
      else
        a->host_free.push_back(b);
    }
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
