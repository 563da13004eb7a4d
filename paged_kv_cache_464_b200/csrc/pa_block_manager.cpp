// pa_block_manager.cpp -- host-side paged KV block manager (include/pa_block_manager.h).
//
// Block pool with a FIFO free list, per-sequence block tables, reference
// counts and copy-on-write, after PagedAttentionManager in "vLLM推理引擎深度解析"
// §三 and the block manager of "vLLM 原理与源码阅读" (Block 管理器); optionally
// prefix caching after the same page's Prefix Caching (自动检测与复用).  Every
// operation checks that it can complete before it changes anything.
#include "pa_block_manager.h"

#include <algorithm>
#include <cstring>
#include <deque>
#include <list>
#include <map>
#include <new>
#include <unordered_map>
#include <vector>

struct pa_block_manager {
  struct Seq {
    std::vector<int32_t> table;
    int32_t len = 0;
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> ref_count;   // per block
  std::vector<int32_t> num_tokens;  // tokens stored in each block
  std::deque<int32_t> free_list;    // taken from the front, returned to the back
  std::map<int64_t, Seq> seqs;      // ordered: pa_bm_sequences lists ascending ids

  // ---- prefix caching (pa_bm_create_prefix_caching); unused otherwise
  bool caching = false;
  std::list<int32_t> evictable;                           // cached, reference count 0, oldest release first
  std::vector<std::list<int32_t>::iterator> evict_pos;    // position of a block in `evictable`
  std::vector<uint8_t> is_evictable;
  std::vector<int64_t> entry;           // cache entry number of a cached block, -1 if not cached
  std::vector<int64_t> parent_entry;    // entry of the block before it in its prompt, -1 for the first
  std::vector<uint64_t> key_hash;
  std::vector<int32_t> key_tokens;      // [num_blocks][block_size] token ids of cached blocks
  std::unordered_map<uint64_t, std::vector<int32_t>> by_hash;
  int64_t next_entry = 0, queried = 0, hit = 0, evictions = 0;

  int64_t slot(const Seq &s, int32_t pos) const {
    return (int64_t)s.table[pos / block_size] * block_size + pos % block_size;
  }
  // blocks an allocation may take: the free list, then evictable cached blocks
  int64_t available() const { return (int64_t)free_list.size() + (int64_t)evictable.size(); }
  int32_t take() {
    if (!free_list.empty()) {
      const int32_t b = free_list.front();
      free_list.pop_front();
      return b;
    }
    const int32_t b = evictable.front();   // the least recently released cached block
    evictable.pop_front();
    is_evictable[b] = 0;
    forget(b);
    ++evictions;
    return b;
  }
  // FNV-1a (64-bit) over the parent entry number and the token ids
  static uint64_t hash_key(int64_t parent, const int32_t *tokens, int32_t n) {
    uint64_t h = 14695981039346656037ull;
    auto mix = [&h](const void *p, size_t bytes) {
      const unsigned char *c = static_cast<const unsigned char *>(p);
      for (size_t i = 0; i < bytes; ++i) {
        h ^= c[i];
        h *= 1099511628211ull;
      }
    };
    mix(&parent, sizeof parent);
    mix(tokens, sizeof(int32_t) * (size_t)n);
    return h;
  }
  // the cached block with exactly this parent entry and these token ids, or -1
  int32_t lookup(int64_t parent, const int32_t *tokens) const {
    auto it = by_hash.find(hash_key(parent, tokens, block_size));
    if (it == by_hash.end()) return -1;
    for (int32_t b : it->second)
      if (parent_entry[b] == parent &&
          std::memcmp(&key_tokens[(size_t)b * block_size], tokens, sizeof(int32_t) * block_size) == 0)
        return b;
    return -1;
  }
  void remember(int32_t b, int64_t parent, const int32_t *tokens) {
    entry[b] = next_entry++;
    parent_entry[b] = parent;
    key_hash[b] = hash_key(parent, tokens, block_size);
    std::memcpy(&key_tokens[(size_t)b * block_size], tokens, sizeof(int32_t) * block_size);
    by_hash[key_hash[b]].push_back(b);
  }
  void forget(int32_t b) {
    auto it = by_hash.find(key_hash[b]);
    if (it != by_hash.end()) {
      auto &v = it->second;
      v.erase(std::find(v.begin(), v.end(), b));
      if (v.empty()) by_hash.erase(it);
    }
    entry[b] = -1;
  }
  // new blocks for `count` tokens, appended to `table`
  void fill(std::vector<int32_t> &table, int32_t count) {
    while (count > 0) {
      const int32_t b = take();
      ref_count[b] = 1;
      num_tokens[b] = std::min(block_size, count);
      count -= num_tokens[b];
      table.push_back(b);
    }
  }
  int32_t blocks_for(int32_t tokens) const { return (tokens + block_size - 1) / block_size; }
};

extern "C" {

pa_block_manager_t *pa_bm_create(int32_t num_blocks, int32_t block_size) {
  if (num_blocks < 0 || block_size <= 0) return nullptr;
  pa_block_manager_t *bm = new (std::nothrow) pa_block_manager_t();
  if (!bm) return nullptr;
  try {
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->ref_count.assign(num_blocks, 0);
    bm->num_tokens.assign(num_blocks, 0);
    for (int32_t b = 0; b < num_blocks; ++b) bm->free_list.push_back(b);
  } catch (...) {
    delete bm;
    return nullptr;
  }
  return bm;
}

void pa_bm_destroy(pa_block_manager_t *bm) { delete bm; }

pa_bm_status_t pa_bm_allocate(pa_block_manager_t *bm, int64_t seq, int32_t num_tokens, int64_t *slots) {
  if (!bm || num_tokens < 0) return PA_BM_BAD_ARG;
  if (bm->seqs.count(seq)) return PA_BM_EXISTS;
  if (bm->blocks_for(num_tokens) > bm->available()) return PA_BM_NO_SPACE;
  pa_block_manager::Seq &s = bm->seqs[seq];
  bm->fill(s.table, num_tokens);
  s.len = num_tokens;
  if (slots)
    for (int32_t p = 0; p < num_tokens; ++p) slots[p] = bm->slot(s, p);
  return PA_BM_OK;
}

pa_bm_status_t pa_bm_share_prefix(pa_block_manager_t *bm, int64_t seq, int64_t src, int32_t num_tokens,
                                  int64_t *unshared_slots, int32_t *num_unshared) {
  if (!bm || num_tokens < 0) return PA_BM_BAD_ARG;
  if (bm->seqs.count(seq)) return PA_BM_EXISTS;
  auto it = bm->seqs.find(src);
  if (it == bm->seqs.end()) return PA_BM_UNKNOWN_SEQ;
  const pa_block_manager::Seq &from = it->second;
  if (num_tokens > from.len) return PA_BM_BAD_ARG;
  // share src's blocks while the tokens they hold fit in the prefix
  size_t shared = 0;
  int32_t covered = 0;
  for (; shared < from.table.size(); ++shared) {
    const int32_t held = std::min(bm->block_size, from.len - covered);
    if (covered + held > num_tokens) break;
    covered += held;
  }
  if (bm->blocks_for(num_tokens - covered) > bm->available()) return PA_BM_NO_SPACE;
  std::vector<int32_t> table(from.table.begin(), from.table.begin() + shared);
  for (int32_t b : table) ++bm->ref_count[b];
  bm->fill(table, num_tokens - covered);
  pa_block_manager::Seq &s = bm->seqs[seq];
  s.table = std::move(table);
  s.len = num_tokens;
  if (unshared_slots)
    for (int32_t p = covered; p < num_tokens; ++p) unshared_slots[p - covered] = bm->slot(s, p);
  if (num_unshared) *num_unshared = num_tokens - covered;
  return PA_BM_OK;
}

pa_bm_status_t pa_bm_append(pa_block_manager_t *bm, int64_t seq, int64_t *slot, int64_t *cow_src,
                            int64_t *cow_dst) {
  if (!bm || !slot) return PA_BM_BAD_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_BM_UNKNOWN_SEQ;
  pa_block_manager::Seq &s = it->second;
  const int32_t offset = s.len % bm->block_size;
  int64_t src = -1, dst = -1;
  int32_t last;
  if (!s.table.empty() && offset != 0) {   // the last block has room
    last = s.table.back();
    if (bm->ref_count[last] > 1) {          // shared: the writer gets its own copy
      if (bm->available() == 0) return PA_BM_NO_SPACE;
      const int32_t fresh = bm->take();
      --bm->ref_count[last];
      bm->ref_count[fresh] = 1;
      bm->num_tokens[fresh] = offset;
      s.table.back() = fresh;
      src = last;
      dst = fresh;
      last = fresh;
    }
    bm->num_tokens[last] = offset + 1;
  } else {                                  // a new block for the token
    if (bm->available() == 0) return PA_BM_NO_SPACE;
    last = bm->take();
    bm->ref_count[last] = 1;
    bm->num_tokens[last] = 1;
    s.table.push_back(last);
  }
  ++s.len;
  *slot = (int64_t)last * bm->block_size + offset;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_BM_OK;
}

pa_bm_status_t pa_bm_append_batch(pa_block_manager_t *bm, const int64_t *seqs, int32_t n, int64_t *slots,
                                  int64_t *cow_pairs, int32_t *num_pairs, int32_t *num_done) {
  if (!bm || n < 0 || (n > 0 && (!seqs || !slots || !cow_pairs))) return PA_BM_BAD_ARG;
  int32_t pairs = 0, done = 0;
  pa_bm_status_t st = PA_BM_OK;
  for (; done < n; ++done) {
    int64_t src, dst;
    st = pa_bm_append(bm, seqs[done], &slots[done], &src, &dst);
    if (st != PA_BM_OK) break;
    if (src >= 0) {
      cow_pairs[2 * pairs] = src;
      cow_pairs[2 * pairs + 1] = dst;
      ++pairs;
    }
  }
  if (num_pairs) *num_pairs = pairs;
  if (num_done) *num_done = done;
  return st;
}

pa_bm_status_t pa_bm_free(pa_block_manager_t *bm, int64_t seq) {
  if (!bm) return PA_BM_BAD_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_BM_UNKNOWN_SEQ;
  const std::vector<int32_t> &t = it->second.table;
  if (!bm->caching) {
    for (int32_t b : t)
      if (--bm->ref_count[b] == 0) {
        bm->num_tokens[b] = 0;
        bm->free_list.push_back(b);
      }
  } else {
    // last to first, so that a prefix outlives its suffixes among the evictable blocks
    for (auto r = t.rbegin(); r != t.rend(); ++r) {
      const int32_t b = *r;
      if (--bm->ref_count[b] != 0) continue;
      if (bm->entry[b] >= 0) {   // cached: content kept for a later prompt
        bm->evict_pos[b] = bm->evictable.insert(bm->evictable.end(), b);
        bm->is_evictable[b] = 1;
      } else {
        bm->num_tokens[b] = 0;
        bm->free_list.push_back(b);
      }
    }
  }
  bm->seqs.erase(it);
  return PA_BM_OK;
}

pa_bm_status_t pa_bm_block_tables(const pa_block_manager_t *bm, const int64_t *seqs, int32_t n, int32_t *tables,
                                  int32_t max_blocks_per_seq, int32_t *context_lens) {
  if (!bm || n < 0 || max_blocks_per_seq < 0 || (n > 0 && (!seqs || (max_blocks_per_seq > 0 && !tables))))
    return PA_BM_BAD_ARG;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PA_BM_UNKNOWN_SEQ;
    if ((int64_t)it->second.table.size() > max_blocks_per_seq) return PA_BM_TABLE_FULL;
  }
  for (int32_t i = 0; i < n; ++i) {
    const pa_block_manager::Seq &s = bm->seqs.find(seqs[i])->second;
    int32_t *row = tables + (size_t)i * max_blocks_per_seq;
    std::copy(s.table.begin(), s.table.end(), row);
    std::fill(row + s.table.size(), row + max_blocks_per_seq, -1);
    if (context_lens) context_lens[i] = s.len;
  }
  return PA_BM_OK;
}

int32_t pa_bm_context_len(const pa_block_manager_t *bm, int64_t seq) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq);
  return it == bm->seqs.end() ? -1 : it->second.len;
}

int32_t pa_bm_ref_count(const pa_block_manager_t *bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->ref_count[block];
}

int32_t pa_bm_free_list(const pa_block_manager_t *bm, int32_t *out, int32_t cap) {
  if (!bm) return -1;
  int32_t i = 0;
  for (int32_t b : bm->free_list) {
    if (out && i < cap) out[i] = b;
    ++i;
  }
  return i;
}

int32_t pa_bm_sequences(const pa_block_manager_t *bm, int64_t *out, int32_t cap) {
  if (!bm) return -1;
  int32_t i = 0;
  for (const auto &kv : bm->seqs) {
    if (out && i < cap) out[i] = kv.first;
    ++i;
  }
  return i;
}

int32_t pa_bm_table(const pa_block_manager_t *bm, int64_t seq, int32_t *out, int32_t cap) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return -1;
  const int32_t n = (int32_t)it->second.table.size();
  for (int32_t i = 0; i < n && i < cap; ++i) out[i] = it->second.table[i];
  return n;
}

void pa_bm_stats(const pa_block_manager_t *bm, pa_bm_stats_t *out) {
  if (!bm || !out) return;
  pa_bm_stats_t s{};
  s.total_blocks = bm->num_blocks;
  s.free_blocks = (int64_t)bm->free_list.size();
  for (int32_t b = 0; b < bm->num_blocks; ++b)
    if (bm->ref_count[b] > 0) {
      ++s.used_blocks;
      s.used_tokens += bm->num_tokens[b];
    }
  for (const auto &kv : bm->seqs) s.logical_tokens += kv.second.len;
  s.num_sequences = (int64_t)bm->seqs.size();
  *out = s;
}

pa_block_manager_t *pa_bm_create_prefix_caching(int32_t num_blocks, int32_t block_size) {
  pa_block_manager_t *bm = pa_bm_create(num_blocks, block_size);
  if (!bm) return nullptr;
  try {
    bm->caching = true;
    bm->evict_pos.resize(num_blocks);
    bm->is_evictable.assign(num_blocks, 0);
    bm->entry.assign(num_blocks, -1);
    bm->parent_entry.assign(num_blocks, -1);
    bm->key_hash.assign(num_blocks, 0);
    bm->key_tokens.assign((size_t)num_blocks * block_size, 0);
  } catch (...) {
    delete bm;
    return nullptr;
  }
  return bm;
}

pa_bm_status_t pa_bm_allocate_prompt(pa_block_manager_t *bm, int64_t seq, const int32_t *token_ids,
                                     int32_t num_tokens, int64_t *slots, int32_t *num_cached_tokens) {
  if (!bm || num_tokens < 0 || (num_tokens > 0 && !token_ids)) return PA_BM_BAD_ARG;
  if (!bm->caching) {
    const pa_bm_status_t st = pa_bm_allocate(bm, seq, num_tokens, slots);
    if (st == PA_BM_OK && num_cached_tokens) *num_cached_tokens = 0;
    return st;
  }
  if (bm->seqs.count(seq)) return PA_BM_EXISTS;
  const int32_t bs = bm->block_size;
  const int32_t full = num_tokens / bs;
  // the longest run of leading full blocks that is cached
  std::vector<int32_t> hits;
  int64_t parent = -1;
  for (int32_t i = 0; i < full; ++i) {
    const int32_t b = bm->lookup(parent, token_ids + (size_t)i * bs);
    if (b < 0) break;
    hits.push_back(b);
    parent = bm->entry[b];
  }
  int64_t revived = 0;
  for (int32_t b : hits) revived += bm->ref_count[b] == 0;
  const int64_t need = bm->blocks_for(num_tokens) - (int64_t)hits.size();
  if (need > bm->available() - revived) return PA_BM_NO_SPACE;
  bm->queried += full;
  bm->hit += (int64_t)hits.size();
  for (int32_t b : hits) {
    if (bm->ref_count[b] == 0) {   // taken back from the evictable blocks
      bm->evictable.erase(bm->evict_pos[b]);
      bm->is_evictable[b] = 0;
    }
    ++bm->ref_count[b];
  }
  pa_block_manager::Seq &s = bm->seqs[seq];
  s.table = hits;
  int32_t left = num_tokens - (int32_t)hits.size() * bs;
  for (int32_t i = (int32_t)hits.size(); i < bm->blocks_for(num_tokens); ++i) {
    const int32_t b = bm->take();
    bm->ref_count[b] = 1;
    bm->num_tokens[b] = std::min(bs, left);
    left -= bm->num_tokens[b];
    s.table.push_back(b);
    if (i < full) {   // a full prompt block: cached under its parent entry and its token ids
      bm->remember(b, parent, token_ids + (size_t)i * bs);
      parent = bm->entry[b];
    }
  }
  s.len = num_tokens;
  if (slots)
    for (int32_t p = 0; p < num_tokens; ++p) slots[p] = bm->slot(s, p);
  if (num_cached_tokens) *num_cached_tokens = (int32_t)hits.size() * bs;
  return PA_BM_OK;
}

int32_t pa_bm_evictable(const pa_block_manager_t *bm, int32_t *out, int32_t cap) {
  if (!bm) return -1;
  int32_t i = 0;
  for (int32_t b : bm->evictable) {
    if (out && i < cap) out[i] = b;
    ++i;
  }
  return i;
}

int32_t pa_bm_cache_entry(const pa_block_manager_t *bm, int32_t block, int64_t *entry, int64_t *parent_entry) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  if (!bm->caching || bm->entry[block] < 0) return 0;
  if (entry) *entry = bm->entry[block];
  if (parent_entry) *parent_entry = bm->parent_entry[block];
  return 1;
}

void pa_bm_prefix_stats(const pa_block_manager_t *bm, pa_bm_prefix_stats_t *out) {
  if (!bm || !out) return;
  pa_bm_prefix_stats_t s{};
  s.queried_blocks = bm->queried;
  s.hit_blocks = bm->hit;
  if (bm->caching)
    for (int32_t b = 0; b < bm->num_blocks; ++b) s.cached_blocks += bm->entry[b] >= 0;
  s.evictable_blocks = (int64_t)bm->evictable.size();
  s.evictions = bm->evictions;
  *out = s;
}

}  // extern "C"
