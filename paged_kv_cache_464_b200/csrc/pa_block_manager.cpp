// pa_block_manager.cpp -- host-side paged KV block manager (include/pa_block_manager.h).
//
// Block pool with a FIFO free list, per-sequence block tables, reference
// counts and copy-on-write, after PagedAttentionManager in "vLLM推理引擎深度解析"
// §三 and the block manager of "vLLM 原理与源码阅读" (Block 管理器).  Every
// operation checks that it can complete before it changes anything.
#include "pa_block_manager.h"

#include <algorithm>
#include <deque>
#include <map>
#include <new>
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

  int64_t slot(const Seq &s, int32_t pos) const {
    return (int64_t)s.table[pos / block_size] * block_size + pos % block_size;
  }
  int32_t take() {
    const int32_t b = free_list.front();
    free_list.pop_front();
    return b;
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
  if (bm->blocks_for(num_tokens) > (int64_t)bm->free_list.size()) return PA_BM_NO_SPACE;
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
  if (bm->blocks_for(num_tokens - covered) > (int64_t)bm->free_list.size()) return PA_BM_NO_SPACE;
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
      if (bm->free_list.empty()) return PA_BM_NO_SPACE;
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
    if (bm->free_list.empty()) return PA_BM_NO_SPACE;
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
  for (int32_t b : it->second.table) {
    if (--bm->ref_count[b] == 0) {
      bm->num_tokens[b] = 0;
      bm->free_list.push_back(b);
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

}  // extern "C"
