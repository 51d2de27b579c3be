// Host-side paged KV block manager (C ABI in include/pagedkv.h).
//
// Keeps the physical block pool's free list and reference counts and each
// sequence's block table, and turns the serving loop's decisions (add a prompt,
// fork a sample, append one token per running sequence, free, swap out / in)
// into the inputs the device kernels take: block tables and context lengths for
// paged_attn_decode, slot mappings for kv_cache_append, copy-on-write pairs for
// kv_block_copy, and block lists for kv_blocks_to_host / kv_blocks_from_host.
//
// Rules ("vLLM PagedAttention and continuous batching", section 4 allocator; "LLM
// Inference 8 - PagedAttention", section "PagedAttention의 동작 방식"; the paper
// digest's framework flowchart):
//   * blocks come from the front of a FIFO free list with reference count 1 and
//     return to its back when their count drops to 0;
//   * a sequence of n tokens holds ceil(n / B) blocks; an append takes a new block
//     only when the last one is full;
//   * an append into a last block shared with other sequences first copies it to a
//     fresh block (copy-on-write) and reports the (src, dst) pair;
//   * a batch of appends changes nothing if the pool cannot serve all of it.
#include <cstdint>
#include <deque>
#include <mutex>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pagedkv.h"

struct pkv_block_manager {
  struct Seq {
    int64_t tokens = 0;
    std::vector<int32_t> table;
  };
  struct Swapped {
    int64_t tokens = 0;
    int32_t blocks = 0;
  };
  int num_blocks = 0;
  int block_size = 0;
  std::deque<int32_t> free_list;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  std::unordered_map<int64_t, Swapped> swapped;
  std::mutex mu;

  int32_t take() {
    const int32_t b = free_list.front();
    free_list.pop_front();
    ref[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--ref[b] == 0) free_list.push_back(b);
  }
  // The partly filled last block an append of `s` writes into, or -1 when the
  // append starts a new block.
  int32_t write_block(const Seq& s) const {
    const int64_t j = s.tokens / block_size;
    return j == (int64_t)s.table.size() ? -1 : s.table[j];
  }
};

namespace {
using Lock = std::lock_guard<std::mutex>;
}

extern "C" {

pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  auto* bm = new (std::nothrow) pkv_block_manager();
  if (!bm) return nullptr;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  if (free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return nullptr;
      }
      seen[b] = 1;
      bm->free_list.push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
  }
  return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int pkv_bm_num_free(pkv_block_manager* bm) {
  if (!bm) return PKV_EINVAL;
  Lock lk(bm->mu);
  return (int)bm->free_list.size();
}

int pkv_bm_ref_count(pkv_block_manager* bm, int block) {
  if (!bm) return PKV_EINVAL;
  Lock lk(bm->mu);
  if (block < 0 || block >= bm->num_blocks) return PKV_EINVAL;
  return bm->ref[block];
}

int pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq, int num_tokens) {
  if (!bm || num_tokens < 0) return PKV_EINVAL;
  Lock lk(bm->mu);
  if (bm->seqs.count(seq) || bm->swapped.count(seq)) return PKV_ESEQ;
  const int64_t need = ((int64_t)num_tokens + bm->block_size - 1) / bm->block_size;
  if (need > (int64_t)bm->free_list.size()) return PKV_ENOMEM;
  pkv_block_manager::Seq s;
  s.tokens = num_tokens;
  for (int64_t i = 0; i < need; ++i) s.table.push_back(bm->take());
  bm->seqs.emplace(seq, std::move(s));
  return PKV_OK;
}

int pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child) {
  if (!bm) return PKV_EINVAL;
  Lock lk(bm->mu);
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end() || bm->seqs.count(child) || bm->swapped.count(child)) return PKV_ESEQ;
  pkv_block_manager::Seq s = it->second;
  for (int32_t b : s.table) ++bm->ref[b];
  bm->seqs.emplace(child, std::move(s));
  return PKV_OK;
}

int pkv_bm_append_tokens(pkv_block_manager* bm, const int64_t* seqs, int n, int64_t* slots, int64_t* cow_pairs,
                         int* num_pairs) {
  if (!bm || n < 0 || (n > 0 && (!seqs || !slots || !cow_pairs)) || !num_pairs) return PKV_EINVAL;
  Lock lk(bm->mu);
  *num_pairs = 0;
  // Free blocks the batch takes: one per sequence whose last block is full, plus
  // the copies of shared last blocks.  The writers of one shared block b are
  // served in order: each copies while b still has another holder, so k writers
  // of a block with r holders make min(k, r - 1) copies (when all r holders write,
  // the last one writes in place).
  std::unordered_set<int64_t> seen;
  std::unordered_map<int32_t, int64_t> writers;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end() || !seen.insert(seqs[i]).second) return PKV_ESEQ;
    const int32_t b = bm->write_block(it->second);
    if (b < 0)
      ++need;
    else if (bm->ref[b] > 1)
      ++writers[b];
  }
  for (const auto& kv : writers) {
    const int64_t holders = bm->ref[kv.first];
    need += kv.second < holders - 1 ? kv.second : holders - 1;
  }
  if (need > (int64_t)bm->free_list.size()) return PKV_ENOMEM;
  int pairs = 0;
  for (int i = 0; i < n; ++i) {
    auto& s = bm->seqs[seqs[i]];
    const int64_t pos = s.tokens;
    const int64_t j = pos / bm->block_size;
    if (j == (int64_t)s.table.size()) {
      s.table.push_back(bm->take());
    } else if (bm->ref[s.table[j]] > 1) {
      const int32_t old = s.table[j];
      const int32_t fresh = bm->take();
      bm->release(old);
      s.table[j] = fresh;
      cow_pairs[2 * pairs] = old;
      cow_pairs[2 * pairs + 1] = fresh;
      ++pairs;
    }
    slots[i] = (int64_t)s.table[j] * bm->block_size + pos % bm->block_size;
    s.tokens = pos + 1;
  }
  *num_pairs = pairs;
  return PKV_OK;
}

int pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq) {
  if (!bm) return PKV_EINVAL;
  Lock lk(bm->mu);
  if (bm->swapped.erase(seq)) return PKV_OK;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PKV_ESEQ;
  for (int32_t b : it->second.table) bm->release(b);
  bm->seqs.erase(it);
  return PKV_OK;
}

int pkv_bm_block_table(pkv_block_manager* bm, int64_t seq, int32_t* row, int max_blocks, int64_t* num_tokens) {
  if (!bm || max_blocks < 0 || (max_blocks > 0 && !row)) return PKV_EINVAL;
  Lock lk(bm->mu);
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PKV_ESEQ;
  const auto& s = it->second;
  if ((int64_t)s.table.size() > max_blocks) return PKV_EINVAL;
  for (int i = 0; i < max_blocks; ++i) row[i] = i < (int)s.table.size() ? s.table[i] : -1;
  if (num_tokens) *num_tokens = s.tokens;
  return (int)s.table.size();
}

int pkv_bm_fill_tables(pkv_block_manager* bm, const int64_t* seqs, int n, int32_t* block_tables, int max_blocks,
                       int32_t* context_lens) {
  if (!bm || n < 0 || max_blocks <= 0 || (n > 0 && (!seqs || !block_tables || !context_lens))) return PKV_EINVAL;
  Lock lk(bm->mu);
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PKV_ESEQ;
    const auto& s = it->second;
    if ((int64_t)s.table.size() > max_blocks || s.tokens > 0x7fffffff) return PKV_EINVAL;
    int32_t* row = block_tables + (size_t)i * max_blocks;
    for (int j = 0; j < max_blocks; ++j) row[j] = j < (int)s.table.size() ? s.table[j] : -1;
    context_lens[i] = (int32_t)s.tokens;
  }
  return PKV_OK;
}

int pkv_bm_swap_out(pkv_block_manager* bm, int64_t seq, int64_t* blocks, int max_blocks, int* n_blocks) {
  if (!bm || !n_blocks || max_blocks < 0 || (max_blocks > 0 && !blocks)) return PKV_EINVAL;
  Lock lk(bm->mu);
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PKV_ESEQ;
  const auto& s = it->second;
  if ((int64_t)s.table.size() > max_blocks) return PKV_EINVAL;
  for (size_t i = 0; i < s.table.size(); ++i) blocks[i] = s.table[i];
  *n_blocks = (int)s.table.size();
  for (int32_t b : s.table) bm->release(b);
  bm->swapped[seq] = {s.tokens, (int32_t)s.table.size()};
  bm->seqs.erase(it);
  return PKV_OK;
}

int pkv_bm_swap_in(pkv_block_manager* bm, int64_t seq, int64_t* blocks, int max_blocks, int* n_blocks) {
  if (!bm || !n_blocks || max_blocks < 0 || (max_blocks > 0 && !blocks)) return PKV_EINVAL;
  Lock lk(bm->mu);
  auto it = bm->swapped.find(seq);
  if (it == bm->swapped.end()) return PKV_ESEQ;
  const int32_t n = it->second.blocks;
  if (n > max_blocks) return PKV_EINVAL;
  if (n > (int64_t)bm->free_list.size()) return PKV_ENOMEM;
  pkv_block_manager::Seq s;
  s.tokens = it->second.tokens;
  for (int32_t i = 0; i < n; ++i) {
    s.table.push_back(bm->take());
    blocks[i] = s.table.back();
  }
  *n_blocks = n;
  bm->swapped.erase(it);
  bm->seqs.emplace(seq, std::move(s));
  return PKV_OK;
}

}  // extern "C"
