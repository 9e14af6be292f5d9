// Host block manager of the paged KV cache (C++, no GPU code).
//
// The bookkeeping half of the method (PagedAttention study notes ch.05):
//   §3   each sequence has a block table, logical block j -> physical block;
//   §5 ② on-demand allocation: a token goes to the next free row after the
//        filled blocks, and a new physical block is taken only when the last
//        one is full, so a sequence wastes less than one block;
//   §6.1 outputs of one prompt share its blocks; a writer to a shared block
//        copies it first (copy on write) and repoints its own table;
//   §6.2 reference counts: dropping a sequence releases one reference per
//        block, and blocks at zero return to the free set;
//   §12 exercise 4: block 7 shared by 4 outputs, the writer copies it to 7',
//        ref counts go 4 -> 3 and 1.
// The free set is first-in first-out (lowest ids first at start), so the
// manager hands out the same blocks as the float64 test oracle's manager.
// Not thread safe: callers serialise access to one manager.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_block_manager {
  struct Seq {
    std::vector<int32_t> blocks;
    int32_t tokens = 0;
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> ref;
  std::deque<int32_t> free_list;
  std::unordered_map<int64_t, Seq> seqs;

  int32_t take() {
    const int32_t b = free_list.front();
    free_list.pop_front();
    ref[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--ref[b] == 0) free_list.push_back(b);
  }
  int32_t blocks_for(int64_t tokens) const { return static_cast<int32_t>((tokens + block_size - 1) / block_size); }
};

namespace {

// What appending one token to `s` needs: 0 (room in an exclusive block), or 1
// block (a new last block, or a copy of a shared one).  `shared_writes`
// counts earlier copies out of the same block within one batch.
int32_t blocks_needed_for_append(const pa_block_manager& bm, const pa_block_manager::Seq& s,
                                 std::unordered_map<int32_t, int32_t>& pending_ref) {
  const int32_t j = s.tokens / bm.block_size;
  if (j == static_cast<int32_t>(s.blocks.size())) return 1;
  const int32_t b = s.blocks[j];
  auto it = pending_ref.find(b);
  int32_t r = (it == pending_ref.end()) ? bm.ref[b] : it->second;
  if (r > 1) {
    pending_ref[b] = r - 1;
    return 1;
  }
  return 0;
}

pa_status append_one(pa_block_manager& bm, pa_block_manager::Seq& s, int64_t* slot, int64_t* cow_src,
                     int64_t* cow_dst) {
  const int32_t j = s.tokens / bm.block_size;
  const int32_t row = s.tokens % bm.block_size;
  int64_t src = -1, dst = -1;
  if (j == static_cast<int32_t>(s.blocks.size())) {
    if (bm.free_list.empty()) return PA_ERR_OUT_OF_BLOCKS;
    s.blocks.push_back(bm.take());
  } else {
    const int32_t b = s.blocks[j];
    if (bm.ref[b] > 1) {
      if (bm.free_list.empty()) return PA_ERR_OUT_OF_BLOCKS;
      const int32_t nb = bm.take();
      bm.ref[b] -= 1;
      s.blocks[j] = nb;
      src = b;
      dst = nb;
    }
  }
  s.tokens += 1;
  if (slot) *slot = static_cast<int64_t>(s.blocks[j]) * bm.block_size + row;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_OK;
}

}  // namespace

extern "C" pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pa_block_manager* bm = new (std::nothrow) pa_block_manager();
  if (bm == nullptr) return nullptr;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  for (int32_t b = 0; b < num_blocks; ++b) bm->free_list.push_back(b);
  return bm;
}

extern "C" void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

extern "C" pa_status pa_bm_add(pa_block_manager* bm, int64_t seq_id, int32_t num_tokens) {
  if (bm == nullptr || num_tokens < 0 || bm->seqs.count(seq_id) != 0) return PA_ERR_INVALID_ARG;
  const int32_t need = bm->blocks_for(num_tokens);
  if (need > static_cast<int32_t>(bm->free_list.size())) return PA_ERR_OUT_OF_BLOCKS;
  pa_block_manager::Seq s;
  s.tokens = num_tokens;
  s.blocks.reserve(need);
  for (int32_t i = 0; i < need; ++i) s.blocks.push_back(bm->take());
  bm->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

extern "C" pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id) {
  if (bm == nullptr || bm->seqs.count(child_id) != 0) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
  pa_block_manager::Seq child = it->second;
  for (int32_t b : child.blocks) bm->ref[b] += 1;
  bm->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

extern "C" pa_status pa_bm_append(pa_block_manager* bm, int64_t seq_id, int64_t* slot, int64_t* cow_src,
                                  int64_t* cow_dst) {
  if (bm == nullptr) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
  return append_one(*bm, it->second, slot, cow_src, cow_dst);
}

extern "C" pa_status pa_bm_free(pa_block_manager* bm, int64_t seq_id) {
  if (bm == nullptr) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
  for (int32_t b : it->second.blocks) bm->release(b);
  bm->seqs.erase(it);
  return PA_OK;
}

extern "C" int32_t pa_bm_num_free_blocks(const pa_block_manager* bm) {
  return bm == nullptr ? -1 : static_cast<int32_t>(bm->free_list.size());
}

extern "C" int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block) {
  if (bm == nullptr || block < 0 || block >= bm->num_blocks) return -1;
  return bm->ref[block];
}

extern "C" pa_status pa_bm_table(const pa_block_manager* bm, int64_t seq_id, int32_t* blocks, int32_t capacity,
                                 int32_t* num_blocks, int32_t* num_tokens) {
  if (bm == nullptr || capacity < 0 || (capacity > 0 && blocks == nullptr)) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
  const auto& s = it->second;
  const int32_t n = static_cast<int32_t>(s.blocks.size());
  if (num_blocks) *num_blocks = n;
  if (num_tokens) *num_tokens = s.tokens;
  if (n > capacity) return PA_ERR_INVALID_ARG;
  std::copy(s.blocks.begin(), s.blocks.end(), blocks);
  return PA_OK;
}

extern "C" void pa_bm_get_stats(const pa_block_manager* bm, pa_bm_stats* out) {
  if (bm == nullptr || out == nullptr) return;
  pa_bm_stats st = {};
  st.num_blocks = bm->num_blocks;
  st.free_blocks = static_cast<int32_t>(bm->free_list.size());
  st.used_blocks = st.num_blocks - st.free_blocks;
  for (int32_t b = 0; b < bm->num_blocks; ++b) st.shared_blocks += bm->ref[b] > 1 ? 1 : 0;
  std::unordered_map<int32_t, int32_t> filled;  // physical block -> rows holding a token
  for (const auto& kv : bm->seqs) {
    const auto& s = kv.second;
    st.num_sequences += 1;
    st.logical_blocks += static_cast<int64_t>(s.blocks.size());
    st.tokens += s.tokens;
    for (size_t j = 0; j < s.blocks.size(); ++j) {
      const int32_t rows = std::min<int32_t>(bm->block_size, s.tokens - static_cast<int32_t>(j) * bm->block_size);
      int32_t& f = filled[s.blocks[j]];
      f = std::max(f, rows);
    }
  }
  for (const auto& kv : filled) st.slots_filled += kv.second;
  *out = st;
}

extern "C" pa_status pa_bm_prepare_step(pa_block_manager* bm, const int64_t* seq_ids, int32_t n,
                                        int32_t max_blocks_per_seq, int32_t* block_tables, int32_t* seq_lens,
                                        int64_t* slot_mapping, int64_t* copy_pairs, int32_t max_pairs,
                                        int32_t* num_pairs) {
  if (bm == nullptr || n < 0 || max_blocks_per_seq <= 0 || max_pairs < 0 || num_pairs == nullptr) {
    return PA_ERR_INVALID_ARG;
  }
  if (n > 0 && (seq_ids == nullptr || block_tables == nullptr || seq_lens == nullptr || slot_mapping == nullptr)) {
    return PA_ERR_INVALID_ARG;
  }
  // Check everything before changing anything: known distinct ids, table
  // width, free blocks and copy-pair room for the whole batch.
  std::vector<pa_block_manager::Seq*> seqs(n);
  std::unordered_map<int64_t, int> seen;
  std::unordered_map<int32_t, int32_t> pending_ref;
  int32_t need_blocks = 0, need_pairs = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || !seen.emplace(seq_ids[i], i).second) return PA_ERR_INVALID_ARG;
    seqs[i] = &it->second;
    if (bm->blocks_for(static_cast<int64_t>(seqs[i]->tokens) + 1) > max_blocks_per_seq) return PA_ERR_INVALID_ARG;
    const int32_t j = seqs[i]->tokens / bm->block_size;
    const bool fresh = j == static_cast<int32_t>(seqs[i]->blocks.size());
    const int32_t k = blocks_needed_for_append(*bm, *seqs[i], pending_ref);
    need_blocks += k;
    need_pairs += (k == 1 && !fresh) ? 1 : 0;
  }
  if (need_blocks > static_cast<int32_t>(bm->free_list.size())) return PA_ERR_OUT_OF_BLOCKS;
  if (need_pairs > max_pairs || (need_pairs > 0 && copy_pairs == nullptr)) return PA_ERR_INVALID_ARG;

  int32_t pairs = 0;
  for (int32_t i = 0; i < n; ++i) {
    int64_t src = -1, dst = -1;
    const pa_status st = append_one(*bm, *seqs[i], &slot_mapping[i], &src, &dst);
    if (st != PA_OK) return st;  // not reached: checked above
    if (src >= 0) {
      copy_pairs[2 * pairs] = src;
      copy_pairs[2 * pairs + 1] = dst;
      ++pairs;
    }
    const auto& s = *seqs[i];
    seq_lens[i] = s.tokens;
    int32_t* row = block_tables + static_cast<size_t>(i) * max_blocks_per_seq;
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    std::fill(row + s.blocks.size(), row + max_blocks_per_seq, -1);
  }
  *num_pairs = pairs;
  return PA_OK;
}

// ---- shared-prefix groups of one step's tables (host planning) --------------

extern "C" pa_status pa_shared_prefix_groups(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                             const int32_t* seq_lens, int32_t num_seqs, int32_t block_size,
                                             int32_t max_group_size, int32_t min_prefix_blocks,
                                             int32_t* group_starts, int32_t* group_prefix_blocks,
                                             int32_t* num_groups) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || max_group_size < 1 || num_groups == nullptr ||
      group_starts == nullptr || (num_seqs > 0 && (block_tables == nullptr || seq_lens == nullptr ||
                                                   group_prefix_blocks == nullptr))) {
    return PA_ERR_INVALID_ARG;
  }
  auto blocks_of = [&](int32_t s) -> int32_t {
    const int64_t n = seq_lens[s];
    if (n <= 0 || n > static_cast<int64_t>(max_blocks_per_seq) * block_size) return 0;
    return static_cast<int32_t>((n + block_size - 1) / block_size);
  };
  auto row = [&](int32_t s) { return block_tables + static_cast<size_t>(s) * max_blocks_per_seq; };
  int32_t g = 0;
  int32_t s = 0;
  while (s < num_seqs) {
    const int32_t first = s;
    const int32_t nb0 = blocks_of(first);
    int32_t prefix = nb0;  // common leading entries so far
    int32_t min_nb = nb0;
    int32_t end = first + 1;
    while (nb0 > 0 && end < num_seqs && end - first < max_group_size) {
      const int32_t nb = blocks_of(end);
      if (nb == 0 || row(end)[0] != row(first)[0]) break;
      int32_t c = 0;
      const int32_t lim = std::min(prefix, nb);
      while (c < lim && row(end)[c] == row(first)[c]) ++c;
      prefix = c;
      min_nb = std::min(min_nb, nb);
      ++end;
    }
    int32_t pb = std::min(prefix, min_nb - 1);
    if (end - first < 2 || pb < std::max(min_prefix_blocks, 1)) pb = 0;
    group_starts[g] = first;
    group_prefix_blocks[g] = pb;
    ++g;
    s = end;
  }
  group_starts[g] = num_seqs;
  *num_groups = g;
  return PA_OK;
}
