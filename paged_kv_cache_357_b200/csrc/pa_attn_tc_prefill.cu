// Query-major multi-query tiles (prefill chunks) on tensor cores: the
// instances at blocks of 16 tokens and the dispatch (blocks of 8 and 32:
// pa_attn_tc_prefill_b8.cu, pa_attn_tc_prefill_b32.cu).  The kernel is in
// pa_attn_tc_prefill.cuh.
#include "pa_attn_tc_prefill.cuh"

namespace pa {

bool select_tc_prefill_variant(const pa_pool_desc& pool, int group, int q_len, Variant& v, int& tiles) {
  if (pool.head_dim != tc::D || (pool.dtype != PA_BF16 && pool.dtype != PA_FP16)) return false;
  if (group <= 0 || tc::pf::kRows % group != 0 || q_len * group < tc::pf::kRows) return false;
  const int positions = tc::pf::kRows / group;
  tiles = (q_len + positions - 1) / positions;
  const bool bf16 = pool.dtype == PA_BF16;
  switch (pool.block_size) {
    case 16: return bf16 ? tc::pf::pick<true, 16>(group, v) : tc::pf::pick<false, 16>(group, v);
    case 8: return select_tc_prefill_b8(bf16, group, v);
    case 32: return select_tc_prefill_b32(bf16, group, v);
    default: return false;
  }
}

}  // namespace pa
