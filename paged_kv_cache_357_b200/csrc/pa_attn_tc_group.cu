// Shared-prefix decode on tensor cores: the instances at blocks of 16 tokens
// and the dispatch (blocks of 8 and 32: pa_attn_tc_group_b8.cu,
// pa_attn_tc_group_b32.cu).  See pa_attn_tc_group.cuh.
#include "pa_attn_tc_group.cuh"

namespace pa {

bool select_tc_group_variant(const pa_pool_desc& pool, int group, int max_members, Variant& v) {
  if (!tc::tc_pool_ok(pool, true)) return false;
  // every member of a group sits in one unit: G x (members rounded up to a
  // power of two) must fit the 32 rows of a unit
  const int rg = tc::row_groups_for(group, max_members);
  if (rg == 0 || rg < max_members) return false;
  const bool bf16 = pool.dtype == PA_BF16;
  switch (pool.block_size) {
    case 16: return bf16 ? tc::pick_group<true, 16>(group, rg, v) : tc::pick_group<false, 16>(group, rg, v);
    case 8: return select_tc_group_b8(bf16, group, rg, v);
    case 32: return select_tc_group_b32(bf16, group, rg, v);
    default: return false;
  }
}

}  // namespace pa
