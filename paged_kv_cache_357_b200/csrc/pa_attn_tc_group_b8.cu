// Shared-prefix decode on tensor cores at blocks of 8 tokens: the kGroup
// instances of the kernel in pa_attn_tc.cuh (the dispatch is in
// pa_attn_tc_group.cu).
#include "pa_attn_tc_group.cuh"

namespace pa {

bool select_tc_group_b8(bool bf16, int group, int rg, Variant& v) {
  return bf16 ? tc::pick_group<true, 8>(group, rg, v) : tc::pick_group<false, 8>(group, rg, v);
}

}  // namespace pa
