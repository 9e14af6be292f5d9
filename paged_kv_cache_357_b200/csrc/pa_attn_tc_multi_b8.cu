// Multi-query paged attention on tensor cores at blocks of 8 tokens: the
// kMulti and kMultiTiled instances of the kernel in pa_attn_tc.cuh (see
// pa_attn_tc_multi.cu for the block-16 instances and the dispatch).
#include "pa_attn_tc.cuh"

namespace pa {

bool select_tc_multi_b8(bool bf16, int group, int rg, bool tiled, Variant& v) {
  return bf16 ? tc::pick_multi<true, 8>(group, rg, tiled, v) : tc::pick_multi<false, 8>(group, rg, tiled, v);
}

}  // namespace pa
