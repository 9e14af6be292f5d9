// Tensor-core decode (one query row per head): the kDecode instances of the
// kernel in pa_attn_tc.cuh.  Used for plain decode where a GQA group of 4 or
// 8 query heads shares each kv head, and for the second pass of the
// shared-prefix decode (groups of 1, 2, 4 or 8), which reads only each
// sequence's own blocks and merges the result with the shared prefix's state.
#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

template <bool kBf16>
static bool pick_decode(int G, Variant& v) {
  switch (G) {
    case 1: v = tc_variant<kBf16, 1, 1, kDecode>(); return true;
    case 2: v = tc_variant<kBf16, 2, 1, kDecode>(); return true;
    case 4: v = tc_variant<kBf16, 4, 1, kDecode>(); return true;
    case 8: v = tc_variant<kBf16, 8, 1, kDecode>(); return true;
    default: return false;
  }
}

}  // namespace tc

bool select_tc_variant(const pa_pool_desc& pool, int group, Variant& v) {
  if (!tc::tc_pool_ok(pool) || (group != 4 && group != 8)) return false;
  return pool.dtype == PA_BF16 ? tc::pick_decode<true>(group, v) : tc::pick_decode<false>(group, v);
}

bool select_tc_suffix_variant(const pa_pool_desc& pool, int group, Variant& v) {
  if (!tc::tc_pool_ok(pool)) return false;
  return pool.dtype == PA_BF16 ? tc::pick_decode<true>(group, v) : tc::pick_decode<false>(group, v);
}

}  // namespace pa
