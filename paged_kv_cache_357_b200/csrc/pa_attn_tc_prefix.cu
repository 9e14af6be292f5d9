// Shared-prefix decode, first pass, on tensor cores: the kPrefix instances of
// the kernel in pa_attn_tc.cuh.  A unit is (group, kv head): the group's
// shared leading blocks are read once for the G query heads of every member
// (up to RG members, G * RG <= 32 rows), and each member row's online-softmax
// state is stored for the second pass (pa_decode_tc.cu).
#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

template <bool kBf16>
static bool pick_prefix(int G, int RG, Variant& v) {
#define PA_PREFIX_CASE(g, rg)                        \
  if (G == g && RG == rg) {                          \
    v = tc_variant<kBf16, g, rg, kPrefix>();         \
    return true;                                     \
  }
  PA_PREFIX_CASE(1, 1) PA_PREFIX_CASE(1, 2) PA_PREFIX_CASE(1, 4) PA_PREFIX_CASE(1, 8) PA_PREFIX_CASE(1, 16)
  PA_PREFIX_CASE(1, 32)
  PA_PREFIX_CASE(2, 1) PA_PREFIX_CASE(2, 2) PA_PREFIX_CASE(2, 4) PA_PREFIX_CASE(2, 8) PA_PREFIX_CASE(2, 16)
  PA_PREFIX_CASE(4, 1) PA_PREFIX_CASE(4, 2) PA_PREFIX_CASE(4, 4) PA_PREFIX_CASE(4, 8)
  PA_PREFIX_CASE(8, 1) PA_PREFIX_CASE(8, 2) PA_PREFIX_CASE(8, 4)
#undef PA_PREFIX_CASE
  return false;
}

}  // namespace tc

bool select_tc_prefix_variant(const pa_pool_desc& pool, int group, int max_members, Variant& v) {
  if (!tc::tc_pool_ok(pool)) return false;
  const int rg = tc::row_groups_for(group, max_members);
  if (rg == 0) return false;
  return pool.dtype == PA_BF16 ? tc::pick_prefix<true>(group, rg, v) : tc::pick_prefix<false>(group, rg, v);
}

}  // namespace pa
