// Shared-prefix decode on tensor cores: the kGroup instances of the kernel in
// pa_attn_tc.cuh.  A unit is (group, kv head): it streams the group's shared
// leading blocks once for the G query heads of every member (up to RG
// members, G * RG <= 32 rows), then each member's own blocks for that
// member's rows, and writes every member's outputs.
#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

template <bool kBf16>
static bool pick_group(int G, int RG, Variant& v) {
#define PA_GROUP_CASE(g, rg)                        \
  if (G == g && RG == rg) {                          \
    v = tc_variant<kBf16, g, rg, kGroup>();         \
    return true;                                     \
  }
  PA_GROUP_CASE(1, 1) PA_GROUP_CASE(1, 2) PA_GROUP_CASE(1, 4) PA_GROUP_CASE(1, 8) PA_GROUP_CASE(1, 16)
  PA_GROUP_CASE(1, 32)
  PA_GROUP_CASE(2, 1) PA_GROUP_CASE(2, 2) PA_GROUP_CASE(2, 4) PA_GROUP_CASE(2, 8) PA_GROUP_CASE(2, 16)
  PA_GROUP_CASE(4, 1) PA_GROUP_CASE(4, 2) PA_GROUP_CASE(4, 4) PA_GROUP_CASE(4, 8)
  PA_GROUP_CASE(8, 1) PA_GROUP_CASE(8, 2) PA_GROUP_CASE(8, 4)
#undef PA_GROUP_CASE
  return false;
}

}  // namespace tc

bool select_tc_group_variant(const pa_pool_desc& pool, int group, int max_members, Variant& v) {
  if (!tc::tc_pool_ok(pool)) return false;
  // every member of a group sits in one unit: G x (members rounded up to a
  // power of two) must fit the 32 rows of a unit
  const int rg = tc::row_groups_for(group, max_members);
  if (rg == 0 || rg < max_members) return false;
  return pool.dtype == PA_BF16 ? tc::pick_group<true>(group, rg, v) : tc::pick_group<false>(group, rg, v);
}

}  // namespace pa
