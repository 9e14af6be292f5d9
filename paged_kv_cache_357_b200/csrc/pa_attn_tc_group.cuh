// Shared-prefix decode on tensor cores: the kGroup instances of the kernel in
// pa_attn_tc.cuh at blocks of B tokens, one per (G, RG) the dispatch can ask
// for.  A unit is (group, kv head): it streams the group's shared leading
// blocks once for the G query heads of every member (up to RG members,
// G * RG <= 32 rows), then each member's own blocks for that member's rows,
// and writes every member's outputs.
#pragma once

#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

template <bool kBf16, int B>
bool pick_group(int G, int RG, Variant& v) {
#define PA_GROUP_CASE(g, rg)                        \
  if (G == g && RG == rg) {                          \
    v = tc_variant<kBf16, g, rg, kGroup, B>();      \
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
}  // namespace pa
