// Tensor-core decode (one query row per head): the kDecode instances of the
// kernel in pa_attn_tc.cuh, for groups of 1, 2, 4 or 8 query heads per kv
// head (head_dim 128, block 16).  Even at one
// row per kv head, where the products are one real column of 16, its
// pipeline streams K/V faster than the CUDA-core kernel (B200: 781.9 against
// 838.3 µs on an 8 x 32k-token MHA layer).
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
  if (!tc::tc_pool_ok(pool)) return false;
  return pool.dtype == PA_BF16 ? tc::pick_decode<true>(group, v) : tc::pick_decode<false>(group, v);
}

}  // namespace pa
