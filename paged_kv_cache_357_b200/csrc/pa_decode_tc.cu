// Tensor-core decode (one query row per head): the kDecode instances of the
// kernel in pa_attn_tc.cuh at block size 16, for groups of 1, 2, 4 or 8
// query heads per kv head (head_dim 128), and the dispatch over block
// sizes; blocks of 8 and 32 tokens are instantiated in
// pa_decode_tc_blocks.cu.  Even at one row per kv head, where the products
// are one real column of 16, its pipeline streams K/V faster than the
// CUDA-core kernel (B200: 781.9 against 838.3 µs on an 8 x 32k-token MHA
// layer).
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
  if (!tc::tc_pool_ok(pool, true)) return false;
  const bool bf16 = pool.dtype == PA_BF16;
  if (pool.block_size != 16) return select_tc_decode_other_block(pool.block_size, bf16, group, v);
  return bf16 ? tc::pick_decode<true>(group, v) : tc::pick_decode<false>(group, v);
}

}  // namespace pa
