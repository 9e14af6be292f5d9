// Tensor-core decode at blocks of 8 and 32 tokens: the kDecode instances of
// the kernel in pa_attn_tc.cuh for groups of 1, 2, 4 or 8 query heads per
// kv head (head_dim 128).  A chunk stays 128 tokens (16 or 4 blocks); the
// block-size trade-off (study notes ch.05 §7: smaller blocks waste less of
// the last block, larger ones cost fewer table lookups and larger copies)
// is the caller's choice, and every choice streams through the same
// pipeline.
#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

template <bool kBf16, int B>
static bool pick_decode_block(int G, Variant& v) {
  switch (G) {
    case 1: v = tc_variant<kBf16, 1, 1, kDecode, B>(); return true;
    case 2: v = tc_variant<kBf16, 2, 1, kDecode, B>(); return true;
    case 4: v = tc_variant<kBf16, 4, 1, kDecode, B>(); return true;
    case 8: v = tc_variant<kBf16, 8, 1, kDecode, B>(); return true;
    default: return false;
  }
}

}  // namespace tc

bool select_tc_decode_other_block(int block_size, bool bf16, int group, Variant& v) {
  switch (block_size) {
    case 8: return bf16 ? tc::pick_decode_block<true, 8>(group, v) : tc::pick_decode_block<false, 8>(group, v);
    case 32: return bf16 ? tc::pick_decode_block<true, 32>(group, v) : tc::pick_decode_block<false, 32>(group, v);
    default: return false;
  }
}

}  // namespace pa
