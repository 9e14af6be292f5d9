// Query-major multi-query tiles (prefill chunks) on tensor cores at blocks
// of 8 tokens: the instances of the kernel in pa_attn_tc_prefill.cuh (the
// dispatch is in pa_attn_tc_prefill.cu).
#include "pa_attn_tc_prefill.cuh"

namespace pa {

bool select_tc_prefill_b8(bool bf16, int group, Variant& v) {
  return bf16 ? tc::pf::pick<true, 8>(group, v) : tc::pf::pick<false, 8>(group, v);
}

}  // namespace pa
