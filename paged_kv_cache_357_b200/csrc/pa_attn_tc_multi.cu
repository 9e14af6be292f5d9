// Multi-query paged attention on tensor cores: the kMulti instances of the
// kernel in pa_attn_tc.cuh.  Each sequence brings q_len new query positions
// (q and out are [num_seqs][q_len][num_q_heads][head_dim]); position i sees
// the sequence's tokens up to seq_len - q_len + i.  A unit holds the G query
// heads of a kv head times RG positions, G * RG <= 32 rows: RG >= q_len
// when they fit, else several units (row tiles of RG = 32 / G positions)
// per sequence.
#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

template <bool kBf16>
static bool pick_multi(int G, int RG, bool tiled, Variant& v) {
#define PA_MULTI_CASE(g, rg)                         \
  if (G == g && RG == rg && !tiled) {                \
    v = tc_variant<kBf16, g, rg, kMulti>();          \
    return true;                                     \
  }
  PA_MULTI_CASE(1, 2) PA_MULTI_CASE(1, 4) PA_MULTI_CASE(1, 8) PA_MULTI_CASE(1, 16) PA_MULTI_CASE(1, 32)
  PA_MULTI_CASE(2, 2) PA_MULTI_CASE(2, 4) PA_MULTI_CASE(2, 8) PA_MULTI_CASE(2, 16)
  PA_MULTI_CASE(4, 2) PA_MULTI_CASE(4, 4) PA_MULTI_CASE(4, 8)
  PA_MULTI_CASE(8, 2) PA_MULTI_CASE(8, 4)
#undef PA_MULTI_CASE
  // row tiles: 32 rows a unit
#define PA_TILED_CASE(g, rg)                         \
  if (G == g && RG == rg && tiled) {                 \
    v = tc_variant<kBf16, g, rg, kMultiTiled>();     \
    return true;                                     \
  }
  PA_TILED_CASE(1, 32) PA_TILED_CASE(2, 16) PA_TILED_CASE(4, 8) PA_TILED_CASE(8, 4)
#undef PA_TILED_CASE
  return false;
}

}  // namespace tc

bool select_tc_multi_variant(const pa_pool_desc& pool, int group, int q_len, Variant& v, int& tiles) {
  if (!tc::tc_pool_ok(pool) || q_len < 2) return false;
  const int rg = tc::row_groups_for(group, q_len);
  if (rg == 0) return false;
  tiles = tc::row_tiles_for(q_len, rg);
  const bool tiled = tiles > 1;
  return pool.dtype == PA_BF16 ? tc::pick_multi<true>(group, rg, tiled, v)
                               : tc::pick_multi<false>(group, rg, tiled, v);
}

}  // namespace pa
