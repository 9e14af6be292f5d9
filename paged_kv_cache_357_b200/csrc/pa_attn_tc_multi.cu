// Multi-query paged attention on tensor cores: the kMulti instances of the
// kernel in pa_attn_tc.cuh.  Each sequence brings q_len new query positions
// (q and out are [num_seqs][q_len][num_q_heads][head_dim]); position i sees
// the sequence's tokens up to seq_len - q_len + i.  A unit holds the G query
// heads of a kv head times RG positions, G * RG <= 32 rows: RG >= q_len
// when they fit, else several units (row tiles of RG = 32 / G positions)
// per sequence.  This unit holds the instances at blocks of 16 tokens and
// the dispatch; blocks of 8 and 32 are instantiated in
// pa_attn_tc_multi_b8.cu and pa_attn_tc_multi_b32.cu.  Once a sequence's
// rows fill a 128-row tile, the query-major kernel of
// pa_attn_tc_prefill.cu takes over.
#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {

}  // namespace tc

bool select_tc_multi_variant(const pa_pool_desc& pool, int group, int q_len, Variant& v, int& tiles) {
  if (!tc::tc_pool_ok(pool, true) || q_len < 2) return false;
  if (select_tc_prefill_variant(pool, group, q_len, v, tiles)) return true;
  const int rg = tc::row_groups_for(group, q_len);
  if (rg == 0) return false;
  tiles = tc::row_tiles_for(q_len, rg);
  const bool tiled = tiles > 1, bf16 = pool.dtype == PA_BF16;
  switch (pool.block_size) {
    case 16: return bf16 ? tc::pick_multi<true, 16>(group, rg, tiled, v) : tc::pick_multi<false, 16>(group, rg, tiled, v);
    case 8: return select_tc_multi_b8(bf16, group, rg, tiled, v);
    case 32: return select_tc_multi_b32(bf16, group, rg, tiled, v);
    default: return false;
  }
}

}  // namespace pa
