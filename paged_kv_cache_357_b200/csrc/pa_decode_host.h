// Host-side description of a decode kernel variant, shared by the
// CUDA-core kernel (pa_decode.cu) and the tensor-core kernel
// (pa_decode_tc.cu).
#pragma once

#include <cuda_runtime.h>

#include "pa_decode_common.cuh"

namespace pa {

struct Variant;
using LaunchFn = cudaError_t (*)(const Variant& v, const DecodeParams& prm, int ctas, cudaStream_t stream);

struct Variant {
  const void* kernel;  // for occupancy queries and attributes
  int threads;
  int smem_bytes;
  int part_stride;  // floats per partial slot: query rows per unit * (D + 2)
  LaunchFn launch;
  int unit_cost;    // partition cost of finishing a unit (DecodeParams::unit_cost)
  bool fuses_update = false;  // tensor-core decode family: takes new tokens (DecodeParams::upd_*) into its launch and writes log normalisers (DecodeParams::lse)
};

// Tensor-core variants (pa_attn_tc.cuh), if one exists for this pool and
// shape.  `group` is the number of query heads per kv head.
// Plain decode (pa_decode_tc.cu): groups of 1, 2, 4 and 8, blocks of 8, 16
// or 32 tokens.
bool select_tc_variant(const pa_pool_desc& pool, int group, Variant& v);
// The plain decode's instances at blocks of 8 and 32 tokens
// (pa_decode_tc_blocks.cu).
bool select_tc_decode_other_block(int block_size, bool bf16, int group, Variant& v);
// Multi-query decode with q_len >= 2 positions (pa_attn_tc_multi.cu); tiles
// = units (row tiles) per sequence.
bool select_tc_multi_variant(const pa_pool_desc& pool, int group, int q_len, Variant& v, int& tiles);
// Its instances at blocks of 8 and 32 tokens (pa_attn_tc_multi_b8.cu,
// pa_attn_tc_multi_b32.cu): rg row groups a unit, tiled = several units a
// sequence.
bool select_tc_multi_b8(bool bf16, int group, int rg, bool tiled, Variant& v);
bool select_tc_multi_b32(bool bf16, int group, int rg, bool tiled, Variant& v);
// Query-major tiles of 128 rows (pa_attn_tc_prefill.cu) when a sequence's
// G x q_len rows fill at least one (blocks of 8, 16 or 32): tiles = units
// per sequence and kv head.  Its instances at blocks of 8 and 32 tokens:
// pa_attn_tc_prefill_b8.cu, pa_attn_tc_prefill_b32.cu.
bool select_tc_prefill_variant(const pa_pool_desc& pool, int group, int q_len, Variant& v, int& tiles);
bool select_tc_prefill_b8(bool bf16, int group, Variant& v);
bool select_tc_prefill_b32(bool bf16, int group, Variant& v);
// Shared-prefix decode over groups of up to max_members sequences
// (pa_attn_tc_group.cu).
bool select_tc_group_variant(const pa_pool_desc& pool, int group, int max_members, Variant& v);
// Its instances at blocks of 8 and 32 tokens (pa_attn_tc_group_b8.cu,
// pa_attn_tc_group_b32.cu), rg row groups (members) a unit.
bool select_tc_group_b8(bool bf16, int group, int rg, Variant& v);
bool select_tc_group_b32(bool bf16, int group, int rg, Variant& v);

}  // namespace pa
