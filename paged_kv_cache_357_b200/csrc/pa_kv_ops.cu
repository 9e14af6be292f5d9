// pa_cache_write and pa_copy_blocks — the two bit-copy kernels beside the
// decode: storing each new token's K/V in its slot (vLLM blog, plain-language section; study
// notes ch.05 §5 item 2) and copying whole blocks for copy on write (study
// notes ch.05 §6.1, §12 exercise 4).
//
// Both are pure data movement, bound by HBM bandwidth and (at the sizes of
// one decode step) by launch latency.  Each thread moves 16-byte chunks with
// a grid-stride loop; consecutive threads touch consecutive chunks of one
// row or block, so every warp reads and writes 512 contiguous bytes.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kCopyThreads = 256;

// Chunk i of new-token tensor k/v ([T][Hkv][D], D/8 chunks per row) goes to
// row slot % B of block slot / B, same kv head.
__global__ void __launch_bounds__(kCopyThreads)
    cache_write_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, const int64_t* __restrict__ slots,
                       long long total_chunks, int Hkv, int chunks_per_row, int B, long long num_slots,
                       uint4* __restrict__ k_pool, uint4* __restrict__ v_pool, int32_t* status) {
  grid_dependency_wait();
  grid_launch_dependents();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_chunks; i += stride) {
    const int chunk = static_cast<int>(i % chunks_per_row);
    const long long th = i / chunks_per_row;  // token * Hkv + head
    const int h = static_cast<int>(th % Hkv);
    const long long t = th / Hkv;
    const long long slot = __ldg(slots + t);
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (chunk == 0 && h == 0) record_status(status, PA_DEV_BAD_SLOT);
      continue;
    }
    const long long blk = slot / B, row = slot % B;
    const size_t dst = (static_cast<size_t>(blk * Hkv + h) * B + row) * chunks_per_row + chunk;
    k_pool[dst] = __ldg(k + i);
    v_pool[dst] = __ldg(v + i);
  }
}

// Work item i = ((pair * 2 + pool) * chunks_per_block + chunk).
__global__ void __launch_bounds__(kCopyThreads)
    copy_blocks_kernel(const int64_t* __restrict__ pairs, long long total_chunks, long long chunks_per_block,
                       long long num_blocks, uint4* k_pool, uint4* v_pool, int32_t* status) {
  grid_dependency_wait();
  grid_launch_dependents();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_chunks; i += stride) {
    const long long chunk = i % chunks_per_block;
    const long long pw = i / chunks_per_block;
    const long long pair = pw >> 1;
    const long long src = __ldg(pairs + 2 * pair), dst = __ldg(pairs + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (chunk == 0 && (pw & 1) == 0) record_status(status, PA_DEV_BAD_PAIR);
      continue;
    }
    if (src == dst) continue;
    uint4* pool = (pw & 1) ? v_pool : k_pool;
    pool[static_cast<size_t>(dst) * chunks_per_block + chunk] = pool[static_cast<size_t>(src) * chunks_per_block + chunk];
  }
}

static bool kv_pool_ok(const pa_pool_desc* pool) {
  return pool != nullptr && pool->num_blocks > 0 && pool->block_size > 0 && pool->num_kv_heads > 0 &&
         pool->head_dim > 0 && pool->head_dim % 8 == 0 && (pool->dtype == PA_FP16 || pool->dtype == PA_BF16);
}

static int copy_grid(long long total_chunks) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (total_chunks + kCopyThreads - 1) / kCopyThreads;
  const long long cap = static_cast<long long>(sms) * 8;
  return static_cast<int>(want < cap ? want : cap);
}

}  // namespace pa

using namespace pa;

extern "C" pa_status pa_cache_write(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                                    void* k_pool, void* v_pool, int32_t* dev_status, const pa_pool_desc* pool,
                                    void* stream) {
  if (!kv_pool_ok(pool) || num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (k == nullptr || v == nullptr || slot_mapping == nullptr || k_pool == nullptr || v_pool == nullptr)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_INVALID_ARG;
  const int cpr = pool->head_dim / 8;
  const long long total = static_cast<long long>(num_tokens) * pool->num_kv_heads * cpr;
  const long long num_slots = static_cast<long long>(pool->num_blocks) * pool->block_size;
  const cudaError_t e = launch_overlapped(
      cache_write_kernel, dim3(copy_grid(total)), dim3(kCopyThreads), 0, static_cast<cudaStream_t>(stream),
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, total, pool->num_kv_heads, cpr,
      pool->block_size, num_slots, static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), dev_status);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_copy_blocks(const int64_t* src_dst_pairs, int32_t num_pairs, void* k_pool, void* v_pool,
                                    int32_t* dev_status, const pa_pool_desc* pool, void* stream) {
  if (!kv_pool_ok(pool) || num_pairs < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (src_dst_pairs == nullptr || k_pool == nullptr || v_pool == nullptr) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_INVALID_ARG;
  const long long cpb = static_cast<long long>(pool->num_kv_heads) * pool->block_size * pool->head_dim / 8;
  const long long total = static_cast<long long>(num_pairs) * 2 * cpb;
  const cudaError_t e = launch_overlapped(copy_blocks_kernel, dim3(copy_grid(total)), dim3(kCopyThreads), 0,
                                          static_cast<cudaStream_t>(stream), src_dst_pairs, total, cpb,
                                          static_cast<long long>(pool->num_blocks), static_cast<uint4*>(k_pool),
                                          static_cast<uint4*>(v_pool), dev_status);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" const char* pa_status_string(int32_t status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size)";
    case PA_ERR_UNSUPPORTED: return "unsupported block_size/head_dim/group/dtype combination";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
    case PA_ERR_SCRATCH_LIMIT: return "batch needs more scratch than pa_decode_no_alloc's fixed array";
    case PA_ERR_OUT_OF_BLOCKS: return "block manager: not enough free blocks";
    case PA_DEV_BAD_BLOCK_ID: return "device: block table entry outside [0, num_blocks)";
    case PA_DEV_BAD_SEQ_LEN: return "device: seq_len negative or beyond the block table";
    case PA_DEV_BAD_SLOT: return "device: slot_mapping entry beyond the pool";
    case PA_DEV_BAD_PAIR: return "device: copy pair block id outside [0, num_blocks)";
    case PA_DEV_TIMEOUT: return "device: a bounded pipeline wait ran out";
    case PA_DEV_BAD_GROUP: return "device: shared-prefix groups do not partition the sequences or exceed max_group_size";
    default: return "unknown status";
  }
}
