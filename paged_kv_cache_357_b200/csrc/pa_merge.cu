// pa_merge_partials — the online-softmax merge (study notes ch.05 §4: the
// running max and running sum carried across blocks) applied to whole
// decodes of disjoint token ranges of the same query rows, for example the
// ranges of one long sequence held by different GPUs.  Part r of a row
// brings its normalised output o_r and its log normaliser lse_r = log sum
// exp(scores of its range); with M = max_r lse_r and w_r = exp(lse_r - M):
//   out = sum_r w_r o_r / sum_r w_r,   lse = M + log sum_r w_r,
// the same rescale-to-a-common-max rule the decode kernels use to merge the
// pieces of a split unit.  A row no part saw (every lse_r = -inf) gets a zero
// output and lse -inf.
//
// HBM-bound and small: one warp per row, each lane a pair of elements per
// 64 columns, the parts read in turn; a grid of the SM count times 8 CTAs
// strides over the rows.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kMergeThreads = 256;

template <bool kBf16, int D>
__global__ void __launch_bounds__(kMergeThreads)
    merge_partials_kernel(const uint32_t* __restrict__ outs, const float* __restrict__ lses, int parts,
                          long long rows, uint32_t* __restrict__ out, float* __restrict__ lse_out) {
  grid_dependency_wait();
  grid_launch_dependents();
  constexpr int kPairs = D / 2 / 32;  // element pairs per lane
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (kMergeThreads / 32);
  for (long long row = (static_cast<long long>(blockIdx.x) * kMergeThreads + threadIdx.x) / 32; row < rows;
       row += warps) {
    float M = -INFINITY;
    for (int r = 0; r < parts; ++r) M = fmaxf(M, __ldg(lses + r * rows + row));
    uint32_t* o = out + row * (D / 2);
    if (M == -INFINITY) {
#pragma unroll
      for (int i = 0; i < kPairs; ++i) o[lane + 32 * i] = 0u;
      if (lse_out != nullptr && lane == 0) lse_out[row] = -INFINITY;
      continue;
    }
    float acc[2 * kPairs] = {};
    float wsum = 0.f;
    for (int r = 0; r < parts; ++r) {
      const float lr = __ldg(lses + r * rows + row);
      if (lr == -INFINITY) continue;  // a part that saw no token adds nothing
      const float w = expf(lr - M);
      wsum += w;
      const uint32_t* src = outs + (r * rows + row) * (D / 2);
#pragma unroll
      for (int i = 0; i < kPairs; ++i) {
        float a, b;
        unpack2<kBf16>(__ldg(src + lane + 32 * i), a, b);
        acc[2 * i] = fmaf(w, a, acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, b, acc[2 * i + 1]);
      }
    }
    const float inv = 1.f / wsum;  // wsum >= 1: the largest part has weight 1
#pragma unroll
    for (int i = 0; i < kPairs; ++i) o[lane + 32 * i] = pack2<kBf16>(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    if (lse_out != nullptr && lane == 0) lse_out[row] = M + logf(wsum);
  }
}

template <bool kBf16, int D>
static cudaError_t launch_merge(const void* outs, const float* lses, int parts, long long rows, void* out,
                                float* lse_out, cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (rows + kMergeThreads / 32 - 1) / (kMergeThreads / 32);
  const long long cap = static_cast<long long>(sms) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  return launch_overlapped(merge_partials_kernel<kBf16, D>, dim3(grid), dim3(kMergeThreads), 0, stream,
                           static_cast<const uint32_t*>(outs), lses, parts, rows, static_cast<uint32_t*>(out),
                           lse_out);
}

}  // namespace pa

using namespace pa;

extern "C" pa_status pa_merge_partials(const void* outs, const float* lses, int32_t num_parts, int32_t num_rows,
                                       int32_t head_dim, int32_t dtype, void* out, float* lse_out, void* stream) {
  if (num_parts < 1 || num_rows < 0 || (head_dim != 64 && head_dim != 128) || (dtype != PA_FP16 && dtype != PA_BF16))
    return PA_ERR_INVALID_ARG;
  if (num_rows == 0) return PA_OK;
  if (outs == nullptr || lses == nullptr || out == nullptr || !aligned16(outs) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lses) & 3u) != 0 || (reinterpret_cast<uintptr_t>(lse_out) & 3u) != 0) {
    return PA_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(num_parts) * num_rows * head_dim > (1LL << 40)) return PA_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == PA_BF16) {
    e = head_dim == 128 ? launch_merge<true, 128>(outs, lses, num_parts, num_rows, out, lse_out, s)
                        : launch_merge<true, 64>(outs, lses, num_parts, num_rows, out, lse_out, s);
  } else {
    e = head_dim == 128 ? launch_merge<false, 128>(outs, lses, num_parts, num_rows, out, lse_out, s)
                        : launch_merge<false, 64>(outs, lses, num_parts, num_rows, out, lse_out, s);
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
