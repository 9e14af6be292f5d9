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
  int part_stride;  // floats per partial slot: G * (D + 2)
  LaunchFn launch;
};

// Tensor-core variant for this pool and group size, if one exists
// (defined in pa_decode_tc.cu).
bool select_tc_variant(const pa_pool_desc& pool, int group, Variant& v);

}  // namespace pa
