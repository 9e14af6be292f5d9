"""paged_kv_cache_357_b200 — PagedAttention's decode hot path on B200 (sm_100a).

The kernels live in ``libpa.so`` (C ABI: ``include/pa.h``), built in-tree by
``python -m paged_kv_cache_357_b200.build``.  This package is a thin binding:

* ``pa_decode``       paged decode attention with online softmax
* ``pa_decode_multi`` q_len causal query positions per sequence (speculative
                      verification, prefill chunks)
* ``pa_decode_shared_prefix``  decode reading shared prompt blocks once per group
* ``pa_cache_write``  slot-mapped write of new tokens' K/V
* ``pa_copy_blocks``  copy-on-write block copies
* ``pa_decode_update`` (and the ``_multi`` / ``_shared_prefix`` forms) a
                      step's copies, writes and decode as one call, one
                      launch on the tensor-core kernel
* ``pa_decode_lse``, ``pa_merge_partials``  decodes of disjoint token ranges
                      with their log normalisers, and their merge
* ``split.gather_partials`` / ``split.decode_split``  a sequence's token ranges
                      held by different ranks, decoded and merged
* ``PagedDecodeStep`` one whole step (copy, write, decode) from host buffers
* ``BlockManager``    host block manager (free set, ref counts, copy on write)

PyTorch supplies device memory and streams only.
"""

from ._lib import (  # noqa: F401
    DEV_STATUS,
    EXPORTED,
    LIB_PATH,
    PA_BF16,
    PA_DECODE_CUDA_CORES_ONLY,
    PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL,
    PA_DECODE_TEST_WITHHOLD_COPIES,
    PA_FP16,
    CacheUpdate,
    DecodeOpts,
    PaError,
    PoolDesc,
    alloc_decode_workspace,
    alloc_multi_workspace,
    alloc_shared_prefix_workspace,
    decode_workspace_bytes,
    multi_workspace_bytes,
    shared_prefix_workspace_bytes,
    shared_prefix_groups,
    pa_decode_multi,
    pa_decode_shared_prefix,
    load,
    pa_cache_write,
    pa_copy_blocks,
    pa_decode,
    pa_decode_lse,
    pa_decode_no_alloc,
    pa_merge_partials,
    pa_decode_multi_update,
    pa_decode_shared_prefix_update,
    pa_decode_update,
    pool_desc,
    status_string,
)
from .block_manager import BlockManager  # noqa: F401
from .step import PagedDecodeStep  # noqa: F401
