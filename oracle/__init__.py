"""CPU float64 oracle for paged decode attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (``cpu_baseline`` and ``--impl reference``) may import anything here.  The
product path (``paged_kv_cache_357_b200``) never imports it and shares no code
with it.

Sources (the three pages this project follows):

* "LLM 注意力与计算内核精读笔记 · 05 PagedAttention 与 KV 显存管理"
  (PagedAttention study notes, ch.05) — the authority on what is computed:
  §3 block table, §4 blockwise attention with online softmax, §5 on-demand
  allocation, §6 copy-on-write, §9/§12 worked examples.
* "vLLM 是什么 PagedAttention 解决了什么" (vLLM blog) — §2 attention
  definition softmax(QK^T/sqrt(d))V and block_table indirection, §1 KV-size
  formula with the Llama-3-8B GQA example.
* "PagedAttention：分页注意力" (CSDN article) — KV-size example for
  LLaMA-7B; its per-block-softmax toy code is NOT followed (it normalises each
  block on its own, which is not attention; the study notes §4 win).

Every function is pinned by tests in ``tests/test_oracle.py``,
``tests/test_oracle_multi.py``, ``tests/test_oracle_bits.py`` and
``tests/test_oracle_lse.py`` against values the pages print, closed forms,
invariants and brute force; none is "parity unpinned".
"""

from .paged_attention import (  # noqa: F401
    bits_to_f64,
    gather_kv,
    attention_dense,
    decode,
    decode_lse,
    merge_outputs,
    decode_one,
    decode_multi,
    decode_blockwise_online,
    partition_states,
    merge_partition_states,
    cache_write,
    copy_blocks,
)
from .bookkeeping import (  # noqa: F401
    blocks_needed,
    block_fills,
    kv_bytes_per_token,
    BlockManager,
)
