"""Block bookkeeping of the paged KV cache (test infrastructure only).

* blocks_needed / block_fills: on-demand allocation — a request of n tokens
  takes ceil(n / B) blocks and only the last one may be partly filled
  (study notes ch.05 §5 item 2, §9.2, §12 exercise 1).
* kv_bytes_per_token: 2 (K and V) x layers x kv heads x head_dim x dtype
  bytes (vLLM blog §"关键细节" 1) KV-size formula; study notes ch.05 §2 for OPT-13B).
* BlockManager: free set, reference counts, fork by sharing, copy on write
  when a writer's target block is shared, free at ref count zero
  (study notes ch.05 §5, §6.1, §6.2, §12 exercise 4).
"""

from __future__ import annotations

from typing import List, Optional, Tuple


def blocks_needed(n_tokens: int, block_size: int) -> int:
    """ceil(n / B): blocks a request of n tokens occupies."""
    if n_tokens < 0 or block_size <= 0:
        raise ValueError("n_tokens >= 0 and block_size > 0 required")
    return (n_tokens + block_size - 1) // block_size


def block_fills(n_tokens: int, block_size: int) -> List[int]:
    """Tokens held by each of the request's blocks: all full but the last."""
    k = blocks_needed(n_tokens, block_size)
    return [min(block_size, n_tokens - j * block_size) for j in range(k)]


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    """2 x layers x kv heads x head_dim x bytes per element."""
    return 2 * num_layers * num_kv_heads * head_dim * dtype_bytes


class BlockManager:
    """A free set plus reference counts over num_blocks physical blocks."""

    def __init__(self, num_blocks: int, block_size: int):
        self.block_size = block_size
        self.free = list(range(num_blocks))
        self.ref = [0] * num_blocks

    def allocate(self) -> int:
        if not self.free:
            raise MemoryError("no free block")
        b = self.free.pop(0)
        self.ref[b] = 1
        return b

    def new_sequence(self, n_tokens: int) -> List[int]:
        """Block table for a fresh request of n tokens."""
        return [self.allocate() for _ in range(blocks_needed(n_tokens, self.block_size))]

    def fork(self, table: List[int]) -> List[int]:
        """A new output that shares every block of ``table`` (ref += 1)."""
        for b in table:
            self.ref[b] += 1
        return list(table)

    def append_slot(self, table: List[int], n_before: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Place token number n_before (0-based) of the sequence owning
        ``table``.  A new block is taken when the last one is full; if the
        target block is shared it is first copied (copy on write): the copy
        gets ref 1, the source loses one reference and the table is repointed.
        Returns (slot, (src, dst) or None)."""
        B = self.block_size
        j, r = divmod(n_before, B)
        cow = None
        if j == len(table):
            table.append(self.allocate())
        elif j > len(table):
            raise ValueError("token position beyond the table")
        else:
            b = table[j]
            if self.ref[b] > 1:
                nb = self.allocate()
                self.ref[b] -= 1
                table[j] = nb
                cow = (b, nb)
        return table[j] * B + r, cow

    def free_sequence(self, table: List[int]) -> None:
        """Drop one reference per block; blocks reaching zero become free."""
        for b in table:
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
            elif self.ref[b] < 0:
                raise RuntimeError("reference count below zero")
