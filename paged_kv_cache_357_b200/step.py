"""One decode step of a paged KV cache driven from host buffers.

The K/V pools are the cache state: they stay resident in device memory
across steps.  What changes every step arrives from the host — q, the block
tables and lengths, the new tokens' K/V with their slots, and any
copy-on-write pairs — and the attention output goes back to the host.  A
step enqueues, on one stream:

    H2D copies -> pa_copy_blocks -> pa_cache_write -> pa_decode -> D2H copy

matching the order of the method: a shared block is copied before a sample
writes into it (study notes ch.05 §6.1), the new token is stored before the
decode reads it (vLLM blog, plain-language section), and the decode reads every block through the
table (vLLM blog §"关键细节" 2)).
"""

from __future__ import annotations

from typing import Optional

from . import _lib


class PagedDecodeStep:
    def __init__(self, k_pool, v_pool, num_seqs: int, num_q_heads: int, max_blocks_per_seq: int,
                 max_new_tokens: int = 0, max_copy_pairs: int = 0, scale: Optional[float] = None,
                 stream=None, num_ctas: int = 0):
        import torch

        self.torch = torch
        self.k_pool, self.v_pool = k_pool, v_pool
        dev = k_pool.device
        NB, Hkv, B, D = k_pool.shape
        self.S, self.Hq, self.D, self.Hkv = num_seqs, num_q_heads, D, Hkv
        self.scale = (1.0 / D**0.5) if scale is None else float(scale)
        self.stream = torch.cuda.Stream(device=dev) if stream is None else stream
        self.num_ctas = num_ctas
        dt = k_pool.dtype
        self.q = torch.empty((num_seqs, num_q_heads, D), dtype=dt, device=dev)
        self.out = torch.empty_like(self.q)
        self.tables = torch.empty((num_seqs, max_blocks_per_seq), dtype=torch.int32, device=dev)
        self.lens = torch.empty((num_seqs,), dtype=torch.int32, device=dev)
        self.new_k = torch.empty((max(max_new_tokens, 1), Hkv, D), dtype=dt, device=dev)
        self.new_v = torch.empty_like(self.new_k)
        self.slots = torch.empty((max(max_new_tokens, 1),), dtype=torch.int64, device=dev)
        self.pairs = torch.empty((max(max_copy_pairs, 1), 2), dtype=torch.int64, device=dev)
        self.workspace = _lib.alloc_decode_workspace(num_seqs, num_q_heads, k_pool, num_ctas)
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.out_host = torch.empty(self.out.shape, dtype=dt, pin_memory=True)
        self.last_h2d_bytes = 0
        self.last_d2h_bytes = 0

    def run(self, q, block_tables, seq_lens, new_k=None, new_v=None, slot_mapping=None, copy_pairs=None):
        """Enqueue one step from host tensors (pinned for overlap); returns the
        pinned host output tensor, valid after ``self.stream`` synchronises."""
        torch = self.torch
        h2d = 0
        with torch.cuda.stream(self.stream):
            for dst, src in ((self.q, q), (self.tables, block_tables), (self.lens, seq_lens)):
                dst.copy_(src, non_blocking=True)
                h2d += src.numel() * src.element_size()
            if copy_pairs is not None and copy_pairs.shape[0] > 0:
                n = copy_pairs.shape[0]
                self.pairs[:n].copy_(copy_pairs, non_blocking=True)
                h2d += copy_pairs.numel() * copy_pairs.element_size()
                _lib.pa_copy_blocks(self.pairs[:n], self.k_pool, self.v_pool, self.status, stream=self.stream)
            if slot_mapping is not None and slot_mapping.shape[0] > 0:
                T = slot_mapping.shape[0]
                self.new_k[:T].copy_(new_k, non_blocking=True)
                self.new_v[:T].copy_(new_v, non_blocking=True)
                self.slots[:T].copy_(slot_mapping, non_blocking=True)
                h2d += sum(t.numel() * t.element_size() for t in (new_k, new_v, slot_mapping))
                _lib.pa_cache_write(self.new_k[:T], self.new_v[:T], self.slots[:T], self.k_pool, self.v_pool,
                                    self.status, stream=self.stream)
            _lib.pa_decode(self.q, self.k_pool, self.v_pool, self.tables, self.lens, self.scale, self.out,
                           self.workspace, self.status, num_ctas=self.num_ctas, stream=self.stream)
            self.out_host.copy_(self.out, non_blocking=True)
        self.last_h2d_bytes = h2d
        self.last_d2h_bytes = self.out.numel() * self.out.element_size()
        return self.out_host

    def device_status(self) -> int:
        """Synchronise the step's stream and return the device status code."""
        self.stream.synchronize()
        return int(self.status.item())
