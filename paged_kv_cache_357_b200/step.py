"""One decode step of a paged KV cache driven from host buffers.

The K/V pools are the cache state: they stay resident in device memory
across steps.  What changes every step arrives from the host — q, the block
tables and lengths, the new tokens' K/V with their slots, and any
copy-on-write pairs — and the attention output goes back to the host.  A
step runs, in the order the method needs:

    H2D copy -> pa_copy_blocks -> pa_cache_write -> pa_decode -> D2H copy

(pa_decode_multi or pa_decode_shared_prefix in place of pa_decode when the
step is built for them); a shared block is copied before a sample writes
into it (study notes ch.05 §6.1), the new token is stored before the decode
reads it (vLLM blog, plain-language section), and the decode reads every
block through the table (vLLM blog §"关键细节" 2).

The step itself is libpa's native executor (``pa_step_*`` in pa.h): per
step one C call, which enqueues one copy of the packed inputs, one CUDA
graph of the step's kernels and one copy of the output, on three streams,
with neighbouring steps overlapping through several buffer sets (three by
default).  This module owns the memory (device input blocks, pinned staging
blocks of the same layout, outputs, workspace) and marshals arguments.
A caller that builds a step's inputs in the staging views (``staging()``)
saves the host-side copy into them.
"""

from __future__ import annotations

import ctypes
from typing import Optional

from . import _lib


class _BufferSet:
    """One step's packed input block (device) with its pinned staging twin,
    and the step's output (device) with its pinned host copy."""

    def __init__(self, torch, dev, dt, layout, fields, out_shape):
        self.dev_bytes = torch.empty(layout.total, dtype=torch.uint8, device=dev)
        self.host_bytes = torch.empty(layout.total, dtype=torch.uint8, pin_memory=True)
        self.host = {}
        self.dev = {}
        for name, (fdt, shape) in fields.items():
            off = getattr(layout, name)
            n = 1
            for d in shape:
                n *= d
            nbytes = n * torch.empty((), dtype=fdt).element_size()
            self.host[name] = self.host_bytes[off:off + nbytes].view(fdt).view(shape)
            self.dev[name] = self.dev_bytes[off:off + nbytes].view(fdt).view(shape)
        self.out = torch.empty(out_shape, dtype=dt, device=dev)
        self.out_host = torch.empty(out_shape, dtype=dt, pin_memory=True)


class PagedDecodeStep:
    def __init__(self, k_pool, v_pool, num_seqs: int, num_q_heads: int, max_blocks_per_seq: int,
                 max_new_tokens: int = 0, max_copy_pairs: int = 0, scale: Optional[float] = None,
                 num_ctas: int = 0, q_len: int = 1, max_group_size: int = 0, num_buffer_sets: int = 3,
                 decode_flags: int = 0):
        """q_len > 1: each step is a multi-query step (pa_decode_multi, q is
        [num_seqs, q_len, num_q_heads, head_dim]).  max_group_size > 0: each
        step decodes with pa_decode_shared_prefix and takes the groups as
        inputs.  Otherwise pa_decode, with decode_flags (e.g.
        PA_DECODE_CUDA_CORES_ONLY)."""
        import torch

        self.torch = torch
        self.k_pool, self.v_pool = k_pool, v_pool
        dev = k_pool.device
        NB, Hkv, B, D = k_pool.shape
        if q_len > 1 and max_group_size > 0:
            raise ValueError("a step is either multi-query or shared-prefix")
        if not 2 <= num_buffer_sets <= _lib.PA_STEP_MAX_SETS:
            raise ValueError(f"between 2 and {_lib.PA_STEP_MAX_SETS} buffer sets")
        self.S, self.Hq, self.D, self.Hkv = num_seqs, num_q_heads, D, Hkv
        self.scale = (1.0 / D**0.5) if scale is None else float(scale)
        self.q_len, self.max_group_size = q_len, max_group_size
        kind = (_lib.PA_STEP_MULTI if q_len > 1 else
                _lib.PA_STEP_SHARED_PREFIX if max_group_size > 0 else _lib.PA_STEP_DECODE)
        self._c = _lib.load()
        self._shape = _lib.StepShape(kind, num_seqs, num_q_heads, max_blocks_per_seq, q_len, max_group_size,
                                     max_new_tokens, max_copy_pairs, self.scale,
                                     _lib.DecodeOpts(num_ctas, decode_flags))
        self._desc = _lib.pool_desc(k_pool)
        layout = _lib.StepLayout()
        _check(self._c.pa_step_layout_of(ctypes.byref(self._shape), ctypes.byref(self._desc), ctypes.byref(layout)),
               "pa_step_layout_of")
        self.layout = layout
        dt, i32, i64 = k_pool.dtype, torch.int32, torch.int64
        S, T, P = num_seqs, max_new_tokens, max_copy_pairs
        q_shape = (S, num_q_heads, D) if q_len == 1 else (S, q_len, num_q_heads, D)
        fields = {"q": (dt, q_shape), "block_tables": (i32, (S, max_blocks_per_seq)), "seq_lens": (i32, (S,)),
                  "copy_pairs": (i64, (P, 2)), "new_k": (dt, (T, Hkv, D)), "new_v": (dt, (T, Hkv, D)),
                  "slot_mapping": (i64, (T,))}
        if max_group_size > 0:
            fields.update(group_starts=(i32, (S + 1,)), group_prefix_blocks=(i32, (S,)))
        self.sets = [_BufferSet(torch, dev, dt, layout, fields, q_shape) for _ in range(num_buffer_sets)]
        if q_len > 1:
            self.workspace = _lib.alloc_multi_workspace(num_seqs, q_len, num_q_heads, k_pool, num_ctas)
        elif max_group_size > 0:
            self.workspace = _lib.alloc_shared_prefix_workspace(num_seqs, max_group_size, num_q_heads, k_pool,
                                                                num_ctas)
        else:
            self.workspace = _lib.alloc_decode_workspace(num_seqs, num_q_heads, k_pool, num_ctas, decode_flags)
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        arr = ctypes.c_void_p * num_buffer_sets
        self._ptrs = [arr(*[getattr(bs, name).data_ptr() for bs in self.sets])
                      for name in ("dev_bytes", "host_bytes", "out", "out_host")]
        handle = ctypes.c_void_p()
        _check(self._c.pa_step_create(ctypes.byref(self._shape), ctypes.byref(self._desc), k_pool.data_ptr(),
                                      v_pool.data_ptr(), self.workspace.data_ptr(),
                                      self.workspace.numel() * self.workspace.element_size(), self.status.data_ptr(),
                                      num_buffer_sets, *self._ptrs, ctypes.byref(handle)), "pa_step_create")
        self._h = handle
        up, ker, down = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(self._c.pa_step_streams(self._h, ctypes.byref(up), ctypes.byref(ker), ctypes.byref(down)),
               "pa_step_streams")
        self.h2d_stream = torch.cuda.ExternalStream(up.value, device=dev)
        self.compute_stream = torch.cuda.ExternalStream(ker.value, device=dev)
        self.d2h_stream = torch.cuda.ExternalStream(down.value, device=dev)
        self._set = ctypes.c_int32()
        self.steps = 0
        self.last_h2d_bytes = 0
        self.last_d2h_bytes = 0

    def staging(self):
        """Pinned host views the next ``run()`` uploads from: q, block_tables,
        seq_lens, new_k, new_v, slot_mapping, copy_pairs (and group_starts,
        group_prefix_blocks for a shared-prefix step), each at its maximum
        size.  A caller that builds its inputs there, and passes them (or
        their leading rows) to ``run()``, saves the host-side copy.  Waits
        until the upload that last read this area is done."""
        _check(self._c.pa_step_next_set(self._h, ctypes.byref(self._set)), "pa_step_next_set")
        return dict(self.sets[self._set.value].host)

    def run(self, q, block_tables, seq_lens, new_k=None, new_v=None, slot_mapping=None, copy_pairs=None,
            group_starts=None, group_prefix_blocks=None):
        """Enqueue one step from host tensors (the ``staging()`` views, or
        any host tensors, which are first copied into them).  Returns the
        pinned host output of this step, valid once ``wait(result)`` or
        ``synchronize()`` returns and until its buffer set comes round again
        (``len(self.sets)`` steps later).  A shared-prefix step also takes
        the groups (int32 host tensors [num_groups + 1] and [num_groups])."""
        _check(self._c.pa_step_next_set(self._h, ctypes.byref(self._set)), "pa_step_next_set")
        bs = self.sets[self._set.value]
        n_groups = 0
        if self.max_group_size > 0:
            if group_starts is None or group_prefix_blocks is None:
                raise ValueError("a shared-prefix step needs group_starts and group_prefix_blocks")
            n_groups = group_prefix_blocks.shape[0]
        n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
        T = 0 if slot_mapping is None else slot_mapping.shape[0]
        inputs = [("q", None, q), ("block_tables", None, block_tables), ("seq_lens", None, seq_lens)]
        if n_groups > 0:
            inputs += [("group_starts", n_groups + 1, group_starts),
                       ("group_prefix_blocks", n_groups, group_prefix_blocks)]
        if n_pairs > 0:
            inputs.append(("copy_pairs", n_pairs, copy_pairs))
        if T > 0:
            inputs += [("new_k", T, new_k), ("new_v", T, new_v), ("slot_mapping", T, slot_mapping)]
        for name, rows, src in inputs:
            dst = bs.host[name] if rows is None else bs.host[name][:rows]
            if tuple(src.shape) != tuple(dst.shape):
                raise ValueError(f"{name}: shape {tuple(src.shape)}, the step holds {tuple(dst.shape)}")
            if src.data_ptr() != dst.data_ptr():
                dst.copy_(src)
        return self.run_staged(n_pairs, T, n_groups)

    def run_staged(self, num_copy_pairs: int = 0, num_new_tokens: int = 0, num_groups: int = 0):
        """Enqueue one step whose inputs already sit in the next buffer
        set's staging views (written after ``staging()`` returned them, or
        left there by an earlier step of the same set): the leading
        num_copy_pairs pairs, num_new_tokens tokens and, for a shared-prefix
        step, num_groups groups are used.  One C call, no host-side copy or
        check of the views; returns the pinned host output as ``run()``."""
        _check(self._c.pa_step_run(self._h, num_copy_pairs, num_new_tokens, num_groups, ctypes.byref(self._set)),
               "pa_step_run")
        self.steps += 1
        L = self.layout
        if num_new_tokens > 0:
            self.last_h2d_bytes = L.slot_mapping + 8 * num_new_tokens
        elif num_copy_pairs > 0:
            self.last_h2d_bytes = L.copy_pairs + 16 * num_copy_pairs
        elif num_groups > 0:
            self.last_h2d_bytes = L.group_prefix_blocks + 4 * num_groups
        else:
            self.last_h2d_bytes = L.seq_lens + 4 * self.S
        self.last_d2h_bytes = L.out_bytes
        return self.sets[self._set.value].out_host

    def wait(self, result) -> None:
        """Block until the step that returned ``result`` has been read back."""
        for k, bs in enumerate(self.sets):
            if bs.out_host is result:
                _check(self._c.pa_step_wait(self._h, k), "pa_step_wait")
                return
        raise ValueError("not a result of this PagedDecodeStep")

    def flush(self) -> None:
        """Enqueue the download of the last step now (it is otherwise issued
        with the next step, behind that step's upload)."""
        _check(self._c.pa_step_flush(self._h), "pa_step_flush")

    def synchronize(self) -> None:
        _check(self._c.pa_step_synchronize(self._h), "pa_step_synchronize")

    def device_status(self) -> int:
        """Synchronise every stream of the step and return the device status."""
        self.synchronize()
        return int(self.status.item())

    def close(self) -> None:
        """Release the executor (its streams, events and graphs); the memory
        stays with this object."""
        h, self._h = getattr(self, "_h", None), None
        if h is not None and h.value:
            self._c.pa_step_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise _lib.PaError(rc, name)
