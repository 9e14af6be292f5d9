"""One decode step of a paged KV cache driven from host buffers.

The K/V pools are the cache state: they stay resident in device memory
across steps.  What changes every step arrives from the host — q, the block
tables and lengths, the new tokens' K/V with their slots, and any
copy-on-write pairs — and the attention output goes back to the host.  A
step runs, in the order the method needs:

    H2D copies -> pa_copy_blocks -> pa_cache_write -> pa_decode -> D2H copy

(pa_decode_multi or pa_decode_shared_prefix in place of pa_decode when the
step is built for them);
a shared block is copied before a sample writes into it (study notes ch.05
§6.1), the new token is stored before the decode reads it (vLLM blog,
plain-language section), and the decode reads every block through the table
(vLLM blog §"关键细节" 2).

Consecutive steps overlap their copies with each other's kernels: the
per-step buffers come in several sets (three by default) used in turn,
uploads run on one stream, kernels on a second and downloads on a third.
Events order the work: a step's kernels wait for its uploads and for the
previous step's kernels (they share the pools); its download waits for its
kernels; the upload into a buffer set waits until the kernels that last read
that set are done, so an upload has the time of (sets - 1) steps.

Per step the host issues little.  Each buffer set is one device allocation
with a pinned host staging area of the same layout: a caller that builds a
step's inputs in the staging views (``staging()``) has them go up in one
copy; other pinned host tensors are copied field by field, straight from
where they are.  After the first step, a set's kernels (copy, write,
decode) are replayed as one CUDA graph captured for that set and those
counts.
"""

from __future__ import annotations

import ctypes
from typing import Optional

from . import _lib

_ALIGN = 256  # byte alignment of every field inside a buffer set


class _BufferSet:
    """One step's inputs and output: the inputs carved from one device
    allocation, mirrored by a pinned host staging area of the same layout."""

    def __init__(self, torch, dev, dt, S, Hq, D, Hkv, max_nb, T, P, q_len, grouped):
        q_shape = (S, Hq, D) if q_len == 1 else (S, q_len, Hq, D)
        fields = [("q", dt, q_shape), ("tables", torch.int32, (S, max_nb)), ("lens", torch.int32, (S,))]
        if grouped:
            fields += [("group_starts", torch.int32, (S + 1,)), ("group_prefix", torch.int32, (max(S, 1),))]
        fields += [("pairs", torch.int64, (max(P, 1), 2)), ("new_k", dt, (max(T, 1), Hkv, D)),
                   ("new_v", dt, (max(T, 1), Hkv, D)), ("slots", torch.int64, (max(T, 1),))]
        self.offsets, off = {}, 0
        for name, fdt, shape in fields:
            n = 1
            for d in shape:
                n *= d
            nbytes = n * torch.empty((), dtype=fdt).element_size()
            self.offsets[name] = (off, off + nbytes, fdt, shape)
            off = (off + nbytes + _ALIGN - 1) // _ALIGN * _ALIGN
        self.dev_bytes = torch.empty(off, dtype=torch.uint8, device=dev)
        self.host_bytes = torch.empty(off, dtype=torch.uint8, pin_memory=True)
        self.dev = {name: self._view(self.dev_bytes, name) for name in self.offsets}
        self.host = {name: self._view(self.host_bytes, name) for name in self.offsets}
        self.q, self.tables, self.lens = self.dev["q"], self.dev["tables"], self.dev["lens"]
        self.group_starts, self.group_prefix = self.dev.get("group_starts"), self.dev.get("group_prefix")
        self.pairs, self.new_k, self.new_v, self.slots = (self.dev[n] for n in ("pairs", "new_k", "new_v", "slots"))
        self.out = torch.empty(q_shape, dtype=dt, device=dev)
        self.out_host = torch.empty(q_shape, dtype=dt, pin_memory=True)
        self.uploaded = torch.cuda.Event()
        self.computed = torch.cuda.Event()
        self.downloaded = torch.cuda.Event()
        self.graphs = {}  # (copy pairs, new tokens, groups) -> captured kernels of this set
        self.used = False

    def _view(self, buf, name):
        a, b, fdt, shape = self.offsets[name]
        return buf[a:b].view(fdt).view(shape)

    def upload_end(self, n_pairs: int, T: int, n_groups: int) -> int:
        """Bytes from the start of the layout through the last field this
        step uses (the whole prefix goes up in one copy)."""
        if T > 0:
            return self.offsets["slots"][1]
        if n_pairs > 0:
            return self.offsets["pairs"][1]
        if n_groups > 0:
            return self.offsets["group_prefix"][1]
        return self.offsets["lens"][1]


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
        self.S, self.Hq, self.D, self.Hkv = num_seqs, num_q_heads, D, Hkv
        self.scale = (1.0 / D**0.5) if scale is None else float(scale)
        self.num_ctas = num_ctas
        self.decode_flags = decode_flags
        if q_len > 1 and max_group_size > 0:
            raise ValueError("a step is either multi-query or shared-prefix")
        self.q_len, self.max_group_size = q_len, max_group_size
        self.h2d_stream = torch.cuda.Stream(device=dev)
        self.compute_stream = torch.cuda.Stream(device=dev)
        self.d2h_stream = torch.cuda.Stream(device=dev)
        if num_buffer_sets < 2:
            raise ValueError("at least two buffer sets")
        self.sets = [_BufferSet(torch, dev, k_pool.dtype, num_seqs, num_q_heads, D, Hkv, max_blocks_per_seq,
                                max_new_tokens, max_copy_pairs, q_len, max_group_size > 0)
                     for _ in range(num_buffer_sets)]
        if q_len > 1:
            self.workspace = _lib.alloc_multi_workspace(num_seqs, q_len, num_q_heads, k_pool, num_ctas)
        elif max_group_size > 0:
            self.workspace = _lib.alloc_shared_prefix_workspace(num_seqs, max_group_size, num_q_heads, k_pool,
                                                                num_ctas)
        else:
            self.workspace = _lib.alloc_decode_workspace(num_seqs, num_q_heads, k_pool, num_ctas, decode_flags)
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        # Every buffer the kernels touch is fixed above, so the C calls are
        # bound here once, checked by the same rules as the Python wrappers
        # (which a first call below goes through); a step then passes only
        # the counts that change.
        self._c = _lib.load()
        self._desc = _lib.pool_desc(k_pool)
        self._desc_ref = ctypes.byref(self._desc)
        self._opts = _lib.DecodeOpts(num_ctas, decode_flags)
        self._opts_ref = ctypes.byref(self._opts)
        self._cs = self.compute_stream.cuda_stream
        self._ws = (self.workspace.data_ptr(), self.workspace.numel() * self.workspace.element_size())
        self._checked = False
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
        bs = self.sets[self.steps % len(self.sets)]
        if bs.used:
            bs.uploaded.synchronize()
        h = bs.host
        views = dict(q=h["q"], block_tables=h["tables"], seq_lens=h["lens"], new_k=h["new_k"], new_v=h["new_v"],
                     slot_mapping=h["slots"], copy_pairs=h["pairs"])
        if self.max_group_size > 0:
            views.update(group_starts=h["group_starts"], group_prefix_blocks=h["group_prefix"])
        return views

    def run(self, q, block_tables, seq_lens, new_k=None, new_v=None, slot_mapping=None, copy_pairs=None,
            group_starts=None, group_prefix_blocks=None):
        """Enqueue one step from host tensors (pinned, or the ``staging()``
        views; leave them unchanged until the step's upload is done).
        Returns the pinned host output of this step, valid once
        ``wait(result)`` or ``synchronize()`` returns and until its buffer set
        comes round again (``len(self.sets)`` steps later).  A shared-prefix
        step also takes the groups (int32 host tensors [num_groups + 1] and
        [num_groups])."""
        torch = self.torch
        bs = self.sets[self.steps % len(self.sets)]
        n_groups = 0
        if self.max_group_size > 0:
            if group_starts is None or group_prefix_blocks is None:
                raise ValueError("a shared-prefix step needs group_starts and group_prefix_blocks")
            n_groups = group_prefix_blocks.shape[0]
        n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
        T = 0 if slot_mapping is None else slot_mapping.shape[0]
        # (field, leading rows or None for all, host tensor) of this step's inputs
        inputs = [("q", None, q), ("tables", None, block_tables), ("lens", None, seq_lens)]
        if n_groups > 0:
            inputs += [("group_starts", n_groups + 1, group_starts), ("group_prefix", n_groups, group_prefix_blocks)]
        if n_pairs > 0:
            inputs.append(("pairs", n_pairs, copy_pairs))
        if T > 0:
            inputs += [("new_k", T, new_k), ("new_v", T, new_v), ("slots", T, slot_mapping)]
        packed = all(src.data_ptr() == bs.host[name].data_ptr() for name, _, src in inputs)
        with torch.cuda.stream(self.h2d_stream):
            if bs.used:
                self.h2d_stream.wait_event(bs.computed)  # the kernels that last read this set
            if packed:
                # every input sits in this set's staging area: one copy of the used prefix
                end = bs.upload_end(n_pairs, T, n_groups)
                bs.dev_bytes[:end].copy_(bs.host_bytes[:end], non_blocking=True)
                h2d = end
            else:
                h2d = 0
                for name, rows, src in inputs:
                    dst = bs.dev[name] if rows is None else bs.dev[name][:rows]
                    dst.copy_(src, non_blocking=True)
                    h2d += src.numel() * src.element_size()
            bs.uploaded.record(self.h2d_stream)
        with torch.cuda.stream(self.compute_stream):
            # the compute stream is in order, so the previous step's kernels
            # (which read the pools this step writes) are already ahead of us
            self.compute_stream.wait_event(bs.uploaded)
            if bs.used:
                self.compute_stream.wait_event(bs.downloaded)  # out of this set was read back
            if not self._checked:
                self._launch_checked(bs, n_pairs, T, n_groups)
                self._checked = True
            else:
                self._launch_graph(bs, n_pairs, T, n_groups)
            bs.computed.record(self.compute_stream)
        with torch.cuda.stream(self.d2h_stream):
            self.d2h_stream.wait_event(bs.computed)
            bs.out_host.copy_(bs.out, non_blocking=True)
            bs.downloaded.record(self.d2h_stream)
        bs.used = True
        self.steps += 1
        self.last_h2d_bytes = h2d
        self.last_d2h_bytes = bs.out.numel() * bs.out.element_size()
        return bs.out_host

    def _launch_graph(self, bs, n_pairs: int, T: int, n_groups: int) -> None:
        """Replay this set's kernels for these counts, capturing them the
        first time (capture records the launches without running them)."""
        key = (n_pairs, T, n_groups)
        g = bs.graphs.get(key)
        if g is None:
            g = self.torch.cuda.CUDAGraph()
            with self.torch.cuda.graph(g, stream=self.compute_stream, capture_error_mode="thread_local"):
                self._launch_bound(bs, n_pairs, T, n_groups)
            bs.graphs[key] = g
        g.replay()

    def _launch_checked(self, bs, n_pairs: int, T: int, n_groups: int) -> None:
        """The step's kernels through the checking Python wrappers."""
        cs = self.compute_stream
        if n_pairs > 0:
            _lib.pa_copy_blocks(bs.pairs[:n_pairs], self.k_pool, self.v_pool, self.status, stream=cs)
        if T > 0:
            _lib.pa_cache_write(bs.new_k[:T], bs.new_v[:T], bs.slots[:T], self.k_pool, self.v_pool, self.status,
                                stream=cs)
        if self.q_len > 1:
            _lib.pa_decode_multi(bs.q, self.k_pool, self.v_pool, bs.tables, bs.lens, self.scale, bs.out,
                                 self.workspace, self.status, num_ctas=self.num_ctas, flags=self.decode_flags,
                                 stream=cs)
        elif self.max_group_size > 0:
            _lib.pa_decode_shared_prefix(bs.q, self.k_pool, self.v_pool, bs.tables, bs.lens,
                                         bs.group_starts[: n_groups + 1], bs.group_prefix[:n_groups],
                                         self.max_group_size, self.scale, bs.out, self.workspace, self.status,
                                         num_ctas=self.num_ctas, flags=self.decode_flags, stream=cs)
        else:
            _lib.pa_decode(bs.q, self.k_pool, self.v_pool, bs.tables, bs.lens, self.scale, bs.out, self.workspace,
                           self.status, num_ctas=self.num_ctas, flags=self.decode_flags, stream=cs)

    def _launch_bound(self, bs, n_pairs: int, T: int, n_groups: int) -> None:
        """The same kernels through the C entry points with the buffers'
        addresses (the buffers, pools, workspace and stream never change);
        captured into a graph by ``_launch_graph``."""
        c, desc, cs, st = self._c, self._desc_ref, self._cs, self.status.data_ptr()
        kp, vp = self.k_pool.data_ptr(), self.v_pool.data_ptr()
        if n_pairs > 0:
            _check(c.pa_copy_blocks(bs.pairs.data_ptr(), n_pairs, kp, vp, st, desc, cs), "pa_copy_blocks")
        if T > 0:
            _check(c.pa_cache_write(bs.new_k.data_ptr(), bs.new_v.data_ptr(), bs.slots.data_ptr(), T, kp, vp, st,
                                    desc, cs), "pa_cache_write")
        S, max_nb = bs.tables.shape
        ws, ws_bytes = self._ws
        if self.q_len > 1:
            _check(c.pa_decode_multi(bs.q.data_ptr(), kp, vp, bs.tables.data_ptr(), max_nb, bs.lens.data_ptr(), S,
                                     self.q_len, self.Hq, self.scale, bs.out.data_ptr(), ws, ws_bytes, st, desc,
                                     self._opts_ref, cs), "pa_decode_multi")
        elif self.max_group_size > 0:
            _check(c.pa_decode_shared_prefix(bs.q.data_ptr(), kp, vp, bs.tables.data_ptr(), max_nb,
                                             bs.lens.data_ptr(), S, self.Hq, bs.group_starts.data_ptr(),
                                             bs.group_prefix.data_ptr(), n_groups, self.max_group_size, self.scale,
                                             bs.out.data_ptr(), ws, ws_bytes, st, desc, self._opts_ref, cs),
                   "pa_decode_shared_prefix")
        else:
            _check(c.pa_decode_ex(bs.q.data_ptr(), kp, vp, bs.tables.data_ptr(), max_nb, bs.lens.data_ptr(), S,
                                  self.Hq, self.scale, bs.out.data_ptr(), ws, ws_bytes, st, desc, self._opts_ref, cs),
                   "pa_decode")

    def wait(self, result) -> None:
        """Block until the step that returned ``result`` has been read back."""
        for bs in self.sets:
            if bs.out_host is result:
                bs.downloaded.synchronize()
                return
        raise ValueError("not a result of this PagedDecodeStep")

    def synchronize(self) -> None:
        for s in (self.h2d_stream, self.compute_stream, self.d2h_stream):
            s.synchronize()

    def device_status(self) -> int:
        """Synchronise every stream of the step and return the device status."""
        self.synchronize()
        return int(self.status.item())


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise _lib.PaError(rc, name)
