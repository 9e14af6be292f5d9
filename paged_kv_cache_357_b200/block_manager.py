"""Python wrapper of libpa's host block manager (C ABI in include/pa.h).

Argument marshalling only; the bookkeeping (free set, reference counts,
copy on write, batched step preparation) runs in C++ inside libpa.
"""

from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence, Tuple

import numpy as np

from . import _lib


class BmStats(ctypes.Structure):
    _fields_ = [
        ("num_blocks", ctypes.c_int32),
        ("free_blocks", ctypes.c_int32),
        ("used_blocks", ctypes.c_int32),
        ("shared_blocks", ctypes.c_int32),
        ("num_sequences", ctypes.c_int32),
        ("logical_blocks", ctypes.c_int64),
        ("tokens", ctypes.c_int64),
        ("slots_filled", ctypes.c_int64),
    ]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


def _declare(lib) -> None:
    if getattr(lib, "_pa_bm_declared", False):
        return
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    p64, p32 = ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32)
    lib.pa_bm_create.argtypes = [i32, i32]
    lib.pa_bm_create.restype = vp
    lib.pa_bm_destroy.argtypes = [vp]
    lib.pa_bm_destroy.restype = None
    lib.pa_bm_add.argtypes = [vp, i64, i32]
    lib.pa_bm_add.restype = i32
    lib.pa_bm_fork.argtypes = [vp, i64, i64]
    lib.pa_bm_fork.restype = i32
    lib.pa_bm_append.argtypes = [vp, i64, p64, p64, p64]
    lib.pa_bm_append.restype = i32
    lib.pa_bm_free.argtypes = [vp, i64]
    lib.pa_bm_free.restype = i32
    lib.pa_bm_num_free_blocks.argtypes = [vp]
    lib.pa_bm_num_free_blocks.restype = i32
    lib.pa_bm_ref_count.argtypes = [vp, i32]
    lib.pa_bm_ref_count.restype = i32
    lib.pa_bm_table.argtypes = [vp, i64, p32, i32, p32, p32]
    lib.pa_bm_table.restype = i32
    lib.pa_bm_get_stats.argtypes = [vp, ctypes.POINTER(BmStats)]
    lib.pa_bm_get_stats.restype = None
    lib.pa_bm_prepare_step.argtypes = [vp, p64, i32, i32, p32, p32, p64, p64, i32, p32]
    lib.pa_bm_prepare_step.restype = i32
    lib._pa_bm_declared = True


class BlockManager:
    """On-demand block allocation with reference counts and copy on write."""

    def __init__(self, num_blocks: int, block_size: int):
        self._lib = _lib.load()
        _declare(self._lib)
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self._h = self._lib.pa_bm_create(self.num_blocks, self.block_size)
        if not self._h:
            raise _lib.PaError(1, "pa_bm_create")

    def close(self) -> None:
        if self._h:
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, rc: int, where: str) -> None:
        if rc != 0:
            raise _lib.PaError(rc, where)

    def add(self, seq_id: int, num_tokens: int) -> None:
        self._check(self._lib.pa_bm_add(self._h, seq_id, num_tokens), "pa_bm_add")

    def fork(self, parent_id: int, child_id: int) -> None:
        self._check(self._lib.pa_bm_fork(self._h, parent_id, child_id), "pa_bm_fork")

    def append(self, seq_id: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        self._check(self._lib.pa_bm_append(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)),
                    "pa_bm_append")
        return slot.value, ((src.value, dst.value) if src.value >= 0 else None)

    def free(self, seq_id: int) -> None:
        self._check(self._lib.pa_bm_free(self._h, seq_id), "pa_bm_free")

    @property
    def num_free(self) -> int:
        return int(self._lib.pa_bm_num_free_blocks(self._h))

    def ref_count(self, block: int) -> int:
        return int(self._lib.pa_bm_ref_count(self._h, block))

    def table(self, seq_id: int) -> Tuple[List[int], int]:
        nb, nt = ctypes.c_int32(), ctypes.c_int32()
        self._lib.pa_bm_table(self._h, seq_id, None, 0, ctypes.byref(nb), ctypes.byref(nt))
        buf = (ctypes.c_int32 * max(nb.value, 1))()
        self._check(self._lib.pa_bm_table(self._h, seq_id, buf, len(buf), ctypes.byref(nb), ctypes.byref(nt)),
                    "pa_bm_table")
        return list(buf[: nb.value]), nt.value

    def stats(self) -> dict:
        st = BmStats()
        self._lib.pa_bm_get_stats(self._h, ctypes.byref(st))
        return st.as_dict()

    def prepare_step(self, seq_ids: Sequence[int], max_blocks_per_seq: int, max_pairs: Optional[int] = None):
        """Append one token to each sequence; returns numpy (block_tables,
        seq_lens, slot_mapping, copy_pairs) ready for the kernels."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        max_pairs = n if max_pairs is None else max_pairs
        tables = np.empty((n, max_blocks_per_seq), np.int32)
        lens = np.empty(n, np.int32)
        slots = np.empty(n, np.int64)
        pairs = np.empty((max(max_pairs, 1), 2), np.int64)
        npairs = ctypes.c_int32()
        p64, p32 = ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32)
        rc = self._lib.pa_bm_prepare_step(
            self._h, ids.ctypes.data_as(p64), n, max_blocks_per_seq, tables.ctypes.data_as(p32),
            lens.ctypes.data_as(p32), slots.ctypes.data_as(p64), pairs.ctypes.data_as(p64), max_pairs,
            ctypes.byref(npairs))
        self._check(rc, "pa_bm_prepare_step")
        return tables, lens, slots, pairs[: npairs.value].copy()
