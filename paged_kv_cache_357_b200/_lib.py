"""ctypes binding of libpa (C ABI declared in include/pa.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their device pointers and sizes are passed to the C entry points,
and non-zero return codes become ``PaError``.  Every step of the hot path runs
in libpa's CUDA kernels; there is no fallback of any kind — if libpa.so is
missing the import of the functions below raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpa.so")

PA_FP16, PA_BF16 = 0, 1
PA_DECODE_TEST_WITHHOLD_COPIES = 1
PA_DECODE_CUDA_CORES_ONLY = 2
PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL = 4
DEV_STATUS = {
    0: "PA_DEV_OK",
    101: "PA_DEV_BAD_BLOCK_ID",
    102: "PA_DEV_BAD_SEQ_LEN",
    103: "PA_DEV_BAD_SLOT",
    104: "PA_DEV_BAD_PAIR",
    105: "PA_DEV_TIMEOUT",
    106: "PA_DEV_BAD_GROUP",
}
EXPORTED = (
    "pa_decode_workspace_bytes",
    "pa_decode_workspace_bytes_ex",
    "pa_decode",
    "pa_decode_ex",
    "pa_decode_no_alloc",
    "pa_decode_multi_workspace_bytes",
    "pa_decode_multi",
    "pa_decode_shared_prefix_workspace_bytes",
    "pa_decode_shared_prefix",
    "pa_shared_prefix_groups",
    "pa_cache_write",
    "pa_copy_blocks",
    "pa_decode_update",
    "pa_decode_lse",
    "pa_merge_partials",
    "pa_decode_multi_update",
    "pa_decode_shared_prefix_update",
    "pa_status_string",
    "pa_bm_create",
    "pa_bm_destroy",
    "pa_bm_add",
    "pa_bm_fork",
    "pa_bm_append",
    "pa_bm_free",
    "pa_bm_num_free_blocks",
    "pa_bm_ref_count",
    "pa_bm_table",
    "pa_bm_get_stats",
    "pa_bm_prepare_step",
    "pa_step_layout_of",
    "pa_step_create",
    "pa_step_next_set",
    "pa_step_run",
    "pa_step_wait",
    "pa_step_flush",
    "pa_step_synchronize",
    "pa_step_streams",
    "pa_step_destroy",
)

PA_STEP_DECODE, PA_STEP_MULTI, PA_STEP_SHARED_PREFIX = 0, 1, 2
PA_STEP_MAX_SETS = 8


class PoolDesc(ctypes.Structure):
    _fields_ = [
        ("num_blocks", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


class DecodeOpts(ctypes.Structure):
    _fields_ = [("num_ctas", ctypes.c_int32), ("flags", ctypes.c_int32)]


class CacheUpdate(ctypes.Structure):
    _fields_ = [
        ("copy_pairs", ctypes.c_void_p),
        ("num_copy_pairs", ctypes.c_int32),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("slot_mapping", ctypes.c_void_p),
        ("num_tokens", ctypes.c_int32),
    ]


class StepShape(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("num_seqs", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("q_len", ctypes.c_int32),
        ("max_group_size", ctypes.c_int32),
        ("max_new_tokens", ctypes.c_int32),
        ("max_copy_pairs", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("opts", DecodeOpts),
    ]


STEP_FIELDS = ("q", "block_tables", "seq_lens", "group_starts", "group_prefix_blocks", "copy_pairs", "new_k", "new_v",
               "slot_mapping")


class StepLayout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_size_t) for name in STEP_FIELDS] + [("total", ctypes.c_size_t),
                                                                     ("out_bytes", ctypes.c_size_t)]


class PaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: libpa returned {code} ({status_string(code)})")


_LIB: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpa.so and declare its signatures (raises if it is not built)."""
    global _LIB
    if _LIB is not None and path == LIB_PATH:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(
            f"libpa.so not found at {path}; build it with `python -m paged_kv_cache_357_b200.build` "
            "(there is no fallback implementation)"
        )
    lib = ctypes.CDLL(path)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    pdesc, popts = ctypes.POINTER(PoolDesc), ctypes.POINTER(DecodeOpts)
    lib.pa_decode_workspace_bytes.argtypes = [i32, i32, pdesc]
    lib.pa_decode_workspace_bytes.restype = sz
    lib.pa_decode_workspace_bytes_ex.argtypes = [i32, i32, pdesc, popts]
    lib.pa_decode_workspace_bytes_ex.restype = sz
    lib.pa_decode.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, f32, vp, vp, sz, vp, pdesc, vp]
    lib.pa_decode.restype = i32
    lib.pa_decode_ex.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, f32, vp, vp, sz, vp, pdesc, popts, vp]
    lib.pa_decode_ex.restype = i32
    lib.pa_decode_no_alloc.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, f32, vp, vp, pdesc, vp]
    lib.pa_decode_no_alloc.restype = i32
    lib.pa_decode_multi_workspace_bytes.argtypes = [i32, i32, i32, pdesc, popts]
    lib.pa_decode_multi_workspace_bytes.restype = sz
    lib.pa_decode_multi.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, f32, vp, vp, sz, vp, pdesc, popts, vp]
    lib.pa_decode_multi.restype = i32
    lib.pa_decode_shared_prefix_workspace_bytes.argtypes = [i32, i32, i32, pdesc, popts]
    lib.pa_decode_shared_prefix_workspace_bytes.restype = sz
    lib.pa_decode_shared_prefix.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, vp, vp, i32, i32, f32, vp, vp, sz,
                                            vp, pdesc, popts, vp]
    lib.pa_decode_shared_prefix.restype = i32
    lib.pa_shared_prefix_groups.argtypes = [vp, i32, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.pa_shared_prefix_groups.restype = i32
    lib.pa_cache_write.argtypes = [vp, vp, vp, i32, vp, vp, vp, pdesc, vp]
    lib.pa_cache_write.restype = i32
    lib.pa_copy_blocks.argtypes = [vp, i32, vp, vp, vp, pdesc, vp]
    pupd = ctypes.POINTER(CacheUpdate)
    lib.pa_decode_update.argtypes = [pupd] + lib.pa_decode_ex.argtypes
    lib.pa_decode_multi_update.argtypes = [pupd] + lib.pa_decode_multi.argtypes
    lib.pa_decode_shared_prefix_update.argtypes = [pupd] + lib.pa_decode_shared_prefix.argtypes
    for name in ("pa_decode_update", "pa_decode_multi_update", "pa_decode_shared_prefix_update"):
        getattr(lib, name).restype = i32
    lib.pa_decode_lse.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, f32, vp, vp, vp, sz, vp, pdesc, popts, vp]
    lib.pa_decode_lse.restype = i32
    lib.pa_merge_partials.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.pa_merge_partials.restype = i32
    lib.pa_copy_blocks.restype = i32
    pshape, playout = ctypes.POINTER(StepShape), ctypes.POINTER(StepLayout)
    vpp = ctypes.POINTER(ctypes.c_void_p)
    lib.pa_step_layout_of.argtypes = [pshape, pdesc, playout]
    lib.pa_step_layout_of.restype = i32
    lib.pa_step_create.argtypes = [pshape, pdesc, vp, vp, vp, sz, vp, i32, vpp, vpp, vpp, vpp, vpp]
    lib.pa_step_create.restype = i32
    lib.pa_step_next_set.argtypes = [vp, ctypes.POINTER(i32)]
    lib.pa_step_next_set.restype = i32
    lib.pa_step_run.argtypes = [vp, i32, i32, i32, ctypes.POINTER(i32)]
    lib.pa_step_run.restype = i32
    lib.pa_step_wait.argtypes = [vp, i32]
    lib.pa_step_wait.restype = i32
    lib.pa_step_flush.argtypes = [vp]
    lib.pa_step_flush.restype = i32
    lib.pa_step_synchronize.argtypes = [vp]
    lib.pa_step_synchronize.restype = i32
    lib.pa_step_streams.argtypes = [vp, vpp, vpp, vpp]
    lib.pa_step_streams.restype = i32
    lib.pa_step_destroy.argtypes = [vp]
    lib.pa_step_destroy.restype = None
    lib.pa_status_string.argtypes = [i32]
    lib.pa_status_string.restype = ctypes.c_char_p
    if path == LIB_PATH:
        _LIB = lib
    return lib


def status_string(code: int) -> str:
    return load().pa_status_string(int(code)).decode()


# ---------------------------------------------------------------------------
# torch-facing helpers (device memory and streams come from PyTorch)
# ---------------------------------------------------------------------------


def _torch():
    import torch

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return PA_FP16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"expected fp16 or bf16, got {t.dtype}")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _need(t, name, *, dtype=None, ndim=None, device=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def pool_desc(k_pool) -> PoolDesc:
    """Descriptor of a [num_blocks, num_kv_heads, block_size, head_dim] pool."""
    nb, hkv, bs, d = k_pool.shape
    return PoolDesc(nb, bs, hkv, d, _dtype_code(k_pool))


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, k_pool, num_ctas: int = 0, flags: int = 0) -> int:
    """Workspace bytes for pa_decode with the same num_ctas and flags."""
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    n = load().pa_decode_workspace_bytes_ex(num_seqs, num_q_heads, ctypes.byref(desc), ctypes.byref(opts))
    if n == 0:
        raise PaError(1, "pa_decode_workspace_bytes")
    return int(n)


def alloc_decode_workspace(num_seqs: int, num_q_heads: int, k_pool, num_ctas: int = 0, flags: int = 0):
    """Zeroed device workspace for pa_decode with the same num_ctas and flags
    (see include/pa.h)."""
    torch = _torch()
    n = decode_workspace_bytes(num_seqs, num_q_heads, k_pool, num_ctas, flags)
    return torch.zeros(n, dtype=torch.uint8, device=k_pool.device)


def pa_decode(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, workspace, dev_status=None,
              num_ctas: int = 0, flags: int = 0, stream=None) -> None:
    """out[s, h] = softmax(scale * q[s, h] . K^T) V over seq_lens[s] paged tokens (pa_decode_ex)."""
    torch = _torch()
    _need(k_pool, "k_pool", ndim=4)
    dev = k_pool.device
    _need(v_pool, "v_pool", dtype=k_pool.dtype, ndim=4, device=dev)
    if v_pool.shape != k_pool.shape:
        raise ValueError("k_pool and v_pool shapes differ")
    _need(q, "q", dtype=k_pool.dtype, ndim=3, device=dev)
    _need(out, "out", dtype=k_pool.dtype, ndim=3, device=dev)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2, device=dev)
    _need(seq_lens, "seq_lens", dtype=torch.int32, ndim=1, device=dev)
    _need(workspace, "workspace", device=dev)
    S, Hq, D = q.shape
    if block_tables.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_tables / seq_lens must have num_seqs rows")
    if D != k_pool.shape[3]:
        raise ValueError("head_dim of q and the pools differ")
    if dev_status is not None:
        _need(dev_status, "dev_status", dtype=torch.int32, device=dev)
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_ex(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), S, Hq,
        float(scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
        ctypes.byref(desc), ctypes.byref(opts), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode")


def _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, q_ndim):
    torch = _torch()
    _need(k_pool, "k_pool", ndim=4)
    dev = k_pool.device
    _need(v_pool, "v_pool", dtype=k_pool.dtype, ndim=4, device=dev)
    if v_pool.shape != k_pool.shape:
        raise ValueError("k_pool and v_pool shapes differ")
    _need(q, "q", dtype=k_pool.dtype, ndim=q_ndim, device=dev)
    _need(out, "out", dtype=k_pool.dtype, ndim=q_ndim, device=dev)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2, device=dev)
    _need(seq_lens, "seq_lens", dtype=torch.int32, ndim=1, device=dev)
    _need(workspace, "workspace", device=dev)
    S = q.shape[0]
    if block_tables.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_tables / seq_lens must have num_seqs rows")
    if q.shape[-1] != k_pool.shape[3]:
        raise ValueError("head_dim of q and the pools differ")
    if dev_status is not None:
        _need(dev_status, "dev_status", dtype=torch.int32, device=dev)


def multi_workspace_bytes(num_seqs: int, q_len: int, num_q_heads: int, k_pool, num_ctas: int = 0,
                          flags: int = 0) -> int:
    """Workspace bytes for pa_decode_multi with the same num_ctas and flags."""
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    n = load().pa_decode_multi_workspace_bytes(num_seqs, q_len, num_q_heads, ctypes.byref(desc),
                                               ctypes.byref(opts))
    if n == 0:
        raise PaError(2, "pa_decode_multi_workspace_bytes")
    return int(n)


def alloc_multi_workspace(num_seqs: int, q_len: int, num_q_heads: int, k_pool, num_ctas: int = 0, flags: int = 0):
    """Zeroed device workspace for pa_decode_multi."""
    torch = _torch()
    n = multi_workspace_bytes(num_seqs, q_len, num_q_heads, k_pool, num_ctas, flags)
    return torch.zeros(n, dtype=torch.uint8, device=k_pool.device)


def pa_decode_multi(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, workspace, dev_status=None,
                    num_ctas: int = 0, flags: int = 0, stream=None) -> None:
    """Causal attention of q_len new positions per sequence over the paged
    cache (pa_decode_multi): q, out are [num_seqs, q_len, num_q_heads, head_dim]."""
    _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, 4)
    S, L, Hq, D = q.shape
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_multi(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), S, L, Hq,
        float(scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
        ctypes.byref(desc), ctypes.byref(opts), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_multi")


def shared_prefix_workspace_bytes(num_seqs: int, max_group_size: int, num_q_heads: int, k_pool, num_ctas: int = 0,
                                  flags: int = 0) -> int:
    """Workspace bytes for pa_decode_shared_prefix with the same num_ctas and flags."""
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    n = load().pa_decode_shared_prefix_workspace_bytes(num_seqs, max_group_size, num_q_heads, ctypes.byref(desc),
                                                       ctypes.byref(opts))
    if n == 0:
        raise PaError(2, "pa_decode_shared_prefix_workspace_bytes")
    return int(n)


def alloc_shared_prefix_workspace(num_seqs: int, max_group_size: int, num_q_heads: int, k_pool, num_ctas: int = 0,
                                  flags: int = 0):
    """Zeroed device workspace for pa_decode_shared_prefix."""
    torch = _torch()
    n = shared_prefix_workspace_bytes(num_seqs, max_group_size, num_q_heads, k_pool, num_ctas, flags)
    return torch.zeros(n, dtype=torch.uint8, device=k_pool.device)


def pa_decode_shared_prefix(q, k_pool, v_pool, block_tables, seq_lens, group_starts, group_prefix_blocks,
                            max_group_size: int, scale: float, out, workspace, dev_status=None, num_ctas: int = 0,
                            flags: int = 0, stream=None) -> None:
    """pa_decode reading each group's shared leading blocks once
    (pa_decode_shared_prefix); group_starts [G + 1] and group_prefix_blocks [G]
    are int32 device tensors (see shared_prefix_groups)."""
    torch = _torch()
    _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, 3)
    dev = k_pool.device
    _need(group_starts, "group_starts", dtype=torch.int32, ndim=1, device=dev)
    _need(group_prefix_blocks, "group_prefix_blocks", dtype=torch.int32, ndim=1, device=dev)
    G = group_prefix_blocks.shape[0]
    if group_starts.shape[0] != G + 1:
        raise ValueError("group_starts must have num_groups + 1 entries")
    S, Hq, D = q.shape
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_shared_prefix(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), S, Hq,
        _ptr(group_starts), _ptr(group_prefix_blocks), G, int(max_group_size), float(scale), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status), ctypes.byref(desc),
        ctypes.byref(opts), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_shared_prefix")


def shared_prefix_groups(block_tables, seq_lens, block_size: int, max_group_size: int, min_prefix_blocks: int = 1):
    """Groups for pa_decode_shared_prefix from host (numpy int32) tables and
    lengths (pa_shared_prefix_groups): returns (group_starts, group_prefix_blocks)."""
    import numpy as np

    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    if bt.ndim != 2 or sl.ndim != 1 or bt.shape[0] != sl.shape[0]:
        raise ValueError("block_tables [S, max_nb] and seq_lens [S] expected")
    S = bt.shape[0]
    starts = np.zeros(S + 1, np.int32)
    prefix = np.zeros(max(S, 1), np.int32)
    ng = ctypes.c_int32(0)
    rc = load().pa_shared_prefix_groups(
        bt.ctypes.data, bt.shape[1], sl.ctypes.data, S, block_size, max_group_size, min_prefix_blocks,
        starts.ctypes.data, prefix.ctypes.data, ctypes.byref(ng),
    )
    if rc != 0:
        raise PaError(rc, "pa_shared_prefix_groups")
    n = ng.value
    return starts[: n + 1].copy(), prefix[:n].copy()


def pa_decode_no_alloc(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, dev_status=None,
                       stream=None) -> None:
    """pa_decode without a caller workspace, for callers that may not
    allocate device memory: the scratch is libpa's own fixed device array
    (8 MiB per device).  Calls that may overlap on the GPU race; order them.
    The first call on a device looks up the array's address, so make it
    before any stream capture."""
    torch = _torch()
    _need(k_pool, "k_pool", ndim=4)
    dev = k_pool.device
    _need(v_pool, "v_pool", dtype=k_pool.dtype, ndim=4, device=dev)
    _need(q, "q", dtype=k_pool.dtype, ndim=3, device=dev)
    _need(out, "out", dtype=k_pool.dtype, ndim=3, device=dev)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2, device=dev)
    _need(seq_lens, "seq_lens", dtype=torch.int32, ndim=1, device=dev)
    S, Hq, D = q.shape
    if out.shape != q.shape or block_tables.shape[0] != S or seq_lens.shape[0] != S or D != k_pool.shape[3]:
        raise ValueError("shapes of q, out, block_tables, seq_lens and the pools disagree")
    if dev_status is not None:
        _need(dev_status, "dev_status", dtype=torch.int32, device=dev)
    desc = pool_desc(k_pool)
    rc = load().pa_decode_no_alloc(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), S, Hq,
        float(scale), _ptr(out), _ptr(dev_status), ctypes.byref(desc), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_no_alloc")


def pa_cache_write(k, v, slot_mapping, k_pool, v_pool, dev_status=None, stream=None) -> None:
    """Store new tokens' K/V ([T, Hkv, D]) into their slots (pa_cache_write)."""
    torch = _torch()
    _need(k_pool, "k_pool", ndim=4)
    dev = k_pool.device
    _need(v_pool, "v_pool", dtype=k_pool.dtype, ndim=4, device=dev)
    _need(k, "k", dtype=k_pool.dtype, ndim=3, device=dev)
    _need(v, "v", dtype=k_pool.dtype, ndim=3, device=dev)
    _need(slot_mapping, "slot_mapping", dtype=torch.int64, ndim=1, device=dev)
    T = k.shape[0]
    if v.shape != k.shape or slot_mapping.shape[0] != T:
        raise ValueError("k, v and slot_mapping disagree on the token count")
    if k.shape[1:] != (k_pool.shape[1], k_pool.shape[3]):
        raise ValueError("new tokens must be [T, num_kv_heads, head_dim]")
    if dev_status is not None:
        _need(dev_status, "dev_status", dtype=torch.int32, device=dev)
    desc = pool_desc(k_pool)
    rc = load().pa_cache_write(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_pool), _ptr(v_pool),
                               _ptr(dev_status), ctypes.byref(desc), _stream(stream))
    if rc != 0:
        raise PaError(rc, "pa_cache_write")


def pa_copy_blocks(src_dst_pairs, k_pool, v_pool, dev_status=None, stream=None) -> None:
    """Copy-on-write block copies: block dst of both pools <- block src (pa_copy_blocks)."""
    torch = _torch()
    _need(k_pool, "k_pool", ndim=4)
    dev = k_pool.device
    _need(v_pool, "v_pool", dtype=k_pool.dtype, ndim=4, device=dev)
    _need(src_dst_pairs, "src_dst_pairs", dtype=torch.int64, ndim=2, device=dev)
    if src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [n, 2]")
    if dev_status is not None:
        _need(dev_status, "dev_status", dtype=torch.int32, device=dev)
    desc = pool_desc(k_pool)
    rc = load().pa_copy_blocks(_ptr(src_dst_pairs), src_dst_pairs.shape[0], _ptr(k_pool), _ptr(v_pool),
                               _ptr(dev_status), ctypes.byref(desc), _stream(stream))
    if rc != 0:
        raise PaError(rc, "pa_copy_blocks")


# ---------------------------------------------------------------------------
# a step's cache update and its decode in one call (pa_decode_update & co.)
# ---------------------------------------------------------------------------


def _cache_update(k_pool, copy_pairs, new_k, new_v, slot_mapping) -> CacheUpdate:
    """The pa_cache_update struct of a step: copy-on-write pairs [n, 2] int64,
    then new tokens' k, v [T, num_kv_heads, head_dim] into slot_mapping [T]
    int64; either part may be None."""
    torch = _torch()
    dev = k_pool.device
    upd = CacheUpdate()
    if copy_pairs is not None:
        _need(copy_pairs, "copy_pairs", dtype=torch.int64, ndim=2, device=dev)
        if copy_pairs.shape[1] != 2:
            raise ValueError("copy_pairs must be [n, 2]")
        upd.copy_pairs, upd.num_copy_pairs = _ptr(copy_pairs), copy_pairs.shape[0]
    if (new_k is None) != (new_v is None) or (new_k is None) != (slot_mapping is None):
        raise ValueError("new_k, new_v and slot_mapping go together")
    if new_k is not None:
        _need(new_k, "new_k", dtype=k_pool.dtype, ndim=3, device=dev)
        _need(new_v, "new_v", dtype=k_pool.dtype, ndim=3, device=dev)
        _need(slot_mapping, "slot_mapping", dtype=torch.int64, ndim=1, device=dev)
        T = new_k.shape[0]
        if new_v.shape != new_k.shape or slot_mapping.shape[0] != T:
            raise ValueError("new_k, new_v and slot_mapping disagree on the token count")
        if new_k.shape[1:] != (k_pool.shape[1], k_pool.shape[3]):
            raise ValueError("new tokens must be [T, num_kv_heads, head_dim]")
        upd.k, upd.v, upd.slot_mapping, upd.num_tokens = _ptr(new_k), _ptr(new_v), _ptr(slot_mapping), T
    return upd


def pa_decode_update(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, workspace, dev_status=None,
                     copy_pairs=None, new_k=None, new_v=None, slot_mapping=None, num_ctas: int = 0, flags: int = 0,
                     stream=None) -> None:
    """pa_copy_blocks, pa_cache_write and pa_decode as one call
    (pa_decode_update): one launch where the tensor-core kernel runs."""
    _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, 3)
    upd = _cache_update(k_pool, copy_pairs, new_k, new_v, slot_mapping)
    S, Hq, D = q.shape
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_update(
        ctypes.byref(upd), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(seq_lens), S, Hq, float(scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_status), ctypes.byref(desc), ctypes.byref(opts), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_update")


def pa_decode_multi_update(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, workspace, dev_status=None,
                           copy_pairs=None, new_k=None, new_v=None, slot_mapping=None, num_ctas: int = 0,
                           flags: int = 0, stream=None) -> None:
    """pa_copy_blocks, pa_cache_write and pa_decode_multi as one call
    (pa_decode_multi_update)."""
    _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, 4)
    upd = _cache_update(k_pool, copy_pairs, new_k, new_v, slot_mapping)
    S, L, Hq, D = q.shape
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_multi_update(
        ctypes.byref(upd), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(seq_lens), S, L, Hq, float(scale), _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), ctypes.byref(desc), ctypes.byref(opts),
        _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_multi_update")


def pa_decode_shared_prefix_update(q, k_pool, v_pool, block_tables, seq_lens, group_starts, group_prefix_blocks,
                                   max_group_size: int, scale: float, out, workspace, dev_status=None,
                                   copy_pairs=None, new_k=None, new_v=None, slot_mapping=None, num_ctas: int = 0,
                                   flags: int = 0, stream=None) -> None:
    """pa_copy_blocks, pa_cache_write and pa_decode_shared_prefix as one call
    (pa_decode_shared_prefix_update)."""
    torch = _torch()
    _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, 3)
    dev = k_pool.device
    _need(group_starts, "group_starts", dtype=torch.int32, ndim=1, device=dev)
    _need(group_prefix_blocks, "group_prefix_blocks", dtype=torch.int32, ndim=1, device=dev)
    G = group_prefix_blocks.shape[0]
    if group_starts.shape[0] != G + 1:
        raise ValueError("group_starts must have num_groups + 1 entries")
    upd = _cache_update(k_pool, copy_pairs, new_k, new_v, slot_mapping)
    S, Hq, D = q.shape
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_shared_prefix_update(
        ctypes.byref(upd), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(seq_lens), S, Hq, _ptr(group_starts), _ptr(group_prefix_blocks), G, int(max_group_size), float(scale),
        _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
        ctypes.byref(desc), ctypes.byref(opts), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_shared_prefix_update")


# ---------------------------------------------------------------------------
# decodes of disjoint token ranges and their merge (pa_decode_lse, pa_merge_partials)
# ---------------------------------------------------------------------------


def pa_decode_lse(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, lse, workspace, dev_status=None,
                  num_ctas: int = 0, flags: int = 0, stream=None) -> None:
    """pa_decode that also writes lse [num_seqs, num_q_heads] float32, the
    natural log of each row's softmax normaliser (pa_decode_lse)."""
    torch = _torch()
    _check_attention_args(q, k_pool, v_pool, block_tables, seq_lens, out, workspace, dev_status, 3)
    S, Hq, D = q.shape
    _need(lse, "lse", dtype=torch.float32, ndim=2, device=k_pool.device)
    if tuple(lse.shape) != (S, Hq):
        raise ValueError("lse must be [num_seqs, num_q_heads]")
    desc = pool_desc(k_pool)
    opts = DecodeOpts(num_ctas, flags)
    rc = load().pa_decode_lse(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), S, Hq,
        float(scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_status), ctypes.byref(desc), ctypes.byref(opts), _stream(stream),
    )
    if rc != 0:
        raise PaError(rc, "pa_decode_lse")


def pa_merge_partials(outs, lses, out, lse_out=None, stream=None) -> None:
    """Merge decodes of disjoint token ranges of the same rows
    (pa_merge_partials): outs [R, ..., head_dim] fp16/bf16 and lses [R, ...]
    float32 from pa_decode_lse; out [..., head_dim], lse_out [...] (optional)."""
    torch = _torch()
    _need(outs, "outs")
    dev = outs.device
    _need(lses, "lses", dtype=torch.float32, device=dev)
    _need(out, "out", dtype=outs.dtype, device=dev)
    R, D = outs.shape[0], outs.shape[-1]
    rows = out.numel() // D if D else 0
    if tuple(outs.shape[1:]) != tuple(out.shape) or tuple(lses.shape) != (R,) + tuple(out.shape[:-1]):
        raise ValueError("outs [R, ..., D], lses [R, ...] and out [..., D] disagree")
    if lse_out is not None:
        _need(lse_out, "lse_out", dtype=torch.float32, device=dev)
        if tuple(lse_out.shape) != tuple(out.shape[:-1]):
            raise ValueError("lse_out must have out's shape without head_dim")
    rc = load().pa_merge_partials(_ptr(outs), _ptr(lses), R, rows, D, _dtype_code(outs), _ptr(out), _ptr(lse_out),
                                  _stream(stream))
    if rc != 0:
        raise PaError(rc, "pa_merge_partials")
