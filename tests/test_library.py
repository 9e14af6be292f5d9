"""The C-ABI library loads, exports every entry point include/pa.h declares,
and rejects bad arguments on the host before touching a GPU (no compute
call runs here)."""

import ctypes
import re
from pathlib import Path

import pytest

import paged_kv_cache_357_b200 as pa
from paged_kv_cache_357_b200 import _lib
from paged_kv_cache_357_b200 import build as pa_build

HEADER = Path(__file__).resolve().parents[1] / "include" / "pa.h"


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return _lib.load()


def declared_entry_points():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"^PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for required in ["pa_decode", "pa_cache_write", "pa_copy_blocks", "pa_decode_workspace_bytes",
                     "pa_status_string"]:
        assert required in names
    assert set(names) == set(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_library_exports_nothing_else(lib):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {n for n in exported if n.startswith("pa_")} == set(declared_entry_points())


def test_status_strings(lib):
    for code in [0, 1, 2, 3, 4, 5, 6, 101, 102, 103, 104, 105, 106]:
        assert pa.status_string(code) != "unknown status"
    assert pa.status_string(12345) == "unknown status"


def _desc(**kw):
    d = dict(num_blocks=64, block_size=16, num_kv_heads=4, head_dim=64, dtype=_lib.PA_FP16)
    d.update(kw)
    return _lib.PoolDesc(**d)


FAKE = 0x100000  # 16-byte aligned, never dereferenced: every case below fails validation first


def _decode(lib, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, max_nb=8, lens=FAKE, S=4, Hq=4, scale=0.125, out=FAKE,
            ws=FAKE, ws_bytes=1 << 20, desc=None):
    desc = desc or _desc()
    return lib.pa_decode(q, k, v, tables, max_nb, lens, S, Hq, scale, out, ws, ws_bytes, None, ctypes.byref(desc),
                         None)


def test_decode_rejects_bad_arguments_on_host(lib):
    assert _decode(lib, S=0) == 0  # empty batch is a no-op
    assert _decode(lib, q=None) == 1
    assert _decode(lib, out=None) == 1
    assert _decode(lib, tables=None) == 1
    assert _decode(lib, q=FAKE + 2) == 1  # misaligned
    assert _decode(lib, S=-1) == 1
    assert _decode(lib, max_nb=0) == 1
    assert _decode(lib, scale=float("nan")) == 1
    assert _decode(lib, desc=_desc(dtype=7)) == 1
    assert _decode(lib, desc=_desc(num_blocks=0)) == 1
    assert _decode(lib, Hq=6) == 1 or _decode(lib, Hq=6) == 2  # 6 % 4 != 0
    assert _decode(lib, Hq=12) == 2  # group 3: no kernel
    assert _decode(lib, desc=_desc(block_size=24)) == 2
    assert _decode(lib, desc=_desc(head_dim=96)) == 2


def test_workspace_query_rejects_bad_arguments(lib):
    d = _desc(head_dim=96)
    assert lib.pa_decode_workspace_bytes(4, 4, ctypes.byref(d)) == 0
    d = _desc()
    assert lib.pa_decode_workspace_bytes(-1, 4, ctypes.byref(d)) == 0
    assert lib.pa_decode_workspace_bytes(4, 12, ctypes.byref(d)) == 0
    opts = _lib.DecodeOpts(7, 0)
    # an explicit CTA count needs no device query
    n = lib.pa_decode_workspace_bytes_ex(4, 4, ctypes.byref(d), ctypes.byref(opts))
    assert n >= 7 * 2 * 1 * (64 + 2) * 4 + 4 * 4


def _multi(lib, q_len=4, S=4, Hq=16, desc=None, flags=0, ws=FAKE):
    desc = desc or _desc(head_dim=128)
    opts = _lib.DecodeOpts(0, flags)
    return lib.pa_decode_multi(FAKE, FAKE, FAKE, FAKE, 8, FAKE, S, q_len, Hq, 0.1, FAKE, ws, 1 << 20, None,
                               ctypes.byref(desc), ctypes.byref(opts), None)


def test_multi_rejects_bad_arguments_on_host(lib):
    assert _multi(lib, S=0) == 0
    assert _multi(lib, q_len=0) == 1
    assert _multi(lib, q_len=-3) == 1
    assert _multi(lib, Hq=12) == 2                     # group 3
    assert _multi(lib, q_len=16) not in (1, 2)         # 4 heads x 16 positions: two row tiles per sequence
    assert _multi(lib, desc=_desc(head_dim=64)) == 2   # tensor-core kernel only
    assert _multi(lib, flags=_lib.PA_DECODE_CUDA_CORES_ONLY) == 2
    assert _multi(lib, flags=64) == 1                  # unknown flag
    d = _desc(head_dim=128)
    opts = _lib.DecodeOpts(7, 0)
    n = lib.pa_decode_multi_workspace_bytes(4, 4, 16, ctypes.byref(d), ctypes.byref(opts))
    assert n >= 7 * 2 * 16 * (128 + 2) * 4 + 4 * 4
    # 4 heads x 16 positions: units of 32 rows, two row tiles (units) per sequence
    n16 = lib.pa_decode_multi_workspace_bytes(4, 16, 16, ctypes.byref(d), ctypes.byref(opts))
    assert n16 >= 7 * 2 * 32 * (128 + 2) * 4 + 4 * 2 * 4 * 4
    assert lib.pa_decode_multi_workspace_bytes(4, 0, 16, ctypes.byref(d), ctypes.byref(opts)) == 0


def _prefix(lib, S=4, G=2, starts=FAKE, prefix=FAKE, max_group=2, Hq=8, desc=None):
    desc = desc or _desc(head_dim=128)
    return lib.pa_decode_shared_prefix(FAKE, FAKE, FAKE, FAKE, 8, FAKE, S, Hq, starts, prefix, G, max_group, 0.1,
                                       FAKE, FAKE, 1 << 20, None, ctypes.byref(desc), None, None)


def test_shared_prefix_rejects_bad_arguments_on_host(lib):
    assert _prefix(lib, S=0, G=0) == 0
    assert _prefix(lib, G=0) == 1          # sequences but no groups
    assert _prefix(lib, G=5) == 1          # more groups than sequences
    assert _prefix(lib, starts=None) == 1
    assert _prefix(lib, prefix=None) == 1
    assert _prefix(lib, max_group=0) == 1
    assert _prefix(lib, max_group=16, Hq=16) == 2  # 4 heads x 16 members > 32 rows
    assert _prefix(lib, desc=_desc(head_dim=64)) == 2
    d = _desc(head_dim=128)
    opts = _lib.DecodeOpts(5, 0)
    n = lib.pa_decode_shared_prefix_workspace_bytes(4, 2, 8, ctypes.byref(d), ctypes.byref(opts))
    # partial states of 2 members x 2 heads per kv head (two slots per CTA), counters per (seq, kv head)
    assert n >= 5 * 2 * 4 * 130 * 4 + 4 * 4 * 4
    assert lib.pa_decode_shared_prefix_workspace_bytes(4, 0, 8, ctypes.byref(d), ctypes.byref(opts)) == 0


def test_cache_write_and_copy_reject_bad_arguments(lib):
    d = _desc()
    assert lib.pa_cache_write(FAKE, FAKE, FAKE, 0, FAKE, FAKE, None, ctypes.byref(d), None) == 0
    assert lib.pa_cache_write(FAKE, FAKE, FAKE, -1, FAKE, FAKE, None, ctypes.byref(d), None) == 1
    assert lib.pa_cache_write(None, FAKE, FAKE, 4, FAKE, FAKE, None, ctypes.byref(d), None) == 1
    assert lib.pa_cache_write(FAKE, FAKE, FAKE, 4, FAKE + 8, FAKE, None, ctypes.byref(d), None) == 1
    bad = _desc(head_dim=12)
    assert lib.pa_cache_write(FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, ctypes.byref(bad), None) == 1
    assert lib.pa_copy_blocks(FAKE, 0, FAKE, FAKE, None, ctypes.byref(d), None) == 0
    assert lib.pa_copy_blocks(None, 3, FAKE, FAKE, None, ctypes.byref(d), None) == 1
    assert lib.pa_copy_blocks(FAKE, -2, FAKE, FAKE, None, ctypes.byref(d), None) == 1


def test_python_binding_checks_tensors_before_calling():
    import torch

    kp = torch.zeros((4, 2, 16, 64), dtype=torch.float16)
    with pytest.raises(ValueError):
        pa.pa_cache_write(kp[0], kp[0], torch.zeros(2, dtype=torch.int64), kp, kp)  # CPU tensors


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        _lib.load(str(tmp_path / "libpa.so"))


def _step_shape(kind=0, S=4, Hq=8, max_nb=5, q_len=1, max_group=0, T=4, P=2):
    return _lib.StepShape(kind, S, Hq, max_nb, q_len, max_group, T, P, 0.125, _lib.DecodeOpts(0, 0))


def test_step_layout_packs_the_fields_in_order(lib):
    """pa_step_layout_of: every field 256-byte aligned, in the documented
    order, each as large as its shape needs; the output is q's size."""
    d = _desc(head_dim=128)
    for kind, q_len, max_group in ((0, 1, 0), (1, 4, 0), (2, 1, 3)):
        sh = _step_shape(kind=kind, q_len=q_len, max_group=max_group)
        L = _lib.StepLayout()
        assert lib.pa_step_layout_of(ctypes.byref(sh), ctypes.byref(d), ctypes.byref(L)) == 0
        offs = [getattr(L, f) for f in _lib.STEP_FIELDS] + [L.total]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        S, Hq, D, Hkv = sh.num_seqs, sh.num_q_heads, d.head_dim, d.num_kv_heads
        q_bytes = S * q_len * Hq * D * 2
        assert L.out_bytes == q_bytes and L.block_tables - L.q >= q_bytes
        assert L.seq_lens - L.block_tables >= S * sh.max_blocks_per_seq * 4
        assert L.new_v - L.new_k >= sh.max_new_tokens * Hkv * D * 2
        assert L.total - L.slot_mapping >= sh.max_new_tokens * 8
        if kind == 2:
            assert L.group_prefix_blocks - L.group_starts >= (S + 1) * 4
        else:
            assert L.group_starts == L.group_prefix_blocks == L.copy_pairs  # unused fields take no room


def test_step_rejects_bad_shapes_and_pointers_on_host(lib):
    d = _desc(head_dim=128)
    L = _lib.StepLayout()
    for bad in (_step_shape(S=0), _step_shape(kind=0, q_len=2), _step_shape(kind=1, q_len=1),
                _step_shape(kind=2, max_group=0), _step_shape(kind=7), _step_shape(T=-1)):
        assert lib.pa_step_layout_of(ctypes.byref(bad), ctypes.byref(d), ctypes.byref(L)) == 1
    sh = _step_shape()
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    bad_ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE + 8)  # misaligned
    h = ctypes.c_void_p()
    for n, arrays in ((1, (ptrs,) * 4), (9, (ptrs,) * 4), (2, (ptrs, bad_ptrs, ptrs, ptrs))):
        rc = lib.pa_step_create(ctypes.byref(sh), ctypes.byref(d), FAKE, FAKE, FAKE, 1 << 20, None, n, *arrays,
                                ctypes.byref(h))
        assert rc == 1 and not h.value
    assert lib.pa_step_run(None, 0, 0, 0, None) == 1
    lib.pa_step_destroy(None)  # a no-op


def test_build_tracks_every_source_and_header():
    """An edited kernel header must make the library stale: the build's
    inputs list every file under csrc/."""
    csrc = Path(pa_build.CSRC)
    on_disk = {p.name for p in csrc.iterdir() if p.suffix in (".cu", ".cuh", ".h", ".cpp")}
    assert on_disk == set(pa_build.SOURCES) | set(pa_build.HEADERS)


def _update(copy_pairs=None, num_copy_pairs=0, k=None, v=None, slots=None, num_tokens=0):
    return _lib.CacheUpdate(copy_pairs, num_copy_pairs, k, v, slots, num_tokens)


def test_update_entry_points_reject_bad_updates_on_host(lib):
    """pa_decode_update and its multi-query and shared-prefix forms check the
    cache update before anything is enqueued (an empty batch included)."""
    desc = _desc()
    opts = _lib.DecodeOpts(0, 0)
    bad = [
        _update(num_copy_pairs=-1),
        _update(num_tokens=-1),
        _update(num_copy_pairs=2),                                             # pairs missing
        _update(copy_pairs=FAKE + 4, num_copy_pairs=2),                        # pairs not 8-byte aligned
        _update(k=FAKE, v=None, slots=FAKE, num_tokens=3),                     # v missing
        _update(k=FAKE + 8, v=FAKE, slots=FAKE, num_tokens=3),                 # k not 16-byte aligned
        _update(k=FAKE, v=FAKE, slots=FAKE + 4, num_tokens=3),                 # slots not 8-byte aligned
    ]
    for u in bad:
        for S in (4, 0):
            rc = lib.pa_decode_update(ctypes.byref(u), FAKE, FAKE, FAKE, FAKE, 8, FAKE, S, 4, 0.125, FAKE, FAKE,
                                      1 << 20, None, ctypes.byref(desc), ctypes.byref(opts), None)
            assert rc == 1, (S, rc)
        rc = lib.pa_decode_multi_update(ctypes.byref(u), FAKE, FAKE, FAKE, FAKE, 8, FAKE, 4, 3, 4, 0.125, FAKE,
                                        FAKE, 1 << 20, None, ctypes.byref(desc), ctypes.byref(opts), None)
        assert rc == 1
        rc = lib.pa_decode_shared_prefix_update(ctypes.byref(u), FAKE, FAKE, FAKE, FAKE, 8, FAKE, 4, 4, FAKE, FAKE,
                                                2, 4, 0.125, FAKE, FAKE, 1 << 20, None, ctypes.byref(desc),
                                                ctypes.byref(opts), None)
        assert rc == 1
    # bad decode arguments are still caught with a valid (here empty) update
    assert lib.pa_decode_update(ctypes.byref(_update()), None, FAKE, FAKE, FAKE, 8, FAKE, 4, 4, 0.125, FAKE, FAKE,
                                1 << 20, None, ctypes.byref(desc), ctypes.byref(opts), None) == 1


def test_lse_and_merge_reject_bad_arguments_on_host(lib):
    desc = _desc(head_dim=128)
    opts = _lib.DecodeOpts(0, 0)
    # pa_decode_lse needs its lse output (4-byte aligned)
    for lse in (None, FAKE + 2):
        rc = lib.pa_decode_lse(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 4, 4, 0.125, FAKE, lse, FAKE, 1 << 20, None,
                               ctypes.byref(desc), ctypes.byref(opts), None)
        assert rc == 1
    merge = lib.pa_merge_partials
    assert merge(FAKE, FAKE, 2, 0, 128, _lib.PA_BF16, FAKE, None, None) == 0  # no rows: a no-op
    assert merge(FAKE, FAKE, 0, 10, 128, _lib.PA_BF16, FAKE, None, None) == 1  # no parts
    assert merge(FAKE, FAKE, 2, -1, 128, _lib.PA_BF16, FAKE, None, None) == 1
    assert merge(FAKE, FAKE, 2, 10, 96, _lib.PA_BF16, FAKE, None, None) == 1  # head_dim
    assert merge(FAKE, FAKE, 2, 10, 128, 7, FAKE, None, None) == 1  # dtype
    assert merge(None, FAKE, 2, 10, 128, _lib.PA_BF16, FAKE, None, None) == 1
    assert merge(FAKE + 8, FAKE, 2, 10, 128, _lib.PA_BF16, FAKE, None, None) == 1  # outs misaligned
    assert merge(FAKE, FAKE + 2, 2, 10, 128, _lib.PA_BF16, FAKE, None, None) == 1  # lses misaligned
    assert merge(FAKE, FAKE, 2, 10, 128, _lib.PA_BF16, FAKE, FAKE + 1, None) == 1  # lse_out misaligned
