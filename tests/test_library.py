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
    for code in [0, 1, 2, 3, 4, 5, 6, 101, 102, 103, 104, 105]:
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
