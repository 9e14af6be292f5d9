"""pa_decode_no_alloc: the decode for callers that cannot allocate device
memory (for instance a plug-in whose host engine owns nearly all device
memory and hands it only inputs and outputs).  Its scratch is libpa's fixed
device array instead of a caller workspace.

The test calls the entry point through the C ABI twice in a row on the same
inputs.  Each call's output is checked against the float64 oracle (the
decode tolerance of tests/pa_testlib.py) and against pa_decode's output
with a caller workspace (within 2e-3 + 1e-2*|ref|).  The second call runs on
the array exactly as the first left it, so it shows that reusing the array
gives the same result.  It does not show that the counter clearing is needed:
a call that completes leaves its counters at zero anyway, and only a call
that stopped partway would leave them set.

This file is collected last; it passes alone in a fresh process and after
the others.
"""

import ctypes

import numpy as np
import pytest

import oracle
from pa_testlib import ATOL, RTOL, assert_attention_close, to_device, torch_f64
from workloads import fill_values_numpy, random_layout

pytestmark = pytest.mark.gpu


def test_no_alloc_decode_matches_oracle_and_pa_decode_on_two_calls(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa
    from paged_kv_cache_357_b200 import _lib

    lib = _lib.load()
    # ragged GQA batch long enough that several CTAs split sequences, so the
    # partial states and arrival counters in the scratch are really used
    lens = [1, 15, 16, 17, 300, 1000, 2500, 4000, 64, 777]
    L = random_layout(2024, lens, dtype="bf16", block_size=16, num_q_heads=32, num_kv_heads=8, head_dim=128,
                      write_new_token=False)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    want = oracle.decode(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)

    ref = torch.full_like(d["q"], float("nan"))
    ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"])
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pa.pa_decode(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, ref, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref64 = torch_f64(ref)

    desc = pa.pool_desc(d["k_pool"])
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(d["q"], float("nan"))
        st.zero_()
        rc = lib.pa_decode_no_alloc(
            d["q"].data_ptr(), d["k_pool"].data_ptr(), d["v_pool"].data_ptr(), d["tables"].data_ptr(),
            L.max_blocks_per_seq, d["lens"].data_ptr(), L.num_seqs, L.num_q_heads, ctypes.c_float(L.scale),
            out.data_ptr(), st.data_ptr(), ctypes.byref(desc), stream)
        torch.cuda.synchronize()
        assert rc == 0, pa.status_string(rc)
        assert int(st.item()) == 0, f"call {call}: device status {int(st.item())}"
        got = torch_f64(out)
        assert_attention_close(got, want, f"no-alloc call {call} vs oracle")
        err = np.abs(got - ref64)
        assert (err <= ATOL + RTOL * np.abs(ref64)).all(), f"call {call}: max abs err {err.max():.3e}"


def test_no_alloc_rejects_batches_beyond_its_scratch(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa

    # 300k sequences x 8 kv heads of arrival counters alone exceed 8 MiB
    S = 300_000
    q = torch.zeros((S, 8, 64), dtype=torch.bfloat16, device=cuda_device)
    kp = torch.zeros((4, 8, 16, 64), dtype=torch.bfloat16, device=cuda_device)
    tables = torch.zeros((S, 1), dtype=torch.int32, device=cuda_device)
    lens = torch.ones((S,), dtype=torch.int32, device=cuda_device)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_no_alloc(q, kp, kp, tables, lens, 0.125, torch.empty_like(q))
    assert e.value.code == 5
