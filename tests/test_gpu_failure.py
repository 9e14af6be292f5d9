"""Failure detection without faulting the GPU: the decode's pipeline waits
are bounded.  With the test hook PA_DECODE_TEST_WITHHOLD_COPIES the producer
issues nothing, every consumer wait runs out (about 20 ms), the kernel
records PA_DEV_TIMEOUT and returns, and the context stays usable."""

import pytest

from pa_testlib import gpu_step, oracle_step, assert_attention_close, to_device, torch_f64
from workloads import fill_values_numpy, random_layout

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,D", [(2, 64), (4, 128)], ids=["cuda-core", "tensor-core"])
def test_bounded_wait_reports_timeout_and_context_survives(cuda_device, G, D):
    import time

    import torch

    import paged_kv_cache_357_b200 as pa

    L = random_layout(31, [40, 70, 5], dtype="bf16", block_size=16, num_q_heads=2 * G, num_kv_heads=2,
                      head_dim=D, write_new_token=False)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = torch.zeros_like(d["q"])
    ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"], num_ctas=4)
    t0 = time.time()
    pa.pa_decode(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st, num_ctas=4,
                 flags=pa.PA_DECODE_TEST_WITHHOLD_COPIES)
    torch.cuda.synchronize()
    assert time.time() - t0 < 10.0
    assert int(st.item()) == 105
    # a normal decode right after, on the same context
    out2, st2 = gpu_step(d, L)
    assert int(st2.item()) == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out2), ref, "after timeout")
