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


def test_prefill_bounded_waits_report_timeout(cuda_device):
    """The query-major prefill kernel (G x q_len of 128 rows or more) under
    the same hook: its issuers' and softmax warps' waits run out, the kernel
    records PA_DEV_TIMEOUT and returns, and a normal call on the same
    context and workspace then matches the oracle."""
    import time

    import numpy as np
    import torch

    import oracle
    import paged_kv_cache_357_b200 as pa
    from workloads import bits_to_torch, f32_to_bits

    G, q_len, Hkv = 4, 64, 2
    L = random_layout(33, [64, 200, 97], dtype="bf16", block_size=16, num_q_heads=G * Hkv, num_kv_heads=Hkv,
                      head_dim=128, write_new_token=False)
    V = fill_values_numpy(L)
    rng = np.random.default_rng(33)
    q_bits = f32_to_bits(rng.standard_normal((L.num_seqs, q_len, L.num_q_heads, 128), dtype=np.float32), "bf16")
    kp = bits_to_torch(V.k_pool, "bf16").to(cuda_device)
    vp = bits_to_torch(V.v_pool, "bf16").to(cuda_device)
    q = bits_to_torch(q_bits, "bf16").to(cuda_device)
    tables = torch.from_numpy(L.block_tables).to(cuda_device)
    lens = torch.from_numpy(L.seq_lens).to(cuda_device)
    out = torch.zeros_like(q)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = pa.alloc_multi_workspace(L.num_seqs, q_len, L.num_q_heads, kp, 4)
    t0 = time.time()
    pa.pa_decode_multi(q, kp, vp, tables, lens, L.scale, out, ws, st, num_ctas=4,
                       flags=pa.PA_DECODE_TEST_WITHHOLD_COPIES)
    torch.cuda.synchronize()
    assert time.time() - t0 < 10.0
    assert int(st.item()) == 105
    ws.zero_()  # a workspace is zeroed again after a non-zero device status
    st.zero_()
    pa.pa_decode_multi(q, kp, vp, tables, lens, L.scale, out, ws, st, num_ctas=4)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.decode_multi(q_bits, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads,
                              "bf16")
    assert_attention_close(torch_f64(out), ref, "prefill after timeout")
