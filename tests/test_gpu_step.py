"""PagedDecodeStep: whole steps from pinned host buffers, several in flight
at once (uploads, kernels and downloads on three streams, two buffer sets).
Each step writes new tokens into the shared pools and decodes; every result
must match the oracle applied to the same sequence of steps."""

import numpy as np
import pytest

from pa_testlib import assert_attention_close, torch_bits
from workloads import bits_to_torch, f32_to_bits, fill_values_numpy, random_layout
import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G", [1, 4])
def test_overlapped_steps_match_oracle(cuda_device, G):
    import torch

    import paged_kv_cache_357_b200 as pa

    L = random_layout(55 + G, [3, 16, 17, 200, 900, 45, 1], dtype="bf16", block_size=16, num_q_heads=2 * G,
                      num_kv_heads=2, head_dim=128, write_new_token=True)
    V = fill_values_numpy(L)
    rng = np.random.default_rng(9)
    nsteps = 5
    qs = [f32_to_bits(rng.standard_normal(V.q.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]
    nks = [f32_to_bits(rng.standard_normal(V.new_k.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]
    nvs = [f32_to_bits(rng.standard_normal(V.new_v.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]

    kp = bits_to_torch(V.k_pool, L.dtype).to(cuda_device)
    vp = bits_to_torch(V.v_pool, L.dtype).to(cuda_device)
    step = pa.PagedDecodeStep(kp, vp, L.num_seqs, L.num_q_heads, L.max_blocks_per_seq,
                              max_new_tokens=L.num_new_tokens, scale=L.scale)
    pin = lambda x: x.pin_memory()  # noqa: E731
    tables, lens, slots = (pin(torch.from_numpy(a)) for a in (L.block_tables, L.seq_lens, L.slot_mapping))
    host_in = [(pin(bits_to_torch(qs[i], L.dtype)), pin(bits_to_torch(nks[i], L.dtype)),
                pin(bits_to_torch(nvs[i], L.dtype))) for i in range(nsteps)]

    results, pending = [], []
    for i in range(nsteps):
        q_h, k_h, v_h = host_in[i]
        pending.append(step.run(q_h, tables, lens, k_h, v_h, slots))
        if len(pending) == 2:  # keep two steps in flight; a result is reused two steps later
            r = pending.pop(0)
            step.wait(r)
            results.append(r.clone())
    for r in pending:
        step.wait(r)
        results.append(r.clone())
    assert step.device_status() == 0

    k_ref, v_ref = V.k_pool, V.v_pool
    for i in range(nsteps):
        k_ref, v_ref = oracle.cache_write(k_ref, v_ref, nks[i], nvs[i], L.slot_mapping)
        ref = oracle.decode(qs[i], k_ref, v_ref, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
        assert_attention_close(results[i].double().numpy(), ref, f"step {i}")
    assert np.array_equal(torch_bits(kp), k_ref) and np.array_equal(torch_bits(vp), v_ref)
