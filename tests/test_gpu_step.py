"""PagedDecodeStep: whole steps from pinned host buffers, several in flight
at once (uploads, kernels and downloads on three streams, two or three buffer
sets).  Each step writes new tokens into the shared pools and decodes (plain,
multi-query or shared-prefix); every result must match the oracle applied to
the same sequence of steps."""

import numpy as np
import pytest

from pa_testlib import assert_attention_close, torch_bits
from workloads import bits_to_torch, f32_to_bits, fill_values_numpy, random_layout
import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,sets", [(1, 2), (4, 2), (4, 3)])
def test_overlapped_steps_match_oracle(cuda_device, G, sets):
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
                              max_new_tokens=L.num_new_tokens, scale=L.scale, num_buffer_sets=sets)
    pin = lambda x: x.pin_memory()  # noqa: E731
    tables, lens, slots = (pin(torch.from_numpy(a)) for a in (L.block_tables, L.seq_lens, L.slot_mapping))
    host_in = [(pin(bits_to_torch(qs[i], L.dtype)), pin(bits_to_torch(nks[i], L.dtype)),
                pin(bits_to_torch(nvs[i], L.dtype))) for i in range(nsteps)]

    results, pending = [], []
    for i in range(nsteps):
        q_h, k_h, v_h = host_in[i]
        pending.append(step.run(q_h, tables, lens, k_h, v_h, slots))
        if len(pending) == sets:  # a result stays valid until its buffer set comes round again
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


def _run_steps(step, host_steps, sets, **kw):
    results, pending = [], []
    for args in host_steps:
        pending.append(step.run(*args, **kw))
        if len(pending) == sets:
            r = pending.pop(0)
            step.wait(r)
            results.append(r.clone())
    for r in pending:
        step.wait(r)
        results.append(r.clone())
    return results


def test_multi_query_steps_match_oracle(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa

    qlen = 3
    L = random_layout(71, [3, 16, 40, 200, 777], dtype="bf16", block_size=16, num_q_heads=8, num_kv_heads=2,
                      head_dim=128, write_new_token=True, q_len=qlen)
    V = fill_values_numpy(L)
    rng = np.random.default_rng(10)
    nsteps = 4
    qs = [f32_to_bits(rng.standard_normal(V.q.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]
    nks = [f32_to_bits(rng.standard_normal(V.new_k.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]
    nvs = [f32_to_bits(rng.standard_normal(V.new_v.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]
    kp = bits_to_torch(V.k_pool, L.dtype).to(cuda_device)
    vp = bits_to_torch(V.v_pool, L.dtype).to(cuda_device)
    step = pa.PagedDecodeStep(kp, vp, L.num_seqs, L.num_q_heads, L.max_blocks_per_seq,
                              max_new_tokens=L.num_new_tokens, scale=L.scale, q_len=qlen)
    pin = lambda x: x.pin_memory()  # noqa: E731
    tables, lens, slots = (pin(torch.from_numpy(a)) for a in (L.block_tables, L.seq_lens, L.slot_mapping))
    host = [(pin(bits_to_torch(qs[i], L.dtype)), tables, lens, pin(bits_to_torch(nks[i], L.dtype)),
             pin(bits_to_torch(nvs[i], L.dtype)), slots) for i in range(nsteps)]
    results = _run_steps(step, host, 3)
    assert step.device_status() == 0
    k_ref, v_ref = V.k_pool, V.v_pool
    for i in range(nsteps):
        k_ref, v_ref = oracle.cache_write(k_ref, v_ref, nks[i], nvs[i], L.slot_mapping)
        ref = oracle.decode_multi(qs[i], k_ref, v_ref, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads,
                                  L.dtype)
        assert_attention_close(results[i].double().numpy(), ref, f"multi step {i}")


def test_shared_prefix_steps_match_oracle(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa
    from test_gpu_shared_prefix import _forked_layout

    L = _forked_layout(72, [(300, [1, 9, 40]), (64, [2, 2]), (33, [5])], G=4)
    V = fill_values_numpy(L)
    rng = np.random.default_rng(11)
    nsteps = 4
    qs = [f32_to_bits(rng.standard_normal(V.q.shape, dtype=np.float32), L.dtype) for _ in range(nsteps)]
    kp = bits_to_torch(V.k_pool, L.dtype).to(cuda_device)
    vp = bits_to_torch(V.v_pool, L.dtype).to(cuda_device)
    step = pa.PagedDecodeStep(kp, vp, L.num_seqs, L.num_q_heads, L.max_blocks_per_seq,
                              max_new_tokens=L.num_new_tokens, scale=L.scale, max_group_size=3)
    gs, gp = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, 3)
    pin = lambda x: x.pin_memory()  # noqa: E731
    tables, lens, slots = (pin(torch.from_numpy(a)) for a in (L.block_tables, L.seq_lens, L.slot_mapping))
    nk, nv = pin(bits_to_torch(V.new_k, L.dtype)), pin(bits_to_torch(V.new_v, L.dtype))
    host = [(pin(bits_to_torch(qs[i], L.dtype)), tables, lens, nk, nv, slots) for i in range(nsteps)]
    results = _run_steps(step, host, 3, group_starts=pin(torch.from_numpy(gs)),
                         group_prefix_blocks=pin(torch.from_numpy(gp)))
    assert step.device_status() == 0
    k_ref, v_ref = oracle.cache_write(V.k_pool, V.v_pool, V.new_k, V.new_v, L.slot_mapping)
    for i in range(nsteps):
        ref = oracle.decode(qs[i], k_ref, v_ref, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
        assert_attention_close(results[i].double().numpy(), ref, f"shared-prefix step {i}")


def test_staged_steps_upload_one_packed_block(cuda_device):
    """Inputs built in the step's pinned staging views go up as one copy of
    the used part of the packed block; results match the oracle step by
    step (through run() and through run_staged(), alternately), and the
    uploaded byte count is that part's size."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = random_layout(58, [3, 16, 17, 200, 900, 45, 1], dtype="bf16", block_size=16, num_q_heads=8,
                      num_kv_heads=2, head_dim=128, write_new_token=True)
    V = fill_values_numpy(L)
    rng = np.random.default_rng(12)
    kp = bits_to_torch(V.k_pool, L.dtype).to(cuda_device)
    vp = bits_to_torch(V.v_pool, L.dtype).to(cuda_device)
    step = pa.PagedDecodeStep(kp, vp, L.num_seqs, L.num_q_heads, L.max_blocks_per_seq,
                              max_new_tokens=L.num_new_tokens, scale=L.scale)
    k_ref, v_ref = V.k_pool, V.v_pool
    for i in range(5):
        q = f32_to_bits(rng.standard_normal(V.q.shape, dtype=np.float32), L.dtype)
        nk = f32_to_bits(rng.standard_normal(V.new_k.shape, dtype=np.float32), L.dtype)
        nv = f32_to_bits(rng.standard_normal(V.new_v.shape, dtype=np.float32), L.dtype)
        s = step.staging()
        s["q"].copy_(bits_to_torch(q, L.dtype))
        s["block_tables"].copy_(torch.from_numpy(L.block_tables))
        s["seq_lens"].copy_(torch.from_numpy(L.seq_lens))
        s["new_k"].copy_(bits_to_torch(nk, L.dtype))
        s["new_v"].copy_(bits_to_torch(nv, L.dtype))
        s["slot_mapping"].copy_(torch.from_numpy(L.slot_mapping))
        if i % 2 == 0:
            out = step.run(s["q"], s["block_tables"], s["seq_lens"], s["new_k"], s["new_v"], s["slot_mapping"])
        else:
            out = step.run_staged(num_new_tokens=L.num_new_tokens)
        step.wait(out)
        assert step.last_h2d_bytes == step.layout.slot_mapping + 8 * L.num_new_tokens
        k_ref, v_ref = oracle.cache_write(k_ref, v_ref, nk, nv, L.slot_mapping)
        ref = oracle.decode(q, k_ref, v_ref, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
        assert_attention_close(out.double().numpy(), ref, f"staged step {i}")
    assert step.device_status() == 0
    assert np.array_equal(torch_bits(kp), k_ref) and np.array_equal(torch_bits(vp), v_ref)
    step.close()


def test_executor_reports_device_errors_and_recovers(cuda_device):
    """A step whose slot mapping points past the pool: the cache write skips
    the token and records PA_DEV_BAD_SLOT (103) in the device status, nothing
    traps, and the next good step on the same executor matches the oracle."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = random_layout(59, [5, 40, 300], dtype="bf16", block_size=16, num_q_heads=8, num_kv_heads=2, head_dim=128,
                      write_new_token=True)
    V = fill_values_numpy(L)
    kp = bits_to_torch(V.k_pool, L.dtype).to(cuda_device)
    vp = bits_to_torch(V.v_pool, L.dtype).to(cuda_device)
    step = pa.PagedDecodeStep(kp, vp, L.num_seqs, L.num_q_heads, L.max_blocks_per_seq,
                              max_new_tokens=L.num_new_tokens, scale=L.scale)
    q = bits_to_torch(V.q, L.dtype)
    nk, nv = bits_to_torch(V.new_k, L.dtype), bits_to_torch(V.new_v, L.dtype)
    tables, lens = torch.from_numpy(L.block_tables), torch.from_numpy(L.seq_lens)
    bad = torch.from_numpy(L.slot_mapping.copy())
    bad[1] = L.num_blocks * L.block_size + 5  # past the pool
    out = step.run(q, tables, lens, nk, nv, bad)
    step.wait(out)
    assert step.device_status() == 103
    step.status.zero_()
    torch.cuda.synchronize()  # the reset is on torch's stream, the step's kernels on the executor's
    out = step.run(q, tables, lens, nk, nv, torch.from_numpy(L.slot_mapping))
    step.wait(out)
    assert step.device_status() == 0
    # the bad step wrote tokens 0 and 2 only; the good step wrote all three
    k_ref, v_ref = oracle.cache_write(V.k_pool, V.v_pool, V.new_k, V.new_v, L.slot_mapping)
    ref = oracle.decode(V.q, k_ref, v_ref, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
    assert_attention_close(out.double().numpy(), ref, "after the bad step")
    step.close()
