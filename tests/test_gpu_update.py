"""GPU parity of the one-call step: pa_decode_update, pa_decode_multi_update
and pa_decode_shared_prefix_update run the step's copy-on-write block copies
(study notes ch.05 §6.1, a kernel of their own), then the new tokens' stores
(vLLM blog, plain-language section), then the decode; the stores run inside
the launch of the tensor-core decode kernel (a grid-wide barrier before its
first K/V load), or as pa_cache_write where that kernel does not run.

Each case is checked three ways:
* the pools, bit for bit, against the oracle's copy_blocks and cache_write;
* the outputs against the float64 oracle, within the decode tolerance
  (max-abs 2e-3 where |oracle| < 0.5, max-rel 1e-2 where |oracle| >= 0.1);
* the outputs, bit for bit, against the same decode launched after separate
  pa_copy_blocks / pa_cache_write kernels: the same kernel with the same
  partition does the same arithmetic, so any difference would be a read
  that ran ahead of a copy or a store.
"""

import numpy as np
import pytest

import oracle
from pa_testlib import assert_attention_close, oracle_step, to_device, torch_bits, torch_f64
from workloads import config_llama2_70b_shared, config_llama3_8b, fill_values_numpy, random_layout

pytestmark = pytest.mark.gpu


def _pools_match(d, kp, vp, what):
    assert np.array_equal(torch_bits(d["k_pool"]), kp), f"{what}: k_pool differs from the oracle"
    assert np.array_equal(torch_bits(d["v_pool"]), vp), f"{what}: v_pool differs from the oracle"


def _update_kwargs(L, d):
    kw = {}
    if L.copy_pairs.shape[0] > 0:
        kw["copy_pairs"] = d["pairs"]
    if L.num_new_tokens > 0:
        kw.update(new_k=d["new_k"], new_v=d["new_v"], slot_mapping=d["slots"])
    return kw


def _run_plain(L, V, device, *, fused, num_ctas=0, flags=0):
    import torch

    import paged_kv_cache_357_b200 as pa

    d = to_device(L, V, device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    out = torch.full_like(d["q"], float("nan"))
    ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"], num_ctas, flags)
    if fused:
        pa.pa_decode_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                            num_ctas=num_ctas, flags=flags, **_update_kwargs(L, d))
    else:
        if L.copy_pairs.shape[0] > 0:
            pa.pa_copy_blocks(d["pairs"], d["k_pool"], d["v_pool"], st)
        if L.num_new_tokens > 0:
            pa.pa_cache_write(d["new_k"], d["new_v"], d["slots"], d["k_pool"], d["v_pool"], st)
        pa.pa_decode(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                     num_ctas=num_ctas, flags=flags)
    torch.cuda.synchronize()
    return out, int(st.item()), d, ws


@pytest.mark.parametrize("num_ctas", [0, 1, 5, 400])
@pytest.mark.parametrize("B", [8, 16, 32])
def test_update_decode_with_copies_and_writes(cuda_device, B, num_ctas):
    """Forked samples at the Llama-2-70B layer shape (64 q / 8 kv heads):
    nine copy-on-write pairs and twelve new tokens, some of them stored into
    a block copied by the same call, then the GQA-8 decode.  With 400 CTAs,
    more than fit on the GPU at once, the stores run as their own launch
    (the in-launch barrier needs the whole grid resident)."""
    L = config_llama2_70b_shared(prompt_len=256, num_prompts=3, samples=4, max_tail=60, block_size=B)
    assert L.copy_pairs.shape[0] > 0 and L.num_new_tokens > 0
    V = fill_values_numpy(L)
    out, st, d, _ = _run_plain(L, V, cuda_device, fused=True, num_ctas=num_ctas)
    assert st == 0
    ref, kp, vp = oracle_step(L, V)
    _pools_match(d, kp, vp, f"B={B} ctas={num_ctas}")
    assert_attention_close(torch_f64(out), ref, f"update decode B={B} ctas={num_ctas}")
    sep, st2, _, _ = _run_plain(L, V, cuda_device, fused=False, num_ctas=num_ctas)
    assert st2 == 0
    assert np.array_equal(torch_bits(out), torch_bits(sep)), "one-launch step differs from separate kernels"


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_update_decode_write_only_gqa4(cuda_device, dtype):
    """Llama-3-8B GQA-4 step (the new token of each of 48 sequences, no
    copies); fp16 runs on a relabelled layout with the same structure."""
    L = config_llama3_8b(batch=48)
    if dtype == "fp16":
        L.dtype = "fp16"
    V = fill_values_numpy(L)
    out, st, d, _ = _run_plain(L, V, cuda_device, fused=True)
    assert st == 0
    ref, kp, vp = oracle_step(L, V)
    _pools_match(d, kp, vp, f"llama3 {dtype}")
    assert_attention_close(torch_f64(out), ref, f"update decode llama3 {dtype}")
    sep, _, _, _ = _run_plain(L, V, cuda_device, fused=False)
    assert np.array_equal(torch_bits(out), torch_bits(sep))


def test_update_repeated_calls_reuse_the_workspace(cuda_device):
    """Three one-call steps in a row on one workspace: the barrier words are
    left as found (the arrival count back at zero), so each call completes
    with the same pools and outputs (the update is idempotent here: the
    copies rewrite the same blocks, the stores the same slots)."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared(prompt_len=128, num_prompts=2, samples=4, max_tail=30, block_size=16)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"])
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    outs = []
    for _ in range(3):
        out = torch.full_like(d["q"], float("nan"))
        pa.pa_decode_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                            **_update_kwargs(L, d))
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append(torch_bits(out))
    ref, kp, vp = oracle_step(L, V)
    _pools_match(d, kp, vp, "after three calls")
    assert_attention_close(torch_f64(out), ref, "third call")
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


@pytest.mark.parametrize("B", [8, 16, 32])
def test_update_shared_prefix(cuda_device, B):
    """Shared-prefix decode (group units of 4 members x 8 heads) with its
    step's copies and stores in the same call."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared(prompt_len=256, num_prompts=3, samples=4, max_tail=60, block_size=B)
    V = fill_values_numpy(L)
    starts, prefix = pa.shared_prefix_groups(L.block_tables, L.seq_lens, B, 4)
    outs = {}
    for fused in (True, False):
        d = to_device(L, V, cuda_device)
        gs, gp = torch.from_numpy(starts).to(cuda_device), torch.from_numpy(prefix).to(cuda_device)
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        out = torch.full_like(d["q"], float("nan"))
        ws = pa.alloc_shared_prefix_workspace(L.num_seqs, 4, L.num_q_heads, d["k_pool"])
        if fused:
            pa.pa_decode_shared_prefix_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], gs, gp, 4,
                                              L.scale, out, ws, st, **_update_kwargs(L, d))
        else:
            pa.pa_copy_blocks(d["pairs"], d["k_pool"], d["v_pool"], st)
            pa.pa_cache_write(d["new_k"], d["new_v"], d["slots"], d["k_pool"], d["v_pool"], st)
            pa.pa_decode_shared_prefix(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], gs, gp, 4,
                                       L.scale, out, ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs[fused] = out
        if fused:
            ref, kp, vp = oracle_step(L, V)
            _pools_match(d, kp, vp, f"shared prefix B={B}")
            assert_attention_close(torch_f64(out), ref, f"update shared prefix B={B}")
    assert np.array_equal(torch_bits(outs[True]), torch_bits(outs[False]))


@pytest.mark.parametrize("q_len,G", [(4, 4), (3, 8), (64, 4)])
def test_update_multi(cuda_device, q_len, G):
    """Multi-query steps whose q_len new tokens are stored by the same call:
    q_len 4 and 3 run on the tensor-core row-tile kernel (stores in its
    launch); q_len
    64 at GQA-4 fills 128-row tiles and runs the query-major prefill kernel,
    after the update's own kernels."""
    import torch

    import paged_kv_cache_357_b200 as pa

    lens = [q_len, q_len + 5, 130, 517, 1000 + q_len]
    L = random_layout(9100 + q_len * 10 + G, lens, dtype="bf16", block_size=16, num_q_heads=2 * G, num_kv_heads=2,
                      head_dim=128, q_len=q_len)
    assert L.num_new_tokens == q_len * len(lens)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = torch.full_like(d["q"], float("nan"))
    ws = pa.alloc_multi_workspace(L.num_seqs, q_len, L.num_q_heads, d["k_pool"])
    pa.pa_decode_multi_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                              **_update_kwargs(L, d))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    kp, vp = oracle.cache_write(V.k_pool, V.v_pool, V.new_k, V.new_v, L.slot_mapping)
    _pools_match(d, kp, vp, f"multi q_len={q_len}")
    ref = oracle.decode_multi(V.q, kp, vp, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
    assert_attention_close(torch_f64(out), ref, f"update multi q_len={q_len} G={G}")


def test_update_on_cuda_cores_runs_separate_kernels(cuda_device):
    """Where the CUDA-core kernel runs (here forced by the flag), the update
    goes ahead of it as its own kernels, with the same results."""
    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared(prompt_len=128, num_prompts=2, samples=4, max_tail=30, block_size=16)
    V = fill_values_numpy(L)
    out, st, d, _ = _run_plain(L, V, cuda_device, fused=True, flags=pa.PA_DECODE_CUDA_CORES_ONLY)
    assert st == 0
    ref, kp, vp = oracle_step(L, V)
    _pools_match(d, kp, vp, "cuda cores")
    assert_attention_close(torch_f64(out), ref, "update decode on CUDA cores")


def test_update_with_no_sequences_still_updates(cuda_device):
    """A step with no sequence to decode still applies its copies and stores."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared(prompt_len=128, num_prompts=2, samples=4, max_tail=30, block_size=16)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    q0 = d["q"][:0]
    ws = pa.alloc_decode_workspace(1, L.num_q_heads, d["k_pool"])
    pa.pa_decode_update(q0, d["k_pool"], d["v_pool"], d["tables"][:0], d["lens"][:0], L.scale, q0.clone(), ws, st,
                        **_update_kwargs(L, d))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _, kp, vp = oracle_step(L, V)
    _pools_match(d, kp, vp, "no sequences")


def test_update_reports_bad_slots_and_pairs(cuda_device):
    """A slot past the pool and a pair naming a block past the pool are
    reported in the device status and skipped; the launch completes."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared(prompt_len=128, num_prompts=2, samples=4, max_tail=30, block_size=16)
    V = fill_values_numpy(L)
    for bad in ("slot", "pair"):
        d = to_device(L, V, cuda_device)
        if bad == "slot":
            d["slots"][1] = L.num_blocks * L.block_size + 3
            want = 103
        else:
            d["pairs"][0, 1] = L.num_blocks + 7
            want = 104
        out, st = torch.full_like(d["q"], float("nan")), torch.zeros(1, dtype=torch.int32, device=cuda_device)
        ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"])
        pa.pa_decode_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                            **_update_kwargs(L, d))
        torch.cuda.synchronize()
        assert int(st.item()) == want, (bad, int(st.item()))


def test_update_barrier_wait_runs_out(cuda_device):
    """Failure detection: with the test hook CTA 0 never arrives at the
    stores' barrier, every wait for it runs out (about 20 ms), the
    kernel returns PA_DEV_TIMEOUT, and the context stays usable: a normal
    step on a zeroed workspace then matches the oracle."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared(prompt_len=128, num_prompts=2, samples=4, max_tail=30, block_size=16)
    V = fill_values_numpy(L)
    for with_copies in (True, False):
        d = to_device(L, V, cuda_device)
        kw = _update_kwargs(L, d)
        if not with_copies:
            kw.pop("copy_pairs")
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        out = torch.full_like(d["q"], float("nan"))
        flags = pa.PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL
        ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"], 0, flags)
        pa.pa_decode_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                            flags=flags, **kw)
        torch.cuda.synchronize()
        assert int(st.item()) == 105, int(st.item())
    out, st, d, _ = _run_plain(L, V, cuda_device, fused=True)
    assert st == 0
    ref, kp, vp = oracle_step(L, V)
    _pools_match(d, kp, vp, "after the timeout")
    assert_attention_close(torch_f64(out), ref, "step after the timeout")
