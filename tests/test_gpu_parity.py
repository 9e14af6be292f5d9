"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle.

Bit-exact: cache write, block copy, the pools after a step, and everything
the block tables index.  Decode: max-abs 2e-3 where |oracle| < 0.5
and max-rel 1e-2 where |oracle| >= 0.1, per element (tests/pa_testlib.py).  Inputs are the seeded workloads; padding rows and
unused blocks of every pool hold NaN.
"""

import numpy as np
import pytest

from pa_testlib import (
    assert_attention_close,
    gpu_step,
    oracle_step,
    to_device,
    torch_bits,
    torch_f64,
)
from workloads import config_llama2_70b_shared, config_tiny, fill_values_numpy, random_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa_mod(cuda_device):
    import paged_kv_cache_357_b200 as pa

    pa.load()
    return pa


def _run_and_check(layout, values, device, num_ctas=0, what=""):
    dev_t = to_device(layout, values, device)
    out, st = gpu_step(dev_t, layout, num_ctas=num_ctas)
    ref_out, ref_k, ref_v = oracle_step(layout, values)
    assert int(st.item()) == 0, f"{what}: device status {int(st.item())}"
    assert np.array_equal(torch_bits(dev_t["k_pool"]), ref_k), f"{what}: K pool differs after copy/write"
    assert np.array_equal(torch_bits(dev_t["v_pool"]), ref_v), f"{what}: V pool differs after copy/write"
    assert_attention_close(torch_f64(out), ref_out, what)
    return out


def test_tiny_config_step(pa_mod, cuda_device):
    L = config_tiny()
    _run_and_check(L, fill_values_numpy(L), cuda_device, what="tiny")


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("B", [8, 16, 32])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_shape_sweep(pa_mod, cuda_device, dtype, B, D, G):
    Hkv = 2
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 9 * B, 250]
    L = random_layout(1000 * B + 10 * D + G, lens, dtype=dtype, block_size=B, num_q_heads=Hkv * G,
                      num_kv_heads=Hkv, head_dim=D, write_new_token=True)
    _run_and_check(L, fill_values_numpy(L), cuda_device, what=f"{dtype} B={B} D={D} G={G}")


@pytest.mark.parametrize("B", [8, 16, 32])
@pytest.mark.parametrize("num_ctas", [1, 3, 7, 64, 1000])
def test_split_counts_agree(pa_mod, cuda_device, num_ctas, B):
    """One CTA (no split at all) through far more CTAs than blocks: every
    split of the work list merges to the same result, at every block size."""
    L = random_layout(77 + B, [1, 5, 16, 17, 40, 100, 333, 700, 1029], dtype="bf16", block_size=B, num_q_heads=8,
                      num_kv_heads=2, head_dim=128)
    _run_and_check(L, fill_values_numpy(L), cuda_device, num_ctas=num_ctas, what=f"B={B} ctas={num_ctas}")


def test_physical_placement_does_not_change_bits(pa_mod, cuda_device):
    import torch

    L = random_layout(5, [3, 40, 129, 600], dtype="bf16", block_size=16, num_q_heads=8, num_kv_heads=2,
                      head_dim=128, write_new_token=False)
    V = fill_values_numpy(L)
    d1 = to_device(L, V, cuda_device)
    out1, _ = gpu_step(d1, L)
    pi = np.random.default_rng(3).permutation(L.num_blocks)
    kp, vp = np.empty_like(V.k_pool), np.empty_like(V.v_pool)
    kp[pi], vp[pi] = V.k_pool, V.v_pool
    L2 = random_layout(5, [3, 40, 129, 600], dtype="bf16", block_size=16, num_q_heads=8, num_kv_heads=2,
                       head_dim=128, write_new_token=False)
    L2.block_tables = np.where(L.block_tables >= 0, pi[np.maximum(L.block_tables, 0)], -1).astype(np.int32)
    V.k_pool, V.v_pool = kp, vp
    d2 = to_device(L2, V, cuda_device)
    out2, _ = gpu_step(d2, L2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_shared_blocks_and_cow_fork(pa_mod, cuda_device):
    """Fork with a partly filled last prompt block (prompt of 2040 tokens,
    8/16 rows in the last block): samples 1-3 copy it, every sample writes its
    own first token, then all four decode."""
    L = config_llama2_70b_shared(prompt_len=2040, num_prompts=4, samples=4, max_tail=0)
    V = fill_values_numpy(L)
    out = _run_and_check(L, V, cuda_device, what="cow fork")
    # samples of one prompt read the same prompt but their own newest token
    o = torch_f64(out)
    for grp in L.share_groups:
        assert not np.array_equal(o[grp[0]], o[grp[1]])


def test_workspace_reuse_is_stable(pa_mod, cuda_device):
    import torch

    L = random_layout(9, [17, 400, 999, 2000, 31], dtype="fp16", block_size=16, num_q_heads=4, num_kv_heads=4,
                      head_dim=128, write_new_token=False)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    ws = pa_mod.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"])
    outs = [gpu_step(d, L, workspace=ws)[0] for _ in range(3)]
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(outs[2]), ref, "reuse")


def test_zero_length_sequences_give_zeros(pa_mod, cuda_device):
    import torch

    L = random_layout(4, [0, 20, 0, 3], dtype="bf16", block_size=16, num_q_heads=4, num_kv_heads=2,
                      head_dim=64, write_new_token=False)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    out, st = gpu_step(d, L)
    assert int(st.item()) == 0
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, "zero-length")


def test_cache_write_bit_exact_random_slots(pa_mod, cuda_device):
    import torch

    rng = np.random.default_rng(12)
    NB, Hkv, B, D = 50, 3, 16, 64
    kp = rng.integers(0, 1 << 15, size=(NB, Hkv, B, D), dtype=np.uint16)
    vp = rng.integers(0, 1 << 15, size=(NB, Hkv, B, D), dtype=np.uint16)
    T = 200
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[::7] = -1
    nk = rng.integers(0, 1 << 15, size=(T, Hkv, D), dtype=np.uint16)
    nv = rng.integers(0, 1 << 15, size=(T, Hkv, D), dtype=np.uint16)
    from workloads import bits_to_torch

    tk, tv = bits_to_torch(kp, "bf16").to(cuda_device), bits_to_torch(vp, "bf16").to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pa_mod.pa_cache_write(bits_to_torch(nk, "bf16").to(cuda_device), bits_to_torch(nv, "bf16").to(cuda_device),
                          torch.from_numpy(slots).to(cuda_device), tk, tv, st)
    torch.cuda.synchronize()
    import oracle

    rk, rv = oracle.cache_write(kp, vp, nk, nv, slots)
    assert int(st.item()) == 0
    assert np.array_equal(torch_bits(tk), rk) and np.array_equal(torch_bits(tv), rv)


def test_copy_blocks_bit_exact(pa_mod, cuda_device):
    import torch

    import oracle
    from workloads import bits_to_torch

    rng = np.random.default_rng(13)
    NB, Hkv, B, D = 40, 8, 16, 128
    kp = rng.integers(0, 1 << 15, size=(NB, Hkv, B, D), dtype=np.uint16)
    vp = rng.integers(0, 1 << 15, size=(NB, Hkv, B, D), dtype=np.uint16)
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:12], perm[12:24]], axis=1).astype(np.int64)
    pairs[3] = [pairs[3, 0], pairs[3, 0]]  # src == dst: no-op
    tk, tv = bits_to_torch(kp, "fp16").to(cuda_device), bits_to_torch(vp, "fp16").to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pa_mod.pa_copy_blocks(torch.from_numpy(pairs).to(cuda_device), tk, tv, st)
    torch.cuda.synchronize()
    rk, rv = oracle.copy_blocks(kp, vp, pairs)
    assert int(st.item()) == 0
    assert np.array_equal(torch_bits(tk), rk) and np.array_equal(torch_bits(tv), rv)


def test_device_errors_are_reported_not_trapped(pa_mod, cuda_device):
    import torch

    L = random_layout(6, [10, 50], dtype="bf16", block_size=16, num_q_heads=2, num_kv_heads=2, head_dim=64,
                      write_new_token=False)
    V = fill_values_numpy(L)
    # a block id past the pool
    d = to_device(L, V, cuda_device)
    d["tables"][1, 2] = L.num_blocks + 5
    _, st = gpu_step(d, L)
    assert int(st.item()) == 101
    # a length past the table
    d = to_device(L, V, cuda_device)
    d["lens"][0] = L.max_blocks_per_seq * 16 + 1
    _, st = gpu_step(d, L)
    assert int(st.item()) == 102
    # a slot past the pool
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    d = to_device(L, V, cuda_device)
    bad_slots = torch.tensor([L.num_blocks * 16 + 3], dtype=torch.int64, device=cuda_device)
    pa_mod.pa_cache_write(d["q"][:1, :2], d["q"][:1, :2], bad_slots, d["k_pool"], d["v_pool"], st)
    torch.cuda.synchronize()
    assert int(st.item()) == 103
    # a copy pair past the pool
    st.zero_()
    pa_mod.pa_copy_blocks(torch.tensor([[0, L.num_blocks]], dtype=torch.int64, device=cuda_device), d["k_pool"],
                          d["v_pool"], st)
    torch.cuda.synchronize()
    assert int(st.item()) == 104
    # the context is still usable
    L3 = config_tiny()
    _run_and_check(L3, fill_values_numpy(L3), cuda_device, what="after errors")


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [8, 16, 32])
def test_tensor_core_and_cuda_core_paths_agree(pa_mod, cuda_device, dtype, G, B):
    """Every group size at head_dim 128 and blocks of 8, 16 or 32 tokens runs
    on the tensor-core kernel by default; the CUDA-core kernel is forced with
    a flag.  Both must match the oracle, and each other to within the
    combined tolerance."""
    import torch

    lens = [1, 2, B - 1, B, B + 1, 127, 128, 129, 300, 1000, 2049, 5]
    L = random_layout(4000 + 10 * B + G, lens, dtype=dtype, block_size=B, num_q_heads=2 * G, num_kv_heads=2,
                      head_dim=128, write_new_token=True)
    V = fill_values_numpy(L)
    ref, _, _ = oracle_step(L, V)
    outs = {}
    for name, flags in (("tensor", 0), ("cuda", pa_mod.PA_DECODE_CUDA_CORES_ONLY)):
        d = to_device(L, V, cuda_device)
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        pa_mod.pa_cache_write(d["new_k"], d["new_v"], d["slots"], d["k_pool"], d["v_pool"], st)
        out = torch.full_like(d["q"], float("nan"))
        ws = pa_mod.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"], flags=flags)
        pa_mod.pa_decode(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st,
                         flags=flags)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, name
        outs[name] = torch_f64(out)
        assert_attention_close(outs[name], ref, f"{name} G={G} {dtype}")
    # both sit within the tolerance of the oracle, so they differ by at most twice it
    diff = np.abs(outs["tensor"] - outs["cuda"])
    assert (diff <= 2 * (2e-3 + 1e-2 * np.abs(ref))).all(), diff.max()
