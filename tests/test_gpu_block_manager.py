"""The host block manager driving the kernels, step by step: prompts forked
into samples (shared blocks), one token appended per live sequence per step
(copy on write of shared blocks, new blocks when full), finished sequences
freed and new prompts reusing their blocks.  The oracle follows the same
history with its own manager; the C++ manager's arrays must equal the
oracle manager's bit for bit, and every decode must match the oracle."""

import numpy as np
import pytest

import oracle
from pa_testlib import assert_attention_close, oracle_manager_step, run_beam_trace, torch_bits
from workloads import bits_to_torch, f32_to_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G", [1, 4])
def test_block_manager_drives_decode_steps(cuda_device, G):
    import torch

    import paged_kv_cache_357_b200 as pa

    rng = np.random.default_rng(40 + G)
    B, NB, Hkv, D, dtype = 16, 160, 2, 128, "bf16"
    Hq = Hkv * G
    scale = 1.0 / np.sqrt(D)
    max_nb = 24
    ours = pa.BlockManager(NB, B)
    ref = oracle.BlockManager(NB, B)
    ref_tables = {}

    # pools: random values everywhere (slots are written before they are read)
    kp_bits = f32_to_bits(rng.standard_normal((NB, Hkv, B, D), dtype=np.float32), dtype)
    vp_bits = f32_to_bits(rng.standard_normal((NB, Hkv, B, D), dtype=np.float32), dtype)
    kp = bits_to_torch(kp_bits, dtype).to(cuda_device)
    vp = bits_to_torch(vp_bits, dtype).to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)

    def new_prompt(sid, n, samples):
        ours.add(sid, n)
        ref_tables[sid] = [ref.new_sequence(n), n]
        for k in range(1, samples):
            ours.fork(sid, sid + k)
            ref_tables[sid + k] = [ref.fork(ref_tables[sid][0]), n]

    new_prompt(0, 40, 3)      # 3 samples share a 2.5-block prompt
    new_prompt(10, 100, 2)    # 2 samples share a 6.25-block prompt
    new_prompt(20, 17, 1)
    live = [0, 1, 2, 10, 11, 20]
    ws = pa.alloc_decode_workspace(16, Hq, kp)
    for step in range(30):
        if step == 12:  # a sample finishes; a new prompt takes its blocks
            ours.free(1)
            ref.free_sequence(ref_tables.pop(1)[0])
            live.remove(1)
            new_prompt(30, 70, 2)
            live += [30, 31]
        tables, lens, slots, pairs = ours.prepare_step(live, max_nb)
        rt, rl, rs, rp = oracle_manager_step(ref, ref_tables, live, max_nb)
        assert np.array_equal(tables, rt) and np.array_equal(lens, rl)
        assert np.array_equal(slots, rs) and np.array_equal(pairs, rp)

        n = len(live)
        q = f32_to_bits(rng.standard_normal((n, Hq, D), dtype=np.float32), dtype)
        nk = f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
        nv = f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)  # noqa: E731
        if pairs.shape[0]:
            pa.pa_copy_blocks(dev(pairs), kp, vp, st)
        pa.pa_cache_write(bits_to_torch(nk, dtype).to(cuda_device), bits_to_torch(nv, dtype).to(cuda_device),
                          dev(slots), kp, vp, st)
        out = torch.full((n, Hq, D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        pa.pa_decode(bits_to_torch(q, dtype).to(cuda_device), kp, vp, dev(tables), dev(lens), scale, out, ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0

        kp_bits, vp_bits = oracle.copy_blocks(kp_bits, vp_bits, rp)
        kp_bits, vp_bits = oracle.cache_write(kp_bits, vp_bits, nk, nv, rs)
        ref_out = oracle.decode(q, kp_bits, vp_bits, rt, rl, scale, Hkv, dtype)
        assert_attention_close(out.double().cpu().numpy(), ref_out, f"step {step}")
    assert np.array_equal(torch_bits(kp), kp_bits) and np.array_equal(torch_bits(vp), vp_bits)
    st_ours = ours.stats()
    assert st_ours["shared_blocks"] > 0 and st_ours["free_blocks"] == len(ref.free)


def test_beam_search_drives_decode_steps(cuda_device):
    """A beam-search trace (study notes ch.05 §6.2: beams share the blocks
    of their common history, branch by fork, copy a shared partial block
    before writing, free the beams that die) driven step by step through the
    copy, write and decode kernels; every step's pools and outputs must
    match the oracle's."""
    import torch

    import paged_kv_cache_357_b200 as pa

    rng = np.random.default_rng(77)
    B, Hkv, D, G, dtype = 16, 2, 128, 4, "bf16"
    Hq, width, steps, prompt = Hkv * G, 6, 24, 203
    max_nb = (prompt + steps) // B + 2
    NB = 4 * width * max_nb
    scale = 1.0 / np.sqrt(D)
    state = {}
    state["kb"] = f32_to_bits(rng.standard_normal((NB, Hkv, B, D), dtype=np.float32), dtype)
    state["vb"] = f32_to_bits(rng.standard_normal((NB, Hkv, B, D), dtype=np.float32), dtype)
    kp = bits_to_torch(state["kb"], dtype).to(cuda_device)
    vp = bits_to_torch(state["vb"], dtype).to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = pa.alloc_decode_workspace(width, Hq, kp)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)  # noqa: E731
    copies = []

    def on_step(i, live, arrays):
        tables, lens, slots, pairs = arrays
        n = len(live)
        q = f32_to_bits(rng.standard_normal((n, Hq, D), dtype=np.float32), dtype)
        nk = f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
        nv = f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
        if pairs.shape[0]:
            pa.pa_copy_blocks(dev(pairs), kp, vp, st)
        copies.append(pairs.shape[0])
        pa.pa_cache_write(bits_to_torch(nk, dtype).to(cuda_device), bits_to_torch(nv, dtype).to(cuda_device),
                          dev(slots), kp, vp, st)
        out = torch.full((n, Hq, D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        pa.pa_decode(bits_to_torch(q, dtype).to(cuda_device), kp, vp, dev(tables), dev(lens), scale, out, ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"beam step {i}"
        state["kb"], state["vb"] = oracle.copy_blocks(state["kb"], state["vb"], pairs)
        state["kb"], state["vb"] = oracle.cache_write(state["kb"], state["vb"], nk, nv, slots)
        ref_out = oracle.decode(q, state["kb"], state["vb"], tables, lens, scale, Hkv, dtype)
        assert_attention_close(out.double().cpu().numpy(), ref_out, f"beam step {i}")

    hist = run_beam_trace(pa.BlockManager(NB, B), oracle.BlockManager(NB, B), prompt, width, steps, seed=12,
                          max_nb=max_nb, on_step=on_step, keep=0.5)
    assert np.array_equal(torch_bits(kp), state["kb"]) and np.array_equal(torch_bits(vp), state["vb"])
    assert sum(copies) > 0  # branching beams copied shared partial blocks
    print(f"beam decode: {steps} steps, {sum(copies)} block copies, final KV saved "
          f"{100 * (1 - hist[-1][0] / hist[-1][1]):.1f} %")
