"""GPU parity of the shared-prefix decode (pa_decode_shared_prefix: one unit
per (group, kv head) streams the group's shared blocks once for every
member's heads, then each member's own blocks for its heads) against the
float64 decode oracle — the result is plain decode; only the memory reads
differ — element by element: max-abs 2e-3 where |oracle| < 0.5, max-rel
1e-2 where |oracle| >= 0.1.  Groups come from
pa_shared_prefix_groups on the host tables."""

import numpy as np
import pytest

import oracle
from pa_testlib import assert_attention_close, gpu_step, oracle_step, subproblem, oracle_subproblem, to_device
from pa_testlib import torch_f64
from workloads import (
    bits_to_torch,
    config_llama2_70b_shared,
    f32_to_bits,
    fill_values_numpy,
    fill_values_torch,
)
from workloads.generate import PAD_ENTRY, PagedLayout, _finish_layout

pytestmark = pytest.mark.gpu


def _forked_layout(seed, prompts, dtype="bf16", G=4, Hkv=2, B=16, extra_blocks=8):
    """Prompts forked into samples: `prompts` is a list of (prompt_len,
    [tail lengths]); every sample shares the prompt's full blocks and owns a
    copy of a partly filled last prompt block plus its tail (the layout the
    block manager leaves after forking and one copy on write per sample)."""
    rng = np.random.default_rng(seed)
    lens, rows = [], []
    need = 0
    for plen, tails in prompts:
        full = plen // B
        for t in tails:
            n = plen + t
            lens.append(n)
            need += -(-n // B) - full
        need += full
    NB = need + extra_blocks
    perm = rng.permutation(NB).astype(np.int32)
    cur = 0
    for plen, tails in prompts:
        full = plen // B
        shared = perm[cur:cur + full]
        cur += full
        for t in tails:
            n = plen + t
            own = -(-n // B) - full
            rows.append(np.concatenate([shared, perm[cur:cur + own]]))
            cur += own
    max_nb = max(len(r) for r in rows)
    tables = np.full((len(rows), max_nb), PAD_ENTRY, np.int32)
    for s, r in enumerate(rows):
        tables[s, : len(r)] = r
    return _finish_layout("forked", seed, dtype, B, NB, Hkv * G, Hkv, 128, np.asarray(lens, np.int32), tables, True)


def _run(device, layout, values, groups, max_group, num_ctas=0):
    import torch

    import paged_kv_cache_357_b200 as pa

    d = to_device(layout, values, device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    if layout.copy_pairs.shape[0] > 0:
        pa.pa_copy_blocks(d["pairs"], d["k_pool"], d["v_pool"], st)
    if layout.num_new_tokens > 0:
        pa.pa_cache_write(d["new_k"], d["new_v"], d["slots"], d["k_pool"], d["v_pool"], st)
    starts, prefix = groups
    gs = torch.from_numpy(starts).to(device)
    gp = torch.from_numpy(prefix).to(device)
    out = torch.full_like(d["q"], float("nan"))
    ws = pa.alloc_shared_prefix_workspace(layout.num_seqs, max_group, layout.num_q_heads, d["k_pool"], num_ctas)
    pa.pa_decode_shared_prefix(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], gs, gp, max_group,
                               layout.scale, out, ws, st, num_ctas=num_ctas)
    torch.cuda.synchronize()
    return out, int(st.item()), d, ws


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_forked_samples_match_oracle(cuda_device, G, dtype):
    import paged_kv_cache_357_b200 as pa

    prompts = [(40, [1, 5, 30]), (300, [1, 2, 17, 64]), (17, [1]), (128, [1, 129]), (1000, [3, 40, 200, 7])]
    max_group = 4
    L = _forked_layout(8000 + G, prompts, dtype=dtype, G=G)
    V = fill_values_numpy(L)
    groups = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, max_group)
    starts, prefix = groups
    # every prompt is one group sharing its full prompt blocks (capped below each member's own blocks)
    assert starts.tolist() == [0, 3, 7, 8, 10, 14]
    assert prefix.tolist() == [2, 18, 0, 8, 62]
    out, st, _, _ = _run(cuda_device, L, V, groups, max_group)
    assert st == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, f"shared prefix G={G} {dtype}")


@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("G", [2, 8])
def test_forked_samples_other_block_sizes(cuda_device, G, B):
    """The same forked prompts at blocks of 8 and 32 tokens: 16 or 4 blocks
    a 128-token chunk, the shared prefix and each member's own blocks in
    whole granules of them; with 8-token blocks a prompt's partly filled
    last block is private to every sample more often."""
    import paged_kv_cache_357_b200 as pa

    prompts = [(40, [1, 5, 30]), (300, [1, 2, 17, 64]), (17, [1]), (128, [1, 129]), (1000, [3, 40, 200, 7])]
    dtype = "bf16" if B == 8 else "fp16"
    L = _forked_layout(8050 + 10 * G + B, prompts, dtype=dtype, G=G, B=B)
    V = fill_values_numpy(L)
    groups = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, 4)
    out, st, _, _ = _run(cuda_device, L, V, groups, 4)
    assert st == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, f"shared prefix G={G} B={B} {dtype}")


@pytest.mark.parametrize("num_ctas", [1, 2, 5, 33, 0])
def test_split_group_units(cuda_device, num_ctas):
    import paged_kv_cache_357_b200 as pa

    prompts = [(2048, [1, 100, 513]), (64, [1, 2]), (700, [260])]
    L = _forked_layout(8100 + num_ctas, prompts, G=8)
    V = fill_values_numpy(L)
    groups = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, 4)
    out, st, _, _ = _run(cuda_device, L, V, groups, 4, num_ctas)
    assert st == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, f"num_ctas={num_ctas}")


@pytest.mark.parametrize("members", [5, 8])
def test_large_groups(cuda_device, members):
    import paged_kv_cache_357_b200 as pa

    prompts = [(500, list(range(1, members + 1))), (90, [3] * members)]
    L = _forked_layout(8200 + members, prompts, G=4)
    V = fill_values_numpy(L)
    groups = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, members)
    assert len(groups[0]) == 3
    out, st, _, _ = _run(cuda_device, L, V, groups, members)
    assert st == 0
    ref, _, _ = oracle_step(L, V)
    assert_attention_close(torch_f64(out), ref, f"{members} members")


def test_workspace_reuse_and_changing_groups(cuda_device):
    """Two calls with different groupings on one workspace: the second must
    not see the first call's prefix lengths or states."""
    import paged_kv_cache_357_b200 as pa

    L = _forked_layout(8300, [(400, [1, 9, 20, 33]), (260, [4, 4])], G=4)
    V = fill_values_numpy(L)
    g1 = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, 4)
    ref, _, _ = oracle_step(L, V)
    out1, st1, d, ws = _run(cuda_device, L, V, g1, 4)
    assert st1 == 0
    assert_attention_close(torch_f64(out1), ref, "grouped")
    # now every sequence alone (prefix 0): a plain decode through the same workspace
    import torch

    starts = np.arange(L.num_seqs + 1, dtype=np.int32)
    prefix = np.zeros(L.num_seqs, np.int32)
    out2 = torch.full_like(d["q"], float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pa.pa_decode_shared_prefix(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"],
                               torch.from_numpy(starts).to(cuda_device), torch.from_numpy(prefix).to(cuda_device),
                               4, L.scale, out2, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_attention_close(torch_f64(out2), ref, "ungrouped")


def test_bad_partition_is_flagged(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa

    L = _forked_layout(8400, [(100, [1, 2]), (50, [1])], G=2)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    ws = pa.alloc_shared_prefix_workspace(L.num_seqs, 2, L.num_q_heads, d["k_pool"])
    out = torch.empty_like(d["q"])
    for starts, prefix in (([0, 2], [6]), ([0, 2, 2, 4], [6, 0, 0]), ([0, 3, 3], [2, 0])):
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        pa.pa_decode_shared_prefix(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"],
                                   torch.tensor(starts, dtype=torch.int32, device=cuda_device),
                                   torch.tensor(prefix, dtype=torch.int32, device=cuda_device), 2, L.scale, out,
                                   ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 106, (starts, prefix)


def test_unsupported_group_size_is_refused(cuda_device):
    import paged_kv_cache_357_b200 as pa

    L = _forked_layout(8500, [(100, [1, 2])], G=8)
    kp = bits_to_torch(fill_values_numpy(L).k_pool, "bf16").to(cuda_device)
    with pytest.raises(pa.PaError) as e:
        pa.shared_prefix_workspace_bytes(L.num_seqs, 5, L.num_q_heads, kp)  # 8 heads x 8 members > 32 rows
    assert e.value.code == 2


@pytest.mark.parametrize("one_launch", [True, False], ids=["one_launch", "separate"])
def test_llama2_70b_shared_full_size(cuda_device, one_launch):
    """The 70B shared-prefix workload at full size through the shared-prefix
    decode: sampled sequences (whole groups among them) against the oracle,
    with the step's writes inside the decode's launch (what the benchmark
    times) or as their own launch.  The oracle applies the step's copies and
    writes to the sampled sequences' blocks before its decode, so a missed
    or late copy or write shows in their outputs."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama2_70b_shared()
    V = fill_values_torch(L, cuda_device)
    rng = np.random.default_rng(9)
    seqs = sorted({int(np.argmin(L.seq_lens)), int(np.argmax(L.seq_lens)),
                   *map(int, rng.choice(L.num_seqs, 5, replace=False)),
                   *L.share_groups[int(rng.integers(len(L.share_groups)))]})
    sub = subproblem(L, V, seqs)
    d = dict(q=V.q, k_pool=V.k_pool, v_pool=V.v_pool, new_k=V.new_k, new_v=V.new_v,
             tables=torch.from_numpy(L.block_tables).to(cuda_device),
             lens=torch.from_numpy(L.seq_lens).to(cuda_device),
             slots=torch.from_numpy(L.slot_mapping).to(cuda_device),
             pairs=torch.from_numpy(L.copy_pairs.reshape(-1, 2)).to(cuda_device))
    starts, prefix = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, 4)
    assert len(prefix) == len(L.share_groups) and (prefix == 2048 // 16 - 1).all()
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = torch.full_like(d["q"], float("nan"))
    ws = pa.alloc_shared_prefix_workspace(L.num_seqs, 4, L.num_q_heads, d["k_pool"])
    gs, gp = torch.from_numpy(starts).to(cuda_device), torch.from_numpy(prefix).to(cuda_device)
    if one_launch:
        pa.pa_decode_shared_prefix_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], gs, gp, 4,
                                          L.scale, out, ws, st, copy_pairs=d["pairs"], new_k=d["new_k"],
                                          new_v=d["new_v"], slot_mapping=d["slots"])
    else:
        pa.pa_copy_blocks(d["pairs"], d["k_pool"], d["v_pool"], st)
        pa.pa_cache_write(d["new_k"], d["new_v"], d["slots"], d["k_pool"], d["v_pool"], st)
        pa.pa_decode_shared_prefix(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], gs, gp, 4, L.scale,
                                   out, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.isfinite(out).all()
    ref = oracle_subproblem(L, sub)
    assert_attention_close(torch_f64(out)[seqs], ref, "llama2_70b_shared")
