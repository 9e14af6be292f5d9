"""The five workloads at full size, in the launch configuration the
benchmark times (default CTA count), in both step forms: the writes inside
the decode's launch (pa_decode_update, what the benchmark times) and the
separate pa_copy_blocks / pa_cache_write / pa_decode launches.

* Pools, bit-exact and whole: both pools are copied to the host before the
  step, the oracle applies the step's block copies and cache writes to those
  copies, and after the step every bit of both device pools must equal the
  oracle's (every written row, every copy-on-write destination, and every
  block the step must leave alone).
* Decode, against the oracle on sampled sequences — the shortest, the
  longest and a seeded random few, every query head (a subset of heads for
  the 32k-token sequences) — within the tolerance of tests/pa_testlib.py,
  whose max-abs and max-rel errors are printed per workload; plus properties
  that hold for every output: finite, and inside the range of the values
  attended."""

import numpy as np
import pytest

import oracle
from pa_testlib import assert_attention_close, gpu_step, oracle_subproblem, subproblem, torch_bits, torch_f64
from workloads import CONFIGS, fill_values_numpy, fill_values_torch

pytestmark = pytest.mark.gpu


def _device_inputs(L, V, device):
    import torch

    return dict(q=V.q, k_pool=V.k_pool, v_pool=V.v_pool, new_k=V.new_k, new_v=V.new_v,
                tables=torch.from_numpy(L.block_tables).to(device), lens=torch.from_numpy(L.seq_lens).to(device),
                slots=torch.from_numpy(L.slot_mapping).to(device),
                pairs=torch.from_numpy(L.copy_pairs.reshape(-1, 2)).to(device))


def _sample(L, k, seed):
    rng = np.random.default_rng(seed)
    lens = L.seq_lens
    pick = {int(np.argmin(lens)), int(np.argmax(lens))}
    pick.update(int(s) for s in rng.choice(L.num_seqs, size=min(k, L.num_seqs), replace=False))
    if L.share_groups:
        pick.update(L.share_groups[int(rng.integers(len(L.share_groups)))])
    return sorted(pick)


@pytest.mark.parametrize("one_launch", [True, False], ids=["one_launch", "separate"])
@pytest.mark.parametrize("name", ["tiny", "llama7b", "llama3_8b", "llama2_70b_shared", "opt13b_long_b8",
                                  "opt13b_long_b16", "opt13b_long_b32"])
def test_config_full_size(cuda_device, name, one_launch):
    import torch

    import paged_kv_cache_357_b200 as pa

    pa.load()
    L = CONFIGS[name]()
    if name == "tiny":
        from workloads.generate import PagedValues

        Vn = fill_values_numpy(L)
        from workloads import bits_to_torch

        V = PagedValues(*(bits_to_torch(x, L.dtype).to(cuda_device) for x in
                          (Vn.q, Vn.k_pool, Vn.v_pool, Vn.new_k, Vn.new_v)))
    else:
        V = fill_values_torch(L, cuda_device)
    long_ctx = name.startswith("opt13b")
    seqs = _sample(L, 2 if long_ctx else 8, seed=len(name))
    heads = [0, 7, 21, 39] if long_ctx else None
    sub = subproblem(L, V, seqs)  # pre-step state, captured before any kernel runs
    k_before, v_before = torch_bits(V.k_pool), torch_bits(V.v_pool)
    vmax = float(V.v_pool.float().nan_to_num(0).abs().max())
    if V.new_v.numel() > 0:
        vmax = max(vmax, float(V.new_v.float().abs().max()))
    d = _device_inputs(L, V, cuda_device)
    out, st = gpu_step(d, L, one_launch=one_launch)
    assert int(st.item()) == 0

    # the whole pools after the step, bit for bit, against the oracle's copy and write
    want_k, want_v = k_before, v_before
    if L.copy_pairs.shape[0] > 0:
        want_k, want_v = oracle.copy_blocks(want_k, want_v, L.copy_pairs)
    if L.num_new_tokens > 0:
        want_k, want_v = oracle.cache_write(want_k, want_v, torch_bits(V.new_k), torch_bits(V.new_v),
                                            L.slot_mapping)
    del k_before, v_before
    for pool, dev_pool, want in (("k", d["k_pool"], want_k), ("v", d["v_pool"], want_v)):
        got_bits = torch_bits(dev_pool)
        diff = np.flatnonzero((got_bits != want).reshape(got_bits.shape[0], -1).any(axis=1))
        assert diff.size == 0, f"{name}: {pool} pool differs from the oracle in blocks {diff[:8].tolist()}"
        del got_bits
    print(f"{name}: pools bit-exact ({L.copy_pairs.shape[0]} block copies, {L.num_new_tokens} written tokens, "
          f"{want_k.shape[0]} blocks)")
    del want_k, want_v
    assert torch.isfinite(out).all()
    assert float(out.float().abs().max()) <= vmax * (1 + 1e-2)
    ref = oracle_subproblem(L, sub, heads)
    got = torch_f64(out)[seqs]
    if heads is not None:
        got = got[:, heads]
    max_abs, max_rel, max_all = assert_attention_close(got, ref, name)
    print(f"{name}: decode max-abs {max_abs:.2e} (|ref| < 0.5), max-rel {max_rel:.2e} (|ref| >= 0.1), "
          f"max-abs over all {max_all:.2e}")
