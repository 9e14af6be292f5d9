"""The five workloads at full size, in the launch configuration the
benchmark times (default CTA count), against the oracle on sampled
sequences — the shortest, the longest and a seeded random few, every query
head (a subset of heads for the 32k-token sequences) — plus properties that
hold for every output: finite, and inside the range of the values attended."""

import numpy as np
import pytest

from pa_testlib import assert_attention_close, gpu_step, oracle_subproblem, subproblem, torch_f64
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


@pytest.mark.parametrize("name", ["tiny", "llama7b", "llama3_8b", "llama2_70b_shared", "opt13b_long_b8",
                                  "opt13b_long_b16", "opt13b_long_b32"])
def test_config_full_size(cuda_device, name):
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
    vmax = float(V.v_pool.float().nan_to_num(0).abs().max())
    if V.new_v.numel() > 0:
        vmax = max(vmax, float(V.new_v.float().abs().max()))
    d = _device_inputs(L, V, cuda_device)
    out, st = gpu_step(d, L)
    assert int(st.item()) == 0
    assert torch.isfinite(out).all()
    assert float(out.float().abs().max()) <= vmax * (1 + 1e-2)
    ref = oracle_subproblem(L, sub, heads)
    got = torch_f64(out)[seqs]
    if heads is not None:
        got = got[:, heads]
    assert_attention_close(got, ref, name)
