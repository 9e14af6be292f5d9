"""GPU parity of the pieces that split a sequence across GPUs by blocks:
pa_decode_lse (the decode plus each row's log normaliser) and
pa_merge_partials (the online-softmax merge of decodes of disjoint token
ranges, study notes ch.05 §4), against the oracle's decode_lse and
merge_outputs.

Tolerances:
* outputs of pa_decode_lse: the decode's (tests/pa_testlib.py);
* log normalisers: |gpu - oracle| <= 1e-3 + 1e-5 |oracle|.  The scores are
  fp32 sums of 128 products of 16-bit values; a shift of 1e-3 in a part's
  normaliser moves its merge weight by 0.1 %, a tenth of the output bound;
* merged outputs: the decode's bound plus 2^-8 max_r |out_r| per element,
  since each part's output was already rounded to the 16-bit type (half a
  unit in the last place, 2^-9 relative, for bf16) before the merge.
"""

import numpy as np
import pytest

import oracle
from pa_testlib import ATOL, RTOL, assert_attention_close, to_device, torch_f64
from workloads import fill_values_numpy, random_layout

pytestmark = pytest.mark.gpu

LSE_ATOL, LSE_RTOL = 1e-3, 1e-5


def _assert_lse_close(got, want, what):
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf rows differ"
    fin = np.isfinite(want)
    err = np.abs(got[fin] - want[fin])
    assert (err <= LSE_ATOL + LSE_RTOL * np.abs(want[fin])).all(), f"{what}: lse max err {err.max():.3e}"


def _run_lse(L, V, device, num_ctas=0, tables=None, lens=None):
    import torch

    import paged_kv_cache_357_b200 as pa

    d = to_device(L, V, device)
    if tables is not None:
        d["tables"] = torch.from_numpy(tables).to(device)
        d["lens"] = torch.from_numpy(lens).to(device)
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full(d["q"].shape[:2], float("nan"), dtype=torch.float32, device=device)
    ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"], num_ctas)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    pa.pa_decode_lse(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, lse, ws, st,
                     num_ctas=num_ctas)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out, lse


@pytest.mark.parametrize("num_ctas", [0, 3])
@pytest.mark.parametrize("B", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_lse_matches_oracle(cuda_device, G, B, num_ctas):
    lens = [0, 1, B - 1, B, B + 1, 300, 2500, 4097]
    L = random_layout(7000 + 100 * G + B + num_ctas, lens, dtype="bf16", block_size=B, num_q_heads=2 * G,
                      num_kv_heads=2, head_dim=128, write_new_token=False)
    V = fill_values_numpy(L)
    out, lse = _run_lse(L, V, cuda_device, num_ctas)
    want_out, want_lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                           L.num_kv_heads, L.dtype)
    assert_attention_close(torch_f64(out), want_out, f"decode_lse G={G} B={B}")
    _assert_lse_close(lse.double().cpu().numpy(), want_lse, f"decode_lse G={G} B={B}")


@pytest.mark.parametrize("R", [2, 3, 5])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_block_ranges_merge_to_the_whole_decode(cuda_device, R, dtype):
    """Each sequence cut at block boundaries into R ranges, as R ranks each
    holding one range would decode them (ranges past a short sequence are
    empty), then merged on the GPU: the whole decode and its normaliser."""
    import torch

    import paged_kv_cache_357_b200 as pa

    B = 16
    lens = [1, 100, 4096, 10000, 0, 777]
    L = random_layout(8100 + R, lens, dtype=dtype, block_size=B, num_q_heads=8, num_kv_heads=2, head_dim=128,
                      write_new_token=False)
    V = fill_values_numpy(L)
    step = -(-max(lens) // (R * B)) * B  # range length, a block multiple
    outs, lses = [], []
    for r in range(R):
        a, b = r * step, (r + 1) * step
        lens_r = np.clip(L.seq_lens - a, 0, b - a).astype(np.int32)
        tables_r = np.zeros_like(L.block_tables)
        tables_r[:, : L.block_tables.shape[1] - a // B] = L.block_tables[:, a // B:]
        o, l = _run_lse(L, V, cuda_device, tables=tables_r, lens=lens_r)
        outs.append(o)
        lses.append(l)
    outs_t, lses_t = torch.stack(outs), torch.stack(lses)
    out = torch.full_like(outs[0], float("nan"))
    lse = torch.full_like(lses[0], float("nan"))
    pa.pa_merge_partials(outs_t, lses_t, out, lse)
    torch.cuda.synchronize()
    want_out, want_lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                           L.num_kv_heads, L.dtype)
    got = torch_f64(out)
    parts = np.abs(torch_f64(outs_t)).max(axis=0)
    err = np.abs(got - want_out)
    bound = ATOL + RTOL * np.abs(want_out) + 2.0 ** -8 * parts
    assert np.isfinite(got).all() and (err <= bound).all(), f"R={R}: max err {err.max():.3e}"
    _assert_lse_close(lse.double().cpu().numpy(), want_lse, f"merged lse R={R}")
    assert (got[L.seq_lens == 0] == 0).all()


@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "fp16"), (64, "bf16")])
def test_merge_kernel_matches_oracle_merge(cuda_device, D, dtype):
    """The merge kernel on the same 16-bit inputs as the oracle's merge:
    random parts with some -inf normalisers, whole rows that no part saw
    among them."""
    import torch

    import paged_kv_cache_357_b200 as pa
    from workloads import bits_to_torch, f32_to_bits

    rng = np.random.default_rng(D)
    R, rows = 4, 1000
    outs_bits = f32_to_bits(rng.standard_normal((R, rows, D)).astype(np.float32), dtype)
    lses = (rng.standard_normal((R, rows)) * 20).astype(np.float32)
    lses[rng.random((R, rows)) < 0.2] = -np.inf
    lses[:, 7] = -np.inf  # a row no part saw
    outs = bits_to_torch(outs_bits, dtype).to(cuda_device)
    out = torch.full((rows, D), float("nan"), dtype=outs.dtype, device=cuda_device)
    lse = torch.full((rows,), float("nan"), dtype=torch.float32, device=cuda_device)
    pa.pa_merge_partials(outs, torch.from_numpy(lses).to(cuda_device), out, lse)
    torch.cuda.synchronize()
    want_out, want_lse = oracle.merge_outputs(oracle.bits_to_f64(outs_bits, dtype), lses.astype(np.float64))
    assert_attention_close(torch_f64(out), want_out, f"merge D={D} {dtype}")
    _assert_lse_close(lse.double().cpu().numpy(), want_lse, f"merge lse D={D}")
    assert (torch_f64(out)[7] == 0).all()


def test_decode_lse_only_on_tensor_cores(cuda_device):
    """The log normalisers come from the tensor-core kernel: head_dim 64 (the
    CUDA-core kernel's shapes) and the CUDA-cores flag are refused."""
    import torch

    import paged_kv_cache_357_b200 as pa

    for D, flags in ((64, 0), (128, pa.PA_DECODE_CUDA_CORES_ONLY)):
        L = random_layout(5, [10, 20], dtype="bf16", block_size=16, num_q_heads=4, num_kv_heads=2, head_dim=D,
                          write_new_token=False)
        V = fill_values_numpy(L)
        d = to_device(L, V, cuda_device)
        lse = torch.empty((2, 4), dtype=torch.float32, device=cuda_device)
        ws = pa.alloc_decode_workspace(2, 4, d["k_pool"], 0, flags)
        with pytest.raises(pa.PaError) as e:
            pa.pa_decode_lse(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale,
                             torch.empty_like(d["q"]), lse, ws, flags=flags)
        assert e.value.code == 2


def test_decode_split_end_to_end_on_one_nccl_rank(cuda_device):
    """split.decode_split through a one-rank NCCL process group on this GPU:
    pa_decode_lse of the rank's range (here the whole sequences), the
    all-gather, pa_merge_partials; the result is the whole decode."""
    import datetime
    import os
    import socket

    import torch
    import torch.distributed as dist

    import paged_kv_cache_357_b200 as pa
    from paged_kv_cache_357_b200.split import decode_split

    L = random_layout(8300, [0, 1, 100, 4097, 777], dtype="bf16", block_size=16, num_q_heads=8, num_kv_heads=2,
                      head_dim=128, write_new_token=False)
    V = fill_values_numpy(L)
    d = to_device(L, V, cuda_device)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=cuda_device)
    try:
        out = torch.full_like(d["q"], float("nan"))
        lse = torch.full(d["q"].shape[:2], float("nan"), dtype=torch.float32, device=cuda_device)
        ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, d["k_pool"])
        st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        decode_split(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], L.scale, out, ws, st, lse_out=lse)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
    finally:
        dist.destroy_process_group()
    want_out, want_lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                           L.num_kv_heads, L.dtype)
    got = torch_f64(out)
    err = np.abs(got - want_out)
    # one part: the merge rescales by exactly 1, so only the part's own rounding and the merge's add up
    assert (err <= ATOL + RTOL * np.abs(want_out) + 2.0 ** -8 * np.abs(got)).all(), err.max()
    _assert_lse_close(lse.double().cpu().numpy(), want_lse, "decode_split")
