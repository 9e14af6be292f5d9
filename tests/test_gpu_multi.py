"""GPU parity of multi-query paged attention (pa_decode_multi, the
tensor-core kernel with q_len causal positions per sequence) against the
float64 oracle's decode_multi, element by element: max-abs
2e-3 where |oracle| < 0.5, max-rel 1e-2 where |oracle| >= 0.1.  Inputs: seeded layouts whose cache already holds every
token (the q_len new ones included), padding rows and unused blocks NaN."""

import numpy as np
import pytest

import oracle
from pa_testlib import assert_attention_close, subproblem, torch_bits, torch_f64
from workloads import (bits_to_torch, config_llama3_8b, config_llama3_8b_prefill, f32_to_bits, fill_values_numpy,
                       fill_values_torch, random_layout)

pytestmark = pytest.mark.gpu


def _inputs(seed, lens, G, L, dtype, Hkv=2, block_size=16, head_dim=128):
    layout = random_layout(seed, lens, dtype=dtype, block_size=block_size, num_q_heads=Hkv * G, num_kv_heads=Hkv,
                           head_dim=head_dim, write_new_token=False)
    vals = fill_values_numpy(layout)
    rng = np.random.default_rng([seed, 99])
    q = f32_to_bits(rng.standard_normal((layout.num_seqs, L, layout.num_q_heads, head_dim), dtype=np.float32),
                    dtype)
    return layout, vals, q


def _run(device, layout, vals, q_bits, num_ctas=0):
    import torch

    import paged_kv_cache_357_b200 as pa

    dt = layout.dtype
    kp = bits_to_torch(vals.k_pool, dt).to(device)
    vp = bits_to_torch(vals.v_pool, dt).to(device)
    q = bits_to_torch(q_bits, dt).to(device)
    tables = torch.from_numpy(layout.block_tables).to(device)
    lens = torch.from_numpy(layout.seq_lens).to(device)
    S, L, Hq, _ = q.shape
    out = torch.full_like(q, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=device)
    ws = pa.alloc_multi_workspace(S, L, Hq, kp, num_ctas)
    pa.pa_decode_multi(q, kp, vp, tables, lens, layout.scale, out, ws, st, num_ctas=num_ctas)
    torch.cuda.synchronize()
    return out, int(st.item())


def _oracle(layout, vals, q_bits):
    return oracle.decode_multi(q_bits, vals.k_pool, vals.v_pool, layout.block_tables, layout.seq_lens,
                               layout.scale, layout.num_kv_heads, layout.dtype)


CASES = [(G, L) for G in (1, 2, 4, 8) for L in (2, 3, 4, 5, 8, 16, 32) if G * L <= 32 and L <= 32 // G]


@pytest.mark.parametrize("G,L", CASES, ids=[f"G{g}-L{l}" for g, l in CASES])
def test_multi_shapes(cuda_device, G, L):
    dtype = "bf16" if (G + L) % 2 else "fp16"
    lens = [n for n in (L, L + 1, 15, 16, 17, 127, 128, 129, 300, 1000) if n >= L] + [0]
    layout, vals, q = _inputs(7000 + 40 * G + L, lens, G, L, dtype)
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"G={G} q_len={L} {dtype}")


TILED = [(1, 64), (2, 33), (4, 16), (4, 64), (4, 256), (8, 8), (8, 16), (8, 64), (8, 256)]


@pytest.mark.parametrize("G,L", TILED, ids=[f"G{g}-L{l}" for g, l in TILED])
def test_multi_row_tiles(cuda_device, G, L):
    """G x q_len beyond the 32 rows of one unit (prefill chunks): each
    sequence's positions are cut into row tiles of 32 / G positions, each a
    unit reading only the blocks its last position sees; the last tile may
    be partial."""
    dtype = "bf16" if L % 2 == 0 else "fp16"
    lens = [L, L + 1, 2 * L + 3, L + 130, 1000, 2049]
    layout, vals, q = _inputs(7500 + 40 * G + L, lens, G, L, dtype)
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"G={G} q_len={L} {dtype}")


BLOCK_CASES = [(B, G, L) for B in (8, 32) for G, L in ((1, 3), (4, 4), (8, 4), (4, 64))]


@pytest.mark.parametrize("B,G,L", BLOCK_CASES, ids=[f"B{b}-G{g}-L{l}" for b, g, l in BLOCK_CASES])
def test_multi_block_sizes(cuda_device, B, G, L):
    """Multi-query at blocks of 8 and 32 tokens: a chunk is still 128 tokens
    (16 or 4 blocks); one unit per sequence up to 32 rows, row tiles beyond."""
    dtype = "bf16" if (B + L) % 2 == 0 else "fp16"
    lens = [n for n in (L, L + 1, B - 1, B, B + 1, 129, 300, 1000) if n >= L]
    layout, vals, q = _inputs(7700 + 10 * B + 3 * G + L, lens, G, L, dtype, block_size=B)
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"B={B} G={G} q_len={L} {dtype}")


@pytest.mark.parametrize("num_ctas", [1, 5, 0])
def test_multi_row_tiles_split_units(cuda_device, num_ctas):
    G, L = 4, 64
    layout, vals, q = _inputs(7600 + num_ctas, [64, 300, 2500, 97], G, L, "bf16")
    out, st = _run(cuda_device, layout, vals, q, num_ctas)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"tiles num_ctas={num_ctas}")


PREFILL = [(1, 128), (1, 200), (2, 64), (2, 100), (4, 32), (4, 40), (4, 256), (8, 16), (8, 33), (8, 256)]


@pytest.mark.parametrize("G,L", PREFILL, ids=[f"G{g}-L{l}" for g, l in PREFILL])
def test_prefill_tiles(cuda_device, G, L):
    """G x q_len of at least 128 rows: the query-major kernel, one unit per
    128 rows (128 / G positions x G heads), 64-token chunks, the last tile
    ragged when q_len is not a multiple of 128 / G; sequences from exactly
    q_len tokens (the first position sees one) to past two thousand."""
    dtype = "bf16" if (G + L) % 2 == 0 else "fp16"
    lens = [L, L + 1, L + 15, L + 64, L + 65, 1000 + L, 2049]
    layout, vals, q = _inputs(7800 + 50 * G + L, lens, G, L, dtype)
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"prefill G={G} q_len={L} {dtype}")


PREFILL_BLOCKS = [(8, 4, 40), (8, 1, 200), (32, 2, 100), (32, 8, 33)]


@pytest.mark.parametrize("B,G,L", PREFILL_BLOCKS, ids=[f"B{b}-G{g}-L{l}" for b, g, l in PREFILL_BLOCKS])
def test_prefill_tiles_other_block_sizes(cuda_device, B, G, L):
    """The query-major kernel at blocks of 8 and 32 tokens: a 128-token
    chunk is 16 or 4 blocks (K as one 3-D box per 8-token block, or two
    2-D boxes per 32-token block); ragged last tiles."""
    dtype = "bf16" if B == 8 else "fp16"
    lens = [L, L + 1, L + B - 1, L + 129, 1000 + L, 2049]
    layout, vals, q = _inputs(7950 + 10 * B + G + L, lens, G, L, dtype, block_size=B)
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"prefill B={B} G={G} q_len={L} {dtype}")


@pytest.mark.parametrize("num_ctas", [1, 3, 37, 200, 0])
def test_prefill_split_units(cuda_device, num_ctas):
    """Query-major units cut between CTAs: with 200 CTAs a long unit spans
    several, so the merging CTA combines more than one published piece, and
    pieces that start past a row's causal limit carry no token for it."""
    G, L = 4, 128
    layout, vals, q = _inputs(7900 + num_ctas, [128, 700, 3000, 129, 4100], G, L, "bf16")
    out, st = _run(cuda_device, layout, vals, q, num_ctas)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"prefill num_ctas={num_ctas}")


def _bits_to_f32(bits, dtype):
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


RISING = [("bf16", 0), ("fp16", 0), ("bf16", 37)]


@pytest.mark.parametrize("dtype,num_ctas", RISING, ids=[f"{d}-ctas{n}" for d, n in RISING])
def test_prefill_rising_scores(cuda_device, dtype, num_ctas):
    """Keys whose magnitude grows along the sequence (x (1 + t / 256) at
    token t) and queries of mixed magnitude (x 0.05 .. 1.6 per row): later
    chunks pass a row's reference max by more than the lazy-rescale gap for
    some rows of a warp and not for others, so references move, and O is
    rescaled, in the middle of a unit, row by row; with 37 CTAs also across
    the pieces of split units."""
    G, L = 4, 128
    layout, vals, _ = _inputs(8100 + num_ctas, [L, L + 70, 700, 1500, 3000], G, L, dtype)
    B = layout.block_size
    k = _bits_to_f32(vals.k_pool, dtype)
    for s, n in enumerate(layout.seq_lens):
        for t in range(int(n)):
            k[layout.block_tables[s, t // B], :, t % B, :] *= 1.0 + t / 256.0
    vals.k_pool = f32_to_bits(k, dtype)
    rng = np.random.default_rng([8100, 5])
    S, Hq, D = layout.num_seqs, layout.num_q_heads, layout.head_dim
    q = f32_to_bits(rng.standard_normal((S, L, Hq, D), dtype=np.float32) *
                    rng.uniform(0.05, 1.6, size=(S, L, Hq, 1)).astype(np.float32), dtype)
    out, st = _run(cuda_device, layout, vals, q, num_ctas)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"rising scores {dtype} num_ctas={num_ctas}")


@pytest.mark.parametrize("num_ctas", [1, 3, 37, 0])
def test_multi_split_units(cuda_device, num_ctas):
    G, L = 4, 4
    lens = [4, 129, 700, 2049, 3000, 33]
    layout, vals, q = _inputs(7100 + num_ctas, lens, G, L, "bf16")
    out, st = _run(cuda_device, layout, vals, q, num_ctas)
    assert st == 0
    assert_attention_close(torch_f64(out), _oracle(layout, vals, q), f"num_ctas={num_ctas}")


def test_multi_short_sequence_is_flagged_and_zero(cuda_device):
    G, L = 2, 4
    layout, vals, q = _inputs(7200, [40, 3, 0, 100], G, L, "bf16")
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 102  # PA_DEV_BAD_SEQ_LEN for the 3-token sequence
    got = torch_f64(out)
    assert not got[1].any() and not got[2].any()
    ref = _oracle(layout, vals, q)
    assert_attention_close(got[[0, 3]], ref[[0, 3]], "other sequences")


def test_single_position_is_the_decode_kernel(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa

    layout, vals, q = _inputs(7300, [5, 130, 999], 4, 1, "bf16")
    out, st = _run(cuda_device, layout, vals, q)
    assert st == 0
    dt = layout.dtype
    kp = bits_to_torch(vals.k_pool, dt).to(cuda_device)
    vp = bits_to_torch(vals.v_pool, dt).to(cuda_device)
    q1 = bits_to_torch(q[:, 0], dt).to(cuda_device).contiguous()
    out1 = torch.empty_like(q1)
    ws = pa.alloc_decode_workspace(layout.num_seqs, layout.num_q_heads, kp)
    pa.pa_decode(q1, kp, vp, torch.from_numpy(layout.block_tables).to(cuda_device),
                 torch.from_numpy(layout.seq_lens).to(cuda_device), layout.scale, out1, ws)
    torch.cuda.synchronize()
    assert np.array_equal(torch_bits(out[:, 0]), torch_bits(out1))


def test_unsupported_shapes_are_refused(cuda_device):
    import torch

    import paged_kv_cache_357_b200 as pa

    # multi-query runs on the tensor-core kernel only: head_dim 128
    layout, vals, q = _inputs(7400, [64, 80], 8, 8, "bf16", head_dim=64)
    kp = bits_to_torch(vals.k_pool, "bf16").to(cuda_device)
    with pytest.raises(pa.PaError) as e:
        pa.multi_workspace_bytes(2, 8, layout.num_q_heads, kp)
    assert e.value.code == 2
    qd = bits_to_torch(q, "bf16").to(cuda_device)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_multi(qd, kp, kp, torch.from_numpy(layout.block_tables).to(cuda_device),
                           torch.from_numpy(layout.seq_lens).to(cuda_device), 0.1, torch.empty_like(qd), ws)
    assert e.value.code == 2
    q2 = qd[:, :2].contiguous()
    with pytest.raises(pa.PaError) as e:  # CUDA cores have no multi-query kernel
        pa.pa_decode_multi(q2, kp, kp, torch.from_numpy(layout.block_tables).to(cuda_device),
                           torch.from_numpy(layout.seq_lens).to(cuda_device), 0.1, torch.empty_like(q2), ws,
                           flags=pa.PA_DECODE_CUDA_CORES_ONLY)
    assert e.value.code == 2


def test_llama3_8b_full_size_speculative_verify(cuda_device):
    """The Llama-3-8B decode workload at full size with 4 positions per
    sequence (the newest tokens written first), sampled sequences against
    the oracle; every output finite and inside the range of V."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama3_8b()
    V = fill_values_torch(L, cuda_device)
    qlen = 4
    g = torch.Generator(device=cuda_device)
    g.manual_seed(8081)
    dt = V.q.dtype
    q = torch.randn((L.num_seqs, qlen, L.num_q_heads, L.head_dim), generator=g, device=cuda_device).to(dt)
    rng = np.random.default_rng(5)
    seqs = sorted({int(np.argmin(L.seq_lens)), int(np.argmax(L.seq_lens)),
                   *map(int, rng.choice(L.num_seqs, 6, replace=False))})
    sub = subproblem(L, V, seqs)
    q_host = torch_bits(q[seqs])
    tables = torch.from_numpy(L.block_tables).to(cuda_device)
    lens = torch.from_numpy(L.seq_lens).to(cuda_device)
    slots = torch.from_numpy(L.slot_mapping).to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pa.pa_cache_write(V.new_k, V.new_v, slots, V.k_pool, V.v_pool, st)
    out = torch.full_like(q, float("nan"))
    ws = pa.alloc_multi_workspace(L.num_seqs, qlen, L.num_q_heads, V.k_pool)
    pa.pa_decode_multi(q, V.k_pool, V.v_pool, tables, lens, L.scale, out, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.isfinite(out).all()
    vmax = max(float(V.v_pool.float().nan_to_num(0).abs().max()), float(V.new_v.float().abs().max()))
    assert float(out.float().abs().max()) <= vmax * (1 + 1e-2)
    kp, vp = oracle.cache_write(sub["k_pool"], sub["v_pool"], sub["new_k"], sub["new_v"], sub["slots"])
    ref = oracle.decode_multi(q_host, kp, vp, sub["tables"], sub["lens"], L.scale, L.num_kv_heads, L.dtype)
    assert_attention_close(torch_f64(out)[seqs], ref, "llama3_8b q_len=4")


def test_llama3_8b_prefill256_full_size(cuda_device):
    """The 256-token prefill workload at full size, as the bench runs it:
    the cache write of every sequence's 256 new tokens, then the query-major
    kernel over all 64 sequences; the shortest sequence (whose first position
    sees one token), the median and the longest one and three more against
    the oracle, every output finite and inside the range of V."""
    import torch

    import paged_kv_cache_357_b200 as pa

    L = config_llama3_8b_prefill()
    V = fill_values_torch(L, cuda_device)
    rng = np.random.default_rng(6)
    order = np.argsort(L.seq_lens)
    seqs = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1]),
                   *map(int, rng.choice(L.num_seqs, 3, replace=False))})
    sub = subproblem(L, V, seqs)
    tables = torch.from_numpy(L.block_tables).to(cuda_device)
    lens = torch.from_numpy(L.seq_lens).to(cuda_device)
    slots = torch.from_numpy(L.slot_mapping).to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pa.pa_cache_write(V.new_k, V.new_v, slots, V.k_pool, V.v_pool, st)
    out = torch.full_like(V.q, float("nan"))
    ws = pa.alloc_multi_workspace(L.num_seqs, L.q_len, L.num_q_heads, V.k_pool)
    pa.pa_decode_multi(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, out, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.isfinite(out).all()
    vmax = max(float(V.v_pool.float().nan_to_num(0).abs().max()), float(V.new_v.float().abs().max()))
    assert float(out.float().abs().max()) <= vmax * (1 + 1e-2)
    kp, vp = oracle.cache_write(sub["k_pool"], sub["v_pool"], sub["new_k"], sub["new_v"], sub["slots"])
    ref = oracle.decode_multi(sub["q"], kp, vp, sub["tables"], sub["lens"], L.scale, L.num_kv_heads, L.dtype)
    assert_attention_close(torch_f64(out)[seqs], ref, "llama3_8b prefill q_len=256")
