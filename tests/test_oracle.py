"""Pins of the float64 oracle against things other than itself: values the
pages print, brute force on tiny inputs, closed forms and invariants.  A
mutation test at the end plants plausible mistakes in copies of the oracle
and checks that at least one pin catches each."""

import json
import math
from pathlib import Path

import numpy as np
import pytest

import oracle
from oracle import (
    BlockManager,
    attention_dense,
    bits_to_f64,
    block_fills,
    blocks_needed,
    cache_write,
    copy_blocks,
    decode,
    decode_blockwise_online,
    decode_one,
    kv_bytes_per_token,
    merge_partition_states,
    partition_states,
)
from workloads import (
    config_llama2_70b_shared,
    config_llama3_8b,
    config_tiny,
    f32_to_bits,
    fill_values_numpy,
    random_layout,
)

GOLDEN = json.loads((Path(__file__).parent / "golden" / "bookkeeping.json").read_text())

# ---------------------------------------------------------------------------
# values printed on the pages
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("ex", GOLDEN["block_examples"], ids=lambda e: str(e["tokens"]))
def test_block_examples_from_pages(ex):
    B = ex["block_size"]
    assert blocks_needed(ex["tokens"], B) == ex["blocks"]
    fills = block_fills(ex["tokens"], B)
    assert len(fills) == ex["blocks"]
    if "fills" in ex:
        assert fills == ex["fills"]
    if "full_blocks" in ex:
        assert sum(f == B for f in fills) == ex["full_blocks"]
        assert sum(f for f in fills if f == B) == ex["tokens_in_full_blocks"]
        assert fills[-1] == ex["last_block_tokens"]
        assert 100 * fills[-1] // B == ex["last_block_fill_percent"]


def test_kv_bytes_from_pages():
    kib = 1024
    for ex in GOLDEN["kv_bytes"]:
        if "kv_heads" in ex:
            per_tok = kv_bytes_per_token(ex["layers"], ex["kv_heads"], ex["head_dim"], ex["dtype_bytes"])
            assert per_tok == ex["kib_per_token"] * kib, ex["model"]
            if "kib_per_token_per_layer" in ex:
                assert kv_bytes_per_token(1, ex["kv_heads"], ex["head_dim"], ex["dtype_bytes"]) == \
                    ex["kib_per_token_per_layer"] * kib
            if "request_mib" in ex:
                assert per_tok * ex["request_tokens"] == ex["request_mib"] * kib * kib
            if "concurrent_gib_approx" in ex:
                total = per_tok * ex["request_tokens"] * ex["concurrent_requests"]
                assert round(total / kib**3) == ex["concurrent_gib_approx"]
        else:
            # LLaMA-7B: 32 layers x hidden 4096 x 2 bytes x 8192 tokens x 2 (K and V)
            head_dim = 128
            per_tok = kv_bytes_per_token(ex["layers"], ex["hidden"] // head_dim, head_dim, ex["dtype_bytes"])
            assert per_tok * ex["context"] == ex["total_gib_approx"] * kib**3


def test_copy_on_write_example_from_pages():
    ex = GOLDEN["copy_on_write"]
    mgr = BlockManager(num_blocks=16, block_size=16)
    mgr.free.remove(ex["shared_block"])
    mgr.ref[ex["shared_block"]] = 1
    first = [ex["shared_block"]]
    outputs = [first] + [mgr.fork(first) for _ in range(ex["samples"] - 1)]
    assert mgr.ref[ex["shared_block"]] == ex["ref_before"]
    writer = outputs[ex["writer"] - 1]
    slot, cow = mgr.append_slot(writer, n_before=8)  # the block holds 8 prompt tokens
    assert cow is not None and cow[0] == ex["shared_block"]
    new_block = cow[1]
    assert writer == [new_block] and slot == new_block * 16 + 8
    assert mgr.ref[ex["shared_block"]] == ex["ref_source_after"]
    assert mgr.ref[new_block] == ex["ref_copy_after"]
    for i, t in enumerate(outputs):
        if i != ex["writer"] - 1:
            assert t == [ex["shared_block"]]
    # finishing an output drops one reference; zero frees the block
    mgr.free_sequence(writer)
    assert mgr.ref[new_block] == 0 and new_block in mgr.free


def test_on_demand_allocation_wastes_less_than_one_block():
    mgr = BlockManager(num_blocks=1000, block_size=16)
    for n in [1, 15, 16, 17, 40, 1000]:
        t = mgr.new_sequence(n)
        assert len(t) * 16 - n < 16
        # appending grows the table only when the last block is full
        before = len(t)
        mgr.append_slot(t, n)
        assert len(t) == before + (1 if n % 16 == 0 else 0)


# ---------------------------------------------------------------------------
# brute force: contiguous dense attention in plain Python loops
# ---------------------------------------------------------------------------


def _brute_attention(qv, Krows, Vrows, scale):
    n = len(Krows)
    D = len(qv)
    if n == 0:
        return [0.0] * D
    z = [scale * sum(qv[d] * Krows[t][d] for d in range(D)) for t in range(n)]
    top = max(z)
    w = [math.exp(x - top) for x in z]
    tot = sum(w)
    return [sum(w[t] * Vrows[t][d] for t in range(n)) / tot for d in range(D)]


def _scatter_contiguous(rng, seqs_k, seqs_v, B, NB, dtype):
    """Place contiguous per-sequence K/V ([n, Hkv, D] bit arrays) into a NaN
    pool at shuffled blocks; return pools and tables built here, not by the
    workload generator."""
    Hkv, D = seqs_k[0].shape[1], seqs_k[0].shape[2]
    nan = np.uint16(0x7E00 if dtype == "fp16" else 0x7FC0)
    kp = np.full((NB, Hkv, B, D), nan, np.uint16)
    vp = np.full((NB, Hkv, B, D), nan, np.uint16)
    perm = rng.permutation(NB)
    max_nb = max(1, max((k.shape[0] + B - 1) // B for k in seqs_k))
    tables = np.full((len(seqs_k), max_nb), -1, np.int32)
    off = 0
    for s, (K, V) in enumerate(zip(seqs_k, seqs_v)):
        n = K.shape[0]
        for t in range(n):
            j = t // B
            if t % B == 0:
                tables[s, j] = perm[off]
                off += 1
            kp[tables[s, j], :, t % B, :] = K[t]
            vp[tables[s, j], :, t % B, :] = V[t]
    return kp, vp, tables


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (4, 1)])
def test_oracle_matches_bruteforce_dense(dtype, Hq, Hkv):
    rng = np.random.default_rng(11)
    B, D = 4, 8
    lens = [1, 3, 4, 5, 13]
    seqs_k = [f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype) for n in lens]
    seqs_v = [f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype) for n in lens]
    q = f32_to_bits(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), dtype)
    NB = sum((n + B - 1) // B for n in lens) + 4
    kp, vp, tables = _scatter_contiguous(rng, seqs_k, seqs_v, B, NB, dtype)
    scale = 0.37
    out = decode(q, kp, vp, tables, np.array(lens, np.int32), scale, Hkv, dtype)
    g = Hq // Hkv
    for s, n in enumerate(lens):
        for h in range(Hq):
            kvh = h // g
            qv = bits_to_f64(q[s, h], dtype).tolist()
            Kr = bits_to_f64(seqs_k[s][:, kvh, :], dtype).tolist()
            Vr = bits_to_f64(seqs_v[s][:, kvh, :], dtype).tolist()
            ref = _brute_attention(qv, Kr, Vr, scale)
            np.testing.assert_allclose(out[s, h], ref, rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv_heads():
    """Grouped heads read the same K/V as an MHA pool in which kv head
    h // g is repeated g times in a row."""
    L = random_layout(5, [7, 33, 16], dtype="bf16", block_size=8, num_q_heads=8, num_kv_heads=2,
                      head_dim=16, write_new_token=False)
    V = fill_values_numpy(L)
    g = L.group
    out_gqa = decode(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 2, L.dtype)
    kp = np.repeat(V.k_pool, g, axis=1)
    vp = np.repeat(V.v_pool, g, axis=1)
    out_mha = decode(V.q, kp, vp, L.block_tables, L.seq_lens, L.scale, 8, L.dtype)
    assert np.array_equal(out_gqa, out_mha)


# ---------------------------------------------------------------------------
# invariants and closed forms
# ---------------------------------------------------------------------------


def test_physical_placement_invariance():
    L = random_layout(3, [1, 17, 40, 100], dtype="fp16", block_size=16, num_q_heads=4, num_kv_heads=2,
                      head_dim=32, write_new_token=False)
    V = fill_values_numpy(L)
    out = decode(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 2, L.dtype)
    pi = np.random.default_rng(9).permutation(L.num_blocks)
    kp = np.empty_like(V.k_pool)
    vp = np.empty_like(V.v_pool)
    kp[pi] = V.k_pool
    vp[pi] = V.v_pool
    tables = np.where(L.block_tables >= 0, pi[np.maximum(L.block_tables, 0)], -1).astype(np.int32)
    out2 = decode(V.q, kp, vp, tables, L.seq_lens, L.scale, 2, L.dtype)
    assert np.array_equal(out, out2)


def test_shared_blocks_give_identical_outputs():
    L = config_llama2_70b_shared(prompt_len=64, num_prompts=2, samples=3, max_tail=0)
    V = fill_values_numpy(L)
    kp, vp = copy_blocks(V.k_pool, V.v_pool, L.copy_pairs)
    q = V.q.copy()
    for grp in L.share_groups:
        q[grp] = q[grp[0]]
    # before the write every sample of a prompt attends the same prompt tokens
    lens = L.seq_lens - 1
    out = decode(q, kp, vp, L.block_tables, lens, L.scale, L.num_kv_heads, L.dtype)
    for grp in L.share_groups:
        for s in grp[1:]:
            assert np.array_equal(out[s], out[grp[0]])


def test_seq_len_one_returns_v0_exactly():
    L = random_layout(4, [1, 1, 1], dtype="bf16", block_size=16, num_q_heads=2, num_kv_heads=2,
                      head_dim=16, write_new_token=False)
    V = fill_values_numpy(L)
    out = decode(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 2, L.dtype)
    for s in range(3):
        for h in range(2):
            v0 = bits_to_f64(V.v_pool[L.block_tables[s, 0], h, 0], L.dtype)
            assert np.array_equal(out[s, h], v0)


def test_equal_keys_and_zero_query_give_mean_of_values():
    rng = np.random.default_rng(2)
    n, D = 37, 16
    V = rng.standard_normal((n, D))
    K_same = np.tile(rng.standard_normal(D), (n, 1))
    q = rng.standard_normal(D)
    np.testing.assert_allclose(attention_dense(q, K_same, V, 0.3), V.mean(axis=0), atol=1e-13)
    np.testing.assert_allclose(attention_dense(np.zeros(D), rng.standard_normal((n, D)), V, 0.3),
                               V.mean(axis=0), atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(3)
    n, D = 50, 8
    K = rng.standard_normal((n, D)) * 0.01
    V = rng.standard_normal((n, D))
    q = np.ones(D)
    K[17] = 40.0 / D  # score gap ~40 with scale 1
    out = attention_dense(q, K, V, 1.0)
    np.testing.assert_allclose(out, V[17], atol=n * math.exp(-39) * np.abs(V).max())


def test_zero_length_sequence_gives_zeros():
    out = attention_dense(np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)), 1.0)
    assert np.array_equal(out, np.zeros(4))


@pytest.mark.parametrize("seed", range(6))
def test_online_softmax_equals_direct(seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 90, size=5)
    L = random_layout(seed, lens, dtype="bf16", block_size=int(rng.choice([4, 8, 16])), num_q_heads=4,
                      num_kv_heads=2, head_dim=16, write_new_token=False)
    V = fill_values_numpy(L)
    for s in range(L.num_seqs):
        for h in range(4):
            a = decode_one(s, h, V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 2, L.dtype)
            b = decode_blockwise_online(s, h, V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                        2, L.dtype)
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_partition_merge_equals_direct(seed):
    rng = np.random.default_rng(100 + seed)
    L = random_layout(seed, [int(rng.integers(2, 300))], dtype="fp16", block_size=16, num_q_heads=2,
                      num_kv_heads=1, head_dim=16, write_new_token=False)
    V = fill_values_numpy(L)
    n = int(L.seq_lens[0])
    k = int(rng.integers(1, min(n, 8)))
    bounds = sorted(rng.choice(np.arange(1, n), size=k, replace=False).tolist())
    for h in range(2):
        st = partition_states(0, h, V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 1, L.dtype,
                              bounds)
        direct = decode_one(0, h, V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 1, L.dtype)
        np.testing.assert_allclose(merge_partition_states(st), direct, rtol=0, atol=1e-12)


def test_oracle_ignores_nan_padding_rows():
    L = random_layout(8, [5, 21], dtype="bf16", block_size=16, num_q_heads=2, num_kv_heads=2, head_dim=8,
                      write_new_token=False)
    V = fill_values_numpy(L)
    out = decode(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, 2, L.dtype)
    assert np.isfinite(out).all()
    # the pool really is poisoned past each sequence's last token
    assert np.isnan(bits_to_f64(V.k_pool[L.block_tables[0, 0], 0, 5], L.dtype)).all()


# ---------------------------------------------------------------------------
# cache write and block copy
# ---------------------------------------------------------------------------


def test_cache_write_places_tokens_where_the_gather_reads_them():
    L = config_tiny()
    V = fill_values_numpy(L)
    kp, vp = cache_write(V.k_pool, V.v_pool, V.new_k, V.new_v, L.slot_mapping)
    B = L.block_size
    changed = np.zeros(kp.shape[:1] + kp.shape[2:3], bool)
    for s in range(L.num_seqs):
        t = int(L.seq_lens[s]) - 1
        b, r = int(L.block_tables[s, t // B]), t % B
        assert np.array_equal(kp[b, :, r, :], V.new_k[s]) and np.array_equal(vp[b, :, r, :], V.new_v[s])
        changed[b, r] = True
    keep = ~changed[:, None, :, None].repeat(L.num_kv_heads, 1).repeat(L.head_dim, 3)
    assert np.array_equal(kp[keep], V.k_pool[keep]) and np.array_equal(vp[keep], V.v_pool[keep])
    # after the write the decode sees no NaN
    out = decode(V.q, kp, vp, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
    assert np.isfinite(out).all()


def test_cache_write_skips_negative_slots():
    L = config_tiny()
    V = fill_values_numpy(L)
    slots = L.slot_mapping.copy()
    slots[1] = -1
    kp, _ = cache_write(V.k_pool, V.v_pool, V.new_k, V.new_v, slots)
    t = int(L.seq_lens[1]) - 1
    b, r = int(L.block_tables[1, t // 16]), t % 16
    assert np.array_equal(kp[b, :, r], V.k_pool[b, :, r])


def test_copy_blocks_copies_whole_blocks_only():
    rng = np.random.default_rng(1)
    kp = rng.integers(0, 65535, size=(10, 2, 4, 8), dtype=np.uint16)
    vp = rng.integers(0, 65535, size=(10, 2, 4, 8), dtype=np.uint16)
    pairs = np.array([[3, 7], [0, 9], [5, 5]])
    k2, v2 = copy_blocks(kp, vp, pairs)
    for src, dst in pairs:
        assert np.array_equal(k2[dst], kp[src]) and np.array_equal(v2[dst], vp[src])
    for b in set(range(10)) - {7, 9}:
        assert np.array_equal(k2[b], kp[b]) and np.array_equal(v2[b], vp[b])


# ---------------------------------------------------------------------------
# workload structure (the configs' bookkeeping)
# ---------------------------------------------------------------------------


def test_tiny_config_structure():
    L = config_tiny()
    assert L.seq_lens.tolist() == [1, 17, 40, 100]
    assert [L.blocks_of(s) for s in range(4)] == [1, 2, 3, 7]
    assert L.num_blocks == 64 and L.unique_blocks_touched() == 13
    assert L.num_new_tokens == 4


def test_shared_prefix_config_refcounts_and_cow_pairs():
    L = config_llama2_70b_shared()
    assert L.num_seqs == 128 and L.copy_pairs.shape == (96, 2)
    npb = 2048 // 16
    for grp in L.share_groups:
        rows = L.block_tables[grp]
        assert (rows[:, : npb - 1] == rows[0, : npb - 1]).all()
        assert (L.refcounts[rows[0, : npb - 1]] == 4).all()
        lasts = rows[:, npb - 1]
        assert len(set(lasts.tolist())) == 4 and (L.refcounts[lasts] == 1).all()
    assert set(L.copy_pairs[:, 1].tolist()).isdisjoint(set(L.copy_pairs[:, 0].tolist()))


def test_llama3_config_lengths():
    L = config_llama3_8b()
    assert L.num_seqs == 256 and L.group == 4
    assert L.seq_lens.min() >= 16 and L.seq_lens.max() <= 8192
    assert 700 < np.median(L.seq_lens) < 1400
    # every slot targets the newest token's row
    B = L.block_size
    for s in range(0, 256, 17):
        t = int(L.seq_lens[s]) - 1
        assert L.slot_mapping[s] == L.block_tables[s, t // B] * B + t % B


# ---------------------------------------------------------------------------
# mutation test: plausible mistakes planted in copies of the oracle fail a pin
# ---------------------------------------------------------------------------


def _mutant_decode_one(kind):
    def f(s, h, q, k_pool, v_pool, block_tables, seq_lens, scale, num_kv_heads, dtype):
        Hq = q.shape[1]
        g = Hq // num_kv_heads
        kvh = (h % num_kv_heads) if kind == "kv_head_modulo" else h // g
        B = k_pool.shape[2]
        n = int(seq_lens[s])
        t = np.arange(n)
        if kind == "swap_block_row":
            blocks, rows = np.asarray(block_tables[s])[np.minimum(t % B, len(block_tables[s]) - 1)], t // B % B
        else:
            blocks, rows = np.asarray(block_tables[s])[t // B], t % B
        K = bits_to_f64(k_pool[blocks, kvh, rows, :], dtype)
        Vp = k_pool if kind == "v_from_k" else v_pool
        Vv = bits_to_f64(Vp[blocks, kvh, rows, :], dtype)
        qv = bits_to_f64(q[s, h], dtype)
        if kind == "no_scale":
            scale = 1.0
        if kind == "per_block_softmax":
            out = np.zeros(qv.shape[0])
            for j in range(0, n, B):
                z = scale * (K[j : j + B] @ qv)
                w = np.exp(z - z.max())
                out += (w / w.sum()) @ Vv[j : j + B]
            return out
        return attention_dense(qv, K, Vv, scale)

    return f


@pytest.mark.parametrize("kind", ["no_scale", "per_block_softmax", "kv_head_modulo", "swap_block_row",
                                  "v_from_k"])
def test_planted_mistakes_are_caught_by_bruteforce_pin(kind):
    rng = np.random.default_rng(21)
    dtype, B, D, Hq, Hkv = "bf16", 4, 8, 4, 2
    lens = [3, 9, 14]
    seqs_k = [f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype) for n in lens]
    seqs_v = [f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype) for n in lens]
    q = f32_to_bits(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), dtype)
    kp, vp, tables = _scatter_contiguous(rng, seqs_k, seqs_v, B, 20, dtype)
    f = _mutant_decode_one(kind)
    worst = 0.0
    for s, n in enumerate(lens):
        for h in range(Hq):
            got = f(s, h, q, kp, vp, tables, np.array(lens), 0.5, Hkv, dtype)
            kvh = h // (Hq // Hkv)
            ref = _brute_attention(bits_to_f64(q[s, h], dtype).tolist(),
                                   bits_to_f64(seqs_k[s][:, kvh], dtype).tolist(),
                                   bits_to_f64(seqs_v[s][:, kvh], dtype).tolist(), 0.5)
            err = np.abs(np.asarray(got) - np.asarray(ref))
            worst = max(worst, float(np.nanmax(err)) if np.isfinite(err).any() else math.inf)
            if not np.isfinite(err).all():
                worst = math.inf
    assert worst > 1e-6, f"mutant {kind} slipped through the brute-force pin"


def test_oracle_module_exports():
    for name in ["decode", "decode_one", "cache_write", "copy_blocks", "BlockManager"]:
        assert hasattr(oracle, name)
