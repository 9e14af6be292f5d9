"""Pins of the oracle's log normaliser (decode_lse) and of its merge of
decodes over disjoint token ranges (merge_outputs), the online-softmax
merge of study notes ch.05 §4 applied to ranges of a sequence:

* closed forms: one token gives lse = scale * q . k exactly; n equal scores
  give lse = score + log n and the plain mean of the V rows;
* brute force: lse against Python's math.fsum of exp over explicit dot
  products, on small random paged layouts;
* the merge invariant: a sequence cut at block boundaries into ranges,
  each range decoded on its own and merged, equals the whole decode and its
  lse (any cut, any number of ranges, empty ranges included);
* planted mistakes in copies of the two functions (log2 for log, a plain
  mean for the weighted merge, the maximum's shift left out), each of which
  must fail one of these pins.
"""

import math

import numpy as np
import pytest

import oracle
from oracle.paged_attention import bits_to_f64
from workloads import f32_to_bits, fill_values_numpy, random_layout


def _one_token_layout(qv, kv, vv, dtype="bf16"):
    """A pool of one block holding one token; q, k, v given as float lists."""
    D = len(qv)
    q = f32_to_bits(np.asarray(qv, np.float32).reshape(1, 1, D), dtype)
    kp = f32_to_bits(np.asarray(kv, np.float32).reshape(1, 1, 1, D), dtype)
    vp = f32_to_bits(np.asarray(vv, np.float32).reshape(1, 1, 1, D), dtype)
    return q, kp, vp, np.zeros((1, 1), np.int32), np.ones(1, np.int32)


def test_one_token_lse_is_the_scaled_score():
    # values exact in bf16: the score is a short exact sum
    qv, kv, vv = [1.0, 2.0, -0.5, 0.25], [3.0, 0.5, 4.0, 8.0], [1.0, -1.0, 2.0, 0.5]
    q, kp, vp, tables, lens = _one_token_layout(qv, kv, vv)
    out, lse = oracle.decode_lse(q, kp, vp, tables, lens, 0.125, 1, "bf16")
    assert lse[0, 0] == 0.125 * (3 + 1 - 2 + 2) == 0.5
    assert np.array_equal(out[0, 0], np.asarray(vv, np.float64))


def test_equal_scores_give_log_n_and_the_mean():
    # k rows all zero: every score is 0, so lse = log n and out = mean of the V rows
    D, B, n = 8, 4, 7
    rng = np.random.default_rng(3)
    q = f32_to_bits(rng.standard_normal((1, 1, D)).astype(np.float32), "bf16")
    kp = f32_to_bits(np.zeros((2, 1, B, D), np.float32), "bf16")
    vvals = rng.integers(-4, 5, size=(2, 1, B, D)).astype(np.float32)
    vp = f32_to_bits(vvals, "bf16")
    tables = np.array([[1, 0]], np.int32)
    out, lse = oracle.decode_lse(q, kp, vp, tables, np.array([n], np.int32), 0.3, 1, "bf16")
    assert abs(lse[0, 0] - math.log(n)) < 1e-15
    rows = [vvals[tables[0, t // B], 0, t % B] for t in range(n)]
    assert np.allclose(out[0, 0], np.mean(np.asarray(rows, np.float64), axis=0), rtol=0, atol=1e-15)


def _bruteforce_lse(L, V):
    q = bits_to_f64(V.q, L.dtype)
    kp = bits_to_f64(V.k_pool, L.dtype)
    g = L.num_q_heads // L.num_kv_heads
    B = L.block_size
    want = np.full((L.num_seqs, L.num_q_heads), -np.inf)
    for s in range(L.num_seqs):
        for h in range(L.num_q_heads):
            terms = []
            for t in range(int(L.seq_lens[s])):
                krow = kp[L.block_tables[s, t // B], h // g, t % B]
                terms.append(math.exp(L.scale * math.fsum(float(a) * float(b) for a, b in zip(q[s, h], krow))))
            if terms:
                want[s, h] = math.log(math.fsum(terms))
    return want


def _small_layout(seed=5, lens=(1, 3, 16, 17, 40, 0)):
    L = random_layout(seed, list(lens), dtype="bf16", block_size=8, num_q_heads=4, num_kv_heads=2, head_dim=16,
                      write_new_token=False)
    return L, fill_values_numpy(L)


def test_lse_matches_bruteforce():
    L, V = _small_layout()
    _, lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads,
                               L.dtype)
    want = _bruteforce_lse(L, V)
    assert np.array_equal(np.isinf(lse), np.isinf(want))
    fin = np.isfinite(want)
    assert np.abs(lse[fin] - want[fin]).max() < 1e-12


def _ranges_decode(L, V, cuts, decode_lse=oracle.decode_lse):
    """Decode each sequence's token ranges [cuts[i], cuts[i+1]) (block
    multiples) on their own: returns outs [R, S, Hq, D], lses [R, S, Hq]."""
    B = L.block_size
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        lens = np.clip(L.seq_lens - a, 0, b - a).astype(np.int32)
        tables = np.zeros_like(L.block_tables)
        w = L.block_tables.shape[1] - a // B
        tables[:, :w] = L.block_tables[:, a // B:]
        o, l = decode_lse(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, L.num_kv_heads, L.dtype)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("cuts", [[0, 8, 1000], [0, 16, 24, 1000], [0, 8, 16, 24, 32, 1000], [0, 1000, 2000]])
def test_merged_ranges_equal_the_whole_decode(cuts):
    L, V = _small_layout()
    full, full_lse = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                       L.num_kv_heads, L.dtype)
    outs, lses = _ranges_decode(L, V, cuts)
    out, lse = oracle.merge_outputs(outs, lses)
    assert np.abs(out - full).max() < 1e-12
    assert np.array_equal(np.isinf(lse), np.isinf(full_lse))
    fin = np.isfinite(full_lse)
    assert np.abs(lse[fin] - full_lse[fin]).max() < 1e-12
    assert np.array_equal(out[L.seq_lens == 0], np.zeros_like(out[L.seq_lens == 0]))


def test_merge_of_one_part_is_that_part():
    L, V = _small_layout()
    o, l = oracle.decode_lse(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
    out, lse = oracle.merge_outputs(o[None], l[None])
    assert np.array_equal(out, o) and np.array_equal(lse, l)


# planted mistakes, each in a copy of the oracle function, must fail a pin

def _mutant_decode_lse(kind):
    def f(q, k_pool, v_pool, block_tables, seq_lens, scale, num_kv_heads, dtype):
        out, lse = oracle.decode_lse(q, k_pool, v_pool, block_tables, seq_lens, scale, num_kv_heads, dtype)
        S, Hq, _ = q.shape
        g = Hq // num_kv_heads
        B = k_pool.shape[2]
        for s in range(S):
            n = int(seq_lens[s])
            for h in range(Hq):
                if n == 0:
                    continue
                K = bits_to_f64(oracle.gather_kv(k_pool, block_tables[s], n, h // g, B), dtype)
                z = scale * (K @ bits_to_f64(q[s, h], dtype))
                m = z.max()
                if kind == "log2":
                    lse[s, h] = m + np.log2(np.exp(z - m).sum())
                elif kind == "no_shift":
                    lse[s, h] = np.log(np.exp(z - m).sum())
        return out, lse
    return f


def _mutant_merge(kind):
    def f(outs, lses):
        outs, lses = np.asarray(outs, np.float64), np.asarray(lses, np.float64)
        if kind == "plain_mean":
            return outs.mean(axis=0), lses.max(axis=0)
        if kind == "max_only":  # the largest part's output, no weighting
            idx = lses.argmax(axis=0)
            return np.take_along_axis(outs, idx[None, ..., None], 0)[0], lses.max(axis=0)
        raise ValueError(kind)
    return f


@pytest.mark.parametrize("kind", ["log2", "no_shift"])
def test_planted_lse_mistakes_are_caught(kind):
    L, V = _small_layout()
    _, lse = _mutant_decode_lse(kind)(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale,
                                      L.num_kv_heads, L.dtype)
    want = _bruteforce_lse(L, V)
    fin = np.isfinite(want)
    assert np.abs(lse[fin] - want[fin]).max() > 1e-6


@pytest.mark.parametrize("kind", ["plain_mean", "max_only"])
def test_planted_merge_mistakes_are_caught(kind):
    L, V = _small_layout()
    full = oracle.decode(V.q, V.k_pool, V.v_pool, L.block_tables, L.seq_lens, L.scale, L.num_kv_heads, L.dtype)
    outs, lses = _ranges_decode(L, V, [0, 8, 16, 1000])
    out, _ = _mutant_merge(kind)(outs, lses)
    assert np.abs(out - full).max() > 1e-6
