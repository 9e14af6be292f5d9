"""Pins of the oracle's multi-query attention (q_len causal positions per
sequence) against things other than itself: pure-Python brute force over
contiguous rows, the decode oracle on truncated sequences, the q_len = 1
case, causality invariants, and planted mistakes that one of these pins must
catch."""

import math

import numpy as np
import pytest

from oracle import bits_to_f64, decode, decode_multi
from test_oracle import _brute_attention, _scatter_contiguous
from workloads import f32_to_bits


def _case(seed, lens, Hq, Hkv, L, dtype="bf16", B=4, D=8):
    rng = np.random.default_rng(seed)
    seqs_k = [f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype) for n in lens]
    seqs_v = [f32_to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype) for n in lens]
    q = f32_to_bits(rng.standard_normal((len(lens), L, Hq, D), dtype=np.float32), dtype)
    NB = sum((n + B - 1) // B for n in lens) + 5
    kp, vp, tables = _scatter_contiguous(rng, [k if k.shape[0] else k.reshape(0, Hkv, D) for k in seqs_k],
                                         seqs_v, B, NB, dtype)
    return q, kp, vp, tables, np.array(lens, np.int32), seqs_k, seqs_v


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv,L", [(2, 2, 3), (4, 1, 2), (4, 2, 5)])
def test_multi_matches_bruteforce(dtype, Hq, Hkv, L):
    lens = [L, L + 1, 7, 13, 16]
    q, kp, vp, tables, sl, seqs_k, seqs_v = _case(31, lens, Hq, Hkv, L, dtype)
    out = decode_multi(q, kp, vp, tables, sl, 0.41, Hkv, dtype)
    g = Hq // Hkv
    for s, n in enumerate(lens):
        for i in range(L):
            last = n - L + i  # the last token position i may see
            for h in range(Hq):
                kvh = h // g
                ref = _brute_attention(bits_to_f64(q[s, i, h], dtype).tolist(),
                                       bits_to_f64(seqs_k[s][: last + 1, kvh], dtype).tolist(),
                                       bits_to_f64(seqs_v[s][: last + 1, kvh], dtype).tolist(), 0.41)
                np.testing.assert_allclose(out[s, i, h], ref, rtol=0, atol=1e-12)


def test_single_position_is_decode():
    lens = [1, 5, 9, 20]
    q, kp, vp, tables, sl, _, _ = _case(32, lens, 4, 2, 1)
    got = decode_multi(q, kp, vp, tables, sl, 0.3, 2, "bf16")
    ref = decode(q[:, 0], kp, vp, tables, sl, 0.3, 2, "bf16")
    np.testing.assert_allclose(got[:, 0], ref, rtol=0, atol=1e-13)


def test_each_position_is_decode_of_the_truncated_sequence():
    L = 4
    lens = [4, 6, 11, 17]
    q, kp, vp, tables, sl, _, _ = _case(33, lens, 4, 2, L)
    got = decode_multi(q, kp, vp, tables, sl, 0.5, 2, "bf16")
    for i in range(L):
        trunc = sl - L + i + 1
        ref = decode(np.ascontiguousarray(q[:, i]), kp, vp, tables, trunc, 0.5, 2, "bf16")
        np.testing.assert_allclose(got[:, i], ref, rtol=0, atol=1e-13)


def test_tokens_past_a_position_do_not_reach_it():
    L, B = 3, 4
    lens = [10]
    q, kp, vp, tables, sl, _, _ = _case(34, lens, 2, 2, L, B=B)
    base = decode_multi(q, kp, vp, tables, sl, 0.5, 2, "bf16")
    # change the K/V rows of the last token: positions 0 .. L-2 cannot see it
    t = lens[0] - 1
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[tables[0, t // B], :, t % B, :] ^= np.uint16(0x0100)
    vp2[tables[0, t // B], :, t % B, :] ^= np.uint16(0x0100)
    moved = decode_multi(q, kp2, vp2, tables, sl, 0.5, 2, "bf16")
    np.testing.assert_array_equal(moved[:, : L - 1], base[:, : L - 1])
    assert np.abs(moved[:, L - 1] - base[:, L - 1]).max() > 1e-6


def test_short_sequences_give_zeros():
    L = 3
    lens = [0, 2, 3]
    q, kp, vp, tables, sl, _, _ = _case(35, lens, 2, 2, L)
    out = decode_multi(q, kp, vp, tables, sl, 0.5, 2, "bf16")
    assert not out[:2].any()
    assert np.abs(out[2]).max() > 0


def _mutant_multi(kind):
    """decode_multi with one plausible mistake planted (on the CPU only)."""

    def f(q, k_pool, v_pool, block_tables, seq_lens, scale, num_kv_heads, dtype):
        S, L, Hq, D = q.shape
        g = Hq // num_kv_heads
        B = k_pool.shape[2]
        out = np.zeros((S, L, Hq, D))
        for s in range(S):
            n = int(seq_lens[s])
            if n < L:
                continue
            limit = n - L + np.arange(L)
            if kind == "mask_off_by_one":
                limit = limit - 1
            if kind == "mask_reversed_rows":
                limit = limit[::-1]
            if kind == "mask_from_start":
                limit = np.arange(L)
            t = np.arange(n)
            vis = t[None, :] <= limit[:, None]
            if kind == "no_mask":
                vis = np.ones_like(vis)
            for h in range(Hq):
                blocks, rows = np.asarray(block_tables[s])[t // B], t % B
                K = bits_to_f64(k_pool[blocks, h // g, rows, :], dtype)
                V = bits_to_f64(v_pool[blocks, h // g, rows, :], dtype)
                Z = scale * (bits_to_f64(q[s, :, h], dtype) @ K.T)
                Z = np.where(vis, Z, -np.inf)
                W = np.exp(Z - Z.max(axis=1, keepdims=True))
                out[s, :, h] = (W / W.sum(axis=1, keepdims=True)) @ V
        return out

    return f


@pytest.mark.parametrize("kind", ["mask_off_by_one", "mask_reversed_rows", "mask_from_start", "no_mask"])
def test_planted_mask_mistakes_are_caught_by_bruteforce_pin(kind):
    L = 3
    lens = [3, 9, 14]
    q, kp, vp, tables, sl, seqs_k, seqs_v = _case(36, lens, 4, 2, L)
    got = _mutant_multi(kind)(q, kp, vp, tables, sl, 0.5, 2, "bf16")
    worst = 0.0
    for s, n in enumerate(lens):
        for i in range(L):
            for h in range(4):
                kvh = h // 2
                last = n - L + i
                ref = _brute_attention(bits_to_f64(q[s, i, h], "bf16").tolist(),
                                       bits_to_f64(seqs_k[s][: last + 1, kvh], "bf16").tolist(),
                                       bits_to_f64(seqs_v[s][: last + 1, kvh], "bf16").tolist(), 0.5)
                err = np.abs(got[s, i, h] - np.asarray(ref))
                worst = max(worst, float(err.max()) if np.isfinite(err).all() else math.inf)
    assert worst > 1e-6, f"mutant {kind} slipped through the brute-force pin"
