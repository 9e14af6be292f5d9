"""Float64 reference of the paged decode step (test infrastructure only).

Written from the pages, slow and literal:

* decode = softmax(q K^T * scale) V over the gathered sequence
  (vLLM blog §"关键细节" 2) "PagedAttention 算子": Attn(Q,K,V) = softmax(QK^T/sqrt(d))V,
  K/V reached block by block through block_table).
* the blockwise form with a running max and running sum merged block by block
  (PagedAttention study notes ch.05 §4: S_ij = Q_i K_j^T, O_i = sum_j P_ij V_j,
  normalisation across blocks via online softmax).
* the partition-then-merge form used for long sequences: each partition keeps
  (max, sum, unnormalised output) and the merge rescales them to a common max
  — the same online-softmax merge rule as ch.05 §4, applied to partitions.
* cache write (vLLM blog, plain-language section: each generated token's
  K/V is written down for later steps) and
  block copy for copy-on-write (study notes ch.05 §6.1, §12 exercise 4).

Readings where the pages are silent (each listed in the design notes):
q head h uses kv head h // (Hq / Hkv) (contiguous GQA groups); token t of a
sequence is row t % B of block block_tables[s, t // B]; seq_len 0 gives a zero
output; the output is returned in float64 (rounding to the 16-bit output type
is the kernel's business and is covered by the comparison tolerance).
"""

from __future__ import annotations

import numpy as np


def bits_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact upcast of raw fp16/bf16 bit patterns (uint16) to float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def gather_kv(pool: np.ndarray, table_row: np.ndarray, n: int, kv_head: int, block_size: int) -> np.ndarray:
    """Rows of tokens 0..n-1 of one sequence for one kv head, reached through
    the block table: token t lives in row t % B of block table_row[t // B]
    (study notes ch.05 §3 and §9.2; vLLM blog §"关键细节" 2)).  pool is [NB, Hkv, B, D]."""
    t = np.arange(n)
    blocks = np.asarray(table_row, dtype=np.int64)[t // block_size]
    rows = t % block_size
    return pool[blocks, kv_head, rows, :]


def attention_dense(q_vec: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q) V for one query vector over contiguous K, V [n, D]
    (vLLM blog §"关键细节" 2)).  n == 0 gives zeros."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    z = scale * (K @ q_vec)
    z = z - z.max()
    w = np.exp(z)
    return (w / w.sum()) @ V


def decode_one(s: int, h: int, q, k_pool, v_pool, block_tables, seq_lens, scale: float,
               num_kv_heads: int, dtype: str) -> np.ndarray:
    """Output row out[s, h, :] of the decode step, in float64.  q, pools are
    uint16 bit arrays; the kv head of q head h is h // (Hq / Hkv)."""
    Hq = q.shape[1]
    g = Hq // num_kv_heads
    kvh = h // g
    B = k_pool.shape[2]
    n = int(seq_lens[s])
    K = bits_to_f64(gather_kv(k_pool, block_tables[s], n, kvh, B), dtype)
    V = bits_to_f64(gather_kv(v_pool, block_tables[s], n, kvh, B), dtype)
    return attention_dense(bits_to_f64(q[s, h], dtype), K, V, scale)


def decode(q, k_pool, v_pool, block_tables, seq_lens, scale: float, num_kv_heads: int, dtype: str) -> np.ndarray:
    """Full decode step: out [S, Hq, D] float64, one decode_one per (s, h)."""
    S, Hq, D = q.shape
    out = np.zeros((S, Hq, D), dtype=np.float64)
    for s in range(S):
        for h in range(Hq):
            out[s, h] = decode_one(s, h, q, k_pool, v_pool, block_tables, seq_lens, scale, num_kv_heads, dtype)
    return out


def decode_multi(q, k_pool, v_pool, block_tables, seq_lens, scale: float, num_kv_heads: int,
                 dtype: str) -> np.ndarray:
    """Attention of q_len new query positions per sequence over the paged
    cache, causal among them (the speculative-decoding and chunked-prefill
    items of the CSDN article's "2026年最新进展" list; the attention itself is
    the vLLM blog's §"关键细节" 2 definition).  q is [S, q_len, Hq, D] bits;
    seq_lens counts every cached token including the q_len new ones, so
    position i sees tokens 0 .. seq_lens[s] - q_len + i.  Computed as one
    masked score matrix per (sequence, head): Z = scale * Q K^T, entries past a
    row's limit removed, softmax along each row, times V.  A sequence with
    fewer than q_len tokens gives zeros.  Returns [S, q_len, Hq, D] float64."""
    S, L, Hq, D = q.shape
    g = Hq // num_kv_heads
    B = k_pool.shape[2]
    out = np.zeros((S, L, Hq, D), dtype=np.float64)
    for s in range(S):
        n = int(seq_lens[s])
        if n < L:
            continue
        limit = n - L + np.arange(L)                        # last visible token of each row
        visible = np.arange(n)[None, :] <= limit[:, None]   # [L, n]
        for h in range(Hq):
            K = bits_to_f64(gather_kv(k_pool, block_tables[s], n, h // g, B), dtype)
            V = bits_to_f64(gather_kv(v_pool, block_tables[s], n, h // g, B), dtype)
            Z = scale * (bits_to_f64(q[s, :, h], dtype) @ K.T)  # [L, n]
            Z = np.where(visible, Z, -np.inf)
            Z = Z - Z.max(axis=1, keepdims=True)
            W = np.exp(Z)
            out[s, :, h] = (W / W.sum(axis=1, keepdims=True)) @ V
    return out


def decode_blockwise_online(s: int, h: int, q, k_pool, v_pool, block_tables, seq_lens, scale: float,
                            num_kv_heads: int, dtype: str) -> np.ndarray:
    """The same output computed the way the study notes ch.05 §4 describe it:
    walk the logical blocks j = 0, 1, ..., take S_j = q K_j^T * scale for the
    block's valid rows, keep a running max m and running sum l, rescale the
    running output by exp(m_old - m_new) and add exp(S_j - m_new) V_j."""
    Hq = q.shape[1]
    kvh = h // (Hq // num_kv_heads)
    B = k_pool.shape[2]
    n = int(seq_lens[s])
    qv = bits_to_f64(q[s, h], dtype)
    D = qv.shape[0]
    m, l, acc = -np.inf, 0.0, np.zeros(D, dtype=np.float64)
    nblocks = (n + B - 1) // B
    for j in range(nblocks):
        valid = min(B, n - j * B)
        phys = int(block_tables[s, j])
        Kj = bits_to_f64(k_pool[phys, kvh, :valid, :], dtype)
        Vj = bits_to_f64(v_pool[phys, kvh, :valid, :], dtype)
        Sj = scale * (Kj @ qv)
        m_new = max(m, float(Sj.max()))
        alpha = np.exp(m - m_new)
        p = np.exp(Sj - m_new)
        l = l * alpha + p.sum()
        acc = acc * alpha + p @ Vj
        m = m_new
    if nblocks == 0:
        return acc
    return acc / l


def partition_states(s: int, h: int, q, k_pool, v_pool, block_tables, seq_lens, scale: float,
                     num_kv_heads: int, dtype: str, bounds):
    """Per-partition softmax state for a sequence split at token positions
    ``bounds`` (ascending, 0 < b < n): for each token range [a, b) return
    (m, l, acc) with m = max score, l = sum exp(score - m),
    acc = sum exp(score - m) v (unnormalised)."""
    Hq = q.shape[1]
    kvh = h // (Hq // num_kv_heads)
    B = k_pool.shape[2]
    n = int(seq_lens[s])
    K = bits_to_f64(gather_kv(k_pool, block_tables[s], n, kvh, B), dtype)
    V = bits_to_f64(gather_kv(v_pool, block_tables[s], n, kvh, B), dtype)
    z = scale * (K @ bits_to_f64(q[s, h], dtype))
    edges = [0] + list(bounds) + [n]
    states = []
    for a, b in zip(edges[:-1], edges[1:]):
        m = float(z[a:b].max())
        w = np.exp(z[a:b] - m)
        states.append((m, float(w.sum()), w @ V[a:b]))
    return states


def merge_partition_states(states) -> np.ndarray:
    """Combine partition states: M = max m_p, out = sum e^(m_p-M) acc_p /
    sum e^(m_p-M) l_p (online-softmax merge, study notes ch.05 §4)."""
    M = max(m for m, _, _ in states)
    num = sum(np.exp(m - M) * acc for m, _, acc in states)
    den = sum(np.exp(m - M) * l for m, l, _ in states)
    return num / den


def decode_lse(q, k_pool, v_pool, block_tables, seq_lens, scale: float, num_kv_heads: int, dtype: str):
    """The decode step's outputs [S, Hq, D] together with, per (s, h), the
    natural log of the softmax normaliser over the sequence's tokens,
    lse = log sum_t exp(scale * q . K_t) [S, Hq] (-inf for no token): the
    quantity that lets decodes of disjoint token ranges be merged afterwards
    (study notes ch.05 §4, the online-softmax merge).  Written out per row
    with the shift by the row's maximum, as the softmax itself."""
    S, Hq, D = q.shape
    g = Hq // num_kv_heads
    B = k_pool.shape[2]
    out = np.zeros((S, Hq, D), dtype=np.float64)
    lse = np.full((S, Hq), -np.inf, dtype=np.float64)
    for s in range(S):
        n = int(seq_lens[s])
        for h in range(Hq):
            out[s, h] = decode_one(s, h, q, k_pool, v_pool, block_tables, seq_lens, scale, num_kv_heads, dtype)
            if n == 0:
                continue
            K = bits_to_f64(gather_kv(k_pool, block_tables[s], n, h // g, B), dtype)
            z = scale * (K @ bits_to_f64(q[s, h], dtype))
            m = z.max()
            lse[s, h] = m + np.log(np.exp(z - m).sum())
    return out, lse


def merge_outputs(outs, lses):
    """Merge decodes of disjoint token ranges of the same rows (study notes
    ch.05 §4: partial results rescaled to a common maximum).  outs
    [R, ..., D] and lses [R, ...] per range; with M = max_r lse_r and
    w_r = e^(lse_r - M): out = sum_r w_r out_r / sum_r w_r and
    lse = M + log sum_r w_r.  A row no range saw (every lse_r = -inf) gets a
    zero output and -inf.  Returns (out, lse) in float64."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    M = lses.max(axis=0)
    seen = np.isfinite(M)
    Ms = np.where(seen, M, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - Ms), 0.0)  # [R, ...]
    wsum = w.sum(axis=0)
    out = np.zeros(outs.shape[1:], dtype=np.float64)
    out[seen] = (np.einsum("r...,r...d->...d", w, outs))[seen] / wsum[seen][..., None]
    lse = np.where(seen, Ms + np.log(np.where(seen, wsum, 1.0)), -np.inf)
    return out, lse


def cache_write(k_pool: np.ndarray, v_pool: np.ndarray, new_k: np.ndarray, new_v: np.ndarray,
                slot_mapping: np.ndarray):
    """Store each new token's K/V rows in its slot (vLLM blog, plain-language section: each
    generated token's K/V is written to the cache).  slot = block * B + row;
    a negative slot skips the token.  Returns new pool arrays (bit copies)."""
    k_out, v_out = k_pool.copy(), v_pool.copy()
    B = k_pool.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        b, r = int(slot) // B, int(slot) % B
        k_out[b, :, r, :] = new_k[t]
        v_out[b, :, r, :] = new_v[t]
    return k_out, v_out


def copy_blocks(k_pool: np.ndarray, v_pool: np.ndarray, pairs: np.ndarray):
    """Copy-on-write block copies (study notes ch.05 §6.1, §12 exercise 4):
    for each (src, dst) in order, block dst of both pools becomes a bit copy
    of block src.  Returns new pool arrays."""
    k_out, v_out = k_pool.copy(), v_pool.copy()
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        k_out[int(dst)] = k_out[int(src)]
        v_out[int(dst)] = v_out[int(src)]
    return k_out, v_out
