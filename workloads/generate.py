"""Seeded generators for paged-KV decode workloads.

Conventions (the same on both sides of every comparison):

* A sequence of ``n`` tokens keeps token ``t`` in row ``t % B`` of the physical
  block ``block_tables[s, t // B]`` (block table indirection, PagedAttention
  notes ch.05 §3 and §9.2; vLLM blog §"关键细节" 2) "PagedAttention 算子").
* ``seq_lens[s]`` counts every token the decode step attends, the newest one
  included.  When a layout writes new tokens, token ``seq_lens[s] - 1`` of each
  sequence is the one written this step (the last ``q_len`` tokens for a
  multi-query layout): its row is NaN in the pool until the cache write
  stores it.
* Pool layout is ``[num_blocks, num_kv_heads, block_size, head_dim]``.  Rows
  that hold no token and blocks that no table references are NaN, so a kernel
  that reads past ``seq_lens`` or multiplies a masked V row by zero shows up.
* Values are N(0, 1) float32 draws rounded once to fp16/bf16; the arrays hold
  the raw 16-bit patterns (uint16) so the same bits reach the GPU and the CPU.

Nothing here computes attention.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Dict, List, Optional

import numpy as np

DTYPES = ("fp16", "bf16")
NAN_BITS = {"fp16": 0x7E00, "bf16": 0x7FC0}
PAD_ENTRY = -1


def f32_to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to fp16/bf16 (nearest-even) and return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        u = x.view(np.uint32).astype(np.uint64)
        lsb = (u >> np.uint64(16)) & np.uint64(1)
        return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    raise ValueError(f"unknown dtype {dtype!r}")


def bits_to_torch(bits: np.ndarray, dtype: str):
    """View a uint16 bit array as a torch fp16/bf16 CPU tensor (no rounding)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "fp16" else torch.bfloat16)


@dataclass
class PagedLayout:
    """Structure of one decode step over a paged KV pool (no values)."""

    name: str
    seed: int
    dtype: str
    block_size: int
    num_blocks: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    scale: float
    seq_lens: np.ndarray  # int32 [S]
    block_tables: np.ndarray  # int32 [S, max_blocks_per_seq], PAD_ENTRY past the last block
    slot_mapping: np.ndarray  # int64 [T]; slot = phys_block * B + row; negative = skip
    copy_pairs: np.ndarray  # int64 [n, 2] (src, dst) copy-on-write pairs, applied before the write
    block_fill: np.ndarray  # int32 [num_blocks]: leading rows holding a token before this step
    refcounts: Optional[np.ndarray] = None  # int32 [num_blocks] after the step (shared-prefix layouts)
    share_groups: List[List[int]] = field(default_factory=list)  # sequences sharing a prompt
    note: str = ""
    q_len: int = 1  # query positions per sequence; q is [S, Hq, D] if 1 else [S, q_len, Hq, D]

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def num_new_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])

    def blocks_of(self, s: int) -> int:
        n = int(self.seq_lens[s])
        return (n + self.block_size - 1) // self.block_size

    def total_blocks_touched(self) -> int:
        """Per-sequence count of (block) entries one decode reads, summed over sequences."""
        B = self.block_size
        return int(((self.seq_lens.astype(np.int64) + B - 1) // B).sum())

    def unique_blocks_touched(self) -> int:
        ids = [self.block_tables[s, : self.blocks_of(s)] for s in range(self.num_seqs)]
        return int(np.unique(np.concatenate(ids)).size) if ids else 0


@dataclass
class PagedValues:
    """16-bit bit patterns (uint16 numpy) or torch tensors for one layout."""

    q: object  # [S, Hq, D], or [S, q_len, Hq, D] for a multi-query layout
    k_pool: object  # [NB, Hkv, B, D]
    v_pool: object
    new_k: object  # [T, Hkv, D]
    new_v: object


# --------------------------------------------------------------------------
# structure builders
# --------------------------------------------------------------------------


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _finish_layout(
    name, seed, dtype, B, NB, Hq, Hkv, D, seq_lens, tables, write_new_token, copy_pairs=None,
    refcounts=None, share_groups=None, note="", scale=None, q_len=1,
) -> PagedLayout:
    """With write_new_token, the last q_len tokens of every sequence are the
    ones this step writes (their rows are unfilled before the step)."""
    S = seq_lens.shape[0]
    copy_pairs = np.zeros((0, 2), np.int64) if copy_pairs is None else np.asarray(copy_pairs, np.int64)
    fill = np.zeros(NB, np.int32)
    slots = []
    for s in range(S):
        n = int(seq_lens[s])
        before = max(n - q_len, 0) if write_new_token else n
        for j in range(_ceil_div(n, B)):
            b = int(tables[s, j])
            rows = min(B, max(0, before - j * B))
            fill[b] = max(fill[b], rows)
        if write_new_token:
            for t in range(before, n):
                slots.append(int(tables[s, t // B]) * B + t % B)
    for _, dst in copy_pairs:
        fill[int(dst)] = 0
    return PagedLayout(
        name=name, seed=seed, dtype=dtype, block_size=B, num_blocks=NB, num_q_heads=Hq,
        num_kv_heads=Hkv, head_dim=D, scale=(1.0 / math.sqrt(D)) if scale is None else scale,
        seq_lens=seq_lens.astype(np.int32), block_tables=tables.astype(np.int32),
        slot_mapping=np.asarray(slots, np.int64), copy_pairs=copy_pairs, block_fill=fill,
        refcounts=refcounts, share_groups=share_groups or [], note=note, q_len=q_len,
    )


def _scatter_tables(rng, seq_lens, B, NB, max_nb=None):
    nb = [_ceil_div(int(n), B) for n in seq_lens]
    total = sum(nb)
    assert total <= NB, (total, NB)
    max_nb = max(max(nb) if nb else 1, 1) if max_nb is None else max_nb
    tables = np.full((len(seq_lens), max_nb), PAD_ENTRY, np.int32)
    perm = rng.permutation(NB).astype(np.int32)
    off = 0
    for s, k in enumerate(nb):
        tables[s, :k] = perm[off : off + k]
        off += k
    return tables


def random_layout(
    seed: int,
    seq_lens,
    *,
    dtype: str = "bf16",
    block_size: int = 16,
    num_q_heads: int = 4,
    num_kv_heads: int = 4,
    head_dim: int = 64,
    pool_factor: float = 1.5,
    extra_blocks: int = 3,
    max_blocks_per_seq: Optional[int] = None,
    write_new_token: bool = True,
    scale: Optional[float] = None,
    name: str = "random",
    q_len: int = 1,
) -> PagedLayout:
    """A layout with the given decode lengths scattered over a shuffled pool
    (with q_len > 1: q_len query positions per sequence, and the last q_len
    tokens of each sequence written this step when write_new_token)."""
    rng = np.random.default_rng(seed)
    seq_lens = np.asarray(seq_lens, np.int32)
    B = block_size
    total = sum(_ceil_div(int(n), B) for n in seq_lens)
    NB = max(int(math.ceil(total * pool_factor)) + extra_blocks, 1)
    tables = _scatter_tables(rng, seq_lens, B, NB, max_blocks_per_seq)
    return _finish_layout(
        name, seed, dtype, B, NB, num_q_heads, num_kv_heads, head_dim, seq_lens, tables,
        write_new_token and seq_lens.size > 0 and int(seq_lens.min()) >= q_len, scale=scale, q_len=q_len,
    )


def config_tiny() -> PagedLayout:
    """Tiny paged decode: 4 sequences {1, 17, 40, 100}, 4/4 heads, D=64, B=16,
    a 64-block pool placed by a seeded permutation, fp16, scale 1/8, and the
    newest token of each sequence written by the cache write (4 tokens)."""
    seed = 1001
    rng = np.random.default_rng(seed)
    seq_lens = np.array([1, 17, 40, 100], np.int32)
    tables = _scatter_tables(rng, seq_lens, 16, 64)
    return _finish_layout("tiny", seed, "fp16", 16, 64, 4, 4, 64, seq_lens, tables, True,
                          scale=1.0 / 8.0, note="4 seqs {1,17,40,100}, 4/4 heads, D=64, B=16, fp16")


def config_llama7b(batch: int = 64) -> PagedLayout:
    """LLaMA-7B-shaped layer: 32/32 heads (MHA), D=128, bf16, B=16, 64
    sequences with lengths uniform in [128, 2048], shuffled pool of 1.1x the
    blocks needed."""
    seed = 1002
    rng = np.random.default_rng(seed)
    seq_lens = rng.integers(128, 2048 + 1, size=batch).astype(np.int32)
    total = sum(_ceil_div(int(n), 16) for n in seq_lens)
    NB = int(math.ceil(1.1 * total))
    tables = _scatter_tables(rng, seq_lens, 16, NB)
    return _finish_layout("llama7b", seed, "bf16", 16, NB, 32, 32, 128, seq_lens, tables, False,
                          note=f"{batch} seqs U[128,2048], 32/32 heads, D=128, B=16, bf16")


def config_llama3_8b(batch: int = 256, q_len: int = 1) -> PagedLayout:
    """Llama-3-8B-shaped GQA layer: 32 q heads / 8 kv heads, D=128, bf16, B=16,
    256 sequences with lognormal lengths (median 1024, sigma 0.75, clipped to
    [16, 8192]), shuffled pool of 1.1x, and the cache write of 256 new tokens.
    With q_len > 1 (speculative verification of q_len tokens): the same
    lengths, the last q_len tokens of each sequence written this step and
    attended by q_len causal query positions."""
    seed = 1003
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(batch)
    seq_lens = np.clip(np.rint(1024.0 * np.exp(0.75 * z)), 16, 8192).astype(np.int32)
    total = sum(_ceil_div(int(n), 16) for n in seq_lens)
    NB = int(math.ceil(1.1 * total))
    tables = _scatter_tables(rng, seq_lens, 16, NB)
    name = "llama3_8b" if q_len == 1 else f"llama3_8b_spec{q_len}"
    what = "cache write" if q_len == 1 else f"cache write, {q_len} causal query positions per sequence"
    return _finish_layout(name, seed, "bf16", 16, NB, 32, 8, 128, seq_lens, tables, True, q_len=q_len,
                          note=f"{batch} seqs lognormal(median 1024, sigma 0.75) in [16,8192], "
                               f"32/8 heads, D=128, B=16, bf16, {batch * q_len}-token {what}")


def config_llama3_8b_prefill(batch: int = 64, q_len: int = 256) -> PagedLayout:
    """A chunked-prefill step on the Llama-3-8B GQA layer: 64 sequences with
    the lognormal lengths of the decode workload (median 1024, sigma 0.75,
    clipped to [q_len, 8192]), each writing its newest q_len tokens (one
    prefill chunk) and attending them with q_len causal query positions
    over everything cached before them."""
    seed = 1006
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(batch)
    seq_lens = np.clip(np.rint(1024.0 * np.exp(0.75 * z)), q_len, 8192).astype(np.int32)
    total = sum(_ceil_div(int(n), 16) for n in seq_lens)
    NB = int(math.ceil(1.1 * total))
    tables = _scatter_tables(rng, seq_lens, 16, NB)
    return _finish_layout(f"llama3_8b_prefill{q_len}", seed, "bf16", 16, NB, 32, 8, 128, seq_lens, tables, True,
                          q_len=q_len,
                          note=f"{batch} seqs lognormal(median 1024, sigma 0.75) in [{q_len},8192], 32/8 heads, "
                               f"D=128, B=16, bf16, a {q_len}-token prefill chunk per sequence "
                               f"({batch * q_len}-token cache write, {q_len} causal query positions)")


def config_llama2_70b_shared(
    prompt_len: int = 2048, num_prompts: int = 32, samples: int = 4, max_tail: int = 512,
    block_size: int = 16,
) -> PagedLayout:
    """Shared-prefix parallel sampling at the Llama-2-70B layer shape: 64 q /
    8 kv heads, D=128, bf16.  Each prompt's blocks are shared by its samples
    (ref count = samples); samples 1.. copy the last prompt block (copy on
    write) and own their generated tokens, 0..max_tail of them before this
    step plus the one written now.  Sample 0 keeps the original block."""
    seed = 1004
    B = block_size
    if prompt_len % B != 0 and max_tail != 0:
        raise ValueError("a partly filled last prompt block is copied at fork time only (max_tail=0)")
    rng = np.random.default_rng(seed)
    tails = rng.integers(0, max_tail + 1, size=(num_prompts, samples))
    seq_lens = (prompt_len + tails + 1).reshape(-1).astype(np.int32)
    npb = _ceil_div(prompt_len, B)
    nb_seq = [_ceil_div(int(n), B) for n in seq_lens]
    total = num_prompts * npb + num_prompts * (samples - 1) + sum(k - npb for k in nb_seq)
    NB = int(math.ceil(1.1 * total))
    perm = rng.permutation(NB).astype(np.int32)
    cursor = [0]

    def take(k):
        out = perm[cursor[0] : cursor[0] + k]
        cursor[0] += k
        return out

    max_nb = max(nb_seq)
    tables = np.full((num_prompts * samples, max_nb), PAD_ENTRY, np.int32)
    pairs, groups = [], []
    refs = np.zeros(NB, np.int32)
    for p in range(num_prompts):
        prompt_ids = take(npb)
        refs[prompt_ids] += samples
        group = []
        for i in range(samples):
            s = p * samples + i
            group.append(s)
            row = prompt_ids.copy()
            if i >= 1:
                c = int(take(1)[0])
                pairs.append((int(prompt_ids[-1]), c))
                refs[prompt_ids[-1]] -= 1
                refs[c] += 1
                row[-1] = c
            tables[s, :npb] = row
            priv = take(nb_seq[s] - npb)
            tables[s, npb : nb_seq[s]] = priv
            refs[priv] += 1
        groups.append(group)
    return _finish_layout(
        "llama2_70b_shared", seed, "bf16", B, NB, 64, 8, 128, seq_lens, tables, True,
        copy_pairs=np.asarray(pairs, np.int64), refcounts=refs, share_groups=groups,
        note=f"{num_prompts} prompts x {prompt_len} tok x {samples} samples, tails U[0,{max_tail}]+1, "
             "64/8 heads, D=128, B=16, bf16, COW of the last prompt block",
    )


def config_opt13b_long(block_size: int = 16, batch: int = 8, seq_len: int = 32768) -> PagedLayout:
    """Long-context OPT-13B layer: 40/40 heads, D=128, fp16, 8 sequences of
    32768 tokens, exact-size shuffled pool, block size 8, 16 or 32."""
    seed = 1005
    rng = np.random.default_rng(seed * 100 + block_size)
    seq_lens = np.full(batch, seq_len, np.int32)
    NB = sum(_ceil_div(int(n), block_size) for n in seq_lens)
    tables = _scatter_tables(rng, seq_lens, block_size, NB)
    return _finish_layout(f"opt13b_long_b{block_size}", seed, "fp16", block_size, NB, 40, 40, 128,
                          seq_lens, tables, False,
                          note=f"{batch} seqs x {seq_len} tok, 40/40 heads, D=128, B={block_size}, fp16")


CONFIGS: Dict[str, Callable[[], PagedLayout]] = {
    "tiny": config_tiny,
    "llama7b": config_llama7b,
    "llama3_8b": config_llama3_8b,
    "llama3_8b_spec4": lambda: config_llama3_8b(q_len=4),
    "llama3_8b_prefill256": config_llama3_8b_prefill,
    "llama2_70b_shared": config_llama2_70b_shared,
    "opt13b_long_b8": lambda: config_opt13b_long(8),
    "opt13b_long_b16": lambda: config_opt13b_long(16),
    "opt13b_long_b32": lambda: config_opt13b_long(32),
}


# --------------------------------------------------------------------------
# value fillers
# --------------------------------------------------------------------------


def _row_mask(layout: PagedLayout) -> np.ndarray:
    """bool [NB, B]: True where the pool row holds a token before this step."""
    rows = np.arange(layout.block_size)[None, :]
    return rows < layout.block_fill[:, None]


def fill_values_numpy(layout: PagedLayout, value_seed: Optional[int] = None) -> PagedValues:
    """Draw q, pools and new tokens on the host as uint16 bit arrays."""
    L = layout
    rng = np.random.default_rng([L.seed if value_seed is None else value_seed, 7])
    S, Hq, Hkv, D, B, NB = L.num_seqs, L.num_q_heads, L.num_kv_heads, L.head_dim, L.block_size, L.num_blocks
    q_shape = (S, Hq, D) if L.q_len == 1 else (S, L.q_len, Hq, D)
    q = f32_to_bits(rng.standard_normal(q_shape, dtype=np.float32), L.dtype)
    nan = np.uint16(NAN_BITS[L.dtype])
    mask = _row_mask(L)[:, None, :, None]  # [NB,1,B,1]
    pools = []
    for _ in range(2):
        vals = f32_to_bits(rng.standard_normal((NB, Hkv, B, D), dtype=np.float32), L.dtype)
        pools.append(np.where(mask, vals, nan).astype(np.uint16))
    T = L.num_new_tokens
    new_k = f32_to_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32), L.dtype)
    new_v = f32_to_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32), L.dtype)
    return PagedValues(q=q, k_pool=pools[0], v_pool=pools[1], new_k=new_k, new_v=new_v)


def fill_values_torch(layout: PagedLayout, device, value_seed: Optional[int] = None,
                      chunk_blocks: int = 4096) -> PagedValues:
    """Draw the same kind of values with torch's seeded generator directly on
    ``device`` (used for pools too large to draw on the host quickly)."""
    import torch

    L = layout
    tdt = torch.float16 if L.dtype == "fp16" else torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(int(L.seed if value_seed is None else value_seed) * 7919 + 13)
    S, Hq, Hkv, D, B, NB = L.num_seqs, L.num_q_heads, L.num_kv_heads, L.head_dim, L.block_size, L.num_blocks
    q_shape = (S, Hq, D) if L.q_len == 1 else (S, L.q_len, Hq, D)
    q = torch.randn(q_shape, generator=g, device=device, dtype=torch.float32).to(tdt)
    mask_all = torch.from_numpy(_row_mask(L)).to(device)
    nan = float("nan")
    pools = []
    for _ in range(2):
        pool = torch.empty((NB, Hkv, B, D), device=device, dtype=tdt)
        for b0 in range(0, NB, chunk_blocks):
            b1 = min(NB, b0 + chunk_blocks)
            v = torch.randn((b1 - b0, Hkv, B, D), generator=g, device=device, dtype=torch.float32)
            m = mask_all[b0:b1][:, None, :, None]
            pool[b0:b1] = torch.where(m, v, torch.full_like(v, nan)).to(tdt)
        pools.append(pool)
    T = L.num_new_tokens
    new_k = torch.randn((T, Hkv, D), generator=g, device=device, dtype=torch.float32).to(tdt)
    new_v = torch.randn((T, Hkv, D), generator=g, device=device, dtype=torch.float32).to(tdt)
    return PagedValues(q=q, k_pool=pools[0], v_pool=pools[1], new_k=new_k, new_v=new_v)


def restrict_layout(layout: PagedLayout, seqs) -> PagedLayout:
    """The same workload limited to sequences ``seqs``: their blocks (and the
    copy sources feeding them) renumbered into a compact pool, the tables,
    lengths, slots and copy pairs remapped.  Used to draw bounded samples of
    a large workload for the CPU baseline."""
    L = layout
    B = L.block_size
    seqs = [int(s) for s in seqs]
    ids = []
    for s in seqs:
        ids.extend(int(b) for b in L.block_tables[s, : L.blocks_of(s)])
    dst = set(ids)
    pairs = [(int(a), int(b)) for a, b in L.copy_pairs.reshape(-1, 2) if int(b) in dst]
    ids.extend(a for a, _ in pairs)
    uniq = sorted(set(ids))
    remap = {b: i for i, b in enumerate(uniq)}
    max_nb = max([L.blocks_of(s) for s in seqs] + [1])
    tables = np.full((len(seqs), max_nb), PAD_ENTRY, np.int32)
    for i, s in enumerate(seqs):
        nb = L.blocks_of(s)
        tables[i, :nb] = [remap[int(b)] for b in L.block_tables[s, :nb]]
    slots = []
    per = L.num_new_tokens // max(L.num_seqs, 1)  # new tokens per sequence (1, or q_len)
    for s in seqs:
        for slot in L.slot_mapping[s * per:(s + 1) * per]:
            slots.append(remap[int(slot) // B] * B + int(slot) % B)
    fill = np.zeros(len(uniq), np.int32)
    for b, i in remap.items():
        fill[i] = L.block_fill[b]
    return PagedLayout(
        name=f"{L.name}[{len(seqs)} seqs]", seed=L.seed, dtype=L.dtype, block_size=B, num_blocks=len(uniq),
        num_q_heads=L.num_q_heads, num_kv_heads=L.num_kv_heads, head_dim=L.head_dim, scale=L.scale,
        seq_lens=L.seq_lens[seqs].astype(np.int32), block_tables=tables, slot_mapping=np.asarray(slots, np.int64),
        copy_pairs=np.asarray([(remap[a], remap[b]) for a, b in pairs], np.int64).reshape(-1, 2),
        block_fill=fill, note=f"sample of {L.name}", q_len=L.q_len,
    )
