"""Helpers shared by the GPU parity tests: move generator bits to the device,
run one step through the C-ABI binding, run the oracle step on the same bits,
and compare.

Tolerance (the reading used throughout).  The stated bounds are max-abs 2e-3
and max-rel 1e-2.  Each is asserted where the 16-bit output can meet it:

* max-abs: |gpu - oracle| <= 2e-3 for every element with |oracle| < 0.5.
  There, rounding to bf16 alone moves a value by at most 2^-10 = 9.8e-4, so
  the bound leaves about 1e-3 for the arithmetic.  Above 0.5 the rounding
  alone can reach 2^-9 = 1.95e-3 (and 3.9e-3 in [1, 2)), so an exact answer
  correctly rounded could fail an absolute bound there.
* max-rel: |gpu - oracle| / |oracle| <= 1e-2 for every element with
  |oracle| >= 0.1 (bf16 rounding is at most 2^-9 = 0.39 % relative).
* and every element, whatever its size, within 2e-3 + 1e-2 * |oracle|.
"""

from __future__ import annotations

import numpy as np

import oracle
from workloads import PagedLayout, PagedValues, bits_to_torch

ATOL = 2e-3
RTOL = 1e-2


def to_device(layout: PagedLayout, values: PagedValues, device):
    """Torch device tensors for one layout (numpy bit arrays or torch tensors)."""
    import torch

    def t16(x):
        if isinstance(x, np.ndarray):
            return bits_to_torch(x, layout.dtype).to(device)
        return x.to(device)

    return dict(
        q=t16(values.q),
        k_pool=t16(values.k_pool).contiguous(),
        v_pool=t16(values.v_pool).contiguous(),
        new_k=t16(values.new_k),
        new_v=t16(values.new_v),
        tables=torch.from_numpy(layout.block_tables).to(device),
        lens=torch.from_numpy(layout.seq_lens).to(device),
        slots=torch.from_numpy(layout.slot_mapping).to(device),
        pairs=torch.from_numpy(layout.copy_pairs.reshape(-1, 2)).to(device),
    )


def torch_bits(t) -> np.ndarray:
    """uint16 bit array of a 16-bit torch tensor (any device)."""
    import torch

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def torch_f64(t) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def gpu_step(dev_t, layout: PagedLayout, *, num_ctas: int = 0, do_copy=True, do_write=True, status=None,
             workspace=None, one_launch=False):
    """copy -> write -> decode through the C ABI; returns (out tensor, status tensor).
    With one_launch the three go through pa_decode_update (the writes inside
    the decode's launch), as the benchmark's step does."""
    import torch

    import paged_kv_cache_357_b200 as pa

    d = dev_t
    st = torch.zeros(1, dtype=torch.int32, device=d["q"].device) if status is None else status
    copy = do_copy and layout.copy_pairs.shape[0] > 0
    write = do_write and layout.num_new_tokens > 0
    out = torch.full_like(d["q"], float("nan"))
    ws = workspace
    if ws is None:
        ws = pa.alloc_decode_workspace(layout.num_seqs, layout.num_q_heads, d["k_pool"], num_ctas)
    if one_launch:
        upd = {}
        if copy:
            upd["copy_pairs"] = d["pairs"]
        if write:
            upd.update(new_k=d["new_k"], new_v=d["new_v"], slot_mapping=d["slots"])
        pa.pa_decode_update(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], layout.scale, out, ws, st,
                            num_ctas=num_ctas, **upd)
        torch.cuda.synchronize()
        return out, st
    if copy:
        pa.pa_copy_blocks(d["pairs"], d["k_pool"], d["v_pool"], st)
    if write:
        pa.pa_cache_write(d["new_k"], d["new_v"], d["slots"], d["k_pool"], d["v_pool"], st)
    pa.pa_decode(d["q"], d["k_pool"], d["v_pool"], d["tables"], d["lens"], layout.scale, out, ws, st,
                 num_ctas=num_ctas)
    torch.cuda.synchronize()
    return out, st


def oracle_step(layout: PagedLayout, values: PagedValues, *, do_copy=True, do_write=True):
    """The same step on the host in float64: returns (out, k_pool, v_pool)."""
    kp, vp = values.k_pool, values.v_pool
    if do_copy and layout.copy_pairs.shape[0] > 0:
        kp, vp = oracle.copy_blocks(kp, vp, layout.copy_pairs)
    if do_write and layout.num_new_tokens > 0:
        kp, vp = oracle.cache_write(kp, vp, values.new_k, values.new_v, layout.slot_mapping)
    out = oracle.decode(values.q, kp, vp, layout.block_tables, layout.seq_lens, layout.scale,
                        layout.num_kv_heads, layout.dtype)
    return out, kp, vp


ABS_BELOW = 0.5   # max-abs is asserted for |oracle| below this
REL_ABOVE = 0.1   # max-rel is asserted for |oracle| at or above this


def attention_errors(got: np.ndarray, ref: np.ndarray):
    """(max abs error over |ref| < ABS_BELOW, max rel error over |ref| >=
    REL_ABOVE, max abs error over all elements)."""
    err = np.abs(got - ref)
    mag = np.abs(ref)
    small, big = mag < ABS_BELOW, mag >= REL_ABOVE
    max_abs = float(err[small].max()) if small.any() else 0.0
    max_rel = float((err[big] / mag[big]).max()) if big.any() else 0.0
    return max_abs, max_rel, float(err.max()) if err.size else 0.0


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Assert the tolerance reading above; returns attention_errors."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside 2e-3 + 1e-2*|ref|; "
            f"max abs err {err.max():.3e}; first bad {idx}; got {got[bad][:5]} ref {ref[bad][:5]}"
        )
    max_abs, max_rel, max_all = attention_errors(got, ref)
    assert max_abs <= ATOL, f"{what}: max abs err {max_abs:.3e} over |ref| < {ABS_BELOW} exceeds {ATOL}"
    assert max_rel <= RTOL, f"{what}: max rel err {max_rel:.3e} over |ref| >= {REL_ABOVE} exceeds {RTOL}"
    return max_abs, max_rel, max_all


def subproblem(layout: PagedLayout, values_dev, seqs):
    """Host bits (pre-step state) of the blocks that sequences `seqs` read,
    plus the copy sources feeding them, renumbered into a compact pool.
    values_dev are the generator's torch device tensors, captured before any
    kernel runs.  Returns (compact layout fields, compact values)."""
    import torch

    B = layout.block_size
    seqs = list(seqs)
    ids = []
    for s in seqs:
        ids.extend(layout.block_tables[s, : layout.blocks_of(s)].tolist())
    dst_set = set(ids)
    pairs = [(int(a), int(b)) for a, b in layout.copy_pairs.reshape(-1, 2) if int(b) in dst_set]
    ids.extend(a for a, _ in pairs)
    uniq = sorted(set(ids))
    remap = {b: i for i, b in enumerate(uniq)}
    idx = torch.tensor(uniq, dtype=torch.long, device=values_dev.k_pool.device)
    kp = torch_bits(values_dev.k_pool.index_select(0, idx))
    vp = torch_bits(values_dev.v_pool.index_select(0, idx))
    max_nb = max(layout.blocks_of(s) for s in seqs)
    tables = np.full((len(seqs), max_nb), -1, np.int32)
    for i, s in enumerate(seqs):
        nb = layout.blocks_of(s)
        tables[i, :nb] = [remap[int(b)] for b in layout.block_tables[s, :nb]]
    cpairs = np.array([(remap[a], remap[b]) for a, b in pairs], np.int64).reshape(-1, 2)
    q = torch_bits(values_dev.q[seqs])
    slots, nk, nv = [], [], []
    if layout.num_new_tokens > 0:
        # every sequence writes the same number of new tokens, in sequence order
        per = layout.num_new_tokens // layout.num_seqs
        assert per * layout.num_seqs == layout.num_new_tokens
        toks = [s * per + i for s in seqs for i in range(per)]
        for t in toks:
            slot = int(layout.slot_mapping[t])
            blk, row = slot // B, slot % B
            slots.append(remap[blk] * B + row)
        nk = torch_bits(values_dev.new_k[toks])
        nv = torch_bits(values_dev.new_v[toks])
    return dict(q=q, k_pool=kp, v_pool=vp, tables=tables, lens=layout.seq_lens[seqs].copy(), pairs=cpairs,
                slots=np.asarray(slots, np.int64), new_k=nk, new_v=nv)


def oracle_subproblem(layout: PagedLayout, sub, heads=None) -> np.ndarray:
    """Oracle outputs [len(seqs), len(heads), D] of a subproblem after its
    copies and writes (heads: the q heads to compute, default all)."""
    kp, vp = sub["k_pool"], sub["v_pool"]
    if sub["pairs"].shape[0] > 0:
        kp, vp = oracle.copy_blocks(kp, vp, sub["pairs"])
    if sub["slots"].shape[0] > 0:
        kp, vp = oracle.cache_write(kp, vp, sub["new_k"], sub["new_v"], sub["slots"])
    heads = list(range(layout.num_q_heads)) if heads is None else list(heads)
    out = np.zeros((sub["q"].shape[0], len(heads), layout.head_dim))
    for i in range(sub["q"].shape[0]):
        for k, h in enumerate(heads):
            out[i, k] = oracle.decode_one(i, h, sub["q"], kp, vp, sub["tables"], sub["lens"], layout.scale,
                                          layout.num_kv_heads, layout.dtype)
    return out


def oracle_manager_step(mgr, tables, seq_ids, max_nb):
    """The oracle manager's arrays for one step that appends one token to
    each of seq_ids: (block_tables, seq_lens, slot_mapping, copy_pairs).
    tables maps a sequence id to [its oracle block table, its token count]."""
    n = len(seq_ids)
    bt = np.full((n, max_nb), -1, np.int32)
    lens = np.zeros(n, np.int32)
    slots = np.zeros(n, np.int64)
    pairs = []
    for i, s in enumerate(seq_ids):
        t, ntok = tables[s]
        slot, cow = mgr.append_slot(t, ntok)
        tables[s][1] = ntok + 1
        slots[i] = slot
        if cow is not None:
            pairs.append(cow)
        bt[i, : len(t)] = t
        lens[i] = ntok + 1
    return bt, lens, slots, np.asarray(pairs, np.int64).reshape(-1, 2)


def run_beam_trace(ours, ref, prompt_len: int, width: int, steps: int, seed: int, max_nb: int, on_step=None,
                   keep: float = 0.0):
    """Beam search over one prompt (study notes ch.05 §6.2), driven through
    the C++ manager `ours` and the oracle manager `ref` side by side: the
    first step branches the prompt into `width` beams, later steps follow
    workloads.beam's seeded trace with continuation probability `keep` (free
    the beams that die, fork the ones that branch, append one token to every
    live beam).  Every step's kernel
    arrays must agree between the two managers.  on_step(i, live, arrays)
    sees each step's arrays.  Returns per step (used blocks, logical
    blocks), logical = what the live beams would hold without sharing."""
    from workloads.beam import beam_parents, beam_step

    ours.add(0, prompt_len)
    tables = {0: [ref.new_sequence(prompt_len), prompt_len]}
    live, next_id = [0], 1
    history = []
    for i, parents in enumerate([[0] * width] + beam_parents(seed, width, steps - 1, keep=keep)):
        st, next_id = beam_step(live, parents, next_id)
        for sid in st.frees:
            ours.free(sid)
            ref.free_sequence(tables.pop(sid)[0])
        for parent, child in st.forks:
            ours.fork(parent, child)
            tables[child] = [ref.fork(tables[parent][0]), tables[parent][1]]
        live = st.live
        arrays = ours.prepare_step(live, max_nb)
        want = oracle_manager_step(ref, tables, live, max_nb)
        for got, exp in zip(arrays, want):
            assert np.array_equal(got, exp), f"beam step {i}: the managers differ"
        stats = ours.stats()
        used = len(ref.ref) - len(ref.free)
        assert stats["used_blocks"] == used
        assert stats["logical_blocks"] == sum(len(tables[s][0]) for s in live)
        history.append((stats["used_blocks"], stats["logical_blocks"]))
        if on_step is not None:
            on_step(i, live, arrays)
    return history


def bits_to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values of fp16/bf16 bit patterns (exact)."""
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def rising_scores(layout: PagedLayout, values: PagedValues, q_bits: np.ndarray, seed: int, rate: float = 1 / 256):
    """Inputs whose scores rise along each sequence: every cached key (and
    every new key, at the position it is written to) scaled by 1 + rate * t
    at token position t, and each query row (a sequence's position and
    head) scaled by a factor drawn from [0.05, 1.6].  A row's running max is
    then passed by a wide margin in the middle of a sequence, for some rows
    of a tile and not for others.  Returns (values with the scaled keys,
    scaled query bits)."""
    from dataclasses import replace

    from workloads import f32_to_bits

    dt, B = layout.dtype, layout.block_size
    k = bits_to_f32(values.k_pool, dt)
    pos = {}
    for s, n in enumerate(layout.seq_lens):
        for t in range(int(n)):
            pos[(int(layout.block_tables[s, t // B]), t % B)] = t
    for (blk, off), t in pos.items():  # a shared slot once, at its position
        k[blk, :, off, :] *= 1.0 + rate * t
    new_k = values.new_k
    if layout.num_new_tokens > 0:
        nk = bits_to_f32(new_k, dt)
        for i, sl in enumerate(layout.slot_mapping):
            nk[i] *= 1.0 + rate * pos[(int(sl) // B, int(sl) % B)]
        new_k = f32_to_bits(nk, dt)
    rng = np.random.default_rng([seed, 5])
    qf = bits_to_f32(q_bits, dt)
    row_scale = rng.uniform(0.05, 1.6, size=qf.shape[:-1] + (1,)).astype(np.float32)
    return replace(values, k_pool=f32_to_bits(k, dt), new_k=new_k), f32_to_bits(qf * row_scale, dt)
