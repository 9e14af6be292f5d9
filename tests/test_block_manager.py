"""The C++ host block manager against the pages' worked examples and, op by
op, against the float64 test oracle's manager (whose semantics the oracle
pins to the study notes' exercises)."""

import json
from pathlib import Path

import numpy as np
import pytest

from oracle import BlockManager as OracleBM
from oracle import block_fills, blocks_needed
from paged_kv_cache_357_b200 import BlockManager, PaError
from paged_kv_cache_357_b200 import build as pa_build
from pa_testlib import run_beam_trace

GOLDEN = json.loads((Path(__file__).parent / "golden" / "bookkeeping.json").read_text())


@pytest.fixture(scope="module", autouse=True)
def _built():
    pa_build.build()


def test_block_examples_from_pages():
    for ex in GOLDEN["block_examples"]:
        bm = BlockManager(num_blocks=100, block_size=ex["block_size"])
        bm.add(1, ex["tokens"])
        table, ntok = bm.table(1)
        assert len(table) == ex["blocks"] and ntok == ex["tokens"]
        assert bm.num_free == 100 - ex["blocks"]
        st = bm.stats()
        assert st["slots_filled"] == ex["tokens"] and st["used_blocks"] == ex["blocks"]


def test_copy_on_write_example_from_pages():
    ex = GOLDEN["copy_on_write"]
    bm = BlockManager(num_blocks=16, block_size=16)
    # make the shared block number 7 as in the exercise: consume blocks 0..6 first
    bm.add(100, 7 * 16)
    bm.add(1, 8)  # 8 prompt tokens -> block 7
    assert bm.table(1)[0] == [ex["shared_block"]]
    for i in range(2, ex["samples"] + 1):
        bm.fork(1, i)
    assert bm.ref_count(ex["shared_block"]) == ex["ref_before"]
    slot, cow = bm.append(ex["writer"])
    assert cow is not None and cow[0] == ex["shared_block"]
    new_block = cow[1]
    assert slot == new_block * 16 + 8
    assert bm.ref_count(ex["shared_block"]) == ex["ref_source_after"]
    assert bm.ref_count(new_block) == ex["ref_copy_after"]
    for i in range(1, ex["samples"] + 1):
        if i != ex["writer"]:
            assert bm.table(i)[0] == [ex["shared_block"]]
    bm.free(ex["writer"])
    assert bm.ref_count(new_block) == 0


def test_on_demand_allocation_wastes_less_than_a_block():
    bm = BlockManager(num_blocks=200, block_size=16)
    for sid, n in enumerate([1, 15, 16, 17, 40, 1000]):
        bm.add(sid, n)
        table, ntok = bm.table(sid)
        assert len(table) == blocks_needed(n, 16)
        assert len(table) * 16 - ntok < 16
        assert block_fills(n, 16)[-1] == n - (len(table) - 1) * 16


@pytest.mark.parametrize("seed", range(8))
def test_matches_oracle_manager_op_by_op(seed):
    rng = np.random.default_rng(seed)
    NB, B = 64, int(rng.choice([4, 8, 16]))
    ours, ref = BlockManager(NB, B), OracleBM(NB, B)
    ref_tables, next_id = {}, 0
    for _ in range(400):
        op = rng.choice(["add", "fork", "append", "append", "append", "free"])
        live = sorted(ref_tables)
        if op == "add":
            n = int(rng.integers(0, 3 * B))
            if blocks_needed(n, B) > len(ref.free):
                with pytest.raises(PaError):
                    ours.add(next_id, n)
                continue
            ours.add(next_id, n)
            ref_tables[next_id] = [ref.new_sequence(n), n]
            next_id += 1
        elif op == "fork" and live:
            p = int(rng.choice(live))
            ours.fork(p, next_id)
            ref_tables[next_id] = [ref.fork(ref_tables[p][0]), ref_tables[p][1]]
            next_id += 1
        elif op == "append" and live:
            s = int(rng.choice(live))
            t, n = ref_tables[s]
            needs_block = n // B == len(t) or ref.ref[t[n // B]] > 1
            if needs_block and not ref.free:
                with pytest.raises(PaError):
                    ours.append(s)
                continue
            got = ours.append(s)
            want = ref.append_slot(t, n)
            ref_tables[s][1] = n + 1
            assert got == want
        elif op == "free" and live:
            s = int(rng.choice(live))
            ours.free(s)
            ref.free_sequence(ref_tables.pop(s)[0])
        for s, (t, n) in ref_tables.items():
            assert ours.table(s) == (t, n)
        assert ours.num_free == len(ref.free)
        assert [ours.ref_count(b) for b in range(NB)] == ref.ref


def test_prepare_step_copy_on_write_fork():
    B = 16
    bm = BlockManager(num_blocks=64, block_size=B)
    bm.add(10, 40)  # 3 blocks, last 8/16 full
    for c in (11, 12, 13):
        bm.fork(10, c)
    tables, lens, slots, pairs = bm.prepare_step([10, 11, 12, 13], max_blocks_per_seq=4)
    # the first three writers copy the shared last block, the fourth finds it exclusive
    shared = bm.table(13)[0][2]
    assert pairs.shape == (3, 2) and (pairs[:, 0] == shared).all()
    assert len(set(pairs[:, 1].tolist())) == 3
    assert lens.tolist() == [41] * 4
    for i, sid in enumerate((10, 11, 12, 13)):
        t, n = bm.table(sid)
        assert tables[i, : len(t)].tolist() == t and (tables[i, len(t):] == -1).all()
        assert slots[i] == t[40 // B] * B + 40 % B
    assert tables[3, 2] == shared and all(tables[i, 2] != shared for i in range(3))
    assert bm.ref_count(shared) == 1
    assert all(bm.ref_count(int(d)) == 1 for d in pairs[:, 1])


def test_prepare_step_is_all_or_nothing():
    B = 8
    bm = BlockManager(num_blocks=4, block_size=B)
    bm.add(0, 8)   # 1 full block
    bm.add(1, 16)  # 2 full blocks
    before = (bm.table(0), bm.table(1), bm.num_free)
    with pytest.raises(PaError) as e:  # both need a fresh block, only 1 free
        bm.prepare_step([0, 1], max_blocks_per_seq=4)
    assert e.value.code == 6
    assert (bm.table(0), bm.table(1), bm.num_free) == before
    with pytest.raises(PaError):  # duplicate id
        bm.prepare_step([0, 0], max_blocks_per_seq=4)
    with pytest.raises(PaError):  # table too narrow for the grown sequence
        bm.prepare_step([1], max_blocks_per_seq=2)
    assert (bm.table(0), bm.table(1), bm.num_free) == before
    tables, lens, slots, pairs = bm.prepare_step([1], max_blocks_per_seq=3)
    assert lens.tolist() == [17] and pairs.shape == (0, 2)


def test_sharing_statistics_for_beam_style_forks():
    """Four outputs forked from one 1000-token prompt (study notes §6.2):
    unshared storage would need 4 x 63 blocks, sharing keeps 63."""
    B = 16
    bm = BlockManager(num_blocks=300, block_size=B)
    bm.add(0, 1000)
    for c in (1, 2, 3):
        bm.fork(0, c)
    st = bm.stats()
    assert st["logical_blocks"] == 4 * 63 and st["used_blocks"] == 63 and st["shared_blocks"] == 63
    assert 1 - st["used_blocks"] / st["logical_blocks"] == pytest.approx(0.75)
    # each output then decodes 24 tokens of its own: the shared 50%-full last
    # block is copied by three of them and the rest is private
    for _ in range(24):
        bm.prepare_step([0, 1, 2, 3], max_blocks_per_seq=70)
    st = bm.stats()
    assert st["tokens"] == 4 * 1024 and st["logical_blocks"] == 4 * 64
    assert st["used_blocks"] == 62 + 4 * 2 and st["shared_blocks"] == 62


BEAM_CASES = [(512, 4, 160, 0.0), (64, 8, 256, 0.0), (1000, 6, 96, 0.9), (128, 4, 512, 0.95)]


@pytest.mark.parametrize("prompt_len,width,steps,keep", BEAM_CASES)
def test_beam_search_trace_shares_blocks(prompt_len, width, steps, keep):
    """Beam search as a process tree (study notes ch.05 §6.2): beams that
    descend from one beam share the blocks of their common history, dropped
    beams free theirs, branching beams fork and copy a shared partial block
    before writing.  The C++ manager follows the oracle manager op by op
    over a seeded trace; the KV saved by sharing is reported per step."""
    B = 16
    max_nb = (prompt_len + steps) // B + 2
    nb = 4 * width * max_nb
    hist = run_beam_trace(BlockManager(nb, B), OracleBM(nb, B), prompt_len, width, steps, seed=prompt_len + width,
                          max_nb=max_nb, keep=keep)
    saving = [1 - u / l for u, l in hist]
    mean, final = float(np.mean(saving)), saving[-1]
    print(f"beam search, prompt {prompt_len}, width {width}, {steps} steps, keep {keep}: KV saved by sharing "
          f"mean {100 * mean:.1f} %, final {100 * final:.1f} %, "
          f"blocks stored {hist[-1][0]} vs {hist[-1][1]} unshared")
    # the prompt alone is shared by every beam at first: at most 1 - 1/width saved
    assert 0 < saving[0] <= 1 - 1 / width + 1e-12
    assert all(0 <= s < 1 for s in saving)
    assert final > 0  # the beams still share at least the prompt's full blocks


@pytest.mark.parametrize("prompt_len", [1000, 512, 40])
def test_beam_search_without_coalescing_shares_the_prompt_only(prompt_len):
    """keep = 1: every beam continues itself, so after the first step's
    branching the beams share exactly the prompt's full blocks.  The prompt's
    partly filled last block is copied by every writer but the last, so the
    stored blocks are floor(P/B) + width * (ceil(n/B) - floor(P/B)) for n =
    P + steps tokens per beam."""
    B, width, steps = 16, 4, 100
    max_nb = (prompt_len + steps) // B + 2
    nb = 4 * width * max_nb
    hist = run_beam_trace(BlockManager(nb, B), OracleBM(nb, B), prompt_len, width, steps, seed=3, max_nb=max_nb,
                          keep=1.0)
    for i, (used, logical) in enumerate(hist):
        n = prompt_len + i + 1
        shared = prompt_len // B
        assert logical == width * blocks_needed(n, B)
        assert used == shared + width * (blocks_needed(n, B) - shared), (i, used)
