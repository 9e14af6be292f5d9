"""The host planner of shared-prefix groups (pa_shared_prefix_groups): hand
cases, and random tables against a direct Python statement of its rule —
consecutive sequences whose first blocks agree form a group of at most
max_group_size; the group shares the leading blocks every member has in
common with the first, capped so each member keeps a block of its own; a
group of one or a prefix under min_prefix_blocks shares nothing."""

import numpy as np
import pytest

import paged_kv_cache_357_b200 as pa
from paged_kv_cache_357_b200 import build as pa_build


@pytest.fixture(scope="module", autouse=True)
def _built():
    pa_build.build()


def _rule(tables, lens, B, max_group, min_prefix=1):
    nb = [(-(-int(n) // B)) if 0 < n <= tables.shape[1] * B else 0 for n in lens]
    starts, prefix, s = [], [], 0
    S = len(lens)
    while s < S:
        first, members = s, [s]
        s += 1
        if nb[first] > 0:
            while s < S and len(members) < max_group and nb[s] > 0 and tables[s, 0] == tables[first, 0]:
                members.append(s)
                s += 1
        common = min(
            next((j for j in range(min(nb[first], nb[m])) if tables[m, j] != tables[first, j]),
                 min(nb[first], nb[m]))
            for m in members
        )
        pb = min(common, min(nb[m] for m in members) - 1)
        if len(members) < 2 or pb < max(min_prefix, 1):
            pb = 0
        starts.append(first)
        prefix.append(pb)
    starts.append(S)
    return starts, prefix


def test_hand_cases():
    B = 16
    bt = np.array([[5, 6, 7, -1], [5, 6, 8, 9], [5, 6, 10, -1], [1, 2, -1, -1], [3, -1, -1, -1], [3, 4, -1, -1]],
                  np.int32)
    lens = np.array([40, 60, 35, 20, 5, 17], np.int32)
    starts, prefix = pa.shared_prefix_groups(bt, lens, B, 4)
    assert starts.tolist() == [0, 3, 4, 6] and prefix.tolist() == [2, 0, 0]  # [3] and [3,4]: 1 own block needed
    starts, prefix = pa.shared_prefix_groups(bt, lens, B, 2)
    assert starts.tolist() == [0, 2, 3, 4, 6] and prefix.tolist() == [2, 0, 0, 0]
    starts, prefix = pa.shared_prefix_groups(bt, lens, B, 4, min_prefix_blocks=3)
    assert prefix.tolist() == [0, 0, 0]
    starts, prefix = pa.shared_prefix_groups(bt[:0], lens[:0], B, 4)
    assert starts.tolist() == [0] and prefix.tolist() == []


@pytest.mark.parametrize("seed", range(6))
def test_random_tables_follow_the_rule(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.choice([8, 16]))
    S, max_nb = 40, 12
    tables = np.full((S, max_nb), -1, np.int32)
    lens = np.zeros(S, np.int32)
    s, nxt = 0, 0
    while s < S:
        k = min(int(rng.integers(1, 6)), S - s)
        shared = int(rng.integers(0, 6))
        base = np.arange(nxt, nxt + shared)
        nxt += shared
        for m in range(k):
            n = int(rng.integers(0, max_nb * B + 1)) if rng.random() < 0.9 else int(rng.integers(-3, 0))
            nb = -(-max(n, 0) // B)
            row = np.concatenate([base, np.arange(nxt, nxt + max_nb)])[:nb]
            nxt += max_nb
            tables[s + m, :nb] = row
            lens[s + m] = n
        s += k
    for max_group in (1, 2, 4, 8):
        got = pa.shared_prefix_groups(tables, lens, B, max_group)
        want = _rule(tables, lens, B, max_group)
        assert got[0].tolist() == want[0] and got[1].tolist() == want[1], max_group
