"""Seeded beam-search traces for the block manager (structure only: which
beam continues which, no scores or attention arithmetic).

Study notes ch.05 §6.2 describe beam search over a paged cache as a process
tree: beams that descend from the same beam share the blocks of their common
history, a beam that is dropped frees its blocks, and one that branches
forks; a writer to a shared block copies it first.  A trace here is, per
step, the parent (an index into the current beams) of each of the `width`
beams that continue.  Parents are drawn with skewed weights (a Dirichlet
draw per step), so some beams branch several times and others die, the way
the best-scoring beams take over a search.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple

import numpy as np


def beam_parents(seed: int, width: int, steps: int, concentration: float = 0.5,
                 keep: float = 0.0) -> List[List[int]]:
    """For each step, the sorted parent indices (0 .. width-1) of the
    `width` beams that continue.  Beam i continues itself with probability
    `keep`; otherwise its parent is drawn with skewed weights (smaller
    `concentration`: fewer parents with more children each).  keep = 0 is a
    neutral genealogy, in which the beams descend from one beam of about
    `width` steps back; keep near 1 keeps them apart for longer."""
    rng = np.random.default_rng([seed, width, steps, int(round(keep * 1000))])
    out = []
    for _ in range(steps):
        w = rng.dirichlet(np.full(width, concentration))
        drawn = rng.choice(width, size=width, p=w)
        stay = rng.random(width) < keep
        out.append(sorted(int(i) if stay[i] else int(drawn[i]) for i in range(width)))
    return out


@dataclass
class BeamStep:
    """What one step of a trace does to the live beams (by sequence id):
    free the beams with no child, fork each extra child from its parent
    (before any token of this step is appended), then append one token to
    every beam in `live` (the parents that continue, then the new children)."""

    frees: List[int] = field(default_factory=list)
    forks: List[Tuple[int, int]] = field(default_factory=list)  # (parent id, child id)
    live: List[int] = field(default_factory=list)


def beam_step(live: List[int], parents: List[int], next_id: int) -> Tuple[BeamStep, int]:
    """Turn one step's parent indices into operations on sequence ids.  The
    first child of a parent keeps the parent's id; further children get new
    ids from `next_id` on.  Returns the step and the next unused id."""
    step = BeamStep()
    counts = [0] * len(live)
    for p in parents:
        counts[p] += 1
    for i, sid in enumerate(live):
        if counts[i] == 0:
            step.frees.append(sid)
    kept, children = [], []
    for i, sid in enumerate(live):
        if counts[i] == 0:
            continue
        kept.append(sid)
        for _ in range(counts[i] - 1):
            step.forks.append((sid, next_id))
            children.append(next_id)
            next_id += 1
    step.live = kept + children
    return step, next_id
