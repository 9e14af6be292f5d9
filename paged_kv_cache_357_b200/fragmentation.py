"""KV-memory waste of three allocation schemes on a synthetic request trace.

The study notes ch.05 §2 name three kinds of waste in KV-cache memory:
slots reserved for a maximum length that is never reached, internal
fragmentation (reserved but unfilled), and external fragmentation (holes
between contiguous allocations).  Exercise 6 asks for a simulator that
compares reserving the maximum length, reserving exactly what a request
will use, and paging, and checks that paging drives fragmentation towards
zero.  This module is that simulator:

* ``reserve_max``:   each request takes ``max_len`` contiguous slots (first
                     fit in one arena) for its whole life.
* ``reserve_exact``: each request takes exactly its final length contiguous
                     slots (an allocator that knows the future: no internal
                     waste, but holes between requests remain).
* ``paged``:         blocks of ``block_size`` slots taken on demand from the
                     C++ block manager as tokens are generated; a request
                     never holds more than one partly filled block.  When a
                     step finds no free block for any waiting request, the
                     most recently admitted request is preempted: its blocks
                     are freed and it goes back to the front of the queue
                     (study notes §5 ③); no request is admitted again until
                     one finishes, so the preempted one cannot starve anew.

Requests arrive with a prompt and an output length, are admitted first come
first served while memory allows, generate one token per step and leave
when done.  Reported: the fraction of allocated KV slots that hold a token
(time-averaged; the quantity behind the notes' 20.4%-38.2% for existing
systems), waste per request, steps to finish the trace, peak concurrency,
admissions blocked by memory, and preemptions.
"""

from __future__ import annotations

import bisect
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np


@dataclass
class Request:
    prompt: int
    output: int

    @property
    def total(self) -> int:
        return self.prompt + self.output


def reservation_waste(final_lengths: Sequence[int], reserved: int) -> List[int]:
    """Slots a fixed reservation leaves unused per request (study notes §2's
    first waste; the CSDN article's example: 4000 reserved, 2000 and 500
    used, 5500 wasted in total)."""
    return [reserved - n for n in final_lengths]


def synthetic_trace(n: int, seed: int = 0, mean_prompt: float = 300.0, mean_output: float = 200.0,
                    max_len: int = 2048) -> List[Request]:
    """Exponentially distributed prompt and output lengths, capped so that
    prompt + output <= max_len (the kind of mix the notes' §2 describes:
    actual lengths far below the maximum)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        p = int(min(max_len - 1, max(1, rng.exponential(mean_prompt))))
        o = int(min(max_len - p, max(1, rng.exponential(mean_output))))
        out.append(Request(p, o))
    return out


class _Arena:
    """First-fit contiguous allocator over [0, capacity) slots."""

    def __init__(self, capacity: int):
        self.free: List[Tuple[int, int]] = [(0, capacity)]  # sorted (start, length)

    def alloc(self, n: int) -> Optional[int]:
        for i, (start, length) in enumerate(self.free):
            if length >= n:
                if length == n:
                    self.free.pop(i)
                else:
                    self.free[i] = (start + n, length - n)
                return start
        return None

    def release(self, start: int, n: int) -> None:
        i = bisect.bisect_left(self.free, (start, 0))
        self.free.insert(i, (start, n))
        merged: List[Tuple[int, int]] = []
        for s, l in self.free:
            if merged and merged[-1][0] + merged[-1][1] == s:
                merged[-1] = (merged[-1][0], merged[-1][1] + l)
            else:
                merged.append((s, l))
        self.free = merged


def simulate(requests: Sequence[Request], capacity_tokens: int, policy: str, block_size: int = 16,
             max_len: int = 2048) -> Dict[str, float]:
    """Run the trace to completion under one policy."""
    if policy not in ("reserve_max", "reserve_exact", "paged"):
        raise ValueError(policy)
    queue = list(range(len(requests)))
    active: Dict[int, int] = {}  # request -> tokens generated so far (prompt included)
    where: Dict[int, int] = {}
    arena = _Arena(capacity_tokens) if policy != "paged" else None
    bm = None
    if policy == "paged":
        from .block_manager import BlockManager

        bm = BlockManager(capacity_tokens // block_size, block_size)
    stored_sum, held_sum, steps, peak, blocked, waste_sum, waste_n, preempted = 0, 0, 0, 0, 0, 0.0, 0, 0

    def held(r: int) -> int:
        if policy == "reserve_max":
            return max_len
        if policy == "reserve_exact":
            return requests[r].total
        return -(-active[r] // block_size) * block_size

    admit = True
    while queue or active:
        # admit first come first served while the head of the queue fits
        while queue and admit:
            r = queue[0]
            req = requests[r]
            if policy == "paged":
                need = -(-req.prompt // block_size)
                if need > bm.num_free:
                    break
                bm.add(r, req.prompt)
            else:
                size = max_len if policy == "reserve_max" else req.total
                start = arena.alloc(size)
                if start is None:
                    break
                where[r] = start
            active[r] = req.prompt
            queue.pop(0)
        if queue and not active:
            raise RuntimeError("a request does not fit in an empty pool")
        if queue:
            blocked += 1
        peak = max(peak, len(active))
        steps += 1
        for r in list(active):
            h = held(r)
            stored_sum += active[r]
            held_sum += h
            waste_sum += h - active[r]
            waste_n += 1
        # one decode step: every active request generates a token
        done, starved = [], []
        for r in list(active):
            if policy == "paged":
                try:
                    bm.append(r)
                except Exception:
                    starved.append(r)  # no block this step: the request waits
                    continue
            active[r] += 1
            if active[r] >= requests[r].total:
                done.append(r)
        if starved and not done and len(starved) == len(active):
            victim = max(active)  # requests are admitted in index order
            bm.free(victim)
            del active[victim]
            queue.insert(0, victim)
            preempted += 1
            admit = False
        if done:
            admit = True
        for r in done:
            if policy == "paged":
                bm.free(r)
            else:
                size = max_len if policy == "reserve_max" else requests[r].total
                arena.release(where.pop(r), size)
            del active[r]
    if bm is not None:
        bm.close()
    return {
        "policy": policy,
        "steps": steps,
        "fill": stored_sum / max(held_sum, 1),
        "mean_waste_per_request_tokens": waste_sum / max(waste_n, 1),
        "peak_concurrency": peak,
        "steps_with_blocked_admission": blocked,
        "preemptions": preempted,
    }


def compare(n_requests: int = 400, capacity_tokens: int = 16 * 2048, block_size: int = 16, seed: int = 0,
            max_len: int = 2048) -> List[Dict[str, float]]:
    trace = synthetic_trace(n_requests, seed=seed, max_len=max_len)
    return [simulate(trace, capacity_tokens, p, block_size, max_len) for p in ("reserve_max", "reserve_exact", "paged")]


if __name__ == "__main__":
    import json

    for row in compare():
        print(json.dumps(row))
