"""A model of the Newton-Schulz chain's tile schedule, checked for progress (CPU).

The persistent kernel lists every tile of every step, phase and matrix in one
order; CTA pair p takes tiles p, p + P, p + 2P, ... A tile waits on a
per-matrix counter of the phase it reads (Gram(k) on Apply(k-1), a split
Gram's Reduce(k) on Gram(k), Poly(k) on Gram(k) or Reduce(k), Apply(k) on
Poly(k)). In a pair, the MMA issuer runs at most two tiles ahead of the
epilogue (two TMEM accumulators; one is handed back when every epilogue warp
of both CTAs has its last chunk in registers). Each of the 16 epilogue warps
(8 per CTA) confirms its part of an MMA tile late: after its next tile's
chunk loop, or at once when that next tile's dependency is not met when the
warp starts it (the rule that keeps the late publish from holding up a tile
that needs it); the last of a CTA's 8 warps to confirm adds the CTA's part
to the counter. A Reduce sub-tile is summed by the epilogue warps alone:
each warp confirms any pending tile, waits for the tile's dependency, and
publishes its own part at once.

This module simulates that protocol with random durations, phase by phase
for small banks (including a split Gram) and a few pairs, and checks that
every tile completes and that no tile's MMA or epilogue loads started before
its dependency was met. The same model without the early-confirm rule
deadlocks when a pair's next tile needs its previous one, which shows that
the check can see a deadlock.
"""
import random
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import pytest

GRAM, POLY, APPLY, REDUCE = 0, 1, 2, 3
TILE_PARTS = 2          # one part per CTA of a pair
WARPS = 8               # epilogue warps per CTA
RED_PARTS = 2 * WARPS   # a Reduce sub-tile: one part per epilogue warp of both CTAs
RED_SUB = 4


@dataclass
class Bank:
    count: int
    nb: int          # 256-blocks of the Gram side (rp / 256)
    napply: int      # Apply tiles per matrix
    ksplit: int = 1  # K splits of the Gram product


@dataclass
class Tile:
    phase: int
    iter: int
    bank: int
    mat: int
    dep: Optional[Tuple[int, int, int]]   # (bank, mat, phase) counter
    target: int


def tile_list(banks: List[Bank], steps: int) -> List[Tile]:
    """The kernel's order: step by step, phase by phase (Gram, Reduce, Poly,
    Apply), bank by bank, matrix by matrix."""
    out = []
    for k in range(steps):
        for phase in (GRAM, REDUCE, POLY, APPLY):
            for b, bk in enumerate(banks):
                sym = bk.nb * (bk.nb + 1) // 2
                for m in range(bk.count):
                    if phase == GRAM:
                        n, dep = sym * bk.ksplit, (b, m, APPLY)
                        target = TILE_PARTS * bk.napply * k
                    elif phase == REDUCE:
                        if bk.ksplit == 1:
                            continue
                        n, dep = sym * RED_SUB, (b, m, GRAM)
                        target = TILE_PARTS * sym * bk.ksplit * (k + 1)
                    elif phase == POLY:
                        n = sym
                        if bk.ksplit > 1:
                            dep, target = (b, m, REDUCE), RED_PARTS * sym * RED_SUB * (k + 1)
                        else:
                            dep, target = (b, m, GRAM), TILE_PARTS * sym * (k + 1)
                    else:
                        n, dep = bk.napply, (b, m, POLY)
                        target = TILE_PARTS * sym * (k + 1)
                    out += [Tile(phase, k, b, m, dep, target) for _ in range(n)]
    return out


@dataclass
class Warp:
    pair: int
    cta: int
    pos: int = 0                    # index into the pair's tile list
    busy_until: int = 0
    state: str = "start"            # start, wait_dep, wait_full, chunks, done
    pending: Optional[int] = None   # global tile index whose confirm is late


@dataclass
class Pair:
    tiles: List[int]
    mma_pos: int = 0                # next tile (index into tiles) the MMA will run
    mma_busy_until: int = 0
    mma_running: Optional[int] = None
    full: Dict[int, int] = field(default_factory=dict)        # pos -> time the accumulator is full
    released: Dict[int, int] = field(default_factory=dict)    # pos -> warps that handed it back


def simulate(banks, steps, pairs, seed, early_confirm=True, max_time=2_000_000):
    rng = random.Random(seed)
    tiles = tile_list(banks, steps)
    counters: Dict[Tuple[int, int, int], int] = {}
    cta_parts: Dict[Tuple[int, int], int] = {}
    P = [Pair([t for t in range(p, len(tiles), pairs)]) for p in range(pairs)]
    W = [Warp(p, c) for p in range(pairs) for c in range(2) for _ in range(WARPS)]
    done_tiles = set()
    violations = []

    def met(t: Tile) -> bool:
        return t.target <= 0 or counters.get(t.dep, 0) >= t.target

    def confirm(w: Warp, g: int):
        key = (g, w.cta)
        cta_parts[key] = cta_parts.get(key, 0) + 1
        if cta_parts[key] == WARPS:
            t = tiles[g]
            c = (t.bank, t.mat, t.phase)
            counters[c] = counters.get(c, 0) + 1
            if cta_parts.get((g, 1 - w.cta), 0) == WARPS:
                done_tiles.add(g)

    now = 0
    while now < max_time:
        progressed = False
        # ---- MMA issuers: at most two tiles ahead of the epilogue
        for pr in P:
            if pr.mma_running is not None and pr.mma_busy_until <= now:
                pr.full[pr.mma_running] = now
                pr.mma_running = None
                progressed = True
            while pr.mma_running is None and pr.mma_pos < len(pr.tiles):
                t = tiles[pr.tiles[pr.mma_pos]]
                if t.phase == REDUCE:           # no MMA
                    pr.mma_pos += 1
                    continue
                # the accumulator of two MMA tiles ago must have been handed back
                mma_before = [q for q in range(pr.mma_pos) if tiles[pr.tiles[q]].phase != REDUCE]
                if len(mma_before) >= 2 and pr.released.get(mma_before[-2], 0) < 2 * WARPS:
                    break
                if not met(t):
                    break
                pr.mma_running = pr.mma_pos
                pr.mma_busy_until = now + rng.randint(1, 40)
                pr.mma_pos += 1
                progressed = True
        # ---- epilogue warps
        for w in W:
            if w.busy_until > now or w.state == "done":
                continue
            pr = P[w.pair]
            if w.pos >= len(pr.tiles):
                if w.pending is not None:
                    confirm(w, w.pending)
                    w.pending = None
                w.state = "done"
                progressed = True
                continue
            g = pr.tiles[w.pos]
            t = tiles[g]
            if t.phase == REDUCE:
                if w.state == "start":
                    if w.pending is not None:
                        confirm(w, w.pending)
                        w.pending = None
                    w.state = "wait_dep"
                    progressed = True
                if w.state == "wait_dep":
                    if not met(t):
                        continue
                    w.state = "chunks"
                    w.busy_until = now + rng.randint(1, 10)
                    progressed = True
                    continue
                if w.state == "chunks":      # publish this warp's part at once
                    c = (t.bank, t.mat, REDUCE)
                    counters[c] = counters.get(c, 0) + 1
                    w.pos += 1
                    w.state = "start"
                    progressed = True
                continue
            if w.state == "start":
                if early_confirm and w.pending is not None and not met(t):
                    confirm(w, w.pending)
                    w.pending = None
                w.state = "wait_dep" if t.phase != GRAM else "wait_full"
                progressed = True
            if w.state == "wait_dep":        # the epilogue's own loads read the finished phase
                if not met(t):
                    continue
                w.state = "wait_full"
                progressed = True
            if w.state == "wait_full":
                if w.pos not in pr.full:
                    continue
                if not met(t):
                    violations.append((g, "accumulator full before the dependency was met"))
                pr.released[w.pos] = pr.released.get(w.pos, 0) + 1   # last chunk in registers
                w.state = "chunks"
                w.busy_until = now + rng.randint(1, 30)
                progressed = True
                continue
            if w.state == "chunks":
                if w.pending is not None:
                    confirm(w, w.pending)
                w.pending = g
                w.pos += 1
                w.state = "start"
                progressed = True
        if all(w.state == "done" for w in W) and all(pr.mma_running is None for pr in P):
            mma = {i for i, t in enumerate(tiles) if t.phase != REDUCE}
            return mma <= done_tiles, violations, now
        if not progressed:
            busy = [w.busy_until for w in W if w.busy_until > now] + \
                   [pr.mma_busy_until for pr in P if pr.mma_running is not None]
            if not busy:
                return False, violations, now      # nothing runs and nothing can start
            now = min(busy)
            continue
        now += 1
    return False, violations, now


BANKS = [
    [Bank(3, 1, 2), Bank(2, 2, 4)],             # 256 x 512 and 512 x 1024-like banks
    [Bank(2, 3, 9), Bank(1, 3, 36)],            # GPT-bank-like shapes (768 wide)
    [Bank(1, 3, 9, ksplit=4), Bank(2, 1, 1)],   # a split Gram (readout-like) with a small bank
]


@pytest.mark.parametrize("banks", BANKS, ids=["small", "gpt-like", "split-gram"])
@pytest.mark.parametrize("pairs", [1, 3, 5])
def test_every_tile_completes_in_the_right_order(banks, pairs):
    for seed in range(12):
        ok, violations, _ = simulate(banks, 3, pairs, seed)
        assert ok, (pairs, seed)
        assert not violations, violations[:3]


def test_late_confirm_without_the_early_rule_can_deadlock():
    """Without confirming a pending tile before waiting on an unmet
    dependency, the schedule stalls for good when a pair's next tile needs its
    previous one (one matrix, one tile per phase, one pair): the check is able
    to see a deadlock. With the rule the same schedule completes."""
    for seed in range(5):
        ok, _, _ = simulate([Bank(1, 1, 1)], 3, 1, seed, early_confirm=False)
        assert not ok
        ok, violations, _ = simulate([Bank(1, 1, 1)], 3, 1, seed)
        assert ok and not violations
