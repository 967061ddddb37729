"""A CPU model of the one-launch front end's cross-CTA protocol
(`front_kernel` in csrc/front.cu).

The launch holds two kinds of work item in one linear grid: tile items (one
tensor of one head, 256 tiled rows: one 256-token block or four 64-token
blocks) and score items (8 query blocks of one head).  A tile item whose
block means the scoring needs writes them and then adds one to its head's
arrival counter; a score item waits until every such item of its head has
arrived, reads the means, and adds one to its head's finished counter; the
head's last score item sets both counters back to zero, so the caller's
workspace is zero again after the launch.

The model decodes every grid index exactly as the kernel does, makes CTAs
resident in index order into a fixed number of slots (the hardware hands out
blocks in order as slots free up), and runs the resident CTAs' steps under
random schedules.  It checks that every item is decoded exactly once, that no
schedule deadlocks (a score item only ever waits on lower-numbered items), that
no score item reads a block mean before it is written, that no counter is reset
while a score item of its head still has to pass its wait, and that the
workspace ends at zero.  Planted mistakes must be caught.
"""
import random

import pytest

ROWS = 8  # query blocks per score item


class Deadlock(AssertionError):
    pass


class Hazard(AssertionError):
    pass


def decode(L, NB, BH, BS, select, compress):
    """(kind, head, item) of grid index L, as the kernel decodes it."""
    score = select or compress
    kb = 256 // BS
    nT = (NB + kb - 1) // kb
    nA = 3 * nT if (compress or not score) else 2 * nT
    nB = (NB + ROWS - 1) // ROWS if score else 0
    per = nA + nB
    if not score:
        return "tile", L // nA, L % nA
    if L < nA:
        return "tile", 0, L
    if L < BH * per:
        s = (L - nA) // per + 1
        off = (L - nA) - (s - 1) * per
        if s < BH and off < nA:
            return "tile", s, off
        if s < BH:
            return "score", s - 1, off - nA
        return "score", BH - 1, off
    vi = L - BH * per
    return "tile", vi // nT, 2 * nT + vi % nT


def grid_size(NB, BH, BS, select, compress):
    kb = 256 // BS
    nT = (NB + kb - 1) // kb
    nB = (NB + ROWS - 1) // ROWS if (select or compress) else 0
    return BH * (3 * nT + nB)


class FrontModel:
    def __init__(self, NB, BH, BS, select, compress, slots, seed, plant=None):
        self.NB, self.BH, self.BS, self.select, self.compress = NB, BH, BS, select, compress
        self.score = select or compress
        self.kb = 256 // BS
        self.nT = (NB + self.kb - 1) // self.kb
        self.nB = (NB + ROWS - 1) // ROWS if self.score else 0
        self.target = (3 if compress else 2) * self.nT  # pooled items per head
        self.slots, self.rng, self.plant = slots, random.Random(seed), plant
        self.arrive = [0] * BH
        self.done = [0] * BH
        self.means = set()          # (head, tensor, block) written
        self.passed = [0] * BH      # score items of the head past their wait
        self.grid = grid_size(NB, BH, BS, select, compress)

    def items(self):
        order = list(range(self.grid))
        if self.plant == "scores_first":  # every score item ahead of the tile items
            kinds = [decode(L, self.NB, self.BH, self.BS, self.select, self.compress)[0] for L in order]
            order = [L for L in order if kinds[L] == "score"] + [L for L in order if kinds[L] == "tile"]
        return order

    def cta(self, L):
        kind, head, item = decode(L, self.NB, self.BH, self.BS, self.select, self.compress)
        if kind == "tile":
            tensor, g = item // self.nT, item % self.nT
            blocks = [b for b in range(g * self.kb, (g + 1) * self.kb) if b < self.NB]
            pools = self.score and (tensor < 2 or self.compress)
            yield ("copy",)
            if pools:
                for b in blocks:
                    yield ("write_mean", head, tensor, b)
                if self.plant != "no_arrival":
                    yield ("arrive", head)
            return
        # score item
        yield ("wait", head)
        yield ("passed", head)
        for tensor in range(3 if self.compress else 2):
            for b in range(self.NB):
                yield ("read_mean", head, tensor, b)
        last = self.nB - 1 if self.plant != "first_resets" else 0
        yield ("finish", head, last)

    def step(self, op):
        kind = op[0]
        if kind == "write_mean":
            self.means.add(op[1:])
        elif kind == "arrive":
            self.arrive[op[1]] += 1
        elif kind == "passed":
            self.passed[op[1]] += 1
        elif kind == "read_mean":
            if op[1:] not in self.means:
                raise Hazard(f"score item of head {op[1]} reads mean {op[2:]} before it is written")
        elif kind == "finish":
            _, h, last = op
            d = self.done[h]
            self.done[h] += 1
            if d == last:
                if self.passed[h] < self.nB:
                    raise Hazard(f"head {h}: counters reset with {self.nB - self.passed[h]} score items still to wait")
                self.arrive[h] = 0
                self.done[h] = 0

    def ready(self, op):
        return op[0] != "wait" or self.arrive[op[1]] >= self.target

    def run(self):
        seen = {}
        for L in range(self.grid):
            key = decode(L, self.NB, self.BH, self.BS, self.select, self.compress)
            assert key not in seen, f"grid index {L} decodes to {key}, as does {seen[key]}"
            seen[key] = L
        n_tiles = self.BH * 3 * self.nT
        assert len(seen) == n_tiles + self.BH * self.nB
        pending = self.items()
        resident = {}
        while pending or resident:
            while pending and len(resident) < self.slots:
                L = pending.pop(0)
                gen = self.cta(L)
                resident[L] = [gen, next(gen, None)]
            runnable = [L for L, (g, op) in resident.items() if op is not None and self.ready(op)]
            finished = [L for L, (g, op) in resident.items() if op is None]
            for L in finished:
                del resident[L]
            if finished:
                continue
            if not runnable:
                raise Deadlock(f"resident CTAs all wait: {sorted(resident)}")
            L = self.rng.choice(runnable)
            gen, op = resident[L]
            self.step(op)
            resident[L][1] = next(gen, None)
        if any(self.arrive) or any(self.done):
            raise Hazard(f"workspace not zero after the launch: {self.arrive} {self.done}")


CASES = [
    # NB, heads, block tokens, select, compress
    (8, 2, 256, True, False),      # tiny: one score item per head
    (120, 3, 256, True, False),    # fastwan-like: 15 score items per head
    (264, 3, 64, True, False),     # tile-64: four blocks per tile item
    (7, 2, 64, True, True),        # a partial last tile item, compression branch
    (14, 3, 64, False, True),      # compression branch alone
    (30, 2, 256, False, False),    # tiles only
]


@pytest.mark.parametrize("case", CASES, ids=[f"NB{c[0]}-H{c[1]}-bs{c[2]}-s{int(c[3])}-c{int(c[4])}" for c in CASES])
@pytest.mark.parametrize("slots", [1, 3, 16])
def test_front_protocol_has_no_deadlock_or_hazard(case, slots):
    for seed in range(6):
        FrontModel(*case, slots=slots, seed=seed).run()


@pytest.mark.parametrize("plant", ["scores_first", "first_resets", "no_arrival"])
def test_front_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(10):
        for case in CASES[:4]:
            try:
                FrontModel(*case, slots=3, seed=seed, plant=plant).run()
            except (Deadlock, Hazard):
                caught += 1
    assert caught > 0, plant
