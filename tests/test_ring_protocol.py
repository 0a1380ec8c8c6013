"""Event-level model of the accept-statistics ring (CPU only).

The statistics kernel streams rows through a ring of shared-memory slots:
producer lanes issue bulk copies whose completion is counted on a "full"
mbarrier per slot, groups of consumer warps read a copy and arrive on the
slot's "empty" mbarrier.  Waits are parity waits, which cannot tell a
phase from the one two before it.  The kernel's rule against that: the
slot count is a multiple of the number of consumer groups, so every use of
a slot goes to one group, in order.

This model runs the producer and consumer steps of the kernel (constants
read from csrc/accept.cu) under random interleavings with copies that land
out of order, with the mbarrier semantics written out: a phase completes
when its arrivals and transaction bytes are all in; a parity wait succeeds
when the barrier's current phase has the other parity.  It checks that
every consumer reads exactly the copy meant for it, that no phase receives
more arrivals than it expects, and that everything terminates.  A negative
control (one warp per production, slots not owned) must be caught.
"""

import math
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(__file__), "..",
                   "introspective_strided_decoding_b200", "csrc", "accept.cu")


def _constants():
    text = open(SRC).read()
    names = ("kSub", "kCopyBytes", "kSlots", "kGroups", "kGroupWarps",
             "kIssuers")
    out = {}
    for n in names:
        m = re.search(r"constexpr int %s = ([0-9 *]+);" % n, text)
        assert m, n
        out[n] = math.prod(int(f) for f in m.group(1).split("*"))
    return out


class Bar:
    """mbarrier: expected arrivals per phase, pending transaction bytes."""

    def __init__(self, expected):
        self.expected, self.arrived, self.tx, self.phases = expected, 0, 0, 0

    def arrive(self, tx=0):
        self.arrived += 1
        self.tx += tx
        assert self.arrived <= self.expected, "phase got an extra arrival"
        self._complete()

    def land(self, tx):
        self.tx -= tx
        assert self.tx >= 0
        self._complete()

    def _complete(self):
        if self.arrived == self.expected and self.tx == 0:
            self.phases += 1
            self.arrived = 0

    def try_wait(self, parity):
        return (self.phases & 1) != parity


def simulate(copies_of_cta, slots, groups, group_warps, issuers, seed):
    """copies_of_cta: list of (copy id, sub-chunks in it) this CTA owns, in
    candidate order, None for a candidate whose row is unused."""
    rng = random.Random(seed)
    full = [Bar(1) for _ in range(slots)]
    empty = [Bar(group_warps) for _ in range(slots)]
    item = [None] * slots
    landed = [None] * slots
    in_flight = []
    seen = {}

    def wait(bar, parity):
        while not bar.try_wait(parity):
            yield

    def producer():
        q0 = 0
        for at in range(0, len(copies_of_cta), issuers):
            batch = copies_of_cta[at:at + issuers]
            lanes = []
            for cand in batch:
                if cand is not None:
                    lanes.append((q0, cand))
                    q0 += 1
            rng.shuffle(lanes)
            for q, cand in lanes:
                s = q % slots
                if q >= slots:
                    yield from wait(empty[s], (q // slots - 1) & 1)
                item[s] = (q, cand)
                full[s].arrive(tx=1)
                in_flight.append((s, q))
                yield
        for m in range(0, groups, issuers):
            marks = list(range(min(issuers, groups - m)))
            rng.shuffle(marks)
            for lane in marks:
                q = q0 + lane
                s = q % slots
                if q >= slots:
                    yield from wait(empty[s], (q // slots - 1) & 1)
                item[s] = (q, None)
                full[s].arrive()
                yield
            q0 += len(marks)

    def consumer(g, i):
        t = 0
        while True:
            q = g + t * groups
            s = q % slots
            yield from wait(full[s], (q // slots) & 1)
            assert item[s] is not None, f"group {g} read an unwritten slot"
            qq, cand = item[s]
            assert qq == q, f"group {g} wanted production {q}, got {qq}"
            if cand is not None and i < cand[1]:
                assert landed[s] == q, "read a slot before its copy landed"
                seen[(cand[0], i)] = seen.get((cand[0], i), 0) + 1
            yield
            empty[s].arrive()
            if cand is None:
                return
            t += 1

    procs = [producer()] + [consumer(g, i) for g in range(groups)
                            for i in range(group_warps)]
    alive = list(range(len(procs)))
    for _ in range(2_000_000):
        if not alive and not in_flight:
            break
        if in_flight and (not alive or rng.random() < 0.3):
            s, q = in_flight.pop(rng.randrange(len(in_flight)))
            landed[s] = q
            full[s].land(1)
            continue
        k = rng.choice(alive)
        try:
            next(procs[k])
        except StopIteration:
            alive.remove(k)
    else:
        raise AssertionError("no progress (deadlock)")
    want = {(c[0], i) for c in copies_of_cta if c is not None
            for i in range(c[1])}
    assert set(seen) == want and all(v == 1 for v in seen.values())


def cta_copies(B, RU, C, S, rows_of, grid, cta):
    """The kernel's decomposition: copies it = (b*RU + j)*CC + cc, CTA k
    takes k, k + grid, ...; a copy of an unused row is skipped."""
    CC = (C + S - 1) // S
    out = []
    for it in range(cta, B * RU * CC, grid):
        b, j, cc = it // (RU * CC), (it // CC) % RU, it % CC
        out.append((it, min(S, C - cc * S)) if j < rows_of(b) else None)
    return out


LAYOUTS = [
    # B, RU, C (sub-chunks per row), used rows of sequence b, grid
    (2, 7, 9, lambda b: 4 if b else 7, 3),   # S and R mode rows, ragged row
    (1, 3, 1, lambda b: 2, 3),               # tiny: one sub-chunk per row
    (2, 3, 128, lambda b: 2, 5),             # the largest vocabulary
]


@pytest.mark.parametrize("esize", [2, 4], ids=["bf16", "f32"])
@pytest.mark.parametrize("layout", range(len(LAYOUTS)))
def test_ring_protocol_of_the_kernel(esize, layout):
    k = _constants()
    S = k["kCopyBytes"] // (k["kSub"] * esize)
    assert k["kSlots"] % k["kGroups"] == 0 and S <= k["kGroupWarps"]
    B, RU, C, rows_of, grid = LAYOUTS[layout]
    for seed in range(2):
        for cta in range(min(grid, B * RU * ((C + S - 1) // S))):
            simulate(cta_copies(B, RU, C, S, rows_of, grid, cta),
                     k["kSlots"], k["kGroups"], k["kGroupWarps"],
                     k["kIssuers"], seed)


def test_model_catches_unowned_slots():
    # One warp per production, 31 consumers cycling over 24 slots: a warp
    # can wait on a slot whose previous use is another warp's and pending.
    copies = cta_copies(1, 3, 1, 1, lambda b: 2, 3, 0)
    with pytest.raises(AssertionError):
        simulate(copies, slots=24, groups=31, group_warps=1, issuers=16,
                 seed=0)
