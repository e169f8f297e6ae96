"""Host-side model of the barrier protocol of the grouped linear layer's kernel
(w4a4_grouped.cu), checked under random interleavings of its roles.

Roles: the TMA producer fills a ring of 6 operand stages; the MMA issuer takes a
CTA pair's output tiles two at a time and alternates between them group by group
(tile 2c group g, tile 2c+1 group g, ...), writing group products into four TMEM
slots, two per tile of the couple; two epilogue teams each read their own tile's
groups. Barriers are modelled with mbarrier phase semantics: a wait on parity P
returns once the barrier's completed-phase count has parity != P, so a waiter that
falls two phases behind sees a phase that has not completed as complete, or blocks
for ever.

The kernel's protocol (a full and an empty barrier per TMEM slot) must finish for
every tile and group count with each team reading exactly its own group from the
slot; the alternative of reading group completion off the operand stage's empty
barrier must be caught failing when a pair has an odd number of tiles (the lone
last tile's team runs ahead of the other by more than the ring), which is why the
kernel has slot barriers."""
import random

import pytest

STAGES, SLOTS = 6, 4


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def try_wait(self, parity):
        return (self.phase & 1) != parity


def simulate(ntl, G, seed, stage_signal=False):
    """Run the roles to completion or deadlock; returns (finished, problems)."""
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(STAGES)]
    empty = [Bar(1) for _ in range(STAGES)]
    tfull = [Bar(1) for _ in range(SLOTS)]
    tempty = [Bar(1) for _ in range(SLOTS)]
    order = []   # issue order: (local tile, group, team)
    for c in range((ntl + 1) // 2):
        nt = 2 if 2 * c + 1 < ntl else 1
        for g in range(G):
            for t in range(nt):
                order.append((2 * c + t, g, t))
    smem, tmem = [None] * STAGES, [None] * SLOTS
    loads, mmas, problems = [], [], []
    prod = {"i": 0, "stage": 0, "phase": 0}
    mma = {"i": 0, "stage": 0, "phase": 0, "gc": [0, 0]}
    teams = [{"t": t, "todo": [(i, g) for i in range(t, ntl, 2) for g in range(G)], "k": 0} for t in range(2)]

    def producer():
        if prod["i"] == len(order) or not empty[prod["stage"]].try_wait(prod["phase"] ^ 1):
            return False
        loads.append((prod["stage"], order[prod["i"]]))
        prod["i"] += 1
        prod["stage"] += 1
        if prod["stage"] == STAGES:
            prod["stage"], prod["phase"] = 0, prod["phase"] ^ 1
        return True

    def tma_lands():
        if not loads:
            return False
        st, what = loads.pop(0)
        if smem[st] is not None:
            problems.append("stage refilled before its MMA")
        smem[st] = what
        full[st].arrive()
        return True

    def mma_issue():
        if mma["i"] == len(order):
            return False
        tile, g, t = order[mma["i"]]
        gc = mma["gc"][t]
        slot = 2 * t + (gc & 1)
        if not tempty[slot].try_wait(((gc >> 1) & 1) ^ 1) or not full[mma["stage"]].try_wait(mma["phase"]):
            return False
        if smem[mma["stage"]] != (tile, g, t):
            problems.append("MMA read the wrong stage")
        mmas.append((mma["stage"], slot, (tile, g)))
        mma["gc"][t] = gc + 1
        mma["i"] += 1
        mma["stage"] += 1
        if mma["stage"] == STAGES:
            mma["stage"], mma["phase"] = 0, mma["phase"] ^ 1
        return True

    def mma_completes():   # in issue order, like tcgen05 commits
        if not mmas:
            return False
        st, slot, what = mmas.pop(0)
        smem[st], tmem[slot] = None, what
        empty[st].arrive()
        tfull[slot].arrive()
        return True

    def team_step(tm):
        if tm["k"] == len(tm["todo"]):
            return False
        i, g = tm["todo"][tm["k"]]
        c = i >> 1
        ga = G * c + g
        slot = 2 * tm["t"] + (ga & 1)
        if stage_signal:
            nt = 2 if 2 * c + 1 < ntl else 1
            seq = 2 * G * c + g * nt + tm["t"]
            ready = empty[seq % STAGES].try_wait((seq // STAGES) & 1)
        else:
            ready = tfull[slot].try_wait((ga >> 1) & 1)
        if not ready:
            return False
        if tmem[slot] != (i, g):
            problems.append(f"team {tm['t']} read {tmem[slot]} for {(i, g)}")
        tmem[slot] = None
        tempty[slot].arrive()
        tm["k"] += 1
        return True

    roles = [producer, tma_lands, mma_issue, mma_completes, lambda: team_step(teams[0]),
             lambda: team_step(teams[1])]
    bias = [rnd.random() + 0.05 for _ in roles]
    while not problems:
        for r in sorted(range(len(roles)), key=lambda r: -bias[r] * rnd.random()):
            if roles[r]():
                break
        else:
            break
    finished = prod["i"] == len(order) and mma["i"] == len(order) and all(
        tm["k"] == len(tm["todo"]) for tm in teams)
    return finished, problems


@pytest.mark.parametrize("ntl", [1, 2, 3, 4, 5, 38, 39])
@pytest.mark.parametrize("G", [1, 3, 5, 9, 16])
def test_slot_barriers_finish_and_deliver_each_group(ntl, G):
    for seed in range(12):
        finished, problems = simulate(ntl, G, seed)
        assert not problems, (ntl, G, seed, problems[:2])
        assert finished, f"deadlock: {ntl} tiles, {G} groups, seed {seed}"


def test_stage_barrier_signal_fails_with_an_odd_tile_count():
    bad = 0
    for ntl in (3, 5, 7):
        for G in (5, 8, 9):
            for seed in range(12):
                finished, problems = simulate(ntl, G, seed, stage_signal=True)
                bad += bool(problems) or not finished
    assert bad > 0
    # with an even tile count the teams stay in step and the stage signal is sound
    for seed in range(12):
        finished, problems = simulate(4, 8, seed, stage_signal=True)
        assert finished and not problems
