"""Host-side model of the barrier protocol of the grouped linear layer's kernel
(w4a4_grouped.cu), checked under random interleavings of its roles.

Roles: the TMA producer fills a ring of 5 operand stages, one per (tile, group),
each holding the tile's A rows and the B rows of both 128-column halves; the MMA
issuer takes each stage's two halves in turn, writing half h's group product into
one of team h's two TMEM slots (groups alternate between them), and frees the stage
after the second half; two epilogue teams each read their own half of every tile,
group by group. Barriers are modelled with mbarrier phase semantics: a wait on
parity P returns once the barrier's completed-phase count has parity != P, so a
waiter that falls two phases behind sees a phase that has not completed as
complete, or blocks for ever.

The kernel's protocol (a full and an empty barrier per TMEM slot) must finish for
every tile and group count with each team reading exactly its own half of each
group from the slot. The model must also catch a broken protocol: an issuer that
does not wait for a slot's empty barrier overwrites products the team has not read."""
import random

import pytest

STAGES, SLOTS = 5, 4


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


def simulate(ntl, G, seed, skip_slot_wait=False):
    """Run the roles to completion or deadlock; returns (finished, problems)."""
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(STAGES)]
    empty = [Bar(1) for _ in range(STAGES)]
    tfull = [Bar(1) for _ in range(SLOTS)]
    tempty = [Bar(1) for _ in range(SLOTS)]
    order = [(i, g) for i in range(ntl) for g in range(G)]   # stage order: (local tile, group)
    smem, tmem = [None] * STAGES, [None] * SLOTS
    loads, mmas, problems = [], [], []
    prod = {"i": 0, "stage": 0, "phase": 0}
    mma = {"i": 0, "h": 0, "stage": 0, "phase": 0}
    teams = [{"t": t, "todo": list(order), "k": 0} for t in range(2)]

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
            problems.append("stage refilled before its MMAs")
        smem[st] = what
        full[st].arrive()
        return True

    def mma_issue():   # one half per step; the stage is freed after half 1
        if mma["i"] == len(order):
            return False
        gc, h = mma["i"], mma["h"]
        slot = 2 * h + (gc & 1)
        if not skip_slot_wait and not tempty[slot].try_wait(((gc >> 1) & 1) ^ 1):
            return False
        if not full[mma["stage"]].try_wait(mma["phase"]):
            return False
        if smem[mma["stage"]] != order[gc]:
            problems.append("MMA read the wrong stage")
        mmas.append((mma["stage"] if h == 1 else None, slot, order[gc] + (h,)))
        if h == 0:
            mma["h"] = 1
        else:
            mma["h"] = 0
            mma["i"] += 1
            mma["stage"] += 1
            if mma["stage"] == STAGES:
                mma["stage"], mma["phase"] = 0, mma["phase"] ^ 1
        return True

    def mma_completes():   # in issue order, like tcgen05 commits
        if not mmas:
            return False
        st, slot, what = mmas.pop(0)
        if st is not None:
            smem[st] = None
            empty[st].arrive()
        tmem[slot] = what
        tfull[slot].arrive()
        return True

    def team_step(tm):
        if tm["k"] == len(tm["todo"]):
            return False
        i, g = tm["todo"][tm["k"]]
        ga = G * i + g
        slot = 2 * tm["t"] + (ga & 1)
        if not tfull[slot].try_wait((ga >> 1) & 1):
            return False
        if tmem[slot] != (i, g, tm["t"]):
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


@pytest.mark.parametrize("ntl", [1, 2, 3, 4, 5, 19, 20])
@pytest.mark.parametrize("G", [1, 3, 5, 9, 16])
def test_slot_barriers_finish_and_deliver_each_group(ntl, G):
    for seed in range(12):
        finished, problems = simulate(ntl, G, seed)
        assert not problems, (ntl, G, seed, problems[:2])
        assert finished, f"deadlock: {ntl} tiles, {G} groups, seed {seed}"


def test_issuer_without_the_slot_wait_is_caught():
    bad = 0
    for ntl in (1, 3):
        for G in (5, 9):
            for seed in range(12):
                finished, problems = simulate(ntl, G, seed, skip_slot_wait=True)
                bad += bool(problems) or not finished
    assert bad > 0
