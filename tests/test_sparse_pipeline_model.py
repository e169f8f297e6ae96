"""Host-side model of the barrier protocol of the 2:4-sparse layer's pair kernel with
resident metadata (w4a4_sparse.cu, K up to 2048), checked under random interleavings.

Roles: the TMA producer walks the pair's tiles (weight-major runs, so the weight tile
changes only a few times); when it changes, it waits for the metadata buffer's empty
barrier and loads the whole reduction's metadata of the new weight tile into shared
memory (the metadata full barrier counts it), then fills the operand ring stage by
stage. The MMA issuer takes each tile into one of two accumulators (after that
accumulator's empty barrier); on a weight-tile change it waits for the previous tile's
accumulator barrier and for the metadata, issues the copy of the metadata into TMEM and
commits the metadata buffer's empty barrier, then issues one MMA per stage and commits
the stage's empty barrier and, last, the accumulator's full barrier. The tensor pipe
runs the copies, MMAs and commits in issue order. The epilogue waits for each tile's
accumulator, reads it and arrives on its empty barrier. TMA loads in flight land in any
order. Barriers follow mbarrier phase semantics (a wait on parity P returns once the
completed-phase count has parity != P).

Every MMA must read its own stage and its weight tile's metadata, the epilogue must read
complete accumulators, and no buffer may be refilled before its reader is done. The
model must also catch the protocol with the metadata buffer's empty wait or the
accumulator's empty wait left out. (With the pipe in issue order, the issuer's wait for
the previous tile's accumulator before the metadata copy is a second guard: the model
finds no fault without it. The kernel keeps it so that the copy never overtakes an
earlier MMA that still reads the metadata columns, whatever the pipe's ordering.)"""
import random

import pytest

STAGES = 4


class Bar:
    def __init__(self, count=1):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def try_wait(self, parity):
        return (self.phase & 1) != parity


def simulate(tiles, nk, seed, skip_meta_empty=False, skip_acc_empty=False):
    """tiles: the pair's walk, a list of weight-tile ids. Returns (finished, problems)."""
    rnd = random.Random(seed)
    full = [Bar() for _ in range(STAGES)]
    empty = [Bar() for _ in range(STAGES)]
    tfull, tempty = [Bar(), Bar()], [Bar(), Bar()]
    mfull, mempty = Bar(), Bar()
    smem = [None] * STAGES          # operand stage contents: (local tile, k block)
    smeta = None                     # metadata buffer in shared memory: weight tile id
    tmeta = None                     # metadata columns in TMEM
    acc = [None, None]               # accumulator: (local tile, k blocks accumulated, read?)
    inflight, pipe, problems = [], [], []
    prod = {"t": 0, "kb": 0, "stage": 0, "phase": 0, "mphase": 0, "cur": None, "meta_done": False}
    mma = {"t": 0, "kb": -1, "stage": 0, "phase": 0, "mphase": 0, "cur": None}
    epi = {"t": 0}

    def producer():
        t = prod["t"]
        if t == len(tiles):
            return False
        if tiles[t] != prod["cur"] and not prod["meta_done"]:
            if not skip_meta_empty and not mempty.try_wait(prod["mphase"] ^ 1):
                return False
            inflight.append(("meta", tiles[t]))
            prod["mphase"] ^= 1
            prod["meta_done"] = True
            return True
        if not empty[prod["stage"]].try_wait(prod["phase"] ^ 1):
            return False
        inflight.append(("stage", prod["stage"], (t, prod["kb"])))
        prod["stage"] += 1
        if prod["stage"] == STAGES:
            prod["stage"], prod["phase"] = 0, prod["phase"] ^ 1
        prod["kb"] += 1
        if prod["kb"] == nk:
            prod["kb"], prod["cur"], prod["meta_done"] = 0, tiles[t], False
            prod["t"] += 1
        return True

    def tma_lands():
        nonlocal smeta
        if not inflight:
            return False
        op = inflight.pop(rnd.randrange(len(inflight)))
        if op[0] == "meta":
            if smeta is not None and ("cp", smeta) in [(p[0], p[1]) for p in pipe]:
                problems.append("metadata buffer refilled before its copy into TMEM")
            smeta = op[1]
            mfull.arrive()
        else:
            _, st, what = op
            if smem[st] is not None:
                problems.append("operand stage refilled before its MMA")
            smem[st] = what
            full[st].arrive()
        return True

    def mma_issue():
        t = mma["t"]
        if t == len(tiles):
            return False
        buf, bph = t & 1, (t >> 1) & 1
        if mma["kb"] == -1:   # tile start: accumulator, then metadata on a weight-tile change
            if not skip_acc_empty and not tempty[buf].try_wait(bph ^ 1):
                return False
            if tiles[t] != mma["cur"]:
                if mma["cur"] is not None:
                    pb, pph = (t - 1) & 1, ((t - 1) >> 1) & 1
                    if not tfull[pb].try_wait(pph):
                        return False
                if not mfull.try_wait(mma["mphase"]):
                    return False
                pipe.append(("cp", tiles[t]))
                pipe.append(("commit", mempty))
                mma["mphase"] ^= 1
                mma["cur"] = tiles[t]
            pipe.append(("start", buf, t))
            mma["kb"] = 0
            return True
        if not full[mma["stage"]].try_wait(mma["phase"]):
            return False
        pipe.append(("mma", mma["stage"], (t, mma["kb"]), tiles[t], buf))
        pipe.append(("commit", empty[mma["stage"]]))
        mma["stage"] += 1
        if mma["stage"] == STAGES:
            mma["stage"], mma["phase"] = 0, mma["phase"] ^ 1
        mma["kb"] += 1
        if mma["kb"] == nk:
            pipe.append(("commit", tfull[buf]))
            mma["kb"] = -1
            mma["t"] += 1
        return True

    def pipe_runs():   # the tensor pipe, in issue order
        nonlocal tmeta
        if not pipe:
            return False
        op = pipe.pop(0)
        if op[0] == "cp":
            if smeta != op[1]:
                problems.append(f"metadata copy read {smeta} for weight tile {op[1]}")
            tmeta = smeta
        elif op[0] == "start":
            _, buf, t = op
            if acc[buf] is not None and not acc[buf][2]:
                problems.append(f"accumulator {buf} overwritten before the epilogue read tile {acc[buf][0]}")
            acc[buf] = [t, 0, False]
        elif op[0] == "mma":
            _, st, what, wt, buf = op
            if smem[st] != what:
                problems.append(f"MMA read stage {smem[st]} for {what}")
            if tmeta != wt:
                problems.append(f"MMA used metadata of weight tile {tmeta} for {wt}")
            if acc[buf][0] != what[0]:
                problems.append("MMA into another tile's accumulator")
            acc[buf][1] += 1
            smem[st] = None
        else:
            op[1].arrive()
        return True

    def epilogue():
        t = epi["t"]
        if t == len(tiles):
            return False
        buf, bph = t & 1, (t >> 1) & 1
        if not tfull[buf].try_wait(bph):
            return False
        if acc[buf] is None or acc[buf][0] != t or acc[buf][1] != nk:
            problems.append(f"epilogue read {acc[buf]} for tile {t}")
        else:
            acc[buf][2] = True
        tempty[buf].arrive()
        epi["t"] += 1
        return True

    roles = [producer, tma_lands, mma_issue, pipe_runs, epilogue]
    bias = [rnd.random() + 0.05 for _ in roles]
    while not problems:
        for r in sorted(range(len(roles)), key=lambda r: -bias[r] * rnd.random()):
            if roles[r]():
                break
        else:
            break
    finished = prod["t"] == len(tiles) and mma["t"] == len(tiles) and epi["t"] == len(tiles) and not pipe
    return finished, problems


WALKS = [[0], [0, 0, 0], [0, 1], [0, 0, 1, 1, 1], [3, 3, 4], [0, 1, 2, 3], [5] * 7 + [6] * 6]


@pytest.mark.parametrize("tiles", WALKS)
@pytest.mark.parametrize("nk", [1, 2, 5, 16])
def test_resident_metadata_protocol_delivers(tiles, nk):
    for seed in range(10):
        finished, problems = simulate(tiles, nk, seed)
        assert not problems, (tiles, nk, seed, problems[:2])
        assert finished, f"deadlock: {tiles}, {nk} k blocks, seed {seed}"


def test_missing_metadata_empty_wait_is_caught():
    bad = 0
    for tiles in ([0, 1, 2], [0, 1, 2, 3]):
        for nk in (1, 2, 5):
            for seed in range(20):
                finished, problems = simulate(tiles, nk, seed, skip_meta_empty=True)
                bad += bool(problems) or not finished
    assert bad > 0


def test_missing_accumulator_empty_wait_is_caught():
    bad = 0
    for tiles in ([0, 0, 0, 0], [0, 0, 1, 1, 1]):
        for nk in (1, 2):
            for seed in range(20):
                finished, problems = simulate(tiles, nk, seed, skip_acc_empty=True)
                bad += bool(problems) or not finished
    assert bad > 0
