"""CPU model of the block-scaled GEMM's barrier protocol on CTA pairs (no
GPU).

The kernel's roles, reduced to their mbarrier traffic:
  * per CTA, a TMA producer filling a ring of STAGES stages -- the A and B
    tiles and their scale atoms -- that land on the leader CTA's full
    barrier and are freed by the MMA commit on empty (sent to both CTAs);
  * in the leader, the scale-copy thread: once stage s has landed it copies
    the stage's scales (both CTAs' shared memory) into TMEM scale columns of
    its own for stage s and commits sf_full[s];
  * the leader's MMA thread: waits full[s] and sf_full[s], issues the stage's
    MMAs and commits empty[s]; after the tile it commits tfull;
  * one tensor pipe that runs the copies and MMAs in the order they were
    issued, whichever thread issued them; a commit arrives once everything
    its thread issued before it has run;
  * per CTA the epilogue (one accumulator, drained before the next tile's
    MMAs start; both CTAs' epilogues arrive on the leader's tempty).
Barriers follow mbarrier parity semantics: a phase completes when its
expected arrivals are in; a wait on parity P returns once the phase of that
parity has completed -- so a waiter two phases behind waits forever, which
the model reports as a deadlock.

Random interleavings must finish without a copy reading scales of another
K step, a TMEM scale column being overwritten before the MMAs that read it
ran, the MMA reading an operand stage or scale column that holds another K
step, a stage being reloaded while it is read, or the accumulator being
reused before it is drained; planted protocol mistakes must be caught.  The
ring depth is that of the E4M3 mode (6 stages) and of the NVFP4 mode (5
stages, the same barriers with four times the scale copies per stage).
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phases = count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count, "more arrivals than the phase expects"
        if self.pending == self.count:
            self.pending, self.phases = 0, self.phases + 1

    def done(self, parity):
        return (self.phases & 1) != parity


class Deadlock(Exception):
    pass


def run(num_tiles, KB, seed, mutation=None, STAGES=6):
    rnd = random.Random(seed)
    bars = {}
    for cta in range(2):
        for s in range(STAGES):
            bars[cta, "full", s] = Bar(2)
            bars[cta, "empty", s] = Bar(1)
            bars[cta, "sf_full", s] = Bar(1)
        bars[cta, "tfull"] = Bar(1)
        bars[cta, "tempty"] = Bar(2)
    smem = {}                    # (cta, stage) -> (tile, k step) of the A, B and scale tiles there
    tcol = {}                    # TMEM scale columns of a stage -> (tile, k step, consumed)
    reading = set()              # stages being read by the tensor pipe right now
    acc = {"tile": None, "drained": True}
    pipe = []                    # issued tensor-pipe work, executed in issue order
    issued = {"copy": 0, "mma": 0}
    ran = {"copy": 0, "mma": 0}

    def wait(key, parity):
        while not bars[key].done(parity):
            yield

    def steps():
        for t in range(num_tiles):
            for kb in range(KB):
                yield t, kb

    def commit(thread, targets):
        """tcgen05.commit: arrive on the targets once everything the thread
        has issued so far has run."""
        pipe.append(("commit", thread, issued[thread], targets))

    def producer(cta):
        for it, (t, kb) in enumerate(steps()):
            s = it % STAGES
            yield from wait((cta, "empty", s), ((it // STAGES) & 1) ^ 1)
            assert (cta, s) not in reading, "stage reloaded while read"
            smem.pop((cta, s), None)
            for _ in range(rnd.randint(1, 4)):
                yield
            smem[cta, s] = (t, kb)
            bars[0, "full", s].arrive()

    def copier():
        for it, (t, kb) in enumerate(steps()):
            s = it % STAGES
            if mutation != "copy_skips_full":
                yield from wait((0, "full", s), (it // STAGES) & 1)
            for _ in range(rnd.randint(0, 2)):
                yield
            pipe.append(("copy", t, kb, s))
            issued["copy"] += 1
            commit("copy", [(0, "sf_full", s)])

    def mma():
        it = 0
        for tl in range(num_tiles):
            parity = (tl & 1) ^ 1 if mutation != "tempty_parity" else tl & 1
            yield from wait((0, "tempty"), parity)
            assert acc["drained"], "accumulator overwritten before drained"
            acc["tile"], acc["drained"] = tl, False
            for kb in range(KB):
                s = it % STAGES
                ph = (it // STAGES) & 1
                yield from wait((0, "full", s), ph)
                if mutation != "mma_skips_sf_full":
                    yield from wait((0, "sf_full", s), ph)
                pipe.append(("mma", tl, kb, s))
                issued["mma"] += 1
                if mutation == "empty_at_issue":
                    for c in range(2):
                        bars[c, "empty", s].arrive()
                else:
                    commit("mma", [(c, "empty", s) for c in range(2)])
                it += 1
            commit("mma", [(c, "tfull") for c in range(2)])

    def tensor_pipe():
        total = num_tiles * KB * 4 + num_tiles
        done = 0
        while done < total:
            if not pipe:
                yield
                continue
            item = pipe[0]
            if item[0] == "copy":
                _, t, kb, s = item
                for c in range(2):
                    assert smem.get((c, s)) == (t, kb), "copied scales of another K step"
                old = tcol.get(s)
                assert old is None or old[2], "TMEM scale columns overwritten before their MMAs ran"
                reading.update({(0, s), (1, s)})
                for _ in range(rnd.randint(1, 3)):
                    yield
                reading.difference_update({(0, s), (1, s)})
                tcol[s] = (t, kb, False)
                ran["copy"] += 1
            elif item[0] == "mma":
                _, tl, kb, s = item
                for c in range(2):
                    assert smem.get((c, s)) == (tl, kb), "MMA read a stage holding another K step"
                col = tcol.get(s)
                assert col is not None and col[:2] == (tl, kb), "MMA read scale columns of another K step"
                assert acc["tile"] == tl, "MMA accumulated into another tile"
                reading.update({(0, s), (1, s)})
                for _ in range(rnd.randint(1, 6)):
                    yield
                reading.difference_update({(0, s), (1, s)})
                tcol[s] = (tl, kb, True)
                ran["mma"] += 1
            else:
                _, thread, upto, targets = item
                while ran[thread] < upto:    # cannot happen in one in-order pipe; kept as a guard
                    yield
                for key in targets:
                    bars[key].arrive()
            pipe.pop(0)
            done += 1

    def epilogue(cta):
        for tl in range(num_tiles):
            yield from wait((cta, "tfull"), tl & 1)
            assert acc["tile"] == tl, "epilogue drained another tile"
            for _ in range(rnd.randint(1, 3)):
                yield
            bars[0, "tempty"].arrive()
            if bars[0, "tempty"].pending == 0:
                acc["drained"] = True

    roles = [producer(0), producer(1), copier(), mma(), tensor_pipe(), epilogue(0), epilogue(1)]
    live, idle, last = roles, 0, None
    while live:
        rnd.shuffle(live)
        nxt = []
        for role in live:
            try:
                next(role)
                nxt.append(role)
            except StopIteration:
                pass
        state = tuple(sorted((str(k), b.phases, b.pending) for k, b in bars.items())) + (len(pipe),)
        idle = idle + 1 if (state == last and len(nxt) == len(live)) else 0
        if idle > 200:
            raise Deadlock(f"tiles={num_tiles} KB={KB}")
        last, live = state, nxt


@pytest.mark.parametrize("stages", [6, 5])
@pytest.mark.parametrize("KB", [1, 2, 5, 7, 11, 40])
@pytest.mark.parametrize("tiles", [1, 2, 3, 5])
def test_protocol_completes_and_hands_off_the_right_buffers(KB, tiles, stages):
    for seed in range(3):
        run(tiles, KB, seed, STAGES=stages)


@pytest.mark.parametrize("mutation,KB,tiles", [
    ("copy_skips_full", 40, 2),        # scales copied before the stage has landed
    ("mma_skips_sf_full", 40, 2),      # MMA issued before its stage's scales reached TMEM
    ("empty_at_issue", 40, 2),         # stage freed when its MMAs are issued, not when they ran
    ("tempty_parity", 8, 4),           # MMA waits for the wrong accumulator phase
])
def test_planted_mistakes_are_caught(mutation, KB, tiles):
    with pytest.raises((AssertionError, Deadlock)):
        for seed in range(32):
            run(tiles, KB, seed, mutation)
