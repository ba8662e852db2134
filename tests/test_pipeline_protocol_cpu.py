"""CPU model of the NVFP4 GEMM's barrier protocol (no GPU).

The kernel's roles, reduced to their mbarrier traffic: per CTA of the pair a
producer (code-stage ring of RS slots), sixteen expand/epilogue warps (FP16
operand ring of FS slots, two K steps per pass, the previous tile's epilogue
after the next tile's first FS K steps) and, in the leader, the MMA thread
(two accumulators).  Barriers follow mbarrier parity semantics: a phase
completes when its expected arrivals are in; a wait on parity P returns once
the phase of that parity has completed.

Random interleavings must finish (no deadlock) without a consumer ever
reading a slot that holds the wrong K step or an accumulator that the
epilogue has not drained; planted protocol mistakes must be caught.
"""
import random

import pytest

FS, RS, SUB, XW = 4, 3, 2, 16


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


def run(num_tiles, K, seed, mutation=None):
    rnd = random.Random(seed)
    KB, KRN = K // 64, (K + 127) // 128
    bars = {}
    for cta in range(2):
        for s in range(FS):
            bars[cta, "full", s] = Bar(2 * XW)
            bars[cta, "empty", s] = Bar(1)
        for r in range(RS):
            bars[cta, "rfull", r] = Bar(1)
            bars[cta, "rempty", r] = Bar(XW)
        for b in range(2):
            bars[cta, "tfull", b] = Bar(1)
            bars[cta, "tempty", b] = Bar(2 * XW)
    slot = {}                    # what each ring slot holds
    acc_tile = {0: None, 1: None}
    drained = {}                 # tile -> warps that drained its accumulator

    def wait(key, parity):
        while not bars[key].done(parity):
            yield

    def producer(cta):
        ir = 0
        for t in range(num_tiles):
            for kr in range(KRN):
                s = ir % RS
                yield from wait((cta, "rempty", s), ((ir // RS) & 1) ^ 1)
                slot[cta, "code", s] = (t, kr)
                bars[cta, "rfull", s].arrive()
                ir += 1

    def mma():
        it = 0
        for tl in range(num_tiles):
            ab = tl & 1 if mutation != "one_accumulator_index" else 0
            use = tl >> 1
            parity = (use & 1) ^ 1 if mutation != "tempty_parity" else use & 1
            yield from wait((0, "tempty", ab), parity)
            prev = acc_tile[ab]
            assert prev is None or drained.get(prev, 0) == 2 * XW, "accumulator overwritten before drained"
            acc_tile[ab] = tl
            for kb in range(KB):
                s = it % FS
                yield from wait((0, "full", s), (it // FS) & 1)
                for cta in range(2):
                    assert slot[cta, "fp16", s] == (tl, kb), "MMA read a slot holding another K step"
                yield                                   # the MMAs run; their commit comes later
                for cta in range(2):
                    assert slot[cta, "fp16", s] == (tl, kb), "slot overwritten while its MMAs ran"
                for cta in range(2):
                    bars[cta, "empty", s].arrive()
                it += 1
            for cta in range(2):
                bars[cta, "tfull", ab].arrive()

    def expander(cta):
        it = ir = tl_done = 0
        pending = None

        def epilogue(tile):
            nonlocal tl_done
            ab = tl_done & 1
            yield from wait((cta, "tfull", ab), (tl_done >> 1) & 1)
            assert acc_tile[ab] == tile, "epilogue drained another tile's accumulator"
            yield
            drained[tile] = drained.get(tile, 0) + 1
            bars[0, "tempty", ab].arrive()
            tl_done += 1

        for t in range(num_tiles):
            kb = 0
            while kb < KB:
                trigger = FS if mutation != "late_epilogue_never" else KB + 1
                if pending is not None and kb == trigger:
                    yield from epilogue(pending)
                    pending = None
                ns = 2 if kb + 1 < KB else 1
                j0 = kb % SUB
                rs = ir % RS
                s0, s1 = it % FS, (it + 1) % FS
                if j0 == 0:
                    yield from wait((cta, "rfull", rs), (ir // RS) & 1)
                yield from wait((cta, "empty", s0), ((it // FS) & 1) ^ 1)
                if ns == 2 and mutation != "skip_second_empty_wait":
                    yield from wait((cta, "empty", s1), (((it + 1) // FS) & 1) ^ 1)
                assert slot[cta, "code", rs] == (t, kb // SUB), "expanded a code stage not yet loaded"
                for q, s in enumerate((s0, s1)[:ns]):
                    slot[cta, "fp16", s] = (t, kb + q)
                for s in (s0, s1)[:ns]:
                    bars[0, "full", s].arrive()
                if j0 + ns == SUB or kb + ns == KB:
                    if mutation != "no_code_release_at_odd_end" or kb + ns != KB or j0 + ns == SUB:
                        bars[cta, "rempty", rs].arrive()
                    ir += 1
                kb += ns
                it += ns
            if pending is not None:
                yield from epilogue(pending)
                pending = None
            pending = t
        if pending is not None:
            yield from epilogue(pending)

    roles = [producer(0), producer(1), mma()] + [expander(c) for c in range(2) for _ in range(XW)]
    live, idle, last = roles, 0, None
    while live:
        rnd.shuffle(live)
        nxt = []
        for r in live:
            try:
                next(r)
                nxt.append(r)
            except StopIteration:
                pass
        state = tuple(sorted((str(k), b.phases, b.pending) for k, b in bars.items()))
        idle = idle + 1 if (state == last and len(nxt) == len(live)) else 0
        if idle > 200:
            raise Deadlock(f"tiles={num_tiles} K={K}")
        last, live = state, nxt


@pytest.mark.parametrize("K", [64, 128, 192, 320, 1088, 5120])
@pytest.mark.parametrize("tiles", [1, 2, 3, 5])
def test_protocol_completes_and_hands_off_the_right_buffers(K, tiles):
    for seed in range(2):
        run(tiles, K, seed)


@pytest.mark.parametrize("mutation,K,tiles", [
    ("tempty_parity", 128, 3),               # MMA waits for the wrong accumulator phase
    ("one_accumulator_index", 320, 3),       # epilogue and MMA disagree on the buffer
    ("skip_second_empty_wait", 512, 3),      # second slot of a pass overwritten while read
    ("no_code_release_at_odd_end", 320, 4),  # code stage never released at an odd K end
])
def test_planted_mistakes_are_caught(mutation, K, tiles):
    with pytest.raises((AssertionError, Deadlock)):
        for seed in range(4):
            run(tiles, K, seed, mutation)


def test_epilogue_at_tile_end_is_also_safe():
    """With two accumulators, draining a tile only after the next tile's
    last K step is still deadlock-free (the model checks safety, not
    speed): the early epilogue is an overlap choice, not a requirement."""
    for seed in range(2):
        run(4, 512, seed, "late_epilogue_never")
