"""The mbarrier protocol of the fused prefill kernel (fused_kernel in
csrc/sfa_prefill.cu), modelled on the CPU.

Each warp role is a generator that waits on barriers and arrives on them in
the kernel's order:

  * loads: the key/value span per KV head, the queries per head;
  * slot blocks: a warp of their own;
  * MMAs: for step j, QK(j), PV(j-1), POOL(j-2), with PV first where step j
    opens a new span;
  * band softmax: four warps, each finishing a tile after the first head of
    the next;
  * x epilogue: eight warps.

A barrier completes a phase when its count of arrivals is in.  A wait passes
as the hardware's parity wait does: when the barrier's completed-phase count
differs in parity from the phase waited for.  Random interleavings of the
roles must finish (no deadlock), and every wait must pass on exactly the
phase it means and never see a phase two ahead (parity aliasing).  Commits
and copies are modelled as completing at once; that only removes waits.
"""
import random

import pytest


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, log):
        self.pending += 1
        assert self.pending <= self.count, f"{self.name}: more arrivals than its count"
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1
        log.append(self.name)


def _run(nq, G, ntiles, first_tile, seed, sq_handshake=True):
    nsteps = ntiles * nq
    log = []
    bars = {}
    for name, count in [("kv_full", 1), ("kv_fix", 1), ("kv_empty", 1), ("p_full", 4), ("p_empty", 1),
                        ("x_full", 8), ("x_empty", 1), ("sc_full", 1), ("sc_empty", 4), ("sq_full", 8),
                        ("sq_empty", 4)]:
        bars[name] = _Bar(name, count)
    for b in (0, 1):
        for name, count in [("q_full", 1), ("q_empty", 1), ("sl_full", 1), ("sl_empty", 1), ("s_full", 1),
                            ("s_empty", 4), ("o_full", 1), ("o_empty", 8)]:
            bars[f"{name}{b}"] = _Bar(f"{name}{b}", count)
    arrive = lambda name: bars[name].arrive(log)
    wait = lambda name, phase: ("wait", name, phase)

    def loads():
        spans = 0
        for j in range(nsteps):
            h, ti, b = j % nq, j // nq, j & 1
            if h % G == 0:
                if spans > 0:
                    yield wait("kv_empty", spans - 1)
                arrive("kv_full")
                if first_tile and ti == 0:  # rows before the call patched in after the copy
                    yield wait("kv_full", spans)
                    arrive("kv_fix")
                spans += 1
            if j >= 2:
                yield wait(f"q_empty{b}", (j >> 1) - 1)
            arrive(f"q_full{b}")

    def slot_loads():
        for j in range(nsteps):
            b = j & 1
            if j >= 2:
                yield wait(f"sl_empty{b}", (j >> 1) - 1)
            arrive(f"sl_full{b}")

    def mmas():
        spans = [0]

        def qk(j):
            h, ti, b = j % nq, j // nq, j & 1
            if h % G == 0:
                yield wait("kv_full", spans[0])
                if first_tile and ti == 0:
                    yield wait("kv_fix", spans[0])
                spans[0] += 1
            yield wait(f"q_full{b}", j >> 1)
            if j >= 2:
                yield wait(f"s_empty{b}", (j >> 1) - 1)
            arrive(f"s_full{b}")
            arrive(f"q_empty{b}")

        def pv(j):
            h, b = j % nq, j & 1
            yield wait("p_full", j)
            if j >= 2:
                yield wait(f"o_empty{b}", (j >> 1) - 1)
            arrive(f"o_full{b}")
            arrive("p_empty")
            if h % G == G - 1 or j == nsteps - 1:
                arrive("kv_empty")

        def pool(j):
            h, ti, b = j % nq, j // nq, j & 1
            yield wait("x_full", j)
            yield wait(f"sl_full{b}", j >> 1)
            if h == 0 and ti >= 1:
                yield wait("sc_empty", ti - 1)
            arrive("x_empty")
            arrive(f"sl_empty{b}")
            if h == nq - 1:
                arrive("sc_full")

        for j in range(nsteps + 2):
            if j < nsteps and (j % nq) % G == 0:
                if j >= 1:
                    yield from pv(j - 1)
                yield from qk(j)
            else:
                if j < nsteps:
                    yield from qk(j)
                if 1 <= j <= nsteps:
                    yield from pv(j - 1)
            if j >= 2:
                yield from pool(j - 2)

    def softmax():
        def finish(ti):
            yield wait("sc_full", ti)
            yield wait("sq_full", ti)
            arrive("sc_empty")
            arrive("sq_empty")

        for j in range(nsteps):
            ti, b = j // nq, j & 1
            yield wait(f"s_full{b}", j >> 1)
            arrive(f"s_empty{b}")
            if j >= 1:
                yield wait("p_empty", j - 1)
            arrive("p_full")
            if j % nq == 0 and ti >= 1:
                yield from finish(ti - 1)
        yield from finish((nsteps - 1) // nq)

    def epilogue():
        for j in range(nsteps):
            h, ti, b = j % nq, j // nq, j & 1
            yield wait(f"o_full{b}", j >> 1)
            arrive(f"o_empty{b}")  # the accumulator is in registers
            if j >= 1:
                yield wait("x_empty", j - 1)
            arrive("x_full")
            if h == nq - 1:
                if ti >= 1 and sq_handshake:
                    yield wait("sq_empty", ti - 1)
                arrive("sq_full")
        yield wait("x_empty", nsteps - 1)

    roles = [loads(), slot_loads(), mmas()] + [softmax() for _ in range(4)] + [epilogue() for _ in range(8)]
    pending = [None] * len(roles)
    alive = set(range(len(roles)))
    rng = random.Random(seed)
    # each role gets its own speed: the chance of yielding the processor after
    # a step, so that some roles fall far behind others
    pause = [rng.choice((0.05, 0.3, 0.9)) for _ in roles]
    # and a chance of sitting out a whole sweep (a starved warp)
    skip = [rng.choice((0.0, 0.0, 0.5, 0.9)) for _ in roles]
    all_in = False  # a sweep that skips nobody (after one without progress)
    while alive:
        progress = 0  # waits passed, roles started or finished in this sweep
        order = sorted(alive)
        rng.shuffle(order)
        for r in order:
            if not all_in and rng.random() < skip[r]:
                continue
            while True:
                if pending[r] is not None:
                    _, name, phase = pending[r]
                    done = bars[name].done
                    if (done & 1) != (phase & 1):  # the hardware's parity wait passes
                        assert done == phase + 1, f"{name}: wait for phase {phase} passed at {done}"
                        pending[r] = None
                        progress += 1
                    else:
                        assert done == phase, f"{name}: waiting for phase {phase} with {done} done"
                        break
                try:
                    pending[r] = next(roles[r])
                    progress += 1
                except StopIteration:
                    alive.discard(r)
                    progress += 1
                    break
                if rng.random() < pause[r]:
                    break
        if progress == 0 and not all_in:
            all_in = True
            continue
        assert progress > 0, f"deadlock: {[pending[r] for r in sorted(alive)]}"
        all_in = False
    return log


@pytest.mark.parametrize("nq,G", [(1, 1), (2, 1), (2, 2), (4, 2), (4, 4), (14, 7), (28, 7), (6, 3)])
@pytest.mark.parametrize("ntiles", [1, 2, 5])
@pytest.mark.parametrize("first_tile", [False, True])
def test_fused_prefill_protocol_has_no_deadlock_or_parity_aliasing(nq, G, ntiles, first_tile):
    for seed in range(8):
        log = _run(nq, G, ntiles, first_tile, seed)
        nsteps = ntiles * nq
        assert log.count("sc_full") == ntiles and log.count("x_full") == 8 * nsteps


def test_the_model_catches_a_missing_release():
    """A planted mistake (the epilogue never releases its accumulator) must be
    reported as a deadlock, not pass silently."""

    def run_without_release(*args):
        saved = _Bar.arrive

        def arrive(self, log):
            if self.name.startswith("o_empty"):
                log.append(self.name)
                return
            saved(self, log)
        _Bar.arrive = arrive
        try:
            return _run(*args)
        finally:
            _Bar.arrive = saved

    with pytest.raises(AssertionError, match="deadlock|waiting"):
        run_without_release(4, 2, 3, False, 0)


def test_the_model_catches_parity_aliasing():
    """Without the epilogue's wait for the tile finish to take |x|^2 (sq_empty),
    one head per tile lets the epilogue complete the |x|^2 barrier twice
    before the softmax warps wait for the first phase: the model must report
    the aliased wait (or the deadlock it causes)."""
    with pytest.raises(AssertionError, match="deadlock|waiting|passed"):
        for seed in range(50):
            _run(1, 1, 4, False, seed, sq_handshake=False)
