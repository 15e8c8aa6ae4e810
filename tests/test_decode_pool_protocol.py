"""The mbarrier and cluster-barrier protocol of the batched decode's pool
kernel (decode_pool_kernel in csrc/sfa_decode_tile.cu), modelled on the CPU.

A cluster of two CTAs serves 16 sequences. CTA rank 0 owns the first
ceil(chunks / 2) 64-column chunks of the hidden size, rank 1 the rest (which
can be none). Per CTA:

  * the MMA lane: slot-block loads four deep, then
    - pass 1: the score MMAs of every chunk;
    - the two cluster-barrier phases;
    - pass 2: the sem MMAs of every chunk;
  * eight compute warps:
    - pass 1: split x into the x^T ring;
    - the partial exchange between the two cluster phases, then the weights;
    - pass 2: warps 0-3 move each sem chunk from tensor memory into the
      staging ring, and all eight read it there.

Each role is a generator that waits and arrives in the kernel's order. A
wait passes as the hardware's parity wait does. Random interleavings of both
CTAs must finish, and every wait must pass on exactly the phase it means.
Copies and commits complete at once in the model; that only removes waits.
"""
import random

import pytest

SLOT_STAGES, A_BUFS, SEM_BUFS, WARPS = 4, 4, 4, 8


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count, f"{self.name}: more arrivals than its count"
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


def _cta(rank, nch, bars, cluster, st_handshake=True):
    half = (nch + 1) // 2
    nloc = half if rank == 0 else nch - half
    B = {}
    for name, count in [("scores", 1), ("w_full", WARPS)]:
        B[name] = bars[(rank, name)] = _Bar(f"{rank}.{name}", count)
    for i in range(SLOT_STAGES):
        for name in ("sl_full", "sl_empty"):
            B[(name, i)] = bars[(rank, name, i)] = _Bar(f"{rank}.{name}{i}", 1)
    for i in range(A_BUFS):
        B[("a_full", i)] = bars[(rank, "a_full", i)] = _Bar(f"{rank}.a_full{i}", WARPS)
        B[("a_empty", i)] = bars[(rank, "a_empty", i)] = _Bar(f"{rank}.a_empty{i}", 1)
    for i in range(SEM_BUFS):
        for name, count in [("sem_full", 1), ("sem_empty", 4), ("st_full", 4), ("st_empty", WARPS)]:
            B[(name, i)] = bars[(rank, name, i)] = _Bar(f"{rank}.{name}{i}", count)
    wait = lambda key, phase: ("wait", B[key], phase)
    cwait = lambda phase: ("wait", cluster, phase)

    def mma():
        cluster.arrive()
        for q in range(min(SLOT_STAGES, 2 * nloc)):  # slot blocks are constant: loaded up front
            B[("sl_full", q % SLOT_STAGES)].arrive()

        def refill(q):  # after load q's MMAs: load q-1's stage takes load q+3
            if q < 1 or q + SLOT_STAGES - 1 >= 2 * nloc:
                return
            yield wait(("sl_empty", (q - 1) % SLOT_STAGES), (q - 1) // SLOT_STAGES)
            B[("sl_full", (q + SLOT_STAGES - 1) % SLOT_STAGES)].arrive()

        for c in range(nloc):  # pass 1
            yield wait(("sl_full", c % SLOT_STAGES), c // SLOT_STAGES)
            yield wait(("a_full", c % A_BUFS), c // A_BUFS)
            B[("a_empty", c % A_BUFS)].arrive()
            B[("sl_empty", c % SLOT_STAGES)].arrive()
            yield from refill(c)
        B["scores"].arrive()
        yield cwait(0)
        cluster.arrive()
        yield cwait(1)
        yield wait("w_full", 0)
        for c in range(nloc):  # pass 2
            q = nloc + c
            yield wait(("sl_full", q % SLOT_STAGES), q // SLOT_STAGES)
            if c >= SEM_BUFS:
                yield wait(("sem_empty", c % SEM_BUFS), c // SEM_BUFS - 1)
            B[("sem_full", c % SEM_BUFS)].arrive()
            B[("sl_empty", q % SLOT_STAGES)].arrive()
            yield from refill(q)

    def compute(warp):
        cluster.arrive()
        for c in range(nloc):  # pass 1
            if c >= A_BUFS:
                yield wait(("a_empty", c % A_BUFS), c // A_BUFS - 1)
            B[("a_full", c % A_BUFS)].arrive()
        yield cwait(0)  # the peer has started: partials may be written into it
        if warp < 4:
            yield wait("scores", 0)
        cluster.arrive()
        yield cwait(1)
        B["w_full"].arrive()
        for c in range(nloc):  # pass 2
            b, ph = c % SEM_BUFS, c // SEM_BUFS
            if warp < 4:
                yield wait(("sem_full", b), ph)
                B[("sem_empty", b)].arrive()
                if c >= SEM_BUFS and st_handshake:
                    yield wait(("st_empty", b), ph - 1)
                B[("st_full", b)].arrive()
            yield wait(("st_full", b), ph)
            B[("st_empty", b)].arrive()

    return [mma()] + [compute(w) for w in range(WARPS)]


def _run(nch, seed, st_handshake=True):
    bars = {}
    cluster = _Bar("cluster", 2 * (WARPS + 1))  # every warp of both CTAs, per phase
    roles = _cta(0, nch, bars, cluster, st_handshake) + _cta(1, nch, bars, cluster, st_handshake)
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
        progress = 0
        order = sorted(alive)
        rng.shuffle(order)
        for r in order:
            if not all_in and rng.random() < skip[r]:
                continue
            while True:
                if pending[r] is not None:
                    _, bar, phase = pending[r]
                    if (bar.done & 1) != (phase & 1):  # the hardware's parity wait passes
                        assert bar.done == phase + 1, f"{bar.name}: wait for phase {phase} passed at {bar.done}"
                        pending[r] = None
                        progress += 1
                    else:
                        assert bar.done == phase, f"{bar.name}: waiting for phase {phase} with {bar.done} done"
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
        assert progress > 0, f"deadlock: {[(p[1].name, p[2]) for p in pending if p]}"
        all_in = False
    return bars, cluster


@pytest.mark.parametrize("nch", [1, 2, 3, 5, 8, 9, 14, 56])
def test_decode_pool_protocol_has_no_deadlock_or_parity_aliasing(nch):
    """nch 64-column chunks (hidden 64 .. 3,584); rank 1 has none at nch = 1."""
    for seed in range(12):
        bars, cluster = _run(nch, seed)
        assert cluster.done == 2
        for rank, nloc in ((0, (nch + 1) // 2), (1, nch - (nch + 1) // 2)):
            assert sum(bars[(rank, "sl_empty", i)].done for i in range(SLOT_STAGES)) == 2 * nloc
            assert sum(bars[(rank, "st_empty", i)].done for i in range(SEM_BUFS)) == nloc


def test_the_model_catches_a_missing_staging_handshake():
    """A planted mistake: warps 0-3 restage a sem chunk without waiting for
    every warp to have read the buffer's previous chunk (st_empty).  The
    staging barrier then runs ahead of its readers, and the model must report
    the aliased or early wait."""
    with pytest.raises(AssertionError, match="waiting|passed|more arrivals|deadlock"):
        for seed in range(50):
            _run(56, seed, st_handshake=False)
