"""A model of the tensor-core prefill kernel's barrier protocol, on the CPU.

The kernel (csrc/prefill_tc.cu) runs three roles per CTA -- one copying
thread, one MMA-issuing thread, four softmax warps -- that hand tiles to each
other through mbarriers waited on by phase parity.  A parity wait is only
sound if the barrier cannot complete the phase after the awaited one before
the waiter looks: two completions ahead, the parity matches again and the
waiter blocks (or passes) on the wrong phase.  The kernel keeps this rule by
construction: the next completion of every barrier depends on its waiter's
own progress.

This test replays the kernel's sequence of waits, arrives and commits (the
same ring sizes, the same conditions) under random timing of every role and
of the asynchronous copies and MMAs, and checks that

* every unit completes (no deadlock), and
* at every wait the barrier has completed at most one phase past the
  awaited one.

A planted protocol mistake -- one "weights ready" barrier shared by all four
S buffers instead of one per buffer, which the kernel first had -- must be
caught.  The model covers the protocol only; the GPU parity tests cover the
arithmetic.
"""

import random

TILE = 32          # tokens per K/V tile
NS = 4             # copy ring stages
NB = 4             # S / P buffers in tensor memory


class Barrier:
    """An mbarrier: `count` arrivals (plus any expected bytes) complete a phase."""

    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.tx, self.done = name, count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        self._check()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def passed(self, phase):
        """Parity test for `phase` (0-based); records a violation if the barrier
        is two or more phases past it."""
        if self.done > phase + 1:
            raise AssertionError(f"{self.name}: waiter on phase {phase} but {self.done} phases completed")
        return self.done == phase + 1


class Sim:
    def __init__(self, seed, shared_p_full=False):
        self.rng = random.Random(seed)
        self.now = 0
        self.events = []          # (time, seq, fn)
        self.seq = 0
        self.mma_free_at = 0      # the tensor pipe runs the MMAs of the CTA in order
        nb_p = 1 if shared_p_full else NB
        self.full = [Barrier(f"full[{i}]") for i in range(NS)]
        self.empty = [Barrier(f"empty[{i}]") for i in range(NS)]
        self.s_bar = [Barrier(f"s_bar[{i}]") for i in range(NB)]
        self.buf_free = [Barrier(f"buf_free[{i}]") for i in range(NB)]
        self.p_full = [Barrier(f"p_full[{i}]") for i in range(nb_p)]

    def at(self, dt, fn):
        self.seq += 1
        self.events.append((self.now + dt, self.seq, fn))

    def copy(self, bar, nbytes):
        self.at(self.rng.randint(1, 60), lambda: bar.complete_tx(nbytes))

    def mma(self, cycles):
        self.mma_free_at = max(self.mma_free_at, self.now) + cycles

    def commit(self, bar):
        done_at = max(self.mma_free_at, self.now) + 1
        self.seq += 1
        self.events.append((done_at, self.seq, lambda: bar.arrive()))

    def pause(self, most):
        for _ in range(self.rng.randint(0, most)):
            yield


def copy_role(sim, units):
    gt = 0
    for nt in units:
        for j in range(nt):
            g = gt + j
            if g >= NS:                                    # P.V of the stage's previous tile done
                while not sim.empty[g % NS].passed(g // NS - 1):
                    yield
            yield from sim.pause(3)
            sim.full[g % NS].arrive(tx=4096)
            sim.copy(sim.full[g % NS], 4096)
        yield "sync"
        gt += nt


def mma_role(sim, units, p_full_of):
    gt = 0
    for nt in units:
        n1 = n2 = 0
        while n2 < nt:
            if n1 < nt:
                g1 = gt + n1
                if sim.full[g1 % NS].passed(g1 // NS) and \
                        (g1 < NB or sim.buf_free[g1 % NB].passed(g1 // NB - 1)):
                    sim.mma(8)
                    sim.commit(sim.s_bar[g1 % NB])
                    n1 += 1
            if n2 < n1:
                g2 = gt + n2
                bar, phase = p_full_of(g2)
                if bar.passed(phase):
                    sim.mma(4)
                    sim.commit(sim.empty[g2 % NS])
                    sim.commit(sim.buf_free[g2 % NB])
                    n2 += 1
            yield
            yield from sim.pause(2)
        yield "sync"
        gt += nt


def compute_role(sim, units, p_full_of):
    gt = 0
    for nt in units:
        for j in range(nt):
            g = gt + j
            while not sim.s_bar[g % NB].passed(g // NB):
                yield
            while not sim.full[g % NS].passed(g // NS):
                yield
            if j > 0 and sim.rng.random() < 0.3:            # the running max grew: rescale O
                while not sim.buf_free[(g - 1) % NB].passed((g - 1) // NB):
                    yield
            yield from sim.pause(6)
            bar, _ = p_full_of(g)
            bar.arrive()
        if nt:
            last = gt + nt - 1
            while not sim.buf_free[last % NB].passed(last // NB):
                yield
        yield "sync"
        gt += nt


def run(units, seed, shared_p_full=False, max_steps=200000):
    sim = Sim(seed, shared_p_full)
    if shared_p_full:
        p_full_of = lambda g: (sim.p_full[0], g)             # noqa: E731
    else:
        p_full_of = lambda g: (sim.p_full[g % NB], g // NB)  # noqa: E731
    roles = {"copy": copy_role(sim, units), "mma": mma_role(sim, units, p_full_of),
             "compute": compute_role(sim, units, p_full_of)}
    at_sync, finished = set(), set()
    for _ in range(max_steps):
        if len(finished) == len(roles):
            return True
        order = list(roles)
        sim.rng.shuffle(order)
        for name in order:
            if name in finished or name in at_sync:
                continue
            for _ in range(sim.rng.randint(1, 3)):
                try:
                    r = next(roles[name])
                except StopIteration:
                    finished.add(name)
                    break
                if r == "sync":
                    at_sync.add(name)
                    break
        if at_sync and len(at_sync | finished) == len(roles):
            at_sync.clear()                                  # __syncthreads between units
        if sim.events:
            sim.events.sort()
            sim.now = sim.events[0][0]
            while sim.events and sim.events[0][0] <= sim.now:
                _, _, fn = sim.events.pop(0)
                fn()
        else:
            sim.now += 1
    return False


def random_units(rng):
    """Units of one CTA: tiles per unit as the kernel computes them
    (pos_max // 32 + 1), a few units per CTA, empty units included."""
    units = []
    for _ in range(rng.randint(1, 4)):
        pos_max = rng.randint(-1, 700)
        units.append(pos_max // TILE + 1 if pos_max >= 0 else 0)
    return units


def test_kernel_protocol_completes_and_no_wait_falls_two_phases_behind():
    for seed in range(300):
        rng = random.Random(seed)
        assert run(random_units(rng), seed), f"deadlock, seed {seed}"


def test_a_shared_weights_barrier_is_caught():
    """One p_full for all four S buffers: the weights of tile j + 1 may be
    written before P.V(j) looked, so the barrier runs two phases ahead."""
    caught = 0
    for seed in range(300):
        rng = random.Random(seed)
        try:
            ok = run(random_units(rng), seed, shared_p_full=True)
        except AssertionError:
            ok = False
        caught += not ok
    assert caught > 0
