"""A small simulator for models of the decode kernels' synchronisation: roles are
Python generators that yield ('wait', barrier, phase) to block on an mbarrier phase;
the scheduler resumes a role only when that phase's parity has completed (mbarrier
try_wait.parity semantics) and checks that it is exactly the phase the role meant.
Buffers carry versions; a read asserts the version it expects.  Used by the protocol
model tests; it contains no kernel arithmetic."""
import random


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phases = name, count, 0, 0

    def arrive(self, sim):
        self.pending += 1
        assert self.pending <= self.count, f"{self.name}: too many arrivals"
        if self.pending == self.count:
            self.pending = 0
            self.phases += 1
            for (b, k) in sim.blocked_on():
                if b is self:
                    assert self.phases <= k + 1, f"{self.name}: phase {k} overrun by a waiter's barrier"


class Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.bars = {}
        self.buf = {}
        self.actors = []  # [generator, pending wait (bar, phase) or None, name]

    def bar(self, name, count=1):
        if name not in self.bars:
            self.bars[name] = Barrier(name, count)
        return self.bars[name]

    def write(self, buf, version):
        self.buf[buf] = version

    def read(self, buf, version):
        assert self.buf.get(buf) == version, f"read of {buf}: expected {version}, found {self.buf.get(buf)}"

    def arrive(self, name):
        self.bars[name].arrive(self)

    def spawn(self, gen, name):
        self.actors.append([gen, None, name])

    def blocked_on(self):
        return [a[1] for a in self.actors if a[1] is not None]

    def run(self, limit=200000):
        steps = 0
        while self.actors:
            steps += 1
            assert steps < limit, "no progress"
            runnable = []
            for a in self.actors:
                w = a[1]
                if w is None or (w[0].phases & 1) != (w[1] & 1):
                    runnable.append(a)
            assert runnable, "deadlock: " + ", ".join(f"{a[2]} waits {a[1][0].name} phase {a[1][1]}"
                                                      for a in self.actors)
            a = self.rng.choice(runnable)
            if a[1] is not None:
                b, k = a[1]
                assert b.phases == k + 1, f"{a[2]}: wait on {b.name} for phase {k} passed at phase count {b.phases}"
                a[1] = None
            try:
                req = next(a[0])
            except StopIteration:
                self.actors.remove(a)
                continue
            if req is not None:  # ('wait', barrier name, phase index)
                a[1] = (self.bars[req[1]], req[2])


def wait(name, k):
    return ("wait", name, k)


def units_of(tiles_per_item, first_tile=0):
    """A CTA's range of (item, tile) units over items of the given tile counts."""
    out = []
    for i, n in enumerate(tiles_per_item):
        t0 = first_tile if i == 0 else 0
        out += [(i, t0 + t) for t in range(n)]
    return out
