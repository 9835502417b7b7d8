"""A model of the pre-fill kernel's synchronisation (prefill_tc_kernel), run over
random interleavings.

This restates the roles of one CTA and the mbarriers between them:
- the Q and K producer;
- the V producer;
- the MMA thread, which issues S_0(0), S_1(0), then per key tile j the sequence
  PV_0(j), S_0(j+1), PV_1(j), S_1(j+1);
- one softmax warpgroup per query tile;
- the asynchronous agents: each TMA load and the in-order tensor-core queue.
Barrier names, counts (one arrival per role) and phase arithmetic follow the kernel.

Tensor memory is modelled as buffers with versions.  S_t holds S_t(j) after its
product.  The softmax then writes P_t(j) over it, which PV_t(j) reads before S_t(j+1)
overwrites it: products of one thread complete in issue order.  O_t holds the sum
through tile j.  The softmax rescales O_t in place once S_t(j) has landed: by then
PV_t(j-1) has landed and PV_t(j) has not been issued.
The checks are those of the decode models (tests/protocol_sim.py):
- no deadlock;
- every wait passes on exactly the phase it means;
- every read sees the version it expects.
"""
import pytest

from protocol_sim import Sim, wait

KQ, KK, KV = 2, 2, 2   # query tiles per CTA, K stages, V stages


def prefill_cta(sim, nt, k_stages=KK, v_stages=KV, pv_before_next_s=True):
    """One CTA over nt key tiles.  The keyword arguments exist to plant mistakes."""
    sim.bar("Q")
    for s in range(k_stages):
        sim.bar(f"KFull{s}")
        sim.bar(f"KEmpty{s}")
    for s in range(v_stages):
        sim.bar(f"VFull{s}")
        sim.bar(f"VEmpty{s}")
    for t in range(KQ):
        sim.bar(f"SFull{t}")
        sim.bar(f"PFull{t}")
        sim.bar(f"OFull{t}")
    queue, done = [], set()

    def load(buf, version, bar):
        yield None
        sim.write(buf, version)
        sim.arrive(bar)

    def qk_producer():
        sim.spawn(load("q", "Q", "Q"), "tmaQ")
        for j in range(nt):
            s = j % k_stages
            if j >= k_stages:
                yield wait(f"KEmpty{s}", j // k_stages - 1)
            sim.spawn(load(f"k{s}", ("K", j), f"KFull{s}"), f"tmaK{j}")
            yield None

    def v_producer():
        for j in range(nt):
            s = j % v_stages
            if j >= v_stages:
                yield wait(f"VEmpty{s}", j // v_stages - 1)
            sim.spawn(load(f"v{s}", ("V", j), f"VFull{s}"), f"tmaV{j}")
            yield None

    def engine():
        while True:
            if not queue:
                if "mma" in done:
                    return
                yield None
                continue
            queue.pop(0)()
            yield None

    def s_product(t, j):
        def op():
            sim.read("q", "Q")
            sim.read(f"k{j % k_stages}", ("K", j))
            sim.write(f"s{t}", ("S", j))
            sim.arrive(f"SFull{t}")
        return op

    def pv_product(t, j):
        def op():
            sim.read(f"s{t}", ("P", j))
            sim.read(f"v{j % v_stages}", ("V", j))
            if j > 0:
                sim.read(f"o{t}", ("O", j - 1))
            sim.write(f"o{t}", ("O", j))
        return op

    def arrival(name):
        return lambda: sim.arrive(name)

    def mma_thread():
        if nt > 0:
            yield wait("Q", 0)
            yield wait("KFull0", 0)
            for t in range(KQ):
                queue.append(s_product(t, 0))
            queue.append(arrival("KEmpty0"))
        for j in range(nt):
            for t in range(KQ):
                yield wait(f"PFull{t}", j)
                if t == 0:
                    yield wait(f"VFull{j % v_stages}", j // v_stages)
                nxt = []
                if j + 1 < nt:
                    if t == 0:
                        yield wait(f"KFull{(j + 1) % k_stages}", (j + 1) // k_stages)
                    nxt.append(s_product(t, j + 1))
                    if t == KQ - 1:
                        nxt.append(arrival(f"KEmpty{(j + 1) % k_stages}"))
                else:
                    nxt.append(arrival(f"OFull{t}"))
                pv = [pv_product(t, j)] + ([arrival(f"VEmpty{j % v_stages}")] if t == KQ - 1 else [])
                queue.extend(pv + nxt if pv_before_next_s else nxt + pv)
                yield None
        done.add("mma")

    def softmax(t):
        for j in range(nt):
            yield wait(f"SFull{t}", j)
            sim.read(f"s{t}", ("S", j))
            if j >= 1:                       # the lazy rescale of O_t, when the max moved
                sim.read(f"o{t}", ("O", j - 1))
                sim.write(f"o{t}", ("O", j - 1))
            sim.write(f"s{t}", ("P", j))     # P_t(j) over the first 64 columns of S_t
            sim.arrive(f"PFull{t}")
            yield None
        if nt > 0:
            yield wait(f"OFull{t}", 0)
            sim.read(f"o{t}", ("O", nt - 1))

    sim.spawn(qk_producer(), "qk")
    sim.spawn(v_producer(), "v")
    sim.spawn(mma_thread(), "mma_thread")
    sim.spawn(engine(), "mma")
    for t in range(KQ):
        sim.spawn(softmax(t), f"softmax{t}")


@pytest.mark.parametrize("nt", [1, 2, 3, 5, 16])
def test_prefill_protocol_random_interleavings(nt):
    for seed in range(400):
        sim = Sim(seed)
        prefill_cta(sim, nt)
        sim.run()


def _caught(nt, seeds=300, **mistake):
    n = 0
    for seed in range(seeds):
        sim = Sim(seed)
        prefill_cta(sim, nt, **mistake)
        try:
            sim.run()
        except AssertionError:
            n += 1
    return n


def test_model_catches_s_issued_before_pv():
    """Issuing S_t(j+1) before PV_t(j) lets the new logits overwrite P_t(j) before the
    product has read it (P lives in S_t's tensor memory)."""
    assert _caught(4, pv_before_next_s=False) > 0
