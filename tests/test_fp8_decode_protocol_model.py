"""A model of the FP8 decode kernel's synchronisation, run over random interleavings.

The roles of one CTA of decode_fp8_kernel, and the mbarriers between them, are
restated as Python generators:
- the TMA producer;
- the S^T issuer, which also writes the query limbs;
- the O^T issuer;
- two softmax groups;
- the asynchronous agents: each TMA load, and the in-order tensor-core queue behind
  each issuer.
The model keeps the kernel's barrier names, counts and phase arithmetic (one arrival
stands for a warp group's per-warp arrivals).  A scheduler runs the roles in random
order and checks mbarrier parity semantics.  A wait passes only when the phase with
its parity has completed, and it must then be exactly the phase the role meant, not
one before (a premature pass) nor two after (an overrun).  Each buffer carries the
version its writer gave it: the stages, the query limbs and 2^-e_q, the S^T, P'^T and
O^T buffers.  Every read checks that it sees the version it expects, which catches a
read before the write as well as an overwrite before the read.  A state where nothing
can run and some role is unfinished is a deadlock.

The model runs on the CPU and no GPU fault can come from it.  It checks the protocol
the kernel implements, including items of a single tile, where one softmax group
releases an item's queries unread.  It does not check the kernel itself.  It is
sequentially consistent.  A wait that exists for memory visibility cannot be shown
necessary here: the QInfo wait, before the softmax reads 2^-e_q, is already implied by
S^T having landed.
"""
import pytest

from protocol_sim import Sim, units_of, wait

K_STAGES = 5


def fp8_cta(sim, units, ring=4, sfree_wait=True):
    """One CTA over `units` = [(item, tile), ...] (its contiguous range of tiles).
    `ring` (P'^T and O^T buffers) and `sfree_wait` exist to plant mistakes."""
    nu = len(units)
    K = K_STAGES
    for s in range(K):
        sim.bar(f"Full{s}")
        sim.bar(f"Empty{s}")
    for b in range(2):
        sim.bar(f"SFull{b}")
        sim.bar(f"SFree{b}")
        sim.bar(f"QFree{b}", 3)   # the item's last S^T product + each softmax group
        sim.bar(f"QInfo{b}")
    for b in range(ring):
        sim.bar(f"PFull{b}")
        sim.bar(f"OFull{b}")
    sim.bar("Joint", 2)           # named barrier 3: both softmax groups

    s_queue, o_queue = [], []     # in-order tensor-core work of each issuer

    def tma_load(j, s):
        yield None
        sim.write(f"stage{s}", ("tile", j))     # codes, scales, and the queries at an item's first tile
        sim.arrive(f"Full{s}")

    def producer():
        for j in range(nu):
            s = j % K
            if j >= K:
                yield wait(f"Empty{s}", j // K - 1)
            sim.spawn(tma_load(j, s), f"tma{j}")
            yield None

    def mma_engine(queue, name):
        while True:
            if not queue:
                if name in done:
                    return
                yield None
                continue
            op = queue.pop(0)
            op()
            yield None

    done = set()

    def s_issuer():
        nitem, prev_item = -1, None
        for js, (item, _) in enumerate(units):
            first = item != prev_item
            if first:
                prev_item = item
                nitem += 1
            s, b = js % K, nitem & 1
            yield wait(f"Full{s}", js // K)
            if first:
                if nitem >= 2:
                    yield wait(f"QFree{b}", (nitem - 2) // 2)
                sim.read(f"stage{s}", ("tile", js))      # the bf16 queries
                sim.write(f"ql{b}", ("item", nitem))
                sim.write(f"qinfo{b}", ("item", nitem))
                sim.arrive(f"QInfo{b}")
            if js >= 2 and sfree_wait:
                yield wait(f"SFree{js & 1}", (js - 2) // 2)
            last_of_item = js + 1 == nu or units[js + 1][0] != item

            def mma(js=js, s=s, b=b, nitem=nitem, last=last_of_item):
                sim.read(f"stage{s}", ("tile", js))      # K codes
                sim.read(f"ql{b}", ("item", nitem))
                sim.write(f"sbuf{js & 1}", ("tile", js))
                sim.arrive(f"SFull{js & 1}")
                if last:
                    sim.arrive(f"QFree{b}")
            s_queue.append(mma)
            yield None
        done.add("s")

    def o_issuer():
        for jo in range(nu):
            yield wait(f"PFull{jo % ring}", jo // ring)
            s = jo % K

            def mma(jo=jo, s=s):
                sim.read(f"stage{s}", ("tile", jo))      # V codes
                sim.read(f"pbuf{jo % ring}", ("tile", jo))
                sim.write(f"obuf{jo % ring}", ("tile", jo))
                sim.arrive(f"OFull{jo % ring}")
                sim.arrive(f"Empty{s}")
            o_queue.append(mma)
            yield None
        done.add("o")

    def joint_sync():
        k = sim.bars["Joint"].phases
        sim.arrive("Joint")
        yield wait("Joint", k)

    def softmax(grp):
        cur_item, nitem, jp, qread = None, -1, -1, True

        def fold(jj):
            yield wait(f"OFull{jj % ring}", jj // ring)
            sim.read(f"obuf{jj % ring}", ("tile", jj))

        def flush(item, final):
            yield from joint_sync()        # every product of the item has been folded
            if grp == 1:
                for b in range(ring):
                    sim.write(f"pbuf{b}", ("exchange", item))
            yield from joint_sync()
            if grp == 1:
                yield from joint_sync()
                return
            for b in range(ring):
                sim.read(f"pbuf{b}", ("exchange", item))
            yield from joint_sync()
            if final:                      # the merging CTA's bulk copy into the idle stages
                for s in range(K):
                    sim.write(f"stage{s}", ("merge", item))

        for j, (item, _) in enumerate(units):
            if item != cur_item:
                if cur_item is not None:
                    if jp >= 0:
                        yield from fold(jp)
                    jp = -1
                    if not qread:
                        sim.arrive(f"QFree{nitem & 1}")
                    qread = True
                    yield from flush(cur_item, False)
                nitem += 1
                qread = False
                cur_item = item
            if (j & 1) != grp:
                yield None
                continue
            s = j % K
            yield wait(f"SFull{grp}", j >> 1)
            sim.read(f"sbuf{grp}", ("tile", j))
            sim.arrive(f"SFree{grp}")
            if jp >= 0:  # fold_issue: the TMEM load of O^T(jp) is issued here ...
                yield wait(f"OFull{jp % ring}", jp // ring)
            yield wait(f"Full{s}", j // K)
            sim.read(f"stage{s}", ("tile", j))            # scale rows
            if not qread:
                yield wait(f"QInfo{nitem & 1}", nitem >> 1)
                sim.read(f"qinfo{nitem & 1}", ("item", nitem))
                sim.arrive(f"QFree{nitem & 1}")
                qread = True
            sim.write(f"pbuf{j % ring}", ("tile", j))
            sim.arrive(f"PFull{j % ring}")
            yield None
            if jp >= 0:  # ... and has landed by fold_finish, after P'(j) is published
                sim.read(f"obuf{jp % ring}", ("tile", jp))
            jp = j
            yield None
        if nu > 0:
            if jp >= 0:
                yield from fold(jp)
            if not qread:
                sim.arrive(f"QFree{nitem & 1}")
            yield from flush(cur_item, True)

    sim.spawn(producer(), "producer")
    sim.spawn(s_issuer(), "s_issuer")
    sim.spawn(o_issuer(), "o_issuer")
    sim.spawn(mma_engine(s_queue, "s"), "s_mma")
    sim.spawn(mma_engine(o_queue, "o"), "o_mma")
    sim.spawn(softmax(0), "softmax0")
    sim.spawn(softmax(1), "softmax1")


CASES = [
    [1], [2], [7], [30],                       # one item
    [1, 1, 1, 1, 1, 1, 1],                     # items of one tile: a group never reads every item
    [3, 1, 2, 1, 4],
    [1, 5, 1, 5],
    [2, 2, 2, 2, 2, 2],
    [10, 3], [4, 12, 1],
]


@pytest.mark.parametrize("tiles", CASES, ids=[".".join(map(str, c)) for c in CASES])
def test_fp8_protocol_random_interleavings(tiles):
    units = units_of(tiles)
    for seed in range(300):
        sim = Sim(seed)
        fp8_cta(sim, units)
        sim.run()


def _caught(units, seeds=300, **mistake):
    n = 0
    for seed in range(seeds):
        sim = Sim(seed)
        fp8_cta(sim, units, **mistake)
        try:
            sim.run()
        except AssertionError:
            n += 1
    return n


def test_model_catches_a_missing_wait():
    """Without the S^T issuer's wait for its S buffer, some interleaving overwrites
    S^T(j - 2) before the softmax has read it."""
    assert _caught(units_of([9]), sfree_wait=False) > 0


def test_model_catches_a_two_buffer_p_ring():
    """With two P'^T / O^T buffers instead of four, O^T(j) can overwrite O^T(j - 2)
    while its load into the softmax is still in flight: the group publishes P'(j)
    before it finishes folding tile j - 2.  This is why the kernel keeps four."""
    assert _caught(units_of([12]), ring=2) > 0
