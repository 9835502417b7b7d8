"""A model of the INT4 decode kernel's synchronisation, run over random interleavings.

This restates the roles of one CTA of decode_int4_kernel and the mbarriers between
them:
- the TMA producer;
- the prep warps: the K low nibbles into tensor memory, the V low nibbles, scales and
  the tile's largest s_v into the stage, and the query limbs at an item's first tile;
- the S^T issuer, which waits on each stage's prep and on the S buffer;
- the O^T issuer;
- two softmax groups on alternate tiles;
- the asynchronous agents: each TMA load and the in-order tensor-core queue behind each
  issuer.
Barrier names, counts (one arrival per role) and phase arithmetic follow the kernel.
The checks are those of the FP8 model (tests/protocol_sim.py):
- no deadlock;
- every wait passes on exactly the phase it means;
- every read sees the version it expects: stage data, the prep's outputs, the query
  limbs and sigma, and the S^T, P'^T and O^T buffers.
The queries' sigma and sum(q) reach the softmax with no barrier of their own.  The
prep writes them before it arrives on that tile's stage barrier, which the softmax
waits for; the model checks that ordering too.

The model is sequentially consistent: a wait that exists only for memory visibility
(the softmax's wait on the stage's prep barrier, once S^T of the tile has already
landed) cannot be shown necessary here; the kernel keeps it for the memory model.
"""
import pytest

from protocol_sim import Sim, units_of, wait

K_STAGES = 6


def int4_cta(sim, units, ring=4, qfree_wait_in_prep=True):
    """One CTA over `units` = [(item, tile), ...].  `ring` (P'^T and O^T buffers) and
    `qfree_wait_in_prep` exist to plant mistakes."""
    nu = len(units)
    K = K_STAGES
    for s in range(K):
        sim.bar(f"Full{s}")
        sim.bar(f"Empty{s}")
        sim.bar(f"Cvt{s}")         # the prep of the stage's tile is done (4 warps: one role here)
    for b in range(2):
        sim.bar(f"SFull{b}")
        sim.bar(f"SFree{b}")
        sim.bar(f"QFree{b}", 3)    # the item's last S^T product + each softmax group
    for b in range(ring):
        sim.bar(f"PFull{b}")
        sim.bar(f"OFull{b}")
    sim.bar("Joint", 2)

    s_queue, o_queue, done = [], [], set()

    def items():
        """(tile index, item, item count so far, first tile of the item?) for each unit."""
        nitem, prev = -1, None
        for j, (item, _) in enumerate(units):
            first = item != prev
            if first:
                nitem += 1
                prev = item
            yield j, item, nitem, first

    def tma_load(j, s):
        yield None
        sim.write(f"stage{s}", ("tile", j))      # code rows, scale rows, queries at a first tile
        sim.arrive(f"Full{s}")

    def producer():
        for j in range(nu):
            s = j % K
            if j >= K:
                yield wait(f"Empty{s}", j // K - 1)
            sim.spawn(tma_load(j, s), f"tma{j}")
            yield None

    def prep():
        for j, item, nitem, first in items():
            s, b = j % K, nitem & 1
            yield wait(f"Full{s}", j // K)
            sim.read(f"stage{s}", ("tile", j))
            sim.write(f"lk{s}", ("tile", j))       # K low nibbles, tensor memory
            sim.write(f"lv{s}", ("tile", j))       # V low nibbles, beside the V codes
            sim.write(f"misc{s}", ("tile", j))     # s_k, z_k, s_v, z_v and the tile's largest s_v
            if first:
                if nitem >= 2 and qfree_wait_in_prep:
                    yield wait(f"QFree{b}", (nitem - 2) // 2)
                sim.write(f"ql{b}", ("item", nitem))
                sim.write(f"qinfo{b}", ("item", nitem))
            sim.arrive(f"Cvt{s}")
            yield None

    def mma_engine(queue, name):
        while True:
            if not queue:
                if name in done:
                    return
                yield None
                continue
            queue.pop(0)()
            yield None

    def s_issuer():
        for js, item, nitem, first in items():
            s, b = js % K, nitem & 1
            yield wait(f"Cvt{s}", js // K)
            if js >= 2:
                yield wait(f"SFree{js & 1}", (js - 2) // 2)
            last = js + 1 == nu or units[js + 1][0] != item

            def mma(js=js, s=s, b=b, nitem=nitem, last=last):
                sim.read(f"stage{s}", ("tile", js))   # K code bytes
                sim.read(f"lk{s}", ("tile", js))
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
                sim.read(f"stage{s}", ("tile", jo))   # V code bytes
                sim.read(f"lv{s}", ("tile", jo))
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

        def flush(item):
            yield from joint_sync()              # every product of the item has been folded
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

        for j, item, n, first in items():
            if item != cur_item:
                if cur_item is not None:
                    if jp >= 0:
                        yield from fold(jp)
                    jp = -1
                    if not qread:
                        sim.arrive(f"QFree{nitem & 1}")
                    qread = True
                    yield from flush(cur_item)
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
            if jp >= 0:                          # fold_issue: O^T(jp) load issued ...
                yield wait(f"OFull{jp % ring}", jp // ring)
            yield wait(f"Cvt{s}", j // K)
            sim.read(f"misc{s}", ("tile", j))
            if not qread:
                sim.read(f"qinfo{nitem & 1}", ("item", nitem))
                sim.arrive(f"QFree{nitem & 1}")
                qread = True
            sim.write(f"pbuf{j % ring}", ("tile", j))
            sim.arrive(f"PFull{j % ring}")
            yield None
            if jp >= 0:                          # ... landed by fold_finish
                sim.read(f"obuf{jp % ring}", ("tile", jp))
            jp = j
            yield None
        if nu > 0:
            if jp >= 0:
                yield from fold(jp)
            if not qread:
                sim.arrive(f"QFree{nitem & 1}")
            yield from flush(cur_item)

    sim.spawn(producer(), "producer")
    sim.spawn(prep(), "prep")
    sim.spawn(s_issuer(), "s_issuer")
    sim.spawn(o_issuer(), "o_issuer")
    sim.spawn(mma_engine(s_queue, "s"), "s_mma")
    sim.spawn(mma_engine(o_queue, "o"), "o_mma")
    sim.spawn(softmax(0), "softmax0")
    sim.spawn(softmax(1), "softmax1")


CASES = [
    [1], [2], [8], [30],
    [1, 1, 1, 1, 1, 1, 1],
    [3, 1, 2, 1, 4],
    [1, 6, 1, 6],
    [2, 2, 2, 2, 2, 2],
    [13, 2], [4, 12, 1],
]


@pytest.mark.parametrize("tiles", CASES, ids=[".".join(map(str, c)) for c in CASES])
def test_int4_protocol_random_interleavings(tiles):
    units = units_of(tiles)
    for seed in range(300):
        sim = Sim(seed)
        int4_cta(sim, units)
        sim.run()


def _caught(units, seeds=300, **mistake):
    n = 0
    for seed in range(seeds):
        sim = Sim(seed)
        int4_cta(sim, units, **mistake)
        try:
            sim.run()
        except AssertionError:
            n += 1
    return n


def test_model_catches_query_limbs_overwritten_early():
    """Without the prep's wait on the query-buffer barrier, the limbs of item n + 2 can
    replace those of item n before item n's last S^T product has read them."""
    assert _caught(units_of([1, 1, 1, 1, 1, 1]), qfree_wait_in_prep=False) > 0


def test_model_catches_a_two_buffer_p_ring():
    """Two P'^T / O^T buffers instead of four: O^T(j) can overwrite O^T(j - 2) while its
    load into the softmax is still in flight."""
    assert _caught(units_of([12]), ring=2) > 0
