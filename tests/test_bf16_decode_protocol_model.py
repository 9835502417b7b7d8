"""A model of the bf16 decode kernel's synchronisation (decode_tc_kernel, the fused
append-and-decode path), run over random interleavings.

This restates the roles of one CTA and the mbarriers between them:
- the TMA producer, which holds back the tile that contains the appended row until
  the append warp has written it;
- the append warp;
- the single MMA issuer, which issues S^T(j) and then O^T(j - 1);
- the softmax warpgroup;
- the asynchronous agents: each TMA load and the in-order tensor-core queue.
Barrier names, counts (one arrival per role) and phase arithmetic follow the kernel.
The checks are those of the quantised kernels' models (tests/protocol_sim.py):
- no deadlock;
- every wait passes on exactly the phase it means;
- every read sees the version it expects.
"Every read" includes the TMA's read of the appended row: it must see the token the
append warp wrote, not the row before it.  The model is sequentially consistent; the
proxy fences around the append are beyond it.
"""
import pytest

from protocol_sim import Sim, units_of, wait

K_STAGES = 3


def bf16_cta(sim, units, append_tiles, p_ring=2, append_wait=True, sfree_wait=True):
    """One CTA over `units`; `append_tiles` holds the units whose tile contains the
    appended row.  The keyword arguments exist to plant mistakes."""
    nu = len(units)
    K = K_STAGES
    for s in range(K):
        sim.bar(f"Full{s}")
        sim.bar(f"Empty{s}")
    for b in range(2):
        sim.bar(f"SFull{b}")
        sim.bar(f"SFree{b}")
    for b in range(p_ring):
        sim.bar(f"PFull{b}")
        sim.bar(f"OFull{b}")
    sim.bar("Append")
    queue, done = [], set()

    def tma_load(j, s):
        yield None
        if j in append_tiles:
            sim.read(f"row{units[j][0]}", "appended")
        sim.write(f"stage{s}", ("tile", j))
        sim.arrive(f"Full{s}")

    def producer():
        appended = False
        for j in range(nu):
            s = j % K
            if j >= K:
                yield wait(f"Empty{s}", j // K - 1)
            if not appended and j in append_tiles and append_wait:
                yield wait("Append", 0)
                appended = True
            sim.spawn(tma_load(j, s), f"tma{j}")
            yield None

    def append_warp():
        for j in sorted(append_tiles):
            sim.write(f"row{units[j][0]}", "appended")
            yield None
        sim.arrive("Append")

    def engine():
        while True:
            if not queue:
                if "mma" in done:
                    return
                yield None
                continue
            queue.pop(0)()
            yield None

    def issue_o(jj):
        s = jj % K

        def mma():
            sim.read(f"stage{s}", ("tile", jj))   # V rows
            sim.read(f"pbuf{jj % p_ring}", ("tile", jj))
            sim.write(f"obuf{jj % p_ring}", ("tile", jj))
            sim.arrive(f"OFull{jj % p_ring}")
            sim.arrive(f"Empty{s}")
        queue.append(mma)

    def mma_issuer():
        for j in range(nu):
            s = j % K
            yield wait(f"Full{s}", j // K)
            if j >= 2 and sfree_wait:
                yield wait(f"SFree{j & 1}", (j - 2) // 2)

            def mma(j=j, s=s):
                sim.read(f"stage{s}", ("tile", j))    # K rows and the queries
                sim.write(f"sbuf{j & 1}", ("tile", j))
                sim.arrive(f"SFull{j & 1}")
            queue.append(mma)
            if j >= 1:
                yield wait(f"PFull{(j - 1) % p_ring}", (j - 1) // p_ring)
                issue_o(j - 1)
            yield None
        if nu > 0:
            yield wait(f"PFull{(nu - 1) % p_ring}", (nu - 1) // p_ring)
            issue_o(nu - 1)
        done.add("mma")

    def softmax():
        cur, pending = None, False

        def fold(jj):
            yield wait(f"OFull{jj % p_ring}", jj // p_ring)
            sim.read(f"obuf{jj % p_ring}", ("tile", jj))

        for j, (item, _) in enumerate(units):
            yield wait(f"SFull{j & 1}", j >> 1)
            sim.read(f"sbuf{j & 1}", ("tile", j))
            sim.arrive(f"SFree{j & 1}")
            if item != cur:
                if cur is not None and pending:
                    yield from fold(j - 1)
                pending = False
                cur = item
            sim.write(f"pbuf{j % p_ring}", ("tile", j))
            sim.arrive(f"PFull{j % p_ring}")
            yield None
            if pending:
                yield from fold(j - 1)
            pending = True
        if nu > 0:
            if pending:
                yield from fold(nu - 1)
            for s in range(K):  # the final merge's bulk copy into the idle stages
                sim.write(f"stage{s}", ("merge", 0))

    sim.spawn(producer(), "producer")
    sim.spawn(append_warp(), "append")
    sim.spawn(mma_issuer(), "mma_issuer")
    sim.spawn(engine(), "mma")
    sim.spawn(softmax(), "softmax")


def _append_tiles(units):
    """The last tile of each item (the appended token is the item's newest row)."""
    last = {}
    for j, (item, _) in enumerate(units):
        last[item] = j
    return set(last.values())


CASES = [[1], [2], [9], [40], [1, 1, 1, 1, 1], [3, 1, 4, 1, 5], [2, 7, 2], [12, 12]]


@pytest.mark.parametrize("tiles", CASES, ids=[".".join(map(str, c)) for c in CASES])
def test_bf16_protocol_random_interleavings(tiles):
    units = units_of(tiles)
    for seed in range(300):
        sim = Sim(seed)
        bf16_cta(sim, units, _append_tiles(units))
        sim.run()


@pytest.mark.parametrize("tiles", [[5], [1, 2, 3, 4], [8, 8, 1]], ids=["5", "1.2.3.4", "8.8.1"])
def test_bf16_protocol_pool_plan(tiles):
    """The pooled cache's plan: the same roles with no fused append (the pool appends
    in a launch of its own before the decode)."""
    units = units_of(tiles)
    for seed in range(300):
        sim = Sim(seed)
        bf16_cta(sim, units, set())
        sim.run()


def _caught(tiles, seeds=300, **mistake):
    units = units_of(tiles)
    n = 0
    for seed in range(seeds):
        sim = Sim(seed)
        bf16_cta(sim, units, _append_tiles(units), **mistake)
        try:
            sim.run()
        except AssertionError:
            n += 1
    return n


def test_model_catches_loading_the_appended_tile_early():
    """Without the producer's wait on the append warp, the tile holding the new token
    can be loaded before the token is written."""
    assert _caught([3, 2], append_wait=False) > 0


def test_s_buffer_wait_is_implied_by_the_p_wait():
    """In this single-issuer kernel the MMA thread's wait for S buffer j % 2 (the
    softmax has read S^T(j - 2)) is implied by an earlier wait.  Before it issues
    S^T(j), the thread has waited for P(j - 2) to issue O^T(j - 2).  The softmax
    publishes P(j - 2) only after its S^T(j - 2) load has completed, and a
    tensor-core fence comes before that arrival.  Without the wait no interleaving
    goes wrong: the wait costs the MMA thread a barrier round trip per tile and
    guards nothing.  (The two-group quantised kernels need theirs.)"""
    assert _caught([9], sfree_wait=False) == 0
    assert _caught([3, 1, 4, 1, 5], sfree_wait=False) == 0


def test_model_catches_a_single_p_buffer():
    """One P^T / O^T buffer instead of two: P(j) overwrites P(j - 1) before O^T(j - 1)
    has read it (the issuer takes P(j - 1) only after issuing S^T(j))."""
    assert _caught([9], p_ring=1) > 0
