"""CPU tests of the paged pool's host side (ragged batching): argument checks, page
accounting and the length contract, with launches skipped (duo_debug_launch_controls
dry run) so that no GPU is needed.  A fake, never dereferenced address stands in for the
device buffer."""
import numpy as np
import pytest

from head_split_kv_duo_b200 import duo

FAKE = 1 << 40


@pytest.fixture
def dry_run():
    assert duo.duo_debug_launch_controls(1, -1) == duo.DUO_OK
    yield
    assert duo.duo_debug_launch_controls(0, -1) == duo.DUO_OK


def _pool(layers=2, Hkv=4, Hq=8, mask=None, S=4, W=16, max_seqs=4, max_len=1000, num_pages=20, opts=None):
    if mask is None:
        mask = np.array([[1, 0, 1, 0]] * layers, dtype=np.uint8)
    if opts is None:
        opts = duo._opts(q_heads=Hq)
    need = duo.duo_pool_bytes(layers, Hkv, 128, mask, S, W, max_seqs, max_len, num_pages, opts)
    st, h = duo.duo_pool_create(layers, Hkv, 128, mask, S, W, max_seqs, max_len, num_pages, opts, FAKE, need)
    return st, h, need


def test_pool_create_checks():
    st, h, need = _pool()
    assert st == duo.DUO_OK and need > 0
    duo.duo_pool_destroy(h)
    assert _pool(opts=duo._opts(q_heads=8, dtype=duo.DUO_FP32))[0] == duo.DUO_ERR_UNSUPPORTED
    assert _pool(opts=duo._opts(q_heads=8, retr_fmt=duo.DUO_KV_INT4_G128))[0] == duo.DUO_ERR_UNSUPPORTED
    assert _pool(Hq=128, opts=duo._opts(q_heads=128))[0] == duo.DUO_ERR_UNSUPPORTED  # group of 32
    assert _pool(mask=np.array([[1, 2, 0, 0]] * 2, np.uint8))[0] == duo.DUO_ERR_INVALID
    assert _pool(W=0)[0] == duo.DUO_ERR_INVALID
    assert _pool(num_pages=0)[0] == duo.DUO_ERR_INVALID
    m = np.array([[1, 0, 1, 0]] * 2, np.uint8)
    need = duo.duo_pool_bytes(2, 4, 128, m, 4, 16, 4, 1000, 20, duo._opts(q_heads=8))
    st, h = duo.duo_pool_create(2, 4, 128, m, 4, 16, 4, 1000, 20, duo._opts(q_heads=8), FAKE, need - 1)
    assert st == duo.DUO_ERR_INVALID
    st, h = duo.duo_pool_create(2, 4, 128, m, 4, 16, 4, 1000, 20, duo._opts(q_heads=8), FAKE + 16, need)
    assert st == duo.DUO_ERR_INVALID


def test_pool_pages_follow_lengths(dry_run):
    """Each open sequence holds ceil(len / 128) pages of its longest layer, distinct
    across sequences; closing returns them; running out of pages or past max_len is
    refused with nothing changed."""
    st, h, _ = _pool(num_pages=10, max_len=1000)
    seqs = [duo.duo_pool_open(h)[1] for _ in range(3)]
    assert len(set(seqs)) == 3
    lens = {s: [0, 0] for s in seqs}
    for s, layer, n in [(seqs[0], 0, 1), (seqs[0], 0, 127), (seqs[0], 1, 300), (seqs[1], 0, 129), (seqs[2], 1, 5)]:
        assert duo.duo_pool_append_kv(h, layer, s, FAKE, FAKE, n) == duo.DUO_OK
        lens[s][layer] += n
    used = sum(-(-max(v) // 128) for v in lens.values())
    assert duo.duo_pool_free_pages(h) == (duo.DUO_OK, 10 - used)
    held = []
    for s in seqs:
        for layer in range(2):
            assert duo.duo_pool_len(h, s, layer) == (duo.DUO_OK, lens[s][layer])
        held += [duo.duo_pool_page(h, s, i)[1] for i in range(-(-max(lens[s]) // 128))]
    assert len(held) == len(set(held)) == used
    # 10 pages: 3 + 2 + 1 used; 5 more pages for one sequence do not fit (4 are free)
    before = duo.duo_pool_free_pages(h)[1]
    assert duo.duo_pool_append_kv(h, 0, seqs[2], FAKE, FAKE, 128 * 6) == duo.DUO_ERR_CAPACITY
    assert duo.duo_pool_free_pages(h)[1] == before and duo.duo_pool_len(h, seqs[2], 0)[1] == 0
    assert duo.duo_pool_append_kv(h, 1, seqs[1], FAKE, FAKE, 1000) == duo.DUO_ERR_CAPACITY  # max_len
    assert duo.duo_pool_close(h, seqs[0]) == duo.DUO_OK
    assert duo.duo_pool_free_pages(h)[1] == before + 3
    assert duo.duo_pool_len(h, seqs[0], 0)[0] == duo.DUO_ERR_INVALID  # closed
    assert duo.duo_pool_open(h)[1] == seqs[0]  # the slot is reused, at length 0
    assert duo.duo_pool_len(h, seqs[0], 1) == (duo.DUO_OK, 0)
    duo.duo_pool_destroy(h)


def test_pool_slots_run_out(dry_run):
    st, h, _ = _pool(max_seqs=2)
    assert duo.duo_pool_open(h)[0] == duo.DUO_OK and duo.duo_pool_open(h)[0] == duo.DUO_OK
    assert duo.duo_pool_open(h)[0] == duo.DUO_ERR_CAPACITY
    duo.duo_pool_destroy(h)


def test_pool_decode_step_bookkeeping(dry_run):
    """A ragged step advances every listed (sequence, layer) by one token and opens a page
    exactly when a sequence crosses a multiple of 128; the step's arguments are checked
    before any launch."""
    st, h, _ = _pool(layers=3, num_pages=40)
    a, b, c = (duo.duo_pool_open(h)[1] for _ in range(3))
    for s, n in [(a, 127), (b, 5), (c, 256)]:
        for layer in range(3):
            assert duo.duo_pool_append_kv(h, layer, s, FAKE, FAKE, n) == duo.DUO_OK
    free0 = duo.duo_pool_free_pages(h)[1]
    P = FAKE
    assert duo.duo_pool_decode_step(h, 0, 3, [a, b, c], P, P, P, P, None) == duo.DUO_OK
    assert [duo.duo_pool_len(h, s, 2)[1] for s in (a, b, c)] == [128, 6, 257]
    assert duo.duo_pool_free_pages(h)[1] == free0 - 1  # c opened its third page
    assert duo.duo_pool_decode_step(h, 0, 3, [a, b], P, P, P, P, None) == duo.DUO_OK
    assert duo.duo_pool_free_pages(h)[1] == free0 - 2  # a opened its second page
    # one layer only: lengths then differ across layers
    assert duo.duo_pool_decode_step(h, 1, 1, [b], P, P, P, P, None) == duo.DUO_OK
    assert [duo.duo_pool_len(h, b, layer)[1] for layer in range(3)] == [7, 8, 7]
    # refused: a sequence listed twice, a closed slot, unequal lengths over the listed
    # layers, too many (layer, sequence) pairs, unaligned buffers, layers out of range
    assert duo.duo_pool_decode_step(h, 0, 1, [a, a], P, P, P, P, None) == duo.DUO_ERR_INVALID
    assert duo.duo_pool_decode_step(h, 0, 1, [3], P, P, P, P, None) == duo.DUO_ERR_INVALID
    assert duo.duo_pool_decode_step(h, 0, 3, [b], P, P, P, P, None) == duo.DUO_ERR_INVALID
    assert duo.duo_pool_decode_step(h, 0, 3, [a, b, c] * 400, P, P, P, P, None) == duo.DUO_ERR_INVALID
    assert duo.duo_pool_decode_step(h, 0, 1, [a], P + 8, P, P, P, None) == duo.DUO_ERR_INVALID
    assert duo.duo_pool_decode_step(h, 2, 2, [a], P, P, P, P, None) == duo.DUO_ERR_INVALID
    assert [duo.duo_pool_len(h, s, 0)[1] for s in (a, b, c)] == [129, 7, 257]
    duo.duo_pool_destroy(h)


def _fail(n, call):
    assert duo.duo_debug_launch_controls(1, n) == duo.DUO_OK
    st = call()
    assert duo.duo_debug_launch_controls(1, -1) == duo.DUO_OK
    return st


def test_pool_launch_failures_keep_the_contract(dry_run):
    """A failed append launch leaves lengths and free pages as they were; a decode step
    whose attention launch fails keeps its appended tokens (lengths advance); a failed
    slot-clearing launch leaves the slot closed."""
    st, h, _ = _pool(num_pages=8)
    s = duo.duo_pool_open(h)[1]
    free0 = duo.duo_pool_free_pages(h)[1]
    assert _fail(0, lambda: duo.duo_pool_append_kv(h, 0, s, FAKE, FAKE, 300)) == duo.DUO_ERR_CUDA
    assert duo.duo_pool_len(h, s, 0)[1] == 0 and duo.duo_pool_free_pages(h)[1] == free0
    for layer in range(2):
        assert duo.duo_pool_append_kv(h, layer, s, FAKE, FAKE, 128) == duo.DUO_OK
    free1 = duo.duo_pool_free_pages(h)[1]
    step = lambda: duo.duo_pool_decode_step(h, 0, 2, [s], FAKE, FAKE, FAKE, FAKE, None)
    assert _fail(0, step) == duo.DUO_ERR_CUDA  # the append: nothing written, no page kept
    assert duo.duo_pool_len(h, s, 1)[1] == 128 and duo.duo_pool_free_pages(h)[1] == free1
    assert _fail(1, step) == duo.DUO_ERR_CUDA  # the attention: the token stays appended
    assert duo.duo_pool_len(h, s, 1)[1] == 129 and duo.duo_pool_free_pages(h)[1] == free1 - 1
    assert _fail(0, lambda: duo.duo_pool_open(h)[0]) == duo.DUO_ERR_CUDA
    assert duo.duo_pool_open(h) == (duo.DUO_OK, 1)  # slot 1 was not taken by the failed call
    duo.duo_pool_destroy(h)
