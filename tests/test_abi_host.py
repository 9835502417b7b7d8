"""CPU tests of the C ABI: the library loads, exports every declared symbol, and its
host-side checks and bookkeeping behave as include/duo.h states.  No kernel is
launched; a fake (never dereferenced) device address stands in for the buffer."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
from head_split_kv_duo_b200 import duo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 40  # 256-byte aligned address that is never touched without a GPU


def _declared():
    text = open(os.path.join(ROOT, "include", "duo.h")).read()
    return re.findall(r"DUO_API\s+[\w\s\*]*?\b(duo_\w+)\s*\(", text)


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 12
    lib = duo.lib()
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", duo._build.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (duo_\w+)", out))
    assert set(names) <= exported
    assert exported <= set(names), f"undeclared exports: {exported - set(names)}"


def _create(layers=2, Hkv=4, d=128, mask=None, S=4, W=16, max_len=1000, opts=None, buf=FAKE, nbytes=None):
    if mask is None:
        mask = np.array([[1, 0, 1, 0]] * layers, dtype=np.uint8)
    if opts is None:
        opts = duo._opts(batch=2, q_heads=8)
    need = duo.duo_cache_bytes(layers, Hkv, d, mask, S, W, max_len, opts)
    st, h = duo.duo_cache_create(layers, Hkv, d, mask, S, W, max_len, opts, buf, need if nbytes is None else nbytes)
    return st, h, need


def test_create_is_host_only_and_reports_lengths():
    st, h, need = _create()
    assert st == duo.DUO_OK and need > 0
    for layer in range(2):
        assert duo.duo_cache_len(h, layer) == (duo.DUO_OK, 0)
    assert duo.duo_cache_len(h, 2)[0] == duo.DUO_ERR_INVALID
    duo.duo_cache_destroy(h)


@pytest.mark.parametrize("kw,status", [
    (dict(layers=0), duo.DUO_ERR_INVALID),
    (dict(d=96), duo.DUO_ERR_INVALID),
    (dict(W=0), duo.DUO_ERR_INVALID),
    (dict(S=-1), duo.DUO_ERR_INVALID),
    (dict(max_len=0), duo.DUO_ERR_INVALID),
    (dict(opts=duo._opts(q_heads=6)), duo.DUO_ERR_INVALID),
    (dict(opts=duo._opts(batch=0)), duo.DUO_ERR_INVALID),
    (dict(opts=duo._opts(dtype=7)), duo.DUO_ERR_INVALID),
    (dict(opts=duo._opts(dtype=duo.DUO_FP32, retr_fmt=duo.DUO_KV_INT4_G128)), duo.DUO_ERR_UNSUPPORTED),
    (dict(d=64, opts=duo._opts(retr_fmt=duo.DUO_KV_INT4_G128)), duo.DUO_ERR_UNSUPPORTED),
    (dict(buf=FAKE + 16), duo.DUO_ERR_INVALID),
    (dict(buf=0), duo.DUO_ERR_INVALID),
])
def test_create_rejects(kw, status):
    if "d" in kw and kw["d"] == 96:
        st, h = duo.duo_cache_create(2, 4, 96, np.zeros((2, 4), np.uint8), 4, 16, 100, None, FAKE, 1 << 30)
    else:
        st, h, _ = _create(**kw)
    assert st == status
    assert not h.value


def test_create_rejects_small_buffer_and_bad_mask():
    st, _, need = _create()
    st, h, _ = _create(nbytes=need - 1)
    assert st == duo.DUO_ERR_INVALID
    st, h, _ = _create(mask=np.array([[1, 2, 0, 0]] * 2, dtype=np.uint8))
    assert st == duo.DUO_ERR_INVALID


def test_calls_check_arguments_before_any_launch():
    st, h, _ = _create(max_len=100)
    p = FAKE  # aligned stand-in pointers: every call below must fail before touching them
    assert duo.duo_append_kv(h, 0, p, p, 0) == duo.DUO_ERR_INVALID
    assert duo.duo_append_kv(h, 5, p, p, 1) == duo.DUO_ERR_INVALID
    assert duo.duo_append_kv(h, 0, p + 8, p, 1) == duo.DUO_ERR_INVALID
    assert duo.duo_append_kv(h, 0, None, p, 1) == duo.DUO_ERR_INVALID
    assert duo.duo_append_kv(h, 0, p, p, 101) == duo.DUO_ERR_CAPACITY
    assert duo.duo_prefill_chunk(h, 0, p, p, p, 101, p, None) == duo.DUO_ERR_CAPACITY
    assert duo.duo_prefill_chunk(h, 0, p, p, p, 0, p, None) == duo.DUO_ERR_INVALID
    assert duo.duo_prefill_chunk(h, 0, p, p, p, 4, p, p + 2) == duo.DUO_ERR_INVALID
    assert duo.duo_decode_attention(h, 0, p, p, None) == duo.DUO_ERR_INVALID  # empty layer
    assert duo.duo_cache_len(h, 0) == (duo.DUO_OK, 0)
    duo.duo_cache_destroy(h)


@pytest.mark.parametrize("fmt", [duo.DUO_KV_INT4_G128, duo.DUO_KV_FP8_E4M3])
def test_quantised_prefill_is_unsupported(fmt):
    st, h, _ = _create(opts=duo._opts(retr_fmt=fmt))
    assert st == duo.DUO_OK
    assert duo.duo_prefill_chunk(h, 0, FAKE, FAKE, FAKE, 4, FAKE, None) == duo.DUO_ERR_UNSUPPORTED
    duo.duo_cache_destroy(h)


def test_fp8_layout_and_bytes():
    """FP8 retrieval rows are d code bytes plus a 4-byte fp32 scale; fp32 or head_dim 64
    caches cannot take the format; an unknown format is invalid."""
    st, h, need = _create(layers=1, Hkv=4, mask=np.array([[1, 1, 0, 0]], np.uint8), S=16, W=512, max_len=1 << 20,
                          opts=duo._opts(retr_fmt=duo.DUO_KV_FP8_E4M3))
    assert st == duo.DUO_OK
    st, r, f = duo.duo_kv_bytes(h, 1 << 20)
    assert r == 2 * (2 * (1 << 20) * (128 + 4) + 2 * 528 * 256)
    st, ptr, nb, cap = duo.duo_debug_region(h, 0, duo.DUO_REGION_RETR_K)
    assert nb == 2 * cap * 128
    st, ptr, nb, cap = duo.duo_debug_region(h, 0, duo.DUO_REGION_RETR_VSZ)
    assert st == duo.DUO_OK and nb == 2 * cap * 4
    duo.duo_cache_destroy(h)
    assert _create(opts=duo._opts(dtype=duo.DUO_FP32, retr_fmt=duo.DUO_KV_FP8_E4M3))[0] == duo.DUO_ERR_UNSUPPORTED
    assert _create(d=64, opts=duo._opts(retr_fmt=duo.DUO_KV_FP8_E4M3))[0] == duo.DUO_ERR_UNSUPPORTED
    assert _create(opts=duo._opts(retr_fmt=3))[0] == duo.DUO_ERR_INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device failure path")
def test_launch_without_device_fails_cleanly():
    st, h, _ = _create(max_len=100)
    assert duo.duo_append_kv(h, 0, FAKE, FAKE, 3) == duo.DUO_ERR_CUDA
    assert duo.duo_cache_len(h, 0) == (duo.DUO_OK, 0)
    duo.duo_cache_destroy(h)


def test_kv_bytes_closed_forms():
    """duo_kv_bytes against the oracle's (H_r L + H_s min(L, S+W)) d and 2 D H L d."""
    mask = np.array([[1, 0, 0, 0, 1, 0, 0, 0]] * 3, dtype=np.uint8)
    st, h, _ = _create(layers=3, Hkv=8, mask=mask, S=16, W=512, max_len=1 << 20, opts=duo._opts(batch=2))
    for L in [1, 100, 528, 529, 32768, 1 << 20]:
        st, r, f = duo.duo_kv_bytes(h, L)
        assert st == duo.DUO_OK
        assert r == 2 * 2 * 3 * 2 * oracle.layer_kv_elems(2, 6, L, 16, 512, 128)
        assert f == 2 * 3 * oracle.full_kv_bytes(1, 8, 128, L, 2)
    duo.duo_cache_destroy(h)


def test_kv_bytes_int4_counts_codes_and_scales():
    st, h, _ = _create(layers=1, Hkv=4, mask=np.array([[1, 1, 0, 0]], np.uint8), S=16, W=512, max_len=1 << 20,
                       opts=duo._opts(retr_fmt=duo.DUO_KV_INT4_G128))
    st, r, f = duo.duo_kv_bytes(h, 1 << 20)
    assert r == 2 * (2 * (1 << 20) * (64 + 4) + 2 * 528 * 256)
    duo.duo_cache_destroy(h)


def test_slot_positions_before_any_token():
    st, h, _ = _create()
    for slot in range(20):
        assert duo.duo_debug_slot_position(h, 0, 1, slot) == (duo.DUO_OK, -1)
    assert duo.duo_debug_slot_position(h, 0, 1, 20)[0] == duo.DUO_ERR_INVALID  # S + W slots
    assert duo.duo_debug_slot_position(h, 0, 0, 999) == (duo.DUO_OK, -1)
    duo.duo_cache_destroy(h)


def test_regions_are_disjoint_and_inside_the_buffer():
    st, h, need = _create(opts=duo._opts(batch=2, q_heads=8, retr_fmt=duo.DUO_KV_INT4_G128))
    spans = []
    for layer in range(2):
        for which in range(6):
            st, ptr, nb, cap = duo.duo_debug_region(h, layer, which)
            assert st == duo.DUO_OK and cap == 1024
            assert FAKE <= ptr and ptr + nb <= FAKE + need and ptr % 1024 == 0
            spans.append((ptr, ptr + nb))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    duo.duo_cache_destroy(h)


def test_status_strings():
    for s in range(6):
        assert duo.duo_status_str(s)


# ------------------------------------------------------- gated mixed attention

def test_gated_checks_arguments_before_any_launch():
    B, L, Hq, Hkv, d, S, W = 1, 100, 4, 2, 64, 2, 8
    p = FAKE

    def call(**kw):
        a = dict(q=p, k=p, v=p, alpha=p, out=p, scale=0.0, L=L, d=d, Hq=Hq, W=W)
        a.update(kw)
        return duo.duo_gated_attention(a["q"], a["k"], a["v"], B, a["L"], a["Hq"], Hkv, a["d"], duo.DUO_FP32,
                                       a["alpha"], S, a["W"], a["scale"], a["out"])

    assert call(q=0) == duo.DUO_ERR_INVALID
    assert call(alpha=0) == duo.DUO_ERR_INVALID
    assert call(out=p + 8) == duo.DUO_ERR_INVALID       # 16-byte alignment
    assert call(alpha=p + 2) == duo.DUO_ERR_INVALID     # 4-byte alignment
    assert call(scale=-1.0) == duo.DUO_ERR_INVALID
    assert call(L=0) == duo.DUO_ERR_INVALID             # empty sequence
    assert call(d=96) == duo.DUO_ERR_INVALID            # head_dim
    assert call(Hq=5) == duo.DUO_ERR_INVALID            # Hq % Hkv
    assert call(W=0) == duo.DUO_ERR_INVALID             # W >= 1


def test_append_decode_checks_arguments_before_any_launch():
    st, h, _ = _create(max_len=10)
    assert st == duo.DUO_OK
    p = FAKE
    try:
        assert duo.duo_append_decode(h, 0, 0, p, p, p, None) == duo.DUO_ERR_INVALID   # no q
        assert duo.duo_append_decode(h, 0, p, 0, p, p, None) == duo.DUO_ERR_INVALID   # no k
        assert duo.duo_append_decode(h, 0, p, p, p + 8, p, None) == duo.DUO_ERR_INVALID  # unaligned v
        assert duo.duo_append_decode(h, 5, p, p, p, p, None) == duo.DUO_ERR_INVALID   # no such layer
        assert duo.duo_append_decode(h, 0, p, p, p, p, p + 2) == duo.DUO_ERR_INVALID  # unaligned lse
        assert duo.duo_cache_len(h, 0) == (duo.DUO_OK, 0)
    finally:
        duo.duo_cache_destroy(h)


# ------------------------------------- host bookkeeping under the test launch controls

@pytest.fixture
def dry_run():
    """Launches skipped and reported as accepted (duo_debug_launch_controls)."""
    assert duo.duo_debug_launch_controls(1, -1) == duo.DUO_OK
    yield
    assert duo.duo_debug_launch_controls(0, -1) == duo.DUO_OK


def test_device_stall_control_checks_its_argument():
    assert duo.duo_debug_device_stall(2) == duo.DUO_ERR_INVALID
    assert duo.duo_debug_device_stall(-1) == duo.DUO_ERR_INVALID
    assert duo.duo_debug_device_stall(1) == duo.DUO_OK
    assert duo.duo_debug_device_stall(0) == duo.DUO_OK


def test_launch_controls_reject_bad_values():
    assert duo.duo_debug_launch_controls(2, -1) == duo.DUO_ERR_INVALID
    assert duo.duo_debug_launch_controls(0, -2) == duo.DUO_ERR_INVALID
    assert duo.duo_debug_launch_controls(0, -1) == duo.DUO_OK


def test_dry_run_lengths_and_slots_follow_the_slot_rule(dry_run):
    """Appends and pre-fill chunks of assorted sizes: len advances by n, and every
    streaming slot reports the position the oracle's replay of the slot rule puts there."""
    S, W = 3, 7
    mask = np.array([[1, 0, 0, 1]], dtype=np.uint8)
    st, h, _ = _create(layers=1, mask=mask, S=S, W=W, max_len=200)
    assert st == duo.DUO_OK
    chunks, n_total = [1, 5, 2, 9, 1, 30, 4], 0
    for i, n in enumerate(chunks):
        if i % 2:
            assert duo.duo_prefill_chunk(h, 0, FAKE, FAKE, FAKE, n, FAKE, None) == duo.DUO_OK
        else:
            assert duo.duo_append_kv(h, 0, FAKE, FAKE, n) == duo.DUO_OK
        n_total += n
        assert duo.duo_cache_len(h, 0) == (duo.DUO_OK, n_total)
        replay = oracle.ring_replay(S, W, chunks[:i + 1])[-1]
        for slot in range(S + W):
            assert duo.duo_debug_slot_position(h, 0, 1, slot) == (duo.DUO_OK, int(replay[slot]))
    assert duo.duo_decode_attention(h, 0, FAKE, FAKE, None) == duo.DUO_OK
    assert duo.duo_get_device_status(h) == duo.DUO_OK
    duo.duo_cache_destroy(h)


def _fail_nth(h, call, n):
    """Runs `call` with launch attempt n (0-based) failing; returns its status and len."""
    assert duo.duo_debug_launch_controls(1, n) == duo.DUO_OK
    st = call()
    assert duo.duo_debug_launch_controls(1, -1) == duo.DUO_OK
    return st, duo.duo_cache_len(h, 0)[1]


@pytest.mark.parametrize("call,launches,appends_at", [
    # (call, its launches here, index of the launch that writes the cache)
    ("append_kv", 1, 0),
    ("prefill_first", 2, 1),      # attention, append (no streaming history yet)
    ("prefill_later", 3, 2),      # history staging, attention, append
    ("decode", 1, None),
    ("append_decode", 2, 0),      # append, then attention (the two-launch path)
])
def test_failed_launch_keeps_the_length_contract(dry_run, call, launches, appends_at):
    """Each launch of each call fails in turn: the call returns DUO_ERR_CUDA, and len
    advances exactly when the launch that writes the cache was accepted -- which, the
    cache being written by the last launch of every call but duo_append_decode's
    two-launch path, means a failed call leaves the cache unchanged."""
    mask = np.array([[1, 0, 0, 1]], dtype=np.uint8)
    n = 6
    for k in range(launches + 1):
        st, h, _ = _create(layers=1, mask=mask, S=2, W=4, max_len=100)
        if call in ("prefill_later", "decode", "append_decode"):
            assert duo.duo_append_kv(h, 0, FAKE, FAKE, 10) == duo.DUO_OK
        len0 = duo.duo_cache_len(h, 0)[1]
        fns = {
            "append_kv": lambda: duo.duo_append_kv(h, 0, FAKE, FAKE, n),
            "prefill_first": lambda: duo.duo_prefill_chunk(h, 0, FAKE, FAKE, FAKE, n, FAKE, None),
            "prefill_later": lambda: duo.duo_prefill_chunk(h, 0, FAKE, FAKE, FAKE, n, FAKE, None),
            "decode": lambda: duo.duo_decode_attention(h, 0, FAKE, FAKE, None),
            "append_decode": lambda: duo.duo_append_decode(h, 0, FAKE, FAKE, FAKE, FAKE, None),
        }
        st, len1 = _fail_nth(h, fns[call], k)
        grew = {"append_decode": 1, "decode": 0}.get(call, n)
        if k == launches:  # no launch failed
            assert st == duo.DUO_OK and len1 == len0 + grew
        else:
            assert st == duo.DUO_ERR_CUDA
            appended = appends_at is not None and k > appends_at
            assert len1 == len0 + (grew if appended else 0), (call, k)
        duo.duo_cache_destroy(h)


def test_gated_launch_failure_is_reported(dry_run):
    for k, want in [(0, duo.DUO_ERR_CUDA), (1, duo.DUO_ERR_CUDA), (2, duo.DUO_OK)]:
        assert duo.duo_debug_launch_controls(1, k) == duo.DUO_OK
        st = duo.duo_gated_attention(FAKE, FAKE, FAKE, 1, 100, 4, 2, 64, duo.DUO_FP32, FAKE, 2, 8, 0.0, FAKE)
        assert st == want, k
    assert duo.duo_debug_launch_controls(1, -1) == duo.DUO_OK
