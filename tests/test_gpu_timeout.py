"""The device timeout path on a GPU, made without a fault: a test control
(duo_debug_device_stall) makes the bf16 decode's softmax wait for a barrier that nothing
arrives at.  The bounded wait runs out (about 2 s), the kernel latches the timeout in the
cache's status word and every role drains and exits; the context stays usable, and the
same cache then decodes like the oracle (the split merge's tickets were left consistent)."""
import time

import pytest
import torch

import oracle
from head_split_kv_duo_b200 import duo, inputs
from head_split_kv_duo_b200.duo import DuoCache
from parity import assert_close, bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_decode_wait_runs_out_and_the_context_survives():
    """Llama-3-8B layer shape (32 q / 8 kv heads, 4 retrieval, S 16, W 512) at 3000
    tokens: a stalled decode reports DUO_ERR_TIMEOUT after about the wait limit; the
    next decode of the same cache and of a fresh cache match the oracle."""
    mask = inputs.retrieval_mask(1, 8, 4, seed=1)
    T = 3000
    k = inputs.randn((1, T, 8, 128), 600, device=DEV)
    v = inputs.randn((1, T, 8, 128), 601, device=DEV)
    q = inputs.randn((1, 32, 128), 602, device=DEV)
    cache = DuoCache(1, 8, 128, mask, 16, 512, T + 8, q_heads=32, dtype=torch.bfloat16)
    cache.append_kv(0, k, v)
    torch.cuda.synchronize()
    assert cache.device_status() == duo.DUO_OK
    assert duo.duo_debug_device_stall(1) == duo.DUO_OK
    try:
        t0 = time.perf_counter()
        cache.decode_attention(0, q)      # the launch itself is accepted
        status = cache.device_status()    # synchronises, reads and clears the status word
        seconds = time.perf_counter() - t0
    finally:
        assert duo.duo_debug_device_stall(0) == duo.DUO_OK
    assert status == duo.DUO_ERR_TIMEOUT
    assert 1.0 < seconds < 60.0, seconds
    assert cache.device_status() == duo.DUO_OK  # the word was cleared by the read

    want, want_lse = oracle.attend(bits(q[:, None]), bits(k), bits(v), mask[0].numpy().astype(bool), 16, 512,
                                   pos0=T - 1)
    for c in (cache, None):
        if c is None:
            c = DuoCache(1, 8, 128, mask, 16, 512, T + 8, q_heads=32, dtype=torch.bfloat16)
            c.append_kv(0, k, v)
        o, lse = c.decode_attention(0, q)
        torch.cuda.synchronize()
        assert c.device_status() == duo.DUO_OK
        assert_close(o.float().cpu().numpy()[:, None], want, torch.bfloat16, lse.cpu().numpy()[:, None], want_lse,
                     "decode after a timed-out decode")
