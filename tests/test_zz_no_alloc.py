"""The allocation-free decode entry point (duo_decode_attention_static_scratch).

Some callers cannot allocate device memory when they decode: a serving runtime whose
device memory is a pool it sized once at start-up, or a caller held to a fixed memory
budget.  The entry point keeps its split-KV scratch in a static device array instead;
this test calls it through the C ABI, twice in a row, and checks each result against
the regular duo_decode_attention on the same cache and query and against the fp64
oracle, within the bf16 parity tolerance of the other tests; it also checks the
requests the entry point refuses.  The file is collected last so that a failure here
leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

from head_split_kv_duo_b200 import duo, inputs
from head_split_kv_duo_b200.duo import DuoCache
from parity import assert_close, oracle_rows

pytestmark = pytest.mark.gpu


def _static_decode(cache, layer, q, out, lse):
    fn = duo.lib().duo_decode_attention_static_scratch
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return fn(cache.handle, layer, q.data_ptr(), out.data_ptr(), lse.data_ptr(),
              torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,Hq,Hkv,nret,ctx", [(1, 32, 8, 4, 20000), (2, 32, 32, 8, 3000)])
def test_static_scratch_decode_matches_regular_decode(B, Hq, Hkv, nret, ctx):
    mask = inputs.retrieval_mask(1, Hkv, nret, seed=3)
    steps = 2
    T = ctx + steps
    q = inputs.randn((B, steps, Hq, 128), 300, device="cuda")
    k = inputs.randn((B, T, Hkv, 128), 301, device="cuda")
    v = inputs.randn((B, T, Hkv, 128), 302, device="cuda")
    cache = DuoCache(1, Hkv, 128, mask, 16, 512, T, batch=B, q_heads=Hq, dtype=torch.bfloat16)
    cache.append_kv(0, k[:, :ctx].contiguous(), v[:, :ctx].contiguous())
    for t in range(steps):  # two calls in a row, each after one more appended token
        cache.append_kv(0, k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous())
        qt = q[:, t].contiguous()
        want, want_lse = cache.decode_attention(0, qt)
        out = torch.empty_like(qt)
        lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        assert _static_decode(cache, 0, qt, out, lse) == duo.DUO_OK
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        assert_close(out.float().cpu().numpy(), want.float().cpu().numpy(), torch.bfloat16,
                     lse.cpu().numpy(), want_lse.cpu().numpy(), f"static scratch call {t}")
        ref, ref_lse = oracle_rows(q[:, t:t + 1], k[:, :ctx + t + 1], v[:, :ctx + t + 1], mask[0], 16, 512, ctx + t)
        assert_close(out.float().cpu().numpy()[:, None], ref, torch.bfloat16, lse.cpu().numpy()[:, None], ref_lse,
                     f"static scratch call {t} against the oracle")


def test_static_scratch_refusals():
    """Requests outside the entry point's limits are refused before any launch: a layer
    with no token yet (DUO_ERR_INVALID), an INT4 retrieval cache (DUO_ERR_UNSUPPORTED),
    and more heads' partial results than the 4 MiB array holds at one CTA
    (DUO_ERR_CAPACITY: 256 sequences x 32 KV heads x (128 + 4) floats)."""
    d = 128
    k = inputs.randn((1, 1, 8, d), 310, device="cuda")
    q = inputs.randn((1, 8, d), 311, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty(1, 8, dtype=torch.float32, device="cuda")
    empty = DuoCache(2, 8, d, inputs.retrieval_mask(2, 8, 4, seed=4), 16, 512, 64, dtype=torch.bfloat16)
    empty.append_kv(0, k, k)  # layer 1 stays empty
    assert _static_decode(empty, 1, q, out, lse) == duo.DUO_ERR_INVALID
    i4 = DuoCache(1, 8, d, inputs.retrieval_mask(1, 8, 4, seed=4), 16, 512, 64, dtype=torch.bfloat16,
                  retr_fmt="int4")
    i4.append_kv(0, k, k)
    assert _static_decode(i4, 0, q, out, lse) == duo.DUO_ERR_UNSUPPORTED
    B, Hkv = 256, 32
    mask = torch.zeros(1, Hkv, dtype=torch.uint8)
    mask[0, 0] = 1
    big = DuoCache(1, Hkv, d, mask, 1, 1, 4, batch=B, dtype=torch.bfloat16)
    kb = inputs.randn((B, 1, Hkv, d), 312, device="cuda")
    big.append_kv(0, kb, kb)
    qb = inputs.randn((B, Hkv, d), 313, device="cuda")
    ob = torch.empty_like(qb)
    lb = torch.empty(B, Hkv, dtype=torch.float32, device="cuda")
    assert _static_decode(big, 0, qb, ob, lb) == duo.DUO_ERR_CAPACITY
    torch.cuda.synchronize()
    for cache in (empty, i4, big):
        assert cache.device_status() == 0
