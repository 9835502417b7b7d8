"""The allocation-free decode entry point (duo_decode_attention_static_scratch).

Some callers cannot allocate device memory when they decode (code under CUDA graph
capture, runtimes whose device memory is a pool sized at start-up).  The entry point
keeps its split-KV scratch in a static device array instead; this test calls it
through the C ABI, twice in a row, and checks each result against the regular
duo_decode_attention on the same cache and query, within the bf16 parity tolerance
of the other tests.  The file is collected last so that a failure here leaves every
other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

from head_split_kv_duo_b200 import duo, inputs
from head_split_kv_duo_b200.duo import DuoCache
from parity import assert_close

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
