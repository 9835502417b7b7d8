"""GPU parity: the C-ABI path (libduo.so kernels) against the fp64 oracle, element
by element on seeded inputs, for the five workloads (reduced sizes that span
several tiles and a ragged tail, plus sampled outputs at full size) and the
degenerate cases of the method."""
import math

import numpy as np
import pytest
import torch

import oracle
from head_split_kv_duo_b200 import inputs
from head_split_kv_duo_b200 import duo
from head_split_kv_duo_b200.duo import DuoCache, DuoError
from parity import assert_close, bits, errors, oracle_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _seq(B, T, Hq, Hkv, d, dtype, seed):
    q = inputs.randn((B, T, Hq, d), seed, dtype, DEV)
    k = inputs.randn((B, T, Hkv, d), seed + 1, dtype, DEV)
    v = inputs.randn((B, T, Hkv, d), seed + 2, dtype, DEV)
    return q, k, v


def _run(cache, q, k, v, chunks, decode_steps):
    """Pre-fill the first sum(chunks) tokens in the given chunks, then decode
    `decode_steps` tokens (append then attend).  Returns per-position outputs
    [B][T][Hq][d] (fp32) and lse [B][T][Hq]."""
    outs, lses = [], []
    pos = 0
    for n in chunks:
        o, l = cache.prefill_chunk(0, q[:, pos:pos + n].contiguous(), k[:, pos:pos + n].contiguous(),
                                   v[:, pos:pos + n].contiguous())
        outs.append(o.float())
        lses.append(l)
        pos += n
    for _ in range(decode_steps):
        cache.append_kv(0, k[:, pos:pos + 1].contiguous(), v[:, pos:pos + 1].contiguous())
        o, l = cache.decode_attention(0, q[:, pos].contiguous())
        outs.append(o.float()[:, None])
        lses.append(l[:, None])
        pos += 1
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    return torch.cat(outs, 1).cpu().numpy(), torch.cat(lses, 1).cpu().numpy()


# ------------------------------------------------------------ tiny hybrid MHA

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunks", [[256], [37] * 6 + [34], [1] * 40 + [216]])
def test_tiny_mha_prefill_then_decode(dtype, chunks):
    """8 heads, d 64, heads {1,5} retrieval, S 4, W 16; pre-fill 256 tokens (whole,
    in chunks of 37, token by token), then 16 decode steps."""
    B, Hq, Hkv, d, S, W, steps = 1, 8, 8, 64, 4, 16, 16
    mask = inputs.fixed_mask(8, (1, 5))
    T = 256 + steps
    q, k, v = _seq(B, T, Hq, Hkv, d, dtype, 0)
    cache = DuoCache(1, Hkv, d, mask, S, W, T, q_heads=Hq, dtype=dtype)
    got, got_lse = _run(cache, q, k, v, chunks, steps)
    want, want_lse = oracle_rows(q, k, v, mask[0], S, W, 0)
    assert_close(got, want, dtype, got_lse, want_lse, f"tiny {dtype} {chunks[:2]}")


def test_chunking_does_not_change_results():
    """Chunked pre-fill with any partition equals single-chunk pre-fill (reading: every
    query row uses the Lambda mask of its own position)."""
    B, Hq, Hkv, d, S, W = 2, 8, 4, 128, 8, 100
    mask = torch.tensor([[0, 1, 0, 0]], dtype=torch.uint8)
    T = 700
    q, k, v = _seq(B, T, Hq, Hkv, d, torch.float32, 5)
    res = []
    for chunks in ([700], [128, 200, 1, 371], [99] * 7 + [7]):
        cache = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=torch.float32)
        res.append(_run(cache, q, k, v, chunks, 0))
    for o, l in res[1:]:
        np.testing.assert_allclose(o, res[0][0], atol=2e-6, rtol=0)
        np.testing.assert_allclose(l, res[0][1], atol=2e-6, rtol=0)


# ------------------------------------------------------ cache bookkeeping

def _check_cache_rows(cache, k, v, T):
    """Every retrieval row equals its input row; every streaming slot holds the input
    row of the position the host bookkeeping reports, bit for bit; slot positions
    match the oracle's replay."""
    B, Hkv, d = cache.batch, cache.kv_heads, cache.head_dim
    esize = 2 if cache.dtype == torch.bfloat16 else 4
    mask = cache.mask[0].tolist()
    ridx = [g for g in range(Hkv) if mask[g]]
    sidx = [g for g in range(Hkv) if not mask[g]]
    rk, cap = cache.region(0, duo.DUO_REGION_RETR_K)
    rv, _ = cache.region(0, duo.DUO_REGION_RETR_V)
    sk, _ = cache.region(0, duo.DUO_REGION_STRM_K)
    sv, _ = cache.region(0, duo.DUO_REGION_STRM_V)
    tdt = cache.dtype
    kb = k.view(torch.int16) if esize == 2 else k.view(torch.int32)
    vb = v.view(torch.int16) if esize == 2 else v.view(torch.int32)
    idt = torch.int16 if esize == 2 else torch.int32
    if ridx:
        R = rk.view(idt).view(B, len(ridx), cap, d)
        RV = rv.view(idt).view(B, len(ridx), cap, d)
        for i, g in enumerate(ridx):
            assert torch.equal(R[:, i, :T], kb[:, :T, g]) and torch.equal(RV[:, i, :T], vb[:, :T, g])
    if sidx:
        nsl = cache.S + cache.W
        SK = sk.view(idt).view(B, len(sidx), nsl, d)
        SV = sv.view(idt).view(B, len(sidx), nsl, d)
        replay = oracle.ring_replay(cache.S, cache.W, [T])[0]
        for i, g in enumerate(sidx):
            for slot in range(nsl):
                pos = cache.slot_position(0, g, slot)
                assert pos == replay[slot], (slot, pos, replay[slot])
                if pos >= 0:
                    assert torch.equal(SK[:, i, slot], kb[:, pos, g]) and torch.equal(SV[:, i, slot], vb[:, pos, g])


@pytest.mark.parametrize("chunks", [[5], [3, 4, 9], [1] * 23, [64, 1, 1, 70], [600]])
@pytest.mark.parametrize("S,W", [(1, 2), (4, 16), (0, 7), (16, 64)])
def test_cache_rows_and_slots_bit_exact(chunks, S, W):
    B, Hkv, d = 2, 4, 64
    mask = torch.tensor([[1, 0, 0, 1]], dtype=torch.uint8)
    T = sum(chunks)
    _, k, v = _seq(B, T, Hkv, Hkv, d, torch.bfloat16, 9)
    cache = DuoCache(1, Hkv, d, mask, S, W, T + 3, batch=B, dtype=torch.bfloat16)
    pos = 0
    for n in chunks:
        cache.append_kv(0, k[:, pos:pos + n].contiguous(), v[:, pos:pos + n].contiguous())
        pos += n
        torch.cuda.synchronize()
        _check_cache_rows(cache, k, v, pos)
    assert cache.len(0) == T


def test_fig5_worked_example_on_device():
    """'Chunked Pre-filling', Figure 5 (right): S 1, W 2, chunks of 4 -> the streaming
    head holds {0, 2, 3} after chunk 1 and {0, 6, 7} after chunk 2."""
    d = 64
    mask = torch.tensor([[0]], dtype=torch.uint8)
    q, k, v = _seq(1, 8, 1, 1, d, torch.float32, 3)
    cache = DuoCache(1, 1, d, mask, 1, 2, 8, dtype=torch.float32)
    held = []
    for c in range(2):
        sl = slice(4 * c, 4 * c + 4)
        cache.prefill_chunk(0, q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous())
        torch.cuda.synchronize()
        held.append(sorted(p for p in (cache.slot_position(0, 0, s) for s in range(3)) if p >= 0))
        _check_cache_rows(cache, k, v, 4 * c + 4)
    assert held == [[0, 2, 3], [0, 6, 7]]


# ------------------------------------------------------------- decode shapes

def _fill_and_decode(Hq, Hkv, d, mask, S, W, B, ctx, steps, seed, dtype=torch.bfloat16, retr_fmt="same",
                     rows_per_check=None):
    T = ctx + steps
    q = inputs.randn((B, steps, Hq, d), seed, dtype, DEV)
    k = inputs.randn((B, T, Hkv, d), seed + 1, dtype, DEV)
    v = inputs.randn((B, T, Hkv, d), seed + 2, dtype, DEV)
    cache = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=dtype, retr_fmt=retr_fmt)
    if ctx > 0:
        cache.append_kv(0, k[:, :ctx].contiguous(), v[:, :ctx].contiguous())
    outs, lses = [], []
    for t in range(steps):
        cache.append_kv(0, k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous())
        o, l = cache.decode_attention(0, q[:, t].contiguous())
        outs.append(o.float()[:, None])
        lses.append(l[:, None])
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    return cache, q, k, v, torch.cat(outs, 1).cpu().numpy(), torch.cat(lses, 1).cpu().numpy()


def _decode_oracle(q, k, v, mask_row, S, W, ctx, steps):
    """Oracle for each decode step t (query position ctx + t, history 0..ctx+t)."""
    ws, ls = [], []
    for t in range(steps):
        w, l = oracle_rows(q[:, t:t + 1], k[:, :ctx + t + 1], v[:, :ctx + t + 1], mask_row, S, W, ctx + t)
        ws.append(w)
        ls.append(l)
    return np.concatenate(ws, 1), np.concatenate(ls, 1)


@pytest.mark.parametrize("B,ctx", [(1, 4095), (8, 3000), (1, 32768), (8, 32768)])
def test_llama2_mha_decode(B, ctx):
    """Llama-2-7B-shaped layer: 32 heads, d 128, 8 retrieval (seeded), S 16, W 512."""
    mask = inputs.retrieval_mask(1, 32, 8, seed=0)
    steps = 2
    _, q, k, v, got, got_lse = _fill_and_decode(32, 32, 128, mask, 16, 512, B, ctx, steps, 10)
    want, want_lse = _decode_oracle(q, k, v, mask[0], 16, 512, ctx, steps)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"llama2 B{B} ctx{ctx}")


@pytest.mark.parametrize("B,ctx", [(1, 5000), (4, 1 << 17), (1, 1 << 17)])
def test_llama3_gqa_decode(B, ctx):
    """Llama-3-8B-shaped layer: 32 q / 8 kv heads (group 4), d 128, 4 retrieval, S 16, W 512."""
    mask = inputs.retrieval_mask(1, 8, 4, seed=1)
    steps = 2
    _, q, k, v, got, got_lse = _fill_and_decode(32, 8, 128, mask, 16, 512, B, ctx, steps, 20)
    want, want_lse = _decode_oracle(q, k, v, mask[0], 16, 512, ctx, steps)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"llama3 B{B} ctx{ctx}")


@pytest.mark.parametrize("ctx", [1, 2, 15, 16, 17, 113, 120, 128, 250, 256, 400, 500, 512, 513, 527, 528, 529,
                                 1000])
def test_decode_short_contexts_and_boundaries(ctx):
    """len around S and S + W; the first query sees only itself.  Before the ring wraps
    (S < len <= W) position p sits in slot S + p, so the newest tokens lie in slots past
    len: lengths whose last slots cross into a further 128-slot tile (113..128, 250,
    256, 400, 500, 512) catch a kernel that scans only the first len slots."""
    mask = torch.tensor([[1, 0]], dtype=torch.uint8)
    _, q, k, v, got, got_lse = _fill_and_decode(4, 2, 128, mask, 16, 512, 2, ctx - 1, 1, 30)
    want, want_lse = _decode_oracle(q, k, v, mask[0], 16, 512, ctx - 1, 1)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"ctx {ctx}")


@pytest.mark.parametrize("S,W,mask", [(0, 1, [0, 0]), (0, 64, [0, 0]), (3, 1, [0, 1]), (0, 5, [1, 1]),
                                      (700, 9, [0, 0]), (2, 3000, [0, 0])])
def test_degenerate_settings(S, W, mask):
    """S = 0 (pure sliding window), W = 1 (only the current token), all-retrieval,
    all-streaming, S or W beyond the sequence."""
    m = torch.tensor([mask], dtype=torch.uint8)
    for dtype in (torch.bfloat16, torch.float32):
        T = 1200
        q, k, v = _seq(1, T, 4, 2, 64, dtype, 40)
        cache = DuoCache(1, 2, 64, m, S, W, T, q_heads=4, dtype=dtype)
        got, got_lse = _run(cache, q, k, v, [500, 300, 390], 10)
        want, want_lse = oracle_rows(q, k, v, m[0], S, W, 0)
        assert_close(got, want, dtype, got_lse, want_lse, f"S{S} W{W} {mask} {dtype}")


def test_capacity_is_enforced_on_device():
    mask = torch.tensor([[1, 0]], dtype=torch.uint8)
    q, k, v = _seq(1, 10, 2, 2, 64, torch.bfloat16, 50)
    cache = DuoCache(1, 2, 64, mask, 2, 4, 8, dtype=torch.bfloat16, q_heads=2)
    cache.append_kv(0, k[:, :8].contiguous(), v[:, :8].contiguous())
    with pytest.raises(DuoError) as e:
        cache.append_kv(0, k[:, 8:9].contiguous(), v[:, 8:9].contiguous())
    assert e.value.status == duo.DUO_ERR_CAPACITY and cache.len(0) == 8
    o, _ = cache.decode_attention(0, q[:, 7].contiguous())  # still usable at capacity
    want, _ = oracle_rows(q[:, 7:8], k[:, :8], v[:, :8], mask[0], 2, 4, 7)
    assert_close(o.float().cpu().numpy()[:, None], want, torch.bfloat16)


# ------------------------------------------------------ planted needle, masks

def _planted(ctx, d=128, seed=60):
    """GQA 8 q / 2 kv heads (kv 0 retrieval, kv 1 streaming), S 16, W 512: keys at a
    middle position and at the window / sink boundaries planted to dominate."""
    Hq, Hkv, S, W = 8, 2, 16, 512
    mask = torch.tensor([[1, 0]], dtype=torch.uint8)
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(1, 1, Hq, d, generator=g)
    k = torch.randn(1, ctx, Hkv, d, generator=g)
    v = torch.randn(1, ctx, Hkv, d, generator=g)
    i = ctx - 1
    needles = {"middle": ctx // 2, "window_edge": i - W + 1, "outside": i - W, "sink_edge": S - 1, "post_sink": S}
    values = {"middle": 0.2, "window_edge": 0.6, "outside": 1.0, "sink_edge": 1.8, "post_sink": 2.6}
    for name, j in needles.items():
        for kv in range(Hkv):
            qq = q[0, 0, kv * 4]
            k[0, j, kv] = 6.0 * qq / qq.norm() * math.sqrt(d) * (1.05 if name == "outside" else 1.0)
            v[0, j, kv] = values[name]
    return [t.to(torch.bfloat16).to(DEV) for t in (q, k, v)], mask, needles, S, W


def test_planted_needle_and_mask_discrimination():
    ctx = 9000
    (q, k, v), mask, needles, S, W = _planted(ctx)
    cache = DuoCache(1, 2, 128, mask, S, W, ctx, q_heads=8, dtype=torch.bfloat16)
    cache.append_kv(0, k.contiguous(), v.contiguous())
    o, lse = cache.decode_attention(0, q[:, 0].contiguous())
    torch.cuda.synchronize()
    got = o.float().cpu().numpy()[:, None]
    want, want_lse = oracle_rows(q, k, v, mask[0], S, W, ctx - 1)
    assert_close(got, want, torch.bfloat16, lse.cpu().numpy()[:, None], want_lse, "planted")
    # retrieval query head 0 recovers the strongest needle (value 1.0, outside the
    # window); streaming query head 4 sees only the window-edge and sink needles
    # (values 0.6 and 1.8, equal logits) and nothing of the middle or outside ones
    # (planted values stay O(1) so that bf16 output rounding is within tolerance)
    assert abs(got[0, 0, 0].mean() - 1.0) < 0.1
    assert abs(got[0, 0, 4].mean() - 1.2) < 0.1
    # each wrong reading of the mask moves the answer by far more than the tolerance
    for wrong in [dict(W=W + 1), dict(W=W - 1), dict(S=S + 1), dict(S=S - 1), dict(mask=[1, 1]), dict(mask=[0, 0])]:
        m = wrong.get("mask", mask[0].tolist())
        w2, _ = oracle_rows(q, k, v, m, wrong.get("S", S), wrong.get("W", W), ctx - 1)
        assert np.abs(w2 - got).max() > 0.1, f"reading {wrong} is not distinguishable"


# ------------------------------------------------------------------- INT4

def _int4_reference(k_rows):
    """oracle quantisation of bf16 rows [..., 128] -> codes, scale bits, zero bits, dequantised fp64."""
    b = bits(k_rows).reshape(-1, 128)
    codes, sb, zb = oracle.int4_quantize(b)
    return codes, sb, zb, oracle.int4_dequantize(codes, sb, zb)


@pytest.mark.parametrize("B,ctx", [(1, 3000), (2, 20000)])
def test_int4_codes_bit_exact_and_decode(B, ctx):
    Hq, Hkv, d, S, W = 32, 8, 128, 16, 512
    mask = inputs.retrieval_mask(1, 8, 4, seed=2)
    steps = 2
    cache, q, k, v, got, got_lse = _fill_and_decode(Hq, Hkv, d, mask, S, W, B, ctx, steps, 70, retr_fmt="int4")
    T = ctx + steps
    ridx = [g for g in range(Hkv) if mask[0, g]]
    rk, cap = cache.region(0, duo.DUO_REGION_RETR_K)
    rv, _ = cache.region(0, duo.DUO_REGION_RETR_V)
    ks, _ = cache.region(0, duo.DUO_REGION_RETR_KSZ)
    vs, _ = cache.region(0, duo.DUO_REGION_RETR_VSZ)
    RK = rk.view(B, len(ridx), cap, 64)[:, :, :T].cpu().numpy()
    RV = rv.view(B, len(ridx), cap, 64)[:, :, :T].cpu().numpy()
    KS = ks.view(torch.int16).view(B, len(ridx), cap, 2)[:, :, :T].cpu().numpy().view(np.uint16)
    VS = vs.view(torch.int16).view(B, len(ridx), cap, 2)[:, :, :T].cpu().numpy().view(np.uint16)
    # the oracle's own quantisation, dequantised in fp64, stands in for the retrieval rows
    kq = k.float().cpu().numpy().astype(np.float64)
    vq = v.float().cpu().numpy().astype(np.float64)
    for i, g in enumerate(ridx):
        for src, C, Z, dst in ((k, RK, KS, kq), (v, RV, VS, vq)):
            codes, sb, zb, deq = _int4_reference(src[:, :, g])
            assert np.array_equal(C[:, i].reshape(-1, 64), codes), "INT4 codes differ"
            assert np.array_equal(Z[:, i, :, 0].reshape(-1), sb) and np.array_equal(Z[:, i, :, 1].reshape(-1), zb)
            dst[:, :, g] = deq.reshape(B, T, 128)
    ws, ls = [], []
    for t in range(steps):
        w, l = oracle.attend(bits(q[:, t:t + 1]), kq[:, :ctx + t + 1], vq[:, :ctx + t + 1], mask[0].numpy().astype(bool),
                             S, W, pos0=ctx + t)
        ws.append(w)
        ls.append(l)
    assert_close(got, np.concatenate(ws, 1), torch.bfloat16, got_lse, np.concatenate(ls, 1), "int4 decode")
    # for information: distance to attention over the unquantised bf16 values
    ref, _ = _decode_oracle(q, k, v, mask[0], S, W, ctx, steps)
    print("int4 vs unquantised:", errors(got, ref))


def _int4_decode_check(Hq, Hkv, mask_row, S, W, B, ctx, steps, seed, plant=False):
    """Append ctx tokens, then `steps` decode steps, on an INT4 retrieval cache; compare
    with the oracle over the oracle's own dequantisation of the retrieval rows.  With
    `plant`, one middle key of every retrieval head is set to 3x the first query of its
    group (so that query's attention concentrates there) and its value to a ramp."""
    d, T, G = 128, ctx + steps, Hq // Hkv
    mask = torch.tensor([mask_row], dtype=torch.uint8)
    q = inputs.randn((B, steps, Hq, d), seed, torch.bfloat16, DEV)
    k = inputs.randn((B, T, Hkv, d), seed + 1, torch.bfloat16, DEV)
    v = inputs.randn((B, T, Hkv, d), seed + 2, torch.bfloat16, DEV)
    ridx = [g for g in range(Hkv) if mask_row[g]]
    if plant and ctx > 2:
        P = ctx // 2
        ramp = torch.linspace(-2.0, 2.0, d, device=DEV).to(torch.bfloat16)
        for g in ridx:
            k[:, P, g] = (3.0 * q[:, 0, g * G].float()).to(torch.bfloat16)
            v[:, P, g] = ramp
    cache = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=torch.bfloat16, retr_fmt="int4")
    if ctx > 0:
        cache.append_kv(0, k[:, :ctx].contiguous(), v[:, :ctx].contiguous())
    outs, lses = [], []
    for t in range(steps):
        cache.append_kv(0, k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous())
        o, l = cache.decode_attention(0, q[:, t].contiguous())
        outs.append(o.float()[:, None])
        lses.append(l[:, None])
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    got, got_lse = torch.cat(outs, 1).cpu().numpy(), torch.cat(lses, 1).cpu().numpy()
    kq = k.float().cpu().numpy().astype(np.float64)
    vq = v.float().cpu().numpy().astype(np.float64)
    for g in ridx:
        for src, dst in ((k, kq), (v, vq)):
            dst[:, :, g] = _int4_reference(src[:, :, g])[3].reshape(B, T, d)
    ws, ls = [], []
    for t in range(steps):
        w, l = oracle.attend(bits(q[:, t:t + 1]), kq[:, :ctx + t + 1], vq[:, :ctx + t + 1],
                             np.asarray(mask_row, dtype=bool), S, W, pos0=ctx + t)
        ws.append(w)
        ls.append(l)
    want, want_lse = np.concatenate(ws, 1), np.concatenate(ls, 1)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"int4 decode Hq{Hq} Hkv{Hkv} B{B} ctx{ctx}")
    return got, want


@pytest.mark.parametrize("Hq,Hkv,mask_row,S,W,B,ctx", [
    (8, 8, [1, 0, 1, 0, 0, 0, 0, 1], 4, 32, 1, 0),        # first token: sees only itself
    (8, 8, [1, 0, 1, 0, 0, 0, 0, 1], 4, 32, 2, 37),       # MHA, one ragged tile
    (16, 8, [1] * 8, 16, 64, 1, 3000),                     # all retrieval, group 2
    (32, 4, [0, 0, 0, 0], 16, 512, 2, 2000),               # all streaming (bf16 pieces only)
    (64, 4, [1, 0, 1, 1], 16, 512, 1, 5000),               # group 16
    (32, 4, [0, 1, 1, 0], 0, 100, 3, 1000),                # group 8, no sinks
    (32, 8, [0, 1, 0, 1, 1, 0, 0, 1], 16, 512, 1, 1 << 18),  # Llama-3 shape, 256K
    (32, 8, [0, 1, 0, 1, 1, 0, 0, 1], 16, 512, 1, 250),      # ring slots past len (tile 2)
    (32, 8, [1, 0, 1, 0, 1, 0, 1, 0], 16, 512, 2, 118),      # ring slots past len (tile 1)
])
def test_int4_tc_decode_shapes(Hq, Hkv, mask_row, S, W, B, ctx):
    _int4_decode_check(Hq, Hkv, mask_row, S, W, B, ctx, 2, 90)


@pytest.mark.parametrize("Hq,Hkv,B,ctx", [(32, 8, 1, 20000), (8, 8, 2, 5000)])
def test_int4_tc_decode_planted_needle(Hq, Hkv, B, ctx):
    """Concentrated attention: the bf16 rounding of p s_v that the MMA sees is
    compensated exactly, so the output still matches the oracle to bf16 accuracy."""
    mask_row = [1, 0] * (Hkv // 2)
    got, want = _int4_decode_check(Hq, Hkv, mask_row, 16, 512, B, ctx, 1, 95, plant=True)
    G = Hq // Hkv
    ramp = np.linspace(-2.0, 2.0, 128)
    for g in range(0, Hkv, 2):  # retrieval heads recover the planted ramp
        assert np.abs(want[:, 0, g * G] - ramp).max() < 0.3
        assert np.abs(got[:, 0, g * G] - ramp).max() < 0.3


# -------------------------------------------------- tensor-core pre-fill (bf16, d 128)

@pytest.mark.parametrize("B,Hq,Hkv,mask,S,W,chunks", [
    (1, 8, 2, [1, 0], 4, 32, [300]),
    (2, 4, 4, [1, 0, 1, 0], 16, 512, [1000, 129, 1, 500]),
    (1, 32, 8, [1, 0, 0, 1, 1, 0, 0, 1], 16, 512, [1024, 1024, 1024, 1024]),
    (1, 4, 2, [0, 0], 0, 1, [257, 255]),
    (1, 4, 2, [0, 0], 200, 3, [130, 140, 90]),
    (1, 4, 2, [1, 1], 3, 7, [640, 17]),
    (1, 8, 1, [0], 5, 300, [77, 600, 129]),
])
def test_tc_prefill_parity(B, Hq, Hkv, mask, S, W, chunks):
    """Chunked pre-fill through the tensor-core kernel against the oracle, rows of
    every chunk; shapes cover ragged tails, sinks inside and beyond one tile,
    windows narrower and wider than a tile, MHA and GQA, B > 1."""
    m = torch.tensor([mask], dtype=torch.uint8)
    T = sum(chunks)
    q, k, v = _seq(B, T, Hq, Hkv, 128, torch.bfloat16, 80)
    cache = DuoCache(1, Hkv, 128, m, S, W, T, batch=B, q_heads=Hq, dtype=torch.bfloat16)
    got, got_lse = _run(cache, q, k, v, chunks, 0)
    want, want_lse = oracle_rows(q, k, v, m[0], S, W, 0)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"tc prefill {chunks}")


def test_llama3_prefill_reduced():
    """Llama-3-8B GQA shape (32 q / 8 kv, 4 retrieval, S 16, W 512), 8K prompt in 2K
    chunks, every output row against the oracle."""
    mask = inputs.retrieval_mask(1, 8, 4, seed=1)
    T, chunk = 8192, 2048
    q, k, v = _seq(1, T, 32, 8, 128, torch.bfloat16, 90)
    cache = DuoCache(1, 8, 128, mask, 16, 512, T, q_heads=32, dtype=torch.bfloat16)
    got, got_lse = _run(cache, q, k, v, [chunk] * (T // chunk), 0)
    want, want_lse = oracle_rows(q, k, v, mask[0], 16, 512, 0)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, "llama3 prefill 8K")


def test_llama3_prefill_full_size_sampled():
    """The benchmarked workload: 256K-token prompt in 32K chunks, Llama-3-8B GQA shape.
    Sampled rows of the first, a middle and the last chunk (first/last rows, rows at
    the S and W boundaries, random rows; all 32 heads) against the oracle."""
    mask = inputs.retrieval_mask(1, 8, 4, seed=1)
    T, chunk = 262144, 32768
    k = inputs.randn((1, T, 8, 128), 200, device=DEV)
    v = inputs.randn((1, T, 8, 128), 201, device=DEV)
    q = inputs.randn((1, chunk, 32, 128), 202, device=DEV)
    cache = DuoCache(1, 8, 128, mask, 16, 512, T, q_heads=32, dtype=torch.bfloat16)
    kb, vb = bits(k), bits(v)
    rng = np.random.default_rng(0)
    for c in range(T // chunk):
        sl = slice(c * chunk, (c + 1) * chunk)
        o, lse = cache.prefill_chunk(0, q, k[:, sl], v[:, sl])
        if c not in (0, 3, 7):
            continue
        torch.cuda.synchronize()
        rows_r = sorted(set([0, 1, 15, 16, 17, 510, 511, 512, 513, chunk - 1] + rng.integers(0, chunk, 12).tolist()))
        ids = [r * 32 + h for r in rows_r for h in range(32)]
        want, want_lse = oracle.attend(bits(q), kb[:, :(c + 1) * chunk], vb[:, :(c + 1) * chunk],
                                       mask[0].numpy().astype(bool), 16, 512, pos0=c * chunk, rows=ids)
        got = o.float()[0, rows_r].reshape(-1, 128).cpu().numpy()
        got_lse = lse[0, rows_r].reshape(-1).cpu().numpy()
        assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"256K prefill chunk {c}")
    assert cache.device_status() == 0


@pytest.mark.parametrize("B,Hq,Hkv,mask,S,W,ctx", [
    (3, 24, 3, [1, 0, 1], 4, 100, 777),
    (2, 16, 2, [0, 1], 16, 512, 20000),
    (1, 16, 1, [1], 0, 8, 300),
    (2, 32, 2, [1, 0], 2, 129, 4097),
    (5, 10, 5, [0, 0, 1, 0, 1], 3, 300, 2500),
])
def test_decode_group_sizes_and_batches(B, Hq, Hkv, mask, S, W, ctx):
    """Query groups of 2, 8, 16 (and 8 on one KV head), odd batch sizes: every item of
    the work split (retrieval and streaming heads of every sequence) against the oracle."""
    m = torch.tensor([mask], dtype=torch.uint8)
    steps = 2
    _, q, k, v, got, got_lse = _fill_and_decode(Hq, Hkv, 128, m, S, W, B, ctx, steps, 110)
    want, want_lse = _decode_oracle(q, k, v, m[0], S, W, ctx, steps)
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, f"decode B{B} G{Hq // Hkv}")


# ------------------------------------------------- gated mixed attention

@pytest.mark.parametrize("dtype,B,L,Hq,Hkv,d,S,W", [
    (torch.float32, 1, 200, 8, 8, 64, 4, 16),        # SIMT pre-fill path
    (torch.bfloat16, 2, 1500, 8, 2, 128, 16, 64),    # tcgen05 pre-fill path, GQA
    (torch.bfloat16, 1, 700, 4, 4, 128, 0, 33),      # no sinks, ragged tiles
])
def test_gated_attention(dtype, B, L, Hq, Hkv, d, S, W):
    """alpha * causal + (1 - alpha) * Lambda per KV head against the oracle, gates
    including the end points 0 and 1."""
    q, k, v = _seq(B, L, Hq, Hkv, d, dtype, 120)
    alpha = torch.linspace(0.0, 1.0, Hkv, dtype=torch.float32)
    got = duo.gated_attention(q, k, v, alpha.to(DEV), S, W)
    torch.cuda.synchronize()
    want = oracle.gated(bits(q), bits(k), bits(v), alpha.numpy(), S, W)
    assert_close(got.float().cpu().numpy(), want, dtype, what=f"gated {dtype} L{L}")


def test_gated_attention_llama3_sampled():
    """Llama-3-8B shape (32 q / 8 kv heads, d 128, S 16, W 512) over an 8K sequence;
    sampled rows: first and last positions, around S and W, and random rows."""
    B, L, Hq, Hkv, d, S, W = 1, 8192, 32, 8, 128, 16, 512
    q, k, v = _seq(B, L, Hq, Hkv, d, torch.bfloat16, 130)
    alpha = torch.rand(Hkv, generator=torch.Generator().manual_seed(5))
    got = duo.gated_attention(q, k, v, alpha.to(DEV), S, W).float().cpu().numpy().reshape(-1, d)
    pos = np.unique(np.concatenate([[0, 1, S - 1, S, S + 1, W - 1, W, W + 1, S + W, L - 1],
                                    np.random.default_rng(7).integers(0, L, 24)]))
    rows = (pos[:, None] * Hq + np.arange(Hq)[None, :]).reshape(-1)
    want = oracle.gated(bits(q), bits(k), bits(v), alpha.numpy(), S, W, rows=rows)
    assert_close(got[rows], want, torch.bfloat16, what="gated llama3 8K sampled")


# ---------------------------------------------- fused append + decode (one launch)

@pytest.mark.parametrize("Hq,Hkv,mask_row,S,W,B,ctx,dtype,fmt", [
    (32, 8, [0, 1, 0, 1, 1, 0, 0, 1], 16, 64, 2, 300, torch.bfloat16, "same"),   # tcgen05 path, ring wraps
    (8, 8, [1, 0, 0, 0, 0, 0, 0, 1], 4, 16, 1, 0, torch.bfloat16, "same"),       # from the first token
    (32, 32, [1] * 8 + [0] * 24, 16, 512, 1, 2000, torch.bfloat16, "same"),       # MHA
    (8, 8, [1, 0, 1, 0, 0, 0, 0, 1], 4, 16, 1, 50, torch.float32, "same"),       # CUDA-core path (two launches)
    (32, 8, [0, 1, 1, 0, 0, 1, 0, 1], 16, 64, 1, 400, torch.bfloat16, "int4"),   # INT4 path (two launches)
])
def test_append_decode_equals_append_then_decode(Hq, Hkv, mask_row, S, W, B, ctx, dtype, fmt):
    """duo_append_decode leaves exactly the cache duo_append_kv writes and returns exactly
    what duo_decode_attention returns, step after step across ring wrap-around."""
    d = 128 if dtype == torch.bfloat16 else 64
    steps = 70
    T = ctx + steps
    mask = torch.tensor([mask_row], dtype=torch.uint8)
    q = inputs.randn((B, steps, Hq, d), 140, dtype, DEV)
    k = inputs.randn((B, T, Hkv, d), 141, dtype, DEV)
    v = inputs.randn((B, T, Hkv, d), 142, dtype, DEV)
    c1 = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=dtype, retr_fmt=fmt)
    c2 = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=dtype, retr_fmt=fmt)
    if ctx > 0:
        for c in (c1, c2):
            c.append_kv(0, k[:, :ctx].contiguous(), v[:, :ctx].contiguous())
    for t in range(steps):
        kt, vt = k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous()
        c1.append_kv(0, kt, vt)
        o1, l1 = c1.decode_attention(0, q[:, t].contiguous())
        o2, l2 = c2.append_decode(0, q[:, t].contiguous(), kt, vt)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {t}"
    torch.cuda.synchronize()
    assert c1.len(0) == c2.len(0) == T and c1.device_status() == 0 and c2.device_status() == 0
    regions = [duo.DUO_REGION_RETR_K, duo.DUO_REGION_RETR_V, duo.DUO_REGION_STRM_K, duo.DUO_REGION_STRM_V]
    if fmt == "int4":
        regions += [duo.DUO_REGION_RETR_KSZ, duo.DUO_REGION_RETR_VSZ]
    for r in regions:
        a, _ = c1.region(0, r)
        b, _ = c2.region(0, r)
        assert torch.equal(a, b), f"region {r}"
    # and the last step matches the oracle
    want, want_lse = _decode_oracle(q[:, steps - 1:], k, v, mask[0], S, W, T - 1, 1)
    if fmt == "same":
        assert_close(o2.float().cpu().numpy()[:, None], want, dtype, l2.cpu().numpy()[:, None], want_lse, "append_decode")


# ------------------------------------------- the 1M-token INT4 stack at its own size

def test_int4_decode_1m_llama3_one_layer():
    """One layer of the 1M-token Llama-3-8B stack at its own size (32 q / 8 kv heads, 4
    INT4 retrieval + 4 bf16 streaming heads chosen by the seed, S 16, W 512, batch 1):
    2^20 - 2 tokens appended, then two decode steps.  Every INT4 code and fp16
    scale/zero is bit-exact with the oracle's quantiser; the outputs and lse of all 32
    query heads match the oracle over its own dequantisation.  The oracle runs one KV
    head (and its four query heads) at a time to bound host memory."""
    Hq, Hkv, d, S, W, G = 32, 8, 128, 16, 512, 4
    T, steps = 1 << 20, 2
    ctx = T - steps
    mask = inputs.retrieval_mask(1, Hkv, 4, seed=1)
    q = inputs.randn((1, steps, Hq, d), 150, device=DEV)
    k = inputs.randn((1, T, Hkv, d), 151, device=DEV)
    v = inputs.randn((1, T, Hkv, d), 152, device=DEV)
    cache = DuoCache(1, Hkv, d, mask, S, W, T, q_heads=Hq, dtype=torch.bfloat16, retr_fmt="int4")
    for t0 in range(0, ctx, 1 << 18):
        t1 = min(ctx, t0 + (1 << 18))
        cache.append_kv(0, k[:, t0:t1].contiguous(), v[:, t0:t1].contiguous())
    outs, lses = [], []
    for t in range(steps):
        cache.append_kv(0, k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous())
        o, l = cache.decode_attention(0, q[:, t].contiguous())
        outs.append(o.float()[0].cpu().numpy())
        lses.append(l[0].cpu().numpy())
    torch.cuda.synchronize()
    assert cache.device_status() == 0 and cache.len(0) == T
    got, got_lse = np.stack(outs), np.stack(lses)          # [steps][Hq][d], [steps][Hq]
    ridx = [g for g in range(Hkv) if mask[0, g]]
    rk, cap = cache.region(0, duo.DUO_REGION_RETR_K)
    rv, _ = cache.region(0, duo.DUO_REGION_RETR_V)
    ks, _ = cache.region(0, duo.DUO_REGION_RETR_KSZ)
    vs, _ = cache.region(0, duo.DUO_REGION_RETR_VSZ)
    qb = bits(q)
    want = np.zeros_like(got, dtype=np.float64)
    want_lse = np.zeros_like(got_lse, dtype=np.float64)
    for g in range(Hkv):
        kg, vg = bits(k[:, :, g:g + 1]), bits(v[:, :, g:g + 1])   # [1][T][1][d] bf16 bits
        if mask[0, g]:
            i = ridx.index(g)
            kd, vd = [], []
            for src, codes_r, sz_r in ((kg, rk, ks), (vg, rv, vs)):
                codes, sb, zb = oracle.int4_quantize(src.reshape(T, d))
                dev_codes = codes_r.view(1, len(ridx), cap, 64)[0, i, :T].cpu().numpy()
                dev_sz = sz_r.view(torch.int16).view(1, len(ridx), cap, 2)[0, i, :T].cpu().numpy().view(np.uint16)
                assert np.array_equal(dev_codes, codes), f"INT4 codes of kv head {g} differ"
                assert np.array_equal(dev_sz[:, 0], sb) and np.array_equal(dev_sz[:, 1], zb), f"scale/zero of {g}"
                (kd if src is kg else vd).append(oracle.int4_dequantize(codes, sb, zb).reshape(1, T, 1, d))
            kg, vg = kd[0], vd[0]
            del kd, vd
        for t in range(steps):
            w, l = oracle.attend(qb[:, t:t + 1, g * G:(g + 1) * G], kg[:, :ctx + t + 1], vg[:, :ctx + t + 1],
                                 [bool(mask[0, g])], S, W, pos0=ctx + t)
            want[t, g * G:(g + 1) * G] = w[0, 0]
            want_lse[t, g * G:(g + 1) * G] = l[0, 0]
        del kg, vg
    assert_close(got, want, torch.bfloat16, got_lse, want_lse, "int4 decode at 1M")


# ------------------------------------------------------------------- FP8

def _fp8_decode_check(Hq, Hkv, mask_row, S, W, B, ctx, steps, seed, plant=False, k_gain=1.0, v_gain=1.0, q_gain=1.0):
    """Append ctx tokens, then `steps` decode steps, on an FP8 (E4M3) retrieval cache.
    Every retrieval code byte and fp32 scale must equal the oracle's quantiser bit for
    bit; outputs are compared with the oracle over its own dequantisation of the
    retrieval rows (streaming heads keep bf16).  k_gain, v_gain and q_gain scale the
    N(0,1) draws (then rounded to bf16) to exercise the kernel's query and value-scale
    normalisation."""
    d, T, G = 128, ctx + steps, Hq // Hkv
    mask = torch.tensor([mask_row], dtype=torch.uint8)
    q = (inputs.randn((B, steps, Hq, d), seed, torch.float32, DEV) * q_gain).to(torch.bfloat16)
    k = (inputs.randn((B, T, Hkv, d), seed + 1, torch.float32, DEV) * k_gain).to(torch.bfloat16)
    v = (inputs.randn((B, T, Hkv, d), seed + 2, torch.float32, DEV) * v_gain).to(torch.bfloat16)
    ridx = [g for g in range(Hkv) if mask_row[g]]
    if plant and ctx > 2:
        P = ctx // 2
        ramp = torch.linspace(-2.0, 2.0, d, device=DEV).to(torch.bfloat16)
        for g in ridx:
            k[:, P, g] = (3.0 * q[:, 0, g * G].float()).to(torch.bfloat16)
            v[:, P, g] = ramp
    cache = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=torch.bfloat16, retr_fmt="fp8")
    if ctx > 0:
        cache.append_kv(0, k[:, :ctx].contiguous(), v[:, :ctx].contiguous())
    outs, lses = [], []
    for t in range(steps):
        cache.append_kv(0, k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous())
        o, l = cache.decode_attention(0, q[:, t].contiguous())
        outs.append(o.float()[:, None])
        lses.append(l[:, None])
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    got, got_lse = torch.cat(outs, 1).cpu().numpy(), torch.cat(lses, 1).cpu().numpy()
    rk, cap = cache.region(0, duo.DUO_REGION_RETR_K)
    rv, _ = cache.region(0, duo.DUO_REGION_RETR_V)
    ks, _ = cache.region(0, duo.DUO_REGION_RETR_KSZ)
    vs, _ = cache.region(0, duo.DUO_REGION_RETR_VSZ)
    kq = k.float().cpu().numpy().astype(np.float64)
    vq = v.float().cpu().numpy().astype(np.float64)
    for i, g in enumerate(ridx):
        for src, C, Z, dst in ((k, rk, ks, kq), (v, rv, vs, vq)):
            codes, scales = oracle.fp8_quantize(bits(src[:, :, g]).reshape(-1, d))
            dev_codes = C.view(B, len(ridx), cap, d)[:, i, :T].cpu().numpy().reshape(-1, d)
            dev_sc = Z.view(torch.float32).view(B, len(ridx), cap)[:, i, :T].cpu().numpy().reshape(-1)
            assert np.array_equal(dev_codes, codes), f"FP8 codes of kv head {g} differ"
            assert np.array_equal(dev_sc.view(np.uint32), scales.view(np.uint32)), f"FP8 scales of kv head {g} differ"
            dst[:, :, g] = oracle.fp8_dequantize(codes, scales).reshape(B, T, d)
    ws, ls = [], []
    for t in range(steps):
        w, l = oracle.attend(bits(q[:, t:t + 1]), kq[:, :ctx + t + 1], vq[:, :ctx + t + 1],
                             np.asarray(mask_row, dtype=bool), S, W, pos0=ctx + t)
        ws.append(w)
        ls.append(l)
    want, want_lse = np.concatenate(ws, 1), np.concatenate(ls, 1)
    scale = max(1.0, float(np.abs(want).max()))
    assert_close(got / scale, want / scale, torch.bfloat16, got_lse, want_lse,
                 f"fp8 decode Hq{Hq} Hkv{Hkv} B{B} ctx{ctx} gains {k_gain},{v_gain},{q_gain}")
    return got, want


@pytest.mark.parametrize("Hq,Hkv,mask_row,S,W,B,ctx", [
    (8, 8, [1, 0, 1, 0, 0, 0, 0, 1], 4, 32, 1, 0),        # first token: sees only itself
    (8, 8, [1, 0, 1, 0, 0, 0, 0, 1], 4, 32, 2, 37),       # MHA, one ragged tile
    (16, 8, [1] * 8, 16, 64, 1, 3000),                     # all retrieval, group 2
    (32, 4, [0, 0, 0, 0], 16, 512, 2, 2000),               # all streaming (bf16 pieces only)
    (64, 4, [1, 0, 1, 1], 16, 512, 1, 5000),               # group 16
    (32, 4, [0, 1, 1, 0], 0, 100, 3, 1000),                # group 8, no sinks
    (32, 8, [0, 1, 0, 1, 1, 0, 0, 1], 16, 512, 1, 1 << 17),  # Llama-3 shape, 128K
    (32, 8, [0, 1, 0, 1, 1, 0, 0, 1], 16, 512, 4, 20000),    # batch 4
    (32, 8, [1, 0, 1, 0, 1, 0, 1, 0], 16, 512, 2, 118),      # ring slots past len (tile 1)
])
def test_fp8_tc_decode_shapes(Hq, Hkv, mask_row, S, W, B, ctx):
    _fp8_decode_check(Hq, Hkv, mask_row, S, W, B, ctx, 2, 160)


@pytest.mark.parametrize("k_gain,v_gain,q_gain", [(1000.0, 1000.0, 1e-3), (1e-4, 1e-4, 1e4), (1 / 300, 1.0, 300.0),
                                                   (100.0, 1.0, 1e-2)])
def test_fp8_tc_decode_value_ranges(k_gain, v_gain, q_gain):
    """K and V far above or below 1 (the per-row scales and the tile's largest V scale
    carry them) and queries far from 1 (the power-of-two query prescale keeps them in
    fp16); the logits keep their N(0,1) size (k_gain * q_gain = 1)."""
    _fp8_decode_check(32, 8, [1, 0, 0, 1, 1, 0, 0, 1], 16, 512, 1, 3000, 1, 165, k_gain=k_gain, v_gain=v_gain,
                      q_gain=q_gain)


@pytest.mark.parametrize("Hq,Hkv,B,ctx", [(32, 8, 1, 20000), (8, 8, 2, 5000)])
def test_fp8_tc_decode_planted_needle(Hq, Hkv, B, ctx):
    mask_row = [1, 0] * (Hkv // 2)
    got, want = _fp8_decode_check(Hq, Hkv, mask_row, 16, 512, B, ctx, 1, 170, plant=True)
    G = Hq // Hkv
    ramp = np.linspace(-2.0, 2.0, 128)
    for g in range(0, Hkv, 2):  # retrieval heads recover the planted ramp
        assert np.abs(want[:, 0, g * G] - ramp).max() < 0.3
        assert np.abs(got[:, 0, g * G] - ramp).max() < 0.3


def test_fp8_append_decode_equals_append_then_decode():
    """duo_append_decode on an FP8 cache (two launches) leaves the same cache and returns
    the same outputs as duo_append_kv followed by duo_decode_attention."""
    Hq, Hkv, d, S, W, B, ctx, steps = 32, 8, 128, 16, 64, 1, 400, 20
    mask = torch.tensor([[0, 1, 1, 0, 0, 1, 0, 1]], dtype=torch.uint8)
    T = ctx + steps
    q = inputs.randn((B, steps, Hq, d), 175, device=DEV)
    k = inputs.randn((B, T, Hkv, d), 176, device=DEV)
    v = inputs.randn((B, T, Hkv, d), 177, device=DEV)
    c1 = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=torch.bfloat16, retr_fmt="fp8")
    c2 = DuoCache(1, Hkv, d, mask, S, W, T, batch=B, q_heads=Hq, dtype=torch.bfloat16, retr_fmt="fp8")
    for c in (c1, c2):
        c.append_kv(0, k[:, :ctx].contiguous(), v[:, :ctx].contiguous())
    for t in range(steps):
        kt, vt = k[:, ctx + t:ctx + t + 1].contiguous(), v[:, ctx + t:ctx + t + 1].contiguous()
        c1.append_kv(0, kt, vt)
        o1, l1 = c1.decode_attention(0, q[:, t].contiguous())
        o2, l2 = c2.append_decode(0, q[:, t].contiguous(), kt, vt)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {t}"
    torch.cuda.synchronize()
    for r in [duo.DUO_REGION_RETR_K, duo.DUO_REGION_RETR_V, duo.DUO_REGION_RETR_KSZ, duo.DUO_REGION_RETR_VSZ,
              duo.DUO_REGION_STRM_K, duo.DUO_REGION_STRM_V]:
        assert torch.equal(c1.region(0, r)[0], c2.region(0, r)[0]), f"region {r}"
