"""Pins for the fp64 oracle: values the pages print, closed forms, library special
cases and brute force on tiny inputs.  None of these re-uses the oracle's own code
path to produce its expected value.

Sources: the paper-graph-ui explainer of DuoAttention (arXiv 2410.10819) and the
paperhub.cn OpenReview discussion of the same paper; each test names its section.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _rand(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


# ---------------------------------------------------------------- cache pins

def test_fig5_worked_example(golden_dir):
    """'Chunked Pre-filling', Figure 5 (right): retained tokens after each chunk."""
    g = json.load(open(os.path.join(golden_dir, "fig5_chunked_prefill.json")))
    S, W, lens = g["S"], g["W"], g["chunk_lens"]
    slots = oracle.ring_replay(S, W, lens)
    total = 0
    for c, n in enumerate(lens):
        total += n
        held = sorted(int(p) for p in slots[c] if p >= 0)
        assert held == g["retained_after_chunk"][c]
        closed = [p for p in range(total) if oracle.retained(total, S, W)[p]]
        assert closed == g["retained_after_chunk"][c]
    # what chunk 2 may read is what chunk 1 left behind
    assert sorted(int(p) for p in slots[0] if p >= 0) == g["cached_before_chunk"][1]


def _partitions(L):
    for cuts in itertools.product([0, 1], repeat=L - 1):
        lens, run = [], 1
        for c in cuts:
            if c:
                lens.append(run)
                run = 1
            else:
                run += 1
        lens.append(run)
        yield lens


def test_ring_replay_brute_force_all_partitions():
    """Every chunk partition of L <= 9 tokens, every S and W: the slots hold exactly
    the sinks plus the last W tokens ('Decoding Procedure' step 3/4, Figure 5), and
    no slot holds a position twice."""
    for L in range(1, 10):
        for S in range(0, L + 1):
            for W in range(1, L + 1):
                for lens in _partitions(L):
                    slots = oracle.ring_replay(S, W, lens)
                    total = 0
                    for c, n in enumerate(lens):
                        total += n
                        held = [int(p) for p in slots[c] if p >= 0]
                        assert len(held) == len(set(held))
                        # set-level statement: first S tokens, plus the W newest non-sinks
                        want = set(range(min(S, total))) | set(range(max(S, total - W), total))
                        assert set(held) == want, (L, S, W, lens, c)


def test_retained_equals_decode_query_visible_set():
    """The newest query must see exactly what the streaming cache keeps, and a
    later query of any chunk never needs a key the cache dropped (reading R2)."""
    for L in range(1, 14):
        for S in range(0, L + 1):
            for W in range(1, L + 1):
                ret = oracle.retained(L, S, W)
                vis = [oracle.visible(L - 1, j, False, S, W) for j in range(L)]
                assert list(ret) == vis
                for c0 in range(1, L):
                    kept = oracle.retained(c0, S, W)
                    for i in range(c0, L):
                        for j in range(c0):
                            if oracle.visible(i, j, False, S, W):
                                assert kept[j], (L, S, W, c0, i, j)


def test_memory_formula(golden_dir):
    """'Decoding Procedure': Memory = (H_r L + H_s (S+R)) d, by the golden values and by
    counting what the caches keep."""
    g = json.load(open(os.path.join(golden_dir, "kv_memory.json")))
    for c in g["memory_formula"]["cases"]:
        assert oracle.layer_kv_elems(c["Hr"], c["Hs"], c["L"], c["S"], c["W"], c["d"]) == c["elems"]
    for L in range(1, 40):
        for S, W in [(0, 1), (2, 3), (4, 16), (16, 5)]:
            counted = 3 * L + 5 * int(oracle.retained(L, S, W).sum())
            assert oracle.layer_kv_elems(3, 5, L, S, W, 1) == counted


def test_budget_ratio(golden_dir):
    """OpenReview reply, 'RazorAttention and Echo Heads': 0.5025 for 64K / 50% / 320."""
    g = json.load(open(os.path.join(golden_dir, "kv_memory.json")))["budget_ratio"]
    for c in g["cases"]:
        got = oracle.budget_ratio(c["L"], c["retrieval_fraction"], c["sink_plus_recent"])
        assert abs(got - c["ratio"]) < 1e-12, c
    # the ratio is the memory formula divided by full attention's H L d
    for Hr, Hs, L, S, W in [(8, 24, 32768, 16, 512), (4, 4, 131072, 16, 512), (1, 3, 1000, 4, 60)]:
        r = Hr / (Hr + Hs)
        assert abs(oracle.budget_ratio(L, r, S + W) - oracle.layer_kv_elems(Hr, Hs, L, S, W, 1) / ((Hr + Hs) * L)) < 1e-12


def test_full_kv_137gb(golden_dir):
    """'The Core Problem': Llama-3-8B, FP16 KV, 1M tokens needs at least 137 GB."""
    g = json.load(open(os.path.join(golden_dir, "kv_memory.json")))["full_kv_bytes"]
    b = oracle.full_kv_bytes(g["layers"], g["kv_heads"], g["head_dim"], g["tokens"], g["elem_bytes"])
    assert b == g["bytes"]
    assert math.floor(b / 1e9) == g["gb_floor"]


# ------------------------------------------------------------ attention pins

def _sdpa(q, k, v, mask):
    """torch's scaled_dot_product_attention in float64 on CPU; q [B][nq][Hq][d],
    k/v [B][L][Hkv][d], mask bool [nq][L] (True = attend)."""
    Hq, Hkv = q.shape[2], k.shape[2]
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask))
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("B,Hq,Hkv,d,L,nq", [(1, 4, 4, 16, 37, 37), (2, 8, 2, 32, 50, 19), (1, 6, 3, 8, 9, 1)])
def test_all_retrieval_is_causal_sdpa(B, Hq, Hkv, d, L, nq):
    """'Gate Parameterization': alpha = 1 on every head gives full causal attention."""
    q, k, v = _rand((B, nq, Hq, d), 1), _rand((B, L, Hkv, d), 2), _rand((B, L, Hkv, d), 3)
    pos0 = L - nq
    mask = np.tril(np.ones((nq, L), dtype=bool), k=pos0)
    out, _ = oracle.attend(q, k, v, [True] * Hkv, S=2, W=3, pos0=pos0)
    np.testing.assert_allclose(out, _sdpa(q, k, v, mask), rtol=0, atol=1e-12)


@pytest.mark.parametrize("S,W", [(3, 40), (0, 64), (64, 1), (10, 30)])
def test_streaming_with_large_window_is_full(S, W):
    """A streaming head whose sinks + window cover the whole sequence (S + W >= L) is
    full causal attention."""
    B, Hq, Hkv, d, L = 1, 4, 2, 16, 40
    q, k, v = _rand((B, L, Hq, d), 4), _rand((B, L, Hkv, d), 5), _rand((B, L, Hkv, d), 6)
    out, _ = oracle.attend(q, k, v, [False, False], S=S, W=W, pos0=0)
    np.testing.assert_allclose(out, _sdpa(q, k, v, np.tril(np.ones((L, L), dtype=bool))), rtol=0, atol=1e-12)


@pytest.mark.parametrize("W", [1, 2, 7, 16])
def test_streaming_without_sinks_is_sliding_window(W):
    """S = 0 leaves only the recent tokens: a causal band of width W (counting the
    query), built here with tril/triu and handed to torch SDPA."""
    B, Hq, Hkv, d, L = 2, 2, 1, 8, 33
    q, k, v = _rand((B, L, Hq, d), 7), _rand((B, L, Hkv, d), 8), _rand((B, L, Hkv, d), 9)
    band = np.tril(np.ones((L, L), dtype=bool)) & np.triu(np.ones((L, L), dtype=bool), k=-(W - 1))
    out, _ = oracle.attend(q, k, v, [False], S=0, W=W, pos0=0)
    np.testing.assert_allclose(out, _sdpa(q, k, v, band), rtol=0, atol=1e-12)


# ------------------------------------------------------- gated mixed attention

def _lambda_mask(L, S, W):
    """The Lambda mask of 'The Full and Streaming Attention Masks' as a union of a
    causal band of width W (query included) and the first S columns, below the diagonal."""
    causal = np.tril(np.ones((L, L), dtype=bool))
    band = causal & np.triu(np.ones((L, L), dtype=bool), k=-(W - 1))
    sinks = causal & (np.arange(L)[None, :] < S)
    return band | sinks


@pytest.mark.parametrize("B,Hq,Hkv,d,L,S,W", [(1, 4, 2, 16, 40, 3, 7), (2, 6, 3, 8, 25, 0, 4), (1, 2, 1, 32, 19, 5, 1)])
def test_gated_is_mixture_of_causal_and_lambda_sdpa(B, Hq, Hkv, d, L, S, W):
    """'Gate Parameterization': attn = alpha * full_attn + (1 - alpha) * streaming_attn
    per KV head; both terms from torch SDPA (float64) under the two masks."""
    q, k, v = _rand((B, L, Hq, d), 31), _rand((B, L, Hkv, d), 32), _rand((B, L, Hkv, d), 33)
    alpha = np.linspace(0.0, 1.0, Hkv) if Hkv > 1 else np.array([0.37])
    full = _sdpa(q, k, v, np.tril(np.ones((L, L), dtype=bool)))
    lam = _sdpa(q, k, v, _lambda_mask(L, S, W))
    a = np.repeat(alpha, Hq // Hkv)[None, None, :, None]
    want = a * full + (1.0 - a) * lam
    np.testing.assert_allclose(oracle.gated(q, k, v, alpha, S, W), want, rtol=0, atol=1e-12)


def test_gated_end_points_and_sampled_rows():
    """alpha = 1 is the retrieval (causal) head and alpha = 0 the streaming head of the
    cache attention; sampled rows equal the same rows of the full evaluation."""
    B, Hq, Hkv, d, L, S, W = 1, 4, 2, 16, 30, 2, 5
    q, k, v = _rand((B, L, Hq, d), 34), _rand((B, L, Hkv, d), 35), _rand((B, L, Hkv, d), 36)
    g = oracle.gated(q, k, v, [1.0, 0.0], S, W)
    att, _ = oracle.attend(q, k, v, [True, False], S=S, W=W, pos0=0)
    np.testing.assert_allclose(g, att, rtol=0, atol=1e-12)
    rows = np.array([0, 7, 33, L * Hq - 1])
    np.testing.assert_array_equal(oracle.gated(q, k, v, [0.2, 0.9], S, W, rows=rows),
                                  oracle.gated(q, k, v, [0.2, 0.9], S, W).reshape(-1, d)[rows])


def test_gated_wrong_gate_is_caught():
    """A gate applied to the wrong KV head (or swapped terms) moves the output far
    outside any tolerance on these inputs."""
    B, Hq, Hkv, d, L, S, W = 1, 4, 2, 16, 60, 2, 5
    q, k, v = _rand((B, L, Hq, d), 37), _rand((B, L, Hkv, d), 38), _rand((B, L, Hkv, d), 39)
    good = oracle.gated(q, k, v, [0.1, 0.8], S, W)
    assert np.abs(oracle.gated(q, k, v, [0.8, 0.1], S, W) - good).max() > 0.05
    assert np.abs(oracle.gated(q, k, v, [0.9, 0.2], S, W) - good).max() > 0.05


def _enumerated_visible(i, is_retrieval, S, W):
    """Visible keys of query i as a union of ranges: all earlier keys for a retrieval
    head; the first S tokens plus the W newest (query included) for a streaming head."""
    if is_retrieval:
        return list(range(i + 1))
    return sorted(set(range(min(S, i + 1))) | set(range(max(0, i - W + 1), i + 1)))


def test_brute_force_tiny_attention():
    """L <= 12: softmax over explicitly enumerated visible keys (scipy softmax and
    logsumexp) equals the oracle's output and lse on every row."""
    rng = np.random.default_rng(11)
    for L in range(1, 13):
        for S, W in [(0, 1), (1, 2), (2, 3), (4, 4), (0, 12), (3, 1)]:
            d, Hkv, Hq = 4, 2, 4
            q, k, v = (rng.standard_normal(s) for s in [(1, L, Hq, d), (1, L, Hkv, d), (1, L, Hkv, d)])
            retr = [True, False]
            out, lse = oracle.attend(q, k, v, retr, S=S, W=W, pos0=0)
            for i in range(L):
                for h in range(Hq):
                    g = h // (Hq // Hkv)
                    js = _enumerated_visible(i, retr[g], S, W)
                    logits = np.array([q[0, i, h] @ k[0, j, g] for j in js]) / math.sqrt(d)
                    p = softmax(logits)
                    np.testing.assert_allclose(out[0, i, h], p @ v[0, js, g], rtol=0, atol=1e-12)
                    assert abs(lse[0, i, h] - logsumexp(logits)) < 1e-12


def test_zero_queries_average_the_visible_values():
    """All-zero queries make every visible logit 0: the output is the plain mean of
    the visible value rows and lse = ln(#visible)."""
    L, d, S, W = 30, 8, 3, 5
    q = np.zeros((1, L, 2, d))
    k, v = _rand((1, L, 2, d), 12), _rand((1, L, 2, d), 13)
    out, lse = oracle.attend(q, k, v, [True, False], S=S, W=W, pos0=0)
    for i in range(L):
        for h, is_r in [(0, True), (1, False)]:
            js = _enumerated_visible(i, is_r, S, W)
            np.testing.assert_allclose(out[0, i, h], v[0, js, h].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[0, i, h] - math.log(len(js))) < 1e-13


def test_softmax_rows_sum_to_one():
    """With one-hot value rows the output is the probability row itself: it sums to 1
    and is exactly zero on masked keys."""
    L, S, W = 24, 2, 6
    q, k = _rand((1, L, 2, L), 14), _rand((1, L, 2, L), 15)
    v = np.broadcast_to(np.eye(L)[None, :, None, :], (1, L, 2, L)).copy()
    out, _ = oracle.attend(q, k, v, [True, False], S=S, W=W, pos0=0)
    for i in range(L):
        for h, is_r in [(0, True), (1, False)]:
            p = out[0, i, h]
            assert abs(p.sum() - 1.0) < 1e-12
            hidden = [j for j in range(L) if j not in _enumerated_visible(i, is_r, S, W)]
            assert np.all(p[hidden] == 0.0)


def test_planted_needle():
    """A key planted as c * q at a middle position dominates a retrieval head's
    softmax; a streaming head cannot see it once it has left the window."""
    L, d, S, W = 64, 16, 2, 8
    rng = np.random.default_rng(16)
    q = rng.standard_normal((1, 1, 2, d))
    k, v = rng.standard_normal((1, L, 2, d)), rng.standard_normal((1, L, 2, d))
    j_star = 30
    for g in range(2):
        k[0, j_star, g] = 40.0 * q[0, 0, g] / np.linalg.norm(q[0, 0, g]) * math.sqrt(d)
    out, _ = oracle.attend(q, k, v, [True, False], S=S, W=W, pos0=L - 1)
    np.testing.assert_allclose(out[0, 0, 0], v[0, j_star, 0], atol=1e-6)
    assert np.abs(out[0, 0, 1] - v[0, j_star, 1]).max() > 0.1


def test_explicit_scale_and_default_scale_agree():
    """'The Full and Streaming Attention Masks' omit the 1/sqrt(d) factor; the default
    is the standard scaled dot product (reading R3)."""
    q, k, v = _rand((1, 5, 2, 16), 17), _rand((1, 5, 2, 16), 18), _rand((1, 5, 2, 16), 19)
    a, la = oracle.attend(q, k, v, [True, False], S=1, W=2, pos0=0)
    b, lb = oracle.attend(q, k, v, [True, False], S=1, W=2, pos0=0, scale=0.25)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_sampled_rows_equal_full_rows():
    q, k, v = _rand((2, 6, 4, 8), 20), _rand((2, 9, 2, 8), 21), _rand((2, 9, 2, 8), 22)
    full, lfull = oracle.attend(q, k, v, [False, True], S=1, W=3, pos0=3)
    rows = [0, 5, 17, 47, 30]
    part, lpart = oracle.attend(q, k, v, [False, True], S=1, W=3, pos0=3, rows=rows)
    assert np.array_equal(part, full.reshape(-1, 8)[rows])
    assert np.array_equal(lpart, lfull.reshape(-1)[rows])


def test_bf16_inputs_convert_exactly():
    x = torch.randn(2, 7, 2, 8, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    as64 = x.to(torch.float64).numpy()
    a, la = oracle.attend(bits, bits, bits, [True, False], S=1, W=2, pos0=0)
    b, lb = oracle.attend(as64, as64, as64, [True, False], S=1, W=2, pos0=0)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


# ----------------------------------------------------------------- INT4 pins

def test_int4_worked_example():
    """Row 0..15 repeated: min 0, max 15, scale 1, zero 0, codes equal the values;
    element 2t sits in the low nibble of byte t."""
    row = np.tile(np.arange(16, dtype=np.float32), 8)[None, :]
    codes, sb, zb = oracle.int4_quantize(row)
    assert sb[0] == 0x3C00 and zb[0] == 0x0000  # fp16 1.0 and 0.0
    want = [(2 * t % 16) | ((2 * t + 1) % 16) << 4 for t in range(64)]
    assert codes[0].tolist() == want
    np.testing.assert_array_equal(oracle.int4_dequantize(codes, sb, zb)[0], row[0].astype(np.float64))


def test_int4_round_half_even():
    row = np.zeros((1, 128), dtype=np.float32)
    row[0, 1] = 15.0  # scale 1, zero 0
    row[0, 2], row[0, 3], row[0, 4] = 2.5, 3.5, 0.5
    codes, _, _ = oracle.int4_quantize(row)
    c = [(codes[0, e // 2] >> (4 * (e & 1))) & 15 for e in range(5)]
    assert c == [0, 15, 2, 4, 0]


def test_int4_round_trip_bound_and_order():
    """Dequantised values stay within half a step of the input (plus the fp16 rounding
    of the step and zero); codes are monotone in x; the row's min and max land on
    codes 0 and 15."""
    x = torch.randn(500, 128, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    xf = x.to(torch.float64).numpy()
    codes, sb, zb = oracle.int4_quantize(bits)
    deq = oracle.int4_dequantize(codes, sb, zb)
    scale = sb.view(np.float16).astype(np.float64)
    err = np.abs(deq - xf).max(axis=1)
    assert np.all(err <= scale * 0.5 * (1 + 4e-3) + 1e-6)
    full = np.stack([(codes >> 0) & 15, (codes >> 4) & 15], axis=-1).reshape(500, 128)
    for r in range(500):
        order = np.argsort(xf[r], kind="stable")
        assert np.all(np.diff(full[r][order].astype(int)) >= 0)
        assert full[r][np.argmin(xf[r])] == 0 and full[r][np.argmax(xf[r])] == 15


def test_int4_constant_row():
    row = np.full((1, 128), 0.71875, dtype=np.float32)  # exact in bf16 and fp16
    codes, sb, zb = oracle.int4_quantize(row)
    assert sb[0] == 0 and np.all(codes == 0)
    np.testing.assert_array_equal(oracle.int4_dequantize(codes, sb, zb), row.astype(np.float64))


# ------------------------------------------------------------------ FP8 pins

def test_fp8_worked_example():
    """amax 3.5 gives the scale 3.5 / 448 = 2^-7, so y = 128 x: values worked out by hand
    from the OCP E4M3 layout (bias 7, 3 mantissa bits, 448 the largest finite value):
    1 -> 128 = 0x70, -2 -> -256 = 0xF8, 0.5 -> 64 = 0x68, 3.5 -> 448 = 0x7E; ties go to
    the even mantissa (8.5 -> 8 = 0x50, 9.5 -> 10 = 0x52); 3 * 2^-9 is the subnormal
    0x03; 0 -> 0x00."""
    vals = [1.0, -2.0, 0.5, 3.5, 8.5 * 2.0 ** -7, 9.5 * 2.0 ** -7, 3 * 2.0 ** -16, 0.0]
    row = np.zeros((1, 128), dtype=np.float32)
    row[0, :len(vals)] = vals
    codes, scales = oracle.fp8_quantize(row)
    assert scales[0] == np.float32(2.0 ** -7)
    assert codes[0, :8].tolist() == [0x70, 0xF8, 0x68, 0x7E, 0x50, 0x52, 0x03, 0x00]
    deq = oracle.fp8_dequantize(codes, scales)[0, :8]
    np.testing.assert_array_equal(deq, [1.0, -2.0, 0.5, 3.5, 8 * 2.0 ** -7, 10 * 2.0 ** -7, 3 * 2.0 ** -16, 0.0])


def test_fp8_encoder_matches_torch_float8_e4m3fn():
    """The oracle's E4M3 rounding equals torch's float32 -> float8_e4m3fn conversion (an
    independent implementation of the same format) on random values, exact ties and
    subnormals within +-448, and its decoding equals torch's for every finite code."""
    rng = np.random.default_rng(11)
    y = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(2000) * 2.0 ** rng.integers(-12, 6, 2000),
                        (np.arange(-64, 64) + 0.5) * 2.0 ** -3, (np.arange(0, 16) + 0.5) * 2.0 ** -9]).astype(np.float32)
    y = y[np.abs(y) <= 448]
    want = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in y], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    tv = torch.tensor(finite, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal([oracle.e4m3_value(c) for c in finite], tv)


def test_fp8_round_trip_bound_and_order():
    """Dequantised values stay within half an E4M3 step of x (relative 2^-4 in the normal
    range, 2^-10 of the scale below it); codes are monotone in x; a row's largest
    magnitude lands on +-448; no NaN code is produced."""
    x = torch.randn(500, 128, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    xf = x.to(torch.float64).numpy()
    codes, scales = oracle.fp8_quantize(bits)
    deq = oracle.fp8_dequantize(codes, scales)
    sc = scales.astype(np.float64)[:, None]
    bound = sc * np.maximum(np.abs(xf) / sc * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - xf) <= bound)
    assert not np.any((codes & 0x7F) == 0x7F)
    for r in range(500):
        order = np.argsort(xf[r], kind="stable")
        assert np.all(np.diff(deq[r][order]) >= 0)
        i = np.argmax(np.abs(xf[r]))
        assert codes[r, i] == (0xFE if xf[r, i] < 0 else 0x7E)


def test_fp8_zero_row():
    codes, scales = oracle.fp8_quantize(np.zeros((2, 128), dtype=np.float32))
    assert np.all(scales == 0) and np.all(codes == 0)
    assert np.all(oracle.fp8_dequantize(codes, scales) == 0)


# ------------------------------------------------------------- mutation check

def _pin_failures(mutant):
    """Run a compact battery of the pins above against a mutated oracle; return the
    names of the pins that catch the mutation."""
    fails = []
    rng = np.random.default_rng(23)
    B, L, Hq, Hkv, d = 1, 20, 4, 2, 8
    q, k, v = (rng.standard_normal(s) for s in [(B, L, Hq, d), (B, L, Hkv, d), (B, L, Hkv, d)])
    # all-retrieval equals causal SDPA
    out, _ = oracle.attend(q, k, v, [True, True], S=1, W=3, pos0=0, mutant=mutant)
    if not np.allclose(out, _sdpa(q, k, v, np.tril(np.ones((L, L), dtype=bool))), atol=1e-10):
        fails.append("causal_sdpa")
    # brute force on a mixed head set
    out, lse = oracle.attend(q, k, v, [True, False], S=2, W=3, pos0=0, mutant=mutant)
    bad = False
    for i in range(L):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            js = _enumerated_visible(i, g == 0, 2, 3)
            logits = np.array([q[0, i, h] @ k[0, j, g] for j in js]) / math.sqrt(d)
            if not np.allclose(out[0, i, h], softmax(logits) @ v[0, js, g], atol=1e-10) or \
                    abs(lse[0, i, h] - logsumexp(logits)) > 1e-10:
                bad = True
    if bad:
        fails.append("brute_force")
    return fails


@pytest.mark.parametrize("mutant", sorted(oracle.MUTANTS))
def test_every_planted_mistake_is_caught(mutant):
    assert _pin_failures(None) == []
    assert _pin_failures(mutant), f"mutation {mutant} slipped through every pin"
