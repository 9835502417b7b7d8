"""The arithmetic the FP8 decode kernel rests on, checked on the CPU.

The kernel multiplies the stored E4M3 codes on the 8-bit tensor cores, with the fp32
operands (queries times 2^e_q, and P' = p s_v 2^6 / smax) entering as three E4M3 limbs
each, limb l scaled by 16^l:
    x ~= v0 + v1 / 16 + v2 / 256,  v0 = e4m3(x), v1 = e4m3(16 (x - v0)), v2 = e4m3(16 (...)).
These tests restate that split in float32 / float64 numpy, with torch's float8_e4m3fn
conversion (round to nearest even) as the E4M3 rounding, and check the bounds the kernel
relies on.  The split is exact when done in fp32, its error is at most 2^-12 |x|, and the
residuals never leave the E4M3 range.  A bf16 query scaled into [2^7, 2^8) is reproduced
exactly.  P' stays below 448.  The recombined products keep the bf16 output tolerance.
A wrong limb scale fails the bound.
"""
import numpy as np
import pytest
import torch

E4M3_MAX = 448.0


def e4m3(x):
    """Round float32 values to the nearest E4M3 value (ties to even), as float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float32).numpy()


def limbs3(x, scale=16.0):
    """The kernel's split, step by step in float32: returns v0, v1, v2 and the residuals."""
    x = np.asarray(x, dtype=np.float32)
    v0 = e4m3(x)
    r1 = ((x - v0) * np.float32(scale)).astype(np.float32)
    v1 = e4m3(r1)
    r2 = ((r1 - v1) * np.float32(scale)).astype(np.float32)
    v2 = e4m3(r2)
    return v0, v1, v2, r1, r2


def recombine(v0, v1, v2, scale=16.0):
    return v0.astype(np.float64) + v1.astype(np.float64) / scale + v2.astype(np.float64) / scale ** 2


def test_e4m3_rounding_reference_points():
    """The E4M3 grid: 3 mantissa bits, ties to even, largest finite 448, subnormal step 2^-9."""
    x = np.array([1.0625, 1.1875, 17.0, 19.0, 448.0, 2.0 ** -9, 3 * 2.0 ** -10, -0.3], dtype=np.float32)
    want = np.array([1.0, 1.25, 16.0, 20.0, 448.0, 2.0 ** -9, 2.0 ** -8, -0.3125], dtype=np.float32)
    assert np.array_equal(e4m3(x), want)


def test_split_is_exact_in_fp32_and_stays_in_range():
    """x - v is exact in float32 (v is x rounded to E4M3), and 16 |x - v| <= |x| in
    E4M3's normal range (below it, 16 |x - v| <= 2^-6 instead): no residual exceeds
    max(|x|, 2^-6) <= 2^8 < 448."""
    rng = np.random.default_rng(11)
    x = (rng.uniform(-1, 1, 200000) * 2.0 ** rng.uniform(-20, 8, 200000)).astype(np.float32)
    x = np.clip(x, -256, 256).astype(np.float32)
    v0, v1, v2, r1, r2 = limbs3(x)
    exact_r1 = (x.astype(np.float64) - v0.astype(np.float64)) * 16.0
    assert np.array_equal(r1.astype(np.float64), exact_r1)
    exact_r2 = (r1.astype(np.float64) - v1.astype(np.float64)) * 16.0
    assert np.array_equal(r2.astype(np.float64), exact_r2)
    assert np.all(np.abs(r1) <= np.maximum(np.abs(x), 2.0 ** -6))
    assert np.all(np.abs(r2) <= np.maximum(np.abs(r1), 2.0 ** -6))
    normal = np.abs(x) >= 2.0 ** -6
    assert np.all(np.abs(r1[normal]) <= np.abs(x[normal]))
    assert max(np.abs(v0).max(), np.abs(v1).max(), np.abs(v2).max()) <= 256.0 < E4M3_MAX


def test_split_error_bound():
    """|x - (v0 + v1/16 + v2/256)| <= 2^-12 |x| in E4M3's normal range, and at most
    half a subnormal step / 256 (2^-18) below it."""
    rng = np.random.default_rng(12)
    x = (rng.uniform(0, 1, 200000) * 2.0 ** rng.uniform(-24, 8, 200000)).astype(np.float32)
    x = np.minimum(x, 256).astype(np.float32)
    v0, v1, v2, _, _ = limbs3(x)
    err = np.abs(x.astype(np.float64) - recombine(v0, v1, v2))
    assert np.all(err <= np.maximum(2.0 ** -12 * np.abs(x), 2.0 ** -18))
    # over the whole range the split is much better than one E4M3 value (2^-4)
    normal = x >= 2.0 ** -6
    assert np.median(err[normal] / x[normal]) < 2.0 ** -14


def test_wrong_limb_scale_breaks_the_bound():
    """Recombining with a limb scale of 8 (or splitting with 8) is caught."""
    rng = np.random.default_rng(13)
    x = rng.uniform(1, 256, 5000).astype(np.float32)
    v0, v1, v2, _, _ = limbs3(x)
    bad = np.abs(x - recombine(v0, v1, v2, scale=8.0))
    assert np.any(bad > 2.0 ** -12 * x)
    w0, w1, w2, _, _ = limbs3(x, scale=8.0)
    bad2 = np.abs(x - recombine(w0, w1, w2, scale=16.0))
    assert np.any(bad2 > 2.0 ** -12 * x)


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def _query_scale(q):
    """2^e putting the largest |q| in [2^7, 2^8), from its exponent as the kernel does."""
    amax = np.float32(np.abs(q).max())
    ex = int(np.frexp(amax)[1]) - 1  # floor(log2 amax)
    return np.float32(2.0 ** (7 - ex))


@pytest.mark.parametrize("gain", [1e-3, 1.0, 300.0, 1e4])
def test_query_limbs_reproduce_bf16_queries(gain):
    """Every bf16 query element at least 2^-13 of its head's largest is reproduced exactly
    by v0 + v1/16 (v2 = 0): 8 significant bits need two 4-bit limbs.  Smaller ones keep
    an absolute error below 2^-19 of the head's largest."""
    rng = np.random.default_rng(14)
    q = _bf16(rng.standard_normal((16, 128)) * gain)
    for row in q:
        sc = _query_scale(row)
        x = (row * sc).astype(np.float32)
        assert 128 <= np.abs(x).max() < 256
        v0, v1, v2, _, _ = limbs3(x)
        got = recombine(v0, v1, v2)
        big = np.abs(x) >= 2.0 ** -6
        assert np.array_equal(got[big], x[big].astype(np.float64))
        assert np.all(v2[big] == 0)
        assert np.all(np.abs(got - x) <= 2.0 ** -12 * 128)


def test_probability_limb_operand_stays_in_e4m3_range():
    """P' = p s_v 2^6 / smax with p <= 2^2 (the running max trails the true one by at
    most 2 in log2 units) and s_v <= smax: at most 2^8 even with the approximate
    division and exponential (relative errors of a few 2^-22), below 448."""
    p_max = 2.0 ** 2 * (1 + 2.0 ** -21)
    factor = 64.0 * (1 + 2.0 ** -21)
    assert p_max * factor < 256.01 < E4M3_MAX
    # and the split of such values never saturates
    x = np.float32(p_max * factor)
    v0, v1, v2, _, _ = limbs3(np.array([x]))
    assert abs(recombine(v0, v1, v2)[0] - float(x)) <= 2.0 ** -12 * float(x)


def test_recombined_products_within_output_tolerance():
    """One 128-token tile: sum_t P'_t c_t with P' split into limbs against the exact sum
    (fp64), and q . c with the query split likewise: both far inside the bf16 output
    tolerance (relative 2^-9), as the fp32 accumulators add limb columns separately."""
    rng = np.random.default_rng(15)
    codes = e4m3(np.clip(rng.standard_normal((128, 128)) * 100, -448, 448))  # stored E4M3 codes
    p = np.exp2(-rng.exponential(3.0, 128)).astype(np.float32)       # probabilities <= 1
    sv = rng.uniform(0.5, 2.0, 128).astype(np.float32)
    x = (p * sv * np.float32(64.0) / np.float32(sv.max())).astype(np.float32)
    v0, v1, v2, _, _ = limbs3(x)
    got = v0 @ codes.astype(np.float64) + (v1 @ codes.astype(np.float64)) / 16 + (v2 @ codes.astype(np.float64)) / 256
    want = x.astype(np.float64) @ codes.astype(np.float64)
    assert np.abs(got - want).max() <= 2.0 ** -12 * (np.abs(x).astype(np.float64) @ np.abs(codes).astype(np.float64)).max()
    q = _bf16(rng.standard_normal(128))
    xq = (q * _query_scale(q)).astype(np.float32)
    w0, w1, w2, _, _ = limbs3(xq)
    s_got = codes.astype(np.float64) @ recombine(w0, w1, w2)
    s_want = codes.astype(np.float64) @ xq.astype(np.float64)
    assert np.abs(s_got - s_want).max() <= 2.0 ** -12 * (np.abs(codes).astype(np.float64) @ np.abs(xq)).max()
