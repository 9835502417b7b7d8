"""The algebra the INT4 decode kernel rests on, checked in exact arithmetic on the CPU.

The kernel feeds each token's stored code bytes U_j = c_2j + 16 c_2j+1 to integer MMAs,
with the low nibbles L_j = c_2j as the only derived operand, and enters the fp32 operands
as 8-bit limbs.  These tests restate the identities and the limb error bounds (plain
int64 / float64 numpy, independent of the kernel and of the oracle): a wrong coefficient,
a swapped nibble or a limb scale off by a factor fails one of them.
"""
import numpy as np
import pytest


def _codes(rng, n):
    return rng.integers(0, 16, size=(n, 128), dtype=np.int64)


def _bytes_of(c):
    # element 2j in the low nibble of byte j, element 2j + 1 in the high nibble
    return c[:, 0::2] + 16 * c[:, 1::2], c[:, 0::2]


def test_dot_product_from_bytes_and_low_nibbles():
    """q . c = sum_j (q_2j+1 / 16) U_j + (q_2j - q_2j+1 / 16) L_j, exactly."""
    rng = np.random.default_rng(1)
    c = _codes(rng, 64)
    U, L = _bytes_of(c)
    # dyadic query values (exact in float64 through the /16)
    q = rng.integers(-2 ** 20, 2 ** 20, size=128).astype(np.float64) / 2 ** 12
    want = c.astype(np.float64) @ q
    qa = q[1::2] / 16.0
    qb = q[0::2] - q[1::2] / 16.0
    got = U.astype(np.float64) @ qa + L.astype(np.float64) @ qb
    assert np.array_equal(got, want)
    # the swapped reading (high nibble first) is wrong
    bad = U.astype(np.float64) @ (q[0::2] / 16.0) + L.astype(np.float64) @ (q[1::2] - q[0::2] / 16.0)
    assert not np.allclose(bad, want)


def test_output_pairs_from_byte_and_low_nibble_sums():
    """sum_t p'_t L_tj = O_2j and sum_t p'_t U_tj = O_2j + 16 O_2j+1 (integer p')."""
    rng = np.random.default_rng(2)
    c = _codes(rng, 128)
    U, L = _bytes_of(c)
    p = rng.integers(-127, 128, size=128, dtype=np.int64)  # one signed limb of P'
    O = p @ c                                                # [128] exact
    RU, RL = p @ U, p @ L
    assert np.array_equal(RL, O[0::2])
    assert np.array_equal((RU - RL) // 16, O[1::2]) and np.all((RU - RL) % 16 == 0)
    # int32 accumulators suffice: |R| < 2^22 for one M128 N16 K32 chain over 128 tokens
    assert np.abs(RU).max() < 2 ** 22 and 128 * 255 * 127 < 2 ** 22


def _limbs(x, n, first, rest):
    """x (array scaled so |x| <= first) into n limbs: rint, then residual * rest."""
    out, r = [], x.copy()
    for i in range(n):
        li = np.rint(r)
        out.append(li)
        r = (r - li) * (rest if i < n - 1 else 1.0)
    return out


def test_query_limbs_three_int8_within_2_pow_minus_21():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(4096) * 3.0
    amax = np.abs(x).max()
    y = x * (127.0 / amax)
    l0, l1, l2 = _limbs(y, 3, 127, 128.0)
    assert np.abs(l0).max() <= 127 and np.abs(l1).max() <= 64 and np.abs(l2).max() <= 64
    back = (amax / 127.0) * (l0 + l1 / 128.0 + l2 / 16384.0)
    assert np.abs(back - x).max() <= amax * 2.0 ** -21


def test_probability_limbs_two_int8_within_2_pow_minus_15():
    """P' = p s_v in [0, tmax]: l0 = rint(x) in [0, 127], l1 = rint(254 (x - l0))."""
    rng = np.random.default_rng(4)
    tmax = 0.37
    pv = rng.random(8192) * tmax
    pv[:3] = [0.0, tmax, tmax * 0.5]
    x = pv * (126.99 / tmax)
    l0 = np.rint(x)
    l1 = np.rint((x - l0) * 254.0)
    assert l0.min() >= 0 and l0.max() <= 127 and np.abs(l1).max() <= 127
    back = (tmax / 126.99) * (l0 + l1 / 254.0)
    assert np.abs(back - pv).max() <= tmax * 2.0 ** -15


@pytest.mark.parametrize("x", [0, 1, -1, 4194303, -4194304, 2087551, -123456])
def test_magic_number_int_to_float_is_exact(x):
    """float(x) = bits(x + 0x4B400000) - 1.5 * 2^23 for |x| < 2^22 (the kernel's conversion)."""
    magic = np.float32(12582912.0)
    as_float = np.array([x + 0x4B400000], dtype=np.int32).view(np.float32)[0]
    assert float(as_float - magic) == float(x)


def test_magic_number_rounding_gives_the_low_byte():
    """t = x + 1.5 * 2^23 rounds x to an integer whose low byte sits in t's low bits."""
    magic = np.float32(12582912.0)
    for x in [0.0, 0.49, 0.51, 126.99, -0.5, -63.7, 127.0, 1.5, 2.5]:
        t = np.float32(np.float32(x) + magic)
        rounded = float(t - magic)
        assert rounded == float(np.rint(np.float32(x)))
        low = int(np.array([t], dtype=np.float32).view(np.int32)[0]) & 0xFF
        assert low == (int(rounded) & 0xFF)
