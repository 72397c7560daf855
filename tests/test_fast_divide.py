"""The attention kernel splits key-block ids into (time, row, column) with a
float reciprocal instead of an integer division: q = trunc(float32(n) *
float32(1 / d)), then one correction step (q - 1 if n - q d < 0, q + 1 if
n - q d >= d). The kernel's comment and the host's 2^22 limit rest on that
being exact for every 0 <= n < 2^22 and d >= 1: n and the quotient are below
2^23, so the float product is within one of n / d. Checked here on the CPU
with numpy's float32 arithmetic (round to nearest, like the kernel's
__int2float_rn, the reciprocal and the multiply), against exact integer
division."""
import numpy as np
import pytest


def fast_divmod(n: np.ndarray, d: int):
    inv = np.float32(1.0) / np.float32(d)
    q = np.trunc(n.astype(np.float32) * inv).astype(np.int64)
    r = n - q * d
    lo = r < 0
    q[lo] -= 1
    r[lo] += d
    hi = r >= d
    q[hi] += 1
    r[hi] -= d
    return q, r


@pytest.mark.parametrize("d", [1, 2, 3, 7, 11, 66, 88, 252, 1000, 4095, 65537, (1 << 22) - 1])
def test_every_id_below_2_22(d):
    n = np.arange(0, 1 << 22, dtype=np.int64)
    q, r = fast_divmod(n, d)
    assert np.array_equal(q, n // d) and np.array_equal(r, n % d)


def test_random_divisors_and_multiples():
    rng = np.random.default_rng(5)
    for d in rng.integers(1, 1 << 20, size=200):
        d = int(d)
        # every multiple of d below 2^22 and its neighbours: where a float
        # product just below an integer would truncate one too low
        k = np.arange(0, (1 << 22) // d + 1, dtype=np.int64) * d
        n = np.concatenate([k, k + 1, np.maximum(k - 1, 0)])
        n = n[n < (1 << 22)]
        q, r = fast_divmod(n, d)
        assert np.array_equal(q, n // d) and np.array_equal(r, n % d), d


def test_a_limit_is_needed():
    """Above 2^25 the float32 conversion of n itself can be off by two, and
    one correction step no longer suffices (first at n = 2^25 + 2 for d = 1):
    the kernel's ids must stay below a bound, and 2^22 leaves a margin."""
    n = np.array([(1 << 25) + 2, (1 << 26) + 2], dtype=np.int64)
    q, _ = fast_divmod(n, 1)
    assert np.all(q != n)
