"""Pins for the oracle's exact node score x = sum_n sum_d q[n,d] k[d].

The oracle computes x with a long fixed-point accumulator.  These tests pin it
to values that do not come from the oracle: Python's exact rational arithmetic,
closed forms on hand-built inputs, and algebraic identities (exact scaling by
powers of two, additivity over tokens, sign symmetry).
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _bits_f32(x):
    return np.array(x, dtype=np.float32)


def _frac_of_storage(a):
    return [Fraction(float(v)) for v in oracle.widen(np.asarray(a)).ravel()]


def _exact_int(q, k):
    return oracle.digits_to_int(oracle.exact_digits(q, k))


def _fraction_score(q, k):
    qf = oracle.widen(q)
    kf = oracle.widen(k)
    N, D = q.shape
    s = Fraction(0)
    for n in range(N):
        for d in range(D):
            s += Fraction(float(qf[n, d])) * Fraction(float(kf[d]))
    return s


def _to_scaled_int(fr):
    origin = oracle.exact_origin()
    v = fr * (1 << origin)
    assert v.denominator == 1, "an exact score must be a multiple of 2^-origin"
    return v.numerator


def _special_values(rng, n):
    pool = [0.0, -0.0, 1.0, -1.0, 2.0 ** -149, -(2.0 ** -149), 2.0 ** -126, 2.0 ** 100, -(2.0 ** 120),
            3.0 * 2.0 ** -140, 1.0 + 2.0 ** -23, 65504.0, 1e-30, -7e-39]
    v = rng.standard_normal(n) * np.exp2(rng.integers(-40, 40, n))
    pick = rng.random(n) < 0.3
    v[pick] = rng.choice(pool, pick.sum())
    return v


@pytest.mark.parametrize("seed", range(6))
def test_fp32_matches_fraction(seed):
    rng = np.random.default_rng(seed)
    N, D = int(rng.integers(1, 5)), int(rng.integers(1, 9))
    q = _special_values(rng, N * D).astype(np.float32).reshape(N, D)
    k = _special_values(rng, D).astype(np.float32)
    assert _exact_int(q, k) == _to_scaled_int(_fraction_score(q, k))


@pytest.mark.parametrize("seed", range(6))
def test_bf16_matches_fraction(seed):
    rng = np.random.default_rng(100 + seed)
    N, D = int(rng.integers(1, 6)), int(rng.integers(1, 17))
    # random bfloat16 bit patterns over the whole finite range (exponent field != 255)
    def rand_bf16(n):
        sign = rng.integers(0, 2, n).astype(np.uint16) << 15
        exp = rng.integers(0, 255, n).astype(np.uint16) << 7
        man = rng.integers(0, 128, n).astype(np.uint16)
        return sign | exp | man
    q = rand_bf16(N * D).reshape(N, D)
    k = rand_bf16(D)
    assert _exact_int(q, k) == _to_scaled_int(_fraction_score(q, k))


def test_cancellation_keeps_tiny_residual():
    # 2^100*1 + 1*2^-140 - 2^100*1 = 2^-140: float64 summation would return 0.
    q = np.array([[2.0 ** 100, 1.0, -(2.0 ** 100)]], dtype=np.float32)
    k = np.array([1.0, 2.0 ** -140, 1.0], dtype=np.float32)
    assert _exact_int(q, k) == 1 << (oracle.exact_origin() - 140)


def test_smallest_products_and_sign():
    tiny = 2.0 ** -149
    q = np.array([[tiny, -tiny]], dtype=np.float32)
    k = np.array([tiny, tiny], dtype=np.float32)
    assert _exact_int(q, k) == 0
    q2 = np.array([[tiny, tiny]], dtype=np.float32)
    k2 = np.array([-tiny, -tiny], dtype=np.float32)
    assert _exact_int(q2, k2) == -2 * (1 << (oracle.exact_origin() - 298))


def test_largest_products_do_not_overflow():
    big = float(np.finfo(np.float32).max)
    N, D = 64, 128
    q = np.full((N, D), big, dtype=np.float32)
    k = np.full(D, big, dtype=np.float32)
    expected = Fraction(big) * Fraction(big) * N * D
    assert _exact_int(q, k) == _to_scaled_int(expected)
    assert _exact_int(-q, k) == -_to_scaled_int(expected)


def test_basis_vectors_closed_form():
    D = 16
    for i in range(D):
        q = np.zeros((2, D), np.float32)
        q[0, i] = 3.0
        q[1, i] = 0.5
        k = np.zeros(D, np.float32)
        k[i] = -2.0
        k[(i + 1) % D] = 100.0   # orthogonal direction contributes nothing
        assert _exact_int(q, k) == -7 * (1 << oracle.exact_origin())


@pytest.mark.parametrize("seed", range(4))
def test_identities(seed):
    rng = np.random.default_rng(200 + seed)
    N, D = 5, 32
    q = rng.standard_normal((N, D)).astype(np.float32)
    k = rng.standard_normal(D).astype(np.float32)
    x = _exact_int(q, k)
    # exact scaling by a power of two
    assert _exact_int(q * np.float32(8.0), k) == 8 * x
    # additivity over tokens
    assert _exact_int(q[:2], k) + _exact_int(q[2:], k) == x
    # sign symmetry
    assert _exact_int(-q, k) == -x
    # agreement with float64 rounding bound: |x - fl64| <= gamma * sum|q||k|
    ref = float(np.sum(q.astype(np.float64) * k.astype(np.float64)))
    bound = N * D * 2.0 ** -52 * float(np.sum(np.abs(q.astype(np.float64)) * np.abs(k.astype(np.float64))))
    assert abs(x / 2.0 ** oracle.exact_origin() - ref) <= bound


@pytest.mark.parametrize("seed", range(4))
def test_digits_are_canonical(seed):
    # The ranking compares digit strings from the top down, which orders the
    # values only when every digit below the top one lies in [0, 2^32) (the
    # top one carries the sign).  Mixed signs exercise the borrows.
    rng = np.random.default_rng(100 + seed)
    for _ in range(50):
        N, D = int(rng.integers(1, 4)), int(rng.integers(1, 9))
        q = _bits_f32(_special_values(rng, N * D).reshape(N, D))
        k = _bits_f32(_special_values(rng, D))
        dig = oracle.exact_digits(q, k)
        assert all(0 <= int(d) < 1 << 32 for d in dig[:-1]), dig
