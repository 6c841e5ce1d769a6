"""Pins for the oracle's GEMM references.  The exact product of the decoded
operands is recomputed here in Python integers (every finite E4M3 value is an
integer multiple of 2^-9, taken from the bit fields), and closed forms
(selection matrices, all-ones operands, unit scales) fix the results."""
from fractions import Fraction

import numpy as np
import pytest


def _units(code: int) -> int:
    """E4M3 code -> value * 2^9 as an integer (finite codes only)."""
    s, E, m = code >> 7, (code >> 3) & 15, code & 7
    u = m if E == 0 else (8 + m) << (E - 1)
    return -u if s else u


def _rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C                      # no NaN codes
    return c


@pytest.mark.parametrize("m,n,k", [(1, 1, 1), (3, 5, 16), (8, 7, 64), (2, 9, 33)])
def test_rowwise_exact_against_integer_brute_force(orc, m, n, k):
    rng = np.random.default_rng(m * 100 + n * 10 + k)
    qa, qb = _rand_codes(rng, (m, k)), _rand_codes(rng, (n, k))
    sa = (rng.random(m) * 3).astype(np.float32)
    sb = (rng.random(n) * 3 - 1).astype(np.float32)
    c, bound = orc.gemm_rowwise(qa, qb, sa, sb)
    for i in range(m):
        for j in range(n):
            d = sum(_units(int(qa[i, t])) * _units(int(qb[j, t])) for t in range(k))
            da = sum(abs(_units(int(qa[i, t])) * _units(int(qb[j, t]))) for t in range(k))
            sab = Fraction(float(sa[i])) * Fraction(float(sb[j]))
            exact = sab * Fraction(d, 2 ** 18)
            assert abs(Fraction(c[i, j]) - exact) <= abs(exact) * Fraction(1, 2 ** 52)
            exb = abs(sab) * Fraction(da, 2 ** 18)            # one fp64 rounding of sab * sum
            assert abs(Fraction(bound[i, j]) - exb) <= exb * Fraction(1, 2 ** 52)


@pytest.mark.parametrize("m,n,k", [(1, 1, 32), (3, 4, 64), (5, 2, 128)])
def test_mx_exact_against_integer_brute_force(orc, m, n, k):
    rng = np.random.default_rng(7 + m + n + k)
    qa, qb = _rand_codes(rng, (m, k)), _rand_codes(rng, (n, k))
    sfa = rng.integers(100, 160, size=(m, k // 32), dtype=np.uint8)
    sfb = rng.integers(90, 150, size=(n, k // 32), dtype=np.uint8)
    c, bound = orc.gemm_mx(qa, sfa, qb, sfb)
    for i in range(m):
        for j in range(n):
            exact = Fraction(0)
            exabs = Fraction(0)
            for b in range(k // 32):
                d = sum(_units(int(qa[i, t])) * _units(int(qb[j, t])) for t in range(32 * b, 32 * b + 32))
                da = sum(abs(_units(int(qa[i, t])) * _units(int(qb[j, t]))) for t in range(32 * b, 32 * b + 32))
                sc = Fraction(2) ** (int(sfa[i, b]) + int(sfb[j, b]) - 254) / 2 ** 18
                exact += sc * d
                exabs += sc * da
            tol = exabs * Fraction(k // 32 + 1, 2 ** 52)
            assert abs(Fraction(c[i, j]) - exact) <= tol
            assert abs(Fraction(bound[i, j]) - exabs) <= tol


def test_selection_matrix_reproduces_rows_of_b(orc):
    """A with a single 1.0 (code 0x38) per row selects rows of B^T, so C is
    a copy of decoded B scaled by sa*sb -- and a transposed operand would not."""
    rng = np.random.default_rng(5)
    n, k = 6, 48
    qb = _rand_codes(rng, (n, k))
    qa = np.zeros((k, k), dtype=np.uint8)
    for i in range(k):
        qa[i, (5 * i + 3) % k] = 0x38
    sa = np.full(k, 2.0, dtype=np.float32)
    sb = np.full(n, 0.25, dtype=np.float32)
    c, _ = orc.gemm_rowwise(qa, qb, sa, sb)
    dec = orc.e4m3_decode_table()
    for i in range(k):
        assert np.array_equal(c[i], 0.5 * dec[qb[:, (5 * i + 3) % k]])


def test_all_ones_closed_form(orc):
    m, n, k = 4, 3, 96
    qa = np.full((m, k), 0x38, dtype=np.uint8)
    qb = np.full((n, k), 0x38, dtype=np.uint8)
    sa = np.array([1, 2, 3, 4], dtype=np.float32)
    sb = np.array([0.5, 1, -1], dtype=np.float32)
    c, bound = orc.gemm_rowwise(qa, qb, sa, sb)
    assert np.array_equal(c, k * np.outer(sa, sb).astype(np.float64))
    assert np.array_equal(bound, np.abs(c))
    sfa = np.full((m, k // 32), 127, dtype=np.uint8)
    sfb = np.full((n, k // 32), 128, dtype=np.uint8)
    cm, _ = orc.gemm_mx(qa, sfa, qb, sfb)
    assert np.all(cm == 2.0 * k)


def test_mx_with_unit_scales_equals_rowwise_with_unit_scales(orc):
    rng = np.random.default_rng(9)
    m, n, k = 7, 5, 160
    qa, qb = _rand_codes(rng, (m, k)), _rand_codes(rng, (n, k))
    c1, b1 = orc.gemm_rowwise(qa, qb, np.ones(m, np.float32), np.ones(n, np.float32))
    c2, b2 = orc.gemm_mx(qa, np.full((m, k // 32), 127, np.uint8), qb, np.full((n, k // 32), 127, np.uint8))
    assert np.array_equal(c1, c2) and np.array_equal(b1, b2)


def test_bound_dominates(orc):
    rng = np.random.default_rng(3)
    qa, qb = _rand_codes(rng, (9, 64)), _rand_codes(rng, (11, 64))
    c, b = orc.gemm_rowwise(qa, qb, rng.random(9).astype(np.float32), rng.random(11).astype(np.float32))
    assert np.all(b >= np.abs(c))
