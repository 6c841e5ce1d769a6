"""Pins for the oracle's E4M3 and UE8M0 format code against facts that do not
come from the oracle itself: the page-stated maximum (448), the closed-form
bit definition evaluated independently here in exact integer arithmetic,
torch's own float8_e4m3fn conversion (a library routine), and exhaustive
bracketing of the MX exponent in exact rational arithmetic."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return json.load(f)


def _e4m3_exact(code: int):
    """Exact value of a finite E4M3 code as a Fraction, from the bit fields
    (integer arithmetic only).  Every finite value is an integer multiple of
    2^-9: subnormal m * 2^-9, normal (8+m) * 2^(E-1) * 2^-9."""
    s, E, m = code >> 7, (code >> 3) & 15, code & 7
    if E == 15 and m == 7:
        return None
    units = m if E == 0 else (8 + m) << (E - 1)
    v = Fraction(units, 512)
    return -v if s else v


def _all_bf16_finite():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float()
    keep = torch.isfinite(x)
    return bits[keep.numpy()], x[keep]


# ------------------------------------------------------------------ decode

def test_decode_matches_bitfield_definition(orc):
    t = orc.e4m3_decode_table()
    for c in range(256):
        ref = _e4m3_exact(c)
        if ref is None:
            assert math.isnan(t[c])
        else:
            assert Fraction(t[c]) == ref, hex(c)


def test_decode_invariants(orc):
    t = orc.e4m3_decode_table()
    finite = np.isfinite(t)
    assert finite.sum() == 254
    assert set(np.nonzero(~finite)[0].tolist()) == {0x7F, 0xFF}
    assert not np.isinf(t).any()                      # no infinities in E4M3fn
    assert t[0x7E] == _facts()["e4m3_max_finite"]["value"] == np.nanmax(t)
    assert t[0x01] == 2.0 ** -9                       # smallest subnormal
    assert t[0x08] == 2.0 ** -6                       # smallest normal
    for c in range(0x7F):                             # sign symmetry
        assert t[c | 0x80] == -t[c] or (c == 0 and t[0x80] == 0.0)
    assert np.all(np.diff(t[0x00:0x7F]) > 0)          # increasing over 0x00..0x7E


def test_decode_matches_torch_float8(orc):
    t = orc.e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    same = (t == ref) | (np.isnan(t) & np.isnan(ref))
    assert same.all()


# ------------------------------------------------------------------ encode

def test_encode_exhaustive_bf16_against_torch(orc):
    bits, x = _all_bf16_finite()
    ours = orc.e4m3_encode(x.double().numpy())
    ref = torch.clamp(x, -448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(hex(int(bits[i])), float(x[i]), ours[i], ref[i]) for i in bad[:10]]


def test_encode_midpoints_go_to_even_code(orc):
    t = orc.e4m3_decode_table()
    for c in range(0x7E):
        mid = (Fraction(t[c]) + Fraction(t[c + 1])) / 2
        even = c if c % 2 == 0 else c + 1
        assert orc.e4m3_encode([float(mid)])[0] == even
        assert orc.e4m3_encode([-float(mid)])[0] == (0x80 | even)


def test_encode_is_nearest_brute_force(orc):
    """Random doubles against an independent argmin over the exact table."""
    rng = np.random.default_rng(123)
    v = np.concatenate([rng.standard_normal(3000) * 50,
                        rng.standard_normal(1000) * 1e-2,
                        rng.uniform(-500, 500, 1000)])
    vals = [_e4m3_exact(c) for c in range(0x7F)]
    ours = orc.e4m3_encode(v)
    for x, q in zip(v, ours):
        a = min(abs(Fraction(float(x))), Fraction(448))
        d = [abs(a - val) for val in vals]
        best = min(d)
        cands = [c for c in range(0x7F) if d[c] == best]
        c = cands[0] if len(cands) == 1 else [cc for cc in cands if cc % 2 == 0][0]
        exp = c | (0x80 if math.copysign(1.0, x) < 0 else 0)
        assert q == exp, (x, q, exp)


def test_encode_round_trip_and_saturation(orc):
    t = orc.e4m3_decode_table()
    for c in range(256):
        if np.isfinite(t[c]):
            v = -0.0 if c == 0x80 else t[c]
            assert orc.e4m3_encode([v])[0] == c
    assert list(orc.e4m3_encode([448.0, 449.0, 463.9, 464.0, 465.0, 1e30])) == [0x7E] * 6
    assert list(orc.e4m3_encode([-448.0, -1e30])) == [0xFE] * 2
    assert list(orc.e4m3_encode([0.0, -0.0, -1e-30, 2.0 ** -11])) == [0x00, 0x80, 0x80, 0x00]


# --------------------------------------------------------------- UE8M0 / MX

def test_mx_exponent_brackets_exactly_for_every_bf16(orc):
    """e = ceil(log2(a/448)) + 127 is the unique integer with
    448 * 2^(e-128) < a <= 448 * 2^(e-127); checked in exact rationals for
    every positive finite bf16 a, with the [0, 254] clamp."""
    bits, x = _all_bf16_finite()
    pos = x > 0
    a = x[pos].double().numpy()
    e = orc.mx_exponent(a)
    M = 448
    for ai, ei in zip(a, e):
        fa = Fraction(float(ai))
        assert 0 <= ei <= 254
        assert fa <= M * Fraction(2) ** (int(ei) - 127)
        if ei > 0:
            assert fa > M * Fraction(2) ** (int(ei) - 128)


def test_mx_exponent_integer_closed_form(orc):
    """For a bf16 a with exponent field Ea and mantissa field m:
    a/448 = (1+m/128)/1.75 * 2^(Ea-127-8), so e = Ea - 8 + [m > 96]
    (1 + m/128 > 1.75 iff m > 96), clamped at 0; subnormals give 0."""
    bits, x = _all_bf16_finite()
    pos = (x > 0).numpy()
    b = bits[pos].astype(np.int64)
    Ea = (b >> 7) & 0xFF
    m = b & 0x7F
    closed = np.where(Ea == 0, 0, np.clip(Ea - 8 + (m > 96), 0, 254))
    e = orc.mx_exponent(x[torch.from_numpy(pos)].double().numpy())
    assert np.array_equal(e, closed)


def test_mx_exponent_special_values(orc):
    assert orc.mx_exponent([0.0])[0] == 127                  # zero block: scale 1
    assert orc.mx_exponent([448.0])[0] == 127
    assert orc.mx_exponent([448.0 * 2 ** -20])[0] == 107
    assert orc.mx_exponent([1e-38])[0] == 0                   # low clamp
    scale = [math.ldexp(1.0, int(e) - 127) for e in orc.mx_exponent([1.0, 1e6])]
    assert scale == [2.0 ** -8, 2.0 ** 12]                    # UE8M0 = 2^(e-127)
