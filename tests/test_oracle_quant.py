"""Pins of the quantizer oracle against what the definition and the mathematics fix.

None of these re-type the oracle's formula: they check invariants (code range, constant
groups), a closed-form error bound, brute-force optimality over all 16 codes with exact
rational arithmetic, exact rational rounding of the stored scale and of the dequantized
value, hand-worked cases (tests/golden/quant_hand_cases.json), the axis-0/axis-1
transposition identity, and the storage cost against the README's "about 70 %" weight
memory saving (FlexGen README mirror, "Handle out-of-memory" tips).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import fg_synth
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------------------
# exact rounding of a rational to a binary float format (independent of numpy)
def round_to_format(x: Fraction, mant_bits: int, emin: int, emax: int) -> Fraction:
    """Round-to-nearest-even of the rational x to a float with `mant_bits` fraction bits,
    minimum normal exponent emin and maximum exponent emax (overflow -> inf not needed)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - mant_bits)
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    assert e <= emax
    return sign * fl * ulp


def rn16(x: Fraction) -> Fraction:
    return round_to_format(x, 10, -14, 15)


def rn32(x: Fraction) -> Fraction:
    return round_to_format(x, 23, -126, 127)


def F(v) -> Fraction:
    return Fraction(float(v))


def _groups(dist, n_groups, g, seed=7, stream=3, scale=1.0):
    x = fg_synth.tensor(seed, stream, (n_groups, g), dist, scale)
    return x


DISTS = [("normal", 0.02), ("normal", 1.0), ("uniform", 1.0), ("t3", 1.0), ("outlier", 1.0)]


# ----------------------------------------------------------------------------------------
def test_hand_worked_cases():
    cases = json.load(open(os.path.join(GOLDEN, "quant_hand_cases.json")))["cases"]
    for c in cases:
        x = np.array(c["x"], dtype=np.float16)[None, :]
        q, mn, s = oracle.quantize_groups(x)
        assert q[0].tolist() == c["codes"], c["why"]
        assert float(mn[0]) == c["min"], c["why"]
        if c["min"] == 0:
            assert not np.signbit(mn[0]), c["why"]
        if "scale_bits" in c:
            assert int(s.view(np.uint16)[0]) == c["scale_bits"], c["why"]
        else:
            assert float(s[0]) == c["scale"] and not np.signbit(s[0]), c["why"]   # s >= +0
        dq = oracle.dequantize_groups(q, mn, s)[0]
        if "dequant_bits" in c:
            assert dq.view(np.uint16).tolist() == c["dequant_bits"], c["why"]
        else:
            assert dq.astype(np.float64).tolist() == [float(v) for v in c["dequant"]], c["why"]


@pytest.mark.parametrize("dist,scale", DISTS)
@pytest.mark.parametrize("g", [32, 64, 128])
def test_codes_in_range_and_error_bound(dist, scale, g):
    x = _groups(dist, 512, g, scale=scale)
    q, mn, s = oracle.quantize_groups(x)
    assert q.dtype == np.uint8 and q.max() <= 15 and q.min() >= 0
    xd = oracle.dequantize_groups(q, mn, s).astype(np.float64)
    xf = x.astype(np.float64)
    sf = s.astype(np.float64)[:, None]
    # ulp of the fp16 result: 2^(floor(log2|x'|) - 10), at least the subnormal step 2^-24
    mag = np.maximum(np.abs(xd), 2.0 ** -14)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 10)
    err = np.abs(xf - xd)
    pos = sf[:, 0] > 0
    bound = sf * 0.5 * (1 + 2.0 ** -20) + 0.5 * ulp
    assert np.all(err[pos] <= bound[pos])
    # min reproduced exactly at code 0; max element gets code 15 when s > 0
    assert np.all(xd.min(axis=1) == xf.min(axis=1))
    rows = np.where(pos)[0]
    amax = xf[rows].argmax(axis=1)
    assert np.all(q[rows, amax] == 15)


def test_constant_groups_round_trip_exactly():
    vals = [0.0, -0.0, 1.0, -3.5, 65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -20), 0.1, 1234.0]
    x = np.array([[v] * 64 for v in vals], dtype=np.float16)
    q, mn, s = oracle.quantize_groups(x)
    assert np.all(q == 0) and np.all(s == 0)
    xd = oracle.dequantize_groups(q, mn, s)
    # exact round trip (zeros come back as +0, which compares equal to -0)
    assert np.all(xd.astype(np.float64) == x.astype(np.float64))


def test_underflow_groups():
    # d/15 below half the smallest subnormal -> s == 0, codes 0, error <= d
    x = np.array([[1.0] * 63 + [1.0 + 2.0 ** -10]], dtype=np.float16)
    q, mn, s = oracle.quantize_groups(x)
    assert s[0] != 0          # d = 2^-10: d/15 is representable -> not underflow
    tiny = np.array([[0.0] * 63 + [2.0 ** -24]], dtype=np.float16)
    q, mn, s = oracle.quantize_groups(tiny)
    assert s[0] == 0 and np.all(q == 0)
    d = 2.0 ** -24
    assert np.all(np.abs(oracle.dequantize_groups(q, mn, s).astype(np.float64) - tiny) <= d)


def test_scale_is_exact_double_rounding_of_range():
    x = _groups("t3", 300, 64, seed=11)
    _, mn, s = oracle.quantize_groups(x)
    for i in range(x.shape[0]):
        vals = [F(v) for v in x[i]]
        lo, hi = min(vals), max(vals)
        assert F(mn[i]) == lo
        d = rn32(hi - lo)
        expect = rn16(rn32(d / 15))
        assert F(s[i]) == expect


@pytest.mark.parametrize("g", [4, 8, 16, 64])
def test_brute_force_rne_optimal(g):
    rng = np.random.default_rng(1000 + g)
    groups = []
    for _ in range(60):
        groups.append(rng.standard_normal(g).astype(np.float16))
    # adversarial: exact ties (x - mn)/s = k + 1/2 with s = 1 and s = 2
    for k in range(15):
        base = [0.0, 15.0] + [k + 0.5] * (g - 2)
        groups.append(np.array(base, np.float16))
        base2 = [-30.0, 0.0] + [-30.0 + 2 * k + 1.0] * (g - 2)
        groups.append(np.array(base2, np.float16))
    x = np.stack(groups)
    q, mn, s = oracle.quantize_groups(x)
    for i in range(x.shape[0]):
        sm, ss = F(mn[i]), F(s[i])
        if ss == 0:
            continue
        for j in range(g):
            xv = F(x[i, j])
            errs = [abs(xv - (sm + c * ss)) for c in range(16)]
            best = min(errs)
            chosen = int(q[i, j])
            exact_ratio = (xv - sm) / ss
            # within fp32 rounding of a half-integer either neighbour is optimal-equivalent
            near_tie = abs(exact_ratio - (exact_ratio.numerator // exact_ratio.denominator) - Fraction(1, 2)) \
                < Fraction(1, 2 ** 20) * max(1, abs(exact_ratio))
            if near_tie and exact_ratio < 15:
                assert errs[chosen] - best <= ss * Fraction(1, 2 ** 19)
            else:
                assert errs[chosen] == best, (i, j, chosen, errs)
            ties = [c for c in range(16) if errs[c] == best]
            if len(ties) == 2:
                # exact tie in exact arithmetic: the even code wins
                assert chosen == [c for c in ties if c % 2 == 0][0]


def test_dequant_is_single_rounding_of_exact_value():
    rng = np.random.default_rng(5)
    mn = rng.standard_normal(400).astype(np.float16)
    s = np.abs(rng.standard_normal(400) * 0.3).astype(np.float16)
    # include subnormal scales and mins and large magnitudes
    s[:20] = np.float16(2.0 ** -24) * np.arange(1, 21, dtype=np.float16)
    mn[20:40] = np.float16(2.0 ** -20)
    mn[40:60] = np.float16(-60000.0)
    s[40:60] = np.float16(8000.0)
    q = rng.integers(0, 16, size=(400, 8)).astype(np.uint8)
    xd = oracle.dequantize_groups(q, mn, s)
    for i in range(400):
        for j in range(8):
            expect = rn16(F(mn[i]) + int(q[i, j]) * F(s[i]))
            assert F(xd[i, j]) == expect


@pytest.mark.parametrize("g", [32, 64])
def test_axis0_is_transpose_of_axis1(g):
    x = fg_synth.tensor(3, 9, (2 * g, 96), "uniform", 2.0)
    c0, p0 = oracle.quantize_pack(x, g, axis=0)
    c1, p1 = oracle.quantize_pack(np.ascontiguousarray(x.T), g, axis=1)
    assert np.array_equal(oracle.unpack_nibbles(c0), oracle.unpack_nibbles(c1).T)
    assert np.array_equal(p0.view(np.uint16), p1.transpose(1, 0, 2).view(np.uint16))
    d0 = oracle.dequantize(c0, p0, 2 * g, 96, g, 0)
    d1 = oracle.dequantize(c1, p1, 96, 2 * g, g, 1)
    assert np.array_equal(d0.view(np.uint16), d1.T.view(np.uint16))


def test_packing_layout():
    codes = np.arange(16, dtype=np.uint8)[None, :].repeat(2, 0)
    packed = oracle.pack_nibbles(codes)
    assert packed[0].tolist() == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    assert np.array_equal(oracle.unpack_nibbles(packed), codes)


@pytest.mark.parametrize("g,expect_pct", [(32, 68.75), (64, 71.875), (128, 73.4375)])
def test_storage_matches_readme_about_70_percent(g, expect_pct):
    rows, cols = 4 * g, 256
    x = fg_synth.tensor(1, 1, (rows, cols), "normal", 0.02)
    codes, params = oracle.quantize_pack(x, g, 1)
    nbytes = codes.nbytes + params.nbytes
    assert nbytes == oracle.storage_bytes(rows * cols, g) == rows * cols // 2 + 4 * rows * cols // g
    saving = 100.0 * (1 - nbytes / (2 * rows * cols))
    assert saving == pytest.approx(expect_pct)
    assert abs(saving - 70.0) < 4.0          # the README mirror states a saving of roughly 70 %


# ----------------------------------------------------------------------------------------
def test_oracle_fp16_rounding_is_exact_rne():
    """The oracle's own double -> fp16 rounding against exact rational rounding: halfway
    points between neighbours (ties to even), values just off them, subnormals, the
    smallest normal, and the overflow boundary (65520 = halfway between 65504 and 2^16)."""
    from oracle import _lib
    L = _lib.lib()
    rng = np.random.default_rng(3)
    vals = []
    for bits in rng.integers(0, 0x7BFF, 300):        # finite fp16 values and their midpoints
        a = float(np.uint16(bits).view(np.float16))
        b = float(np.uint16(bits + 1).view(np.float16))
        mid = (a + b) / 2
        vals += [a, mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf)]
    vals += [2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 65504.0, 65519.99, 65520.0, 1e-30]
    vals += list(rng.standard_normal(200) * 10.0 ** rng.integers(-6, 4, 200))
    for v in vals:
        for sv in (v, -v):
            got = int(L.orc_d2h(sv))
            if abs(sv) >= 65520.0:
                assert got & 0x7FFF == 0x7C00
                continue
            exp = rn16(F(sv))
            assert F(np.uint16(got).view(np.float16)) == exp, (sv, hex(got))
            assert (got >> 15) == (1 if np.signbit(sv) else 0)
