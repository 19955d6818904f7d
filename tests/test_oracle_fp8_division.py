"""Pin of the quantisation rule's arithmetic: the scale is s = amax / 448 and
the code is e4m3_rn(h / s), each a correctly rounded float32 DIVISION (the
reading of XTuner PR #2089 §Changes this library takes), not the product with
a rounded reciprocal that the PR's review thread constant ``1.0 / FP8_MAX``
suggests (s = amax * RN(1/448), q = e4m3_rn(h * RN(1/s))).

The two readings differ only where a one-ulp float32 difference crosses an E4M3
rounding midpoint, which random inputs almost never hit. Here the inputs are
constructed: for seeded float32 maxima and every E4M3 midpoint m, the float32
values x next to m*s are scanned for one where the two readings give different
codes. The expected codes are worked out in exact rational arithmetic
(``fractions.Fraction``: float32 rounding and E4M3 rounding to nearest, ties
to even, written out here from the IEEE-754 and OCP FP8 definitions), never by
the oracle, and the oracle must give the division reading's code and scale."""
from fractions import Fraction as Q

import numpy as np
import pytest

from oracle import moe_oracle as O


def _rhe(q: Q) -> int:
    """Round a non-negative rational to the nearest integer, ties to even."""
    n = q.numerator // q.denominator
    r = q - n
    if r > Q(1, 2) or (r == Q(1, 2) and n % 2 == 1):
        n += 1
    return n


def _floor_log2(a: Q) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Q(2) ** e > a:
        e -= 1
    if Q(2) ** (e + 1) <= a:
        e += 1
    return e


def rn_f32(q: Q) -> Q:
    """The float32 nearest to q (ties to even), as an exact rational."""
    if q == 0:
        return Q(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = max(_floor_log2(a), -126)
    ulp = Q(2) ** (e - 23)
    return sign * _rhe(a / ulp) * ulp


def e4m3_code(v: Q) -> int:
    """OCP E4M3FN code of a value, round to nearest even, saturating at 448."""
    sign = 0x80 if v < 0 else 0
    a = abs(v)
    if a >= 448:
        return sign | 0x7E
    if a < Q(1, 64):                      # subnormals: multiples of 2**-9
        return sign | _rhe(a * 512)       # 8 lands on 0x08 = 2**-6, also right
    e = _floor_log2(a)
    n = _rhe(a / Q(2) ** (e - 3))         # 8 .. 16
    if n == 16:
        e, n = e + 1, 8
    return sign | min(((e + 7) << 3) | (n - 8), 0x7E)


def f32(v) -> Q:
    return Q(float(np.float32(v)))


def _midpoints():
    """Every midpoint between neighbouring positive finite E4M3 values below 448."""
    vals = sorted({Q(float(x)) for x in O.e4m3_decode_table() if np.isfinite(x) and x >= 0})
    return [(a + b) / 2 for a, b in zip(vals, vals[1:])]


def _find_split(max_tries=400):
    rng = np.random.default_rng(2089)
    mids = _midpoints()
    for _ in range(max_tries):
        amax = f32(rng.uniform(0.5, 8.0))
        s = rn_f32(amax / 448)
        r = rn_f32(1 / s)
        for m in mids[8:]:                # normal range: codes differ in the mantissa
            x0 = rn_f32(m * s)
            ulp = Q(2) ** (_floor_log2(x0) - 23)
            for k in range(-2, 3):
                x = x0 + k * ulp
                if not 0 < x < amax:
                    continue
                div = e4m3_code(rn_f32(x / s))
                rcp = e4m3_code(rn_f32(x * r))
                if div != rcp:
                    return amax, x, s, div, rcp
    return None


def test_exact_helpers_agree_with_the_format_definitions():
    # rn_f32 against numpy's float64 -> float32 rounding where float64 is exact
    rng = np.random.default_rng(1)
    for v in rng.standard_normal(200) * 10.0 ** rng.integers(-30, 30, 200):
        assert rn_f32(Q(float(v))) == Q(float(np.float32(v)))
    # the E4M3 code of every finite value is that value's code
    table = O.e4m3_decode_table()
    for c in range(0x7F):
        assert e4m3_code(Q(float(table[c]))) == c
        # (an exact rational has no negative zero: -0 encodes as 0x00 here)
        assert e4m3_code(-Q(float(table[c]))) == (c | 0x80 if c else 0)


def test_quant_1x128_code_is_a_division_by_the_scale():
    found = _find_split()
    assert found is not None, "no input separating the two readings was found"
    amax, x, s, div, rcp = found
    assert div != rcp
    h = np.zeros((2, 128), dtype=np.float32)
    h[0, 0] = float(amax)
    h[0, 1] = float(x)
    h[1, 5] = -float(amax)                # the same through the sign
    h[1, 9] = -float(x)
    q, sc = O.quant_1x128(h)
    assert Q(float(sc[0, 0])) == s and Q(float(sc[1, 0])) == s
    assert int(q[0, 1]) == div and int(q[1, 9]) == div | 0x80
    assert int(q[0, 0]) == 0x7E and int(q[1, 5]) == 0xFE
    # the 128x128 weight quantiser takes the same rule over its block
    w = np.zeros((128, 128), dtype=np.float32)
    w[17, 3] = float(amax)
    w[90, 64] = float(x)
    qw, sw = O.quant_weight_128x128(w)
    assert Q(float(sw[0, 0])) == s
    assert int(qw[90, 64]) == div and int(qw[17, 3]) == 0x7E


def test_scale_is_a_division_by_448():
    """Scales: s = RN(amax / 448), which differs from RN(amax * RN(1/448)) for
    some maxima; the oracle must give the division, in both quantisers."""
    rng = np.random.default_rng(448)
    r448 = rn_f32(Q(1, 448))
    hits = 0
    for v in rng.uniform(0.01, 100.0, 4000):
        amax = f32(v)
        div = rn_f32(amax / 448)
        if div == rn_f32(amax * r448):
            continue
        hits += 1
        h = np.zeros((1, 128), dtype=np.float32)
        h[0, 3] = float(amax)
        _, sc = O.quant_1x128(h)
        assert Q(float(sc[0, 0])) == div
        w = np.zeros((128, 128), dtype=np.float32)
        w[7, 100] = -float(amax)
        _, sw = O.quant_weight_128x128(w)
        assert Q(float(sw[0, 0])) == div
        if hits >= 20:
            break
    assert hits >= 20


@pytest.mark.parametrize("seed", [0, 1])
def test_exact_reference_matches_oracle_codes_on_random_tiles(seed):
    """Away from constructed midpoints too, every code and scale is the exact
    division reading."""
    rng = np.random.default_rng(seed)
    h = (rng.standard_normal((4, 256)) * rng.uniform(0.01, 50.0, (4, 1))).astype(np.float32)
    q, sc = O.quant_1x128(h)
    for r in range(4):
        for t in range(2):
            tile = h[r, t * 128:(t + 1) * 128]
            s = rn_f32(max(abs(f32(v)) for v in tile) / 448)
            assert Q(float(sc[r, t])) == s
            for c in range(0, 128, 7):
                assert int(q[r, t * 128 + c]) == e4m3_code(rn_f32(f32(tile[c]) / s))
