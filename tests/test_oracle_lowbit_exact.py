"""The low-bit cache oracle against exact rational arithmetic (CPU only).

Every rounding the quantiser defines -- inv = RN32(448 / amax), scale =
RN32(amax / 448), y = RN32(x * inv), code = the e4m3 value nearest to y (ties to
the even code, saturating at 448) -- is redone here with Fractions, so the
check does not rest on numpy's float32 arithmetic or on the oracle's encoder.
"""

from fractions import Fraction

import numpy as np

from oracle import lowbit_cache as L


def _rn32(q: Fraction) -> Fraction:
    """q rounded to the nearest float32, ties to even (normal range)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    assert -126 <= e <= 127
    m = a / Fraction(2) ** (e - 23)           # in [2^23, 2^24)
    r = m.numerator // m.denominator
    rem = m - r
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and r % 2 == 1):
        r += 1
    return sign * r * Fraction(2) ** (e - 23)


def _e4m3_values():
    """(value, code) of the finite non-negative e4m3 codes, ascending."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        v = Fraction(m, 512) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        out.append((v, c))
    return out


VALS = _e4m3_values()


def _e4m3_exact(y: Fraction) -> int:
    a = abs(y)
    if a >= 448:
        code = 0x7E
    else:
        code = None
        for (v0, c0), (v1, c1) in zip(VALS, VALS[1:]):
            if v0 <= a <= v1:
                d0, d1 = a - v0, v1 - a
                code = c0 if d0 < d1 else c1 if d1 < d0 else (c0 if c0 % 2 == 0 else c1)
                break
    return code | (0x80 if y < 0 else 0)


def _bf16_values(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = x.view(np.uint32)
    bits = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    return bits


def _exact_group(bits):
    xs = [Fraction(float((np.uint32(b) << np.uint32(16)).view(np.float32))) for b in bits]
    amax = max(abs(x) for x in xs)
    if amax == 0:
        return [0] * len(xs), Fraction(0)
    inv = _rn32(Fraction(448) / amax)
    scale = _rn32(amax / Fraction(448))
    return [_e4m3_exact(_rn32(x * inv)) for x in xs], scale


def test_quantiser_matches_exact_rounding():
    rng = np.random.default_rng(11)
    rows = np.concatenate([_bf16_values(rng, (6, 128)), _bf16_values(rng, (6, 128), scale=1e-3),
                           _bf16_values(rng, (6, 128), scale=300.0)])
    codes, scale = L.quantize_latent(rows)
    for r in range(rows.shape[0]):
        for g in range(2):
            want_codes, want_scale = _exact_group(rows[r, 64 * g:64 * (g + 1)])
            assert codes[r, 64 * g:64 * (g + 1)].tolist() == want_codes, (r, g)
            assert Fraction(float(scale[r, g])) == want_scale, (r, g)


def test_quantiser_matches_exact_rounding_at_the_midpoint_cases():
    # groups built around the two inputs whose code the float32 product decides
    for amax, x in ((1.53125, 1.3671875), (1.9375, 1.453125)):
        g = np.zeros(64, dtype=np.float32)
        g[0], g[1], g[2] = amax, x, -x
        bits = (g.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
        codes, scale = L.quantize_latent(bits[None, :])
        want_codes, want_scale = _exact_group(bits)
        assert codes[0].tolist() == want_codes
        assert Fraction(float(scale[0, 0])) == want_scale


def test_e4m3_encoder_matches_exact_nearest_value():
    rng = np.random.default_rng(12)
    y = (rng.standard_normal(3000) * np.exp2(rng.uniform(-12, 9, 3000))).astype(np.float32)
    got = L.e4m3_encode(y)
    want = [_e4m3_exact(Fraction(float(v))) for v in y]
    assert got.tolist() == want
