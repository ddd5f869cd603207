"""Pins of the low-bit cache oracle (CPU only).

The e4m3 values come from the format's definition (OCP FP8 E4M3: bias 7,
3 mantissa bits, no infinities, 0x7F NaN, largest finite 448) and, as a
library special case, from torch's float8_e4m3fn conversions; the quantiser
is pinned by a hand-worked group, its invariants (the group maximum maps to
+-448, groups are independent, scaling a group by a power of two leaves its
codes alone) and the round-to-nearest error bound.
"""

import numpy as np
import torch

from oracle import lowbit_cache as L


def _bf16(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def _finite_codes():
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def test_e4m3_code_values_from_the_format():
    table = {
        0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
        0x30: 0.5, 0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x76: 224.0, 0x77: 240.0,
        0x78: 256.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0,
    }
    got = L.e4m3_decode(np.array(list(table), dtype=np.uint8))
    assert np.array_equal(got, np.array(list(table.values())))
    assert np.signbit(L.e4m3_decode(np.array([0x80], dtype=np.uint8)))[0]
    assert np.isnan(L.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(L.e4m3_decode(codes), ref, equal_nan=True)


def test_e4m3_encode_round_trips_every_finite_code():
    codes = _finite_codes()
    vals = L.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(L.e4m3_encode(vals), codes)


def test_e4m3_encode_ties_to_even():
    pos = np.array([c for c in range(0x7F)], dtype=np.uint8)     # 0 .. 448 in increasing order
    v = L.e4m3_decode(pos)
    assert (np.diff(v) > 0).all()
    mid = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (v[:-1] + v[1:]) / 2)   # midpoints are exact in float32
    got = L.e4m3_encode(mid)
    even = np.where(pos[:-1] % 2 == 0, pos[:-1], pos[1:])             # the neighbour with an even mantissa
    assert np.array_equal(got, even)
    # just off the midpoint the nearer code wins
    lo = np.nextafter(mid, np.float32(0)).astype(np.float32)
    hi = np.nextafter(mid, np.float32(1e9)).astype(np.float32)
    assert np.array_equal(L.e4m3_encode(lo), pos[:-1])
    assert np.array_equal(L.e4m3_encode(hi), pos[1:])


def test_e4m3_encode_matches_torch_float8():
    rng = np.random.default_rng(3)
    y = (rng.standard_normal(100000) * np.exp2(rng.uniform(-14, 9, 100000))).astype(np.float32)
    y = y[np.abs(y) <= 448]
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(L.e4m3_encode(y), ref)


def test_e4m3_encode_saturates():
    y = np.array([448.0, 463.9, 464.0, 480.0, 500.0, 1e6, -470.0, -1e30], dtype=np.float32)
    assert L.e4m3_encode(y).tolist() == [0x7E] * 6 + [0xFE] * 2


def test_quantize_hand_example():
    # one group of 64 with amax 1.0: inv = 448, scale = 1/448 rounded to float32
    x = np.zeros(64, dtype=np.float32)
    x[0], x[1], x[2], x[3] = 1.0, -0.5, 0.25, 0.0009765625            # the last is 2^-10
    codes, scale = L.quantize_latent(_bf16(x)[None, :])
    assert scale.shape == (1, 1) and scale[0, 0] == np.float32(1.0) / np.float32(448.0)
    # 1 * 448 = 448 -> 0x7E;  -0.5 * 448 = -224 = -1.75 * 2^7 -> sign, E = 14, M = 6 -> 0xF6;
    # 0.25 * 448 = 112 = 1.75 * 2^6 -> E = 13, M = 6 -> 0x6E;  2^-10 * 448 = 0.4375 = 1.75 * 2^-2
    # -> E = 5, M = 6 -> 0x2E;  zeros -> 0x00
    assert codes[0, :4].tolist() == [0x7E, 0xF6, 0x6E, 0x2E]
    assert (codes[0, 4:] == 0).all()
    back = L.dequantize_latent(codes, scale)[0]
    assert back[0] == 448.0 * float(scale[0, 0]) and back[3] == 0.4375 * float(scale[0, 0])


def test_quantize_group_maximum_maps_to_448():
    rng = np.random.default_rng(5)
    c = _bf16(rng.standard_normal((16, 512)).astype(np.float32))
    codes, scale = L.quantize_latent(c)
    x = (c.astype(np.uint32) << np.uint32(16)).view(np.float32).reshape(16, 8, 64)
    k = np.argmax(np.abs(x), axis=-1)
    top = np.take_along_axis(codes.reshape(16, 8, 64), k[..., None], axis=-1)[..., 0]
    assert ((top & 0x7F) == 0x7E).all()
    assert np.array_equal(scale, (np.max(np.abs(x), axis=-1) / np.float32(448)).astype(np.float32))


def test_quantize_groups_are_independent():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 256)).astype(np.float32)
    c0 = _bf16(x)
    x2 = (c0.astype(np.uint32) << np.uint32(16)).view(np.float32).copy()
    x2[:, 64:128] *= 8.0                                              # one group, by a power of two
    codes0, s0 = L.quantize_latent(c0)
    codes1, s1 = L.quantize_latent(_bf16(x2))
    assert np.array_equal(codes0, codes1)
    assert np.array_equal(s1[:, 1], s0[:, 1] * np.float32(8.0))
    assert np.array_equal(np.delete(s1, 1, axis=1), np.delete(s0, 1, axis=1))


def test_dequantize_error_bound():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    c = _bf16(x)
    codes, scale = L.quantize_latent(c)
    xb = (c.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    back = L.dequantize_latent(codes, scale)
    s = np.repeat(scale.astype(np.float64), 64, axis=1)
    # half a unit in the last place of a 3-bit significand (2^-4 relative), a
    # subnormal step of 2^-9 units below 2^-6, and the float32 roundings of
    # inv, the product and the scale
    bound = (2.0 ** -4 + 2.0 ** -20) * np.abs(xb) + 2.0 ** -10 * s
    assert (np.abs(back - xb) <= bound).all()
    assert np.abs(back - xb).max() > 0


def test_zero_group():
    c = np.zeros((2, 128), dtype=np.uint16)
    c[1, 64:] = _bf16(np.linspace(-1, 1, 64).astype(np.float32))
    codes, scale = L.quantize_latent(c)
    assert (codes[0] == 0).all() and (codes[1, :64] == 0).all()
    assert scale[0].tolist() == [0.0, 0.0] and scale[1, 0] == 0.0 and scale[1, 1] > 0
    assert (L.dequantize_latent(codes, scale)[0] == 0).all()


def test_row_layout_and_size():
    assert L.row_layout(512, 64) == (512, 544, 672)     # DeepSeek-V2: 58 % of the bf16 row (1,152 bytes)
    assert L.row_layout(64, 32) == (64, 80, 144)
    assert L.row_layout(256, 64) == (256, 272, 400)
    so, ko, rb = L.row_layout(512, 64)
    assert 8.0 * rb / (512 + 64) == 9.333333333333334


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(8)
    c = _bf16(rng.standard_normal((5, 512)).astype(np.float32))
    kr = _bf16(rng.standard_normal((5, 64)).astype(np.float32))
    codes, scale = L.quantize_latent(c)
    rows = L.pack_rows(codes, scale, kr)
    assert rows.shape == (5, 672)
    c2, s2, k2 = L.unpack_rows(rows, 512, 64)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scale) and np.array_equal(k2, kr)
    # the scales sit at byte 512 as little-endian float32, the key at byte 544 as bf16
    assert rows[0, 512:516].tobytes() == np.float32(scale[0, 0]).tobytes()
    assert rows[0, 544:546].tobytes() == np.uint16(kr[0, 0]).tobytes()


def test_row_padding_is_zero():
    rng = np.random.default_rng(9)
    c = _bf16(rng.standard_normal((3, 64)).astype(np.float32))
    kr = _bf16(rng.standard_normal((3, 32)).astype(np.float32))
    codes, scale = L.quantize_latent(c)
    rows = L.pack_rows(codes, scale, kr)
    assert rows.shape == (3, 144)
    assert (rows[:, 68:80] == 0).all()                  # between the one scale and the key
    assert np.array_equal(rows[:, 80:144].view("<u2"), kr)


def test_codes_are_decided_in_float32():
    # amax 1.53125, x 1.3671875: x * 448 / amax is exactly 400, the midpoint of
    # 384 (code 0x7C) and 416 (0x7D); float32 rounds inv = 448 / amax up to
    # 292.57144165..., so the float32 product is 400 + 2^-15 and the code 0x7D.
    # amax 1.9375, x 1.453125: x * inv rounds to exactly 336, the midpoint of
    # 320 (0x7A) and 352 (0x7B), which goes to the even 0x7A (x / scale would
    # give 336 + 2^-15 and 0x7B).
    for amax, x, code in ((1.53125, 1.3671875, 0x7D), (1.9375, 1.453125, 0x7A)):
        g = np.zeros(64, dtype=np.float32)
        g[0], g[1] = amax, x
        inv = np.float32(448.0) / np.float32(amax)
        assert (np.float32(x) * inv == np.float32(400.0 + 2.0 ** -15)) == (code == 0x7D)
        codes, _ = L.quantize_latent(_bf16(g)[None, :])
        assert codes[0, 0] == 0x7E and codes[0, 1] == code
