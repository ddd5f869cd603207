"""fp64 CPU oracle of the low-bit latent cache: 8-bit e4m3 latent codes with one
float32 scale per 64 latent columns, the decoupled RoPE key kept in bf16.

TEST INFRASTRUCTURE ONLY, like ``mla_oracle``: only the tests, the smoke check
and the CPU-baseline leg of ``bench.py`` may call it, and it shares no code with
the CUDA path.

The pages report that the served DeepSeek-V2 model keeps its KV cache at about
6 bits per element ("DeepSeek-V2 review", 4.2 Evaluation, "Inference
efficiency"; "Техотчёт DeepSeek-V2 (2024): MLA и экономика инференса",
"Откуда берутся 93,3%") and give no format.  The reading taken here:

* Only the latent c^KV is quantised.  The decoupled RoPE key k^R is a single
  64-wide vector per token whose rotation carries the position ("Идея 2:
  отделённый RoPE"); it stays bf16, exactly as the bf16 cache stores it.
* Codes are OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
  bits; no infinities; magnitude code 0x7F is NaN; largest finite value 448;
  subnormals m * 2^-9), the narrowest format the B200 converts in one
  instruction.  A 64-column group's codes share one scale: amax = max |x| over
  the group, x the bf16 latent widened to float32, and

      inv   = 448 / amax          (float32 division, round to nearest even)
      scale = amax / 448          (float32 division, round to nearest even)
      code  = e4m3(x * inv)       (float32 product, then round to nearest even,
                                   ties to even, saturating at +-448)

  so the group's largest value maps to +-448.  An all-zero group stores
  scale 0 and zero codes.  The dequantised value is e4m3(code) * scale.
  Both roundings are decided in float32 on both sides, as the GPU does them.
* Row layout, little-endian bytes: the d_c codes; then the d_c / 64 scales as
  float32 from the next 16-byte boundary; then the d_r bf16 RoPE values from
  the 16-byte boundary after that; the row padded to a multiple of 16 bytes.
  At the DeepSeek-V2 shape (d_c 512, d_r 64) a row is 512 + 32 + 128 = 672
  bytes against 1,152 in bf16 (58 %, 9.3 bits per cached element).
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
GROUP = 64


def _r16(x: int) -> int:
    return (x + 15) // 16 * 16


def row_layout(d_c: int, d_r: int):
    """(scale offset, RoPE-key offset, row bytes) of one cache row."""
    assert d_c % GROUP == 0 and d_r % 8 == 0
    scale_off = _r16(d_c)
    kr_off = _r16(scale_off + 4 * (d_c // GROUP))
    return scale_off, kr_off, _r16(kr_off + 2 * d_r)


# ---------------------------------------------------------------------------
# E4M3 (OCP FP8): the value of every code, and round-to-nearest-even encoding
# ---------------------------------------------------------------------------


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """float64 value of each e4m3 code (NaN for 0x7F and 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    out = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """e4m3 codes of finite float32 values: round to nearest, ties to even,
    magnitudes past the largest finite value saturate to +-448."""
    v = np.asarray(y, dtype=np.float32).astype(np.float64)
    assert np.isfinite(v).all()
    sign = np.signbit(v).astype(np.int64) << 7
    a = np.abs(v)
    _, ex = np.frexp(a)                        # a = f * 2**ex, 0.5 <= f < 1 (a > 0)
    e = ex.astype(np.int64) - 1                # a = (2 f) * 2**e
    normal = a >= 2.0 ** -6
    # normal: the significand in units of its last place, q in [8, 16)
    q_n = np.rint(np.where(normal, a / np.exp2(np.where(normal, e, 0) - 3.0), 0.0)).astype(np.int64)
    carry = q_n == 16                          # rounded up into the next binade
    big_e = np.where(carry, e + 1, e) + 7      # biased exponent
    mant = np.where(carry, 0, q_n - 8)
    code_n = (big_e << 3) | mant
    code_n = np.where((big_e > 15) | ((big_e == 15) & (mant == 7)), 0x7E, code_n)
    # subnormal: units of 2^-9; a rounded value of 8 is the smallest normal (code 0x08)
    code_s = np.rint(np.where(normal, 0.0, a / 2.0 ** -9)).astype(np.int64)
    code = np.where(normal, code_n, code_s)
    return (code | sign).astype(np.uint8)


# ---------------------------------------------------------------------------
# latent quantisation per 64-column group
# ---------------------------------------------------------------------------


def quantize_latent(c_bits: np.ndarray):
    """Codes (uint8, same shape) and float32 scales (..., d_c / 64) of bf16
    latent rows c_bits (uint16, last axis d_c)."""
    c = np.asarray(c_bits, dtype=np.uint16)
    d_c = c.shape[-1]
    x = (c.astype(np.uint32) << np.uint32(16)).view(np.float32).reshape(c.shape[:-1] + (d_c // GROUP, GROUP))
    amax = np.max(np.abs(x), axis=-1)                                   # float32, exact
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    inv = np.where(zero, np.float32(0.0), np.float32(E4M3_MAX) / safe).astype(np.float32)
    scale = np.where(zero, np.float32(0.0), safe / np.float32(E4M3_MAX)).astype(np.float32)
    y = (x * inv[..., None]).astype(np.float32)                         # one float32 rounding
    codes = e4m3_encode(y).reshape(c.shape)
    return codes, scale


def dequantize_latent(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """float64 latent rows from codes and their group scales."""
    q = e4m3_decode(codes)
    d_c = q.shape[-1]
    q = q.reshape(q.shape[:-1] + (d_c // GROUP, GROUP))
    return (q * np.asarray(scale, dtype=np.float64)[..., None]).reshape(codes.shape)


def pack_rows(codes: np.ndarray, scale: np.ndarray, k_r_bits: np.ndarray) -> np.ndarray:
    """Cache rows (uint8, (n, row bytes)) from codes (n, d_c), scales (n, d_c/64)
    and the rotated bf16 RoPE keys (n, d_r); padding bytes are zero."""
    n, d_c = codes.shape
    d_r = k_r_bits.shape[-1]
    so, ko, rb = row_layout(d_c, d_r)
    out = np.zeros((n, rb), dtype=np.uint8)
    out[:, :d_c] = codes
    out[:, so:so + 4 * (d_c // GROUP)] = np.ascontiguousarray(scale, dtype="<f4").view(np.uint8).reshape(n, -1)
    out[:, ko:ko + 2 * d_r] = np.ascontiguousarray(k_r_bits, dtype="<u2").view(np.uint8).reshape(n, -1)
    return out


def unpack_rows(rows: np.ndarray, d_c: int, d_r: int):
    """(codes, scales, RoPE-key bits) of cache rows (uint8, (n, row bytes))."""
    so, ko, _ = row_layout(d_c, d_r)
    r = np.ascontiguousarray(rows, dtype=np.uint8)
    codes = r[:, :d_c].copy()
    scale = np.ascontiguousarray(r[:, so:so + 4 * (d_c // GROUP)]).view("<f4").astype(np.float32)
    k_r = np.ascontiguousarray(r[:, ko:ko + 2 * d_r]).view("<u2").astype(np.uint16)
    return codes, scale, k_r
