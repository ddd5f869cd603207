"""Planted-mistake check of the low-bit cache pins (CPU only): each entry plants
one plausible slip in a private copy of the oracle module and asserts that at
least one pin in ``test_oracle_lowbit_pins`` fails on it, and, where the slip
is in the quantiser, that the exact-arithmetic check in
``test_oracle_lowbit_exact`` fails too."""

import inspect
import os
import types

import pytest

import tests.test_oracle_lowbit_exact as exact
import tests.test_oracle_lowbit_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "lowbit_cache.py")

MUTATIONS = {
    "encode_truncates": ("q_n = np.rint(np.where(normal,", "q_n = np.floor(np.where(normal,"),
    "encode_bias_8": ("big_e = np.where(carry, e + 1, e) + 7", "big_e = np.where(carry, e + 1, e) + 8"),
    "encode_subnormal_step": ("code_s = np.rint(np.where(normal, 0.0, a / 2.0 ** -9))",
                              "code_s = np.rint(np.where(normal, 0.0, a / 2.0 ** -10))"),
    "encode_no_saturation": ("code_n = np.where((big_e > 15) | ((big_e == 15) & (mant == 7)), 0x7E, code_n)",
                             "code_n = code_n & 0x7F"),
    "encode_drops_sign": ("return (code | sign).astype(np.uint8)", "return code.astype(np.uint8)"),
    "decode_bias_6": ("(1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)",
                      "(1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 6.0)"),
    "decode_subnormal_step": ("mag = np.where(e == 0, m * 2.0 ** -9,", "mag = np.where(e == 0, m * 2.0 ** -10,"),
    "scale_stored_inverted": ("scale = np.where(zero, np.float32(0.0), safe / np.float32(E4M3_MAX))",
                              "scale = np.where(zero, np.float32(0.0), np.float32(E4M3_MAX) / safe)"),
    "one_scale_per_row": ("amax = np.max(np.abs(x), axis=-1)                                   # float32, exact",
                          "amax = np.max(np.abs(x), axis=(-2, -1))[..., None] * np.ones(x.shape[-2], np.float32)"),
    "product_in_double": ("y = (x * inv[..., None]).astype(np.float32)",
                          "y = (x.astype(np.float64) * (448.0 / np.where(zero, 1.0, amax.astype(np.float64)))[..., None])"),
    "divide_by_scale": ("y = (x * inv[..., None]).astype(np.float32)",
                        "y = (x / np.where(zero, np.float32(1.0), scale)[..., None]).astype(np.float32)"),
    "key_before_scales": ("kr_off = _r16(scale_off + 4 * (d_c // GROUP))", "kr_off = scale_off"),
}


def _mutated_module(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("lowbit_cache_mutant")
    exec(compile(src.replace(old, new), "lowbit_cache_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    mod = _mutated_module(*MUTATIONS[name])
    monkeypatch.setattr(pins, "L", mod)
    failures = 0
    for fname, fn in inspect.getmembers(pins, inspect.isfunction):
        if not fname.startswith("test_"):
            continue
        try:
            fn()
        except Exception:
            failures += 1
    assert failures >= 1, f"no pin caught mutation {name}"


# slips in the quantiser's arithmetic (not in the layout or the decoder), which
# the exact-rounding check must catch on its own
QUANTISER = ("encode_truncates", "encode_bias_8", "encode_subnormal_step", "encode_drops_sign",
             "scale_stored_inverted", "one_scale_per_row", "product_in_double", "divide_by_scale")


@pytest.mark.parametrize("name", QUANTISER)
def test_exact_check_catches_planted_mistake(name, monkeypatch):
    mod = _mutated_module(*MUTATIONS[name])
    monkeypatch.setattr(exact, "L", mod)
    failures = 0
    for fname, fn in inspect.getmembers(exact, inspect.isfunction):
        if not fname.startswith("test_"):
            continue
        try:
            fn()
        except Exception:
            failures += 1
    assert failures >= 1, f"the exact check missed mutation {name}"
