"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each test below is chosen so that a plausible slip in the oracle (a transposed
weight, a wrong RoPE sign or pairing, a missing term, an off-by-one in the mask,
the wrong score scale) fails at least one of them. None of them re-types the
oracle's own formula.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# bf16 rounding helper vs a library routine
# --------------------------------------------------------------------------

def test_f32_to_bf16_matches_torch_including_ties():
    r = _rng(1)
    x = r.standard_normal(20000).astype(np.float32)
    # plant exact ties: low 16 bits = 0x8000 with both parities of the kept LSB
    u = x.view(np.uint32).copy()
    u[:2000] = (u[:2000] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = u.view(np.float32)
    ours = O.f32_to_bf16_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# RoPE ("MLA 논문정리", "MLA 코드 구현")
# --------------------------------------------------------------------------

def test_rope_inv_freq_closed_form():
    # base^(-2m/d): d=4 -> [1, base^-1/2]; with base 10000 that is [1, 0.01]
    assert np.allclose(O.rope_inv_freq(4, 10000.0), [1.0, 0.01], rtol=0, atol=1e-15)
    f = O.rope_inv_freq(64, 10000.0)
    assert f.shape == (32,)
    assert f[0] == 1.0 and abs(f[31] - 10000.0 ** (-31 / 32)) < 1e-18
    assert np.all(np.diff(f) < 0)


def test_rope_position_zero_is_identity():
    x = _rng(2).standard_normal((5, 64))
    assert np.array_equal(O.rope_rotate(x, np.zeros(5)), x)


def test_rope_matches_complex_rotation():
    # Half-split pairing (m, m + d/2) rotated by +theta is multiplication of
    # the complex number x_m + i x_{m+d/2} by exp(i theta).
    r = _rng(3)
    d = 16
    x = r.standard_normal((7, d))
    pos = r.integers(0, 5000, size=7)
    z = (x[:, : d // 2] + 1j * x[:, d // 2:]) * np.exp(
        1j * pos[:, None] * (10000.0 ** (-np.arange(0, d, 2) / d)))
    want = np.concatenate([z.real, z.imag], axis=1)
    assert np.allclose(O.rope_rotate(x, pos), want, rtol=0, atol=1e-12)


def test_rope_preserves_pair_norms():
    r = _rng(4)
    x = r.standard_normal((9, 64))
    y = O.rope_rotate(x, r.integers(0, 131072, size=9))
    n_in = x[:, :32] ** 2 + x[:, 32:] ** 2
    n_out = y[:, :32] ** 2 + y[:, 32:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-12, atol=0)


def test_rope_scores_depend_on_relative_position_only():
    r = _rng(5)
    q, k = r.standard_normal(64), r.standard_normal(64)
    for p, pk, shift in [(10, 3, 100), (4000, 17, 2), (0, 0, 777)]:
        a = O.rope_rotate(q, p) @ O.rope_rotate(k, pk)
        b = O.rope_rotate(q, p + shift) @ O.rope_rotate(k, pk + shift)
        assert abs(a - b) < 1e-9


def test_rope_f32_table_emulation_tracks_fp64_rotation():
    # The bit-level emulation of the GPU arithmetic stays within bf16 rounding
    # (plus float32 table error) of the fp64 rotation.
    r = _rng(6)
    xb = O.f32_to_bf16_rne(r.standard_normal((300, 64)).astype(np.float32))
    pos = r.integers(0, 4096, size=300)
    tab = O.rope_table_f32(4096, 64)
    got = O.bf16_to_f64(O.rope_emulate_bf16(xb, pos, tab))
    want = O.rope_rotate(O.bf16_to_f64(xb), pos)
    assert np.max(np.abs(got - want) / (np.abs(want) + 1e-3)) < 2 ** -8 + 1e-4


def _round_rne(x, mant_bits):
    """Exact round-to-nearest-even of a rational to `mant_bits` significand bits
    (normal range only), written out on fractions.Fraction."""
    from fractions import Fraction
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    x, e = abs(Fraction(x)), 0
    while x >= 2:
        x, e = x / 2, e + 1
    while x < 1:
        x, e = x * 2, e - 1
    scaled = x * 2 ** (mant_bits - 1)
    q, rem = divmod(scaled.numerator, scaled.denominator)
    half = Fraction(rem, scaled.denominator)
    if half > Fraction(1, 2) or (half == Fraction(1, 2) and q % 2 == 1):
        q += 1
    return sign * Fraction(q, 2 ** (mant_bits - 1)) * Fraction(2) ** e


def test_rope_emulation_rounds_each_product_then_the_sum():
    """The GPU's RoPE rounds x1*c and x2*s to float32 separately, then their
    difference (sum) to float32, then to bf16.  On these inputs the two
    products nearly cancel, so a fused multiply-add (one rounding of
    x1*c - fl(x2*s)) or a single rounding of the exact value lands on another
    bf16 -- the expected bits below are the separately rounded result,
    evaluated in exact rational arithmetic."""
    from fractions import Fraction
    f32 = lambda v: _round_rne(v, 24)
    bf16 = lambda v: _round_rne(v, 8)

    def bits_value(b):
        return Fraction(float(O.bf16_to_f64(np.array([b], np.uint16))[0]))

    # (x1 bits, x2 bits, cos, sin as float32), d_r = 2: out = [x1 c - x2 s, x2 c + x1 s]
    cases = [
        (0x3F31, 0x3F91, np.float32(0.8069711), np.float32(0.59059095), 0, 0xBDE4),   # a: -0.111328125
        (0xBF73, 0x3F74, np.float32(0.70473045), np.float32(0.70947516), 1, 0xBAE6),  # b: -0.0017547607421875
    ]
    for x1b, x2b, c, sn, which, want_bits in cases:
        x1, x2 = bits_value(x1b), bits_value(x2b)
        cf, sf = Fraction(float(c)), Fraction(float(sn))
        if which == 0:
            sep = bf16(f32(f32(x1 * cf) - f32(x2 * sf)))
            fused = bf16(f32(x1 * cf - f32(x2 * sf)))
            once = bf16(x1 * cf - x2 * sf)
        else:
            sep = bf16(f32(f32(x2 * cf) + f32(x1 * sf)))
            fused = bf16(f32(x2 * cf + f32(x1 * sf)))
            once = bf16(x2 * cf + x1 * sf)
        assert sep != fused and sep != once          # the case tells the schemes apart
        assert sep == bits_value(want_bits)          # the expected bits, written out
        table = np.array([[c, sn]], np.float32)      # one position, cos | sin
        got = O.rope_emulate_bf16(np.array([[x1b, x2b]], np.uint16), np.array([0]), table)
        assert int(got[0, which]) == want_bits, (hex(int(got[0, which])), hex(want_bits))


# --------------------------------------------------------------------------
# YaRN on the decoupled RoPE ("Техотчёт DeepSeek-V2 (2024)", long context;
# "DeepSeek-V2 review", 4): s = 40, alpha = 1, beta = 32, 4K -> 160K
# --------------------------------------------------------------------------

def test_yarn_with_no_stretch_is_plain_rope():
    for d_r in (16, 64):
        np.testing.assert_allclose(O.yarn_inv_freq(d_r, s=1.0), O.rope_inv_freq(d_r), rtol=1e-15, atol=0)
    assert O.yarn_score_scale(128, 64, s=1.0) == O.default_scale(128, 64)


def test_yarn_regimes_at_the_v2_shape():
    # Derived by hand for d_r = 64, base 10000, a 4096-token training length:
    # pair m turns 4096 * 10000^(-m/32) / (2 pi) times.  More than 32 turns
    # (kept) for m <= 10; fewer than 1 turn (interpolated by s) for m >= 23;
    # the 12 pairs m = 11 .. 22 lie on the ramp.
    ratio = O.yarn_inv_freq(64) / O.rope_inv_freq(64)
    kept = np.isclose(ratio, 1.0, rtol=1e-12)
    interp = np.isclose(ratio, 1.0 / 40.0, rtol=1e-12)
    assert list(np.flatnonzero(kept)) == list(range(11))
    assert list(np.flatnonzero(interp)) == list(range(23, 32))
    ramp = ratio[11:23]
    assert np.all((ramp > 1.0 / 40.0) & (ramp < 1.0))
    assert np.all(np.diff(ratio) <= 1e-15)          # slower pairs are stretched more


def test_yarn_interpolated_pairs_reach_old_angles_at_stretched_positions():
    # a pair that turns less than once over the training length makes, over
    # s times that length, the turn it used to make: its angle at s p equals
    # the plain angle at p; a fast pair keeps its angle at every position
    x = _rng(21).standard_normal((5, 64))
    p = np.array([0, 7, 100, 1000, 4095], np.float64)
    yarn = O.yarn_inv_freq(64)
    slow = np.r_[23:32]
    fast = np.r_[0:11]
    got = O.rope_rotate(x, 40.0 * p, inv_freq=yarn)
    want = O.rope_rotate(x, p)
    np.testing.assert_allclose(got[:, slow], want[:, slow], atol=1e-9)
    np.testing.assert_allclose(got[:, 32 + slow], want[:, 32 + slow], atol=1e-9)
    got_fast = O.rope_rotate(x, p, inv_freq=yarn)
    np.testing.assert_allclose(got_fast[:, fast], want[:, fast], atol=1e-12)


def test_yarn_keeps_the_relative_position_property():
    r = _rng(22)
    q, k = r.standard_normal(64), r.standard_normal(64)
    f = O.yarn_inv_freq(64)
    a = O.rope_rotate(q, 130000, inv_freq=f) @ O.rope_rotate(k, 129000, inv_freq=f)
    b = O.rope_rotate(q, 1000, inv_freq=f) @ O.rope_rotate(k, 0, inv_freq=f)
    assert abs(a - b) < 1e-8


def test_yarn_temperature_and_target_length():
    # the page's numbers: s = 40 stretches the 4K training length to 160K
    assert 40 * 4096 == 160 * 1024
    # sqrt(t) = 0.0707 ln s + 1 (DeepSeek-V2's coefficient; 0.1 in the generic
    # rule): ln 40 = 3.6888795, so sqrt(t) = 1.2608038 and t = 1.5896262;
    # every score is multiplied by t
    assert abs(O.yarn_sqrt_temperature(40.0) - 1.2608038) < 1e-6
    assert abs(O.yarn_sqrt_temperature(40.0, 0.1) - 1.3688879) < 1e-6
    assert abs(O.yarn_score_scale(128, 64) * math.sqrt(192) - 1.5896262) < 1e-6


# --------------------------------------------------------------------------
# Hand-computed tiny case: n_h = 1, d_c = 2, d_h = 1, d_r = 2, L = 2, T_q = 1
# --------------------------------------------------------------------------

def test_hand_computed_tiny_case():
    # W^UK picks latent component 0, W^UV picks component 1:
    #   k^C_j = c_j[0], v^C_j = c_j[1].
    w_uk = np.array([[[1.0, 0.0]]])
    w_uv = np.array([[[0.0, 1.0]]])
    c = np.array([[1.0, 2.0], [3.0, -1.0]])
    # k^R pre-RoPE: token 0 at position 0 stays [1, 0]; token 1 at position 1
    # becomes [cos 1, sin 1] (d_r = 2, inv_freq = [1]).
    k_r = np.array([[1.0, 0.0], [1.0, 0.0]])
    # The single query is token 1, position L - T_q = 1: q^R = [0, 1] becomes
    # [0*cos1 - 1*sin1, 1*cos1 + 0*sin1] = [-sin 1, cos 1].
    q_c = np.array([[[2.0]]])
    q_r = np.array([[[0.0, 1.0]]])
    # Scores before scaling:
    #   s0 = q^C k^C_0 + q^R.k^R_0 = 2*1 + (-sin1*1 + cos1*0) = 2 - sin 1
    #   s1 = 2*3 + (-sin1*cos1 + cos1*sin1) = 6
    # Scale 1/sqrt(d_h + d_r) = 1/sqrt(3).
    s0 = (2.0 - math.sin(1.0)) / math.sqrt(3.0)
    s1 = 6.0 / math.sqrt(3.0)
    e0, e1 = math.exp(s0), math.exp(s1)
    p0, p1 = e0 / (e0 + e1), e1 / (e0 + e1)
    o_want = p0 * 2.0 + p1 * (-1.0)               # sum p_j v^C_j
    lat_want = [p0 * 1 + p1 * 3, p0 * 2 + p1 * -1]  # sum p_j c_j
    lse_want = math.log(e0 + e1)
    got = O.mla_decode_reference(c, k_r, q_c, q_r, w_uk, w_uv, want_p=True)
    assert abs(got["o"][0, 0, 0] - o_want) < 1e-14
    assert np.allclose(got["latent"][0, 0], lat_want, rtol=0, atol=1e-14)
    assert abs(got["lse"][0, 0] - lse_want) < 1e-14
    assert np.allclose(got["p"][0, 0], [p0, p1], rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# Absorption identities ("Key에 대한 수식 전개", "Value에 대한 수식 전개";
# "Техотчёт ...", exercise 2 of "Что сделать руками")
# --------------------------------------------------------------------------

def _random_problem(r, L=37, T_q=1, n_h=3, d_c=16, d_h=8, d_r=8):
    return dict(
        c=r.standard_normal((L, d_c)),
        k_r=r.standard_normal((L, d_r)),
        q_c=r.standard_normal((T_q, n_h, d_h)),
        q_r=r.standard_normal((T_q, n_h, d_r)),
        w_uk=r.standard_normal((n_h, d_h, d_c)) / 4,
        w_uv=r.standard_normal((n_h, d_h, d_c)) / 4,
    )


def test_absorbed_form_equals_explicit_oracle():
    # Absorbed evaluation, written here from the identities:
    #   q^T (W^UK c) = (W^UK^T q)^T c   and   W^UV sum_j p_j c_j = sum_j p_j W^UV c_j
    r = _rng(7)
    for T_q in (1, 3):
        P = _random_problem(r, T_q=T_q)
        L, n_h = P["c"].shape[0], P["q_c"].shape[1]
        d_h, d_r = P["q_c"].shape[2], P["k_r"].shape[1]
        ref = O.mla_decode_reference(P["c"], P["k_r"], P["q_c"], P["q_r"], P["w_uk"], P["w_uv"])
        kr = O.rope_rotate(P["k_r"], np.arange(L))
        for t in range(T_q):
            qr = O.rope_rotate(P["q_r"][t], L - T_q + t)
            for i in range(n_h):
                q_abs = P["w_uk"][i].T @ P["q_c"][t, i]            # (d_c,)
                s = (P["c"] @ q_abs + kr @ qr[i]) / math.sqrt(d_h + d_r)
                s = s[: L - T_q + t + 1]
                p = np.exp(s - s.max())
                p /= p.sum()
                lat = p @ P["c"][: L - T_q + t + 1]
                assert np.allclose(ref["latent"][t, i], lat, rtol=1e-12, atol=1e-13)
                assert np.allclose(ref["o"][t, i], P["w_uv"][i] @ lat, rtol=1e-12, atol=1e-13)


def test_absorb_q_and_up_v_definitions_match_identities():
    r = _rng(8)
    q_c = r.standard_normal((5, 4, 8))
    w = r.standard_normal((4, 8, 16))
    c = r.standard_normal(16)
    qa = O.absorb_q(q_c, w)
    for n in range(5):
        for i in range(4):
            assert abs(qa[n, i] @ c - q_c[n, i] @ (w[i] @ c)) < 1e-12
    lat = r.standard_normal((5, 4, 16))
    o = O.up_v(lat, w)
    # W^UV applied to a weighted sum equals the weighted sum of W^UV applied
    a = r.random(3)
    cs = r.standard_normal((3, 16))
    lat2 = np.broadcast_to(a @ cs, (1, 4, 16))
    o2 = O.up_v(lat2, w)
    for i in range(4):
        assert np.allclose(o2[0, i], sum(a[j] * (w[i] @ cs[j]) for j in range(3)), atol=1e-12)
    assert o.shape == (5, 4, 8)


def test_rope_on_compressed_keys_breaks_absorption():
    # Exercise 3 of "Что сделать руками" / "Decoupled Rotary Position
    # Embedding" step 1: rotating k^C = W^UK c by a position-dependent R puts
    # R between the query and W^UK, so one position-free absorbed query can no
    # longer reproduce the scores.  With decoupled RoPE it can.
    r = _rng(9)
    d_c, d_h, L = 16, 8, 12
    w = r.standard_normal((d_h, d_c))
    c = r.standard_normal((L, d_c))
    q = r.standard_normal(d_h)
    p_q = L - 1
    q_abs = w.T @ q
    absorbed = c @ q_abs
    rotated = np.array([O.rope_rotate(q, p_q) @ O.rope_rotate(w @ c[j], j) for j in range(L)])
    assert np.max(np.abs(rotated - absorbed)) > 1e-2
    plain = np.array([q @ (w @ c[j]) for j in range(L)])
    assert np.max(np.abs(plain - absorbed)) < 1e-12


# --------------------------------------------------------------------------
# Softmax invariants and degenerate cases
# --------------------------------------------------------------------------

def test_probability_rows_sum_to_one_and_mask_is_causal():
    r = _rng(10)
    P = _random_problem(r, L=50, T_q=4)
    got = O.mla_decode_reference(P["c"], P["k_r"], P["q_c"], P["q_r"], P["w_uk"], P["w_uv"],
                                 want_p=True)
    p = got["p"]
    assert np.allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    for t in range(4):
        vis = 50 - 4 + t + 1
        assert np.all(p[t, :, vis:] == 0.0)
        assert np.all(p[t, :, :vis] > 0.0)


def test_one_token_context_returns_v_exactly():
    r = _rng(11)
    P = _random_problem(r, L=1, T_q=1)
    got = O.mla_decode_reference(P["c"], P["k_r"], P["q_c"], P["q_r"], P["w_uk"], P["w_uv"])
    for i in range(P["q_c"].shape[1]):
        assert np.array_equal(got["latent"][0, i], P["c"][0])
        assert np.allclose(got["o"][0, i], P["w_uv"][i] @ P["c"][0], rtol=0, atol=1e-15)


def test_equal_keys_give_uniform_weights():
    r = _rng(12)
    L = 9
    P = _random_problem(r, L=L, T_q=1, d_r=8)
    P["c"][:] = P["c"][0]
    P["k_r"][:] = 0.0        # RoPE of a zero vector is zero at every position
    got = O.mla_decode_reference(P["c"], P["k_r"], P["q_c"], P["q_r"], P["w_uk"], P["w_uv"],
                                 want_p=True)
    assert np.allclose(got["p"], 1.0 / L, rtol=0, atol=1e-15)
    # lse = log(L) + the common score
    n_h = P["q_c"].shape[1]
    for i in range(n_h):
        s = (P["q_c"][0, i] @ (P["w_uk"][i] @ P["c"][0])) / math.sqrt(8 + 8)
        assert abs(got["lse"][0, i] - (s + math.log(L))) < 1e-12


def test_multi_token_decode_equals_single_token_steps():
    # "학습 시와 디코딩 시의 흐름": one generalised causal mask serves prefill and
    # decode; row t of a T_q = 4 step equals a T_q = 1 step at length L-3+t.
    r = _rng(13)
    L = 70
    P = _random_problem(r, L=L, T_q=4)
    multi = O.mla_decode_reference(P["c"], P["k_r"], P["q_c"], P["q_r"], P["w_uk"], P["w_uv"])
    for t in range(4):
        Lt = L - 3 + t
        single = O.mla_decode_reference(P["c"][:Lt], P["k_r"][:Lt], P["q_c"][t:t + 1],
                                        P["q_r"][t:t + 1], P["w_uk"], P["w_uv"])
        assert np.allclose(multi["o"][t], single["o"][0], rtol=1e-12, atol=1e-13)
        assert np.allclose(multi["lse"][t], single["lse"][0], rtol=1e-12, atol=1e-13)


def test_split_merge_equals_unsplit():
    r = _rng(14)
    L = 64
    P = _random_problem(r, L=L, T_q=1)
    full = O.mla_decode_reference(P["c"], P["k_r"], P["q_c"], P["q_r"], P["w_uk"], P["w_uv"])
    kr = O.rope_rotate(P["k_r"], np.arange(L))
    qr = O.rope_rotate(P["q_r"], np.array([[L - 1]]))
    for cuts in ([0, 64], [0, 20, 64], [0, 1, 2, 30, 63, 64], [0, 10, 19, 28, 37, 46, 55, 64]):
        parts_o, parts_l = [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            # a T_q = 1 query sees all of a key range: attention over the range
            g = O.mla_attention_explicit(P["c"][a:b], kr[a:b], P["q_c"], qr, P["w_uk"],
                                         P["w_uv"],
                                         scale=1 / math.sqrt(8 + 8))
            parts_o.append(g["latent"])
            parts_l.append(g["lse"])
        lat, lse = O.merge_partials(np.stack(parts_o), np.stack(parts_l))
        assert np.allclose(lat, full["latent"], rtol=1e-12, atol=1e-13)
        assert np.allclose(lse, full["lse"], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Paged cache index arithmetic: brute force on a tiny permuted pool
# --------------------------------------------------------------------------

def test_gather_through_permuted_block_table():
    bs, nb, B = 4, 10, 2
    perm = np.array([7, 2, 9, 0, 5, 1, 8, 3, 6, 4])
    table = perm.reshape(B, nb // B)
    pool = np.full((nb, bs, 3), -1, dtype=np.int64)
    for b in range(B):
        for p in range(17):
            blk, slot = O.cache_slot(table, b, p, bs)
            pool[blk, slot] = [b, p, 0]
    for b in range(B):
        rows = O.gather_rows(pool, table, b, 17, bs)
        assert np.array_equal(rows[:, 0], np.full(17, b))
        assert np.array_equal(rows[:, 1], np.arange(17))
    # worked by hand: sequence 0 owns blocks 7 2 9 0 5, sequence 1 owns 1 8 3 6 4;
    # token p sits in the table's block p // 4 at slot p % 4
    assert O.cache_slot(table, 0, 0, bs) == (7, 0)
    assert O.cache_slot(table, 0, 16, bs) == (5, 0)
    assert O.cache_slot(table, 1, 5, bs) == (8, 1)
    assert O.cache_slot(table, 1, 15, bs) == (6, 3)
    # a pool written without the oracle's index helper gathers back in order
    pool2 = np.full((nb, bs, 2), -1, dtype=np.int64)
    for b in range(B):
        for p in range(17):
            pool2[table[b][p // bs], p % bs] = [b, p]
    for b in range(B):
        rows = O.gather_rows(pool2, table, b, 17, bs)
        assert np.array_equal(rows[:, 1], np.arange(17)) and (rows[:, 0] == b).all()


# --------------------------------------------------------------------------
# Cache-size closed forms printed on the pages
# --------------------------------------------------------------------------

def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                vals[k] = float(v)
    return vals


def test_cache_sizes_printed_on_pages():
    g = _golden("cache_sizes.txt")
    f = O.cache_numbers_per_token
    v2 = dict(n_h=128, d_h=128, layers=60)
    assert f("MHA", **v2) == g["v2_mha_numbers"]
    assert f("MQA", **v2) == g["v2_mqa_numbers"]
    mla = f("MLA", d_c=512, d_r=64, layers=60)
    assert mla == g["v2_mla_numbers"]
    assert mla / f("MQA", d_h=128, layers=60) == g["v2_mla_equiv_gqa_groups"]
    gqa67 = f("GQA", n_g=8, d_h=128, layers=95)
    assert gqa67 == g["ds67b_gqa8_numbers"]
    assert gqa67 * 2 / 1024 == g["ds67b_gqa8_kib_bf16"]
    assert mla * 6 / 8 == g["v2_mla_bytes_6bit"]
    assert round(100 * (1 - (mla * 6 / 8) / (gqa67 * 2)), 1) == g["v2_reduction_percent"]
    # d_c = 4 d_h and d_h^R = d_h / 2 ("DeepSeek-V2 review", 2.4)
    assert f("MLA", d_c=4 * 128, d_r=128 // 2, layers=1) == 4.5 * 128
    code_mha = f("MHA", n_h=96, d_h=8, layers=1)
    code_mla = f("MLA", d_c=64, d_r=16, layers=1)
    assert code_mha == g["code_mha_numbers"] and code_mla == g["code_mla_numbers"]
    assert round(code_mha / code_mla) == g["code_ratio_approx"]


# ---------------------------------------------------------------------------
# Folded projections ("MLA 논문정리", "Key에 대한 수식 전개": W'^Q = (W^Q)^T W^UK;
# "Value에 대한 수식 전개": W'^O = W^O W^UV).  Each definition is pinned by a
# brute-force sum over its indices, written out here with plain loops, and the
# folded forms by the identity with the two-step products they replace.
# ---------------------------------------------------------------------------

def _fold_case(seed=7, n_h=2, d_h=3, d_c=4, d_cq=5, d_model=6, n_tok=2):
    r = np.random.default_rng(seed)
    return dict(w_uq=r.standard_normal((n_h, d_h, d_cq)), w_uk=r.standard_normal((n_h, d_h, d_c)),
                w_uv=r.standard_normal((n_h, d_h, d_c)), w_o=r.standard_normal((d_model, n_h, d_h)),
                c_q=r.standard_normal((n_tok, d_cq)), lat=r.standard_normal((n_tok, n_h, d_c)),
                o=r.standard_normal((n_tok, n_h, d_h)))


def test_query_up_projection_and_output_projection_by_brute_force():
    z = _fold_case()
    n_h, d_h, d_cq = z["w_uq"].shape
    d_model = z["w_o"].shape[0]
    q = O.q_up(z["c_q"], z["w_uq"])
    u = O.o_proj(z["o"], z["w_o"])
    for n in range(z["c_q"].shape[0]):
        for i in range(n_h):
            for k in range(d_h):
                want = sum(z["w_uq"][i, k, d] * z["c_q"][n, d] for d in range(d_cq))
                assert abs(q[n, i, k] - want) < 1e-12
        for m in range(d_model):
            want = sum(z["w_o"][m, i, k] * z["o"][n, i, k] for i in range(n_h) for k in range(d_h))
            assert abs(u[n, m] - want) < 1e-12


def test_folded_weights_by_brute_force():
    z = _fold_case()
    n_h, d_h, d_cq = z["w_uq"].shape
    d_c = z["w_uk"].shape[2]
    d_model = z["w_o"].shape[0]
    f = O.fold_q(z["w_uq"], z["w_uk"])
    g = O.fold_o(z["w_o"], z["w_uv"])
    assert f.shape == (n_h, d_c, d_cq) and g.shape == (d_model, n_h, d_c)
    for i in range(n_h):
        for c in range(d_c):
            for d in range(d_cq):
                want = sum(z["w_uk"][i, k, c] * z["w_uq"][i, k, d] for k in range(d_h))
                assert abs(f[i, c, d] - want) < 1e-12
            for m in range(d_model):
                want = sum(z["w_o"][m, i, k] * z["w_uv"][i, k, c] for k in range(d_h))
                assert abs(g[m, i, c] - want) < 1e-12


def test_folded_projections_equal_the_two_step_products():
    z = _fold_case(seed=11, n_h=4, d_h=8, d_c=16, d_cq=24, d_model=20, n_tok=5)
    f = O.fold_q(z["w_uq"], z["w_uk"])
    g = O.fold_o(z["w_o"], z["w_uv"])
    two_step_q = O.absorb_q(O.q_up(z["c_q"], z["w_uq"]), z["w_uk"])
    two_step_u = O.o_proj(O.up_v(z["lat"], z["w_uv"]), z["w_o"])
    np.testing.assert_allclose(O.folded_q(z["c_q"], f), two_step_q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.folded_o(z["lat"], g), two_step_u, rtol=1e-12, atol=1e-12)
