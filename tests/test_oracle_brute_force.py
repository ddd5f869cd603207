"""Brute-force pin of the fp64 oracle on whole workload cases.

Every bf16 input is a dyadic rational, so the bilinear parts of MLA attention
(k^C_j = W^UK_i c_j, v^C_j = W^UV_i c_j, q^C . k^C_j) are computed here in
exact integer arithmetic, with no absorption and no rounding at all.  The
transcendental parts (the RoPE angles base^(-2m/d_r) p, cos and sin, the score
scale 1/sqrt(d_h + d_h^R), exp and log) are taken at 50 significant digits
with mpmath; RoPE is written as a complex rotation of the pair
(x_m, x_{m + d_r/2}), softmax with no max subtraction.  The oracle, run on the
same seeded workload through its per-sequence evaluation, must agree with this
to fp64 accuracy.

Passages: "MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리", eq. (9)-(11),
"Decoupled Rotary Position Embedding" and "MLA 코드 구현" (positions and the
causal mask of the forward pass); DeepSeek-V3 Technical Report notes, eq. (10)
(score scale).
"""

import mpmath as mp
import numpy as np
import pytest

from mla_latent_kv_38_b200.workloads import CaseSpec, config_specs
from oracle import evaluate
from oracle import mla_oracle as O

SHIFT = 160          # every bf16 value used here is an integer multiple of 2^-SHIFT
mp.mp.dps = 50


def _exact_ints(bits):
    """bf16 bit patterns -> Python ints v * 2^SHIFT (exact)."""
    vals = (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)
    out = []
    for v in vals.ravel().tolist():
        num, den = float(v).as_integer_ratio()
        assert (1 << SHIFT) % den == 0
        out.append(num * ((1 << SHIFT) // den))
    return np.array(out, dtype=object).reshape(vals.shape)


def _idot(a, b):
    return sum(x * y for x, y in zip(a, b))


def _rope_mp(x_int, pos, d_r, base=10000):
    """Rotate pair (x_m, x_{m+d_r/2}) by the angle pos * base^(-2m/d_r), as the
    complex number x_m + i x_{m+d_r/2}; returns mp floats (true values)."""
    h = d_r // 2
    out = [None] * d_r
    for m in range(h):
        z = mp.mpc(mp.ldexp(x_int[m], -SHIFT), mp.ldexp(x_int[m + h], -SHIFT))
        theta = mp.mpf(pos) * mp.power(base, mp.mpf(-2 * m) / d_r)
        z = z * mp.expj(theta)
        out[m], out[m + h] = z.real, z.imag
    return out


def _brute_sequence(spec, b):
    """(o, latent, lse) of sequence b for every query and head."""
    L, T_q = int(spec.seq_lens[b]), spec.T_q
    d_h, d_r = spec.d_h, spec.d_r
    c = _exact_ints(spec.c_kv_rows(b, 0, L))                  # (L, d_c)
    k_r = _exact_ints(spec.k_r_rows(b, 0, L))                 # (L, d_r)
    q_c = _exact_ints(spec.q_c()[b * T_q:(b + 1) * T_q])      # (T_q, n_h, d_h)
    q_r = _exact_ints(spec.q_r()[b * T_q:(b + 1) * T_q])
    w_uk, w_uv = _exact_ints(spec.w_uk()), _exact_ints(spec.w_uv())
    scale = 1 / mp.sqrt(d_h + d_r)
    k_rot = [_rope_mp(k_r[j], j, d_r) for j in range(L)]
    o = np.empty((T_q, spec.n_h, d_h))
    lat = np.empty((T_q, spec.n_h, spec.d_c))
    lse = np.empty((T_q, spec.n_h))
    for i in range(spec.n_h):
        # explicit reconstruction, exact: integers scaled by 2^(2 SHIFT)
        k_c = [[_idot(w_uk[i, r], c[j]) for r in range(d_h)] for j in range(L)]
        v_c = [[_idot(w_uv[i, r], c[j]) for r in range(d_h)] for j in range(L)]
        for t in range(T_q):
            pos = L - T_q + t
            q_rot = _rope_mp(q_r[t, i], pos, d_r)
            e = []
            for j in range(pos + 1):                          # keys 0 .. L - T_q + t
                dot_c = mp.ldexp(_idot(q_c[t, i], k_c[j]), -3 * SHIFT)
                dot_r = mp.fsum(a * bb for a, bb in zip(q_rot, k_rot[j]))
                e.append(mp.exp(scale * (dot_c + dot_r)))
            z = mp.fsum(e)
            lse[t, i] = float(mp.log(z))
            for r in range(d_h):
                o[t, i, r] = float(mp.fsum(e[j] * mp.ldexp(v_c[j][r], -2 * SHIFT)
                                           for j in range(len(e))) / z)
            for r in range(spec.d_c):
                lat[t, i, r] = float(mp.fsum(e[j] * mp.ldexp(c[j, r], -SHIFT)
                                             for j in range(len(e))) / z)
    return o, lat, lse


def _check(spec, b):
    want_o, want_lat, want_lse = _brute_sequence(spec, b)
    got = evaluate.reference(spec, b)
    for name, g, w in (("o", got["o"], want_o), ("latent", got["latent"], want_lat),
                       ("lse", got["lse"], want_lse)):
        err = np.abs(g - w).max()
        assert err <= 1e-12 * max(1.0, np.abs(w).max()), (name, err)


def test_tiny_workload_against_exact_arithmetic():
    """The 4-head, d_c = 64, 128-token case, query at position 127."""
    spec = config_specs()["tiny"]
    _check(spec, 0)


@pytest.mark.parametrize("b", [0, 1])
def test_multi_token_batch_against_exact_arithmetic(b):
    """Two sequences, three new tokens each: the causal mask among the new
    tokens and the per-sequence slicing of the query batch."""
    spec = CaseSpec(n_h=2, d_c=16, d_h=8, d_r=8, seq_lens=np.array([5, 23], np.int32), T_q=3, seed=4)
    _check(spec, b)


def test_brute_force_sees_a_planted_mask_slip(monkeypatch):
    """The comparison is sharp: an oracle whose queries saw one key too many
    fails it."""
    spec = CaseSpec(n_h=2, d_c=16, d_h=8, d_r=8, seq_lens=np.array([9], np.int32), T_q=2, seed=5)
    real = O.mla_attention_explicit

    def leaky(c_kv, k_r_rot, q_c, q_r_rot, *a, **kw):
        # query 0 of 2 now also sees the last key
        out0 = real(c_kv, k_r_rot, q_c[:1], q_r_rot[:1], *a, **kw)
        out1 = real(c_kv, k_r_rot, q_c[1:], q_r_rot[1:], *a, **kw)
        return {k: np.concatenate([out0[k], out1[k]]) for k in out0}

    monkeypatch.setattr(O, "mla_attention_explicit", leaky)
    with pytest.raises(AssertionError):
        _check(spec, 0)
