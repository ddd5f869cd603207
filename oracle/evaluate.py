"""Oracle evaluation of one sequence of a workload (test infrastructure only).

Takes a workload spec (head shapes, lengths, seed; inputs drawn by the seeded
generator) and runs :func:`mla_oracle.mla_decode_reference` on the bf16-rounded
inputs of sequence ``b``, widened to float64.
"""

from __future__ import annotations

from . import mla_oracle as O

_CACHE = {}


def _cached(kind, spec):
    key = (kind,) + _key(spec)
    if key not in _CACHE:
        if len(_CACHE) > 16:
            _CACHE.clear()
        if kind == "w":
            _CACHE[key] = (O.bf16_to_f64(spec.w_uk()), O.bf16_to_f64(spec.w_uv()))
        else:
            _CACHE[key] = (O.bf16_to_f64(spec.q_c()), O.bf16_to_f64(spec.q_r()))
    return _CACHE[key]


def _key(spec):
    return (spec.n_h, spec.d_c, spec.d_h, spec.d_r, spec.T_q, spec.seed, spec.B,
            tuple(int(x) for x in spec.seq_lens))


def reference(spec, b: int, heads=None, want_p=False, inv_freq=None, scale=None, cache="bf16"):
    """Oracle outputs for sequence b: dict(o, latent, lse[, p]) over `heads`.

    inv_freq / scale: RoPE frequencies and score scale other than the
    defaults (YaRN: mla_oracle.yarn_inv_freq, mla_oracle.yarn_score_scale).
    cache "e4m3": every cached latent row is read back from its e4m3 codes and
    group scales (``lowbit_cache``); the RoPE key as in the bf16 cache."""
    L = int(spec.seq_lens[b])
    T_q = spec.T_q
    c = O.bf16_to_f64(spec.c_kv_rows(b, 0, L))
    if cache == "e4m3":
        from . import lowbit_cache as LB
        c = LB.dequantize_latent(*LB.quantize_latent(spec.c_kv_rows(b, 0, L)))
    k = O.bf16_to_f64(spec.k_r_rows(b, 0, L))
    w_uk, w_uv = _cached("w", spec)
    q_c, q_r = _cached("q", spec)
    sl = slice(b * T_q, (b + 1) * T_q)
    return O.mla_decode_reference(c, k, q_c[sl], q_r[sl], w_uk, w_uv, scale=scale, inv_freq=inv_freq, heads=heads,
                                  want_p=want_p)

