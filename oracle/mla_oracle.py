"""fp64 CPU oracle for MLA decode over a latent KV cache.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module: only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may call it. It shares no code with the CUDA path (only the seeded input
generator module is common to both, and that draws numbers and nothing else).

What it computes is the plain, un-absorbed definition of multi-head latent
attention with decoupled RoPE, evaluated in float64 on the bf16-rounded inputs
the GPU receives:

* RoPE with the half-split ``rotate_half`` convention and ``inv_freq =
  base^(-2m/d_r)`` -- "MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리",
  section "MLA 코드 구현" (``build_rope_cache`` / ``rotate_half`` / ``apply_rope``).
* Explicit up-projection of every cached latent: ``k^C = W^UK c^KV`` and
  ``v^C = W^UV c^KV`` -- same page, "Low-Rank Key-Value Joint Compression",
  eq. (10) and (11); "Техотчёт DeepSeek-V2 (2024): MLA и экономика инференса",
  section "Идея 1".
* One decoupled RoPE key shared by all heads, concatenated to each head's key;
  the query is ``[q^C; q^R]`` -- "Техотчёт DeepSeek-V2 ...", section "Идея 2:
  отделённый RoPE"; "DeepSeek-V2 review", section 2.3 (Decoupled RoPE).
* Scores scaled by ``1/sqrt(d_h + d_h^R)``, causal softmax, weighted sum of the
  reconstructed values -- DeepSeek-V3 report notes, "Multi-Head Attention 및
  Output 계산 (식 10, 11)", eq. (10); "Техотчёт DeepSeek-V2 ...", "Идея 2".
* The generalised causal mask for ``T_q`` new tokens at the end of a ``T_k``
  long cache (``triu(-inf, diagonal = T_k - T_q + 1)``) -- "MLA 논문정리",
  "MLA 코드 구현" (forward) and "학습 시와 디코딩 시의 흐름".

Also here, for tests that need them: the absorbed-query and value up-projection
definitions (eq. 10/11 applied to a query or a latent, "Key에 대한 수식 전개",
"Value에 대한 수식 전개"), the query up-projection and output projection on
either side of the path and their folded weights (W^UK into W^UQ, W^UV into
W^O, same sections), the paged-cache index arithmetic, the log-sum-exp
merge of split partials, an emulation of the GPU's float32 RoPE arithmetic for
the bit-exact append check, and the per-token cache-size formulas of the
"Сколько получилось" table.

Where the pages are silent or disagree, the functions below say which reading
they take (score scale, shared RoPE key, half-split pairing, query positions,
weight standard deviations).
"""

from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# bf16 helpers (oracle-local; the CUDA path has its own conversions)
# ---------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 bits, round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    out = r.astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


# ---------------------------------------------------------------------------
# RoPE ("MLA 논문정리", "MLA 코드 구현": build_rope_cache / rotate_half / apply_rope)
# ---------------------------------------------------------------------------


def rope_inv_freq(d_r: int, base: float = 10000.0) -> np.ndarray:
    """Frequencies base^(-2m/d_r) for pair index m = 0 .. d_r/2 - 1."""
    assert d_r % 2 == 0
    m = np.arange(d_r // 2, dtype=np.float64)
    return base ** (-(2.0 * m) / d_r)


def yarn_inv_freq(d_r: int, base: float = 10000.0, s: float = 40.0, alpha: float = 1.0, beta: float = 32.0,
                  orig_len: int = 4096) -> np.ndarray:
    """YaRN frequencies (NTK-by-parts) of the decoupled RoPE.

    "Техотчёт DeepSeek-V2 (2024)", "Обучение: данные, гиперпараметры,
    инфраструктура" (long context) and "DeepSeek-V2 review", 4 (Long context):
    the context grows from 4K to 128K by YaRN on k^R only; each frequency pair
    is scaled by how many turns it makes over the training length, with
    s = 40, alpha = 1, beta = 32 (target length s x 4K = 160K).  Reading taken
    here (the page states the rule in words): pair m with frequency
    f_m = base^(-2m/d_r) makes r_m = orig_len f_m / (2 pi) turns over the
    training length; gamma_m = clamp((r_m - alpha) / (beta - alpha), 0, 1);
    the new frequency is f_m ((1 - gamma_m) / s + gamma_m): pairs that turn
    fewer than alpha times are interpolated by s, pairs that turn more than
    beta times are kept, the ramp in between is linear in r_m.
    """
    f = rope_inv_freq(d_r, base)
    turns = orig_len * f / (2.0 * math.pi)
    gamma = np.clip((turns - alpha) / (beta - alpha), 0.0, 1.0)
    return f * ((1.0 - gamma) / s + gamma)


def yarn_sqrt_temperature(s: float = 40.0, coeff: float = 0.0707) -> float:
    """sqrt(t) = coeff ln s + 1: the attention temperature of YaRN (0.1 in the
    generic rule; DeepSeek-V2 tuned it to 0.0707, "Техотчёт DeepSeek-V2",
    long context).  Reading taken here: both q and k are multiplied by
    sqrt(t), so every score is multiplied by t."""
    return coeff * math.log(s) + 1.0


def yarn_score_scale(d_h: int, d_r: int, s: float = 40.0, coeff: float = 0.0707) -> float:
    """t / sqrt(d_h + d_h^R): the score scale with the YaRN temperature."""
    return yarn_sqrt_temperature(s, coeff) ** 2 / math.sqrt(d_h + d_r)


def rope_rotate(x: np.ndarray, pos, base: float = 10000.0, inv_freq=None) -> np.ndarray:
    """Apply RoPE to the last axis of ``x`` at positions ``pos`` (fp64).

    Half-split pairing: element m rotates with element m + d_r/2 by angle
    ``pos * inv_freq[m]``:  x'_m = x_m cos - x_{m+h} sin,
    x'_{m+h} = x_{m+h} cos + x_m sin  (``x*cos + rotate_half(x)*sin`` with
    ``rotate_half(x) = [-x2, x1]``).
    ``pos`` broadcasts against ``x.shape[:-1]``.
    """
    x = np.asarray(x, dtype=np.float64)
    d_r = x.shape[-1]
    h = d_r // 2
    f = rope_inv_freq(d_r, base) if inv_freq is None else np.asarray(inv_freq, dtype=np.float64)
    theta = np.asarray(pos, dtype=np.float64)[..., None] * f
    c, s = np.cos(theta), np.sin(theta)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_table_f32(max_pos: int, d_r: int, base: float = 10000.0, inv_freq=None) -> np.ndarray:
    """float32 table (max_pos, d_r): row p = [cos(p*f_0..), sin(p*f_0..)] from fp64."""
    f = rope_inv_freq(d_r, base) if inv_freq is None else np.asarray(inv_freq, dtype=np.float64)
    theta = np.arange(max_pos, dtype=np.float64)[:, None] * f
    return np.concatenate([np.cos(theta), np.sin(theta)], axis=1).astype(np.float32)


def rope_emulate_bf16(x_bits: np.ndarray, pos: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Bit-level model of the GPU's RoPE: float32 products and sums, no fused
    multiply-add, then bf16 round-to-nearest-even.

    x_bits: (..., d_r) bf16 bits; pos: integer array broadcasting to x[..., 0];
    table: float32 (max_pos, d_r) as from :func:`rope_table_f32`.
    """
    x = bf16_to_f64(x_bits).astype(np.float32)
    d_r = x.shape[-1]
    h = d_r // 2
    row = table[np.asarray(pos)]
    c = row[..., :h].astype(np.float32)
    s = row[..., h:].astype(np.float32)
    x1, x2 = x[..., :h], x[..., h:]
    # each product rounded to float32, then the difference / sum rounded
    # (numpy evaluates float32 array arithmetic one rounded operation at a time)
    a = (x1 * c) - (x2 * s)
    b = (x2 * c) + (x1 * s)
    assert a.dtype == np.float32 and b.dtype == np.float32
    return f32_to_bf16_rne(np.concatenate([a, b], axis=-1))


# ---------------------------------------------------------------------------
# Paged cache index arithmetic
# ---------------------------------------------------------------------------


def cache_slot(block_table: np.ndarray, b: int, pos: int, block_size: int):
    """(physical block, slot) holding token ``pos`` of sequence ``b``."""
    return int(block_table[b, pos // block_size]), pos % block_size


def gather_rows(pool: np.ndarray, block_table: np.ndarray, b: int, length: int,
                block_size: int) -> np.ndarray:
    """Rows 0..length-1 of sequence b, read through the block table."""
    out = np.empty((length,) + pool.shape[2:], dtype=pool.dtype)
    for p in range(length):
        blk, slot = cache_slot(block_table, b, p, block_size)
        out[p] = pool[blk, slot]
    return out


# ---------------------------------------------------------------------------
# Absorption-side definitions (eq. 10 / 11 applied per head)
# ---------------------------------------------------------------------------


def absorb_q(q_c: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """q_abs[n, i, :] = W^UK_i^T q^C[n, i, :].

    q_c: (n_tok, n_h, d_h); w_uk: (n_h, d_h, d_c) -> (n_tok, n_h, d_c).
    "MLA 논문정리", "Key에 대한 수식 전개": the key weight moves onto the query.
    """
    q_c = np.asarray(q_c, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    out = np.empty((q_c.shape[0], q_c.shape[1], w_uk.shape[2]))
    for i in range(q_c.shape[1]):
        out[:, i, :] = q_c[:, i, :] @ w_uk[i]
    return out


def up_v(latent: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """o[n, i, :] = W^UV_i latent[n, i, :].

    latent: (n_tok, n_h, d_c); w_uv: (n_h, d_h, d_c) -> (n_tok, n_h, d_h).
    "MLA 논문정리", "Value에 대한 수식 전개": the value weight is applied once to
    the probability-weighted latent.
    """
    latent = np.asarray(latent, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    out = np.empty((latent.shape[0], latent.shape[1], w_uv.shape[1]))
    for i in range(latent.shape[1]):
        out[:, i, :] = latent[:, i, :] @ w_uv[i].T
    return out


# ---------------------------------------------------------------------------
# The projections on either side of the path, and their folded forms
# ("MLA 논문정리", "Key에 대한 수식 전개": W'^Q = (W^Q)^T W^UK, and "Value에
# 대한 수식 전개": W'^O = W^O W^UV; "Техотчёт DeepSeek-V2 (2024)", "Идея 1")
# ---------------------------------------------------------------------------


def q_up(c_q: np.ndarray, w_uq: np.ndarray) -> np.ndarray:
    """q^C[n, i, :] = W^UQ_i c^Q[n]: the query up-projection from the query latent.

    c_q: (n_tok, d_cq); w_uq: (n_h, d_h, d_cq) -> (n_tok, n_h, d_h)."""
    c_q = np.asarray(c_q, dtype=np.float64)
    w_uq = np.asarray(w_uq, dtype=np.float64)
    return np.einsum("hkd,nd->nhk", w_uq, c_q)


def o_proj(o: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """u[n] = W^O [o[n, 0, :]; ...; o[n, n_h - 1, :]] = sum_i W^O_i o[n, i, :].

    o: (n_tok, n_h, d_h); w_o: (d_model, n_h, d_h) -> (n_tok, d_model)."""
    o = np.asarray(o, dtype=np.float64)
    w_o = np.asarray(w_o, dtype=np.float64)
    return np.einsum("mhk,nhk->nm", w_o, o)


def fold_q(w_uq: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """F_i = W^UK_i^T W^UQ_i, so that q_abs[n, i, :] = F_i c^Q[n] in one product.

    w_uq: (n_h, d_h, d_cq); w_uk: (n_h, d_h, d_c) -> (n_h, d_c, d_cq)."""
    w_uq = np.asarray(w_uq, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    return np.einsum("hkc,hkd->hcd", w_uk, w_uq)


def fold_o(w_o: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """G_i = W^O_i W^UV_i, so that u[n] = sum_i G_i latent[n, i, :]: one product
    with K = n_h d_c over the whole latent output.

    w_o: (d_model, n_h, d_h); w_uv: (n_h, d_h, d_c) -> (d_model, n_h, d_c)."""
    w_o = np.asarray(w_o, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    return np.einsum("mhk,hkc->mhc", w_o, w_uv)


def folded_q(c_q: np.ndarray, f: np.ndarray) -> np.ndarray:
    """q_abs[n, i, :] = F_i c^Q[n]; c_q: (n_tok, d_cq), f: (n_h, d_c, d_cq)."""
    return np.einsum("hcd,nd->nhc", np.asarray(f, dtype=np.float64), np.asarray(c_q, dtype=np.float64))


def folded_o(latent: np.ndarray, g: np.ndarray) -> np.ndarray:
    """u[n] = sum_i G_i latent[n, i, :]; latent: (n_tok, n_h, d_c), g: (d_model, n_h, d_c)."""
    return np.einsum("mhc,nhc->nm", np.asarray(g, dtype=np.float64), np.asarray(latent, dtype=np.float64))


# ---------------------------------------------------------------------------
# The attention itself, explicit reconstruction, no absorption
# ---------------------------------------------------------------------------


def default_scale(d_h: int, d_r: int) -> float:
    """1/sqrt(d_h + d_h^R) (DeepSeek-V3 notes eq. 10; "Идея 2")."""
    return 1.0 / math.sqrt(d_h + d_r)


def mla_attention_explicit(c_kv, k_r_rot, q_c, q_r_rot, w_uk, w_uv, scale=None,
                           heads=None, want_p=False):
    """Causal MLA attention of T_q new queries over a cache of T_k rows.

    c_kv: (T_k, d_c) latents; k_r_rot: (T_k, d_r) RoPE'd shared keys;
    q_c: (T_q, n_h, d_h); q_r_rot: (T_q, n_h, d_r) RoPE'd queries;
    w_uk, w_uv: (n_h, d_h, d_c).  The T_q queries are the last T_q cache rows,
    so query t sees keys 0 .. T_k - T_q + t.

    Returns a dict with, for the selected heads (all by default):
      o      (T_q, H, d_h)  sum_j p_tj v^C_j         (the head output)
      latent (T_q, H, d_c)  sum_j p_tj c_j           (what absorbed decode emits)
      lse    (T_q, H)       log sum_j exp(s_tj)
      p      (T_q, H, T_k)  probabilities (if want_p)
    """
    c_kv = np.asarray(c_kv, dtype=np.float64)
    k_r_rot = np.asarray(k_r_rot, dtype=np.float64)
    q_c = np.asarray(q_c, dtype=np.float64)
    q_r_rot = np.asarray(q_r_rot, dtype=np.float64)
    T_k, d_c = c_kv.shape
    T_q, n_h, d_h = q_c.shape
    d_r = k_r_rot.shape[1]
    assert 1 <= T_q <= T_k
    if scale is None:
        scale = default_scale(d_h, d_r)
    heads = list(range(n_h)) if heads is None else list(heads)
    H = len(heads)
    o = np.empty((T_q, H, d_h))
    lat = np.empty((T_q, H, d_c))
    lse = np.empty((T_q, H))
    p_all = np.empty((T_q, H, T_k)) if want_p else None
    # mask[t, j] = True where key j is visible to query t
    j_idx = np.arange(T_k)[None, :]
    t_idx = np.arange(T_q)[:, None]
    visible = j_idx <= (T_k - T_q + t_idx)
    for hi, i in enumerate(heads):
        wk = np.asarray(w_uk[i], dtype=np.float64)      # (d_h, d_c)
        wv = np.asarray(w_uv[i], dtype=np.float64)
        k_c = c_kv @ wk.T                                # (T_k, d_h)   eq. (10)
        v_c = c_kv @ wv.T                                # (T_k, d_h)   eq. (11)
        k = np.concatenate([k_c, k_r_rot], axis=1)       # shared k^R for every head
        q = np.concatenate([q_c[:, i, :], q_r_rot[:, i, :]], axis=1)   # (T_q, d_h+d_r)
        s = (q @ k.T) * scale                            # (T_q, T_k)
        s = np.where(visible, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        p = e / z
        o[:, hi, :] = p @ v_c
        lat[:, hi, :] = p @ c_kv
        lse[:, hi] = (m + np.log(z))[:, 0]
        if want_p:
            p_all[:, hi, :] = p
    out = {"o": o, "latent": lat, "lse": lse}
    if want_p:
        out["p"] = p_all
    return out


def mla_decode_reference(c_kv, k_r, q_c, q_r, w_uk, w_uv, base=10000.0, scale=None, inv_freq=None,
                         heads=None, want_p=False):
    """One decode step of one sequence from raw (pre-RoPE) inputs.

    c_kv: (L, d_c) and k_r: (L, d_r) for every cached token, the last T_q of
    which are the new tokens; q_c: (T_q, n_h, d_h); q_r: (T_q, n_h, d_r)
    pre-RoPE.  Token j sits at position j; query t at position L - T_q + t
    ("MLA 논문정리", forward: new tokens take positions past_len .. T_total-1).
    """
    L = np.asarray(c_kv).shape[0]
    T_q = np.asarray(q_c).shape[0]
    k_r_rot = rope_rotate(k_r, np.arange(L), base, inv_freq)
    qpos = np.arange(L - T_q, L)
    q_r_rot = rope_rotate(q_r, qpos[:, None], base, inv_freq)
    return mla_attention_explicit(c_kv, k_r_rot, q_c, q_r_rot, w_uk, w_uv, scale,
                                  heads=heads, want_p=want_p)


# ---------------------------------------------------------------------------
# Split-KV log-sum-exp merge
# ---------------------------------------------------------------------------


def merge_partials(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Combine S normalised partial results over disjoint key ranges.

    o_parts: (S, ..., d); lse_parts: (S, ...).  With w_s = exp(lse_s - max),
    o = sum_s w_s o_s / sum_s w_s and lse = max + log sum_s w_s.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m)
    z = w.sum(axis=0)
    o = (w[..., None] * o_parts).sum(axis=0) / z[..., None]
    return o, m + np.log(z)


# ---------------------------------------------------------------------------
# Cache-size accounting ("Техотчёт DeepSeek-V2 ...", table "Сколько получилось";
# "DeepSeek-V2 review", section 2.4)
# ---------------------------------------------------------------------------


def cache_numbers_per_token(mechanism: str, *, n_h=0, d_h=0, layers=1, n_g=0,
                            d_c=0, d_r=0) -> int:
    """Cached numbers per token over ``layers`` layers for each mechanism."""
    if mechanism == "MHA":
        return 2 * n_h * d_h * layers
    if mechanism == "GQA":
        return 2 * n_g * d_h * layers
    if mechanism == "MQA":
        return 2 * d_h * layers
    if mechanism == "MLA":
        return (d_c + d_r) * layers
    raise ValueError(mechanism)
