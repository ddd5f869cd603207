"""Folded projections through the C ABI against the fp64 oracle.

"MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리", "Key에 대한 수식 전개"
(W^UK folds into the query projection) and "Value에 대한 수식 전개" (W^UV folds
into the output projection).  The GPU folds the weights once (fp32 sums, bf16
results), then q_abs comes from the query latent in one product and the model
output from the decode's latent in one product with K = n_h d_c.  The oracle
computes the unfolded two-step products in fp64 (q^C = W^UQ c^Q, q_abs =
W^UK^T q^C; o = W^UV latent, u = W^O o).
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec
from oracle import mla_oracle as O
from oracle.evaluate import reference

from tests.test_gpu_parity import V2, _dc, _f64, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def _folded(M, spec):
    cfg = M.MlaConfig(spec.n_h, spec.d_c, spec.d_h, spec.d_r, 64, 0.0, 0)
    w = {k: getattr(spec, k)() for k in ("w_uq", "w_uk", "w_uv", "w_o")}
    f = torch.empty((spec.n_h, spec.d_c, spec.d_cq), dtype=torch.bfloat16, device="cuda")
    g = torch.empty((spec.d_model, spec.n_h, spec.d_c), dtype=torch.bfloat16, device="cuda")
    M.mla_fold_weights(cfg, spec.d_cq, spec.d_model, _dev(w["w_uq"]), _dev(w["w_uk"]), _dev(w["w_uv"]),
                       _dev(w["w_o"]), f, g)
    torch.cuda.synchronize()
    return cfg, {k: O.bf16_to_f64(v) for k, v in w.items()}, f, g


SHAPES = {
    "small": dict(n_h=4, d_c=256, d_h=64, d_r=64, d_cq=192, d_model=384),
    "v2": dict(n_h=128, d_c=512, d_h=128, d_r=64, d_cq=1536, d_model=5120),
}


@pytest.mark.parametrize("shape", sorted(SHAPES))
def test_folded_weights_match_the_oracle(M, shape):
    z = SHAPES[shape]
    spec = CaseSpec(n_h=z["n_h"], d_c=z["d_c"], d_h=z["d_h"], d_r=z["d_r"], seq_lens=np.array([64], np.int32),
                    d_cq=z["d_cq"], d_model=z["d_model"], seed=41)
    cfg, w, f, g = _folded(M, spec)
    heads = [0, spec.n_h - 1]
    want_f = O.fold_q(w["w_uq"][heads], w["w_uk"][heads])
    got_f = _f64(f)[heads]
    rows = [0, 1, spec.d_model // 2, spec.d_model - 1]
    want_g = O.fold_o(w["w_o"][rows], w["w_uv"])
    got_g = _f64(g)[rows]
    for got, want, what in ((got_f, want_f, "F"), (got_g, want_g, "G")):
        # fp32 sums of d_h products, one bf16 rounding: within 2^-8 of each element's size
        err = np.abs(got - want)
        assert (err <= 2.0 ** -8 * np.abs(want) + 1e-6).all(), (what, float(err.max()))


@pytest.mark.parametrize("n_tok", [1, 15, 32, 300])
@pytest.mark.parametrize("shape", sorted(SHAPES))
def test_folded_query_side_matches_the_two_step_oracle(M, shape, n_tok):
    z = SHAPES[shape]
    if shape == "v2" and n_tok == 300:
        pytest.skip("covered by the small shape; the oracle's W^UQ product is large")
    spec = CaseSpec(n_h=z["n_h"], d_c=z["d_c"], d_h=z["d_h"], d_r=z["d_r"],
                    seq_lens=np.full(n_tok, 64, np.int32), d_cq=z["d_cq"], d_model=z["d_model"], seed=42)
    cfg, w, f, g = _folded(M, spec)
    c_q = spec.c_q()
    q_abs = torch.empty((n_tok, spec.n_h, spec.d_c), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.mla_absorb_q_folded(cfg, spec.d_cq, _dev(c_q), f, q_abs, n_tok, status)
    torch.cuda.synchronize()
    assert M.mla_read_status(status) == 0
    want = O.absorb_q(O.q_up(O.bf16_to_f64(c_q), w["w_uq"]), w["w_uk"])
    assert_close(_f64(q_abs), want, f"folded q_abs {shape} n_tok={n_tok}")


@pytest.mark.parametrize("n_tok", [1, 32, 300])
@pytest.mark.parametrize("shape", sorted(SHAPES))
def test_folded_output_side_matches_the_two_step_oracle(M, shape, n_tok):
    z = SHAPES[shape]
    spec = CaseSpec(n_h=z["n_h"], d_c=z["d_c"], d_h=z["d_h"], d_r=z["d_r"],
                    seq_lens=np.full(n_tok, 64, np.int32), d_cq=z["d_cq"], d_model=z["d_model"], seed=43)
    cfg, w, f, g = _folded(M, spec)
    # a latent of the decode output's size: N(0, 1/16) (a softmax average of N(0, 1) rows)
    r = np.random.default_rng(7)
    lat = O.f32_to_bf16_rne((0.25 * r.standard_normal((n_tok, spec.n_h, spec.d_c))).astype(np.float32))
    u = torch.empty((n_tok, spec.d_model), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(M.mla_up_o_folded_workspace_bytes(cfg, spec.d_model, n_tok), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.mla_up_o_folded(cfg, spec.d_model, _dev(lat), g, u, n_tok, ws, status)
    torch.cuda.synchronize()
    assert M.mla_read_status(status) == 0
    want = O.o_proj(O.up_v(O.bf16_to_f64(lat), w["w_uv"]), w["w_o"])
    assert_close(_f64(u), want, f"folded u {shape} n_tok={n_tok}")


def test_folded_step_matches_the_full_oracle(M):
    """c^Q -> q_abs (folded) -> RoPE + append -> decode -> u (folded), against
    the oracle's explicit attention with q^C = W^UQ c^Q and u = W^O o."""
    spec = CaseSpec(**V2, seq_lens=np.array([300, 97], np.int32), T_q=2, seed=44)
    dc = _dc(spec)
    cfg, w, f, g = _folded(M, spec)
    c_q = spec.c_q()
    M.mla_absorb_q_folded(dc.cfg, spec.d_cq, _dev(c_q), f, dc.q_abs, spec.n_tok, dc.status)
    M.mla_rope_append(dc.cfg, dc.q_r, dc.k_r_new, dc.c_kv_new, dc.positions, dc.rope_table, dc.max_pos,
                      dc.block_table, spec.max_blocks, dc.pool, spec.num_blocks, spec.B, spec.T_q, dc.status)
    dc.decode_only()
    u = torch.empty((spec.n_tok, spec.d_model), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(M.mla_up_o_folded_workspace_bytes(dc.cfg, spec.d_model, spec.n_tok), dtype=torch.uint8,
                     device="cuda")
    M.mla_up_o_folded(dc.cfg, spec.d_model, dc.latent, g, u, spec.n_tok, ws, dc.status)
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    q_c = O.q_up(O.bf16_to_f64(c_q), w["w_uq"])            # (n_tok, n_h, d_h), fp64, not rounded
    got = _f64(u).reshape(spec.B, spec.T_q, spec.d_model)
    for b in range(spec.B):
        L = int(spec.seq_lens[b])
        sl = slice(b * spec.T_q, (b + 1) * spec.T_q)
        ref = O.mla_decode_reference(O.bf16_to_f64(spec.c_kv_rows(b, 0, L)), O.bf16_to_f64(spec.k_r_rows(b, 0, L)),
                                     q_c[sl], O.bf16_to_f64(spec.q_r())[sl], w["w_uk"], w["w_uv"])
        want = O.o_proj(ref["o"], w["w_o"])
        assert_close(got[b], want, f"folded step u seq {b}")
