"""The low-bit latent cache through the C ABI against the oracle.

The pages quote a cache of about 6 bits per element ("DeepSeek-V2 review", 4.2
"Inference efficiency"; "Техотчёт DeepSeek-V2 (2024)", "Откуда берутся 93,3%")
without a format; the library stores e4m3 latent codes with one float32 scale
per 64 columns and the rotated RoPE key in bf16 (``oracle.lowbit_cache``).
Bars: the appended rows byte for byte (codes, scales, key, padding) through the
block table; the decode over the e4m3 pool against the oracle's attention over
the dequantised cache, with the bf16 path's tolerances (the quantisation is the
same on both sides, so only float32 arithmetic separates them).
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec, config_specs
from oracle import lowbit_cache as LB
from oracle import mla_oracle as O
from oracle.evaluate import reference

from tests.test_gpu_parity import LSE_ABS, V2, _f64, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def _dc(spec, **kw):
    from mla_latent_kv_38_b200.runner import DeviceCase
    return DeviceCase(spec, cache="e4m3", **kw)


def check_e4m3(dc, seqs, heads=None):
    s = dc.spec
    out = _f64(dc.out).reshape(s.B, s.T_q, s.n_h, s.d_h)
    lat = _f64(dc.latent).reshape(s.B, s.T_q, s.n_h, s.d_c)
    lse = dc.lse.cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h)
    hs = list(range(s.n_h)) if heads is None else list(heads)
    for b in seqs:
        ref = reference(s, b, heads=hs, cache="e4m3")
        assert_close(out[b][:, hs], ref["o"], f"o seq {b}")
        assert_close(lat[b][:, hs], ref["latent"], f"latent seq {b}")
        d = np.abs(lse[b][:, hs] - ref["lse"]).max()
        assert d <= LSE_ABS, f"lse seq {b}: {d:.3e}"


CASES = {
    "tiny_config": config_specs()["tiny"],
    "v2_ragged": CaseSpec(**V2, seq_lens=np.array([1, 63, 64, 65, 300], np.int32), seed=21),
    "v2_permuted": CaseSpec(**V2, seq_lens=np.array([700, 129, 2], np.int32), seed=22, permute_blocks=True),
    "v2_multi_token": CaseSpec(**V2, seq_lens=np.array([4, 5, 67, 200], np.int32), T_q=4, seed=23),
    "small_heads": CaseSpec(n_h=12, d_c=128, d_h=64, d_r=32, seq_lens=np.array([33, 97], np.int32), seed=24),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_e4m3_append_bit_exact(M, name):
    spec = CASES[name]
    dc = _dc(spec)
    dc.step()
    torch.cuda.synchronize()
    assert dc.append_status() == 0
    pool = dc.pool.cpu().numpy()
    tab = O.rope_table_f32(dc.max_pos, spec.d_r)
    for b, L in enumerate(spec.seq_lens):
        L = int(L)
        rows = O.gather_rows(pool, dc.block_table_np, b, L, spec.block_size)
        codes, scale = LB.quantize_latent(spec.c_kv_rows(b, 0, L))
        kr = O.rope_emulate_bf16(spec.k_r_rows(b, 0, L), np.arange(L), tab)
        want = LB.pack_rows(codes, scale, kr)
        assert rows.shape == want.shape
        bad = np.nonzero((rows != want).any(axis=1))[0]
        assert bad.size == 0, f"seq {b}: {bad.size} rows differ, first {bad[:4]}"
    want_q = O.rope_emulate_bf16(spec.q_r(), spec.positions()[:, None], tab)
    assert np.array_equal(dc.bits(dc.q_r), want_q)


@pytest.mark.parametrize("splits", [0, 1, 3])
@pytest.mark.parametrize("name", sorted(CASES))
def test_e4m3_step_matches_the_oracle(M, name, splits):
    spec = CASES[name]
    dc = _dc(spec, max_splits=splits)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    check_e4m3(dc, range(spec.B))


def test_e4m3_full_size_v2_decode(M):
    """DeepSeek-V2 decode at full size (32 sequences of 4,096 keys) over the
    e4m3 pool: all 128 heads of two sequences and six heads of eight more."""
    spec = config_specs()["v2_decode"]
    dc = _dc(spec)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    check_e4m3(dc, [0, 31])
    check_e4m3(dc, [3, 7, 11, 15, 19, 23, 27, 30], heads=[0, 1, 63, 64, 65, 127])


def test_e4m3_bad_block_is_flagged(M):
    spec = CaseSpec(**V2, seq_lens=np.array([130, 64], np.int32), seed=25)
    dc = _dc(spec)
    dc.step()
    bt = dc.block_table.clone()
    bt[0, 1] = spec.num_blocks + 5                         # keys 64 .. 127 of sequence 0
    M.mla_decode_e4m3(dc.cfg, dc.q_abs, dc.q_r, dc.pool, spec.num_blocks, bt, spec.max_blocks, dc.seq_lens,
                      spec.B, spec.T_q, 0, dc.ws, dc.ws_bytes, dc.latent, dc.lse)
    torch.cuda.synchronize()
    assert dc.decode_status() & M.MLA_STATUS_BAD_BLOCK
    assert torch.isfinite(dc.latent.float()).all()


def test_e4m3_pool_is_smaller(M):
    spec = config_specs()["v2_decode"]
    assert M.mla_e4m3_row_bytes(spec.d_c, spec.d_r) * 1.0 / (2 * (spec.d_c + spec.d_r)) == 672 / 1152
