"""YaRN-scaled decoupled RoPE on the CUDA path, against the fp64 oracle.

DeepSeek-V2 extends its context from 4K to 128K by YaRN on the decoupled key
only ("Техотчёт DeepSeek-V2 (2024)", long context; "DeepSeek-V2 review", 4):
the cos/sin table (NTK-by-parts frequencies, s = 40, alpha = 1, beta = 32)
and the score scale (temperature t = (0.0707 ln s + 1)^2) change; the
kernels do not.  The library builds the table and the scale
(mla_rope_table_yarn, mla_yarn_score_scale); the oracle uses its own
definitions (mla_oracle.yarn_inv_freq, yarn_score_scale).
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec, config_specs
from oracle import mla_oracle as O
from oracle.evaluate import reference

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_REL = 5e-3
LSE_ABS = 1e-2
YARN = dict(s=40.0, alpha=1.0, beta=32.0, orig_len=4096, coeff=0.0707)
V2 = dict(n_h=128, d_c=512, d_h=128, d_r=64)


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def _check(dc, seqs, heads=None):
    s = dc.spec
    f = O.yarn_inv_freq(s.d_r)
    scale = O.yarn_score_scale(s.d_h, s.d_r)
    out = dc.out.float().cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h, s.d_h)
    lat = dc.latent.float().cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h, s.d_c)
    lse = dc.lse.cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h)
    hs = list(range(s.n_h)) if heads is None else list(heads)
    for b in seqs:
        ref = reference(s, b, heads=hs, inv_freq=f, scale=scale)
        for got, want, what in ((out[b][:, hs], ref["o"], "o"), (lat[b][:, hs], ref["latent"], "latent")):
            err = np.abs(got - want)
            assert np.isfinite(got).all(), what
            assert err.max() <= MAX_ABS and err.sum() / np.abs(want).sum() <= MEAN_REL, \
                (what, b, err.max(), err.sum() / np.abs(want).sum())
        assert np.abs(lse[b][:, hs] - ref["lse"]).max() <= LSE_ABS, b


@pytest.mark.parametrize("impl", [0, 1])
@pytest.mark.parametrize("T_q,lens", [(1, [5000, 300, 65]), (2, [4100, 129])])
def test_yarn_full_path_past_the_training_length(M, impl, T_q, lens):
    from mla_latent_kv_38_b200.runner import DeviceCase
    spec = CaseSpec(**V2, seq_lens=np.array(lens, np.int32), T_q=T_q, seed=41)
    dc = DeviceCase(spec, impl=impl, yarn=YARN)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    _check(dc, range(spec.B))
    # the appended rows' RoPE part against the oracle's model of the kernel
    # arithmetic on the oracle's own YaRN table (the same floats here)
    tab = O.rope_table_f32(dc.max_pos, spec.d_r, inv_freq=O.yarn_inv_freq(spec.d_r))
    assert np.array_equal(tab, dc.rope_table.cpu().numpy())
    pool = dc.bits(dc.pool)
    for b, L in enumerate(spec.seq_lens):
        L = int(L)
        rows = O.gather_rows(pool, dc.block_table_np, b, L, spec.block_size)
        assert np.array_equal(rows[:, :spec.d_c], spec.c_kv_rows(b, 0, L))
        assert np.array_equal(rows[:, spec.d_c:], O.rope_emulate_bf16(spec.k_r_rows(b, 0, L), np.arange(L), tab))


def test_yarn_long_context_full_size(M):
    """The long workload (B=4, context 131072, 32x the training length) with
    YaRN, in the benchmark's launch configuration, sampled heads."""
    from mla_latent_kv_38_b200.runner import DeviceCase
    spec = config_specs()["long"]
    dc = DeviceCase(spec, yarn=YARN)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    _check(dc, [0, 3], [0, 63, 64, 127])
