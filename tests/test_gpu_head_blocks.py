"""Parity of the tensor-core decode with more than one block of 128 heads.

The tcgen05 decode takes heads in blocks of 128 (one block per unit of work),
so a layer with 256 heads has two units per query row that read the same
cache pages.  These cases check both head blocks (and both CTAs of each pair:
heads 0-63 and 64-127 of a block) against the oracle, with split units
(merged partials), whole units and T_q = 2.
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec
from oracle.evaluate import reference

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_REL = 5e-3
LSE_ABS = 1e-2

H256 = dict(n_h=256, d_c=512, d_h=128, d_r=64)
HEADS = [0, 1, 63, 64, 127, 128, 129, 191, 192, 255]


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def _close(got, want, what):
    err = np.abs(got - want)
    max_abs = float(err.max())
    mre = float(err.sum() / max(np.abs(want).sum(), 1e-300))
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert max_abs <= MAX_ABS and mre <= MEAN_REL, f"{what}: max_abs={max_abs:.3e} mean_rel={mre:.3e}"


def _run_and_check(M, spec, seqs):
    from mla_latent_kv_38_b200.runner import DeviceCase
    dc = DeviceCase(spec, impl=M.IMPL_TCGEN05)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    s = spec
    out = dc.out.float().cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h, s.d_h)
    lat = dc.latent.float().cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h, s.d_c)
    lse = dc.lse.cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h)
    for b in seqs:
        ref = reference(s, b, heads=HEADS)
        _close(out[b][:, HEADS], ref["o"], f"o seq {b}")
        _close(lat[b][:, HEADS], ref["latent"], f"latent seq {b}")
        d = np.abs(lse[b][:, HEADS] - ref["lse"]).max()
        assert d <= LSE_ABS, f"lse seq {b}: {d:.3e}"


@pytest.mark.parametrize("T_q,lens", [(1, [700, 130, 64, 1]), (2, [300, 65, 2])])
def test_two_head_blocks_split_units(M, T_q, lens):
    # few pages: every cluster gets at most a page or two, so units are split
    # across clusters and merged
    spec = CaseSpec(**H256, seq_lens=np.array(lens, np.int32), T_q=T_q, seed=21, permute_blocks=True)
    _run_and_check(M, spec, range(spec.B))


def test_two_head_blocks_whole_units(M):
    # 128 units of 10 pages over 74 clusters: most units lie inside one
    # cluster's page range and are written without a merge
    spec = CaseSpec(**H256, seq_lens=np.full(64, 600, np.int32), seed=22)
    _run_and_check(M, spec, [0, 1, 31, 62, 63])
