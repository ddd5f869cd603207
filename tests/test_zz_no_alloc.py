"""mla_decode_noalloc: decode for callers that cannot allocate device memory.

Callers such as plugins handed only their input and output buffers, or code
inside a framework that owns every device allocation, cannot supply
mla_decode's workspace.  mla_decode_noalloc keeps the split-KV partials in a
fixed device array of the library instead.  This test calls it through the C
ABI twice in a row and checks each result against mla_decode's within the
parity tolerances used everywhere else; it must pass alone in a fresh process
and after the other tests (the array keeps earlier calls' contents).
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_REL = 5e-3
LSE_ABS = 1e-2


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def _close(got, want, what):
    g = got.float().cpu().numpy().astype(np.float64)
    w = want.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - w)
    assert np.isfinite(g).all(), what
    assert err.max() <= MAX_ABS, (what, err.max())
    assert err.sum() / np.abs(w).sum() <= MEAN_REL, (what, err.sum() / np.abs(w).sum())


def test_noalloc_matches_workspace_decode_twice(M):
    from mla_latent_kv_38_b200.runner import DeviceCase
    spec = CaseSpec(n_h=128, d_c=512, d_h=128, d_r=64,
                    seq_lens=np.array([700, 65, 2, 300], np.int32), T_q=2, seed=21)
    dc = DeviceCase(spec, impl=M.IMPL_SIMT, max_splits=3)
    dc.step()                                   # reference: mla_decode with a workspace
    torch.cuda.synchronize()
    ref_lat, ref_lse = dc.latent.clone(), dc.lse.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # calls in a row: more splits, then fewer (the partials' lse block moves,
    # and the array still holds the larger call's values), then none (the
    # array is not used at all)
    for call, splits in enumerate((5, 3, 1)):
        lat = torch.full_like(dc.latent, float("nan"))
        lse = torch.full_like(dc.lse, float("nan"))
        M.mla_decode_noalloc(dc.cfg, dc.q_abs, dc.q_r, dc.pool, spec.num_blocks, dc.block_table,
                             spec.max_blocks, dc.seq_lens, spec.B, spec.T_q, splits, lat, lse,
                             status)
        torch.cuda.synchronize()
        assert M.mla_read_status(status) == 0
        _close(lat, ref_lat, f"latent, call {call} ({splits} splits)")
        d = (lse - ref_lse).abs().max().item()
        assert d <= LSE_ABS, (call, d)


def test_noalloc_reports_a_bad_block(M):
    """A block-table entry outside the pool is flagged in the caller's status
    word; that row is read as zeros, never out of bounds, so the outputs stay
    finite."""
    from mla_latent_kv_38_b200.runner import DeviceCase
    spec = CaseSpec(n_h=128, d_c=512, d_h=128, d_r=64, seq_lens=np.array([130, 70], np.int32), seed=23)
    dc = DeviceCase(spec, impl=M.IMPL_SIMT)
    dc.step()
    torch.cuda.synchronize()
    dc.block_table[0, 1] = spec.num_blocks + 5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lat = torch.full_like(dc.latent, float("nan"))
    lse = torch.full_like(dc.lse, float("nan"))
    M.mla_decode_noalloc(dc.cfg, dc.q_abs, dc.q_r, dc.pool, spec.num_blocks, dc.block_table,
                         spec.max_blocks, dc.seq_lens, spec.B, spec.T_q, 3, lat, lse, status)
    torch.cuda.synchronize()
    assert M.mla_read_status(status) & M.MLA_STATUS_BAD_BLOCK
    assert torch.isfinite(lat.float()).all() and torch.isfinite(lse).all()


def test_noalloc_rejects_requests_beyond_the_array(M):
    from mla_latent_kv_38_b200.runner import DeviceCase
    spec = CaseSpec(n_h=128, d_c=512, d_h=128, d_r=64, seq_lens=np.full(64, 64, np.int32), seed=22)
    dc = DeviceCase(spec, fill_history=False)
    # 64 splits * 64 rows * 128 heads * 2 KiB of partials is far beyond 16 MiB
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_noalloc(dc.cfg, dc.q_abs, dc.q_r, dc.pool, spec.num_blocks, dc.block_table,
                             spec.max_blocks, dc.seq_lens, spec.B, spec.T_q, 64, dc.latent, dc.lse)
    assert e.value.code == -3
