"""The split-KV merge of the tensor-core decode, through the C ABI.

A (query row, block of 128 heads) unit whose keys are split over several SM
pairs is combined by log-sum-exp weights (the pages' split-KV decode: each
part's softmax is renormalised by exp(lse_part - lse)).  The merge kernel
reads every part's fp32 row and log-sum-exp; these cases cover units of 2 to
10 parts side by side, repeated calls on the same workspace, and multi-token
units, each against the fp64 oracle.
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec

from tests.test_gpu_parity import V2, _dc, check_sequences

pytestmark = pytest.mark.gpu

# 10, 5, 4 and 2 tiles of 256 keys: with max_splits = 0 every tile gets its
# own SM pair (fewer tiles than pairs), so the units have 10, 5, 4 and 2 parts
MIXED = dict(seq_lens=np.array([2560, 1280, 1024, 300], np.int32), seed=21)


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


@pytest.mark.parametrize("splits, want", [(0, [10, 5, 4, 2]), (5, [5, 5, 4, 2]), (2, [2, 2, 2, 2])])
def test_units_of_many_parts_merge_to_the_oracle(M, splits, want):
    spec = CaseSpec(**V2, **MIXED)
    dc = _dc(spec, impl=0, max_splits=splits)
    U = spec.B
    for _ in range(3):   # repeated calls reuse the workspace's partial slots
        dc.reset_step_inputs()
        dc.latent.fill_(float("nan"))
        dc.step()
        torch.cuda.synchronize()
        assert dc.decode_status() == 0
        check_sequences(dc, range(spec.B))
    assert M.mla_decode_split_counts(dc.cfg, spec.B, 1, splits, dc.ws, U).tolist() == want


def test_multi_token_units_merge_to_the_oracle(M):
    """T_q = 2 doubles the units; each sequence's two query rows are split and
    merged separately (token-major unit order)."""
    spec = CaseSpec(**V2, seq_lens=np.array([700, 1100, 90], np.int32), T_q=2, seed=22)
    dc = _dc(spec, impl=0, max_splits=3)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0
    check_sequences(dc, range(spec.B))
    parts = M.mla_decode_split_counts(dc.cfg, spec.B, spec.T_q, 3, dc.ws, spec.B * spec.T_q).tolist()
    assert max(parts) == 3 and min(parts) >= 1, parts
