"""Chunked prefill on the paged latent cache, through the C ABI, against the fp64 oracle.

"MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리", "MLA 코드 구현" (the
forward's mask `triu(diagonal = T_k - T_q + 1)`) and "학습 시와 디코딩 시의 흐름":
a chunk of T_q new tokens is appended to the cache and attends to the cached
prefix and causally to itself; T_q = L is prefill from an empty cache.  The
calls are those of the decode step (mla_absorb_q, mla_rope_append with T_q
tokens per sequence, mla_decode with T_q > 1, mla_up_v); the oracle is the same
explicit reconstruction with the generalised mask.
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_38_b200.workloads import CaseSpec, prefill_specs

from tests.test_gpu_parity import V2, SAMPLE_HEADS, _dc, check_sequences

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


SMALL = {
    # a 64-token chunk over prefixes of 236 and 37 rows
    "chunk_over_prefix": CaseSpec(**V2, seq_lens=np.array([300, 101], np.int32), T_q=64, seed=31),
    # sequence 1 has no prefix (L = T_q): prefill from an empty cache
    "from_empty_cache": CaseSpec(**V2, seq_lens=np.array([200, 129], np.int32), T_q=129, seed=32),
    # ragged pages, permuted block table, a chunk that starts mid-page
    "ragged_chunk": CaseSpec(**V2, seq_lens=np.array([257, 1000, 64], np.int32), T_q=64, seed=33,
                             permute_blocks=True),
    # head shapes the tensor-core kernels do not take: portable kernels
    "small_heads": CaseSpec(n_h=4, d_c=64, d_h=32, d_r=16, seq_lens=np.array([40, 90], np.int32), T_q=40,
                            seed=34),
}


@pytest.mark.parametrize("impl", [0, 1])
@pytest.mark.parametrize("name", sorted(SMALL))
def test_prefill_small(M, name, impl):
    spec = SMALL[name]
    dc = _dc(spec, impl=impl)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    check_sequences(dc, range(spec.B))


@pytest.mark.parametrize("splits", [1, 3])
def test_prefill_split_bound(M, splits):
    """The bound on parts per unit holds for prefill units too (units of a
    sequence have kv = L - T_q + t + 1 keys, from the prefix up to L)."""
    spec = SMALL["ragged_chunk"]
    dc = _dc(spec, impl=0, max_splits=splits)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0
    check_sequences(dc, range(spec.B))
    U = spec.B * spec.T_q
    parts = M.mla_decode_split_counts(dc.cfg, spec.B, spec.T_q, splits, dc.ws, U).numpy()
    assert parts.max() <= splits


@pytest.mark.parametrize("name, all_heads, sampled", [("prefill_chunk", [0], [3]), ("prefill", [], [0])])
def test_prefill_full_size(M, name, all_heads, sampled):
    """The benchmark's prefill workloads in its launch configuration: every
    head of a whole 512-token chunk, sampled heads elsewhere."""
    spec = prefill_specs()[name]
    dc = _dc(spec)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    if all_heads:
        check_sequences(dc, all_heads)
    check_sequences(dc, sampled, SAMPLE_HEADS)
