"""The tensor-core decode's bounded waits, exercised without a GPU fault.

Every mbarrier wait of the decode kernel gives up after a time limit, sets
MLA_STATUS_TIMEOUT in the status word, lets issued tensor-core work drain,
frees its tensor memory and returns.  mla_test_arm_decode_timeout makes the
next decode call withhold one cache load (a barrier that nothing completes)
and bounds its waits by a few milliseconds.  The call must return, report
MLA_STATUS_TIMEOUT, and leave the context usable: an ordinary call right
after it matches the fp64 oracle.
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


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_38_b200 import build
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def test_withheld_load_times_out_and_the_next_call_is_clean(M):
    from mla_latent_kv_38_b200.runner import DeviceCase
    spec = CaseSpec(n_h=128, d_c=512, d_h=128, d_r=64, seq_lens=np.array([300, 65], np.int32), seed=31)
    dc = DeviceCase(spec, impl=M.IMPL_TCGEN05)
    dc.step()                                   # RoPE'd query and the appended rows in place
    torch.cuda.synchronize()
    assert dc.decode_status() == 0

    M.mla_clear_status(dc.ws)
    M.mla_test_arm_decode_timeout(5_000_000)    # 5 ms per wait
    dc.decode_only()
    torch.cuda.synchronize()                    # the call returned: nothing hangs
    assert dc.decode_status() & M.MLA_STATUS_TIMEOUT

    # the same context, an ordinary call: tensor memory was freed, no state leaked
    M.mla_clear_status(dc.ws)
    dc.latent.fill_(float("nan"))
    dc.decode_only()
    M.mla_up_v(dc.cfg, dc.latent, dc.w_uv, dc.out, spec.n_tok)
    torch.cuda.synchronize()
    assert dc.decode_status() == 0
    s = spec
    out = dc.out.float().cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h, s.d_h)
    lat = dc.latent.float().cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h, s.d_c)
    lse = dc.lse.cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h)
    for b in range(s.B):
        ref = reference(s, b)
        for got, want, what in ((out[b], ref["o"], "o"), (lat[b], ref["latent"], "latent")):
            err = np.abs(got - want)
            assert np.isfinite(got).all(), what
            assert err.max() <= MAX_ABS and err.sum() / np.abs(want).sum() <= MEAN_REL, (what, b)
        assert np.abs(lse[b] - ref["lse"]).max() <= LSE_ABS


def test_arm_rejects_out_of_range_limits(M):
    with pytest.raises(M.MlaError) as e:
        M.mla_test_arm_decode_timeout(0)
    assert e.value.code == -3
    with pytest.raises(M.MlaError) as e:
        M.mla_test_arm_decode_timeout(3_000_000_000)
    assert e.value.code == -3
