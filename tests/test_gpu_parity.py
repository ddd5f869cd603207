"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bars: bit-exact for the cache append and the page-table gather; for floating
point, max-abs error <= 2e-2 and mean relative error sum|gpu-ref|/sum|ref|
<= 5e-3 on the head output o and on the latent output, and |lse error| <= 1e-2.
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
    return DeviceCase(spec, **kw)


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got, want, what):
    err = np.abs(got - want)
    max_abs = float(err.max())
    mre = float(err.sum() / max(np.abs(want).sum(), 1e-300))
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert max_abs <= MAX_ABS and mre <= MEAN_REL, f"{what}: max_abs={max_abs:.3e} mean_rel={mre:.3e}"
    return max_abs, mre


def check_sequences(dc, seqs, heads=None):
    s = dc.spec
    out = _f64(dc.out).reshape(s.B, s.T_q, s.n_h, s.d_h)
    lat = _f64(dc.latent).reshape(s.B, s.T_q, s.n_h, s.d_c)
    lse = dc.lse.cpu().numpy().astype(np.float64).reshape(s.B, s.T_q, s.n_h)
    hs = list(range(s.n_h)) if heads is None else list(heads)
    for b in seqs:
        ref = reference(s, b, heads=hs)
        assert_close(out[b][:, hs], ref["o"], f"o seq {b}")
        assert_close(lat[b][:, hs], ref["latent"], f"latent seq {b}")
        d = np.abs(lse[b][:, hs] - ref["lse"]).max()
        assert d <= LSE_ABS, f"lse seq {b}: {d:.3e}"


V2 = dict(n_h=128, d_c=512, d_h=128, d_r=64)

SMALL_CASES = {
    "tiny_config": config_specs()["tiny"],
    "v2_ragged": CaseSpec(**V2, seq_lens=np.array([1, 63, 64, 65, 300], np.int32), seed=1),
    "v2_permuted": CaseSpec(**V2, seq_lens=np.array([700, 129, 2], np.int32), seed=2,
                            permute_blocks=True),
    "v2_multi_token": CaseSpec(**V2, seq_lens=np.array([4, 5, 67, 200], np.int32), T_q=4, seed=3),
    "tiny_multi_token": CaseSpec(n_h=4, d_c=64, d_h=32, d_r=16,
                                 seq_lens=np.array([2, 64, 129], np.int32), T_q=2, seed=4),
    "odd_heads": CaseSpec(n_h=12, d_c=128, d_h=64, d_r=32, seq_lens=np.array([33, 97], np.int32),
                          seed=5),
}


@pytest.mark.parametrize("name", sorted(SMALL_CASES))
@pytest.mark.parametrize("impl", [0, 1])
def test_full_path_small(M, name, impl):
    spec = SMALL_CASES[name]
    dc = _dc(spec, impl=impl)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    check_sequences(dc, range(spec.B))


@pytest.mark.parametrize("name", sorted(SMALL_CASES))
def test_append_and_gather_bit_exact(M, name):
    spec = SMALL_CASES[name]
    dc = _dc(spec)
    dc.step()
    torch.cuda.synchronize()
    pool = dc.bits(dc.pool)
    table = dc.block_table_np
    tab = O.rope_table_f32(dc.max_pos, spec.d_r)
    for b, L in enumerate(spec.seq_lens):
        L = int(L)
        rows = O.gather_rows(pool, table, b, L, spec.block_size)     # through the block table
        assert np.array_equal(rows[:, :spec.d_c], spec.c_kv_rows(b, 0, L))
        want_kr = O.rope_emulate_bf16(spec.k_r_rows(b, 0, L), np.arange(L), tab)
        assert np.array_equal(rows[:, spec.d_c:], want_kr)
    # the step's query RoPE, in place
    q_r = dc.bits(dc.q_r)
    want_q = O.rope_emulate_bf16(spec.q_r(), spec.positions()[:, None], tab)
    assert np.array_equal(q_r, want_q)


def test_many_units_whole_and_split(M):
    # 300 units of 9 pages each (last page partial): most units fit inside one
    # cluster's page range (written directly), the rest straddle two clusters
    spec = CaseSpec(**V2, seq_lens=np.full(300, 517, np.int32), seed=12, permute_blocks=True)
    dc = _dc(spec)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0
    check_sequences(dc, [0, 1, 150, 298, 299])


def test_schedule_kernel_for_many_units(M):
    """Above 2,048 units (query row, block of 128 heads) the schedule is
    computed by a separate one-block kernel before the decode (three launches
    instead of two).  2,100 sequences: most of 70 to 260 keys (one 256-key
    tile, never split: cuts fall between tiles), every seventh of 600 to 899
    keys (3 or 4 tiles), so that some cuts fall inside a unit, which is then
    split and merged."""
    lens = np.array([600 + (37 * b) % 300 if b % 7 == 0 else 70 + (37 * b) % 191 for b in range(2100)], np.int32)
    spec = CaseSpec(**V2, seq_lens=lens, seed=13, permute_blocks=True)
    dc = _dc(spec)
    assert M.mla_decode_launches(dc.cfg, spec.B, 1, 0) == 3
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0
    parts = M.mla_decode_split_counts(dc.cfg, spec.B, 1, 0, dc.ws, spec.B).numpy()
    assert parts.min() >= 1 and parts.max() >= 2
    split = [int(b) for b in np.nonzero(parts >= 2)[0]]
    whole = [int(b) for b in np.nonzero(parts == 1)[0]]
    check_sequences(dc, sorted(set(split[:3] + split[-2:] + whole[:2] + whole[-2:] + [1049])))


SPLIT_SPEC = dict(seq_lens=np.array([1000, 37, 513], np.int32), seed=6)


@pytest.mark.parametrize("splits", [0, 1, 2, 3, 7])
@pytest.mark.parametrize("impl", [0, 1])
def test_split_count_invariance(M, splits, impl):
    spec = CaseSpec(**V2, **SPLIT_SPEC)
    dc = _dc(spec, impl=impl, max_splits=splits)
    dc.step()
    torch.cuda.synchronize()
    check_sequences(dc, range(spec.B))
    U = spec.B * spec.T_q * spec.n_h // 128
    parts = M.mla_decode_split_counts(dc.cfg, spec.B, spec.T_q, splits, dc.ws, U).tolist()
    if impl == 1:
        assert parts == [splits if splits else parts[0]] * U
        return
    # tensor-core decode: 4, 1 and 3 tiles of 256 keys over 74 SM pairs; the
    # bound caps the parts of every unit, and each unit is split as far as the
    # bound and its tile count allow (the equal cut gives every tile its own
    # range)
    tiles = [4, 1, 3]
    want = [min(splits, n) if splits else n for n in tiles]
    assert parts == want, (splits, parts)


def test_split_counts_differ_with_the_bound(M):
    """The tensor-core decode's per-unit split counts, read back from the
    workspace, follow max_splits (and the results stay within tolerance)."""
    spec = CaseSpec(**V2, **SPLIT_SPEC)
    seen = []
    for splits in (1, 2, 3, 7):
        dc = _dc(spec, impl=0, max_splits=splits)
        dc.step()
        torch.cuda.synchronize()
        check_sequences(dc, range(spec.B))
        seen.append(tuple(M.mla_decode_split_counts(dc.cfg, spec.B, 1, splits, dc.ws, 3).tolist()))
        assert max(seen[-1]) <= splits
    assert len(set(seen)) == 4, seen


# Head shapes for the projections: the DeepSeek-V2 shape, and shapes that take
# the other tiling branches (d_h = 64 or 192 for absorb_q's contraction, two
# 128-feature tiles for up_v) or fall back to the CUDA-core kernels.
PROJ_SHAPES = {
    "v2": dict(n_h=128, d_c=512, d_h=128),
    "small": dict(n_h=12, d_c=128, d_h=64),
    "wide": dict(n_h=6, d_c=256, d_h=192),
    "tall": dict(n_h=5, d_c=192, d_h=256),
}
# token counts: one token, below one 16-row MMA step, the V2 decode batch, and
# more than one token tile with a ragged last tile
PROJ_TOKENS = [1, 15, 32, 300]
_proj_inputs = {}


def _proj_case(shape, n_tok):
    key = (shape, n_tok)
    if key not in _proj_inputs:
        from mla_latent_kv_38_b200 import synth
        d = PROJ_SHAPES[shape]
        n_h, d_c, d_h = d["n_h"], d["d_c"], d["d_h"]
        seed = 11 + n_tok
        q_c = synth.normal_bf16(seed, 1, (n_tok, n_h, d_h))
        lat = synth.normal_bf16(seed, 2, (n_tok, n_h, d_c), std=0.05)
        w_uk = synth.normal_bf16(seed, 3, (n_h, d_h, d_c), std=synth.weight_std(d_c))
        w_uv = synth.normal_bf16(seed, 4, (n_h, d_h, d_c), std=synth.weight_std(d_c))
        want_q = O.absorb_q(O.bf16_to_f64(q_c), O.bf16_to_f64(w_uk))
        want_o = O.up_v(O.bf16_to_f64(lat), O.bf16_to_f64(w_uv))
        _proj_inputs[key] = (q_c, lat, w_uk, w_uv, want_q, want_o)
    return _proj_inputs[key]


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("impl", [0, 1])
@pytest.mark.parametrize("n_tok", PROJ_TOKENS)
@pytest.mark.parametrize("shape", sorted(PROJ_SHAPES))
def test_projection_parity(M, shape, n_tok, impl):
    d = PROJ_SHAPES[shape]
    q_c, lat, w_uk, w_uv, want_q, want_o = _proj_case(shape, n_tok)
    cfg = M.MlaConfig(d["n_h"], d["d_c"], d["d_h"], 16, 64, 0.0, impl)
    q_abs = torch.full((n_tok, d["n_h"], d["d_c"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = torch.full((n_tok, d["n_h"], d["d_h"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.mla_absorb_q(cfg, _dev(q_c), _dev(w_uk), q_abs, n_tok)
    M.mla_up_v(cfg, _dev(lat), _dev(w_uv), out, n_tok)
    torch.cuda.synchronize()
    assert_close(_f64(q_abs), want_q, f"q_abs {shape} n_tok={n_tok}")
    assert_close(_f64(out), want_o, f"up_v {shape} n_tok={n_tok}")


def test_projection_tcgen05_shapes(M):
    """impl = 2 forces the tensor-core projections and rejects shapes they do
    not tile; the shapes they do tile match the CUDA-core kernels' results."""
    for shape, absorb_ok, up_v_ok in [("v2", True, True), ("small", True, False),
                                      ("wide", True, False), ("tall", False, True)]:
        d = PROJ_SHAPES[shape]
        q_c, lat, w_uk, w_uv, want_q, want_o = _proj_case(shape, 32)
        cfg = M.MlaConfig(d["n_h"], d["d_c"], d["d_h"], 16, 64, 0.0, M.IMPL_TCGEN05)
        q_abs = torch.empty((32, d["n_h"], d["d_c"]), dtype=torch.bfloat16, device="cuda")
        out = torch.empty((32, d["n_h"], d["d_h"]), dtype=torch.bfloat16, device="cuda")
        if absorb_ok:
            M.mla_absorb_q(cfg, _dev(q_c), _dev(w_uk), q_abs, 32)
            torch.cuda.synchronize()
            assert_close(_f64(q_abs), want_q, f"q_abs {shape} tcgen05")
        else:
            with pytest.raises(M.MlaError) as e:
                M.mla_absorb_q(cfg, _dev(q_c), _dev(w_uk), q_abs, 32)
            assert e.value.code == -2, shape
        if up_v_ok:
            M.mla_up_v(cfg, _dev(lat), _dev(w_uv), out, 32)
            torch.cuda.synchronize()
            assert_close(_f64(out), want_o, f"up_v {shape} tcgen05")
        else:
            with pytest.raises(M.MlaError) as e:
                M.mla_up_v(cfg, _dev(lat), _dev(w_uv), out, 32)
            assert e.value.code == -2, shape


def test_device_checks_flag_bad_rows(M):
    spec = CaseSpec(**V2, seq_lens=np.array([130, 70], np.int32), seed=9)
    dc = _dc(spec)
    # sequence 1 claims fewer rows than its query tokens need
    dc.seq_lens[1] = 0
    M.mla_clear_status(dc.ws)
    dc.decode_only()
    assert dc.decode_status() & M.MLA_STATUS_BAD_SEQ_LEN
    # a block-table entry outside the pool
    dc.seq_lens[1] = 70
    dc.block_table[0, 1] = spec.num_blocks + 5
    M.mla_clear_status(dc.ws)
    dc.decode_only()
    assert dc.decode_status() & M.MLA_STATUS_BAD_BLOCK
    # an append through the bad entry (sequence 0, block 1) and one position
    # beyond the RoPE table (sequence 1): both rows skipped and flagged
    M.mla_clear_status(dc.status)
    dc.positions[0] = 64 + 3
    dc.positions[1] = dc.max_pos + 1
    dc.step()
    st = dc.append_status()
    assert st & M.MLA_STATUS_BAD_POSITION and st & M.MLA_STATUS_BAD_BLOCK
    torch.cuda.synchronize()


def test_host_argument_errors(M):
    spec = CaseSpec(**V2, seq_lens=np.array([64], np.int32), seed=10)
    dc = _dc(spec, fill_history=False)
    with pytest.raises(M.MlaError) as e:
        M.mla_decode(dc.cfg, dc.q_abs, dc.q_r, dc.pool, spec.num_blocks, dc.block_table,
                     spec.max_blocks, dc.seq_lens, 1, 1, 0, dc.ws, 16, dc.latent, dc.lse)
    assert e.value.code == -4
    with pytest.raises(M.MlaError) as e:
        M.mla_decode(dc.cfg, dc.q_abs, dc.q_r, dc.pool, spec.num_blocks, dc.block_table,
                     spec.max_blocks, dc.seq_lens, 1, 65536, 0, dc.ws, dc.ws_bytes, dc.latent, dc.lse)
    assert e.value.code == -3
    bad = M.MlaConfig(128, 512, 128, 64, block_size=32)
    with pytest.raises(M.MlaError) as e:
        M.mla_absorb_q(bad, dc.q_c, dc.w_uk, dc.q_abs, 1)
    assert e.value.code == -2


# ---------------------------------------------------------------------------
# Full sizes of the five workloads, in the benchmark's launch configuration:
# every head of at least two sequences, plus at least eight seeded sequences
# (all of them where the workload has fewer) at sampled heads.
# ---------------------------------------------------------------------------

def _sampled(B, n, seed):
    rng = np.random.default_rng(seed)
    return sorted(int(x) for x in rng.choice(B, size=min(n, B), replace=False))


# workload: (sequences checked on all heads, sequences checked on SAMPLE_HEADS)
FULL = {
    "tiny": ([0], []),
    "v2_decode": ([0, 31], _sampled(32, 8, 101)),
    "varlen": ([0, 77], _sampled(128, 8, 102)),
    "long": ([0, 3], [1, 2]),
    "multi_token": ([0, 63], _sampled(64, 8, 103)),
}
SAMPLE_HEADS = [0, 1, 63, 64, 65, 127]


@pytest.mark.parametrize("name", ["tiny", "v2_decode", "multi_token", "long", "varlen"])
def test_full_size(M, name):
    spec = config_specs()[name]
    all_heads, sampled = FULL[name]
    dc = _dc(spec)
    dc.step()
    torch.cuda.synchronize()
    assert dc.decode_status() == 0 and dc.append_status() == 0
    check_sequences(dc, all_heads)
    if sampled:
        check_sequences(dc, sampled, [h for h in SAMPLE_HEADS if h < spec.n_h])
    # page-table gather of the fully checked sequences' cache rows, bit exact
    pool = dc.bits(dc.pool)
    tab = O.rope_table_f32(dc.max_pos, spec.d_r)
    for b in all_heads:
        L = int(spec.seq_lens[b])
        rows = O.gather_rows(pool, dc.block_table_np, b, L, spec.block_size)
        assert np.array_equal(rows[:, :spec.d_c], spec.c_kv_rows(b, 0, L))
        assert np.array_equal(rows[:, spec.d_c:],
                              O.rope_emulate_bf16(spec.k_r_rows(b, 0, L), np.arange(L), tab))
