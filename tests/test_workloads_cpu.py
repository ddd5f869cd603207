"""The benchmark's workloads and roofline arithmetic, checked on the CPU.

The five workloads carry the shapes and lengths of the pages' DeepSeek-V2
setting ("Техотчёт DeepSeek-V2 (2024): MLA и экономика инференса", "Сколько
получилось": n_h = 128, d_c = 512, d_h = 128, d_h^R = 64), and the roofline's
numerators are plain counts: every cached row read once (d_c + d_r bf16),
the absorbed query and the outputs; 2 (d_c + d_r) + 2 d_c FLOPs per visible
(query, head, key) triple ("DeepSeek-V2 review", 2.1: T = max(B / BW, F / P)).
"""

import numpy as np
import pytest

from mla_latent_kv_38_b200 import synth
from mla_latent_kv_38_b200.workloads import CaseSpec, config_specs

V2 = dict(n_h=128, d_c=512, d_h=128, d_r=64)


def test_workload_shapes():
    specs = config_specs()
    tiny = specs["tiny"]
    assert (tiny.B, tiny.n_h, tiny.d_c, tiny.d_h, tiny.d_r, tiny.T_q) == (1, 4, 64, 32, 16, 1)
    assert list(tiny.seq_lens) == [128]
    for name in ("v2_decode", "varlen", "long", "multi_token"):
        s = specs[name]
        assert (s.n_h, s.d_c, s.d_h, s.d_r, s.block_size) == (128, 512, 128, 64, 64), name
    assert specs["v2_decode"].B == 32 and set(specs["v2_decode"].seq_lens) == {4096}
    assert specs["long"].B == 4 and set(specs["long"].seq_lens) == {131072}
    mt = specs["multi_token"]
    assert mt.B == 64 and mt.T_q == 4 and set(mt.seq_lens) == {8192}
    vl = specs["varlen"]
    assert vl.B == 128 and vl.permute_blocks
    assert vl.seq_lens.min() >= 512 and vl.seq_lens.max() <= 32768


def test_algorithmic_bytes_and_flops_closed_forms():
    specs = config_specs()
    s = specs["v2_decode"]
    # cache 32 x 4096 rows x 1152 B, q 32 x 128 x 1152 B, out 32 x 128 x (1024 + 4) B
    assert s.algorithmic_bytes() == 32 * 4096 * 1152 + 32 * 128 * 1152 + 32 * 128 * 1028
    assert abs(s.algorithmic_bytes() / 1e6 - 159.9) < 0.1
    # 2176 FLOPs per (query, head, visible key)
    assert s.algorithmic_flops() == 128 * 32 * 4096 * 2176
    assert abs(s.algorithmic_flops() / 1e9 - 36.5) < 0.05
    lg = specs["long"]
    assert abs(lg.algorithmic_bytes() / 1e6 - 605) < 1 and abs(lg.algorithmic_flops() / 1e9 - 146) < 0.5
    mt = specs["multi_token"]
    # the 4 new tokens see 8189 .. 8192 keys
    assert mt.visible_keys() == 64 * (8189 + 8190 + 8191 + 8192)
    assert abs(mt.algorithmic_flops() / 1e9 - 584) < 1


@pytest.mark.parametrize("T_q", [1, 3])
def test_visible_keys_follow_the_causal_mask(T_q):
    lens = np.array([5, 64, 130], np.int32)
    s = CaseSpec(**V2, seq_lens=lens, T_q=T_q)
    # query t of a sequence of length L sees keys 0 .. L - T_q + t
    want = sum(L - T_q + t + 1 for L in lens for t in range(T_q))
    assert s.visible_keys() == want


def test_block_tables_cover_every_block_once():
    s = CaseSpec(**V2, seq_lens=np.array([1, 64, 65, 700], np.int32), permute_blocks=True, seed=3)
    t = s.block_table()
    nb = s.blocks_per_seq()
    assert nb == [1, 1, 2, 11]
    used = np.concatenate([t[b, :n] for b, n in enumerate(nb)])
    assert sorted(used.tolist()) == list(range(s.num_blocks))
    for b, n in enumerate(nb):
        assert (t[b, n:] == -1).all()


def test_seeded_inputs_are_reproducible_and_keyed():
    a = synth.normal_bf16(5, 1, (4, 8))
    b = synth.normal_bf16(5, 1, (4, 8))
    c = synth.normal_bf16(6, 1, (4, 8))
    d = synth.normal_bf16(5, 2, (4, 8))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # one sequence's cache rows regenerate alone, from the same counter base
    s = CaseSpec(**V2, seq_lens=np.array([70, 70], np.int32), seed=9)
    whole = s.c_kv_rows(1, 0, 70)
    assert np.array_equal(whole[10:20], s.c_kv_rows(1, 10, 20))
    assert not np.array_equal(whole, s.c_kv_rows(0, 0, 70))
