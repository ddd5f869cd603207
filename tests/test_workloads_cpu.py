"""The benchmark's workloads, roofline arithmetic and input generator, checked
on the CPU.

The generator is pinned to SplitMix64's published outputs, its bf16 rounding to
round-to-nearest-even (ties included), and its torch form (used to fill the
cache history on the device) to its numpy form (used by the oracle).

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


def test_splitmix64_matches_its_published_outputs():
    """SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) from state 0 starts
    0xe220a8397b1dcdaf, 0x6e789e6aa1b965f4, 0x06c45d188009454f,
    0xf88bb8a8724c81ec; the counter form used here is output k of the stream
    seeded with the tensor's key."""
    gamma = 0x9E3779B97F4A7C15
    mask = (1 << 64) - 1

    def mix(z):
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
        return z ^ (z >> 31)

    def stream(state, n):
        out = []
        for _ in range(n):
            state = (state + gamma) & mask
            out.append(mix(state))
        return out

    assert stream(0, 4) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]
    for seed, tid in ((0, 1), (7, 5), (123456789, 8)):
        key = int(synth._key(seed, tid))
        got = synth.uniform_u64(seed, tid, np.arange(6, dtype=np.uint64))
        assert [int(x) for x in got] == stream(key, 6)


def test_bf16_rounding_is_nearest_even_in_one_step():
    r = np.random.default_rng(5)
    x = np.concatenate([r.standard_normal(20000) * 10.0 ** r.integers(-6, 6, 20000),
                        # exact halfway points between neighbouring bf16 values: odd
                        # 9-bit significands 257 .. 511 at a few scales, both signs
                        np.outer(np.arange(257, 512, 2), 2.0 ** np.array([-20, -9, 0, 7])).ravel(),
                        -np.outer(np.arange(257, 512, 2), 2.0 ** np.array([-3, 11])).ravel()])
    bits = synth.to_bf16_bits(x)
    got = synth.bf16_bits_to_f64(bits)
    ties = [0]
    for v, g in zip(x.tolist(), got.tolist()):
        # neighbours of v with 8 significant bits, in exact float arithmetic
        m, e = np.frexp(abs(v))                     # v = m 2^e, 0.5 <= m < 1
        ulp = 2.0 ** (int(e) - 8)
        lo = np.floor(abs(v) / ulp) * ulp
        hi = lo + ulp
        if abs(v) - lo < hi - abs(v):
            want = lo
        elif abs(v) - lo > hi - abs(v):
            want = hi
        else:                                       # tie: the even significand
            ties[0] += 1
            want = lo if int(lo / ulp) % 2 == 0 else hi
        assert g == np.copysign(want, v), (v, g, want)
    assert ties[0] == 128 * 6


def test_torch_generator_matches_numpy_generator():
    """The cache history is drawn with the torch form of the generator; the
    oracle draws the same rows with the numpy form."""
    torch = pytest.importorskip("torch")
    for seed, tid, start, count in ((0, 1, 0, 50000), (3, 2, (5 << 20) * 64, 4096), (9, 4, 12345, 777)):
        a = synth.normal_bf16(seed, tid, (count,), start=start)
        b = synth.normal_bf16_torch(seed, tid, count, start=start, device="cpu", chunk=1 << 14)
        b = b.view(torch.int16).numpy().view(np.uint16)
        assert (a != b).sum() == 0


def test_box_muller_normals_have_unit_moments():
    z = synth.normal_f64(11, 3, 0, 200000)
    n = z.size
    assert abs(z.mean()) < 5 / np.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    # a tail fraction: P(|z| > 2) = 0.0455
    assert abs((np.abs(z) > 2).mean() - 0.0455) < 0.003
