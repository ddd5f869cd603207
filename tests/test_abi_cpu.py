"""CPU-side checks of the C ABI library: it builds for sm_100a, loads, exports
every function include/mla.h declares, and rejects bad arguments on the host
before touching a device (so these calls are safe without a GPU)."""

import ctypes
import os
import re

import numpy as np
import pytest

from mla_latent_kv_38_b200 import build
from oracle import mla_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    build.build()
    from mla_latent_kv_38_b200 import binding
    return binding


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(M):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(M._lib, n), n
    assert set(M.EXPORTED) == set(names)


def test_status_strings(M):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert M.mla_status_str(code) not in ("", "unknown status")
    assert M.mla_status_str(-99) == "unknown status"


def test_library_rope_table_matches_oracle_table(M):
    for d_r, max_pos in ((16, 300), (64, 5000)):
        lib = M.mla_rope_table(d_r, 10000.0, max_pos).numpy()
        ref = O.rope_table_f32(max_pos, d_r)
        ulps = np.abs(lib.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
        assert ulps.max() <= 1
        assert (ulps > 0).mean() < 1e-3


FAKE = 0x10000  # 16-byte aligned non-null value; never dereferenced by these calls


def _cfg(M, **kw):
    base = dict(n_h=128, d_c=512, d_h=128, d_r=64)
    base.update(kw)
    return M.MlaConfig(**base)


def test_host_validation_without_device(M):
    raw = M.raw_call
    cfg = _cfg(M)
    bad_block = _cfg(M, block_size=32)
    bad_dc = _cfg(M, d_c=520)
    p = ctypes.c_void_p(FAKE)
    assert raw("mla_absorb_q", ctypes.byref(bad_block), p, p, p, 4, None, None) == -2
    assert raw("mla_absorb_q", ctypes.byref(bad_dc), p, p, p, 4, None, None) == -2
    assert raw("mla_absorb_q", ctypes.byref(cfg), None, p, p, 4, None, None) == -1
    assert raw("mla_absorb_q", ctypes.byref(cfg), ctypes.c_void_p(FAKE + 2), p, p, 4, None, None) == -7
    assert raw("mla_absorb_q", ctypes.byref(cfg), p, p, p, 0, None, None) == -3
    assert raw("mla_absorb_q", ctypes.byref(cfg), p, p, p, 4, ctypes.c_void_p(FAKE + 2), None) == -7
    assert raw("mla_up_v", ctypes.byref(cfg), p, p, p, 70000, None, None) == -3
    assert raw("mla_up_v", ctypes.byref(cfg), p, p, p, 4, ctypes.c_void_p(FAKE + 2), None) == -7
    ws = M.mla_decode_workspace_bytes(cfg, 32, 1, 0)
    assert ws >= 256 and ws % 256 == 0
    assert M.mla_decode_workspace_bytes(cfg, 32, 1, 4) >= M.mla_decode_workspace_bytes(cfg, 32, 1, 1)
    args = [ctypes.byref(cfg), p, p, p, 10, p, 1, p, 32, 1, 0, p, ws - 1, p, p, None]
    assert raw("mla_decode", *args) == -4
    args[12] = ws
    args[11] = ctypes.c_void_p(FAKE + 16)          # workspace must be 256-byte aligned
    assert raw("mla_decode", *args) == -4
    args[11] = p
    args[9] = 2048                                  # B * T_q = 65,536 query rows: one too many
    assert raw("mla_decode", *args) == -3
    args[9] = 1
    args[1] = None
    assert raw("mla_decode", *args) == -1
    impl_tc_tiny = _cfg(M, n_h=4, d_c=64, d_h=32, d_r=16, impl=2)
    args = [ctypes.byref(impl_tc_tiny), p, p, p, 10, p, 1, p, 1, 1, 0, p,
            M.mla_decode_workspace_bytes(impl_tc_tiny, 1, 1, 0), p, p, None]
    assert raw("mla_decode", *args) == -2           # tcgen05 kernel needs the V2 shape
    assert raw("mla_rope_table", 64, ctypes.c_double(10000.0), 0, p) == -3
    assert raw("mla_clear_status", None, None) == -1


def test_rope_append_host_validation(M):
    raw = M.raw_call
    cfg = _cfg(M)
    p = ctypes.c_void_p(FAKE)

    def call(c=cfg, q_r=p, k_r=p, c_kv=p, pos=p, table=p, max_pos=4096, bt=p, mbps=64,
             pool=p, num_blocks=2048, B=32, T_q=1, status=None):
        return raw("mla_rope_append", ctypes.byref(c), q_r, k_r, c_kv, pos, table, max_pos, bt, mbps,
                   pool, num_blocks, B, T_q, status, None)

    assert call(c=_cfg(M, block_size=16)) == -2
    assert call(c=_cfg(M, d_r=72)) == -2
    for name in ("k_r", "c_kv", "pos", "table", "bt", "pool"):
        assert call(**{name: None}) == -1, name
    odd16 = ctypes.c_void_p(FAKE + 8)               # 8-byte but not 16-byte aligned
    odd4 = ctypes.c_void_p(FAKE + 2)
    for name in ("q_r", "k_r", "c_kv", "pool"):
        assert call(**{name: odd16}) == -7, name
    for name in ("pos", "table", "bt", "status"):
        assert call(**{name: odd4}) == -7, name
    assert call(B=0) == -3 and call(T_q=0) == -3
    assert call(B=1 << 13, T_q=1 << 12) == -3       # more than 2^24 tokens
    assert call(max_pos=0) == -3 and call(mbps=0) == -3 and call(num_blocks=0) == -3


def test_decode_launch_counts(M):
    v2 = _cfg(M)
    # tensor-core kernels: decode (which computes its own schedule) + merge; a
    # separate scheduling kernel only beyond 2048 units of (query row, 128 heads)
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 32, 1, 0) == 2
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 32, 1, 3) == 2
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 2048, 1, 0) == 2
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 2049, 1, 0) == 3
    assert M.raw_call("mla_decode_launches", ctypes.byref(_cfg(M, n_h=256)), 1025, 1, 0) == 3
    # portable kernels: one launch without splits, decode + merge with them
    simt = _cfg(M, impl=1)
    assert M.raw_call("mla_decode_launches", ctypes.byref(simt), 32, 1, 1) == 1
    assert M.raw_call("mla_decode_launches", ctypes.byref(simt), 32, 1, 4) == 2
    # automatic choice: 32 rows x 16 head groups fill 8 x 148 slots with 3 splits
    assert M.raw_call("mla_decode_launches", ctypes.byref(simt), 32, 1, 0) == 2
    assert M.raw_call("mla_decode_launches", ctypes.byref(simt), 4095, 16, 0) == 1
    # prefill-sized chunks: T_q is limited only by the row and unit counts
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 1, 2048, 0) == 2
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 4, 4096, 0) == 3
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 2, 32768, 0) == -3
    assert M.raw_call("mla_decode_launches", ctypes.byref(_cfg(M, n_h=256)), 1, 40000, 0) == -3
    tiny = _cfg(M, n_h=4, d_c=64, d_h=32, d_r=16)
    assert M.raw_call("mla_decode_launches", ctypes.byref(tiny), 1, 1, 0) == 2
    tiny_tc = _cfg(M, n_h=4, d_c=64, d_h=32, d_r=16, impl=2)
    assert M.raw_call("mla_decode_launches", ctypes.byref(tiny_tc), 1, 1, 0) == -2
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 32, 2048, 0) == -3
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 0, 1, 0) == -3
    assert M.raw_call("mla_decode_launches", ctypes.byref(v2), 32, 1, -1) == -3
    # the workspace query answers 0 for arguments the decode call would reject
    assert M.mla_decode_workspace_bytes(v2, 0, 1, 0) == 0
    assert M.mla_decode_workspace_bytes(_cfg(M, block_size=32), 32, 1, 0) == 0


def test_workspace_covers_only_the_kernels_that_run(M):
    """The tensor-core decode's workspace holds its schedule arrays and its
    (74 + U) partial slots of 128 rows x (512 + 1) fp32, and nothing for the
    portable kernel's partials (and the other way round)."""
    v2 = _cfg(M)
    U = 32
    slots = (74 + U) * 128 * (512 + 1) * 4
    tc = M.mla_decode_workspace_bytes(v2, 32, 1, 0)
    assert slots < tc < slots + (1 << 16), tc
    assert M.mla_decode_workspace_bytes(v2, 32, 1, 7) == tc           # max_splits changes no size
    simt = M.mla_decode_workspace_bytes(_cfg(M, impl=1), 32, 1, 3)
    assert 3 * 32 * 128 * (512 + 1) * 4 <= simt < 3 * 32 * 128 * (512 + 1) * 4 + 1024, simt
    assert M.mla_decode_workspace_bytes(_cfg(M, impl=1), 32, 1, 1) == 256   # no splits: the status word only


def test_noalloc_rejects_before_touching_a_device(M):
    raw = M.raw_call
    cfg = _cfg(M)
    p = ctypes.c_void_p(FAKE)

    def call(c=cfg, B=32, T_q=1, splits=2, status=None, **ptrs):
        a = dict(q_abs=p, q_r=p, pool=p, bt=p, lens=p, out=p, lse=p)
        a.update(ptrs)
        return raw("mla_decode_noalloc", ctypes.byref(c), a["q_abs"], a["q_r"], a["pool"], 2048, a["bt"],
                   64, a["lens"], B, T_q, splits, a["out"], a["lse"], status, None)

    assert call(c=_cfg(M, block_size=32)) == -2
    for name in ("q_abs", "q_r", "pool", "bt", "lens", "out", "lse"):
        assert call(**{name: None}) == -1, name
    assert call(q_abs=ctypes.c_void_p(FAKE + 8)) == -7
    assert call(status=ctypes.c_void_p(FAKE + 2)) == -7
    assert call(splits=0) == -3 and call(splits=257) == -3 and call(T_q=17) == -3
    # 2 splits x 4096 rows x (512 + 1) fp32 is 32 KiB over the fixed 16 MiB array
    assert 2 * 32 * 128 * (4 * 512 + 4) > 16 << 20
    assert call(splits=2) == -3
    assert call(B=8, splits=64) == -3


@pytest.mark.parametrize("field,value,ok", [
    ("n_h", 0, False), ("n_h", 1, True), ("n_h", 1024, True), ("n_h", 1025, False),
    ("d_c", 0, False), ("d_c", 8, True), ("d_c", 12, False), ("d_c", 512, True), ("d_c", 520, False),
    ("d_r", 0, False), ("d_r", 8, True), ("d_r", 12, False), ("d_r", 64, True), ("d_r", 72, False),
    ("d_h", 0, False), ("d_h", 8, True), ("d_h", 12, False), ("d_h", 256, True), ("d_h", 264, False),
    ("block_size", 32, False), ("block_size", 128, False),
    ("impl", -1, False), ("impl", 3, False),
    ("scale", float("nan"), False), ("scale", -1.0, True), ("scale", 0.125, True),
])
def test_config_limits(M, field, value, ok):
    """The shape limits the header states, at their boundaries (the launch-count
    query runs the same configuration check as every compute call)."""
    cfg = _cfg(M, impl=1)
    setattr(cfg, field, value)
    rc = M.raw_call("mla_decode_launches", ctypes.byref(cfg), 4, 1, 0)
    if ok:
        assert rc in (1, 2), rc
        assert M.mla_decode_workspace_bytes(cfg, 4, 1, 0) > 0
    else:
        assert rc == -2, rc
        assert M.mla_decode_workspace_bytes(cfg, 4, 1, 0) == 0


def test_rope_table_argument_checks(M):
    buf = (ctypes.c_float * 64)()
    assert M.raw_call("mla_rope_table", 16, ctypes.c_double(10000.0), 4, None) == -1
    for d_r, base, max_pos in ((15, 10000.0, 4), (0, 10000.0, 4), (16, 0.0, 4), (16, -2.0, 4),
                               (16, float("nan"), 4), (16, 10000.0, 0)):
        assert M.raw_call("mla_rope_table", d_r, ctypes.c_double(base), max_pos, buf) == -3, (d_r, base, max_pos)
    assert M.raw_call("mla_rope_table", 16, ctypes.c_double(10000.0), 4, buf) == 0
    # position 0 is the identity rotation: cos = 1, sin = 0 for every pair
    assert list(buf[:8]) == [1.0] * 8 and list(buf[8:16]) == [0.0] * 8


def test_yarn_table_and_scale_match_the_oracle(M):
    """The library's host-side YaRN table and score scale against the oracle's
    definitions.  The two sides use different libm implementations, so an
    entry may differ by one float ulp, or near zero by the rounding of a
    large angle (about 1e-11 absolute at positions near 1.4e5)."""
    from oracle import mla_oracle as O
    for d_r, max_pos in ((64, 140000), (16, 5000)):
        lib = M.mla_rope_table_yarn(d_r, 10000.0, max_pos).numpy()
        ref = O.rope_table_f32(max_pos, d_r, inv_freq=O.yarn_inv_freq(d_r))
        ulp = np.maximum(np.spacing(np.abs(ref).astype(np.float32)), 1e-9)
        assert np.all(np.abs(lib.astype(np.float64) - ref) <= ulp), d_r
        assert np.mean(lib != ref) < 1e-4
    # no stretch: the plain table
    np.testing.assert_array_equal(M.mla_rope_table_yarn(64, 10000.0, 64, 1.0).numpy(),
                                  M.mla_rope_table(64, 10000.0, 64).numpy())
    assert abs(M.mla_yarn_score_scale(128, 64) - O.yarn_score_scale(128, 64)) < 1e-7
    assert abs(M.mla_yarn_score_scale(128, 64, 40.0, 0.1) - O.yarn_score_scale(128, 64, 40.0, 0.1)) < 1e-7
    buf = (ctypes.c_float * 64)()
    assert M.raw_call("mla_rope_table_yarn", 16, ctypes.c_double(10000.0), 4, ctypes.c_double(0.5),
                      ctypes.c_double(1.0), ctypes.c_double(32.0), 4096, buf) == -3      # s < 1
    assert M.raw_call("mla_rope_table_yarn", 16, ctypes.c_double(10000.0), 4, ctypes.c_double(40.0),
                      ctypes.c_double(32.0), ctypes.c_double(1.0), 4096, buf) == -3      # beta <= alpha
    with pytest.raises(M.MlaError):
        M.mla_yarn_score_scale(128, 64, 0.5)


def test_e4m3_row_bytes_match_the_oracle_layout(M):
    from oracle import lowbit_cache as LB
    for d_c in (64, 128, 192, 256, 512):
        for d_r in (8, 16, 32, 64):
            assert M.mla_e4m3_row_bytes(d_c, d_r) == LB.row_layout(d_c, d_r)[2], (d_c, d_r)
    for d_c, d_r in ((0, 64), (100, 64), (576, 64), (512, 0), (512, 12), (512, 72)):
        assert M.mla_e4m3_row_bytes(d_c, d_r) == 0, (d_c, d_r)


def test_e4m3_host_validation(M):
    raw = M.raw_call
    cfg = _cfg(M)
    p = ctypes.c_void_p(FAKE)

    def append(c=cfg, q_r=p, k_r=p, c_kv=p, pos=p, table=p, max_pos=4096, bt=p, mbps=64,
               pool=p, num_blocks=2048, B=32, T_q=1, status=None):
        return raw("mla_rope_append_e4m3", ctypes.byref(c), q_r, k_r, c_kv, pos, table, max_pos, bt, mbps,
                   pool, num_blocks, B, T_q, status, None)

    def decode(c=cfg, q_abs=p, q_r=p, pool=p, num_blocks=2048, bt=p, mbps=64, lens=p, B=32, T_q=1,
               max_splits=0, ws=p, ws_bytes=1 << 30, out=p, lse=p):
        return raw("mla_decode_e4m3", ctypes.byref(c), q_abs, q_r, pool, num_blocks, bt, mbps, lens, B, T_q,
                   max_splits, ws, ctypes.c_size_t(ws_bytes), out, lse, None)

    assert append(c=_cfg(M, d_c=96)) == -2 and decode(c=_cfg(M, d_c=96)) == -2   # not whole 64-column groups
    assert decode(c=_cfg(M, impl=2)) == -2                                        # portable kernels only
    for name in ("k_r", "c_kv", "pos", "table", "bt", "pool"):
        assert append(**{name: None}) == -1, name
    for name in ("q_abs", "q_r", "pool", "bt", "lens", "ws", "out", "lse"):
        assert decode(**{name: None}) == -1, name
    odd16 = ctypes.c_void_p(FAKE + 8)
    assert append(pool=odd16) == -7 and decode(pool=odd16) == -7 and decode(out=odd16) == -7
    assert append(B=0) == -3 and decode(B=0) == -3 and decode(B=65536) == -3
    assert decode(ws=ctypes.c_void_p(FAKE + 16)) == -4                            # not 256-byte aligned
    need = M.mla_decode_e4m3_workspace_bytes(cfg, 32, 1, 0)
    assert need > 0 and decode(ws_bytes=need - 1) == -4
    assert M.mla_decode_e4m3_workspace_bytes(_cfg(M, d_c=96), 32, 1, 0) == 0
    assert M.mla_decode_e4m3_workspace_bytes(_cfg(M, impl=2), 32, 1, 0) == 0
    # the portable kernel's split partials: splits x rows x (4 d_c + 4) bytes after the status word
    rows, splits = 32 * 128, 3
    r256 = lambda x: (x + 255) // 256 * 256
    assert M.mla_decode_e4m3_workspace_bytes(cfg, 32, 1, splits) == 256 + r256(splits * rows * 512 * 4) + \
        r256(splits * rows * 4)


def test_portable_split_choice(M):
    """The portable kernels' automatic split count: enough (token, 32-head
    group) CTAs for about 8 per SM, between 1 and 64 parts; visible through
    the workspace size of the e4m3 decode (splits x rows x (4 d_c + 4) bytes)."""
    r256 = lambda x: (x + 255) // 256 * 256

    def ws(n_h, d_c, B, T_q):
        rows = B * T_q * n_h
        work = B * T_q * ((n_h + 31) // 32)
        s = min(64, max(1, -(-8 * 148 // work)))
        return 256 + (r256(s * rows * d_c * 4) + r256(s * rows * 4) if s > 1 else 0)

    for n_h, d_c, B, T_q in ((128, 512, 32, 1), (128, 512, 1, 1), (4, 64, 1, 1), (128, 512, 64, 4),
                             (12, 128, 2, 1), (128, 512, 512, 4)):
        cfg = _cfg(M, n_h=n_h, d_c=d_c, d_r=64 if d_c == 512 else 16)
        assert M.mla_decode_e4m3_workspace_bytes(cfg, B, T_q, 0) == ws(n_h, d_c, B, T_q), (n_h, d_c, B, T_q)
