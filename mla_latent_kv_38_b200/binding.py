"""Python binding of the B200 MLA latent-KV decode library (libmla_b200.so).

Argument marshalling only: every step runs in the library's CUDA kernels.  The
functions carry the C ABI's names (see include/mla.h) and take torch CUDA
tensors (bf16 tensors for the mla_bf16 arguments, int32 / float32 otherwise);
the stream defaults to torch's current stream.  A non-zero return code raises
:class:`MlaError`.  Importing this module without the built library raises
immediately: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MLA_B200_LIB") or os.path.join(_HERE, "libmla_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing; build it with `python -m mla_latent_kv_38_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

EXPORTED = (
    "mla_status_str", "mla_check_device", "mla_rope_table", "mla_rope_table_yarn",
    "mla_yarn_score_scale", "mla_absorb_q",
    "mla_rope_append", "mla_decode_workspace_bytes", "mla_decode", "mla_decode_launches",
    "mla_decode_noalloc", "mla_decode_split_counts", "mla_test_arm_decode_timeout", "mla_up_v",
    "mla_fold_weights", "mla_absorb_q_folded", "mla_up_o_folded_workspace_bytes", "mla_up_o_folded",
    "mla_e4m3_row_bytes", "mla_rope_append_e4m3", "mla_decode_e4m3_workspace_bytes", "mla_decode_e4m3",
    "mla_clear_status", "mla_read_status",
)

MLA_ERR_SIZE = -3
MLA_STATUS_BAD_POSITION = 1
MLA_STATUS_BAD_BLOCK = 2
MLA_STATUS_BAD_SEQ_LEN = 4
MLA_STATUS_TIMEOUT = 8

IMPL_AUTO, IMPL_SIMT, IMPL_TCGEN05 = 0, 1, 2


class MlaConfig(ctypes.Structure):
    """Mirror of ``mla_config_t``."""

    _fields_ = [
        ("n_h", ctypes.c_int),
        ("d_c", ctypes.c_int),
        ("d_h", ctypes.c_int),
        ("d_r", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("impl", ctypes.c_int),
    ]

    def __init__(self, n_h, d_c, d_h, d_r, block_size=64, scale=0.0, impl=IMPL_AUTO):
        super().__init__(n_h, d_c, d_h, d_r, block_size, scale, impl)


class MlaError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {code} ({mla_status_str(code)})")
        self.code = code


_vp, _i, _sz, _cfgp = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.POINTER(MlaConfig)
_lib.mla_status_str.restype = ctypes.c_char_p
_lib.mla_status_str.argtypes = [_i]
_lib.mla_check_device.argtypes = []
_lib.mla_rope_table.argtypes = [_i, ctypes.c_double, _i, _vp]
_lib.mla_rope_table_yarn.argtypes = [_i, ctypes.c_double, _i, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                     _i, _vp]
_lib.mla_yarn_score_scale.restype = ctypes.c_float
_lib.mla_yarn_score_scale.argtypes = [_i, _i, ctypes.c_double, ctypes.c_double]
_lib.mla_absorb_q.argtypes = [_cfgp, _vp, _vp, _vp, _i, _vp, _vp]
_lib.mla_rope_append.argtypes = [_cfgp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp, _vp]
_lib.mla_decode_workspace_bytes.restype = _sz
_lib.mla_decode_workspace_bytes.argtypes = [_cfgp, _i, _i, _i]
_lib.mla_decode.argtypes = [_cfgp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp, _sz, _vp, _vp, _vp]
_lib.mla_decode_launches.argtypes = [_cfgp, _i, _i, _i]
_lib.mla_decode_noalloc.argtypes = [_cfgp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp, _vp, _vp,
                                    _vp]
_lib.mla_decode_split_counts.argtypes = [_cfgp, _i, _i, _i, _vp, _vp, _i, _vp]
_lib.mla_test_arm_decode_timeout.argtypes = [ctypes.c_uint64]
_lib.mla_up_v.argtypes = [_cfgp, _vp, _vp, _vp, _i, _vp, _vp]
_lib.mla_fold_weights.argtypes = [_cfgp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.mla_absorb_q_folded.argtypes = [_cfgp, _i, _vp, _vp, _vp, _i, _vp, _vp]
_lib.mla_up_o_folded_workspace_bytes.restype = _sz
_lib.mla_up_o_folded_workspace_bytes.argtypes = [_cfgp, _i, _i]
_lib.mla_up_o_folded.argtypes = [_cfgp, _i, _vp, _vp, _vp, _i, _vp, _sz, _vp, _vp]
_lib.mla_e4m3_row_bytes.restype = _sz
_lib.mla_e4m3_row_bytes.argtypes = [_i, _i]
_lib.mla_rope_append_e4m3.argtypes = [_cfgp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp, _vp]
_lib.mla_decode_e4m3_workspace_bytes.restype = _sz
_lib.mla_decode_e4m3_workspace_bytes.argtypes = [_cfgp, _i, _i, _i]
_lib.mla_decode_e4m3.argtypes = [_cfgp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp, _sz, _vp, _vp, _vp]
_lib.mla_clear_status.argtypes = [_vp, _vp]
_lib.mla_read_status.argtypes = [_vp, _vp, _vp]


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn, rc):
    if rc != 0:
        raise MlaError(fn, rc)


def mla_status_str(code: int) -> str:
    return _lib.mla_status_str(int(code)).decode()


def mla_check_device() -> int:
    return _lib.mla_check_device()


def mla_rope_table(d_r: int, base: float, max_pos: int) -> torch.Tensor:
    """Host float32 table (max_pos, d_r) built by the library (cos | sin)."""
    out = torch.empty((max_pos, d_r), dtype=torch.float32)
    _check("mla_rope_table", _lib.mla_rope_table(d_r, float(base), max_pos, out.data_ptr()))
    return out


def mla_rope_table_yarn(d_r: int, base: float, max_pos: int, s: float = 40.0, alpha: float = 1.0,
                        beta: float = 32.0, orig_len: int = 4096) -> torch.Tensor:
    """Host float32 YaRN table (max_pos, d_r) built by the library (cos | sin)."""
    out = torch.empty((max_pos, d_r), dtype=torch.float32)
    _check("mla_rope_table_yarn", _lib.mla_rope_table_yarn(d_r, float(base), max_pos, float(s), float(alpha),
                                                           float(beta), int(orig_len), out.data_ptr()))
    return out


def mla_yarn_score_scale(d_h: int, d_r: int, s: float = 40.0, coeff: float = 0.0707) -> float:
    v = float(_lib.mla_yarn_score_scale(int(d_h), int(d_r), float(s), float(coeff)))
    if v <= 0.0:
        raise MlaError("mla_yarn_score_scale", MLA_ERR_SIZE)
    return v


def mla_absorb_q(cfg: MlaConfig, q_c, w_uk, q_abs, n_tok: int, dev_status=None, stream=None):
    _check("mla_absorb_q", _lib.mla_absorb_q(ctypes.byref(cfg), _ptr(q_c), _ptr(w_uk), _ptr(q_abs),
                                             int(n_tok), _ptr(dev_status), _stream(stream)))


def mla_rope_append(cfg: MlaConfig, q_r, k_r, c_kv, positions, rope_table, max_pos: int,
                    block_table, max_blocks_per_seq: int, pool, num_blocks: int, B: int, T_q: int,
                    dev_status=None, stream=None):
    _check("mla_rope_append", _lib.mla_rope_append(
        ctypes.byref(cfg), _ptr(q_r), _ptr(k_r), _ptr(c_kv), _ptr(positions), _ptr(rope_table),
        int(max_pos), _ptr(block_table), int(max_blocks_per_seq), _ptr(pool), int(num_blocks),
        int(B), int(T_q), _ptr(dev_status), _stream(stream)))


def mla_decode_workspace_bytes(cfg: MlaConfig, B: int, T_q: int, max_splits: int = 0) -> int:
    return int(_lib.mla_decode_workspace_bytes(ctypes.byref(cfg), int(B), int(T_q), int(max_splits)))


def mla_decode(cfg: MlaConfig, q_abs, q_r, pool, num_blocks: int, block_table,
               max_blocks_per_seq: int, seq_lens, B: int, T_q: int, max_splits: int,
               workspace, ws_bytes: int, out_latent, out_lse, stream=None):
    _check("mla_decode", _lib.mla_decode(
        ctypes.byref(cfg), _ptr(q_abs), _ptr(q_r), _ptr(pool), int(num_blocks), _ptr(block_table),
        int(max_blocks_per_seq), _ptr(seq_lens), int(B), int(T_q), int(max_splits), _ptr(workspace),
        int(ws_bytes), _ptr(out_latent), _ptr(out_lse), _stream(stream)))


def mla_decode_launches(cfg: MlaConfig, B: int, T_q: int, max_splits: int = 0) -> int:
    n = _lib.mla_decode_launches(ctypes.byref(cfg), int(B), int(T_q), int(max_splits))
    if n < 0:
        raise MlaError("mla_decode_launches", n)
    return n


def mla_decode_noalloc(cfg: MlaConfig, q_abs, q_r, pool, num_blocks: int, block_table,
                       max_blocks_per_seq: int, seq_lens, B: int, T_q: int, splits: int,
                       out_latent, out_lse, dev_status=None, stream=None):
    """mla_decode without a workspace, for callers that cannot allocate: the
    split partials live in the library's fixed 16 MiB device array."""
    _check("mla_decode_noalloc", _lib.mla_decode_noalloc(
        ctypes.byref(cfg), _ptr(q_abs), _ptr(q_r), _ptr(pool), int(num_blocks), _ptr(block_table),
        int(max_blocks_per_seq), _ptr(seq_lens), int(B), int(T_q), int(splits), _ptr(out_latent),
        _ptr(out_lse), _ptr(dev_status), _stream(stream)))


def mla_decode_split_counts(cfg: MlaConfig, B: int, T_q: int, max_splits: int, workspace, n_counts: int,
                            stream=None):
    """Parts per unit of work of the last completed mla_decode call (host int32 tensor)."""
    out = torch.zeros(n_counts, dtype=torch.int32)
    _check("mla_decode_split_counts", _lib.mla_decode_split_counts(
        ctypes.byref(cfg), int(B), int(T_q), int(max_splits), _ptr(workspace), out.data_ptr(), int(n_counts),
        _stream(stream)))
    return out


def mla_test_arm_decode_timeout(wait_limit_ns: int):
    """Test hook: the next tensor-core mla_decode call withholds one load and
    bounds its waits by wait_limit_ns (it then reports MLA_STATUS_TIMEOUT)."""
    _check("mla_test_arm_decode_timeout", _lib.mla_test_arm_decode_timeout(int(wait_limit_ns)))


def mla_up_v(cfg: MlaConfig, latent, w_uv, out, n_tok: int, dev_status=None, stream=None):
    _check("mla_up_v", _lib.mla_up_v(ctypes.byref(cfg), _ptr(latent), _ptr(w_uv), _ptr(out),
                                     int(n_tok), _ptr(dev_status), _stream(stream)))


def mla_fold_weights(cfg: MlaConfig, d_cq: int, d_model: int, w_uq, w_uk, w_uv, w_o, w_fold_q, w_fold_o,
                     stream=None):
    _check("mla_fold_weights", _lib.mla_fold_weights(
        ctypes.byref(cfg), int(d_cq), int(d_model), _ptr(w_uq), _ptr(w_uk), _ptr(w_uv), _ptr(w_o),
        _ptr(w_fold_q), _ptr(w_fold_o), _stream(stream)))


def mla_absorb_q_folded(cfg: MlaConfig, d_cq: int, c_q, w_fold_q, q_abs, n_tok: int, dev_status=None,
                        stream=None):
    _check("mla_absorb_q_folded", _lib.mla_absorb_q_folded(
        ctypes.byref(cfg), int(d_cq), _ptr(c_q), _ptr(w_fold_q), _ptr(q_abs), int(n_tok), _ptr(dev_status),
        _stream(stream)))


def mla_up_o_folded_workspace_bytes(cfg: MlaConfig, d_model: int, n_tok: int) -> int:
    return int(_lib.mla_up_o_folded_workspace_bytes(ctypes.byref(cfg), int(d_model), int(n_tok)))


def mla_up_o_folded(cfg: MlaConfig, d_model: int, latent, w_fold_o, u, n_tok: int, workspace, dev_status=None,
                    stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("mla_up_o_folded", _lib.mla_up_o_folded(
        ctypes.byref(cfg), int(d_model), _ptr(latent), _ptr(w_fold_o), _ptr(u), int(n_tok), _ptr(workspace),
        ws_bytes, _ptr(dev_status), _stream(stream)))


def mla_e4m3_row_bytes(d_c: int, d_r: int) -> int:
    return int(_lib.mla_e4m3_row_bytes(int(d_c), int(d_r)))


def mla_rope_append_e4m3(cfg: MlaConfig, q_r, k_r, c_kv, positions, rope_table, max_pos: int,
                         block_table, max_blocks_per_seq: int, pool, num_blocks: int, B: int, T_q: int,
                         dev_status=None, stream=None):
    _check("mla_rope_append_e4m3", _lib.mla_rope_append_e4m3(
        ctypes.byref(cfg), _ptr(q_r), _ptr(k_r), _ptr(c_kv), _ptr(positions), _ptr(rope_table),
        int(max_pos), _ptr(block_table), int(max_blocks_per_seq), _ptr(pool), int(num_blocks),
        int(B), int(T_q), _ptr(dev_status), _stream(stream)))


def mla_decode_e4m3_workspace_bytes(cfg: MlaConfig, B: int, T_q: int, max_splits: int = 0) -> int:
    return int(_lib.mla_decode_e4m3_workspace_bytes(ctypes.byref(cfg), int(B), int(T_q), int(max_splits)))


def mla_decode_e4m3(cfg: MlaConfig, q_abs, q_r, pool, num_blocks: int, block_table,
                    max_blocks_per_seq: int, seq_lens, B: int, T_q: int, max_splits: int,
                    workspace, ws_bytes: int, out_latent, out_lse, stream=None):
    _check("mla_decode_e4m3", _lib.mla_decode_e4m3(
        ctypes.byref(cfg), _ptr(q_abs), _ptr(q_r), _ptr(pool), int(num_blocks), _ptr(block_table),
        int(max_blocks_per_seq), _ptr(seq_lens), int(B), int(T_q), int(max_splits), _ptr(workspace),
        int(ws_bytes), _ptr(out_latent), _ptr(out_lse), _stream(stream)))


def mla_clear_status(dev_status, stream=None):
    _check("mla_clear_status", _lib.mla_clear_status(_ptr(dev_status), _stream(stream)))


def mla_read_status(dev_status, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check("mla_read_status", _lib.mla_read_status(_ptr(dev_status), ctypes.addressof(out),
                                                   _stream(stream)))
    return int(out.value)


def raw_call(name: str, *args) -> int:
    """Call an exported function with raw ctypes arguments; returns its code."""
    return getattr(_lib, name)(*args)
