"""Device-side driver of one MLA decode step through the C ABI.

:class:`DeviceCase` allocates a workload's buffers with torch, fills the paged
latent cache with the history rows (through ``mla_rope_append``), and runs the
step ``mla_rope_append -> mla_absorb_q -> mla_decode -> mla_up_v``.  Used by
the GPU tests, the benchmark and the smoke check.
"""

from __future__ import annotations

import numpy as np
import torch

from . import binding as M
from . import synth
from .workloads import ROW_SHIFT, CaseSpec

NAN_BF16 = 0x7FC0


def _bits_to_dev(bits: np.ndarray, dev) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(dev).view(torch.bfloat16)


class DeviceCase:
    """Buffers and the step of one workload on one GPU."""

    def __init__(self, spec: CaseSpec, impl: int = M.IMPL_AUTO, max_splits: int = 0,
                 device: str = "cuda:0", rope_base: float = 10000.0, fill_history: bool = True,
                 yarn=None, cache: str = "bf16"):
        """yarn: None (plain RoPE, scale 1/sqrt(d_h + d_r)) or a dict of
        mla_rope_table_yarn / mla_yarn_score_scale arguments (s, alpha, beta,
        orig_len, coeff); the library builds the table and the scale.
        cache: "bf16" (rows of d_c + d_r bf16 values) or "e4m3" (the low-bit
        rows of mla_rope_append_e4m3 / mla_decode_e4m3)."""
        assert cache in ("bf16", "e4m3")
        self.cache = cache
        self.spec = spec
        self.dev = torch.device(device)
        self.impl = impl
        self.max_splits = max_splits
        s = spec
        self.yarn = dict(yarn) if yarn is not None else None
        scale = 0.0
        if self.yarn is not None:
            scale = M.mla_yarn_score_scale(s.d_h, s.d_r, self.yarn.get("s", 40.0), self.yarn.get("coeff", 0.0707))
        self.cfg = M.MlaConfig(s.n_h, s.d_c, s.d_h, s.d_r, s.block_size, scale, impl)
        dev = self.dev
        self.max_pos = int(np.max(s.seq_lens))
        if self.yarn is None:
            self.rope_table = M.mla_rope_table(s.d_r, rope_base, self.max_pos).to(dev)
        else:
            y = self.yarn
            self.rope_table = M.mla_rope_table_yarn(s.d_r, rope_base, self.max_pos, y.get("s", 40.0),
                                                    y.get("alpha", 1.0), y.get("beta", 32.0),
                                                    y.get("orig_len", 4096)).to(dev)
        self.block_table_np = s.block_table()
        self.block_table = torch.from_numpy(self.block_table_np).to(dev)
        self.seq_lens = torch.from_numpy(s.seq_lens.astype(np.int32)).to(dev)
        # Unwritten cache slots hold NaN so that any read past a sequence's end
        # shows (e4m3: NaN codes, scales and key values of 0x7F7F... bytes).
        if cache == "bf16":
            self.pool = torch.full((s.num_blocks, s.block_size, s.D), NAN_BF16, dtype=torch.int16,
                                   device=dev).view(torch.bfloat16)
        else:
            self.row_bytes = M.mla_e4m3_row_bytes(s.d_c, s.d_r)
            self.pool = torch.full((s.num_blocks, s.block_size, self.row_bytes), 0x7F, dtype=torch.uint8,
                                   device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.w_uk = _bits_to_dev(s.w_uk(), dev)
        self.w_uv = _bits_to_dev(s.w_uv(), dev)

        # step inputs (host copies kept for the end-to-end leg)
        self.h_q_c = s.q_c()
        self.h_q_r = s.q_r()
        pos = s.positions()
        self.h_positions = pos
        self.h_c_kv_new = np.concatenate([s.c_kv_rows(b, int(L) - s.T_q, int(L))
                                          for b, L in enumerate(s.seq_lens)])
        self.h_k_r_new = np.concatenate([s.k_r_rows(b, int(L) - s.T_q, int(L))
                                         for b, L in enumerate(s.seq_lens)])
        self.q_c = _bits_to_dev(self.h_q_c, dev)
        self.q_r_pre = _bits_to_dev(self.h_q_r, dev)
        self.q_r = self.q_r_pre.clone()
        self.c_kv_new = _bits_to_dev(self.h_c_kv_new, dev)
        self.k_r_new = _bits_to_dev(self.h_k_r_new, dev)
        self.positions = torch.from_numpy(pos).to(dev)

        n = s.n_tok
        self.q_abs = torch.empty((n, s.n_h, s.d_c), dtype=torch.bfloat16, device=dev)
        self.latent = torch.empty((n, s.n_h, s.d_c), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((n, s.n_h), dtype=torch.float32, device=dev)
        self.out = torch.empty((n, s.n_h, s.d_h), dtype=torch.bfloat16, device=dev)
        self.ws_bytes = (M.mla_decode_workspace_bytes(self.cfg, s.B, s.T_q, max_splits) if cache == "bf16" else
                         M.mla_decode_e4m3_workspace_bytes(self.cfg, s.B, s.T_q, max_splits))
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        if fill_history:
            self.fill_history()
        torch.cuda.synchronize(dev)

    # -- cache history ------------------------------------------------------

    def fill_history(self, chunk_rows: int = 1 << 16):
        """Append rows 0 .. L_b - T_q - 1 of every sequence (positions equal
        to row indices), drawing them on the device from the seeded stream."""
        s = self.spec
        for b, L in enumerate(s.seq_lens):
            hist = int(L) - s.T_q
            for j0 in range(0, hist, chunk_rows):
                j1 = min(hist, j0 + chunk_rows)
                base = (b << ROW_SHIFT) + j0
                c = synth.normal_bf16_torch(s.seed, synth.TID["c_kv"], (j1 - j0) * s.d_c,
                                            start=base * s.d_c, device=self.dev)
                k = synth.normal_bf16_torch(s.seed, synth.TID["k_r"], (j1 - j0) * s.d_r,
                                            start=base * s.d_r, device=self.dev)
                pos = torch.arange(j0, j1, dtype=torch.int32, device=self.dev)
                self._append()(self.cfg, None, k, c, pos, self.rope_table, self.max_pos,
                               self.block_table[b:b + 1], s.max_blocks, self.pool, s.num_blocks,
                               1, j1 - j0, self.status)

    def _append(self):
        return M.mla_rope_append if self.cache == "bf16" else M.mla_rope_append_e4m3

    # -- the step -------------------------------------------------------------

    def reset_step_inputs(self):
        """Restore the pre-RoPE query part (the step rotates it in place)."""
        self.q_r.copy_(self.q_r_pre)

    def step(self, stream=None):
        """One pass of the whole hot path for the batch.

        RoPE + append and the query absorption read disjoint inputs, so either
        may go first; the append goes first: the absorption's CTAs then start
        while it runs and fetch their weight tiles before they wait for it."""
        s = self.spec
        self.rope_append(stream)
        M.mla_absorb_q(self.cfg, self.q_c, self.w_uk, self.q_abs, s.n_tok, self.status, stream)
        self.decode_only(stream)
        M.mla_up_v(self.cfg, self.latent, self.w_uv, self.out, s.n_tok, self.status, stream)

    def rope_append(self, stream=None):
        """RoPE on q^R in place and the new cache rows appended."""
        s = self.spec
        self._append()(self.cfg, self.q_r, self.k_r_new, self.c_kv_new, self.positions,
                       self.rope_table, self.max_pos, self.block_table, s.max_blocks, self.pool,
                       s.num_blocks, s.B, s.T_q, self.status, stream)

    def decode_only(self, stream=None):
        s = self.spec
        decode = M.mla_decode if self.cache == "bf16" else M.mla_decode_e4m3
        decode(self.cfg, self.q_abs, self.q_r, self.pool, s.num_blocks, self.block_table,
               s.max_blocks, self.seq_lens, s.B, s.T_q, self.max_splits, self.ws,
               self.ws_bytes, self.latent, self.lse, stream)

    def decode_status(self) -> int:
        return M.mla_read_status(self.ws)

    def append_status(self) -> int:
        return M.mla_read_status(self.status)

    # -- readback helpers ----------------------------------------------------

    @staticmethod
    def bits(t: torch.Tensor) -> np.ndarray:
        return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
