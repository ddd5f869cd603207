"""Workload definitions: head shapes, cache lengths, block tables and seeded
inputs of an MLA decode batch.

A case is a batch of sequences with their cache lengths (after the step's
append), the head shapes, and a seed.  Inputs come from the seeded generator in
``synth``; the oracle (in the tests) and the CUDA path each take them from
there, never from each other.  Nothing here computes any part of the method.

Element streams are keyed by (sequence, token) so that one sequence's inputs
can be regenerated alone: cache row j of sequence b uses counter base
``(b << 20) + j``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from mla_latent_kv_38_b200 import synth

ROW_SHIFT = 20  # supports cache lengths up to 2^20 per sequence


@dataclass
class CaseSpec:
    n_h: int
    d_c: int
    d_h: int
    d_r: int
    seq_lens: np.ndarray            # (B,) cache length after the append
    T_q: int = 1
    seed: int = 0
    permute_blocks: bool = False
    block_size: int = 64
    name: str = ""
    d_cq: int = 1536                # query latent (W^UQ's input), DeepSeek-V2
    d_model: int = 5120             # model width (W^O's output), DeepSeek-V2

    @property
    def B(self):
        return int(len(self.seq_lens))

    @property
    def n_tok(self):
        return self.B * self.T_q

    @property
    def D(self):
        return self.d_c + self.d_r

    def blocks_per_seq(self):
        return [(int(L) + self.block_size - 1) // self.block_size for L in self.seq_lens]

    @property
    def max_blocks(self):
        return max(self.blocks_per_seq())

    @property
    def num_blocks(self):
        return int(sum(self.blocks_per_seq()))

    def block_table(self) -> np.ndarray:
        """(B, max_blocks) int32; physical blocks in order, or a seeded
        permutation of all blocks.  Unused entries hold -1."""
        nb = self.blocks_per_seq()
        phys = np.arange(self.num_blocks, dtype=np.int32)
        if self.permute_blocks:
            phys = synth.permutation(self.seed, self.num_blocks)
        t = np.full((self.B, self.max_blocks), -1, dtype=np.int32)
        k = 0
        for b, n in enumerate(nb):
            t[b, :n] = phys[k:k + n]
            k += n
        return t

    # ---- seeded inputs (bf16 bit patterns) -------------------------------

    def _rows(self, tid, b, j0, j1, width, std=1.0):
        base = (b << ROW_SHIFT) + j0
        return synth.normal_bf16(self.seed, tid, (j1 - j0, width), std=std, start=base * width)

    def c_kv_rows(self, b, j0, j1):
        return self._rows(synth.TID["c_kv"], b, j0, j1, self.d_c)

    def k_r_rows(self, b, j0, j1):
        """Pre-RoPE shared keys of tokens j0..j1-1 of sequence b."""
        return self._rows(synth.TID["k_r"], b, j0, j1, self.d_r)

    def q_c(self):
        return synth.normal_bf16(self.seed, synth.TID["q_c"], (self.n_tok, self.n_h, self.d_h))

    def q_r(self):
        """Pre-RoPE per-head query RoPE parts."""
        return synth.normal_bf16(self.seed, synth.TID["q_r"], (self.n_tok, self.n_h, self.d_r))

    def w_uk(self):
        return synth.normal_bf16(self.seed, synth.TID["w_uk"], (self.n_h, self.d_h, self.d_c),
                                 std=synth.weight_std(self.d_c))

    def c_q(self):
        """Query latents c^Q (the input of W^UQ), one per token."""
        return synth.normal_bf16(self.seed, synth.TID["c_q"], (self.n_tok, self.d_cq))

    def w_uq(self):
        return synth.normal_bf16(self.seed, synth.TID["w_uq"], (self.n_h, self.d_h, self.d_cq),
                                 std=synth.weight_std(self.d_cq))

    def w_o(self):
        return synth.normal_bf16(self.seed, synth.TID["w_o"], (self.d_model, self.n_h, self.d_h),
                                 std=synth.weight_std(self.n_h * self.d_h))

    def w_uv(self):
        return synth.normal_bf16(self.seed, synth.TID["w_uv"], (self.n_h, self.d_h, self.d_c),
                                 std=synth.weight_std(self.d_c))

    def positions(self):
        return np.concatenate([np.arange(L - self.T_q, L, dtype=np.int32) for L in self.seq_lens])

    # ---- accounting -------------------------------------------------------

    def visible_keys(self):
        return sum(int(L) - self.T_q + t + 1 for L in self.seq_lens for t in range(self.T_q))

    def algorithmic_bytes(self, row_bytes=None):
        """Cache read once + q (bf16) + latent out (bf16) + lse (fp32); a cache
        row is D bf16 values unless row_bytes says otherwise (the e4m3 rows)."""
        cache = int(np.sum(self.seq_lens)) * (self.D * 2 if row_bytes is None else int(row_bytes))
        q = self.n_tok * self.n_h * self.D * 2
        out = self.n_tok * self.n_h * (self.d_c * 2 + 4)
        return cache + q + out

    def algorithmic_flops(self):
        """2*(d_c+d_r) for the score and 2*d_c for the weighted sum, per
        (query token, head, visible key)."""
        return self.n_h * self.visible_keys() * (2 * self.D + 2 * self.d_c)


def config_specs():
    """The five workloads: shapes, lengths and structure as the pages give them."""
    v2 = dict(n_h=128, d_c=512, d_h=128, d_r=64)
    return {
        "tiny": CaseSpec(n_h=4, d_c=64, d_h=32, d_r=16, seq_lens=np.array([128], np.int32),
                         name="tiny B=1 n_h=4 d_c=64 d_h=32 d_r=16 L=128"),
        "v2_decode": CaseSpec(**v2, seq_lens=np.full(32, 4096, np.int32),
                              name="DeepSeek-V2 decode B=32 L=4096"),
        "varlen": CaseSpec(**v2, seq_lens=synth.seq_lens_uniform(0, 128, 512, 32768),
                           permute_blocks=True,
                           name="var-len B=128 L~U[512,32768] permuted blocks"),
        "long": CaseSpec(**v2, seq_lens=np.full(4, 131072, np.int32),
                         name="long context B=4 L=131072"),
        "multi_token": CaseSpec(**v2, seq_lens=np.full(64, 8192, np.int32), T_q=4,
                                name="multi-token B=64 T_q=4 L=8192"),
    }


def prefill_specs():
    """Chunked prefill on the same paged cache (the decode call with T_q new
    tokens per sequence under the generalised causal mask): a 512-token chunk
    appended to a 3,584-token prefix, and prefill of 2,048 tokens from an empty
    cache.  DeepSeek-V2 head shapes."""
    v2 = dict(n_h=128, d_c=512, d_h=128, d_r=64)
    return {
        "prefill_chunk": CaseSpec(**v2, seq_lens=np.full(4, 4096, np.int32), T_q=512,
                                  name="chunked prefill B=4 chunk 512 L=4096"),
        "prefill": CaseSpec(**v2, seq_lens=np.full(1, 2048, np.int32), T_q=2048,
                            name="prefill B=1 T=2048 from an empty cache"),
    }


def workload_specs():
    """Every named workload: the five decode configurations and the prefill ones."""
    out = config_specs()
    out.update(prefill_specs())
    return out

