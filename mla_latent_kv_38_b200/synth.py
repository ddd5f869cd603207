"""Seeded synthetic inputs for the MLA decode path.

This module only draws numbers. It holds none of the attention arithmetic, so
both the CUDA path (through the tests and the benchmark) and the fp64 oracle can
take their inputs from it without sharing any of the method.

Generator: a counter-based SplitMix64 stream (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014) keyed by
(seed, tensor id, element index), turned into standard normals with the
Box-Muller transform (Box and Muller, 1958). Every element is a pure function of
its key, so any slice of a tensor (one sequence of a long cache, say) can be
regenerated without drawing the rest.

Values are rounded to bfloat16 with round-to-nearest-even here, once, and both
sides receive the same 16-bit patterns.
"""

from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Tensor ids: fixed small integers so that a tensor's stream does not depend on
# which other tensors a caller draws.
TID = {
    "c_kv": 1,
    "k_r": 2,
    "q_c": 3,
    "q_r": 4,
    "w_uk": 5,
    "w_uv": 6,
    "seq_lens": 7,
    "block_perm": 8,
    "c_q": 9,
    "w_uq": 10,
    "w_o": 11,
}


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, tid: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k = _mix(np.array([np.uint64(seed) * _GOLDEN + np.uint64(tid)], dtype=np.uint64))
        return _mix(k + _GOLDEN)[0]


def uniform_u64(seed: int, tid: int, index: np.ndarray) -> np.ndarray:
    """SplitMix64 output for counters `index` (uint64) of stream (seed, tid)."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(_key(seed, tid) + (idx + np.uint64(1)) * _GOLDEN)


def _unit(u: np.ndarray) -> np.ndarray:
    # top 53 bits -> (0, 1]
    return ((u >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)


def normal_f64(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    """Standard normals for flat element indices [start, start+count)."""
    i = np.arange(start, start + count, dtype=np.uint64)
    u1 = _unit(uniform_u64(seed, tid, np.uint64(2) * i))
    u2 = _unit(uniform_u64(seed, tid, np.uint64(2) * i + np.uint64(1)))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (round to nearest, ties to even); uint16 bits.

    The float64 significand is rounded directly to 8 significant bits; going
    through float32 first would round twice.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    # bf16 keeps 8 significant bits (7 stored). Round the float64 at bit 45
    # (52 - 7 fraction bits), ties to even, then re-encode through float32.
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    rounded = b + np.uint64(0x0000_0FFF_FFFF_FFFF) + lsb
    rounded &= ~np.uint64(0x0000_1FFF_FFFF_FFFF)
    r = rounded.view(np.float64)
    f = r.astype(np.float32)  # exact: r has at most 8 significant bits
    out = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def normal_bf16(seed: int, tid: int, shape, std: float = 1.0, start: int = 0) -> np.ndarray:
    """bf16 bit patterns of N(0, std^2) draws for a tensor of `shape` (flat order)."""
    n = int(np.prod(shape))
    return to_bf16_bits(std * normal_f64(seed, tid, start, n)).reshape(shape)


def seq_lens_uniform(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    """B integer lengths uniform in [lo, hi] (inclusive)."""
    u = uniform_u64(seed, TID["seq_lens"], np.arange(B, dtype=np.uint64))
    span = np.uint64(hi - lo + 1)
    return (lo + (u % span).astype(np.int64)).astype(np.int32)


def permutation(seed: int, n: int) -> np.ndarray:
    """A seeded permutation of range(n) (sort by SplitMix64 keys)."""
    u = uniform_u64(seed, TID["block_perm"], np.arange(n, dtype=np.uint64))
    return np.argsort(u, kind="stable").astype(np.int32)


def weight_std(fan_in: int) -> float:
    """Standard deviation 1/sqrt(fan_in) for the up-projection weights."""
    return 1.0 / float(np.sqrt(fan_in))


# ---------------------------------------------------------------------------
# The same generator evaluated with torch on a CUDA device, for bulk inputs.
# Integer steps use int64 with wrapping multiplication (the same bits as the
# unsigned arithmetic above) and masked shifts for the logical right shifts.
# ---------------------------------------------------------------------------

def _i64(v: int) -> int:
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def _torch_mix(z):
    import torch

    def shr(x, k):
        return (x >> k) & ((1 << (64 - k)) - 1)

    z = (z ^ shr(z, 30)) * _i64(int(_M1))
    z = (z ^ shr(z, 27)) * _i64(int(_M2))
    return z ^ shr(z, 31)


def normal_bf16_torch(seed: int, tid: int, count: int, start: int = 0, std: float = 1.0,
                      device="cuda", chunk: int = 1 << 24):
    """bf16 tensor of `count` draws for flat indices [start, start+count); the
    same values as :func:`normal_bf16` up to the last bit of the float64
    log/cos, which bf16 rounding hides except with probability ~2^-44."""
    import torch

    key = _i64(int(_key(seed, tid)))
    golden = _i64(int(_GOLDEN))
    out = torch.empty(count, dtype=torch.bfloat16, device=device)
    for c0 in range(0, count, chunk):
        n = min(chunk, count - c0)
        i = torch.arange(start + c0, start + c0 + n, dtype=torch.int64, device=device)
        u1 = _torch_mix(key + (2 * i + 1) * golden)
        u2 = _torch_mix(key + (2 * i + 2) * golden)
        f1 = ((u1 >> 11) & ((1 << 53) - 1)).to(torch.float64).add_(1.0).mul_(1.0 / 9007199254740992.0)
        f2 = ((u2 >> 11) & ((1 << 53) - 1)).to(torch.float64).add_(1.0).mul_(1.0 / 9007199254740992.0)
        z = torch.sqrt(-2.0 * torch.log(f1)) * torch.cos((2.0 * np.pi) * f2) * std
        out[c0:c0 + n] = _torch_f64_to_bf16(z)
    return out


def _torch_f64_to_bf16(z):
    """float64 -> bf16 with one rounding (round half to even on the float64
    significand), matching :func:`to_bf16_bits`."""
    import torch

    b = z.view(torch.int64)
    lsb = (b >> 45) & 1
    r = (b + ((1 << 44) - 1) + lsb) & ~((1 << 45) - 1)
    f = r.view(torch.float64).to(torch.float32)  # exact
    return f.to(torch.bfloat16)                  # exact
