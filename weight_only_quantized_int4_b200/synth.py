"""Seeded synthetic inputs: activations, fp32 weights and lookup tables.

This module only draws random numbers and casts them to the input dtypes.  It
holds no step of the quantized matmul (no scale, zero-point, code or decode
arithmetic), so the CPU oracle and the CUDA path can both be fed from it.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used as a counter-based generator -- value i
of a stream is mix(key + (i + 1) * gamma) -- so any element of a matrix can be
produced without producing the ones before it.  Normal deviates come from the
Box-Muller transform over the pair of uniforms (2j, 2j + 1): element 2j takes
the cosine branch and element 2j + 1 the sine branch.
"""
from __future__ import annotations

import math
import zlib

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: str) -> np.uint64:
    """Key of a named sub-stream: mix(seed * 2^32 + crc32(stream))."""
    base = np.array([((seed & 0xFFFFFFFF) << 32) | zlib.crc32(stream.encode())],
                    dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(base)[0]


def uniform(seed: int, stream: str, index: np.ndarray) -> np.ndarray:
    """Uniform doubles in [0, 1) for the given counter values (53-bit)."""
    key = stream_key(seed, stream)
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(key + (idx + np.uint64(1)) * _GAMMA)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_at(seed: int, stream: str, index: np.ndarray) -> np.ndarray:
    """Standard normal deviates for element indices `index` (float64)."""
    idx = np.asarray(index, dtype=np.uint64)
    pair = idx & ~np.uint64(1)
    u1 = 1.0 - uniform(seed, stream, pair)          # (0, 1]
    u2 = uniform(seed, stream, pair + np.uint64(1))
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * math.pi * u2
    odd = (idx & np.uint64(1)).astype(bool)
    return np.where(odd, r * np.sin(ang), r * np.cos(ang))


def normal_rows(seed: int, stream: str, n_rows: int, n_cols: int,
                rows=None, chunk_elems: int = 1 << 24) -> np.ndarray:
    """Rows of an [n_rows, n_cols] standard-normal matrix (float64).

    Element (n, k) is stream element n * n_cols + k, so a subset of rows is the
    same numbers the full matrix holds at those rows.
    """
    rows = np.arange(n_rows) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), n_cols), dtype=np.float64)
    per = max(1, chunk_elems // max(1, n_cols))
    cols = np.arange(n_cols, dtype=np.uint64)
    for s in range(0, len(rows), per):
        r = rows[s:s + per].astype(np.uint64)
        idx = r[:, None] * np.uint64(n_cols) + cols[None, :]
        out[s:s + per] = normal_at(seed, stream, idx)
    return out


def weights(seed: int, stream: str, N: int, K: int, sigma: float, rows=None) -> np.ndarray:
    """fp32 weights W[N, K] ~ N(0, sigma^2) (rows subset optional)."""
    return (sigma * normal_rows(seed, stream, N, K, rows)).astype(np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    nan = (b & 0x7FFFFFFF) > 0x7F800000
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return np.where(nan, np.uint16(0x7FC0), r)


def activations(seed: int, stream: str, M: int, K: int, dtype: str) -> np.ndarray:
    """x[M, K] ~ N(0, 1) as uint16 bit patterns of fp16 or bf16."""
    z = normal_rows(seed, stream, M, K)
    if dtype == "f16":
        return z.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        return to_bf16_bits(z.astype(np.float32))
    raise ValueError(dtype)


def _norm_ppf(p: float) -> float:
    """Inverse standard normal CDF by bisection on Phi(x) = erfc(-x/sqrt2)/2."""
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * math.erfc(-mid / math.sqrt(2.0)) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def nf_table(bits: int) -> np.ndarray:
    """2^bits-entry normal-quantile table over [-1, 1] as fp16 bits.

    T[i] = q((i + 0.5) / 2^bits) / q((2^bits - 0.5) / 2^bits) with q the standard
    normal quantile: symmetric, ascending, endpoints exactly -1 and 1.
    """
    n = 1 << bits
    top = _norm_ppf((n - 0.5) / n)
    t = np.array([_norm_ppf((i + 0.5) / n) / top for i in range(n)])
    return t.astype(np.float16).view(np.uint16)


def nf4_table() -> np.ndarray:
    """The 16-entry NF4-style table (nf_table(4))."""
    return nf_table(4)


def nf3_table() -> np.ndarray:
    """The 8-entry NF3-style table (nf_table(3))."""
    return nf_table(3)


def lut2_table(seed: int = 0) -> np.ndarray:
    """4-entry seeded table: 4 N(0,1) draws / max|.|, sorted, fp16 bits."""
    v = normal_at(seed, "lut2", np.arange(4, dtype=np.uint64))
    v = np.sort(v / np.max(np.abs(v)))
    return v.astype(np.float16).view(np.uint16)


# ------------------------------------------------------------------ torch twin
#
# The same generator written with torch int64 tensors, for inputs too large to
# draw on the host (the benchmark's weights): uint64 wrapping arithmetic on
# two's-complement int64, logical right shifts by masking.  The uniforms match
# the numpy functions above bit for bit; the Box-Muller step runs in the
# device's float64 log / sqrt / sin / cos, whose last bits may differ from the
# host's, so the normal deviates agree to a few ulps of float64.

def _i64(u: int) -> int:
    """uint64 constant as the int64 with the same bits."""
    return u - (1 << 64) if u >= (1 << 63) else u


_T_GAMMA = _i64(0x9E3779B97F4A7C15)
_T_M1 = _i64(0xBF58476D1CE4E5B9)
_T_M2 = _i64(0x94D049BB133111EB)


def _srl(z, k: int):
    """Logical right shift of an int64 tensor holding uint64 bits."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix_t(z):
    z = (z ^ _srl(z, 30)) * _T_M1
    z = (z ^ _srl(z, 27)) * _T_M2
    return z ^ _srl(z, 31)


def weights_torch(seed: int, stream: str, N: int, K: int, sigma: float, device="cpu"):
    """weights() as an fp32 torch tensor on `device`."""
    import torch

    W = torch.empty(N, K, dtype=torch.float32, device=device)
    rows = max(1, (1 << 24) // max(1, K))
    for r0 in range(0, N, rows):
        r1 = min(N, r0 + rows)
        W[r0:r1] = (sigma * _rows_torch(seed, stream, r0, r1, K, device)).to(torch.float32)
    return W


def _rows_torch(seed, stream, r0, r1, K, device):
    """Rows [r0, r1) of normal_rows(seed, stream, ., K) as float64 on `device`."""
    import torch

    key = _i64(int(stream_key(seed, stream)))
    idx = torch.arange(r0 * K, r1 * K, dtype=torch.int64, device=device)
    pair = idx & ~1

    def uni(ctr):
        z = _mix_t(key + (ctr + 1) * _T_GAMMA)
        return _srl(z, 11).to(torch.float64) * (1.0 / 9007199254740992.0)

    u1 = 1.0 - uni(pair)
    u2 = uni(pair + 1)
    r = torch.sqrt(-2.0 * torch.log(u1))
    ang = (2.0 * math.pi) * u2
    return torch.where((idx & 1).bool(), r * torch.sin(ang), r * torch.cos(ang)).view(r1 - r0, K)


def activations_torch(seed: int, stream: str, M: int, K: int, dtype: str, device="cpu"):
    """activations() as an fp16 / bf16 torch tensor on `device`."""
    import torch

    z = _rows_torch(seed, stream, 0, M, K, device)
    if dtype == "f16":
        return z.to(torch.float16)
    if dtype == "bf16":
        return z.to(torch.float32).to(torch.bfloat16)
    raise ValueError(dtype)
