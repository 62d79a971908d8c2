"""Problem construction and comparison helpers shared by the GPU tests.

Inputs come from the seeded generator; expected values come from the oracle
only.  Nothing here reads anything produced by the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle
from weight_only_quantized_int4_b200 import synth

# Element bound on |y_gpu - y_oracle| relative to sum_k |x_mk| |w~_nk|, and the
# bound on the relative L2 error over a whole output.
ELEM_TOL = 4e-3
REL_L2_TOL = 2e-3

SIGMA = {"sym": 0.02, "asym": 0.015, "lut": 0.02}


def table(mode, bits):
    if mode != "lut":
        return None
    return {4: synth.nf4_table, 3: synth.nf3_table, 2: lambda: synth.lut2_table(0)}[bits]()


@dataclass
class Problem:
    mode: str
    bits: int
    group: int
    M: int
    N: int
    K: int
    xdtype: str
    rows: np.ndarray           # row indices the oracle covers (whole 16-row blocks)
    W_rows: np.ndarray         # fp32 weights of those rows
    x: np.ndarray              # uint16 bits [M, K]
    lut: np.ndarray | None
    codes: np.ndarray          # oracle logical codes of `rows`
    scales: np.ndarray
    zeros: np.ndarray | None
    qw: np.ndarray             # oracle packed buffers of `rows`
    sp: np.ndarray
    zp: np.ndarray | None

    @property
    def zl(self):
        return self.zp if self.mode == "asym" else self.lut


def row_blocks(N, n_blocks, seed):
    """A seeded choice of whole 16-row blocks (always the first and the last)."""
    nrb = N // 16
    if n_blocks >= nrb:
        blocks = np.arange(nrb)
    else:
        rng = np.random.default_rng(seed)
        mid = rng.choice(np.arange(1, nrb - 1), size=n_blocks - 2, replace=False)
        blocks = np.sort(np.concatenate([[0], mid, [nrb - 1]]))
    return (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)


def make(mode, bits, group, M, N, K, xdtype="f16", seed=0, n_blocks=None, wstream="W"):
    rows = np.arange(N) if n_blocks is None else row_blocks(N, n_blocks, seed + 1)
    W_rows = synth.weights(seed, wstream, N, K, SIGMA[mode], rows=rows)
    lut = table(mode, bits)
    codes, scales, zeros = oracle.quantize(W_rows, mode, bits, group, lut=lut)
    qw, sp, zp = oracle.pack(codes, scales, zeros, mode, bits, group)
    x = synth.activations(seed, "x", M, K, xdtype)
    return Problem(mode, bits, group, M, N, K, xdtype, rows, W_rows, x, lut, codes, scales, zeros,
                   qw, sp, zp)


def expected(p: Problem):
    """(y_ref [M, rows], bound [M, rows]) from the oracle."""
    y = oracle.qmm(p.x, p.xdtype, p.qw, p.sp, p.zl, p.M, len(p.rows), p.K, p.mode, p.bits,
                   p.group)
    zl = p.zeros if p.mode == "asym" else p.lut
    Wt = oracle.dequant(p.codes, p.scales, zl, p.mode, p.bits, p.group)
    xv = oracle.widen(p.x, p.xdtype)
    bound = ELEM_TOL * (np.abs(xv) @ np.abs(Wt).T)
    return y, bound


def compare(y_gpu: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what=""):
    """Element bound and relative L2 bound; returns (max err/bound, rel L2)."""
    err = np.abs(y_gpu - y_ref)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements over the bound, first at {tuple(i)}: "
                             f"gpu {y_gpu[tuple(i)]} oracle {y_ref[tuple(i)]} "
                             f"bound {bound[tuple(i)]}")
    ref_norm = np.linalg.norm(y_ref)
    rel = np.linalg.norm(err) / ref_norm if ref_norm > 0 else np.linalg.norm(err)
    assert rel <= REL_L2_TOL, f"{what}: relative L2 error {rel:.3e} > {REL_L2_TOL}"
    worst = float(np.max(np.where(bound > 0, err / np.maximum(bound, 1e-300), 0.0)))
    return worst, rel
