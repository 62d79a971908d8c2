"""CPU oracle for the weight-only quantized matmul (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The arithmetic lives in ``oracle.cpp``
(plain C++, compiled with g++ into ``_build/liboracle.so``); this file only
builds it and converts numpy arrays to pointers.

Every function mirrors one entry point of ``oracle.cpp``; see that file for the
passages each one follows and for the readings taken where the sources are
silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

MODES = {"sym": 0, "asym": 1, "lut": 2}
DTYPES = {"f16": 0, "bf16": 1}


def build(force: bool = False) -> str:
    """Compile oracle.cpp with g++ (strict IEEE: no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared",
                           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC])
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            lib.oracle_quantize.argtypes = [P, I, I, I, I, I, P, P, P, P]
            lib.oracle_pack.argtypes = [P, P, P, I, I, I, I, I, P, P, P]
            lib.oracle_unpack.argtypes = [P, P, P, I, I, I, I, I, P, P, P]
            lib.oracle_dequant.argtypes = [P, P, P, I, I, I, I, I, P]
            lib.oracle_round.argtypes = [P, S, I, P]
            lib.oracle_widen.argtypes = [P, S, I, P]
            lib.oracle_qmm.argtypes = [P, I, P, P, P, I, I, I, I, I, I, I, I, P]
            lib.oracle_qmm_gated.argtypes = [P, I, P, P, P, I, I, I, I, I, I, I, I, P]
            lib.oracle_quantize_asym.argtypes = [P, I, I, I, I, P, P, P]
            lib.oracle_pack_asym.argtypes = [P, P, P, I, I, I, I, I, P, P, P]
            lib.oracle_dequant_asym.argtypes = [P, P, P, I, I, I, I, P]
            lib.oracle_qmm_asym.argtypes = [P, I, P, P, P, I, I, I, I, I, I, I, I, P]
            lib.oracle_zeros_bytes.argtypes = [I, I, I, I]
            lib.oracle_zeros_bytes.restype = S
            lib.oracle_quantize_gidx.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
            lib.oracle_dequant_gidx.argtypes = [P, P, P, I, I, I, I, I, P, P]
            lib.oracle_pack_gidx.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P]
            lib.oracle_qmm_gidx.argtypes = [P, I, P, P, P, P, I, I, I, I, I, I, I, I, P]
            lib.oracle_packed_bytes.argtypes = [I, I, I]
            lib.oracle_packed_bytes.restype = S
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name} rejected its arguments (status {rc})")


def n_groups(K, group):
    return 1 if group == -1 else K // group


def quantize(W, mode, bits, group, lut=None):
    """fp32 W[N, K] -> (codes uint8[N, K], scales fp16-bits[N, G], zeros or None)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    G = n_groups(K, group)
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, G), np.uint16)
    zeros = np.empty((N, G), np.uint16) if mode == "asym" else None
    lut = None if lut is None else np.ascontiguousarray(lut, dtype=np.uint16)
    _check(_load().oracle_quantize(_p(W), N, K, MODES[mode], bits, group, _p(lut),
                                   _p(codes), _p(scales), _p(zeros)), "oracle_quantize")
    return codes, scales, zeros


def pack(codes, scales, zeros, mode, bits, group):
    """Logical (codes, scales, zeros) -> packed (qweight uint8, scales, zeros)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    qweight = np.empty(N * K * bits // 8, np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    sp = np.empty(scales.size, np.uint16)
    zp = None
    if mode == "asym":
        zeros = np.ascontiguousarray(zeros, dtype=np.uint16)
        zp = np.empty(zeros.size, np.uint16)
    _check(_load().oracle_pack(_p(codes), _p(scales), _p(zeros), N, K, MODES[mode], bits,
                               group, _p(qweight), _p(sp), _p(zp)), "oracle_pack")
    return qweight, sp, zp


def unpack(qweight, scales_p, zeros_p, N, K, mode, bits, group):
    """Packed buffers -> logical (codes, scales, zeros)."""
    G = n_groups(K, group)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint8)
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, G), np.uint16) if scales_p is not None else None
    zeros = np.empty((N, G), np.uint16) if (mode == "asym" and zeros_p is not None) else None
    sp = None if scales_p is None else np.ascontiguousarray(scales_p, dtype=np.uint16)
    zp = None if zeros_p is None else np.ascontiguousarray(zeros_p, dtype=np.uint16)
    _check(_load().oracle_unpack(_p(qweight), _p(sp), _p(zp), N, K, MODES[mode], bits, group,
                                 _p(codes), _p(scales), _p(zeros)), "oracle_unpack")
    return codes, scales, zeros


def dequant(codes, scales, zeros_or_lut, mode, bits, group):
    """Logical codes -> exact W~[N, K] (float64)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.empty((N, K), np.float64)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zl = None if zeros_or_lut is None else np.ascontiguousarray(zeros_or_lut, dtype=np.uint16)
    _check(_load().oracle_dequant(_p(codes), _p(scales), _p(zl), N, K, MODES[mode], bits,
                                  group, _p(out)), "oracle_dequant")
    return out


def round_to(values, dtype):
    """Values -> fp16/bf16 bits (round to nearest even), the oracle's own rounding."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _check(_load().oracle_round(_p(v), v.size, DTYPES[dtype], _p(out)), "oracle_round")
    return out


def widen(bits16, dtype):
    """fp16/bf16 bit patterns -> exact float64 values."""
    b = np.ascontiguousarray(bits16, dtype=np.uint16)
    out = np.empty(b.shape, np.float64)
    _check(_load().oracle_widen(_p(b), b.size, DTYPES[dtype], _p(out)), "oracle_widen")
    return out


def qmm(x, xdtype, qweight, scales_p, zeros_or_lut, M, N, K, mode, bits, group,
        n0=0, n1=None):
    """y[M, n1 - n0] (float64) from the packed buffers, for columns [n0, n1)."""
    n1 = N if n1 is None else n1
    x = np.ascontiguousarray(x, dtype=np.uint16)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint8)
    sp = np.ascontiguousarray(scales_p, dtype=np.uint16)
    zl = None if zeros_or_lut is None else np.ascontiguousarray(zeros_or_lut, dtype=np.uint16)
    y = np.empty((M, n1 - n0), np.float64)
    _check(_load().oracle_qmm(_p(x), DTYPES[xdtype], _p(qweight), _p(sp), _p(zl), M, N, K,
                              MODES[mode], bits, group, n0, n1, _p(y)), "oracle_qmm")
    return y


def qmm_gated(x, xdtype, qweight, scales_p, zeros_or_lut, M, I, K, mode, bits, group,
              i0=0, i1=None):
    """silu(gate) * up [M, i1 - i0] (float64) from a gated packed buffer (2I rows
    whose 16-row blocks alternate gate, up), for outputs [i0, i1)."""
    i1 = I if i1 is None else i1
    x = np.ascontiguousarray(x, dtype=np.uint16)
    qweight = np.ascontiguousarray(qweight, dtype=np.uint8)
    sp = np.ascontiguousarray(scales_p, dtype=np.uint16)
    zl = None if zeros_or_lut is None else np.ascontiguousarray(zeros_or_lut, dtype=np.uint16)
    y = np.empty((M, i1 - i0), np.float64)
    _check(_load().oracle_qmm_gated(_p(x), DTYPES[xdtype], _p(qweight), _p(sp), _p(zl), M, I, K,
                                    MODES[mode], bits, group, i0, i1, _p(y)), "oracle_qmm_gated")
    return y


# ---- zero-point options: zero group inside the scale group, fp16 or 4-bit zeros

def quantize_asym(W, group, zgroup):
    """fp32 W[N, K] -> (codes uint8[N, K], scales fp16-bits[N, G], zeros fp16-bits[N, Gz])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, n_groups(K, group)), np.uint16)
    zeros = np.empty((N, n_groups(K, zgroup)), np.uint16)
    _check(_load().oracle_quantize_asym(_p(W), N, K, group, zgroup, _p(codes), _p(scales),
                                        _p(zeros)), "oracle_quantize_asym")
    return codes, scales, zeros


def pack_asym(codes, scales, zeros, group, zgroup, zbits):
    """Logical -> packed (qweight uint8, scales uint16, zeros uint8 bytes)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    qweight = np.empty(N * K // 2, np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint16)
    sp = np.empty(scales.size, np.uint16)
    zp = np.empty(_load().oracle_zeros_bytes(N, K, zgroup, zbits), np.uint8)
    _check(_load().oracle_pack_asym(_p(codes), _p(scales), _p(zeros), N, K, group, zgroup, zbits,
                                    _p(qweight), _p(sp), _p(zp)), "oracle_pack_asym")
    return qweight, sp, zp


def dequant_asym(codes, scales, zeros, group, zgroup):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.empty((N, K), np.float64)
    _check(_load().oracle_dequant_asym(_p(codes), _p(np.ascontiguousarray(scales, np.uint16)),
                                       _p(np.ascontiguousarray(zeros, np.uint16)), N, K, group,
                                       zgroup, _p(out)), "oracle_dequant_asym")
    return out


def qmm_asym(x, xdtype, qweight, scales_p, zeros_p, M, N, K, group, zgroup, zbits, n0=0, n1=None):
    n1 = N if n1 is None else n1
    y = np.empty((M, n1 - n0), np.float64)
    _check(_load().oracle_qmm_asym(
        _p(np.ascontiguousarray(x, np.uint16)), DTYPES[xdtype],
        _p(np.ascontiguousarray(qweight, np.uint8)), _p(np.ascontiguousarray(scales_p, np.uint16)),
        _p(np.ascontiguousarray(zeros_p, np.uint8)), M, N, K, group, zgroup, zbits, n0, n1, _p(y)),
        "oracle_qmm_asym")
    return y


# ---- act-order: per-column groups g_idx

def _gidx(g_idx):
    return np.ascontiguousarray(g_idx, dtype=np.int32)


def quantize_gidx(W, mode, bits, group, g_idx, lut=None):
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    G = n_groups(K, group)
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, G), np.uint16)
    zeros = np.empty((N, G), np.uint16) if mode == "asym" else None
    lut = None if lut is None else np.ascontiguousarray(lut, dtype=np.uint16)
    _check(_load().oracle_quantize_gidx(_p(W), N, K, MODES[mode], bits, group, _p(_gidx(g_idx)),
                                        _p(lut), _p(codes), _p(scales), _p(zeros)),
           "oracle_quantize_gidx")
    return codes, scales, zeros


def dequant_gidx(codes, scales, zeros_or_lut, mode, bits, group, g_idx):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.empty((N, K), np.float64)
    zl = None if zeros_or_lut is None else np.ascontiguousarray(zeros_or_lut, dtype=np.uint16)
    _check(_load().oracle_dequant_gidx(_p(codes), _p(np.ascontiguousarray(scales, np.uint16)),
                                       _p(zl), N, K, MODES[mode], bits, group, _p(_gidx(g_idx)),
                                       _p(out)), "oracle_dequant_gidx")
    return out


def pack_gidx(codes, scales, zeros, g_idx, mode, bits, group):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    qweight = np.empty(N * K * bits // 8, np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    sp = np.empty(scales.size, np.uint16)
    zp = None
    if mode == "asym":
        zeros = np.ascontiguousarray(zeros, dtype=np.uint16)
        zp = np.empty(zeros.size, np.uint16)
    _check(_load().oracle_pack_gidx(_p(codes), _p(scales), _p(zeros), _p(_gidx(g_idx)), N, K,
                                    MODES[mode], bits, group, _p(qweight), _p(sp), _p(zp)),
           "oracle_pack_gidx")
    return qweight, sp, zp


def qmm_gidx(x, xdtype, qweight, scales_p, zeros_or_lut, g_idx, M, N, K, mode, bits, group,
             n0=0, n1=None):
    n1 = N if n1 is None else n1
    zl = None if zeros_or_lut is None else np.ascontiguousarray(zeros_or_lut, dtype=np.uint16)
    y = np.empty((M, n1 - n0), np.float64)
    _check(_load().oracle_qmm_gidx(
        _p(np.ascontiguousarray(x, np.uint16)), DTYPES[xdtype],
        _p(np.ascontiguousarray(qweight, np.uint8)), _p(np.ascontiguousarray(scales_p, np.uint16)),
        _p(zl), _p(_gidx(g_idx)), M, N, K, MODES[mode], bits, group, n0, n1, _p(y)),
        "oracle_qmm_gidx")
    return y
