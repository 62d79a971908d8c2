"""Python binding of libqmm, the weight-only quantized matmul for B200.

Argument marshalling only: torch tensors are passed to the C ABI
(include/qmm.h) as raw device pointers together with the current CUDA
stream; every step of the computation runs in the library's CUDA kernels.
There is no fallback: if libqmm.so is missing or cannot be loaded, every call
raises.

    import weight_only_quantized_int4_b200 as q
    qw, s, z = q.pack(W, "sym", bits=4, group=128)          # W: fp32 [N, K] on cuda
    y = q.qmm(x, qw, s, None, N=N, K=K, mode="sym", bits=4, group=128)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmm.so")

MODES = {"sym": 0, "asym": 1, "lut": 2}
DTYPES = {torch.float16: 0, torch.bfloat16: 1}
PATHS = {"auto": 0, "skinny": 1, "tensor": 2, "skinny_streamk": 3}
PATH_NAMES = {1: "skinny", 2: "tensor"}

SYMBOLS = ("qmm_packed_size", "qmm_pack", "qmm_workspace_size", "qmm_workspace_size_for", "qmm",
           "qmm_with_path",
           "qmm_path", "qmm_path_ex", "qmm_dequant", "qmm_check_error", "qmm_strerror", "qmm_noalloc",
           "qmm_pack_gated", "qmm_gated", "qmm_zeros_size", "qmm_pack_asym",
           "qmm_workspace_size_asym", "qmm_asym", "qmm_dequant_asym", "qmm_actorder_perm",
           "qmm_pack_actorder", "qmm_workspace_size_actorder", "qmm_actorder",
           "qmm_set_wait_limit")

_lib = None
_lock = threading.Lock()


class QmmError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {strerror(status)} (status {status})")
        self.status = status


def load(path: str = LIB_PATH):
    """Load libqmm.so (raises OSError if it is absent: build it first)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise OSError(f"{path} not found; build it with "
                              "`python -m weight_only_quantized_int4_b200.build`")
            lib = ctypes.CDLL(path)
            P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            lib.qmm_packed_size.argtypes = [I, I, I, I, I, P, P]
            lib.qmm_packed_size.restype = S
            lib.qmm_pack.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
            lib.qmm_workspace_size.argtypes = [I, I, I, I, I, I]
            lib.qmm_workspace_size.restype = S
            lib.qmm_workspace_size_for.argtypes = [I, I, I, I, I, I, I]
            lib.qmm_workspace_size_for.restype = S
            lib.qmm.argtypes = [P, I, P, P, P, I, I, I, I, I, I, P, P, S, P]
            lib.qmm_with_path.argtypes = [P, I, P, P, P, I, I, I, I, I, I, P, P, S, P, I]
            lib.qmm_path.argtypes = [I, I, I, I, I, I]
            lib.qmm_path_ex.argtypes = [I, I, I, I, I, I, I, I]
            lib.qmm_noalloc.argtypes = [P, I, P, P, P, I, I, I, I, I, I, P, P]
            lib.qmm_pack_gated.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P]
            lib.qmm_gated.argtypes = [P, I, P, P, P, I, I, I, I, I, I, P, P, S, P]
            lib.qmm_dequant.argtypes = [P, P, P, I, I, I, I, I, I, P, P]
            lib.qmm_zeros_size.argtypes = [I, I, I, I, I]
            lib.qmm_zeros_size.restype = S
            lib.qmm_pack_asym.argtypes = [P, I, I, I, I, I, P, P, P, P]
            lib.qmm_workspace_size_asym.argtypes = [I, I, I, I, I, I]
            lib.qmm_workspace_size_asym.restype = S
            lib.qmm_asym.argtypes = [P, I, P, P, P, I, I, I, I, I, I, P, P, S, P]
            lib.qmm_dequant_asym.argtypes = [P, P, P, I, I, I, I, I, I, P, P]
            lib.qmm_actorder_perm.argtypes = [P, I, I, P, P, P]
            lib.qmm_pack_actorder.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P]
            lib.qmm_workspace_size_actorder.argtypes = [I, I, I, I, I, I]
            lib.qmm_workspace_size_actorder.restype = S
            lib.qmm_actorder.argtypes = [P, I, P, P, P, P, I, I, I, I, I, I, P, P, S, P]
            lib.qmm_check_error.argtypes = [P]
            lib.qmm_set_wait_limit.argtypes = [ctypes.c_longlong]
            lib.qmm_set_wait_limit.restype = ctypes.c_longlong
            lib.qmm_strerror.argtypes = [I]
            lib.qmm_strerror.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def strerror(status: int) -> str:
    return load().qmm_strerror(status).decode()


# Pointer arguments go to ctypes as plain ints (every entry point declares its
# argtypes, so ctypes converts them): no c_void_p object per argument.
def _ptr(t):
    return None if t is None else t.data_ptr()


# The current device's current stream as a raw cudaStream_t.  torch's raw
# accessor skips building a torch.cuda.Stream object on every call; the public
# route stays for builds that lack it.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream():
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, what: str):
    if status != 0:
        raise QmmError(status, what)


def _dev(t, name):
    if t is not None and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def packed_size(N, K, mode, bits=4, group=128):
    """(qweight bytes, scale bytes, zero bytes) for an [N, K] weight."""
    sb, zb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    q = load().qmm_packed_size(N, K, bits, group, MODES[mode], ctypes.byref(sb), ctypes.byref(zb))
    if q == 0:
        raise QmmError(-2, "qmm_packed_size")
    return q, sb.value, zb.value


def pack(W, mode, bits=4, group=128, lut=None, out=None):
    """Quantize fp32 W[N, K] (CUDA) -> (qweight uint8, scales fp16-bits int16, zeros or None)."""
    _dev(W, "W")
    N, K = W.shape
    qb, sb, zb = packed_size(N, K, mode, bits, group)
    if out is None:
        qw = torch.empty(qb, dtype=torch.uint8, device=W.device)
        sc = torch.empty(sb // 2, dtype=torch.int16, device=W.device)
        ze = torch.empty(zb // 2, dtype=torch.int16, device=W.device) if zb else None
    else:
        qw, sc, ze = out
    _check(load().qmm_pack(_ptr(W), N, K, MODES[mode], bits, group, _ptr(lut), _ptr(qw),
                           _ptr(sc), _ptr(ze), _stream()), "qmm_pack")
    return qw, sc, ze


def pack_gated(Wg, Wu, mode, bits=4, group=128, lut=None):
    """Quantize the FFN gate and up projections (fp32 [I, K] each, CUDA) into
    one packed [2I, K] buffer with alternating 16-row gate / up blocks."""
    _dev(Wg, "Wg")
    _dev(Wu, "Wu")
    I, K = Wg.shape
    if tuple(Wu.shape) != (I, K):
        raise ValueError("Wg and Wu must have the same shape")
    qb, sb, zb = packed_size(2 * I, K, mode, bits, group)
    qw = torch.empty(qb, dtype=torch.uint8, device=Wg.device)
    sc = torch.empty(sb // 2, dtype=torch.int16, device=Wg.device)
    ze = torch.empty(zb // 2, dtype=torch.int16, device=Wg.device) if zb else None
    _check(load().qmm_pack_gated(_ptr(Wg), _ptr(Wu), I, K, MODES[mode], bits, group, _ptr(lut),
                                 _ptr(qw), _ptr(sc), _ptr(ze), _stream()), "qmm_pack_gated")
    return qw, sc, ze


def qmm_gated(x, qweight, scales, zeros_or_lut, I, K, mode, bits=4, group=128, y=None, ws=None):
    """y[M, I] = silu(x . dequant(Wg)^T) * (x . dequant(Wu)^T) on a pack_gated buffer."""
    _dev(x, "x")
    if x.dtype not in DTYPES:
        raise ValueError("x must be fp16 or bf16")
    M = x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x.shape[1] != K")
    if y is None:
        y = torch.empty(M, I, dtype=x.dtype, device=x.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(load().qmm_gated(_ptr(x), DTYPES[x.dtype], _ptr(qweight), _ptr(scales),
                            _ptr(zeros_or_lut), M, I, K, bits, group, MODES[mode], _ptr(y),
                            _ptr(ws), nbytes, _stream()), "qmm_gated")
    return y


def workspace_size(M, N, K, mode, bits=4, group=128, path="auto"):
    return load().qmm_workspace_size_for(M, N, K, bits, group, MODES[mode], PATHS[path])


def workspace(M, N, K, mode, bits=4, group=128, device="cuda", path="auto"):
    """A zero-filled workspace for this problem (None if it needs none)."""
    n = workspace_size(M, N, K, mode, bits, group, path)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def path(M, N, K, mode, bits=4, group=128, xdtype=None, request="auto"):
    """The kernel ("skinny" or "tensor") a call runs: with xdtype None, qmm's
    choice for fp16 activations; else for that activation dtype ("f16",
    "bf16" or a torch dtype) when `request` (a path name) is asked for."""
    if xdtype is None and request == "auto":
        st = load().qmm_path(M, N, K, bits, group, MODES[mode])
        if st < 0:
            raise QmmError(st, "qmm_path")
        return PATH_NAMES[st]
    dt = {"f16": 0, "bf16": 1, None: 0}.get(xdtype, None)
    if dt is None:
        dt = DTYPES[xdtype]
    st = load().qmm_path_ex(M, N, K, bits, group, MODES[mode], dt, PATHS[request])
    if st < 0:
        raise QmmError(st, "qmm_path_ex")
    return PATH_NAMES[st]


def qmm(x, qweight, scales, zeros_or_lut, N, K, mode, bits=4, group=128, y=None, ws=None,
        path="auto"):
    """y[M, N] = x[M, K] . dequant(qweight)^T on the current device and stream.

    ws: a workspace from workspace() (split-K over all SMs; reusable by later
    calls on the same stream), or None: then every CTA owns whole row tiles,
    which is slower when there are few row tiles (large N / K at small M)."""
    _dev(x, "x")
    if x.dtype not in DTYPES:
        raise ValueError("x must be fp16 or bf16")
    M = x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x.shape[1] != K")
    if y is None:
        y = torch.empty(M, N, dtype=x.dtype, device=x.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(load().qmm_with_path(_ptr(x), DTYPES[x.dtype], _ptr(qweight), _ptr(scales),
                                _ptr(zeros_or_lut), M, N, K, bits, group, MODES[mode], _ptr(y),
                                _ptr(ws), nbytes, _stream(), PATHS[path]), "qmm")
    return y


def qmm_noalloc(x, qweight, scales, zeros_or_lut, N, K, mode, bits=4, group=128, y=None):
    """y = x . dequant(qweight)^T with the library's static scratch buffer
    (no workspace, no allocation by the library); M <= 16."""
    _dev(x, "x")
    if x.dtype not in DTYPES:
        raise ValueError("x must be fp16 or bf16")
    M = x.shape[0]
    if y is None:
        y = torch.empty(M, N, dtype=x.dtype, device=x.device)
    _check(load().qmm_noalloc(_ptr(x), DTYPES[x.dtype], _ptr(qweight), _ptr(scales),
                              _ptr(zeros_or_lut), M, N, K, bits, group, MODES[mode], _ptr(y),
                              _stream()), "qmm_noalloc")
    return y


def dequant(qweight, scales, zeros_or_lut, N, K, mode, bits=4, group=128, dtype=torch.float16,
            out=None):
    """Decoded weights W~[N, K] (fp16 or bf16), for checks and inspection."""
    if out is None:
        out = torch.empty(N, K, dtype=dtype, device=qweight.device)
    _check(load().qmm_dequant(_ptr(qweight), _ptr(scales), _ptr(zeros_or_lut), N, K, bits, group,
                              MODES[mode], DTYPES[out.dtype], _ptr(out), _stream()),
           "qmm_dequant")
    return out


# ---- zero-point options: zero group inside the scale group, fp16 or 4-bit zeros

def pack_asym(W, group=-1, zgroup=8, zbits=4):
    """Quantize fp32 W[N, K] (CUDA) into ASYM codes with zero-points per group
    of `zgroup` (fp16 or 4-bit) -> (qweight uint8, scales int16 bits, zeros uint8 bytes)."""
    _dev(W, "W")
    N, K = W.shape
    qb, sb, _ = packed_size(N, K, "asym", 4, group)
    zb = load().qmm_zeros_size(N, K, group, zgroup, zbits)
    if zb == 0:
        raise QmmError(-2, "qmm_zeros_size")
    qw = torch.empty(qb, dtype=torch.uint8, device=W.device)
    sc = torch.empty(sb // 2, dtype=torch.int16, device=W.device)
    ze = torch.empty(zb, dtype=torch.uint8, device=W.device)
    _check(load().qmm_pack_asym(_ptr(W), N, K, group, zgroup, zbits, _ptr(qw), _ptr(sc), _ptr(ze),
                                _stream()), "qmm_pack_asym")
    return qw, sc, ze


def workspace_asym(M, N, K, group, zgroup, zbits, device="cuda"):
    n = load().qmm_workspace_size_asym(M, N, K, group, zgroup, zbits)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def qmm_asym(x, qweight, scales, zeros, N, K, group=-1, zgroup=8, zbits=4, y=None, ws=None):
    """y = x . dequant(qweight)^T for a pack_asym buffer."""
    _dev(x, "x")
    if x.dtype not in DTYPES:
        raise ValueError("x must be fp16 or bf16")
    M = x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x.shape[1] != K")
    if y is None:
        y = torch.empty(M, N, dtype=x.dtype, device=x.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(load().qmm_asym(_ptr(x), DTYPES[x.dtype], _ptr(qweight), _ptr(scales), _ptr(zeros), M,
                           N, K, group, zgroup, zbits, _ptr(y), _ptr(ws), nbytes, _stream()),
           "qmm_asym")
    return y


def dequant_asym(qweight, scales, zeros, N, K, group=-1, zgroup=8, zbits=4, dtype=torch.float16):
    out = torch.empty(N, K, dtype=dtype, device=qweight.device)
    _check(load().qmm_dequant_asym(_ptr(qweight), _ptr(scales), _ptr(zeros), N, K, group, zgroup,
                                   zbits, DTYPES[out.dtype], _ptr(out), _stream()),
           "qmm_dequant_asym")
    return out


# ---- act-order: per-column groups

def actorder_perm(g_idx, group):
    """perm (int32 [K], CUDA) from g_idx (int32 [K], CUDA); raises if a group
    does not hold exactly `group` columns (synchronizes the stream)."""
    _dev(g_idx, "g_idx")
    K = g_idx.shape[0]
    perm = torch.empty(K, dtype=torch.int32, device=g_idx.device)
    bad = torch.zeros(1, dtype=torch.int32, device=g_idx.device)
    _check(load().qmm_actorder_perm(_ptr(g_idx), K, group, _ptr(perm), _ptr(bad), _stream()),
           "qmm_actorder_perm")
    if int(bad.item()) != 0:
        raise ValueError(f"g_idx: {int(bad.item())} groups do not hold exactly {group} columns")
    return perm


def pack_actorder(W, perm, mode, bits=4, group=128, lut=None):
    """Quantize fp32 W[N, K] with act-order groups: packed column j = W[:, perm[j]]."""
    _dev(W, "W")
    _dev(perm, "perm")
    N, K = W.shape
    qb, sb, zb = packed_size(N, K, mode, bits, group)
    qw = torch.empty(qb, dtype=torch.uint8, device=W.device)
    sc = torch.empty(sb // 2, dtype=torch.int16, device=W.device)
    ze = torch.empty(zb // 2, dtype=torch.int16, device=W.device) if zb else None
    _check(load().qmm_pack_actorder(_ptr(W), _ptr(perm), N, K, MODES[mode], bits, group, _ptr(lut),
                                    _ptr(qw), _ptr(sc), _ptr(ze), _stream()), "qmm_pack_actorder")
    return qw, sc, ze


def workspace_actorder(M, N, K, mode, bits=4, group=128, device="cuda"):
    n = load().qmm_workspace_size_actorder(M, N, K, bits, group, MODES[mode])
    return torch.zeros(n, dtype=torch.uint8, device=device)


def qmm_actorder(x, perm, qweight, scales, zeros_or_lut, N, K, mode, bits=4, group=128, y=None,
                 ws=None):
    """y = x . W~^T over the original columns for a pack_actorder buffer."""
    _dev(x, "x")
    if x.dtype not in DTYPES:
        raise ValueError("x must be fp16 or bf16")
    M = x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x.shape[1] != K")
    if y is None:
        y = torch.empty(M, N, dtype=x.dtype, device=x.device)
    if ws is None:
        ws = workspace_actorder(M, N, K, mode, bits, group, device=x.device)
    nbytes = ws.numel() * ws.element_size()
    _check(load().qmm_actorder(_ptr(x), DTYPES[x.dtype], _ptr(perm), _ptr(qweight), _ptr(scales),
                               _ptr(zeros_or_lut), M, N, K, bits, group, MODES[mode], _ptr(y),
                               _ptr(ws), nbytes, _stream()), "qmm_actorder")
    return y


def check_error():
    """Raise if a kernel abandoned a bounded wait since the last check."""
    _check(load().qmm_check_error(_stream()), "qmm_check_error")


def set_wait_limit(cycles):
    """Clock cycles a kernel wait may take before the call gives up (<= 0: the
    default of about 2 s); returns the previous value."""
    return load().qmm_set_wait_limit(int(cycles))
