"""qmm_noalloc: the decode path on the library's own static scratch buffer.

Callers that cannot allocate device memory (code being recorded into a CUDA
graph under stream capture, or an engine whose device memory is fixed at
start-up) cannot provide qmm's workspace; qmm_noalloc runs the same kernel on
a scratch array the library holds.  This file checks, through the C ABI, that
two calls in a row agree with qmm (with its own workspace) within the
tolerance of the parity tests, and that oversized problems are refused.

The file name sorts last on purpose: a run that stops at the first failure has
already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

import weight_only_quantized_int4_b200 as q
from tests import cases

pytestmark = pytest.mark.gpu


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


@pytest.mark.parametrize("mode,bits,group,xdtype,M,N,K", [
    ("sym", 4, 128, "f16", 5, 1024, 2048),
    ("asym", 4, 128, "bf16", 16, 4096, 4096),     # needs the reduced worker count
    ("lut", 4, 64, "f16", 1, 2048, 4096),
])
def test_noalloc_matches_qmm_twice(mode, bits, group, xdtype, M, N, K):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from weight_only_quantized_int4_b200 import build
    build.build()
    lib = q.load()
    p = cases.make(mode, bits, group, M, N, K, xdtype, seed=77)
    tdt = torch.float16 if xdtype == "f16" else torch.bfloat16
    x = _dev16(p.x).view(tdt)
    qw = torch.from_numpy(p.qw).cuda()
    sp = _dev16(p.sp)
    zl = None if p.zl is None else _dev16(p.zl)
    ws = q.workspace(M, N, K, mode, bits, group)
    y_ref = q.qmm(x, qw, sp, zl, N, K, mode, bits, group, ws=ws)
    _, bound = cases.expected(p)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    dt = 0 if xdtype == "f16" else 1
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
        st = lib.qmm_noalloc(ptr(x), dt, ptr(qw), ptr(sp), ptr(zl), M, N, K, bits, group,
                             q.MODES[mode], ptr(y), stream)
        assert st == 0, q.strerror(st)
        torch.cuda.synchronize()
        cases.compare(y.float().cpu().numpy().astype(np.float64),
                      y_ref.float().cpu().numpy().astype(np.float64), bound, f"noalloc {mode}")


def test_noalloc_rejects_more_than_one_slab():
    lib = q.load()
    fake = ctypes.c_void_p(0x1000)
    st = lib.qmm_noalloc(fake, 0, fake, fake, None, 17, 256, 256, 4, 128, 0,
                         ctypes.c_void_p(0x900000), None)
    assert st == -7
    assert "static scratch" in q.strerror(st)
