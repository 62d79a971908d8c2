"""qmm_noalloc: the decode path on the library's own static scratch buffer.

Some callers cannot allocate device memory while they run the product: code
being recorded into a CUDA graph under stream capture, or an engine whose
device memory is planned once at start-up and may not grow.  They cannot hand
qmm its split-K workspace, so qmm_noalloc runs the same kernel on a scratch
array the library holds.  This file checks, through the C ABI, two calls in a
row against the oracle (the parity tests' element bound and relative L2
bound), on shapes whose decode plan splits K across CTAs -- so the shared
buffer's arrival counters and partial sums are really used, and must be back
at zero for the second call -- and that oversized problems are refused.

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

SCRATCH_BYTES = 8 << 20   # the library's static buffer


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


# N = 9600: 300 row tiles of 32 rows, more than one resident CTA per tile
# can take, so the plan is the split-K one that needs a workspace.  The bf16
# case with 16 tokens needs more partial-sum slots than the buffer holds and
# runs with fewer split-K workers.
@pytest.mark.parametrize("mode,bits,group,xdtype,M,N,K", [
    ("sym", 4, 128, "f16", 1, 9600, 1024),
    ("asym", 4, 128, "bf16", 16, 9600, 2048),
    ("lut", 4, 64, "f16", 5, 9600, 1024),
])
def test_noalloc_matches_oracle_twice(mode, bits, group, xdtype, M, N, K):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from weight_only_quantized_int4_b200 import build
    build.build()
    lib = q.load()
    need = q.workspace_size(M, N, K, mode, bits, group)
    assert need > 0, "the shape must use split-K partials (and so the static buffer)"
    if mode == "asym":
        assert need > SCRATCH_BYTES, "this case must take the fewer-workers plan"
    p = cases.make(mode, bits, group, M, N, K, xdtype, seed=77)
    y_ref, bound = cases.expected(p)
    tdt = torch.float16 if xdtype == "f16" else torch.bfloat16
    x = _dev16(p.x).view(tdt)
    qw = torch.from_numpy(p.qw).cuda()
    sp = _dev16(p.sp)
    zl = None if p.zl is None else _dev16(p.zl)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    dt = 0 if xdtype == "f16" else 1
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
        st = lib.qmm_noalloc(ptr(x), dt, ptr(qw), ptr(sp), ptr(zl), M, N, K, bits, group,
                             q.MODES[mode], ptr(y), stream)
        assert st == 0, q.strerror(st)
        torch.cuda.synchronize()
        cases.compare(y.float().cpu().numpy().astype(np.float64), y_ref, bound,
                      f"noalloc {mode} call {call}")
    assert lib.qmm_check_error(stream) == 0


def test_noalloc_rejects_more_than_one_slab():
    lib = q.load()
    fake = ctypes.c_void_p(0x1000)
    st = lib.qmm_noalloc(fake, 0, fake, fake, None, 17, 256, 256, 4, 128, 0,
                         ctypes.c_void_p(0x900000), None)
    assert st == -7
    assert "static scratch" in q.strerror(st)
