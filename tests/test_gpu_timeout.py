"""Failure detection without a GPU fault: a kernel wait that runs out.

Every wait of the tensor-core kernel on another part of itself (a copy landing,
a stage freed, an MMA done) has a limit in clock cycles; a wait that runs out
makes the CTA drain what it issued, free its tensor memory and exit, and
qmm_check_error reports QMM_ERR_TIMEOUT.  Here the limit is cut to a few
dozen cycles, so the first wait for a copy gives up on purpose; then, back at
the default limit, an ordinary call on the same context must pass parity.
Nothing hangs or faults: every wait on that path is bounded.
"""
import numpy as np
import pytest
import torch

import weight_only_quantized_int4_b200 as q
from tests import cases

pytestmark = pytest.mark.gpu

TIMEOUT = -5


def _upload(p):
    tdt = torch.float16 if p.xdtype == "f16" else torch.bfloat16
    dev16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    x = dev16(p.x).view(tdt)
    return x, torch.from_numpy(p.qw).cuda(), dev16(p.sp), None if p.zl is None else dev16(p.zl)


def test_wait_that_runs_out_reports_timeout_then_a_normal_call_passes():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from weight_only_quantized_int4_b200 import build
    build.build()
    q.load()
    M, N, K = 64, 272, 1024
    assert q.path(M, N, K, "sym", 4, 128, "f16", "tensor") == "tensor"
    p = cases.make("sym", 4, 128, M, N, K, "f16", seed=41)
    y_ref, bound = cases.expected(p)
    x, qw, sp, _ = _upload(p)
    q.check_error()                                  # nothing pending before
    previous = q.set_wait_limit(64)
    try:
        q.qmm(x, qw, sp, None, N, K, "sym", 4, 128, ws=None, path="tensor")
        with pytest.raises(q.QmmError) as e:
            q.check_error()
        assert e.value.status == TIMEOUT
    finally:
        q.set_wait_limit(previous)
    assert q.set_wait_limit(0) == previous           # restored (0 = the default)
    # the context is usable: the same call at the default limit, a fresh workspace
    ws = q.workspace(M, N, K, "sym", path="tensor")
    y = q.qmm(x, qw, sp, None, N, K, "sym", 4, 128, ws=ws, path="tensor")
    torch.cuda.synchronize()
    q.check_error()
    cases.compare(y.float().cpu().numpy().astype(np.float64), y_ref, bound, "after timeout")
