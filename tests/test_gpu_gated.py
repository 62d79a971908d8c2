"""The fused feed-forward gate (qmm_pack_gated / qmm_gated) against the oracle
(needs a B200).

Packing: qmm_pack_gated(Wg, Wu) must write, byte for byte, what the oracle's
quantize + pack give for the interleaved [2I, K] matrix (16-row blocks
alternating gate, up).

Output: y = silu(g) u element by element against the oracle's double result.
The bound propagates the plain parity bound of each sum through the product:
|dy| <= |silu'(g)| |u| bound_g + |silu(g)| bound_u with |silu'| <= 1.1, plus one
rounding of y to the output type; the relative L2 bar is twice the plain one
(two sums enter each output).
"""
import numpy as np
import pytest
import torch

import oracle
import weight_only_quantized_int4_b200 as q
from tests import cases

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from weight_only_quantized_int4_b200 import build
    build.build()
    q.load()


def _split(rows):
    """Gate and up rows of an interleaved [2I, K] matrix."""
    n2 = rows.shape[0]
    blk = np.arange(n2) // 16
    return rows[blk % 2 == 0], rows[blk % 2 == 1]


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


CASES = [("sym", 4, 128, "f16"), ("sym", 4, -1, "bf16"), ("asym", 4, 128, "bf16"),
         ("asym", 4, 64, "f16"), ("lut", 4, 64, "f16"), ("lut", 2, 64, "f16"), ("sym", 4, 32, "f16")]


@pytest.mark.parametrize("mode,bits,group,xdtype", CASES)
def test_gated_pack_and_product(mode, bits, group, xdtype):
    I, K = 176, 1024                 # 11 output blocks: ragged tiles on both paths
    tdt = torch.float16 if xdtype == "f16" else torch.bfloat16
    out_eps = 2.0 ** -10 if xdtype == "f16" else 2.0 ** -7
    for M in (1, 5, 16, 17, 64, 130):
        p = cases.make(mode, bits, group, M, 2 * I, K, xdtype, seed=500 + M)
        Wg, Wu = _split(p.W_rows)
        lut = None if p.lut is None else _dev16(p.lut)
        qw, sc, ze = q.pack_gated(torch.from_numpy(Wg).cuda(), torch.from_numpy(Wu).cuda(), mode,
                                  bits, group, lut=lut)
        torch.cuda.synchronize()
        assert np.array_equal(qw.cpu().numpy(), p.qw), f"{mode} codes"
        assert np.array_equal(sc.cpu().numpy().view(np.uint16), p.sp), f"{mode} scales"
        if mode == "asym":
            assert np.array_equal(ze.cpu().numpy().view(np.uint16), p.zp), f"{mode} zeros"
        zl = ze if mode == "asym" else lut
        x = _dev16(p.x).view(tdt)
        ws = q.workspace(M, 2 * I, K, mode, bits, group)
        y = q.qmm_gated(x, qw, sc, zl, I, K, mode, bits, group, ws=ws)
        torch.cuda.synchronize()
        y_ref = oracle.qmm_gated(p.x, xdtype, p.qw, p.sp, p.zl, M, I, K, mode, bits, group)
        plain, plain_bound = cases.expected(p)
        g, u = _split(plain.T)
        bg, bu = _split(plain_bound.T)
        g, u, bg, bu = g.T, u.T, bg.T, bu.T
        silu_g = g / (1.0 + np.exp(-np.clip(g, -700, 700)))
        bound = 1.1 * np.abs(u) * bg + np.abs(silu_g) * bu + out_eps * np.abs(y_ref) + 1e-30
        y_gpu = y.float().cpu().numpy().astype(np.float64)
        err = np.abs(y_gpu - y_ref)
        assert np.all(err <= bound), (
            f"{mode}{bits} g{group} {xdtype} M{M}: {int((err > bound).sum())} over the bound, "
            f"max err/bound {float(np.max(err / bound)):.3f}")
        rel = np.linalg.norm(err) / np.linalg.norm(y_ref)
        assert rel <= 2 * cases.REL_L2_TOL, f"{mode} M{M}: relative L2 {rel:.3e}"
    q.check_error()


def test_gated_rejects_bad_sizes():
    lib = q.load()
    fake = torch.zeros(64, dtype=torch.uint8, device="cuda")
    import ctypes
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    # I not a multiple of 16
    assert lib.qmm_gated(vp(fake), 0, vp(fake), vp(fake), None, 1, 24, 128, 4, 128, 0, vp(fake),
                         None, 0, None) == -2
    assert lib.qmm_pack_gated(vp(fake), vp(fake), 24, 128, 0, 4, 128, None, vp(fake), vp(fake),
                              None, None) == -2
    # I <= 0
    assert lib.qmm_gated(vp(fake), 0, vp(fake), vp(fake), None, 1, 0, 128, 4, 128, 0, vp(fake),
                         None, 0, None) == -1
