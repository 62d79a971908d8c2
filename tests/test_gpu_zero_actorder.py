"""Zero-point options and act-order groups: the CUDA path against the oracle
(needs a B200).

Zero-point options (Marlin zero-point issue, efrantar's and mobicham's
replies): ASYM codes with a zero group nested in the scale group and fp16 or
4-bit integer zero-points.  Act-order (GPTQ-Triton summary, "Limitations &
Caveats"): groups given per column by g_idx, the packed columns sorted by
group.

Packing and decoding are compared byte for byte; the product element by
element against the oracle's double result with |err| <= 4e-3 sum|x||w~| and
relative L2 <= 2e-3.  Shapes cover ragged row tiles (11 row blocks), a K that
ends halfway through a 128-column stage, an odd number of 4-bit zero records
per row block, and M on both sides of the 16-token slab.
"""
import numpy as np
import pytest
import torch

import oracle
import weight_only_quantized_int4_b200 as q
from tests import cases
from weight_only_quantized_int4_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from weight_only_quantized_int4_b200 import build
    build.build()
    q.load()


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def tdtype(xdtype):
    return torch.float16 if xdtype == "f16" else torch.bfloat16


def bound_of(x, xdtype, Wt):
    return cases.ELEM_TOL * (np.abs(oracle.widen(x, xdtype)) @ np.abs(Wt).T)


# ------------------------------------------------------ zero-point options

ZCASES = [  # group, zgroup, zbits, xdtype, K
    (-1, 8, 4, "f16", 1088),      # mobicham's scale per row / zero per 8; K ends mid-stage
    (-1, 8, 16, "bf16", 1088),
    (-1, 64, 4, "f16", 1088),     # 17 zero groups per row block: odd 8-byte record count
    (-1, 256, 4, "bf16", 1280),
    (-1, -1, 4, "f16", 1024),     # one 4-bit zero-point per row
    (128, 128, 4, "f16", 1152),   # quantized zero-points only
    (128, 32, 4, "bf16", 1152),
    (64, 16, 16, "f16", 1152),
    (256, 64, 16, "bf16", 1280),
]


@pytest.mark.parametrize("group,zgroup,zbits,xdtype,K", ZCASES)
def test_zero_options_pack_dequant_qmm(group, zgroup, zbits, xdtype, K):
    N = 176
    W = synth.weights(70, "W", N, K, 0.015)
    codes, scales, zeros = oracle.quantize_asym(W, group, zgroup)
    qw_o, sp_o, zp_o = oracle.pack_asym(codes, scales, zeros, group, zgroup, zbits)
    qw, sc, ze = q.pack_asym(torch.from_numpy(W).cuda(), group, zgroup, zbits)
    torch.cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy(), qw_o), "codes"
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sp_o), "scales"
    assert np.array_equal(ze.cpu().numpy(), zp_o), "zero-points"
    Wt = oracle.dequant_asym(codes, scales, zeros, group, zgroup)
    for odt in ("f16", "bf16"):
        d = q.dequant_asym(qw, sc, ze, N, K, group, zgroup, zbits, dtype=tdtype(odt))
        assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16),
                              oracle.round_to(Wt, odt)), odt
    for M in (1, 5, 16, 17, 40):
        x = synth.activations(71 + M, "x", M, K, xdtype)
        ws = q.workspace_asym(M, N, K, group, zgroup, zbits)
        y = q.qmm_asym(dev(x).view(tdtype(xdtype)), qw, sc, ze, N, K, group, zgroup, zbits, ws=ws)
        torch.cuda.synchronize()
        y_ref = oracle.qmm_asym(x, xdtype, qw_o, sp_o, zp_o, M, N, K, group, zgroup, zbits)
        cases.compare(y.float().cpu().numpy().astype(np.float64), y_ref, bound_of(x, xdtype, Wt),
                      f"g{group} zg{zgroup} z{zbits} {xdtype} M{M}")
        # no workspace: every CTA owns whole tiles
        y2 = q.qmm_asym(dev(x).view(tdtype(xdtype)), qw, sc, ze, N, K, group, zgroup, zbits)
        torch.cuda.synchronize()
        cases.compare(y2.float().cpu().numpy().astype(np.float64), y_ref,
                      bound_of(x, xdtype, Wt), f"no workspace M{M}")
    q.check_error()


def test_zero_options_same_group_fp16_is_plain_asym():
    """zgroup == group with fp16 zeros runs the plain ASYM format: same bytes,
    same result bits as qmm_pack / qmm."""
    N, K, M = 96, 1024, 3
    W = torch.from_numpy(synth.weights(72, "W", N, K, 0.015)).cuda()
    qw, sc, ze = q.pack_asym(W, 128, 128, 16)
    qw0, sc0, ze0 = q.pack(W, "asym", 4, 128)
    torch.cuda.synchronize()
    assert torch.equal(qw, qw0) and torch.equal(sc, sc0)
    assert torch.equal(ze, ze0.view(torch.uint8))
    x = dev(synth.activations(72, "x", M, K, "bf16")).view(torch.bfloat16)
    y = q.qmm_asym(x, qw, sc, ze, N, K, 128, 128, 16)
    y0 = q.qmm(x, qw0, sc0, ze0, N, K, "asym", 4, 128)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)


def test_zero_options_zero_point_codes_give_zero():
    """Every code at its (4-bit) zero-point: y = 0 exactly, any x."""
    N, K, M, zg = 64, 512, 4, 8
    rng = np.random.default_rng(73)
    z = rng.integers(0, 16, (N, K // zg))
    codes = np.repeat(z, zg, axis=1).astype(np.uint8)
    scales = np.full((N, 1), 0x3C00, np.uint16)
    zeros = oracle.round_to(z.astype(np.float64), "f16")
    qw, sp, zp = oracle.pack_asym(codes, scales, zeros, -1, zg, 4)
    x = dev(synth.activations(73, "x", M, K, "f16")).view(torch.float16)
    y = q.qmm_asym(x, dev(qw), dev(sp), dev(zp), N, K, -1, zg, 4)
    torch.cuda.synchronize()
    assert not torch.any(y != 0)


def test_zero_options_reject_bad_groups():
    import ctypes
    lib = q.load()
    fake = torch.zeros(64, dtype=torch.uint8, device="cuda")
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    # zero group larger than the scale group; not a power of two; zbits 8
    for group, zgroup, zbits, want in ((64, 128, 4, -2), (-1, 24, 4, -2), (-1, 8, 8, -1),
                                       (-1, 4, 4, -2)):
        assert lib.qmm_asym(vp(fake), 0, vp(fake), vp(fake), vp(fake), 1, 16, 1024, group, zgroup,
                            zbits, vp(fake), None, 0, None) == want
        assert lib.qmm_zeros_size(16, 1024, group, zgroup, zbits) == 0


# ------------------------------------------------------------ act-order

def _gidx(K, group, seed):
    order = np.random.default_rng(seed).permutation(K)
    gidx = np.empty(K, np.int32)
    gidx[order] = np.arange(K) // group
    return gidx


ACASES = [("sym", 4, 128, "f16", 1088 - 64), ("sym", 4, 64, "bf16", 1088),
          ("asym", 4, 128, "bf16", 1152), ("lut", 4, 64, "f16", 1024), ("lut", 2, 32, "f16", 1152),
          ("lut", 3, 64, "f16", 1152), ("sym", 4, 16, "f16", 1024)]


@pytest.mark.parametrize("mode,bits,group,xdtype,K", ACASES)
def test_actorder_pack_and_qmm(mode, bits, group, xdtype, K):
    N = 176
    W = synth.weights(80, "W", N, K, cases.SIGMA[mode])
    lut = cases.table(mode, bits)
    gidx = _gidx(K, group, 81)
    codes, scales, zeros = oracle.quantize_gidx(W, mode, bits, group, gidx, lut=lut)
    qw_o, sp_o, zp_o = oracle.pack_gidx(codes, scales, zeros, gidx, mode, bits, group)
    # perm from g_idx on the device = numpy's stable argsort
    perm = q.actorder_perm(torch.from_numpy(gidx).cuda(), group)
    torch.cuda.synchronize()
    assert np.array_equal(perm.cpu().numpy(), np.argsort(gidx, kind="stable"))
    lut_d = None if lut is None else dev(lut)
    qw, sc, ze = q.pack_actorder(torch.from_numpy(W).cuda(), perm, mode, bits, group, lut=lut_d)
    torch.cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy(), qw_o), "codes"
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sp_o), "scales"
    if mode == "asym":
        assert np.array_equal(ze.cpu().numpy().view(np.uint16), zp_o), "zeros"
    zl_o = zp_o if mode == "asym" else lut
    zl = ze if mode == "asym" else lut_d
    zl_log = zeros if mode == "asym" else lut
    Wt = oracle.dequant_gidx(codes, scales, zl_log, mode, bits, group, gidx)
    for M in (1, 7, 16, 33, 80):
        x = synth.activations(82 + M, "x", M, K, xdtype)
        y = q.qmm_actorder(dev(x).view(tdtype(xdtype)), perm, qw, sc, zl, N, K, mode, bits, group)
        torch.cuda.synchronize()
        y_ref = oracle.qmm_gidx(x, xdtype, qw_o, sp_o, zl_o, gidx, M, N, K, mode, bits, group)
        cases.compare(y.float().cpu().numpy().astype(np.float64), y_ref, bound_of(x, xdtype, Wt),
                      f"{mode}{bits} g{group} {xdtype} M{M} path {q.path(M, N, K, mode, bits, group)}")
    q.check_error()


def test_actorder_perm_reports_unequal_groups():
    K, g = 1024, 128
    gidx = _gidx(K, g, 83)
    gidx[5] = (gidx[5] + 1) % (K // g)       # one group short, one over
    with pytest.raises(ValueError):
        q.actorder_perm(torch.from_numpy(gidx).cuda(), g)
    gidx[5] = K // g                          # out of range: matches no group
    with pytest.raises(ValueError):
        q.actorder_perm(torch.from_numpy(gidx).cuda(), g)


def test_actorder_needs_workspace():
    import ctypes
    lib = q.load()
    fake = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    assert lib.qmm_actorder(vp(fake), 0, vp(fake), vp(fake), vp(fake), None, 1, 16, 1024, 4, 128,
                            0, vp(fake[2048:]), None, 0, None) == -6


# ------------------------------------------- full-size shapes, sampled rows
#
# The benchmark's shapes: every weight row is packed on the GPU, the oracle
# computes four sampled row blocks (the first, the last and two seeded ones);
# their bytes and their outputs are compared.

def _sampled_weights(N, K, sigma, seed):
    rows = cases.row_blocks(N, 4, seed + 1)
    W_rows = synth.weights(seed, "W", N, K, sigma, rows=rows)
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = torch.randn(N, K, generator=g, device="cuda") * sigma
    W[torch.from_numpy(rows).cuda()] = torch.from_numpy(W_rows).cuda()
    return rows, W_rows, W


def _blocks(buf, rows, per_block):
    blocks = np.unique(rows // 16)
    return np.concatenate([buf[b * per_block:(b + 1) * per_block] for b in blocks])


@pytest.mark.parametrize("K,N,group,zgroup,xdtype,Ms", [
    (4096, 14336, -1, 8, "f16", (1, 8, 32)),          # bench asym_rowscale_zg8_u4
    (8192, 57344, 128, 128, "bf16", (1, 16)),         # bench llama70b_asym_zq4_bf16
])
def test_zero_options_fullsize(K, N, group, zgroup, xdtype, Ms):
    rows, W_rows, W = _sampled_weights(N, K, 0.015, 90)
    qw, sc, ze = q.pack_asym(W, group, zgroup, 4)
    del W
    torch.cuda.synchronize()
    c, s_, z = oracle.quantize_asym(W_rows, group, zgroup)
    qw_o, sp_o, zp_o = oracle.pack_asym(c, s_, z, group, zgroup, 4)
    G, GZ = (1 if group == -1 else K // group), K // zgroup
    assert np.array_equal(_blocks(qw.cpu().numpy(), rows, K * 8), qw_o)
    assert np.array_equal(_blocks(sc.cpu().numpy().view(np.uint16), rows, 16 * G), sp_o)
    assert np.array_equal(_blocks(ze.cpu().numpy(), rows, 8 * GZ), zp_o)
    Wt = oracle.dequant_asym(c, s_, z, group, zgroup)
    for M in Ms:
        x = synth.activations(91 + M, "x", M, K, xdtype)
        ws = q.workspace_asym(M, N, K, group, zgroup, 4)
        y = q.qmm_asym(dev(x).view(tdtype(xdtype)), qw, sc, ze, N, K, group, zgroup, 4, ws=ws)
        torch.cuda.synchronize()
        y_ref = oracle.qmm_asym(x, xdtype, qw_o, sp_o, zp_o, M, len(rows), K, group, zgroup, 4)
        y_s = y[:, torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
        cases.compare(y_s, y_ref, bound_of(x, xdtype, Wt), f"zero options K{K} N{N} M{M}")
    q.check_error()


@pytest.mark.parametrize("K,N", [(4096, 22016), (11008, 4096)])
def test_actorder_fullsize(K, N):
    """bench actorder_llama7b shapes, on both paths (M = 1, 16 decode; 64 tensor for N > 4096)."""
    group = 128
    rows, W_rows, W = _sampled_weights(N, K, 0.02, 92)
    gidx = _gidx(K, group, 93)
    perm = q.actorder_perm(torch.from_numpy(gidx).cuda(), group)
    qw, sc, _ = q.pack_actorder(W, perm, "sym", 4, group)
    del W
    torch.cuda.synchronize()
    c, s_, _ = oracle.quantize_gidx(W_rows, "sym", 4, group, gidx)
    qw_o, sp_o, _ = oracle.pack_gidx(c, s_, None, gidx, "sym", 4, group)
    assert np.array_equal(_blocks(qw.cpu().numpy(), rows, K * 8), qw_o)
    assert np.array_equal(_blocks(sc.cpu().numpy().view(np.uint16), rows, 16 * (K // group)), sp_o)
    Wt = oracle.dequant_gidx(c, s_, None, "sym", 4, group, gidx)
    for M in (1, 16, 64):
        x = synth.activations(94 + M, "x", M, K, "f16")
        y = q.qmm_actorder(dev(x).view(torch.float16), perm, qw, sc, None, N, K, "sym", 4, group)
        torch.cuda.synchronize()
        y_ref = oracle.qmm_gidx(x, "f16", qw_o, sp_o, None, gidx, M, len(rows), K, "sym", 4, group)
        y_s = y[:, torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
        cases.compare(y_s, y_ref, bound_of(x, "f16", Wt), f"act-order K{K} N{N} M{M}")
    q.check_error()
