"""Pins for the oracle's zero-point options and act-order groups.

Zero-point options ("Does Marlin support zero-point quantization?", efrantar's
and mobicham's replies): zero-points stored as 4-bit integers, and a zero-point
group nested inside the scale group.  Act-order (GPTQ-Triton summary,
"Limitations & Caveats"): every column carries its group index g_idx.

Each function is checked against hand-worked values (tests/golden), against
the already-pinned plain oracle in the cases where the new one must reduce to
it, against library routines (numpy's stable argsort for the act-order column
placement, numpy matmul on the decoded weights) and against invariants
(permutation equivariance, y = 0 when every code sits at its zero-point).
"""
import numpy as np
import pytest

import oracle
from tests import golden_io as gio
from weight_only_quantized_int4_b200 import synth


def h2f(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


@pytest.fixture(scope="module")
def hz():
    return gio.read("hand_zero_groups_actorder.txt")


def _f(hz, name):
    return gio.floats(hz[name][0])


def _i(hz, name):
    return gio.ints(hz[name][0])


# ------------------------------------------------------ zero-point options

def test_hand_zero_group_8(hz):
    row = np.array([_f(hz, "zrow")], np.float32)
    codes, scales, zeros = oracle.quantize_asym(row, 16, 8)
    assert scales[0].tolist() == [_i(hz, "zrow_scale")[0]]
    assert zeros[0].tolist() == _i(hz, "zrow_zeros_z8")
    assert codes[0].tolist() == _i(hz, "zrow_q_z8")
    d = oracle.dequant_asym(codes, scales, zeros, 16, 8)
    assert d[0].tolist() == _f(hz, "zrow_d_z8")
    # one zero-point for the whole scale group
    c16, s16, z16 = oracle.quantize_asym(row, 16, 16)
    assert z16[0].tolist() == _i(hz, "zrow_zero_z16")
    assert c16[0].tolist() == _i(hz, "zrow_q_z16")


def _asym_problem(N, K, group, seed):
    W = synth.weights(seed, "w", N, K, 0.015)
    return W


@pytest.mark.parametrize("group", [64, 128, -1])
def test_same_zero_group_is_plain_asym(group):
    """zero group = scale group, fp16 zeros: exactly the plain asymmetric oracle."""
    N, K, M = 32, 256, 3
    W = _asym_problem(N, K, group, 31)
    c, s, z = oracle.quantize_asym(W, group, group)
    c0, s0, z0 = oracle.quantize(W, "asym", 4, group)
    assert np.array_equal(c, c0) and np.array_equal(s, s0) and np.array_equal(z, z0)
    qw, sp, zp = oracle.pack_asym(c, s, z, group, group, 16)
    qw0, sp0, zp0 = oracle.pack(c0, s0, z0, "asym", 4, group)
    assert np.array_equal(qw, qw0) and np.array_equal(sp, sp0)
    assert np.array_equal(zp, zp0.view(np.uint8))
    x = synth.activations(0, "x", M, K, "bf16")
    y = oracle.qmm_asym(x, "bf16", qw, sp, zp, M, N, K, group, group, 16)
    assert np.array_equal(y, oracle.qmm(x, "bf16", qw0, sp0, zp0, M, N, K, "asym", 4, group))


@pytest.mark.parametrize("group,zgroup", [(128, 8), (-1, 8), (-1, 32), (64, 16)])
def test_zero_bits_4_and_16_agree(group, zgroup):
    """The same integer zero-points stored in 4 bits or in fp16 decode alike."""
    N, K, M = 32, 256, 2
    W = _asym_problem(N, K, group, 32)
    c, s, z = oracle.quantize_asym(W, group, zgroup)
    qw16, sp16, zp16 = oracle.pack_asym(c, s, z, group, zgroup, 16)
    qw4, sp4, zp4 = oracle.pack_asym(c, s, z, group, zgroup, 4)
    assert np.array_equal(qw16, qw4) and np.array_equal(sp16, sp4)
    assert zp4.size * 4 == zp16.size
    x = synth.activations(1, "x", M, K, "f16")
    y16 = oracle.qmm_asym(x, "f16", qw16, sp16, zp16, M, N, K, group, zgroup, 16)
    y4 = oracle.qmm_asym(x, "f16", qw4, sp4, zp4, M, N, K, group, zgroup, 4)
    assert np.array_equal(y16, y4)
    # and the qmm from packed buffers is x . W~^T (numpy matmul on the decoded weights)
    Wt = oracle.dequant_asym(c, s, z, group, zgroup)
    xv = oracle.widen(x, "f16")
    assert np.allclose(y4, xv @ Wt.T, rtol=1e-12, atol=1e-12 * np.abs(xv).sum(1).max())


def test_zero_nibble_hand_position(hz):
    N, K, zg = 16, 64, 8
    codes = np.zeros((N, K), np.uint8)
    scales = np.full((N, 1), 0x3C00, np.uint16)
    zeros = np.zeros((N, K // zg), np.uint16)
    r, gi = _i(hz, "zq_row")[0], _i(hz, "zq_group")[0]
    zeros[r, gi] = 0x4980        # 11.0
    _, _, zp = oracle.pack_asym(codes, scales, zeros, -1, zg, 4)
    b, sh = _i(hz, "zq_byte")[0], _i(hz, "zq_shift")[0]
    assert zp[b] == 11 << sh
    assert np.count_nonzero(zp) == 1
    # a zero-point that is not an integer in [0, 15] has no 4-bit form
    zeros[r, gi] = 0x3800        # 0.5
    with pytest.raises(ValueError):
        oracle.pack_asym(codes, scales, zeros, -1, zg, 4)


def test_zero_group_codes_at_zero_point_give_zero():
    N, K, M, zg = 32, 128, 3, 8
    rng = np.random.default_rng(5)
    z = rng.integers(0, 16, (N, K // zg))
    codes = np.repeat(z, zg, axis=1).astype(np.uint8)
    scales = np.full((N, 1), 0x3C00, np.uint16)
    zeros = oracle.round_to(z.astype(np.float64), "f16")
    for zbits in (16, 4):
        qw, sp, zp = oracle.pack_asym(codes, scales, zeros, -1, zg, zbits)
        y = oracle.qmm_asym(synth.activations(0, "x", M, K, "f16"), "f16", qw, sp, zp, M, N, K,
                            -1, zg, zbits)
        assert np.all(y == 0.0)
    # moving one zero-point by one makes exactly that group's columns non-zero
    zeros2 = zeros.copy()
    zeros2[3, 5] = oracle.round_to(np.array([z[3, 5] + 1.0]), "f16")[0]
    qw, sp, zp = oracle.pack_asym(codes, scales, zeros2, -1, zg, 16)
    d = oracle.dequant_asym(codes, scales, zeros2, -1, zg)
    assert np.count_nonzero(d) == zg and np.all(d[3, 40:48] == -1.0)


def test_zero_group_rounding_bound():
    """|w - w~| <= s/2 wherever the code is not at a clamp, <= 1.5 s everywhere
    (data with min <= 0 <= max in every scale group)."""
    N, K = 64, 512
    W = _asym_problem(N, K, -1, 33)
    for group, zg in ((-1, 8), (128, 16), (256, 32)):
        c, s, z = oracle.quantize_asym(W, group, zg)
        d = oracle.dequant_asym(c, s, z, group, zg)
        L = K if group == -1 else group
        sv = np.repeat(h2f(s), L, axis=1)
        err = np.abs(W.astype(np.float64) - d)
        inner = (c > 0) & (c < 15)
        assert np.all(err[inner] <= sv[inner] / 2 * (1 + 1e-6))
        assert np.all(err <= 1.5 * sv)
        # a zero group's own zero-point: the group's minimum maps to code 0 or
        # (when the group is all positive) the group's codes start at rint(min/s)
        zmin = W.reshape(N, K // zg, zg).min(axis=2)
        zv = h2f(z)
        sg = np.repeat(h2f(s), L // zg, axis=1)
        expect = np.clip(np.rint(-zmin / sg), 0, 15)
        assert np.array_equal(zv, expect)


# ------------------------------------------------------------ act-order

def test_hand_actorder_groups(hz):
    row = np.array([_f(hz, "arow")], np.float32)
    gidx = np.array(_i(hz, "arow_gidx"))
    codes, scales, _ = oracle.quantize_gidx(row, "sym", 4, 4, gidx)
    assert scales[0].tolist() == _i(hz, "arow_scales")
    assert codes[0].tolist() == _i(hz, "arow_q")
    d = oracle.dequant_gidx(codes, scales, None, "sym", 4, 4, gidx)
    assert d[0].tolist() == _f(hz, "arow_d")
    assert d[0].sum() == _f(hz, "arow_sum")[0]
    _, s_nat, _ = oracle.quantize(row, "sym", 4, 4)
    assert s_nat[0].tolist() == _i(hz, "arow_natural_scales")
    assert np.argsort(gidx, kind="stable").tolist() == _i(hz, "arow_perm")


def _gidx(K, group, seed):
    """GPTQ act-order g_idx: a random column order, groups along it."""
    order = np.random.default_rng(seed).permutation(K)
    gidx = np.empty(K, np.int32)
    gidx[order] = np.arange(K) // group
    return gidx


@pytest.mark.parametrize("mode,bits", [("sym", 4), ("asym", 4), ("lut", 4), ("lut", 2)])
def test_natural_gidx_is_plain(mode, bits):
    """g_idx[k] = k / group reduces every act-order function to the plain one."""
    N, K, M, g = 32, 256, 3, 64
    W = synth.weights(40, "w", N, K, 0.02)
    lut = synth.nf4_table() if (mode == "lut" and bits == 4) else (
        synth.lut2_table(0) if mode == "lut" else None)
    gidx = np.arange(K) // g
    c, s, z = oracle.quantize_gidx(W, mode, bits, g, gidx, lut=lut)
    c0, s0, z0 = oracle.quantize(W, mode, bits, g, lut=lut)
    assert np.array_equal(c, c0) and np.array_equal(s, s0)
    if mode == "asym":
        assert np.array_equal(z, z0)
    zl = z if mode == "asym" else lut
    assert np.array_equal(oracle.dequant_gidx(c, s, zl, mode, bits, g, gidx),
                          oracle.dequant(c0, s0, zl, mode, bits, g))
    qw, sp, zp = oracle.pack_gidx(c, s, z, gidx, mode, bits, g)
    qw0, sp0, zp0 = oracle.pack(c0, s0, z0, mode, bits, g)
    assert np.array_equal(qw, qw0) and np.array_equal(sp, sp0)
    x = synth.activations(0, "x", M, K, "f16")
    zlp = zp if mode == "asym" else lut
    assert np.array_equal(oracle.qmm_gidx(x, "f16", qw, sp, zlp, gidx, M, N, K, mode, bits, g),
                          oracle.qmm(x, "f16", qw0, sp0, zlp, M, N, K, mode, bits, g))


@pytest.mark.parametrize("mode,group", [("sym", 64), ("asym", 128), ("lut", 32)])
def test_actorder_quantize_is_permutation_equivariant(mode, group):
    """Quantizing W[:, pi] with g_idx[pi] gives the codes [:, pi] and the same
    scales: a group is a set of columns, its order is immaterial."""
    N, K = 32, 256
    W = synth.weights(41, "w", N, K, 0.02)
    lut = synth.nf4_table() if mode == "lut" else None
    gidx = _gidx(K, group, 7)
    pi = np.random.default_rng(8).permutation(K)
    c, s, z = oracle.quantize_gidx(W, mode, 4, group, gidx, lut=lut)
    c2, s2, z2 = oracle.quantize_gidx(W[:, pi], mode, 4, group, gidx[pi], lut=lut)
    assert np.array_equal(c2, c[:, pi]) and np.array_equal(s2, s)
    if mode == "asym":
        assert np.array_equal(z2, z)
    # and it is the plain quantizer on the columns sorted by group
    perm = np.argsort(gidx, kind="stable")
    c0, s0, z0 = oracle.quantize(W[:, perm], mode, 4, group, lut=lut)
    assert np.array_equal(c0, c[:, perm]) and np.array_equal(s0, s)


@pytest.mark.parametrize("mode,bits,group", [("sym", 4, 64), ("asym", 4, 128), ("lut", 4, 32),
                                             ("lut", 3, 64), ("sym", 4, -1)])
def test_actorder_pack_and_qmm(mode, bits, group):
    """Packed bytes = the plain packing of the codes with their columns sorted
    by group (numpy's stable argsort gives the order); qmm from those bytes is
    x . W~^T over the original columns."""
    N, K, M = 32, 256, 4
    W = synth.weights(42, "w", N, K, 0.02)
    lut = {4: synth.nf4_table(), 3: synth.nf3_table(), 2: synth.lut2_table(0)}[bits] \
        if mode == "lut" else None
    gidx = _gidx(K, K if group == -1 else group, 9)
    c, s, z = oracle.quantize_gidx(W, mode, bits, group, gidx, lut=lut)
    qw, sp, zp = oracle.pack_gidx(c, s, z, gidx, mode, bits, group)
    perm = np.argsort(gidx, kind="stable")
    qw0, sp0, zp0 = oracle.pack(c[:, perm], s, z, mode, bits, group)
    assert np.array_equal(qw, qw0) and np.array_equal(sp, sp0)
    x = synth.activations(2, "x", M, K, "bf16")
    zl = z if mode == "asym" else lut
    zlp = zp if mode == "asym" else lut
    y = oracle.qmm_gidx(x, "bf16", qw, sp, zlp, gidx, M, N, K, mode, bits, group)
    Wt = oracle.dequant_gidx(c, s, zl, mode, bits, group, gidx)
    xv = oracle.widen(x, "bf16")
    assert np.allclose(y, xv @ Wt.T, rtol=1e-12, atol=1e-12 * np.abs(xv).sum(1).max())
    # the same sums as the plain oracle on the column-permuted activations
    y0 = oracle.qmm(x[:, perm], "bf16", qw0, sp0, zlp, M, N, K, mode, bits, group)
    assert np.allclose(y, y0, rtol=1e-12, atol=1e-12 * np.abs(xv).sum(1).max())
    if group != -1:   # one group: every order is the natural one
        assert not np.allclose(y, oracle.qmm(x, "bf16", qw0, sp0, zlp, M, N, K, mode, bits, group))


def test_actorder_rejects_unequal_groups():
    N, K, g = 16, 64, 16
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((N, K // g), np.uint16)
    gidx = np.arange(K) // g
    gidx[0] = 1                    # group 0 has 15 columns, group 1 has 17
    with pytest.raises(ValueError):
        oracle.pack_gidx(codes, scales, None, gidx, "sym", 4, g)
    gidx[0] = K // g               # out of range
    with pytest.raises(ValueError):
        oracle.dequant_gidx(codes, scales, None, "sym", 4, g, gidx)
