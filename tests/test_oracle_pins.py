"""Pins for the CPU oracle: it is checked against hand-worked values, library
routines, brute force and invariants -- never against itself or the GPU.

A plausible mistake in the oracle (a dropped zero-point, a wrong sign, a
transposed operand, a misplaced nibble, round-half-up instead of half-even,
an fp32 scale where the fp16 one belongs) fails at least one test here.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import golden_io as gio
from weight_only_quantized_int4_b200 import synth


def h2f(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------- hand cases

@pytest.fixture(scope="module")
def hq():
    return gio.read("hand_quantize_4x8.txt")


def _rows(hq, *names):
    return np.array([gio.floats(hq[n][0]) for n in names], np.float32)


def test_hand_sym_g8(hq):
    W = _rows(hq, "w0", "w1", "w2", "w3")
    codes, scales, zeros = oracle.quantize(W, "sym", 4, 8)
    assert zeros is None
    assert scales[:, 0].tolist() == gio.ints(hq["sym_g8_scales"][0])
    for i in range(4):
        assert codes[i].tolist() == gio.ints(hq[f"sym_g8_q{i}"][0]), i
    d = oracle.dequant(codes, scales, None, "sym", 4, 8)
    assert d[0].tolist() == gio.floats(hq["sym_g8_d0"][0])
    assert d[3].tolist() == gio.floats(hq["sym_g8_d3"][0])
    assert not d[2].any()


def test_hand_group_minus_one_vs_8(hq):
    row = np.concatenate([_rows(hq, "w0")[0], _rows(hq, "w3")[0]])[None, :]
    c8, s8, _ = oracle.quantize(row, "sym", 4, 8)
    assert s8[0].tolist() == [0x2C00, 0x3800]
    assert c8[0].tolist() == gio.ints(hq["sym_g8_q0"][0]) + gio.ints(hq["sym_g8_q3"][0])
    c1, s1, _ = oracle.quantize(row, "sym", 4, -1)
    assert s1.shape == (1, 1)
    assert s1[0, 0] == int(hq["sym_row16_gm1_scale"][0][0], 0)
    assert c1[0].tolist() == gio.ints(hq["sym_row16_gm1_q"][0])


def test_hand_asym_g8(hq):
    W = _rows(hq, "w0", "w1", "w2", "w3")
    codes, scales, zeros = oracle.quantize(W, "asym", 4, 8)
    assert scales[:, 0].tolist() == gio.ints(hq["asym_g8_scales"][0])
    assert zeros[:, 0].tolist() == gio.ints(hq["asym_g8_zeros"][0])
    for i in range(4):
        assert codes[i].tolist() == gio.ints(hq[f"asym_g8_q{i}"][0]), i
    P = _rows(hq, "asym_pos")
    c, s, z = oracle.quantize(P, "asym", 4, 8)
    assert s[0, 0] == int(hq["asym_pos_scale"][0][0], 0)
    assert z[0, 0] == int(hq["asym_pos_zero"][0][0], 0)
    assert c[0].tolist() == gio.ints(hq["asym_pos_q"][0])
    # decode (q - z) s
    d = oracle.dequant(codes, scales, zeros, "asym", 4, 8)
    s1 = h2f(scales[1, 0])
    assert d[1].tolist() == [(q - 8) * s1 for q in gio.ints(hq["asym_g8_q1"][0])]


def test_hand_lut4_g8(hq):
    T = np.array(gio.floats(hq["lut4_table"][0]), np.float16).view(np.uint16)
    W = _rows(hq, "w0", "w1", "w2", "w3")
    codes, scales, _ = oracle.quantize(W, "lut", 4, 8, lut=T)
    assert scales[:, 0].tolist() == gio.ints(hq["lut4_g8_scales"][0])
    for i in range(4):
        assert codes[i].tolist() == gio.ints(hq[f"lut4_g8_q{i}"][0]), i
    c, s, _ = oracle.quantize(_rows(hq, "lut4_tie"), "lut", 4, 8, lut=T)
    assert s[0, 0] == int(hq["lut4_tie_scale"][0][0], 0)
    assert c[0].tolist() == gio.ints(hq["lut4_tie_q"][0])
    d = oracle.dequant(c, s, T, "lut", 4, 8)
    assert d[0].tolist() == [h2f(T[q]) * 2.0 for q in c[0]]


def test_hand_lut2(hq):
    T = np.array(gio.floats(hq["lut2_table"][0]), np.float16).view(np.uint16)
    c, s, _ = oracle.quantize(_rows(hq, "lut2_row"), "lut", 2, 8, lut=T)
    assert s[0, 0] == int(hq["lut2_scale"][0][0], 0)
    assert c[0].tolist() == gio.ints(hq["lut2_q"][0])


def test_hand_qmm_sym_g8(hq):
    """The 4x8 SYM case embedded in a 16x64 matrix and quantized with group 16
    (the packed layout's smallest group): each row's first group is the 8 hand
    values plus 8 zeros, so absmax, scale and codes are the group-8 ones, the
    zeros get q = 8, and every later group is all zero and decodes to 0."""
    hy = gio.read("hand_qmm_sym_g8.txt")
    W = np.zeros((16, 64), np.float32)
    W[:4, :8] = _rows(hq, "w0", "w1", "w2", "w3")
    codes, scales, _ = oracle.quantize(W, "sym", 4, 16)
    assert scales[:4, 0].tolist() == gio.ints(hq["sym_g8_scales"][0])
    qw, sp, _ = oracle.pack(codes, scales, None, "sym", 4, 16)
    x = np.zeros((2, 64), np.float16)
    x[0, :8] = gio.floats(hy["x0"][0])
    x[1, :8] = gio.floats(hy["x1"][0])
    y = oracle.qmm(x.view(np.uint16), "f16", qw, sp, None, 2, 16, 64, "sym", 4, 16)
    assert y[0, :4].tolist() == gio.floats(hy["y0"][0])
    assert y[1, :4].tolist() == gio.floats(hy["y1"][0])
    assert not y[:, 4:].any()


def test_hand_layout():
    hl = gio.read("hand_layout.txt")
    for N, K, bits, mode, n, k, code, byte, val in hl["case"]:
        N, K, bits, n, k, code, byte = map(int, (N, K, bits, n, k, code, byte))
        codes = np.zeros((N, K), np.uint8)
        codes[n, k] = code
        G = K // 16
        scales = np.zeros((N, G), np.uint16)
        zeros = np.zeros((N, G), np.uint16) if mode == "asym" else None
        qw, _, _ = oracle.pack(codes, scales, zeros, mode, bits, 16)
        expect = np.zeros(N * K * bits // 8, np.uint8)
        expect[byte] = int(val, 16)
        assert np.array_equal(qw, expect), (mode, n, k, np.nonzero(qw))
        back, _, _ = oracle.unpack(qw, None, None, N, K, mode, bits, 16)
        assert np.array_equal(back, codes)
    for n, gi, G, idx in hl["scale_case"]:
        n, gi, G, idx = map(int, (n, gi, G, idx))
        N, K = ((n // 16) + 1) * 16, 64 * G
        scales = np.zeros((N, G), np.uint16)
        scales[n, gi] = 0x3C00
        _, sp, _ = oracle.pack(np.zeros((N, K), np.uint8), scales, None, "sym", 4, 64)
        assert np.nonzero(sp)[0].tolist() == [idx]


# ------------------------------------------------------ conversions vs libraries

def _edge_values():
    rng = np.random.default_rng(1)
    v = [rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000)]
    # exact fp16 ties: midpoints between neighbouring halves, incl. subnormals
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo, hi = h.view(np.float16).astype(np.float64), (h + 1).view(np.float16).astype(np.float64)
    v.append((lo + hi) / 2)
    v.append(np.array([65504.0, 65519.99, 65520.0, 7e4, 2.0 ** -24, 2.0 ** -25,
                       3 * 2.0 ** -26, 0.0, -0.0, 1 / 7]))
    return np.concatenate([v[0], v[1], -v[1], v[2]])


def test_fp16_rounding_matches_numpy():
    v = _edge_values()
    ours = oracle.round_to(v, "f16")
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)       # IEEE RNE in numpy
    assert np.array_equal(ours, ref)


def test_bf16_rounding_matches_torch():
    v = _edge_values().astype(np.float32).astype(np.float64)   # fp32 inputs
    ours = oracle.round_to(v, "bf16")
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours, ref.view(np.uint16))


def test_widen_all_fp16_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen(bits, "f16")
    ref = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_widen_bf16_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])


# ------------------------------------------------------------ brute force

def _rand_w(N, K, sigma, seed):
    return synth.weights(seed, "pin", N, K, sigma)


@pytest.mark.parametrize("group", [16, 64, -1])
def test_sym_codes_are_nearest_grid_points(group):
    W = _rand_w(32, 128, 0.02, 3)
    codes, scales, _ = oracle.quantize(W, "sym", 4, group)
    G = scales.shape[1]
    s = h2f(scales)[:, np.repeat(np.arange(G), 128 // G)]
    grid = (np.arange(16)[None, None, :] - 8) * s[:, :, None]          # every code's value
    err = np.abs(W.astype(np.float64)[:, :, None] - grid)
    chosen = np.take_along_axis(err, codes[:, :, None].astype(np.int64), 2)[..., 0]
    assert np.all(chosen <= err.min(axis=2) + 1e-6 * s)
    # |w - w~| <= s/2 (up to the fp16 scale's rounding): s = absmax/7 keeps w/s in range
    d = oracle.dequant(codes, scales, None, "sym", 4, group)
    assert np.all(np.abs(W - d) <= 0.5 * s * (1 + 2.0 ** -9))


def test_asym_codes_are_nearest_grid_points():
    W = _rand_w(32, 256, 0.015, 4)
    codes, scales, zeros = oracle.quantize(W, "asym", 4, 128)
    s = np.repeat(h2f(scales), 128, axis=1)
    z = np.repeat(h2f(zeros), 128, axis=1)
    assert np.all(z == np.round(z)) and z.min() >= 0 and z.max() <= 15
    grid = (np.arange(16)[None, None, :] - z[:, :, None]) * s[:, :, None]
    err = np.abs(W.astype(np.float64)[:, :, None] - grid)
    chosen = np.take_along_axis(err, codes[:, :, None].astype(np.int64), 2)[..., 0]
    assert np.all(chosen <= err.min(axis=2) + 1e-6 * s)
    # the group's min and max land within one step of the grid ends
    Wg = W.reshape(32, 2, 128)
    lo = (0 - h2f(zeros)) * h2f(scales)
    hi = (15 - h2f(zeros)) * h2f(scales)
    assert np.all(np.abs(Wg.min(axis=2) - lo) <= h2f(scales) * 0.51)
    assert np.all(Wg.max(axis=2) <= hi + h2f(scales) * 0.51)


@pytest.mark.parametrize("bits", [4, 3, 2])
def test_lut_codes_are_nearest_entries(bits):
    T = {4: synth.nf4_table(), 3: synth.nf3_table(), 2: synth.lut2_table(0)}[bits]
    W = _rand_w(32, 128, 0.02, 5)
    codes, scales, _ = oracle.quantize(W, "lut", bits, 64, lut=T)
    s = np.repeat(h2f(scales).astype(np.float32), 64, axis=1)
    u = (W / s).astype(np.float32)                                      # fp32 division
    dist = np.abs(u[:, :, None] - h2f(T).astype(np.float32)[None, None, :])
    best = dist.min(axis=2)
    chosen = np.take_along_axis(dist, codes[:, :, None].astype(np.int64), 2)[..., 0]
    assert np.array_equal(chosen, best)
    # lowest index among equals: no smaller index attains the minimum
    first = np.argmax(dist == best[:, :, None], axis=2)
    assert np.array_equal(first, codes)
    absmax = np.abs(W).reshape(32, 2, 64).max(axis=2)
    assert np.array_equal(scales, absmax.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------- layout & packing

@pytest.mark.parametrize("bits,mode", [(4, "sym"), (4, "lut"), (2, "lut")])
def test_layout_is_a_bijection(bits, mode):
    """Every (n, k) gets its own bit field and every bit of the buffer is used."""
    N, K = 32, 256
    seen = np.zeros(N * K * bits // 8 * 8, np.int32)
    qmax = (1 << bits) - 1
    for n in range(0, N, 3):
        for k in range(0, K, 5):
            codes = np.zeros((N, K), np.uint8)
            codes[n, k] = qmax
            qw, _, _ = oracle.pack(codes, np.zeros((N, K // 64), np.uint16), None, mode, bits, 64)
            on = np.nonzero(np.unpackbits(qw, bitorder="little"))[0]
            assert len(on) == bits
            assert on[-1] - on[0] == bits - 1 and on[0] % bits == 0
            seen[on] += 1
    assert seen.max() == 1
    # full coverage: all codes at max set every bit
    qw, _, _ = oracle.pack(np.full((N, K), qmax, np.uint8), np.zeros((N, 4), np.uint16), None,
                           mode, bits, 64)
    assert np.all(qw == 0xFF)


def test_layout3_fields_and_bijection():
    """3-bit codes: every code owns three consecutive bits of its lane's 24
    bytes; the two members of a pair are adjacent (one 6-bit field, the lower
    column first); no bit is shared and all bits are used."""
    N, K = 32, 256
    seen = np.zeros(N * K * 3, np.int32)
    for n in range(0, N, 3):
        for k in range(0, K, 5):
            codes = np.zeros((N, K), np.uint8)
            codes[n, k] = 7
            qw, _, _ = oracle.pack(codes, np.zeros((N, K // 64), np.uint16), None, "lut", 3, 64)
            on = np.nonzero(np.unpackbits(qw, bitorder="little"))[0]
            assert len(on) == 3 and on[1] == on[0] + 1 and on[2] == on[0] + 2
            # the lane's string: 192 bits starting at a multiple of 192
            assert (on[0] // 192) == (on[2] // 192)
            seen[on] += 1
            if k % 2 == 0:   # the pair's other member (column k + 1) follows
                codes[n, k + 1] = 7
                qw2, _, _ = oracle.pack(codes, np.zeros((N, K // 64), np.uint16), None, "lut",
                                        3, 64)
                on2 = np.nonzero(np.unpackbits(qw2, bitorder="little"))[0]
                assert list(on2) == list(range(on[0], on[0] + 6))
    assert seen.max() == 1
    qw, _, _ = oracle.pack(np.full((N, K), 7, np.uint8), np.zeros((N, 4), np.uint16), None,
                           "lut", 3, 64)
    assert np.all(qw == 0xFF)


def test_layout3_hand_position():
    """Code 5 (binary 101) at row 9, column 21, worked out from the layout's
    definition: g = 1, h = 1, tile j = 1, t = 1, c = 1 -> lane 5 (bytes
    120..143 of chunk 0, bits 960..1151), pair p = 1, member 1: bit 960 + 24 j
    + 6 p + 3 = 993 = byte 124 bit 1, so bits 1 and 3 of byte 124 are set."""
    N, K = 16, 128
    codes = np.zeros((N, K), np.uint8)
    codes[9, 21] = 5
    qw, _, _ = oracle.pack(codes, np.zeros((N, 2), np.uint16), None, "lut", 3, 64)
    expect = np.zeros(N * K * 3 // 8, np.uint8)
    expect[124] = 0x0A
    assert np.array_equal(qw, expect)


@pytest.mark.parametrize("bits,mode", [(4, "sym"), (4, "asym"), (4, "lut"), (3, "lut"),
                                       (2, "lut")])
def test_pack_unpack_round_trip(bits, mode):
    rng = np.random.default_rng(7)
    N, K, g = 48, 384, 128
    G = K // g
    codes = rng.integers(0, 1 << bits, (N, K)).astype(np.uint8)
    scales = rng.integers(0, 0x7BFF, (N, G)).astype(np.uint16)
    zeros = rng.integers(0, 16, (N, G)).astype(np.uint16) if mode == "asym" else None
    qw, sp, zp = oracle.pack(codes, scales, zeros, mode, bits, g)
    assert qw.size == N * K * bits // 8
    c2, s2, z2 = oracle.unpack(qw, sp, zp, N, K, mode, bits, g)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    if mode == "asym":
        assert np.array_equal(z2, zeros)
    raw = rng.integers(0, 256, qw.size).astype(np.uint8)
    c3, _, _ = oracle.unpack(raw, None, None, N, K, mode, bits, g)
    qw3, _, _ = oracle.pack(c3, scales, zeros, mode, bits, g)
    assert np.array_equal(qw3, raw)


# ---------------------------------------------------------------- matmul

def _problem(mode, bits, group, M, N, K, seed, xdtype="f16"):
    W = _rand_w(N, K, 0.02, seed)
    lut = None
    if mode == "lut":
        lut = {4: synth.nf4_table(), 3: synth.nf3_table(), 2: synth.lut2_table(0)}[bits]
    codes, scales, zeros = oracle.quantize(W, mode, bits, group, lut=lut)
    qw, sp, zp = oracle.pack(codes, scales, zeros, mode, bits, group)
    x = synth.activations(seed, "x", M, K, xdtype)
    zl = zp if mode == "asym" else lut
    return dict(codes=codes, scales=scales, zeros=zeros, lut=lut, qw=qw, sp=sp, zl=zl, x=x)


@pytest.mark.parametrize("mode,bits,group,xdt", [("sym", 4, 128, "f16"), ("sym", 4, -1, "f16"),
                                                 ("asym", 4, 64, "bf16"), ("lut", 4, 64, "f16"),
                                                 ("lut", 3, 64, "f16"), ("lut", 2, 64, "f16")])
def test_qmm_matches_numpy_matmul(mode, bits, group, xdt):
    """x . W~^T through numpy's matmul (a library routine) on the decoded weights."""
    M, N, K = 5, 48, 256
    p = _problem(mode, bits, group, M, N, K, 11, xdt)
    zl = p["zeros"] if mode == "asym" else p["lut"]
    Wt = oracle.dequant(p["codes"], p["scales"], zl, mode, bits, group)
    xv = oracle.widen(p["x"], xdt)
    ref = xv @ Wt.T
    y = oracle.qmm(p["x"], xdt, p["qw"], p["sp"], p["zl"], M, N, K, mode, bits, group)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(xv).sum(1).max())
    # a transposed or shifted operand would not survive a brute-force element
    m, n = 3, 17
    assert abs(y[m, n] - sum(xv[m, k] * Wt[n, k] for k in range(K))) <= 1e-12


def test_qmm_column_range():
    p = _problem("sym", 4, 128, 3, 64, 256, 12)
    full = oracle.qmm(p["x"], "f16", p["qw"], p["sp"], None, 3, 64, 256, "sym", 4, 128)
    part = oracle.qmm(p["x"], "f16", p["qw"], p["sp"], None, 3, 64, 256, "sym", 4, 128, 16, 40)
    assert np.array_equal(full[:, 16:40], part)


@pytest.mark.parametrize("mode", ["sym", "asym"])
def test_all_codes_at_zero_point_give_zero(mode):
    M, N, K, g = 4, 32, 128, 64
    codes = np.full((N, K), 8, np.uint8)
    scales = np.full((N, K // g), 0x3C00, np.uint16)
    zeros = None
    if mode == "asym":
        z = np.random.default_rng(2).integers(0, 16, (N, K // g))
        codes = np.repeat(z, g, axis=1).astype(np.uint8)
        zeros = oracle.round_to(z.astype(np.float64), "f16")
    qw, sp, zp = oracle.pack(codes, scales, zeros, mode, 4, g)
    x = synth.activations(0, "x", M, K, "f16")
    y = oracle.qmm(x, "f16", qw, sp, zp, M, N, K, mode, 4, g)
    assert np.all(y == 0.0)


def test_linearity_in_scale():
    M, N, K, g = 3, 32, 256, 128
    p = _problem("sym", 4, g, M, N, K, 13)
    y1 = oracle.qmm(p["x"], "f16", p["qw"], p["sp"], None, M, N, K, "sym", 4, g)
    s2 = oracle.round_to(h2f(p["sp"]) * 4.0, "f16")           # exact: power of two
    y4 = oracle.qmm(p["x"], "f16", p["qw"], s2, None, M, N, K, "sym", 4, g)
    assert np.array_equal(y4, 4.0 * y1)
    s3 = oracle.round_to(h2f(p["sp"]) * 0.75, "f16")
    y3 = oracle.qmm(p["x"], "f16", p["qw"], s3, None, M, N, K, "sym", 4, g)
    # 0.75 s is rounded to fp16 again: each term moves by at most 2^-11 of itself
    Wt = oracle.dequant(p["codes"], p["scales"], None, "sym", 4, g)
    bound = 0.75 * 2.0 ** -11 * (np.abs(oracle.widen(p["x"], "f16")) @ np.abs(Wt).T)
    assert np.all(np.abs(y3 - 0.75 * y1) <= bound * (1 + 1e-9))
    assert not np.array_equal(y3, 0.75 * y1)


def test_lut_with_integer_table_equals_sym():
    """LUT mode with T[i] = i - 8 and the SYM codes/scales reproduces SYM exactly."""
    M, N, K, g = 4, 32, 256, 64
    p = _problem("sym", 4, g, M, N, K, 14)
    T = np.arange(-8, 8).astype(np.float16).view(np.uint16)
    qw_l, sp_l, _ = oracle.pack(p["codes"], p["scales"], None, "lut", 4, g)
    ys = oracle.qmm(p["x"], "f16", p["qw"], p["sp"], None, M, N, K, "sym", 4, g)
    yl = oracle.qmm(p["x"], "f16", qw_l, sp_l, T, M, N, K, "lut", 4, g)
    assert np.array_equal(ys, yl)


def test_integer_weights_reduce_to_exact_matmul():
    """With s = 1 every W~ is the small integer q - 8 and x is fp16: the products
    and sums are exact in double, so the result equals torch's fp64 matmul."""
    M, N, K = 6, 32, 128
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    scales = np.full((N, 1), 0x3C00, np.uint16)
    qw, sp, _ = oracle.pack(codes, scales, None, "sym", 4, -1)
    x = rng.integers(-64, 64, (M, K)).astype(np.float16)
    y = oracle.qmm(x.view(np.uint16), "f16", qw, sp, None, M, N, K, "sym", 4, -1)
    ref = torch.from_numpy(x.astype(np.float64)) @ torch.from_numpy(codes.astype(np.float64) - 8).T
    assert np.array_equal(y, ref.numpy())


# ---------------------------------------------------------------- inputs

def test_generator_is_counter_based():
    a = synth.normal_rows(0, "w", 40, 96)
    b = synth.normal_rows(0, "w", 40, 96, rows=[3, 17, 39])
    assert np.array_equal(a[[3, 17, 39]], b)
    assert not np.array_equal(a, synth.normal_rows(0, "x", 40, 96))
    big = synth.normal_rows(0, "w", 512, 1024)
    assert abs(big.mean()) < 0.01 and abs(big.std() - 1) < 0.01


def test_tables():
    t = h2f(synth.nf4_table())
    assert t[0] == -1.0 and t[-1] == 1.0 and np.all(np.diff(t) > 0)
    assert np.array_equal(t, -t[::-1])
    t2 = h2f(synth.lut2_table(0))
    assert np.all(np.diff(t2) > 0) and np.max(np.abs(t2)) == 1.0
    t3 = h2f(synth.nf3_table())
    assert len(t3) == 8 and t3[0] == -1.0 and t3[-1] == 1.0 and np.all(np.diff(t3) > 0)
    assert np.array_equal(t3, -t3[::-1])
    # T[5] = q(5.5 / 8) / q(7.5 / 8) with q the normal quantile (values from scipy)
    assert abs(t3[5] - 0.48877641 / 1.53412054) < 1e-3


# ------------------------------------------------- fused feed-forward gate

def _negate_f16(x):
    """-x for fp16 bit patterns (flip the sign bit: exact)."""
    return (np.asarray(x, np.uint16) ^ np.uint16(0x8000)).astype(np.uint16)


@pytest.mark.parametrize("mode,bits,group", [("sym", 4, 128), ("asym", 4, 64), ("lut", 4, 64)])
def test_gated_odd_even_identity(mode, bits, group):
    """silu(g) u + silu(-g) (-u) = g u for any g, u (silu(v) - silu(-v) = v), so
    gated(x) + gated(-x) equals the product of the plain sums of the gate and
    up rows.  The interleave (which packed rows are the gate and the up rows of
    output i) and the composition are checked against the pinned plain oracle;
    the exponential cancels out."""
    M, I, K = 3, 32, 256
    p = _problem(mode, bits, group, M, 2 * I, K, 21)
    x = p["x"]
    g_plus = oracle.qmm_gated(x, "f16", p["qw"], p["sp"], p["zl"], M, I, K, mode, bits, group)
    g_minus = oracle.qmm_gated(_negate_f16(x), "f16", p["qw"], p["sp"], p["zl"], M, I, K, mode,
                               bits, group)
    y = oracle.qmm(x, "f16", p["qw"], p["sp"], p["zl"], M, 2 * I, K, mode, bits, group)
    gate = np.concatenate([y[:, 32 * b: 32 * b + 16] for b in range(I // 16)], axis=1)
    up = np.concatenate([y[:, 32 * b + 16: 32 * b + 32] for b in range(I // 16)], axis=1)
    assert np.allclose(g_plus + g_minus, gate * up, rtol=1e-9, atol=1e-12)


def test_gated_gate_and_up_roles():
    """Gate rows with a large negative sum switch the output off (silu -> 0);
    a large positive one passes the up sum through (silu(v) -> v); a zero gate
    gives exactly 0.  Swapping gate and up would break each of these."""
    I, K, g = 48, 128, 128
    x = oracle.round_to(np.ones((1, K)), "f16")
    codes = np.full((2 * I, K), 8, np.uint8)
    blocks = [slice(32 * b, 32 * b + 16) for b in range(I // 16)]
    ups = [slice(32 * b + 16, 32 * b + 32) for b in range(I // 16)]
    codes[blocks[0]] = 0          # outputs 0..15: gate sum -8 K s = -1024 s
    codes[blocks[1]] = 15         # outputs 16..31: gate sum +7 K s
    codes[blocks[2]] = 8          # outputs 32..47: gate sum 0
    for u in ups:
        codes[u] = 11             # up sum +3 K s
    scales = np.full((2 * I, 1), 0x3C00, np.uint16)     # s = 1
    qw, sp, _ = oracle.pack(codes, scales, None, "sym", 4, g)
    y = oracle.qmm_gated(x, "f16", qw, sp, None, 1, I, K, "sym", 4, g)[0]
    up = 3.0 * K
    assert np.all(np.abs(y[0:16]) < 1e-300 * up + 1e-200)          # silu(-1024) ~ -1024 e^-1024
    assert np.allclose(y[16:32], 7.0 * K * up, rtol=1e-12)         # silu(896) = 896 (to 1e-300)
    assert np.all(y[32:48] == 0.0)


def test_gated_silu_at_moderate_sums():
    """Gate sums of moderate size, exact in the codes: the output must be
    silu(v) u with silu in its tanh form, v/2 (1 + tanh(v/2)).  The two
    tests above hold for any v sigma(c v) (the odd-even identity and the
    limits do not see the constant c); this one pins c = 1."""
    import math
    I, K, g = 80, 128, 128
    x = oracle.round_to(np.ones((1, K)), "f16")
    s = 1.0 / 16.0                                   # fp16 0x2C00, exact
    codes = np.full((2 * I, K), 8, np.uint8)
    vs = [-3.0, -1.0, 0.5, 1.0, 2.5]                 # gate sums: 16 v codes one step off 8
    for b, v in enumerate(vs):
        n_off = int(round(abs(v) / s))
        codes[32 * b: 32 * b + 16, :n_off] = 9 if v > 0 else 7
        codes[32 * b + 16: 32 * b + 32, :16] = 9     # up sum 16 s = 1
    scales = np.full((2 * I, 1), 0x2C00, np.uint16)
    qw, sp, _ = oracle.pack(codes, scales, None, "sym", 4, g)
    y = oracle.qmm_gated(x, "f16", qw, sp, None, 1, I, K, "sym", 4, g)[0]
    for b, v in enumerate(vs):
        want = 0.5 * v * (1.0 + math.tanh(0.5 * v))
        assert np.allclose(y[16 * b: 16 * b + 16], want, rtol=1e-12, atol=0), (v, y[16 * b], want)
