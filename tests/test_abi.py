"""The C-ABI library: it loads, exports every symbol include/qmm.h declares,
and rejects bad arguments on the host (no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest

import weight_only_quantized_int4_b200 as q
from weight_only_quantized_int4_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "qmm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\**\s+\**(qmm\w*)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return q.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("qmm_pack", "qmm", "qmm_packed_size", "qmm_workspace_size", "qmm_dequant",
                 "qmm_strerror"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(q.SYMBOLS)


def test_sizes_and_paths(lib):
    assert q.packed_size(4096, 4096, "sym", 4, 128) == (4096 * 2048, 4096 * 32 * 2, 0)
    assert q.packed_size(64, 256, "asym", 4, -1) == (64 * 128, 64 * 2, 64 * 2)
    assert q.packed_size(16, 128, "lut", 2, 64) == (16 * 32, 16 * 2 * 2, 0)
    assert q.path(1, 4096, 4096, "sym") == "skinny"
    assert q.path(16, 4096, 4096, "sym") == "skinny"
    # measured crossover: the decode path up to M = 32 (one slab reads the
    # weights once), the tensor path above, for every N; combinations the
    # tensor path does not take stay on the decode path
    assert q.path(32, 11008, 4096, "sym") == "skinny"
    assert q.path(33, 11008, 4096, "sym") == "tensor"
    assert q.path(32, 4096, 4096, "sym") == "skinny"
    assert q.path(33, 4096, 4096, "sym") == "tensor"
    assert q.path(4096, 14336, 4096, "lut", 2, 64) == "skinny"
    # the kernel a forced-path request really runs, per activation dtype
    assert q.path(300, 272, 1024, "sym", 4, 128, "f16", "tensor") == "tensor"
    assert q.path(300, 272, 1024, "lut", 2, 64, "f16", "tensor") == "skinny"
    assert q.path(300, 272, 1024, "lut", 4, 64, "bf16", "tensor") == "tensor"
    assert q.path(300, 272, 1024, "asym", 4, 128, "bf16", "tensor") == "tensor"
    assert q.path(300, 272, 1024, "sym", 4, -1, "bf16", "tensor") == "tensor"
    assert q.path(5, 272, 1024, "sym", 4, 128, "f16", "skinny") == "skinny"
    assert q.path(4096, 11008, 4096, "sym", 4, 128, "f16", "auto") == "tensor"


@pytest.mark.parametrize("N,K,bits,group,mode,status", [
    (100, 4096, 4, 128, "sym", -2),     # N % 16
    (4096, 4000, 4, 128, "sym", -2),    # K % 64
    (4096, 4096, 2, 64, "sym", -2),     # 2-bit needs LUT
    (4096, 4160, 2, 64, "lut", -2),     # 2-bit needs K % 128
    (4096, 4096, 4, 100, "sym", -2),    # group not a multiple of 16
    (4608, 4608, 4, 48, "sym", -2),     # group not a power of two
    (4096, 4096, 4, 384, "sym", -2),    # group does not divide K
    (0, 4096, 4, 128, "sym", -1),
    (4096, 4096, 5, 128, "lut", -1),   # no 5-bit codes
    (4096, 4096, 3, 128, "sym", -2),   # 3-bit needs LUT
    (4096, 4160, 3, 64, "lut", -2),    # 3-bit needs K % 128
])
def test_bad_shapes_are_rejected(lib, N, K, bits, group, mode, status):
    assert lib.qmm_path(1, N, K, bits, group, q.MODES[mode]) == status
    assert lib.qmm_packed_size(N, K, bits, group, q.MODES[mode], None, None) == 0


def test_bad_arguments_return_status_without_launching(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)                      # never dereferenced: checks fail first
    # null x
    assert lib.qmm(None, 0, fake, fake, None, 1, 64, 64, 4, 64, 0, fake, None, 0, None) == -1
    # bad dtype, bad mode, negative M
    assert lib.qmm(fake, 7, fake, fake, None, 1, 64, 64, 4, 64, 0, fake, None, 0, None) == -1
    assert lib.qmm(fake, 0, fake, fake, None, 1, 64, 64, 4, 64, 9, fake, None, 0, None) == -1
    assert lib.qmm(fake, 0, fake, fake, None, -1, 64, 64, 4, 64, 0, fake, None, 0, None) == -1
    # M == 0 is a no-op
    assert lib.qmm(fake, 0, fake, fake, None, 0, 64, 64, 4, 64, 0, fake, None, 0, None) == 0
    # ASYM / LUT need their buffer
    assert lib.qmm(fake, 0, fake, fake, None, 1, 64, 64, 4, 64, 1, fake, None, 0, None) == -1
    # misaligned x
    assert lib.qmm(P(0x1002), 0, fake, fake, None, 1, 64, 64, 4, 64, 0, P(0x90000), None, 0,
                   None) == -3
    # scales / ASYM zeros must be 16-byte aligned (copied in 16-byte pieces)
    assert lib.qmm(fake, 0, fake, P(0x1004), None, 1, 64, 64, 4, 64, 0, P(0x90000), None, 0,
                   None) == -3
    assert lib.qmm(fake, 0, fake, fake, P(0x1008), 1, 64, 64, 4, 64, 1, P(0x90000), None, 0,
                   None) == -3
    assert lib.qmm_noalloc(fake, 0, fake, P(0x1004), None, 1, 64, 64, 4, 64, 0, P(0x90000),
                           None) == -3
    assert lib.qmm_pack(fake, 64, 64, 0, 4, 64, None, fake, P(0x1002), None, None) == -3
    # y overlapping x
    assert lib.qmm(fake, 0, P(0x200000), fake, None, 2, 64, 64, 4, 64, 0, P(0x1040), None, 0,
                   None) == -1
    # bad path
    assert lib.qmm_with_path(fake, 0, fake, fake, None, 1, 64, 64, 4, 64, 0, P(0x90000), None,
                             0, None, 5) == -1
    # pack: null W, misaligned W
    assert lib.qmm_pack(None, 64, 64, 0, 4, 64, None, fake, fake, None, None) == -1
    assert lib.qmm_pack(P(0x1004), 64, 64, 0, 4, 64, None, fake, fake, None, None) == -3
    assert lib.qmm_pack(fake, 64, 64, 2, 4, 64, None, fake, fake, None, None) == -1  # LUT, no table
    assert lib.qmm_dequant(fake, fake, None, 64, 64, 4, 64, 0, 3, fake, None) == -1


def test_strerror_covers_every_status(lib):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert q.strerror(s) != "unknown status"
    assert q.strerror(-99) == "unknown status"


def test_zero_point_options_sizes_and_rejections(lib):
    # 4-bit zero records: N * (K / zgroup) / 2 bytes; fp16: N * (K / zgroup) * 2
    assert lib.qmm_zeros_size(4096, 14336, -1, 8, 4) == 4096 * 1792 // 2
    assert lib.qmm_zeros_size(4096, 14336, -1, 8, 16) == 4096 * 1792 * 2
    assert lib.qmm_zeros_size(64, 1024, 128, 128, 4) == 64 * 8 // 2
    assert lib.qmm_zeros_size(64, 1024, -1, -1, 4) == 64 // 2
    for group, zgroup, zbits in ((64, 128, 4), (-1, 24, 4), (-1, 4, 4), (-1, 8, 8),
                                 (128, 8, 2)):
        assert lib.qmm_zeros_size(64, 1024, group, zgroup, zbits) == 0
    P = ctypes.c_void_p
    fake = P(0x1000)
    # zero group larger than the scale group; zbits not 4 / 16; zeros missing or misaligned
    assert lib.qmm_asym(fake, 0, fake, fake, fake, 1, 64, 1024, 64, 128, 4, P(0x900000), None, 0,
                        None) == -2
    assert lib.qmm_asym(fake, 0, fake, fake, fake, 1, 64, 1024, -1, 8, 8, P(0x900000), None, 0,
                        None) == -1
    assert lib.qmm_asym(fake, 0, fake, fake, None, 1, 64, 1024, -1, 8, 4, P(0x900000), None, 0,
                        None) == -1
    assert lib.qmm_asym(fake, 0, fake, fake, P(0x1008), 1, 64, 1024, -1, 8, 4, P(0x900000), None,
                        0, None) == -3
    assert lib.qmm_pack_asym(fake, 64, 1024, -1, 8, 4, fake, fake, None, None) == -1
    assert lib.qmm_pack_asym(fake, 64, 1024, 64, 128, 4, fake, fake, fake, None) == -2
    assert lib.qmm_dequant_asym(fake, fake, fake, 64, 1024, -1, 8, 4, 3, fake, None) == -1
    # the options only take 4-bit ASYM codes: the shape rules of qmm apply
    assert lib.qmm_asym(fake, 0, fake, fake, fake, 1, 60, 1024, -1, 8, 4, P(0x900000), None, 0,
                        None) == -2


def test_actorder_argument_checks(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)
    # perm from g_idx: bad group, bad K, null pointers
    assert lib.qmm_actorder_perm(fake, 1024, 48, fake, fake, None) == -2
    assert lib.qmm_actorder_perm(fake, 0, 128, fake, fake, None) == -1
    assert lib.qmm_actorder_perm(fake, 1024, 128, None, fake, None) == -1
    # pack: perm required and 16-byte aligned
    assert lib.qmm_pack_actorder(fake, None, 64, 1024, 0, 4, 128, None, fake, fake, None,
                                 None) == -1
    assert lib.qmm_pack_actorder(fake, P(0x1004), 64, 1024, 0, 4, 128, None, fake, fake, None,
                                 None) == -3
    # the product needs its workspace (x is gathered into it)
    n = lib.qmm_workspace_size_actorder(3, 64, 1024, 4, 128, 0)
    plain = lib.qmm_workspace_size(3, 64, 1024, 4, 128, 0)
    assert n == (plain + 255) // 256 * 256 + 3 * 1024 * 2
    assert lib.qmm_actorder(fake, 0, fake, fake, fake, None, 3, 64, 1024, 4, 128, 0,
                            P(0x900000), None, 0, None) == -6
    assert lib.qmm_actorder(fake, 0, fake, fake, fake, None, 3, 64, 1024, 4, 128, 0,
                            P(0x900000), P(0x100000), n - 256, None) == -6
    # y overlapping the workspace
    assert lib.qmm_actorder(fake, 0, fake, fake, fake, None, 3, 64, 1024, 4, 128, 0,
                            P(0x100100), P(0x100000), n, None) == -1
    # M == 0 is a no-op
    assert lib.qmm_actorder(fake, 0, fake, fake, fake, None, 0, 64, 1024, 4, 128, 0,
                            P(0x900000), None, 0, None) == 0
