"""Parity at the full problem sizes of the benchmark workloads (needs a B200).

The GPU runs every row of each weight matrix in the same launch configuration
the benchmark uses; the oracle checks a seeded sample of whole 16-row blocks
(first and last included): packed bytes bit for bit, y columns element by
element.  Rows outside the sample are filled from torch's seeded generator.
"""
import numpy as np
import pytest
import torch

import weight_only_quantized_int4_b200 as q
from tests import cases

pytestmark = pytest.mark.gpu

# (mode, bits, group, xdtype, [(K, N)], [M])  -- LLaMA-7B/70B-shaped layers
CONFIGS = {
    "decode_4096sq": ("sym", 4, 128, "f16", [(4096, 4096)], [1]),
    "llama7b_decode": ("sym", 4, 128, "f16",
                       [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)],
                       [1, 2, 4, 8, 16]),
    "llama70b_asym_bf16": ("asym", 4, 128, "bf16",
                           [(8192, 10240), (8192, 57344), (28672, 8192)], [1, 16, 64]),
    "lut4_nf4": ("lut", 4, 64, "f16", [(4096, 14336)], [1, 8, 32]),
    "lut2": ("lut", 2, 64, "f16", [(4096, 14336)], [1, 8, 32]),
    "lut3_nf3": ("lut", 3, 64, "f16", [(4096, 14336)], [1, 8, 32]),
    "prefill_gm1": ("sym", 4, -1, "f16", [(4096, 11008)], [64, 256, 1024, 4096]),
    "prefill_g128": ("sym", 4, 128, "f16", [(4096, 11008)], [64, 256, 1024, 4096]),
    # the largest K and N the packed layout accepts (2^20), each with the
    # smallest other dimension: 8192 K stages in one row tile, 65536 row blocks
    "max_sizes": ("sym", 4, 128, "f16", [(1 << 20, 16), (128, 1 << 20)], [1, 16, 64]),
}


def _gpu_weights(p, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = torch.randn(p.N, p.K, generator=g, device="cuda") * cases.SIGMA[p.mode]
    W[torch.from_numpy(p.rows).cuda()] = torch.from_numpy(p.W_rows).cuda()
    return W


def _sample_bytes(buf, rows, per_block):
    blocks = np.unique(rows // 16)
    return np.concatenate([buf[b * per_block:(b + 1) * per_block] for b in blocks])


@pytest.mark.parametrize("name", list(CONFIGS))
def test_fullsize(name):
    mode, bits, group, xdtype, shapes, Ms = CONFIGS[name]
    tdt = torch.float16 if xdtype == "f16" else torch.bfloat16
    for si, (K, N) in enumerate(shapes):
        p0 = cases.make(mode, bits, group, max(Ms), N, K, xdtype, seed=si, n_blocks=4)
        W = _gpu_weights(p0, 1000 + si)
        lut = None if p0.lut is None else torch.from_numpy(p0.lut.view(np.int16)).cuda()
        qw, sc, ze = q.pack(W, mode, bits, group, lut=lut)
        del W
        torch.cuda.synchronize()
        G = 1 if group == -1 else K // group
        per_blk = K * bits // 8 * 16
        assert np.array_equal(_sample_bytes(qw.cpu().numpy(), p0.rows, per_blk), p0.qw), name
        assert np.array_equal(_sample_bytes(sc.cpu().numpy().view(np.uint16), p0.rows, 16 * G),
                              p0.sp), name
        if mode == "asym":
            assert np.array_equal(_sample_bytes(ze.cpu().numpy().view(np.uint16), p0.rows, 16 * G),
                                  p0.zp), name
        zl = ze if mode == "asym" else lut
        for M in Ms:
            p = cases.make(mode, bits, group, M, N, K, xdtype, seed=si, n_blocks=4)
            x = torch.from_numpy(p.x.view(np.int16)).cuda().view(tdt)
            ws = q.workspace(M, N, K, mode, bits, group)
            y = q.qmm(x, qw, sc, zl, N, K, mode, bits, group, ws=ws)
            torch.cuda.synchronize()
            y_ref, bound = cases.expected(p)
            y_s = y[:, torch.from_numpy(p.rows).cuda()].float().cpu().numpy().astype(np.float64)
            cases.compare(y_s, y_ref, bound, f"{name} K{K} N{N} M{M}")
        del qw, sc, ze
        torch.cuda.empty_cache()
