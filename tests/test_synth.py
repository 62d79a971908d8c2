"""The seeded input generator's torch twin (used by the benchmark to draw its
inputs on the device) against the host generator, and the benchmark's table of
configurations against the five configurations it times.  CPU only."""
import os
import sys

import numpy as np
import pytest
import torch

from weight_only_quantized_int4_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("seed,stream,N,K", [(0, "W0.0", 48, 256), (0, "W3.1", 17, 96),
                                             (5, "x", 3, 1024)])
def test_torch_weights_equal_host_weights(seed, stream, N, K):
    W = synth.weights(seed, stream, N, K, 0.02)
    Wt = synth.weights_torch(seed, stream, N, K, 0.02).numpy()
    assert np.array_equal(W.view(np.uint32), Wt.view(np.uint32))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_torch_activations_equal_host_activations(dtype):
    x = synth.activations(0, "x2", 7, 640, dtype)
    xt = synth.activations_torch(0, "x2", 7, 640, dtype)
    assert np.array_equal(x, xt.view(torch.int16).numpy().view(np.uint16))


def test_bench_configurations_cover_the_five_configs():
    W = bench.WORKLOADS
    for names in bench.CONFIG_WORKLOADS.values():
        for n in names:
            assert n in W, n
    # configs[0]: M = 1, K = N = 4096, SYM g128 fp16
    assert W["decode_4096sq"] == ("sym", 4, 128, "f16", [(4096, 4096)], [1])
    # configs[1]: the headline (LLaMA-7B decode layers, M = 1..16)
    assert W["llama7b_decode"][5] == [1, 2, 4, 8, 16]
    # configs[2]: 70B ASYM bf16, M in {1, 16, 64}
    assert W["llama70b_asym_bf16"][:4] == ("asym", 4, 128, "bf16")
    assert W["llama70b_asym_bf16"][5] == [1, 16, 64]
    # configs[3]: LUT4 and LUT2, g64, M in {1, 8, 32}, K 4096, N 14336
    for n, bits in (("lut4_nf4", 4), ("lut2", 2)):
        assert W[n] == ("lut", bits, 64, "f16", [(4096, 14336)], [1, 8, 32])
    # configs[4]: the prefill sweep, g128 and per-row scales
    sweep = bench.CONFIG_WORKLOADS["5_prefill_k4096_n11008"]
    got = sorted((W[n][2], W[n][5][0]) for n in sweep)
    assert got == sorted((g, m) for g in (128, -1) for m in (64, 256, 1024, 4096))
