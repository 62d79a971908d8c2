"""bench.py with several ranks, on the CPU: world size 2 over gloo.

The decode path has no data exchange between GPUs (each rank is an
independent replica), so the only multi-rank logic is the timing: every rank
times its own K steps, the job time is the slowest rank's, and the reported
throughput is all ranks' bytes over that time.  These tests run that logic in
two real processes, and check that the reference arm under torchrun does its
work on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # the bench's collective sequence: barrier, max of the device time,
        # barrier, max of the end-to-end time -- same steps on every rank
        dist.barrier()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist)
        dist.barrier()
        e2e = bench.max_over_ranks(30.0 - 7.0 * rank, dist)
        value = bench.whole_job_gbs(world, 2.0e9, 100, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "e2e": e2e, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_two_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms"] == 15.0            # the slowest rank's device time
        assert r["e2e"] == 30.0
        # 2 ranks x 2 GB per step x 100 steps in 15 ms
        assert r["value"] == pytest.approx(2 * 2.0e9 * 100 / 0.015 / 1e9)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_gbs(1, 1.0e9, 10, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_workload_units_and_bytes():
    """Tensor-bound workloads (every call M >= 256) are reported in TFLOP/s,
    the rest in GB/s; algorithmic bytes count the zero-point records and the
    act-order permutation."""
    assert bench.tensor_bound("prefill_m4096") and bench.tensor_bound("prefill_m256")
    assert not bench.tensor_bound("llama7b_decode") and not bench.tensor_bound("prefill_m64")
    assert bench.alg_flops(2, 3, 5) == 60.0
    K, N = 4096, 14336
    plain = bench.alg_bytes("asym", 4, -1, 1, K, N)
    zg8 = bench.alg_bytes("asym", 4, -1, 1, K, N, zopts=(8, 4))
    # fp16 row zero (N * 2 bytes) replaced by 4-bit zeros per 8 columns (N * K / 16)
    assert zg8 - plain == N * K // 16 - N * 2
    assert bench.alg_bytes("sym", 4, 128, 1, K, N, actorder=True) == \
        bench.alg_bytes("sym", 4, 128, 1, K, N) + 4 * K
    assert bench.alg_bytes("sym", 4, 128, 2, K, 2 * 64, gated=True) == \
        bench.alg_bytes("sym", 4, 128, 2, K, 2 * 64) - 2 * 64 * 2


def test_arena_views_hold_the_tensors_at_aligned_offsets():
    # the end-to-end leg copies one buffer each way: its views must be the
    # tensors themselves (same values, dtype, shape, contiguous) at offsets the
    # C ABI accepts, and the copied bytes are the buffer's size
    import torch
    g = torch.Generator().manual_seed(0)
    ts = [torch.randn(1, 4096, generator=g).half(),
          torch.randn(3, 40, generator=g).to(torch.bfloat16),   # 240 bytes: padded to 256
          torch.randn(16, 11008, generator=g).half()]
    arena, views = bench.arena_of(ts)
    assert arena.dtype == torch.uint8
    assert arena.numel() == 8192 + 256 + 16 * 11008 * 2
    base = arena.data_ptr()
    for t, v in zip(ts, views):
        assert v.dtype == t.dtype and v.shape == t.shape and v.is_contiguous()
        assert torch.equal(v, t)
        assert (v.data_ptr() - base) % 256 == 0
        assert v.untyped_storage().data_ptr() == arena.untyped_storage().data_ptr()
    # writing through the arena is seen by the views (one copy moves them all)
    arena.zero_()
    assert all(int(v.abs().sum()) == 0 for v in views)


@pytest.mark.parametrize("mode,bits,group,K,N,mb", [
    ("sym", 4, 128, 4096, 4096, 8.65), ("sym", 4, 128, 4096, 12288, 25.95),
    ("sym", 4, 128, 4096, 22016, 46.50), ("sym", 4, 128, 11008, 4096, 23.25),
    ("asym", 4, 128, 8192, 10240, 44.56), ("asym", 4, 128, 8192, 57344, 249.56),
    ("asym", 4, 128, 28672, 8192, 124.78), ("lut", 4, 64, 4096, 14336, 31.20),
    ("lut", 2, 64, 4096, 14336, 16.52), ("sym", 4, -1, 4096, 11008, 22.57),
    ("sym", 4, 128, 4096, 11008, 23.25)])
def test_weight_bytes_match_the_stated_figures(mode, bits, group, K, N, mb):
    """Codes + scales (+ zeros) of each benchmark shape against the figures
    worked out from the format: b/8 bytes per weight plus 2 bytes per group
    (4 with ASYM zeros), i.e. 0.516 B/weight for SYM4 g128, 0.531 for ASYM4
    g128 and LUT4 g64, 0.281 for LUT2 g64.  M = 0 leaves out x and y."""
    got = bench.alg_bytes(mode, bits, group, 0, K, N)
    assert round(got / 1e6, 2) == mb
    per_weight = {("sym", 4, 128): 0.515625, ("asym", 4, 128): 0.53125,
                  ("lut", 4, 64): 0.53125, ("lut", 2, 64): 0.28125}.get((mode, bits, group))
    if per_weight is not None:
        assert got == N * K * per_weight
