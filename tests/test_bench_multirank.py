"""bench.py's multi-rank plumbing on CPU: two gloo ranks, the step time is the
max over ranks and the throughput counts every rank's tokens."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port), LASP_BENCH_BACKEND="gloo")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_setup()
    try:
        seconds = 1.0 + r  # rank 1 is the slow one
        value, t = bench.aggregate(1000.0, seconds, w)
        bench.barrier(w)
        out[r] = (value, t)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    for r in (0, 1):
        value, t = res[r]
        assert t == 2.0
        assert value == pytest.approx(2 * 1000.0 / 2.0)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(500.0, 0.5, 1) == (1000.0, 0.5)
    assert bench.algorithmic_bytes("state_scan", 1, 128, 128, 1024, 2) == 2 * 128 * 128 * 4 / 128
    s4 = 4 * 128 * 128
    assert bench.algorithmic_bytes("fwd_walk_tc", 1, 128, 128, 1024, 2) == 4 * 128 * 2 + s4 / 1024 + s4 / 256
    assert bench.algorithmic_bytes("fwd_walk_tc", 1, 128, 256, 1024, 2) == 4 * 128 * 2 + s4 / 256
    # chunks inside a tile: one cached bf16 tile per 128 tokens whatever C is
    assert bench.algorithmic_bytes("fwd_walk_tc", 1, 128, 64, 1024, 2) == 4 * 128 * 2 + s4 / 1024 + s4 / 256
    assert bench.algorithmic_bytes("bwd_walk_tc", 1, 128, 32, 1024, 2) == 7 * 128 * 2 + s4 / 256 + s4 / 1024


def test_algorithmic_bytes_of_the_segment_kernels():
    """Bytes per token-head of the kernels that work per segment of G tokens:
    the state total reads the segment states once; the gated segment states
    write one state per segment; the forward walk reads one state per segment
    and writes a bf16 state tile per 128 tokens, which the backward walk reads
    back with one gradient state per segment."""
    sys.path.insert(0, ROOT)
    import bench
    d, G, e = 128, 1024, 2
    s = 4 * d * d
    assert bench.algorithmic_bytes("state_total", 1, d, 128, G, e) == s / G
    assert bench.algorithmic_bytes("gla_segment_states_tc", 1, d, 128, G, e) == 2 * d * e + 4 * d + s / G
    assert bench.algorithmic_bytes("gla_segment_scan", 1, d, 128, G, e) == 2 * s / G + 4 * d / G
    assert bench.algorithmic_bytes("gla_out_tc", 1, d, 128, G, e) == 4 * d * e + 4 * d + s / G + s / 256
    assert bench.algorithmic_bytes("gla_bwd_tc", 1, d, 128, G, e) == 7 * d * e + 8 * d + s / 256 + s / G
    # per-tile kernels do not depend on the segment
    assert bench.algorithmic_bytes("gla_states_tc", 1, d, 128, G, e) == bench.algorithmic_bytes(
        "gla_states_tc", 1, d, 128, 128, e)
