"""The multi-process path on CPU: two gloo ranks.

Rows are independent, so N GPUs run N independent batches (weak scaling):
there is no data-path collective, only the barrier and the max-over-ranks
timing reduction of the benchmark.  These tests run that host logic with
world_size 2 on the gloo backend, and check that splitting a batch's rows
over ranks reproduces the whole batch (each rank running the oracle on its
row block), which is what makes the replicas equivalent to one large call.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_rows_partitions_exactly():
    for rows in (0, 1, 7, 37, 64, 8192):
        for world in (1, 2, 3, 4, 8):
            spans = [bench.shard_rows(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        # timing plumbing: barrier and the max over ranks
        bench.barrier()
        t = bench.max_over_ranks(0.25 + rank)
        # the data path: this rank's row block of one seeded batch
        c = workloads.make_case("odd", 37)
        start, stop = bench.shard_rows(c.rows, world, rank)
        bits = workloads.bits
        part = oracle.sum_rmsnorm_fp8([bits(x) for x in c.inputs], c.rows, c.cols,
                                      bits(c.gamma), c.eps, c.weight_offset, c.scale_ub,
                                      residual=bits(c.residual), row_start=start,
                                      row_count=stop - start)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), t=t, start=start, stop=stop,
                 **part)
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    # every rank saw the maximum of the per-rank values
    assert all(float(p["t"]) == 1.25 for p in parts)
    # the row blocks tile the batch and reproduce the single-process oracle
    import oracle
    import workloads
    c = workloads.make_case("odd", 37)
    bits = workloads.bits
    whole = oracle.sum_rmsnorm_fp8([bits(x) for x in c.inputs], c.rows, c.cols, bits(c.gamma),
                                   c.eps, c.weight_offset, c.scale_ub,
                                   residual=bits(c.residual))
    assert int(parts[0]["start"]) == 0 and int(parts[-1]["stop"]) == c.rows
    for key in ("q", "scales", "res_out"):
        assert np.array_equal(np.concatenate([p[key] for p in parts]), whole[key]), key


def test_weak_scaling_value_formula():
    """value = all ranks' bytes / max-over-ranks time (whole-job GB/s)."""
    per_step = bench.step_bytes("decode")
    steps, world, t = 100, 4, 2e-3
    assert per_step == sum(
        __import__("workloads").fused_bytes(8, r, 7168, True) for r in (1, 8, 32, 64))
    value = world * per_step * steps / t / 1e9
    assert value == pytest.approx(4 * 15863204 * 100 / 2e-3 / 1e9)
