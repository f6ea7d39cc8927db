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


def _two_shot_worker(rank, world, port, out_dir):
    """The two-shot data flow of the multi-GPU call with gloo as the
    transport: rank k holds partial k only; it fetches the partials of its
    row block from every rank (an all-gather here, peer loads on GPUs),
    computes those rows, and every rank gathers all blocks' codes, scales and
    residual rows."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import workloads
    from reduce_rmsnorm_fp8_b200.allreduce import two_shot_rows
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        c = workloads.make_case("odd", 37, R=world)
        bits = workloads.bits
        mine = torch.from_numpy(bits(c.inputs[rank]).view(np.uint8).copy())  # bytes: gloo has no 16-bit ints
        parts = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine)
        start, stop = two_shot_rows(c.rows, world, rank)
        per = -(-c.rows // world)
        blk = oracle.sum_rmsnorm_fp8([p.numpy().view(np.uint16) for p in parts], c.rows, c.cols,
                                     bits(c.gamma), c.eps, c.weight_offset, c.scale_ub,
                                     residual=bits(c.residual), row_start=start,
                                     row_count=stop - start)
        gathered = {}
        for key, width in (("q", c.cols), ("res_out", c.cols), ("scales", 1)):
            pad = np.zeros((per, width), dtype=blk[key].dtype)
            pad[:stop - start] = blk[key].reshape(stop - start, width)
            t = torch.from_numpy(pad.view(np.uint8).copy())
            out = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(out, t)
            whole = np.concatenate([o.numpy().view(blk[key].dtype).reshape(per, width)
                                    for o in out])[:c.rows]
            gathered[key] = whole.reshape((c.rows,) + blk[key].shape[1:])
        np.savez(os.path.join(out_dir, f"ts{rank}.npz"), **gathered)
    finally:
        dist.destroy_process_group()


def test_two_shot_flow_on_gloo(tmp_path):
    world, port = 2, free_port()
    mp.start_processes(_two_shot_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    import oracle
    import workloads
    c = workloads.make_case("odd", 37, R=world)
    bits = workloads.bits
    whole = oracle.sum_rmsnorm_fp8([bits(x) for x in c.inputs], c.rows, c.cols, bits(c.gamma),
                                   c.eps, c.weight_offset, c.scale_ub,
                                   residual=bits(c.residual))
    for r in range(world):
        got = np.load(tmp_path / f"ts{r}.npz")
        for key in ("q", "scales", "res_out"):
            assert np.array_equal(got[key], whole[key]), (r, key)
