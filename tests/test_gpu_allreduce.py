"""GPU parity of the multi-GPU form (rrf_allreduce_rmsnorm_fp8).

All ranks run in one launch on one GPU (LocalGroup): each rank's partial,
residual, outputs and signal pad are separate buffers, and the ranks' blocks
meet at the same start and end barriers as in a job with one GPU per rank.
Every rank's outputs must equal the oracle's on the whole problem (the
partials as the inputs, in rank order) within the fused call's tolerances,
and every rank must hold the same bits.
"""
import dataclasses

import numpy as np
import pytest
import torch

import parity
import workloads

pytestmark = pytest.mark.gpu

ONE, TWO = 1, 2


@pytest.fixture(scope="module")
def rrf():
    import reduce_rmsnorm_fp8_b200 as m
    return m


@pytest.fixture(scope="module")
def allreduce():
    from reduce_rmsnorm_fp8_b200 import allreduce as m
    return m


def rank_case(name, rows, world, sub=None):
    """The seeded problem with `world` partials (one per rank)."""
    return parity.to_device(workloads.make_case(name, rows, R=world, sub=sub))


def run_local(allreduce, c, mode, in_place=False, group=None):
    """One call over c's partials; returns the per-rank outputs as numpy."""
    world = len(c.inputs)
    g = group or allreduce.LocalGroup(world)
    res_in = None if c.residual is None else [c.residual.clone() for _ in range(world)]
    res_out = res_in if in_place else None
    q, scales, res_out = g(c.inputs, c.gamma, c.eps, c.weight_offset, c.scale_ub,
                           residual_in=res_in, residual_out=res_out, mode=mode)
    torch.cuda.synchronize()
    outs = []
    for k in range(world):
        o = {"q": q[k].view(torch.uint8).cpu().numpy(),
             "scales": scales[k].reshape(-1).cpu().numpy()}
        if res_out is not None:
            o["res_out"] = workloads.bits(res_out[k])
        outs.append(o)
    return outs


def assert_ranks_agree(outs):
    for o in outs[1:]:
        for k in outs[0]:
            assert np.array_equal(o[k], outs[0][k]), f"ranks disagree on {k}"


CASES = [("decode", 1), ("decode", 8), ("decode", 64), ("odd", 37), ("tiny", 4), ("sweep", 48)]


@pytest.mark.parametrize("name,rows", CASES)
@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("mode", [ONE, TWO])
def test_local_group_matches_oracle(rrf, allreduce, name, rows, world, mode):
    c = rank_case(name, rows, world)
    outs = run_local(allreduce, c, mode)
    assert_ranks_agree(outs)
    # the workload's own input count keeps the strict cap; other rank counts
    # may put many values exactly on a midpoint (see parity.assert_fused_parity)
    own_R = workloads.WORKLOADS[name].R == world
    parity.assert_fused_parity(outs[0], parity.oracle_fused(c), f"{name} {rows} w{world} m{mode}",
                               cap_at_ties=not own_R)


@pytest.mark.parametrize("name,rows,world", [("decode", 64, 8), ("decode", 8, 8), ("odd", 37, 4),
                                             ("sweep", 48, 4)])
@pytest.mark.parametrize("mode", [ONE, TWO])
def test_same_shape_same_bits_as_fused_call(rrf, allreduce, name, rows, world, mode):
    """Where the multi-GPU call splits a row as the single-GPU call does, the
    two reduce the statistics in the same order: identical bits."""
    c = rank_case(name, rows, world)
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    m, cluster, threads, vpt = rrf.rrf_plan_allreduce(world, rows, c.cols, sm,
                                                       c.residual is not None, mode)
    outs = run_local(allreduce, c, mode)
    # the single-GPU call forced to the same row split (cluster size, block size)
    fused = parity.gpu_fused(c, variant=2 if cluster > 1 else 1,
                             cluster_size=cluster if cluster > 1 else 0, block_threads=threads)
    for k in fused:
        assert np.array_equal(outs[0][k], fused[k]), k


@pytest.mark.parametrize("mode", [ONE, TWO])
def test_in_place_residual(allreduce, mode):
    c = rank_case("decode", 32, 8)
    ref = parity.oracle_fused(c)
    outs = run_local(allreduce, c, mode, in_place=True)
    assert_ranks_agree(outs)
    parity.assert_fused_parity(outs[0], ref, "in place")


def test_repeated_calls_on_one_group(rrf, allreduce):
    """Six calls on the same pads (the blocks' call counters), new data and
    shapes each time, alternating modes."""
    g = allreduce.LocalGroup(4)
    for i in range(6):
        c = rank_case("odd", 37 if i % 3 else 64, 4, sub=20 + i)
        outs = run_local(allreduce, c, ONE if i % 2 else TWO, group=g)
        assert_ranks_agree(outs)
        parity.assert_fused_parity(outs[0], parity.oracle_fused(c), f"call {i + 1}")
    assert rrf.rrf_device_error() == 0


def test_graph_replay(rrf, allreduce):
    """A call captured in a CUDA graph and replayed three times over new
    inputs copied into the captured buffers: every replay synchronises the
    ranks afresh and is correct."""
    world = 8
    g = allreduce.LocalGroup(world)
    c0 = rank_case("decode", 32, world, sub=40)
    xs = [x.clone() for x in c0.inputs]
    res = [c0.residual.clone() for _ in range(world)]
    q = [torch.empty(x.shape, dtype=torch.float8_e4m3fn, device="cuda") for x in xs]
    sc = [torch.empty((x.shape[0], 1), dtype=torch.float32, device="cuda") for x in xs]
    call = lambda: g(xs, c0.gamma, c0.eps, c0.weight_offset, c0.scale_ub, residual_in=res,
                     residual_out=res, q_out=q, scales_out=sc, mode=TWO)
    call()  # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for i in range(3):
        # new partials and residual; gamma stays the captured one
        c = dataclasses.replace(rank_case("decode", 32, world, sub=41 + i), gamma=c0.gamma)
        for x, src in zip(xs, c.inputs):
            x.copy_(src)
        for r in res:
            r.copy_(c.residual)
        graph.replay()
        torch.cuda.synchronize()
        outs = [{"q": q[k].view(torch.uint8).cpu().numpy(),
                 "scales": sc[k].reshape(-1).cpu().numpy(),
                 "res_out": workloads.bits(res[k])} for k in range(world)]
        assert_ranks_agree(outs)
        parity.assert_fused_parity(outs[0], parity.oracle_fused(c), f"replay {i}")
    assert rrf.rrf_device_error() == 0


def test_two_shot_full_prefill(allreduce):
    """8 ranks, 8192 x 8192 (each rank computes 1024 rows): sampled rows
    against the oracle, all rows equal on every rank."""
    c = rank_case("prefill", 8192, 8)
    outs = run_local(allreduce, c, TWO)
    assert_ranks_agree(outs)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 509), np.arange(1020, 1030),
                                     [8191]]))
    parity.assert_fused_parity(parity.select_rows(outs[0], rows),
                               parity.oracle_fused(c, rows=rows), "prefill two-shot")


def test_empty_call(rrf, allreduce):
    g = allreduce.LocalGroup(2)
    x = [torch.empty((0, 64), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    gamma = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    q, s, r = g(x, gamma, 1e-6, 0.0, 1.0)
    assert q[0].shape == (0, 64) and s[0].shape == (0, 1) and r is None


def test_missing_peer_times_out(rrf, allreduce):
    """Rank 0 of a two-rank group launched alone: both barrier waits run out
    (1 ms each), the kernel finishes and reports the timeout in the device
    error word; the library stays usable."""
    rrf.rrf_device_error(clear=True)
    rows, cols = 16, 1024
    mk = lambda dt: [torch.zeros((rows, cols), dtype=dt, device="cuda") for _ in range(2)]
    xs, qs = mk(torch.bfloat16), mk(torch.uint8)
    scales = [torch.zeros(rows, dtype=torch.float32, device="cuda") for _ in range(2)]
    pads = [torch.zeros(rrf.RRF_AR_SIGNAL_WORDS, dtype=torch.int32, device="cuda")
            for _ in range(2)]
    gamma = torch.ones(cols, dtype=torch.bfloat16, device="cuda")
    ptr = lambda ts: [t.data_ptr() for t in ts]
    rrf.rrf_allreduce_rmsnorm_fp8_ptr(ptr(xs), None, None, ptr(qs), ptr(scales), ptr(pads), 0, 1,
                                      rows, cols, gamma.data_ptr(), 1e-6, 0.0, 1.0,
                                      mode=TWO, timeout_ns=1_000_000,
                                      stream=torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rrf.rrf_device_error(clear=True) & rrf.RRF_DEVICE_ERROR_PEER_TIMEOUT
    c = rank_case("decode", 8, 2)
    parity.assert_fused_parity(run_local(allreduce, c, TWO)[0], parity.oracle_fused(c), "after",
                               cap_at_ties=True)
    assert rrf.rrf_device_error() == 0


def test_peer_group_nccl_group_of_one(rrf, allreduce, tmp_path):
    """The symmetric-memory path (PeerGroup) on a real NCCL process group of
    one rank: allocation, rendezvous, pointer marshalling and the call."""
    import torch.distributed as dist
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        c = rank_case("decode", 32, 1)
        pg = allreduce.PeerGroup(dist.group.WORLD, max_rows=64, cols=c.cols)
        pg.input(32).copy_(c.inputs[0])
        pg.residual(32).copy_(c.residual)
        q, scales, res = pg(32, c.gamma, c.eps, c.weight_offset, c.scale_ub)
        torch.cuda.synchronize()
        got = {"q": q.view(torch.uint8).cpu().numpy(), "scales": scales.reshape(-1).cpu().numpy(),
               "res_out": workloads.bits(res)}
        parity.assert_fused_parity(got, parity.oracle_fused(c), "peer group of one",
                                   cap_at_ties=True)
        del pg
    finally:
        dist.destroy_process_group()
