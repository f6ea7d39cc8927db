"""GPU parity of the sharded form (a row's hidden dimension split into S
column shards): phase 1 on every shard, the statistics stacked as an
all-gather would, phase 2 on every shard; the concatenated result must match
the oracle on the whole rows with the same tolerances as the fused call.
The shards are emulated on one GPU (each shard's data in its own buffers)."""
import numpy as np
import pytest
import torch

import parity
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rrf():
    import reduce_rmsnorm_fp8_b200 as m
    return m


def shard(t, s, S):
    w = t.shape[-1] // S
    return t[..., s * w:(s + 1) * w].contiguous()


def run_sharded(rrf, c, S, in_place=False):
    """Both phases over S column shards of case c; returns the gathered
    outputs (as the fused call's) and the per-shard statistics and scales."""
    stats, hs = [], []
    for s in range(S):
        xs = [shard(x, s, S) for x in c.inputs]
        res = None if c.residual is None else shard(c.residual, s, S)
        st, h = rrf.rrf_sum_rmsnorm_fp8_pre(xs, shard(c.gamma, s, S), c.weight_offset,
                                            residual_in=res,
                                            residual_out=res if in_place else None)
        stats.append(st)
        hs.append(h)
    gathered = torch.stack(stats).contiguous()
    qs, scales = [], []
    for s in range(S):
        q, sc = rrf.rrf_rmsnorm_fp8_post(hs[s], shard(c.gamma, s, S), gathered, c.cols, c.eps,
                                         c.weight_offset, c.scale_ub)
        qs.append(q)
        scales.append(sc)
    torch.cuda.synchronize()
    out = {"q": torch.cat([q.view(torch.uint8) for q in qs], dim=-1).cpu().numpy(),
           "scales": scales[0].reshape(-1).cpu().numpy()}
    if c.residual is not None:
        out["res_out"] = workloads.bits(torch.cat(hs, dim=-1))
    h_all = workloads.bits(torch.cat(hs, dim=-1))
    return out, gathered.cpu().numpy(), [s.reshape(-1).cpu().numpy() for s in scales], h_all


@pytest.mark.parametrize("name,rows", [("decode", 1), ("decode", 32), ("decode", 64),
                                       ("odd", 37), ("sweep", 64), ("tiny", 4)])
@pytest.mark.parametrize("S", [1, 2, 4, 8])
def test_sharded_matches_whole_rows(rrf, name, rows, S):
    c = parity.to_device(workloads.make_case(name, rows))
    if (c.cols // S) % 8:
        pytest.skip("shard width not a multiple of 8")
    out, stats, scales, h_all = run_sharded(rrf, c, S)
    ref = parity.oracle_fused(c)
    parity.assert_fused_parity(out, ref, f"{name} {rows} S={S}")
    for sc in scales[1:]:  # every shard derives the same scales
        assert np.array_equal(sc, scales[0])
    # the norm input (h_out without a residual) is the oracle's, bit for bit
    assert np.array_equal(h_all, ref["h"])


@pytest.mark.parametrize("name,rows", [("decode", 64), ("odd", 37), ("sweep", 16)])
def test_one_shard_equals_fused_call(rrf, name, rows):
    """With one shard the two phases reproduce the fused call bit for bit:
    the same launch computes the same statistics, and merging one shard's
    pair changes nothing."""
    c = parity.to_device(workloads.make_case(name, rows))
    out, _, _, _ = run_sharded(rrf, c, 1)
    fused = parity.gpu_fused(c)
    for k in fused:
        assert np.array_equal(out[k], fused[k]), k


def test_shard_statistics_pinned(rrf):
    """Phase 1's statistics: max |h * g'| equals the fp32 products' maximum
    computed from the oracle's h (exactly: a max does not depend on order);
    the sum of squares agrees with float64 within 1e-6."""
    c = parity.to_device(workloads.make_case("odd", 37))
    S = 4
    _, stats, _, _ = run_sharded(rrf, c, S)
    ref = parity.oracle_fused(c)
    h = parity.oracle.bf16_to_float(ref["h"])  # float32
    g = workloads.bits(c.gamma)
    gp = (parity.oracle.bf16_to_float(g) + np.float32(c.weight_offset)).astype(np.float32)
    w = c.cols // S
    for s in range(S):
        hs, gs = h[:, s * w:(s + 1) * w], gp[s * w:(s + 1) * w]
        key = np.abs(hs * gs).max(axis=1)  # fp32 products, as the kernel rounds them
        assert np.array_equal(stats[s, :, 1], key)
        ss = (hs.astype(np.float64) ** 2).sum(axis=1)
        assert np.all(np.abs(stats[s, :, 0] - ss) <= 1e-6 * ss)


def test_sharded_in_place_residual(rrf):
    c = parity.to_device(workloads.make_case("decode", 8))
    ref = parity.oracle_fused(c)  # before the in-place update
    out, _, _, _ = run_sharded(rrf, c, 4, in_place=True)
    parity.assert_fused_parity(out, ref, "in place")


def test_sharded_glue_with_nccl_group_of_one(rrf, tmp_path):
    """The torch.distributed path (all-gather of the statistics) on a real
    NCCL process group of one rank."""
    import torch.distributed as dist

    from reduce_rmsnorm_fp8_b200 import sharded
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        c = parity.to_device(workloads.make_case("decode", 32))
        q, scales, res_out = sharded.sharded_sum_rmsnorm_fp8(
            c.inputs, c.gamma, c.eps, c.weight_offset, c.scale_ub, residual_in=c.residual)
        torch.cuda.synchronize()
        got = {"q": q.view(torch.uint8).cpu().numpy(), "scales": scales.reshape(-1).cpu().numpy(),
               "res_out": workloads.bits(res_out)}
        parity.assert_fused_parity(got, parity.oracle_fused(c), "nccl group of one")
    finally:
        dist.destroy_process_group()


def test_post_validation(rrf):
    c = parity.to_device(workloads.make_case("decode", 8))
    stats, h = rrf.rrf_sum_rmsnorm_fp8_pre(c.inputs, c.gamma, c.weight_offset,
                                           residual_in=c.residual)
    with pytest.raises(ValueError):  # stats must be [shards, rows, 2]
        rrf.rrf_rmsnorm_fp8_post(h, c.gamma, stats, c.cols, c.eps, c.weight_offset, c.scale_ub)
    with pytest.raises(rrf.RrfError) as e:  # fewer total columns than the shard's
        rrf.rrf_rmsnorm_fp8_post(h, c.gamma, stats[None], c.cols - 8, c.eps, c.weight_offset,
                                 c.scale_ub)
    assert e.value.status == rrf.Status.ERR_SHAPE
