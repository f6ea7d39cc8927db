"""GPU parity of the MX output (rrf_sum_rmsnorm_mxfp8): one E8M0 scale per
32 elements, against the oracle (tolerances in parity.assert_mx_parity)."""
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


def gpu_mx(rrf, c, in_place=False):
    res_in = None if c.residual is None else c.residual.clone()
    q, sc, res = rrf.rrf_sum_rmsnorm_mxfp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                           residual_in=res_in,
                                           residual_out=res_in if in_place else None)
    torch.cuda.synchronize()
    out = {"q": q.view(torch.uint8).cpu().numpy(), "scales_mx": sc.cpu().numpy()}
    if res is not None:
        out["res_out"] = workloads.bits(res)
    return out


CASES = [("tiny", 4), ("decode", 1), ("decode", 8), ("decode", 32), ("decode", 64),
         ("odd", 37), ("odd", 64), ("sweep", 16), ("sweep", 64), ("sweep", 256)]


@pytest.mark.parametrize("name,rows", CASES)
def test_mx_matches_oracle(rrf, name, rows):
    c = parity.to_device(workloads.make_case(name, rows))
    parity.assert_mx_parity(gpu_mx(rrf, c), parity.oracle_mx(c), f"{name} {rows}")


def test_mx_prefill_sampled_rows(rrf):
    c = parity.to_device(workloads.make_case("prefill", 8192))
    got = gpu_mx(rrf, c)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 397), [1, 8191]]))
    parity.assert_mx_parity(parity.select_rows(got, rows), parity.oracle_mx(c, rows=rows),
                            "prefill")


def test_mx_in_place_and_rows_of_the_row_scaled_call(rrf):
    """In place; and the norm input h (residual_out) is the row-scaled call's."""
    c = parity.to_device(workloads.make_case("decode", 32))
    ref = parity.oracle_mx(c)
    got = gpu_mx(rrf, c, in_place=True)
    parity.assert_mx_parity(got, ref, "in place")
    assert np.array_equal(got["res_out"], parity.gpu_fused(c)["res_out"])


@pytest.mark.parametrize("R,cols", [(1, 32), (3, 96), (16, 4096), (5, 131072)])
def test_mx_edges(rrf, R, cols):
    c = parity.to_device(workloads.make_case("odd", 3, R=R, cols=cols))
    parity.assert_mx_parity(gpu_mx(rrf, c), parity.oracle_mx(c), f"R={R} cols={cols}",
                            cap_at_ties=True)


def test_mx_zero_rows_and_blocks(rrf):
    """Zero inputs: every block takes code 0 and every code is +-0."""
    c = parity.to_device(workloads.make_case("decode", 8))
    for x in c.inputs:
        x.zero_()
    c.residual.zero_()
    got = gpu_mx(rrf, c)
    assert np.all(got["scales_mx"] == 0) and np.all((got["q"] & 0x7F) == 0)
    parity.assert_mx_parity(got, parity.oracle_mx(c), "zeros")


def test_mx_empty(rrf):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, sc, _ = rrf.rrf_sum_rmsnorm_mxfp8([x], torch.ones(64, dtype=torch.bfloat16,
                                                         device="cuda"), 1e-6, 0.0)
    assert q.shape == (0, 64) and sc.shape == (0, 2)
