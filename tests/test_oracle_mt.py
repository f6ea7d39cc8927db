"""The oracle's row-parallel driver (the CPU baseline's all-cores leg) gives
the single-threaded oracle's outputs bit for bit, whatever the thread count:
it only splits the rows into contiguous chunks."""
import numpy as np
import pytest

import workloads


@pytest.mark.parametrize("threads", [1, 2, 3, 5, 8, 0, 64])
@pytest.mark.parametrize("residual", [True, False])
def test_row_parallel_equals_single_threaded(oracle_impl, threads, residual):
    c = workloads.make_case("odd", 37, cols=264, R=3, residual=residual)
    xs = [workloads.bits(x) for x in c.inputs]
    res = workloads.bits(c.residual) if residual else None
    g = workloads.bits(c.gamma)
    one = oracle_impl.sum_rmsnorm_fp8(xs, c.rows, c.cols, g, c.eps, c.weight_offset, c.scale_ub,
                                      residual=res)
    mt = oracle_impl.sum_rmsnorm_fp8_mt(xs, c.rows, c.cols, g, c.eps, c.weight_offset,
                                        c.scale_ub, residual=res, threads=threads)
    assert 1 <= mt["threads"] <= c.rows
    if threads:
        assert mt["threads"] == min(threads, c.rows)
    for k in one:
        assert np.array_equal(one[k], mt[k]), k


def test_cores_is_positive(oracle_impl):
    assert oracle_impl.cores() >= 1
