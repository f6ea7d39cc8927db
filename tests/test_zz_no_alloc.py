"""rrf_allreduce_rmsnorm_fp8_static: the multi-GPU call for callers that
cannot allocate device memory (a program whose device memory belongs to
another allocator's pool, a latency-bound loop that must not risk the
device-wide synchronisation cudaMalloc / cudaFree can cause, a plug-in whose
host forbids allocation).  It runs every rank in one launch on this GPU and
takes the signal pads from a fixed array inside the library, so the caller
passes only inputs and outputs.

The GPU test calls it twice in a row through the C ABI, on two different
problems, and compares each result with the same problem run through
rrf_allreduce_rmsnorm_fp8 with pads the caller allocated, at the tolerances
of the parity tests (residual bit for bit, scales within 1e-6 relative, codes
equal except at most 0.1% one step apart).  This file is collected last so
that a run stopping at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
import workloads

ONE, TWO = 1, 2


@pytest.fixture(scope="module")
def rrf():
    import reduce_rmsnorm_fp8_b200 as m
    return m


def test_world_beyond_the_fixed_pads_is_rejected(rrf):
    """A world the fixed array has no pads for is refused on the host,
    before any CUDA call (so this runs without a GPU)."""
    n = rrf.RRF_AR_STATIC_MAX_WORLD + 1
    fake = (ctypes.c_void_p * n)(*[16 * (i + 1) for i in range(n)])
    st = rrf.lib.rrf_allreduce_rmsnorm_fp8_static(fake, None, None, fake, fake, n, 4, 64,
                                                  ctypes.c_void_p(16), 1e-6, 0.0, 1.0, 0, 0,
                                                  None)
    assert st == rrf.Status.ERR_RANKS
    st = rrf.lib.rrf_allreduce_rmsnorm_fp8_static(fake, None, None, fake, fake, 0, 4, 64,
                                                  ctypes.c_void_p(16), 1e-6, 0.0, 1.0, 0, 0,
                                                  None)
    assert st == rrf.Status.ERR_RANKS


def _outputs(q, scales, res):
    out = []
    for k in range(len(q)):
        o = {"q": q[k].view(torch.uint8).cpu().numpy(),
             "scales": scales[k].reshape(-1).cpu().numpy()}
        if res is not None:
            o["res_out"] = workloads.bits(res[k])
        out.append(o)
    return out


def _static_call(rrf, c, mode):
    """One call of the new entry point on c's partials (every rank's buffers
    on this GPU); returns the per-rank outputs as tensors."""
    world = len(c.inputs)
    shape = c.inputs[0].shape
    res_in = None if c.residual is None else [c.residual.clone() for _ in range(world)]
    res_out = None if res_in is None else [torch.empty_like(r) for r in res_in]
    q = [torch.empty(shape, dtype=torch.float8_e4m3fn, device="cuda") for _ in range(world)]
    sc = [torch.empty((shape[0], 1), dtype=torch.float32, device="cuda") for _ in range(world)]
    ptrs = lambda ts: None if ts is None else [t.data_ptr() for t in ts]
    rrf.rrf_allreduce_rmsnorm_fp8_static_ptr(
        ptrs(c.inputs), ptrs(res_in), ptrs(res_out), ptrs(q), ptrs(sc), shape[0], shape[1],
        c.gamma.data_ptr(), c.eps, c.weight_offset, c.scale_ub, mode=mode,
        stream=torch.cuda.current_stream().cuda_stream)
    return q, sc, res_out


def _assert_within_tolerance(got, ref, label):
    if "res_out" in ref:
        assert np.array_equal(got["res_out"], ref["res_out"]), f"{label}: residual differs"
    rel = np.abs(got["scales"].astype(np.float64) - ref["scales"]) / ref["scales"]
    assert rel.max() <= parity.SCALE_RTOL, f"{label}: scale rel err {rel.max():.3g}"
    diff = got["q"] != ref["q"]
    assert diff.sum() <= parity.CODE_MISMATCH_FRACTION * diff.size, f"{label}: codes differ"
    a, b = got["q"][diff], ref["q"][diff]
    assert ((a & 0x80) == (b & 0x80)).all(), f"{label}: a code changed sign"
    assert (np.abs((a & 0x7F).astype(int) - (b & 0x7F).astype(int)) == 1).all(), \
        f"{label}: a code differs by more than one step"


@pytest.mark.gpu
def test_matches_the_allocating_entry_point_on_two_calls_in_a_row(rrf):
    from reduce_rmsnorm_fp8_b200 import allreduce
    rrf.rrf_device_error(clear=True)
    problems = [(parity.to_device(workloads.make_case("decode", 64, R=8, sub=60)), TWO),
                (parity.to_device(workloads.make_case("odd", 37, R=4, sub=61)), ONE)]
    # two calls of the new entry point back to back on the same stream
    static = [_static_call(rrf, c, mode) for c, mode in problems]
    torch.cuda.synchronize()
    static = [_outputs(*o) for o in static]
    for (c, mode), got in zip(problems, static):
        world = len(c.inputs)
        res = [c.residual.clone() for _ in range(world)]
        q, sc, res_out = allreduce.LocalGroup(world)(c.inputs, c.gamma, c.eps, c.weight_offset,
                                                    c.scale_ub, residual_in=res, mode=mode)
        torch.cuda.synchronize()
        ref = _outputs(q, sc, res_out)
        for k in range(world):
            _assert_within_tolerance(got[k], ref[k], f"{c.name} {c.rows} rows, rank {k}")
    assert rrf.rrf_device_error() == 0
