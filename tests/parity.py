"""Helpers for the GPU parity tests: run the CUDA library and the oracle on
the same seeded inputs and compare them at the stated tolerances.

Tolerances (stated for this operation):
  * the bf16 sum and the residual output are bit-exact;
  * scales agree within 1e-6 relative;
  * fp8 codes are equal, except that at most 0.1% of a call's elements may
    differ by one code step, and only where the oracle's pre-quantisation
    value y / scale lies within 1e-6 relative of an e4m3 rounding midpoint.
"""
from __future__ import annotations

import ml_dtypes
import numpy as np
import torch

import oracle
import workloads

SCALE_RTOL = 1e-6
CODE_MIDPOINT_RTOL = 1e-6
CODE_MISMATCH_FRACTION = 1e-3

_mags = np.unique(np.arange(0, 0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn)
                  .astype(np.float64))
_mids = (_mags[:-1] + _mags[1:]) / 2.0


def midpoint_distance(v: np.ndarray) -> np.ndarray:
    """Relative distance of |v| to the nearest e4m3 rounding midpoint."""
    a = np.abs(v.astype(np.float64)).reshape(-1)
    idx = np.clip(np.searchsorted(_mids, a), 1, len(_mids) - 1)
    d = np.minimum(np.abs(a - _mids[idx - 1]), np.abs(a - _mids[idx]))
    return (d / np.maximum(a, 2.0 ** -10)).reshape(v.shape)


def to_device(case: workloads.Case, device="cuda") -> workloads.Case:
    mv = lambda t: None if t is None else t.to(device).contiguous()
    return workloads.Case(case.name, case.R, case.rows, case.cols,
                          [mv(x) for x in case.inputs], mv(case.residual), mv(case.gamma),
                          case.eps, case.weight_offset, case.scale_ub)


def oracle_fused(case: workloads.Case, rows=None) -> dict:
    """The oracle on the case (all rows, or the listed rows)."""
    bits = workloads.bits
    if rows is None:
        xs = [bits(x) for x in case.inputs]
        res = None if case.residual is None else bits(case.residual)
        n = case.rows
    else:
        idx = torch.as_tensor(np.asarray(rows), device=case.inputs[0].device)
        xs = [bits(x.index_select(0, idx)) for x in case.inputs]
        res = None if case.residual is None else bits(case.residual.index_select(0, idx))
        n = len(rows)
    return oracle.sum_rmsnorm_fp8(xs, n, case.cols, bits(case.gamma), case.eps,
                                  case.weight_offset, case.scale_ub, residual=res, detail=True)


def oracle_sum(case: workloads.Case) -> np.ndarray:
    return oracle.sum_bf16([workloads.bits(x) for x in case.inputs], case.rows, case.cols)


def gpu_fused(case: workloads.Case, variant=0, cluster_size=0, block_threads=0,
              in_place=False, flags=0) -> dict:
    import reduce_rmsnorm_fp8_b200 as rrf
    res_in = None if case.residual is None else case.residual.clone()
    res_out = res_in if in_place else None
    q, scales, res_out = rrf.rrf_sum_rmsnorm_fp8_ex(
        case.inputs, case.gamma, case.eps, case.weight_offset, case.scale_ub,
        residual_in=res_in, residual_out=res_out, variant=variant,
        cluster_size=cluster_size, block_threads=block_threads, flags=flags)
    torch.cuda.synchronize()
    out = {"q": q.view(torch.uint8).cpu().numpy(), "scales": scales.reshape(-1).cpu().numpy()}
    if res_out is not None:
        out["res_out"] = workloads.bits(res_out)
    return out


def select_rows(gpu: dict, rows) -> dict:
    out = {k: v[rows] for k, v in gpu.items()}
    return out


def assert_fused_parity(gpu: dict, ref: dict, label: str = "", cap_at_ties: bool = False) -> dict:
    """Compare one call's outputs; returns a summary of the comparison.

    cap_at_ties: for problems outside the workloads' own input counts, where
    the bf16 inputs can put many y / scale values exactly on an e4m3 midpoint
    (ratios of short-mantissa products), the cap on differing codes is the
    larger of 0.1% and the number of oracle values within 1e-6 of a midpoint;
    every differing code must still sit at a midpoint and differ by one step."""
    if "res_out" in ref:
        assert np.array_equal(gpu["res_out"], ref["res_out"]), f"{label}: residual_out differs"
    rel = np.abs(gpu["scales"].astype(np.float64) - ref["scales"]) / ref["scales"]
    assert rel.max() <= SCALE_RTOL, f"{label}: scale rel err {rel.max():.3g}"
    qg, qr = gpu["q"], ref["q"]
    diff = qg != qr
    n_diff = int(diff.sum())
    if n_diff:
        near = midpoint_distance(ref["v"]) <= CODE_MIDPOINT_RTOL
        cap = CODE_MISMATCH_FRACTION * qr.size
        if cap_at_ties:
            cap = max(cap, int(near.sum()))
        assert n_diff <= cap, f"{label}: {n_diff} codes differ"
        assert near[diff].all(), f"{label}: a code differs away from a rounding midpoint"
        same_sign = (qg[diff] & 0x80) == (qr[diff] & 0x80)
        step = np.abs((qg[diff] & 0x7F).astype(int) - (qr[diff] & 0x7F).astype(int))
        assert same_sign.all() and (step == 1).all(), f"{label}: a code differs by > 1 step"
    return {"scale_max_rel": float(rel.max()), "codes_differing": n_diff}


def oracle_mx(case: workloads.Case, rows=None) -> dict:
    """The oracle's MX output on the case (all rows, or the listed rows)."""
    bits = workloads.bits
    if rows is None:
        xs = [bits(x) for x in case.inputs]
        res = None if case.residual is None else bits(case.residual)
        n = case.rows
    else:
        idx = torch.as_tensor(np.asarray(rows), device=case.inputs[0].device)
        xs = [bits(x.index_select(0, idx)) for x in case.inputs]
        res = None if case.residual is None else bits(case.residual.index_select(0, idx))
        n = len(rows)
    return oracle.sum_rmsnorm_mxfp8(xs, n, case.cols, bits(case.gamma), case.eps,
                                    case.weight_offset, residual=res, detail=True)


def assert_mx_parity(gpu: dict, ref: dict, label: str = "", cap_at_ties: bool = False) -> dict:
    """MX output: the residual bit for bit; the E8M0 codes equal except in
    blocks whose max |y| lies within 1e-6 of a power of two (where the last
    bit of r decides floor(log2)), and there at most one step apart; within
    blocks of equal codes, the element codes as for the row-scaled output
    (one step, at an e4m3 midpoint, on at most 0.1% of them)."""
    if "res_out" in ref:
        assert np.array_equal(gpu["res_out"], ref["res_out"]), f"{label}: residual_out differs"
    sg, sr = gpu["scales_mx"].astype(int), ref["scales_mx"].astype(int)
    rows, nb = sr.shape
    vmax = np.abs(ref["v"].astype(np.float64)).reshape(rows, nb, 32).max(axis=2)
    edge = (vmax * (1 - CODE_MIDPOINT_RTOL) < 256.0) | (vmax * (1 + CODE_MIDPOINT_RTOL) >= 512.0)
    diff = sg != sr
    assert not np.any(diff & ~edge), f"{label}: a block scale differs away from a power of two"
    assert np.all(np.abs(sg - sr)[diff] <= 1), f"{label}: a block scale differs by > 1"
    same = np.repeat(~diff, 32, axis=1)
    qg, qr = gpu["q"][same], ref["q"][same]
    dq = qg != qr
    n_diff = int(dq.sum())
    if n_diff:
        near = midpoint_distance(ref["v"][same]) <= CODE_MIDPOINT_RTOL
        cap = CODE_MISMATCH_FRACTION * qr.size
        if cap_at_ties:
            cap = max(cap, int(near.sum()))
        assert n_diff <= cap, f"{label}: {n_diff} codes differ"
        assert near[dq].all(), f"{label}: a code differs away from a rounding midpoint"
        step = np.abs((qg[dq] & 0x7F).astype(int) - (qr[dq] & 0x7F).astype(int))
        assert ((qg[dq] & 0x80) == (qr[dq] & 0x80)).all() and (step == 1).all(), \
            f"{label}: a code differs by > 1 step"
    return {"scale_blocks_differing": int(diff.sum()), "codes_differing": n_diff}
