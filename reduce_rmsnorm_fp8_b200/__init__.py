"""Fused bf16 sum + residual + RMSNorm + per-row FP8 (e4m3fn) for B200.

A thin Python binding over the C ABI in ``include/rrf.h`` (``librrf.so``,
hand-written sm_100a CUDA kernels).  The functions here only marshal torch
tensors into pointers, sizes and the current CUDA stream; every step of the
operation runs in the library's kernels.  Importing this package fails if
``librrf.so`` has not been built (``python -m reduce_rmsnorm_fp8_b200.build``):
there is no fallback.

Functions, named after the C entry points:
  rrf_sum(inputs, out=None)
  rrf_sum_rmsnorm_fp8(inputs, gamma, eps, weight_offset, scale_ub,
                      residual_in=None, residual_out=None, q_out=None,
                      scales_out=None) -> (q, scales, residual_out)
  rrf_sum_rmsnorm_fp8_ex(..., variant=0, cluster_size=0, block_threads=0)
  rrf_plan_fused(num_inputs, rows, cols, sm_count) -> (cluster, threads, vpt)
  rrf_check_sum_args / rrf_check_fused_args (raw pointers, host only)
"""
from __future__ import annotations

from ._lib import (  # noqa: F401
    LIB_PATH,
    RRF_MAX_COLS,
    RRF_FLAG_NO_PDL,
    RRF_MAX_INPUTS,
    RRF_VARIANT_AUTO,
    RRF_VARIANT_CLUSTER,
    RRF_VARIANT_ROW,
    RrfError,
    Status,
    lib,
    rrf_check_fused_args,
    rrf_check_sum_args,
    rrf_debug_fail_next_launch,
    rrf_last_cuda_error,
    rrf_plan_fused,
    rrf_status_string,
    rrf_sum,
    rrf_sum_ptr,
    rrf_sum_rmsnorm_fp8,
    rrf_sum_rmsnorm_fp8_ex,
    rrf_sum_rmsnorm_fp8_ptr,
    rrf_version,
)
