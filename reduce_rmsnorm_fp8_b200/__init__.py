"""Fused bf16 sum + residual + RMSNorm + per-row FP8 (e4m3fn) for B200.

A thin Python binding over the C ABI in ``include/rrf.h`` (``librrf.so``,
hand-written sm_100a CUDA kernels).  The functions here only marshal torch
tensors into pointers, sizes and the current CUDA stream; every step of the
operation runs in the library's kernels.  The library is loaded on first use
of any function or constant; if ``librrf.so`` has not been built
(``python -m reduce_rmsnorm_fp8_b200.build``) that first use raises
ImportError: there is no fallback.  (Importing the package alone does not
load it, so the build step itself can run from a fresh checkout.)

Functions, named after the C entry points:
  rrf_sum(inputs, out=None)
  rrf_sum_rmsnorm_fp8(inputs, gamma, eps, weight_offset, scale_ub,
                      residual_in=None, residual_out=None, q_out=None,
                      scales_out=None) -> (q, scales, residual_out)
  rrf_sum_rmsnorm_fp8_ex(..., variant=0, cluster_size=0, block_threads=0,
                         flags=0)
  rrf_plan_fused(num_inputs, rows, cols, sm_count) -> (cluster, threads, vpt)
  rrf_check_sum_args / rrf_check_fused_args (raw pointers, host only)
  rrf_device_error(clear=False) -> RRF_DEVICE_ERROR_* bits
  rrf_sum_rmsnorm_fp8_pre / rrf_rmsnorm_fp8_post: the two phases of the
      sharded form (a row's hidden dimension split across devices); the
      torch.distributed glue between them is in ``sharded.py``
"""
from __future__ import annotations

_EXPORTS = (
    "LIB_PATH", "RRF_MAX_COLS", "RRF_MAX_INPUTS", "RRF_VARIANT_AUTO", "RRF_VARIANT_CLUSTER",
    "RRF_VARIANT_ROW", "RRF_FLAG_NO_PDL", "RRF_FLAG_BARRIER_EXCHANGE",
    "RRF_FLAG_DEBUG_STARVE_EXCHANGE", "RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT", "RrfError",
    "Status", "lib", "rrf_check_fused_args", "rrf_check_sum_args",
    "rrf_debug_fail_next_launch", "rrf_debug_starve_next_gemm", "rrf_device_error", "rrf_last_cuda_error", "rrf_plan_fused",
    "rrf_status_string", "rrf_sum", "rrf_sum_ptr", "rrf_sum_rmsnorm_fp8",
    "rrf_sum_rmsnorm_fp8_ex", "rrf_sum_rmsnorm_fp8_ptr", "rrf_version", "RRF_MAX_SHARDS",
    "rrf_sum_rmsnorm_fp8_pre", "rrf_rmsnorm_fp8_post", "rrf_check_pre_args",
    "rrf_check_post_args", "RRF_DEVICE_ERROR_PEER_TIMEOUT", "RRF_AR_MAX_WORLD",
    "RRF_AR_MAX_BLOCKS", "RRF_AR_SIGNAL_WORDS", "RRF_AR_AUTO", "RRF_AR_ONE_SHOT",
    "RRF_AR_TWO_SHOT", "rrf_check_allreduce_args", "rrf_plan_allreduce",
    "rrf_allreduce_rmsnorm_fp8_ptr", "RRF_DEVICE_ERROR_GEMM_TIMEOUT", "rrf_scaled_mm_fp8",
    "rrf_check_scaled_mm_args", "rrf_sum_rmsnorm_mxfp8", "rrf_check_mxfp8_args",
    "mx_blocked", "mx_blocked_bytes", "rrf_scaled_mm_mxfp8", "rrf_check_scaled_mm_mx_args",
    "RRF_AR_STATIC_MAX_WORLD", "rrf_allreduce_rmsnorm_fp8_static_ptr",
    "rrf_plan_scaled_mm", "RRF_GEMM_KERNEL_PAIR", "RRF_GEMM_KERNEL_TILE",
    "RRF_GEMM_KERNEL_SWAP", "RRF_FLAG_NO_PREFETCH", "RRF_FLAG_PREFETCH", "rrf_plan_fused_ex",
    "RRF_DEVICE_ERROR_BOUNDS",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import _lib  # raises ImportError if librrf.so is missing
        return getattr(_lib, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(list(globals()) + list(_EXPORTS))
