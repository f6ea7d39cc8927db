"""The sharded form across devices: each rank holds a column shard of every
row (Tenstorrent rmsnorm_2d.py, decode_forward / prefill_forward:
pre-all-gather statistics, all-gather, post-all-gather normalisation).

    stats, h = rrf_sum_rmsnorm_fp8_pre(...)      # this rank's shard
    all_gather(stats)                             # rows * 8 bytes per rank
    q, scales = rrf_rmsnorm_fp8_post(h, ..., gathered stats)

Both phases are the library's kernels; this module is the torch.distributed
glue (the collective is the only step here, and it moves statistics only).
"""
from __future__ import annotations

from . import _lib


def sharded_sum_rmsnorm_fp8(inputs, gamma, eps, weight_offset, scale_ub, residual_in=None,
                            residual_out=None, group=None):
    """The fused operation on this rank's column shard of every row.

    ``inputs``: R bf16 CUDA tensors [rows, cols_shard] (every rank the same
    shape); ``gamma``: this rank's bf16 [cols_shard]; ``group``: the process
    group of the ranks sharing the rows (None or a single rank: no exchange).
    Returns (q [rows, cols_shard], scales [rows, 1], h) -- every rank derives
    the same scales; h is the norm input (residual_out with a residual).
    """
    import torch
    import torch.distributed as dist
    stats, h = _lib.rrf_sum_rmsnorm_fp8_pre(inputs, gamma, weight_offset,
                                            residual_in=residual_in, residual_out=residual_out)
    world = 1
    if group is not None or (dist.is_available() and dist.is_initialized()):
        world = dist.get_world_size(group)
    rows, cols = stats.shape[0], inputs[0].shape[-1]
    if world > 1:
        gathered = torch.empty((world, rows, 2), dtype=stats.dtype, device=stats.device)
        dist.all_gather_into_tensor(gathered, stats, group=group)
    else:
        gathered = stats.reshape(1, rows, 2)
    q, scales = _lib.rrf_rmsnorm_fp8_post(h, gamma, gathered, cols * world, eps, weight_offset,
                                          scale_ub)
    return q, scales, h
