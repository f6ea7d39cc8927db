"""The multi-GPU form: all-reduce of per-GPU bf16 partials fused with the
residual, RMSNorm and per-row FP8 quantisation (rrf_allreduce_rmsnorm_fp8).

The kernel reads and writes the other ranks' buffers directly, so every
buffer a rank touches must be addressable from its GPU:

* ``PeerGroup``: one process per GPU; the buffers are allocated as torch
  symmetric memory (every rank maps every peer's allocation) and exchanged
  through the process group once, at construction.
* ``LocalGroup``: all ranks' buffers on one GPU and one launch that runs
  every rank (the same kernel and barriers; this GPU's memory stands in for
  the links), which is how the exchange is exercised on a single GPU.

This module marshals arguments only; the all-reduce, the norm and the
quantisation run in librrf.so (Modular docs `allreduce_rmsnorm_fp8`: 1-stage
and 2-stage paths; b12x PR #283: fixed rank order, rounded once).
"""
from __future__ import annotations

# Entries of the C header, for the helpers below that need no library.
RRF_AR_MAX_WORLD = 8
RRF_AR_SIGNAL_WORDS = (2 * RRF_AR_MAX_WORLD + 1) * 1024
RRF_AR_AUTO = 0


def _lib():
    from . import _lib as lib  # raises ImportError if librrf.so is missing
    return lib


def two_shot_rows(rows: int, world: int, rank: int) -> tuple[int, int]:
    """The rows [start, stop) rank ``rank`` computes in the two-shot mode:
    blocks of ceil(rows / world) rows in rank order (the last ones may be
    short or empty)."""
    per = -(-rows // world) if world else 0
    start = min(rank * per, rows)
    return start, min(start + per, rows)


def _torch():
    import torch
    return torch


def _check_rank_tensors(ts, like, what, dtype=None):
    torch = _torch()
    if len(ts) != len(like):
        raise ValueError(f"{what}: need one tensor per rank")
    for t, x in zip(ts, like):
        if t.device != x.device or not t.is_contiguous():
            raise ValueError(f"{what}: contiguous tensors on the partials' device")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{what}: dtype {dtype}")
    return torch


class LocalGroup:
    """``world`` ranks whose buffers all live on one GPU; every call runs all
    of them in one launch (each rank's blocks meet the others' at the same
    barriers as in a multi-GPU job).  Keeps the ranks' signal pads (which
    carry the calls' numbering themselves, so calls may be captured in a
    CUDA graph and replayed)."""

    def __init__(self, world: int, device=None):
        torch = _torch()
        if not 1 <= world <= RRF_AR_MAX_WORLD:
            raise ValueError(f"world must be in [1, {RRF_AR_MAX_WORLD}]")
        self.world = world
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.pads = [torch.zeros(RRF_AR_SIGNAL_WORDS, dtype=torch.int32, device=self.device)
                     for _ in range(world)]

    def reset(self):
        """Zero the pads (needed after a barrier wait ran out)."""
        for p in self.pads:
            p.zero_()

    def __call__(self, partials, gamma, eps, weight_offset, scale_ub, residual_in=None,
                 residual_out=None, q_out=None, scales_out=None, mode=RRF_AR_AUTO,
                 timeout_ns=0):
        """One call over the ranks' partials (``world`` bf16 tensors of one
        shape).  residual_in: one tensor per rank (the same values on every
        rank) or None; residual_out defaults to new tensors (pass residual_in
        for the in-place update).  Returns (q, scales, residual_out), lists
        with one tensor per rank."""
        torch = _torch()
        if len(partials) != self.world:
            raise ValueError("need one partial per rank")
        rows, cols = _lib()._rows_cols(partials)
        x0 = partials[0]
        if x0.device != self.device:
            raise ValueError("partials must be on the group's device")
        if gamma.dtype != torch.bfloat16 or gamma.numel() != cols or gamma.device != x0.device:
            raise ValueError("gamma must be a bf16 tensor of length cols on the same device")
        if residual_in is not None:
            _check_rank_tensors(residual_in, partials, "residual_in", torch.bfloat16)
            if residual_out is None:
                residual_out = [torch.empty_like(r) for r in residual_in]
            _check_rank_tensors(residual_out, partials, "residual_out", torch.bfloat16)
        if q_out is None:
            q_out = [torch.empty(x0.shape, dtype=torch.float8_e4m3fn, device=x0.device)
                     for _ in range(self.world)]
        if scales_out is None:
            scales_out = [torch.empty(tuple(x0.shape[:-1]) + (1,), dtype=torch.float32,
                                      device=x0.device) for _ in range(self.world)]
        _check_rank_tensors(q_out, partials, "q_out", torch.float8_e4m3fn)
        _check_rank_tensors(scales_out, partials, "scales_out", torch.float32)
        ptrs = (lambda ts: None if ts is None else [t.data_ptr() for t in ts])
        with torch.cuda.device(x0.device):
            _lib().rrf_allreduce_rmsnorm_fp8_ptr(
                ptrs(partials), ptrs(residual_in), ptrs(residual_out), ptrs(q_out),
                ptrs(scales_out), ptrs(self.pads), 0, self.world, rows, cols, gamma.data_ptr(),
                eps, weight_offset, scale_ub, mode, timeout_ns, _lib()._stream(x0.device))
        return q_out, scales_out, residual_out


def peer_layout(max_rows: int, cols: int, residual: bool = True):
    """Byte offsets of a rank's regions in its symmetric allocation (each
    256-byte aligned): input bf16 [max_rows, cols], residual bf16 (if any),
    codes [max_rows, cols], scales float32 [max_rows], signal pad.  Returns
    ({name: (offset, nbytes)}, total bytes)."""
    regions = [("input", max_rows * cols * 2)]
    if residual:
        regions.append(("residual", max_rows * cols * 2))
    regions += [("q", max_rows * cols), ("scales", max_rows * 4),
                ("pad", RRF_AR_SIGNAL_WORDS * 4)]
    out, off = {}, 0
    for name, nbytes in regions:
        out[name] = (off, nbytes)
        off += -(-nbytes // 256) * 256
    return out, off


class PeerGroup:
    """The multi-GPU call in a job with one process per GPU: every rank's
    input, residual, codes, scales and signal pad live in one torch
    symmetric-memory allocation of up to ``max_rows`` rows, mapped by every
    peer (exchanged once through ``group``).  A producer writes its partial
    into ``input(rows)`` (and the residual into ``residual(rows)``); a call
    then leaves every rank's codes, scales and updated residual in its own
    allocation."""

    def __init__(self, group, max_rows: int, cols: int, residual: bool = True, device=None):
        torch = _torch()
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if not 1 <= self.world <= RRF_AR_MAX_WORLD:
            raise ValueError(f"world must be in [1, {RRF_AR_MAX_WORLD}]")
        if cols % 8:
            raise ValueError("cols must be a multiple of 8")
        self.max_rows, self.cols, self.has_residual = max_rows, cols, residual
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.layout, total = peer_layout(max_rows, cols, residual)
        self.buf = symm_mem.empty(total, dtype=torch.uint8, device=self.device)
        self.handle = symm_mem.rendezvous(self.buf, group)
        bases = [int(p) for p in self.handle.buffer_ptrs]
        local = self.buf.data_ptr() - bases[self.rank]
        self.ptrs = {name: [b + local + off for b in bases]
                     for name, (off, _) in self.layout.items()}
        off, nbytes = self.layout["pad"]
        self.buf[off:off + nbytes].zero_()
        torch.cuda.synchronize(self.device)
        dist.barrier(group)

    def _view(self, name, rows, dtype, shape):
        off, _ = self.layout[name]
        itemsize = _torch().empty((), dtype=dtype).element_size()
        n = 1
        for s in shape:
            n *= s
        return self.buf[off:off + n * itemsize].view(dtype).view(shape)

    def input(self, rows: int):
        """This rank's partial [rows, cols] (bf16), to be written by its
        producer before the call."""
        return self._view("input", rows, _torch().bfloat16, (rows, self.cols))

    def residual(self, rows: int):
        """This rank's residual [rows, cols] (bf16), updated in place."""
        if not self.has_residual:
            raise ValueError("the group was made without a residual")
        return self._view("residual", rows, _torch().bfloat16, (rows, self.cols))

    def __call__(self, rows: int, gamma, eps, weight_offset, scale_ub, mode=RRF_AR_AUTO,
                 timeout_ns=0):
        """One call on the first ``rows`` rows (every rank makes the same
        call).  Returns views of this rank's (codes [rows, cols], scales
        [rows, 1], residual [rows, cols] or None)."""
        torch = _torch()
        if not 0 <= rows <= self.max_rows:
            raise ValueError("rows outside [0, max_rows]")
        if gamma.dtype != torch.bfloat16 or gamma.numel() != self.cols or \
                gamma.device != self.device:
            raise ValueError("gamma must be a bf16 tensor of length cols on the group's device")
        res = self.ptrs["residual"] if self.has_residual else None
        with torch.cuda.device(self.device):
            _lib().rrf_allreduce_rmsnorm_fp8_ptr(
                self.ptrs["input"], res, res, self.ptrs["q"], self.ptrs["scales"],
                self.ptrs["pad"], self.rank, 1, rows, self.cols, gamma.data_ptr(), eps,
                weight_offset, scale_ub, mode, timeout_ns, _lib()._stream(self.device))
        q = self._view("q", rows, torch.float8_e4m3fn, (rows, self.cols))
        scales = self._view("scales", rows, torch.float32, (rows, 1))
        return q, scales, (self.residual(rows) if self.has_residual else None)
