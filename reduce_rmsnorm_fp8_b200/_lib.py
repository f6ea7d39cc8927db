"""ctypes binding of librrf.so: argument marshalling only."""
from __future__ import annotations

import ctypes
import enum
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# RRF_DEBUG_LIBRARY=1 selects the bounds-checking build (librrf_debug.so).
LIB_PATH = os.path.join(_PKG, "librrf_debug.so" if os.environ.get("RRF_DEBUG_LIBRARY") == "1"
                        else "librrf.so")

RRF_MAX_INPUTS = 16
RRF_MAX_COLS = 16 * 256 * 8 * 8
RRF_VARIANT_AUTO = 0
RRF_VARIANT_ROW = 1
RRF_VARIANT_CLUSTER = 2
RRF_FLAG_NO_PDL = 1
RRF_FLAG_BARRIER_EXCHANGE = 2
RRF_FLAG_DEBUG_STARVE_EXCHANGE = 0x100
RRF_FLAG_NO_PREFETCH = 4
RRF_FLAG_PREFETCH = 8
RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT = 1
RRF_MAX_SHARDS = 64
RRF_DEVICE_ERROR_PEER_TIMEOUT = 2
RRF_AR_MAX_WORLD = 8
RRF_AR_MAX_BLOCKS = 1024
RRF_AR_SIGNAL_WORDS = (2 * RRF_AR_MAX_WORLD + 1) * RRF_AR_MAX_BLOCKS
RRF_AR_STATIC_MAX_WORLD = 8  # ranks whose pads the library's fixed array holds
RRF_AR_AUTO = 0
RRF_AR_ONE_SHOT = 1
RRF_AR_TWO_SHOT = 2
RRF_DEVICE_ERROR_GEMM_TIMEOUT = 4
RRF_DEVICE_ERROR_BOUNDS = 8
RRF_GEMM_KERNEL_PAIR = 1
RRF_GEMM_KERNEL_TILE = 2
RRF_GEMM_KERNEL_SWAP = 3


class Status(enum.IntEnum):
    OK = 0
    ERR_NULL = 1
    ERR_RANKS = 2
    ERR_SHAPE = 3
    ERR_ALIGN = 4
    ERR_ALIAS = 5
    ERR_VALUE = 6
    ERR_UNSUPPORTED = 7
    ERR_CUDA = 8


class RrfError(RuntimeError):
    """A non-zero rrf_status from the library."""

    def __init__(self, status: int, cuda_error: int = 0):
        self.status = Status(status)
        self.cuda_error = cuda_error
        msg = f"{self.status.name}: {rrf_status_string(status)}"
        if self.status == Status.ERR_CUDA:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m reduce_rmsnorm_fp8_b200.build` "
        "(the CUDA kernels are the only implementation; there is no fallback)")

lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float
_ptrs = ctypes.POINTER(ctypes.c_void_p)

lib.rrf_sum.restype = _int
lib.rrf_sum.argtypes = [_ptrs, _int, _i64, _i64, _vp, _vp]
_fused_args = [_ptrs, _int, _i64, _i64, _vp, _vp, _vp, _f32, _f32, _f32, _vp, _vp]
lib.rrf_sum_rmsnorm_fp8.restype = _int
lib.rrf_sum_rmsnorm_fp8.argtypes = _fused_args + [_vp]
lib.rrf_sum_rmsnorm_fp8_ex.restype = _int
lib.rrf_sum_rmsnorm_fp8_ex.argtypes = _fused_args + [_int, _int, _int, _int, _vp]
lib.rrf_plan_fused.restype = _int
lib.rrf_plan_fused.argtypes = [_int, _i64, _i64, _int, _int, ctypes.POINTER(_int),
                               ctypes.POINTER(_int), ctypes.POINTER(_int)]
lib.rrf_plan_fused_ex.restype = _int
lib.rrf_plan_fused_ex.argtypes = [_int, _i64, _i64, _int, _int] + [ctypes.POINTER(_int)] * 4
lib.rrf_check_sum_args.restype = _int
lib.rrf_check_sum_args.argtypes = [_ptrs, _int, _i64, _i64, _vp]
lib.rrf_check_fused_args.restype = _int
lib.rrf_check_fused_args.argtypes = _fused_args
lib.rrf_status_string.restype = ctypes.c_char_p
lib.rrf_status_string.argtypes = [_int]
lib.rrf_last_cuda_error.restype = _int
lib.rrf_last_cuda_error.argtypes = []
lib.rrf_debug_fail_next_launch.restype = None
lib.rrf_debug_fail_next_launch.argtypes = [_int]
lib.rrf_debug_starve_next_gemm.restype = None
lib.rrf_debug_starve_next_gemm.argtypes = []
lib.rrf_sum_rmsnorm_fp8_pre.restype = _int
lib.rrf_sum_rmsnorm_fp8_pre.argtypes = [_ptrs, _int, _i64, _i64, _vp, _vp, _vp, _vp, _f32, _vp,
                                        _vp]
lib.rrf_rmsnorm_fp8_post.restype = _int
lib.rrf_rmsnorm_fp8_post.argtypes = [_vp, _i64, _i64, _vp, _int, _i64, _vp, _f32, _f32, _f32,
                                     _vp, _vp, _vp]
lib.rrf_check_pre_args.restype = _int
lib.rrf_check_pre_args.argtypes = [_ptrs, _int, _i64, _i64, _vp, _vp, _vp, _vp, _f32, _vp]
lib.rrf_check_post_args.restype = _int
lib.rrf_check_post_args.argtypes = [_vp, _i64, _i64, _vp, _int, _i64, _vp, _f32, _f32, _f32,
                                    _vp, _vp]
_ar_args = [_ptrs, _ptrs, _ptrs, _ptrs, _ptrs, _ptrs, _int, _int, _int, _i64, _i64, _vp, _f32,
            _f32, _f32, _int]
lib.rrf_allreduce_rmsnorm_fp8.restype = _int
lib.rrf_allreduce_rmsnorm_fp8.argtypes = _ar_args + [ctypes.c_uint64, _vp]
lib.rrf_allreduce_rmsnorm_fp8_static.restype = _int
lib.rrf_allreduce_rmsnorm_fp8_static.argtypes = [_ptrs] * 5 + [_int, _i64, _i64, _vp, _f32, _f32,
                                                               _f32, _int, ctypes.c_uint64, _vp]
lib.rrf_check_allreduce_args.restype = _int
lib.rrf_check_allreduce_args.argtypes = _ar_args
lib.rrf_plan_allreduce.restype = _int
lib.rrf_plan_allreduce.argtypes = [_int, _i64, _i64, _int, _int, _int] + [ctypes.POINTER(_int)] * 4
lib.rrf_sum_rmsnorm_mxfp8.restype = _int
lib.rrf_sum_rmsnorm_mxfp8.argtypes = [_ptrs, _int, _i64, _i64, _vp, _vp, _vp, _f32, _f32, _vp,
                                      _vp, _vp]
lib.rrf_check_mxfp8_args.restype = _int
lib.rrf_check_mxfp8_args.argtypes = [_ptrs, _int, _i64, _i64, _vp, _vp, _vp, _f32, _f32, _vp,
                                     _vp]
lib.rrf_sum_rmsnorm_mxfp8_blocked.restype = _int
lib.rrf_sum_rmsnorm_mxfp8_blocked.argtypes = lib.rrf_sum_rmsnorm_mxfp8.argtypes
lib.rrf_scaled_mm_mxfp8.restype = _int
lib.rrf_scaled_mm_mxfp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
lib.rrf_check_scaled_mm_mx_args.restype = _int
lib.rrf_check_scaled_mm_mx_args.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64]
lib.rrf_scaled_mm_fp8.restype = _int
lib.rrf_scaled_mm_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
lib.rrf_check_scaled_mm_args.restype = _int
lib.rrf_check_scaled_mm_args.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64]
lib.rrf_plan_scaled_mm.restype = _int
lib.rrf_plan_scaled_mm.argtypes = [_i64, _i64, _i64, _int, _int] + [ctypes.POINTER(_int)] * 4 + \
    [ctypes.POINTER(_i64)] * 2
lib.rrf_device_error.restype = _int
lib.rrf_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), _int]
lib.rrf_version.restype = ctypes.c_char_p
lib.rrf_version.argtypes = []


def rrf_status_string(status: int) -> str:
    return lib.rrf_status_string(int(status)).decode()


def rrf_last_cuda_error() -> int:
    return lib.rrf_last_cuda_error()


def rrf_debug_fail_next_launch(cuda_error: int) -> None:
    lib.rrf_debug_fail_next_launch(int(cuda_error))


def rrf_debug_starve_next_gemm() -> None:
    """The next GEMM call on this thread runs its epilogue's bounded wait
    out (test hook; see include/rrf.h)."""
    lib.rrf_debug_starve_next_gemm()


def rrf_device_error(clear: bool = False) -> int:
    """The device error word of the current device (RRF_DEVICE_ERROR_* bits);
    synchronises the device."""
    v = ctypes.c_uint(0)
    _raise_on(lib.rrf_device_error(ctypes.byref(v), int(bool(clear))))
    return v.value


def rrf_version() -> str:
    return lib.rrf_version().decode()


def _raise_on(status: int) -> None:
    if status != 0:
        raise RrfError(status, lib.rrf_last_cuda_error() if status == Status.ERR_CUDA else 0)


def _ptr_table(ptrs):
    return (ctypes.c_void_p * max(1, len(ptrs)))(*[p or None for p in ptrs])


# ------------------------------------------------------- raw pointer calls ---

def rrf_check_sum_args(input_ptrs, rows, cols, out_ptr) -> int:
    return lib.rrf_check_sum_args(_ptr_table(input_ptrs), len(input_ptrs), rows, cols,
                                  out_ptr or None)


def rrf_check_fused_args(input_ptrs, rows, cols, residual_in, residual_out, gamma, eps,
                         weight_offset, scale_ub, q_out, scales_out) -> int:
    return lib.rrf_check_fused_args(_ptr_table(input_ptrs), len(input_ptrs), rows, cols,
                                    residual_in or None, residual_out or None, gamma or None,
                                    eps, weight_offset, scale_ub, q_out or None,
                                    scales_out or None)


def rrf_plan_fused(num_inputs: int, rows: int, cols: int, sm_count: int, residual=True):
    """The launch the library would pick: (cluster_size, block_threads,
    vecs_per_thread)."""
    c, t, v = _int(), _int(), _int()
    _raise_on(lib.rrf_plan_fused(num_inputs, rows, cols, int(bool(residual)), sm_count,
                                 ctypes.byref(c), ctypes.byref(t), ctypes.byref(v)))
    return c.value, t.value, v.value


def rrf_plan_fused_ex(num_inputs: int, rows: int, cols: int, sm_count: int, residual=True):
    """The launch the library would pick, with its L2-prefetch choice:
    (cluster_size, block_threads, vecs_per_thread, prefetch)."""
    out = [_int() for _ in range(4)]
    _raise_on(lib.rrf_plan_fused_ex(num_inputs, rows, cols, int(bool(residual)), sm_count,
                                    *[ctypes.byref(o) for o in out]))
    return tuple(o.value for o in out)


def _ar_tables(inputs, residual_in, residual_out, q_out, scales_out, signals):
    opt = (lambda t: None if t is None else _ptr_table(t))
    return tuple(opt(t) for t in (inputs, residual_in, residual_out, q_out, scales_out, signals))


def rrf_check_allreduce_args(inputs, residual_in, residual_out, q_out, scales_out, signals,
                             rank, local_ranks, rows, cols, gamma, eps, weight_offset, scale_ub,
                             mode, world=None) -> int:
    """Host validation of the multi-GPU call on raw pointers (lists of
    ``world`` ints; residual lists may be None)."""
    world = len(inputs) if world is None else world
    return lib.rrf_check_allreduce_args(
        *_ar_tables(inputs, residual_in, residual_out, q_out, scales_out, signals), world,
        rank, local_ranks, rows, cols, gamma or None, eps, weight_offset, scale_ub, mode)


def rrf_plan_allreduce(world: int, rows: int, cols: int, sm_count: int, residual=True,
                       mode: int = 0):
    """The multi-GPU call's choice: (mode, cluster_size, block_threads,
    vecs_per_thread)."""
    out = [_int() for _ in range(4)]
    _raise_on(lib.rrf_plan_allreduce(world, rows, cols, int(bool(residual)), mode, sm_count,
                                     *[ctypes.byref(o) for o in out]))
    return tuple(o.value for o in out)


def rrf_allreduce_rmsnorm_fp8_ptr(inputs, residual_in, residual_out, q_out, scales_out, signals,
                                  rank, local_ranks, rows, cols, gamma, eps, weight_offset,
                                  scale_ub, mode=0, timeout_ns=0, stream=0) -> None:
    """rrf_allreduce_rmsnorm_fp8 on raw pointers: every list holds one device
    address per rank, as this GPU addresses that rank's buffer."""
    _raise_on(lib.rrf_allreduce_rmsnorm_fp8(
        *_ar_tables(inputs, residual_in, residual_out, q_out, scales_out, signals), len(inputs),
        rank, local_ranks, rows, cols, gamma or None, eps, weight_offset, scale_ub, mode,
        timeout_ns, stream or None))


def rrf_allreduce_rmsnorm_fp8_static_ptr(inputs, residual_in, residual_out, q_out, scales_out,
                                         rows, cols, gamma, eps, weight_offset, scale_ub,
                                         mode=0, timeout_ns=0, stream=0) -> None:
    """rrf_allreduce_rmsnorm_fp8_static on raw pointers: every rank's buffers
    on the current GPU, all ranks in one launch, the signal pads held by the
    library (nothing is allocated)."""
    tables = _ar_tables(inputs, residual_in, residual_out, q_out, scales_out, None)[:5]
    _raise_on(lib.rrf_allreduce_rmsnorm_fp8_static(
        *tables, len(inputs), rows, cols, gamma or None, eps, weight_offset, scale_ub, mode,
        timeout_ns, stream or None))


def rrf_sum_ptr(input_ptrs, rows, cols, out_ptr, stream=0) -> None:
    """rrf_sum on raw device pointers and a raw cudaStream_t handle."""
    _raise_on(lib.rrf_sum(_ptr_table(input_ptrs), len(input_ptrs), rows, cols,
                          out_ptr or None, stream or None))


def rrf_sum_rmsnorm_fp8_ptr(input_ptrs, rows, cols, residual_in, residual_out, gamma, eps,
                            weight_offset, scale_ub, q_out, scales_out, variant=0,
                            cluster_size=0, block_threads=0, flags=0, stream=0) -> None:
    """rrf_sum_rmsnorm_fp8_ex on raw device pointers and a raw stream handle."""
    _raise_on(lib.rrf_sum_rmsnorm_fp8_ex(
        _ptr_table(input_ptrs), len(input_ptrs), rows, cols, residual_in or None,
        residual_out or None, gamma or None, eps, weight_offset, scale_ub, q_out or None,
        scales_out or None, variant, cluster_size, block_threads, flags, stream or None))


# ------------------------------------------------------------ torch calls ---

def _torch():
    import torch
    return torch


def _rows_cols(inputs):
    torch = _torch()
    if len(inputs) == 0:
        raise ValueError("need at least one input")
    x0 = inputs[0]
    for x in inputs:
        if x.dtype != torch.bfloat16:
            raise TypeError("inputs must be bfloat16")
        if x.shape != x0.shape or x.device != x0.device:
            raise ValueError("inputs must share shape and device")
        if x.device.type != "cuda":
            raise ValueError("inputs must be CUDA tensors")
        if not x.is_contiguous():
            raise ValueError("inputs must be contiguous")
    if x0.dim() == 0:
        raise ValueError("inputs must have a last dimension")
    cols = x0.shape[-1]
    rows = x0.numel() // cols if cols else 0
    return rows, cols


def _stream(device):
    return _torch().cuda.current_stream(device).cuda_stream


def rrf_sum(inputs, out=None):
    """Sum of the bf16 CUDA tensors ``inputs`` (fp32 in list order, rounded
    to bf16 once), into ``out`` (allocated if None).  Returns ``out``."""
    torch = _torch()
    rows, cols = _rows_cols(inputs)
    dev = inputs[0].device
    if out is None:
        out = torch.empty_like(inputs[0])
    with torch.cuda.device(dev):
        rrf_sum_ptr([x.data_ptr() for x in inputs], rows, cols, out.data_ptr(),
                    _stream(dev))
    return out


def rrf_sum_rmsnorm_fp8_ex(inputs, gamma, eps, weight_offset, scale_ub, residual_in=None,
                           residual_out=None, q_out=None, scales_out=None, variant=0,
                           cluster_size=0, block_threads=0, flags=0):
    """The fused operation with a forced launch (variant, cluster size, block
    size; 0 = automatic; flags RRF_FLAG_NO_PDL).  Returns (q, scales,
    residual_out)."""
    torch = _torch()
    rows, cols = _rows_cols(inputs)
    x0 = inputs[0]
    dev = x0.device
    if gamma.dtype != torch.bfloat16 or gamma.numel() != cols or gamma.device != dev:
        raise ValueError("gamma must be a bf16 tensor of length cols on the inputs' device")
    if residual_in is not None and residual_out is None:
        residual_out = torch.empty_like(residual_in)
    if q_out is None:
        q_out = torch.empty(x0.shape, dtype=torch.float8_e4m3fn, device=dev)
    if scales_out is None:
        scales_out = torch.empty(tuple(x0.shape[:-1]) + (1,), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rrf_sum_rmsnorm_fp8_ptr(
            [x.data_ptr() for x in inputs], rows, cols,
            residual_in.data_ptr() if residual_in is not None else 0,
            residual_out.data_ptr() if residual_out is not None else 0,
            gamma.data_ptr(), eps, weight_offset, scale_ub, q_out.data_ptr(),
            scales_out.data_ptr(), variant, cluster_size, block_threads, flags, _stream(dev))
    return q_out, scales_out, residual_out


def rrf_sum_rmsnorm_fp8(inputs, gamma, eps, weight_offset, scale_ub, residual_in=None,
                        residual_out=None, q_out=None, scales_out=None):
    """The fused operation.  ``inputs``: R bf16 CUDA tensors [..., cols];
    ``gamma``: bf16 [cols]; ``residual_in`` (optional) bf16 like the inputs,
    written to ``residual_out`` (a new tensor if None; pass residual_in for an
    in-place update).  Returns (q: float8_e4m3fn like the inputs, scales:
    float32 [..., 1], residual_out or None)."""
    return rrf_sum_rmsnorm_fp8_ex(inputs, gamma, eps, weight_offset, scale_ub, residual_in,
                                  residual_out, q_out, scales_out)


def rrf_check_mxfp8_args(input_ptrs, rows, cols, residual_in, residual_out, gamma, eps,
                         weight_offset, q_out, scales_mx_out) -> int:
    return lib.rrf_check_mxfp8_args(_ptr_table(input_ptrs), len(input_ptrs), rows, cols,
                                    residual_in or None, residual_out or None, gamma or None,
                                    eps, weight_offset, q_out or None, scales_mx_out or None)


def mx_blocked_bytes(rows: int, cols: int) -> int:
    """Bytes of MX scale codes in the blocked order (rows rounded up to 128)."""
    return -(-rows // 128) * 128 * (cols // 32)


def mx_blocked(codes):
    """Row-major MX scale codes [rows, cols / 32] (uint8 tensor) -> the
    blocked order that the block-scaled GEMM reads (a flat uint8 tensor of
    mx_blocked_bytes(rows, cols) bytes; rounded-up rows zero).  A layout
    change for preparing weights once, not a step of the call."""
    torch = _torch()
    rows, nb = codes.shape
    if nb % 4:
        raise ValueError("cols must be a multiple of 128")
    pad = -(-rows // 128) * 128
    p = torch.zeros((pad, nb), dtype=torch.uint8, device=codes.device)
    p[:rows] = codes
    # [rows/128, 4 (r/32 % 4), 32 (r % 32), nb/4, 4 (j % 4)] -> [rows/128, nb/4, 32, 4, 4]
    return p.view(pad // 128, 4, 32, nb // 4, 4).permute(0, 3, 2, 1, 4).contiguous().view(-1)


def rrf_sum_rmsnorm_mxfp8(inputs, gamma, eps, weight_offset, residual_in=None,
                          residual_out=None, q_out=None, scales_mx_out=None, blocked=False):
    """The fused operation with MX output: one E8M0 scale code per 32
    elements.  Returns (q: float8_e4m3fn like the inputs, scales_mx: uint8
    [..., cols / 32] or, with ``blocked``, a flat uint8 tensor in the blocked
    order for rrf_scaled_mm_mxfp8, residual_out or None)."""
    torch = _torch()
    rows, cols = _rows_cols(inputs)
    x0 = inputs[0]
    dev = x0.device
    if gamma.dtype != torch.bfloat16 or gamma.numel() != cols or gamma.device != dev:
        raise ValueError("gamma must be a bf16 tensor of length cols on the inputs' device")
    if cols % (128 if blocked else 32):
        raise ValueError(f"cols must be a multiple of {128 if blocked else 32}")
    if residual_in is not None and residual_out is None:
        residual_out = torch.empty_like(residual_in)
    if q_out is None:
        q_out = torch.empty(x0.shape, dtype=torch.float8_e4m3fn, device=dev)
    if scales_mx_out is None:
        shape = (mx_blocked_bytes(rows, cols),) if blocked else \
            tuple(x0.shape[:-1]) + (cols // 32,)
        scales_mx_out = torch.empty(shape, dtype=torch.uint8, device=dev)
    fn = lib.rrf_sum_rmsnorm_mxfp8_blocked if blocked else lib.rrf_sum_rmsnorm_mxfp8
    with torch.cuda.device(dev):
        _raise_on(fn(
            _ptr_table([x.data_ptr() for x in inputs]), len(inputs), rows, cols,
            residual_in.data_ptr() if residual_in is not None else None,
            residual_out.data_ptr() if residual_out is not None else None, gamma.data_ptr(),
            eps, weight_offset, q_out.data_ptr(), scales_mx_out.data_ptr(), _stream(dev)))
    return q_out, scales_mx_out, residual_out


# ------------------------------------------------------------ sharded norm ---

def rrf_check_pre_args(input_ptrs, rows, cols, residual_in, residual_out, h_out, gamma,
                       weight_offset, stats_out) -> int:
    return lib.rrf_check_pre_args(_ptr_table(input_ptrs), len(input_ptrs), rows, cols,
                                  residual_in or None, residual_out or None, h_out or None,
                                  gamma or None, weight_offset, stats_out or None)


def rrf_check_post_args(h, rows, cols, stats, shards, total_cols, gamma, eps, weight_offset,
                        scale_ub, q_out, scales_out) -> int:
    return lib.rrf_check_post_args(h or None, rows, cols, stats or None, shards, total_cols,
                                   gamma or None, eps, weight_offset, scale_ub, q_out or None,
                                   scales_out or None)


def rrf_sum_rmsnorm_fp8_pre(inputs, gamma, weight_offset, residual_in=None, residual_out=None,
                            h_out=None, stats_out=None):
    """Phase 1 of the sharded norm on this device's column shard.  Returns
    (stats float32 [rows, 2], h) where h is residual_out (with a residual) or
    h_out (without)."""
    torch = _torch()
    rows, cols = _rows_cols(inputs)
    x0 = inputs[0]
    dev = x0.device
    if gamma.dtype != torch.bfloat16 or gamma.numel() != cols or gamma.device != dev:
        raise ValueError("gamma must be a bf16 tensor of length cols on the inputs' device")
    if residual_in is not None:
        if residual_out is None:
            residual_out = torch.empty_like(residual_in)
        h = residual_out
    else:
        if h_out is None:
            h_out = torch.empty_like(x0)
        h = h_out
    if stats_out is None:
        stats_out = torch.empty((rows, 2), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _raise_on(lib.rrf_sum_rmsnorm_fp8_pre(
            _ptr_table([x.data_ptr() for x in inputs]), len(inputs), rows, cols,
            residual_in.data_ptr() if residual_in is not None else None,
            residual_out.data_ptr() if residual_out is not None else None,
            h_out.data_ptr() if h_out is not None else None, gamma.data_ptr(), weight_offset,
            stats_out.data_ptr(), _stream(dev)))
    return stats_out, h


def rrf_rmsnorm_fp8_post(h, gamma, stats, total_cols, eps, weight_offset, scale_ub, q_out=None,
                         scales_out=None, write_scales=True):
    """Phase 2 of the sharded norm: ``stats`` float32 [shards, rows, 2] (all
    shards' phase-1 statistics, in shard order).  Returns (q, scales or None)."""
    torch = _torch()
    if h.dtype != torch.bfloat16 or not h.is_contiguous() or h.device.type != "cuda":
        raise ValueError("h must be a contiguous bf16 CUDA tensor")
    cols = h.shape[-1]
    rows = h.numel() // cols if cols else 0
    dev = h.device
    shards = stats.shape[0]
    if stats.dtype != torch.float32 or tuple(stats.shape) != (shards, rows, 2) or \
            not stats.is_contiguous():
        raise ValueError("stats must be a contiguous float32 [shards, rows, 2] tensor")
    if q_out is None:
        q_out = torch.empty(h.shape, dtype=torch.float8_e4m3fn, device=dev)
    if scales_out is None and write_scales:
        scales_out = torch.empty(tuple(h.shape[:-1]) + (1,), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _raise_on(lib.rrf_rmsnorm_fp8_post(
            h.data_ptr(), rows, cols, stats.data_ptr(), shards, total_cols, gamma.data_ptr(),
            eps, weight_offset, scale_ub, q_out.data_ptr(),
            scales_out.data_ptr() if scales_out is not None else None, _stream(dev)))
    return q_out, scales_out


def rrf_check_scaled_mm_args(a, a_scale, b, b_scale, bias, out, M, N, K) -> int:
    """Host validation of the FP8 GEMM on raw pointers."""
    return lib.rrf_check_scaled_mm_args(a or None, a_scale or None, b or None, b_scale or None,
                                        bias or None, out or None, M, N, K)


def rrf_plan_scaled_mm(M: int, N: int, K: int, sm_count: int, mx: bool = False) -> dict:
    """The GEMM kernel rrf_scaled_mm_fp8 (or, mx=True, rrf_scaled_mm_mxfp8)
    runs for an M x N x K product on sm_count SMs (host only)."""
    ints = [_int() for _ in range(4)]
    longs = [_i64() for _ in range(2)]
    _raise_on(lib.rrf_plan_scaled_mm(M, N, K, int(bool(mx)), sm_count,
                                     *[ctypes.byref(o) for o in ints + longs]))
    names = {RRF_GEMM_KERNEL_PAIR: "pair", RRF_GEMM_KERNEL_TILE: "tile",
             RRF_GEMM_KERNEL_SWAP: "swap"}
    return {"kernel": names.get(ints[0].value), "a_rows": ints[1].value,
            "tile_n": ints[2].value, "k_tiles_per_stage": ints[3].value,
            "tiles": longs[0].value, "ctas": longs[1].value}


def rrf_scaled_mm_fp8(a, a_scale, b, b_scale, bias=None, out=None):
    """out = RN_bf16((a @ b^T) * a_scale * b_scale + bias) on the tensor
    cores.  a: float8_e4m3fn [M, K] (e.g. rrf_sum_rmsnorm_fp8's codes), a_scale
    float32 [M] or [M, 1] (its scales), b: float8_e4m3fn [N, K] (a weight
    stored like a linear layer's), b_scale float32 [N], bias bf16 [N] or None.
    Returns out, bf16 [M, N]."""
    torch = _torch()
    for t, name in ((a, "a"), (b, "b")):
        if t.dtype != torch.float8_e4m3fn or t.dim() != 2 or not t.is_contiguous() or \
                t.device.type != "cuda":
            raise ValueError(f"{name} must be a contiguous 2-D float8_e4m3fn CUDA tensor")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b need the same K")
    dev = a.device
    for t, n, name in ((a_scale, M, "a_scale"), (b_scale, N, "b_scale")):
        if t.dtype != torch.float32 or t.numel() != n or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must be a contiguous float32 tensor of {n} values")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N or
                             bias.device != dev):
        raise ValueError("bias must be a bf16 tensor of N values")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _raise_on(lib.rrf_scaled_mm_fp8(
            a.data_ptr(), a_scale.data_ptr(), b.data_ptr(), b_scale.data_ptr(),
            bias.data_ptr() if bias is not None else None, out.data_ptr(), M, N, K,
            _stream(dev)))
    return out


def rrf_check_scaled_mm_mx_args(a, sa, b, sb, bias, out, M, N, K) -> int:
    """Host validation of the MX GEMM on raw pointers."""
    return lib.rrf_check_scaled_mm_mx_args(a or None, sa or None, b or None, sb or None,
                                           bias or None, out or None, M, N, K)


def rrf_scaled_mm_mxfp8(a, sa, b, sb, bias=None, out=None):
    """out = RN_bf16((a * 2^(sa - 127)) @ (b * 2^(sb - 127))^T + bias) on
    the tensor cores' block-scaled MMA.  a: float8_e4m3fn [M, K], b:
    float8_e4m3fn [N, K]; sa / sb: uint8 E8M0 codes in the blocked order
    (rrf_sum_rmsnorm_mxfp8(..., blocked=True) for a, mx_blocked for a
    weight); bias bf16 [N] or None.  Returns out, bf16 [M, N]."""
    torch = _torch()
    for t, name in ((a, "a"), (b, "b")):
        if t.dtype != torch.float8_e4m3fn or t.dim() != 2 or not t.is_contiguous() or \
                t.device.type != "cuda":
            raise ValueError(f"{name} must be a contiguous 2-D float8_e4m3fn CUDA tensor")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b need the same K")
    dev = a.device
    for t, n, name in ((sa, M, "sa"), (sb, N, "sb")):
        if t.dtype != torch.uint8 or t.numel() != mx_blocked_bytes(n, K) or \
                not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must hold the blocked scale codes of {n} rows")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N or
                             bias.device != dev):
        raise ValueError("bias must be a bf16 tensor of N values")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _raise_on(lib.rrf_scaled_mm_mxfp8(
            a.data_ptr(), sa.data_ptr(), b.data_ptr(), sb.data_ptr(),
            bias.data_ptr() if bias is not None else None, out.data_ptr(), M, N, K,
            _stream(dev)))
    return out
