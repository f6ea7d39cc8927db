"""Oracle for the fused bf16 sum + residual + RMSNorm + per-row FP8 operation.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
leg of the benchmark may import this package.  It loads ``rrf_oracle.c`` (plain
single-threaded C, built here with gcc) through ctypes and exposes it on numpy
arrays.  It imports nothing from the CUDA package and the CUDA package imports
nothing from it.

bf16 tensors travel as numpy ``uint16`` arrays of bit patterns, fp8 e4m3fn as
``uint8`` codes, scales as ``float32``.  What each function computes, and the
pages it follows, is stated in ``rrf_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rrf_oracle.c")
# the row-parallel driver (no arithmetic of its own), linked into the same library
_SRC_MT = os.path.join(_HERE, "rrf_oracle_mt.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

# -ffp-contract=off: no fused multiply-add, every fp32 operation rounds once.
CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-msse2", "-mfpmath=sse", "-Wall", "-Wextra"]

_lock = threading.Lock()
_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile ``src`` (default ``rrf_oracle.c``) and the row-parallel driver
    ``rrf_oracle_mt.c`` into a shared library (gcc)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    srcs = [src, _SRC_MT]
    stale = not os.path.exists(out) or any(os.path.getmtime(out) < os.path.getmtime(f)
                                           for f in srcs)
    if force or stale:
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, *srcs, "-lm", "-lpthread"], check=True)
        os.replace(tmp, out)
    return out


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bf16_rows(a, rows: int, cols: int) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 arrays are passed as uint16 bit patterns")
    if a.size != rows * cols:
        raise ValueError(f"expected {rows}x{cols} elements, got {a.size}")
    return a.reshape(rows, cols)


def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


class Oracle:
    """The oracle's functions, bound to one build of ``rrf_oracle.c``."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i64 = ctypes.c_int64
        vp = ctypes.c_void_p
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_bf16_round_array.restype = None
        lib.oracle_bf16_round_array.argtypes = [vp, vp, i64]
        lib.oracle_e4m3_encode_array.restype = None
        lib.oracle_e4m3_encode_array.argtypes = [vp, vp, i64]
        lib.oracle_sum.restype = None
        lib.oracle_sum.argtypes = [ctypes.POINTER(u16p), ctypes.c_int, i64, i64, vp]
        lib.oracle_sum_rmsnorm_fp8_rows.restype = None
        lib.oracle_sum_rmsnorm_fp8_rows.argtypes = [
            ctypes.POINTER(u16p), ctypes.c_int, i64, i64, i64, vp, vp, vp,
            ctypes.c_float, ctypes.c_float, ctypes.c_float, vp, vp, vp, vp]
        lib.oracle_cores.restype = ctypes.c_int
        lib.oracle_cores.argtypes = []
        lib.oracle_sum_rmsnorm_fp8_mt.restype = ctypes.c_int
        lib.oracle_sum_rmsnorm_fp8_mt.argtypes = [
            ctypes.POINTER(u16p), ctypes.c_int, i64, i64, vp, vp, vp, ctypes.c_float,
            ctypes.c_float, ctypes.c_float, vp, vp, ctypes.c_int]
        lib.oracle_mx_scale_code.restype = ctypes.c_uint8
        lib.oracle_mx_scale_code.argtypes = [ctypes.c_float]
        lib.oracle_sum_rmsnorm_mxfp8_rows.restype = None
        lib.oracle_sum_rmsnorm_mxfp8_rows.argtypes = [
            ctypes.POINTER(u16p), ctypes.c_int, i64, i64, i64, vp, vp, vp, ctypes.c_float,
            ctypes.c_float, vp, vp, vp, vp]
        lib.oracle_e8m0_decode.restype = ctypes.c_double
        lib.oracle_e8m0_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_scaled_mm_mx.restype = None
        lib.oracle_scaled_mm_mx.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
        lib.oracle_bf16_round_double.restype = ctypes.c_uint16
        lib.oracle_bf16_round_double.argtypes = [ctypes.c_double]
        lib.oracle_scaled_mm.restype = None
        lib.oracle_scaled_mm.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
        self.lib = lib
        self.path = lib_path

    @staticmethod
    def _table(inputs, rows, cols):
        arrs = [_bf16_rows(x, rows, cols) for x in inputs]
        u16p = ctypes.POINTER(ctypes.c_uint16)
        table = (u16p * len(arrs))(*[a.ctypes.data_as(u16p) for a in arrs])
        return arrs, table

    # ------------------------------------------------------------ scalars ---
    def bf16_round(self, values) -> np.ndarray:
        """float32 -> nearest bf16 (ties to even), as uint16 bit patterns."""
        v = np.ascontiguousarray(values, dtype=np.float32)
        out = np.empty(v.shape, dtype=np.uint16)
        self.lib.oracle_bf16_round_array(_ptr(v), _ptr(out), v.size)
        return out

    def e4m3_decode(self, codes) -> np.ndarray:
        """e4m3fn codes -> float64 values (NaN for 0x7F / 0xFF)."""
        c = np.asarray(codes, dtype=np.uint8)
        return np.array([self.lib.oracle_e4m3_decode(int(k)) for k in c.ravel()],
                        dtype=np.float64).reshape(c.shape)

    def e4m3_encode(self, values) -> np.ndarray:
        """float32 -> nearest e4m3fn code (ties to even, saturating to +-448)."""
        v = np.ascontiguousarray(values, dtype=np.float32)
        out = np.empty(v.shape, dtype=np.uint8)
        self.lib.oracle_e4m3_encode_array(_ptr(v), _ptr(out), v.size)
        return out

    # ---------------------------------------------------------- operation ---
    def sum_bf16(self, inputs, rows: int, cols: int) -> np.ndarray:
        """bf16 sum of the R inputs: fp32 accumulation in rank order, one
        rounding."""
        if not 1 <= len(inputs) <= 64:
            raise ValueError("need 1..64 inputs")
        arrs, table = self._table(inputs, rows, cols)
        out = np.empty((rows, cols), dtype=np.uint16)
        self.lib.oracle_sum(table, len(arrs), rows, cols, _ptr(out))
        return out

    def sum_rmsnorm_fp8(self, inputs, rows: int, cols: int, gamma, eps: float,
                        weight_offset: float, scale_ub: float, residual=None,
                        row_start: int = 0, row_count: int | None = None,
                        detail: bool = False) -> dict:
        """The fused operation on rows [row_start, row_start + row_count).

        Returns ``q`` (uint8 [n, cols]), ``scales`` (float32 [n]) and, with a
        residual, ``res_out`` (uint16 [n, cols]).  ``detail=True`` adds ``h``
        (the bf16 norm input) and ``v`` (float32 y / scale).
        """
        if row_count is None:
            row_count = rows - row_start
        if not (0 <= row_start and row_start + row_count <= rows):
            raise ValueError("row range out of bounds")
        arrs, table = self._table(inputs, rows, cols)
        g = np.ascontiguousarray(gamma, dtype=np.uint16).reshape(cols)
        # full-size buffers, of which only the requested rows are written
        q = np.zeros((rows, cols), dtype=np.uint8)
        scales = np.zeros(rows, dtype=np.float32)
        res_in = res_out = None
        if residual is not None:
            res_in = _bf16_rows(residual, rows, cols)
            res_out = np.zeros((rows, cols), dtype=np.uint16)
        h = np.zeros((rows, cols), dtype=np.uint16) if detail else None
        v = np.zeros((rows, cols), dtype=np.float32) if detail else None
        self.lib.oracle_sum_rmsnorm_fp8_rows(
            table, len(arrs), row_start, row_count, cols, _ptr(res_in), _ptr(res_out),
            _ptr(g), eps, weight_offset, scale_ub, _ptr(q), _ptr(scales), _ptr(h),
            _ptr(v))
        sl = slice(row_start, row_start + row_count)
        out = {"q": q[sl].copy(), "scales": scales[sl].copy()}
        if res_out is not None:
            out["res_out"] = res_out[sl].copy()
        if detail:
            out["h"] = h[sl].copy()
            out["v"] = v[sl].copy()
        return out


    def cores(self) -> int:
        """Cores this process may run on (its CPU affinity)."""
        return int(self.lib.oracle_cores())

    def sum_rmsnorm_fp8_mt(self, inputs, rows: int, cols: int, gamma, eps: float,
                           weight_offset: float, scale_ub: float, residual=None,
                           threads: int = 0) -> dict:
        """sum_rmsnorm_fp8 over all rows, the rows split into contiguous
        chunks over ``threads`` POSIX threads (0: one per core).  Returns the
        outputs of sum_rmsnorm_fp8 and ``threads``, the number used."""
        arrs, table = self._table(inputs, rows, cols)
        g = np.ascontiguousarray(gamma, dtype=np.uint16).reshape(cols)
        q = np.zeros((rows, cols), dtype=np.uint8)
        scales = np.zeros(rows, dtype=np.float32)
        res_in = res_out = None
        if residual is not None:
            res_in = _bf16_rows(residual, rows, cols)
            res_out = np.zeros((rows, cols), dtype=np.uint16)
        used = self.lib.oracle_sum_rmsnorm_fp8_mt(
            table, len(arrs), rows, cols, _ptr(res_in), _ptr(res_out), _ptr(g), eps,
            weight_offset, scale_ub, _ptr(q), _ptr(scales), threads)
        if used < 0:
            raise RuntimeError("a worker thread could not be started")
        out = {"q": q, "scales": scales, "threads": int(used)}
        if res_out is not None:
            out["res_out"] = res_out
        return out

    def mx_scale_code(self, amax: float) -> int:
        """E8M0 code of a block's shared scale from its max |V| (OCP MX)."""
        return int(self.lib.oracle_mx_scale_code(float(amax)))

    def sum_rmsnorm_mxfp8(self, inputs, rows: int, cols: int, gamma, eps: float,
                          weight_offset: float, residual=None, row_start: int = 0,
                          row_count: int | None = None, detail: bool = False) -> dict:
        """The norm with MX output on rows [row_start, row_start + row_count):
        ``q`` (uint8 [n, cols]), ``scales_mx`` (uint8 E8M0 codes
        [n, cols / 32]), ``res_out`` with a residual; ``detail`` adds ``h``
        and ``v`` (float32 y * 2^(127 - code))."""
        if cols % 32:
            raise ValueError("cols must be a multiple of 32")
        if row_count is None:
            row_count = rows - row_start
        if not (0 <= row_start and row_start + row_count <= rows):
            raise ValueError("row range out of bounds")
        arrs, table = self._table(inputs, rows, cols)
        g = np.ascontiguousarray(gamma, dtype=np.uint16).reshape(cols)
        q = np.zeros((rows, cols), dtype=np.uint8)
        sc = np.zeros((rows, cols // 32), dtype=np.uint8)
        res_in = res_out = None
        if residual is not None:
            res_in = _bf16_rows(residual, rows, cols)
            res_out = np.zeros((rows, cols), dtype=np.uint16)
        h = np.zeros((rows, cols), dtype=np.uint16)
        v = np.zeros((rows, cols), dtype=np.float32) if detail else None
        self.lib.oracle_sum_rmsnorm_mxfp8_rows(
            table, len(arrs), row_start, row_count, cols, _ptr(res_in), _ptr(res_out), _ptr(g),
            eps, weight_offset, _ptr(q), _ptr(sc), _ptr(h), _ptr(v))
        sl = slice(row_start, row_start + row_count)
        out = {"q": q[sl].copy(), "scales_mx": sc[sl].copy()}
        if res_out is not None:
            out["res_out"] = res_out[sl].copy()
        if detail:
            out["h"] = h[sl].copy()
            out["v"] = v[sl].copy()
        return out

    def e8m0_decode(self, codes) -> np.ndarray:
        """E8M0 codes -> float64 values (NaN for 0xFF)."""
        c = np.asarray(codes, dtype=np.uint8)
        return np.array([self.lib.oracle_e8m0_decode(int(k)) for k in c.ravel()],
                        dtype=np.float64).reshape(c.shape)

    def scaled_mm_mx(self, a, sa, b, sb, bias=None, exact: bool = False):
        """The MX GEMM: a uint8 e4m3fn codes [M, K], b [N, K], sa / sb E8M0
        codes [M, K / 32] / [N, K / 32], bias bf16 bits [N] or None.  Returns
        out (bf16 bits [M, N]) and, with ``exact``, the float64 values."""
        a = np.ascontiguousarray(a, dtype=np.uint8)
        b = np.ascontiguousarray(b, dtype=np.uint8)
        M, K = a.shape
        N = b.shape[0]
        if b.shape[1] != K or K % 32:
            raise ValueError("a and b need the same K, a multiple of 32")
        sa = np.ascontiguousarray(sa, dtype=np.uint8).reshape(M, K // 32)
        sb = np.ascontiguousarray(sb, dtype=np.uint8).reshape(N, K // 32)
        bi = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16).reshape(N)
        out = np.empty((M, N), dtype=np.uint16)
        ex = np.empty((M, N), dtype=np.float64) if exact else None
        self.lib.oracle_scaled_mm_mx(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(bi), M, N, K,
                                     _ptr(out), _ptr(ex))
        return (out, ex) if exact else out

    def bf16_round_double(self, values) -> np.ndarray:
        """float64 -> nearest bf16 (ties to even) in one rounding, as uint16."""
        v = np.asarray(values, dtype=np.float64)
        return np.array([self.lib.oracle_bf16_round_double(float(x)) for x in v.ravel()],
                        dtype=np.uint16).reshape(v.shape)

    def scaled_mm(self, a, a_scale, b, b_scale, bias=None, exact: bool = False):
        """The FP8 GEMM: a uint8 e4m3fn codes [M, K], b [N, K], scales float32
        [M] and [N], bias bf16 bits [N] or None.  Returns out (bf16 bits
        [M, N]) and, with ``exact``, also the float64 values before the
        rounding."""
        a = np.ascontiguousarray(a, dtype=np.uint8)
        b = np.ascontiguousarray(b, dtype=np.uint8)
        M, K = a.shape
        N = b.shape[0]
        if b.shape[1] != K:
            raise ValueError("a and b need the same K")
        sa = np.ascontiguousarray(a_scale, dtype=np.float32).reshape(M)
        sb = np.ascontiguousarray(b_scale, dtype=np.float32).reshape(N)
        bi = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16).reshape(N)
        out = np.empty((M, N), dtype=np.uint16)
        ex = np.empty((M, N), dtype=np.float64) if exact else None
        self.lib.oracle_scaled_mm(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(bi), M, N, K,
                                  _ptr(out), _ptr(ex))
        return (out, ex) if exact else out


def default() -> Oracle:
    """The oracle built from ``rrf_oracle.c`` (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def bf16_round(values):
    return default().bf16_round(values)


def e4m3_decode(codes):
    return default().e4m3_decode(codes)


def e4m3_encode(values):
    return default().e4m3_encode(values)


def sum_bf16(inputs, rows, cols):
    return default().sum_bf16(inputs, rows, cols)


def sum_rmsnorm_fp8(*args, **kwargs):
    return default().sum_rmsnorm_fp8(*args, **kwargs)


def bf16_round_double(values):
    return default().bf16_round_double(values)


def scaled_mm(*args, **kwargs):
    return default().scaled_mm(*args, **kwargs)


def sum_rmsnorm_mxfp8(*args, **kwargs):
    return default().sum_rmsnorm_mxfp8(*args, **kwargs)


def scaled_mm_mx(*args, **kwargs):
    return default().scaled_mm_mx(*args, **kwargs)
