"""Seeded synthetic inputs for the fused bf16 sum + RMSNorm + FP8 operation.

This module only draws inputs.  It holds none of the operation's arithmetic:
both the CUDA library and the CPU oracle consume what it produces, and neither
is imported here.

Generator: splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-style -- output k of stream
``seed`` mixes ``seed + (k + 1) * 0x9E3779B97F4A7C15`` -- turned into uniforms
in (0, 1] from the top 53 bits and into normals by the Box-Muller transform,
all in float64 with torch operations (on the host or on the GPU), then
narrowed to float32 and to bf16 (torch's conversions).

Seeds: ``1000 * config + 100 * sub + tensor``; ``tensor`` is 0..R-1 for the
inputs, R for the residual and R + 1 for gamma; the outlier mask of input r
uses stream ``seed(r) + 50``.  ``config`` numbers the workloads below, ``sub``
indexes their row counts.

Workloads (each names the shapes and distributions it is drawn from; "N(m, s)"
means mean m and standard deviation s):
  tiny     R=2, 4 x 256, inputs N(0,1), no residual, gamma N(1,0.1),
           eps 1e-6, weight_offset 0, scale_ub 1200.
  decode   R=8, rows {1, 8, 32, 64} x 7168, inputs N(0,0.5), residual N(0,1),
           gamma N(1,0.1), eps 1e-5, weight_offset 0, scale_ub 1200.  The
           shapes of the TensorRT-LLM MNNVL one-shot / two-shot tests (hidden
           7168, 1 to 64 tokens).
  odd      R=4, rows {37, 64} x 7168, inputs N(0,1) with 1% of elements
           multiplied by 50 (a Bernoulli(0.01) mask per input), residual
           N(0,1), gamma N(0,0.1) with weight_offset 1.0 (unit-offset gamma),
           eps 1e-6, scale_ub 8.0 so outlier rows hit the clamp.
  prefill  R=8, 8192 x 8192, inputs N(0,1), residual N(0,1), gamma N(1,0.1),
           eps 1e-5, weight_offset 0, scale_ub 1200 (about 1.3 GiB per call).
  sweep    R=4, 4096 columns, rows {16, 32, 48, 64, 96, 128, 256} (128 KiB to
           2 MiB per input, the payload sizes of the b12x PCIe two-shot
           timing table), inputs N(0,1); the fused form uses no residual,
           gamma N(1,0.1), eps 1e-6, weight_offset 0, scale_ub 1200.
"""
from __future__ import annotations

import dataclasses

import numpy as np

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _i64(u: int) -> int:
    """The int64 with the same 64 bits as the unsigned value u."""
    u &= 0xFFFFFFFFFFFFFFFF
    return u - (1 << 64) if u >= (1 << 63) else u


def _srl(z, s: int):
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(seed: int, n: int, device="cpu"):
    """Outputs 0 .. n-1 of the splitmix64 stream ``seed`` as int64 bit patterns
    (torch wraps int64 arithmetic modulo 2^64, which is what the generator
    needs)."""
    import torch
    k = torch.arange(1, n + 1, dtype=torch.int64, device=device)
    z = k * _i64(_GOLDEN) + _i64(seed)
    z = (z ^ _srl(z, 30)) * _i64(_M1)
    z = (z ^ _srl(z, 27)) * _i64(_M2)
    return z ^ _srl(z, 31)


def uniform(seed: int, n: int, device="cpu"):
    """n uniforms in (0, 1], float64 (top 53 bits of each output, plus one)."""
    z = splitmix64(seed, n, device)
    return (_srl(z, 11).double() + 1.0) * (1.0 / 9007199254740992.0)


def normal(seed: int, n: int, mean: float = 0.0, std: float = 1.0, device="cpu"):
    """n normals N(mean, std) by Box-Muller, float64.  The bit stream is the
    same on every device; the float64 log / sqrt / cos / sin may differ in the
    last place between the host's and the GPU's libraries."""
    import torch
    m = (n + 1) // 2
    u = uniform(seed, 2 * m, device)
    rad = torch.sqrt(-2.0 * torch.log(u[0::2]))
    ang = (2.0 * torch.pi) * u[1::2]
    out = torch.stack((rad * torch.cos(ang), rad * torch.sin(ang)), dim=1).reshape(-1)
    return out[:n] * std + mean


def to_bf16(x):
    """float64 -> float32 -> bf16 (torch's conversions)."""
    import torch
    return x.to(torch.float32).to(torch.bfloat16)


def bits(t) -> np.ndarray:
    """A bf16 torch tensor (any device) as a host numpy array of uint16 bit
    patterns, the form the oracle takes."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    config: int
    R: int
    rows: tuple
    cols: int
    input_std: float
    residual: bool
    gamma_mean: float
    gamma_std: float
    eps: float
    weight_offset: float
    scale_ub: float
    outlier_p: float = 0.0
    outlier_mult: float = 1.0


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, (4,), 256, 1.0, False, 1.0, 0.1, 1e-6, 0.0, 1200.0),
    "decode": Workload("decode", 2, 8, (1, 8, 32, 64), 7168, 0.5, True, 1.0, 0.1,
                       1e-5, 0.0, 1200.0),
    "odd": Workload("odd", 3, 4, (37, 64), 7168, 1.0, True, 0.0, 0.1, 1e-6, 1.0, 8.0,
                    outlier_p=0.01, outlier_mult=50.0),
    "prefill": Workload("prefill", 4, 8, (8192,), 8192, 1.0, True, 1.0, 0.1, 1e-5,
                        0.0, 1200.0),
    "sweep": Workload("sweep", 5, 4, (16, 32, 48, 64, 96, 128, 256), 4096, 1.0, False,
                      1.0, 0.1, 1e-6, 0.0, 1200.0),
}


@dataclasses.dataclass
class Case:
    """One seeded problem: bf16 torch tensors [rows, cols] (gamma [cols])."""
    name: str
    R: int
    rows: int
    cols: int
    inputs: list
    residual: object
    gamma: object
    eps: float
    weight_offset: float
    scale_ub: float


def seed_of(config: int, sub: int, tensor: int) -> int:
    return 1000 * config + 100 * sub + tensor


def draw_input(seed: int, rows: int, cols: int, std: float, outlier_p: float = 0.0,
               outlier_mult: float = 1.0, device="cpu"):
    """One bf16 input [rows, cols] drawn from stream ``seed``."""
    import torch
    x = normal(seed, rows * cols, 0.0, std, device)
    if outlier_p > 0.0:
        mask = uniform(seed + 50, rows * cols, device) < outlier_p
        x = torch.where(mask, x * outlier_mult, x)
    return to_bf16(x).reshape(rows, cols)


def make_case(name: str, rows: int | None = None, *, sub: int | None = None,
              residual: bool | None = None, R: int | None = None,
              cols: int | None = None, device="cpu") -> Case:
    """Draw the seeded problem ``name`` at one of its row counts, as bf16 torch
    tensors on ``device``.

    ``rows`` defaults to the workload's first row count; ``sub`` (the seed's
    row index) defaults to that row count's position in the workload's list,
    else 9.  ``residual``, ``R`` and ``cols`` override the workload's own
    values (for edge cases); the seeds stay the workload's.
    """
    w = WORKLOADS[name]
    if rows is None:
        rows = w.rows[0]
    if sub is None:
        sub = w.rows.index(rows) if rows in w.rows else 9
    R = w.R if R is None else R
    cols = w.cols if cols is None else cols
    use_res = w.residual if residual is None else residual
    inputs = [draw_input(seed_of(w.config, sub, r), rows, cols, w.input_std,
                         w.outlier_p, w.outlier_mult, device) for r in range(R)]
    res = None
    if use_res:
        res = to_bf16(normal(seed_of(w.config, sub, R), rows * cols, 0.0, 1.0,
                             device)).reshape(rows, cols)
    gamma = to_bf16(normal(seed_of(w.config, sub, R + 1), cols, w.gamma_mean,
                           w.gamma_std, device))
    return Case(name, R, rows, cols, inputs, res, gamma, w.eps, w.weight_offset,
                w.scale_ub)


def fused_bytes(R: int, rows: int, cols: int, residual: bool) -> int:
    """Algorithmic HBM bytes of one fused call: each input read once, the
    residual read and written, gamma read once, fp8 codes and fp32 scales
    written."""
    return R * rows * cols * 2 + (4 * rows * cols if residual else 0) + cols * 2 \
        + rows * cols + 4 * rows


def sum_bytes(R: int, rows: int, cols: int) -> int:
    """Algorithmic HBM bytes of one sum-only call: R reads and one write."""
    return (R + 1) * rows * cols * 2


# ------------------------------------------------------------ FP8 GEMM ---
# Operands of the GEMM that consumes the per-row scales.  The activation
# codes and scales normally come from the fused call; these stand-alone
# operands are codes of N(0, 1) samples (torch's saturating float8_e4m3fn
# conversion: input preparation, not the GEMM's arithmetic), per-row scales
# U(0.001, 0.01), weight codes of N(0, 1), per-column scales U(0.0005, 0.002)
# (a weight of magnitude ~1e-3 quantised per output column) and a bf16 bias
# N(0, 0.1).  Seeds: 9000 + 10 * sub + tensor.

GEMM_SHAPES = {
    # decode: the decode batch sizes against a 7168 x 7168 projection
    "gemm_decode": dict(Ms=(1, 8, 32, 64), N=7168, K=7168),
    # prefill: 8192 rows of the 8192-wide prefill hidden state, 8192 outputs
    "gemm_prefill": dict(Ms=(8192,), N=8192, K=8192),
}


@dataclasses.dataclass
class GemmCase:
    M: int
    N: int
    K: int
    a: "torch.Tensor"        # float8_e4m3fn [M, K]
    a_scale: "torch.Tensor"  # float32 [M]
    b: "torch.Tensor"        # float8_e4m3fn [N, K]
    b_scale: "torch.Tensor"  # float32 [N]
    bias: "torch.Tensor | None"  # bf16 [N]


def _e4m3_codes(seed: int, n: int, device):
    import torch
    x = normal(seed, n, 0.0, 1.0, device).float()
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)


def make_gemm_case(M: int, N: int, K: int, sub: int = 0, bias: bool = True,
                   device="cpu") -> GemmCase:
    s = lambda t: 9000 + 10 * sub + t
    a = _e4m3_codes(s(0), M * K, device).reshape(M, K)
    b = _e4m3_codes(s(1), N * K, device).reshape(N, K)
    sa = (0.001 + 0.009 * uniform(s(2), M, device)).float()
    sb = (0.0005 + 0.0015 * uniform(s(3), N, device)).float()
    bi = to_bf16(normal(s(4), N, 0.0, 0.1, device)) if bias else None
    return GemmCase(M, N, K, a, sa, b, sb, bi)


def gemm_bytes(M: int, N: int, K: int, bias: bool = True) -> int:
    """Algorithmic HBM bytes of one GEMM call: each operand read once, the
    bf16 output written once."""
    return M * K + N * K + 4 * M + 4 * N + (2 * N if bias else 0) + 2 * M * N


def gemm_flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K
