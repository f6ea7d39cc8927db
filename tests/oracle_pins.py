"""Pins for the oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises ``AssertionError`` when
the oracle disagrees with what the pages, the number formats or mathematics
fix.  The sources, never the oracle's own code:

* library routines that implement a step on their own: torch's float32 ->
  bf16 conversion and float32 -> float8_e4m3fn conversion, ml_dtypes'
  float8_e4m3fn decoding;
* the e4m3fn landmarks of the OCP 8-bit floating point specification and the
  b12x two-shot precision figure (fixtures under ``golden/``);
* error bounds (one bf16 rounding of the exact sum plus the fp32 recursive
  summation bound), float64 brute force, closed forms worked out by hand,
  invariants, determinism and row independence.

``test_oracle_pins.py`` runs every pin on the oracle; ``test_oracle_mutants.py``
runs them on copies of the oracle with one plausible mistake planted each,
and requires each copy to fail at least one pin.
"""
from __future__ import annotations

import math
import os

import ml_dtypes
import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
U32 = 2.0 ** -24  # unit roundoff of fp32


# ------------------------------------------------------------ library side ---

def lib_bf16(values) -> np.ndarray:
    """float32 -> bf16 bits by torch's conversion (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32(bits) -> np.ndarray:
    """bf16 bits -> float32 (bf16 is the upper half of a binary32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def lib_e4m3_torch(values) -> np.ndarray:
    """float32 -> e4m3fn codes by torch, after clamping to +-448 (saturation)."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def lib_e4m3_mld(values) -> np.ndarray:
    """float32 -> e4m3fn codes by ml_dtypes, after clamping to +-448."""
    v = np.clip(np.asarray(values, dtype=np.float32), -448.0, 448.0)
    return v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def lib_e4m3_decode(codes) -> np.ndarray:
    return np.asarray(codes, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def bf16_ulp(x) -> np.ndarray:
    """Spacing of bf16 numbers at magnitude |x| (normal range)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def e4m3_ulp(x) -> np.ndarray:
    """Spacing of e4m3fn numbers at magnitude |x| (subnormal spacing 2^-9)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -6)
    return np.exp2(np.floor(np.log2(a)) - 3)


def e4m3_midpoint_distance(v) -> np.ndarray:
    """Relative distance of |v| to the nearest midpoint between two adjacent
    finite e4m3fn magnitudes."""
    mags = np.unique(lib_e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (mags[:-1] + mags[1:]) / 2.0
    a = np.abs(np.asarray(v, dtype=np.float64)).reshape(-1)
    idx = np.clip(np.searchsorted(mids, a), 1, len(mids) - 1)
    d = np.minimum(np.abs(a - mids[idx - 1]), np.abs(a - mids[idx]))
    return (d / np.maximum(a, 2.0 ** -10)).reshape(np.shape(v))


def rand_bf16(seed: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return lib_bf16(rng.normal(mean, std, size=shape).astype(np.float32))


def bf16_of(values) -> np.ndarray:
    """bf16 bits of values that are exactly representable (checked)."""
    v = np.asarray(values, dtype=np.float32)
    b = lib_bf16(v)
    assert np.array_equal(f32(b), v), "value not exact in bf16"
    return b


def read_golden(name: str):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ codec ---

def pin_e4m3_decode_table(o):
    """All 256 codes decode as ml_dtypes and the OCP landmarks say."""
    codes = np.arange(256, dtype=np.uint8)
    mine = o.e4m3_decode(codes)
    ref = lib_e4m3_decode(codes)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(mine[fin], ref[fin])
    assert np.array_equal(np.signbit(mine[fin]), np.signbit(ref[fin]))
    for code, value, *_ in read_golden("e4m3fn_landmarks.txt"):
        got = o.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0]
        if value == "nan":
            assert math.isnan(got), code
        else:
            assert got == float(value) and math.copysign(1, got) == math.copysign(1, float(value)), code


def pin_e4m3_encode_roundtrip(o):
    """Every finite code encodes back to itself, -0 included."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = lib_e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(o.e4m3_encode(vals), codes)


def pin_e4m3_encode_ties_and_saturation(o):
    """Midpoints go to the even code, points beside them to the nearer code,
    magnitudes above 448 (and infinities) saturate to +-448."""
    mags = lib_e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))  # 0 .. 448
    lo, hi = mags[:-1], mags[1:]
    mid = ((lo + hi) / 2.0).astype(np.float32)  # exact in fp32
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2.0)
    codes_lo = np.arange(0, 0x7E, dtype=np.uint8)
    even = np.where(codes_lo % 2 == 0, codes_lo, codes_lo + 1).astype(np.uint8)
    assert np.array_equal(o.e4m3_encode(mid), even)
    assert np.array_equal(o.e4m3_encode(-mid), even | 0x80)
    below = np.nextafter(mid, np.float32(0))
    above = np.nextafter(mid, np.float32(np.inf))
    assert np.array_equal(o.e4m3_encode(below), codes_lo)
    assert np.array_equal(o.e4m3_encode(above), codes_lo + 1)
    big = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3e38, np.inf], dtype=np.float32)
    assert np.all(o.e4m3_encode(big) == 0x7E)
    assert np.all(o.e4m3_encode(-big) == 0xFE)
    assert o.e4m3_encode(np.array([np.nan], dtype=np.float32))[0] & 0x7F == 0x7F


def pin_e4m3_encode_vs_libraries(o):
    """Random fp32 over the whole e4m3 range and beyond, tiny values included:
    the oracle's codes equal torch's and ml_dtypes' (after saturation)."""
    rng = np.random.default_rng(7)
    n = 200_000
    mant = rng.uniform(1.0, 2.0, n)
    expo = rng.integers(-14, 11, n)
    sign = rng.choice([-1.0, 1.0], n)
    v = (sign * mant * np.exp2(expo)).astype(np.float32)
    mine = o.e4m3_encode(v)
    assert np.array_equal(mine, lib_e4m3_torch(v))
    assert np.array_equal(mine, lib_e4m3_mld(v))


# ------------------------------------------------------------------- bf16 ---

def pin_bf16_round_vs_torch(o):
    """fp32 -> bf16 equals torch's round-to-nearest-even on random bit
    patterns, exact ties, the overflow edge, subnormals, zeros, infinities."""
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2 ** 32, 300_000, dtype=np.uint64).astype(np.uint32)
    v = u.view(np.float32)
    v = v[np.isfinite(v)]
    ties = (rng.integers(0, 2 ** 16, 20_000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    edge = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 3.4e38,
                     np.finfo(np.float32).max, 1e-40, -1e-45, 1.0039062, 1.0039063],
                    dtype=np.float32)
    for arr in (v, ties, edge):
        assert np.array_equal(o.bf16_round(arr), lib_bf16(arr))


# -------------------------------------------------------------------- sum ---

def pin_sum_identity(o):
    """R = 1: the sum is the input itself, bit for bit (-0 and subnormals too)."""
    x = rand_bf16(1, (5, 24))
    x[0, :4] = np.array([0x8000, 0x0000, 0x0001, 0x807F], dtype=np.uint16)
    assert np.array_equal(o.sum_bf16([x], 5, 24), x)


def pin_sum_two_exact(o):
    """R = 2 with nearby exponents: fp32 holds a + b exactly, so the result is
    the correctly rounded bf16 of the exact sum (torch's conversion of the
    float64 sum)."""
    rng = np.random.default_rng(2)
    a, b = (lib_bf16((rng.choice([-1.0, 1.0], (8, 128)) * rng.uniform(0.5, 4.0, (8, 128)))
                     .astype(np.float32)) for _ in range(2))
    exact = f32(a).astype(np.float64) + f32(b).astype(np.float64)
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)
    assert np.array_equal(o.sum_bf16([a, b], 8, 128), lib_bf16(exact.astype(np.float32)))


def pin_sum_bound(o):
    """Within one bf16 rounding of the exact sum, plus the fp32 recursive
    summation bound (R-1) u sum|x|, for R = 2..16."""
    for R in (2, 3, 5, 8, 16):
        xs = [rand_bf16(100 + R * 17 + r, (4, 96), std=1.0 + r) for r in range(R)]
        s = f32(o.sum_bf16(xs, 4, 96)).astype(np.float64)
        vals = np.stack([f32(x).astype(np.float64) for x in xs])
        exact = vals.sum(axis=0)
        gamma = (R - 1) * U32 / (1 - (R - 1) * U32)
        bound = 0.5 * bf16_ulp(np.maximum(np.abs(s), np.abs(exact))) \
            + gamma * np.abs(vals).sum(axis=0)
        assert np.all(np.abs(s - exact) <= bound), R


def pin_sum_fixed_order_fp32(o):
    """The accumulator is fp32 and runs in rank order 0..R-1: a unit placed
    before +-2^30 is absorbed (result +0), placed after it survives (1)."""
    one, big = bf16_of([1.0]), bf16_of([2.0 ** 30])
    neg = bf16_of([-(2.0 ** 30)])
    col = lambda b: b.reshape(1, 1)
    first = o.sum_bf16([col(one), col(big), col(neg)], 1, 1)
    last = o.sum_bf16([col(big), col(neg), col(one)], 1, 1)
    assert first[0, 0] == 0x0000 and last[0, 0] == bf16_of([1.0])[0]


def pin_sum_signed_zero(o):
    """All -0 inputs give -0 (the accumulator starts from the first input);
    -0 + +0 gives +0 (IEEE round to nearest)."""
    nz = np.full((1, 8), 0x8000, dtype=np.uint16)
    pz = np.zeros((1, 8), dtype=np.uint16)
    assert np.all(o.sum_bf16([nz, nz, nz], 1, 8) == 0x8000)
    assert np.all(o.sum_bf16([nz, pz], 1, 8) == 0x0000)


def pin_sum_twoshot_precision(o):
    """b12x PR #283, Validation: at row magnitude ~16 the error against the
    exact sum is at most 0.0625, one bf16 half-ulp (fixture).  Inputs are bf16
    values in [2, 8), so fp32 adds them exactly and the one bf16 rounding is
    the only error; the bound must be reached, not only respected."""
    (lo, hi, err), = [tuple(map(float, r)) for r in read_golden("twoshot_bf16_precision.txt")]
    assert 0.5 * bf16_ulp(lo) == err
    rng = np.random.default_rng(5)
    xs = [lib_bf16(rng.uniform(2.0, 8.0, (64, 256)).astype(np.float32)) for _ in range(4)]
    s = f32(o.sum_bf16(xs, 64, 256)).astype(np.float64)
    exact = sum(f32(x).astype(np.float64) for x in xs)
    band = (np.abs(exact) >= lo) & (np.abs(exact) < hi)
    assert band.sum() > 1000
    e = np.abs(s - exact)[band]
    assert e.max() <= err and e.max() == err


# ------------------------------------------------------------- residual ---

def pin_residual(o):
    """res_out = RN_bf16(f32(s) + f32(res)) with s the rounded sum: checked by
    torch's rounding of the exact (fp32-exact) sum; res = -s gives +0; the
    in-place form gives the same bits."""
    R, rows, cols = 3, 4, 64
    xs = [rand_bf16(20 + r, (rows, cols)) for r in range(R)]
    res = rand_bf16(30, (rows, cols))
    g = rand_bf16(31, (cols,), 0.1, 1.0)
    out = o.sum_rmsnorm_fp8(xs, rows, cols, g, 1e-5, 0.0, 1200.0, residual=res)
    s = o.sum_bf16(xs, rows, cols)
    exact = f32(s).astype(np.float64) + f32(res).astype(np.float64)
    assert np.array_equal(out["res_out"], lib_bf16(exact.astype(np.float32)))
    neg = (s ^ np.uint16(0x8000)).astype(np.uint16)
    out2 = o.sum_rmsnorm_fp8(xs, rows, cols, g, 1e-5, 0.0, 1200.0, residual=neg)
    assert np.all(out2["res_out"] == 0x0000)


def pin_residual_after_rounding(o):
    """The residual is added to the bf16-rounded sum, not to the fp32
    accumulator: inputs 1, 2^-8, 2^-16 sum to 1 + 2^-8 + 2^-16, which rounds to
    1 + 2^-7; with residual -1 the norm input is 2^-7 (adding -1 before the
    rounding would give the tie 2^-8 + 2^-16 -> 2^-8)."""
    xs = [bf16_of([[v]]) for v in (1.0, 2.0 ** -8, 2.0 ** -16)]
    res = bf16_of([[-1.0]])
    assert o.sum_bf16(xs, 1, 1)[0, 0] == bf16_of([1.0 + 2.0 ** -7])[0]
    out = o.sum_rmsnorm_fp8(xs, 1, 1, bf16_of([1.0]), 1e-6, 0.0, 1200.0, residual=res)
    assert out["res_out"][0, 0] == bf16_of([2.0 ** -7])[0]


# ------------------------------------------------------------------- norm ---

def _independent_h(o, xs, rows, cols, res):
    s = o.sum_bf16(xs, rows, cols)
    if res is None:
        return s
    return lib_bf16((f32(s).astype(np.float64) + f32(res).astype(np.float64)).astype(np.float32))


def pin_norm_brute_force(o):
    """float64 RMSNorm + amax scale from the same bf16 norm input agrees with
    the oracle: scales within 6e-7 relative, y = v * scale within 8e-7, codes
    equal to the library encoding of the float64 y / scale except next to a
    rounding midpoint."""
    cases = [  # R, rows, cols, residual, eps, wo, ub, gamma mean
        (3, 3, 64, True, 1e-5, 0.5, 1200.0, 1.0),
        (1, 2, 40, False, 1e-6, 0.0, 1200.0, 1.0),
        (4, 4, 8, True, 1e-6, 1.0, 0.5, 0.0),      # clamped rows
        (2, 3, 200, False, 0.25, 0.0, 1200.0, -0.5),
    ]
    for k, (R, rows, cols, use_res, eps, wo, ub, gm) in enumerate(cases):
        xs = [rand_bf16(200 + 10 * k + r, (rows, cols), std=2.0) for r in range(R)]
        res = rand_bf16(250 + k, (rows, cols)) if use_res else None
        g = rand_bf16(260 + k, (cols,), 0.3, gm)
        out = o.sum_rmsnorm_fp8(xs, rows, cols, g, eps, wo, ub, residual=res, detail=True)
        h = f32(_independent_h(o, xs, rows, cols, res)).astype(np.float64)
        gp = f32(g).astype(np.float64) + wo
        eps32 = float(np.float32(eps))
        r64 = 1.0 / np.sqrt((h * h).mean(axis=1, keepdims=True) + eps32)
        y64 = h * r64 * gp
        amax = np.abs(y64).max(axis=1)
        sc64 = np.maximum(np.minimum(amax, float(np.float32(ub))), float(np.float32(1e-12))) / 448.0
        assert np.all(np.abs(out["scales"] - sc64) <= 6e-7 * sc64), k
        y_or = out["v"].astype(np.float64) * out["scales"][:, None].astype(np.float64)
        assert np.all(np.abs(y_or - y64) <= 8e-7 * np.abs(y64) + 1e-30), k
        v64 = y64 / sc64[:, None]
        want = lib_e4m3_torch(v64.astype(np.float32))
        diff = out["q"] != want
        if diff.any():
            near = e4m3_midpoint_distance(v64) < 2e-6
            assert np.all(near[diff]), k
            step = np.abs(out["q"][diff].astype(int) - want[diff].astype(int))
            assert np.all(step == 1), k


def pin_norm_constant_row(o):
    """A constant row c gives y_j = c / sqrt(c^2 + eps) * (g_j + wo)."""
    cols = 48
    xs = [np.full((1, cols), bf16_of([1.5])[0], dtype=np.uint16)] * 2  # c = 3
    g = rand_bf16(40, (cols,), 0.2, 1.0)
    for eps, wo in ((1e-6, 0.0), (2.0, 0.25)):
        out = o.sum_rmsnorm_fp8(xs, 1, cols, g, eps, wo, 1200.0, detail=True)
        y = 3.0 / math.sqrt(9.0 + float(np.float32(eps))) * (f32(g).astype(np.float64) + wo)
        got = out["v"][0].astype(np.float64) * float(out["scales"][0])
        assert np.all(np.abs(got - y) <= 6e-7 * np.abs(y)), eps
        assert abs(float(out["scales"][0]) - np.abs(y).max() / 448.0) <= 5e-7 * np.abs(y).max() / 448.0


def pin_norm_one_hot(o):
    """A one-hot row a at j0: y_j0 = a (g + wo) / sqrt(a^2 / cols + eps), which
    encodes to +-448; every other y is a zero carrying the sign of g + wo."""
    cols, j0, a, eps, wo = 16, 3, 5.0, 1e-3, 0.0
    x = np.zeros((1, cols), dtype=np.uint16)
    x[0, j0] = bf16_of([a])[0]
    g = rand_bf16(41, (cols,), 1.0, 0.0)
    out = o.sum_rmsnorm_fp8([x], 1, cols, g, eps, wo, 1200.0, detail=True)
    gp = f32(g).astype(np.float64) + wo
    y0 = a * gp[j0] / math.sqrt(a * a / cols + float(np.float32(eps)))
    assert abs(float(out["scales"][0]) - abs(y0) / 448.0) <= 5e-7 * abs(y0) / 448.0
    assert out["q"][0, j0] == (0xFE if gp[j0] < 0 else 0x7E)
    others = np.arange(cols) != j0
    assert np.array_equal(out["q"][0, others], np.where(gp[others] < 0, 0x80, 0x00))


def pin_norm_zero_row(o):
    """An all-zero row: amax = 0, the scale is the floor 1e-12 / 448 (fp32),
    and every code is a zero carrying the sign of g + wo."""
    cols = 32
    z = np.zeros((2, cols), dtype=np.uint16)
    g = rand_bf16(42, (cols,), 1.0, 0.0)
    out = o.sum_rmsnorm_fp8([z, z], 2, cols, g, 1e-6, 0.0, 1200.0)
    assert np.all(out["scales"] == np.float32(1e-12) / np.float32(448.0))
    want = np.where(f32(g) < 0, 0x80, 0x00)
    assert np.array_equal(out["q"], np.stack([want, want]))


def pin_norm_hand_example(o):
    """Worked by hand: R = 2 inputs of ones, 8 columns, eps = 0, no residual.
    s = 2, mean(s^2) = 4, r = 1/2, y = gamma; amax = 2, scale = fp32(2 / 448);
    y / scale for gamma = 1, 0.5, -1, 2, 0.25, -2, 1.25, 0 is about 224, 112,
    -224, 448, 56, -448, 280, 0, i.e. codes 0x76, 0x6E, 0xF6, 0x7E, 0x66, 0xFE,
    0x79 (280 is nearer 288 than 256), 0x00."""
    ones = np.full((1, 8), bf16_of([1.0])[0], dtype=np.uint16)
    g = bf16_of([1.0, 0.5, -1.0, 2.0, 0.25, -2.0, 1.25, 0.0])
    out = o.sum_rmsnorm_fp8([ones, ones], 1, 8, g, 0.0, 0.0, 1200.0)
    assert out["scales"][0] == np.float32(2.0) / np.float32(448.0)
    assert list(out["q"][0]) == [0x76, 0x6E, 0xF6, 0x7E, 0x66, 0xFE, 0x79, 0x00]


def pin_norm_clamp(o):
    """When amax exceeds scale_ub the scale is fp32(ub / 448) exactly and every
    |y| >= ub * 464 / 448 saturates to +-448."""
    cols, ub = 64, 2.0
    x = rand_bf16(43, (2, cols), 30.0)
    x[:, 5] = bf16_of([4096.0])[0]  # one huge element: amax far above ub
    g = rand_bf16(44, (cols,), 0.1, 1.0)
    out = o.sum_rmsnorm_fp8([x], 2, cols, g, 1e-6, 0.0, ub, detail=True)
    assert np.all(out["scales"] == np.float32(ub) / np.float32(448.0))
    y = out["v"].astype(np.float64) * out["scales"][:, None]
    sat = np.abs(y) >= ub * 464.0 / 448.0
    assert sat.any()
    assert np.all((out["q"][sat] & 0x7F) == 0x7E)


def pin_norm_invariants(o):
    """Seeded rows with outliers: |decode(q)| <= 448; scale <= ub / 448; an
    unclamped row's largest |y| encodes to +-448; every code is the nearest
    e4m3 value to y / scale (within half an e4m3 ulp)."""
    rows, cols, R = 6, 256, 4
    xs = []
    for r in range(R):
        x = f32(rand_bf16(300 + r, (rows, cols))).astype(np.float64)
        x[np.random.default_rng(310 + r).random((rows, cols)) < 0.02] *= 50.0
        xs.append(lib_bf16(x.astype(np.float32)))
    res = rand_bf16(320, (rows, cols))
    g = rand_bf16(321, (cols,), 0.1, 0.0)
    for ub in (8.0, 1200.0):
        out = o.sum_rmsnorm_fp8(xs, rows, cols, g, 1e-6, 1.0, ub, residual=res, detail=True)
        dq = lib_e4m3_decode(out["q"])
        assert np.all(np.abs(dq) <= 448.0)
        assert np.all(out["scales"] <= np.float32(ub) / np.float32(448.0))
        v = out["v"].astype(np.float64)
        amax_v = np.abs(v).max(axis=1)
        unclamped = out["scales"] < np.float32(ub) / np.float32(448.0)
        for i in np.nonzero(unclamped)[0]:
            j = int(np.argmax(np.abs(v[i])))
            assert (out["q"][i, j] & 0x7F) == 0x7E
            assert abs(amax_v[i] - 448.0) <= 448.0 * 4 * U32
        inside = np.abs(v) <= 448.0
        assert np.all(np.abs(dq - v)[inside] <= 0.5 * e4m3_ulp(v)[inside] * (1 + 1e-12))


def pin_norm_mean_square(o):
    """mean((y / (g + wo))^2) = ms / (ms + eps): checked with a large eps so
    that the placement of eps matters."""
    rows, cols = 3, 128
    xs = [rand_bf16(50 + r, (rows, cols)) for r in range(2)]
    g = rand_bf16(52, (cols,), 0.05, 1.0)
    for eps in (0.5, 3.0):
        out = o.sum_rmsnorm_fp8(xs, rows, cols, g, eps, 0.0, 1200.0, detail=True)
        h = f32(o.sum_bf16(xs, rows, cols)).astype(np.float64)
        ms = (h * h).mean(axis=1)
        y = out["v"].astype(np.float64) * out["scales"][:, None]
        lhs = ((y / f32(g).astype(np.float64)) ** 2).mean(axis=1)
        assert np.all(np.abs(lhs - ms / (ms + eps)) <= 3e-6 * ms / (ms + eps)), eps


# ------------------------------------------------------------- structure ---

def pin_determinism(o):
    """Repeated calls give the same bits."""
    xs = [rand_bf16(60 + r, (4, 72)) for r in range(3)]
    res = rand_bf16(63, (4, 72))
    g = rand_bf16(64, (72,), 0.1, 1.0)
    a = o.sum_rmsnorm_fp8(xs, 4, 72, g, 1e-5, 0.0, 1200.0, residual=res)
    b = o.sum_rmsnorm_fp8(xs, 4, 72, g, 1e-5, 0.0, 1200.0, residual=res)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def pin_row_independence(o):
    """Each row depends only on its own data: rows computed one range at a
    time equal the rows computed together (the property row sharding uses)."""
    rows, cols = 7, 40
    xs = [rand_bf16(70 + r, (rows, cols)) for r in range(2)]
    res = rand_bf16(72, (rows, cols))
    g = rand_bf16(73, (cols,), 0.1, 1.0)
    whole = o.sum_rmsnorm_fp8(xs, rows, cols, g, 1e-5, 0.0, 1200.0, residual=res)
    parts = [o.sum_rmsnorm_fp8(xs, rows, cols, g, 1e-5, 0.0, 1200.0, residual=res,
                               row_start=a, row_count=n) for a, n in ((0, 3), (3, 1), (4, 3))]
    for k in whole:
        assert np.array_equal(whole[k], np.concatenate([p[k] for p in parts])), k


# ------------------------------------------------------------- MX output ---
# The OCP MX v1.0 conversion: a block of 32 elements shares X = 2^(floor(
# log2(max |V|)) - 8) (e4m3's largest normal is 1.75 * 2^8), an E8M0 code;
# elements are V / X rounded to e4m3fn, nearest even, saturating.

def e8m0_value(codes) -> np.ndarray:
    """E8M0 codes -> values by ml_dtypes' float8_e8m0fnu decoding."""
    return np.asarray(codes, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)


def pin_mx_scale_code(o):
    """The code's scale X is the power of two with 256 <= amax / X < 512."""
    rng = np.random.default_rng(41)
    amax = np.concatenate([np.exp2(np.arange(-100.0, 120.0)),
                           rng.uniform(0.5, 2.0, 300) * np.exp2(rng.integers(-110, 110, 300))])
    for a in amax.astype(np.float32):
        x = e8m0_value(o.mx_scale_code(float(a)))
        assert 256.0 <= float(a) / x < 512.0, (a, x)
    assert o.mx_scale_code(0.0) == 0


def pin_mx_blocks_vs_row_scaled_oracle(o):
    """On a random problem: every block's largest |v| lies in [256, 512);
    the codes are torch's saturating conversion of v; v * X is the same y as
    the row-scaled (pinned) path's v * scale; h and the residual agree."""
    R, rows, cols = 3, 4, 256
    xs = [rand_bf16(43 + r, (rows, cols)) for r in range(R)]
    res = rand_bf16(50, (rows, cols))
    gamma = rand_bf16(51, cols, 0.1, 1.0)
    mx = o.sum_rmsnorm_mxfp8(xs, rows, cols, gamma, 1e-5, 0.0, residual=res, detail=True)
    ref = o.sum_rmsnorm_fp8(xs, rows, cols, gamma, 1e-5, 0.0, 1e30, residual=res, detail=True)
    v = mx["v"].reshape(rows, cols // 32, 32)
    m = np.abs(v).max(axis=2)
    assert np.all((m >= 256.0) & (m < 512.0))
    assert np.array_equal(mx["q"], lib_e4m3_torch(mx["v"]))
    X = np.repeat(e8m0_value(mx["scales_mx"]), 32, axis=1)
    y_mx = mx["v"].astype(np.float64) * X
    y_row = ref["v"].astype(np.float64) * ref["scales"].astype(np.float64)[:, None]
    assert np.all(np.abs(y_mx - y_row) <= 2.0 ** -22 * np.abs(y_row) + 1e-30)
    assert np.array_equal(mx["h"], ref["h"]) and np.array_equal(mx["res_out"], ref["res_out"])


def pin_mx_block_isolation(o):
    """Row of ones with one 64 at column 52 (R = 1, gamma 1, no residual):
    r = 1 / sqrt((127 + 4096) / 128 + eps); the 64 raises only block 1's
    scale: codes floor(log2(64 r)) + 119 there, floor(log2(r)) + 119 elsewhere."""
    cols = 128
    row = np.ones((1, cols), np.float32)
    row[0, 52] = 64.0
    eps = 1e-6
    mx = o.sum_rmsnorm_mxfp8([bf16_of(row)], 1, cols, bf16_of(np.ones(cols, np.float32)), eps,
                             0.0, detail=True)
    r = 1.0 / math.sqrt((127.0 + 4096.0) / cols + eps)
    want = [math.floor(math.log2(r)) + 119] * 4
    want[1] = math.floor(math.log2(64.0 * r)) + 119
    assert mx["scales_mx"][0].tolist() == want


def pin_mx_zero_block(o):
    """A block of zeros: code 0 and zero codes; the other blocks unaffected."""
    cols = 96
    row = rand_bf16(52, (1, cols))
    row[0, 32:64] = 0
    gamma = bf16_of(np.ones(cols, np.float32))
    mx = o.sum_rmsnorm_mxfp8([row], 1, cols, gamma, 1e-6, 0.0)
    assert mx["scales_mx"][0, 1] == 0 and np.all(mx["q"][0, 32:64] == 0)
    assert mx["scales_mx"][0, 0] > 0 and mx["scales_mx"][0, 2] > 0


# --------------------------------------------------------------- FP8 GEMM ---
# The consumer of the per-row scales (Ascend aclnnAlltoAllQuantMatmul,
# per-token dynamic quantisation): out = RN_bf16((a_q @ b_q^T) * a_scale *
# b_scale + bias).

def _bf16_table():
    """Every finite non-negative bf16 value, ascending, and its bit pattern."""
    bits = np.arange(0, 0x7F80, dtype=np.uint16)
    return f32(bits).astype(np.float64), bits


def brute_bf16_round_double(values) -> np.ndarray:
    """Nearest bf16 of float64 values by search in the table of all finite
    bf16 values; ties to the even pattern; beyond the midpoint between the
    largest finite value and 2^128, infinity."""
    vals, bits = _bf16_table()
    top = np.append(vals, 2.0 ** 128)
    v = np.asarray(values, dtype=np.float64).reshape(-1)
    out = np.empty(v.size, dtype=np.uint16)
    for i, x in enumerate(v):
        a = abs(x)
        j = int(np.searchsorted(top, a, side="right")) - 1  # top[j] <= a < top[j + 1]
        lo, hi = top[j], top[min(j + 1, len(top) - 1)]
        if a - lo < hi - a or a == lo:
            k = j
        elif hi - a < a - lo:
            k = j + 1
        else:
            k = j if j % 2 == 0 else j + 1
        b = 0x7F80 if k >= len(vals) else int(bits[k])
        out[i] = b | (0x8000 if math.copysign(1.0, x) < 0 else 0)
    return out.reshape(np.shape(values))


def rand_e4m3(seed: int, shape, std: float = 1.0) -> np.ndarray:
    """e4m3fn codes of normal samples (torch's conversion, clamped)."""
    rng = np.random.default_rng(seed)
    return lib_e4m3_torch(rng.normal(0.0, std, size=shape).astype(np.float32))


def pin_bf16_round_double_brute_force(o):
    rng = np.random.default_rng(31)
    x = np.concatenate([
        rng.normal(0, 1, 400) * np.exp2(rng.integers(-140, 128, 400)),
        # exact midpoints (ties), and one float64 ulp either side of them
        (np.arange(256, 512) + 0.5) * 2.0 ** -8,
        np.nextafter((np.arange(256, 320) + 0.5) * 2.0 ** -8, np.inf),
        np.nextafter((np.arange(256, 320) + 0.5) * 2.0 ** -8, -np.inf),
        [0.0, -0.0, 2.0 ** -134, 2.0 ** -133 * 1.5, 3.3895313892515355e38,
         2.0 ** 128 - 2.0 ** 119, np.nextafter(2.0 ** 128 - 2.0 ** 119, 0), 1e300]])
    x = np.concatenate([x, -x])
    assert np.array_equal(o.bf16_round_double(x), brute_bf16_round_double(x))


def pin_bf16_round_double_agrees_on_floats(o):
    """On values that are fp32 numbers the one rounding equals the pinned
    float32 rounding (torch's)."""
    rng = np.random.default_rng(32)
    v = (rng.normal(0, 1, 2000) * np.exp2(rng.integers(-100, 100, 2000))).astype(np.float32)
    assert np.array_equal(o.bf16_round_double(v.astype(np.float64)), lib_bf16(v))


def pin_scaled_mm_vs_float64_matmul(o):
    """Sum, scales and bias against numpy's float64 matmul of the codes'
    values (ml_dtypes' decoding); the sum of exact products is exact, so the
    float64 values agree bit for bit."""
    M, N, K = 5, 7, 96
    a, b = rand_e4m3(33, (M, K), 2.0), rand_e4m3(34, (N, K), 0.5)
    rng = np.random.default_rng(35)
    sa = rng.uniform(0.5, 2.0, M).astype(np.float32)
    sb = rng.uniform(0.01, 0.1, N).astype(np.float32)
    bias = lib_bf16(rng.normal(0, 1, N).astype(np.float32))
    S = lib_e4m3_decode(a) @ lib_e4m3_decode(b).T
    want = S * sa.astype(np.float64)[:, None] * sb.astype(np.float64)[None, :] + \
        f32(bias).astype(np.float64)[None, :]
    out, ex = o.scaled_mm(a, sa, b, sb, bias, exact=True)
    assert np.array_equal(ex, want)
    assert np.array_equal(out, brute_bf16_round_double(want))
    out0 = o.scaled_mm(a, sa, b, sb, None)
    assert np.array_equal(out0, brute_bf16_round_double(want - f32(bias)[None, :]))


def pin_scaled_mm_closed_forms(o):
    """All-ones codes give K * a_scale * b_scale; negating a row of a
    negates that row of the output; zero codes give +0."""
    M, N, K = 3, 4, 160
    ones = np.full((M, K), 0x38, np.uint8)  # e4m3fn 1.0
    sa = np.array([1.0, 0.5, 3.0], np.float32)
    sb = np.array([1.0, 2.0, 0.25, 0.125], np.float32)
    out, ex = o.scaled_mm(ones, sa, np.full((N, K), 0x38, np.uint8), sb, exact=True)
    assert np.array_equal(ex, K * sa[:, None].astype(np.float64) * sb[None, :])
    a, b = rand_e4m3(36, (M, K)), rand_e4m3(37, (N, K))
    pos = o.scaled_mm(a, sa, b, sb)
    neg_a = a.copy()
    neg_a[1] ^= 0x80
    neg = o.scaled_mm(neg_a, sa, b, sb)
    assert np.array_equal(neg[0], pos[0]) and np.array_equal(neg[2], pos[2])
    nz = pos[1] & 0x7FFF != 0
    assert np.array_equal(neg[1][nz], pos[1][nz] ^ 0x8000)
    zero = o.scaled_mm(np.zeros((M, K), np.uint8), sa, b, sb)
    assert np.all(zero == 0)


def pin_scaled_mm_rounds_once(o):
    """y = 1 * 1 * (1 + 2^-8) + 2^-40: just above the bf16 midpoint between 1
    and 1 + 2^-7, so one rounding gives 1 + 2^-7 (0x3F81); rounding to fp32
    first would land on the midpoint and then tie to 1.0 (0x3F80)."""
    one = np.full((1, 16), 0, np.uint8)
    one[0, 0] = 0x38
    sb = np.array([1.0 + 2.0 ** -8], np.float32)
    up = o.scaled_mm(one, np.ones(1, np.float32), one, sb, bf16_of([2.0 ** -40]))
    down = o.scaled_mm(one, np.ones(1, np.float32), one, sb, bf16_of([-2.0 ** -40]))
    assert up[0, 0] == 0x3F81 and down[0, 0] == 0x3F80


def pin_scaled_mm_k_split(o):
    """The sum over K is the sum of the sums over two halves (exactly)."""
    M, N, K = 4, 5, 256
    a, b = rand_e4m3(38, (M, K), 3.0), rand_e4m3(39, (N, K), 3.0)
    one_m, one_n = np.ones(M, np.float32), np.ones(N, np.float32)
    _, whole = o.scaled_mm(a, one_m, b, one_n, exact=True)
    _, lo = o.scaled_mm(a[:, :100], one_m, b[:, :100], one_n, exact=True)
    _, hi = o.scaled_mm(a[:, 100:], one_m, b[:, 100:], one_n, exact=True)
    assert np.array_equal(whole, lo + hi)


# ----------------------------------------------------------------- MX GEMM ---
# The Ascend page's mx scenario: out = (x1 * x1Scale) @ (x2 * x2Scale) +
# bias, one E8M0 scale per 32 values of K on both operands.

def rand_e8m0(seed: int, shape, lo: int = 120, hi: int = 134) -> np.ndarray:
    return np.random.default_rng(seed).integers(lo, hi, size=shape).astype(np.uint8)


def pin_scaled_mm_mx_vs_float64_matmul(o):
    """Against numpy's float64 matmul of the dequantised operands (ml_dtypes'
    e4m3fn and E8M0 decodings): the same float64 values, the same bf16."""
    M, N, K = 4, 6, 160
    a, b = rand_e4m3(61, (M, K), 2.0), rand_e4m3(62, (N, K), 2.0)
    sa, sb = rand_e8m0(63, (M, K // 32)), rand_e8m0(64, (N, K // 32))
    bias = lib_bf16(np.random.default_rng(65).normal(0, 1, N).astype(np.float32))
    A = lib_e4m3_decode(a) * np.repeat(e8m0_value(sa), 32, axis=1)
    B = lib_e4m3_decode(b) * np.repeat(e8m0_value(sb), 32, axis=1)
    want = A @ B.T + f32(bias).astype(np.float64)[None, :]
    out, ex = o.scaled_mm_mx(a, sa, b, sb, bias, exact=True)
    assert np.array_equal(ex, want)
    assert np.array_equal(out, brute_bf16_round_double(want))


def pin_scaled_mm_mx_reduces_to_row_scales(o):
    """With one scale code per row of a and per row of b, the MX GEMM is the
    (pinned) per-token GEMM with scales 2^(code - 127)."""
    M, N, K = 3, 5, 128
    a, b = rand_e4m3(66, (M, K)), rand_e4m3(67, (N, K))
    ca, cb = rand_e8m0(68, M), rand_e8m0(69, N)
    sa, sb = np.repeat(ca[:, None], K // 32, axis=1), np.repeat(cb[:, None], K // 32, axis=1)
    mx = o.scaled_mm_mx(a, sa, b, sb)
    row = o.scaled_mm(a, e8m0_value(ca).astype(np.float32), b, e8m0_value(cb).astype(np.float32))
    assert np.array_equal(mx, row)


def pin_scaled_mm_mx_block_linearity(o):
    """Raising one block's scale code of a by one adds exactly that block's
    contribution once more (the blocks are the 32 values of K they cover)."""
    M, N, K = 2, 3, 128
    a, b = rand_e4m3(70, (M, K)), rand_e4m3(71, (N, K))
    sa, sb = rand_e8m0(72, (M, K // 32)), rand_e8m0(73, (N, K // 32))
    _, base = o.scaled_mm_mx(a, sa, b, sb, exact=True)
    sa2 = sa.copy()
    sa2[1, 2] += 1
    _, up = o.scaled_mm_mx(a, sa2, b, sb, exact=True)
    keep = np.zeros_like(a)
    keep[1, 64:96] = a[1, 64:96]
    _, blk = o.scaled_mm_mx(keep, sa, b, sb, exact=True)
    assert np.array_equal(up[0], base[0]) and np.array_equal(up[1], base[1] + blk[1])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
