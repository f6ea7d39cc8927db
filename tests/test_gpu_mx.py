"""GPU parity of the MX output (rrf_sum_rmsnorm_mxfp8): one E8M0 scale per
32 elements, against the oracle (tolerances in parity.assert_mx_parity)."""
import numpy as np
import pytest
import torch

import parity
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rrf():
    import reduce_rmsnorm_fp8_b200 as m
    return m


def gpu_mx(rrf, c, in_place=False):
    res_in = None if c.residual is None else c.residual.clone()
    q, sc, res = rrf.rrf_sum_rmsnorm_mxfp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                           residual_in=res_in,
                                           residual_out=res_in if in_place else None)
    torch.cuda.synchronize()
    out = {"q": q.view(torch.uint8).cpu().numpy(), "scales_mx": sc.cpu().numpy()}
    if res is not None:
        out["res_out"] = workloads.bits(res)
    return out


CASES = [("tiny", 4), ("decode", 1), ("decode", 8), ("decode", 32), ("decode", 64),
         ("odd", 37), ("odd", 64), ("sweep", 16), ("sweep", 64), ("sweep", 256)]


@pytest.mark.parametrize("name,rows", CASES)
def test_mx_matches_oracle(rrf, name, rows):
    c = parity.to_device(workloads.make_case(name, rows))
    parity.assert_mx_parity(gpu_mx(rrf, c), parity.oracle_mx(c), f"{name} {rows}")


def test_mx_prefill_sampled_rows(rrf):
    c = parity.to_device(workloads.make_case("prefill", 8192))
    got = gpu_mx(rrf, c)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 397), [1, 8191]]))
    parity.assert_mx_parity(parity.select_rows(got, rows), parity.oracle_mx(c, rows=rows),
                            "prefill")


def test_mx_in_place_and_rows_of_the_row_scaled_call(rrf):
    """In place; and the norm input h (residual_out) is the row-scaled call's."""
    c = parity.to_device(workloads.make_case("decode", 32))
    ref = parity.oracle_mx(c)
    got = gpu_mx(rrf, c, in_place=True)
    parity.assert_mx_parity(got, ref, "in place")
    assert np.array_equal(got["res_out"], parity.gpu_fused(c)["res_out"])


@pytest.mark.parametrize("R,cols", [(1, 32), (3, 96), (16, 4096), (5, 131072)])
def test_mx_edges(rrf, R, cols):
    c = parity.to_device(workloads.make_case("odd", 3, R=R, cols=cols))
    parity.assert_mx_parity(gpu_mx(rrf, c), parity.oracle_mx(c), f"R={R} cols={cols}",
                            cap_at_ties=True)


def test_mx_zero_rows_and_blocks(rrf):
    """Zero inputs: every block takes code 0 and every code is +-0."""
    c = parity.to_device(workloads.make_case("decode", 8))
    for x in c.inputs:
        x.zero_()
    c.residual.zero_()
    got = gpu_mx(rrf, c)
    assert np.all(got["scales_mx"] == 0) and np.all((got["q"] & 0x7F) == 0)
    parity.assert_mx_parity(got, parity.oracle_mx(c), "zeros")


def test_mx_empty(rrf):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, sc, _ = rrf.rrf_sum_rmsnorm_mxfp8([x], torch.ones(64, dtype=torch.bfloat16,
                                                         device="cuda"), 1e-6, 0.0)
    assert q.shape == (0, 64) and sc.shape == (0, 2)


# ------------------------------------------------------------ blocked order --

def test_blocked_scales_are_the_row_major_ones(rrf):
    """The blocked output is the row-major output in the blocked order (the
    layout the block-scaled GEMM reads), for rows that are and are not a
    multiple of 128."""
    for name, rows in (("decode", 64), ("odd", 37), ("prefill", 8192)):
        c = parity.to_device(workloads.make_case(name, rows))
        q1, s1, _ = rrf.rrf_sum_rmsnorm_mxfp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                              residual_in=c.residual.clone())
        sb = torch.zeros(rrf.mx_blocked_bytes(rows, c.cols), dtype=torch.uint8, device="cuda")
        q2, s2, _ = rrf.rrf_sum_rmsnorm_mxfp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                              residual_in=c.residual.clone(), scales_mx_out=sb,
                                              blocked=True)
        torch.cuda.synchronize()
        assert torch.equal(q1.view(torch.uint8), q2.view(torch.uint8)), name
        assert torch.equal(s2, rrf.mx_blocked(s1)), name


# ----------------------------------------------------------------- MX GEMM --

U = 2.0 ** -24


def mx_operands(M, N, K, seed, bias=True):
    """Codes of N(0, 1) samples and E8M0 codes in [120, 134) for both
    operands (workloads' operand codes; the scale codes drawn here)."""
    c = workloads.make_gemm_case(M, N, K, sub=seed, bias=bias, device="cuda")
    rng = np.random.default_rng(100 + seed)
    sa = rng.integers(120, 134, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(120, 134, (N, K // 32)).astype(np.uint8)
    return c, sa, sb


def check_mx_gemm(c, sa, sb, got, rows=None, label=""):
    """Against the oracle within the fp32-summation bound (as for the FP8
    GEMM): |out - y| <= E + ulp_bf16(|y| + E), E = (K - 1) u sum|terms| +
    u |bias|."""
    import oracle
    rows = np.arange(c.M) if rows is None else np.asarray(rows)
    a = c.a.view(torch.uint8).cpu().numpy()[rows]
    b = c.b.view(torch.uint8).cpu().numpy()
    bias = None if c.bias is None else workloads.bits(c.bias)
    _, y = oracle.scaled_mm_mx(a, sa[rows], b, sb, bias, exact=True)
    e8 = np.exp2(np.arange(256, dtype=np.float64) - 127)
    dec = np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    A = dec[a] * np.repeat(e8[sa[rows]], 32, axis=1)
    B = dec[b] * np.repeat(e8[sb], 32, axis=1)
    bmag = 0.0 if bias is None else np.abs(
        (bias.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)[None, :]
    E = (c.K - 1) * U * (A @ B.T) + U * (np.abs(y) + bmag)
    tol = E + np.exp2(np.floor(np.log2(np.maximum(np.abs(y) + E, 2.0 ** -126))) - 7)
    g = (workloads.bits(got)[rows].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    worst = float((np.abs(g - y) / tol).max())
    assert worst <= 1.0, f"{label}: beyond the bound (ratio {worst:.3g})"


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (8, 384, 512), (13, 320, 1024),
                                   (32, 448, 640), (37, 256, 256), (128, 128, 512),
                                   (200, 272, 384), (130, 400, 1024), (256, 512, 2048),
                                   # an odd number of k-tiles after full boxes: the
                                   # swapped kernel's last pair takes the box's zeros
                                   (3, 256, 1152), (24, 384, 1408),
                                   # a last weight tile in the odd half of its scale
                                   # block, 16 of its 64 rows inside N
                                   (5, 208, 256)])
@pytest.mark.parametrize("bias", [True, False])
def test_mx_gemm_matches_oracle(rrf, M, N, K, bias):
    c, sa, sb = mx_operands(M, N, K, M % 5, bias)
    out = rrf.rrf_scaled_mm_mxfp8(c.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), c.b,
                                  rrf.mx_blocked(torch.from_numpy(sb).cuda()), c.bias)
    torch.cuda.synchronize()
    check_mx_gemm(c, sa, sb, out, label=f"{M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K,bias", [(2200, 2320, 384, True), (2200, 2320, 384, False),
                                        (2100, 2336, 256, True)])
def test_mx_gemm_pair_tiles_with_tails(rrf, M, N, K, bias):
    """Enough 256 x 256 tiles for the SM-pair kernel (every pair takes two,
    so both accumulators and their shared columns are used), with a row tail
    inside the odd CTA's half (2200) or inside the even CTA's half with the
    odd CTA's rows and scale atom wholly past the operand (2100), and a
    column tail that leaves the odd CTA's B half and the second B scale atom
    past the operand; every output checked."""
    c, sa, sb = mx_operands(M, N, K, 4, bias)
    out = rrf.rrf_scaled_mm_mxfp8(c.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), c.b,
                                  rrf.mx_blocked(torch.from_numpy(sb).cuda()), c.bias)
    torch.cuda.synchronize()
    check_mx_gemm(c, sa, sb, out, label=f"pair {M}x{N}x{K}")
    assert rrf.rrf_device_error() == 0


@pytest.mark.parametrize("M,N,K", [(8, 7168, 7168), (64, 7168, 7168), (2000, 2560, 1024),
                                   (8192, 8192, 8192)])
def test_mx_gemm_large_sampled_rows(rrf, M, N, K):
    c, sa, sb = mx_operands(M, N, K, 7)
    out = rrf.rrf_scaled_mm_mxfp8(c.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), c.b,
                                  rrf.mx_blocked(torch.from_numpy(sb).cuda()), c.bias)
    torch.cuda.synchronize()
    check_mx_gemm(c, sa, sb, out, rows=sorted({0, 1, M // 2, M - 1}), label=f"{M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(8, 16384, 1024), (16, 16384, 1024), (24, 16384, 1024),
                                   (64, 16384, 7168), (100, 16384, 1024)])
def test_mx_gemm_several_tiles_per_cta(rrf, M, N, K):
    """More 64-column output tiles than CTAs (N = 16384: 256 tiles on at most
    one CTA per SM), so each persistent CTA walks several tiles with its
    stage ring, both accumulators and the odd tiles' half of the weight's
    scale atoms: the swapped kernel at 8, 16 and 32 rows, the 64- and
    128-row A-stage kernels; sampled rows, every column, against the
    oracle."""
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    p = rrf.rrf_plan_scaled_mm(M, N, K, sm, mx=True)
    want = "swap" if M <= 32 else "tile"
    assert p["kernel"] == want and p["tile_n"] == 64 and p["tiles"] > p["ctas"], p
    c, sa, sb = mx_operands(M, N, K, 8)
    out = rrf.rrf_scaled_mm_mxfp8(c.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), c.b,
                                  rrf.mx_blocked(torch.from_numpy(sb).cuda()), c.bias)
    torch.cuda.synchronize()
    check_mx_gemm(c, sa, sb, out, rows=sorted({0, 1, M // 2, M - 1}), label=f"{M}x{N}x{K}")
    assert rrf.rrf_device_error() == 0


def test_mx_quantizer_feeds_mx_gemm(rrf):
    """The fused call's MX codes and blocked scales feed the MX GEMM."""
    case = parity.to_device(workloads.make_case("decode", 64))
    q, sblk, _ = rrf.rrf_sum_rmsnorm_mxfp8(case.inputs, case.gamma, case.eps,
                                           case.weight_offset,
                                           residual_in=case.residual.clone(), blocked=True)
    _, splain, _ = rrf.rrf_sum_rmsnorm_mxfp8(case.inputs, case.gamma, case.eps,
                                             case.weight_offset,
                                             residual_in=case.residual.clone())
    w, _, sb = mx_operands(1, 1024, case.cols, 9)
    out = rrf.rrf_scaled_mm_mxfp8(q, sblk, w.b, rrf.mx_blocked(torch.from_numpy(sb).cuda()),
                                  w.bias)
    torch.cuda.synchronize()
    c = workloads.GemmCase(64, 1024, case.cols, q, None, w.b, None, w.bias)
    check_mx_gemm(c, splain.cpu().numpy(), sb, out, label="mx quantizer -> mx gemm")


def test_mx_gemm_deterministic_and_empty(rrf):
    c, sa, sb = mx_operands(96, 256, 512, 3)
    args = (c.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), c.b,
            rrf.mx_blocked(torch.from_numpy(sb).cuda()), c.bias)
    o1, o2 = rrf.rrf_scaled_mm_mxfp8(*args), rrf.rrf_scaled_mm_mxfp8(*args)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    e = workloads.make_gemm_case(0, 256, 256, device="cuda")
    out = rrf.rrf_scaled_mm_mxfp8(e.a, torch.empty(0, dtype=torch.uint8, device="cuda"), e.b,
                                  torch.zeros(rrf.mx_blocked_bytes(256, 256), dtype=torch.uint8,
                                              device="cuda"), e.bias)
    assert out.shape == (0, 256)
    assert rrf.rrf_device_error() == 0
