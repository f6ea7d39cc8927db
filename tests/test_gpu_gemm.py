"""GPU parity of the FP8 GEMM that consumes the per-row scales
(rrf_scaled_mm_fp8) against the oracle.

Tolerance, from the arithmetic: the products of two e4m3 values are exact;
the tensor cores sum K of them in fp32, within (K - 1) u sum_k |a_k b_k|
(u = 2^-24, the recursive-summation bound, whatever the order); the
epilogue's two multiplications and the bias add cost 3 u (|y| + |bias|); the
result is rounded once to bf16.  So |out - y| <= E + ulp_bf16(|y| + E) with
E = (K - 1) u sum|a b| sa sb + 3 u (|y| + |bias|), y the oracle's exact value.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def rrf():
    import reduce_rmsnorm_fp8_b200 as m
    return m


def codes(t):
    return t.view(torch.uint8).cpu().numpy()


def bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def check(c, got, rows=None, label=""):
    """Compare the GPU output (bf16 tensor [M, N]) with the oracle on all rows
    or the listed ones; returns the largest error as a fraction of the bound."""
    rows = np.arange(c.M) if rows is None else np.asarray(rows)
    a, b = codes(c.a)[rows], codes(c.b)
    sa, sb = c.a_scale.cpu().numpy()[rows], c.b_scale.cpu().numpy()
    bias = None if c.bias is None else workloads.bits(c.bias)
    _, y = oracle.scaled_mm(a, sa, b, sb, bias, exact=True)
    dec = lambda x: np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))[x]
    mag = dec(a) @ dec(b).T * sa.astype(np.float64)[:, None] * sb.astype(np.float64)[None, :]
    bmag = 0.0 if bias is None else np.abs(bf16_values(bias)).astype(np.float64)[None, :]
    E = (c.K - 1) * U * mag + 3 * U * (np.abs(y) + bmag)
    a_ = np.maximum(np.abs(y) + E, 2.0 ** -126)
    tol = E + np.exp2(np.floor(np.log2(a_)) - 7)
    g = bf16_values(workloads.bits(got)[rows]).astype(np.float64)
    err = np.abs(g - y)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"{label}: error {err.max():.3g} beyond the bound (ratio {worst:.3g})"
    return worst


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (9, 512, 640), (24, 336, 1536),
                                   (5, 256, 144), (37, 256, 256), (128, 128, 128),
                                   (200, 272, 384), (130, 400, 144), (64, 1024, 1024),
                                   (256, 512, 2048),
                                   # an odd number of k-tiles after full boxes: the
                                   # swapped kernel's last pair takes the box's zeros
                                   (3, 320, 1152), (16, 208, 1408), (29, 128, 1664)])
@pytest.mark.parametrize("bias", [True, False])
def test_scaled_mm_matches_oracle(rrf, M, N, K, bias):
    c = workloads.make_gemm_case(M, N, K, sub=M % 7, bias=bias, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    torch.cuda.synchronize()
    check(c, out, label=f"{M}x{N}x{K}")


def test_wide_tiles_sampled_rows(rrf):
    """A grid of 256 x 256 tiles on SM pairs with row and column tails;
    sampled rows against the oracle, including both tails."""
    c = workloads.make_gemm_case(2000, 2576, 1040, sub=3, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    torch.cuda.synchronize()
    check(c, out, rows=[0, 1, 127, 128, 255, 1000, 1919, 1920, 1999], label="wide")


@pytest.mark.parametrize("M", [1, 8, 16, 32, 64])
def test_decode_projection_sampled_rows(rrf, M):
    N = K = 7168
    c = workloads.make_gemm_case(M, N, K, sub=M, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    torch.cuda.synchronize()
    check(c, out, rows=sorted({0, M // 2, M - 1}), label=f"decode {M}")


def sm_count():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("M,N,K,kernel", [(1, 16384, 7168, "swap"), (8, 16384, 7168, "swap"),
                                          (32, 16384, 7168, "swap"), (16, 16384, 1024, "swap"),
                                          (9, 16384, 1024, "swap"), (64, 16384, 1024, "tile"),
                                          (8, 16384, 1040, "tile"), (100, 16384, 1024, "tile")])
def test_several_tiles_per_cta(rrf, M, N, K, kernel):
    """Products with more 64-column weight tiles than CTAs, so every
    persistent CTA walks several tiles and reuses its stage ring and both
    accumulators: the swapped kernel at each row padding (8, 16, 32), the
    64-row and 128-row A-stage kernels, and the one-k-tile-per-box form
    (K % 128 != 0).  The plan query shows which kernel ran; sampled rows
    with every column against the oracle."""
    p = rrf.rrf_plan_scaled_mm(M, N, K, sm_count())
    assert p["kernel"] == kernel and p["tiles"] > p["ctas"], p
    c = workloads.make_gemm_case(M, N, K, sub=M % 5, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    torch.cuda.synchronize()
    check(c, out, rows=sorted({0, M // 2, M - 1}), label=f"{M}x{N}x{K}")
    assert rrf.rrf_device_error() == 0


def test_prefill_sampled_rows(rrf):
    c = workloads.make_gemm_case(8192, 8192, 8192, sub=1, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    torch.cuda.synchronize()
    check(c, out, rows=[0, 4095, 8191], label="prefill")


def test_consumes_the_fused_call(rrf):
    """The fused kernel's codes and scales feed the GEMM directly."""
    case = parity.to_device(workloads.make_case("decode", 64))
    q, scales, _ = rrf.rrf_sum_rmsnorm_fp8(case.inputs, case.gamma, case.eps,
                                           case.weight_offset, case.scale_ub,
                                           residual_in=case.residual.clone())
    w = workloads.make_gemm_case(1, 1024, case.cols, sub=5, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(q, scales, w.b, w.b_scale, w.bias)
    torch.cuda.synchronize()
    c = workloads.GemmCase(64, 1024, case.cols, q, scales.reshape(-1), w.b, w.b_scale, w.bias)
    check(c, out, label="fused -> gemm")


def test_deterministic_and_empty(rrf):
    c = workloads.make_gemm_case(96, 512, 512, sub=2, device="cuda")
    o1 = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    o2 = rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    e = workloads.make_gemm_case(0, 256, 256, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(e.a, e.a_scale, e.b, e.b_scale, e.bias)
    assert out.shape == (0, 256)
    assert rrf.rrf_device_error() == 0


@pytest.mark.parametrize("M,N,K,mx", [(96, 512, 512, False), (8, 1024, 1024, False),
                                      (2048, 2048, 512, False), (4096, 4096, 512, False),
                                      (96, 512, 512, True), (4096, 4096, 512, True)])
def test_wait_timeout_is_reported(rrf, M, N, K, mx):
    """The test hook makes the epilogue's bounded wait run out (one CTA's
    tile, several tiles per CTA, SM pairs; per-token and MX): the call
    finishes, reports RRF_DEVICE_ERROR_GEMM_TIMEOUT, and the next call on the
    same operands matches the oracle."""
    import test_gpu_mx
    rrf.rrf_device_error(clear=True)
    if mx:
        c, sa, sb = test_gpu_mx.mx_operands(M, N, K, 6)
        args = (c.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), c.b,
                rrf.mx_blocked(torch.from_numpy(sb).cuda()), c.bias)
        call = lambda: rrf.rrf_scaled_mm_mxfp8(*args)
    else:
        c = workloads.make_gemm_case(M, N, K, sub=6, device="cuda")
        call = lambda: rrf.rrf_scaled_mm_fp8(c.a, c.a_scale, c.b, c.b_scale, c.bias)
    rrf.rrf_debug_starve_next_gemm()
    call()
    torch.cuda.synchronize()
    assert rrf.rrf_device_error(clear=True) & rrf.RRF_DEVICE_ERROR_GEMM_TIMEOUT
    out = call()
    torch.cuda.synchronize()
    assert rrf.rrf_device_error() == 0
    rows = [0, M // 2, M - 1]
    if mx:
        test_gpu_mx.check_mx_gemm(c, sa, sb, out, rows=rows, label="after the timeout")
    else:
        check(c, out, rows=rows, label="after the timeout")
