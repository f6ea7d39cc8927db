"""GPU parity: the CUDA library against the oracle on the same seeded inputs.

Every workload is run through the C ABI (via the thin binding) and compared
element by element with the oracle: bit-exact bf16 sum and residual, scales
within 1e-6 relative, fp8 codes equal up to the stated midpoint allowance.
The full-size prefill case is checked on sampled rows, in the launch the
benchmark times.
"""
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


def dev_case(name, rows=None, **kw):
    return parity.to_device(workloads.make_case(name, rows, **kw))


# ----------------------------------------------------------- the workloads ---

def test_tiny(rrf):
    c = dev_case("tiny")
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), "tiny")
    assert np.array_equal(workloads.bits(rrf.rrf_sum(c.inputs)), parity.oracle_sum(c))


@pytest.mark.parametrize("rows", [1, 8, 32, 64])
def test_decode(rrf, rows):
    c = dev_case("decode", rows)
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), f"decode {rows}")


@pytest.mark.parametrize("rows", [37, 64])
def test_odd_shapes_with_clamped_rows(rrf, rows):
    c = dev_case("odd", rows)
    ref = parity.oracle_fused(c)
    parity.assert_fused_parity(parity.gpu_fused(c), ref, f"odd {rows}")
    # 1% of the elements are 50x outliers, so every row of 7168 columns holds
    # some and reaches the clamp: the scale is then exactly fp32(ub / 448)
    ub_scale = np.float32(c.scale_ub) / np.float32(448.0)
    assert (ref["scales"] == ub_scale).all(), "a row missed the scale_ub clamp"


@pytest.mark.parametrize("rows", [16, 32, 48, 64, 96, 128, 256])
def test_sweep_sum_and_fused(rrf, rows):
    c = dev_case("sweep", rows)
    assert np.array_equal(workloads.bits(rrf.rrf_sum(c.inputs)), parity.oracle_sum(c))
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), f"sweep {rows}")


def test_prefill_full_size_sampled_rows(rrf):
    """8 x 8192 x 8192 with residual, drawn on the GPU; the outputs of the
    whole call are checked on 40 rows spread over the batch (first and last
    included) against the oracle on exactly those rows."""
    c = workloads.make_case("prefill", device="cuda")
    gpu = parity.gpu_fused(c)
    rows = sorted(set([0, 1, c.rows - 1] + list(np.random.default_rng(4).choice(
        c.rows, 37, replace=False))))
    ref = parity.oracle_fused(c, rows=rows)
    parity.assert_fused_parity(parity.select_rows(gpu, rows), ref, "prefill")
    # every row's scale is positive and finite, and every residual row written
    assert np.isfinite(gpu["scales"]).all() and (gpu["scales"] > 0).all()
    del c
    torch.cuda.empty_cache()


def test_sum_prefill_size(rrf):
    """rrf_sum at 8 x 8192 x 8192: bit-exact on sampled rows."""
    c = workloads.make_case("prefill", device="cuda", residual=False)
    s = rrf.rrf_sum(c.inputs)
    rows = [0, 4095, 8191]
    idx = torch.tensor(rows, device="cuda")
    import oracle
    ref = oracle.sum_bf16([workloads.bits(x.index_select(0, idx)) for x in c.inputs], 3, c.cols)
    assert np.array_equal(workloads.bits(s.index_select(0, idx)), ref)
    del c, s
    torch.cuda.empty_cache()


# ------------------------------------------------------ forced launch shapes ---

@pytest.mark.parametrize("name,rows", [("decode", 64), ("odd", 37), ("decode", 1),
                                       ("sweep", 16)])
@pytest.mark.parametrize("variant,cluster", [(1, 0), (2, 2), (2, 3), (2, 4), (2, 5), (2, 6),
                                             (2, 7), (2, 8), (2, 12), (2, 14), (2, 16)])
def test_forced_variants(rrf, name, rows, variant, cluster):
    """Every cluster size (1 = one block per row; powers of two reduce the
    slots with the butterfly, the others in slot order) gives the same bf16
    outputs and matches the oracle within tolerance."""
    c = dev_case(name, rows)
    gpu = parity.gpu_fused(c, variant=variant, cluster_size=cluster)
    parity.assert_fused_parity(gpu, parity.oracle_fused(c), f"{name} {rows} C={cluster}")


@pytest.mark.parametrize("threads", [32, 64, 128, 256, 512])
def test_forced_block_sizes(rrf, threads):
    c = dev_case("odd", 64)
    ref = parity.oracle_fused(c)
    for variant, cluster in ((1, 0), (2, 4)):
        try:
            gpu = parity.gpu_fused(c, variant=variant, cluster_size=cluster,
                                   block_threads=threads)
        except rrf.RrfError as e:
            assert e.status == rrf.Status.ERR_UNSUPPORTED  # slice too long for the block
            continue
        parity.assert_fused_parity(gpu, ref, f"threads={threads} C={cluster}")


@pytest.mark.parametrize("cluster", [2, 3, 4, 7, 8, 16])
@pytest.mark.parametrize("exchange", ["async", "barrier"])
def test_cluster_exchanges(rrf, cluster, exchange):
    """Both ways for a cluster's blocks to share their statistics -- st.async
    into the peers' shared memory counted on mbarriers, or a cluster barrier
    phase -- match the oracle, and leave the device error word clear."""
    rrf.rrf_device_error(clear=True)
    flags = 0 if exchange == "async" else rrf.RRF_FLAG_BARRIER_EXCHANGE
    for name, rows in (("decode", 8), ("odd", 37)):
        c = dev_case(name, rows)
        gpu = parity.gpu_fused(c, variant=2, cluster_size=cluster, flags=flags)
        parity.assert_fused_parity(gpu, parity.oracle_fused(c), f"{name} C={cluster} {exchange}")
    assert rrf.rrf_device_error() == 0


def test_starved_exchange_times_out_and_reports(rrf):
    """Failure detection without a GPU fault: every block waits for one value
    that no peer sends; the bounded wait runs out (about 2 ms), the kernel
    sets the timeout bit and finishes; the context stays usable and the next
    call is correct."""
    c = dev_case("decode", 8)
    rrf.rrf_device_error(clear=True)
    parity.gpu_fused(c, variant=2, cluster_size=8, flags=rrf.RRF_FLAG_DEBUG_STARVE_EXCHANGE)
    assert rrf.rrf_device_error(clear=True) & rrf.RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT
    assert rrf.rrf_device_error() == 0
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), "after timeout")
    assert rrf.rrf_device_error() == 0
    for variant, flags in ((1, 0), (2, rrf.RRF_FLAG_BARRIER_EXCHANGE)):
        # the hook needs a clustered launch with the transaction-counted exchange
        with pytest.raises(rrf.RrfError) as e:
            parity.gpu_fused(c, variant=variant, cluster_size=0 if variant == 1 else 8,
                             flags=flags | rrf.RRF_FLAG_DEBUG_STARVE_EXCHANGE)
        assert e.value.status == rrf.Status.ERR_UNSUPPORTED


def test_variants_bitwise_identical_bf16(rrf):
    c = dev_case("decode", 32)
    outs = [parity.gpu_fused(c, variant=v, cluster_size=k)
            for v, k in ((1, 0), (2, 2), (2, 4), (2, 7), (2, 8), (2, 16))]
    for o in outs[1:]:
        assert np.array_equal(o["res_out"], outs[0]["res_out"])


def test_programmatic_dependent_launch_flag(rrf):
    """Launching without programmatic dependent launch gives the same bits,
    and a chain of dependent calls (each reading the previous call's residual
    output) matches the oracle: the wait for the previous grid keeps stream
    order."""
    c = dev_case("decode", 64)
    a = parity.gpu_fused(c)
    b = parity.gpu_fused(c, flags=rrf.RRF_FLAG_NO_PDL)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    # chain: residual_out of call i is residual_in of call i + 1
    res = c.residual.clone()
    outs = []
    for i in range(4):
        nxt = torch.empty_like(res)
        rrf.rrf_sum_rmsnorm_fp8(c.inputs, c.gamma, c.eps, c.weight_offset, c.scale_ub,
                                residual_in=res, residual_out=nxt)
        res = nxt
        outs.append(nxt)
    torch.cuda.synchronize()
    expect = c.residual
    for i in range(4):
        step = workloads.Case(c.name, c.R, c.rows, c.cols, c.inputs, expect, c.gamma, c.eps,
                              c.weight_offset, c.scale_ub)
        ref = parity.oracle_fused(step)
        assert np.array_equal(workloads.bits(outs[i]), ref["res_out"]), i
        expect = outs[i]


@pytest.mark.parametrize("name,rows", [("decode", 64), ("decode", 1), ("odd", 37),
                                       ("tiny", None), ("sweep", 256)])
def test_prefetch_flags(rrf, name, rows):
    """The L2 prefetch before the wait for the previous kernel, forced on and
    off: the same bits either way, matching the oracle."""
    c = dev_case(name, rows)
    on = parity.gpu_fused(c, flags=rrf.RRF_FLAG_PREFETCH)
    off = parity.gpu_fused(c, flags=rrf.RRF_FLAG_NO_PREFETCH)
    for k in on:
        assert np.array_equal(on[k], off[k]), k
    parity.assert_fused_parity(on, parity.oracle_fused(c), f"{name} prefetch")
    with pytest.raises(rrf.RrfError):
        parity.gpu_fused(c, flags=rrf.RRF_FLAG_PREFETCH | rrf.RRF_FLAG_NO_PREFETCH)


@pytest.mark.parametrize("cluster", [0, 7])
def test_prefetch_of_data_the_previous_kernel_writes(rrf, cluster):
    """A chain in which every call's inputs are the previous call's residual
    output: each call prefetches (with PDL) the very rows the kernel before it
    is still writing, and must still read the new values after its wait."""
    c = dev_case("decode", 64, R=2)
    x0 = c.inputs[0]
    bufs = [c.inputs[1].clone()] + [torch.empty_like(x0) for _ in range(6)]
    res = c.residual.clone()
    for i in range(6):
        # call i: inputs (x0, bufs[i]), residual res; writes bufs[i + 1]
        rrf.rrf_sum_rmsnorm_fp8_ex([x0, bufs[i]], c.gamma, c.eps, c.weight_offset, c.scale_ub,
                                   residual_in=res, residual_out=bufs[i + 1],
                                   variant=2 if cluster else 0, cluster_size=cluster,
                                   flags=rrf.RRF_FLAG_PREFETCH)
    torch.cuda.synchronize()
    bits = workloads.bits
    prev = bufs[0]
    for i in range(6):
        step = workloads.Case(c.name, 2, c.rows, c.cols, [x0, prev], res, c.gamma, c.eps,
                              c.weight_offset, c.scale_ub)
        assert np.array_equal(bits(bufs[i + 1]), parity.oracle_fused(step)["res_out"]), i
        prev = bufs[i + 1]


# --------------------------------------------------------------- random shapes ---

def test_random_shapes_and_launches(rrf):
    """60 seeded random problems: R, rows, cols (multiples of 8, many ragged),
    residual on/off (in place or not), scalars, and a random forced launch
    (automatic, one block per row, or a cluster of 2-16 with either
    exchange, a random block size); every one matches the oracle."""
    rng = np.random.default_rng(2026)
    checked = 0
    for _ in range(60):
        R = int(rng.integers(1, 17))
        rows = int(rng.choice([1, 2, 3, 5, 7, 16, 33, 64, 150, 300]))
        cols = int(8 * rng.integers(1, 1200))
        c = dev_case("decode", rows, cols=cols, R=R, residual=bool(rng.integers(0, 2)))
        c.eps = float(rng.choice([0.0, 1e-6, 1e-5, 0.1]))
        c.weight_offset = float(rng.choice([0.0, 1.0, -0.5]))
        c.scale_ub = float(rng.choice([1200.0, 8.0, 0.5, float("inf")]))
        variant = int(rng.choice([0, 1, 2]))
        cluster = int(rng.integers(2, 17)) if variant == 2 else 0
        threads = int(rng.choice([0, 0, 32, 64, 128, 256, 512]))
        flags = int(rng.choice([0, rrf.RRF_FLAG_BARRIER_EXCHANGE, rrf.RRF_FLAG_NO_PDL,
                                rrf.RRF_FLAG_PREFETCH, rrf.RRF_FLAG_NO_PREFETCH]))
        in_place = c.residual is not None and bool(rng.integers(0, 2))
        try:
            gpu = parity.gpu_fused(c, variant=variant, cluster_size=cluster,
                                   block_threads=threads, flags=flags, in_place=in_place)
        except rrf.RrfError as e:
            assert e.status == rrf.Status.ERR_UNSUPPORTED  # the forced launch cannot cover it
            continue
        parity.assert_fused_parity(gpu, parity.oracle_fused(c),
                                   f"R={R} {rows}x{cols} v{variant} C{cluster} T{threads} f{flags}")
        checked += 1
    assert checked >= 40
    assert rrf.rrf_device_error() == 0


# --------------------------------------------------------------- edge cases ---

@pytest.mark.parametrize("cols", [8, 16, 264, 2880, 7176, 8200, 16384, 131072, 262144])
def test_column_counts(rrf, cols):
    """Ragged rows (vector counts that are not a multiple of the block) and
    the hidden sizes the TensorRT-LLM padding discussion lists, up to the
    longest row the library accepts."""
    rows = 3 if cols >= 131072 else 5
    c = dev_case("decode", rows, cols=cols, R=3)
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), f"cols {cols}")
    assert np.array_equal(workloads.bits(rrf.rrf_sum(c.inputs)), parity.oracle_sum(c))


@pytest.mark.parametrize("R", [1, 2, 3, 5, 8, 9, 16])
def test_input_counts(rrf, R):
    c = dev_case("odd", 37, R=R)
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), f"R={R}")
    assert np.array_equal(workloads.bits(rrf.rrf_sum(c.inputs)), parity.oracle_sum(c))


def test_in_place_residual(rrf):
    c = dev_case("decode", 8)
    parity.assert_fused_parity(parity.gpu_fused(c, in_place=True), parity.oracle_fused(c),
                               "in place")


def test_empty_batch(rrf):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    q, s, r = rrf.rrf_sum_rmsnorm_fp8([x, x], g, 1e-6, 0.0, 1200.0, residual_in=x)
    assert q.shape == (0, 256) and s.shape == (0, 1) and r.shape == (0, 256)
    assert rrf.rrf_sum([x]).shape == (0, 256)


def test_zero_rows_and_signed_zeros(rrf):
    """All-zero rows: scale = 1e-12 / 448 and codes +-0 following the sign of
    gamma + weight_offset; -0 inputs sum to -0."""
    c = dev_case("tiny")
    c.inputs = [torch.zeros_like(x) for x in c.inputs]
    c.gamma = torch.tensor(np.where(np.arange(c.cols) % 3 == 0, -1.0, 1.0),
                           dtype=torch.bfloat16, device="cuda")
    gpu = parity.gpu_fused(c)
    ref = parity.oracle_fused(c)
    assert np.array_equal(gpu["q"], ref["q"])
    assert (ref["q"][:, 0] == 0x80).all() and (ref["q"][:, 1] == 0x00).all()
    assert np.array_equal(gpu["scales"], ref["scales"])
    negz = [torch.full_like(x, -0.0) for x in c.inputs]
    assert (workloads.bits(rrf.rrf_sum(negz)) == 0x8000).all()


def test_saturation_and_no_clamp(rrf):
    """scale_ub = +inf (no clamp) and a tiny scale_ub (every row clamped, most
    codes saturated)."""
    for ub in (float("inf"), 1e-3):
        c = dev_case("odd", 37)
        c.scale_ub = ub
        ref = parity.oracle_fused(c)
        parity.assert_fused_parity(parity.gpu_fused(c), ref, f"ub={ub}")
    assert ((ref["q"] & 0x7F) == 0x7E).mean() > 0.5


# ------------------------------------------------ determinism and graphs ---

def test_repeat_and_graph_replay_bitwise(rrf):
    """Repeated calls and three replays of a captured CUDA graph give the
    same bits as the first eager call."""
    c = dev_case("decode", 64)
    first = parity.gpu_fused(c)
    for _ in range(2):
        again = parity.gpu_fused(c)
        for k in first:
            assert np.array_equal(first[k], again[k]), k
    res_out = torch.empty_like(c.residual)
    q = torch.empty(c.inputs[0].shape, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty((c.rows, 1), dtype=torch.float32, device="cuda")
    call = lambda: rrf.rrf_sum_rmsnorm_fp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                           c.scale_ub, residual_in=c.residual,
                                           residual_out=res_out, q_out=q, scales_out=s)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        call()  # warm-up outside capture (sets the non-portable cluster attribute)
    torch.cuda.current_stream().wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for _ in range(3):
        q.zero_()
        s.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(q.view(torch.uint8).cpu().numpy(), first["q"])
        assert np.array_equal(s.reshape(-1).cpu().numpy(), first["scales"])
        assert np.array_equal(workloads.bits(res_out), first["res_out"])


# -------------------------------------------------- errors and guard bands ---

def test_validation_on_device_tensors(rrf):
    c = dev_case("tiny")
    x = c.inputs
    with pytest.raises(ValueError):  # the binding checks shapes before marshalling
        rrf.rrf_sum([x[0], x[1][:, 8:]])
    flat = torch.empty(c.rows * c.cols + 8, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x[0])
    with pytest.raises(rrf.RrfError) as e:  # an input misaligned by one element
        rrf.rrf_sum_ptr([x[0].data_ptr(), flat.data_ptr() + 2], c.rows, c.cols,
                        out.data_ptr())
    assert e.value.status == rrf.Status.ERR_ALIGN
    with pytest.raises(rrf.RrfError) as e:  # output over an input
        rrf.rrf_sum_ptr([x[0].data_ptr(), x[1].data_ptr()], c.rows, c.cols, x[1].data_ptr())
    assert e.value.status == rrf.Status.ERR_ALIAS
    with pytest.raises(rrf.RrfError) as e:
        rrf.rrf_sum_rmsnorm_fp8(x, c.gamma, -1.0, 0.0, 1.0)
    assert e.value.status == rrf.Status.ERR_VALUE


def test_injected_launch_failure_reports_cuda_error(rrf):
    c = dev_case("tiny")
    rrf.rrf_debug_fail_next_launch(719)
    with pytest.raises(rrf.RrfError) as e:
        rrf.rrf_sum_rmsnorm_fp8(c.inputs, c.gamma, c.eps, c.weight_offset, c.scale_ub)
    assert e.value.status == rrf.Status.ERR_CUDA and e.value.cuda_error == 719
    assert rrf.rrf_last_cuda_error() == 719
    # the hook is one-shot and nothing was launched: the next call works
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), "after")


def test_guard_bands_untouched(rrf):
    """Outputs sit between canary bytes; a call writes nothing outside them."""
    c = dev_case("odd", 37)
    n = c.rows * c.cols
    pad = 4096
    qbuf = torch.full((n + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((c.rows + 2 * pad // 4,), 7.0, dtype=torch.float32, device="cuda")
    rbuf = torch.full((n + 2 * pad,), 3.0, dtype=torch.bfloat16, device="cuda")
    q = qbuf[pad:pad + n].view(torch.float8_e4m3fn).view(c.rows, c.cols)
    s = sbuf[pad // 4:pad // 4 + c.rows].view(c.rows, 1)
    r = rbuf[pad:pad + n].view(c.rows, c.cols)
    rrf.rrf_sum_rmsnorm_fp8(c.inputs, c.gamma, c.eps, c.weight_offset, c.scale_ub,
                            residual_in=c.residual, residual_out=r, q_out=q, scales_out=s)
    torch.cuda.synchronize()
    assert (qbuf[:pad] == 0xA5).all() and (qbuf[pad + n:] == 0xA5).all()
    assert (sbuf[:pad // 4] == 7.0).all() and (sbuf[pad // 4 + c.rows:] == 7.0).all()
    assert (rbuf[:pad] == 3.0).all() and (rbuf[pad + n:] == 3.0).all()
    got = {"q": q.view(torch.uint8).cpu().numpy(), "scales": s.reshape(-1).cpu().numpy(),
           "res_out": workloads.bits(r)}
    parity.assert_fused_parity(got, parity.oracle_fused(c), "guarded")
