"""Property tests of the host-side validation (no GPU): buffers are placed at
random 16-byte-aligned fake addresses in a small address space, so that they
overlap often, and the library's verdict is compared with the rule the
header states for each call -- an output may overlap no input and no other
output, except the residual written in place (residual_out == residual_in).
Validation never dereferences the pointers."""
import os

import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

BASE = 1 << 24   # fake addresses: BASE + 16 * slot
SLOTS = 64       # a small space, so that overlaps are common

# a fixed seed, so that every run checks the same layouts (RRF_PROPERTY_EXAMPLES
# raises the count for a longer search)
SETTINGS = settings(max_examples=int(os.environ.get("RRF_PROPERTY_EXAMPLES", "400")),
                    deadline=None, derandomize=True, database=None,
                    suppress_health_check=[HealthCheck.function_scoped_fixture])


@pytest.fixture(scope="module")
def rrf():
    from reduce_rmsnorm_fp8_b200 import build
    build.build()
    import reduce_rmsnorm_fp8_b200 as m
    return m


def overlaps(a, b):
    """Half-open byte ranges (start, size) intersect."""
    return a[0] < b[0] + b[1] and b[0] < a[0] + a[1]


def any_alias(writes, reads):
    for i, w in enumerate(writes):
        if any(overlaps(w, r) for r in reads):
            return True
        if any(overlaps(w, w2) for w2 in writes[i + 1:]):
            return True
    return False


addr = st.integers(0, SLOTS).map(lambda k: BASE + 16 * k)


@SETTINGS
@given(R=st.integers(1, 4), rows=st.integers(1, 6), cols=st.sampled_from([8, 16, 24, 64]),
       residual=st.sampled_from(["none", "separate", "in_place"]),
       slots=st.lists(addr, min_size=10, max_size=10))
def test_fused_call_alias_rule(rrf, R, rows, cols, residual, slots):
    inputs = slots[:R]
    gamma, q, scales, res_in, res_out = slots[4:9]
    if residual == "none":
        res_in = res_out = 0
    elif residual == "in_place":
        res_out = res_in
    bf16 = rows * cols * 2
    reads = [(p, bf16) for p in inputs] + [(gamma, cols * 2)]
    if residual != "none" and res_in != res_out:  # equal pointers are in place
        reads.append((res_in, bf16))
    writes = [(q, rows * cols), (scales, rows * 4)]
    if residual != "none":
        writes.append((res_out, bf16))
    want = rrf.Status.ERR_ALIAS if any_alias(writes, reads) else rrf.Status.OK
    got = rrf.rrf_check_fused_args(inputs, rows, cols, res_in, res_out, gamma, 1e-5, 0.0,
                                   1200.0, q, scales)
    assert got == want, (got, want)


@SETTINGS
@given(R=st.integers(1, 4), rows=st.integers(1, 6), cols=st.sampled_from([8, 16, 64]),
       slots=st.lists(addr, min_size=5, max_size=5))
def test_sum_call_alias_rule(rrf, R, rows, cols, slots):
    inputs, out = slots[:R], slots[4]
    bf16 = rows * cols * 2
    want = (rrf.Status.ERR_ALIAS if any(overlaps((out, bf16), (p, bf16)) for p in inputs)
            else rrf.Status.OK)
    assert rrf.rrf_check_sum_args(inputs, rows, cols, out) == want


@SETTINGS
@given(M=st.integers(1, 8), N=st.sampled_from([16, 32, 48]), K=st.sampled_from([16, 32, 64]),
       bias=st.booleans(), slots=st.lists(addr, min_size=6, max_size=6))
def test_scaled_mm_alias_rule(rrf, M, N, K, bias, slots):
    a, a_scale, b, b_scale, bias_p, out = slots
    if not bias:
        bias_p = 0
    reads = [(a, M * K), (a_scale, M * 4), (b, N * K), (b_scale, N * 4)]
    if bias:
        reads.append((bias_p, N * 2))
    want = rrf.Status.ERR_ALIAS if any_alias([(out, M * N * 2)], reads) else rrf.Status.OK
    got = rrf.rrf_check_scaled_mm_args(a, a_scale, b, b_scale, bias_p, out, M, N, K)
    assert got == want, (got, want)


@SETTINGS
@given(rows=st.integers(1, 6), cols=st.sampled_from([8, 64]),
       which=st.sampled_from(["input", "gamma", "q", "residual_in", "residual_out"]),
       offset=st.sampled_from([1, 2, 4, 8]))
def test_fused_call_alignment_rule(rrf, rows, cols, which, offset):
    """A data pointer off its 16-byte alignment is ERR_ALIGN, whatever else
    holds (the buffers here are far apart); the scales need 4 bytes."""
    step = 1 << 20
    p = {"input": BASE, "gamma": BASE + step, "q": BASE + 2 * step,
         "residual_in": BASE + 3 * step, "residual_out": BASE + 4 * step}
    p[which] += offset
    got = rrf.rrf_check_fused_args([p["input"]], rows, cols, p["residual_in"],
                                   p["residual_out"], p["gamma"], 1e-5, 0.0, 1200.0, p["q"],
                                   BASE + 5 * step)
    assert got == rrf.Status.ERR_ALIGN
    ok = rrf.rrf_check_fused_args([BASE], rows, cols, BASE + 3 * step, BASE + 4 * step,
                                  BASE + step, 1e-5, 0.0, 1200.0, BASE + 2 * step,
                                  BASE + 5 * step + 4 * (offset % 2 == 0))
    assert ok == rrf.Status.OK


@SETTINGS
@given(world=st.integers(1, 4), rows=st.integers(1, 4), cols=st.sampled_from([8, 16, 64]),
       residual=st.sampled_from(["none", "separate", "in_place", "mixed"]),
       near_signal=st.booleans(), slots=st.lists(addr, min_size=22, max_size=22))
def test_allreduce_alias_rule(rrf, world, rows, cols, residual, near_signal, slots):
    """The multi-GPU call: no write (codes, scales, signal pads, residual
    outputs) may overlap a read (inputs, gamma, residual inputs not written
    in place) or another write, and a residual written in place serves only
    its own rank."""
    sig_words = rrf.RRF_AR_SIGNAL_WORDS
    gamma = slots[0]
    inputs = slots[1:1 + world]
    q = slots[5:5 + world]
    scales = slots[9:9 + world]
    res_in = slots[13:13 + world]
    res_out = slots[17:17 + world]
    # signal pads far apart (their 4 * RRF_AR_SIGNAL_WORDS bytes would cover
    # the small space), or one of them inside it
    signals = [BASE + (1 << 22) * (j + 1) for j in range(world)]
    if near_signal:
        signals[0] = slots[21]
    if residual == "none":
        res_in = res_out = None
    elif residual == "in_place":
        res_out = list(res_in)
    elif residual == "mixed":
        res_out = [res_in[j] if j % 2 == 0 else res_out[j] for j in range(world)]
    bf16 = rows * cols * 2
    reads = [(gamma, cols * 2)] + [(p, bf16) for p in inputs]
    writes = []
    for j in range(world):
        if res_in is not None and res_in[j] != res_out[j]:
            reads.append((res_in[j], bf16))
        writes += [(q[j], rows * cols), (scales[j], rows * 4), (signals[j], sig_words * 4)]
        if res_in is not None:
            writes.append((res_out[j], bf16))
    alias = any_alias(writes, reads)
    if res_in is not None and not alias:
        alias = any(i != j and overlaps((res_out[j], bf16), (res_in[i], bf16))
                    for j in range(world) for i in range(world))
    want = rrf.Status.ERR_ALIAS if alias else rrf.Status.OK
    got = rrf.rrf_check_allreduce_args(inputs, res_in, res_out, q, scales, signals, 0, 1,
                                       rows, cols, gamma, 1e-5, 0.0, 1200.0,
                                       rrf.RRF_AR_AUTO, world=world)
    assert got == want, (got, want)
