"""The bounds-checking build (librrf_debug.so, compiled with RRF_DEBUG).

Every kernel of that build checks the index of each global and shared
access it is about to make; a check that fails sets RRF_DEVICE_ERROR_BOUNDS
in the device error word and skips the access (no trap, no assert).  It
stands in for a memory checker.  On the CPU: the build compiles and exports
every function of the header.  On the GPU: small cases of every kernel run
through it, match the oracle, and leave the error word clear."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    return set(re.findall(r"\bT (rrf_[a-z0-9_]+)$", out, flags=re.M))


def test_debug_build_exports_what_the_normal_build_does():
    from reduce_rmsnorm_fp8_b200 import build
    normal = build.build()
    debug = build.build(debug=True)
    assert os.path.basename(debug) == "librrf_debug.so"
    assert exported(debug) == exported(normal)


_GPU_SCRIPT = r'''
import sys
sys.path[:0] = [ROOT, HERE]
import numpy as np, torch
import reduce_rmsnorm_fp8_b200 as rrf
from reduce_rmsnorm_fp8_b200 import allreduce
import parity, workloads, oracle
assert rrf.LIB_PATH.endswith("librrf_debug.so"), rrf.LIB_PATH
rrf.rrf_device_error(clear=True)
dev = lambda name, rows, **kw: parity.to_device(workloads.make_case(name, rows, **kw))
for name, rows in (("decode", 1), ("decode", 64), ("odd", 37), ("tiny", None), ("sweep", 256)):
    c = dev(name, rows)
    parity.assert_fused_parity(parity.gpu_fused(c), parity.oracle_fused(c), f"{name} {rows}")
c = dev("odd", 37)
for C in (3, 7, 16):
    for flags in (0, rrf.RRF_FLAG_BARRIER_EXCHANGE):
        parity.assert_fused_parity(parity.gpu_fused(c, variant=2, cluster_size=C, flags=flags),
                                   parity.oracle_fused(c), f"C={C} f={flags}")
c = dev("decode", 8)
q, s, _ = rrf.rrf_sum_rmsnorm_mxfp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                    residual_in=c.residual.clone())
qb, sb, _ = rrf.rrf_sum_rmsnorm_mxfp8(c.inputs, c.gamma, c.eps, c.weight_offset,
                                      residual_in=c.residual.clone(), blocked=True)
torch.cuda.synchronize()
got = {"q": q.view(torch.uint8).cpu().numpy(), "scales_mx": s.cpu().numpy()}
ref = parity.oracle_mx(c)
parity.assert_mx_parity(got, {k: v for k, v in ref.items() if k != "res_out"}, "mx")
from reduce_rmsnorm_fp8_b200 import sharded  # noqa: F401 (import check)
c = dev("decode", 32, cols=2048)
st = torch.empty((32, 2), dtype=torch.float32, device="cuda")
h = torch.empty_like(c.inputs[0])
rrf.rrf_sum_rmsnorm_fp8_pre(c.inputs, c.gamma, c.weight_offset, residual_in=c.residual.clone(),
                            residual_out=h, stats_out=st)
q, sc = rrf.rrf_rmsnorm_fp8_post(h, c.gamma, st.view(1, 32, 2), c.cols, c.eps, c.weight_offset,
                                 c.scale_ub)
torch.cuda.synchronize()
parity.assert_fused_parity({"q": q.view(torch.uint8).cpu().numpy(),
                            "scales": sc.reshape(-1).cpu().numpy()},
                           {k: v for k, v in parity.oracle_fused(c).items() if k != "res_out"},
                           "pre + post, one shard")
for world, mode in ((4, 1), (4, 2), (8, 2)):
    c = dev("decode", 8, R=world)
    g = allreduce.LocalGroup(world)
    qs, ss, rs = g(c.inputs, c.gamma, c.eps, c.weight_offset, c.scale_ub,
                   residual_in=[c.residual.clone() for _ in range(world)], mode=mode)
    torch.cuda.synchronize()
    parity.assert_fused_parity({"q": qs[0].view(torch.uint8).cpu().numpy(),
                                "scales": ss[0].reshape(-1).cpu().numpy(),
                                "res_out": workloads.bits(rs[0])},
                               parity.oracle_fused(c), f"allreduce w{world} m{mode}",
                               cap_at_ties=True)
import test_gpu_gemm as tg
import test_gpu_mx as tm
for M, N, K in ((9, 512, 640), (200, 272, 384), (8, 16384, 1024), (64, 16384, 1024)):
    gc = workloads.make_gemm_case(M, N, K, sub=1, device="cuda")
    out = rrf.rrf_scaled_mm_fp8(gc.a, gc.a_scale, gc.b, gc.b_scale, gc.bias)
    torch.cuda.synchronize()
    tg.check(gc, out, rows=sorted({0, M // 2, M - 1}), label=f"gemm {M}x{N}x{K}")
for M, N, K in ((8, 384, 512), (130, 400, 1024), (16, 16384, 1024)):
    gc, sa, sbb = tm.mx_operands(M, N, K, 2)
    out = rrf.rrf_scaled_mm_mxfp8(gc.a, rrf.mx_blocked(torch.from_numpy(sa).cuda()), gc.b,
                                  rrf.mx_blocked(torch.from_numpy(sbb).cuda()), gc.bias)
    torch.cuda.synchronize()
    tm.check_mx_gemm(gc, sa, sbb, out, rows=sorted({0, M // 2, M - 1}), label=f"mx {M}x{N}x{K}")
c = dev("decode", 64)
s = rrf.rrf_sum(c.inputs)
torch.cuda.synchronize()
assert np.array_equal(workloads.bits(s), parity.oracle_sum(c))
flags = rrf.rrf_device_error()
assert flags == 0, f"device error word {flags:#x}"
print("debug build clean")
'''


@pytest.mark.gpu
def test_checked_build_runs_every_kernel_clean():
    from reduce_rmsnorm_fp8_b200 import build
    build.build(debug=True)
    script = f"ROOT = {ROOT!r}\nHERE = {HERE!r}\n" + _GPU_SCRIPT
    env = dict(os.environ, RRF_DEBUG_LIBRARY="1")
    p = subprocess.run([sys.executable, "-c", script], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=900)
    assert p.returncode == 0, (p.stdout + p.stderr)[-4000:]
    assert "debug build clean" in p.stdout
