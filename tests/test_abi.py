"""The C ABI without a GPU: the library loads, exports every function the
header declares, validates arguments on the host and plans launches.  No
compute entry point is called here."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rrf.h")


@pytest.fixture(scope="module")
def rrf():
    from reduce_rmsnorm_fp8_b200 import build
    build.build()
    import reduce_rmsnorm_fp8_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rrf_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("rrf_sum", "rrf_sum_rmsnorm_fp8", "rrf_sum_rmsnorm_fp8_ex",
                 "rrf_status_string", "rrf_last_cuda_error"):
        assert want in names


def test_library_exports_every_declared_function(rrf):
    out = subprocess.run(["nm", "-D", "--defined-only", rrf.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (rrf_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for name in declared_functions():
        getattr(rrf.lib, name)  # resolvable through ctypes


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "rrf.h"\nint main(void) { return RRF_OK; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(tmp_path / "t")], check=True)


def test_constants_match_header(rrf):
    text = open(HEADER).read()
    assert rrf.RRF_MAX_INPUTS == int(re.search(r"#define RRF_MAX_INPUTS (\d+)", text).group(1))
    expr = re.search(r"#define RRF_MAX_COLS \(([^)]*)\)", text).group(1)
    assert rrf.RRF_MAX_COLS == eval(expr)
    for name in ("RRF_VARIANT_AUTO", "RRF_VARIANT_ROW", "RRF_VARIANT_CLUSTER",
                 "RRF_FLAG_NO_PDL", "RRF_FLAG_BARRIER_EXCHANGE",
                 "RRF_FLAG_DEBUG_STARVE_EXCHANGE", "RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT",
                 "RRF_DEVICE_ERROR_PEER_TIMEOUT", "RRF_DEVICE_ERROR_GEMM_TIMEOUT",
                 "RRF_AR_MAX_WORLD", "RRF_AR_MAX_BLOCKS",
                 "RRF_AR_AUTO", "RRF_AR_ONE_SHOT", "RRF_AR_TWO_SHOT", "RRF_MAX_SHARDS"):
        assert getattr(rrf, name) == int(
            re.search(rf"#define {name} (0x[0-9a-fA-F]+|\d+)u?", text).group(1), 0)
    expr = re.search(r"#define RRF_AR_SIGNAL_WORDS (\(.*\))\s*$", text, flags=re.M).group(1)
    assert rrf.RRF_AR_SIGNAL_WORDS == eval(expr, {"RRF_AR_MAX_WORLD": rrf.RRF_AR_MAX_WORLD,
                                                  "RRF_AR_MAX_BLOCKS": rrf.RRF_AR_MAX_BLOCKS})
    from reduce_rmsnorm_fp8_b200 import allreduce
    assert (allreduce.RRF_AR_SIGNAL_WORDS, allreduce.RRF_AR_MAX_WORLD, allreduce.RRF_AR_AUTO) == \
        (rrf.RRF_AR_SIGNAL_WORDS, rrf.RRF_AR_MAX_WORLD, rrf.RRF_AR_AUTO)
    for st in rrf.Status:
        assert re.search(rf"RRF_{st.name} = {int(st)}\b", text), st


def test_status_strings_and_version(rrf):
    for st in rrf.Status:
        assert rrf.rrf_status_string(st)
    assert rrf.rrf_status_string(99) == "unknown status"
    assert re.fullmatch(r"\d+\.\d+\.\d+", rrf.rrf_version())
    assert rrf.rrf_last_cuda_error() == 0


# ----------------------------------------------------------- validation ---

A = 1 << 20  # fake, 16-byte aligned addresses: validation never dereferences them


def fused_ok_args(R=4, rows=8, cols=64):
    n = rows * cols
    ins = [A * (r + 1) for r in range(R)]
    base = A * 64
    return dict(input_ptrs=ins, rows=rows, cols=cols, residual_in=base,
                residual_out=base + 4 * A, gamma=base + 8 * A, eps=1e-5, weight_offset=0.0,
                scale_ub=1200.0, q_out=base + 12 * A, scales_out=base + 16 * A)


def check(rrf, **kw):
    return rrf.Status(rrf.rrf_check_fused_args(**kw))


def test_fused_validation_accepts_valid(rrf):
    assert check(rrf, **fused_ok_args()) == rrf.Status.OK
    kw = fused_ok_args()
    kw["residual_out"] = kw["residual_in"]  # in-place residual
    assert check(rrf, **kw) == rrf.Status.OK
    kw = fused_ok_args()
    kw["residual_in"] = kw["residual_out"] = 0  # no residual
    assert check(rrf, **kw) == rrf.Status.OK
    kw = fused_ok_args()
    kw["scale_ub"] = float("inf")
    assert check(rrf, **kw) == rrf.Status.OK


@pytest.mark.parametrize("change,status", [
    (dict(input_ptrs=[]), "ERR_RANKS"),
    (dict(input_ptrs=[A * (r + 1) for r in range(17)]), "ERR_RANKS"),
    (dict(rows=-1), "ERR_SHAPE"),
    (dict(cols=0), "ERR_SHAPE"),
    (dict(cols=60), "ERR_SHAPE"),
    (dict(cols=16 * 256 * 8 * 8 + 8), "ERR_SHAPE"),
    (dict(rows=2 ** 40), "ERR_SHAPE"),
    (dict(eps=-1e-6), "ERR_VALUE"),
    (dict(eps=float("nan")), "ERR_VALUE"),
    (dict(eps=float("inf")), "ERR_VALUE"),
    (dict(scale_ub=0.0), "ERR_VALUE"),
    (dict(scale_ub=-1.0), "ERR_VALUE"),
    (dict(scale_ub=float("nan")), "ERR_VALUE"),
    (dict(weight_offset=float("inf")), "ERR_VALUE"),
    (dict(gamma=0), "ERR_NULL"),
    (dict(q_out=0), "ERR_NULL"),
    (dict(scales_out=0), "ERR_NULL"),
    (dict(residual_out=0), "ERR_NULL"),
    (dict(residual_in=0), "ERR_NULL"),
    (dict(input_ptrs=[A, 0]), "ERR_NULL"),
    (dict(input_ptrs=[A, A * 2 + 8]), "ERR_ALIGN"),
    (dict(gamma=A * 72 + 2), "ERR_ALIGN"),
    (dict(q_out=A * 76 + 8), "ERR_ALIGN"),
    (dict(scales_out=A * 80 + 2), "ERR_ALIGN"),
    (dict(residual_in=A * 64 + 16 + 4), "ERR_ALIGN"),
    (dict(q_out=A * 1 + 16), "ERR_ALIAS"),           # inside input 0
    (dict(scales_out=A * 72), "ERR_ALIAS"),          # on gamma
    (dict(residual_out=A * 64 + 16), "ERR_ALIAS"),   # overlaps residual_in, not equal
    (dict(q_out=A * 68 + 256), "ERR_ALIAS"),         # inside residual_out
    (dict(scales_out=A * 76 + 100), "ERR_ALIAS"),    # inside q_out
])
def test_fused_validation_rejects(rrf, change, status):
    kw = fused_ok_args()
    kw.update(change)
    assert check(rrf, **kw) == rrf.Status[status]


def test_empty_rows_is_valid_without_pointers(rrf):
    st = rrf.rrf_check_fused_args([0, 0], 0, 64, 0, 0, 0, 1e-6, 0.0, 1.0, 0, 0)
    assert st == rrf.Status.OK
    assert rrf.rrf_check_sum_args([0], 0, 64, 0) == rrf.Status.OK
    # the scalars and the shape are still checked
    assert rrf.rrf_check_fused_args([0], 0, 64, 0, 0, 0, -1.0, 0.0, 1.0, 0, 0) == \
        rrf.Status.ERR_VALUE
    assert rrf.rrf_check_sum_args([0], 0, 63, 0) == rrf.Status.ERR_SHAPE


def test_sum_validation(rrf):
    ins = [A, 2 * A, 3 * A]
    assert rrf.rrf_check_sum_args(ins, 16, 64, 8 * A) == rrf.Status.OK
    assert rrf.rrf_check_sum_args(ins, 16, 64, 0) == rrf.Status.ERR_NULL
    assert rrf.rrf_check_sum_args(ins, 16, 64, 8 * A + 4) == rrf.Status.ERR_ALIGN
    assert rrf.rrf_check_sum_args(ins, 16, 64, 2 * A + 64) == rrf.Status.ERR_ALIAS
    assert rrf.rrf_check_sum_args(ins, 16, 12, 8 * A) == rrf.Status.ERR_SHAPE
    assert rrf.rrf_check_sum_args([A] * 17, 16, 64, 8 * A) == rrf.Status.ERR_RANKS
    # sum-only has no column limit beyond memory
    assert rrf.rrf_check_sum_args(ins, 1, 1 << 22, 1 << 40) == rrf.Status.OK


# -------------------------------------------------------------- planner ---

TABLE = os.path.join(ROOT, "reduce_rmsnorm_fp8_b200", "csrc", "rrf_plan_table.inc")


def plan_table():
    """The entries of the launch table compiled into the library:
    (input bound, residual, cols, rows, cluster, prefetch, us)."""
    text = re.sub(r"//.*", "", open(TABLE).read())
    return [tuple(float(v) if "." in v else int(v) for v in m.replace("f", "").split(","))
            for m in re.findall(r"RRF_PLAN\(([^)]*)\)", text)]


def test_plan_table_is_measured_and_covers_the_grid():
    """The table holds the sweep's grid: every input bound with and without
    a residual, the workloads' row lengths and batch sizes."""
    entries = plan_table()
    assert entries, "no launch sweep recorded in rrf_plan_table.inc"
    keys = {(e[0], e[1], e[2], e[3]) for e in entries}
    assert len(keys) == len(entries)  # one entry per shape
    for rb in (2, 4, 8, 16):
        for res in (0, 1):
            assert any(k[0] == rb and k[1] == res for k in keys), (rb, res)
    for rb, res, cols, rows in ((8, 1, 7168, 1), (8, 1, 7168, 8), (8, 1, 7168, 32),
                                (8, 1, 7168, 64), (4, 1, 7168, 37), (4, 1, 7168, 64),
                                (2, 0, 1024, 4), (8, 1, 8192, 8192)):
        assert (rb, res, cols, rows) in keys, (rb, res, cols, rows)
    for e in entries:
        assert 1 <= e[4] <= 16 and e[5] in (0, 1) and e[6] > 0


def test_plan_follows_the_table(rrf):
    """For every shape of the table the planner takes the launch measured
    fastest there (cluster size and L2 prefetch)."""
    for rb, res, cols, rows, cluster, prefetch, _ in plan_table():
        c, t, v, p = rrf.rrf_plan_fused_ex(rb, rows, cols, 148, residual=bool(res))
        assert (c, p) == (cluster, prefetch), (rb, res, cols, rows)
        assert c * t * v * 8 >= cols


def test_plan_takes_the_nearest_entry(rrf):
    """Shapes between the table's: the entry of the same input bound and
    residual flag nearest in log2(cols) (weighted 4x) + log2(rows)."""
    import math
    entries = plan_table()
    for R, rows, cols, res in ((3, 5, 7168, True), (6, 40, 6144, False), (12, 300, 12288, True),
                               (8, 100, 7168, True), (1, 3000, 1536, False)):
        rb = 2 if R <= 2 else 4 if R <= 4 else 8 if R <= 8 else 16
        cands = [e for e in entries if e[0] == rb and e[1] == int(res)]
        best = min(cands, key=lambda e: 4 * abs(math.log2(cols / e[2])) +
                   abs(math.log2(rows / e[3])))
        c, t, v, p = rrf.rrf_plan_fused_ex(R, rows, cols, 148, residual=res)
        want = best[4]
        while want > 1 and cols // 8 // want < 32:
            want -= 1
        assert (c, p) == (want, best[5]), (R, rows, cols, res, c, best)


def test_plan_covers_every_row(rrf):
    for R in (1, 3, 8, 16):
        for cols in (8, 256, 2880, 7168, 7176, 8192, 8200, 16384, 131072, 262144):
            for rows in (1, 37, 4096):
                c, t, v = rrf.rrf_plan_fused(R, rows, cols, 148)
                assert 1 <= c <= 16 and 32 <= t <= 1024 and t % 32 == 0
                assert v in (1, 2, 4, 8)
                assert c * t * v * 8 >= cols, (R, rows, cols)


def test_plan_rejects(rrf):
    with pytest.raises(rrf.RrfError) as e:
        rrf.rrf_plan_fused(4, 1, 16 * 256 * 8 * 8 + 8, 148)
    assert e.value.status == rrf.Status.ERR_SHAPE
    with pytest.raises(rrf.RrfError):
        rrf.rrf_plan_fused(0, 1, 64, 148)


def test_use_fails_loudly_without_library(tmp_path):
    """Without librrf.so the first use of the package raises ImportError:
    there is no fallback.  (The bare import succeeds so that the build step
    can run from a fresh checkout.)"""
    import shutil
    pkg = tmp_path / "reduce_rmsnorm_fp8_b200"
    shutil.copytree(os.path.join(ROOT, "reduce_rmsnorm_fp8_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "_build", "__pycache__"))
    code = ("import reduce_rmsnorm_fp8_b200 as r, reduce_rmsnorm_fp8_b200.build as b\n"
            "assert b.LIB.endswith('librrf.so')\n"
            "r.rrf_sum\n")
    res = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True,
                         text=True)
    assert res.returncode != 0 and "librrf.so is missing" in res.stderr
    assert "ImportError" in res.stderr


# ------------------------------------------------------------ sharded form ---

def test_pre_validation(rrf):
    ins = [A, 2 * A]
    ok = dict(input_ptrs=ins, rows=8, cols=64, residual_in=0, residual_out=0, h_out=8 * A,
              gamma=9 * A, weight_offset=0.0, stats_out=10 * A)
    assert rrf.rrf_check_pre_args(**ok) == rrf.Status.OK
    res = dict(ok, residual_in=11 * A, residual_out=12 * A, h_out=0)
    assert rrf.rrf_check_pre_args(**res) == rrf.Status.OK
    for change, status in [
            (dict(h_out=0), "ERR_NULL"),                               # nowhere to put h
            (dict(res, h_out=8 * A), "ERR_NULL"),                      # h twice
            (dict(stats_out=0), "ERR_NULL"),
            (dict(stats_out=10 * A + 4), "ERR_ALIGN"),
            (dict(h_out=8 * A + 8), "ERR_ALIGN"),
            (dict(h_out=A + 64), "ERR_ALIAS"),                        # over an input
            (dict(stats_out=8 * A + 16), "ERR_ALIAS"),                # over h
            (dict(cols=12), "ERR_SHAPE"),
            (dict(weight_offset=float("nan")), "ERR_VALUE")]:
        kw = dict(ok)
        kw.update(change)
        assert rrf.rrf_check_pre_args(**kw) == rrf.Status[status], change


def test_post_validation(rrf):
    ok = dict(h=A, rows=8, cols=64, stats=2 * A, shards=4, total_cols=256, gamma=3 * A,
              eps=1e-5, weight_offset=0.0, scale_ub=1200.0, q_out=4 * A, scales_out=5 * A)
    assert rrf.rrf_check_post_args(**ok) == rrf.Status.OK
    assert rrf.rrf_check_post_args(**dict(ok, scales_out=0)) == rrf.Status.OK
    for change, status in [
            (dict(shards=0), "ERR_SHAPE"), (dict(shards=65), "ERR_SHAPE"),
            (dict(total_cols=56), "ERR_SHAPE"), (dict(cols=60), "ERR_SHAPE"),
            (dict(h=0), "ERR_NULL"), (dict(stats=0), "ERR_NULL"), (dict(q_out=0), "ERR_NULL"),
            (dict(stats=2 * A + 4), "ERR_ALIGN"), (dict(q_out=4 * A + 8), "ERR_ALIGN"),
            (dict(q_out=A + 16), "ERR_ALIAS"), (dict(scales_out=2 * A + 8), "ERR_ALIAS"),
            (dict(eps=-1.0), "ERR_VALUE"), (dict(scale_ub=0.0), "ERR_VALUE")]:
        kw = dict(ok)
        kw.update(change)
        assert rrf.rrf_check_post_args(**kw) == rrf.Status[status], change


def _ar_ok(world=4, residual=True):
    """Valid fake arguments of the multi-GPU call: rank j's buffers at
    distinct aligned addresses (rows 8, cols 64)."""
    at = lambda k: [(k * 16 + j) * A for j in range(world)]
    return dict(inputs=at(1), residual_in=at(2) if residual else None,
                residual_out=at(3) if residual else None, q_out=at(4), scales_out=at(5),
                signals=at(6), rank=0, local_ranks=1, rows=8, cols=64, gamma=A // 2, eps=1e-5,
                weight_offset=0.0, scale_ub=1200.0, mode=0)


def test_allreduce_validation_accepts_valid(rrf):
    for world in (1, 2, 8):
        for res in (True, False):
            assert rrf.rrf_check_allreduce_args(**_ar_ok(world, res)) == rrf.Status.OK
    ok = _ar_ok()
    assert rrf.rrf_check_allreduce_args(**dict(ok, local_ranks=4)) == rrf.Status.OK
    assert rrf.rrf_check_allreduce_args(**dict(ok, rank=3)) == rrf.Status.OK
    in_place = dict(ok, residual_out=ok["residual_in"])
    assert rrf.rrf_check_allreduce_args(**in_place) == rrf.Status.OK
    # rows == 0 is a no-op that looks at no pointer
    empty = {k: (None if isinstance(v, list) else v) for k, v in ok.items()}
    assert rrf.rrf_check_allreduce_args(**dict(empty, rows=0, gamma=0), world=4) == \
        rrf.Status.OK


def _swap(lst, j, value):
    out = list(lst)
    out[j] = value
    return out


@pytest.mark.parametrize("change,status", [
    (lambda o: dict(o, rank=4), "ERR_RANKS"),
    (lambda o: dict(o, rank=-1), "ERR_RANKS"),
    (lambda o: dict(o, rank=1, local_ranks=4), "ERR_RANKS"),
    (lambda o: dict(o, local_ranks=2), "ERR_UNSUPPORTED"),
    (lambda o: dict(o, mode=3), "ERR_UNSUPPORTED"),
    (lambda o: dict(o, eps=-1.0), "ERR_VALUE"),
    (lambda o: dict(o, scale_ub=float("nan")), "ERR_VALUE"),
    (lambda o: dict(o, cols=60), "ERR_SHAPE"),
    (lambda o: dict(o, cols=8 * 8 * 512 * 4 + 8), "ERR_SHAPE"),
    (lambda o: dict(o, rows=-1), "ERR_SHAPE"),
    (lambda o: dict(o, gamma=0), "ERR_NULL"),
    (lambda o: dict(o, residual_out=None), "ERR_NULL"),
    (lambda o: dict(o, q_out=_swap(o["q_out"], 2, 0)), "ERR_NULL"),
    (lambda o: dict(o, signals=_swap(o["signals"], 3, 0)), "ERR_NULL"),
    (lambda o: dict(o, inputs=_swap(o["inputs"], 1, o["inputs"][1] + 8)), "ERR_ALIGN"),
    (lambda o: dict(o, scales_out=_swap(o["scales_out"], 1, o["scales_out"][1] + 2)),
     "ERR_ALIGN"),
    (lambda o: dict(o, signals=_swap(o["signals"], 0, o["signals"][0] + 4)), "ERR_ALIGN"),
    # a rank's codes over another rank's partial
    (lambda o: dict(o, q_out=_swap(o["q_out"], 2, o["inputs"][0] + 64)), "ERR_ALIAS"),
    # two ranks' scales in one buffer
    (lambda o: dict(o, scales_out=_swap(o["scales_out"], 1, o["scales_out"][0])), "ERR_ALIAS"),
    # a pad over another rank's residual
    (lambda o: dict(o, signals=_swap(o["signals"], 1, o["residual_out"][2])), "ERR_ALIAS"),
    # an in-place residual that serves another rank's input
    (lambda o: dict(o, residual_out=_swap(o["residual_out"], 1, o["residual_in"][2])),
     "ERR_ALIAS"),
])
def test_allreduce_validation_rejects(rrf, change, status):
    assert rrf.rrf_check_allreduce_args(**change(_ar_ok())) == rrf.Status[status]


def test_allreduce_world_bounds(rrf):
    ok = _ar_ok(8)
    assert rrf.rrf_check_allreduce_args(**ok, world=9) == rrf.Status.ERR_RANKS
    assert rrf.rrf_check_allreduce_args(**ok, world=0) == rrf.Status.ERR_RANKS


@pytest.mark.parametrize("world,rows,cols,res,mode,want", [
    (8, 64, 7168, True, 0, (2, 8, 128, 1)),     # 8 rows per rank, rows split in clusters of 8
    (8, 1, 7168, True, 0, (1, 8, 128, 1)),      # fewer rows than ranks: one-shot
    (8, 8192, 8192, True, 0, (2, 1, 512, 2)),   # prefill: 1024 rows per rank, a block per row
    (4, 37, 7168, True, 0, (2, 8, 128, 1)),
    (8, 64, 7168, True, 1, (1, 8, 128, 1)),     # forced one-shot: 64 rows per rank
    (2, 4, 256, False, 0, (2, 1, 32, 1)),       # short rows: one block of one warp
    (8, 16, 131072, False, 2, (2, 8, 512, 4)),  # the widest row
])
def test_allreduce_plan(rrf, world, rows, cols, res, mode, want):
    assert rrf.rrf_plan_allreduce(world, rows, cols, 148, res, mode) == want


def test_allreduce_plan_rejects(rrf):
    with pytest.raises(rrf.RrfError) as e:
        rrf.rrf_plan_allreduce(9, 8, 64, 148)
    assert e.value.status == rrf.Status.ERR_RANKS
    with pytest.raises(rrf.RrfError) as e:
        rrf.rrf_plan_allreduce(8, 8, 131072 + 8, 148)
    assert e.value.status == rrf.Status.ERR_SHAPE


def test_two_shot_rows_tile_the_batch():
    from reduce_rmsnorm_fp8_b200 import allreduce
    for rows in (0, 1, 7, 37, 64, 8192):
        for world in (1, 2, 3, 8):
            spans = [allreduce.two_shot_rows(rows, world, k) for k in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert all(b - a <= -(-rows // world) for a, b in spans)


def test_peer_layout_is_aligned_and_disjoint():
    from reduce_rmsnorm_fp8_b200 import allreduce
    for res in (True, False):
        regions, total = allreduce.peer_layout(37, 7168, res)
        spans = sorted(regions.values())
        assert all(off % 256 == 0 for off, _ in spans)
        assert all(a[0] + a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        assert spans[-1][0] + spans[-1][1] <= total
        assert ("residual" in regions) == res


def test_scaled_mm_validation(rrf):
    ok = dict(a=A, a_scale=2 * A, b=3 * A, b_scale=4 * A, bias=5 * A, out=6 * A, M=64, N=256,
              K=512)
    assert rrf.rrf_check_scaled_mm_args(**ok) == rrf.Status.OK
    assert rrf.rrf_check_scaled_mm_args(**dict(ok, bias=0)) == rrf.Status.OK
    # M == 0 is a no-op that looks at no pointer
    assert rrf.rrf_check_scaled_mm_args(0, 0, 0, 0, 0, 0, 0, 256, 512) == rrf.Status.OK
    for change, status in [
            (dict(N=8), "ERR_SHAPE"), (dict(K=8), "ERR_SHAPE"), (dict(N=264), "ERR_SHAPE"),
            (dict(K=520), "ERR_SHAPE"), (dict(M=-1), "ERR_SHAPE"),
            (dict(M=65535 * 128 + 1), "ERR_SHAPE"),
            (dict(a=0), "ERR_NULL"), (dict(b_scale=0), "ERR_NULL"), (dict(out=0), "ERR_NULL"),
            (dict(a=A + 8), "ERR_ALIGN"), (dict(out=6 * A + 4), "ERR_ALIGN"),
            (dict(a_scale=2 * A + 2), "ERR_ALIGN"), (dict(bias=5 * A + 1), "ERR_ALIGN"),
            (dict(out=A + 16), "ERR_ALIAS"),                     # over a
            (dict(b_scale=6 * A + 1024), "ERR_ALIAS"),           # a scale inside out
            (dict(bias=6 * A + 64 * 256 * 2 - 2), "ERR_ALIAS")]:  # bias at out's end
        kw = dict(ok)
        kw.update(change)
        assert rrf.rrf_check_scaled_mm_args(**kw) == rrf.Status[status], change


def test_mxfp8_validation(rrf):
    ins = [A, 2 * A]
    ok = dict(input_ptrs=ins, rows=8, cols=64, residual_in=0, residual_out=0, gamma=3 * A,
              eps=1e-5, weight_offset=0.0, q_out=4 * A, scales_mx_out=5 * A + 1)
    assert rrf.rrf_check_mxfp8_args(**ok) == rrf.Status.OK  # scale codes are bytes
    for change, status in [
            (dict(cols=48), "ERR_SHAPE"),                    # not a multiple of 32
            (dict(scales_mx_out=0), "ERR_NULL"),
            (dict(q_out=4 * A + 8), "ERR_ALIGN"),
            (dict(scales_mx_out=A + 100), "ERR_ALIAS"),      # inside an input
            (dict(scales_mx_out=4 * A + 8 * 64 - 1), "ERR_ALIAS"),  # the codes' last byte
            (dict(eps=-1.0), "ERR_VALUE")]:
        kw = dict(ok)
        kw.update(change)
        assert rrf.rrf_check_mxfp8_args(**kw) == rrf.Status[status], change


def test_scaled_mm_mx_validation(rrf):
    ok = dict(a=A, sa=2 * A, b=3 * A, sb=4 * A, bias=5 * A, out=6 * A, M=64, N=256, K=512)
    assert rrf.rrf_check_scaled_mm_mx_args(**ok) == rrf.Status.OK
    assert rrf.rrf_check_scaled_mm_mx_args(0, 0, 0, 0, 0, 0, 0, 256, 512) == rrf.Status.OK
    for change, status in [
            (dict(K=384 + 64), "ERR_SHAPE"), (dict(K=0), "ERR_SHAPE"), (dict(N=264), "ERR_SHAPE"),
            (dict(sa=0), "ERR_NULL"), (dict(sb=4 * A + 8), "ERR_ALIGN"),
            (dict(sa=2 * A + 4), "ERR_ALIGN"),
            (dict(out=2 * A + 16), "ERR_ALIAS"),          # over sa's blocked bytes
            (dict(sb=6 * A + 64 * 256 * 2 - 16), "ERR_ALIAS")]:  # sb's start inside out
        kw = dict(ok)
        kw.update(change)
        assert rrf.rrf_check_scaled_mm_mx_args(**kw) == rrf.Status[status], change


@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 256), (128, 512), (200, 384), (300, 1024)])
def test_mx_blocked_layout_is_the_header_formula(rrf, rows, cols):
    """The host helper that puts a weight's MX scale codes in the blocked
    order, against the byte position include/rrf.h states, written out as a
    plain loop; the size against RRF_MX_BLOCKED_BYTES."""
    import numpy as np
    import torch
    rng = np.random.default_rng(rows * 7 + cols)
    nb = cols // 32
    codes = rng.integers(0, 256, (rows, nb)).astype(np.uint8)
    got = rrf.mx_blocked(torch.from_numpy(codes)).numpy()
    size = -(-rows // 128) * 128 * nb
    assert got.size == size == rrf.mx_blocked_bytes(rows, cols)
    want = np.zeros(size, dtype=np.uint8)
    for r in range(rows):
        for j in range(nb):
            pos = ((r // 128) * (cols // 128) + j // 4) * 512 + (r % 32) * 16 + \
                ((r // 32) % 4) * 4 + j % 4
            want[pos] = codes[r, j]
    assert np.array_equal(got, want)


def test_mx_blocked_rejects_partial_atoms(rrf):
    import torch
    with pytest.raises(ValueError):
        rrf.mx_blocked(torch.zeros((4, 6), dtype=torch.uint8))


@pytest.mark.parametrize("M,N,K,mx,want", [
    (8, 16384, 7168, False, ("swap", 8, 64, 8, 256, 148)),
    (16, 16384, 1024, False, ("swap", 16, 64, 4, 256, 148)),
    (32, 16384, 7168, False, ("swap", 32, 64, 4, 256, 148)),
    (64, 16384, 7168, False, ("tile", 64, 64, 4, 256, 148)),
    (8, 16384, 1040, False, ("tile", 64, 64, 1, 256, 148)),   # K % 128 != 0: 2-D boxes
    (100, 16384, 1024, False, ("tile", 128, 64, 2, 256, 148)),
    (64, 7168, 7168, False, ("tile", 64, 64, 4, 112, 112)),
    (2048, 2048, 512, False, ("tile", 128, 128, 1, 256, 148)),
    (8192, 8192, 8192, False, ("pair", 256, 256, 1, 1024, 148)),
    (8, 16384, 1024, True, ("swap", 8, 64, 4, 256, 148)),
    (32, 7168, 7168, True, ("swap", 32, 64, 4, 112, 112)),
    (64, 16384, 7168, True, ("tile", 64, 64, 4, 256, 148)),
    (100, 16384, 1024, True, ("tile", 128, 64, 2, 256, 148)),
    (2048, 2048, 512, True, ("tile", 128, 128, 1, 256, 148)),
    (8192, 8192, 8192, True, ("pair", 256, 256, 1, 1024, 148))])
def test_gemm_plan(rrf, M, N, K, mx, want):
    """The host-side GEMM plan on 148 SMs: the kernel a shape takes and how
    many output tiles its CTAs walk (ctas < tiles: several per CTA)."""
    p = rrf.rrf_plan_scaled_mm(M, N, K, 148, mx=mx)
    assert (p["kernel"], p["a_rows"], p["tile_n"], p["k_tiles_per_stage"], p["tiles"],
            p["ctas"]) == want


def test_gemm_plan_invariants_and_rejections(rrf):
    for M in (1, 7, 8, 9, 31, 33, 64, 65, 129, 300, 1000, 4096):
        for N in (16, 256, 1024, 7168, 16384):
            for K in (128, 1024, 7168):
                for mx in (False, True):
                    p = rrf.rrf_plan_scaled_mm(M, N, K, 148, mx=mx)
                    assert 1 <= p["ctas"] <= min(p["tiles"] * (2 if p["kernel"] == "pair" else 1),
                                                 148)
                    assert p["kernel"] != "swap" or M <= p["a_rows"] <= 32
                    if p["kernel"] == "pair":
                        assert p["ctas"] % 2 == 0
    p = rrf.rrf_plan_scaled_mm(0, 256, 256, 148)
    assert (p["kernel"], p["tiles"], p["ctas"]) == (None, 0, 0)
    for args, status in [((8, 8, 128, 148), "ERR_SHAPE"), ((8, 256, 8, 148), "ERR_SHAPE"),
                         ((-1, 256, 256, 148), "ERR_SHAPE"), ((8, 256, 256, 1), "ERR_UNSUPPORTED")]:
        with pytest.raises(rrf.RrfError) as e:
            rrf.rrf_plan_scaled_mm(*args)
        assert e.value.status == rrf.Status[status]
    with pytest.raises(rrf.RrfError):
        rrf.rrf_plan_scaled_mm(8, 256, 1040, 148, mx=True)  # MX needs K % 128 == 0


def test_sweep_writes_a_table_the_planner_reads(tmp_path):
    """bench.py's table writer: the lines it writes parse back to its
    entries, and the header is a C comment (the file is #included)."""
    import bench
    entries = [(2, 0, 1024, 1, 1, 1, 1.25), (8, 1, 7168, 64, 4, 1, 3.2262),
               (16, 1, 16384, 2048, 1, 0, 198.5)]
    out = tmp_path / "table.inc"
    bench.write_plan_table(str(out), entries, "NVIDIA B200", 148, 181.0)
    text = out.read_text()
    assert all(l.startswith("//") or l.startswith("RRF_PLAN(") for l in text.splitlines() if l)
    body = re.sub(r"//.*", "", text)
    got = [tuple(float(v) if "." in v else int(v) for v in m.replace("f", "").split(","))
           for m in re.findall(r"RRF_PLAN\(([^)]*)\)", body)]
    assert [g[:6] for g in got] == [e[:6] for e in entries]
    assert all(abs(g[6] - e[6]) < 5e-4 for g, e in zip(got, entries))
