// rrf_api.cu -- the C ABI declared in include/rrf.h: host-side validation,
// the launch planner and the entry points.  Every argument is checked before
// any CUDA call; the library allocates nothing and keeps only a per-device
// SM-count cache.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "rrf.h"
#include "rrf_internal.h"

namespace rrf {
namespace {

thread_local int t_last_cuda_error = 0;
thread_local int t_fail_next_launch = 0;
thread_local bool t_starve_next_gemm = false;

// The library's device error word: kernels set bits in it (a wait that ran
// out); rrf_device_error reads and clears it.  Static device memory, one per
// device; its address is looked up once per device.
__device__ unsigned int g_device_error;
std::atomic<uintptr_t> g_device_error_addr[64];

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

rrf_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return RRF_ERR_CUDA;
}

// SM count of the current device, cached per device.
rrf_status current_sm_count(int* sm_count) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev >= 0 && dev < kMaxDevices) {
        int cached = g_sm_count[dev].load(std::memory_order_relaxed);
        if (cached > 0) {
            *sm_count = cached;
            return RRF_OK;
        }
    }
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
    *sm_count = n;
    return RRF_OK;
}

// Address of the device error word on the current device.
rrf_status device_error_word(unsigned int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev >= 0 && dev < kMaxDevices) {
        uintptr_t cached = g_device_error_addr[dev].load(std::memory_order_relaxed);
        if (cached != 0) {
            *out = (unsigned int*)cached;
            return RRF_OK;
        }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev >= 0 && dev < kMaxDevices)
        g_device_error_addr[dev].store((uintptr_t)p, std::memory_order_relaxed);
    *out = (unsigned int*)p;
    return RRF_OK;
}

// A pending injected failure (test hook) replaces the launch.
bool take_injected_failure(cudaError_t* e) {
    if (t_fail_next_launch == 0) return false;
    *e = (cudaError_t)t_fail_next_launch;
    t_fail_next_launch = 0;
    return true;
}

int take_starve_gemm() {
    const bool s = t_starve_next_gemm;
    t_starve_next_gemm = false;
    return s ? 1 : 0;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, int64_t bytes) {
    return Range{(uintptr_t)p, (uintptr_t)p + (uintptr_t)bytes};
}

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

rrf_status check_shape(int num_inputs, int64_t rows, int64_t cols, int64_t max_cols) {
    if (num_inputs < 1 || num_inputs > RRF_MAX_INPUTS) return RRF_ERR_RANKS;
    if (rows < 0 || cols <= 0 || cols % 8 != 0 || cols > max_cols) return RRF_ERR_SHAPE;
    // every array's byte size (2 bytes per element) must fit in int64; the
    // grid (at most 16 blocks per row) must fit in 2^31 - 1 blocks
    if (rows > 0 && rows > (INT64_MAX / 2) / cols) return RRF_ERR_SHAPE;
    if (rows > (int64_t)INT32_MAX / 16) return RRF_ERR_SHAPE;
    return RRF_OK;
}

rrf_status check_inputs(const void* const* inputs, int num_inputs) {
    if (inputs == nullptr) return RRF_ERR_NULL;
    for (int r = 0; r < num_inputs; ++r) {
        if (inputs[r] == nullptr) return RRF_ERR_NULL;
        if (!aligned(inputs[r], 16)) return RRF_ERR_ALIGN;
    }
    return RRF_OK;
}

}  // namespace

// --------------------------------------------------------------- planner ---

static int round_up32(int64_t x) { return (int)((x + 31) / 32 * 32); }

// Threads per block and vectors per thread for a row slice of `slice`
// vectors: the fewest vectors per thread that keep the block at <= 512
// threads (any size up to the compiled bound at 8 vectors per thread), or,
// with forced_threads, the fewest that let that many threads cover the slice.
// (On B200 the 8 x 8192-column prefill row runs fastest as 512 threads x 2
// vectors: 2 blocks and 1024 threads per SM keep the most loads in flight.)
static bool pick_block(int R, int64_t slice, int forced_threads, FusedLaunch* l) {
    const int rb = input_bound(R);
    for (int vpt = 1; vpt <= 8; vpt *= 2) {
        const int max_t = fused_max_threads(rb, vpt);
        int t;
        if (forced_threads != 0) {
            t = forced_threads;
            if (t > max_t || (int64_t)t * vpt < slice) continue;
        } else {
            t = round_up32((slice + vpt - 1) / vpt);
            if ((t > 512 && vpt < 8) || t > max_t) continue;
        }
        l->threads = t;
        l->vecs_per_thread = vpt;
        return true;
    }
    return false;
}

// ------------------------------------------------------------ launch table --
// The fused call's launch is read from a table of measured launches
// (rrf_plan_table.inc, written by `bench.py --plan-sweep` on a B200): for
// input bounds 2/4/8/16, with and without a residual, over row lengths and
// batch sizes, the cluster size and L2-prefetch setting whose graph-replayed
// calls over buffer sets larger than L2 ran fastest.  A call takes the entry
// of its input bound and residual flag nearest to its shape (row length
// weighted 4x against batch size, both on a log scale; batch sizes scaled to
// the table's 148 SMs), then adjusts the cluster so that every block keeps
// at least 32 vectors and fits its slice.
struct PlanEntry {
    int rb;        // input bound
    int residual;  // 0 / 1
    int cols;
    int rows;
    int cluster;   // blocks per row
    int prefetch;  // L2 prefetch before the wait for the previous kernel
    float us;      // measured time per call of this launch
};

static const PlanEntry kPlanTable[] = {
#define RRF_PLAN(rb, res, cols, rows, cluster, prefetch, us) \
    {rb, res, cols, rows, cluster, prefetch, us},
#include "rrf_plan_table.inc"
#undef RRF_PLAN
    {0, 0, 0, 0, 0, 0, 0.0f}};

constexpr int kPlanTableSms = 148;

static const PlanEntry* table_entry(int R, int64_t rows, int64_t cols, int sm_count,
                                    bool residual) {
    const int rb = input_bound(R);
    const double r = (double)(rows > 0 ? rows : 1) * kPlanTableSms / sm_count;
    const PlanEntry* best = nullptr;
    double best_d = 0.0;
    for (const PlanEntry* e = kPlanTable; e->rb != 0; ++e) {
        if (e->rb != rb || e->residual != (residual ? 1 : 0)) continue;
        const double d = 4.0 * std::fabs(std::log2((double)cols / e->cols)) +
                         std::fabs(std::log2(r / e->rows));
        if (best == nullptr || d < best_d) {
            best = e;
            best_d = d;
        }
    }
    return best;
}

// The cluster size by formula, from earlier launch-shape sweeps on B200: one
// block per row when the batch has a row per SM or a row moves under ~48 KB
// (a block streams a 37 KB row in about the time a cluster round trip
// costs), else clusters of 8 (150 KB rows: 2.53 us at 1 row vs 4.53 us
// unsplit), or of 4 once 4 blocks per row give two blocks per SM.  The
// multi-GPU kernel uses it; the fused call uses it only without a table
// entry, and then prefetches when its grid is resident at once (at most 4
// blocks per SM).
static int cluster_formula(int64_t rows, double row_bytes, int sm_count) {
    if (rows >= sm_count || row_bytes < 48.0 * 1024.0) return 1;
    return rows * 4 >= 2 * (int64_t)sm_count ? 4 : 8;
}

// Launch for a given cluster size (0 = the planner's choice) and block size
// (0 = automatic).
static rrf_status shape_launch(int R, int64_t rows, int64_t cols, int sm_count, int cluster,
                               int forced_threads, bool residual, FusedLaunch* out) {
    rrf_status st = check_shape(R, rows, cols, RRF_MAX_COLS);
    if (st != RRF_OK) return st;
    if (sm_count < 1) sm_count = 1;
    const int64_t vecs = cols / 8;
    int c = 0;
    bool prefetch = false;
    if (const PlanEntry* e = table_entry(R, rows, cols, sm_count, residual)) {
        c = e->cluster;
        prefetch = e->prefetch != 0;
    } else {
        const double row_bytes = (double)cols * (2.0 * R + (residual ? 4.0 : 0.0) + 1.0);
        c = cluster_formula(rows, row_bytes, sm_count);
        prefetch = rows * c <= 4 * (int64_t)sm_count;
    }
    if (cluster != 0) {
        c = cluster;
    } else {
        // at least 32 vectors per block; then split further, up to 16, while
        // one block cannot hold its slice
        while (c > 1 && vecs / c < 32) --c;
        while (c < 16 && !pick_block(R, (vecs + c - 1) / c, forced_threads, out)) ++c;
    }
    if (!pick_block(R, (vecs + c - 1) / c, forced_threads, out))
        return cluster == 0 && forced_threads == 0 ? RRF_ERR_SHAPE : RRF_ERR_UNSUPPORTED;
    out->cluster = c;
    out->pdl = true;
    out->prefetch = prefetch;
    // Exchange: measured on B200 (residual stores after the exchange in both
    // forms), the st.async + mbarrier exchange ties the cluster barrier at 1-8
    // rows and beats it from 32 rows on (4.03 vs 4.39 us at 64 rows of 7168
    // columns; 0.3 us less at 37 and 64 rows of 4 inputs).
    out->async_exchange = true;
    return RRF_OK;
}

rrf_status plan_fused(int R, int64_t rows, int64_t cols, int sm_count, bool residual,
                      FusedLaunch* out) {
    return shape_launch(R, rows, cols, sm_count, 0, 0, residual, out);
}

rrf_status record_cuda_error(cudaError_t e) { return cuda_fail(e); }

cudaError_t launch_fused(const FusedArgs& a, int64_t rows, const FusedLaunch& l, bool residual,
                         cudaStream_t stream) {
    switch (input_bound(a.R)) {
        case 2: return launch_fused_rb2(a, rows, l, residual, stream);
        case 4: return launch_fused_rb4(a, rows, l, residual, stream);
        case 8: return launch_fused_rb8(a, rows, l, residual, stream);
        default: return launch_fused_rb16(a, rows, l, residual, stream);
    }
}

}  // namespace rrf

using namespace rrf;

// ------------------------------------------------------------ validation ---

extern "C" rrf_status rrf_check_sum_args(const void* const* inputs, int num_inputs,
                                         int64_t rows, int64_t cols, const void* out) {
    rrf_status st = check_shape(num_inputs, rows, cols, INT64_MAX);
    if (st != RRF_OK || rows == 0) return st;
    if ((st = check_inputs(inputs, num_inputs)) != RRF_OK) return st;
    if (out == nullptr) return RRF_ERR_NULL;
    if (!aligned(out, 16)) return RRF_ERR_ALIGN;
    const int64_t bytes = rows * cols * 2;
    const Range o = range_of(out, bytes);
    for (int r = 0; r < num_inputs; ++r)
        if (overlap(o, range_of(inputs[r], bytes))) return RRF_ERR_ALIAS;
    return RRF_OK;
}

extern "C" rrf_status rrf_check_fused_args(const void* const* inputs, int num_inputs,
                                           int64_t rows, int64_t cols,
                                           const void* residual_in,
                                           const void* residual_out, const void* gamma,
                                           float eps, float weight_offset, float scale_ub,
                                           const void* q_out, const void* scales_out) {
    rrf_status st = check_shape(num_inputs, rows, cols, RRF_MAX_COLS);
    if (st != RRF_OK) return st;
    if (!(std::isfinite(eps) && eps >= 0.0f)) return RRF_ERR_VALUE;
    if (!std::isfinite(weight_offset)) return RRF_ERR_VALUE;
    if (std::isnan(scale_ub) || !(scale_ub > 0.0f)) return RRF_ERR_VALUE;
    if (rows == 0) return RRF_OK;
    if ((st = check_inputs(inputs, num_inputs)) != RRF_OK) return st;
    if ((residual_in == nullptr) != (residual_out == nullptr)) return RRF_ERR_NULL;
    if (gamma == nullptr || q_out == nullptr || scales_out == nullptr) return RRF_ERR_NULL;
    if (!aligned(gamma, 16) || !aligned(q_out, 16) || !aligned(scales_out, 4))
        return RRF_ERR_ALIGN;
    if (residual_in != nullptr && (!aligned(residual_in, 16) || !aligned(residual_out, 16)))
        return RRF_ERR_ALIGN;

    const int64_t bf16_bytes = rows * cols * 2;
    Range reads[RRF_MAX_INPUTS + 2];
    int n_reads = 0;
    for (int r = 0; r < num_inputs; ++r) reads[n_reads++] = range_of(inputs[r], bf16_bytes);
    reads[n_reads++] = range_of(gamma, cols * 2);
    const bool in_place = residual_in != nullptr && residual_in == residual_out;
    if (residual_in != nullptr && !in_place)
        reads[n_reads++] = range_of(residual_in, bf16_bytes);

    Range writes[3];
    int n_writes = 0;
    writes[n_writes++] = range_of(q_out, rows * cols);
    writes[n_writes++] = range_of(scales_out, rows * 4);
    if (residual_out != nullptr) writes[n_writes++] = range_of(residual_out, bf16_bytes);

    for (int w = 0; w < n_writes; ++w) {
        for (int r = 0; r < n_reads; ++r)
            if (overlap(writes[w], reads[r])) return RRF_ERR_ALIAS;
        for (int w2 = w + 1; w2 < n_writes; ++w2)
            if (overlap(writes[w], writes[w2])) return RRF_ERR_ALIAS;
    }
    return RRF_OK;
}

// ----------------------------------------------------------- entry points ---

extern "C" rrf_status rrf_sum(const void* const* inputs, int num_inputs, int64_t rows,
                              int64_t cols, void* out, rrf_stream_t stream) {
    rrf_status st = rrf_check_sum_args(inputs, num_inputs, rows, cols, out);
    if (st != RRF_OK || rows == 0) return st;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    SumArgs a = {};
    for (int r = 0; r < num_inputs; ++r) a.in[r] = static_cast<const uint4*>(inputs[r]);
    a.out = static_cast<uint4*>(out);
    a.R = num_inputs;
    a.n_vecs = rows * cols / 8;
    cudaError_t e;
    if (!take_injected_failure(&e)) e = launch_sum(a, sm_count, true, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_sum_rmsnorm_fp8_ex(const void* const* inputs, int num_inputs,
                                             int64_t rows, int64_t cols,
                                             const void* residual_in, void* residual_out,
                                             const void* gamma, float eps,
                                             float weight_offset, float scale_ub,
                                             void* q_out, float* scales_out, int variant,
                                             int cluster_size, int block_threads, int flags,
                                             rrf_stream_t stream) {
    rrf_status st = rrf_check_fused_args(inputs, num_inputs, rows, cols, residual_in,
                                         residual_out, gamma, eps, weight_offset, scale_ub,
                                         q_out, scales_out);
    if (st != RRF_OK) return st;
    if (variant < RRF_VARIANT_AUTO || variant > RRF_VARIANT_CLUSTER) return RRF_ERR_UNSUPPORTED;
    if ((flags & ~(RRF_FLAG_NO_PDL | RRF_FLAG_BARRIER_EXCHANGE | RRF_FLAG_NO_PREFETCH |
                   RRF_FLAG_PREFETCH | RRF_FLAG_DEBUG_STARVE_EXCHANGE)) != 0 ||
        (flags & RRF_FLAG_NO_PREFETCH && flags & RRF_FLAG_PREFETCH))
        return RRF_ERR_UNSUPPORTED;
    if (block_threads != 0 && (block_threads < 32 || block_threads > 1024 || block_threads % 32))
        return RRF_ERR_UNSUPPORTED;
    if (variant == RRF_VARIANT_CLUSTER && cluster_size != 0 &&
        (cluster_size < 2 || cluster_size > 16))
        return RRF_ERR_UNSUPPORTED;
    if (rows == 0) return RRF_OK;

    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    int cluster = 0;
    if (variant == RRF_VARIANT_ROW) cluster = 1;
    if (variant == RRF_VARIANT_CLUSTER) {
        cluster = cluster_size;
        if (cluster == 0) {
            FusedLaunch planned = {};
            if ((st = plan_fused(num_inputs, rows, cols, sm_count, residual_in != nullptr,
                                 &planned)) != RRF_OK)
                return st;
            cluster = planned.cluster > 1 ? planned.cluster : 2;
        }
    }
    FusedLaunch l = {};
    if ((st = shape_launch(num_inputs, rows, cols, sm_count, cluster, block_threads,
                           residual_in != nullptr, &l)) != RRF_OK)
        return st;
    const int64_t vecs = cols / 8;
    l.pdl = (flags & RRF_FLAG_NO_PDL) == 0;
    if (flags & RRF_FLAG_NO_PREFETCH) l.prefetch = false;
    if (flags & RRF_FLAG_PREFETCH) l.prefetch = true;
    if (flags & RRF_FLAG_BARRIER_EXCHANGE) l.async_exchange = false;
    if (flags & RRF_FLAG_DEBUG_STARVE_EXCHANGE) {
        // the hook exercises the bounded wait of the transaction-counted exchange
        if (l.cluster == 1 || (flags & RRF_FLAG_BARRIER_EXCHANGE)) return RRF_ERR_UNSUPPORTED;
        l.async_exchange = true;
    }
    unsigned int* err = nullptr;
    if ((st = device_error_word(&err)) != RRF_OK) return st;

    FusedArgs a = {};
    for (int r = 0; r < num_inputs; ++r) a.in[r] = static_cast<const uint4*>(inputs[r]);
    a.res_in = static_cast<const uint4*>(residual_in);
    a.res_out = static_cast<uint4*>(residual_out);
    a.gamma = static_cast<const uint4*>(gamma);
    a.q = static_cast<uint2*>(q_out);
    a.scales = scales_out;
    a.R = num_inputs;
    a.vecs = (int)vecs;
    a.rows = rows;
    a.cluster = l.cluster;
    a.slice_vecs = (int)((vecs + l.cluster - 1) / l.cluster);
    a.inv_cols = (float)(1.0 / (double)cols);
    a.eps = eps;
    a.weight_offset = weight_offset;
    a.scale_ub = scale_ub;
    a.err = err;
    a.starve = (flags & RRF_FLAG_DEBUG_STARVE_EXCHANGE) ? 1 : 0;
    a.prefetch = l.prefetch ? 1 : 0;
    cudaError_t e;
    if (!take_injected_failure(&e))
        e = launch_fused(a, rows, l, residual_in != nullptr, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_sum_rmsnorm_fp8(const void* const* inputs, int num_inputs,
                                          int64_t rows, int64_t cols,
                                          const void* residual_in, void* residual_out,
                                          const void* gamma, float eps, float weight_offset,
                                          float scale_ub, void* q_out, float* scales_out,
                                          rrf_stream_t stream) {
    return rrf_sum_rmsnorm_fp8_ex(inputs, num_inputs, rows, cols, residual_in, residual_out,
                                  gamma, eps, weight_offset, scale_ub, q_out, scales_out,
                                  RRF_VARIANT_AUTO, 0, 0, 0, stream);
}

// ------------------------------------------------------------ MX output ---

extern "C" rrf_status rrf_check_mxfp8_args(const void* const* inputs, int num_inputs,
                                           int64_t rows, int64_t cols, const void* residual_in,
                                           const void* residual_out, const void* gamma,
                                           float eps, float weight_offset, const void* q_out,
                                           const void* scales_mx_out) {
    rrf_status st = check_shape(num_inputs, rows, cols, RRF_MAX_COLS);
    if (st != RRF_OK) return st;
    if (cols % 32 != 0) return RRF_ERR_SHAPE;
    if (!(std::isfinite(eps) && eps >= 0.0f)) return RRF_ERR_VALUE;
    if (!std::isfinite(weight_offset)) return RRF_ERR_VALUE;
    if (rows == 0) return RRF_OK;
    if ((st = check_inputs(inputs, num_inputs)) != RRF_OK) return st;
    if ((residual_in == nullptr) != (residual_out == nullptr)) return RRF_ERR_NULL;
    if (gamma == nullptr || q_out == nullptr || scales_mx_out == nullptr) return RRF_ERR_NULL;
    if (!aligned(gamma, 16) || !aligned(q_out, 16)) return RRF_ERR_ALIGN;
    if (residual_in != nullptr && (!aligned(residual_in, 16) || !aligned(residual_out, 16)))
        return RRF_ERR_ALIGN;
    const int64_t bf16_bytes = rows * cols * 2;
    Range reads[RRF_MAX_INPUTS + 2];
    int n_reads = 0;
    for (int r = 0; r < num_inputs; ++r) reads[n_reads++] = range_of(inputs[r], bf16_bytes);
    reads[n_reads++] = range_of(gamma, cols * 2);
    if (residual_in != nullptr && residual_in != residual_out)
        reads[n_reads++] = range_of(residual_in, bf16_bytes);
    Range writes[3];
    int n_writes = 0;
    writes[n_writes++] = range_of(q_out, rows * cols);
    writes[n_writes++] = range_of(scales_mx_out, rows * (cols / 32));
    if (residual_out != nullptr) writes[n_writes++] = range_of(residual_out, bf16_bytes);
    for (int w = 0; w < n_writes; ++w) {
        for (int r = 0; r < n_reads; ++r)
            if (overlap(writes[w], reads[r])) return RRF_ERR_ALIAS;
        for (int w2 = w + 1; w2 < n_writes; ++w2)
            if (overlap(writes[w], writes[w2])) return RRF_ERR_ALIAS;
    }
    return RRF_OK;
}

static rrf_status mxfp8_call(const void* const* inputs, int num_inputs, int64_t rows,
                             int64_t cols, const void* residual_in, void* residual_out,
                             const void* gamma, float eps, float weight_offset, void* q_out,
                             void* scales_mx_out, bool blocked, rrf_stream_t stream) {
    rrf_status st = rrf_check_mxfp8_args(inputs, num_inputs, rows, cols, residual_in,
                                         residual_out, gamma, eps, weight_offset, q_out,
                                         scales_mx_out);
    if (st != RRF_OK) return st;
    if (blocked) {
        if (cols % 128 != 0) return RRF_ERR_SHAPE;
        if (rows == 0) return RRF_OK;
        // the blocked buffer is larger than the row-major one (rows rounded
        // up): it must not overlap the data either
        const int64_t bf16_bytes = rows * cols * 2;
        const Range sc = range_of(scales_mx_out, RRF_MX_BLOCKED_BYTES(rows, cols));
        for (int r = 0; r < num_inputs; ++r)
            if (overlap(sc, range_of(inputs[r], bf16_bytes))) return RRF_ERR_ALIAS;
        if (overlap(sc, range_of(gamma, cols * 2)) || overlap(sc, range_of(q_out, rows * cols)))
            return RRF_ERR_ALIAS;
        if (residual_in != nullptr && (overlap(sc, range_of(residual_in, bf16_bytes)) ||
                                       overlap(sc, range_of(residual_out, bf16_bytes))))
            return RRF_ERR_ALIAS;
    }
    if (rows == 0) return RRF_OK;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    FusedLaunch l = {};
    if ((st = shape_launch(num_inputs, rows, cols, sm_count, 0, 0, residual_in != nullptr,
                           &l)) != RRF_OK)
        return st;
    l.mx = true;
    unsigned int* err = nullptr;
    if ((st = device_error_word(&err)) != RRF_OK) return st;
    const int64_t vecs = cols / 8;
    FusedArgs a = {};
    for (int r = 0; r < num_inputs; ++r) a.in[r] = static_cast<const uint4*>(inputs[r]);
    a.res_in = static_cast<const uint4*>(residual_in);
    a.res_out = static_cast<uint4*>(residual_out);
    a.gamma = static_cast<const uint4*>(gamma);
    a.q = static_cast<uint2*>(q_out);
    a.scales_mx = static_cast<uint8_t*>(scales_mx_out);
    a.mx_blocked = blocked ? 1 : 0;
    a.prefetch = l.prefetch ? 1 : 0;
    a.R = num_inputs;
    a.vecs = (int)vecs;
    a.rows = rows;
    a.cluster = l.cluster;
    // a cluster block's slice starts on a 32-element block (4 vectors); the
    // block's threads (a multiple of 32) x vectors per thread still cover it
    a.slice_vecs = (int)(((vecs + l.cluster - 1) / l.cluster + 3) / 4 * 4);
    a.inv_cols = (float)(1.0 / (double)cols);
    a.eps = eps;
    a.weight_offset = weight_offset;
    a.scale_ub = 1.0f;
    a.err = err;
    cudaError_t e;
    if (!take_injected_failure(&e))
        e = launch_fused(a, rows, l, residual_in != nullptr, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_sum_rmsnorm_mxfp8(const void* const* inputs, int num_inputs,
                                            int64_t rows, int64_t cols, const void* residual_in,
                                            void* residual_out, const void* gamma, float eps,
                                            float weight_offset, void* q_out,
                                            void* scales_mx_out, rrf_stream_t stream) {
    return mxfp8_call(inputs, num_inputs, rows, cols, residual_in, residual_out, gamma, eps,
                      weight_offset, q_out, scales_mx_out, false, stream);
}

extern "C" rrf_status rrf_sum_rmsnorm_mxfp8_blocked(const void* const* inputs, int num_inputs,
                                                    int64_t rows, int64_t cols,
                                                    const void* residual_in,
                                                    void* residual_out, const void* gamma,
                                                    float eps, float weight_offset, void* q_out,
                                                    void* scales_mx_out, rrf_stream_t stream) {
    return mxfp8_call(inputs, num_inputs, rows, cols, residual_in, residual_out, gamma, eps,
                      weight_offset, q_out, scales_mx_out, true, stream);
}

// -------------------------------------------------------- sharded norm ---

extern "C" rrf_status rrf_check_pre_args(const void* const* inputs, int num_inputs, int64_t rows,
                                         int64_t cols, const void* residual_in,
                                         const void* residual_out, const void* h_out,
                                         const void* gamma, float weight_offset,
                                         const void* stats_out) {
    rrf_status st = check_shape(num_inputs, rows, cols, RRF_MAX_COLS);
    if (st != RRF_OK) return st;
    if (!std::isfinite(weight_offset)) return RRF_ERR_VALUE;
    if (rows == 0) return RRF_OK;
    if ((st = check_inputs(inputs, num_inputs)) != RRF_OK) return st;
    if ((residual_in == nullptr) != (residual_out == nullptr)) return RRF_ERR_NULL;
    // the norm input goes to residual_out with a residual, to h_out without
    if ((residual_in == nullptr) == (h_out == nullptr)) return RRF_ERR_NULL;
    if (gamma == nullptr || stats_out == nullptr) return RRF_ERR_NULL;
    if (!aligned(gamma, 16) || !aligned(stats_out, 8)) return RRF_ERR_ALIGN;
    if (residual_in != nullptr && (!aligned(residual_in, 16) || !aligned(residual_out, 16)))
        return RRF_ERR_ALIGN;
    if (h_out != nullptr && !aligned(h_out, 16)) return RRF_ERR_ALIGN;
    const int64_t bf16_bytes = rows * cols * 2;
    Range reads[RRF_MAX_INPUTS + 2];
    int n_reads = 0;
    for (int r = 0; r < num_inputs; ++r) reads[n_reads++] = range_of(inputs[r], bf16_bytes);
    reads[n_reads++] = range_of(gamma, cols * 2);
    if (residual_in != nullptr && residual_in != residual_out)
        reads[n_reads++] = range_of(residual_in, bf16_bytes);
    Range writes[2];
    int n_writes = 0;
    writes[n_writes++] = range_of(residual_out != nullptr ? residual_out : h_out, bf16_bytes);
    writes[n_writes++] = range_of(stats_out, rows * 8);
    for (int w = 0; w < n_writes; ++w) {
        for (int r = 0; r < n_reads; ++r)
            if (overlap(writes[w], reads[r])) return RRF_ERR_ALIAS;
        for (int w2 = w + 1; w2 < n_writes; ++w2)
            if (overlap(writes[w], writes[w2])) return RRF_ERR_ALIAS;
    }
    return RRF_OK;
}

extern "C" rrf_status rrf_sum_rmsnorm_fp8_pre(const void* const* inputs, int num_inputs,
                                              int64_t rows, int64_t cols,
                                              const void* residual_in, void* residual_out,
                                              void* h_out, const void* gamma,
                                              float weight_offset, float* stats_out,
                                              rrf_stream_t stream) {
    rrf_status st = rrf_check_pre_args(inputs, num_inputs, rows, cols, residual_in,
                                       residual_out, h_out, gamma, weight_offset, stats_out);
    if (st != RRF_OK || rows == 0) return st;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    FusedLaunch l = {};
    if ((st = shape_launch(num_inputs, rows, cols, sm_count, 0, 0, residual_in != nullptr,
                           &l)) != RRF_OK)
        return st;
    unsigned int* err = nullptr;
    if ((st = device_error_word(&err)) != RRF_OK) return st;
    const int64_t vecs = cols / 8;
    FusedArgs a = {};
    for (int r = 0; r < num_inputs; ++r) a.in[r] = static_cast<const uint4*>(inputs[r]);
    a.res_in = static_cast<const uint4*>(residual_in);
    a.res_out = static_cast<uint4*>(residual_out);
    a.gamma = static_cast<const uint4*>(gamma);
    a.R = num_inputs;
    a.vecs = (int)vecs;
    a.rows = rows;
    a.cluster = l.cluster;
    a.slice_vecs = (int)((vecs + l.cluster - 1) / l.cluster);
    a.inv_cols = (float)(1.0 / (double)cols);
    a.weight_offset = weight_offset;
    a.scale_ub = 1.0f;
    a.err = err;
    a.stats_only = 1;
    a.prefetch = l.prefetch ? 1 : 0;
    a.stats = reinterpret_cast<float2*>(stats_out);
    a.h_out = static_cast<uint4*>(h_out);
    cudaError_t e;
    if (!take_injected_failure(&e))
        e = launch_fused(a, rows, l, residual_in != nullptr, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_check_post_args(const void* h, int64_t rows, int64_t cols,
                                          const float* stats, int shards, int64_t total_cols,
                                          const void* gamma, float eps, float weight_offset,
                                          float scale_ub, const void* q_out,
                                          const void* scales_out) {
    if (shards < 1 || shards > RRF_MAX_SHARDS) return RRF_ERR_SHAPE;
    if (rows < 0 || cols <= 0 || cols % 8 != 0 || total_cols < cols) return RRF_ERR_SHAPE;
    if (rows > 0 && rows > (INT64_MAX / 2) / cols) return RRF_ERR_SHAPE;
    if ((rows + 3) / 4 * ((cols / 8 + 63) / 64) > (int64_t)INT32_MAX) return RRF_ERR_SHAPE;
    if (!(std::isfinite(eps) && eps >= 0.0f)) return RRF_ERR_VALUE;
    if (!std::isfinite(weight_offset)) return RRF_ERR_VALUE;
    if (std::isnan(scale_ub) || !(scale_ub > 0.0f)) return RRF_ERR_VALUE;
    if (rows == 0) return RRF_OK;
    if (h == nullptr || stats == nullptr || gamma == nullptr || q_out == nullptr)
        return RRF_ERR_NULL;
    if (!aligned(h, 16) || !aligned(gamma, 16) || !aligned(q_out, 16) || !aligned(stats, 8))
        return RRF_ERR_ALIGN;
    if (scales_out != nullptr && !aligned(scales_out, 4)) return RRF_ERR_ALIGN;
    const Range reads[3] = {range_of(h, rows * cols * 2), range_of(gamma, cols * 2),
                            range_of(stats, (int64_t)shards * rows * 8)};
    Range writes[2];
    int n_writes = 0;
    writes[n_writes++] = range_of(q_out, rows * cols);
    if (scales_out != nullptr) writes[n_writes++] = range_of(scales_out, rows * 4);
    for (int w = 0; w < n_writes; ++w) {
        for (int r = 0; r < 3; ++r)
            if (overlap(writes[w], reads[r])) return RRF_ERR_ALIAS;
        for (int w2 = w + 1; w2 < n_writes; ++w2)
            if (overlap(writes[w], writes[w2])) return RRF_ERR_ALIAS;
    }
    return RRF_OK;
}

extern "C" rrf_status rrf_rmsnorm_fp8_post(const void* h, int64_t rows, int64_t cols,
                                           const float* stats, int shards, int64_t total_cols,
                                           const void* gamma, float eps, float weight_offset,
                                           float scale_ub, void* q_out, float* scales_out,
                                           rrf_stream_t stream) {
    rrf_status st = rrf_check_post_args(h, rows, cols, stats, shards, total_cols, gamma, eps,
                                        weight_offset, scale_ub, q_out, scales_out);
    if (st != RRF_OK || rows == 0) return st;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    PostArgs a = {};
    a.h = static_cast<const uint4*>(h);
    a.gamma = static_cast<const uint4*>(gamma);
    a.stats = reinterpret_cast<const float2*>(stats);
    a.q = static_cast<uint2*>(q_out);
    a.scales = scales_out;
    a.rows = rows;
    a.vecs = (int)(cols / 8);
    a.shards = shards;
    a.inv_total_cols = (float)(1.0 / (double)total_cols);
    a.eps = eps;
    a.weight_offset = weight_offset;
    a.scale_ub = scale_ub;
    if ((st = device_error_word(&a.err)) != RRF_OK) return st;
    cudaError_t e;
    if (!take_injected_failure(&e)) e = launch_post(a, sm_count, true, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

// ------------------------------------------------------ multi-GPU form ---

namespace rrf {
namespace {

constexpr int64_t kArMaxCols = (int64_t)8 * 8 * kArMaxThreads * 4;  // C * 8 * T * VPT
constexpr uint64_t kArDefaultTimeoutNs = 1000000000ull;             // 1 s

// Two-shot splits the rows over the ranks, so it needs a row per rank; it
// moves (world - 1) / world of the partials over the links where one-shot
// moves world - 1 times them, and both take the same two barriers.
int ar_mode(int world, int64_t rows, int mode) {
    if (mode != RRF_AR_AUTO) return mode;
    return rows >= world ? RRF_AR_TWO_SHOT : RRF_AR_ONE_SHOT;
}

// The row shape for the rows one rank computes, chosen as for the single-GPU
// kernel's formula (cluster_formula), then the fewest vectors per thread (at most 4)
// that keep a block at <= 512 threads, splitting the row further (up to
// clusters of 8) while none does.
rrf_status plan_allreduce(int world, int64_t rows, int64_t cols, bool residual, int mode,
                          int sm_count, ArLaunch* l) {
    if (world < 1 || world > RRF_AR_MAX_WORLD) return RRF_ERR_RANKS;
    rrf_status st = check_shape(world, rows, cols, kArMaxCols);
    if (st != RRF_OK) return st;
    if (mode < RRF_AR_AUTO || mode > RRF_AR_TWO_SHOT) return RRF_ERR_UNSUPPORTED;
    if (sm_count < 1) sm_count = 1;
    l->two_shot = ar_mode(world, rows, mode) == RRF_AR_TWO_SHOT;
    const int64_t mine = l->two_shot ? (rows + world - 1) / world : rows;
    const int64_t vecs = cols / 8;
    const double row_bytes = (double)cols * (2.0 * world + (residual ? 4.0 : 0.0) + 1.0);
    int c = cluster_formula(mine, row_bytes, sm_count);
    while (c > 1 && vecs / c < 32) c /= 2;
    for (;;) {
        const int64_t slice = (vecs + c - 1) / c;
        int vpt = 1;
        while (vpt < 4 && slice > (int64_t)kArMaxThreads * vpt) vpt *= 2;
        if (slice <= (int64_t)kArMaxThreads * vpt) {
            l->cluster = c;
            l->vecs_per_thread = vpt;
            l->threads = round_up32((slice + vpt - 1) / vpt);
            break;
        }
        if (c >= 8) return RRF_ERR_SHAPE;
        c *= 2;
    }
    l->residual = residual;
    l->local_ranks = 1;
    l->blocks = 0;
    return RRF_OK;
}

}  // namespace
}  // namespace rrf

extern "C" rrf_status rrf_check_allreduce_args(
    const void* const* inputs, const void* const* residual_in, void* const* residual_out,
    void* const* q_out, float* const* scales_out, unsigned int* const* signals, int world,
    int rank, int local_ranks, int64_t rows, int64_t cols, const void* gamma, float eps,
    float weight_offset, float scale_ub, int mode) {
    if (world < 1 || world > RRF_AR_MAX_WORLD) return RRF_ERR_RANKS;
    if (local_ranks != 1 && local_ranks != world) return RRF_ERR_UNSUPPORTED;
    if (rank < 0 || rank >= world || (local_ranks > 1 && rank != 0)) return RRF_ERR_RANKS;
    if (mode < RRF_AR_AUTO || mode > RRF_AR_TWO_SHOT) return RRF_ERR_UNSUPPORTED;
    rrf_status st = check_shape(world, rows, cols, kArMaxCols);
    if (st != RRF_OK) return st;
    if (!(std::isfinite(eps) && eps >= 0.0f)) return RRF_ERR_VALUE;
    if (!std::isfinite(weight_offset)) return RRF_ERR_VALUE;
    if (std::isnan(scale_ub) || !(scale_ub > 0.0f)) return RRF_ERR_VALUE;
    if (rows == 0) return RRF_OK;
    if (!inputs || !q_out || !scales_out || !signals || !gamma) return RRF_ERR_NULL;
    if ((residual_in == nullptr) != (residual_out == nullptr)) return RRF_ERR_NULL;
    if (!aligned(gamma, 16)) return RRF_ERR_ALIGN;
    const bool res = residual_in != nullptr;
    for (int j = 0; j < world; ++j) {
        if (!inputs[j] || !q_out[j] || !scales_out[j] || !signals[j]) return RRF_ERR_NULL;
        if (res && (!residual_in[j] || !residual_out[j])) return RRF_ERR_NULL;
        if (!aligned(inputs[j], 16) || !aligned(q_out[j], 16) || !aligned(scales_out[j], 4) ||
            !aligned(signals[j], 16))
            return RRF_ERR_ALIGN;
        if (res && (!aligned(residual_in[j], 16) || !aligned(residual_out[j], 16)))
            return RRF_ERR_ALIGN;
    }
    // No write may overlap a read or another write, except residual_out[j]
    // == residual_in[j] exactly (every rank's buffers, as this GPU sees them).
    const int64_t bf16_bytes = rows * cols * 2;
    Range reads[2 * RRF_AR_MAX_WORLD + 1];
    Range writes[4 * RRF_AR_MAX_WORLD];
    int n_reads = 0, n_writes = 0;
    reads[n_reads++] = range_of(gamma, cols * 2);
    for (int j = 0; j < world; ++j) {
        reads[n_reads++] = range_of(inputs[j], bf16_bytes);
        if (res && residual_in[j] != residual_out[j])
            reads[n_reads++] = range_of(residual_in[j], bf16_bytes);
        writes[n_writes++] = range_of(q_out[j], rows * cols);
        writes[n_writes++] = range_of(scales_out[j], rows * 4);
        writes[n_writes++] = range_of(signals[j], (int64_t)RRF_AR_SIGNAL_WORDS * 4);
        if (res) writes[n_writes++] = range_of(residual_out[j], bf16_bytes);
    }
    for (int w = 0; w < n_writes; ++w) {
        for (int r = 0; r < n_reads; ++r)
            if (overlap(writes[w], reads[r])) return RRF_ERR_ALIAS;
        for (int w2 = w + 1; w2 < n_writes; ++w2)
            if (overlap(writes[w], writes[w2])) return RRF_ERR_ALIAS;
    }
    if (res) {  // an in-place residual may serve only its own rank
        for (int j = 0; j < world; ++j)
            for (int i = 0; i < world; ++i)
                if (i != j && overlap(range_of(residual_out[j], bf16_bytes),
                                      range_of(residual_in[i], bf16_bytes)))
                    return RRF_ERR_ALIAS;
    }
    return RRF_OK;
}

extern "C" rrf_status rrf_allreduce_rmsnorm_fp8(
    const void* const* inputs, const void* const* residual_in, void* const* residual_out,
    void* const* q_out, float* const* scales_out, unsigned int* const* signals, int world,
    int rank, int local_ranks, int64_t rows, int64_t cols, const void* gamma, float eps,
    float weight_offset, float scale_ub, int mode, uint64_t timeout_ns, rrf_stream_t stream) {
    rrf_status st = rrf_check_allreduce_args(inputs, residual_in, residual_out, q_out,
                                             scales_out, signals, world, rank, local_ranks,
                                             rows, cols, gamma, eps, weight_offset, scale_ub,
                                             mode);
    if (st != RRF_OK || rows == 0) return st;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    ArLaunch l = {};
    if ((st = plan_allreduce(world, rows, cols, residual_in != nullptr, mode, sm_count, &l)) !=
        RRF_OK)
        return st;
    l.local_ranks = local_ranks;
    // A persistent grid: every block of every rank in this launch resident
    // at once (the barriers pair block b of every rank), at most one cluster
    // per row of the rank's range.
    int resident = 0;
    cudaError_t e = allreduce_resident_blocks(l, &resident);
    if (e != cudaSuccess) return cuda_fail(e);
    int64_t cap = resident / local_ranks;
    if (cap > RRF_AR_MAX_BLOCKS) cap = RRF_AR_MAX_BLOCKS;
    cap = cap / l.cluster * l.cluster;
    if (cap < l.cluster) return RRF_ERR_UNSUPPORTED;
    const int64_t mine = l.two_shot ? (rows + world - 1) / world : rows;
    const int64_t want = mine * l.cluster;
    l.blocks = (int)(want < cap ? want : cap);
    unsigned int* err = nullptr;
    if ((st = device_error_word(&err)) != RRF_OK) return st;

    ArArgs a = {};
    for (int j = 0; j < world; ++j) {
        a.in[j] = static_cast<const uint4*>(inputs[j]);
        if (residual_in != nullptr) {
            a.res_in[j] = static_cast<const uint4*>(residual_in[j]);
            a.res_out[j] = static_cast<uint4*>(residual_out[j]);
        }
        a.q[j] = static_cast<uint2*>(q_out[j]);
        a.scales[j] = scales_out[j];
        a.sig[j] = signals[j];
    }
    a.gamma = static_cast<const uint4*>(gamma);
    a.world = world;
    a.rank0 = rank;
    a.blocks = l.blocks;
    a.two_shot = l.two_shot;
    a.rows = rows;
    a.rows_per_rank = mine;
    a.vecs = (int)(cols / 8);
    a.cluster = l.cluster;
    a.slice_vecs = (int)((cols / 8 + l.cluster - 1) / l.cluster);
    a.inv_cols = (float)(1.0 / (double)cols);
    a.eps = eps;
    a.weight_offset = weight_offset;
    a.scale_ub = scale_ub;
    a.timeout_ns = timeout_ns != 0 ? timeout_ns : kArDefaultTimeoutNs;
    a.err = err;
    if (!take_injected_failure(&e)) e = launch_allreduce(a, l, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_plan_allreduce(int world, int64_t rows, int64_t cols, int residual,
                                         int mode, int sm_count, int* mode_out,
                                         int* cluster_size, int* block_threads,
                                         int* vecs_per_thread) {
    if (!mode_out || !cluster_size || !block_threads || !vecs_per_thread) return RRF_ERR_NULL;
    ArLaunch l = {};
    rrf_status st = plan_allreduce(world, rows, cols, residual != 0, mode, sm_count, &l);
    if (st != RRF_OK) return st;
    *mode_out = l.two_shot ? RRF_AR_TWO_SHOT : RRF_AR_ONE_SHOT;
    *cluster_size = l.cluster;
    *block_threads = l.threads;
    *vecs_per_thread = l.vecs_per_thread;
    return RRF_OK;
}

// ---------------------------------------------------------- FP8 GEMM ---

extern "C" rrf_status rrf_check_scaled_mm_args(const void* a, const float* a_scale,
                                               const void* b, const float* b_scale,
                                               const void* bias, const void* out, int64_t M,
                                               int64_t N, int64_t K) {
    // N and K: multiples of 16 (16-byte rows for the tensor maps and the
    // stores); M: the grid's second dimension counts 128-row tiles
    if (M < 0 || N < 16 || K < 16 || N % 16 != 0 || K % 16 != 0) return RRF_ERR_SHAPE;
    if (M > 65535LL * 128 || N > (int64_t)INT32_MAX / 2 || K > (int64_t)INT32_MAX / 2)
        return RRF_ERR_SHAPE;
    if (M == 0) return RRF_OK;
    if (!a || !a_scale || !b || !b_scale || !out) return RRF_ERR_NULL;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(a_scale, 4) ||
        !aligned(b_scale, 4) || (bias != nullptr && !aligned(bias, 2)))
        return RRF_ERR_ALIGN;
    const Range o = range_of(out, M * N * 2);
    const Range reads[5] = {range_of(a, M * K), range_of(b, N * K), range_of(a_scale, M * 4),
                            range_of(b_scale, N * 4),
                            bias != nullptr ? range_of(bias, N * 2) : Range{0, 0}};
    for (const Range& r : reads)
        if (overlap(o, r)) return RRF_ERR_ALIAS;
    return RRF_OK;
}

extern "C" rrf_status rrf_scaled_mm_fp8(const void* a, const float* a_scale, const void* b,
                                        const float* b_scale, const void* bias, void* out,
                                        int64_t M, int64_t N, int64_t K, rrf_stream_t stream) {
    rrf_status st = rrf_check_scaled_mm_args(a, a_scale, b, b_scale, bias, out, M, N, K);
    if (st != RRF_OK || M == 0) return st;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    unsigned int* err = nullptr;
    if ((st = device_error_word(&err)) != RRF_OK) return st;
    GemmArgs g = {};
    g.a_scale = a_scale;
    g.b_scale = b_scale;
    g.bias = static_cast<const uint16_t*>(bias);
    g.out = static_cast<uint16_t*>(out);
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.err = err;
    g.starve = take_starve_gemm();
    cudaError_t e;
    if (!take_injected_failure(&e)) e = launch_scaled_mm(g, a, b, sm_count, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_plan_scaled_mm(int64_t M, int64_t N, int64_t K, int mx, int sm_count,
                                         int* kernel, int* a_rows, int* tile_n,
                                         int* k_tiles_per_stage, int64_t* tiles,
                                         int64_t* ctas) {
    if (!kernel || !a_rows || !tile_n || !k_tiles_per_stage || !tiles || !ctas)
        return RRF_ERR_NULL;
    // the calls' own shape rules, checked without operands
    const rrf_status st = mx ? rrf_check_scaled_mm_mx_args(nullptr, nullptr, nullptr, nullptr,
                                                            nullptr, nullptr, M, N, K)
                             : rrf_check_scaled_mm_args(nullptr, nullptr, nullptr, nullptr,
                                                        nullptr, nullptr, M, N, K);
    if (st != RRF_OK && st != RRF_ERR_NULL) return st;
    if (sm_count < 2) return RRF_ERR_UNSUPPORTED;
    if (M == 0) {
        *kernel = *a_rows = *tile_n = *k_tiles_per_stage = 0;
        *tiles = *ctas = 0;
        return RRF_OK;
    }
    const GemmPlan p = plan_scaled_mm(M, N, K, mx != 0, sm_count);
    *kernel = p.kernel;
    *a_rows = p.a_rows;
    *tile_n = p.tile_n;
    *k_tiles_per_stage = p.k_tiles_per_stage;
    *tiles = p.tiles;
    *ctas = p.ctas;
    return RRF_OK;
}

extern "C" rrf_status rrf_check_scaled_mm_mx_args(const void* a, const void* sa,
                                                  const void* b, const void* sb,
                                                  const void* bias, const void* out, int64_t M,
                                                  int64_t N, int64_t K) {
    if (M < 0 || N < 16 || K < 128 || N % 16 != 0 || K % 128 != 0) return RRF_ERR_SHAPE;
    if (M > 65535LL * 128 || N > (int64_t)INT32_MAX / 2 || K > (int64_t)INT32_MAX / 2)
        return RRF_ERR_SHAPE;
    if (M == 0) return RRF_OK;
    if (!a || !sa || !b || !sb || !out) return RRF_ERR_NULL;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(sa, 16) ||
        !aligned(sb, 16) || (bias != nullptr && !aligned(bias, 2)))
        return RRF_ERR_ALIGN;
    const Range o = range_of(out, M * N * 2);
    const Range reads[5] = {range_of(a, M * K), range_of(b, N * K),
                            range_of(sa, RRF_MX_BLOCKED_BYTES(M, K)),
                            range_of(sb, RRF_MX_BLOCKED_BYTES(N, K)),
                            bias != nullptr ? range_of(bias, N * 2) : Range{0, 0}};
    for (const Range& r : reads)
        if (overlap(o, r)) return RRF_ERR_ALIAS;
    return RRF_OK;
}

extern "C" rrf_status rrf_scaled_mm_mxfp8(const void* a, const void* sa, const void* b,
                                          const void* sb, const void* bias, void* out, int64_t M,
                                          int64_t N, int64_t K, rrf_stream_t stream) {
    rrf_status st = rrf_check_scaled_mm_mx_args(a, sa, b, sb, bias, out, M, N, K);
    if (st != RRF_OK || M == 0) return st;
    int sm_count = 0;
    if ((st = current_sm_count(&sm_count)) != RRF_OK) return st;
    unsigned int* err = nullptr;
    if ((st = device_error_word(&err)) != RRF_OK) return st;
    GemmArgs g = {};
    g.bias = static_cast<const uint16_t*>(bias);
    g.out = static_cast<uint16_t*>(out);
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.err = err;
    g.starve = take_starve_gemm();
    cudaError_t e;
    if (!take_injected_failure(&e))
        e = launch_scaled_mm_mx(g, a, b, static_cast<const uint8_t*>(sa),
                                static_cast<const uint8_t*>(sb), sm_count, (cudaStream_t)stream);
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" rrf_status rrf_plan_fused_ex(int num_inputs, int64_t rows, int64_t cols,
                                        int residual, int sm_count, int* cluster_size,
                                        int* block_threads, int* vecs_per_thread,
                                        int* prefetch) {
    if (!cluster_size || !block_threads || !vecs_per_thread || !prefetch) return RRF_ERR_NULL;
    FusedLaunch l = {};
    rrf_status st = plan_fused(num_inputs, rows, cols, sm_count, residual != 0, &l);
    if (st != RRF_OK) return st;
    *cluster_size = l.cluster;
    *block_threads = l.threads;
    *vecs_per_thread = l.vecs_per_thread;
    *prefetch = l.prefetch ? 1 : 0;
    return RRF_OK;
}

extern "C" rrf_status rrf_plan_fused(int num_inputs, int64_t rows, int64_t cols, int residual,
                                     int sm_count, int* cluster_size, int* block_threads,
                                     int* vecs_per_thread) {
    int prefetch = 0;
    return rrf_plan_fused_ex(num_inputs, rows, cols, residual, sm_count, cluster_size,
                             block_threads, vecs_per_thread, &prefetch);
}

extern "C" const char* rrf_status_string(rrf_status status) {
    switch (status) {
        case RRF_OK: return "ok";
        case RRF_ERR_NULL: return "a required pointer is null (or only one residual pointer given)";
        case RRF_ERR_RANKS: return "num_inputs outside [1, 16]";
        case RRF_ERR_SHAPE: return "invalid shape: rows < 0, cols <= 0, cols % 8 != 0, or too large";
        case RRF_ERR_ALIGN: return "misaligned pointer: data needs 16 bytes, scales 4 bytes";
        case RRF_ERR_ALIAS: return "an output overlaps an input or another output";
        case RRF_ERR_VALUE: return "invalid scalar: eps < 0 or not finite, scale_ub <= 0 or NaN, weight_offset not finite";
        case RRF_ERR_UNSUPPORTED: return "the forced launch cannot cover this shape";
        case RRF_ERR_CUDA: return "a CUDA call failed (see rrf_last_cuda_error)";
    }
    return "unknown status";
}

extern "C" int rrf_last_cuda_error(void) { return t_last_cuda_error; }

extern "C" rrf_status rrf_device_error(unsigned int* flags, int clear) {
    if (flags == nullptr) return RRF_ERR_NULL;
    unsigned int* word = nullptr;
    rrf_status st = device_error_word(&word);
    if (st != RRF_OK) return st;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(flags, word, sizeof *flags, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear) e = cudaMemset(word, 0, sizeof *word);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return e == cudaSuccess ? RRF_OK : cuda_fail(e);
}

extern "C" void rrf_debug_fail_next_launch(int cuda_error) { t_fail_next_launch = cuda_error; }

extern "C" void rrf_debug_starve_next_gemm(void) { t_starve_next_gemm = true; }

extern "C" const char* rrf_version(void) { return "0.1.0"; }
