// rrf_post.cu -- the second phase of the sharded norm: quantise one column
// shard of each row from the row statistics of every shard.
//
// The hidden dimension of a row may be split across GPUs (Tenstorrent
// rmsnorm_2d.py, decode_forward / prefill_forward: a pre-all-gather pass
// computes per-device statistics, an all-gather exchanges them, a
// post-all-gather pass normalises).  Here the first phase is the fused
// kernel's statistics-only form (sum, residual, and this shard's
// (sum h^2, max |h * g'|) per row); the statistics of all shards are
// gathered by the caller; this kernel combines them in a fixed order (the
// same butterfly in every warp of every shard, so every shard derives the
// same scale) and writes the codes of its shard.
#include <cuda_runtime.h>

#include "rrf_device.cuh"
#include "rrf_internal.h"

namespace rrf {
namespace {

constexpr int kPostThreads = 128;

__global__ void __launch_bounds__(kPostThreads) post_kernel(const PostArgs a) {
    wait_for_previous_grid();  // see rrf_device.cuh: programmatic dependent launch
    allow_next_grid();

    const int64_t blocks_per_row = (a.vecs + kPostThreads - 1) / kPostThreads;
    const int64_t row = (int64_t)blockIdx.x / blocks_per_row;
    const int v = (int)((int64_t)blockIdx.x % blocks_per_row) * kPostThreads + threadIdx.x;
    const int lane = threadIdx.x & 31;

    // The row's statistics over all shards: lane s (+32k) takes shard s, then a
    // full butterfly -- every warp of every shard reduces the same values in
    // the same order.
    RowStats st = stats_empty();
    for (int s = lane; s < a.shards; s += 32) {
        const float2 p = a.stats[(int64_t)s * a.rows + row];
        st = stats_merge(st, RowStats{p.x, p.y});
    }
    st = stats_butterfly(st, 32);
    const float ms = st.ss / a.total_cols_f;
    const float rinv = 1.0f / sqrtf(ms + a.eps);
    const float amax = __fmul_rn(st.key, rinv);
    const float scale = fmaxf(fminf(amax, a.scale_ub), 1e-12f) / 448.0f;
    const float inv_scale = 1.0f / scale;

    if (v < a.vecs) {
        const int64_t i = row * (int64_t)a.vecs + v;
        float hf[8], gf[8], qv[8];
        bf16x8_to_f32(ld_once(a.h + i), hf);
        bf16x8_to_f32(ld_shared_by_all(a.gamma + v), gf);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float y = __fmul_rn(__fmul_rn(hf[e], rinv), __fadd_rn(gf[e], a.weight_offset));
            qv[e] = __fmul_rn(y, inv_scale);
        }
        st_once(a.q + i, f32_to_e4m3x8(qv));
    }
    if (v == 0 && a.scales != nullptr) a.scales[row] = scale;
}

}  // namespace

cudaError_t launch_post(const PostArgs& a, bool pdl, cudaStream_t stream) {
    const int64_t blocks = a.rows * ((a.vecs + kPostThreads - 1) / kPostThreads);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kPostThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, post_kernel, a);
}

}  // namespace rrf
