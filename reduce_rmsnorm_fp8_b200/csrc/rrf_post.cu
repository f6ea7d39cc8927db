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

constexpr int kPostThreads = 128;         // 4 warps per block
constexpr int kPostVecsPerLane = 2;       // a block's chunk: 64 vectors of each row
constexpr int kPostChunkVecs = 32 * kPostVecsPerLane;

// A block takes 4 * RPW consecutive rows (RPW per warp) and one 64-vector
// chunk of them.  The gathered statistics are shard-major ([shards][rows]
// [2]), so the block's rows are contiguous within each shard: every thread
// stages some of them in shared memory with coalesced loads, then one thread
// per row merges the row's shards in shard order (the same order in every
// block of every shard, so every shard derives the same scale) and derives
// the row's 1/r, scale and 1/scale once; the warps then quantise their rows.
// (Per-row scale work in every thread, and scattered per-row statistics
// reads, measured as the bottlenecks of earlier forms on B200.)
template <int RPW>
__global__ void __launch_bounds__(kPostThreads) post_kernel(const PostArgs a, int chunks) {
    constexpr int RB = 4 * RPW;  // rows per block
    __shared__ float2 stage[RRF_MAX_SHARDS * RB];  // [shard][row]
    __shared__ float3 rowval[RB];                  // (1/r, scale, 1/scale)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (a.prefetch) {
        // This block's rows of h and its chunk of gamma to L2 while the
        // previous kernel (normally the all-gather of the statistics; h was
        // written before it) may still run: a hint, no value read after the
        // wait changes.
        const int64_t r0 = (int64_t)(blockIdx.x / chunks) * RB;
        const int c0 = (int)(blockIdx.x % chunks) * kPostChunkVecs;
        const int64_t rows_here = a.rows - r0 < RB ? a.rows - r0 : RB;
        const int nv = a.vecs - c0 < kPostChunkVecs ? a.vecs - c0 : kPostChunkVecs;
        if (tid < rows_here) prefetch_l2(a.h + (r0 + tid) * a.vecs + c0, (uint32_t)nv * 16u);
        else if (tid == RB) prefetch_l2(a.gamma + c0, (uint32_t)nv * 16u);
    }
    wait_for_previous_grid();  // see rrf_device.cuh: programmatic dependent launch
    allow_next_grid();

    // every address derives from these two, taken after the wait
    const int64_t row0 = opaque((int64_t)(blockIdx.x / chunks) * RB);
    const int v0 = opaque((int)(blockIdx.x % chunks) * kPostChunkVecs);
    const int64_t left = a.rows - row0;
    const int nrows = left < RB ? (int)left : RB;

    // the data of this warp's rows and the chunk's gamma first: every global
    // load of the block is in flight before its first barrier
    uint4 gv[kPostVecsPerLane];
#pragma unroll
    for (int j = 0; j < kPostVecsPerLane; ++j) {
        const int v = v0 + lane + 32 * j;
        gv[j] = v < a.vecs ? ld_shared_by_all(a.gamma + v) : make_uint4(0, 0, 0, 0);
    }
    uint4 hv[RPW][kPostVecsPerLane];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int r = warp + 4 * k;
#pragma unroll
        for (int j = 0; j < kPostVecsPerLane; ++j) {
            const int v = v0 + lane + 32 * j;
            if (r < nrows && v < a.vecs &&
                RRF_IN_BOUNDS(row0 + r < a.rows && v >= 0, a.err))
                hv[k][j] = ld_once(a.h + (row0 + r) * a.vecs + v);
        }
    }
    // the statistics of the block's rows, coalesced per shard
    for (int i = tid; i < a.shards * RB; i += kPostThreads) {
        const int s = i / RB, r = i % RB;
        if (!RRF_IN_BOUNDS(i < RRF_MAX_SHARDS * RB, a.err)) break;  // the stage's size
        stage[i] = r < nrows && RRF_IN_BOUNDS(row0 + r < a.rows, a.err)
                       ? a.stats[(int64_t)s * a.rows + row0 + r]
                       : make_float2(0.0f, 0.0f);
    }
    __syncthreads();
    if (tid < nrows) {
        float ss = 0.0f, key = 0.0f;
        for (int s = 0; s < a.shards; ++s) {
            const float2 p = stage[s * RB + tid];
            ss = ss + p.x;
            key = fmaxf(key, p.y);
        }
        const RowScale rs = row_scale(ss, key, a.inv_total_cols, a.eps, a.scale_ub);
        const float scale = rs.scale;
        rowval[tid] = make_float3(rs.rinv, scale, rs.inv_scale);
        if (v0 == 0 && a.scales != nullptr && RRF_IN_BOUNDS(row0 + tid < a.rows, a.err))
            a.scales[row0 + tid] = scale;
    }
    __syncthreads();

#pragma unroll
    for (int k = 0; k < RPW; ++k) {
        const int r = warp + 4 * k;
        if (r >= nrows) break;  // uniform across the warp
        const float3 rv = rowval[r];
#pragma unroll
        for (int j = 0; j < kPostVecsPerLane; ++j) {
            const int v = v0 + lane + 32 * j;
            if (v < a.vecs && RRF_IN_BOUNDS(row0 + r < a.rows && v >= 0, a.err)) {
                float hf[8], gf[8], qv[8];
                bf16x8_to_f32(hv[k][j], hf);
                bf16x8_to_f32(gv[j], gf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float y =
                        __fmul_rn(__fmul_rn(hf[e], rv.x), __fadd_rn(gf[e], a.weight_offset));
                    qv[e] = __fmul_rn(y, rv.z);
                }
                st_once(a.q + (row0 + r) * a.vecs + v, f32_to_e4m3x8(qv));
            }
        }
    }
}

template <int RPW>
cudaError_t launch_rpw(const PostArgs& a, int chunks, bool pdl, cudaStream_t stream) {
    constexpr int RB = 4 * RPW;
    const int64_t blocks = (a.rows + RB - 1) / RB * chunks;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kPostThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, post_kernel<RPW>, a, chunks);
}

}  // namespace

cudaError_t launch_post(const PostArgs& a, int sm_count, bool pdl, cudaStream_t stream) {
    const int chunks = (a.vecs + kPostChunkVecs - 1) / kPostChunkVecs;
    // Four rows per warp once that still gives every SM several blocks; one
    // row per warp for small calls, which are latency-bound.  Small calls
    // (every block resident at once) also prefetch before the wait.
    PostArgs b = a;
    if ((a.rows + 15) / 16 * chunks >= 4 * (int64_t)sm_count) {
        b.prefetch = 0;
        return launch_rpw<4>(b, chunks, pdl, stream);
    }
    b.prefetch = (a.rows + 3) / 4 * chunks <= 8 * (int64_t)sm_count ? 1 : 0;
    return launch_rpw<1>(b, chunks, pdl, stream);
}

}  // namespace rrf
