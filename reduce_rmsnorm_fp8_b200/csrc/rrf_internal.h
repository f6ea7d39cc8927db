// rrf_internal.h -- shared between the host API (rrf_api.cu) and the kernel
// translation units (rrf_sum.cu, rrf_fused.cu).  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rrf.h"

namespace rrf {

// Everything a launch needs, passed by value as the kernel parameter.  Input
// pointers address 16-byte vectors of 8 bf16 elements.
struct SumArgs {
    const uint4* in[RRF_MAX_INPUTS];
    uint4* out;
    int R;
    int64_t n_vecs;  // rows * cols / 8
};

struct FusedArgs {
    const uint4* in[RRF_MAX_INPUTS];
    const uint4* res_in;   // null without a residual
    uint4* res_out;        // null without a residual
    const uint4* gamma;    // [cols / 8]
    uint2* q;              // 8 e4m3fn codes per 16-byte input vector
    float* scales;         // [rows]
    int R;
    int vecs;              // cols / 8 (vectors per row)
    int slice_vecs;        // vectors per block of a row's cluster: ceil(vecs / C)
    int cluster;           // C, blocks per row (1 = no cluster)
    float inv_cols;        // 1 / cols rounded to fp32: the mean square is sum * inv_cols
    float eps;
    float weight_offset;
    float scale_ub;
    unsigned int* err;     // the library's device error word
    int starve;            // test hook: exchange values a block waits for beyond C
    // Statistics-only form (the first phase of the sharded norm): instead of
    // codes and scales the kernel writes each row's (sum h^2, max |h g'|) and,
    // without a residual, the bf16 norm input h itself.
    int stats_only;
    float2* stats;         // [rows]
    uint4* h_out;          // [rows, cols] or null (with a residual, res_out holds h)
    // MX output: one E8M0 scale code per 32 elements instead of scales
    uint8_t* scales_mx;    // [rows, cols / 32], or blocked (mx_blocked)
    int mx_blocked;        // scales in the block-scaled MMA's 512-byte atom order
    int prefetch;          // prefetch the block's slice into L2 before the PDL wait
    int64_t rows;          // rows of the call (the bounds-checking build's limit)
};

// The second phase of the sharded norm: quantise one column shard from the
// statistics of every shard.
struct PostArgs {
    const uint4* h;        // bf16 norm input of this shard [rows, cols]
    const uint4* gamma;    // this shard's gamma [cols]
    const float2* stats;   // [shards, rows]: (sum h^2, max |h g'|) per shard
    uint2* q;              // [rows, cols] codes
    float* scales;         // [rows] or null (another shard writes them)
    int64_t rows;
    int vecs;              // cols / 8
    int shards;
    float inv_total_cols;  // 1 / (columns of the whole row, all shards), rounded to fp32
    float eps;
    float weight_offset;
    float scale_ub;
    unsigned int* err;     // the library's device error word
    int prefetch;          // prefetch the block's h and gamma into L2 before the PDL wait
};

// The multi-GPU form (rrf_allreduce.cu).  Pointer arrays are indexed by rank
// and hold each rank's buffer as this GPU addresses it (a peer mapping, or,
// with several ranks in one launch, another buffer of this GPU).
struct ArArgs {
    const uint4* in[RRF_AR_MAX_WORLD];      // partials [rows, cols]
    const uint4* res_in[RRF_AR_MAX_WORLD];  // residuals, or null
    uint4* res_out[RRF_AR_MAX_WORLD];
    uint2* q[RRF_AR_MAX_WORLD];             // codes [rows, cols]
    float* scales[RRF_AR_MAX_WORLD];        // [rows]
    unsigned int* sig[RRF_AR_MAX_WORLD];    // signal pads
    const uint4* gamma;
    int world;
    int rank0;             // first rank this launch runs
    int blocks;            // blocks per rank (G, a multiple of the cluster size)
    int two_shot;
    int64_t rows;
    int64_t rows_per_rank; // two-shot: ceil(rows / world)
    int vecs;
    int slice_vecs;
    int cluster;
    float inv_cols;        // 1 / cols rounded to fp32
    float eps;
    float weight_offset;
    float scale_ub;
    unsigned long long timeout_ns;
    unsigned int* err;
};

struct ArLaunch {
    int two_shot;
    int cluster;          // blocks per row (1, 2, 4 or 8)
    int threads;
    int vecs_per_thread;  // 1, 2 or 4
    int blocks;           // per rank
    int local_ranks;      // ranks in one launch
    bool residual;
};

// Largest block of the multi-GPU kernel (RRF_AR_MAX_WORLD loads in flight
// and up to 4 vectors per thread fit the register budget of 512 threads).
constexpr int kArMaxThreads = 512;

// The FP8 GEMM (rrf_gemm.cu); the operands themselves reach the kernel as
// tensor maps.
struct GemmArgs {
    const float* a_scale;  // [M]
    const float* b_scale;  // [N]
    const uint16_t* bias;  // bf16 [N] or null
    uint16_t* out;         // bf16 [M, N]
    int M, N, K;
    unsigned int* err;
    int starve;            // test hook: the epilogue's extra wait runs out
};

struct FusedLaunch {
    int cluster;          // blocks per row
    int threads;          // threads per block
    int vecs_per_thread;  // 1, 2, 4 or 8
    bool pdl;             // launch with programmatic stream serialization
    bool async_exchange;  // clusters meet through st.async + mbarrier waits
    bool mx = false;      // MX output (per-32-element scales)
    bool prefetch = false;  // L2 prefetch of each block's slice before the PDL wait
};

// The fused kernel is compiled for input-count bounds RB in {2, 4, 8, 16}
// (inputs past R are predicated off) and VPT in {1, 2, 4, 8} vectors per
// thread.
constexpr int input_bound(int R) { return R <= 2 ? 2 : (R <= 4 ? 4 : (R <= 8 ? 8 : 16)); }

// Largest block the fused kernel is compiled for: a thread holds RB loads in
// flight and VPT vectors of its row slice in registers, so the register
// budget per thread (65536 / threads) must grow with both.  Chosen from the
// ptxas register counts so that no instantiation spills more than a few bytes.
constexpr int fused_max_threads(int rb, int vpt) {
    return rb <= 4 ? (vpt <= 4 ? 1024 : 512)
                   : (rb == 8 ? (vpt <= 2 ? 1024 : (vpt == 4 ? 512 : 256))
                              : (vpt <= 4 ? 512 : 256));
}

// Kernel launchers (one per translation unit).  They return the CUDA error of
// the launch (cudaSuccess when it was enqueued).
cudaError_t launch_sum(const SumArgs& a, int sm_count, bool pdl, cudaStream_t stream);
// One fused launcher per compiled input bound RB (inputs past R are
// predicated off); launch_fused picks the smallest RB >= R.
cudaError_t launch_fused_rb2(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                             bool residual, cudaStream_t stream);
cudaError_t launch_fused_rb4(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                             bool residual, cudaStream_t stream);
cudaError_t launch_fused_rb8(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                             bool residual, cudaStream_t stream);
cudaError_t launch_fused_rb16(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                              bool residual, cudaStream_t stream);
cudaError_t launch_fused(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                         bool residual, cudaStream_t stream);

cudaError_t launch_post(const PostArgs& a, int sm_count, bool pdl, cudaStream_t stream);

cudaError_t launch_allreduce(const ArArgs& a, const ArLaunch& l, cudaStream_t stream);
// The GEMM kernel a shape takes (pure host arithmetic; the launchers follow
// it).  kernel: kGemmPair (256 x 256 tiles on SM pairs), kGemmTile (a
// persistent CTA per SM walking a_rows-row A stages of 128 x tile_n tiles)
// or kGemmSwap (operands swapped: 64 weight rows on the MMA's M side, the
// call's rows padded to a_rows on its N side); k_tiles_per_stage k-tiles of
// 128 per TMA box; tiles output tiles over ctas CTAs.
constexpr int kGemmPair = RRF_GEMM_KERNEL_PAIR;
constexpr int kGemmTile = RRF_GEMM_KERNEL_TILE;
constexpr int kGemmSwap = RRF_GEMM_KERNEL_SWAP;
struct GemmPlan {
    int kernel;
    int a_rows;
    int tile_n;
    int k_tiles_per_stage;
    int64_t tiles;
    int64_t ctas;
};
GemmPlan plan_scaled_mm(int64_t M, int64_t N, int64_t K, bool mx, int sm_count);
cudaError_t launch_scaled_mm(const GemmArgs& g, const void* a, const void* b, int sm_count,
                             cudaStream_t stream);
// The MX GEMM: sfa / sfb are the scale codes in the blocked order; g.a_scale
// and g.b_scale are null.
cudaError_t launch_scaled_mm_mx(const GemmArgs& g, const void* a, const void* b,
                                const uint8_t* sfa, const uint8_t* sfb, int sm_count,
                                cudaStream_t stream);
// Blocks of the launch shape `l` that can be resident on the current device
// at once (the occupancy query; nothing is launched).
cudaError_t allreduce_resident_blocks(const ArLaunch& l, int* resident);

// Keep `e` as this host thread's last CUDA error (rrf_last_cuda_error) and
// return RRF_ERR_CUDA.
rrf_status record_cuda_error(cudaError_t e);

// The launch shape the library picks (pure host arithmetic).
rrf_status plan_fused(int R, int64_t rows, int64_t cols, int sm_count, bool residual,
                      FusedLaunch* out);

}  // namespace rrf
