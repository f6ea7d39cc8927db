// rrf_fused.cu -- the fused bf16 sum + residual + RMSNorm + per-row FP8 kernel.
//
// One row is covered by C blocks (C = 1: one block per row; C > 1: a
// thread-block cluster, the row's statistics meeting in distributed shared
// memory).  Each block owns a contiguous slice of the row's 16-byte vectors;
// each thread owns up to VPT of them, strided by the block size so that a
// warp's accesses are contiguous.  Every input byte is read from HBM once;
// the row's bf16 norm input h stays in registers between the two passes:
//   1. load the R inputs, the residual and gamma; fp32 sum in rank order,
//      round to bf16, add the residual and round again, store residual_out;
//      accumulate the sum of squares and the largest |h * (gamma +
//      weight_offset)|;
//   2. after one reduction of both statistics (warp -> block -> cluster):
//      r = 1 / sqrt(mean + eps), amax = r * max |h * g'|,
//      scale = max(min(amax, scale_ub), 1e-12) / 448, and the codes of
//      y = (h * r) * (gamma + weight_offset) times 1 / scale.  Sources:
// Modular docs `allreduce_rmsnorm_fp8` (one launch, no HBM round trip between
// the reduction and the norm), b12x PR #283 (fixed-order fp32, round once),
// TensorRT-LLM PR #19836 (cluster partial-sum exchange and its barrier rules).
#include <cuda_runtime.h>

#include <atomic>

#include "rrf_device.cuh"
#include "rrf_internal.h"

#ifndef RRF_RB
#error "compile with -DRRF_RB=<2|4|8|16>"
#endif

namespace rrf {
namespace {

// E8M0 code of an MX block's shared scale 2^(floor(log2(amax)) - 8) (OCP MX
// v1.0, e4m3 elements: 448 = 1.75 * 2^8): the biased exponent field of
// amax minus 8, clamped at 0 (zero, subnormal and tiny maxima).
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
    return e > 8 ? (uint32_t)(e - 8) : 0u;
}

// The 8 codes of one vector: y = (h * r) * (gamma + weight_offset), then
// y * m (m = 1 / scale, or 1 / X of an MX block), each product rounded once.
template <bool PACKED>
__device__ __forceinline__ uint2 quantise_vector(uint4 h, uint4 g, float r, float wo, float m) {
    if constexpr (PACKED) {
        const float2 r2 = make_float2(r, r), w2 = make_float2(wo, wo), m2 = make_float2(m, m);
        float2 hf[4], gf[4], qv[4];
        bf16x8_to_f32x2(h, hf);
        bf16x8_to_f32x2(g, gf);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            qv[e] = __fmul2_rn(__fmul2_rn(__fmul2_rn(hf[e], r2), __fadd2_rn(gf[e], w2)), m2);
        return f32x2_to_e4m3x8(qv);
    } else {
        float hf[8], gf[8], qv[8];
        bf16x8_to_f32(h, hf);
        bf16x8_to_f32(g, gf);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            qv[e] = __fmul_rn(__fmul_rn(__fmul_rn(hf[e], r), __fadd_rn(gf[e], wo)), m);
        return f32_to_e4m3x8(qv);
    }
}

// The same from h and g' = gamma + weight_offset held as fp32 pairs.
__device__ __forceinline__ uint2 quantise_pairs(const float2 hf[4], const float2 gp[4], float r,
                                                float m) {
    const float2 r2 = make_float2(r, r), m2 = make_float2(m, m);
    float2 qv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[e] = __fmul2_rn(__fmul2_rn(__fmul2_rn(hf[e], r2), gp[e]), m2);
    return f32x2_to_e4m3x8(qv);
}

// ASYNC (cluster rows only): the blocks of a cluster meet through the
// transaction-counted exchange (st.async into the peers' shared memory,
// bounded mbarrier waits) instead of a cluster barrier phase.
// MX: the output takes one E8M0 scale per 32 elements (4 vectors held by 4
// consecutive lanes) instead of one scale per row.
template <int RB, int VPT, bool RES, bool CLUSTER, bool ASYNC, bool MX = false>
__global__ void __launch_bounds__(fused_max_threads(RB, VPT)) fused_kernel(const FusedArgs a) {
    static_assert(CLUSTER || !ASYNC, "the exchange is between the blocks of a cluster");
    __shared__ RowStats warp_stats[32];
    __shared__ RowStats cluster_stats[16];
    __shared__ uint64_t exchange_bar;

    if (CLUSTER) {
        if (ASYNC && threadIdx.x == 0) {
            // one arrival (this one) and C blocks' 8 bytes of statistics
            mbar_init(&exchange_bar, 1);
            mbar_arrive_expect_tx(&exchange_bar, 8u * (uint32_t)(a.cluster + a.starve));
            fence_mbar_init_cluster();
        }
        // Phase 0 of the cluster barrier: this block has started (and set up
        // its exchange barrier).  Its wait comes just before the first write
        // into a peer's shared memory.
        cluster_arrive_relaxed();
    }
    const int tid = threadIdx.x;
    const int T = blockDim.x;
    const uint32_t rank = CLUSTER ? cluster_rank() : 0u;
    const int64_t row = CLUSTER ? (int64_t)(blockIdx.x / a.cluster) : (int64_t)blockIdx.x;
    if (a.prefetch) {
        // Ask L2 for this block's slice of every input, the residual and
        // gamma while the previous kernel may still run: a hint that changes
        // no value read after the wait, and the fetch from HBM overlaps that
        // kernel's tail instead of following it.
        const int pb = (int)rank * a.slice_vecs;
        const int pn = min(a.slice_vecs, a.vecs - pb);
        if (pn > 0) {
            const int64_t off = row * (int64_t)a.vecs + pb;
            const uint32_t bytes = (uint32_t)pn * 16u;
            if (tid < a.R) prefetch_l2(a.in[tid] + off, bytes);
            else if (RES && tid == a.R) prefetch_l2(a.res_in + off, bytes);
            else if (tid == a.R + 1) prefetch_l2(a.gamma + pb, bytes);
        }
    }
    // With programmatic dependent launch this block may run ahead of the
    // previous kernel: wait for it before any global access, then let the
    // next kernel launch early (it waits for this grid the same way).
    wait_for_previous_grid();
    allow_next_grid();

    // Every address below derives from these two, taken after the wait.
    const int v_begin = opaque((int)rank * a.slice_vecs);
    const int v_end = min(v_begin + a.slice_vecs, a.vecs);
    const int64_t row_base = opaque(row * (int64_t)a.vecs);
    // One vector per thread keeps gamma in registers between the passes;
    // longer slices re-read it (an L1 hit) to save registers.
    constexpr bool KEEP_GAMMA = VPT == 1;
    // Packed fp32 pairs (the scalar operations' bits in half the
    // instructions) where a thread holds one vector: the decode-sized calls
    // are bound by that chain (0.05-0.17 us per call less on B200).  With
    // several vectors per thread (prefill rows) the scalar form measured
    // faster (209 against 220-230 us at 8 x 8192 x 8192).
    constexpr bool PACKED = VPT == 1;

    uint4 h[VPT];
    uint4 g[KEEP_GAMMA ? VPT : 1];
    // PACKED: the vector's h and g' = gamma + weight_offset also stay as fp32
    // pairs between the passes, so the last pass does not unpack them again
    float2 hk[PACKED ? 4 : 1], gk[PACKED ? 4 : 1];
    RowStats st = stats_empty();
    // MX: max |h * g'| over each vector's 32-element block (4 lanes)
    float bkey[MX ? VPT : 1];

    // ---- pass 1: sum, residual, sum of squares, max |h * g'|
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = v_begin + tid + k * T;
        if (v < v_end && RRF_IN_BOUNDS(v >= 0 && v < a.vecs && row < a.rows, a.err)) {
            uint4 x[RB];
#pragma unroll
            for (int r = 0; r < RB; ++r)
                if (r < a.R) x[r] = ld_once(a.in[r] + row_base + v);
            uint4 res;
            if (RES) res = ld_once_coherent(a.res_in + row_base + v);
            const uint4 gv = ld_shared_by_all(a.gamma + v);
            if (KEEP_GAMMA) g[k] = gv;

            uint4 s;
            if constexpr (PACKED) {
                float2 acc[4];
                bf16x8_to_f32x2(x[0], acc);
#pragma unroll
                for (int r = 1; r < RB; ++r)
                    if (r < a.R) add_bf16x8_x2(acc, x[r]);
                s = f32x2_to_bf16x8(acc);
            } else {
                float acc[8];
                bf16x8_to_f32(x[0], acc);
#pragma unroll
                for (int r = 1; r < RB; ++r)
                    if (r < a.R) add_bf16x8(acc, x[r]);
                s = f32_to_bf16x8(acc);
            }
            if (RES) {
                if constexpr (PACKED) {
                    float2 t[4];
                    bf16x8_to_f32x2(s, t);
                    add_bf16x8_x2(t, res);
                    s = f32x2_to_bf16x8(t);
                } else {
                    float t[8];
                    bf16x8_to_f32(s, t);
                    add_bf16x8(t, res);
                    s = f32_to_bf16x8(t);
                }
                // Cluster rows store the residual in the last pass, after the
                // exchange: with the barrier exchange its release would
                // otherwise wait for the store to land, and with either
                // exchange the early stores measured slower on B200 (0.1-0.2 us
                // at 32-64 rows of 7168 columns).  The statistics-only form
                // has no last pass.
                if (!CLUSTER || a.stats_only) st_once(a.res_out + row_base + v, s);
            } else if (a.stats_only) {
                st_once(a.h_out + row_base + v, s);
            }
            h[k] = s;
            // max |h * g'| of the vector's 8 elements, g' = gamma + weight_offset
            float vkey = 0.0f;
            if constexpr (PACKED) {
                float2 gf[4];
                bf16x8_to_f32x2(s, hk);
                bf16x8_to_f32x2(gv, gf);
                st.ss += sumsq_bf16x8_x2(hk);
                const float2 wo2 = make_float2(a.weight_offset, a.weight_offset);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    gk[e] = __fadd2_rn(gf[e], wo2);
                    const float2 p = __fmul2_rn(hk[e], gk[e]);
                    vkey = fmaxf(vkey, fmaxf(fabsf(p.x), fabsf(p.y)));
                }
            } else {
                float hf[8], gf[8];
                bf16x8_to_f32(s, hf);
                bf16x8_to_f32(gv, gf);
                st.ss += sumsq_bf16x8(s);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    vkey = fmaxf(vkey, fabsf(__fmul_rn(hf[e], __fadd_rn(gf[e], a.weight_offset))));
            }
            if constexpr (MX) bkey[k] = vkey;
            st.key = fmaxf(st.key, vkey);
        } else if constexpr (MX) {
            bkey[k] = 0.0f;
        }
    }
    if constexpr (MX) {
        // A 32-element block is the vectors of lanes 4i .. 4i+3 (slices and
        // block sizes are multiples of 4 vectors); every lane shuffles.
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            bkey[k] = fmaxf(bkey[k], __shfl_xor_sync(0xFFFFFFFFu, bkey[k], 1));
            bkey[k] = fmaxf(bkey[k], __shfl_xor_sync(0xFFFFFFFFu, bkey[k], 2));
        }
    }

    // ---- reduction of the statistics: block, then cluster
    // (a block has at most 32 warps: their slots in warp_stats)
    (void)RRF_IN_BOUNDS(blockDim.x <= 1024, a.err);
    st = block_stats(st, warp_stats);
    if (CLUSTER) {
        // the cluster's slots: C <= 16 blocks, this block's slot inside them
        // (a failed check leaves the exchange to run out its bounded wait)
        (void)RRF_IN_BOUNDS(a.cluster <= 16 && rank < (uint32_t)a.cluster, a.err);
        cluster_wait_acquire();  // phase 0 done: every block of the cluster runs
        st = ASYNC ? cluster_stats_async(st, cluster_stats, &exchange_bar, rank, a.cluster, a.err)
                   : cluster_stats_combine(st, cluster_stats, rank, a.cluster);
    }
    if (a.stats_only) {
        // first phase of the sharded norm: this shard's row statistics
        if (tid == 0 && rank == 0 && RRF_IN_BOUNDS(row < a.rows, a.err))
            a.stats[row] = make_float2(st.ss, st.key);
        return;
    }
    // max_j |y_j| = max_j |(h_j * r) * g'_j| = r * max_j |h_j * g'_j| up to the
    // order of the two roundings (row_scale)
    const RowScale rs = row_scale(st.ss, st.key, a.inv_cols, a.eps, a.scale_ub);
    const float rinv = rs.rinv, scale = rs.scale, inv_scale = rs.inv_scale;

    // ---- last pass: quantise
    if constexpr (MX) {
        // The block's max |y| is r * its max |h * g'| (the same two products
        // rounded in the other order, as for the row scale).
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = v_begin + tid + k * T;
            if (v < v_end && RRF_IN_BOUNDS(v >= 0 && v < a.vecs && row < a.rows, a.err)) {
                const uint32_t code = mx_scale_code(__fmul_rn(bkey[k], rinv));
                const float inv_x = __uint_as_float((254u - code) << 23);  // 2^(127 - code)
                st_once(a.q + row_base + v,
                        PACKED ? quantise_pairs(hk, gk, rinv, inv_x)
                               : quantise_vector<PACKED>(
                                     h[k], KEEP_GAMMA ? g[k] : ld_shared_by_all(a.gamma + v),
                                     rinv, a.weight_offset, inv_x));
                if ((v & 3) == 0) {
                    // row-major [rows, cols / 32], or the tensor cores' blocked
                    // order (512-byte atoms of 128 rows x 4 blocks)
                    const int64_t j = v >> 2;
                    const int64_t off =
                        a.mx_blocked
                            ? ((row >> 7) * (a.vecs >> 4) + (j >> 2)) * 512 + (row & 31) * 16 +
                                  ((row >> 5) & 3) * 4 + (j & 3)
                            : (row_base + v) >> 2;
                    // (the scale buffer: rows, or rows rounded up to 128, of cols / 32)
                    if (RRF_IN_BOUNDS(off >= 0 && off < (a.mx_blocked ? (a.rows + 127) / 128 * 128
                                                                      : a.rows) *
                                                             (a.vecs >> 2),
                                      a.err))
                        a.scales_mx[off] = (uint8_t)code;
                }
                if (RES && CLUSTER) st_once(a.res_out + row_base + v, h[k]);
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = v_begin + tid + k * T;
            if (v < v_end && RRF_IN_BOUNDS(v >= 0 && v < a.vecs && row < a.rows, a.err)) {
                st_once(a.q + row_base + v,
                        PACKED ? quantise_pairs(hk, gk, rinv, inv_scale)
                               : quantise_vector<PACKED>(
                                     h[k], KEEP_GAMMA ? g[k] : ld_shared_by_all(a.gamma + v),
                                     rinv, a.weight_offset, inv_scale));
                if (RES && CLUSTER) st_once(a.res_out + row_base + v, h[k]);
            }
        }
        if (tid == 0 && rank == 0 && RRF_IN_BOUNDS(row < a.rows, a.err)) a.scales[row] = scale;
    }
}

template <int RB, int VPT, bool RES, bool CLUSTER, bool ASYNC, bool MX>
cudaError_t launch_one(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                       cudaStream_t stream) {
    auto kernel = fused_kernel<RB, VPT, RES, CLUSTER, ASYNC, MX>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * l.cluster), 1, 1);
    cfg.blockDim = dim3((unsigned)l.threads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (l.pdl) {
        attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
        ++cfg.numAttrs;
    }
    if (CLUSTER) {
        if (l.cluster > 8) {
            // Clusters of 16 are outside the portable limit of 8 and must be
            // enabled once per kernel and device.
            static std::atomic<uint64_t> enabled_on{0};
            int dev = 0;
            cudaError_t e = cudaGetDevice(&dev);
            if (e != cudaSuccess) return e;
            const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
            if (bit == 0 || (enabled_on.load(std::memory_order_relaxed) & bit) == 0) {
                e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
                if (e != cudaSuccess) return e;
                enabled_on.fetch_or(bit, std::memory_order_relaxed);
            }
        }
        attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
        attr[cfg.numAttrs].val.clusterDim.x = (unsigned)l.cluster;
        attr[cfg.numAttrs].val.clusterDim.y = 1;
        attr[cfg.numAttrs].val.clusterDim.z = 1;
        ++cfg.numAttrs;
    }
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <int RB, bool RES, bool CLUSTER, bool ASYNC, bool MX>
cudaError_t launch_vpt(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                       cudaStream_t stream) {
    switch (l.vecs_per_thread) {
        case 1: return launch_one<RB, 1, RES, CLUSTER, ASYNC, MX>(a, rows, l, stream);
        case 2: return launch_one<RB, 2, RES, CLUSTER, ASYNC, MX>(a, rows, l, stream);
        case 4: return launch_one<RB, 4, RES, CLUSTER, ASYNC, MX>(a, rows, l, stream);
        case 8: return launch_one<RB, 8, RES, CLUSTER, ASYNC, MX>(a, rows, l, stream);
        default: return cudaErrorInvalidValue;
    }
}

// The MX output exists with one block per row or the transaction-counted
// cluster exchange (the library's choice); the barrier exchange is a test
// and benchmark option of the row-scaled output only.
template <int RB, bool RES>
cudaError_t launch_shape(const FusedArgs& a, int64_t rows, const FusedLaunch& l,
                         cudaStream_t stream) {
    if (l.mx) {
        if (l.cluster == 1) return launch_vpt<RB, RES, false, false, true>(a, rows, l, stream);
        if (!l.async_exchange) return cudaErrorInvalidValue;
        return launch_vpt<RB, RES, true, true, true>(a, rows, l, stream);
    }
    if (l.cluster == 1) return launch_vpt<RB, RES, false, false, false>(a, rows, l, stream);
    return l.async_exchange ? launch_vpt<RB, RES, true, true, false>(a, rows, l, stream)
                            : launch_vpt<RB, RES, true, false, false>(a, rows, l, stream);
}

}  // namespace

// This translation unit is compiled once per input bound (RRF_RB = 2, 4, 8,
// 16) so the instantiations build in parallel; it defines launch_fused_rb<RB>.
#define RRF_CAT2(a, b) a##b
#define RRF_CAT(a, b) RRF_CAT2(a, b)
cudaError_t RRF_CAT(launch_fused_rb, RRF_RB)(const FusedArgs& a, int64_t rows,
                                             const FusedLaunch& l, bool residual,
                                             cudaStream_t stream) {
    return residual ? launch_shape<RRF_RB, true>(a, rows, l, stream)
                    : launch_shape<RRF_RB, false>(a, rows, l, stream);
}

}  // namespace rrf
