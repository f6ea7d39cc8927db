// rrf_allreduce.cu -- the multi-GPU form: all-reduce of `world` bf16 partials
// that live on `world` GPUs, fused with the residual, RMSNorm and per-row FP8
// quantisation in one kernel that reads and writes the peers' buffers
// directly (NVLink / NVSwitch loads and stores through peer mappings).
//
// Sources: Modular docs `allreduce_rmsnorm_fp8` (one launch; a 1-stage path
// in which every GPU reduces all rows, and a 2-stage path in which every GPU
// reduces ceil(rows / ngpus) rows and the FP8 rows and scales are gathered);
// b12x PR #283 (each rank takes its share of the rows from every peer and
// accumulates in fp32 in fixed rank order, rounding once); TensorRT-LLM PR
// #19836 (arrivals counted per CTA; one cluster-barrier phase per thread;
// every CTA of a cluster started before its shared memory is written).
//
// Structure of one call on rank k (block b of a persistent grid of G blocks
// per rank; every rank launches the same G):
//   start barrier  block b tells block b of every rank that it runs (so this
//                  rank's input is ready: it was produced earlier in the
//                  rank's stream) and waits until every rank has told it;
//   rows           one-shot: every row, read from all ranks, written to this
//                  rank's outputs; two-shot: rows [k*P, (k+1)*P) with
//                  P = ceil(rows / world), written to every rank's outputs;
//   end barrier    the same after the stores: when every block of rank k has
//                  passed it, every peer block has finished its stores into
//                  k's outputs and its reads of k's input.
// A flag word holds the call's number, which each block keeps in a counter
// word of its own rank's pad and advances at the end of the call: the pads
// are zeroed once, the host passes no number, and a call replayed from a
// CUDA graph is numbered afresh.  Block b's counter has the same history on
// every rank (every rank makes the same calls with the same grid), so block
// b of every rank uses the same number.  Every wait is bounded in time;
// one that runs out sets a bit in the device error word and the kernel goes
// on with the same control flow (no block of a cluster may skip a phase that
// its peers take), so it always finishes.
#include <cuda_runtime.h>

#include "rrf_device.cuh"
#include "rrf_internal.h"

namespace rrf {
namespace {

// ------------------------------------------------------------- signal pads --

// Word (phase, src, block) of a rank's pad: block `block` of rank `src` has
// reached barrier `phase` (0 start, 1 end) of the call numbered by the word.
__device__ __forceinline__ unsigned int* flag_word(unsigned int* pad, int phase, int src,
                                                   int block) {
    return pad + ((size_t)(phase * RRF_AR_MAX_WORLD + src) * RRF_AR_MAX_BLOCKS + block);
}

// The calls block `block` of this rank has completed on this pad.
__device__ __forceinline__ unsigned int* counter_word(unsigned int* pad, int block) {
    return pad + (size_t)2 * RRF_AR_MAX_WORLD * RRF_AR_MAX_BLOCKS + block;
}

__device__ __forceinline__ void st_release_sys(unsigned int* p, unsigned int v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_sys(unsigned int* p, unsigned int v) {
    asm volatile("st.relaxed.sys.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned int ld_relaxed_gpu(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned int ld_acquire_sys(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Barrier `phase` between block `block` of rank `rank` and the same block of
// every rank.  Thread t < world signals rank t and then waits for rank t's
// word in this rank's pad (acquire loads: the flag before every thread's later
// loads, through the __syncthreads after the wait).  At the end barrier the
// signal is a release store, which (after the __syncthreads before it) orders
// every thread's stores into the peers' buffers before the flag.  The start
// barrier orders no store of this kernel: what a peer then reads was written
// by earlier kernels of this rank's stream, which completed before this one
// began.  (On B200 each system-scope release costs about 3 us even with
// nothing to drain, measured with all ranks in one launch; a separate
// __threadfence_system before the release added as much again.)
__device__ void peer_barrier(const ArArgs& a, int phase, int rank, int block,
                             unsigned int call) {
    __syncthreads();
    const int t = threadIdx.x;
    // (the pads' words: world <= RRF_AR_MAX_WORLD ranks, block < RRF_AR_MAX_BLOCKS)
    if (t < a.world && RRF_IN_BOUNDS(a.world <= RRF_AR_MAX_WORLD && rank < a.world &&
                                         block < RRF_AR_MAX_BLOCKS,
                                     a.err)) {
        unsigned int* theirs = flag_word(a.sig[t], phase, rank, block);
        if (phase == 0) st_relaxed_sys(theirs, call);
        else st_release_sys(theirs, call);
        const unsigned int* mine = flag_word(a.sig[rank], phase, t, block);
        if (ld_acquire_sys(mine) != call) {
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_sys(mine) != call) {
                if (global_timer_ns() - t0 > a.timeout_ns) {
                    atomicOr(a.err, RRF_DEVICE_ERROR_PEER_TIMEOUT);
                    break;
                }
            }
        }
    }
    __syncthreads();
}

// Plain 16-byte store (to this GPU's or a peer's memory).
__device__ __forceinline__ void st_any(uint4* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_any(uint2* p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// ------------------------------------------------------------------ kernel --
// One row is covered by C blocks (C = 1, or a cluster of C whose blocks meet
// in distributed shared memory, as in the single-GPU kernel); a cluster walks
// the rows of its rank's range with a stride of the rank's cluster count.
// Each thread holds VPT 16-byte vectors of its block's slice of the row.
// Up to 2 vectors per thread the registers are capped for two 512-thread
// blocks per SM (ptxas: 64 registers, at most 12 bytes spilled), so a
// persistent grid of wide rows still keeps 1024 threads of loads per SM.
template <int VPT, bool RES, bool CLUSTER>
__global__ void __launch_bounds__(kArMaxThreads, VPT <= 2 ? 2 : 1) ar_kernel(const ArArgs a) {
    constexpr int W = RRF_AR_MAX_WORLD;
    constexpr bool KEEP_GAMMA = VPT == 1;
    // Double-buffered by row parity: a fast block may write the next row's
    // statistics while a slow one still reads this row's.
    __shared__ RowStats warp_stats[2][32];
    __shared__ RowStats slots[2][8];

    const int lrank = (int)blockIdx.x / a.blocks;  // rank within this launch
    const int rank = a.rank0 + lrank;
    const int block = (int)blockIdx.x - lrank * a.blocks;
    const int C = CLUSTER ? a.cluster : 1;
    const uint32_t crank = CLUSTER ? cluster_rank() : 0u;
    const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31;
    const int v_begin = (int)crank * a.slice_vecs;
    const int v_end = min(v_begin + a.slice_vecs, a.vecs);

    // This call's number: one more than the calls this block has completed
    // on its rank's pad (written by this block at the end of the previous
    // call, an earlier kernel of the stream).
    __shared__ unsigned int call_s;
    if (tid == 0)
        call_s = RRF_IN_BOUNDS(rank < a.world && block < RRF_AR_MAX_BLOCKS, a.err)
                     ? ld_relaxed_gpu(counter_word(a.sig[rank], block)) + 1u
                     : 0u;
    __syncthreads();
    const unsigned int call = call_s;

    // Cluster phase 0 (every block of the cluster has started) overlaps the
    // start barrier; its wait comes before the first remote shared store.
    if (CLUSTER) cluster_arrive_relaxed();
    peer_barrier(a, 0, rank, block, call);
    if (CLUSTER) cluster_wait_acquire();

    // every address below derives from `first`, taken after the start
    // barrier's acquire (the peers' loads must not move above it)
    const int64_t first = opaque(a.two_shot ? (int64_t)rank * a.rows_per_rank : (int64_t)0);
    const int64_t stop = a.two_shot ? min(first + a.rows_per_rank, a.rows) : a.rows;
    const int nclusters = a.blocks / C;
    const uint4* res_in = RES ? a.res_in[rank] : nullptr;
    int par = 0;
    for (int64_t row = first + block / C; row < stop; row += nclusters, par ^= 1) {
        const int64_t base = row * (int64_t)a.vecs;
        uint4 h[VPT];
        uint4 g[KEEP_GAMMA ? VPT : 1];
        RowStats st = stats_empty();
        // ---- pass 1: the partials of every rank in rank order, the residual
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = v_begin + tid + k * T;
            if (v < v_end && RRF_IN_BOUNDS(v >= 0 && v < a.vecs && row < a.rows, a.err)) {
                uint4 x[W];
#pragma unroll
                for (int j = 0; j < W; ++j)
                    if (j < a.world) x[j] = ld_once_coherent(a.in[j] + base + v);
                uint4 res;
                if (RES) res = ld_once_coherent(res_in + base + v);
                const uint4 gv = ld_shared_by_all(a.gamma + v);
                if (KEEP_GAMMA) g[k] = gv;
                float acc[8];
                bf16x8_to_f32(x[0], acc);
#pragma unroll
                for (int j = 1; j < W; ++j)
                    if (j < a.world) add_bf16x8(acc, x[j]);
                uint4 s = f32_to_bf16x8(acc);
                if (RES) {
                    float t[8];
                    bf16x8_to_f32(s, t);
                    add_bf16x8(t, res);
                    s = f32_to_bf16x8(t);
                }
                h[k] = s;
                st.ss += sumsq_bf16x8(s);
                float hf[8], gf[8];
                bf16x8_to_f32(s, hf);
                bf16x8_to_f32(gv, gf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    stats_offer(st, hf[e], __fadd_rn(gf[e], a.weight_offset));
            }
        }
        // ---- the row's statistics: block, then cluster (one phase per row)
        st = block_stats(st, warp_stats[par]);
        if (CLUSTER) {
            if (tid < C) st_peer_stats(slots[par], crank, tid, st);
            cluster_arrive_release();
            cluster_wait_acquire();
            st = stats_butterfly(slots[par][lane & (C - 1)], C);
        }
        const RowScale rs = row_scale(st.ss, st.key, a.inv_cols, a.eps, a.scale_ub);
        const float rinv = rs.rinv, scale = rs.scale, inv_scale = rs.inv_scale;
        // ---- pass 2: codes; the outputs go to this rank (one-shot) or to
        // every rank (two-shot)
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = v_begin + tid + k * T;
            if (v < v_end && RRF_IN_BOUNDS(v >= 0 && v < a.vecs && row < a.rows, a.err)) {
                float hf[8], gf[8], qv[8];
                bf16x8_to_f32(h[k], hf);
                bf16x8_to_f32(KEEP_GAMMA ? g[k] : ld_shared_by_all(a.gamma + v), gf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float y =
                        __fmul_rn(__fmul_rn(hf[e], rinv), __fadd_rn(gf[e], a.weight_offset));
                    qv[e] = __fmul_rn(y, inv_scale);
                }
                const uint2 code = f32_to_e4m3x8(qv);
                if (a.two_shot) {
#pragma unroll
                    for (int j = 0; j < W; ++j) {
                        if (j < a.world) {
                            st_any(a.q[j] + base + v, code);
                            if (RES) st_any(a.res_out[j] + base + v, h[k]);
                        }
                    }
                } else {
                    st_any(a.q[rank] + base + v, code);
                    if (RES) st_any(a.res_out[rank] + base + v, h[k]);
                }
            }
        }
        if (tid == 0 && crank == 0 && RRF_IN_BOUNDS(row < a.rows, a.err)) {
            if (a.two_shot) {
#pragma unroll
                for (int j = 0; j < W; ++j)
                    if (j < a.world) a.scales[j][row] = scale;
            } else {
                a.scales[rank][row] = scale;
            }
        }
    }
    peer_barrier(a, 1, rank, block, call);
    if (tid == 0 && RRF_IN_BOUNDS(rank < a.world && block < RRF_AR_MAX_BLOCKS, a.err))
        *counter_word(a.sig[rank], block) = call;
}

// Clusters of up to 8 (the portable size) only.
template <int VPT, bool RES, bool CLUSTER>
cudaError_t launch_shape(const ArArgs& a, const ArLaunch& l, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.blocks * l.local_ranks), 1, 1);
    cfg.blockDim = dim3((unsigned)l.threads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (CLUSTER) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)l.cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.numAttrs = 1;
    } else if (l.local_ranks > 1) {
        // Several ranks in one launch wait on one another: a cooperative
        // launch is refused unless all its blocks can be resident at once.
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, ar_kernel<VPT, RES, CLUSTER>, a);
}

template <int VPT, bool RES, bool CLUSTER>
cudaError_t occupancy_shape(const ArLaunch& l, int* resident) {
    if (CLUSTER) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)l.cluster, 1, 1);
        cfg.blockDim = dim3((unsigned)l.threads, 1, 1);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)l.cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        cudaError_t e =
            cudaOccupancyMaxActiveClusters(&clusters, ar_kernel<VPT, RES, CLUSTER>, &cfg);
        *resident = clusters * l.cluster;
        return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, ar_kernel<VPT, RES, CLUSTER>, l.threads, 0);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    *resident = per_sm * sms;
    return cudaSuccess;
}

template <int VPT, bool RES>
cudaError_t dispatch_cluster(const ArArgs* a, const ArLaunch& l, cudaStream_t stream,
                             int* resident) {
    if (l.cluster > 1)
        return a ? launch_shape<VPT, RES, true>(*a, l, stream)
                 : occupancy_shape<VPT, RES, true>(l, resident);
    return a ? launch_shape<VPT, RES, false>(*a, l, stream)
             : occupancy_shape<VPT, RES, false>(l, resident);
}

template <int VPT>
cudaError_t dispatch_res(const ArArgs* a, const ArLaunch& l, cudaStream_t stream,
                         int* resident) {
    return l.residual ? dispatch_cluster<VPT, true>(a, l, stream, resident)
                      : dispatch_cluster<VPT, false>(a, l, stream, resident);
}

// a == nullptr: report the resident-block capacity of the launch shape
// instead of launching.
cudaError_t dispatch(const ArArgs* a, const ArLaunch& l, cudaStream_t stream, int* resident) {
    switch (l.vecs_per_thread) {
        case 1: return dispatch_res<1>(a, l, stream, resident);
        case 2: return dispatch_res<2>(a, l, stream, resident);
        default: return dispatch_res<4>(a, l, stream, resident);
    }
}

}  // namespace

cudaError_t allreduce_resident_blocks(const ArLaunch& l, int* resident) {
    return dispatch(nullptr, l, nullptr, resident);
}

cudaError_t launch_allreduce(const ArArgs& a, const ArLaunch& l, cudaStream_t stream) {
    return dispatch(&a, l, stream, nullptr);
}

}  // namespace rrf
