// rrf_device.cuh -- device-side building blocks of the sum and fused kernels:
// 16-byte memory access, bf16 / e4m3fn conversion, programmatic dependent
// launch, cluster barriers and the warp / block / cluster reduction of a
// row's statistics.  sm_100a only.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace rrf {

// Device error bits (the library's device error word; see rrf_device_error).
constexpr unsigned int kDeviceErrorExchangeTimeout = 1u;
// Set by the bounds-checking build (RRF_DEBUG) when a kernel computed an
// index outside the buffer it was about to access; that access was skipped.
constexpr unsigned int kDeviceErrorBounds = 8u;

// RRF_IN_BOUNDS(ok, err): in a build with RRF_DEBUG defined, `ok` (the
// condition that an index lies inside its buffer) is evaluated and, if it is
// false, the bounds bit is set in the device error word `err` and the macro
// yields false so that the caller skips the access (no trap, no assert: a
// failed check never stops the GPU).  In the normal build it is the constant
// true and `ok` is not evaluated.
#ifdef RRF_DEBUG
__device__ __forceinline__ bool rrf_bounds_check(bool ok, unsigned int* err) {
    if (!ok) atomicOr(err, kDeviceErrorBounds);
    return ok;
}
#define RRF_IN_BOUNDS(ok, err) (::rrf::rrf_bounds_check((ok), (err)))
#else
#define RRF_IN_BOUNDS(ok, err) (true)
#endif

// Bound on a wait for the cluster's statistics: far above the microsecond a
// healthy exchange takes, far below anything that would look like a hang.
constexpr unsigned long long kExchangeWaitLimitNs = 2000000ull;  // 2 ms

// ------------------------------------------------------------------ memory --

// Bulk prefetch of the `bytes` bytes at p (16-byte aligned, a multiple of 16)
// into L2.  No data comes back and nothing waits for it: a hint with no
// effect on the values any load returns, so a kernel may issue it before it
// waits for the previous kernel of its stream (L2 is the GPU's point of
// coherence for its own memory: a line the previous kernel writes afterwards
// is updated in L2).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}

// x, as a value the compiler must take to be produced at this point: the
// address of a load derived from it cannot be formed, so the load cannot be
// issued, before the volatile instructions that precede it (a wait for the
// previous kernel, a barrier's acquire).  The loads below are plain asm that
// the compiler may otherwise schedule freely.
__device__ __forceinline__ int64_t opaque(int64_t x) {
    asm volatile("" : "+l"(x));
    return x;
}

__device__ __forceinline__ int opaque(int x) {
    asm volatile("" : "+r"(x));
    return x;
}

// Streamed 16-byte load of data read exactly once: read-only path, no L1
// allocation, 256-byte L2 prefetch of the surrounding line.
__device__ __forceinline__ uint4 ld_once(const uint4* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// The same for data the kernel may also write (an in-place residual): a
// coherent load, still without L1 allocation.  Each element is loaded once,
// by the thread that later overwrites it, so the load may be scheduled freely.
__device__ __forceinline__ uint4 ld_once_coherent(const uint4* p) {
    uint4 v;
    asm("ld.global.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// 16-byte load of data every block of the grid reads (gamma): read-only path,
// cached.
__device__ __forceinline__ uint4 ld_shared_by_all(const uint4* p) {
    uint4 v;
    asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// Streaming stores (evict-first): results are not re-read by this kernel.
__device__ __forceinline__ void st_once(uint4* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_once(uint2* p, uint2 v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(v.x), "r"(v.y)
                 : "memory");
}

// -------------------------------------------------------------------- bf16 --

// A 16-byte vector holds 8 bf16; 32-bit word k holds elements 2k (low half)
// and 2k+1 (high half).  bf16 -> fp32 widening is exact: the bf16 bits are the
// top half of the fp32 bits.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float f[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f[2 * k] = __uint_as_float(w[k] << 16);
        f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

// Two fp32 -> two bf16, round to nearest even (cvt.rn.bf16x2.f32 puts its
// first source in the upper half).
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint4 f32_to_bf16x8(const float f[8]) {
    uint4 v;
    v.x = f32x2_to_bf16x2(f[0], f[1]);
    v.y = f32x2_to_bf16x2(f[2], f[3]);
    v.z = f32x2_to_bf16x2(f[4], f[5]);
    v.w = f32x2_to_bf16x2(f[6], f[7]);
    return v;
}

// acc += widen(x), one IEEE fp32 add per element (no contraction).
__device__ __forceinline__ void add_bf16x8(float acc[8], const uint4 x) {
    float f[8];
    bf16x8_to_f32(x, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], f[e]);
}

// Sum of squares of 8 bf16 as a balanced tree (each square is exact in fp32).
__device__ __forceinline__ float sumsq_bf16x8(const uint4 v) {
    float f[8];
    bf16x8_to_f32(v, f);
    const float a = __fmaf_rn(f[0], f[0], f[1] * f[1]);
    const float b = __fmaf_rn(f[2], f[2], f[3] * f[3]);
    const float c = __fmaf_rn(f[4], f[4], f[5] * f[5]);
    const float d = __fmaf_rn(f[6], f[6], f[7] * f[7]);
    return (a + b) + (c + d);
}

// ------------------------------------------------------- packed fp32 pairs --
// sm_100a's two-wide FADD / FMUL / FFMA: each half of a pair is one IEEE
// round-to-nearest operation, so the results are the scalar operations' bits
// in half the instructions.  A 16-byte vector of 8 bf16 is handled as 4 pairs
// (elements 2k, 2k+1: the low and high half of word k).

__device__ __forceinline__ void bf16x8_to_f32x2(const uint4 v, float2 f[4]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
        f[k] = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u));
}

__device__ __forceinline__ uint4 f32x2_to_bf16x8(const float2 f[4]) {
    uint4 v;
    v.x = f32x2_to_bf16x2(f[0].x, f[0].y);
    v.y = f32x2_to_bf16x2(f[1].x, f[1].y);
    v.z = f32x2_to_bf16x2(f[2].x, f[2].y);
    v.w = f32x2_to_bf16x2(f[3].x, f[3].y);
    return v;
}

// acc += widen(x), one IEEE fp32 add per element.
__device__ __forceinline__ void add_bf16x8_x2(float2 acc[4], const uint4 x) {
    float2 f[4];
    bf16x8_to_f32x2(x, f);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = __fadd2_rn(acc[k], f[k]);
}

// sumsq_bf16x8 in pairs, the same tree: (a + b) + (c + d) with
// a = f0^2 + f1^2 (one fma over the exact square f1^2), b over f2, f3, c over
// f4, f5, d over f6, f7.
__device__ __forceinline__ float sumsq_bf16x8_x2(const float2 f[4]) {
    const float2 ac = __ffma2_rn(make_float2(f[0].x, f[2].x), make_float2(f[0].x, f[2].x),
                                 __fmul2_rn(make_float2(f[0].y, f[2].y),
                                            make_float2(f[0].y, f[2].y)));
    const float2 bd = __ffma2_rn(make_float2(f[1].x, f[3].x), make_float2(f[1].x, f[3].x),
                                 __fmul2_rn(make_float2(f[1].y, f[3].y),
                                            make_float2(f[1].y, f[3].y)));
    const float2 t = __fadd2_rn(ac, bd);  // (a + b, c + d)
    return t.x + t.y;
}

// ------------------------------------------------------------------ e4m3fn --

// Two fp32 -> two e4m3fn codes, round to nearest even, saturating to +-448
// (cvt.rn.satfinite.e4m3x2.f32 through the cuda_fp8.h intrinsic); the first
// element lands in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint2 f32x2_to_e4m3x8(const float2 f[4]) {
    uint2 q;
    q.x = (uint32_t)__nv_cvt_float2_to_fp8x2(f[0], __NV_SATFINITE, __NV_E4M3) |
          ((uint32_t)__nv_cvt_float2_to_fp8x2(f[1], __NV_SATFINITE, __NV_E4M3) << 16);
    q.y = (uint32_t)__nv_cvt_float2_to_fp8x2(f[2], __NV_SATFINITE, __NV_E4M3) |
          ((uint32_t)__nv_cvt_float2_to_fp8x2(f[3], __NV_SATFINITE, __NV_E4M3) << 16);
    return q;
}

__device__ __forceinline__ uint2 f32_to_e4m3x8(const float f[8]) {
    uint2 q;
    q.x = f32x2_to_e4m3x2(f[0], f[1]) | (f32x2_to_e4m3x2(f[2], f[3]) << 16);
    q.y = f32x2_to_e4m3x2(f[4], f[5]) | (f32x2_to_e4m3x2(f[6], f[7]) << 16);
    return q;
}

// ------------------------------------------------ programmatic dependent launch --
// A kernel launched with programmatic stream serialization may start while the
// previous kernel in the stream is still running.  It must wait for that
// kernel (completion and memory visibility) before it reads or writes global
// memory; without the launch attribute the wait returns at once.

__device__ __forceinline__ void wait_for_previous_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Let the next kernel in the stream be scheduled; it still waits for this
// whole grid before touching memory.
__device__ __forceinline__ void allow_next_grid() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------ thread-block cluster --
// Cluster barrier phases follow the rules the TensorRT-LLM PR #19836 write-up
// spells out: every thread arrives and waits exactly once per phase, no
// thread leaves before the last phase, and a block writes a peer's shared
// memory only after a completed phase has shown that the peer has started.

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ------------------------------------------ transaction-counted exchange --
// The other way for a cluster's blocks to meet: each block pushes its value
// into every peer's shared memory with st.async, which counts the bytes on
// the peer's mbarrier, and waits on its own mbarrier until all C values have
// landed.  No thread waits for the cluster's other threads, and no release
// fence waits for this thread's global stores.  Every wait is bounded in
// time: a wait that runs out sets a bit in the library's device error word
// and the kernel finishes without the missing values instead of hanging.

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t arrivals) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(arrivals)
                 : "memory");
}

// Make this thread's mbarrier initialisations visible to the cluster (for the
// peers' st.async) before the next cluster barrier arrival.
__device__ __forceinline__ void fence_mbar_init_cluster() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival that also announces `bytes` of incoming transactions.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait until phase `parity` of `bar` completes, for at most limit_ns
// nanoseconds; returns false if the wait ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait_cluster(bar, parity))
        if (global_timer_ns() - t0 > limit_ns) return false;
    return true;
}

// Store two floats into shared-memory word pair `local` of cluster block
// `peer` and count 8 bytes on that block's mbarrier `bar` (same offsets in
// every block).
__device__ __forceinline__ void st_async_peer_f32x2(void* local, uint64_t* bar, uint32_t peer,
                                                    float x, float y) {
    uint32_t raddr, rbar;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local)),
                 "r"(peer));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(smem_u32(bar)),
                 "r"(peer));
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
                 :: "r"(raddr), "f"(x), "f"(y), "r"(rbar)
                 : "memory");
}

// --------------------------------------------------------- row statistics --
// What a row's norm needs from all of its elements, reduced in one round: the
// sum of squares of h and the largest |h * g'| (g' = gamma + weight_offset).
// max_j |y_j| with y_j = (h_j * r) * g'_j is then r * max_j |h_j g'_j| up to
// the rounding of the two products (a couple of ulps).
//
// Butterfly (xor) reductions: at every level lane i merges its value with
// lane i ^ off's; fp32 addition and fmaxf are commutative, so every lane ends
// with the same bits, whichever lane reads the result.  A reduction over n
// partials (n a power of two <= 32) runs log2(n) levels on lanes that hold
// partial lane % n, so every lane of the warp ends with the total.

struct __align__(8) RowStats {  // 8-byte aligned: one v2 store per peer
    float ss;   // sum of h^2
    float key;  // max |h * g'|
};

__device__ __forceinline__ RowStats stats_empty() { return RowStats{0.0f, 0.0f}; }

__device__ __forceinline__ void stats_offer(RowStats& s, float h, float g) {
    s.key = fmaxf(s.key, fabsf(__fmul_rn(h, g)));
}

__device__ __forceinline__ RowStats stats_merge(RowStats a, const RowStats& b) {
    a.ss = a.ss + b.ss;
    a.key = fmaxf(a.key, b.key);
    return a;
}

__device__ __forceinline__ RowStats stats_butterfly(RowStats s, int n) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        if (off >= n) break;
        RowStats o;
        o.ss = __shfl_xor_sync(0xFFFFFFFFu, s.ss, off);
        o.key = __shfl_xor_sync(0xFFFFFFFFu, s.key, off);
        s = stats_merge(s, o);
    }
    return s;
}

// Sum and max over the 32 lanes of a warp, every lane getting the result:
// the sum by the same xor butterfly as stats_butterfly (the same bits), the
// max in one instruction (redux.sync.max.f32, sm_100a; like fmaxf it ignores
// a NaN operand unless all are NaN).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) v = v + __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ int pow2_ceil(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Block-wide statistics, returned to every thread (one __syncthreads).
__device__ __forceinline__ RowStats block_stats(RowStats s, RowStats* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    s.ss = warp_sum(s.ss);
    s.key = warp_max(s.key);
    if (lane == 0) scratch[warp] = s;
    __syncthreads();
    const int n = pow2_ceil(nwarps);
    const int i = lane & (n - 1);
    return stats_butterfly(i < nwarps ? scratch[i] : stats_empty(), n);
}

// A row's norm factor, FP8 scale and quantisation multiplier from its
// statistics (ss = sum h^2, key = max |h g'|): the mean square ss * inv_cols
// (inv_cols = 1/cols rounded to fp32), r = rsqrt(mean + eps) (the hardware
// reciprocal square root, within 2 ulp), amax = r * key (max |y| up to the
// order of the two roundings), scale = clamp(amax, scale_ub, 1e-12) *
// fp32(1/448) and 1 / scale.  Against the correctly rounded 1/sqrt and
// divisions this moves a scale by a few ulps, far inside the 1e-6 relative
// tolerance, and takes four dependent IEEE divisions and square roots off
// the end of every row.
struct RowScale {
    float rinv;
    float scale;
    float inv_scale;
};

__device__ __forceinline__ RowScale row_scale(float ss, float key, float inv_cols, float eps,
                                              float scale_ub) {
    RowScale r;
    r.rinv = rsqrtf(__fadd_rn(__fmul_rn(ss, inv_cols), eps));
    const float amax = __fmul_rn(key, r.rinv);
    r.scale = __fmul_rn(fmaxf(fminf(amax, scale_ub), 1e-12f), 1.0f / 448.0f);
    r.inv_scale = 1.0f / r.scale;
    return r;
}

// Store a block's statistics into slot `rank` of cluster block `peer`.
__device__ __forceinline__ void st_peer_stats(RowStats* slots, uint32_t rank, uint32_t peer,
                                              const RowStats& s) {
    const uint32_t laddr = (uint32_t)__cvta_generic_to_shared(&slots[rank]);
    uint32_t raddr;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(laddr), "r"(peer));
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" :: "r"(raddr), "f"(s.ss),
                 "f"(s.key)
                 : "memory");
}

// The statistics of a row from the C slots of a cluster exchange, the same
// bits in every thread of every block: a power-of-two C with the butterfly
// over lanes (every lane of the warp takes part), any other C folded in slot
// order.
__device__ __forceinline__ RowStats reduce_slots(const RowStats* slots, int C) {
    if ((C & (C - 1)) == 0) return stats_butterfly(slots[(threadIdx.x & 31) & (C - 1)], C);
    RowStats s = slots[0];
    for (int i = 1; i < C; ++i) s = stats_merge(s, slots[i]);
    return s;
}

// Cluster-wide statistics through the transaction-counted exchange: thread p
// (p < C) pushes the block's statistics into slot `rank` of block p; every
// thread then waits (bounded) for this block's C slots and reduces them the
// same way in every block (reduce_slots).  The caller has completed barrier phase
// 0 (every block has started and initialised `bar`, which expects C * 8
// bytes).  On a timeout the error bit is set and the slots are used as they
// are.
__device__ __forceinline__ RowStats cluster_stats_async(const RowStats& block, RowStats* slots,
                                                        uint64_t* bar, uint32_t rank, int C,
                                                        unsigned int* err) {
    if ((int)threadIdx.x < C)
        st_async_peer_f32x2(&slots[rank], bar, threadIdx.x, block.ss, block.key);
    if (!mbar_wait_bounded(bar, 0, kExchangeWaitLimitNs)) atomicOr(err, kDeviceErrorExchangeTimeout);
    return reduce_slots(slots, C);
}

// Cluster-wide statistics: block `rank` writes its statistics into slot
// `rank` of every block of the cluster (threads 0..C-1 write one peer each),
// one barrier phase publishes the writes, and every block reduces the C
// slots the same way (reduce_slots), so all blocks hold the same bits.  The
// caller has completed barrier phase 0 (every block has started).
__device__ __forceinline__ RowStats cluster_stats_combine(const RowStats& block, RowStats* slots,
                                                          uint32_t rank, int C) {
    if ((int)threadIdx.x < C) st_peer_stats(slots, rank, threadIdx.x, block);
    cluster_arrive_release();
    cluster_wait_acquire();
    return reduce_slots(slots, C);
}

}  // namespace rrf
