// rrf_gemm.cu -- the FP8 GEMM that consumes the per-row scales:
//   out[m][n] = RN_bf16((sum_k a[m][k] * b[n][k]) * a_scale[m] * b_scale[n] + bias[n])
// on the 5th-generation tensor cores (Ascend CANN docs,
// aclnnAlltoAllQuantMatmul: per-token dynamic quantisation of the
// activations, then (x1_q @ x2) * x1Scale * x2Scale + bias).
//
// Kernels (plan_scaled_mm chooses by shape; the launchers follow its plan):
//   scaled_mm_pair_kernel / scaled_mm_mx_pair_kernel  256 x 256 tiles on SM
//            pairs (tcgen05.mma.cta_group::2) for products that fill every pair;
//   scaled_mm_kernel / scaled_mm_mx_kernel  persistent CTAs on 128 x BN tiles
//            (BN 128 or 64), Z k-tiles per TMA box for short products;
//   scaled_mm_swap_pairk_kernel  at most 32 rows against a weight, the
//            operands swapped (the weight's rows on the MMA's M side, two
//            k-tiles of them per instruction); per-token and MX forms.
// A persistent CTA per SM walks 128 x BN tiles of out (BN 128 or 64).
// Warp roles (the same in every kernel; the swapped kernel's MX form adds a
// seventh warp that rearranges the scale codes of each stage):
//   warp 0   one thread issues the TMA loads of the A (128 x 128 bytes) and
//            B (BN x 128 bytes) k-tiles into a ring of shared-memory stages
//            (128-byte swizzle, the layout the MMA descriptors name);
//   warp 1   allocates two fp32 accumulators in tensor memory (BN columns of
//            128 lanes each) and one thread issues tcgen05.mma (kind::f8f6f4,
//            M = 128, N = BN, K = 32 per instruction, 4 per k-tile); a
//            tcgen05.commit per k-tile hands the stage back to the producer,
//            one per tile hands the accumulator to the epilogue;
//   warps 2-5 the epilogue: tcgen05.ld of its 32 accumulator lanes (rows),
//            the two scales and bias, one rounding to bf16, 64-byte stores,
//            while the MMAs of the next tile fill the other accumulator.
// Every mbarrier wait is bounded in time; a wait that runs out sets
// RRF_DEVICE_ERROR_GEMM_TIMEOUT, and the CTA still waits (bounded) for its
// own loads and MMAs and frees its tensor memory before it returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "rrf_device.cuh"
#include "rrf_internal.h"

namespace rrf {
namespace {

constexpr int kBM = 128;             // rows of a tile (the MMA's M)
constexpr int kBK = 128;             // k per stage: 128 one-byte codes = one swizzle row
constexpr int kThreads = 192;        // 6 warps
constexpr int kMmaK = 32;            // k of one kind::f8f6f4 instruction
constexpr unsigned long long kGemmWaitLimitNs = 100000000ull;  // 100 ms

// ---------------------------------------------------------------- mbarrier --

__device__ __forceinline__ bool mbar_try_wait_cta(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of `bar`; false (and the error bit) if the wait ran
// out.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, unsigned int* err) {
    if (mbar_try_wait_cta(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait_cta(bar, parity)) {
        if (global_timer_ns() - t0 > kGemmWaitLimitNs) {
            atomicOr(err, RRF_DEVICE_ERROR_GEMM_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The epilogue's wait for its accumulator (phase `parity` of `bar`).  Under
// the test hook (g.starve) it then also waits for the accumulator's next
// completion, which cannot come before this epilogue releases it: the
// bounded wait runs out and reports RRF_DEVICE_ERROR_GEMM_TIMEOUT, so the
// failure path runs on a GPU without a fault or a hang.
__device__ __forceinline__ bool epilogue_wait(uint64_t* bar, uint32_t parity, const GemmArgs& g) {
    if (!wait_phase(bar, parity, g.err)) return false;
    return g.starve == 0 || wait_phase(bar, parity ^ 1u, g.err);
}

// ---------------------------------------------------------------------- TMA --

// 2-D tiled load of box {x, y} at coordinates (x, y) into shared memory,
// completing `bytes` on `bar` (this CTA's shared memory only).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :
        : "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// ----------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(dst_smem)), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, both K-major e4m3, fp32 D.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's lane.
__device__ __forceinline__ void tmem_load_32(uint32_t taddr, float v[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major tile stored as rows of 128
// bytes in 128-byte-swizzled 1024-byte atoms (8 rows each), the layout a
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes: start address >> 4,
// leading-dimension offset 1 (unused within a swizzle row), stride between
// 8-row groups 1024 bytes, descriptor version 1, layout SWIZZLE_128B (2).
__device__ __forceinline__ uint64_t kmajor_sw128_desc(const void* tile) {
    const uint64_t addr = smem_u32(tile);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | ((1024ull >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor of kind::f8f6f4: fp32 accumulator, A and B e4m3,
// both K-major, N = bn, M = 128.
__host__ __device__ constexpr uint32_t f8_idesc(int bn) {
    return (1u << 4) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

// ------------------------------------------------------------------ kernel --

// The epilogue of 32 accumulator columns [n, n + 32) of one output row: both
// scales and the bias in fp32, one rounding to bf16, 64-byte stores (16 or
// 32 columns valid: N % 16 == 0).
__device__ __forceinline__ void store_row_chunk(const GemmArgs& g, const float v[32], float sa,
                                                int row, int n) {
    if (!RRF_IN_BOUNDS(row >= 0 && row < g.M && n >= 0 && n < g.N, g.err)) return;
    const int valid = g.N - n < 32 ? g.N - n : 32;
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        // (the MX GEMM has no column scales: its scales act inside the MMA)
        const float s0 = i < valid ? (g.b_scale != nullptr ? g.b_scale[n + i] : 1.0f) : 0.0f;
        const float s1 =
            i + 1 < valid ? (g.b_scale != nullptr ? g.b_scale[n + i + 1] : 1.0f) : 0.0f;
        float y0 = __fmul_rn(__fmul_rn(v[i], sa), s0);
        float y1 = __fmul_rn(__fmul_rn(v[i + 1], sa), s1);
        if (g.bias != nullptr && i < valid) {
            y0 = __fadd_rn(y0, __uint_as_float((uint32_t)g.bias[n + i] << 16));
            y1 = __fadd_rn(y1, __uint_as_float((uint32_t)g.bias[n + i + 1] << 16));
        }
        packed[i / 2] = f32x2_to_bf16x2(y0, y1);
    }
    uint4* dst = reinterpret_cast<uint4*>(g.out + (int64_t)row * g.N + n);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        if (q * 8 < valid)
            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2],
                                packed[4 * q + 3]);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

// AROWS: rows of A loaded per k-tile.  128 normally; 8, 16, 32 or 64 for
// calls of at most that many rows, which shrinks the A stage (the MMA still
// reads 128 rows: the rows past AROWS come from the bytes that follow -- the
// next k-tiles' A rows or the stage's B tiles -- and land in accumulator
// rows that are never stored).
// Z: k-tiles per stage, loaded by one 3-D TMA box per operand (128 bytes x
// rows x Z atoms of 128 values of K).  A TMA operation moves a few KB at a
// fixed cost, and a CTA streams a weight only as fast as it issues them:
// short, wide products (a decode batch against a weight) take Z = 4 or 2,
// which needs K % 128 == 0 (k-atoms past K read as zero).
template <int BN, int AROWS, int Z>
struct Tile {
    static_assert(AROWS == kBM || (AROWS <= 64 && AROWS % 8 == 0 && BN == 64),
                  "the MMA's 128 rows of A must stay inside the stage");
    static_assert((Z - 1) * AROWS * kBK + kBM * kBK <= Z * (AROWS + BN) * kBK,
                  "the MMA's 128 rows of A must stay inside the stage");
    static constexpr int kABytes = AROWS * kBK;        // one k-tile of A
    static constexpr int kBBytes = BN * kBK;           // one k-tile of B
    static constexpr int kBOffset = Z * kABytes;       // B tiles follow the Z A tiles
    static constexpr int kStageBytes = Z * (kABytes + kBBytes);
    // as many stages as fit in 200 KB (220 KB with several k-tiles per
    // stage), at most 12: 4 at BN 256, 6 at 128, 8 at 64, 12 with 64-row A
    // stages, 3 with four k-tiles of 64 rows
    static constexpr int kBudget = (Z > 1 ? 220 : 200) * 1024;
    static constexpr int kStages = kBudget / kStageBytes > 12 ? 12 : kBudget / kStageBytes;
    static constexpr int kTmemCols = 2 * BN;  // two accumulators
    // full / empty per stage, full / empty per accumulator, one for the drain
    static constexpr int kBarriers = 2 * kStages + 4 + 1;
    // 1 KB of slack aligns the stages to the 1024-byte swizzle atom
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarriers * 8 + 16;
    static_assert(kSmemBytes <= 227 * 1024, "stages exceed the shared memory of a CTA");
};

// 3-D tiled load of box {x, y, z} at coordinates (x, y, z), completing on
// `bar` (this CTA's shared memory only).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :
        : "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// The loads of stage group kg (k-tiles kg*Z ...) of A rows m0.. and B rows
// n0..: 2-D boxes for Z = 1, else one 3-D box of Z atoms per operand.
template <int Z, int ABYTES, int BOFFSET>
__device__ __forceinline__ void load_group(uint8_t* dst, const CUtensorMap* ma,
                                           const CUtensorMap* mb, uint64_t* bar, int kg, int m0,
                                           int n0) {
    if constexpr (Z == 1) {
        tma_load_2d(dst, ma, bar, kg * kBK, m0);
        tma_load_2d(dst + BOFFSET, mb, bar, kg * kBK, n0);
    } else {
        tma_load_3d(dst, ma, bar, 0, m0, kg * Z);
        tma_load_3d(dst + BOFFSET, mb, bar, 0, n0, kg * Z);
    }
}

// A persistent grid: CTA c takes tiles c, c + gridDim.x, ... (row-major over
// the 128 x BN tiles, so the CTAs working at one time share A rows and B
// columns in L2).  The accumulator is double-buffered in tensor memory: the
// MMAs of a CTA's next tile run while the epilogue warps drain this one.
template <int BN, int AROWS, int Z>
__global__ void __launch_bounds__(kThreads, 1)
    scaled_mm_kernel(const __grid_constant__ CUtensorMap tma_a,
                     const __grid_constant__ CUtensorMap tma_b, const GemmArgs g) {
    using T = Tile<BN, AROWS, Z>;
    constexpr int S = T::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * T::kStageBytes);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;       // [2]: the tile's MMAs are done
    uint64_t* acc_empty = acc_full + 2;   // [2]: the epilogue has read the tile
    uint64_t* drained = acc_empty + 2;    // every MMA of the CTA is done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_n = (g.N + BN - 1) / BN;
    const int tiles = tiles_n * ((g.M + kBM - 1) / kBM);
    const int ktiles = (g.K + kBK - 1) / kBK;
    const int kgroups = (ktiles + Z - 1) / Z;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
        }
        mbar_init(drained, 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, T::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch: the set-up above overlapped the previous
    // kernel of the stream; the operands, scales and output are touched only
    // after that kernel has completed.  (Measured on B200 at 1-64 x 7168 x
    // 7168: 0.4-0.6 us per call faster than a plain launch; an L2 prefetch of
    // the CTA's weight tile before the wait made the same calls 2 us slower
    // and was dropped.)
    wait_for_previous_grid();
    allow_next_grid();

    if (warp == 0) {
        // ---- producer: TMA loads of every k-tile of every tile of this CTA
        if (lane == 0) {
            int it = 0;  // k-tiles issued, over all tiles
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t / tiles_n) * kBM, n0 = (t % tiles_n) * BN;
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    // a fresh barrier counts as having completed the phase
                    // before phase 0: the first pass over the ring does not wait
                    if (!wait_phase(&empty[s], ((it / S) & 1) ^ 1, g.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], T::kStageBytes);
                    load_group<Z, T::kABytes, T::kBOffset>(smem + s * T::kStageBytes, &tma_a,
                                                           &tma_b, &full[s], kg, m0, n0);
                }
            }
            // the loads still in flight land before the CTA may exit
            for (int i = it > S ? it - S : 0; i < it; ++i)
                wait_phase(&full[i % S], (i / S) & 1, g.err);
        }
    } else if (warp == 1) {
        // ---- MMA issue: 4 instructions of K = 32 per k-tile
        if (lane == 0) {
            constexpr uint32_t idesc = f8_idesc(BN);
            int it = 0, j = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
                const int buf = j & 1;
                // the epilogue has drained this accumulator's previous tile
                if (!wait_phase(&acc_empty[buf], ((j >> 1) & 1) ^ 1, g.err)) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&full[s], (it / S) & 1, g.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t* stage = smem + s * T::kStageBytes;
                    // the k-tiles of the group that lie inside K
                    const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                    for (int j = 0; j < nk; ++j) {
                        const uint64_t ad = kmajor_sw128_desc(stage + j * T::kABytes);
                        const uint64_t bd = kmajor_sw128_desc(stage + T::kBOffset + j * T::kBBytes);
#pragma unroll
                        for (int k = 0; k < kBK / kMmaK; ++k) {
                            // advance the start address by k * 32 bytes in the swizzle row
                            const uint64_t step = (uint64_t)(k * kMmaK) >> 4;
                            mma_f8(d, ad + step, bd + step, idesc, (kg | j | k) != 0);
                        }
                    }
                    mma_commit(&empty[s]);  // the stage is free once these are done
                }
                mma_commit(&acc_full[buf]);
            }
            mma_commit(drained);
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp w reads accumulator lanes 32 * (w % 4) ...
        const int quarter = warp & 3;
        int j = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            const int buf = j & 1;
            const int m0 = (t / tiles_n) * kBM, n0 = (t % tiles_n) * BN;
            bool have = epilogue_wait(&acc_full[buf], (j >> 1) & 1, g);
            if (!__all_sync(0xFFFFFFFFu, have)) break;
            tc_fence_after_sync();
            const int row = m0 + quarter * 32 + lane;
            const float sa = row < g.M ? g.a_scale[row] : 0.0f;
            const uint32_t base = tmem + (uint32_t)(buf * BN) + ((uint32_t)(quarter * 32) << 16);
            for (int c = 0; c < BN; c += 32) {
                float v[32];
                tmem_load_32(base + (uint32_t)c, v);
                const int n = n0 + c;
                if (row >= g.M || n >= g.N) continue;
                store_row_chunk(g, v, sa, row, n);
            }
            // this warp's reads of the accumulator are done: hand it back
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }

    // ---- teardown: tensor memory is freed after the CTA's last MMA and load
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        wait_phase(drained, 0, g.err);
        tc_fence_after_sync();
        tmem_dealloc(tmem, T::kTmemCols);
    }
}

// ------------------------------------------------ block-scaled MMA helpers --
// The mx scenario's GEMM carries one E8M0 code per 32 values of K on both
// operands, on tcgen05.mma kind::mxf8f6f4 with block scaling: the scale codes
// of a k-tile (128 rows x 4 codes, one 512-byte atom of the blocked order:
// row r's 4 codes at byte (r % 32) * 16 + (r / 32) * 4) are loaded next to
// the A and B tiles, copied into tensor memory with tcgen05.cp (32 lanes x
// 128 bits, repeated in the 4 lane quarters: lane l holds rows l, l+32,
// l+64, l+96, 4 codes each, in 4 columns), and the k-tile's four MMAs take
// code (k-step) of each 32-bit word.  Row r of an M = 128 operand reads
// column r / 32 of lane r; column c of the N side reads column c / 32 of
// lane c % 32.

// 1-D bulk copy of `bytes` (a multiple of 16, both addresses 16-byte
// aligned) into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Shared -> tensor memory: 32 rows of 16 bytes, repeated in the 4 lane quarters.
__device__ __forceinline__ void tmem_copy_32x128b_x4(uint32_t taddr, uint64_t src_desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(src_desc)
                 : "memory");
}

// Descriptor of a scale atom as tcgen05.cp's source: 32 rows of 16 bytes,
// contiguous, no swizzle (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_atom_desc(const void* atom) {
    const uint64_t addr = smem_u32(atom);
    return ((addr >> 4) & 0x3FFFull) | ((128ull >> 4) << 32) | (1ull << 46);
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate, uint32_t sfa,
                                       uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa),
           "r"(sfb)
        : "memory");
}

// Instruction descriptor of the block-scaled MMA: A and B e4m3 (0), K-major,
// N = bn, M = 128, E8M0 scales (bit 23), scale codes taken from byte `id` of
// the A and B scale words.
__host__ __device__ constexpr uint32_t mx_idesc(int bn, uint32_t id) {
    return (id << 4) | ((uint32_t)(bn >> 3) << 17) | (1u << 23) | ((uint32_t)(kBM >> 4) << 24) |
           (id << 29);
}

// ------------------------------------- short products: the operands swapped --
// A call of at most 32 rows against a weight (a decode batch): the weight's
// rows are the MMA's M side and the call's rows its N side (NA = the rows
// rounded up to 8, 16 or 32), so no tensor-core row is spent on padding.  A
// CTA streams a 64-row weight tile (Z k-tiles per 3-D TMA box) against the
// call's rows (an L2-resident box of NA rows per stage).  One instruction
// takes two k-tiles: A = the 128 rows of shared memory that hold weight
// k-tiles kt and kt+1 (64 rows each, consecutive), B = the 2 NA rows that
// hold the call's k-tiles kt and kt+1.  In D = A B^T (M = 128, N = 2 NA) the
// block D[0:64, 0:NA] gets k-tile kt's partial product and D[64:128, NA:2NA]
// k-tile kt+1's; the two off-diagonal blocks pair a weight k-tile with the
// other k-tile of the call and are never read.  The epilogue adds the two
// diagonal blocks (the even one first).  Against one M = 64, N = NA
// instruction per k-tile this halves the instructions that hold each stage
// back from the producer.  An odd number of k-tiles pairs the last one with
// the zeros the TMA box holds past K.  D[w][m] of the M = 128 layout sits in
// tensor-memory lane w, column m.
//
// MX (block-scaled) form: the stage also holds the Z scale atoms of the
// weight's 128-row block and the Z of the call's rows, and per pair of
// k-tiles a seventh warp writes two atoms for the pair into the stage (off
// the MMA issue path: the MMA thread waits for them per stage): the A
// atom, line l = the weight tile's rows l and 32 + l for k-tile kt (the
// tile's half of the block's atom), then the same rows for kt+1, so that A
// row r reads its own k-tile's codes in column r / 32; and the B atom, whose
// column c / 32, lane c % 32 holds call row c's codes for kt (c < NA) or row
// c - NA's for kt+1.  The k-tile past an odd count takes kt's codes (its
// data are zeros).
template <int NA, int Z, bool MX = false>
struct SwapPairTile {
    static_assert(NA == 8 || NA == 16 || NA == 32, "the call's rows: 8, 16 or 32");
    static_assert(Z % 2 == 0, "k-tiles go to the MMA in pairs");
    static constexpr int kWRows = 64;                  // weight rows per tile
    static constexpr int kWBytes = kWRows * kBK;       // one k-tile of the weight: 8 KB
    static constexpr int kXBytes = NA * kBK;           // one k-tile of the call's rows
    static constexpr int kXOffset = Z * kWBytes;
    static constexpr int kSfBytes = 512;               // one scale atom
    static constexpr int kSfwOffset = Z * (kWBytes + kXBytes);   // the weight's atoms
    static constexpr int kSfxOffset = kSfwOffset + Z * kSfBytes;  // the call's atoms
    static constexpr int kPairOffset = kSfxOffset + Z * kSfBytes; // per pair: A, B atoms
    static constexpr int kStageBytes =
        MX ? kPairOffset + (Z / 2) * 2 * kSfBytes : Z * (kWBytes + kXBytes);
    static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;
    static constexpr int kCombBytes = NA * kWRows * 4;  // the odd block, handed between warps
    static constexpr int kStages = (218 * 1024 - kCombBytes) / kStageStride > 12
                                       ? 12
                                       : (218 * 1024 - kCombBytes) / kStageStride;
    // two accumulators of 2 NA columns (a power of two of at least 32), then
    // (MX) 4 + 4 scale columns; the allocation a power of two
    static constexpr int kAccStride = 2 * NA < 32 ? 32 : 2 * NA;
    static constexpr int kUsedCols = 2 * kAccStride + (MX ? 8 : 0);
    static constexpr int kTmemCols = kUsedCols <= 64 ? 64 : kUsedCols <= 128 ? 128 : 256;
    // full / empty per stage, full / empty per accumulator, the drain, the
    // odd block's full / empty, and (MX) the pair atoms written per stage
    static constexpr int kBarriers = (MX ? 3 : 2) * kStages + 4 + 1 + 2;
    // the MX form adds a seventh warp that writes the pair atoms
    static constexpr int kThreadsPerCta = MX ? kThreads + 32 : kThreads;
    static constexpr int kSmemBytes =
        1024 + kStages * kStageStride + kCombBytes + kBarriers * 8 + 16;
    static_assert(kSmemBytes <= 227 * 1024, "stages exceed the shared memory of a CTA");
    static_assert(kXBytes % 1024 == 0, "each k-tile must start on a swizzle atom");
};

// Make this thread's shared-memory stores visible to the async proxy
// (tcgen05.cp reads them).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// NA consecutive fp32 accumulator columns of this thread's lane (NA = 8, 16
// or 32).
template <int NA>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, float v[NA]) {
    uint32_t r[NA];
    if constexpr (NA == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                       "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < NA; ++i) v[i] = __uint_as_float(r[i]);
    } else if constexpr (NA == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < NA; ++i) v[i] = __uint_as_float(r[i]);
    } else {
        static_assert(NA == 32, "8, 16 or 32 columns");
        tmem_load_32(taddr, v);
    }
}

// sfx, sfw: the MX form's scale codes of the call's rows and of the weight
// (the blocked order); null in the per-token form.
template <int NA, int Z, bool MX>
__global__ void __launch_bounds__(SwapPairTile<NA, Z, MX>::kThreadsPerCta, 1)
    scaled_mm_swap_pairk_kernel(const __grid_constant__ CUtensorMap tma_x,
                                const __grid_constant__ CUtensorMap tma_w, const GemmArgs g,
                                const uint8_t* sfx, const uint8_t* sfw) {
    using T = SwapPairTile<NA, Z, MX>;
    constexpr int S = T::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    float* comb = reinterpret_cast<float*>(ring + S * T::kStageStride);  // [NA][64]
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + S * T::kStageStride + T::kCombBytes);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drained = acc_empty + 2;
    uint64_t* comb_full = drained + 1;     // the odd block is in comb (64 threads arrive)
    uint64_t* comb_empty = comb_full + 1;  // comb was read (64 threads arrive)
    uint64_t* built = comb_empty + 1;      // (MX) a stage's pair atoms are written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(built + (MX ? S : 0));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (g.N + T::kWRows - 1) / T::kWRows;
    const int ktiles = g.K / kBK;  // K is a multiple of 128
    const int kgroups = (ktiles + Z - 1) / Z;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drained, 1);
        mbar_init(comb_full, 64);
        mbar_init(comb_empty, 64);
        if constexpr (MX)
            for (int s = 0; s < S; ++s) mbar_init(&built[s], 32);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, T::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch (see scaled_mm_kernel).
    wait_for_previous_grid();
    allow_next_grid();

    if (warp == 0) {
        // ---- producer: Z k-tiles of the weight tile and of the call's rows
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int n0 = t * T::kWRows;
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&empty[s], ((it / S) & 1) ^ 1, g.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = ring + s * T::kStageStride;
                    if constexpr (MX) {
                        // the scale atoms of the group's k-tiles inside K (a
                        // 1-D copy must not run past the row block's atoms)
                        const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                        const uint32_t sf_bytes = (uint32_t)(nk * T::kSfBytes);
                        mbar_arrive_expect_tx(&full[s],
                                              Z * (T::kWBytes + T::kXBytes) + 2 * sf_bytes);
                        tma_load_3d(dst, &tma_w, &full[s], 0, n0, kg * Z);
                        tma_load_3d(dst + T::kXOffset, &tma_x, &full[s], 0, 0, kg * Z);
                        bulk_load(dst + T::kSfwOffset,
                                  sfw + ((int64_t)(n0 / 128) * ktiles + kg * Z) * T::kSfBytes,
                                  sf_bytes, &full[s]);
                        bulk_load(dst + T::kSfxOffset, sfx + (int64_t)kg * Z * T::kSfBytes,
                                  sf_bytes, &full[s]);
                    } else {
                        mbar_arrive_expect_tx(&full[s], T::kStageBytes);
                        tma_load_3d(dst, &tma_w, &full[s], 0, n0, kg * Z);
                        tma_load_3d(dst + T::kXOffset, &tma_x, &full[s], 0, 0, kg * Z);
                    }
                }
            }
            for (int i = it > S ? it - S : 0; i < it; ++i)
                wait_phase(&full[i % S], (i / S) & 1, g.err);
        }
    } else if (warp == 1 && MX) {
        // ---- MX: one thread copies each pair's scale atoms (written by the
        // seventh warp) into tensor memory and issues the block-scaled MMAs
        // D[128 x 2NA] += A[128 x 32] * B[2NA x 32]^T
        if (lane == 0) {
            const uint32_t tmem_sfw = tmem + 2 * T::kAccStride, tmem_sfx = tmem_sfw + 4;
            int it = 0, j = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
                const int buf = j & 1;
                if (!wait_phase(&acc_empty[buf], ((j >> 1) & 1) ^ 1, g.err)) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(buf * T::kAccStride);
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&full[s], (it / S) & 1, g.err) ||
                        !wait_phase(&built[s], (it / S) & 1, g.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t* stage = ring + s * T::kStageStride;
                    const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                    for (int kj = 0; kj < nk; kj += 2) {
                        const uint8_t* pair = stage + T::kPairOffset + kj * T::kSfBytes;
                        // tcgen05 operations of this thread run in issue order
                        // (see scaled_mm_mx_kernel)
                        tmem_copy_32x128b_x4(tmem_sfw, sf_atom_desc(pair));
                        tmem_copy_32x128b_x4(tmem_sfx, sf_atom_desc(pair + T::kSfBytes));
                        const uint64_t wd = kmajor_sw128_desc(stage + kj * T::kWBytes);
                        const uint64_t xd = kmajor_sw128_desc(stage + T::kXOffset + kj * T::kXBytes);
#pragma unroll
                        for (int k = 0; k < kBK / kMmaK; ++k) {
                            const uint64_t step = (uint64_t)(k * kMmaK) >> 4;
                            mma_mx(d, wd + step, xd + step, mx_idesc(2 * NA, (uint32_t)k),
                                   (kg | kj | k) != 0, tmem_sfw, tmem_sfx);
                        }
                    }
                    mma_commit(&empty[s]);
                }
                mma_commit(&acc_full[buf]);
            }
            mma_commit(drained);
        }
        __syncwarp();
    } else if (MX && warp == kThreads / 32) {
        // ---- MX, the seventh warp: once a stage has landed, each lane writes
        // line `lane` of every pair's A and B atoms, makes its stores visible
        // to the async proxy and arrives on the stage's `built` barrier
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const int half = t & 1;  // the tile's 64 rows in the weight's 128-row block
            for (int kg = 0; kg < kgroups; ++kg, ++it) {
                const int s = it % S;
                if (!__all_sync(0xFFFFFFFFu, wait_phase(&full[s], (it / S) & 1, g.err))) {
                    ok = false;
                    break;
                }
                uint8_t* stage = ring + s * T::kStageStride;
                const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                constexpr int kWords = T::kSfBytes / 4;
                for (int kj = 0; kj < nk; kj += 2) {
                    const uint32_t* w0 =
                        reinterpret_cast<const uint32_t*>(stage + T::kSfwOffset + kj * T::kSfBytes);
                    const uint32_t* x0 =
                        reinterpret_cast<const uint32_t*>(stage + T::kSfxOffset + kj * T::kSfBytes);
                    const uint32_t* w1 = kj + 1 < nk ? w0 + kWords : w0;
                    const uint32_t* x1 = kj + 1 < nk ? x0 + kWords : x0;
                    uint32_t* pa =
                        reinterpret_cast<uint32_t*>(stage + T::kPairOffset + kj * T::kSfBytes);
                    uint32_t* pb = pa + kWords;
                    // line `lane` of each atom (16 bytes: 4 words)
                    pa[4 * lane + 0] = w0[4 * lane + 2 * half];
                    pa[4 * lane + 1] = w0[4 * lane + 2 * half + 1];
                    pa[4 * lane + 2] = w1[4 * lane + 2 * half];
                    pa[4 * lane + 3] = w1[4 * lane + 2 * half + 1];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c = 32 * q + lane;  // a column of B (call rows < 32: word 0)
                        pb[4 * lane + q] = c < NA       ? x0[4 * c]
                                           : c < 2 * NA ? x1[4 * (c - NA)]
                                                        : 0x7F7F7F7Fu;  // unread: 2^0
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&built[s]);  // each lane releases its own stores
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue: D[128 x 2NA] += A[128 x 32] * B[2NA x 32]^T, A and B
        // each spanning two k-tiles
        if (lane == 0) {
            constexpr uint32_t idesc = f8_idesc(2 * NA);  // M = 128, N = 2 NA
            int it = 0, j = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
                const int buf = j & 1;
                if (!wait_phase(&acc_empty[buf], ((j >> 1) & 1) ^ 1, g.err)) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(buf * T::kAccStride);
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&full[s], (it / S) & 1, g.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t* stage = ring + s * T::kStageStride;
                    const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                    for (int kj = 0; kj < nk; kj += 2) {
                        const uint64_t wd = kmajor_sw128_desc(stage + kj * T::kWBytes);
                        const uint64_t xd = kmajor_sw128_desc(stage + T::kXOffset + kj * T::kXBytes);
#pragma unroll
                        for (int k = 0; k < kBK / kMmaK; ++k) {
                            const uint64_t step = (uint64_t)(k * kMmaK) >> 4;
                            mma_f8(d, wd + step, xd + step, idesc, (kg | kj | k) != 0);
                        }
                    }
                    mma_commit(&empty[s]);
                }
                mma_commit(&acc_full[buf]);
            }
            mma_commit(drained);
        }
        __syncwarp();
    } else {
        // ---- epilogue: lane quarter q of tensor memory holds rows 32q ..
        // 32q+31 of D: quarters 0, 1 the even block's weight rows 0-63,
        // quarters 2, 3 the odd block's; the odd warps hand their NA values
        // per row to the even warps through shared memory, which add them,
        // scale (per-token form; the MX form's scales act inside the MMA)
        // and store (weight row w of the tile is output column n)
        const int quarter = warp & 3;
        const bool odd = quarter >= 2;
        const int w = (quarter & 1) * 32 + lane;
        int j = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
            const int buf = j & 1;
            const int n = t * T::kWRows + w;
            bool have = epilogue_wait(&acc_full[buf], (j >> 1) & 1, g);
            if (!__all_sync(0xFFFFFFFFu, have)) break;
            tc_fence_after_sync();
            float v[NA];
            tmem_load_cols<NA>(tmem + (uint32_t)(buf * T::kAccStride + (odd ? NA : 0)) +
                                   ((uint32_t)(quarter * 32) << 16),
                               v);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
            if (odd) {
                // comb is free once the even warps have read the previous tile's
                if (j > 0 && !wait_phase(comb_empty, (j - 1) & 1, g.err)) ok = false;
#pragma unroll
                for (int m = 0; m < NA; ++m) comb[m * T::kWRows + w] = v[m];  // no bank conflicts
                mbar_arrive(comb_full);  // each thread releases its own stores
            } else {
                if (!wait_phase(comb_full, j & 1, g.err)) ok = false;
                float o[NA];
#pragma unroll
                for (int m = 0; m < NA; ++m) o[m] = comb[m * T::kWRows + w];
                mbar_arrive(comb_empty);
                if (ok && n < g.N && RRF_IN_BOUNDS(n >= 0, g.err)) {
                    const float sb = MX ? 1.0f : g.b_scale[n];
                    const float bias =
                        g.bias != nullptr ? __uint_as_float((uint32_t)g.bias[n] << 16) : 0.0f;
#pragma unroll
                    for (int m = 0; m < NA; ++m) {
                        if (m < g.M) {
                            float y = __fadd_rn(v[m], o[m]);
                            if constexpr (!MX) y = __fmul_rn(__fmul_rn(y, __ldg(g.a_scale + m)), sb);
                            if (g.bias != nullptr) y = __fadd_rn(y, bias);
                            g.out[(int64_t)m * g.N + n] =
                                (uint16_t)(f32x2_to_bf16x2(y, 0.0f) & 0xFFFFu);
                        }
                    }
                }
            }
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        wait_phase(drained, 0, g.err);
        tc_fence_after_sync();
        tmem_dealloc(tmem, T::kTmemCols);
    }
}

// ------------------------------------------------- two-CTA (pair) kernel --
// A cluster of two CTAs on neighbouring SMs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256): each CTA loads 128 rows of A
// and 128 rows of B per k-tile (32 KB instead of the one-CTA kernel's 48 KB
// for the same MMA work per SM) and holds 128 accumulator rows x 256 columns
// of the tile, twice (double buffer).  The even CTA of the pair (the
// leader) arms the stage barriers and issues the MMAs, which read both CTAs'
// shared memory; both CTAs' loads complete on the leader's barriers.

// Shared::cluster address of the same shared-memory location in CTA `rank`
// of the cluster.
__device__ __forceinline__ uint32_t peer_smem(const void* local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)),
                 "r"(rank));
    return r;
}

// One arrival on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(bar)
                 : "memory");
}

// A load of the pair: lands in this CTA's shared memory and completes its
// bytes on the barrier at the same offset in the pair's even CTA.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :
        : "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar) & 0xFEFFFFFFu), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(dst_smem)), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at shared::cluster address `bar` when the
// pair's tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar)
                 : "memory");
}

// Instruction descriptor of the pair's MMA: as f8_idesc with M = 256.
__host__ __device__ constexpr uint32_t f8_idesc_pair(int bn) {
    return (1u << 4) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// Tile t of a tiles_m x tiles_n grid in groups of 8 tile rows: consecutive
// tiles walk down the 8 rows of a group before moving to the next column, so
// the tiles in flight at one time share a few rows of A and columns of B in
// L2 (a row-major walk spans every column of B at once).
__device__ __forceinline__ void grouped_tile(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
    constexpr int G = 8;
    const int group = t / (G * tiles_n);
    const int first = group * G;
    const int rows = tiles_m - first < G ? tiles_m - first : G;
    const int r = t - group * G * tiles_n;
    tm = first + r % rows;
    tn = r / rows;
}

struct PairTile {
    static constexpr int kHalfBytes = 128 * kBK;            // 16 KB: 128 rows of A or of B
    static constexpr int kStageBytes = 2 * kHalfBytes;      // this CTA's A half and B half
    static constexpr int kStages = 6;                       // 192 KB (7 measured no faster)
    static constexpr int kTmemCols = 512;                   // two 256-column accumulators
    static constexpr int kBarriers = 2 * kStages + 4 + 1;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarriers * 8 + 16;
};

__global__ void __launch_bounds__(kThreads, 1)
    scaled_mm_pair_kernel(const __grid_constant__ CUtensorMap tma_a,
                          const __grid_constant__ CUtensorMap tma_b, const GemmArgs g) {
    using T = PairTile;
    constexpr int S = T::kStages;
    constexpr int BN = 256;  // the pair tile is 256 x 256
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * T::kStageBytes);  // leader's are used
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;       // [2]
    uint64_t* acc_empty = acc_full + 2;   // [2], the leader's: both CTAs' epilogue warps
    uint64_t* drained = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0: the leader
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int tiles_n = (g.N + 255) / 256, tiles_m = (g.M + 255) / 256;
    const int tiles = tiles_n * tiles_m;
    const int ktiles = (g.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);  // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(drained, 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, T::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    // both CTAs' barriers and tensor memory exist before either signals the other
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch (see scaled_mm_kernel).
    wait_for_previous_grid();
    allow_next_grid();

    if (warp == 0) {
        // ---- producer (each CTA): its 128 rows of A and of B per k-tile
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs) {
                int tm, tn;
                grouped_tile(t, tiles_m, tiles_n, tm, tn);
                const int m0 = tm * 256 + (int)rank * 128;
                const int n0 = tn * 256 + (int)rank * 128;
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&empty[s], ((it / S) & 1) ^ 1, g.err)) {
                        ok = false;
                        break;
                    }
                    // the leader arms its barrier for both CTAs' bytes; the
                    // odd CTA's loads may land first (the count goes negative)
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * T::kStageBytes);
                    uint8_t* dst = smem + s * T::kStageBytes;
                    tma_load_2d_pair(dst, &tma_a, &full[s], kt * kBK, m0);
                    tma_load_2d_pair(dst + T::kHalfBytes, &tma_b, &full[s], kt * kBK, n0);
                }
            }
            // this CTA's loads in flight have landed once the MMAs released
            // their stages (the empty barriers are this CTA's own)
            for (int i = it > S ? it - S : 0; i < it; ++i)
                wait_phase(&empty[i % S], (i / S) & 1, g.err);
        }
    } else if (warp == 1) {
        // ---- MMA issue (the leader only)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = f8_idesc_pair(BN);
            const uint32_t peer = 1;
            int it = 0, j = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs, ++j) {
                const int buf = j & 1;
                if (!wait_phase(&acc_empty[buf], ((j >> 1) & 1) ^ 1, g.err)) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&full[s], (it / S) & 1, g.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t* tile = smem + s * T::kStageBytes;
                    const uint64_t ad = kmajor_sw128_desc(tile);
                    const uint64_t bd = kmajor_sw128_desc(tile + T::kHalfBytes);
#pragma unroll
                    for (int k = 0; k < kBK / kMmaK; ++k) {
                        const uint64_t step = (uint64_t)(k * kMmaK) >> 4;
                        mma_f8_pair(d, ad + step, bd + step, idesc, (kt | k) != 0);
                    }
                    // both CTAs' stage s is free once these MMAs are done
                    mma_commit_pair(smem_u32(&empty[s]));
                    mma_commit_pair(peer_smem(&empty[s], peer));
                }
                mma_commit_pair(smem_u32(&acc_full[buf]));
                mma_commit_pair(peer_smem(&acc_full[buf], peer));
            }
            mma_commit_pair(smem_u32(drained));
            mma_commit_pair(peer_smem(drained, peer));
        }
        __syncwarp();
    } else {
        // ---- epilogue (each CTA): its 128 accumulator rows of the tile
        const int quarter = warp & 3;
        const uint32_t leader_acc_empty[2] = {peer_smem(&acc_empty[0], 0),
                                              peer_smem(&acc_empty[1], 0)};
        int j = 0;
        for (int t = pair; t < tiles; t += npairs, ++j) {
            const int buf = j & 1;
            int tm, tn;
            grouped_tile(t, tiles_m, tiles_n, tm, tn);
            const int m0 = tm * 256 + (int)rank * 128, n0 = tn * 256;
            bool have = epilogue_wait(&acc_full[buf], (j >> 1) & 1, g);
            if (!__all_sync(0xFFFFFFFFu, have)) break;
            tc_fence_after_sync();
            const int row = m0 + quarter * 32 + lane;
            const float sa = row < g.M ? g.a_scale[row] : 0.0f;
            const uint32_t base = tmem + (uint32_t)(buf * BN) + ((uint32_t)(quarter * 32) << 16);
            for (int c = 0; c < BN; c += 32) {
                float v[32];
                tmem_load_32(base + (uint32_t)c, v);
                const int n = n0 + c;
                if (row >= g.M || n >= g.N) continue;
                store_row_chunk(g, v, sa, row, n);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty[buf]);
        }
    }

    // ---- teardown: every MMA of the pair is done before tensor memory is
    // freed, and neither CTA leaves while the other may still use it
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        wait_phase(drained, 0, g.err);
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, T::kTmemCols);
    }
    cluster_arrive_release();
    cluster_wait_acquire();
}

// ------------------------------------------- MX (block-scaled) GEMM kernel --
// out = (a * 2^(sa - 127)) @ (b * 2^(sb - 127))^T + bias with one E8M0 code
// per 32 values of K (the mx scenario), the scale atoms handled as the
// block-scaled MMA helpers above describe.

// BN 128 or 64 columns per tile; AROWS and Z (k-tiles per stage, one 3-D
// TMA box per operand) as for the per-token kernel (64-row A: the MMA's rows
// 64-127 read the 8 KB that follow and land in accumulator rows that are
// never stored).  A 64-column tile uses half of its B scale atom: the MMA
// reads the scale columns from 2 further on for the odd half (column j of
// the atom holds rows 32j..32j+31).  Stage: Z A tiles, Z B tiles, the Z A
// scale atoms, the Z B scale atoms (consecutive in the blocked order).
template <int BN, int AROWS, int Z>
struct MxTile {
    static_assert(BN == 128 || BN == 64, "one scale atom covers 128 columns");
    static_assert(AROWS == kBM || (AROWS <= 64 && AROWS % 8 == 0 && BN == 64),
                  "the MMA's 128 rows of A must stay inside the stage");
    static_assert((Z - 1) * AROWS * kBK + kBM * kBK <= Z * (AROWS + BN) * kBK,
                  "the MMA's 128 rows of A must stay inside the stage");
    static constexpr int kABytes = AROWS * kBK;      // one k-tile of A
    static constexpr int kBBytes = BN * kBK;         // one k-tile of B
    static constexpr int kSfBytes = 512;             // one atom: 128 rows x 4 codes
    static constexpr int kBOffset = Z * kABytes;
    static constexpr int kSfaOffset = Z * (kABytes + kBBytes);
    static constexpr int kSfbOffset = kSfaOffset + Z * kSfBytes;
    static constexpr int kStageBytes = Z * (kABytes + kBBytes + 2 * kSfBytes);
    static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;
    // as many stages as fit in 200 KB (220 KB with several k-tiles per
    // stage), at most 12: 6 at BN 128, 11 at 64, 3 with four 64-row k-tiles
    static constexpr int kBudget = (Z > 1 ? 220 : 200) * 1024;
    static constexpr int kStages = kBudget / kStageStride > 12 ? 12 : kBudget / kStageStride;
    static constexpr int kAccCols = 2 * BN;          // two accumulators
    // accumulators, then 4 + 4 scale columns (a power of two of at least 32)
    static constexpr int kTmemCols = BN == 128 ? 512 : 256;
    static constexpr int kBarriers = 2 * kStages + 4 + 1;
    static constexpr int kSmemBytes = 1024 + kStages * kStageStride + kBarriers * 8 + 16;
    static_assert(kSmemBytes <= 227 * 1024, "stages exceed the shared memory of a CTA");
};

template <int BN, int AROWS, int Z>
__global__ void __launch_bounds__(kThreads, 1)
    scaled_mm_mx_kernel(const __grid_constant__ CUtensorMap tma_a,
                        const __grid_constant__ CUtensorMap tma_b, const GemmArgs g,
                        const uint8_t* sfa, const uint8_t* sfb) {
    using T = MxTile<BN, AROWS, Z>;
    constexpr int S = T::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * T::kStageStride);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drained = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_n = (g.N + BN - 1) / BN;
    const int tiles = tiles_n * ((g.M + kBM - 1) / kBM);
    const int ktiles = g.K / kBK;  // K is a multiple of 128
    const int kgroups = (ktiles + Z - 1) / Z;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drained, 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, T::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch (see scaled_mm_kernel).
    wait_for_previous_grid();
    allow_next_grid();
    const uint32_t tmem_sfa = tmem + T::kAccCols, tmem_sfb = tmem + T::kAccCols + 4;

    if (warp == 0) {
        // ---- producer: A, B and their scale atoms of every k-tile
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t / tiles_n) * kBM, n0 = (t % tiles_n) * BN;
                const uint8_t* sfa_tile = sfa + (int64_t)(m0 / 128) * ktiles * T::kSfBytes;
                const uint8_t* sfb_tile = sfb + (int64_t)(n0 / 128) * ktiles * T::kSfBytes;
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&empty[s], ((it / S) & 1) ^ 1, g.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = smem + s * T::kStageStride;
                    // the scale atoms of the group's k-tiles inside K (a 1-D
                    // copy must not run past the row block's atoms); the A
                    // and B boxes are whole (atoms past K read as zero)
                    const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                    const uint32_t sf_bytes = (uint32_t)(nk * T::kSfBytes);
                    mbar_arrive_expect_tx(&full[s],
                                          Z * (T::kABytes + T::kBBytes) + 2 * sf_bytes);
                    load_group<Z, T::kABytes, T::kBOffset>(dst, &tma_a, &tma_b, &full[s], kg,
                                                           m0, n0);
                    bulk_load(dst + T::kSfaOffset, sfa_tile + kg * Z * T::kSfBytes, sf_bytes,
                              &full[s]);
                    bulk_load(dst + T::kSfbOffset, sfb_tile + kg * Z * T::kSfBytes, sf_bytes,
                              &full[s]);
                }
            }
            for (int i = it > S ? it - S : 0; i < it; ++i)
                wait_phase(&full[i % S], (i / S) & 1, g.err);
        }
    } else if (warp == 1) {
        // ---- scale copies and MMAs
        if (lane == 0) {
            int it = 0, j = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
                const int buf = j & 1;
                if (!wait_phase(&acc_empty[buf], ((j >> 1) & 1) ^ 1, g.err)) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                // the odd 64-column half of a scale atom: 2 columns further on
                const uint32_t sfb_cols =
                    tmem_sfb + (BN == 64 ? (uint32_t)((t % tiles_n) & 1) * 2u : 0u);
                for (int kg = 0; kg < kgroups; ++kg, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&full[s], (it / S) & 1, g.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t* stage = smem + s * T::kStageStride;
                    const int nk = ktiles - kg * Z < Z ? ktiles - kg * Z : Z;
                    for (int kj = 0; kj < nk; ++kj) {
                        // tcgen05 operations of this thread run in issue order:
                        // the copies land before the MMAs below read the
                        // scales, and the previous k-tile's MMAs have read
                        // theirs before these
                        tmem_copy_32x128b_x4(tmem_sfa,
                                             sf_atom_desc(stage + T::kSfaOffset + kj * T::kSfBytes));
                        tmem_copy_32x128b_x4(tmem_sfb,
                                             sf_atom_desc(stage + T::kSfbOffset + kj * T::kSfBytes));
                        const uint64_t ad = kmajor_sw128_desc(stage + kj * T::kABytes);
                        const uint64_t bd = kmajor_sw128_desc(stage + T::kBOffset + kj * T::kBBytes);
#pragma unroll
                        for (int k = 0; k < kBK / kMmaK; ++k) {
                            const uint64_t step = (uint64_t)(k * kMmaK) >> 4;
                            mma_mx(d, ad + step, bd + step, mx_idesc(BN, (uint32_t)k),
                                   (kg | kj | k) != 0, tmem_sfa, sfb_cols);
                        }
                    }
                    mma_commit(&empty[s]);
                }
                mma_commit(&acc_full[buf]);
            }
            mma_commit(drained);
        }
        __syncwarp();
    } else {
        // ---- epilogue: the scales are inside the accumulator; bias, bf16
        const int quarter = warp & 3;
        int j = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            const int buf = j & 1;
            const int m0 = (t / tiles_n) * kBM, n0 = (t % tiles_n) * BN;
            bool have = epilogue_wait(&acc_full[buf], (j >> 1) & 1, g);
            if (!__all_sync(0xFFFFFFFFu, have)) break;
            tc_fence_after_sync();
            const int row = m0 + quarter * 32 + lane;
            const uint32_t base = tmem + (uint32_t)(buf * BN) + ((uint32_t)(quarter * 32) << 16);
            for (int c = 0; c < BN; c += 32) {
                float v[32];
                tmem_load_32(base + (uint32_t)c, v);
                const int n = n0 + c;
                if (row >= g.M || n >= g.N) continue;
                store_row_chunk(g, v, 1.0f, row, n);  // g.b_scale is null: no scaling
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        wait_phase(drained, 0, g.err);
        tc_fence_after_sync();
        tmem_dealloc(tmem, T::kTmemCols);
    }
}

// --------------------------------------------- MX GEMM on SM pairs (2 CTAs) --
// The block-scaled MMA with cta_group::2 on 256 x 256 tiles, as the per-token
// pair kernel: each CTA loads 128 rows of A and 128 rows of B per k-tile.
// Scales: each CTA loads the atom of its own 128 A rows and both atoms of
// the tile's 256 B rows (the MMA scales each CTA's half of the product with
// the scale codes in that CTA's tensor memory, and every CTA's half spans
// all 256 columns); the leader's tcgen05.cp.cta_group::2 copies each CTA's
// atoms from its own shared memory into its own tensor memory.  The scale
// atoms travel as 3-D TMA boxes, so that the odd CTA's copies, like its A
// and B tiles, complete on the leader's stage barrier.
//
// Tensor memory (512 columns): the 256-column accumulator twice would leave
// no room for the 12 scale columns, so the two accumulators overlap in 32
// columns -- buffer 0 at [0, 256), buffer 1 at [224, 480), scales at
// [480, 492).  The epilogue reads the shared 32 columns first and reports
// that on `ovl_free`; the MMAs of the next tile wait for it.

// A 3-D tiled load of the pair (no swizzle) completing on the leader's barrier.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :
        : "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar) & 0xFEFFFFFFu), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// tcgen05.cp of the pair: in both CTAs, from the CTA's own shared memory at
// the descriptor's address to its own tensor memory at `taddr`.
__device__ __forceinline__ void tmem_copy_32x128b_x4_pair(uint32_t taddr, uint64_t src_desc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(src_desc)
                 : "memory");
}

__device__ __forceinline__ void mma_mx_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate, uint32_t sfa,
                                            uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa),
           "r"(sfb)
        : "memory");
}

// mx_idesc with M = 256.
__host__ __device__ constexpr uint32_t mx_idesc_pair(int bn, uint32_t id) {
    return (id << 4) | ((uint32_t)(bn >> 3) << 17) | (1u << 23) | ((uint32_t)(256 >> 4) << 24) |
           (id << 29);
}

struct MxPairTile {
    static constexpr int BN = 256;
    static constexpr int kHalfBytes = 128 * kBK;                 // 16 KB: 128 rows of A or B
    static constexpr int kSfaBytes = 512;                        // one atom
    static constexpr int kSfbBytes = 1024;                       // two atoms: 256 rows of B
    static constexpr int kSfOffset = 2 * kHalfBytes;
    static constexpr int kStageBytes = 2 * kHalfBytes + kSfaBytes + kSfbBytes;  // 33.5 KB
    static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;     // 34 KB
    static constexpr int kStages = 6;
    static constexpr int kTmemCols = 512;
    static constexpr uint32_t kBuf1 = 224;                       // buffer 1's first column
    static constexpr uint32_t kSfaCol = kBuf1 + BN;              // 480
    static constexpr uint32_t kSfbCol = kSfaCol + 4;             // 484 .. 491
    // full / empty per stage, full / empty per accumulator, overlap, drain
    static constexpr int kBarriers = 2 * kStages + 4 + 1 + 1;
    static constexpr int kSmemBytes = 1024 + kStages * kStageStride + kBarriers * 8 + 16;
};
static_assert(MxPairTile::kSfbCol + 8 <= MxPairTile::kTmemCols, "scale columns past the allocation");
static_assert(MxPairTile::kSmemBytes <= 227 * 1024, "stages exceed the shared memory of a CTA");

__global__ void __launch_bounds__(kThreads, 1)
    scaled_mm_mx_pair_kernel(const __grid_constant__ CUtensorMap tma_a,
                             const __grid_constant__ CUtensorMap tma_b,
                             const __grid_constant__ CUtensorMap tma_sfa,
                             const __grid_constant__ CUtensorMap tma_sfb, const GemmArgs g) {
    using T = MxPairTile;
    constexpr int S = T::kStages;
    constexpr int BN = T::BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * T::kStageStride);  // leader's are used
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;       // [2]
    uint64_t* acc_empty = acc_full + 2;   // [2], the leader's: both CTAs' epilogue warps
    uint64_t* ovl_free = acc_empty + 2;   // the leader's: the shared columns have been read
    uint64_t* drained = ovl_free + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0: the leader
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int tiles_n = (g.N + 255) / 256, tiles_m = (g.M + 255) / 256;
    const int tiles = tiles_n * tiles_m;
    const int ktiles = g.K / kBK;  // K is a multiple of 128

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);  // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(ovl_free, 8);
        mbar_init(drained, 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, T::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Programmatic dependent launch (see scaled_mm_kernel).
    wait_for_previous_grid();
    allow_next_grid();

    if (warp == 0) {
        // ---- producer (each CTA): its 128 rows of A and of B, its A scale
        // atom and both B scale atoms of the tile, per k-tile
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs) {
                int tm, tn;
                grouped_tile(t, tiles_m, tiles_n, tm, tn);
                const int m0 = tm * 256 + (int)rank * 128;
                const int n0 = tn * 256 + (int)rank * 128;
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&empty[s], ((it / S) & 1) ^ 1, g.err)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * T::kStageBytes);
                    uint8_t* dst = smem + s * T::kStageStride;
                    tma_load_2d_pair(dst, &tma_a, &full[s], kt * kBK, m0);
                    tma_load_2d_pair(dst + T::kHalfBytes, &tma_b, &full[s], kt * kBK, n0);
                    tma_load_3d_pair(dst + T::kSfOffset, &tma_sfa, &full[s], 0, kt, m0 / 128);
                    tma_load_3d_pair(dst + T::kSfOffset + T::kSfaBytes, &tma_sfb, &full[s], 0, kt,
                                     tn * 2);
                }
            }
            for (int i = it > S ? it - S : 0; i < it; ++i)
                wait_phase(&empty[i % S], (i / S) & 1, g.err);
        }
    } else if (warp == 1) {
        // ---- scale copies and MMAs (the leader only)
        if (rank == 0 && lane == 0) {
            const uint32_t peer = 1;
            int it = 0, j = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += npairs, ++j) {
                const int buf = j & 1;
                // this buffer's previous tile has been drained, and the
                // previous tile (the other buffer) no longer needs the
                // shared columns
                if (!wait_phase(&acc_empty[buf], ((j >> 1) & 1) ^ 1, g.err)) break;
                if (j > 0 && !wait_phase(ovl_free, (j - 1) & 1, g.err)) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + (buf ? T::kBuf1 : 0u);
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % S;
                    if (!wait_phase(&full[s], (it / S) & 1, g.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint8_t* tile = smem + s * T::kStageStride;
                    const uint8_t* sf = tile + T::kSfOffset;
                    tmem_copy_32x128b_x4_pair(tmem + T::kSfaCol, sf_atom_desc(sf));
                    tmem_copy_32x128b_x4_pair(tmem + T::kSfbCol, sf_atom_desc(sf + T::kSfaBytes));
                    tmem_copy_32x128b_x4_pair(tmem + T::kSfbCol + 4,
                                              sf_atom_desc(sf + T::kSfaBytes + 512));
                    const uint64_t ad = kmajor_sw128_desc(tile);
                    const uint64_t bd = kmajor_sw128_desc(tile + T::kHalfBytes);
#pragma unroll
                    for (int k = 0; k < kBK / kMmaK; ++k) {
                        const uint64_t step = (uint64_t)(k * kMmaK) >> 4;
                        mma_mx_pair(d, ad + step, bd + step, mx_idesc_pair(BN, (uint32_t)k),
                                    (kt | k) != 0, tmem + T::kSfaCol, tmem + T::kSfbCol);
                    }
                    mma_commit_pair(smem_u32(&empty[s]));
                    mma_commit_pair(peer_smem(&empty[s], peer));
                }
                mma_commit_pair(smem_u32(&acc_full[buf]));
                mma_commit_pair(peer_smem(&acc_full[buf], peer));
            }
            mma_commit_pair(smem_u32(drained));
            mma_commit_pair(peer_smem(drained, peer));
        }
        __syncwarp();
    } else {
        // ---- epilogue (each CTA): its 128 accumulator rows; the 32 columns
        // shared by the two buffers first
        const int quarter = warp & 3;
        const uint32_t leader_acc_empty[2] = {peer_smem(&acc_empty[0], 0),
                                              peer_smem(&acc_empty[1], 0)};
        const uint32_t leader_ovl_free = peer_smem(ovl_free, 0);
        int j = 0;
        for (int t = pair; t < tiles; t += npairs, ++j) {
            const int buf = j & 1;
            int tm, tn;
            grouped_tile(t, tiles_m, tiles_n, tm, tn);
            const int m0 = tm * 256 + (int)rank * 128, n0 = tn * 256;
            bool have = epilogue_wait(&acc_full[buf], (j >> 1) & 1, g);
            if (!__all_sync(0xFFFFFFFFu, have)) break;
            tc_fence_after_sync();
            const int row = m0 + quarter * 32 + lane;
            const uint32_t base = tmem + (buf ? T::kBuf1 : 0u) + ((uint32_t)(quarter * 32) << 16);
            // the shared columns are the last 32 of buffer 0, the first of buffer 1
            const int first = buf ? 0 : BN - 32;
            for (int i = 0; i < BN / 32; ++i) {
                const int c = (first + 32 * i) % BN;
                float v[32];
                tmem_load_32(base + (uint32_t)c, v);
                if (i == 0) {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(leader_ovl_free);
                }
                const int n = n0 + c;
                if (row >= g.M || n >= g.N) continue;
                store_row_chunk(g, v, 1.0f, row, n);  // g.b_scale is null: no scaling
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty[buf]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        wait_phase(drained, 0, g.err);
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, T::kTmemCols);
    }
    cluster_arrive_release();
    cluster_wait_acquire();
}

// ------------------------------------------------------------------- host --

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, through the runtime's entry-point query
// (the library links only the runtime).
EncodeTiled encode_tiled() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// Dynamic shared memory above 48 KB is enabled once per device for each
// kernel (KERNEL: the kernel's address; its devices done in a bitmask).
template <auto KERNEL>
cudaError_t enable_dynamic_smem(int bytes) {
    static std::atomic<uint64_t> enabled_on{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
    if (bit != 0 && (enabled_on.load(std::memory_order_relaxed) & bit) != 0) return cudaSuccess;
    e = cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) enabled_on.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// A launch of `pairs` clusters of two CTAs, one SM pair each.
template <class... Params, class... Args>
cudaError_t launch_on_pairs(void (*kernel)(Params...), int64_t pairs, int smem_bytes,
                            cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// One CTA per SM (at most `ctas`) of `threads` threads, launched with
// programmatic dependent launch: the kernel's set-up may overlap the previous
// kernel of the stream.
template <class... Params, class... Args>
cudaError_t launch_persistent_threads(void (*kernel)(Params...), unsigned ctas, int threads,
                                      int smem_bytes, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The same with the GEMM kernels' kThreads threads per CTA.
template <class... Params, class... Args>
cudaError_t launch_persistent(void (*kernel)(Params...), unsigned ctas, int smem_bytes,
                              cudaStream_t stream, Args... args) {
    return launch_persistent_threads(kernel, ctas, kThreads, smem_bytes, stream, args...);
}

// A [rows, K] byte matrix, box of 128 bytes x box_rows rows, 128-byte swizzle;
// rows and columns past the matrix read as zero.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
    EncodeTiled fn = encode_tiled();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    const cuuint32_t elem[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Blocked scale codes of a [rows, K] operand as a 3-D array of 32-bit words:
// 128 words (one 512-byte atom) x K/128 atoms along k x ceil(rows/128) row
// blocks; a box is one atom (box_blocks 1) or the atoms of two consecutive
// row blocks (2).  Row blocks past the operand read as zero.
bool make_sf_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_blocks) {
    EncodeTiled fn = encode_tiled();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {128, (cuuint64_t)(K / 128), (cuuint64_t)((rows + 127) / 128)};
    const cuuint64_t strides[2] = {512, (cuuint64_t)(K / 128) * 512};
    const cuuint32_t box[3] = {128, 1, (cuuint32_t)box_blocks};
    const cuuint32_t elem[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// A [rows, K] byte matrix (K % 128 == 0) as a 3-D array: 128 bytes x rows x
// K/128 atoms; a box is box_rows rows of Z consecutive atoms, which land as
// Z row-major tiles of box_rows x 128 bytes, 128-byte swizzle.  Rows and
// atoms past the matrix read as zero.
bool make_map3(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows, int z) {
    EncodeTiled fn = encode_tiled();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kBK, (cuuint64_t)rows, (cuuint64_t)(K / kBK)};
    const cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)kBK};
    const cuuint32_t box[3] = {(cuuint32_t)kBK, (cuuint32_t)box_rows, (cuuint32_t)z};
    const cuuint32_t elem[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// The operand maps of a kernel that loads Z k-tiles per stage.
bool make_maps(CUtensorMap* ma, CUtensorMap* mb, const GemmArgs& g, const void* a, const void* b,
               int arows, int brows, int z) {
    if (z == 1) return make_map(ma, a, g.M, g.K, arows) && make_map(mb, b, g.N, g.K, brows);
    return make_map3(ma, a, g.M, g.K, arows, z) && make_map3(mb, b, g.N, g.K, brows, z);
}

template <int BN, int AROWS, int Z>
cudaError_t launch_bn(const GemmArgs& g, const void* a, const void* b, int sm_count,
                      cudaStream_t stream) {
    using T = Tile<BN, AROWS, Z>;
    CUtensorMap ma, mb;
    if (!make_maps(&ma, &mb, g, a, b, AROWS, BN, Z)) return cudaErrorInvalidValue;
    constexpr auto kernel = scaled_mm_kernel<BN, AROWS, Z>;
    const cudaError_t e = enable_dynamic_smem<kernel>(T::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)((g.N + BN - 1) / BN) * ((g.M + kBM - 1) / kBM);
    const unsigned grid = (unsigned)(tiles < sm_count ? tiles : sm_count);  // one CTA per SM
    return launch_persistent(kernel, grid, T::kSmemBytes, stream, ma, mb, g);
}

// sfa, sfb: the MX form's scale codes of a and b (the blocked order), else
// null.
template <int NA, int Z, bool MX = false>
cudaError_t launch_swap_pairk(const GemmArgs& g, const void* a, const void* b, int sm_count,
                              cudaStream_t stream, const uint8_t* sfa = nullptr,
                              const uint8_t* sfb = nullptr) {
    using T = SwapPairTile<NA, Z, MX>;
    CUtensorMap mx, mw;
    if (!make_map3(&mx, a, g.M, g.K, NA, Z) || !make_map3(&mw, b, g.N, g.K, T::kWRows, Z))
        return cudaErrorInvalidValue;
    constexpr auto kernel = scaled_mm_swap_pairk_kernel<NA, Z, MX>;
    const cudaError_t e = enable_dynamic_smem<kernel>(T::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (g.N + T::kWRows - 1) / T::kWRows;
    const unsigned grid = (unsigned)(tiles < sm_count ? tiles : sm_count);
    return launch_persistent_threads(kernel, grid, T::kThreadsPerCta, T::kSmemBytes, stream, mx,
                                     mw, g, sfa, sfb);
}

cudaError_t launch_pair(const GemmArgs& g, const void* a, const void* b, int sm_count,
                        cudaStream_t stream) {
    using T = PairTile;
    CUtensorMap ma, mb;
    if (!make_map(&ma, a, g.M, g.K, 128) || !make_map(&mb, b, g.N, g.K, 128))
        return cudaErrorInvalidValue;
    const cudaError_t e = enable_dynamic_smem<scaled_mm_pair_kernel>(T::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)((g.N + 255) / 256) * ((g.M + 255) / 256);
    const int64_t pairs = tiles < sm_count / 2 ? tiles : sm_count / 2;
    return launch_on_pairs(scaled_mm_pair_kernel, pairs, T::kSmemBytes, stream, ma, mb, g);
}

template <int BN, int AROWS, int Z>
cudaError_t launch_mx(const GemmArgs& g, const void* a, const void* b, const uint8_t* sfa,
                      const uint8_t* sfb, int sm_count, cudaStream_t stream) {
    using T = MxTile<BN, AROWS, Z>;
    CUtensorMap ma, mb;
    if (!make_maps(&ma, &mb, g, a, b, AROWS, BN, Z)) return cudaErrorInvalidValue;
    constexpr auto kernel = scaled_mm_mx_kernel<BN, AROWS, Z>;
    const cudaError_t e = enable_dynamic_smem<kernel>(T::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)((g.N + BN - 1) / BN) * ((g.M + kBM - 1) / kBM);
    const unsigned grid = (unsigned)(tiles < sm_count ? tiles : sm_count);
    return launch_persistent(kernel, grid, T::kSmemBytes, stream, ma, mb, g, sfa, sfb);
}

cudaError_t launch_mx_pair(const GemmArgs& g, const void* a, const void* b, const uint8_t* sfa,
                           const uint8_t* sfb, int sm_count, cudaStream_t stream) {
    using T = MxPairTile;
    CUtensorMap ma, mb, msa, msb;
    if (!make_map(&ma, a, g.M, g.K, 128) || !make_map(&mb, b, g.N, g.K, 128) ||
        !make_sf_map(&msa, sfa, g.M, g.K, 1) || !make_sf_map(&msb, sfb, g.N, g.K, 2))
        return cudaErrorInvalidValue;
    const cudaError_t e = enable_dynamic_smem<scaled_mm_mx_pair_kernel>(T::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)((g.N + 255) / 256) * ((g.M + 255) / 256);
    const int64_t pairs = tiles < sm_count / 2 ? tiles : sm_count / 2;
    return launch_on_pairs(scaled_mm_mx_pair_kernel, pairs, T::kSmemBytes, stream, ma, mb, msa,
                           msb, g);
}

}  // namespace

GemmPlan plan_scaled_mm(int64_t M, int64_t N, int64_t K, bool mx, int sm_count) {
    auto tile = [&](int kernel, int arows, int bn, int z) {
        GemmPlan p;
        p.kernel = kernel;
        p.a_rows = arows;
        p.tile_n = bn;
        p.k_tiles_per_stage = z;
        if (kernel == kGemmPair) {
            p.tiles = ((M + 255) / 256) * ((N + 255) / 256);
            const int64_t pairs = p.tiles < sm_count / 2 ? p.tiles : sm_count / 2;
            p.ctas = 2 * pairs;
        } else {
            // the swapped kernel's tiles are 64 weight rows by all the call's rows
            p.tiles = kernel == kGemmSwap ? (N + 63) / 64 : ((N + bn - 1) / bn) * ((M + kBM - 1) / kBM);
            p.ctas = p.tiles < sm_count ? p.tiles : sm_count;  // one CTA per SM
        }
        return p;
    };
    const int64_t row_tiles = (M + kBM - 1) / kBM;
    // large products: 256 x 256 tiles on SM pairs once they fill every pair
    if (((M + 255) / 256) * ((N + 255) / 256) >= sm_count / 2) return tile(kGemmPair, 256, 256, 1);
    if (mx) {
        // else one CTA per 128 x 128 tile once those fill every SM; short, wide
        // problems take 128 x 64 tiles (A stages of the call's rows, up to 64)
        if (row_tiles * ((N + 127) / 128) >= sm_count) return tile(kGemmTile, kBM, 128, 1);
        // (K % 128 == 0 here: several k-tiles per TMA box, as the per-token GEMM)
        // at most 32 rows: the operands swapped, two k-tiles per MMA (M = 128
        // over two weight k-tiles, the scale atoms rebuilt per pair)
        if (M <= 8) return tile(kGemmSwap, 8, 64, 4);
        if (M <= 16) return tile(kGemmSwap, 16, 64, 4);
        if (M <= 32) return tile(kGemmSwap, 32, 64, 4);
        if (M <= 64) return tile(kGemmTile, 64, 64, 4);
        return tile(kGemmTile, kBM, 64, 2);
    }
    // One CTA per 128 x 128 tile once those fill every SM (a 128 x 256 tile
    // never would: ceil(M/128) * ceil(N/256) <= 2 * ceil(M/256) * ceil(N/256),
    // which is below the SM count whenever the pairs are not all busy); short,
    // wide problems (decode batches against a weight) take 64-column tiles,
    // the most CTAs streaming the weight.
    if (row_tiles * ((N + 127) / 128) >= sm_count) return tile(kGemmTile, kBM, 128, 1);
    // the weight-streaming shapes: several k-tiles per TMA box where K allows
    const bool atoms = K % kBK == 0;
    if (M <= 64 && !atoms) return tile(kGemmTile, 64, 64, 1);
    // at most 32 rows: the operands swapped, the call's rows padded to 8, 16
    // or 32 (at 64 the swapped MMA is no cheaper: measured slower); 8 k-tiles
    // per box at 8 rows (3 stages), 4 at 16 and 32 rows (5 and 4 stages).
    // Measured at 1-32 x 7168 x 7168: 8 beats 6 and 4 at 8 rows, 4 beats 8
    // and 6 at 16 rows (12.2 against 13.4 us), 4 beats 2 at 32 rows.
    if (M <= 8) return tile(kGemmSwap, 8, 64, 8);
    if (M <= 16) return tile(kGemmSwap, 16, 64, 4);
    if (M <= 32) return tile(kGemmSwap, 32, 64, 4);
    if (M <= 64) return tile(kGemmTile, 64, 64, 4);
    return tile(kGemmTile, kBM, 64, atoms ? 2 : 1);
}

cudaError_t launch_scaled_mm_mx(const GemmArgs& g, const void* a, const void* b,
                                const uint8_t* sfa, const uint8_t* sfb, int sm_count,
                                cudaStream_t stream) {
    const GemmPlan p = plan_scaled_mm(g.M, g.N, g.K, true, sm_count);
    if (p.kernel == kGemmPair) return launch_mx_pair(g, a, b, sfa, sfb, sm_count, stream);
    if (p.kernel == kGemmSwap) {
        if (p.a_rows == 8) return launch_swap_pairk<8, 4, true>(g, a, b, sm_count, stream, sfa, sfb);
        if (p.a_rows == 16)
            return launch_swap_pairk<16, 4, true>(g, a, b, sm_count, stream, sfa, sfb);
        return launch_swap_pairk<32, 4, true>(g, a, b, sm_count, stream, sfa, sfb);
    }
    if (p.tile_n == 128) return launch_mx<128, kBM, 1>(g, a, b, sfa, sfb, sm_count, stream);
    if (p.a_rows == 64) return launch_mx<64, 64, 4>(g, a, b, sfa, sfb, sm_count, stream);
    return launch_mx<64, kBM, 2>(g, a, b, sfa, sfb, sm_count, stream);
}

cudaError_t launch_scaled_mm(const GemmArgs& g, const void* a, const void* b, int sm_count,
                             cudaStream_t stream) {
    const GemmPlan p = plan_scaled_mm(g.M, g.N, g.K, false, sm_count);
    if (p.kernel == kGemmPair) return launch_pair(g, a, b, sm_count, stream);
    if (p.kernel == kGemmSwap) {
        if (p.a_rows == 8) return launch_swap_pairk<8, 8>(g, a, b, sm_count, stream);
        if (p.a_rows == 16) return launch_swap_pairk<16, 4>(g, a, b, sm_count, stream);
        return launch_swap_pairk<32, 4>(g, a, b, sm_count, stream);
    }
    if (p.tile_n == 128) return launch_bn<128, kBM, 1>(g, a, b, sm_count, stream);
    if (p.a_rows == 64)
        return p.k_tiles_per_stage == 4 ? launch_bn<64, 64, 4>(g, a, b, sm_count, stream)
                                        : launch_bn<64, 64, 1>(g, a, b, sm_count, stream);
    return p.k_tiles_per_stage == 2 ? launch_bn<64, kBM, 2>(g, a, b, sm_count, stream)
                                    : launch_bn<64, kBM, 1>(g, a, b, sm_count, stream);
}

}  // namespace rrf
