// rrf_sum.cu -- the bf16 sum of R buffers: fp32 accumulation in rank order,
// one rounding to bf16 (b12x PR #283 "PCIeTwoShotBF16": fixed-order fp32
// accumulation rounded once, deterministic).
//
// A grid-stride loop over 16-byte vectors: per vector the R loads are issued
// back to back before any add, each input byte is read once, the output is
// written once with streaming stores.
#include <cuda_runtime.h>

#include "rrf_device.cuh"
#include "rrf_internal.h"

namespace rrf {
namespace {

template <int RB>
__global__ void __launch_bounds__(256) sum_kernel(const SumArgs a) {
    wait_for_previous_grid();  // see rrf_device.cuh: programmatic dependent launch
    allow_next_grid();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // every address derives from the first index, taken after the wait
    const int64_t first = opaque((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    for (int64_t i = first; i < a.n_vecs; i += stride) {
        uint4 x[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r)
            if (r < a.R) x[r] = ld_once(a.in[r] + i);
        float acc[8];
        bf16x8_to_f32(x[0], acc);
#pragma unroll
        for (int r = 1; r < RB; ++r)
            if (r < a.R) add_bf16x8(acc, x[r]);
        st_once(a.out + i, f32_to_bf16x8(acc));
    }
}

template <int RB>
cudaError_t launch_rb(const SumArgs& a, int sm_count, bool pdl, cudaStream_t stream) {
    // Large calls: 256-thread blocks, 16 per SM (two full residencies; a
    // streaming probe of the same 8:1 read/write mix peaked there on B200),
    // the grid-stride loop covers the rest.  Small calls (fewer vectors than
    // 256 per SM) are latency-bound: smaller blocks spread them over every SM.
    int threads = 256;
    if (a.n_vecs < (int64_t)sm_count * 256) {
        const int64_t per_sm = (a.n_vecs + sm_count - 1) / sm_count;
        threads = (int)((per_sm + 31) / 32 * 32);
        if (threads < 32) threads = 32;
    }
    const int64_t need = (a.n_vecs + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count * 16;
    const unsigned blocks = (unsigned)(need < cap ? need : cap);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, sum_kernel<RB>, a);
}

}  // namespace

cudaError_t launch_sum(const SumArgs& a, int sm_count, bool pdl, cudaStream_t stream) {
    if (a.R <= 2) return launch_rb<2>(a, sm_count, pdl, stream);
    if (a.R <= 4) return launch_rb<4>(a, sm_count, pdl, stream);
    if (a.R <= 8) return launch_rb<8>(a, sm_count, pdl, stream);
    return launch_rb<16>(a, sm_count, pdl, stream);
}

}  // namespace rrf
