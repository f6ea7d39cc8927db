// rrf_noalloc.cu -- rrf_allreduce_rmsnorm_fp8_static: the multi-GPU form run
// with every rank in one launch on this GPU, its signal pads taken from a
// fixed array the library itself holds instead of from the caller.
//
// Who needs it: a caller that cannot allocate device memory.  Examples are
// a host program whose device memory is all owned by another allocator (a
// framework's caching pool that has reserved the GPU, where a separate
// cudaMalloc can fail or fragment what the pool holds), code that must not
// call cudaMalloc / cudaFree because they can synchronise the whole device
// (a latency-bound serving loop), and plug-ins whose host forbids
// allocation after start-up.  Such a caller still owns and passes every
// input and output; only the scratch (the pads) comes from here.
//
// The pads live in one file-scope __device__ array, so every GPU that loads
// the library holds RRF_AR_STATIC_MAX_WORLD pads (544 KiB) until the process
// exits.  All calls share it: each call zeroes the pads it uses (in stream
// order, before its kernel), and calls that overlap on the GPU (two streams,
// or two host threads without ordering between their streams) race on it.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "rrf.h"
#include "rrf_internal.h"

namespace {

constexpr size_t kPadWords = (size_t)RRF_AR_STATIC_MAX_WORLD * RRF_AR_SIGNAL_WORDS;

static __device__ __align__(256) unsigned int g_static_pads[kPadWords];

constexpr int kMaxDevices = 64;
std::atomic<uintptr_t> g_static_pads_addr[kMaxDevices];

// Device address of g_static_pads on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device (with that device current), and kept.
cudaError_t static_pads(unsigned int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cacheable = dev >= 0 && dev < kMaxDevices;
    if (cacheable) {
        const uintptr_t cached = g_static_pads_addr[dev].load(std::memory_order_acquire);
        if (cached != 0) {
            *out = reinterpret_cast<unsigned int*>(cached);
            return cudaSuccess;
        }
    }
    unsigned int* ptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_static_pads);
    if (e != cudaSuccess) return e;
    if (ptr == nullptr) return cudaErrorInvalidSymbol;
    if (cacheable)
        g_static_pads_addr[dev].store(reinterpret_cast<uintptr_t>(ptr), std::memory_order_release);
    *out = ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" rrf_status rrf_allreduce_rmsnorm_fp8_static(
    const void* const* inputs, const void* const* residual_in, void* const* residual_out,
    void* const* q_out, float* const* scales_out, int world, int64_t rows, int64_t cols,
    const void* gamma, float eps, float weight_offset, float scale_ub, int mode,
    uint64_t timeout_ns, rrf_stream_t stream) {
    // The array holds the pads of at most RRF_AR_STATIC_MAX_WORLD ranks.
    if (world < 1 || world > RRF_AR_STATIC_MAX_WORLD) return RRF_ERR_RANKS;
    unsigned int* base = nullptr;
    cudaError_t e = static_pads(&base);
    if (e != cudaSuccess) return rrf::record_cuda_error(e);
    unsigned int* pads[RRF_AR_MAX_WORLD];
    for (int j = 0; j < world; ++j) pads[j] = base + (size_t)j * RRF_AR_SIGNAL_WORDS;
    // Every rank runs in this one launch (the pads are on this GPU only).
    rrf_status st = rrf_check_allreduce_args(inputs, residual_in, residual_out, q_out,
                                             scales_out, pads, world, 0, world, rows, cols,
                                             gamma, eps, weight_offset, scale_ub, mode);
    if (st != RRF_OK || rows == 0) return st;
    // The pads keep the previous call's flags and counters: start from zero.
    e = cudaMemsetAsync(base, 0, (size_t)world * RRF_AR_SIGNAL_WORDS * sizeof(unsigned int),
                        (cudaStream_t)stream);
    if (e != cudaSuccess) return rrf::record_cuda_error(e);
    return rrf_allreduce_rmsnorm_fp8(inputs, residual_in, residual_out, q_out, scales_out, pads,
                                     world, 0, world, rows, cols, gamma, eps, weight_offset,
                                     scale_ub, mode, timeout_ns, stream);
}
