// quantize_noalloc.cu -- nvfp4_quantize_noalloc: the same quantization as
// nvfp4_quantize, for callers that cannot hand the library any scratch
// memory.
//
// Who needs it: code that runs where no device allocation may happen -- a
// plugin inside a host application that owns every byte of device memory
// through its own allocator, an inference server that forbids allocation
// after start-up, or a foreign-language caller with no binding to a CUDA
// allocator.  Such callers can still pass their input and output buffers, but
// not the workspace that the dynamic-scale path of nvfp4_quantize needs for
// the amax pass (one partial maximum per CTA).
//
// Here that scratch is a fixed array in device memory, reserved when the
// library is loaded on a GPU and held until the process exits.  Host code
// cannot use the array's name as a device address: the first call on each
// device asks the runtime for the address (cudaGetSymbolAddress, with that
// device current) and keeps it.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nvfp4.h"
#include "internal.h"

namespace nvfp4 {

// One partial maximum per CTA of the amax pass; that pass never launches more
// than kAmaxMaxCtas CTAs, whatever the tensor size.  The array's size is the
// one the public header states.
constexpr int kNoAllocPartials = NVFP4_NOALLOC_SCRATCH_FLOATS;
static_assert(kNoAllocPartials == kAmaxMaxCtas, "the public scratch size must cover the amax pass's partials");
static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartials];

static float* g_noalloc_ptr[64];
static std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (looked up once
// per device).
static cudaError_t noalloc_scratch(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

static bool noalloc_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void reset_noalloc_cache() {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (auto& q : g_noalloc_ptr) q = nullptr;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                               uint8_t* codes, uint8_t* sf, float* tensor_scale, unsigned flags,
                                               int* dev_status, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0 || ld_x < k) return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)NVFP4_SCALE_GIVEN) != 0u) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!x_bf16 || !codes || !sf)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > kQuantMaxRows || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!noalloc_aligned16(x_bf16) || !noalloc_aligned16(codes) || !noalloc_aligned16(sf) || (ld_x % 8) != 0 ||
        (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    const bool given = (flags & NVFP4_SCALE_GIVEN) != 0u;
    // a problem that would need more partial maxima than the array holds
    if (!given && rows > 0 && amax_grid(rows, k) > kNoAllocPartials) return NVFP4_ERR_WORKSPACE;

    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0) {
        if (!given) return cudaMemsetAsync(tensor_scale, 0, sizeof(float), s) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
        return NVFP4_OK;
    }
    float* partials = nullptr;
    if (!given && noalloc_scratch(&partials) != cudaSuccess) return NVFP4_ERR_CUDA;
    const cudaError_t e = launch_quantize(static_cast<const uint16_t*>(x_bf16), rows, k, ld_x, codes, sf,
                                          tensor_scale, given, partials, dev_status, s);
    return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
