// api.cu -- the C ABI (include/nvfp4.h): host-side argument checks, device
// capability check, and the kernel launches.  No call allocates device memory
// and none synchronizes the host.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/nvfp4.h"
#include "internal.h"
#include "gemm.h"
#include "tmap.h"

namespace nvfp4 {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

CUresult make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                      uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swizzle) {
    (void)elem_bytes;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// ------------------------------------------------------------------ device
struct DevInfo {
    int checked = 0;   // 0 unknown, 1 ok, -1 unsupported
    int sms = 0;
};
static DevInfo g_dev[64];

static nvfp4_status device_ok(int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    DevInfo& d = g_dev[dev];
    if (d.checked == 0) {
        int major = 0, minor = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.sms = n;
        d.checked = (major == 10 && minor == 0) ? 1 : -1;
    }
    if (d.checked < 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    if (sms) *sms = d.sms;
    return NVFP4_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_sf_bytes(int64_t rows, int64_t k) {
    if (rows < 0 || k <= 0 || (k % 64) != 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(k / 16);
}

size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t k) {
    (void)rows;
    (void)k;
    return kQuantWorkspaceBytes;
}

nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, uint8_t* codes, uint8_t* sf,
                            float* tensor_scale, unsigned flags, void* workspace, size_t workspace_bytes,
                            int* dev_status, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0 || ld_x < k) return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)NVFP4_SCALE_GIVEN) != 0u) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!x_bf16 || !codes || !sf)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > kQuantMaxRows || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const bool given = (flags & NVFP4_SCALE_GIVEN) != 0u;
    if (!given && (!workspace || workspace_bytes < kQuantWorkspaceBytes)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(sf) || (ld_x % 8) != 0 ||
        (!given && !aligned16(workspace)) || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0) {
        if (!given) return cuda_status(cudaMemsetAsync(tensor_scale, 0, sizeof(float), s));
        return NVFP4_OK;
    }
    const uint16_t* xb = static_cast<const uint16_t*>(x_bf16);
    if (!given) {
        // one kernel (amax and quantize with a grid-wide handoff); the
        // two-kernel path when the grid cannot be co-resident
        const cudaError_t e = launch_quantize_fused(xb, rows, k, ld_x, codes, sf, tensor_scale,
                                                    static_cast<unsigned long long*>(workspace), kFusedSlots,
                                                    dev_status, sms, s);
        if (e != cudaErrorNotSupported) return cuda_status(e);
    }
    return cuda_status(launch_quantize(xb, rows, k, ld_x, codes, sf, tensor_scale, given, static_cast<float*>(workspace),
                                       dev_status, s));
}

nvfp4_status nvfp4_layernorm_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, const float* gamma,
                                      const float* beta, int64_t rows_per_group, double eps, uint8_t* codes,
                                      uint8_t* sf, float* tensor_scale, unsigned flags, void* workspace,
                                      size_t workspace_bytes, int* dev_status, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0 || ld_x < k || rows_per_group < 0) return NVFP4_ERR_INVALID_ARG;
    if (!(eps > 0.0) || !(eps < 1.0e300)) return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)NVFP4_SCALE_GIVEN) != 0u) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!x_bf16 || !codes || !sf)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > ((int64_t)1 << 31) || k > layernorm_max_k()) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const bool given = (flags & NVFP4_SCALE_GIVEN) != 0u;
    if (!given && (!workspace || workspace_bytes < kQuantWorkspaceBytes)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(sf) || (ld_x % 8) != 0 || !aligned16(gamma) ||
        !aligned16(beta) || (!given && !aligned16(workspace)) || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0) {
        if (!given) return cuda_status(cudaMemsetAsync(tensor_scale, 0, sizeof(float), s));
        return NVFP4_OK;
    }
    return cuda_status(launch_layernorm_quantize(static_cast<const uint16_t*>(x_bf16), rows, k, ld_x, gamma, beta,
                                                 rows_per_group, eps, codes, sf, tensor_scale, given,
                                                 static_cast<unsigned long long*>(workspace),
                                                 given ? 0u : next_generation(), dev_status, sms, s));
}

nvfp4_status nvfp4_quantize_block(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, int block,
                                  uint8_t* codes, uint8_t* sf, float* tensor_scale, unsigned flags, void* workspace,
                                  size_t workspace_bytes, int* dev_status, nvfp4_stream_t stream) {
    if (block != 16 && block != 32 && block != 64) return NVFP4_ERR_INVALID_ARG;
    if (block == 16)
        return nvfp4_quantize(x_bf16, rows, k, ld_x, codes, sf, tensor_scale, flags, workspace, workspace_bytes,
                              dev_status, stream);
    if (rows < 0 || k <= 0 || ld_x < k) return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)NVFP4_SCALE_GIVEN) != 0u) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!x_bf16 || !codes || !sf)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > kQuantMaxRows || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const bool given = (flags & NVFP4_SCALE_GIVEN) != 0u;
    if (!given && (!workspace || workspace_bytes < kQuantWorkspaceBytes)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(sf) || (ld_x % 8) != 0 ||
        (!given && !aligned16(workspace)) || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0) {
        if (!given) return cuda_status(cudaMemsetAsync(tensor_scale, 0, sizeof(float), s));
        return NVFP4_OK;
    }
    return cuda_status(launch_quantize_block(static_cast<const uint16_t*>(x_bf16), rows, k, ld_x, block, codes, sf,
                                             tensor_scale, given, workspace, dev_status, sms, s));
}

nvfp4_status nvfp4_block_size_errors(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                     const float* tensor_scale, double* errors, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0 || ld_x < k) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_scale || !errors || (rows > 0 && !x_bf16)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > (int64_t)1 << 31 || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || (ld_x % 8) != 0 || (reinterpret_cast<uintptr_t>(errors) & 7u) ||
        (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0) return cuda_status(cudaMemsetAsync(errors, 0, 8 * sizeof(double), s));
    return cuda_status(launch_block_size_errors(static_cast<const uint16_t*>(x_bf16), rows, k, ld_x, tensor_scale,
                                                errors, sms, s));
}

int nvfp4_select_block_size(const double* errors, double lambda) {
    if (!errors || !(lambda >= 0.0)) return 0;
    int best = 1;
    double bestv = 0.0;
    for (int i = 0; i < 7; ++i) {
        const int b = 1 << i;
        const double e = errors[7] > 0.0 ? errors[i] / errors[7] : 0.0;
        const double v = e + lambda * (4.0 + 8.0 / b) / 12.0;
        if (i == 0 || v < bestv) {
            bestv = v;
            best = b;
        }
    }
    return best;
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* sf, const float* tensor_scale, int64_t rows,
                              int64_t k, void* out, int out_dtype, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_DTYPE_BF16 && out_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!codes || !sf || !tensor_scale || !out)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(codes) || !aligned16(sf) || !aligned16(out)) return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = device_ok(nullptr);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return cuda_status(launch_dequantize(codes, sf, tensor_scale, rows, k, out, out_dtype == NVFP4_DTYPE_BF16,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_fake_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, void* y, int y_dtype,
                                 uint8_t* clip_mask, float* tensor_scale, unsigned flags, void* workspace,
                                 size_t workspace_bytes, int* dev_status, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0 || ld_x < k) return NVFP4_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)NVFP4_SCALE_GIVEN) != 0u) return NVFP4_ERR_INVALID_ARG;
    if (y_dtype != NVFP4_DTYPE_BF16 && y_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!x_bf16 || !y)) return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > kQuantMaxRows || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const bool given = (flags & NVFP4_SCALE_GIVEN) != 0u;
    if (!given && (!workspace || workspace_bytes < kQuantWorkspaceBytes)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(y) || (clip_mask && !aligned16(clip_mask)) || (ld_x % 8) != 0 ||
        (!given && !aligned16(workspace)) || (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0) {
        if (!given) return cuda_status(cudaMemsetAsync(tensor_scale, 0, sizeof(float), s));
        return NVFP4_OK;
    }
    return cuda_status(launch_fake_quantize(static_cast<const uint16_t*>(x_bf16), rows, k, ld_x, y,
                                            y_dtype == NVFP4_DTYPE_F32, clip_mask, tensor_scale, given, workspace,
                                            dev_status, sms, s));
}

nvfp4_status nvfp4_ste_backward(const void* grad_y, const uint8_t* clip_mask, int64_t rows, int64_t k, int dtype,
                                void* grad_x, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_DTYPE_BF16 && dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!grad_y || !clip_mask || !grad_x)) return NVFP4_ERR_INVALID_ARG;
    if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > (int64_t)1 << 31 || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(grad_y) || !aligned16(clip_mask) || !aligned16(grad_x)) return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return cuda_status(launch_ste_backward(grad_y, clip_mask, rows, k, dtype == NVFP4_DTYPE_F32, grad_x, sms,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

// Checks of one W4A4 problem (shared by the single and the grouped call).
static nvfp4_status check_gemm_problem(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_scale,
                                       const uint8_t* b_codes, const uint8_t* b_sf, const float* b_scale, int64_t M,
                                       int64_t N, int64_t K, const void* y, int y_dtype, const uint8_t* y_codes,
                                       const uint8_t* y_sf, const float* y_scale) {
    if (M < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return NVFP4_OK;
    if (!a_codes || !a_sf || !b_codes || !b_sf || !a_scale || !b_scale) return NVFP4_ERR_INVALID_ARG;
    if (y) {
        if (y_dtype != NVFP4_DTYPE_BF16 && y_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
        if (y_codes || y_sf) return NVFP4_ERR_INVALID_ARG;
    } else {
        if (!y_codes || !y_sf || !y_scale) return NVFP4_ERR_INVALID_ARG;
    }
    if (y && y_dtype == NVFP4_DTYPE_BF16 && N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (y && y_dtype == NVFP4_DTYPE_F32 && N % 4 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!y && N % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(b_codes) || !aligned16(b_sf) || (y && !aligned16(y)) ||
        (y_codes && !aligned16(y_codes)) || (y_sf && !aligned16(y_sf)))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

nvfp4_status nvfp4_gemm_w4a4(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_scale,
                             const uint8_t* b_codes, const uint8_t* b_sf, const float* b_scale, int64_t M, int64_t N,
                             int64_t K, void* y, int y_dtype, uint8_t* y_codes, uint8_t* y_sf, const float* y_scale,
                             float* y_amax, int act, int* dev_status, nvfp4_stream_t stream) {
    const nvfp4_status chk = check_gemm_problem(a_codes, a_sf, a_scale, b_codes, b_sf, b_scale, M, N, K, y, y_dtype,
                                                y_codes, y_sf, y_scale);
    if (chk != NVFP4_OK) return chk;
    if (act != NVFP4_ACT_NONE && act != NVFP4_ACT_GELU_TANH) return NVFP4_ERR_INVALID_ARG;
    if (M == 0) return NVFP4_OK;                 /* nothing to read or write */
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    GemmW4A4Args a{a_codes, a_sf, a_scale, b_codes, b_sf, b_scale, M, N, K, y, y_dtype,
                   y_codes, y_sf, y_scale, y_amax, dev_status, act};
    return cuda_status(launch_gemm_w4a4(a, sms, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm_w4a4_grouped(const nvfp4_gemm_problem* problems, int count, int y_dtype, int* dev_status,
                                     nvfp4_stream_t stream) {
    if (!problems || count < 1 || count > NVFP4_MAX_GROUP) return NVFP4_ERR_INVALID_ARG;
    if (NVFP4_MAX_GROUP > gemm_w4a4_max_group()) return NVFP4_ERR_INVALID_ARG;
    const bool nvfp4_out = problems[0].y == nullptr;
    const int act = problems[0].act;
    if (act != NVFP4_ACT_NONE && act != NVFP4_ACT_GELU_TANH) return NVFP4_ERR_INVALID_ARG;
    GemmW4A4Args args[NVFP4_MAX_GROUP];
    int n = 0;
    for (int i = 0; i < count; ++i) {
        const nvfp4_gemm_problem& q = problems[i];
        if ((q.y == nullptr) != nvfp4_out || q.act != act) return NVFP4_ERR_INVALID_ARG;   // one kind per launch
        const nvfp4_status st = check_gemm_problem(q.a_codes, q.a_sf, q.a_scale, q.b_codes, q.b_sf, q.b_scale, q.M,
                                                   q.N, q.K, q.y, y_dtype, q.y_codes, q.y_sf, q.y_scale);
        if (st != NVFP4_OK) return st;
        if (q.M == 0) continue;                  // nothing to read or write
        args[n++] = GemmW4A4Args{q.a_codes, q.a_sf, q.a_scale, q.b_codes, q.b_sf, q.b_scale, q.M, q.N, q.K,
                                 q.y, y_dtype, q.y_codes, q.y_sf, q.y_scale, q.y_amax, dev_status, act};
    }
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    if (n == 0) return NVFP4_OK;
    return cuda_status(launch_gemm_w4a4_grouped(args, n, sms, reinterpret_cast<cudaStream_t>(stream)));
}

size_t nvfp4_mx_sf_bytes(int64_t rows, int64_t k) {
    if (rows < 0 || k <= 0 || (k % 128) != 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(k / 32);
}

nvfp4_status nvfp4_mx_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, uint8_t* codes, uint8_t* sf,
                               nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0 || ld_x < k) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!x_bf16 || !codes || !sf)) return NVFP4_ERR_INVALID_ARG;
    if (k % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > (int64_t)65535 * 64 || k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(sf) || (ld_x % 8) != 0) return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = device_ok(nullptr);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return cuda_status(launch_mx_quantize(static_cast<const uint16_t*>(x_bf16), rows, k, ld_x, codes, sf,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_mx_dequantize(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t k, void* out,
                                 int out_dtype, nvfp4_stream_t stream) {
    if (rows < 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if (out_dtype != NVFP4_DTYPE_BF16 && out_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (!codes || !sf || !out)) return NVFP4_ERR_INVALID_ARG;
    if (k % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(codes) || !aligned16(sf) || !aligned16(out)) return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return cuda_status(launch_mx_dequantize(codes, sf, rows, k, out, out_dtype == NVFP4_DTYPE_BF16, sms,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_mx_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* b_codes, const uint8_t* b_sf,
                           int64_t M, int64_t N, int64_t K, void* y, int y_dtype, int act, int* dev_status,
                           nvfp4_stream_t stream) {
    if (M < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return NVFP4_OK;
    if (!a_codes || !a_sf || !b_codes || !b_sf || !y) return NVFP4_ERR_INVALID_ARG;
    if (y_dtype != NVFP4_DTYPE_BF16 && y_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
    if (act != NVFP4_ACT_NONE && act != NVFP4_ACT_GELU_TANH) return NVFP4_ERR_INVALID_ARG;
    if (y_dtype == NVFP4_DTYPE_BF16 && N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (y_dtype == NVFP4_DTYPE_F32 && N % 4 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(b_codes) || !aligned16(b_sf) || !aligned16(y))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    GemmW4A4Args a{a_codes, a_sf, nullptr, b_codes, b_sf, nullptr, M, N, K, y, y_dtype,
                   nullptr, nullptr, nullptr, nullptr, dev_status, act, true};
    return cuda_status(launch_gemm_w4a4(a, sms, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_attention(const uint8_t* q_codes, const uint8_t* q_sf, const float* q_scale,
                             const uint8_t* k_codes, const uint8_t* k_sf, const float* k_scale,
                             const uint8_t* v_codes, const uint8_t* v_sf, const float* v_scale,
                             const float* s_head, int64_t H, int64_t Lq, int64_t Lk, int64_t d, void* out,
                             void* workspace, size_t workspace_bytes, int* dev_status, nvfp4_stream_t stream) {
    if (H <= 0 || Lq <= 0 || Lk <= 0 || d <= 0) return NVFP4_ERR_INVALID_ARG;
    if (!q_codes || !q_sf || !q_scale || !k_codes || !k_sf || !k_scale || !v_codes || !v_sf || !v_scale || !out)
        return NVFP4_ERR_INVALID_ARG;
    if (d != 128 || Lq % 128 != 0 || Lk % 128 != 0 || H > 65535 || H * Lq >= ((int64_t)1 << 31) ||
        H * Lk >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!workspace || workspace_bytes < attention_workspace_bytes(H, Lk, d)) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(q_codes) || !aligned16(q_sf) || !aligned16(k_codes) || !aligned16(k_sf) || !aligned16(v_codes) ||
        !aligned16(v_sf) || !aligned16(out) || !aligned16(workspace) ||
        (s_head && (reinterpret_cast<uintptr_t>(s_head) & 3u)))
        return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = device_ok(nullptr);
    if (st != NVFP4_OK) return st;
    return cuda_status(launch_attention(q_codes, q_sf, q_scale, k_codes, k_sf, k_scale, v_codes, v_sf, v_scale,
                                        s_head, H, Lq, Lk, out, workspace, dev_status,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

size_t nvfp4_attention_workspace_bytes(int64_t H, int64_t Lk, int64_t d) {
    if (H <= 0 || Lk <= 0 || d <= 0) return 0;
    return attention_workspace_bytes(H, Lk, d);
}

nvfp4_status nvfp4_gemm_w4a16(const void* x_bf16, const uint8_t* w_codes, const uint8_t* w_sf, const float* w_scale,
                              int64_t M, int64_t N, int64_t K, void* y, int y_dtype, int* dev_status,
                              nvfp4_stream_t stream) {
    if (M < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return NVFP4_OK;                 /* nothing to read or write */
    if (!x_bf16 || !w_codes || !w_sf || !w_scale || !y) return NVFP4_ERR_INVALID_ARG;
    if (y_dtype != NVFP4_DTYPE_BF16 && y_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
    if (K % 64 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (y_dtype == NVFP4_DTYPE_BF16 && N % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (y_dtype == NVFP4_DTYPE_F32 && N % 4 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(y)) return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = device_ok(&sms);
    if (st != NVFP4_OK) return st;
    GemmW4A16Args a{static_cast<const uint16_t*>(x_bf16), w_codes, w_sf, w_scale, M, N, K, y, y_dtype, dev_status};
    return cuda_status(launch_gemm_w4a16(a, sms, reinterpret_cast<cudaStream_t>(stream)));
}

const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case NVFP4_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
        case NVFP4_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.0 (B200)";
        case NVFP4_ERR_CUDA: return "CUDA error";
        case NVFP4_ERR_TIMEOUT: return "device-side wait timed out";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
        case NVFP4_ERR_NONFINITE: return "input holds Inf or NaN";
    }
    return "unknown status";
}

uint64_t nvfp4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void nvfp4_shutdown(void) {
    for (auto& d : g_dev) d = DevInfo{};
    reset_noalloc_cache();
}

nvfp4_status nvfp4_debug_wait_timeout(int* dev_status, int64_t limit_us, nvfp4_stream_t stream) {
    if (!dev_status || limit_us < 1 || limit_us > 2000000) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0u) return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = device_ok(nullptr);
    if (st != NVFP4_OK) return st;
    return cuda_status(launch_debug_wait_timeout(dev_status, (uint64_t)limit_us * 1000ull,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
