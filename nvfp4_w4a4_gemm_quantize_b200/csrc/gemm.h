// gemm.h -- launch-side declarations of the GEMM kernels (not part of the
// public C ABI).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

struct GemmW4A4Args {
    const uint8_t* a_codes;
    const uint8_t* a_sf;
    const float* a_scale;
    const uint8_t* b_codes;
    const uint8_t* b_sf;
    const float* b_scale;
    int64_t M, N, K;
    void* y;
    int y_dtype;              // 0 bf16, 1 f32
    uint8_t* y_codes;         // fused NVFP4 output (y == nullptr)
    uint8_t* y_sf;
    const float* y_scale;
    float* y_amax;
    int* dev_status;
    int act;                  // epilogue activation: 0 none, 1 GELU (tanh form)
    bool mx;                  // MX operands: blocks of 32, E8M0 scales, no tensor scale
};

cudaError_t launch_gemm_w4a4(const GemmW4A4Args& a, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm_w4a4_grouped(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream);
cudaError_t launch_group_single(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream);
int gemm_w4a4_max_group();
cudaError_t launch_gemm_w4a4_2sm(const GemmW4A4Args& a, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm_w4a4_2sm_grouped(const GemmW4A4Args* probs, int count, int num_sms, cudaStream_t stream);
int gemm_w4a4_2sm_tile_n(const GemmW4A4Args* probs, int count);
bool gemm_w4a4_2sm_supports(int64_t N);

struct GemmW4A16Args {
    const uint16_t* x;
    const uint8_t* w_codes;
    const uint8_t* w_sf;
    const float* w_scale;
    int64_t M, N, K;
    void* y;
    int y_dtype;
    int* dev_status;
};

cudaError_t launch_gemm_w4a16(const GemmW4A16Args& a, int num_sms, cudaStream_t stream);

}  // namespace nvfp4
