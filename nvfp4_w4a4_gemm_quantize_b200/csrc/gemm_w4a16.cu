// gemm_w4a16.cu -- weights-only NVFP4 GEMM (placeholder until the kernel lands).
#include "internal.h"

namespace nvfp4 {

cudaError_t launch_gemm_w4a16(const GemmW4A16Args& a, int num_sms, cudaStream_t stream) {
    (void)a;
    (void)num_sms;
    (void)stream;
    return cudaErrorNotSupported;
}

}  // namespace nvfp4
