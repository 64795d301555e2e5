// internal.h -- launch-side declarations shared by the library's translation
// units (not part of the public C ABI).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kAmaxThreads = 512;
constexpr int kAmaxMaxCtas = 256;        // partial maxima, one float each
constexpr int kQuantThreads = 512;
constexpr int kFusedSlots = 512;         // one-kernel quantize: (generation, max) per CTA
constexpr size_t kQuantWorkspaceBytes = kFusedSlots * sizeof(unsigned long long);
static_assert(kQuantWorkspaceBytes >= kAmaxMaxCtas * sizeof(float), "workspace holds the two-kernel partials too");
// The tile quantizer's two-kernel form puts one 128-row block per grid row
// (gridDim.y <= 65535), so the quantize entry points accept at most this many
// rows (checked before any launch).
constexpr int64_t kQuantMaxRows = (int64_t)65535 * 128;

void count_launch(int n);

// Per-call number tagging the slots of a grid-wide handoff in a caller's
// workspace (never 0; one counter for every kernel that hands over through
// slots, so no two calls in the process share a number).
uint32_t next_generation();

cudaError_t launch_layernorm_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const float* gamma,
                                      const float* beta, int64_t rows_per_group, double eps, uint8_t* codes,
                                      uint8_t* sf, float* tensor_scale, bool scale_given, unsigned long long* slots,
                                      uint32_t gen, int* dev_status, int num_sms, cudaStream_t stream);
int64_t layernorm_max_k();

int amax_grid(int64_t rows, int64_t k);

cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                            uint8_t* sf, float* tensor_scale, bool scale_given, float* partials,
                            int* dev_status, cudaStream_t stream);

cudaError_t launch_quantize_fused(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                                  uint8_t* sf, float* tensor_scale, unsigned long long* slots, int max_slots,
                                  int* dev_status, int num_sms, cudaStream_t stream);

cudaError_t launch_quantize_block(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, int block, uint8_t* codes,
                                  uint8_t* sf, float* tensor_scale, bool scale_given, void* workspace,
                                  int* dev_status, int num_sms, cudaStream_t stream);

cudaError_t launch_block_size_errors(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                                     const float* tensor_scale, double* errors, int num_sms, cudaStream_t stream);

cudaError_t launch_fake_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, void* y, bool y_f32,
                                 uint8_t* mask, float* tensor_scale, bool scale_given, void* workspace,
                                 int* dev_status, int num_sms, cudaStream_t stream);

cudaError_t launch_ste_backward(const void* grad_y, const uint8_t* mask, int64_t rows, int64_t k, bool f32,
                                void* grad_x, int num_sms, cudaStream_t stream);

cudaError_t launch_mx_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes, uint8_t* sf,
                               cudaStream_t stream);

cudaError_t launch_mx_dequantize(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t k, void* out,
                                 bool bf16, int num_sms, cudaStream_t stream);

cudaError_t launch_attention(const uint8_t* q_codes, const uint8_t* q_sf, const float* g_q, const uint8_t* k_codes,
                             const uint8_t* k_sf, const float* g_k, const uint8_t* v_codes, const uint8_t* v_sf,
                             const float* g_v, const float* s_head, int64_t H, int64_t Lq, int64_t Lk, void* out,
                             void* workspace, int* dev_status, cudaStream_t stream);

size_t attention_workspace_bytes(int64_t H, int64_t Lk, int64_t d);

cudaError_t launch_debug_wait_timeout(int* dev_status, uint64_t limit_ns, cudaStream_t stream);

void reset_noalloc_cache();

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* sf, const float* tensor_scale,
                              int64_t rows, int64_t k, void* out, bool bf16, cudaStream_t stream);

}  // namespace nvfp4
