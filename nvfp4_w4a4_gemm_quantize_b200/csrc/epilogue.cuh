// epilogue.cuh -- the GEMM epilogue's activation, applied to alpha * acc
// before the output (bf16, FP32 or the next layer's NVFP4 codes) is formed.
#pragma once
#include <cstdint>

namespace nvfp4 {

// Epilogue activation applied to alpha * acc before the output is formed.
enum EpiAct { ACT_NONE = 0, ACT_GELU_TANH = 1 };

// GELU in its tanh form, 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))),
// with the hardware tanh approximation (tanh.approx.f32, relative error about
// 2^-11): the activation of the DiT family's MLPs.  Saturates cleanly: large
// negative v gives +0, large positive v gives v.
__device__ __forceinline__ float gelu_tanh(float v) {
    const float u = v * fmaf(0.0356774081f * v, v, 0.7978845608f);   // sqrt(2/pi) (v + 0.044715 v^3)
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
    const float hv = 0.5f * v;
    return fmaf(hv, t, hv);
}

template <int ACT>
__device__ __forceinline__ float epi_value(float alpha, uint32_t acc_bits) {
    const float v = __fmul_rn(alpha, __uint_as_float(acc_bits));
    return ACT == ACT_GELU_TANH ? gelu_tanh(v) : v;
}

}  // namespace nvfp4
