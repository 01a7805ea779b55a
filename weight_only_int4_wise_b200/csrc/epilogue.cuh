// The activation of the expert layer's up projection, applied in the GEMM
// epilogues (include/w4a16.h, W4A16_ACT_*).
#pragma once

#include <cuda_fp16.h>

#include "../../include/w4a16.h"

namespace w4a16 {

// Epilogue value: the fp32 accumulator rounded to fp16 (the product's result),
// then, for the expert layer's up projection, the activation evaluated in fp32
// on that fp16 value and rounded to fp16 again. GELU in both of its usual
// forms: x * Phi(x) with Phi the normal CDF (erf form), and the tanh
// approximation with the cubic term 0.044715 x^3. Both are written without
// the sum 1 + (something near -1) that loses all of fp32's digits for negative
// x: Phi(x) = erfc(-x / sqrt 2) / 2, and (1 + tanh u) / 2 = 1 / (1 + e^(-2u)).
__device__ __forceinline__ __half epilogue_value(float acc, int act) {
    const __half h = __float2half_rn(acc);
    if (act == W4A16_ACT_IDENTITY) return h;
    const float x = __half2float(h);
    float y;
    if (act == W4A16_ACT_RELU) {
        y = fmaxf(x, 0.f);
    } else if (act == W4A16_ACT_GELU_ERF) {
        y = 0.5f * x * erfcf(x * -0.70710678118654752f);
    } else {
        const float u = 0.79788456080286536f * (x + 0.044715f * x * x * x);
        y = x / (1.f + expf(-2.f * u));
    }
    return __float2half_rn(y);
}

}  // namespace w4a16
