// softmax.cuh -- the router's fp32 arithmetic, shared by the warp-per-token router (route.cu)
// and the fused router epilogue of the logits GEMM (gemm_tc.cu), so both form bit-identical
// weights from the same logits.
#pragma once

#include <cstdint>

namespace moe {

// exp by Cody-Waite range reduction and a degree-7 Taylor polynomial (W. J. Cody and W. Waite,
// "Software Manual for the Elementary Functions", 1980): x = n ln2 + r, ln2 split into a high
// part with 16 significant bits and a low correction, exp(r) by Horner's rule with fused
// multiply-adds, scaling by 2^n through the exponent field.  Every step is one IEEE single
// operation rounded to nearest even, written with explicit intrinsics so that the compiler can
// neither contract nor reorder them; the result is therefore the same on any IEEE machine that
// evaluates the same steps.  Results below 2^-125 flush to +0 (n < -125), none is subnormal.
__device__ __forceinline__ float exp_cody_waite(float x) {
    if (isnan(x)) return x;
    const float kLog2e = (float)1.4426950408889634074;
    const float kLn2Hi = (float)(45426.0 / 65536.0);
    const float kLn2Lo = (float)(0.6931471805599453094 - 45426.0 / 65536.0);
    const float t = __fmul_rn(x, kLog2e);
    if (t > 200.0f) return __int_as_float(0x7f800000);
    if (t < -200.0f) return 0.0f;
    const float nf = rintf(t);
    const int n = (int)nf;
    if (n < -125) return 0.0f;
    float r = __fmaf_rn(-nf, kLn2Hi, x);
    r = __fmaf_rn(-nf, kLn2Lo, r);
    float p = (float)(1.0 / 5040.0);
    p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    if (n > 127) return __fmul_rn(__fmul_rn(p, __int_as_float(254 << 23)), 2.0f);
    return __fmul_rn(p, __int_as_float((n + 127) << 23));
}

// Order-preserving map of a float (NaN excluded) to uint32; -0 and +0 map to the same key.
__device__ __forceinline__ uint32_t float_key(float v) {
    const uint32_t u = __float_as_uint(__fadd_rn(v, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

}  // namespace moe
