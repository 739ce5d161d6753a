// softmax.cuh -- the router's fp32 arithmetic, shared by the routers of route.cu (warp per
// token, group of lanes per token, the small-batch router), so all of them form bit-identical
// weights from the same logits.
//
// One token is routed by one warp: lane l holds experts l, l+32, ...; the softmax sum adds the
// lane partials left to right, then an xor butterfly 16, 8, 4, 2, 1; the top-k picks experts by
// (logit descending, expert ascending) and divides exp(L - m) by the sum once.
#pragma once

#include <cstdint>

#include "common.cuh"

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

// Lane j < k receives the j-th expert of token t (largest logit first) and its weight, writes
// them to ids[t*k + j], w[t*k + j] and returns the expert id; other lanes return -1.
template <int EPL>
__device__ __forceinline__ int route_token_warp(const float* L, int E, int k, size_t t,
                                                int32_t* __restrict__ ids, float* __restrict__ w,
                                                unsigned flags) {
    constexpr unsigned kFull = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    float v[EPL];
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? L[e] : 0.0f;
        key[i] = e < E ? float_key(v[i]) : 0u;
    }
    uint32_t lmax = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) lmax = max(lmax, key[i]);
    const float m = key_float(__reduce_max_sync(kFull, lmax));
    float u[EPL];
    float part = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        u[i] = e < E ? exp_cody_waite(__fsub_rn(v[i], m)) : 0.0f;
        if (e < E) part = __fadd_rn(part, u[i]);
    }
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) part = __fadd_rn(part, __shfl_xor_sync(kFull, part, h));
    const float S = part;

    int my_id = 0;
    float my_w = 0.0f;
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const bool ok = !((taken >> i) & 1u) && key[i] > bk;
            bk = ok ? key[i] : bk;
            bi = ok ? i : bi;
        }
        const uint32_t wk = __reduce_max_sync(kFull, bk);
        const unsigned cand = (bk == wk && bk != 0u) ? (unsigned)(lane + 32 * bi) : 0x7fffffffu;
        const int we = (int)__reduce_min_sync(kFull, cand);
        float up = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) up = (i == bi) ? u[i] : up;
        const float wu = __shfl_sync(kFull, up, we & 31);
        if (lane == (we & 31)) taken |= 1u << (we >> 5);
        if (lane == j) {
            my_id = we;
            my_w = __fdiv_rn(wu, S);
        }
    }
    if (flags & MOE_FLAG_RENORMALIZE) {
        // Sum of the k weights in j order, then one division each.
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(kFull, my_w, j));
        my_w = __fdiv_rn(my_w, sum);
    }
    if (lane < k) {
        ids[t * k + lane] = my_id;
        w[t * k + lane] = my_w;
    }
    return lane < k ? my_id : -1;
}

}  // namespace moe
