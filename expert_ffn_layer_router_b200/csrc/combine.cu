// combine.cu -- router-weighted combine onto the residual, and the fp32 expert FFN.
//
// Combine ("Expert Networks > Worked Example: Expert Specialization", token-0 trace and the
// dropped token 4; "Some Tokens Do Not Get In", "Past the edge"; the fused-MoE dataflow
// diagram's moe_sum step for top_k > 1):
//   out[t] = x[t] + sum over kept j, ascending, of w[t,j] * Y[offsets[id] + slot]
// accumulated in fp32 and rounded once; a token none of whose pairs was kept is copied bit for
// bit (so -0.0 and every payload survive).  One warp per token, 16-byte loads and stores.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kMaxK = 32;

struct F32Traits {
    using T = float;
    static constexpr int kVec = 4;                                  // elements per 16 bytes
    __device__ static void unpack(const uint4& v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    __device__ static uint4 pack(const float (&f)[4]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
    __device__ static float load1(const void* p, size_t i) { return ((const float*)p)[i]; }
    __device__ static void store1(void* p, size_t i, float v) { ((float*)p)[i] = v; }
};

struct BF16Traits {
    static constexpr int kVec = 8;
    __device__ static void unpack(const uint4& v, float (&f)[8]) {
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(u[i] << 16);
            f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        }
    }
    __device__ static uint4 pack(const float (&f)[8]) {
        return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
    }
    __device__ static float load1(const void* p, size_t i) {
        return __uint_as_float((uint32_t)((const uint16_t*)p)[i] << 16);
    }
    __device__ static void store1(void* p, size_t i, float v) {
        __nv_bfloat16 b = __float2bfloat16_rn(v);
        ((uint16_t*)p)[i] = *reinterpret_cast<uint16_t*>(&b);
    }
};

template <class Tr, bool kVector>
__global__ void __launch_bounds__(256) combine_kernel(
    const void* __restrict__ x, const void* __restrict__ Y, const float* __restrict__ w,
    const int32_t* __restrict__ ids, const int32_t* __restrict__ slot,
    const int32_t* __restrict__ offsets, int T, int d, int E, int k, long long max_rows,
    void* __restrict__ out, DeviceStatus* st) {
    pdl_begin();
    constexpr int V = Tr::kVec;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    // Rows and weights of the kept pairs, j ascending (lane j reads pair j).
    int row = -1;
    float wt = 0.0f;
    if (lane < k) {
        const size_t p = (size_t)t * k + lane;
        const int s = slot[p];
        if (s >= 0) {
            const int e = ids[p];
            if ((unsigned)e < (unsigned)E) {
                const long long r = (long long)offsets[e] + s;
                if (r >= 0 && r < offsets[e + 1] && r < max_rows) { row = (int)r; wt = w[p]; }
                else report(st, MOE_DEV_BAD_INDEX, 301);
            } else {
                report(st, MOE_DEV_BAD_INDEX, 302);
            }
        }
    }
    const unsigned kept_mask = __ballot_sync(0xffffffffu, row >= 0);
    int rows[kMaxK];
    float ws[kMaxK];
    int nk = 0;
    for (unsigned m = kept_mask; m; m &= m - 1) {
        const int j = __ffs(m) - 1;
        rows[nk] = __shfl_sync(0xffffffffu, row, j);
        ws[nk] = __shfl_sync(0xffffffffu, wt, j);
        ++nk;
    }
    if (kVector) {
        const int nv = d / V;                                       // 16-byte vectors per row
        const uint4* xr = reinterpret_cast<const uint4*>(x) + (size_t)t * nv;
        uint4* orow = reinterpret_cast<uint4*>(out) + (size_t)t * nv;
        if (nk == 0) {
            for (int c = lane; c < nv; c += 32) orow[c] = __ldg(xr + c);
            return;
        }
        const uint4* Yv = reinterpret_cast<const uint4*>(Y);
        for (int c = lane; c < nv; c += 32) {
            float acc[V];
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = 0.0f;
            for (int q = 0; q < nk; ++q) {
                float yv[V];
                Tr::unpack(__ldg(Yv + (size_t)rows[q] * nv + c), yv);
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = __fmaf_rn(ws[q], yv[i], acc[i]);
            }
            float xv[V];
            Tr::unpack(__ldg(xr + c), xv);
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = __fadd_rn(xv[i], acc[i]);
            orow[c] = Tr::pack(acc);
        }
    } else {
        for (int c = lane; c < d; c += 32) {
            const size_t xi = (size_t)t * d + c;
            if (nk == 0) {
                if (V == 8) ((uint16_t*)out)[xi] = ((const uint16_t*)x)[xi];
                else ((uint32_t*)out)[xi] = ((const uint32_t*)x)[xi];
                continue;
            }
            float acc = 0.0f;
            for (int q = 0; q < nk; ++q)
                acc = __fmaf_rn(ws[q], Tr::load1(Y, (size_t)rows[q] * d + c), acc);
            Tr::store1(out, xi, __fadd_rn(Tr::load1(x, xi), acc));
        }
    }
}

// One warp per token, 16-byte vectors.  The token's kept pairs (row, weight), in j order, are
// held in registers of every lane (KMAX slots, filled by shuffles); for each vector a lane issues
// the loads of x and of all kept rows before any arithmetic (the pair loop is unrolled to KMAX
// with predicates), so k + 1 reads per lane are in flight together.
template <class Tr, int KMAX>
__global__ void __launch_bounds__(256) combine_vec_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ Y, const float* __restrict__ w,
    const int32_t* __restrict__ ids, const int32_t* __restrict__ slot,
    const int32_t* __restrict__ offsets, int T, int nv, int E, int k, long long max_rows,
    uint4* __restrict__ out, DeviceStatus* st) {
    pdl_begin();
    constexpr int V = Tr::kVec;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    int row = -1;
    float wt = 0.0f;
    if (lane < k) {
        const size_t p = (size_t)t * k + lane;
        const int s = slot[p];
        if (s >= 0) {
            const int e = ids[p];
            if ((unsigned)e < (unsigned)E) {
                const long long r = (long long)offsets[e] + s;
                if (r >= 0 && r < offsets[e + 1] && r < max_rows) { row = (int)r; wt = w[p]; }
                else report(st, MOE_DEV_BAD_INDEX, 303);
            } else {
                report(st, MOE_DEV_BAD_INDEX, 304);
            }
        }
    }
    unsigned m = __ballot_sync(0xffffffffu, row >= 0);
    const int nk = __popc(m);
    const uint4* xr = x + (size_t)t * nv;
    uint4* orow = out + (size_t)t * nv;
    if (nk == 0) {
        for (int c = lane; c < nv; c += 32) orow[c] = __ldg(xr + c);
        return;
    }
    size_t rbase[KMAX];
    float wq[KMAX];
#pragma unroll
    for (int q = 0; q < KMAX; ++q) {
        const int src = m ? __ffs(m) - 1 : 0;
        m &= m - 1;
        rbase[q] = (size_t)__shfl_sync(0xffffffffu, row, src) * nv;
        wq[q] = __shfl_sync(0xffffffffu, wt, src);
    }
    for (int c = lane; c < nv; c += 32) {
        const uint4 xv4 = __ldg(xr + c);
        uint4 yv4[KMAX];
#pragma unroll
        for (int q = 0; q < KMAX; ++q)
            if (q < nk) yv4[q] = __ldg(Y + rbase[q] + c);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int q = 0; q < KMAX; ++q) {
            if (q < nk) {
                float yv[V];
                Tr::unpack(yv4[q], yv);
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = __fmaf_rn(wq[q], yv[i], acc[i]);
            }
        }
        float xv[V];
        Tr::unpack(xv4, xv);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = __fadd_rn(xv[i], acc[i]);
        orow[c] = Tr::pack(acc);
    }
}

// Small batches: one block per token, so a token's row is spread over up to 256 threads and each
// thread issues its x and kept-row loads at once (the warp-per-token kernel would leave most of
// the GPU idle with few tokens).
template <class Tr, int KMAX>
__global__ void __launch_bounds__(256) combine_token_block_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ Y, const float* __restrict__ w,
    const int32_t* __restrict__ ids, const int32_t* __restrict__ slot,
    const int32_t* __restrict__ offsets, int nv, int E, int k, long long max_rows,
    uint4* __restrict__ out, DeviceStatus* st) {
    pdl_begin();
    constexpr int V = Tr::kVec;
    __shared__ int s_rows[KMAX];
    __shared__ float s_w[KMAX];
    __shared__ int s_nk;
    const int t = blockIdx.x;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int row = -1;
        float wt = 0.0f;
        if (lane < k) {
            const size_t p = (size_t)t * k + lane;
            const int s = slot[p];
            if (s >= 0) {
                const int e = ids[p];
                if ((unsigned)e < (unsigned)E) {
                    const long long r = (long long)offsets[e] + s;
                    if (r >= 0 && r < offsets[e + 1] && r < max_rows) { row = (int)r; wt = w[p]; }
                    else report(st, MOE_DEV_BAD_INDEX, 305);
                } else {
                    report(st, MOE_DEV_BAD_INDEX, 306);
                }
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, row >= 0);
        if (row >= 0) {
            const int pos = __popc(m & ((1u << lane) - 1u));
            s_rows[pos] = row;
            s_w[pos] = wt;
        }
        if (lane == 0) s_nk = __popc(m);
    }
    __syncthreads();
    const int nk = s_nk;
    const uint4* xr = x + (size_t)t * nv;
    uint4* orow = out + (size_t)t * nv;
    for (int c = threadIdx.x; c < nv; c += blockDim.x) {
        const uint4 xv4 = __ldg(xr + c);
        if (nk == 0) { orow[c] = xv4; continue; }
        uint4 yv4[KMAX];
#pragma unroll
        for (int q = 0; q < KMAX; ++q)
            if (q < nk) yv4[q] = __ldg(Y + (size_t)s_rows[q] * nv + c);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int q = 0; q < KMAX; ++q) {
            if (q < nk) {
                float yv[V];
                Tr::unpack(yv4[q], yv);
                const float wq = s_w[q];
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = __fmaf_rn(wq, yv[i], acc[i]);
            }
        }
        float xv[V];
        Tr::unpack(xv4, xv);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = __fadd_rn(xv[i], acc[i]);
        orow[c] = Tr::pack(acc);
    }
}

// ---------------------------------------------------------------------------------------------
// fp32 expert FFN on CUDA cores (small fp32 layers): one block per kept row.
//   h = W1[e] x + b1[e]; a = SiLU(h) = h / (1 + exp(-h)); Y = W2[e] a + b2[e]
// ("Expert Networks > Worked Example: Expert Specialization", token-0 trace.)
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) ffn_f32_kernel(
    const float* __restrict__ x, const int32_t* __restrict__ rowtok,
    const int32_t* __restrict__ offsets, int E, int T, int d, int F,
    const float* __restrict__ W1, const float* __restrict__ b1, const float* __restrict__ W2,
    const float* __restrict__ b2, float* __restrict__ H, float* __restrict__ Y,
    DeviceStatus* st, int gated) {
    pdl_begin();
    extern __shared__ float s_mem[];
    float* xs = s_mem;          // [d]
    float* as = s_mem + d;      // [F]
    __shared__ int s_e;
    const int r = blockIdx.x;
    // Row ranges given by the caller: offsets[0] = 0, non-decreasing, offsets[E] <= the rows of H
    // and Y (the grid).  Bad offsets: nothing is stored, MOE_DEV_BAD_INDEX is recorded.
    int bad = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) bad |= offsets[e + 1] < offsets[e];
    if (threadIdx.x == 0) bad |= offsets[0] != 0 || offsets[E] > (long long)gridDim.x;
    if (__syncthreads_or(bad)) {
        if (r == 0 && threadIdx.x == 0) report(st, MOE_DEV_BAD_INDEX, 402);
        return;
    }
    if (r >= offsets[E]) return;
    if (threadIdx.x == 0) {
        int lo = 0, hi = E - 1;                  // expert e with offsets[e] <= r < offsets[e+1]
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
        }
        s_e = lo;
    }
    __syncthreads();
    const int e = s_e;
    const int t = rowtok[r];
    if ((unsigned)t >= (unsigned)T) { if (threadIdx.x == 0) report(st, MOE_DEV_BAD_INDEX, 401); return; }
    for (int i = threadIdx.x; i < d; i += blockDim.x) xs[i] = x[(size_t)t * d + i];
    __syncthreads();
    const size_t F1 = gated ? 2 * (size_t)F : (size_t)F;    // W1 rows per expert
    const float* W1e = W1 + (size_t)e * F1 * d;
    for (int f = threadIdx.x; f < F; f += blockDim.x) {
        float h = 0.0f;
        for (int i = 0; i < d; ++i) h = __fmaf_rn(W1e[(size_t)f * d + i], xs[i], h);
        if (b1) h += b1[(size_t)e * F1 + f];
        float a = h / (1.0f + expf(-h));
        if (gated) {                                  // a = SiLU(gate) * up
            float u = 0.0f;
            for (int i = 0; i < d; ++i) u = __fmaf_rn(W1e[(size_t)(F + f) * d + i], xs[i], u);
            if (b1) u += b1[(size_t)e * F1 + F + f];
            a *= u;
        }
        if (H) H[(size_t)r * F + f] = a;
        as[f] = a;
    }
    __syncthreads();
    const float* W2e = W2 + (size_t)e * d * F;
    for (int o = threadIdx.x; o < d; o += blockDim.x) {
        float y = 0.0f;
        for (int f = 0; f < F; ++f) y = __fmaf_rn(W2e[(size_t)o * F + f], as[f], y);
        if (b2) y += b2[(size_t)e * d + o];
        Y[(size_t)r * d + o] = y;
    }
}

// fp32 router logits on CUDA cores: L[t, e] = sum_i x[t, i] Wr[i, e] + br[e], i ascending.
__global__ void logits_f32_kernel(const float* __restrict__ x, const float* __restrict__ Wr,
                                  const float* __restrict__ br, int T, int d, int E,
                                  float* __restrict__ L, int32_t* __restrict__ zero, int zero_n) {
    pdl_begin();
    if (zero)
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < zero_n; i += gridDim.x * blockDim.x)
            zero[i] = 0;
    const long long n = (long long)T * E;
    for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < n;
         q += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(q / E), e = (int)(q % E);
        float acc = 0.0f;
        for (int i = 0; i < d; ++i) acc = __fmaf_rn(x[(size_t)t * d + i], Wr[(size_t)i * E + e], acc);
        L[q] = br ? __fadd_rn(acc, br[e]) : acc;
    }
}

}  // namespace

void launch_logits_f32(const float* x, const float* Wr, const float* br, int T, int d, int E,
                       float* logits, int32_t* zero, int zero_n, cudaStream_t s, int* launches) {
    const long long n = (long long)T * E;
    if (n == 0) return;
    const int blocks = (int)std::min<long long>((n + 255) / 256, 148 * 8);
    launch_pdl(logits_f32_kernel, dim3(blocks), dim3(256), 0, s, x, Wr, br, T, d, E, logits, zero,
               zero_n);
    *launches += 1;
}

void launch_combine(int dtype, const void* x, const void* Y, const float* w, const int32_t* ids,
                    const int32_t* slot, const int32_t* offsets, int T, int d, int E, int k,
                    long long max_rows, void* out, DeviceStatus* st, cudaStream_t s,
                    int* launches) {
    if (T == 0) return;
    const int blocks = (T + 7) / 8;
    const bool aligned = ((uintptr_t)x % 16 == 0) && ((uintptr_t)Y % 16 == 0) &&
                         ((uintptr_t)out % 16 == 0);
    if (dtype == MOE_BF16 && aligned && d % 8 == 0 && k <= 8 && T < 4 * 148) {
        const int nv = d / 8;
        const int threads = std::min(256, ((nv + 31) / 32) * 32);
        launch_pdl(combine_token_block_kernel<BF16Traits, 8>, dim3(T), dim3(threads), 0, s,
                   (const uint4*)x, (const uint4*)Y, w, ids, slot, offsets, nv, E, k, max_rows,
                   (uint4*)out, st);
        *launches += 1;
        return;
    }
    if (dtype == MOE_BF16 && aligned && d % 8 == 0 && k <= 8) {
        launch_pdl(combine_vec_kernel<BF16Traits, 8>, dim3(blocks), dim3(256), 0, s,
                   (const uint4*)x, (const uint4*)Y, w, ids, slot, offsets, T, d / 8, E, k,
                   max_rows, (uint4*)out, st);
        *launches += 1;
        return;
    }
    if (dtype == MOE_BF16) {
        if (aligned && d % 8 == 0)
            launch_pdl(combine_kernel<BF16Traits, true>, dim3(blocks), dim3(256), 0, s, x, Y, w,
                       ids, slot, offsets, T, d, E, k, max_rows, out, st);
        else
            launch_pdl(combine_kernel<BF16Traits, false>, dim3(blocks), dim3(256), 0, s, x, Y, w,
                       ids, slot, offsets, T, d, E, k, max_rows, out, st);
    } else {
        if (aligned && d % 4 == 0)
            launch_pdl(combine_kernel<F32Traits, true>, dim3(blocks), dim3(256), 0, s, x, Y, w, ids,
                       slot, offsets, T, d, E, k, max_rows, out, st);
        else
            launch_pdl(combine_kernel<F32Traits, false>, dim3(blocks), dim3(256), 0, s, x, Y, w,
                       ids, slot, offsets, T, d, E, k, max_rows, out, st);
    }
    *launches += 1;
}

void launch_ffn_f32(const float* x, const int32_t* rowtok, const int32_t* offsets, int E, int T,
                    int d, int F, long long max_rows, const float* W1, const float* b1,
                    const float* W2, const float* b2, float* H, float* Y, DeviceStatus* st,
                    cudaStream_t s, int* launches, bool gated) {
    if (max_rows <= 0) return;
    const size_t smem = sizeof(float) * ((size_t)d + F);
    launch_pdl(ffn_f32_kernel, dim3((unsigned)max_rows), dim3(256), smem, s, x, rowtok, offsets, E,
               T, d, F, W1, b1, W2, b2, H, Y, st, gated ? 1 : 0);
    *launches += 1;
}

}  // namespace moe
