// route.cu -- router softmax/top-k and capacity-limited dispatch (sm_100a).
//
// Step 1, router ("Dynamic Token Routing AI", How it works): a warp, or a group of lanes, per
// token computes the softmax of its E logits in fp32 and keeps the k largest in registers.
// Step 2, capacity ("Expert Networks > Worked Example: Expert Specialization", capacity
// paragraph; "Some Tokens Do Not Get In", "Why there is a buffer" / "Past the edge"): each
// expert keeps at most K pairs, those with the highest router weight (ties: lower token), and
// the slot of a kept pair is its rank among the expert's kept tokens in ascending token order.
//
// Dispatch, two launches, deterministic (no result depends on the order of atomics):
//   route + place: the router (a group of 8, 16 or 32 lanes per token for E <= 64, 128, 256 and
//            k <= the group, one warp per token otherwise) also appends every (token, expert)
//            pair to its expert's candidate list cand[e][.] and counts its weight in a
//            2048-bin histogram of the expert's weights; list positions come from per-block
//            counters in shared memory plus one global atomic per (block, expert) on gcnt[e].
//            The order inside a list is arbitrary.
//   select : one block per expert; if n_e > K the histogram gives the bin that holds the K-th
//            largest weight, and ranking that bin's candidates (ties: lower token first) gives
//            the exact boundary; a radix select on the weight bits covers the cases the
//            histogram cannot (arrival order, a bin of more than 1024 candidates).  The kept
//            tokens are marked in a bitmap over the batch, whose prefix popcounts give each kept
//            pair its slot (its rank in token order), so the result does not depend on the list
//            order.
// The counters and histograms must be zero when the route kernel starts; a launch before it in
// the same call clears them (the router's weight split, the router GEMM itself when the split was
// prepared beforehand, the fp32 logits kernel, or a memset).
#include <atomic>
#include <cfloat>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "softmax.cuh"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------------------------
// Router: softmax over E + top-k, one warp per token (route_token_warp, softmax.cuh).
// ---------------------------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T,
                                                         int E, int k, int32_t* __restrict__ ids,
                                                         float* __restrict__ w, unsigned flags) {
    pdl_begin();
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    route_token_warp<EPL>(logits + (size_t)t * E, E, k, (size_t)t, ids, w, flags);
}

// Router for small batches of bf16 tokens: one block per token computes its E logits on CUDA
// cores and warp 0 routes the token with the same arithmetic as route_topk_kernel.  Thread
// (part, e) reduces d/P consecutive products with four interleaved accumulators (products
// i = i0 + 4j + r go to accumulator r), combined as (a0 + a1) + (a2 + a3); the P parts are then
// added in part order, plus the bias.  Fixed order, so the logits are deterministic.
template <int EPL>
__global__ void __launch_bounds__(1024) router_small_kernel(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ Wr,
    const float* __restrict__ br, int T, int d, int E, int k, float* __restrict__ logits_out,
    int32_t* __restrict__ ids, float* __restrict__ w, unsigned flags) {
    pdl_trigger();                                    // the dispatch after it may be scheduled
    pdl_wait();
    extern __shared__ float s_x[];                    // [d]
    __shared__ float s_part[1024];
    __shared__ float s_L[256];
    const int t = blockIdx.x;
    for (int i = threadIdx.x; i < d; i += blockDim.x)
        s_x[i] = __bfloat162float(x[(size_t)t * d + i]);
    __syncthreads();
    const int P = (int)blockDim.x / E;                // parts of the reduction per expert
    const int tid = threadIdx.x;
    if (tid < P * E) {
        const int e = tid % E, part = tid / E;
        const int i0 = (int)((long long)d * part / P), i1 = (int)((long long)d * (part + 1) / P);
        float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
        int i = i0;
        // 32 weights in flight per thread (the loads do not wait on one another), then the
        // products in the same order as four at a time.
        for (; i + 31 < i1; i += 32) {
            float wv[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) wv[j] = __ldg(Wr + (size_t)(i + j) * E + e);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                a0 = __fmaf_rn(s_x[i + j], wv[j], a0);
                a1 = __fmaf_rn(s_x[i + j + 1], wv[j + 1], a1);
                a2 = __fmaf_rn(s_x[i + j + 2], wv[j + 2], a2);
                a3 = __fmaf_rn(s_x[i + j + 3], wv[j + 3], a3);
            }
        }
        for (; i + 3 < i1; i += 4) {
            const float w0 = __ldg(Wr + (size_t)i * E + e);
            const float w1 = __ldg(Wr + (size_t)(i + 1) * E + e);
            const float w2 = __ldg(Wr + (size_t)(i + 2) * E + e);
            const float w3 = __ldg(Wr + (size_t)(i + 3) * E + e);
            a0 = __fmaf_rn(s_x[i], w0, a0);
            a1 = __fmaf_rn(s_x[i + 1], w1, a1);
            a2 = __fmaf_rn(s_x[i + 2], w2, a2);
            a3 = __fmaf_rn(s_x[i + 3], w3, a3);
        }
        for (; i < i1; ++i) a0 = __fmaf_rn(s_x[i], __ldg(Wr + (size_t)i * E + e), a0);
        s_part[part * E + e] = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    }
    __syncthreads();
    if (tid < E) {
        float L = s_part[tid];
        for (int part = 1; part < P; ++part) L = __fadd_rn(L, s_part[part * E + tid]);
        if (br) L = __fadd_rn(L, br[tid]);
        s_L[tid] = L;
        if (logits_out) logits_out[(size_t)t * E + tid] = L;
    }
    __syncthreads();
    if (tid < 32) route_token_warp<EPL>(s_L, E, k, (size_t)t, ids, w, flags);
}

// Block-wide exclusive scan of one value per thread (blockDim.x a multiple of 32, <= 1024).
// Returns the exclusive prefix; *total receives the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nw ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) s_warp[lane] = s;       // inclusive prefix of warp totals
    }
    __syncthreads();
    const int before = warp ? s_warp[warp - 1] : 0;
    *total = s_warp[nw - 1];
    __syncthreads();
    return before + x - v;
}

// ---------------------------------------------------------------------------------------------
// Route + place.
// ---------------------------------------------------------------------------------------------
// A group of G lanes per token (G = 8, 16, 32 for E <= 64, 128, 256; k <= G).  Lane q of a group
// owns the warp router's lanes l in [q*32/G, (q+1)*32/G) and, for each, experts l, l+32, ...; so
// the fp32 arithmetic is exactly route_token_warp's: m = max; u_e = exp(L_e - m); lane partials
// added left to right; then the pairwise tree p[l] += p[l + h], h = 16, 8, 4, 2, 1 (shuffles down
// within the group where l + h belongs to another lane), which adds the same pairs as the warp's
// xor butterfly; top-k by (logit desc, expert asc); w = u / S.  A block of 16 warps routes 64
// consecutive tokens and places their pairs (block counters in shared memory, one global atomic
// per (block, expert)).
constexpr int kGroupBlockTokens = 64;
constexpr int kGroupWarps = 16;                        // one round of 4 tokens per warp (G = 8)

// Per-expert histogram of the weight keys, built while routing: bin = bits 29..19 of the fp32
// weight (weights are in [0, 1], so bit 30 is 0 and the bin grows with the weight: 7 exponent
// bits and the top 4 mantissa bits).
constexpr int kHistBins = 2048;
__device__ __forceinline__ int hist_bin(float wv) {
    return (int)min(__float_as_uint(wv) >> 19, (uint32_t)(kHistBins - 1));
}

template <int G>
__global__ void __launch_bounds__(kGroupWarps * 32) route_place_group_kernel(
    const float* __restrict__ logits, int T, int E, int k, unsigned flags,
    int32_t* __restrict__ ids, float* __restrict__ w, int32_t* __restrict__ gcnt,
    int32_t* __restrict__ cand, uint32_t* __restrict__ hist, DeviceStatus* st) {
    pdl_begin();
    constexpr int LPL = 32 / G;                        // warp-router lanes per group lane
    constexpr int NI = G / 4;                          // experts per warp-router lane: E <= 32 NI
    constexpr int TPW = kGroupBlockTokens / kGroupWarps;   // tokens per warp
    constexpr int TPP = 32 / G;                        // tokens per warp per round
    constexpr int R = TPW / TPP;                       // rounds
    __shared__ int s_n[32 * NI], s_base[32 * NI];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane / G, q = lane % G;
    for (int e = tid; e < 32 * NI; e += blockDim.x) s_n[e] = 0;
    __syncthreads();
    int my_e[R], my_pos[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        my_e[r] = -1;
        my_pos[r] = 0;
        const int t = blockIdx.x * kGroupBlockTokens + warp * TPW + r * TPP + g;
        const bool active = t < T;                     // group-uniform
        const float* Lr = logits + (size_t)(active ? t : 0) * E;
        float v[LPL][NI];
#pragma unroll
        for (int li = 0; li < LPL; ++li)
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int e = q * LPL + li + 32 * i;
                v[li][i] = (active && e < E) ? __ldg(Lr + e) : 0.0f;
            }
        float m = -INFINITY;
#pragma unroll
        for (int li = 0; li < LPL; ++li)
#pragma unroll
            for (int i = 0; i < NI; ++i)
                if (q * LPL + li + 32 * i < E && v[li][i] > m) m = v[li][i];
#pragma unroll
        for (int o = G / 2; o >= 1; o >>= 1) {
            const float y = __shfl_xor_sync(kFull, m, o, G);
            m = y > m ? y : m;
        }
        float p[LPL];
#pragma unroll
        for (int li = 0; li < LPL; ++li) {
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < NI; ++i)
                if (q * LPL + li + 32 * i < E)
                    acc = __fadd_rn(acc, exp_cody_waite(__fsub_rn(v[li][i], m)));
            p[li] = acc;
        }
#pragma unroll
        for (int h = 16; h >= 1; h >>= 1) {
            if (h >= LPL) {
                const int dl = h / LPL;                // partner lane offset within the group
#pragma unroll
                for (int li = 0; li < LPL; ++li) {
                    const float y = __shfl_down_sync(kFull, p[li], dl, G);
                    if (q < dl) p[li] = __fadd_rn(p[li], y);
                }
            } else {
#pragma unroll
                for (int li = 0; li < LPL; ++li)
                    if (li < h) p[li] = __fadd_rn(p[li], p[li + h]);
            }
        }
        const float S = __shfl_sync(kFull, p[0], 0, G);
        // Top-k: each lane sorts its candidates once by (logit desc, expert asc), invalid ones
        // (e >= E) last; each round the group takes the best head and its owner pops it.
        constexpr int NC = LPL * NI;
        float cl[NC];
        int ce[NC];
#pragma unroll
        for (int li = 0; li < LPL; ++li)
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int e = q * LPL + li + 32 * i;
                cl[li * NI + i] = e < E ? v[li][i] : 0.0f;
                ce[li * NI + i] = e < E ? e : 0x7fffffff;
            }
        // Odd-even transposition sort (NC rounds of neighbour compare-exchange).
#pragma unroll
        for (int rnd = 0; rnd < NC; ++rnd)
#pragma unroll
            for (int a = rnd & 1; a + 1 < NC; a += 2) {
                const bool sw = ce[a + 1] != 0x7fffffff &&
                                (ce[a] == 0x7fffffff || cl[a + 1] > cl[a] ||
                                 (cl[a + 1] == cl[a] && ce[a + 1] < ce[a]));
                const float tl = sw ? cl[a + 1] : cl[a];
                const int te = sw ? ce[a + 1] : ce[a];
                cl[a + 1] = sw ? cl[a] : cl[a + 1];
                ce[a + 1] = sw ? ce[a] : ce[a + 1];
                cl[a] = tl;
                ce[a] = te;
            }
        float my_l = 0.0f;
        int id_j = 0;
        for (int j = 0; j < k; ++j) {
            float bl = cl[0];
            int be = ce[0];
#pragma unroll
            for (int o = G / 2; o >= 1; o >>= 1) {
                const float yl = __shfl_xor_sync(kFull, bl, o, G);
                const int ye = __shfl_xor_sync(kFull, be, o, G);
                if (ye != 0x7fffffff && (be == 0x7fffffff || yl > bl || (yl == bl && ye < be))) {
                    bl = yl;
                    be = ye;
                }
            }
            if (ce[0] == be) {                         // the owner pops its head
#pragma unroll
                for (int a = 0; a + 1 < NC; ++a) { cl[a] = cl[a + 1]; ce[a] = ce[a + 1]; }
                cl[NC - 1] = 0.0f;
                ce[NC - 1] = 0x7fffffff;
            }
            if (q == j) { id_j = be; my_l = bl; }
        }
        // Lane j < k forms weight j: w = exp(L - m) / S; the renormalised form divides by the sum
        // of the k weights added in j order.
        const float w_j = __fdiv_rn(exp_cody_waite(__fsub_rn(my_l, m)), S);
        float wsum = 0.0f;
        if (flags & MOE_FLAG_RENORMALIZE)
            for (int j = 0; j < k; ++j) wsum = __fadd_rn(wsum, __shfl_sync(kFull, w_j, j, G));
        if (active && q < k) {
            const size_t pj = (size_t)t * k + q;
            const float wf = (flags & MOE_FLAG_RENORMALIZE) ? __fdiv_rn(w_j, wsum) : w_j;
            ids[pj] = id_j;
            w[pj] = wf;
            my_e[r] = id_j;
            my_pos[r] = atomicAdd(&s_n[id_j], 1);
            if (hist) atomicAdd(&hist[(size_t)id_j * kHistBins + hist_bin(wf)], 1u);
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) s_base[e] = s_n[e] ? atomicAdd(&gcnt[e], s_n[e]) : 0;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (my_e[r] < 0) continue;
        const int t = blockIdx.x * kGroupBlockTokens + warp * TPW + r * TPP + g;
        const long long pos = (long long)s_base[my_e[r]] + my_pos[r];
        if (pos < T) cand[(size_t)my_e[r] * T + pos] = t * k + q;
        else report(st, MOE_DEV_BAD_INDEX, 131);        // counters were not zero at entry
    }
}

// One warp per token (any E <= 1024, k <= 32): route_token_warp, then the same placement.  A
// block of 8 warps takes 64 consecutive tokens, 8 per warp; lane j keeps pair j of each.
constexpr int kWarpRouteTokens = 64;

template <int EPL>
__global__ void __launch_bounds__(256) route_place_warp_kernel(
    const float* __restrict__ logits, int T, int E, int k, unsigned flags,
    int32_t* __restrict__ ids, float* __restrict__ w, int32_t* __restrict__ gcnt,
    int32_t* __restrict__ cand, uint32_t* __restrict__ hist, DeviceStatus* st) {
    pdl_begin();
    extern __shared__ int s_nb[];                       // [E] counts, then [E] bases
    int* s_n = s_nb;
    int* s_base = s_nb + E;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < E; e += blockDim.x) s_n[e] = 0;
    __syncthreads();
    constexpr int kPer = kWarpRouteTokens / 8;
    int my_e[kPer], my_pos[kPer];
    const int t0 = blockIdx.x * kWarpRouteTokens + warp * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        my_e[i] = -1;
        const int t = t0 + i;
        if (t < T) {
            my_e[i] = route_token_warp<EPL>(logits + (size_t)t * E, E, k, (size_t)t, ids, w, flags);
            if (my_e[i] >= 0) {
                my_pos[i] = atomicAdd(&s_n[my_e[i]], 1);
                if (hist)
                    atomicAdd(&hist[(size_t)my_e[i] * kHistBins + hist_bin(w[(size_t)t * k + lane])],
                              1u);
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) s_base[e] = s_n[e] ? atomicAdd(&gcnt[e], s_n[e]) : 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (my_e[i] >= 0) {
            const long long pos = (long long)s_base[my_e[i]] + my_pos[i];
            if (pos < T) cand[(size_t)my_e[i] * T + pos] = (t0 + i) * k + lane;
            else report(st, MOE_DEV_BAD_INDEX, 132);    // counters were not zero at entry
        }
}

// ---------------------------------------------------------------------------------------------
// Placement of a given routing (no router): pairs p in [0, T*k) with expert ids[p] and weight
// w[p] go to their experts' candidate lists and weight histograms, as the routers above place
// theirs.  Each thread takes kGivenPairs pairs; per-block counters in shared memory ([E] ints,
// dynamic), one global atomic per (block, expert).  An id outside [0, E) is recorded as
// MOE_DEV_BAD_INDEX (site 135) and its pair left out; a weight that is not >= +0 (negative, -0,
// NaN) is recorded (site 134): the selection orders weights by their bit patterns.
// ---------------------------------------------------------------------------------------------
constexpr int kGivenPairs = 4;

__global__ void __launch_bounds__(256) place_given_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ w, long long P, int T, int E,
    int32_t* __restrict__ gcnt, int32_t* __restrict__ cand, uint32_t* __restrict__ hist,
    DeviceStatus* st) {
    pdl_begin();
    extern __shared__ int s_given[];                   // [E] block counts, then [E] bases
    int* s_n = s_given;
    int* s_base = s_given + E;
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) s_n[e] = 0;
    __syncthreads();
    const long long p0 = (long long)blockIdx.x * blockDim.x * kGivenPairs;
    int my_e[kGivenPairs], my_pos[kGivenPairs];
#pragma unroll
    for (int i = 0; i < kGivenPairs; ++i) {
        const long long p = p0 + (long long)i * blockDim.x + tid;
        my_e[i] = -1;
        my_pos[i] = 0;
        if (p >= P) continue;
        const int e = ids[p];
        const float wv = w[p];
        if ((unsigned)e >= (unsigned)E) { report(st, MOE_DEV_BAD_INDEX, 135); continue; }
        if (!(wv >= 0.0f) || (__float_as_uint(wv) >> 31)) report(st, MOE_DEV_BAD_INDEX, 134);
        my_e[i] = e;
        my_pos[i] = atomicAdd(&s_n[e], 1);
        if (hist) atomicAdd(&hist[(size_t)e * kHistBins + hist_bin(wv)], 1u);
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) s_base[e] = s_n[e] ? atomicAdd(&gcnt[e], s_n[e]) : 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kGivenPairs; ++i) {
        if (my_e[i] < 0) continue;
        const long long p = p0 + (long long)i * blockDim.x + tid;
        const long long pos = (long long)s_base[my_e[i]] + my_pos[i];
        if (pos < T) cand[(size_t)my_e[i] * T + pos] = (int32_t)p;
        else report(st, MOE_DEV_BAD_INDEX, 133);       // a token listed one expert twice, or
    }                                                  // the counters were not zero at entry
}

// ---------------------------------------------------------------------------------------------
// Capacity selection from unordered candidate lists: one block per expert.
// ---------------------------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelSmem = 200 * 1024;  // dynamic shared memory of the selection kernel (the
                                      // static arrays take about 9 KB more)
constexpr int kSelBitWords = 8192;    // token-bitmap words kept on chip (T <= 262144)

// Radix select over the keys of candidates i < n (most significant byte first), restricted to
// those with filter(i): finds the `want`-th largest key; returns it, and in *rem how many
// candidates equal to it are among the `want` largest.
template <class KeyFn, class FilterFn>
__device__ __forceinline__ uint32_t radix_select(int n, int want, KeyFn key_of, FilterFn filter,
                                                 int* s_hist, uint32_t* s_prefix, int* s_rem,
                                                 int* rem) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0, mask = 0;
    int remaining = want;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < 256; b += blockDim.x) s_hist[b] = 0;
        __syncthreads();
        // Keys share few values in their high bytes (softmax weights differ mostly in the
        // mantissa): one atomic per distinct bin per warp, not per key.
        for (int i0 = 0; i0 < n; i0 += blockDim.x) {
            const int i = i0 + tid;
            int bin = -1;
            if (i < n && filter(i)) {
                const uint32_t key = key_of(i);
                if ((key & mask) == prefix) bin = (int)((key >> shift) & 255u);
            }
            const unsigned peers = __match_any_sync(kFull, bin);
            if (bin >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1)
                atomicAdd(&s_hist[bin], __popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            // Lane l owns bins 255-8l .. 248-8l (top-down); find the bin where the running
            // count from the top reaches `remaining`.
            int loc = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) loc += s_hist[255 - 8 * tid - q];
            int inc = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, inc, o);
                if (tid >= o) inc += y;
            }
            const int exc = inc - loc;
            const unsigned hit = __ballot_sync(kFull, inc >= remaining && exc < remaining);
            const int owner = __ffs(hit) - 1;
            if (tid == owner) {
                int run = exc;
                for (int q = 0; q < 8; ++q) {
                    const int b = 255 - 8 * tid - q;
                    if (run + s_hist[b] >= remaining) {
                        *s_prefix = prefix | ((uint32_t)b << shift);
                        *s_rem = remaining - run;
                        break;
                    }
                    run += s_hist[b];
                }
            }
        }
        __syncthreads();
        prefix = *s_prefix;
        remaining = *s_rem;
        mask |= 255u << shift;
        __syncthreads();
    }
    *rem = remaining;
    return prefix;
}

// Keys order candidates by priority, larger first: the weight's bit pattern (weights are >= +0,
// so their bits order like their values), or for MOE_FLAG_ARRIVAL_ORDER the complement of the
// pair index (earlier tokens first).  Among equal weights the lower pair index (the lower
// token) wins.  `gbits` (null when the bitmap fits on chip) is [E][2 * ceil(T/32)] words.
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const int32_t* __restrict__ cand, const int32_t* __restrict__ gcnt,
    const float* __restrict__ w, int T, int E, int k, long long K, unsigned flags,
    uint32_t* __restrict__ gbits, int keys_cap, const uint32_t* __restrict__ hist,
    int32_t* __restrict__ slot, uint8_t* __restrict__ drop, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ rowtok, DeviceStatus* st) {
    pdl_begin();
    extern __shared__ uint32_t s_dyn[];
    __shared__ int s_warp[32];
    __shared__ uint32_t s_tk[kSelThreads];    // tie bin: keys and pair indices
    __shared__ int32_t s_tp[kSelThreads];
    __shared__ int s_nt, s_bstar, s_need, s_found, s_b2, s_need2;
    __shared__ int s_hist[256];
    __shared__ int s_h2[kHistBins];           // second-level histogram of the threshold bin
    __shared__ uint32_t s_prefix;
    __shared__ int s_rem;
    const int e = blockIdx.x, tid = threadIdx.x;
    const int nw = (T + 31) / 32;
    uint32_t* bits = gbits ? gbits + (size_t)e * 2 * nw : s_dyn;       // [nw] kept tokens
    uint32_t* pre = bits + nw;                                          // [nw] prefix popcounts
    uint32_t* s_keys = s_dyn + (gbits ? 0 : 2 * nw);                   // [keys_cap]
    int32_t* s_list = reinterpret_cast<int32_t*>(s_keys + keys_cap);   // [keys_cap]
    const long long P = (long long)T * k;

    int n = gcnt[e];
    if (n < 0 || n > T) {
        if (tid == 0) report(st, MOE_DEV_BAD_INDEX, 121);
        n = n < 0 ? 0 : T;
    }
    const int kept = (int)min((long long)n, K);
    // Row offset of this expert: kept counts of the experts before it.
    int part = 0;
    for (int q = tid; q < e; q += blockDim.x) part += (int)min((long long)min(max(gcnt[q], 0), T), K);
    int off;
    (void)block_exclusive_scan(part, s_warp, &off);
    if (tid == 0) {
        if (counts) { counts[e] = n; counts[E + e] = kept; }
        if (offsets) {
            offsets[e] = off;
            if (e == E - 1) offsets[E] = off + kept;
        }
    }
    if (n == 0) return;
    const int32_t* list = cand + (size_t)e * T;
    const bool arrival = (flags & MOE_FLAG_ARRIVAL_ORDER) != 0;
    const bool on_chip = n <= keys_cap;
    auto pair_of = [&](int i) -> int32_t {
        const int32_t p = on_chip ? s_list[i] : list[i];
        return p;
    };
    auto key_from = [&](int32_t p) -> uint32_t {
        return arrival ? ~(uint32_t)p : __float_as_uint(w[p]);
    };
    const bool need_keys = n > K && K > 0;      // otherwise every candidate is kept
    if (on_chip) {
        // Eight candidates per thread in flight: their list entries, then their weights.
        for (int i0 = 0; i0 < n; i0 += 8 * kSelThreads) {
            int32_t pv[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const int i = i0 + b * kSelThreads + tid;
                pv[b] = i < n ? list[i] : -1;
            }
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const int i = i0 + b * kSelThreads + tid;
                if (i >= n) continue;
                int32_t p = pv[b];
                if (p < 0 || p >= P) { report(st, MOE_DEV_BAD_INDEX, 122); p = -1; }
                s_list[i] = p;
                s_keys[i] = (p < 0 || !need_keys) ? 0u : key_from(p);
            }
        }
    }
    for (int i = tid; i < nw; i += blockDim.x) bits[i] = 0;
    __syncthreads();
    auto key_of = [&](int i) -> uint32_t {
        if (on_chip) return s_keys[i];
        const int32_t p = list[i];
        return (p < 0 || p >= P) ? 0u : key_from(p);
    };
    auto valid = [&](int i) -> bool {
        const int32_t p = pair_of(i);
        return p >= 0 && p < P;
    };

    uint32_t tau = 0;                 // keys > tau are kept; keys == tau when pair <= p_tau
    int32_t p_tau = 0x7fffffff;
    bool select_all = n <= K;
    bool by_hist = false;
    int bstar = 0;
    if (!select_all && K > 0 && hist && !arrival) {
        // Threshold bin from the histogram: thread t holds bins 2047 - 2t and 2046 - 2t (top
        // down); b* is the bin where the count from the top reaches K.  Keys above b* are kept,
        // below dropped; the `need` largest (ties: lower pair) of bin b* are kept.  A second
        // histogram of bin b*'s keys over their next 11 bits (18..8) narrows the boundary to one
        // sub-bin b2, whose few candidates are ranked exactly by (key desc, pair asc).  Any
        // inconsistency (histogram total != n, the top bin, more than one candidate per thread
        // in b2) falls back to the radix selection below.
        const uint32_t* h = hist + (size_t)e * kHistBins;
        const int b_hi = kHistBins - 1 - 2 * tid, b_lo = b_hi - 1;
        const int c_hi = (int)h[b_hi], c_lo = (int)h[b_lo];
        if (tid == 0) { s_nt = 0; s_bstar = -1; s_found = 0; s_b2 = -1; }
        s_h2[b_hi] = 0;
        s_h2[b_lo] = 0;
        int tot;
        const int above = block_exclusive_scan(c_hi + c_lo, s_warp, &tot);
        if (above < K && above + c_hi >= K) {
            s_bstar = b_hi;
            s_need = (int)(K - above);
        } else if (above + c_hi < K && above + c_hi + c_lo >= K) {
            s_bstar = b_lo;
            s_need = (int)(K - above - c_hi);
        }
        __syncthreads();
        bstar = s_bstar;
        const int need = s_need;
        if (tot == n && bstar >= 0 && bstar < kHistBins - 1) {
            for (int i = tid; i < n; i += blockDim.x) {
                if (!valid(i)) continue;
                const uint32_t key = key_of(i);
                if ((int)(key >> 19) == bstar) atomicAdd(&s_h2[(key >> 8) & (kHistBins - 1)], 1);
            }
            __syncthreads();
            const int d_hi = s_h2[b_hi], d_lo = s_h2[b_lo];
            int tot2;
            const int above2 = block_exclusive_scan(d_hi + d_lo, s_warp, &tot2);
            if (above2 < need && above2 + d_hi >= need) {
                s_b2 = b_hi;
                s_need2 = need - above2;
            } else if (above2 + d_hi < need && above2 + d_hi + d_lo >= need) {
                s_b2 = b_lo;
                s_need2 = need - above2 - d_hi;
            }
            __syncthreads();
            const int b2 = s_b2, need2 = s_need2;
            const int mt = b2 >= 0 ? s_h2[b2] : kSelThreads + 1;
            if (mt <= kSelThreads) {
                const uint32_t pre24 = ((uint32_t)bstar << 11) | (uint32_t)b2;   // key bits 29..8
                for (int i = tid; i < n; i += blockDim.x) {
                    if (!valid(i)) continue;
                    const uint32_t key = key_of(i);
                    if ((key >> 8) == pre24) {
                        const int at = atomicAdd(&s_nt, 1);
                        if (at < kSelThreads) { s_tk[at] = key; s_tp[at] = pair_of(i); }
                    }
                }
                __syncthreads();
                const int m = s_nt;
                // Rank of each candidate of b2 by (key desc, pair asc); the need2-th one bounds
                // the kept set: key > tau, or key == tau and pair <= p_tau.
                if (m == mt && tid < m) {
                    const uint32_t kt = s_tk[tid];
                    const int32_t pt = s_tp[tid];
                    int rank = 0;
                    for (int j = 0; j < m; ++j) {
                        const uint32_t kj = s_tk[j];
                        rank += (kj > kt || (kj == kt && s_tp[j] < pt)) ? 1 : 0;
                    }
                    if (rank == need2 - 1) { s_prefix = kt; s_rem = pt; s_found = 1; }
                }
                __syncthreads();
                if (s_found) {
                    by_hist = true;
                    tau = s_prefix;
                    p_tau = s_rem;
                }
            }
        }
    }
    if (!select_all && K > 0 && !by_hist) {
        int need_eq;
        tau = radix_select(n, (int)K, key_of, valid, s_hist, &s_prefix, &s_rem, &need_eq);
        // Candidates equal to tau: are all of them among the K largest?  Count them.
        int eqc = 0;
        for (int i = tid; i < n; i += blockDim.x) eqc += (valid(i) && key_of(i) == tau) ? 1 : 0;
        int eq_tot;
        (void)block_exclusive_scan(eqc, s_warp, &eq_tot);
        if (eq_tot > need_eq) {
            // Ties straddle the boundary: keep the need_eq tied pairs with the lowest index.
            int dummy;
            p_tau = (int32_t)~radix_select(
                n, need_eq, [&](int i) -> uint32_t { return ~(uint32_t)pair_of(i); },
                [&](int i) -> bool { return valid(i) && key_of(i) == tau; }, s_hist, &s_prefix,
                &s_rem, &dummy);
        }
    }
    // Mark kept tokens.  (With the histogram, tau lies in bin b*: keys in higher bins are above
    // tau and keys in lower bins below it, so the same rule holds.)
    for (int i = tid; i < n; i += blockDim.x) {
        if (!valid(i)) continue;
        const int32_t p = pair_of(i);
        const uint32_t key = key_of(i);
        const bool keep = K > 0 && (select_all || key > tau || (key == tau && p <= p_tau));
        if (keep) {
            const int t = p / k;
            atomicOr(&bits[t >> 5], 1u << (t & 31));
        }
    }
    __syncthreads();
    // Exclusive prefix of popcounts over the bitmap words, 1024 words per round.
    int carry = 0;
    for (int w0 = 0; w0 < nw; w0 += blockDim.x) {
        const int wi = w0 + tid;
        const int c = wi < nw ? __popc(bits[wi]) : 0;
        int tot;
        const int ex = block_exclusive_scan(c, s_warp, &tot);
        if (wi < nw) pre[wi] = carry + ex;
        carry += tot;
    }
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
        if (!valid(i)) continue;
        const int32_t p = pair_of(i);
        const int t = p / k;
        const uint32_t word = bits[t >> 5], bit = 1u << (t & 31);
        if (word & bit) {
            const int sl = (int)pre[t >> 5] + __popc(word & (bit - 1u));
            if (sl >= kept) {                   // only with duplicated pairs in the list
                report(st, MOE_DEV_BAD_INDEX, 123);
                continue;
            }
            slot[p] = sl;
            drop[p] = 0;
        } else {
            slot[p] = -1;
            drop[p] = 1;
        }
    }
    // Row map in token order, one bitmap word per thread: each thread writes the rows of its
    // word's kept tokens, and neighbouring threads write neighbouring rows.
    if (rowtok) {
        for (int wi = tid; wi < nw; wi += blockDim.x) {
            uint32_t word = bits[wi];
            int sl = (int)pre[wi];
            while (word) {
                const int j = __ffs(word) - 1;
                word &= word - 1u;
                if (sl < kept) rowtok[off + sl] = wi * 32 + j;
                ++sl;
            }
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Small batches (T*k <= kSmallPairs): counting, capacity selection, slots, offsets and the row
// map in one block, one launch.  Same results as the two-launch dispatch above: candidates of an
// expert are kept in ascending token order (warp-serial stable placement), an overflowing
// expert keeps its K pairs of largest (weight, then lower token) -- or its first K with
// MOE_FLAG_ARRIVAL_ORDER -- and slots rank the kept tokens in ascending token order.
// ---------------------------------------------------------------------------------------------
constexpr int kSmallPairs = 1024;

__device__ __forceinline__ void dispatch_small_block(
    const int32_t* __restrict__ ids, const float* __restrict__ w, int T, int E, int k,
    long long K, unsigned flags, int32_t* __restrict__ slot, uint8_t* __restrict__ drop,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ rowtok,
    DeviceStatus* st, int32_t* sm) {
    __shared__ int s_warp[32];
    const int P = T * k;
    int32_t* cnt = sm;                 // [E]
    int32_t* start = cnt + E;          // [E + 1]
    int32_t* run = start + E + 1;      // [E]
    int32_t* koff = run + E;           // [E + 1] kept offsets
    int32_t* list = koff + E + 1;      // [P] pair index, grouped by expert, ascending token
    int32_t* lexp = list + P;          // [P] expert of each list position
    int32_t* s_ids = lexp + P;         // [P] the routing, read from global memory once
    float* s_w = reinterpret_cast<float*>(s_ids + P);      // [P]
    uint8_t* keep = reinterpret_cast<uint8_t*>(s_w + P);   // [P]
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = ids[p];
        s_ids[p] = e;
        s_w[p] = w[p];
        if ((unsigned)e < (unsigned)E) atomicAdd(&cnt[e], 1);
        else report(st, MOE_DEV_BAD_INDEX, 111);
    }
    __syncthreads();
    // start = exclusive prefix of received counts, koff = of kept counts.
    int carry = 0, kcarry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + tid;
        const int v = e < E ? cnt[e] : 0;
        const int kv = e < E ? (int)min((long long)v, K) : 0;
        int tot, ktot;
        const int ex = block_exclusive_scan(v, s_warp, &tot);
        const int kex = block_exclusive_scan(kv, s_warp, &ktot);
        if (e < E) { start[e] = carry + ex; run[e] = carry + ex; koff[e] = kcarry + kex; }
        carry += tot;
        kcarry += ktot;
    }
    if (tid == 0) { start[E] = carry; koff[E] = kcarry; }
    __syncthreads();
    if (tid < 32) {                                   // stable placement, 32 pairs at a time
        for (int pb = 0; pb < P; pb += 32) {
            const int p = pb + tid;
            int e = p < P ? s_ids[p] : -1;
            if ((unsigned)e >= (unsigned)E) e = -1;
            const unsigned peers = __match_any_sync(kFull, e);
            const int rank = __popc(peers & ((1u << tid) - 1u));
            const int pos = e >= 0 ? run[e] + rank : 0;
            __syncwarp();
            if (e >= 0) {
                list[pos] = p;
                lexp[pos] = e;
                if (tid == __ffs(peers) - 1) run[e] = pos + __popc(peers);
            }
            __syncwarp();
        }
    }
    __syncthreads();
    const bool arrival = (flags & MOE_FLAG_ARRIVAL_ORDER) != 0;
    for (int i = tid; i < carry; i += blockDim.x) {
        const int e = lexp[i];
        const int b0 = start[e], n = start[e + 1] - b0, pos = i - b0;
        bool kp;
        if (n <= K || arrival) {
            kp = pos < K;
        } else {
            const int p = list[i];
            const float wi = s_w[p];
            int rank = 0;
            for (int j = b0; j < b0 + n; ++j) {
                const float wj = s_w[list[j]];
                rank += (wj > wi || (wj == wi && j < i)) ? 1 : 0;
            }
            kp = rank < K;
        }
        keep[i] = kp ? 1 : 0;
    }
    __syncthreads();
    for (int i = tid; i < carry; i += blockDim.x) {
        const int e = lexp[i];
        const int b0 = start[e];
        const int p = list[i];
        if (keep[i]) {
            int s = 0;
            for (int j = b0; j < i; ++j) s += keep[j];
            slot[p] = s;
            drop[p] = 0;
            if (rowtok) rowtok[koff[e] + s] = p / k;
        } else {
            slot[p] = -1;
            drop[p] = 1;
        }
    }
    for (int e = tid; e < E; e += blockDim.x) {
        if (counts) { counts[e] = cnt[e]; counts[E + e] = koff[e + 1] - koff[e]; }
        if (offsets) offsets[e] = koff[e];
    }
    if (tid == 0 && offsets) offsets[E] = koff[E];
}

__global__ void __launch_bounds__(1024) dispatch_small_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ w, int T, int E, int k,
    long long K, unsigned flags, int32_t* __restrict__ slot, uint8_t* __restrict__ drop,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ rowtok,
    DeviceStatus* st) {
    pdl_trigger();                                    // the expert GEMM may be scheduled (it
    pdl_wait();                                       // prefetches its weights, then waits)
    extern __shared__ int32_t sm[];
    dispatch_small_block(ids, w, T, E, k, K, flags, slot, drop, counts, offsets, rowtok, st, sm);
}

// ---------------------------------------------------------------------------------------------
// Dispatch from a given routing (moe_dispatch).
// ---------------------------------------------------------------------------------------------
__global__ void kept_count_kernel(const int32_t* __restrict__ ids,
                                  const int32_t* __restrict__ slot, long long P, int E, int T,
                                  int32_t* __restrict__ kept, DeviceStatus* st) {
    pdl_begin();
    for (long long p = blockIdx.x * (long long)blockDim.x + threadIdx.x; p < P;
         p += (long long)gridDim.x * blockDim.x) {
        const int s = slot[p];
        if (s < 0) continue;
        const int e = ids[p];
        if ((unsigned)e >= (unsigned)E || s >= T) { report(st, MOE_DEV_BAD_INDEX, 201); continue; }
        atomicAdd(&kept[e], 1);
    }
}

__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ kept, int E,
                                                       int32_t* __restrict__ offsets) {
    pdl_begin();
    __shared__ int s_warp[32];
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        const int v = e < E ? kept[e] : 0;
        int tot;
        const int ex = block_exclusive_scan(v, s_warp, &tot);
        if (e < E) offsets[e] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) offsets[E] = carry;
}

__global__ void rowtok_scatter_kernel(const int32_t* __restrict__ ids,
                                      const int32_t* __restrict__ slot, long long P, int E, int k,
                                      const int32_t* __restrict__ offsets,
                                      int32_t* __restrict__ rowtok, DeviceStatus* st) {
    pdl_begin();
    for (long long p = blockIdx.x * (long long)blockDim.x + threadIdx.x; p < P;
         p += (long long)gridDim.x * blockDim.x) {
        const int s = slot[p];
        if (s < 0) continue;
        const int e = ids[p];
        if ((unsigned)e >= (unsigned)E) continue;
        const int r = offsets[e] + s;
        if (r >= offsets[e + 1]) { report(st, MOE_DEV_BAD_INDEX, 202); continue; }
        rowtok[r] = (int32_t)(p / k);
    }
}

// x_perm[r] = x[rowtok[r]], 16-byte vectors (row bytes a multiple of 16) or 4-byte words.
template <typename V>
__global__ void permute_rows_kernel(const V* __restrict__ x, const int32_t* __restrict__ rowtok,
                                    const int32_t* __restrict__ offsets, int E, int vpr, int T,
                                    V* __restrict__ xp, DeviceStatus* st) {
    pdl_begin();
    const int rows = offsets[E];
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)rows * vpr;
         i += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(i / vpr), c = (int)(i % vpr);
        const int t = rowtok[r];
        if ((unsigned)t >= (unsigned)T) { report(st, MOE_DEV_BAD_INDEX, 203); continue; }
        xp[i] = x[(size_t)t * vpr + c];
    }
}

template <int EPL>
void launch_route_t(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                    cudaStream_t s, unsigned flags) {
    const int blocks = (T + 7) / 8;
    launch_pdl(route_topk_kernel<EPL>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, ids, w,
               flags);
}

}  // namespace

void launch_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                       cudaStream_t s, unsigned flags) {
    const int epl = (E + 31) / 32;
    if (epl <= 1) launch_route_t<1>(logits, T, E, k, ids, w, s, flags);
    else if (epl <= 2) launch_route_t<2>(logits, T, E, k, ids, w, s, flags);
    else if (epl <= 4) launch_route_t<4>(logits, T, E, k, ids, w, s, flags);
    else if (epl <= 8) launch_route_t<8>(logits, T, E, k, ids, w, s, flags);
    else if (epl <= 16) launch_route_t<16>(logits, T, E, k, ids, w, s, flags);
    else launch_route_t<32>(logits, T, E, k, ids, w, s, flags);
}


bool dispatch_small_fits(int T, int k) { return (long long)T * k <= kSmallPairs; }

bool router_small_fits(int T, int E, int d) { return T <= 1024 && E <= 256 && d <= 12288; }

void launch_router_small(const void* x, const float* Wr, const float* br, int T, int d, int E,
                         int k, float* logits_out, int32_t* ids, float* w, unsigned flags,
                         cudaStream_t s, int* launches) {
    const size_t smem = sizeof(float) * (size_t)d;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    const int epl = (E + 31) / 32;
    if (epl <= 1)
        launch_pdl(router_small_kernel<1>, dim3(T), dim3(1024), smem, s, xb, Wr, br, T, d, E, k,
                   logits_out, ids, w, flags);
    else if (epl <= 2)
        launch_pdl(router_small_kernel<2>, dim3(T), dim3(1024), smem, s, xb, Wr, br, T, d, E, k,
                   logits_out, ids, w, flags);
    else if (epl <= 4)
        launch_pdl(router_small_kernel<4>, dim3(T), dim3(1024), smem, s, xb, Wr, br, T, d, E, k,
                   logits_out, ids, w, flags);
    else
        launch_pdl(router_small_kernel<8>, dim3(T), dim3(1024), smem, s, xb, Wr, br, T, d, E, k,
                   logits_out, ids, w, flags);
    *launches += 1;
}

namespace {
// Failure-detection self-test: waits on an mbarrier that nothing arrives on, with the same
// bounded wait the pipelines use; the wait gives up and records MOE_DEV_TIMEOUT.
__global__ void wait_timeout_selftest_kernel(DeviceStatus* st, unsigned long long limit_ns) {
    pdl_begin();
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) mbar_init(b, 1);
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(b, 0, st, 901, limit_ns);
    __syncthreads();
}
}  // namespace

void launch_wait_timeout_selftest(DeviceStatus* st, long long limit_ns, cudaStream_t s) {
    launch_pdl(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0, s, st,
               (unsigned long long)limit_ns);
}

void launch_dispatch_small(const int32_t* ids, const float* w, int T, int E, int k, long long K,
                           unsigned flags, int32_t* slot, uint8_t* drop, int32_t* counts,
                           int32_t* offsets, int32_t* rowtok, DeviceStatus* st, cudaStream_t s,
                           int* launches) {
    const int P = T * k;
    const size_t smem = sizeof(int32_t) * (4 * (size_t)E + 2 + 4 * (size_t)P) + (size_t)P;
    launch_pdl(dispatch_small_kernel, dim3(1), dim3(1024), smem, s, ids, w, T, E, k, K, flags, slot,
               drop, counts, offsets, rowtok, st);
    *launches += 1;
}

// Lanes per token of the group router (0: the warp router with more experts per lane).
int route_group_lanes(int E, int k) {
    const int G = E <= 64 ? 8 : (E <= 128 ? 16 : (E <= 256 ? 32 : 0));
    return (G > 0 && k <= G) ? G : 0;
}

size_t dispatch_counter_ints(int E) { return (size_t)E * (1 + kHistBins); }

void launch_route_place(const float* logits, int T, int E, int k, unsigned flags, int32_t* ids,
                        float* w, int32_t* gcnt, int32_t* cand, DeviceStatus* st, cudaStream_t s,
                        int* launches) {
    // The histogram follows the counters; arrival-order selection does not use it.
    uint32_t* hist = (flags & MOE_FLAG_ARRIVAL_ORDER) ? nullptr
                                                      : reinterpret_cast<uint32_t*>(gcnt + E);
    if (T == 0) return;
    const int G = route_group_lanes(E, k);
    if (G > 0) {
        const dim3 g((T + kGroupBlockTokens - 1) / kGroupBlockTokens);
        if (G == 8)
            launch_pdl(route_place_group_kernel<8>, g, dim3(kGroupWarps * 32), 0, s, logits, T, E,
                       k, flags, ids, w, gcnt, cand, hist, st);
        else if (G == 16)
            launch_pdl(route_place_group_kernel<16>, g, dim3(kGroupWarps * 32), 0, s, logits, T, E,
                       k, flags, ids, w, gcnt, cand, hist, st);
        else
            launch_pdl(route_place_group_kernel<32>, g, dim3(kGroupWarps * 32), 0, s, logits, T, E,
                       k, flags, ids, w, gcnt, cand, hist, st);
    } else {
        const dim3 g((T + kWarpRouteTokens - 1) / kWarpRouteTokens);
        const size_t smem = 2 * sizeof(int) * (size_t)E;
        const int epl = (E + 31) / 32;
        if (epl <= 1)
            launch_pdl(route_place_warp_kernel<1>, g, dim3(256), smem, s, logits, T, E, k, flags,
                       ids, w, gcnt, cand, hist, st);
        else if (epl <= 2)
            launch_pdl(route_place_warp_kernel<2>, g, dim3(256), smem, s, logits, T, E, k, flags,
                       ids, w, gcnt, cand, hist, st);
        else if (epl <= 4)
            launch_pdl(route_place_warp_kernel<4>, g, dim3(256), smem, s, logits, T, E, k, flags,
                       ids, w, gcnt, cand, hist, st);
        else if (epl <= 8)
            launch_pdl(route_place_warp_kernel<8>, g, dim3(256), smem, s, logits, T, E, k, flags,
                       ids, w, gcnt, cand, hist, st);
        else if (epl <= 16)
            launch_pdl(route_place_warp_kernel<16>, g, dim3(256), smem, s, logits, T, E, k, flags,
                       ids, w, gcnt, cand, hist, st);
        else
            launch_pdl(route_place_warp_kernel<32>, g, dim3(256), smem, s, logits, T, E, k, flags,
                       ids, w, gcnt, cand, hist, st);
    }
    *launches += 1;
}

void launch_place_given(const int32_t* ids, const float* w, int T, int E, int k, unsigned flags,
                        int32_t* gcnt, int32_t* cand, DeviceStatus* st, cudaStream_t s,
                        int* launches) {
    uint32_t* hist = (flags & MOE_FLAG_ARRIVAL_ORDER) ? nullptr
                                                      : reinterpret_cast<uint32_t*>(gcnt + E);
    const long long P = (long long)T * k;
    if (P == 0) return;
    const long long per_block = 256LL * kGivenPairs;
    const dim3 g((unsigned)((P + per_block - 1) / per_block));
    launch_pdl(place_given_kernel, g, dim3(256), 2 * sizeof(int) * (size_t)E, s, ids, w, P, T, E,
               gcnt, cand, hist, st);
    *launches += 1;
}

size_t select_bits_bytes(int T, int E) {
    const size_t nw = ((size_t)T + 31) / 32;
    return nw <= (size_t)kSelBitWords ? 0 : (size_t)E * 2 * nw * sizeof(uint32_t);
}

void launch_select(const int32_t* cand, const int32_t* gcnt, const float* w, int T, int E, int k,
                   long long K, unsigned flags, uint32_t* gbits, int32_t* slot, uint8_t* drop,
                   int32_t* counts, int32_t* offsets, int32_t* rowtok, DeviceStatus* st,
                   cudaStream_t s, int* launches) {
    const size_t nw = ((size_t)T + 31) / 32;
    const bool bits_on_chip = nw <= (size_t)kSelBitWords;
    // Candidates whose keys and pair indices fit next to the bitmap stay on chip; an expert with
    // more keeps reading them from global memory.
    const size_t bits_smem = bits_on_chip ? 2 * nw * 4 : 0;
    const int keys_cap = (int)((kSelSmem - bits_smem) / 8);
    const size_t smem = kSelSmem;
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load() & bit)) {
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmem);
        attr_done.fetch_or(bit);
    }
    const uint32_t* hist = (flags & MOE_FLAG_ARRIVAL_ORDER)
                               ? nullptr
                               : reinterpret_cast<const uint32_t*>(gcnt + E);
    launch_pdl(select_kernel, dim3(E), dim3(kSelThreads), smem, s, cand, gcnt, w, T, E, k, K,
               flags, bits_on_chip ? nullptr : gbits, keys_cap, hist, slot, drop, counts, offsets,
               rowtok, st);
    *launches += 1;
}

void launch_dispatch(const int32_t* ids, const int32_t* slot, int T, int E, int k,
                     int32_t* kept_tmp, int32_t* offsets, int32_t* rowtok, DeviceStatus* st,
                     cudaStream_t s, int* launches) {
    const long long P = (long long)T * k;
    const int blocks = (int)std::min<long long>((P + 255) / 256, 148 * 8);
    note_launch(cudaMemsetAsync(kept_tmp, 0, sizeof(int32_t) * E, s));
    if (P > 0) launch_pdl(kept_count_kernel, dim3(blocks), dim3(256), 0, s, ids, slot, P, E, T,
                          kept_tmp, st);
    launch_pdl(offsets_kernel, dim3(1), dim3(1024), 0, s, kept_tmp, E, offsets);
    if (P > 0)
        launch_pdl(rowtok_scatter_kernel, dim3(blocks), dim3(256), 0, s, ids, slot, P, E, k,
                   offsets, rowtok, st);
    *launches += (P > 0) ? 3 : 1;
}

void launch_permute_rows(const void* x, const int32_t* rowtok, const int32_t* offsets, int E,
                         size_t row_bytes, int T, long long max_rows, void* xp, DeviceStatus* st,
                         cudaStream_t s, int* launches) {
    const int blocks = 148 * 8;
    if (row_bytes % 16 == 0 && ((uintptr_t)x % 16 == 0) && ((uintptr_t)xp % 16 == 0)) {
        launch_pdl(permute_rows_kernel<uint4>, dim3(blocks), dim3(256), 0, s, (const uint4*)x,
                   rowtok, offsets, E, (int)(row_bytes / 16), T, (uint4*)xp, st);
    } else {
        launch_pdl(permute_rows_kernel<uint32_t>, dim3(blocks), dim3(256), 0, s, (const uint32_t*)x,
                   rowtok, offsets, E, (int)(row_bytes / 4), T, (uint32_t*)xp, st);
    }
    (void)max_rows;
    *launches += 1;
}

}  // namespace moe
