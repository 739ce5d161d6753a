// route.cu -- router softmax/top-k and capacity-limited dispatch (sm_100a).
//
// Step 1, router ("Dynamic Token Routing AI", How it works): one warp per token computes the
// softmax of its E logits in fp32 and keeps the k largest in registers.
// Step 2, capacity ("Expert Networks > Worked Example: Expert Specialization", capacity
// paragraph; "Some Tokens Do Not Get In", "Why there is a buffer" / "Past the edge"): each
// expert keeps at most K pairs, those with the highest router weight (ties: lower token), and
// the slot of a kept pair is its rank among the expert's kept tokens in ascending token order.
//
// Dispatch pipeline, all deterministic (no result depends on the order of atomics):
//   count  : one warp per chunk of 32 tokens counts its pairs per expert  -> cnt[E][nC]
//   scan   : one block per expert, exclusive prefix over chunks           -> base[E][nC], n[E]
//   scatter: one warp per chunk writes its pairs into the expert's candidate list at
//            base + (rank among equal experts inside the chunk)             -> cand[E][T]
//            (a stable counting sort: every list is in ascending token order)
//   select : one block per expert; if n_e > K a 4-pass radix select on the fp32 weight bits
//            finds the K-th largest weight, then one ordered pass with block scans assigns
//            slots, drop flags, rowtok and the counts.
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
// Router: softmax over E + top-k, one warp per token.  Lane l holds experts l, l+32, ...
// Softmax sum order: lane partials left to right, then xor-butterfly 16, 8, 4, 2, 1.
// ---------------------------------------------------------------------------------------------
// One token's routing by one warp: L points at the token's E logits (global or shared).
template <int EPL>
__device__ __forceinline__ void route_token_warp(const float* L, int E, int k, size_t t,
                                                 int32_t* __restrict__ ids,
                                                 float* __restrict__ w, unsigned flags) {
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
}

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
    pdl_begin();
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

// ---------------------------------------------------------------------------------------------
// Dispatch: count pairs per (expert, 32-token chunk).
// ---------------------------------------------------------------------------------------------
constexpr int kChunk = 32;   // tokens per chunk

__global__ void __launch_bounds__(128) count_chunks_kernel(const int32_t* __restrict__ ids, int T,
                                                           int E, int k, int nC,
                                                           int32_t* __restrict__ cnt,
                                                           DeviceStatus* st) {
    pdl_begin();
    extern __shared__ int32_t s_cnt[];                 // [4][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* my = s_cnt + warp * E;
    for (int e = lane; e < E; e += 32) my[e] = 0;
    __syncwarp();
    const int c = blockIdx.x * 4 + warp;
    if (c >= nC) return;
    const long long p0 = (long long)c * kChunk * k;
    const long long p1 = (long long)min(T, (c + 1) * kChunk) * k;
    for (long long p = p0 + lane; p < p1; p += 32) {
        const int e = ids[p];
        if ((unsigned)e >= (unsigned)E) { report(st, MOE_DEV_BAD_INDEX, 101); continue; }
        atomicAdd(&my[e], 1);
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) cnt[(size_t)e * nC + c] = my[e];
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

// One block per expert: base[e][c] = sum of cnt[e][c' < c]; n[e] = total.
__global__ void __launch_bounds__(256) scan_chunks_kernel(const int32_t* __restrict__ cnt, int nC,
                                                          int32_t* __restrict__ base,
                                                          int32_t* __restrict__ nrecv) {
    pdl_begin();
    __shared__ int s_warp[32];
    const int e = blockIdx.x;
    const int32_t* in = cnt + (size_t)e * nC;
    int32_t* out = base + (size_t)e * nC;
    int carry = 0;
    for (int c0 = 0; c0 < nC; c0 += blockDim.x) {
        const int c = c0 + threadIdx.x;
        const int v = c < nC ? in[c] : 0;
        int tot;
        const int ex = block_exclusive_scan(v, s_warp, &tot);
        if (c < nC) out[c] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) nrecv[e] = carry;
}

// One warp per chunk: stable scatter of the chunk's pairs into cand[e][.] (ascending tokens).
__global__ void __launch_bounds__(128) scatter_chunks_kernel(const int32_t* __restrict__ ids,
                                                             int T, int E, int k, int nC,
                                                             const int32_t* __restrict__ base,
                                                             int32_t* __restrict__ cand) {
    pdl_begin();
    extern __shared__ int32_t s_run[];                 // [4][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 4 + warp;
    if (c >= nC) return;
    int32_t* run = s_run + warp * E;
    for (int e = lane; e < E; e += 32) run[e] = base[(size_t)e * nC + c];
    __syncwarp();
    const long long p0 = (long long)c * kChunk * k;
    const long long p1 = (long long)min(T, (c + 1) * kChunk) * k;
    // The chunk's ids are loaded 8 rounds of 32 at a time (independent loads in flight), then
    // placed round by round in pair order.
    for (long long pg = p0; pg < p1; pg += 8 * 32) {
        int ev[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const long long p = pg + 32 * r + lane;
            ev[r] = p < p1 ? ids[p] : -1;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const long long p = pg + 32 * r + lane;
            if (pg + 32 * r >= p1) break;               // warp-uniform
            int e = ev[r];
            if ((unsigned)e >= (unsigned)E) e = -1;    // bad ids were reported by the count pass
            const unsigned peers = __match_any_sync(kFull, e);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            const int pos = (e >= 0) ? run[e] + rank : 0;
            __syncwarp();
            if (p < p1 && e >= 0) {
                cand[(size_t)e * T + pos] = (int32_t)p;
                if (lane == __ffs(peers) - 1) run[e] = pos + __popc(peers);
            }
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Capacity selection: one block per expert.
// ---------------------------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelSmemKeys = 16384;   // candidates of one expert whose list and keys stay on chip

__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const int32_t* __restrict__ cand, const int32_t* __restrict__ nrecv,
    const float* __restrict__ w, int T, int E, int k, long long K, int32_t* __restrict__ slot,
    uint8_t* __restrict__ drop, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ rowtok, unsigned flags) {
    pdl_begin();
    extern __shared__ uint32_t s_keys[];              // [kSelSmemKeys] keys, then the list
    int32_t* s_list = reinterpret_cast<int32_t*>(s_keys + kSelSmemKeys);
    __shared__ int s_warp[32];
    __shared__ int s_hist[256];
    __shared__ uint32_t s_prefix;
    __shared__ int s_remaining;
    const int e = blockIdx.x;
    const int tid = threadIdx.x;
    const int n = nrecv[e];
    const int kept = (int)min((long long)n, K);

    // Row offset of this expert: sum of kept counts of the experts before it.
    int part = 0;
    for (int q = tid; q < e; q += blockDim.x) part += (int)min((long long)nrecv[q], K);
    int off_tot;
    (void)block_exclusive_scan(part, s_warp, &off_tot);
    const int off = off_tot;
    if (tid == 0) {
        if (counts) { counts[e] = n; counts[E + e] = kept; }
        if (offsets) {
            offsets[e] = off;
            if (e == E - 1) offsets[E] = off + kept;
        }
    }
    const int32_t* list = cand + (size_t)e * T;

    if (K == 0) {                       // no slots: every pair of this expert is dropped
        for (int i = tid; i < n; i += blockDim.x) {
            const int p = list[i];
            slot[p] = -1;
            drop[p] = 1;
        }
        return;
    }
    if (n <= K || (flags & MOE_FLAG_ARRIVAL_ORDER)) {
        // Everything fits, or arrival order: the first K candidates (ascending token) get in.
        for (int i = tid; i < n; i += blockDim.x) {
            const int p = list[i];
            const bool keep = i < K;
            slot[p] = keep ? i : -1;
            drop[p] = keep ? 0 : 1;
            if (keep && rowtok) rowtok[off + i] = p / k;
        }
        return;
    }

    // Weight bit patterns of the candidates (weights are >= +0, so the bits order like the
    // values), gathered once into shared memory when they fit.
    const bool on_chip = n <= kSelSmemKeys;
    if (on_chip)
        for (int i = tid; i < n; i += blockDim.x) {
            const int p = list[i];
            s_list[i] = p;
            s_keys[i] = __float_as_uint(w[p]);
        }
    __syncthreads();
    auto key_of = [&](int i) -> uint32_t {
        return on_chip ? s_keys[i] : __float_as_uint(w[list[i]]);
    };

    // Radix select (most significant byte first) of the K-th largest key.
    uint32_t prefix = 0, mask = 0;
    int remaining = (int)K;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < 256; b += blockDim.x) s_hist[b] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t key = key_of(i);
            if ((key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & 255u], 1);
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
                        s_prefix = prefix | ((uint32_t)b << shift);
                        s_remaining = remaining - run;
                        break;
                    }
                    run += s_hist[b];
                }
            }
        }
        __syncthreads();
        prefix = s_prefix;
        remaining = s_remaining;
        mask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t tau = prefix;        // K-th largest weight bits
    const int need_eq = remaining;      // how many weights equal to tau are kept (lowest t first)
    // After the last pass s_hist[tau & 255] counts the keys equal to tau.  When all of them are
    // kept (no tie straddles the capacity boundary, the usual case) keep = (key >= tau) and the
    // tie ranks are not needed.
    const bool all_eq_kept = s_hist[tau & 255u] == need_eq;

    int eq_carry = 0, keep_carry = 0;
    for (int i0 = 0; i0 < n; i0 += blockDim.x) {
        const int i = i0 + tid;
        int p = 0;
        uint32_t key = 0;
        if (i < n) { p = on_chip ? s_list[i] : list[i]; key = key_of(i); }
        const int is_eq = (i < n && key == tau) ? 1 : 0;
        int eq_tot = 0, eq_rank = 0;
        if (!all_eq_kept) eq_rank = eq_carry + block_exclusive_scan(is_eq, s_warp, &eq_tot);
        const int keep =
            (i < n) && (key > tau || (is_eq && (all_eq_kept || eq_rank < need_eq))) ? 1 : 0;
        int keep_tot;
        const int s = keep_carry + block_exclusive_scan(keep, s_warp, &keep_tot);
        if (i < n) {
            slot[p] = keep ? s : -1;
            drop[p] = keep ? 0 : 1;
            if (keep && rowtok) rowtok[off + s] = p / k;
        }
        eq_carry += eq_tot;
        keep_carry += keep_tot;
    }
}

// ---------------------------------------------------------------------------------------------
// Small batches (T*k <= kSmallPairs): counting, capacity selection, slots, offsets and the row
// map in one block, one launch.  Same results as the chunked pipeline above: candidates of an
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
    pdl_begin();
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

int chunk_count(int T) { return (T + kChunk - 1) / kChunk; }

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

void launch_capacity_select(const int32_t* ids, const float* w, int T, int E, int k, long long K,
                            int32_t* cnt, int32_t* base, int32_t* nrecv, int32_t* cand,
                            int32_t* slot, uint8_t* drop, int32_t* counts, int32_t* offsets,
                            int32_t* rowtok, DeviceStatus* st, cudaStream_t s, int* launches,
                            bool counts_ready, unsigned flags) {
    const int nC = chunk_count(T);
    const int blocks = (nC + 3) / 4;
    const size_t smem = (size_t)4 * E * sizeof(int32_t);
    if (!counts_ready) {
        launch_pdl(count_chunks_kernel, dim3(blocks), dim3(128), smem, s, ids, T, E, k, nC, cnt,
                   st);
        *launches += 1;
    }
    launch_pdl(scan_chunks_kernel, dim3(E), dim3(256), 0, s, cnt, nC, base, nrecv);
    launch_pdl(scatter_chunks_kernel, dim3(blocks), dim3(128), smem, s, ids, T, E, k, nC, base,
               cand);
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load() & bit)) {
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelSmemKeys * 8);
        attr_done.fetch_or(bit);
    }
    launch_pdl(select_kernel, dim3(E), dim3(kSelThreads), kSelSmemKeys * 8, s, cand, nrecv, w, T, E,
               k, K, slot, drop, counts, offsets, rowtok, flags);
    *launches += 3;
}

void launch_dispatch(const int32_t* ids, const int32_t* slot, int T, int E, int k,
                     int32_t* kept_tmp, int32_t* offsets, int32_t* rowtok, DeviceStatus* st,
                     cudaStream_t s, int* launches) {
    const long long P = (long long)T * k;
    const int blocks = (int)std::min<long long>((P + 255) / 256, 148 * 8);
    cudaMemsetAsync(kept_tmp, 0, sizeof(int32_t) * E, s);
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
