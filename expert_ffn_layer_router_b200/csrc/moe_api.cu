// moe_api.cu -- the C ABI of include/moe_b200.h: argument checks, workspace layout and the
// launch sequence of each call.  Nothing here allocates device memory or synchronises the host
// (except moe_get_device_status, which by contract reads the status word back).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local int32_t g_last_launches = 0;
thread_local cudaEvent_t g_stage_events[MOE_STAGE_EVENTS];
thread_local bool g_stage_on = false;

void stage_mark(int i, cudaStream_t s) {
    if (g_stage_on) cudaEventRecord(g_stage_events[i], s);
}

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool bad_problem(const moe_problem* p) {
    if (!p) return true;
    if (p->T < 0 || p->d_model < 1 || p->d_ff < 1 || p->E < 1 || p->E > 1024) return true;
    if (p->k < 1 || p->k > p->E || p->k > 32) return true;
    if (std::isnan(p->capacity_factor) || p->capacity_factor < 0.0f) return true;
    if (p->dtype != MOE_F32 && p->dtype != MOE_BF16) return true;
    if (p->flags & ~(MOE_FLAG_RENORMALIZE | MOE_FLAG_ARRIVAL_ORDER | MOE_FLAG_GATED |
                     MOE_FLAG_ROUTER_PREPARED))
        return true;
    if ((long long)p->T * p->k > 0x7fffffffLL) return true;
    if ((long long)p->T * p->E > 0x7fffffffLL) return true;
    return false;
}

bool unsupported(const moe_problem* p) {
    if (p->dtype == MOE_BF16) {
        if ((p->d_model % 64) != 0 || (p->d_ff % 64) != 0) return true;
        if ((p->flags & MOE_FLAG_GATED) && (p->d_ff % 128) != 0) return true;
    }
    return false;
}

long long capacity_of(const moe_problem* p) {
    if (std::isinf(p->capacity_factor)) return p->T;
    const double v = std::floor((double)p->capacity_factor * (double)p->T * (double)p->k /
                                (double)p->E);
    return v > (double)p->T ? (long long)p->T : (long long)v;
}

size_t esize(const moe_problem* p) { return p->dtype == MOE_BF16 ? 2 : 4; }

// Rows of the expert-sorted buffers: at most every pair, at most K per expert.
long long max_rows_of(const moe_problem* p, long long K) {
    return std::min<long long>((long long)p->T * p->k, (long long)p->E * K);
}

struct Plan {
    size_t status, gcnt, logits, ids, w, slot, drop, counts, cand, bits, offsets, rowtok,
        kept_tmp, H, Y, split, total;
};

Plan make_plan(const moe_problem* p) {
    const long long K = capacity_of(p);
    const size_t P = (size_t)p->T * p->k;
    const size_t R = (size_t)max_rows_of(p, K);
    Plan q{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + std::max<size_t>(bytes, 1));
        return at;
    };
    q.status = take(sizeof(moe::DeviceStatus));
    q.gcnt = take(moe::dispatch_counter_ints(p->E) * 4);
    q.logits = take((size_t)p->T * p->E * 4);
    q.ids = take(P * 4);
    q.w = take(P * 4);
    q.slot = take(P * 4);
    q.drop = take(P);
    q.counts = take((size_t)2 * p->E * 4);
    q.cand = take((size_t)p->E * p->T * 4);
    q.bits = take(moe::select_bits_bytes(p->T, p->E));
    q.offsets = take((size_t)(p->E + 1) * 4);
    q.rowtok = take(R * 4);
    q.kept_tmp = take((size_t)p->E * 4);
    q.H = take(R * p->d_ff * esize(p));
    q.Y = take(R * p->d_model * esize(p));
    q.split = take(p->dtype == MOE_BF16 ? moe::router_split_bytes(p->d_model, p->E) : 0);
    q.total = off;
    return q;
}

template <class T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ws) + off);
}

bool misaligned(const void* ptr, size_t a) { return ptr && (reinterpret_cast<uintptr_t>(ptr) % a); }

moe_status check_ws(const moe_problem* p, const void* ws, size_t ws_bytes, Plan* plan) {
    *plan = make_plan(p);
    if (!ws || ws_bytes < plan->total || misaligned(ws, kAlign)) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

moe_status finish(int launches) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || moe::g_launch_error != cudaSuccess) return MOE_ERR_CUDA;
    g_last_launches = launches;
    return MOE_OK;
}

// Common entry check.  `needs_ffn`: the call runs the expert GEMMs, whose tensor-core tiles need
// d_model and d_ff to be multiples of 64 in bf16; routing, dispatch and combine take any width.
moe_status pre(const moe_problem* p, bool needs_ffn) {
    if (bad_problem(p)) return MOE_ERR_INVALID_ARG;
    if (needs_ffn && unsupported(p)) return MOE_ERR_UNSUPPORTED;
    cudaGetLastError();   // a stale error from unrelated work must not be blamed on this call
    moe::g_launch_error = cudaSuccess;
    return MOE_OK;
}

// Scratch of the routing and capacity selection (the workspace's, or the static array's).
struct RouteScratch {
    moe::DeviceStatus* st;
    int32_t* gcnt;      // [E] pairs received per expert, then [E][2048] weight-key histograms;
                        // dispatch_counter_ints(E) ints, zero at entry of the route kernel
    int32_t* cand;      // [E][T] candidate lists
    uint32_t* bits;     // select_bits_bytes(T, E) bytes, or null when that is 0
};

// Steps 1-2 on device data from given logits.  rowtok/offsets may be null (moe_route); counts is
// always written.  Small batches: the warp router, then the single-block dispatch.  Otherwise:
// the dispatch counters are cleared, the router places every pair in its expert's candidate
// list, and the capacity selection runs per expert.
void route_steps(const moe_problem* p, const float* logits, int32_t* ids, float* w,
                 int32_t* slot, uint8_t* drop, int32_t* counts, int32_t* offsets,
                 int32_t* rowtok, const RouteScratch& rs, cudaStream_t s, int* launches) {
    const long long K = capacity_of(p);
    if (moe::dispatch_small_fits(p->T, p->k)) {
        moe::launch_route_topk(logits, p->T, p->E, p->k, ids, w, s, p->flags);
        *launches += 1;
        moe::launch_dispatch_small(ids, w, p->T, p->E, p->k, K, p->flags, slot, drop, counts,
                                   offsets, rowtok, rs.st, s, launches);
        return;
    }
    moe::note_launch(cudaMemsetAsync(rs.gcnt, 0, sizeof(int32_t) * moe::dispatch_counter_ints(p->E), s));
    moe::launch_route_place(logits, p->T, p->E, p->k, p->flags, ids, w, rs.gcnt, rs.cand, rs.st,
                            s, launches);
    moe::launch_select(rs.cand, rs.gcnt, w, p->T, p->E, p->k, K, p->flags, rs.bits, slot, drop,
                       counts, offsets, rowtok, rs.st, s, launches);
}

RouteScratch scratch_of(void* ws, const Plan& q) {
    return RouteScratch{at<moe::DeviceStatus>(ws, q.status), at<int32_t>(ws, q.gcnt),
                        at<int32_t>(ws, q.cand), q.bits ? at<uint32_t>(ws, q.bits) : nullptr};
}

moe_status ffn_steps(const moe_problem* p, const void* x, const int32_t* offsets,
                     const int32_t* rowtok, const void* W1, const float* b1, const void* W2,
                     const float* b2, void* Y, void* ws, const Plan& q, cudaStream_t s,
                     int* launches) {
    moe::DeviceStatus* st = at<moe::DeviceStatus>(ws, q.status);
    const long long R = max_rows_of(p, capacity_of(p));
    if (R == 0) return MOE_OK;
    const bool gated = (p->flags & MOE_FLAG_GATED) != 0;
    if (p->dtype == MOE_F32) {
        moe::launch_ffn_f32((const float*)x, rowtok, offsets, p->E, p->T, p->d_model, p->d_ff, R,
                            (const float*)W1, b1, (const float*)W2, b2, at<float>(ws, q.H),
                            (float*)Y, st, s, launches, gated);
        return MOE_OK;
    }
    void* H = at<void>(ws, q.H);
    if (moe::launch_expert_gemm(gated ? 2 : 0, x, p->d_model, rowtok, p->T, offsets, p->E, p->d_model,
                                p->d_ff, W1, b1, H, p->d_ff, R, st, s, launches) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (moe::launch_expert_gemm(1, H, p->d_ff, nullptr, (int)R, offsets, p->E, p->d_ff,
                                p->d_model, W2, b2, Y, p->d_model, R, st, s, launches) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

// ------------------------------------------------------------------------------------------------
// moe_route_static: moe_route for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: plug-ins inside an inference engine
// that owns all device memory and gives its plug-ins no allocator, and latency-bound serving
// loops whose policy forbids cudaMalloc/cudaFree on the request path (an allocation can
// synchronise the device and stall every stream).  This entry point runs the same router and
// capacity kernels as moe_route, with their scratch (per-expert counters and weight histograms,
// candidate lists, the status word) placed in one file-scope __device__ array below.
//
// The array is a fixed kRouteStaticBytes per GPU, held by every GPU that loads the library until
// the process exits.  Host code only sees a stand-in for it, so the device address is fetched
// with cudaGetSymbolAddress on the first call in each CUDA context (the first call on a device,
// for callers of the runtime's primary context) and cached per context.  The call allocates
// nothing and calls no allocating routine.
// ------------------------------------------------------------------------------------------------
constexpr size_t kRouteStaticBytes = 8u << 20;   // 8 MiB per device
constexpr int kStaticSlots = 64;      // cached (context, address) pairs

__device__ __align__(256) unsigned char g_route_static_scratch[kRouteStaticBytes];

struct StaticSlot {
    std::atomic<void*> ctx{nullptr};
    std::atomic<void*> ptr{nullptr};
};
StaticSlot g_static_slots[kStaticSlots];
std::mutex g_static_mu;

using CtxGetCurrentFn = int (*)(void**);     // cuCtxGetCurrent(CUcontext*)
CtxGetCurrentFn g_ctx_get = nullptr;
std::once_flag g_ctx_once;

// The CUDA context current on this thread (null if none is bound yet).  The array has one
// device address per context that loaded the library's module.
void* current_context() {
    std::call_once(g_ctx_once, []() {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
    });
    void* ctx = nullptr;
    if (!g_ctx_get || g_ctx_get(&ctx) != 0) return nullptr;
    return ctx;
}

// Scratch layout of moe_route inside the static array; returns the bytes it needs.
size_t route_static_layout(const moe_problem* p, size_t* gcnt, size_t* cand, size_t* bits) {
    size_t off = align_up(sizeof(moe::DeviceStatus));
    *gcnt = off;
    off = align_up(off + moe::dispatch_counter_ints(p->E) * 4);
    *cand = off;
    off = align_up(off + (size_t)p->E * p->T * 4);
    *bits = off;
    off = align_up(off + moe::select_bits_bytes(p->T, p->E));
    return off;
}

// Device address of the static array in the current context: the cached one, else looked up
// (cudaGetSymbolAddress, which binds the device's primary context if none is current) and
// cached.  With every slot taken the address is looked up on each call, uncached.
void* static_scratch_for_current_context(cudaError_t* err) {
    *err = cudaSuccess;
    void* ctx = current_context();
    if (ctx)
        for (int i = 0; i < kStaticSlots; ++i)
            if (g_static_slots[i].ctx.load(std::memory_order_acquire) == ctx)
                return g_static_slots[i].ptr.load(std::memory_order_acquire);
    std::lock_guard<std::mutex> lock(g_static_mu);
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_route_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    ctx = current_context();
    if (!ctx) return ptr;
    for (int i = 0; i < kStaticSlots; ++i) {
        void* c = g_static_slots[i].ctx.load(std::memory_order_relaxed);
        if (c == ctx) return g_static_slots[i].ptr.load(std::memory_order_relaxed);
        if (c == nullptr) {
            g_static_slots[i].ptr.store(ptr, std::memory_order_relaxed);
            g_static_slots[i].ctx.store(ctx, std::memory_order_release);
            return ptr;
        }
    }
    return ptr;
}

}  // namespace

extern "C" {

moe_status moe_capacity(const moe_problem* p, int64_t* K) {
    if (bad_problem(p) || !K) return MOE_ERR_INVALID_ARG;
    *K = capacity_of(p);
    return MOE_OK;
}

moe_status moe_workspace_size(const moe_problem* p, size_t* bytes) {
    if (bad_problem(p) || !bytes) return MOE_ERR_INVALID_ARG;
    *bytes = make_plan(p).total;
    return MOE_OK;
}

moe_status moe_route(const moe_problem* p, const float* logits, int32_t* ids, float* w,
                     int32_t* slot, uint8_t* drop, int32_t* counts, void* ws, size_t ws_bytes,
                     void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (!counts || (p->T > 0 && (!logits || !ids || !w || !slot || !drop)))
        return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    if (p->T == 0) {
        moe::note_launch(cudaMemsetAsync(counts, 0, sizeof(int32_t) * 2 * p->E, s));
        return finish(0);
    }
    route_steps(p, logits, ids, w, slot, drop, counts, nullptr, nullptr, scratch_of(ws, q), s,
                &launches);
    return finish(launches);
}

moe_status moe_capacity_dispatch(const moe_problem* p, long long K, const int32_t* ids,
                                 const float* w, int32_t* slot, uint8_t* drop, int32_t* counts,
                                 int32_t* offsets, int32_t* rowtok, void* ws, size_t ws_bytes,
                                 void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (K < 0 || !counts || (p->T > 0 && (!ids || !w || !slot || !drop)) ||
        (rowtok && !offsets))
        return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    if (p->T == 0) {
        moe::note_launch(cudaMemsetAsync(counts, 0, sizeof(int32_t) * 2 * p->E, s));
        if (offsets)
            moe::note_launch(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (p->E + 1), s));
        return finish(0);
    }
    const RouteScratch rs = scratch_of(ws, q);
    if (moe::dispatch_small_fits(p->T, p->k)) {
        moe::launch_dispatch_small(ids, w, p->T, p->E, p->k, K, p->flags, slot, drop, counts,
                                   offsets, rowtok, rs.st, s, &launches);
        return finish(launches);
    }
    moe::note_launch(cudaMemsetAsync(rs.gcnt, 0, sizeof(int32_t) * moe::dispatch_counter_ints(p->E), s));
    moe::launch_place_given(ids, w, p->T, p->E, p->k, p->flags, rs.gcnt, rs.cand, rs.st, s,
                            &launches);
    moe::launch_select(rs.cand, rs.gcnt, w, p->T, p->E, p->k, K, p->flags, rs.bits, slot, drop,
                       counts, offsets, rowtok, rs.st, s, &launches);
    return finish(launches);
}

moe_status moe_prepare_router(const moe_problem* p, const float* Wr, void* ws, size_t ws_bytes,
                              void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (!Wr) return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    int launches = 0;
    // Only the tensor-core router (bf16, more than 1024 tokens) reads the split.
    if (p->dtype == MOE_BF16 && p->T > 0 && !moe::router_small_fits(p->T, p->E, p->d_model)) {
        if (p->d_model % 64 != 0) return MOE_ERR_UNSUPPORTED;
        moe::launch_router_split(Wr, p->d_model, p->E, at<void>(ws, q.split), nullptr, 0,
                                 (cudaStream_t)stream, &launches);
    }
    return finish(launches);
}

moe_status moe_router_logits(const moe_problem* p, const void* x, const float* Wr,
                             const float* br, float* logits, void* ws, size_t ws_bytes,
                             void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (!Wr || (p->T > 0 && (!x || !logits))) return MOE_ERR_INVALID_ARG;
    if (p->dtype == MOE_BF16 && misaligned(x, 16)) return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    if (p->T == 0) return finish(0);
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    // The kernels of moe_forward's first stage, so the logits are the forward's bit for bit.
    if (p->dtype == MOE_BF16 && moe::router_small_fits(p->T, p->E, p->d_model)) {
        moe::launch_router_small(x, Wr, br, p->T, p->d_model, p->E, p->k, logits,
                                 at<int32_t>(ws, q.ids), at<float>(ws, q.w), p->flags, s,
                                 &launches);
    } else if (p->dtype == MOE_BF16) {
        if (p->d_model % 64 != 0) return MOE_ERR_UNSUPPORTED;
        if (moe::launch_router_gemm(x, p->T, p->d_model, Wr, br, p->E, at<void>(ws, q.split),
                                    (p->flags & MOE_FLAG_ROUTER_PREPARED) != 0, logits, nullptr,
                                    0, at<moe::DeviceStatus>(ws, q.status), s,
                                    &launches) != cudaSuccess)
            return MOE_ERR_CUDA;
    } else {
        moe::launch_logits_f32((const float*)x, Wr, br, p->T, p->d_model, p->E, logits, nullptr,
                               0, s, &launches);
    }
    return finish(launches);
}

moe_status moe_dispatch(const moe_problem* p, const int32_t* ids, const int32_t* slot,
                        int32_t* offsets, int32_t* rowtok, const void* x, void* x_perm,
                        void* ws, size_t ws_bytes, void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (!offsets || (p->T > 0 && (!ids || !slot || !rowtok))) return MOE_ERR_INVALID_ARG;
    if (x_perm && !x) return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    moe::DeviceStatus* st = at<moe::DeviceStatus>(ws, q.status);
    moe::launch_dispatch(ids, slot, p->T, p->E, p->k, at<int32_t>(ws, q.kept_tmp), offsets,
                         rowtok, st, s, &launches);
    if (x_perm && p->T > 0)
        moe::launch_permute_rows(x, rowtok, offsets, p->E, (size_t)p->d_model * esize(p), p->T,
                                 max_rows_of(p, capacity_of(p)), x_perm, st, s, &launches);
    return finish(launches);
}

moe_status moe_expert_ffn(const moe_problem* p, const void* x, const int32_t* offsets,
                          const int32_t* rowtok, const void* W1, const float* b1,
                          const void* W2, const float* b2, void* Y, void* ws, size_t ws_bytes,
                          void* stream) {
    moe_status r = pre(p, true);
    if (r != MOE_OK) return r;
    if (!offsets || !W1 || !W2 || (p->T > 0 && (!x || !rowtok || !Y))) return MOE_ERR_INVALID_ARG;
    if (p->dtype == MOE_BF16 &&
        (misaligned(x, 16) || misaligned(W1, 16) || misaligned(W2, 16) || misaligned(Y, 16) ||
         misaligned(b1, 16) || misaligned(b2, 16)))
        return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    int launches = 0;
    if (p->T == 0) return finish(0);
    r = ffn_steps(p, x, offsets, rowtok, W1, b1, W2, b2, Y, ws, q, (cudaStream_t)stream,
                  &launches);
    if (r != MOE_OK) return r;
    return finish(launches);
}

moe_status moe_combine(const moe_problem* p, const void* x, const void* Y, const float* w,
                       const int32_t* ids, const int32_t* slot, const int32_t* offsets,
                       void* out, void* ws, size_t ws_bytes, void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (p->T > 0 && (!x || !Y || !w || !ids || !slot || !offsets || !out))
        return MOE_ERR_INVALID_ARG;
    if (out && (out == x || out == Y)) return MOE_ERR_INVALID_ARG;
    if (ws && (ws_bytes < kAlign || misaligned(ws, kAlign))) return MOE_ERR_WORKSPACE;
    int launches = 0;
    moe::launch_combine(p->dtype, x, Y, w, ids, slot, offsets, p->T, p->d_model, p->E, p->k,
                        max_rows_of(p, capacity_of(p)), out,
                        ws ? at<moe::DeviceStatus>(ws, 0) : nullptr, (cudaStream_t)stream,
                        &launches);
    return finish(launches);
}

moe_status moe_forward(const moe_problem* p, const void* x, const float* Wr, const float* br,
                       const void* W1, const float* b1, const void* W2, const float* b2,
                       void* out, float* logits_out, int32_t* ids_out, float* w_out,
                       int32_t* slot_out, uint8_t* drop_out, int32_t* counts_out, void* ws,
                       size_t ws_bytes, void* stream) {
    moe_status r = pre(p, true);
    if (r != MOE_OK) return r;
    if (!Wr || !W1 || !W2 || (p->T > 0 && (!x || !out))) return MOE_ERR_INVALID_ARG;
    if (out && out == x) return MOE_ERR_INVALID_ARG;
    if (p->dtype == MOE_BF16 &&
        (misaligned(x, 16) || misaligned(W1, 16) || misaligned(W2, 16) || misaligned(out, 16) ||
         misaligned(b1, 16) || misaligned(b2, 16)))
        return MOE_ERR_INVALID_ARG;
    Plan q;
    if ((r = check_ws(p, ws, ws_bytes, &q)) != MOE_OK) return r;
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, q.counts);
    if (p->T == 0) {
        moe::note_launch(cudaMemsetAsync(counts, 0, sizeof(int32_t) * 2 * p->E, s));
        return finish(0);
    }
    moe::DeviceStatus* st = at<moe::DeviceStatus>(ws, q.status);
    float* logits = logits_out ? logits_out : at<float>(ws, q.logits);
    int32_t* ids = ids_out ? ids_out : at<int32_t>(ws, q.ids);
    float* w = w_out ? w_out : at<float>(ws, q.w);
    int32_t* slot = slot_out ? slot_out : at<int32_t>(ws, q.slot);
    uint8_t* drop = drop_out ? drop_out : at<uint8_t>(ws, q.drop);
    int32_t* offsets = at<int32_t>(ws, q.offsets);
    int32_t* rowtok = at<int32_t>(ws, q.rowtok);
    void* Y = at<void>(ws, q.Y);

    stage_mark(0, s);
    // Small bf16 batches: logits on CUDA cores and routing in one launch (a 128-row tensor-core
    // tile would leave the GPU idle), then the single-block dispatch.  Larger batches: logits
    // from the tensor cores (bf16) or CUDA cores (fp32), whose launch also clears the dispatch
    // counters; then the router that places each pair in its expert's candidate list, and the
    // per-expert capacity selection.
    const bool small = p->dtype == MOE_BF16 && moe::router_small_fits(p->T, p->E, p->d_model);
    const bool small_dispatch = moe::dispatch_small_fits(p->T, p->k);
    int32_t* gcnt = small_dispatch ? nullptr : at<int32_t>(ws, q.gcnt);
    const int zero_n = small_dispatch ? 0 : (int)moe::dispatch_counter_ints(p->E);
    if (small) {
        // The large dispatch re-reads the logits: keep them (in the workspace if not asked for).
        moe::launch_router_small(x, Wr, br, p->T, p->d_model, p->E, p->k,
                                 small_dispatch ? logits_out : logits, ids, w, p->flags, s,
                                 &launches);
        if (!small_dispatch) moe::note_launch(cudaMemsetAsync(gcnt, 0, sizeof(int32_t) * (size_t)zero_n, s));
    } else if (p->dtype == MOE_BF16) {
        if (moe::launch_router_gemm(x, p->T, p->d_model, Wr, br, p->E, at<void>(ws, q.split),
                                    (p->flags & MOE_FLAG_ROUTER_PREPARED) != 0, logits, gcnt,
                                    zero_n, st, s, &launches) != cudaSuccess)
            return MOE_ERR_CUDA;
    } else {
        moe::launch_logits_f32((const float*)x, Wr, br, p->T, p->d_model, p->E, logits, gcnt,
                               zero_n, s, &launches);
    }
    stage_mark(1, s);
    const long long K = capacity_of(p);
    if (small_dispatch) {
        if (!small) {
            moe::launch_route_topk(logits, p->T, p->E, p->k, ids, w, s, p->flags);
            launches += 1;
        }
        stage_mark(2, s);
        moe::launch_dispatch_small(ids, w, p->T, p->E, p->k, K, p->flags, slot, drop, counts,
                                   offsets, rowtok, st, s, &launches);
    } else {
        const RouteScratch rs = scratch_of(ws, q);
        // (After the small router this routes the T <= 1024 tokens a second time, with the
        // same arithmetic, to place the pairs.)
        moe::launch_route_place(logits, p->T, p->E, p->k, p->flags, ids, w, gcnt, rs.cand, st,
                                s, &launches);
        stage_mark(2, s);
        moe::launch_select(rs.cand, gcnt, w, p->T, p->E, p->k, K, p->flags, rs.bits, slot, drop,
                           counts, offsets, rowtok, st, s, &launches);
    }
    stage_mark(3, s);
    const long long R = max_rows_of(p, K);
    if (R > 0 && p->dtype == MOE_BF16) {
        void* H = at<void>(ws, q.H);
        const int g1 = (p->flags & MOE_FLAG_GATED) ? 2 : 0;
        if (moe::launch_expert_gemm(g1, x, p->d_model, rowtok, p->T, offsets, p->E, p->d_model,
                                    p->d_ff, W1, b1, H, p->d_ff, R, st, s, &launches) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        stage_mark(4, s);
        if (moe::launch_expert_gemm(1, H, p->d_ff, nullptr, (int)R, offsets, p->E, p->d_ff,
                                    p->d_model, W2, b2, Y, p->d_model, R, st, s, &launches) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        stage_mark(5, s);
    } else {
        r = ffn_steps(p, x, offsets, rowtok, W1, b1, W2, b2, Y, ws, q, s, &launches);
        if (r != MOE_OK) return r;
        stage_mark(4, s);
        stage_mark(5, s);
    }
    moe::launch_combine(p->dtype, x, Y, w, ids, slot, offsets, p->T, p->d_model, p->E, p->k, R,
                        out, st, s, &launches);
    stage_mark(6, s);
    return finish(launches);
}

moe_status moe_get_device_status(const void* ws, size_t ws_bytes, void* stream, int32_t* code) {
    if (!code) return MOE_ERR_INVALID_ARG;
    if (!ws) {
        // The status word of moe_route_static's scratch on the current device.
        cudaError_t err;
        ws = static_scratch_for_current_context(&err);
        if (!ws) return MOE_ERR_CUDA;
        ws_bytes = sizeof(moe::DeviceStatus);
    }
    if (ws_bytes < sizeof(moe::DeviceStatus)) return MOE_ERR_INVALID_ARG;
    moe::DeviceStatus h{};
    if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, (cudaStream_t)stream) !=
            cudaSuccess ||
        cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    *code = h.code;
    return h.code == MOE_DEV_OK ? MOE_OK : MOE_ERR_DEVICE;
}

moe_status moe_reset_device_status(void* ws, size_t ws_bytes, void* stream) {
    if (!ws) {
        cudaError_t err;
        ws = static_scratch_for_current_context(&err);
        if (!ws) return MOE_ERR_CUDA;
        ws_bytes = sizeof(moe::DeviceStatus);
    }
    if (ws_bytes < sizeof(moe::DeviceStatus)) return MOE_ERR_INVALID_ARG;
    if (cudaMemsetAsync(ws, 0, sizeof(moe::DeviceStatus), (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int32_t moe_last_launch_count(void) { return g_last_launches; }

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, int32_t limit_us, void* stream) {
    if (!ws || ws_bytes < sizeof(moe::DeviceStatus) || limit_us < 1 || limit_us > 10000000)
        return MOE_ERR_INVALID_ARG;
    cudaGetLastError();
    moe::g_launch_error = cudaSuccess;
    moe::launch_wait_timeout_selftest(reinterpret_cast<moe::DeviceStatus*>(ws),
                                      (long long)limit_us * 1000, (cudaStream_t)stream);
    return finish(1);
}

moe_status moe_set_stage_events(void* const* events, int32_t n) {
    if (!events || n == 0) {
        g_stage_on = false;
        return MOE_OK;
    }
    if (n < MOE_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < MOE_STAGE_EVENTS; ++i) {
        if (!events[i]) return MOE_ERR_INVALID_ARG;
        g_stage_events[i] = (cudaEvent_t)events[i];
    }
    g_stage_on = true;
    return MOE_OK;
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported problem shape";
        case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE: return "device reported an error in the status word";
    }
    return "unknown status";
}

}  // extern "C"

extern "C" moe_status moe_route_static(const moe_problem* p, const float* logits, int32_t* ids,
                                       float* w, int32_t* slot, uint8_t* drop, int32_t* counts,
                                       void* stream) {
    moe_status r = pre(p, false);
    if (r != MOE_OK) return r;
    if (!counts || (p->T > 0 && (!logits || !ids || !w || !slot || !drop)))
        return MOE_ERR_INVALID_ARG;
    size_t o_gcnt, o_cand, o_bits;
    if (route_static_layout(p, &o_gcnt, &o_cand, &o_bits) > kRouteStaticBytes)
        return MOE_ERR_WORKSPACE;
    cudaError_t err;
    void* scratch = static_scratch_for_current_context(&err);
    if (!scratch) return MOE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    if (p->T == 0) {
        moe::note_launch(cudaMemsetAsync(counts, 0, sizeof(int32_t) * 2 * p->E, s));
        return finish(0);
    }
    // The array keeps the previous call's contents: the status word must start at zero (the
    // dispatch counters are cleared by route_steps); every other region is fully written by this
    // call before it is read.
    moe::DeviceStatus* st = at<moe::DeviceStatus>(scratch, 0);
    moe::note_launch(cudaMemsetAsync(st, 0, sizeof(moe::DeviceStatus), s));
    int launches = 0;
    const RouteScratch rs{st, at<int32_t>(scratch, o_gcnt), at<int32_t>(scratch, o_cand),
                          moe::select_bits_bytes(p->T, p->E) ? at<uint32_t>(scratch, o_bits)
                                                             : nullptr};
    route_steps(p, logits, ids, w, slot, drop, counts, nullptr, nullptr, rs, s, &launches);
    return finish(launches);
}
