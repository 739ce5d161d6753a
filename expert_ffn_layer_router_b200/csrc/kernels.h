// kernels.h -- launchers of the MoE kernels (internal to the library).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace moe {

struct DeviceStatus;

// route.cu
// flags: MOE_FLAG_RENORMALIZE divides each token's k weights by their sum.
void launch_route_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                       cudaStream_t s, unsigned flags);
// Routing of T tokens from their logits (ids, w) that also appends every pair p = t*k + j to its
// expert's candidate list cand[e][.] ([E][T]), counts it in gcnt[e] and in a per-expert histogram
// of weight keys that follows gcnt; the dispatch_counter_ints(E) ints at gcnt must be zero at
// entry.
// A group of route_group_lanes(E, k) lanes routes each token when that is not 0, else a warp.
size_t dispatch_counter_ints(int E);
int route_group_lanes(int E, int k);
void launch_route_place(const float* logits, int T, int E, int k, unsigned flags, int32_t* ids,
                        float* w, int32_t* gcnt, int32_t* cand, DeviceStatus* st, cudaStream_t s,
                        int* launches);
// Candidate lists and weight histograms of a given routing (ids, w [T*k]), as launch_route_place
// builds them; the same counters must be zero at entry.
void launch_place_given(const int32_t* ids, const float* w, int T, int E, int k, unsigned flags,
                        int32_t* gcnt, int32_t* cand, DeviceStatus* st, cudaStream_t s,
                        int* launches);
// Capacity selection from the candidate lists: slot, drop, counts (nullable), offsets and rowtok
// (nullable).  flags: MOE_FLAG_ARRIVAL_ORDER keeps an overflowing expert's first K pairs in token
// order.  gbits: select_bits_bytes(T, E) bytes of scratch (unused and nullable when that is 0).
size_t select_bits_bytes(int T, int E);
void launch_select(const int32_t* cand, const int32_t* gcnt, const float* w, int T, int E, int k,
                   long long K, unsigned flags, uint32_t* gbits, int32_t* slot, uint8_t* drop,
                   int32_t* counts, int32_t* offsets, int32_t* rowtok, DeviceStatus* st,
                   cudaStream_t s, int* launches);
// Small batches (T*k <= 1024): the whole capacity selection in one single-block launch.
bool dispatch_small_fits(int T, int k);
void launch_dispatch_small(const int32_t* ids, const float* w, int T, int E, int k, long long K,
                           unsigned flags, int32_t* slot, uint8_t* drop, int32_t* counts,
                           int32_t* offsets, int32_t* rowtok, DeviceStatus* st, cudaStream_t s,
                           int* launches);
// Small batches of bf16 tokens (T <= 1024, E <= 256, d <= 12288): logits on CUDA cores and routing in one
// launch, one block per token.  logits_out may be null.
bool router_small_fits(int T, int E, int d);
void launch_router_small(const void* x, const float* Wr, const float* br, int T, int d, int E,
                         int k, float* logits_out, int32_t* ids, float* w, unsigned flags,
                         cudaStream_t s, int* launches);
void launch_wait_timeout_selftest(DeviceStatus* st, long long limit_ns, cudaStream_t s);
void launch_dispatch(const int32_t* ids, const int32_t* slot, int T, int E, int k,
                     int32_t* kept_tmp, int32_t* offsets, int32_t* rowtok, DeviceStatus* st,
                     cudaStream_t s, int* launches);
void launch_permute_rows(const void* x, const int32_t* rowtok, const int32_t* offsets, int E,
                         size_t row_bytes, int T, long long max_rows, void* xp, DeviceStatus* st,
                         cudaStream_t s, int* launches);

// combine.cu
// max_rows: rows of Y; a kept pair whose row falls outside [0, max_rows) or outside its
// expert's range is skipped and recorded as MOE_DEV_BAD_INDEX (st may be null).
void launch_combine(int dtype, const void* x, const void* Y, const float* w, const int32_t* ids,
                    const int32_t* slot, const int32_t* offsets, int T, int d, int E, int k,
                    long long max_rows, void* out, DeviceStatus* st, cudaStream_t s,
                    int* launches);
void launch_ffn_f32(const float* x, const int32_t* rowtok, const int32_t* offsets, int E, int T,
                    int d, int F, long long max_rows, const float* W1, const float* b1,
                    const float* W2, const float* b2, float* H, float* Y, DeviceStatus* st,
                    cudaStream_t s, int* launches, bool gated);
// Also clears zero[0, zero_n) (the dispatch counters).
void launch_logits_f32(const float* x, const float* Wr, const float* br, int T, int d, int E,
                       float* logits, int32_t* zero, int zero_n, cudaStream_t s, int* launches);

// gemm_tc.cu
int pick_bn(int nout, long long max_rows, int E, int num_sm);
int router_group(int E);
size_t router_split_bytes(int d, int E);
// which = 0: D = SiLU(A W^T + bias) (GEMM1); which = 1: D = A W^T + bias (GEMM2);
// which = 2: gated GEMM1, W [E, 2*Nout, K] (gate rows, up rows), bias [E, 2*Nout],
// D = SiLU(A W_gate^T + b_gate) * (A W_up^T + b_up) (Nout a multiple of 128).
cudaError_t launch_expert_gemm(int which, const void* A, long long lda, const int32_t* a_rows,
                               int a_row_limit, const int32_t* offsets, int E, int K, int Nout,
                               const void* W, const float* bias, void* D, long long ldd,
                               long long max_rows, DeviceStatus* st, cudaStream_t s,
                               int* launches);
// Router logits L = x Wr + br [T, E] on the tensor cores, from Wr split into two bf16 terms in
// split_buf (router_split_bytes): split here, or already (prepared); either way zero[0, zero_n)
// (the dispatch counters) is cleared.
cudaError_t launch_router_gemm(const void* x, int T, int d, const float* Wr, const float* br,
                               int E, void* split_buf, bool prepared, float* logits,
                               int32_t* zero, int zero_n, DeviceStatus* st, cudaStream_t s,
                               int* launches);
// The split alone (also clears zero[0, zero_n)).
void launch_router_split(const float* Wr, int d, int E, void* split_buf, int32_t* zero,
                         int zero_n, cudaStream_t s, int* launches);

}  // namespace moe
