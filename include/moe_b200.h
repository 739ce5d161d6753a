/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) forward pass of one capacity-limited
 * Mixture-of-Experts layer.
 *
 * The layer (sources are the pages' titles and sections):
 *   1. router: softmax over the E router logits of each token, keep the k largest
 *      ("Dynamic Token Routing AI", How it works: a gating network scores each token and
 *      picks experts);
 *   2. capacity: every expert has K = floor(C * T * k / E) slots (at most T); an expert that
 *      receives more than K (token, expert) pairs keeps the K with the highest router weight
 *      and drops the rest ("Expert Networks > Worked Example: Expert Specialization", capacity
 *      paragraph: K = 1.25 * (8/4) rounded down to 2, the lowest-confidence token is dropped;
 *      "Some Tokens Do Not Get In", "Why there is a buffer": t*k slots, fixed buffer per
 *      expert);
 *   3. expert FFN on the kept pairs: h = W1 x + b1, a = SiLU(h), y = W2 a + b2 (worked
 *      example, trace of token 0);
 *   4. combine: out = x + sum_j w_j * y_j over the token's kept pairs; a token whose pairs
 *      were all dropped leaves the layer exactly as it entered (worked example, token 4;
 *      "Some Tokens Do Not Get In", "Past the edge"; the k outputs of a token are summed back
 *      in token order as in the fused-MoE dataflow diagram's moe_sum step).
 *
 * Conventions for every call:
 *   - All pointers except `p` and the out-parameters of the host-only queries are DEVICE
 *     pointers owned by the caller.  The library never allocates device memory: scratch comes
 *     from the caller's workspace `ws` of `ws_bytes` bytes (size from moe_workspace_size,
 *     256-byte aligned).
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and performs no host synchronisation.  Kernels are launched with programmatic
 *     stream serialization: a kernel may be scheduled while the preceding work on `stream`
 *     drains, but it waits for that work to complete (griddepcontrol.wait) before it reads or
 *     writes any memory, so stream order is kept for every input and output.
 *   - Host-checkable errors (bad shapes, k > E, negative or NaN capacity factor, null or
 *     misaligned pointers, workspace too small, unsupported shape) return a non-zero status
 *     BEFORE anything is launched; outputs are then untouched.
 *   - Errors the device detects (a pipeline wait that ran out, an index out of range) are
 *     recorded in a status word at the start of `ws`; read it with moe_get_device_status.
 *     The calls never clear it (the first error stays), so clear it once with
 *     moe_reset_device_status after allocating a workspace, and again after handling an error.
 *   - Layouts are row-major and dense.  Pair p = t * k + j addresses the j-th expert of token
 *     t (j = 0 is the largest logit).  W1 is [E, d_ff, d_model] and W2 is [E, d_model, d_ff]
 *     ("out x in", so h = W1 x).  b1 is [E, d_ff] and b2 is [E, d_model], float32 always.
 *   - dtype MOE_BF16: x, W1, W2, out and expert outputs are bfloat16, accumulation is float32
 *     on the tensor cores; d_model and d_ff must be multiples of 64, and bf16 pointers and the
 *     biases 16-byte aligned.  dtype MOE_F32: everything float32 on CUDA cores (small layers).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* bad shape, pointer, alignment or capacity factor */
    MOE_ERR_UNSUPPORTED = 2,  /* well-formed problem this build does not run */
    MOE_ERR_WORKSPACE = 3,    /* workspace null or smaller than moe_workspace_size */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE = 5        /* the device status word holds an error */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Device status codes (moe_get_device_status). */
#define MOE_DEV_OK 0
#define MOE_DEV_TIMEOUT 1      /* a pipeline wait in a kernel gave up after about 2 s */
#define MOE_DEV_BAD_INDEX 2    /* an index read from an input was out of range */

typedef struct {
    int32_t T;                /* tokens, >= 0 */
    int32_t d_model;          /* model width, >= 1 */
    int32_t d_ff;             /* expert hidden width, >= 1 */
    int32_t E;                /* experts, 1..1024 */
    int32_t k;                /* experts per token, 1..min(E, 32) */
    float capacity_factor;    /* C >= 0; +INFINITY = dropless (K = T) */
    int32_t dtype;            /* moe_dtype */
    uint32_t flags;           /* MOE_FLAG_* below; other bits must be 0 */
} moe_problem;

/* Routing-policy variants (flags of moe_problem).  Default (0): softmax weights over all E,
 * not renormalised; an overflowing expert keeps its K highest-weight pairs.
 *   MOE_FLAG_RENORMALIZE: each token's k weights are divided by their sum (formed in fp32 over
 *     j = 0..k-1, one correctly rounded division each); the renormalised weights are the ones
 *     reported, used for drop priority and in the combine.
 *   MOE_FLAG_ARRIVAL_ORDER: an overflowing expert keeps the first K pairs in token order, the
 *     reading of "Some Tokens Do Not Get In", "Past the edge" (each expert's fixed buffer fills
 *     first come, first served, and later tokens are turned away), instead of the highest
 *     weights. */
#define MOE_FLAG_RENORMALIZE 1u
#define MOE_FLAG_ARRIVAL_ORDER 2u
/* Expert variant: gated FFN, after the fused-MoE dataflow diagram (GEMM 1 writes gate and up
 * halves, "SiLU x mul" combines them, GEMM 2 follows).  W1 is then [E, 2*d_ff, d_model] (rows
 * [0, d_ff) the gate, [d_ff, 2*d_ff) the up projection) and b1 [E, 2*d_ff]; the expert computes
 * a = SiLU(W1_gate x + b1_gate) * (W1_up x + b1_up), y = W2 a + b2.  bf16 needs d_ff % 128 == 0. */
#define MOE_FLAG_GATED 4u
/* Router weights prepared once: moe_forward skips splitting Wr into its two bfloat16 terms and
 * reads the terms moe_prepare_router left in the workspace (bf16 batches above 1024 tokens; the
 * other paths use Wr directly and ignore the flag).  The caller prepares again after Wr changes
 * or after the workspace was used for another problem; with stale terms the logits are wrong. */
#define MOE_FLAG_ROUTER_PREPARED 8u

/* Host only.  Per-expert capacity K = min(T, floor(C * T * k / E)) evaluated in double
 * (worked example, capacity paragraph; generalised to k slots per token as in "Some Tokens Do
 * Not Get In").  Returns MOE_ERR_INVALID_ARG for a malformed problem. */
moe_status moe_capacity(const moe_problem* p, int64_t* K);

/* Host only.  Workspace bytes needed by any call below for problem p (the largest, moe_forward,
 * decides).  A workspace of this size serves every call for that problem. */
moe_status moe_workspace_size(const moe_problem* p, size_t* bytes);

/* Router + capacity (steps 1-2).
 *   logits [T, E] float32 in;  ids [T*k] int32, w [T*k] float32 (softmax weight, not
 *   renormalised), slot [T*k] int32 (rank of t among the expert's kept tokens in ascending
 *   token order, -1 if dropped), drop [T*k] uint8 (1 = dropped), counts [2E] int32 (pairs
 *   received per expert, then pairs kept per expert).
 * Drop priority inside one expert: weight descending, then token index ascending.  Top-k ties
 * in the logits go to the lower expert index.  The softmax uses a fixed summation order and
 * its own exp, so ids, w, slot and drop are bit-for-bit functions of the logits.  NaN logits
 * are a precondition violation (result unspecified). */
moe_status moe_route(const moe_problem* p, const float* logits, int32_t* ids, float* w,
                     int32_t* slot, uint8_t* drop, int32_t* counts, void* ws, size_t ws_bytes,
                     void* stream);

/* Capacity-limited dispatch of a given routing, steps 2-3 without the router ("Expert Networks >
 * Worked Example: Expert Specialization", capacity paragraph; "Some Tokens Do Not Get In",
 * "Past the edge"): for routings formed elsewhere, and for the owner of a set of experts under
 * expert parallelism, which selects among candidates gathered from every rank.
 *   p: T, E, k and flags (MOE_FLAG_ARRIVAL_ORDER keeps an overflowing expert's first K pairs in
 *   token order; MOE_FLAG_RENORMALIZE is ignored: the weights are given); capacity_factor,
 *   d_model and d_ff size the workspace only (moe_workspace_size with the same p).
 *   K >= 0: the capacity of every expert, given explicitly (it need not be C*T*k/E of p).
 *   ids [T*k] int32 in: pair p = t*k + j goes to expert ids[p]; a token's k ids must be
 *   distinct (as a top-k gives them).  w [T*k] float32 in: its weight, >= +0 and finite.
 *   slot, drop [T*k] and counts [2E] out, as moe_route gives them for the same ids and w.
 *   offsets [E+1] int32 out (nullable): exclusive prefix of the kept counts.
 *   rowtok (nullable; needs offsets) int32 out, min(T*k, E*K) entries: rowtok[offsets[e] +
 *   slot] = token t of that kept pair.
 * Errors: MOE_ERR_INVALID_ARG for K < 0 or missing buffers; device-detected bad ids (outside
 * [0, E)) or weights (negative, -0, NaN) go to the status word as MOE_DEV_BAD_INDEX. */
moe_status moe_capacity_dispatch(const moe_problem* p, long long K, const int32_t* ids,
                                 const float* w, int32_t* slot, uint8_t* drop, int32_t* counts,
                                 int32_t* offsets, int32_t* rowtok, void* ws, size_t ws_bytes,
                                 void* stream);

/* Splits Wr [d_model, E] float32 into the two bfloat16 terms the tensor-core router reads (hi =
 * bf16(w), mid = bf16(w - hi)) and keeps them in ws, for moe_forward calls with
 * MOE_FLAG_ROUTER_PREPARED on the same p and ws.  Weights are constant during inference, so the
 * split need not be repeated per call.  A no-op for problems that do not use the tensor-core
 * router (fp32, or at most 1024 tokens). */
moe_status moe_prepare_router(const moe_problem* p, const float* Wr, void* ws, size_t ws_bytes,
                              void* stream);

/* Router logits alone, step 1's first half ("Dynamic Token Routing AI", How it works: the gating
 * network scores every token): logits [T, E] float32 = x Wr + br, with moe_forward's kernels, so
 * the values equal its logits_out bit for bit.  x [T, d_model] in p's dtype (16-byte aligned for
 * bf16), Wr [d_model, E] float32, br [E] float32 or NULL.  bf16 batches above 1024 tokens need
 * d_model a multiple of 64 (else MOE_ERR_UNSUPPORTED). */
moe_status moe_router_logits(const moe_problem* p, const void* x, const float* Wr,
                             const float* br, float* logits, void* ws, size_t ws_bytes,
                             void* stream);

/* Dispatch layout from a routing.
 *   ids, slot [T*k] in;  offsets [E+1] int32 out (exclusive prefix of kept counts);
 *   rowtok [min(T*k, E*K)] int32 out: rowtok[offsets[e] + slot] = token of that kept pair.
 *   x_perm (nullable) [rows, d_model] in x's dtype: when given, receives x[rowtok[r]] in row
 *   r (the permuted token buffer; the FFN does not need it, it gathers rows itself). */
moe_status moe_dispatch(const moe_problem* p, const int32_t* ids, const int32_t* slot,
                        int32_t* offsets, int32_t* rowtok, const void* x, void* x_perm,
                        void* ws, size_t ws_bytes, void* stream);

/* Expert FFN over the kept rows (step 3): for each expert e and row r in
 * [offsets[e], offsets[e+1]): Y[r] = W2[e] SiLU(W1[e] x[rowtok[r]] + b1[e]) + b2[e].
 * The token gather is folded into the first GEMM's operand load; nothing is materialised but
 * the hidden activations (in ws, x's dtype).  Y is [min(T*k, E*K), d_model] in x's dtype.
 * b1, b2 may be NULL (zero bias).
 * The kernels check offsets on the device: offsets[0] = 0, non-decreasing, offsets[E] <=
 * min(T*k, E*K).  If not, nothing is written to Y or H and MOE_DEV_BAD_INDEX is recorded.  A
 * rowtok entry outside [0, T) is recorded the same way and its row is computed from zeros. */
moe_status moe_expert_ffn(const moe_problem* p, const void* x, const int32_t* offsets,
                          const int32_t* rowtok, const void* W1, const float* b1,
                          const void* W2, const float* b2, void* Y, void* ws, size_t ws_bytes,
                          void* stream);

/* Combine (step 4): out[t] = x[t] + sum over kept j (ascending) of w[t*k+j] * Y[offsets[id]
 * + slot], accumulated in float32 and rounded once; out[t] = x[t] bit for bit when no pair of
 * t is kept.  out must not alias x or Y.  Y has min(T*k, E*K) rows.
 *   ws (nullable, 256-byte aligned, ws_bytes >= 256): only its status word is used.  A kept
 *   pair whose expert id is out of range, or whose row offsets[id] + slot lies outside
 *   [offsets[id], offsets[id+1]) or outside Y, is skipped (its term is left out) and recorded
 *   as MOE_DEV_BAD_INDEX in ws's status word; with ws = NULL it is skipped silently. */
moe_status moe_combine(const moe_problem* p, const void* x, const void* Y, const float* w,
                       const int32_t* ids, const int32_t* slot, const int32_t* offsets,
                       void* out, void* ws, size_t ws_bytes, void* stream);

/* The whole layer: logits = x Wr + br (Wr [d_model, E] float32, br [E] float32 or NULL), then
 * the four steps.  out [T, d_model] in x's dtype.  Optional outputs (NULL = keep in ws):
 * logits_out [T, E], ids_out, w_out, slot_out [T*k], drop_out [T*k], counts_out [2E].
 * With dtype MOE_BF16 the logits come from the tensor cores with Wr split into two bfloat16 terms
 * (hi = bf16(Wr), mid = bf16(Wr - hi); the remainder is below 2^-18 |Wr|) and float32
 * accumulation; the routing of those logits is bit for bit the routing moe_route gives for them
 * (logits_out exports them). */
moe_status moe_forward(const moe_problem* p, const void* x, const float* Wr, const float* br,
                       const void* W1, const float* b1, const void* W2, const float* b2,
                       void* out, float* logits_out, int32_t* ids_out, float* w_out,
                       int32_t* slot_out, uint8_t* drop_out, int32_t* counts_out, void* ws,
                       size_t ws_bytes, void* stream);

/* Profiling aid, host only, per calling thread.  With n >= MOE_STAGE_EVENTS, moe_forward records
 * events[0..6] (cudaEvent_t handles owned by the caller) on its stream at: entry, after the
 * router logits, after softmax/top-k, after capacity selection and dispatch, after the first
 * expert GEMM, after the second expert GEMM, after the combine.  n = 0 (or events NULL) turns
 * it off.  Recording adds no synchronisation; the handles must outlive the calls that use them. */
#define MOE_STAGE_EVENTS 7
moe_status moe_set_stage_events(void* const* events, int32_t n);

/* moe_route without a workspace, for callers that cannot allocate device memory: plug-ins of an
 * inference engine that owns all device memory and gives its plug-ins no allocator, and serving
 * loops that may not call cudaMalloc/cudaFree on the request path (an allocation can
 * synchronise the device).  The source pages describe no such call; it is a deployment aid.
 *   Same arguments, outputs and results as moe_route (bit for bit), minus ws/ws_bytes.  The
 *   router/capacity scratch lives in one fixed 8 MiB array of device memory per GPU, part of the
 *   library image and held by every GPU that loads the library until the process exits.  Needs
 *   256 + 4*E*2049 + 4*E*T bytes (each part rounded up to 256; above T = 262144 tokens also
 *   8*E*ceil(T/32) for the selection's token bitmaps); larger problems get MOE_ERR_WORKSPACE
 *   before anything is launched (T=16384 with E=64 fits; T=65536 with E=128 does not).
 *   The first call in a CUDA context (for runtime-API callers: the first call on a device) looks
 *   up the array's device address in that context and caches it.  The cached address dies with
 *   its context: do not call it across a cudaDeviceReset of that device.
 *   The status word lives in the array too: each call clears it when it starts, and
 *   moe_get_device_status(NULL, 0, stream, &code) reads it (MOE_DEV_BAD_INDEX for an id out of
 *   range).
 *   Every call on a device shares the one array: calls that overlap on the GPU (other streams,
 *   other host threads) race and corrupt each other's results; serialise them.  Nothing is
 *   allocated, and no allocating routine is called. */
moe_status moe_route_static(const moe_problem* p, const float* logits, int32_t* ids, float* w,
                            int32_t* slot, uint8_t* drop, int32_t* counts, void* stream);

/* Failure-detection self-test: launches one kernel that waits on a pipeline barrier nothing
 * ever arrives on, using the same bounded wait as the layer's kernels but with a limit of
 * `limit_us` microseconds (1..10^7).  The wait gives up, records MOE_DEV_TIMEOUT in the status
 * word of `ws` and the kernel returns; the GPU context stays usable.  Asynchronous on `stream`;
 * read the result with moe_get_device_status. */
moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, int32_t limit_us, void* stream);

/* Reads the device status word of `ws` (synchronises `stream`).  ws = NULL reads the status word
 * of moe_route_static's fixed scratch on the current device, which that call clears when it
 * starts: it holds the result of the latest moe_route_static call there. */
moe_status moe_get_device_status(const void* ws, size_t ws_bytes, void* stream, int32_t* code);

/* Clears the device status word of `ws` (asynchronous on `stream`); ws = NULL: the status word of
 * moe_route_static's scratch on the current device. */
moe_status moe_reset_device_status(void* ws, size_t ws_bytes, void* stream);

/* Kernel launches made by the most recent successful compute call on this host thread. */
int32_t moe_last_launch_count(void);

/* Static, never NULL. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
