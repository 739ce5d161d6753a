// gemm_tc.cu -- grouped GEMM on the 5th-generation tensor cores (tcgen05, accumulators in
// tensor memory) for the expert FFN and the router logits (sm_100a).
//
// Expert FFN ("Expert Networks > Worked Example: Expert Specialization", token-0 trace: h = W1 x
// + b1, a = SiLU(h), y = W2 a + b2; closing paragraph: each expert processes its kept tokens as
// one batch):
//   GEMM1: H[r, :] = SiLU(x[rowtok[r]] . W1[e]^T + b1[e])   rows r of expert e, gather folded
//          into the A-operand load (the fused-MoE dataflow diagram's "GEMM 1 reads row p //
//          top_k" idea, here indexed by expert-sorted row rather than pair order);
//   GEMM2: Y[r, :] = H[r] . W2[e]^T + b2[e].
// Router logits: L = x . (Wr_hi + Wr_mid) with the fp32 Wr split into two bf16 terms (hi =
// bf16(Wr), mid = bf16(Wr - hi); the rest is below 2^-18 |Wr|) by router_split_kernel; the
// epilogue adds the two fp32 partial products and the router bias.
//
// One persistent CTA per SM (or CTA pair per two SMs) walks a static list of (expert, m-tile,
// BN-column n-tile) tiles, n-tile fastest.  Warp roles (448 threads):
//   warp 0       TMA producer for B (weights, K-major, 128-byte swizzle), and for A when its
//                rows are contiguous
//   warp 1       TMEM allocator and the single thread that issues tcgen05.mma
//   warps 2-9    epilogue: tcgen05.ld from TMEM, bias + activation, bf16 blocks staged in
//                shared memory and written by TMA stores (fp32 stores for the router)
//   warps 10-13  A producers when A is gathered: 16-byte cp.async of the m-tile's rows
//                (through rowtok for GEMM1) into the 128-byte-swizzled K-major layout
// Pipeline: STAGES shared-memory stages (full/empty mbarriers) and two TMEM accumulators
// (tmem_full/tmem_empty) so the epilogue of tile i overlaps the main loop of tile i+1.
// Every wait is bounded (about 2 s) and reports MOE_DEV_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "softmax.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;            // rows per CTA tile (TMEM lanes)
constexpr int kBK = 64;             // K per stage: one 128-byte swizzle atom of bf16
constexpr int kThreads = 448;       // 14 warps (roles below)
constexpr int kEpiWarps = 8;        // two per TMEM lane quadrant, each half of the columns
constexpr int kTmemCols = 512;      // two accumulators at column 0 and 256
constexpr int kMaxGroups = 1024;

// kEpiRouter: fp32 logits hi + mid (+ bias), staged in shared memory and written row by row.
// kEpiSwiGLU: gated experts; the tile's 256 B rows are 128 gate rows and the matching 128 up
// rows, and the epilogue writes SiLU(gate) * up for 128 hidden features.
enum Epi { kEpiSiLU = 0, kEpiBias = 1, kEpiRouter = 2, kEpiSwiGLU = 4 };

struct GemmArgs {
    const __nv_bfloat16* A;   // [*, lda] row-major
    long long lda;            // elements
    const int32_t* a_rows;    // nullable: A row of tile row r is a_rows[r] (gather)
    int a_row_limit;          // rows of A (bound for gathered indices)
    const int32_t* offsets;   // [E+1] row ranges of the groups; null = one group of rows0 rows
    int rows0;
    int max_rows;             // rows of D (and of a contiguous A): offsets[E] must not exceed it
    int E;                    // groups
    int K;                    // reduction length, multiple of 64
    int n_tiles;              // column tiles per group
    int b_rows_per_group;     // row stride between groups in B's tensor map
    int Nout;                 // valid output columns per group
    const float* bias;        // [E, Nout] (FFN) or [router_E] (router); nullable
    void* D;                  // output
    long long ldd;            // elements
    int router_E;             // router epilogue: number of experts (columns of D)
    DeviceStatus* st;
    int32_t* zero;            // router: ints to clear (the dispatch counters), when its weight
    int zero_n;               // split did not run in the same call (else null / 0)
    const void* W;            // B's base address (the L2 prefetch below)
    long long pf_bytes;       // > 0: before waiting for its predecessor, each CTA prefetches up
                              // to this many bytes of its first tile's weight rows into L2
};

// PAIR: two CTAs of a cluster share one 256-row tile; each holds its 128 A rows and half of the
// BN B rows in shared memory, the pair's tensor cores compute the 256 x BN product together.
// The router epilogue (BN = 2 Eg: hi and mid columns of Eg experts) stages the tile's logits in a
// padded [128][Eg + 1] fp32 array instead of the bf16 staging buffers.
//
// HALFM (weight streaming, single CTAs): m-tiles of 64 rows.  The MMAs stay M = 128; A stages are
// 8 KB apart and each MMA reads 16 KB from its stage, so rows 64-127 of the product come from the
// next stage (or, for the last A stage, from the first B stage) and are never stored.  Halving
// the A stages leaves room for more weight stages in flight.
template <int BN, bool PAIR, int EPI, bool HALFM = false>
struct Cfg {
    static constexpr bool kRouter = EPI == kEpiRouter;
    static constexpr int kEg = BN / 2;
    static constexpr int kLStride = kEg + 1;                      // floats per staged logits row
    static constexpr int kTileM = PAIR ? 256 : (HALFM ? 64 : 128);
    static constexpr int kCtaRows = HALFM ? 64 : 128;             // A rows of one CTA's tile
    static constexpr int kMmaM = PAIR ? 256 : 128;
    static constexpr int kBRows = PAIR ? BN / 2 : BN;          // B rows held by this CTA
    static constexpr int kABytes = kCtaRows * kBK * 2;           // 16 KB (8 KB with HALFM)
    static constexpr int kBBytes = kBRows * kBK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStageBudget = (kRouter ? 168 : 200) * 1024;
    static constexpr int kStages = kStageBudget / kStageBytes > 8 ? 8 : kStageBudget / kStageBytes;
    static constexpr int kStgOff = kStages * kStageBytes;        // epilogue staging
    static constexpr int kStgBytes =
        kRouter ? kBM * kLStride * 4 : kEpiWarps * 2048;
    static constexpr int kBarOff = kStgOff + kStgBytes;
    static constexpr int kTableOff = kBarOff + 512;
    static constexpr int kSmemBytes = 1024 + kTableOff + (kMaxGroups + 1) * 4;
    static_assert(kStages >= 2, "at least two stages");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 N for M=128 / M=256");
    static_assert(kBBytes % 1024 == 0, "B stage must stay 1024-byte aligned");
    static_assert(8 * (3 * kStages + 4) + 4 <= 512, "barrier area");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kStgBytes % 8 == 0, "barriers stay 8-byte aligned");
    static_assert(!HALFM || (!PAIR && !kRouter), "64-row tiles: single-CTA FFN GEMMs only");
    // With HALFM the MMA of the last A stage reads 8 KB past the A stages: inside B stage 0.
    static_assert(!HALFM || kBBytes >= 8192, "the last A stage's read stays in shared memory");
};

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane, waited for inside the same asm
// statement so that no use of the registers can be scheduled before the load has landed.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 consecutive fp32 columns, load and wait in one statement.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---- pair (cta_group::2) primitives ----
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `cta` of this cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t addr, uint32_t cta) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(cta));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                     cluster_addr)
                 : "memory");
}
// TMA 2-D load whose completion is counted on a barrier of either CTA of the pair.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar,
                                                 int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(tmap), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc,
                                                 uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on the barrier at this shared offset in both CTAs of the pair once the pair's MMAs
// issued so far have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(bar)
        : "memory");
}

// TMA tile store from shared memory (bulk-group completion) and its waits.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     tmap),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The shared-memory sources of all committed stores have been read (the buffer may be reused).
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// All committed stores have completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// Tile t -> (group, first row of this CTA, valid rows of this CTA, column tile).
// s_mt[e] = tiles of kTileM rows before group e; `half` = this CTA's 128-row half (pairs).
struct TileCoord {
    int e, row0, rows, nt;
};

template <int kTileM, int kCtaRows>
__device__ __forceinline__ TileCoord tile_coord(int tile, const int* s_mt, int E, int n_tiles,
                                                const GemmArgs& a, int half) {
    TileCoord c;
    const int mt = tile / n_tiles;
    c.nt = tile - mt * n_tiles;
    int lo = 0, hi = E - 1;                 // largest e with s_mt[e] <= mt
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_mt[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    c.e = lo;
    const int g0 = a.offsets ? __ldg(a.offsets + lo) : 0;
    const int g1 = a.offsets ? __ldg(a.offsets + lo + 1) : a.rows0;
    c.row0 = g0 + (mt - s_mt[lo]) * kTileM + half * kCtaRows;
    c.rows = min(kCtaRows, g1 - c.row0);    // <= 0: this CTA's half of the tile is empty
    return c;
}

// Writers of the router GEMM's logits: the 8 epilogue warps (index 0-7) and warps 10-13 (index
// 8-11).  Per tile: barrier 1 (the staged logits are complete), then warp r writes rows r, r + 12,
// ... (coalesced along the experts); barrier 2 (the staging array may be refilled).  Every writer
// warp meets both barriers for every tile; wr = -1 only meets them (an epilogue warp whose
// pipeline wait failed).
constexpr int kRouteWarps = kEpiWarps + 4;

__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void router_tile(const float* sL, int LS, int Eg, const TileCoord& tc,
                                            const GemmArgs& a, int wr) {
    const int lane = threadIdx.x & 31;
    named_bar(1, kRouteWarps * 32);
    if (wr >= 0) {
        const int e0 = tc.nt * Eg;                         // first expert of this column tile
        const int ne = min(Eg, a.router_E - e0);
        for (int r = wr; r < tc.rows; r += kRouteWarps) {
            float* out = reinterpret_cast<float*>(a.D) + ((long long)tc.row0 + r) * a.ldd + e0;
            for (int e = lane; e < ne; e += 32) out[e] = sL[r * LS + e];
        }
    }
    named_bar(2, kRouteWarps * 32);
}

template <int BN, int EPI, bool GATHER, bool PAIR, bool HALFM>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmD, const GemmArgs args) {
    // Weight-streaming kernels do their set-up (and an L2 prefetch of their weights) before
    // waiting for the previous kernel; the others wait first.  (Measured on B200: moving the wait,
    // or adding the prefetch branch, in the compute-bound kernels slowed them by 2%.)
    if constexpr (!HALFM) pdl_begin();
    using C = Cfg<BN, PAIR, EPI, HALFM>;
    constexpr int S = C::kStages;
    constexpr int TM = C::kTileM;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const uint32_t bar0 = base + C::kBarOff;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (3 * S + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (3 * S + 2 + b); };
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base_ptr + C::kBarOff + 8 * (3 * S + 4));
    int* s_mt = reinterpret_cast<int*>(base_ptr + C::kTableOff);
    auto sA = [&](int s) { return base + (uint32_t)s * C::kABytes; };
    auto sB = [&](int s) { return base + (uint32_t)S * C::kABytes + (uint32_t)s * C::kBBytes; };

    // Gathered rows run on single-CTA tiles: the pipeline is limited by the rows in flight, not
    // by the weight traffic that pairs would halve (measured on B200: pairs with a relay of the
    // peer's gathered stages were 4% slower).
    static_assert(!(GATHER && PAIR), "gathered A uses single-CTA tiles");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E;
    DeviceStatus* st = args.st;
    const uint32_t crank = PAIR ? cluster_rank() : 0u;
    const bool leader = crank == 0;
    const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;      // tile walker id
    const int ncl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < S; ++s) {
            // producer arrive + expected bytes; gathered rows add one arrival per A thread
            mbar_init(full_bar(s), GATHER ? 1 + 128 : 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), (PAIR ? 2 : 1) * kEpiWarps * 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        if (!GATHER) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        if (EPI == kEpiSiLU || EPI == kEpiBias || EPI == kEpiSwiGLU)
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmD) : "memory");
    }
    if (warp == 1) {
        __syncwarp();
        if (PAIR) {
            tmem_alloc_pair(smem_u32(s_tmem), kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(s_tmem), kTmemCols);
            tmem_relinquish();
        }
    }
    if constexpr (HALFM) {
        if (args.pf_bytes > 0 && warp == 3) {
            // Weight streaming (few rows per group): start reading this CTA's first weight tile
            // into L2 while the kernels before it still run, its first k-blocks for all of the
            // tile's rows (the boxes the producer loads first).  The tile is the one a schedule
            // of one m-tile per group gives (tile = group * n_tiles + column tile), which is exact
            // when every group has 1 to TM rows; otherwise some prefetched bytes go unused.
            const int e = cid / args.n_tiles, nt = cid % args.n_tiles;
            if (e < E) {
                const int brow = e * args.b_rows_per_group + nt * BN;
                const int nkb_pf =
                    (int)min((long long)(args.K / kBK), args.pf_bytes / C::kBBytes);
                for (int kb = lane; kb < nkb_pf; kb += 32)
                    asm volatile(
                        "cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                        ::"l"(&tmB), "r"(kb * kBK), "r"(brow) : "memory");
            }
        }
        // Nothing above reads memory that a predecessor writes.
        pdl_wait();
        pdl_trigger();
    }
    if (warp == 2) {
        // Tile prefix over groups: lane l sums groups [l*per, (l+1)*per).  Row ranges given by
        // the caller are checked first: offsets[0] = 0, non-decreasing, offsets[E] <= max_rows,
        // so every row of every tile lies inside D.  Bad offsets: no tile runs, nothing is
        // stored, MOE_DEV_BAD_INDEX is recorded.
        const int per = (E + 31) / 32;
        int loc = 0;
        bool bad = false;
        for (int q = 0; q < per; ++q) {
            const int e = lane * per + q;
            if (e < E) {
                const int n = args.offsets ? __ldg(args.offsets + e + 1) - __ldg(args.offsets + e)
                                           : args.rows0;
                bad |= n < 0;
                loc += (max(n, 0) + TM - 1) / TM;
            }
        }
        if (args.offsets && lane == 0)
            bad |= __ldg(args.offsets) != 0 || __ldg(args.offsets + E) > args.max_rows;
        bad = __any_sync(0xffffffffu, bad);
        if (bad && lane == 0) report(st, MOE_DEV_BAD_INDEX, 510);
        int inc = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        int run = inc - loc;
        for (int q = 0; q < per; ++q) {
            const int e = lane * per + q;
            if (e < E) {
                s_mt[e] = run;
                const int n = args.offsets ? __ldg(args.offsets + e + 1) - __ldg(args.offsets + e)
                                           : args.rows0;
                run += (max(n, 0) + TM - 1) / TM;
            }
        }
        if (lane == 31) s_mt[E] = bad ? 0 : inc;
    }
    tc_fence_before();
    __syncwarp();
    if (PAIR) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int n_tiles = args.n_tiles;
    if constexpr (EPI == kEpiRouter) {
        // The routing kernel after this one counts into these (the weight split clears them when
        // it runs in the same call).
        const int nthr = (int)(gridDim.x * blockDim.x);
        for (int i = (int)(blockIdx.x * blockDim.x + threadIdx.x); i < args.zero_n; i += nthr)
            args.zero[i] = 0;
    }
    const int total = s_mt[E] * n_tiles;
    const int nkb = args.K / kBK;
    constexpr uint32_t kIdesc = idesc_bf16(C::kMmaM, BN);
    // A last column tile with at most BN/2 valid columns (d_ff = 1408 on 256-wide tiles) runs
    // N = BN/2 MMAs: the padded half is neither multiplied nor read back.  On pairs each CTA then
    // supplies BN/4 of the tile's weight rows (the first BN/4 rows of its B stage).
    constexpr bool kHalfOk = (EPI == kEpiSiLU || EPI == kEpiBias) && (BN / 2) % 16 == 0;
    constexpr uint32_t kIdescHalf = idesc_bf16(C::kMmaM, kHalfOk ? BN / 2 : BN);
    const bool last_half = kHalfOk && (n_tiles * BN - args.Nout) >= BN / 2;
    // Barriers of the pair's leader that both CTAs signal.
    auto lead = [&](uint32_t addr) { return PAIR ? map_to_cta(addr, 0) : addr; };

    if (warp == 0) {
        // ---------------- TMA producer: B (weights), and A when its rows are contiguous --------
        if (lane == 0) {
            constexpr uint32_t kTx = (PAIR ? 2u : 1u) * ((GATHER ? 0u : (uint32_t)C::kABytes) +
                                                         (uint32_t)C::kBBytes);
            uint32_t it = 0;
            bool ok = true;
            for (int tile = cid; ok && tile < total; tile += ncl) {
                const TileCoord tc = tile_coord<TM, C::kCtaRows>(tile, s_mt, E, n_tiles, args, (int)crank);
                const bool half = last_half && tc.nt == n_tiles - 1;
                const int brow = tc.e * args.b_rows_per_group + tc.nt * BN +
                                 (int)crank * (half ? BN / 4 : C::kBRows);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (!mbar_wait<PAIR>(empty_bar(s), ph ^ 1u, st, 1)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(full_bar(s), kTx);
                    if (EPI == kEpiSwiGLU) {
                        // gate rows [e*2F + nt*128, +128) and up rows [e*2F + F + nt*128, +128)
                        // (a pair CTA holds one of the two 128-row halves).
                        const int g0 = tc.e * args.b_rows_per_group + tc.nt * 128;
                        const int u0 = g0 + args.Nout;
                        if (PAIR) {
                            if (!GATHER)
                                tma_load_2d_pair(sA(s), &tmA, lead(full_bar(s)), kb * kBK, tc.row0);
                            tma_load_2d_pair(sB(s), &tmB, lead(full_bar(s)), kb * kBK,
                                             crank ? u0 : g0);
                        } else {
                            if (!GATHER) tma_load_2d(sA(s), &tmA, full_bar(s), kb * kBK, tc.row0);
                            tma_load_2d(sB(s), &tmB, full_bar(s), kb * kBK, g0);
                            tma_load_2d(sB(s) + 128u * 128u, &tmB, full_bar(s), kb * kBK, u0);
                        }
                    } else if (PAIR) {
                        const uint32_t fb = lead(full_bar(s));
                        if (!GATHER) tma_load_2d_pair(sA(s), &tmA, fb, kb * kBK, tc.row0);
                        tma_load_2d_pair(sB(s), &tmB, fb, kb * kBK, brow);
                    } else {
                        if (!GATHER) tma_load_2d(sA(s), &tmA, full_bar(s), kb * kBK, tc.row0);
                        tma_load_2d(sB(s), &tmB, full_bar(s), kb * kBK, brow);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (the pair's leader only) ----------------
        if (lane == 0 && leader) {
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int tile = cid; ok && tile < total; tile += ncl, ++lt) {
                const uint32_t b = lt & 1u, use = lt >> 1;
                if (!mbar_wait<PAIR>(tempty_bar(b), (use & 1u) ^ 1u, st, 2)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * 256u;
                const uint32_t idesc =
                    (last_half && tile % n_tiles == n_tiles - 1) ? kIdescHalf : kIdesc;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (!mbar_wait<PAIR>(full_bar(s), ph, st, 3)) { ok = false; break; }
                    if (GATHER) fence_proxy_async_smem();   // cp.async rows -> tensor-core reads
                    tc_fence_after();
                    const uint64_t da = smem_desc_sw128(sA(s));
                    const uint64_t db = smem_desc_sw128(sB(s));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        if (PAIR)
                            tc_mma_bf16_pair(d_tmem, da + 2u * kk, db + 2u * kk, idesc,
                                             (kb | kk) != 0 ? 1u : 0u);
                        else
                            tc_mma_bf16(d_tmem, da + 2u * kk, db + 2u * kk, idesc,
                                        (kb | kk) != 0 ? 1u : 0u);
                    }
                    if (PAIR) tc_commit_pair(empty_bar(s)); else tc_commit(empty_bar(s));
                }
                if (!ok) break;
                if (PAIR) tc_commit_pair(tfull_bar(b)); else tc_commit(tfull_bar(b));
            }
        }
    } else if (warp < 2 + kEpiWarps) {
        // ---------------- epilogue (this CTA's 128 rows) ----------------
        // Warp w reads TMEM lane quadrant w % 4 (rows 32q..32q+31) and half h of the tile's
        // 32-column chunks.  Each 32x32 block goes through a 2 KB staging buffer (64-byte rows,
        // 16-byte chunks swizzled by (row / 2) % 4, conflict-free both ways) and leaves with
        // stores that cover whole 64-byte row segments, 8 rows per warp instruction.
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const uint32_t tempty_target0 = lead(tempty_bar(0));
        const uint32_t tempty_target1 = lead(tempty_bar(1));
        const uint32_t stg = base + C::kStgOff + (uint32_t)(warp - 2) * 2048u;
        uint32_t lt = 0;
        for (int tile = cid; tile < total; tile += ncl, ++lt) {
            const TileCoord tc = tile_coord<TM, C::kCtaRows>(tile, s_mt, E, n_tiles, args, (int)crank);
            const uint32_t b = lt & 1u, use = lt >> 1;
            if (!mbar_wait<PAIR>(tfull_bar(b), use & 1u, st, 4)) {
                // The router's routing warps meet two barriers per tile: keep meeting them.
                if (EPI == kEpiRouter) {
                    router_tile(nullptr, 0, 0, tc, args, -1);
                    continue;
                }
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + b * 256u;
            const int wrows = min(32, max(0, tc.rows - q * 32));      // valid rows of the warp
            const long long wrow0 = (long long)tc.row0 + q * 32;
            if (EPI == kEpiRouter) {
                // Logits of this warp's 32 rows, hi + mid (+ bias), into the staging array; a
                // warp pair splits the tile's experts.  Then the TMEM buffer is released and the
                // writer warps store the tile (router_tile).
                constexpr int Eg = C::kEg, LS = C::kLStride;
                constexpr int kCols = Eg >= 32 ? Eg / 2 : Eg;
                float* sL = reinterpret_cast<float*>(base_ptr + C::kStgOff);
                if (Eg >= 32 || h == 0) {
#pragma unroll 1
                    for (int c0 = h * kCols; c0 < (h + 1) * kCols; c0 += 16) {
                        float hi[16], mi[16];
                        __syncwarp();
                        tmem_ld16_wait(taddr + c0, hi);
                        tmem_ld16_wait(taddr + Eg + c0, mi);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int e = tc.nt * Eg + c0 + i;
                            float v = __fadd_rn(hi[i], mi[i]);
                            if (args.bias && e < args.router_E) v = __fadd_rn(v, __ldg(args.bias + e));
                            sL[(q * 32 + lane) * LS + c0 + i] = v;
                        }
                    }
                }
                __syncwarp();
                tc_fence_before();
                mbar_arrive(tempty_bar(b));
                router_tile(sL, LS, Eg, tc, args, warp - 2);
                continue;
            } else {
                // Output columns of this tile: BN (128 hidden features for gated experts).
                constexpr int kOut = EPI == kEpiSwiGLU ? 128 : BN;
                constexpr int kOutChunks = (kOut + 31) / 32;
                constexpr int kOutHalf = (kOutChunks + 1) / 2;
                const int n0 = tc.nt * kOut;
                const float* bias = args.bias ? args.bias + (size_t)tc.e * args.b_rows_per_group + n0
                                              : nullptr;
#pragma unroll 1
                for (int ci = h * kOutHalf; ci < kOutChunks && ci < (h + 1) * kOutHalf; ++ci) {
                    const int c0 = ci * 32;
                    const int ncol = (kOut - c0) >= 32 ? 32 : 16;
                    float v[32];
                    float u[32];
                    // warp-uniform: columns past the group's width (padding) or no rows
                    if (n0 + c0 >= args.Nout || wrows == 0) continue;
                    __syncwarp();
                    if (ncol == 32) tmem_ld32_wait(taddr + c0, v);
                    else tmem_ld16_wait(taddr + c0, v);
                    if (EPI == kEpiSwiGLU) tmem_ld32_wait(taddr + 128 + c0, u);
                    const int nc = min(ncol, args.Nout - (n0 + c0));     // 16 or 32
                    if (bias) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            if (i >= nc) break;
                            const float4 bv = __ldg(reinterpret_cast<const float4*>(bias + c0 + i));
                            v[i] += bv.x; v[i + 1] += bv.y; v[i + 2] += bv.z; v[i + 3] += bv.w;
                            if (EPI == kEpiSwiGLU) {
                                const float4 bu = __ldg(reinterpret_cast<const float4*>(
                                    bias + args.Nout + c0 + i));
                                u[i] += bu.x; u[i + 1] += bu.y; u[i + 2] += bu.z; u[i + 3] += bu.w;
                            }
                        }
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        if (i >= nc) break;
                        float a0 = v[i], a1 = v[i + 1];
                        if (EPI == kEpiSiLU || EPI == kEpiSwiGLU) {
                            a0 = __fdividef(a0, 1.0f + __expf(-a0));
                            a1 = __fdividef(a1, 1.0f + __expf(-a1));
                        }
                        if (EPI == kEpiSwiGLU) {
                            a0 *= u[i];
                            a1 *= u[i + 1];
                        }
                        pk[i >> 1] = pack_bf16x2(a0, a1);
                    }
                    // The previous block's TMA store must have read the staging buffer.
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                    // Stage: this thread's row (= lane), nc/8 chunks of 16 bytes.  The XOR of the
                    // chunk index with (row / 2) % 4 is the tensor map's 64-byte swizzle.
                    const uint32_t rowp = stg + (uint32_t)lane * 64u;
                    const uint32_t sw = (uint32_t)((lane >> 1) & 3);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (j < nc / 8)
                            st_shared_v4(rowp + ((j ^ sw) << 4), pk[4 * j], pk[4 * j + 1],
                                         pk[4 * j + 2], pk[4 * j + 3]);
                    if (wrows == 32 && nc == 32) {
                        // A whole 32 x 32 block of this group's rows: one TMA store.
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmD, stg, n0 + c0, (int)wrow0);
                            bulk_commit();
                        }
                        continue;
                    }
                    // A block that crosses the end of the group (the rows past it belong to the
                    // next group) or a 16-column block: plain stores of the valid part.
                    __syncwarp();
                    // Copy out: lane handles chunk lane % 4 of rows lane / 4 + 8 i.
                    const int cc = lane & 3;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int R = (lane >> 2) + 8 * i;
                        if (R < wrows && cc < nc / 8) {
                            const uint4 val = ld_shared_v4(
                                stg + (uint32_t)R * 64u + ((uint32_t)(cc ^ ((R >> 1) & 3)) << 4));
                            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(args.D) +
                                                 (wrow0 + R) * args.ldd + n0 + c0 + cc * 8;
                            st_global_v4(out, val.x, val.y, val.z, val.w);
                        }
                    }
                }
            }
            __syncwarp();
            tc_fence_before();
            if (PAIR) mbar_arrive_cluster(b ? tempty_target1 : tempty_target0);
            else mbar_arrive(tempty_bar(b));
        }
    } else if (GATHER) {
        // ---------------- A producers (cp.async, gathered rows) ----------------
        // Each thread issues its 16-byte copies for a stage and lets the hardware arrive on the
        // stage's full barrier when they have landed (cp.async.mbarrier.arrive.noinc), so all
        // stages can be in flight at once and no producer thread ever blocks on its own copies.
        // The MMA thread makes the landed rows visible to the tensor cores with a proxy fence.
        const int at = threadIdx.x - 32 * (2 + kEpiWarps);   // 0..127
        const int chunk = at & 7;                             // 16-byte chunk of the row
        const int rbase = at >> 3;                            // rows rbase + 16 i
        // The row indices of the CTA's next tile are loaded early in the current one, so that
        // the first copies of the next tile do not wait on them.
        uint32_t it = 0;
        bool ok = true;
        bool have_next = false;
        int nidx[8];
        for (int tile = cid; ok && tile < total; tile += ncl) {
            const TileCoord tc = tile_coord<TM, C::kCtaRows>(tile, s_mt, E, n_tiles, args, (int)crank);
            const __nv_bfloat16* src[8];
            uint32_t dst_off[8];
            bool valid[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = rbase + 16 * i;
                valid[i] = r < tc.rows;
                long long ar = 0;
                if (valid[i]) {
                    const int g = have_next ? nidx[i] : __ldg(args.a_rows + tc.row0 + r);
                    if ((unsigned)g >= (unsigned)args.a_row_limit) {
                        report(st, MOE_DEV_BAD_INDEX, 501);
                        valid[i] = false;
                    } else {
                        ar = g;
                    }
                }
                src[i] = args.A + ar * args.lda + chunk * 8;
                dst_off[i] = (uint32_t)r * 128u + (uint32_t)((chunk ^ (r & 7)) << 4);
            }
            const int next = tile + ncl;
            TileCoord nc{0, 0, 0, 0};
            if (next < total) nc = tile_coord<TM, C::kCtaRows>(next, s_mt, E, n_tiles, args, (int)crank);
            have_next = false;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1u;
                if (!mbar_wait<PAIR>(empty_bar(s), ph ^ 1u, st, 5)) { ok = false; break; }
                const uint32_t dA = sA(s);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (valid[i]) cp_async_16(dA + dst_off[i], src[i] + kb * kBK);
                cp_async_arrive_noinc(full_bar(s));
                if (kb == 0 && next < total) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = rbase + 16 * i;
                        nidx[i] = r < nc.rows ? __ldg(args.a_rows + nc.row0 + r) : 0;
                    }
                    have_next = true;
                }
            }
        }
        cp_async_commit();     // no copy of this thread may still be in flight at exit
        cp_async_wait<0>();
    } else if (EPI == kEpiRouter) {
        // ---------------- router: warps 10-13 help write each tile's logits ----------------
        float* sL = reinterpret_cast<float*>(base_ptr + C::kStgOff);
        for (int tile = cid; tile < total; tile += ncl) {
            const TileCoord tc = tile_coord<TM, C::kCtaRows>(tile, s_mt, E, n_tiles, args, 0);
            router_tile(sL, C::kLStride, C::kEg, tc, args, warp - 2);
        }
    }

    if (warp >= 2 && warp < 2 + kEpiWarps && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncwarp();
    if (PAIR) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        if (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
        else tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Wr [d, E] fp32 -> B [ntl * 2Eg, d] bf16, the router GEMM's weight rows; also clears zero[0,
// zero_n).  For column tile nt, row
// nt*2Eg + c holds hi = bf16(Wr[:, nt*Eg + c]) and row nt*2Eg + Eg + c holds mid = bf16(Wr - hi)
// (Wr - hi is exact in fp32); experts past E are zero.  One block per 16 x Eg piece of Wr: every
// thread issues its (at most 4) coalesced loads before using any, the piece is transposed through
// shared memory, and each of the first 2 Eg threads writes 16 consecutive k of one hi or mid row.
constexpr int kSplitK = 16;

template <int Eg>
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ Wr, int d,
                                                           int E, __nv_bfloat16* __restrict__ B,
                                                           int32_t* __restrict__ zero,
                                                           int zero_n) {
    pdl_begin();
    // The dispatch counters and histograms of this call start at zero (the routing kernel after
    // the logits GEMM adds to them); every block clears a slice.
    if (zero) {
        const int nb = gridDim.x * gridDim.y, bid = blockIdx.y * gridDim.x + blockIdx.x;
        for (int i = bid * blockDim.x + threadIdx.x; i < zero_n; i += nb * blockDim.x) zero[i] = 0;
    }
    constexpr int kPer = (kSplitK * Eg + 255) / 256;
    __shared__ float s_w[kSplitK][Eg + 1];
    const int k0 = blockIdx.x * kSplitK, nt = blockIdx.y;
    float v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x + 256 * j, kk = i / Eg, c = i % Eg, e = nt * Eg + c;
        v[j] = (i < kSplitK * Eg && e < E) ? __ldg(Wr + (size_t)(k0 + kk) * E + e) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x + 256 * j;
        if (i < kSplitK * Eg) s_w[i / Eg][i % Eg] = v[j];
    }
    __syncthreads();
    if (threadIdx.x < 2 * Eg) {
        const int c = threadIdx.x % Eg, t = threadIdx.x / Eg;
        uint32_t pk[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float a = s_w[2 * q][c], b = s_w[2 * q + 1][c];
            const uint32_t h = pack_bf16x2(a, b);
            pk[q] = t == 0 ? h
                           : pack_bf16x2(__fsub_rn(a, __uint_as_float(h << 16)),
                                         __fsub_rn(b, __uint_as_float(h & 0xffff0000u)));
        }
        uint4* dst =
            reinterpret_cast<uint4*>(B + ((size_t)nt * 2 * Eg + t * Eg + c) * d + k0);
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encode_fn_ready() {
    std::call_once(g_encode_once, []() {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// 2-D bf16 tensor map over rows x cols (cols contiguous, row pitch `ld` elements).
bool make_tmap_2d(CUtensorMap* tm, const void* ptr, long long rows, int cols, long long ld,
                  int box_cols, int box_rows, CUtensorMapSwizzle swz) {
    if (!encode_fn_ready()) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Operand tile map: rows x K (K contiguous), box 64 x box_rows, 128-byte swizzle.
bool make_tmap(CUtensorMap* tm, const void* ptr, long long rows, int K, int box_rows) {
    return make_tmap_2d(tm, ptr, rows, K, K, kBK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Output map of the expert GEMMs: rows x cols bf16 (row pitch ld), 32 x 32 boxes with the
// 64-byte swizzle of the epilogue's staging buffers.
bool make_tmap_out(CUtensorMap* tm, const void* ptr, long long rows, int cols, long long ld) {
    return make_tmap_2d(tm, ptr, rows, cols, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

int g_num_sms = 0;

int num_sms() {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    return g_num_sms;
}

// The dynamic shared-memory attribute is per device; remember which devices have it.
template <int BN, int EPI, bool GATHER, bool PAIR, bool HALFM = false>
cudaError_t launch_gemm_t(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                          const GemmArgs& a, long long tiles, cudaStream_t s) {
    using C = Cfg<BN, PAIR, EPI, HALFM>;
    auto kern = grouped_gemm_kernel<BN, EPI, GATHER, PAIR, HALFM>;
    static std::atomic<uint64_t> attr_done{0};
    static std::atomic<int> pair_slots[64];
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_done.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (PAIR) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = 2;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(2 * 74, 1, 1);
            cfg.blockDim = dim3(kThreads, 1, 1);
            cfg.dynamicSmemBytes = C::kSmemBytes;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int nclusters = 0;
            e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
            if (e != cudaSuccess || nclusters <= 0) nclusters = num_sms() / 2;
            pair_slots[dev & 63].store(nclusters);
        }
        attr_done.fetch_or(bit);
    }
    if (!PAIR) {
        const int grid = (int)std::min<long long>(num_sms(), std::max<long long>(tiles, 1));
        launch_pdl(kern, dim3(grid), dim3(kThreads), C::kSmemBytes, s, tmA, tmB, tmD, a);
        return cudaGetLastError();
    }
    const int clusters =
        (int)std::min<long long>(pair_slots[dev & 63].load(), std::max<long long>(tiles, 1));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute at2[2] = {at[0], {}};
    at2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at2[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at2;
    cfg.numAttrs = 2;
    return note_launch(cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmD, a));
}

template <int EPI, bool GATHER, bool PAIR, bool HALFM = false>
cudaError_t launch_gemm_bn(int BN, const CUtensorMap& tmA, const CUtensorMap& tmB,
                           const CUtensorMap& tmD, const GemmArgs& a, long long tiles,
                           cudaStream_t s) {
    switch (BN) {
        case 256: return launch_gemm_t<256, EPI, GATHER, PAIR, HALFM>(tmA, tmB, tmD, a, tiles, s);
        case 192: return launch_gemm_t<192, EPI, GATHER, PAIR, HALFM>(tmA, tmB, tmD, a, tiles, s);
        case 176: return launch_gemm_t<176, EPI, GATHER, PAIR, HALFM>(tmA, tmB, tmD, a, tiles, s);
        case 128: return launch_gemm_t<128, EPI, GATHER, PAIR, HALFM>(tmA, tmB, tmD, a, tiles, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int EPI>
cudaError_t launch_router_bn(int BN, const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const GemmArgs& a, long long tiles, cudaStream_t s) {
    switch (BN) {
        case 128: return launch_gemm_t<128, EPI, false, false>(tmA, tmB, tmB, a, tiles, s);
        case 64: return launch_gemm_t<64, EPI, false, false>(tmA, tmB, tmB, a, tiles, s);
        case 32: return launch_gemm_t<32, EPI, false, false>(tmA, tmB, tmB, a, tiles, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// Column tile for an output width.
//  - Groups of many rows (compute-bound): a column tile costs BN + 128, for the per-tile work
//    that does not shrink with BN (A operand loads, pipeline turn-around), about half a 256-wide
//    tile's MMA time.  Measured on B200 at d_ff = 1408: 256-wide tiles (with a half-width last
//    tile) beat the exact 176-wide ones by 15%.
//  - At most 64 rows per group on average (decode, weight streaming): a tile costs about its
//    weight bytes, BN + 32, and the persistent grid finishes with its last partial wave, so
//    the cost is ceil(tiles / SMs) x (BN + 32).  Measured on B200 at T = 64, E = 64, k = 8:
//    d_model = 2048 outputs on 128-wide tiles (6.9 waves) beat 256-wide ones (3.5) by 13%.
bool weight_streaming(long long max_rows, int E) { return max_rows <= 64LL * E; }

int pick_bn(int nout, long long max_rows, int E, int num_sm) {
    const bool streaming = weight_streaming(max_rows, E);
    const long long m_tiles = streaming ? E : (max_rows + 127) / 128 + E;
    // Ties go to the wider tile when compute-bound, to the narrower one (finer waves) when
    // streaming.
    const int wide_first[] = {256, 192, 176, 128};
    const int narrow_first[] = {128, 176, 192, 256};
    const int* cands = streaming ? narrow_first : wide_first;
    int best = 256;
    long long best_cost = -1;
    for (int c = 0; c < 4; ++c) {
        const int bn = cands[c];
        const long long n_tiles = (nout + bn - 1) / bn;
        const long long cost =
            streaming ? (m_tiles * n_tiles + num_sm - 1) / num_sm * (bn + 32) : n_tiles * (bn + 128);
        if (best_cost < 0 || cost < best_cost) { best = bn; best_cost = cost; }
    }
    return best;
}

int router_group(int E) { return E <= 16 ? 16 : (E <= 32 ? 32 : 64); }


// Gated experts' first GEMM: W is [E, 2F, K] (gate rows then up rows), bias [E, 2F]; D = H [rows,
// F] = SiLU(A W_gate^T + b_gate) * (A W_up^T + b_up).  256-wide tiles = 128 gate + 128 up rows.
cudaError_t launch_gated_gemm(const void* A, long long lda, const int32_t* a_rows,
                              int a_row_limit, const int32_t* offsets, int E, int K, int F,
                              const void* W, const float* bias, void* D, long long ldd,
                              long long max_rows, DeviceStatus* st, cudaStream_t s,
                              int* launches);

// Pair (2-SM, M = 256) tiles when the experts' rows fill 256-row tiles well enough; 1-SM
// otherwise.  A 128 x 256 single-CTA tile moves about 96 KB through shared memory per 512 tensor
// cycles (its operand fills plus the MMA's operand reads), above what shared memory delivers; a
// pair's 256 x 256 tile holds half of the weight rows in each CTA and needs about 64 KB per SM.
bool use_pair(long long max_rows, int E) { return max_rows >= 256LL * E; }

cudaError_t launch_expert_gemm(int which, const void* A, long long lda, const int32_t* a_rows,
                               int a_row_limit, const int32_t* offsets, int E, int K, int Nout,
                               const void* W, const float* bias, void* D, long long ldd,
                               long long max_rows, DeviceStatus* st, cudaStream_t s,
                               int* launches) {
    if (which == 2) {
        return launch_gated_gemm(A, lda, a_rows, a_row_limit, offsets, E, K, Nout, W, bias, D,
                                 ldd, max_rows, st, s, launches);
    }
    const int BN = pick_bn(Nout, max_rows, E, num_sms());
    const bool pair = use_pair(max_rows, E) && a_rows == nullptr;
    CUtensorMap tm;
    if (!make_tmap(&tm, W, (long long)E * Nout, K, pair ? BN / 2 : BN)) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.A = reinterpret_cast<const __nv_bfloat16*>(A);
    a.lda = lda;
    a.a_rows = a_rows;
    a.a_row_limit = a_row_limit;
    a.offsets = offsets;
    a.rows0 = 0;
    a.max_rows = (int)max_rows;
    a.E = E;
    a.K = K;
    a.n_tiles = (Nout + BN - 1) / BN;
    a.b_rows_per_group = Nout;
    a.Nout = Nout;
    a.bias = bias;
    a.D = D;
    a.ldd = ldd;
    a.router_E = 0;
    a.st = st;
    // Weight streaming: 64-row m-tiles (more weight stages in flight), and each CTA reads up to
    // 512 KB of its first weight tile into L2 before it waits for the dispatch (at most 76 MB on
    // 148 SMs, well inside the 126 MB L2).
    const bool halfm = weight_streaming(max_rows, E) && !pair;
    a.W = W;
    a.pf_bytes = halfm ? 512 * 1024 : 0;
    const int tm_rows = pair ? 256 : (halfm ? 64 : kBM);
    const long long max_tiles = ((max_rows + tm_rows - 1) / tm_rows + E) * a.n_tiles;
    // Contiguous A rows: a TMA tile map over the A buffer, 128-row boxes (64 with 64-row tiles;
    // unused when gathering).
    CUtensorMap tmA = tm;
    const bool gather = a_rows != nullptr;
    if (!gather && !make_tmap(&tmA, A, (long long)a_row_limit, K, halfm ? 64 : kBM))
        return cudaErrorInvalidValue;
    CUtensorMap tmD;
    if (!make_tmap_out(&tmD, D, max_rows, Nout, ldd)) return cudaErrorInvalidValue;
    cudaError_t e;
    if (halfm) {
        if (gather)
            e = which == 0
                    ? launch_gemm_bn<kEpiSiLU, true, false, true>(BN, tmA, tm, tmD, a, max_tiles, s)
                    : launch_gemm_bn<kEpiBias, true, false, true>(BN, tmA, tm, tmD, a, max_tiles, s);
        else
            e = which == 0
                    ? launch_gemm_bn<kEpiSiLU, false, false, true>(BN, tmA, tm, tmD, a, max_tiles, s)
                    : launch_gemm_bn<kEpiBias, false, false, true>(BN, tmA, tm, tmD, a, max_tiles, s);
    } else if (gather) {
        e = which == 0 ? launch_gemm_bn<kEpiSiLU, true, false>(BN, tmA, tm, tmD, a, max_tiles, s)
                       : launch_gemm_bn<kEpiBias, true, false>(BN, tmA, tm, tmD, a, max_tiles, s);
    } else if (pair) {
        e = which == 0 ? launch_gemm_bn<kEpiSiLU, false, true>(BN, tmA, tm, tmD, a, max_tiles, s)
                       : launch_gemm_bn<kEpiBias, false, true>(BN, tmA, tm, tmD, a, max_tiles, s);
    } else {
        e = which == 0 ? launch_gemm_bn<kEpiSiLU, false, false>(BN, tmA, tm, tmD, a, max_tiles, s)
                       : launch_gemm_bn<kEpiBias, false, false>(BN, tmA, tm, tmD, a, max_tiles, s);
    }
    if (e == cudaSuccess) *launches += 1;
    return e;
}

cudaError_t launch_gated_gemm(const void* A, long long lda, const int32_t* a_rows,
                              int a_row_limit, const int32_t* offsets, int E, int K, int F,
                              const void* W, const float* bias, void* D, long long ldd,
                              long long max_rows, DeviceStatus* st, cudaStream_t s,
                              int* launches) {
    if (F % 128 != 0) return cudaErrorInvalidValue;
    const bool pair = use_pair(max_rows, E) && a_rows == nullptr;
    CUtensorMap tm;
    if (!make_tmap(&tm, W, (long long)E * 2 * F, K, 128)) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.A = reinterpret_cast<const __nv_bfloat16*>(A);
    a.lda = lda;
    a.a_rows = a_rows;
    a.a_row_limit = a_row_limit;
    a.offsets = offsets;
    a.max_rows = (int)max_rows;
    a.E = E;
    a.K = K;
    a.n_tiles = F / 128;
    a.b_rows_per_group = 2 * F;
    a.Nout = F;
    a.bias = bias;
    a.D = D;
    a.ldd = ldd;
    a.st = st;
    const int tm_rows = pair ? 256 : kBM;
    const long long max_tiles = ((max_rows + tm_rows - 1) / tm_rows + E) * a.n_tiles;
    CUtensorMap tmA = tm;
    const bool gather = a_rows != nullptr;
    if (!gather && !make_tmap(&tmA, A, (long long)a_row_limit, K, kBM))
        return cudaErrorInvalidValue;
    CUtensorMap tmD;
    if (!make_tmap_out(&tmD, D, max_rows, F, ldd)) return cudaErrorInvalidValue;
    cudaError_t e;
    if (gather)
        e = launch_gemm_t<256, kEpiSwiGLU, true, false>(tmA, tm, tmD, a, max_tiles, s);
    else if (pair)
        e = launch_gemm_t<256, kEpiSwiGLU, false, true>(tmA, tm, tmD, a, max_tiles, s);
    else
        e = launch_gemm_t<256, kEpiSwiGLU, false, false>(tmA, tm, tmD, a, max_tiles, s);
    if (e == cudaSuccess) *launches += 1;
    return e;
}

size_t router_split_bytes(int d, int E) {
    const int Eg = router_group(E);
    const int ntl = (E + Eg - 1) / Eg;
    return (size_t)ntl * 2 * Eg * d * 2;
}

void launch_router_split(const float* Wr, int d, int E, void* split_buf, int32_t* zero,
                         int zero_n, cudaStream_t s, int* launches) {
    const int Eg = router_group(E);
    const int ntl = (E + Eg - 1) / Eg;
    const dim3 sg(d / kSplitK, ntl);
    __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(split_buf);
    if (Eg == 16)
        launch_pdl(router_split_kernel<16>, sg, dim3(256), 0, s, Wr, d, E, sb, zero, zero_n);
    else if (Eg == 32)
        launch_pdl(router_split_kernel<32>, sg, dim3(256), 0, s, Wr, d, E, sb, zero, zero_n);
    else
        launch_pdl(router_split_kernel<64>, sg, dim3(256), 0, s, Wr, d, E, sb, zero, zero_n);
    *launches += 1;
}

cudaError_t launch_router_gemm(const void* x, int T, int d, const float* Wr, const float* br,
                               int E, void* split_buf, bool prepared, float* logits,
                               int32_t* zero, int zero_n, DeviceStatus* st, cudaStream_t s,
                               int* launches) {
    const int Eg = router_group(E);
    const int ntl = (E + Eg - 1) / Eg;
    const int BN = 2 * Eg;
    if (!prepared) launch_router_split(Wr, d, E, split_buf, zero, zero_n, s, launches);
    CUtensorMap tm;
    if (!make_tmap(&tm, split_buf, (long long)ntl * BN, d, BN)) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.A = reinterpret_cast<const __nv_bfloat16*>(x);
    a.lda = d;
    a.a_rows = nullptr;
    a.a_row_limit = T;
    a.offsets = nullptr;
    a.rows0 = T;
    a.max_rows = T;
    a.E = 1;
    a.K = d;
    a.n_tiles = ntl;
    a.b_rows_per_group = 0;
    a.Nout = ntl * Eg;
    a.bias = br;
    a.D = logits;
    a.ldd = E;
    a.router_E = E;
    a.st = st;
    a.zero = prepared ? zero : nullptr;
    a.zero_n = prepared ? zero_n : 0;
    const long long tiles = (long long)((T + kBM - 1) / kBM) * ntl;
    CUtensorMap tmA;
    if (!make_tmap(&tmA, x, (long long)T, d, kBM)) return cudaErrorInvalidValue;
    cudaError_t e = launch_router_bn<kEpiRouter>(BN, tmA, tm, a, tiles, s);
    if (e == cudaSuccess) *launches += 1;
    return e;
}


}  // namespace moe
