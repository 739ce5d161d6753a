// moe_oracle.cpp -- plain CPU oracle for the capacity-limited Mixture-of-Experts layer forward.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file: only
// the tests, the package's smoke check and the bench's CPU-baseline leg use it.  It shares no
// code, header, constant table or helper with the CUDA library; the two are written separately
// from the same statement of the method.
//
// What the layer computes (sources are the pages' titles and sections):
//   * "Expert Networks > Worked Example: Expert Specialization" (mbrenndoerfer.com), the
//     capacity paragraph: K = C * (tokens / experts), rounded down; an expert that receives more
//     than K tokens drops the ones with the lowest router confidence; a dropped token leaves the
//     layer unchanged through the residual.
//   * same page, the trace of token 0: h = W1 x + b1, a = SiLU(h), y = W2 a + b2, and the output
//     is x + w * y, w being how confident the router is in that expert.
//   * same page, closing paragraph: each expert processes its kept tokens as one batch.
//   * "Some Tokens Do Not Get In" (getbasislab.com), sections "Why there is a buffer" and "Past
//     the edge": t*k token slots to fill, a fixed buffer per expert, overflow tokens take the
//     residual path and arrive exactly as they entered.
//   * the fused-MoE dataflow diagram (monishver11.github.io, moe-vllm flow.excalidraw): with
//     top_k > 1 the k expert outputs of a token are summed back in token order ("moe_sum").
//
// Readings where the pages are silent (each is listed with its reason in the design notes):
//   R1 router weights are a softmax over all E logits, not renormalised after top-k;
//   R2 the softmax uses this file's own exp (Cody-Waite reduction + degree-7 Taylor polynomial)
//      and a fixed summation order, so that the weights are a deterministic fp32 function of the
//      logits that an independent GPU implementation can reproduce bit for bit;
//   R3 top-k orders experts by (logit descending, expert index ascending);
//   R4 capacity with top-k: K = min(T, floor(C*T*k/E)); C = +inf means dropless (K = T);
//   R5 drop priority inside one expert: (weight descending, token index ascending), keep K;
//   R6 slot = rank of the token among the expert's kept tokens in ascending token order;
//   R7 FFN and combine accumulate in double from the stored-precision inputs; the result is
//      rounded once to x's type; a token with no kept pair is returned bit for bit.
//
// Build: g++ -O2 -std=c++17 -fno-fast-math -ffp-contract=off -shared -fPIC (see build_oracle.py).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ------------------------------------------------------------------------------------------------
// Own exp, float in / float out.  Method: W. J. Cody and W. Waite, "Software Manual for the
// Elementary Functions" (1980): x = n*ln2 + r with n = nearest integer to x/ln2 and ln2 split
// into a short high part (exact products n*hi for |n| < 2^8) and a low correction; then
// exp(r) by its Taylor series to r^7/7! (|r| <= ln2/2 makes the truncation error < 0.1 ulp),
// evaluated by Horner's rule with fused multiply-adds; then scale by 2^n through the exponent
// field.  All steps are IEEE-754 single operations with round-to-nearest-even, so the result
// is reproducible on any conforming machine.  Results below 2^-125 are flushed to +0 (n < -125)
// so no subnormal is ever produced; n > 127 overflows to +inf.
// ------------------------------------------------------------------------------------------------
float own_exp(float x) {
    if (std::isnan(x)) return x;
    const float kLog2e = (float)1.4426950408889634074;          // 1/ln 2 rounded to float
    const float kLn2Hi = (float)(45426.0 / 65536.0);             // floor(ln2 * 2^16) / 2^16
    const float kLn2Lo = (float)(0.6931471805599453094 - 45426.0 / 65536.0);
    float t = x * kLog2e;
    if (t > 200.0f) return INFINITY;
    if (t < -200.0f) return 0.0f;
    float nf = std::nearbyint(t);                                // ties to even (default mode)
    int n = (int)nf;
    if (n < -125) return 0.0f;
    float r = std::fma(-nf, kLn2Hi, x);
    r = std::fma(-nf, kLn2Lo, r);
    float p = (float)(1.0 / 5040.0);
    p = std::fma(p, r, (float)(1.0 / 720.0));
    p = std::fma(p, r, (float)(1.0 / 120.0));
    p = std::fma(p, r, (float)(1.0 / 24.0));
    p = std::fma(p, r, (float)(1.0 / 6.0));
    p = std::fma(p, r, 0.5f);
    p = std::fma(p, r, 1.0f);
    p = std::fma(p, r, 1.0f);
    if (n > 127) {                                               // 2^n not a float: two steps
        uint32_t b127 = (uint32_t)(127 + 127) << 23;
        float s127; std::memcpy(&s127, &b127, 4);
        return (p * s127) * 2.0f;
    }
    uint32_t bits = (uint32_t)(n + 127) << 23;
    float scale; std::memcpy(&scale, &bits, 4);
    return p * scale;
}

// Softmax of one row of E logits (reading R1/R2).  m = max; u_e = own_exp(L_e - m); the sum is
// formed in a fixed order: 32 partial sums, partial_l = u_l + u_{l+32} + u_{l+64} + ...
// (left to right), then combined pairwise as s_l <- s_l + s_{l xor h} for h = 16, 8, 4, 2, 1;
// p_e = u_e / S with one correctly rounded division.
void softmax_row(const float* L, int E, float* p) {
    float m = L[0];
    for (int e = 1; e < E; ++e) if (L[e] > m) m = L[e];
    std::vector<float> u(E);
    for (int e = 0; e < E; ++e) u[e] = own_exp(L[e] - m);
    float part[32];
    for (int l = 0; l < 32; ++l) {
        float acc = 0.0f;
        for (int e = l; e < E; e += 32) acc = acc + u[e];
        part[l] = acc;
    }
    for (int h = 16; h >= 1; h >>= 1) {
        float nxt[32];
        for (int l = 0; l < 32; ++l) nxt[l] = part[l] + part[l ^ h];
        std::memcpy(part, nxt, sizeof(part));
    }
    const float S = part[0];
    for (int e = 0; e < E; ++e) p[e] = u[e] / S;
}

// "a before b" in the top-k order of reading R3.
inline bool topk_before(float La, int a, float Lb, int b) {
    return La > Lb || (La == Lb && a < b);
}

inline double load_elem(const void* base, size_t i, int dtype) {
    if (dtype == 0) return (double)((const float*)base)[i];
    uint16_t h = ((const uint16_t*)base)[i];
    uint32_t bits = (uint32_t)h << 16;
    float f; std::memcpy(&f, &bits, 4);
    return (double)f;
}

// Round a double to the nearest bfloat16, ties to even, directly (no intermediate float).
uint16_t bf16_from_double(double v) {
    if (std::isnan(v)) return 0x7FC0;
    uint16_t sign = std::signbit(v) ? 0x8000 : 0;
    double a = std::fabs(v);
    if (a == 0.0) return sign;
    if (std::isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    std::frexp(a, &e);                         // a = m * 2^e, m in [0.5, 1)
    int q = std::max(e - 8, -133);             // exponent of the last kept significand bit
    double r = std::nearbyint(std::ldexp(a, -q));
    double res = std::ldexp(r, q);
    if (res >= 0x1p128) return (uint16_t)(sign | 0x7F80);
    float f = (float)res;                      // exact: res has at most 8 significant bits
    uint32_t bits; std::memcpy(&bits, &f, 4);
    return (uint16_t)(sign | (bits >> 16));
}

// One expert FFN on one token (worked-example trace): h = W1 x + b1, a = SiLU(h) = h / (1 +
// e^{-h}), y = W2 a + b2.  W1e is [F, d] and W2e is [d, F], row-major ("out x in").
// gated (the fused-MoE dataflow diagram's "SiLU x mul" between GEMM 1 and GEMM 2): W1e is
// [2F, d] and b1e [2F], rows [0, F) the gate g and rows [F, 2F) the up projection u, and
// a = SiLU(g) * u.  h_out receives a.
void expert_ffn(int d, int F, int dtype, const double* x, const void* W1, size_t w1_off,
                const float* b1e, const void* W2, size_t w2_off, const float* b2e,
                double* h_out, double* y, bool gated = false) {
    std::vector<double> a(F);
    auto row_dot = [&](int row) {
        double h = 0.0;
        for (int i = 0; i < d; ++i) h += load_elem(W1, w1_off + (size_t)row * d + i, dtype) * x[i];
        if (b1e) h += (double)b1e[row];
        return h;
    };
    for (int f = 0; f < F; ++f) {
        const double g = row_dot(f);
        const double silu = g / (1.0 + std::exp(-g));
        a[f] = gated ? silu * row_dot(F + f) : silu;
        if (h_out) h_out[f] = gated ? a[f] : g;
    }
    for (int o = 0; o < d; ++o) {
        double s = 0.0;
        for (int f = 0; f < F; ++f) s += load_elem(W2, w2_off + (size_t)o * F + f, dtype) * a[f];
        if (b2e) s += (double)b2e[o];
        y[o] = s;
    }
}

template <class Fn>
void parallel_for(int n, int nthreads, Fn fn) {
    if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
    nthreads = std::min(nthreads, std::max(n, 1));
    if (nthreads <= 1) { for (int i = 0; i < n; ++i) fn(i); return; }
    std::vector<std::thread> pool;
    for (int w = 0; w < nthreads; ++w)
        pool.emplace_back([=]() { for (int i = w; i < n; i += nthreads) fn(i); });
    for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Capacity per expert, reading R4.  Returns -1 for a negative or NaN capacity factor.
long long oracle_capacity(long long T, long long E, long long k, double C) {
    if (std::isnan(C) || C < 0.0 || T < 0 || E <= 0 || k <= 0) return -1;
    if (std::isinf(C)) return T;
    double v = std::floor(C * (double)T * (double)k / (double)E);
    if (v > (double)T) return T;
    return (long long)v;
}

float oracle_own_exp(float x) { return own_exp(x); }

void oracle_own_exp_n(long long n, const float* x, float* y) {
    for (long long i = 0; i < n; ++i) y[i] = own_exp(x[i]);
}

void oracle_softmax(int T, int E, const float* logits, float* p) {
    for (int t = 0; t < T; ++t) softmax_row(logits + (size_t)t * E, E, p + (size_t)t * E);
}

// Router logits L = x Wr + br with a double sum rounded once to float.  x is [T, d] (dtype 0 =
// float, 1 = bfloat16 bits), Wr is [d, E] float, br is [E] float or null.
void oracle_logits(int T, int d, int E, int dtype, const void* x, const float* Wr,
                   const float* br, float* L, int nthreads) {
    parallel_for(T, nthreads, [&](int t) {
        std::vector<double> acc(E, 0.0);
        for (int i = 0; i < d; ++i) {
            double xv = load_elem(x, (size_t)t * d + i, dtype);
            for (int e = 0; e < E; ++e) acc[e] += xv * (double)Wr[(size_t)i * E + e];
        }
        for (int e = 0; e < E; ++e) {
            double v = acc[e] + (br ? (double)br[e] : 0.0);
            L[(size_t)t * E + e] = (float)v;
        }
    });
}

// Capacity selection of a given routing ("Expert Networks > Worked Example: Expert
// Specialization", capacity paragraph; "Some Tokens Do Not Get In", "Past the edge"):
//   ids[T*k], w[T*k]: pair p = t*k + j routed to expert ids[p] with router weight w[p];
//   each expert keeps at most K of its pairs, by (weight descending, token ascending) -- or, with
//   flags & 2, its first K pairs in token order;
//   slot[T*k]: rank among the expert's kept tokens (ascending t), -1 if dropped;
//   drop[T*k]: 1 if dropped;  counts[2E]: received per expert, then kept per expert.
// Returns 0, or -1 on bad arguments (an id outside [0, E)).
int oracle_select(int T, int E, int k, long long K, const int32_t* ids, const float* w,
                  int32_t* slot, uint8_t* drop, int32_t* counts, int flags) {
    if (T < 0 || E <= 0 || k <= 0 || K < 0) return -1;
    for (long long p = 0; p < (long long)T * k; ++p)
        if (ids[p] < 0 || ids[p] >= E) return -1;
    // Candidate pairs of each expert, ascending token index.
    std::vector<std::vector<int>> cand(E);
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) cand[ids[(size_t)t * k + j]].push_back(t * k + j);
    for (int e = 0; e < E; ++e) {
        const std::vector<int>& c = cand[e];
        // order[] holds positions into c, sorted by (weight descending, token ascending).
        std::vector<int> order(c.size());
        for (size_t i = 0; i < c.size(); ++i) order[i] = (int)i;
        if (!(flags & 2))                               // by weight; else keep arrival order
            std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
                float wa = w[c[a]], wb = w[c[b]];
                if (wa != wb) return wa > wb;
                return c[a] / k < c[b] / k;
            });
        std::vector<char> keep(c.size(), 0);
        long long nkeep = std::min<long long>(K, (long long)order.size());
        for (long long i = 0; i < nkeep; ++i) keep[order[i]] = 1;
        int s = 0;
        for (size_t i = 0; i < c.size(); ++i) {
            int pi = c[i];
            if (keep[i]) { slot[pi] = s++; drop[pi] = 0; }
            else { slot[pi] = -1; drop[pi] = 1; }
        }
        counts[e] = (int32_t)c.size();
        counts[E + e] = s;
    }
    return 0;
}

// Routing: softmax, top-k, then the capacity selection above.
//   ids[T*k], w[T*k]: pair p = t*k + j, j = 0 is the largest logit.
// flags: 1 = renormalise each token's k weights by their sum (fp32, j ascending, one division
// each); 2 = capacity by arrival (token) order instead of by weight.
int oracle_route(int T, int E, int k, long long K, const float* logits, int32_t* ids, float* w,
                 int32_t* slot, uint8_t* drop, int32_t* counts, int flags) {
    if (T < 0 || E <= 0 || k <= 0 || k > E || K < 0) return -1;
    std::vector<float> p(E);
    for (int t = 0; t < T; ++t) {
        const float* L = logits + (size_t)t * E;
        softmax_row(L, E, p.data());
        std::vector<char> taken(E, 0);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || topk_before(L[e], e, L[best], best)) best = e;
            }
            taken[best] = 1;
            ids[(size_t)t * k + j] = best;
            w[(size_t)t * k + j] = p[best];
        }
        if (flags & 1) {
            float sum = 0.0f;
            for (int j = 0; j < k; ++j) sum = sum + w[(size_t)t * k + j];
            for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = w[(size_t)t * k + j] / sum;
        }
    }
    return oracle_select(T, E, k, K, ids, w, slot, drop, counts, flags);
}

// Expert-sorted row layout: offsets[E+1] (exclusive prefix of kept counts) and
// rowtok[offsets[e] + slot] = token index of that kept pair.
int oracle_dispatch(int T, int E, int k, const int32_t* ids, const int32_t* slot,
                    int32_t* offsets, int32_t* rowtok) {
    std::vector<long long> kept(E, 0);
    for (long long pi = 0; pi < (long long)T * k; ++pi)
        if (slot[pi] >= 0) kept[ids[pi]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = (int32_t)(offsets[e] + kept[e]);
    for (long long pi = 0; pi < (long long)T * k; ++pi)
        if (slot[pi] >= 0) rowtok[offsets[ids[pi]] + slot[pi]] = (int32_t)(pi / k);
    return 0;
}

// Expert FFN outputs for a list of (token, expert) rows: Y[r] = W2e SiLU(W1e x_t + b1e) + b2e in
// double; H[r] (optional) is the pre-activation h.  W1 is [E, F, d], W2 is [E, d, F] in x's
// dtype; b1 [E, F], b2 [E, d] float or null.
// flags bit 4: gated experts (W1 [E, 2F, d], b1 [E, 2F]).
int oracle_expert_rows(int d, int F, int E, int dtype, const void* x, const void* W1,
                       const float* b1, const void* W2, const float* b2, int nrows,
                       const int32_t* row_tok, const int32_t* row_exp, double* Y, double* H,
                       int nthreads, int flags) {
    for (int r = 0; r < nrows; ++r) if (row_exp[r] < 0 || row_exp[r] >= E) return -1;
    const bool gated = (flags & 4) != 0;
    const size_t F1 = gated ? 2 * (size_t)F : (size_t)F;   // rows of W1 per expert
    parallel_for(nrows, nthreads, [&](int r) {
        int t = row_tok[r], e = row_exp[r];
        std::vector<double> xv(d);
        for (int i = 0; i < d; ++i) xv[i] = load_elem(x, (size_t)t * d + i, dtype);
        expert_ffn(d, F, dtype, xv.data(), W1, (size_t)e * F1 * d, b1 ? b1 + (size_t)e * F1 : nullptr,
                   W2, (size_t)e * d * F, b2 ? b2 + (size_t)e * d : nullptr,
                   H ? H + (size_t)r * F : nullptr, Y + (size_t)r * d, gated);
    });
    return 0;
}

// Layer output for a list of tokens given the routing: out = x + sum over kept j (ascending) of
// w_tj * y_tj, in double, rounded once to x's dtype.  A token with no kept pair is copied bit for
// bit.  out_f64 [ntok, d] receives the unrounded value, out_x [ntok, d] the rounded one.
int oracle_combine_tokens(int T, int d, int F, int E, int k, int dtype, const void* x,
                          const void* W1, const float* b1, const void* W2, const float* b2,
                          const int32_t* ids, const float* w, const int32_t* slot, int ntok,
                          const int32_t* tok, double* out_f64, void* out_x, int nthreads,
                          int flags) {
    for (int i = 0; i < ntok; ++i) if (tok[i] < 0 || tok[i] >= T) return -1;
    const bool gated = (flags & 4) != 0;
    const size_t F1 = gated ? 2 * (size_t)F : (size_t)F;
    parallel_for(ntok, nthreads, [&](int i) {
        int t = tok[i];
        std::vector<double> xv(d), y(d), s(d, 0.0);
        for (int c = 0; c < d; ++c) xv[c] = load_elem(x, (size_t)t * d + c, dtype);
        bool any = false;
        for (int j = 0; j < k; ++j) {
            size_t pi = (size_t)t * k + j;
            if (slot[pi] < 0) continue;
            int e = ids[pi];
            expert_ffn(d, F, dtype, xv.data(), W1, (size_t)e * F1 * d,
                       b1 ? b1 + (size_t)e * F1 : nullptr, W2, (size_t)e * d * F,
                       b2 ? b2 + (size_t)e * d : nullptr, nullptr, y.data(), gated);
            for (int c = 0; c < d; ++c) s[c] += (double)w[pi] * y[c];
            any = true;
        }
        for (int c = 0; c < d; ++c) {
            double v = xv[c] + s[c];
            if (out_f64) out_f64[(size_t)i * d + c] = v;
            if (!out_x) continue;
            if (dtype == 0) {
                float* o = (float*)out_x + (size_t)i * d + c;
                *o = any ? (float)v : ((const float*)x)[(size_t)t * d + c];
            } else {
                uint16_t* o = (uint16_t*)out_x + (size_t)i * d + c;
                *o = any ? bf16_from_double(v) : ((const uint16_t*)x)[(size_t)t * d + c];
            }
        }
    });
    return 0;
}

// Combine alone, given the expert outputs: out[t] = x[t] + sum over kept j (ascending) of
// w[t*k+j] * Y[offsets[id] + slot] in double, rounded once to x's dtype; a token with no kept
// pair is copied bit for bit.  Y is [rows, d] in x's dtype.
int oracle_combine_given_y(int T, int d, int E, int k, int dtype, const void* x, const void* Y,
                           long long rows, const float* w, const int32_t* ids,
                           const int32_t* slot, const int32_t* offsets, double* out_f64,
                           void* out_x) {
    for (int t = 0; t < T; ++t) {
        std::vector<double> s(d, 0.0);
        bool any = false;
        for (int j = 0; j < k; ++j) {
            size_t pi = (size_t)t * k + j;
            if (slot[pi] < 0) continue;
            int e = ids[pi];
            if (e < 0 || e >= E) return -1;
            long long r = (long long)offsets[e] + slot[pi];
            if (r < 0 || r >= rows || r >= offsets[e + 1]) return -1;
            for (int c = 0; c < d; ++c) s[c] += (double)w[pi] * load_elem(Y, (size_t)r * d + c, dtype);
            any = true;
        }
        for (int c = 0; c < d; ++c) {
            size_t xi = (size_t)t * d + c;
            double v = load_elem(x, xi, dtype) + s[c];
            if (out_f64) out_f64[xi] = v;
            if (dtype == 0) ((float*)out_x)[xi] = any ? (float)v : ((const float*)x)[xi];
            else ((uint16_t*)out_x)[xi] = any ? bf16_from_double(v) : ((const uint16_t*)x)[xi];
        }
    }
    return 0;
}

uint16_t oracle_bf16_from_double(double v) { return bf16_from_double(v); }

}  // extern "C"
