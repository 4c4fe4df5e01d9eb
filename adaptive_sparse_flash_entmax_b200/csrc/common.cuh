// common.cuh -- device-side pieces shared by every kernel of the library:
// the alpha-entmax power terms, the per-row tau solver state and its
// Halley-bisection update, the sliding score histogram, and the workspace
// header layout.
//
// Method (AdaSplash pages, by title and section):
//   "AdaSplash: Adaptive Sparse Flash Attention", Technical Deep Dive /
//   Accelerated Alpha-Entmax Transformation: tau is the root of
//   f(tau) = sum_j (x_j - tau)_+^gamma - 1, x = (alpha-1) s, gamma = 1/(alpha-1);
//   f' and f'' are again shifted powers times constants; Halley's step is taken
//   when it stays inside the bracket, otherwise the bracket is bisected.
//   "AdaSplash-2: ...", Sparse Attention Makes Waves: the iteration starts from
//   a coarse histogram of the row's scores kept on chip.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ent {

constexpr int kBlk = 128;          // query-tile rows and key-block columns
constexpr int kBins = 64;          // histogram slots per row
constexpr float kBinsPerUnit = 63.f;  // bin width 1/63: 64 slots cover [m-1, m]
constexpr int kMaxPass = 24;       // solver pass cap (bisection alone needs ~20-23)

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
    unsigned int status;           // 0 = ok, 1 = a bounded wait gave up
    unsigned int timeout_site;     // where it gave up (debug)
    unsigned int tile_counter;     // forward: CTAs finished (the last one re-solves failed tiles)
    unsigned int fail_count;       // forward: tiles on the failure list
    unsigned long long counters[8];
    unsigned int claim;            // forward: failure-list entries taken for solving again
    unsigned char pad1[256 - 16 - 64 - 4];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

enum Counter { kCtrQkBlocks = 0, kCtrPvBlocks = 1, kCtrPasses = 2, kCtrTiles = 3,
               kCtrBwdBlocks = 4, kCtrGvBlocks = 5, kCtrSkipped = 6, kCtrListEntries = 7 };

__device__ __forceinline__ float load_f(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_f(float* p, size_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, size_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}

// Power terms of u = x - tau > 0: t0 = u^gamma (the probability), t1 = u^(gamma-1)
// (the backward's g and -f'/gamma), t2 = u^(gamma-2) (f''/(gamma(gamma-1))).
// GM = 1..4 is an exact integer gamma (alpha = 2, 1.5, 4/3, 1.25); GM = 0 any
// gamma >= 1 via exp2/log2.  u <= 0 gives zeros (strict support).
template <int GM>
__device__ __forceinline__ void entmax_terms(float u, float gamma, float& t0, float& t1,
                                             float& t2) {
    if (!(u > 0.f)) { t0 = t1 = t2 = 0.f; return; }
    if (GM == 1) { t0 = u; t1 = 1.f; t2 = 0.f; }
    else if (GM == 2) { t0 = u * u; t1 = u; t2 = 1.f; }
    else if (GM == 3) { const float u2 = u * u; t0 = u2 * u; t1 = u2; t2 = u; }
    else if (GM == 4) { const float u2 = u * u; t0 = u2 * u2; t1 = u2 * u; t2 = u2; }
    else {
        t2 = exp2f((gamma - 2.f) * __log2f(u));
        t1 = t2 * u;
        t0 = t1 * u;
    }
}

template <int GM>
__device__ __forceinline__ float entmax_p(float u, float gamma) {
    if (!(u > 0.f)) return 0.f;
    if (GM == 1) return u;
    if (GM == 2) return u * u;
    if (GM == 3) return u * u * u;
    if (GM == 4) { const float u2 = u * u; return u2 * u2; }
    return exp2f(gamma * __log2f(u));
}

template <int GM>
__device__ __forceinline__ float entmax_g(float u, float gamma) {
    if (!(u > 0.f)) return 0.f;
    if (GM == 1) return 1.f;
    if (GM == 2) return u;
    if (GM == 3) return u * u;
    if (GM == 4) return u * u * u;
    return exp2f((gamma - 1.f) * __log2f(u));
}

// Per-row solver state.  `unv`: the row stopped on a Halley step it did not
// evaluate (the forward verifies it afterwards); `down`: that step went down, so the
// support may have grown past the blocks live in the last pass.
struct RowSolver {
    float tau, lo, hi;
    int done;
    int iters;
    int unv = 0;
    int down = 0;
};

// Unverified-step rules of solver_update (all 0: every stop is at an evaluated tau).
struct AcceptRule {
    float step = 0.f;      // largest step, either way
    float cert_up = 0.f;   // bound on the change in f from elements crossing the support
    float cert_down = 0.f; // boundary within an upward / a downward step
};

// One Halley-bisection update after a pass evaluated F0 = sum u^gamma,
// F1 = sum u^(gamma-1), F2 = sum u^(gamma-2) at the current tau.  Stops (keeping
// the evaluated tau) when |f| <= ftol, when the proposed step is below
// stol*max(1,|tau|), or at the pass cap.  The Halley point is taken when it lies
// within the closed bracket [lo, hi] (a point that rounding put a few ulps
// outside is clamped onto it: a root on a bracket end, such as tau = m - 1 for
// a one-element support, must stay reachable); otherwise the bracket is bisected.
// The rule `acc` may also stop a row on a Halley step it takes without evaluating
// it, when f at the new point is small by two counts.  (1) With the support fixed, f
// after the step is f + dl f' + dl^2 f''/2 (exact for gamma = 2, whose f is then a
// quadratic, and for gamma = 1, a line; a Taylor estimate otherwise): Halley's own
// miss, which is not small where f is not.  (2) Each element that crosses the
// boundary within a step h changes f by at most h^gamma.  Upward, only elements of the
// support (u <= h) can leave: together at most h^2 F2 (gamma >= 2) or h F1
// (gamma < 2), from the sums just evaluated.  Downward, the elements that can enter
// are not counted by the sums; h^min(gamma,2) per entering element is what the rule
// bounds.  Either way the caller checks f at the new tau afterwards.
__device__ __forceinline__ void solver_update(RowSolver& st, float F0, float F1, float F2,
                                              float gamma, bool gamma_is_one, int pass,
                                              float ftol, float stol,
                                              const AcceptRule& acc = AcceptRule()) {
    if (st.done) return;
    const float f = F0 - 1.f;
    if (fabsf(f) <= ftol || pass >= kMaxPass) { st.done = 1; st.iters = pass; return; }
    if (f > 0.f) st.lo = st.tau; else st.hi = st.tau;
    const float fp = -gamma * F1;
    const float fpp = gamma_is_one ? 0.f : gamma * (gamma - 1.f) * F2;
    const float h = st.tau - 2.f * f * fp / (2.f * fp * fp - f * fpp);
    const float scale = fmaxf(1.f, fabsf(st.tau));
    const float tol = stol * scale;
    const bool halley = isfinite(h) && h >= st.lo - tol && h <= st.hi + tol;
    const float next = halley ? fminf(fmaxf(h, st.lo), st.hi) : 0.5f * (st.lo + st.hi);
    const float dl = next - st.tau;
    if (fabsf(dl) <= tol) { st.done = 1; st.iters = pass; return; }
    if (halley && fabsf(dl) <= acc.step) {
        const float h = fabsf(dl);
        const float cross = (dl > 0.f) ? ((gamma >= 2.f) ? F2 * h * h : F1 * h)
                                       : ((gamma >= 2.f) ? h * h : exp2f(gamma * __log2f(h)));
        const float miss = fabsf(f + dl * (fp + 0.5f * dl * fpp));   // fixed-support f after it
        if (miss + cross <= (dl > 0.f ? acc.cert_up : acc.cert_down)) {
            st.tau = next; st.done = 1; st.unv = 1; st.down = dl < 0.f; st.iters = pass; return;
        }
    }
    st.tau = next;
}

// ---------------------------------------------------------------- histogram
// Absolute bin of x: a = floor(x * 63).  A row whose running maximum m has bin
// A keeps the 64 bins A-63..A in slots (a & 63).  Anything below bin A-63 lies
// under (A-63)/63 <= m - 1 <= tau and can never be in the support.
__device__ __forceinline__ int abs_bin(float x) { return __float2int_rd(x * kBinsPerUnit); }

constexpr int kNoBin = -(1 << 29);

// Slots of hist (stride `stride` between slots of one row) that leave the
// window when the top bin moves from A_old to A_new are cleared.
template <typename C>
__device__ __forceinline__ void hist_slide(C* hist, int stride, int A_old, int A_new) {
    if (A_new <= A_old) return;
    const int moved = A_new - A_old;
    if (moved >= kBins) {
        for (int s = 0; s < kBins; ++s) hist[s * stride] = 0;
    } else {
        for (int k = 0; k < moved; ++k) hist[((A_old - (kBins - 1) + k) & (kBins - 1)) * stride] = 0;
    }
}

// Bracket and start for tau from a row histogram (top bin A, max m, n admissible
// keys), using ptab[k] = (k/63)^gamma, k = 0..64.
// With k = A - a (k = 0 the top bin) and the edge index j = A + 1 - e of the edge
// E = e/63 (j = 0 the top edge), let
//     G(j) = sum_{k < j} c_k (j - k)^gamma.
// The bins give rigorous bounds of f at the edges:
//     F_up(E)  = G(j)     / 63^gamma - 1  >=  f(E),
//     F_low(E) = G(j - 1) / 63^gamma - 1  <=  f(E)
// (every element of bin a lies in [a/63, (a+1)/63)).  G grows with j, so
// hi = the lowest edge with F_up <= 0 (the largest j with G(j) <= 63^gamma) and
// lo = the highest edge with F_low >= 0 (j = j* + 1 for the smallest j* with
// G(j*) >= 63^gamma).  For an integer gamma (1..4) G comes from running moments
// M_r = sum_{k<j} c_k k^r in one sweep over the bins (exact: double holds these
// integers); otherwise G is evaluated directly inside two binary searches.
// Both ends are widened by a few ulps of m against rounding in the bin
// assignment and intersected with the plain bracket [m-1, m - n^(1-alpha)].
// tau_0 is the root of the straight line through the bin-centre model
// F_c(E) = sum_a c_a ((a+1/2)/63 - E)_+^gamma - 1 at E = lo and E = hi.
// `count(a)` returns the number of elements in absolute bin a (a in [ebot, A]);
// every element at or above edge ebot/63 is counted (the window may be narrower
// than 64 bins; edges below ebot are not used).
template <int GM, typename CountFn>
__device__ __forceinline__ void hist_start_fn(CountFn count, int A, int ebot, float m, int n,
                                              float alpha, float gamma, const float* ptab,
                                              float& lo, float& hi, float& tau0) {
    const int jmax = A + 1 - ebot;        // usable edges j = 0 .. jmax
    int h_j = 0;                          // largest j with G(j) <= 63^gamma
    int l_j = -1;                         // smallest j with G(j) >= 63^gamma
    if (GM >= 1 && GM <= 4) {
        // Exact sweep from the top edge down: finite differences of G in j are
        // integer recurrences (64-bit: G <= 65535 * 64^4),
        //   D_r(j) = sum_{k<j} c_k (j-k)^r,
        //   D_r(j+1) = sum_{i<=r} C(r,i) D_i(j) + c_j   (binomial expansion of (j-k+1)^r).
        // G = D_gamma grows with j, so the sweep stops at the first edge with
        // G >= 63^gamma.  A compact loop: this code runs once per row, and an
        // unrolled version costs more in instruction fetch than in arithmetic.
        const long long thr = (GM == 1) ? 63ll : (GM == 2) ? 3969ll : (GM == 3) ? 250047ll : 15752961ll;
        long long D0 = 0, D1 = 0, D2 = 0, D3 = 0, D4 = 0;
        unsigned int c_next = (jmax > 0) ? count(A) : 0u;
#pragma unroll 1
        for (int j = 0; j <= jmax; ++j) {
            const long long G = (GM == 1) ? D1 : (GM == 2) ? D2 : (GM == 3) ? D3 : D4;
            if (G >= thr) { l_j = j; h_j = (G == thr) ? j : j - 1; break; }
            h_j = j;
            const long long c = (long long)c_next;
            c_next = (j + 1 < jmax) ? count(A - j - 1) : 0u;
            if (GM >= 4) D4 = D4 + 4 * D3 + 6 * D2 + 4 * D1 + D0 + c;
            if (GM >= 3) D3 = D3 + 3 * D2 + 3 * D1 + D0 + c;
            if (GM >= 2) D2 = D2 + 2 * D1 + D0 + c;
            D1 = D1 + D0 + c;
            D0 = D0 + c;
        }
    } else {
        auto Gn = [&](int j) {   // G(j) / 63^gamma
            float acc = 0.f;
            for (int k = 0; k < j; ++k) acc = fmaf((float)count(A - k), ptab[j - k], acc);
            return acc;
        };
        int ok_ = 0, bad = jmax + 1;               // Gn(0) = 0 <= 1; Gn(jmax+1) treated as > 1
        while (bad - ok_ > 1) { const int mid = (ok_ + bad) >> 1; if (Gn(mid) <= 1.f) ok_ = mid; else bad = mid; }
        h_j = ok_;
        if (Gn(jmax) >= 1.f) {
            int lo_ = 0, hi_ = jmax;               // Gn(0) = 0 < 1, Gn(jmax) >= 1
            while (hi_ - lo_ > 1) { const int mid = (lo_ + hi_) >> 1; if (Gn(mid) >= 1.f) hi_ = mid; else lo_ = mid; }
            l_j = hi_;
        }
    }
    const float slack = 4.f * 1.1920929e-7f * fmaxf(1.f, fabsf(m));
    const float plain_lo = m - 1.f;
    const float plain_hi = m - exp2f((1.f - alpha) * __log2f((float)n));
    lo = (l_j >= 0 && l_j + 1 <= jmax) ? fmaxf((float)(A - l_j) / kBinsPerUnit - slack, plain_lo) : plain_lo;
    hi = fminf((float)(A + 1 - h_j) / kBinsPerUnit + slack, plain_hi);
    if (hi < lo) hi = lo;
    // Bins whose centre lies below lo add nothing to either model value; with lo
    // from the histogram those are the bins k > l_j (k = A - a).
    const int kend = (l_j >= 0 && l_j + 1 <= jmax) ? min(jmax, l_j + 2) : jmax;
    float fcl = -1.f, fch = -1.f;
#pragma unroll 1
    for (int k = 0; k < kend; ++k) {
        const unsigned int c = count(A - k);
        const float centre = ((float)(A - k) + 0.5f) / kBinsPerUnit;
        fcl = fmaf((float)c, entmax_p<GM>(centre - lo, gamma), fcl);
        fch = fmaf((float)c, entmax_p<GM>(centre - hi, gamma), fch);
    }
    float t0 = 0.5f * (lo + hi);
    if (fcl > 0.f && fch < 0.f) t0 = lo + (hi - lo) * (fcl / (fcl - fch));
    tau0 = fminf(fmaxf(t0, lo), hi);
}

// Single histogram with slots hist[(a & 63) * stride].
template <int GM>
__device__ __forceinline__ void hist_start(const unsigned int* hist, int stride, int A, float m,
                                           int n, float alpha, float gamma, const float* ptab,
                                           float& lo, float& hi, float& tau0) {
    hist_start_fn<GM>([&](int a) { return hist[(a & (kBins - 1)) * stride]; }, A,
                      A - (kBins - 1), m, n, alpha, gamma, ptab, lo, hi, tau0);
}

// Branch-free power terms for the streaming passes: u <= 0 gives zeros through
// max(u, 0) and selects instead of branches.
template <int GM>
__device__ __forceinline__ void entmax_terms_bf(float u, float gamma, float& t0, float& t1,
                                                float& t2) {
    const float up = fmaxf(u, 0.f);
    if (GM == 1) { t0 = up; t1 = (u > 0.f) ? 1.f : 0.f; t2 = 0.f; }
    else if (GM == 2) { t0 = up * up; t1 = up; t2 = (u > 0.f) ? 1.f : 0.f; }
    else if (GM == 3) { t2 = up; t1 = up * up; t0 = t1 * up; }
    else if (GM == 4) { t2 = up * up; t1 = t2 * up; t0 = t2 * t2; }
    else {
        const float l = __log2f(up);                      // -inf at up = 0
        const float v = exp2f((gamma - 2.f) * l);         // inf at up = 0 when gamma < 2
        t2 = (u > 0.f) ? v : 0.f;
        t1 = t2 * up;
        t0 = t1 * up;
    }
}

template <int GM>
__device__ __forceinline__ float entmax_g_bf(float u, float gamma) {
    const float up = fmaxf(u, 0.f);
    if (GM == 1) return (u > 0.f) ? 1.f : 0.f;
    if (GM == 2) return up;
    if (GM == 3) return up * up;
    if (GM == 4) return up * up * up;
    const float v = exp2f((gamma - 1.f) * __log2f(up));   // inf at up = 0 when gamma < 1 (not used)
    return (u > 0.f) ? v : 0.f;
}

// Packed (two-lane f32x2) accumulation of the power terms for the streaming
// passes: a0 += u^gamma, a1 += u^(gamma-1), a2 += u^(gamma-2) for both lanes of
// u, zeros where u <= 0.  The sm_100 packed FMA/ADD/MUL issue two fp32 lanes per
// instruction.
__device__ __forceinline__ float step_pos(float u) { return (u > 0.f) ? 1.f : 0.f; }

template <int GM>
__device__ __forceinline__ void entmax_acc_x2(float2 u, float gamma, float2& a0, float2& a1,
                                              float2& a2) {
    const float2 up = make_float2(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f));
    if (GM == 1) {
        a0 = __fadd2_rn(a0, up);
        a1 = __fadd2_rn(a1, make_float2(step_pos(u.x), step_pos(u.y)));
    } else if (GM == 2) {
        a0 = __ffma2_rn(up, up, a0);
        a1 = __fadd2_rn(a1, up);
        a2 = __fadd2_rn(a2, make_float2(step_pos(u.x), step_pos(u.y)));
    } else if (GM == 3) {
        const float2 t1 = __fmul2_rn(up, up);
        a0 = __ffma2_rn(t1, up, a0);
        a1 = __fadd2_rn(a1, t1);
        a2 = __fadd2_rn(a2, up);
    } else if (GM == 4) {
        const float2 t2 = __fmul2_rn(up, up);
        a0 = __ffma2_rn(t2, t2, a0);
        a1 = __ffma2_rn(t2, up, a1);
        a2 = __fadd2_rn(a2, t2);
    } else {
        const float vx = exp2f((gamma - 2.f) * __log2f(up.x));   // inf at 0 when gamma < 2
        const float vy = exp2f((gamma - 2.f) * __log2f(up.y));
        const float2 t2 = make_float2((u.x > 0.f) ? vx : 0.f, (u.y > 0.f) ? vy : 0.f);
        const float2 t1 = __fmul2_rn(t2, up);
        a0 = __ffma2_rn(t1, up, a0);
        a1 = __fadd2_rn(a1, t1);
        a2 = __fadd2_rn(a2, t2);
    }
}

// Packed p = u_+^gamma for both lanes.
template <int GM>
__device__ __forceinline__ float2 entmax_p_x2(float2 u, float gamma) {
    const float2 up = make_float2(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f));
    if (GM == 1) return up;
    if (GM == 2) return __fmul2_rn(up, up);
    if (GM == 3) return __fmul2_rn(__fmul2_rn(up, up), up);
    if (GM == 4) { const float2 u2 = __fmul2_rn(up, up); return __fmul2_rn(u2, u2); }
    return make_float2(exp2f(gamma * __log2f(up.x)), exp2f(gamma * __log2f(up.y)));
}

// Packed g = u_+^(gamma-1) for both lanes (the backward's weights).
template <int GM>
__device__ __forceinline__ float2 entmax_g_x2(float2 u, float gamma) {
    const float2 up = make_float2(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f));
    if (GM == 1) return make_float2(step_pos(u.x), step_pos(u.y));
    if (GM == 2) return up;
    if (GM == 3) return __fmul2_rn(up, up);
    if (GM == 4) return __fmul2_rn(__fmul2_rn(up, up), up);
    const float vx = exp2f((gamma - 1.f) * __log2f(up.x)), vy = exp2f((gamma - 1.f) * __log2f(up.y));
    return make_float2((u.x > 0.f) ? vx : 0.f, (u.y > 0.f) ? vy : 0.f);
}

// Packed p = u_+^gamma and g = u_+^(gamma-1) together.
template <int GM>
__device__ __forceinline__ void entmax_pg_x2(float2 u, float gamma, float2& p, float2& g) {
    const float2 up = make_float2(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f));
    if (GM == 1) { p = up; g = make_float2(step_pos(u.x), step_pos(u.y)); }
    else if (GM == 2) { g = up; p = __fmul2_rn(up, up); }
    else if (GM == 3) { g = __fmul2_rn(up, up); p = __fmul2_rn(g, up); }
    else if (GM == 4) { const float2 t = __fmul2_rn(up, up); g = __fmul2_rn(t, up); p = __fmul2_rn(t, t); }
    else {
        const float lx = __log2f(up.x), ly = __log2f(up.y);
        p = make_float2(exp2f(gamma * lx), exp2f(gamma * ly));
        g = make_float2((u.x > 0.f) ? exp2f((gamma - 1.f) * lx) : 0.f,
                        (u.y > 0.f) ? exp2f((gamma - 1.f) * ly) : 0.f);
    }
}

template <int GM>
__device__ __forceinline__ float entmax_p_bf(float u, float gamma) {
    const float up = fmaxf(u, 0.f);
    if (GM == 1) return up;
    if (GM == 2) return up * up;
    if (GM == 3) return up * up * up;
    if (GM == 4) { const float u2 = up * up; return u2 * u2; }
    return exp2f(gamma * __log2f(up));                    // 0 at up = 0 (gamma > 0)
}

}  // namespace ent
