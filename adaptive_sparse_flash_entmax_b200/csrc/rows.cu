// rows.cu -- row-wise alpha-entmax of a [rows][n] score matrix z (no attention):
//     x = (alpha-1) z,   p = (x - tau)_+^gamma,   sum p = 1 per row,
// and its vector-Jacobian product dz = g (dp - delta), g = u^(gamma-1) on u > 0,
// delta = sum g dp / sum g (the same Jacobian the attention backward applies to S).
// One CTA of 256 threads per row; the row stays in registers (n <= 256 * 64), so
// every solver pass works on chip and the kernel reads z once and writes p once.
// Root finders ("AdaSplash: Adaptive Sparse Flash Attention", Technical Deep Dive /
// Accelerated Alpha-Entmax Transformation; "AdaSplash-2: ...", Sparse Attention
// Makes Waves):
//   ENT_SOLVE_HIST    Halley-bisection from the bracket and start of a 64-bin
//                     histogram of the row (the attention path's solver);
//   ENT_SOLVE_HALLEY  Halley-bisection from the plain bracket [m-1, m - n^(1-alpha)],
//                     midpoint start;
//   ENT_SOLVE_BISECT  bisection on the plain bracket (the baseline of the pages'
//                     iteration-count comparison).
#include "kernels.h"

namespace ent {

namespace {

constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kBisectCap = 48;   // bisection halves a bracket of width <= 1 to float rounding

// Sum of three values over the CTA; every thread gets the totals.
__device__ __forceinline__ void block_sum3(float& a, float& b, float& c, float (*red)[kRowWarps]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    __syncthreads();   // the previous use of red is finished
    if (lane == 0) { red[0][warp] = a; red[1][warp] = b; red[2][warp] = c; }
    __syncthreads();
    a = b = c = 0.f;
#pragma unroll
    for (int w = 0; w < kRowWarps; ++w) { a += red[0][w]; b += red[1][w]; c += red[2][w]; }
}

__device__ __forceinline__ float block_max(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = red[0];
#pragma unroll
    for (int w = 1; w < kRowWarps; ++w) v = fmaxf(v, red[w]);
    return v;
}

// One bisection step after a pass evaluated F0 at tau: keeps the half of the bracket
// that holds the root.  Stops like the Halley-bisection update (|f| <= ftol, or the
// step below stol*max(1,|tau|), keeping the evaluated tau) or at the pass cap.
__device__ __forceinline__ void bisect_update(RowSolver& st, float F0, int pass, float ftol,
                                              float stol) {
    if (st.done) return;
    const float f = F0 - 1.f;
    if (fabsf(f) <= ftol || pass >= kBisectCap) { st.done = 1; st.iters = pass; return; }
    if (f > 0.f) st.lo = st.tau; else st.hi = st.tau;
    const float next = 0.5f * (st.lo + st.hi);
    if (fabsf(next - st.tau) <= stol * fmaxf(1.f, fabsf(st.tau))) { st.done = 1; st.iters = pass; return; }
    st.tau = next;
}

// Bracket and start from a full 64-bin row histogram, computed by one warp: the
// bounds of hist_start_fn (the same G(j) = sum_{k<j} c_k (j-k)^gamma at the edges,
// c_k the count k bins below the top bin A), with lane l evaluating the edges
// j = l and l + 32 by direct sums and ballots locating the two crossings (G grows
// with j); the bin-centre model at lo and hi is a warp sum.  All lanes return
// the same values.
template <int GM>
__device__ __forceinline__ void hist_bracket_warp(const unsigned int* hist, int A, float m, int n,
                                                  float alpha, float gamma, const float* ptab,
                                                  float& lo, float& hi, float& tau0) {
    const int lane = threadIdx.x & 31;
    auto cnt = [&](int k) { return hist[(A - k) & (kBins - 1)]; };
    // G(j) <= 63^gamma  and  G(j) >= 63^gamma at edge j (exact integers for gamma 1..4)
    auto test = [&](int j, bool& le, bool& ge) {
        if (GM >= 1 && GM <= 4) {
            unsigned long long g = 0;
            for (int k = 0; k < j; ++k) {
                const unsigned long long w = (unsigned long long)(j - k);
                const unsigned long long pw = (GM == 1) ? w : (GM == 2) ? w * w : (GM == 3) ? w * w * w : w * w * w * w;
                g += (unsigned long long)cnt(k) * pw;
            }
            const unsigned long long thr = (GM == 1) ? 63ull : (GM == 2) ? 3969ull : (GM == 3) ? 250047ull : 15752961ull;
            le = g <= thr;
            ge = g >= thr;
        } else {
            float g = 0.f;   // G(j) / 63^gamma
            for (int k = 0; k < j; ++k) g = fmaf((float)cnt(k), ptab[j - k], g);
            le = g <= 1.f;
            ge = g >= 1.f;
        }
    };
    bool le0, ge0, le1, ge1, le2 = false, ge2 = false;
    test(lane, le0, ge0);
    test(lane + 32, le1, ge1);
    if (lane == 0) test(64, le2, ge2);
    const int nle = __popc(__ballot_sync(0xffffffffu, le0)) + __popc(__ballot_sync(0xffffffffu, le1)) +
                    __shfl_sync(0xffffffffu, (int)le2, 0);
    const int nge = __popc(__ballot_sync(0xffffffffu, ge0)) + __popc(__ballot_sync(0xffffffffu, ge1)) +
                    __shfl_sync(0xffffffffu, (int)ge2, 0);
    const int h_j = nle - 1;                   // edges 0 .. h_j have G <= 63^gamma (G(0) = 0)
    const int l_j = nge > 0 ? 65 - nge : -1;   // edges l_j .. 64 have G >= 63^gamma
    const float slack = 4.f * 1.1920929e-7f * fmaxf(1.f, fabsf(m));
    const float plain_lo = m - 1.f;
    const float plain_hi = m - exp2f((1.f - alpha) * __log2f((float)n));
    lo = (l_j >= 0 && l_j + 1 <= kBins) ? fmaxf((float)(A - l_j) / kBinsPerUnit - slack, plain_lo) : plain_lo;
    hi = fminf((float)(A + 1 - h_j) / kBinsPerUnit + slack, plain_hi);
    if (hi < lo) hi = lo;
    float fcl = 0.f, fch = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int k = lane + 32 * h;
        const float c = (float)cnt(k);
        const float centre = ((float)(A - k) + 0.5f) / kBinsPerUnit;
        fcl = fmaf(c, entmax_p<GM>(centre - lo, gamma), fcl);
        fch = fmaf(c, entmax_p<GM>(centre - hi, gamma), fch);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        fcl += __shfl_xor_sync(0xffffffffu, fcl, o);
        fch += __shfl_xor_sync(0xffffffffu, fch, o);
    }
    fcl -= 1.f;
    fch -= 1.f;
    float t0 = 0.5f * (lo + hi);
    if (fcl > 0.f && fch < 0.f) t0 = lo + (hi - lo) * (fcl / (fcl - fch));
    tau0 = fminf(fmaxf(t0, lo), hi);
}

// HIST: the histogram start (ENT_SOLVE_HIST); the other solvers take a kernel without it.
// The kernels are bound by the latency of each row's passes, so the rows in flight per SM
// set their rate: the register caps below (CTAs per SM) are the fastest measured on
// [16384, 1024], [16384, 4096] and [4096, 16384] bf16 rows (the forward at eight CTAs per
// SM spills a few words and is still 16 % faster than at three).
template <int E> constexpr int rows_fwd_ctas() { return E <= 16 ? 8 : 2; }
template <int E> constexpr int rows_bwd_ctas() { return E <= 4 ? 8 : E <= 16 ? 5 : 1; }

template <typename T, int E, int GM, bool HIST>
__global__ void __launch_bounds__(kRowThreads, rows_fwd_ctas<E>()) rows_fwd_kernel(const RowArgs a) {
    __shared__ float red[3][kRowWarps];
    __shared__ unsigned int hist[kBins];
    __shared__ float ptab[68];
    __shared__ float bc[2];          // tau, done (broadcast by thread 0)
    const int tid = threadIdx.x;
    const size_t off = (size_t)blockIdx.x * a.n;
    const T* z = static_cast<const T*>(a.z) + off;
    const float gamma = a.gamma, cx = a.cx;
    float x[E];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid + e * kRowThreads;
        x[e] = (j < a.n) ? cx * load_f(z, j) : -INFINITY;
        m = fmaxf(m, x[e]);
    }
    m = block_max(m, red[0]);

    RowSolver sv;
    sv.done = 0;
    sv.iters = 0;
    sv.lo = m - 1.f;
    sv.hi = fmaxf(sv.lo, m - exp2f((1.f - a.alpha) * __log2f((float)a.n)));
    sv.tau = 0.5f * (sv.lo + sv.hi);
    if constexpr (HIST) {
        // 64 bins of width 1/63 on the absolute grid under the row max: [m-1, m]
        const int A = abs_bin(m);
        if (tid < kBins) hist[tid] = 0u;
        if (tid < 65) ptab[tid] = entmax_p<GM>((float)tid / kBinsPerUnit, gamma);
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if (x[e] == -INFINITY) continue;
            const int b = abs_bin(x[e]);
            if (b >= A - (kBins - 1)) atomicAdd(&hist[b & (kBins - 1)], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            hist_bracket_warp<GM>(hist, A, m, a.n, a.alpha, gamma, ptab, sv.lo, sv.hi, sv.tau);
            if (tid == 0) { bc[0] = sv.tau; red[0][0] = sv.lo; red[1][0] = sv.hi; }
        }
        __syncthreads();
        sv.tau = bc[0];
        sv.lo = red[0][0];
        sv.hi = red[1][0];
    }
    for (int pass = 1;; ++pass) {
        float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0;
        const float2 nt2 = make_float2(-sv.tau, -sv.tau);
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const float2 xx = (e + 1 < E) ? make_float2(x[e], x[e + 1]) : make_float2(x[e], -INFINITY);
            entmax_acc_x2<GM>(__fadd2_rn(xx, nt2), gamma, s0, s1, s2);
        }
        float F0 = s0.x + s0.y, F1 = s1.x + s1.y, F2 = s2.x + s2.y;
        block_sum3(F0, F1, F2, red);
        if (tid == 0) {
            if (a.method == kSolveBisect) bisect_update(sv, F0, pass, a.ftol, a.stol);
            else solver_update(sv, F0, F1, F2, gamma, gamma == 1.f, pass, a.ftol, a.stol);
            bc[0] = sv.tau;
            bc[1] = sv.done ? 1.f : 0.f;
        }
        __syncthreads();
        sv.tau = bc[0];
        if (bc[1] != 0.f) break;
    }
    T* p = static_cast<T*>(a.p) + off;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid + e * kRowThreads;
        if (j < a.n) store_f(p, j, entmax_p<GM>(x[e] - sv.tau, gamma));
    }
    if (tid == 0) {
        a.tau[blockIdx.x] = sv.tau;
        if (a.iters) a.iters[blockIdx.x] = (uint8_t)sv.iters;
    }
}

template <typename T, int E, int GM>
__global__ void __launch_bounds__(kRowThreads, rows_bwd_ctas<E>()) rows_bwd_kernel(const RowArgs a) {
    __shared__ float red[3][kRowWarps];
    const int tid = threadIdx.x;
    const size_t off = (size_t)blockIdx.x * a.n;
    const T* z = static_cast<const T*>(a.z) + off;
    const T* dp = static_cast<const T*>(a.dp) + off;
    const float gamma = a.gamma, cx = a.cx, tau = a.tau_in[blockIdx.x];
    float g[E], d[E];
    float sg = 0.f, sgd = 0.f, unused = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid + e * kRowThreads;
        g[e] = (j < a.n) ? entmax_g<GM>(cx * load_f(z, j) - tau, gamma) : 0.f;
        d[e] = (j < a.n) ? load_f(dp, j) : 0.f;
        sg += g[e];
        sgd = fmaf(g[e], d[e], sgd);
    }
    block_sum3(sg, sgd, unused, red);
    const float delta = (sg > 0.f) ? sgd / sg : 0.f;
    T* dz = static_cast<T*>(a.dz) + off;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = tid + e * kRowThreads;
        if (j < a.n) store_f(dz, j, g[e] * (d[e] - delta));
    }
}

template <typename T, int GM>
cudaError_t rows_launch(const RowArgs& a, bool bwd, cudaStream_t s) {
    const dim3 grid(a.rows), block(kRowThreads);
    const int e = (a.n + kRowThreads - 1) / kRowThreads;
    if (bwd) {
        if (e <= 4) rows_bwd_kernel<T, 4, GM><<<grid, block, 0, s>>>(a);
        else if (e <= 16) rows_bwd_kernel<T, 16, GM><<<grid, block, 0, s>>>(a);
        else rows_bwd_kernel<T, 64, GM><<<grid, block, 0, s>>>(a);
    } else if (a.method == kSolveHist) {
        if (e <= 4) rows_fwd_kernel<T, 4, GM, true><<<grid, block, 0, s>>>(a);
        else if (e <= 16) rows_fwd_kernel<T, 16, GM, true><<<grid, block, 0, s>>>(a);
        else rows_fwd_kernel<T, 64, GM, true><<<grid, block, 0, s>>>(a);
    } else {
        if (e <= 4) rows_fwd_kernel<T, 4, GM, false><<<grid, block, 0, s>>>(a);
        else if (e <= 16) rows_fwd_kernel<T, 16, GM, false><<<grid, block, 0, s>>>(a);
        else rows_fwd_kernel<T, 64, GM, false><<<grid, block, 0, s>>>(a);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t rows_dispatch(const RowArgs& a, int gm, bool bwd, cudaStream_t s) {
    switch (gm) {
        case 1: return rows_launch<T, 1>(a, bwd, s);
        case 2: return rows_launch<T, 2>(a, bwd, s);
        default: return rows_launch<T, 0>(a, bwd, s);
    }
}

}  // namespace

cudaError_t rows_entmax(const RowArgs& a, int dtype_bf16, int gm, bool bwd, cudaStream_t s) {
    // alpha = 4/3 and 1.25 take the general (exp2/log2) kernels here
    const int g = (gm == 1 || gm == 2) ? gm : 0;
    return dtype_bf16 ? rows_dispatch<__nv_bfloat16>(a, g, bwd, s) : rows_dispatch<float>(a, g, bwd, s);
}

}  // namespace ent
