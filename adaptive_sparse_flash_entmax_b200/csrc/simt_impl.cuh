// simt_impl.cuh -- the FP32 CUDA-core path of the fused alpha-entmax attention.
//
// It runs the whole method in true fp32 (scores by FMA, not on tensor cores):
// float32 inputs always take this path, because TF32 tensor-core products carry
// ~1e-3 relative score error, far above what an fp32 caller expects.
//
// Forward (one CTA per 128-row query tile; thread = query row), following
// "AdaSplash: Adaptive Sparse Flash Attention", Technical Deep Dive /
// AdaSplash: Fused GPU Kernel for Attention, with the AdaSplash-2 histogram
// start ("AdaSplash-2: ...", Sparse Attention Makes Waves):
//   pass 0      stream K: row max + sliding 64-bin score histogram,
//               then a rigorous bracket and tau_0 per row;
//   passes 1..k stream K: F0 = sum u^g, F1 = sum u^(g-1), F2 = sum u^(g-2),
//               u = x - tau; Halley-bisection update; the last pass also
//               marks which key blocks hold any u > 0 (Exploiting Sparsity);
//   P.V pass    stream K, V of the live blocks only: O = sum p v.
// Backward (Experimental Setup & Results / Backward Pass: the zero blocks are
// skipped): per query tile delta and dQ; per key block dK and dV.
#pragma once
#include "common.cuh"
#include "kernels.h"

namespace ent {

constexpr int kSub = 32;    // keys per shared-memory sub-block (forward)
constexpr int kSubB = 16;   // keys / rows per sub-block (backward)

template <typename TIn, int D>
__device__ __forceinline__ void load_rows_f32(float* dst, int dst_stride, const TIn* src,
                                              int row0, int nrows, int N, int tid, int nthr) {
    for (int idx = tid; idx < nrows * D; idx += nthr) {
        const int r = idx / D, c = idx - r * D;
        const int g = row0 + r;
        dst[r * dst_stride + c] = (g < N) ? load_f(src, (size_t)g * D + c) : 0.f;
    }
}

// r[jj] = q_row . K_s[jj] for kSub keys; q from padded smem row, K broadcast.
template <int D, int NK>
__device__ __forceinline__ void dot_rows(float (&r)[NK], const float* qrow, const float* Ks) {
#pragma unroll
    for (int jj = 0; jj < NK; ++jj) r[jj] = 0.f;
#pragma unroll 2
    for (int c = 0; c < D; c += 4) {
        const float q0 = qrow[c], q1 = qrow[c + 1], q2 = qrow[c + 2], q3 = qrow[c + 3];
#pragma unroll
        for (int jj = 0; jj < NK; ++jj) {
            const float4 kv = *reinterpret_cast<const float4*>(Ks + jj * D + c);
            r[jj] = fmaf(q0, kv.x, r[jj]);
            r[jj] = fmaf(q1, kv.y, r[jj]);
            r[jj] = fmaf(q2, kv.z, r[jj]);
            r[jj] = fmaf(q3, kv.w, r[jj]);
        }
    }
}

template <int D>
constexpr size_t simt_fwd_smem(int T) {
    return sizeof(float) * (128 * (D + 1) + 2 * kSub * D + kBins * 128 + 68) + (size_t)((T + 15) / 16) * 16;
}

template <typename TIn, int D, int GM>
__global__ void __launch_bounds__(128, 1) simt_fwd_kernel(FwdArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* Qs = reinterpret_cast<float*>(smem_raw);            // [128][D+1]
    float* Ks = Qs + 128 * (D + 1);                             // [kSub][D]
    float* Vs = Ks + kSub * D;                                  // [kSub][D]
    unsigned int* hist = reinterpret_cast<unsigned int*>(Vs + kSub * D);   // [64][128]
    float* ptab = reinterpret_cast<float*>(hist + kBins * 128);            // [65] (+pad)
    unsigned char* live = reinterpret_cast<unsigned char*>(ptab + 68);     // [T]

    const int tid = threadIdx.x;
    const int T = a.T, N = a.N;
    const int t = a.causal ? (T - 1 - (int)blockIdx.x) : (int)blockIdx.x;  // long tiles first
    const int bh = blockIdx.y;
    const size_t head = (size_t)bh * N * D;
    const TIn* q = static_cast<const TIn*>(a.q) + head;
    const TIn* k = static_cast<const TIn*>(a.k) + head;
    const TIn* v = static_cast<const TIn*>(a.v) + head;
    const int i = t * kBlk + tid;
    const bool row_valid = i < N;
    const int last_row = min(t * kBlk + kBlk - 1, N - 1);
    const int nblk = a.causal ? t + 1 : T;
    const int key_end = !row_valid ? 0 : (a.causal ? i + 1 : N);   // admissible keys [0, key_end)
    const float gamma = a.gamma, cx = a.cx;

    load_rows_f32<TIn, D>(Qs, D + 1, q, t * kBlk, kBlk, N, tid, 128);
    if (tid < 65) ptab[tid] = entmax_p<GM>((float)tid / kBinsPerUnit, gamma);
    for (int s = 0; s < kBins; ++s) hist[s * 128 + tid] = 0u;
    for (int b = tid; b < T; b += 128) live[b] = 0;
    const float* qrow = Qs + tid * (D + 1);

    float m = -INFINITY;
    int A = kNoBin;
    RowSolver st;
    st.tau = 0.f; st.lo = 0.f; st.hi = 0.f;
    st.done = row_valid ? 0 : 1;
    st.iters = 0;
    int pass = 0;
    for (;; ++pass) {
        float F0 = 0.f, F1 = 0.f, F2 = 0.f;
        for (int b = 0; b < nblk; ++b) {
            int any = 0;
            for (int sb = 0; sb < kBlk / kSub; ++sb) {
                const int j0 = b * kBlk + sb * kSub;
                if (j0 >= N || (a.causal && j0 > last_row)) break;   // CTA-uniform
                __syncthreads();
                load_rows_f32<TIn, D>(Ks, D, k, j0, kSub, N, tid, 128);
                __syncthreads();
                float r[kSub];
                dot_rows<D, kSub>(r, qrow, Ks);
                const int nv = key_end - j0;   // valid keys of this sub-block: jj < nv
                if (pass == 0) {
                    float bm = -INFINITY;
#pragma unroll
                    for (int jj = 0; jj < kSub; ++jj)
                        if (jj < nv) bm = fmaxf(bm, __fmul_rn(cx, r[jj]));
                    if (bm > m) {
                        m = bm;
                        const int An = abs_bin(m);
                        hist_slide(hist + tid, 128, A, An);
                        A = An;
                    }
#pragma unroll
                    for (int jj = 0; jj < kSub; ++jj) {
                        if (jj < nv) {
                            const int ab = abs_bin(__fmul_rn(cx, r[jj]));
                            if (ab >= A - (kBins - 1)) hist[(ab & (kBins - 1)) * 128 + tid] += 1u;
                        }
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < kSub; ++jj) {
                        if (jj < nv) {
                            const float u = __fmaf_rn(cx, r[jj], -st.tau);
                            float t0, t1, t2;
                            entmax_terms<GM>(u, gamma, t0, t1, t2);
                            F0 += t0; F1 += t1; F2 += t2;
                            any |= (u > 0.f);
                        }
                    }
                }
            }
            if (pass > 0) {
                const int blk_live = __syncthreads_or(any);
                if (tid == 0) live[b] = (unsigned char)blk_live;
            }
        }
        if (pass == 0) {
            if (row_valid) {
                hist_start<GM>(hist + tid, 128, A, m, key_end, a.alpha, gamma, ptab, st.lo, st.hi,
                               st.tau);
            }
        } else {
            solver_update(st, F0, F1, F2, gamma, gamma == 1.f, pass, a.ftol, a.stol);
        }
        if (pass > 0 && __syncthreads_and(st.done)) break;
    }
    const int npass = pass;   // solver passes after the statistics pass

    // P.V over live blocks; with otilde a second sweep accumulates G.V and sum_j g
    // (g = u^(gamma-1)) for otilde = G.V / sum_j g.
    int nlive = 0;
    const int nsweep = a.otilde ? 2 : 1;
#pragma unroll 1
    for (int sweep = 0; sweep < nsweep; ++sweep) {
        float acc[D];
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = 0.f;
        float wsum = 0.f;
        for (int b = 0; b < nblk; ++b) {
            if (!live[b]) continue;   // CTA-uniform (shared flag, written before the last barrier)
            if (sweep == 0) ++nlive;
            for (int sb = 0; sb < kBlk / kSub; ++sb) {
                const int j0 = b * kBlk + sb * kSub;
                if (j0 >= N || (a.causal && j0 > last_row)) break;
                __syncthreads();
                load_rows_f32<TIn, D>(Ks, D, k, j0, kSub, N, tid, 128);
                load_rows_f32<TIn, D>(Vs, D, v, j0, kSub, N, tid, 128);
                __syncthreads();
                float r[kSub];
                dot_rows<D, kSub>(r, qrow, Ks);
                const int nv = key_end - j0;
#pragma unroll
                for (int jj = 0; jj < kSub; ++jj) {
                    const float u = __fmaf_rn(cx, r[jj], -st.tau);
                    const float p = (jj >= nv) ? 0.f : (sweep == 0) ? entmax_p<GM>(u, gamma) : entmax_g<GM>(u, gamma);
                    wsum += p;
#pragma unroll
                    for (int c = 0; c < D; c += 4) {
                        const float4 vv = *reinterpret_cast<const float4*>(Vs + jj * D + c);
                        acc[c] = fmaf(p, vv.x, acc[c]);
                        acc[c + 1] = fmaf(p, vv.y, acc[c + 1]);
                        acc[c + 2] = fmaf(p, vv.z, acc[c + 2]);
                        acc[c + 3] = fmaf(p, vv.w, acc[c + 3]);
                    }
                }
            }
        }
        if (row_valid && sweep == 0) {
            TIn* o = static_cast<TIn*>(a.o) + head + (size_t)i * D;
#pragma unroll
            for (int c = 0; c < D; ++c) store_f(o, c, acc[c]);
        } else if (row_valid) {
            float* ot = a.otilde + head + (size_t)i * D;
            const float rs = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
            for (int c = 0; c < D; ++c) ot[c] = acc[c] * rs;
        }
    }
    if (row_valid) {
        a.tau[(size_t)bh * N + i] = st.tau;
        if (a.iters) a.iters[(size_t)bh * N + i] = (unsigned char)st.iters;
    }
    uint8_t* mrow = a.mask + ((size_t)bh * T + t) * T;
    for (int b = tid; b < T; b += 128) mrow[b] = (b < nblk) ? live[b] : 0;
    if (tid == 0) {
        atomicAdd(&a.hdr->counters[kCtrQkBlocks], (unsigned long long)nblk * (npass + 1));
        atomicAdd(&a.hdr->counters[kCtrPvBlocks], (unsigned long long)nlive);
        atomicAdd(&a.hdr->counters[kCtrPasses], (unsigned long long)npass);
        atomicAdd(&a.hdr->counters[kCtrTiles], 1ull);
        if (a.otilde) atomicAdd(&a.hdr->counters[kCtrGvBlocks], (unsigned long long)nlive);
    }
}

// ------------------------------------------------------------------ backward
// delta and dQ for one 128-row query tile (thread = query row).
template <int D>
constexpr size_t simt_bwd_dq_smem() {
    return sizeof(float) * (2 * 128 * (D + 1) + 2 * kSubB * D);
}

template <typename TIn, int D, int GM>
__global__ void __launch_bounds__(128, 1) simt_bwd_dq_kernel(BwdArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* Qs = reinterpret_cast<float*>(smem_raw);   // [128][D+1]
    float* dOs = Qs + 128 * (D + 1);                   // [128][D+1]
    float* Ks = dOs + 128 * (D + 1);                   // [kSubB][D]
    float* Vs = Ks + kSubB * D;                        // [kSubB][D]
    const int tid = threadIdx.x;
    const int T = a.T, N = a.N;
    const int t = a.causal ? (T - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int bh = blockIdx.y;
    const size_t head = (size_t)bh * N * D;
    const TIn* k = static_cast<const TIn*>(a.k) + head;
    const TIn* v = static_cast<const TIn*>(a.v) + head;
    const int i = t * kBlk + tid;
    const bool row_valid = i < N;
    const int last_row = min(t * kBlk + kBlk - 1, N - 1);
    const int nblk = a.causal ? t + 1 : T;
    const int key_end = !row_valid ? 0 : (a.causal ? i + 1 : N);
    const float gamma = a.gamma, cx = a.cx;
    const uint8_t* mrow = a.mask + ((size_t)bh * T + t) * T;

    load_rows_f32<TIn, D>(Qs, D + 1, static_cast<const TIn*>(a.q) + head, t * kBlk, kBlk, N, tid, 128);
    load_rows_f32<TIn, D>(dOs, D + 1, static_cast<const TIn*>(a.dout) + head, t * kBlk, kBlk, N, tid, 128);
    const float* qrow = Qs + tid * (D + 1);
    const float* dorow = dOs + tid * (D + 1);
    const float tau = row_valid ? a.tau[(size_t)bh * N + i] : 0.f;

    float sg = 0.f, sgdp = 0.f, delta = 0.f;
    float acc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) acc[c] = 0.f;
    int nvis = 0, nphase0 = 0;
    if (a.otilde) {
        // delta_i = dO_i . otilde_i (dP = dO V^T), so the delta phase is not needed
        __syncthreads();   // the dO tile is loaded cooperatively
        if (row_valid) {
            const float* ot = a.otilde + head + (size_t)i * D;
            for (int c = 0; c < D; ++c) delta = fmaf(dorow[c], ot[c], delta);
            a.delta[(size_t)bh * N + i] = delta;
        }
    }
    for (int phase = a.otilde ? 1 : 0; phase < 2; ++phase) {
        for (int b = 0; b < nblk; ++b) {
            if (!mrow[b]) continue;   // CTA-uniform
            ++nvis;
            if (phase == 0) ++nphase0;
            for (int sb = 0; sb < kBlk / kSubB; ++sb) {
                const int j0 = b * kBlk + sb * kSubB;
                if (j0 >= N || (a.causal && j0 > last_row)) break;
                __syncthreads();
                load_rows_f32<TIn, D>(Ks, D, k, j0, kSubB, N, tid, 128);
                load_rows_f32<TIn, D>(Vs, D, v, j0, kSubB, N, tid, 128);
                __syncthreads();
                float r[kSubB], dp[kSubB];
                dot_rows<D, kSubB>(r, qrow, Ks);
                dot_rows<D, kSubB>(dp, dorow, Vs);
                const int nv = key_end - j0;
#pragma unroll
                for (int jj = 0; jj < kSubB; ++jj) {
                    const float g = (jj < nv) ? entmax_g<GM>(__fmaf_rn(cx, r[jj], -tau), gamma) : 0.f;
                    if (phase == 0) {
                        sg += g;
                        sgdp = fmaf(g, dp[jj], sgdp);
                    } else {
                        const float ds = g * (dp[jj] - delta);
#pragma unroll
                        for (int c = 0; c < D; c += 4) {
                            const float4 kv = *reinterpret_cast<const float4*>(Ks + jj * D + c);
                            acc[c] = fmaf(ds, kv.x, acc[c]);
                            acc[c + 1] = fmaf(ds, kv.y, acc[c + 1]);
                            acc[c + 2] = fmaf(ds, kv.z, acc[c + 2]);
                            acc[c + 3] = fmaf(ds, kv.w, acc[c + 3]);
                        }
                    }
                }
            }
        }
        if (phase == 0) {
            delta = (sg > 0.f) ? sgdp / sg : 0.f;
            if (row_valid) a.delta[(size_t)bh * N + i] = delta;
        }
    }
    if (row_valid) {
        TIn* dq = static_cast<TIn*>(a.dq) + head + (size_t)i * D;
#pragma unroll
        for (int c = 0; c < D; ++c) store_f(dq, c, acc[c] * a.scale);
    }
    // block GEMMs: the delta phase computes S and dP (2), the dQ phase S, dP and dS K (3)
    if (tid == 0)
        atomicAdd(&a.hdr->counters[kCtrBwdBlocks], (unsigned long long)(2 * nphase0 + 3 * (nvis - nphase0)));
}

// dV (WHICH = 0) or dK (WHICH = 1) for one 128-key block (thread = key).
// Needs delta from simt_bwd_dq_kernel for dK.
template <int D>
constexpr size_t simt_bwd_dkv_smem() {
    return sizeof(float) * (2 * 128 * (D + 1) + 2 * kSubB * D + 2 * kSubB);
}

template <typename TIn, int D, int GM, int WHICH>
__global__ void __launch_bounds__(128, 1) simt_bwd_dkv_kernel(BwdArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* Ks = reinterpret_cast<float*>(smem_raw);   // [128][D+1]
    float* Vs = Ks + 128 * (D + 1);                    // [128][D+1]
    float* Qr = Vs + 128 * (D + 1);                    // [kSubB][D]
    float* dOr = Qr + kSubB * D;                       // [kSubB][D]
    float* tau_s = dOr + kSubB * D;                    // [kSubB]
    float* delta_s = tau_s + kSubB;                    // [kSubB]
    const int tid = threadIdx.x;
    const int T = a.T, N = a.N;
    const int b = blockIdx.x;
    const int bh = blockIdx.y;
    const size_t head = (size_t)bh * N * D;
    const TIn* q = static_cast<const TIn*>(a.q) + head;
    const TIn* dout = static_cast<const TIn*>(a.dout) + head;
    const int j = b * kBlk + tid;
    const bool key_valid = j < N;
    const float gamma = a.gamma, cx = a.cx;

    load_rows_f32<TIn, D>(Ks, D + 1, static_cast<const TIn*>(a.k) + head, b * kBlk, kBlk, N, tid, 128);
    if (WHICH == 1)
        load_rows_f32<TIn, D>(Vs, D + 1, static_cast<const TIn*>(a.v) + head, b * kBlk, kBlk, N, tid, 128);
    const float* krow = Ks + tid * (D + 1);
    const float* vrow = Vs + tid * (D + 1);

    float acc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) acc[c] = 0.f;
    int nvis = 0;
    for (int t = a.causal ? b : 0; t < T; ++t) {
        if (!a.mask[((size_t)bh * T + t) * T + b]) continue;   // CTA-uniform
        ++nvis;
        for (int rs = 0; rs < kBlk / kSubB; ++rs) {
            const int i0 = t * kBlk + rs * kSubB;
            if (i0 >= N) break;
            __syncthreads();
            load_rows_f32<TIn, D>(Qr, D, q, i0, kSubB, N, tid, 128);
            load_rows_f32<TIn, D>(dOr, D, dout, i0, kSubB, N, tid, 128);
            if (tid < kSubB) {
                const int ii = i0 + tid;
                tau_s[tid] = ii < N ? a.tau[(size_t)bh * N + ii] : 0.f;
                delta_s[tid] = (WHICH == 1 && ii < N) ? a.delta[(size_t)bh * N + ii] : 0.f;
            }
            __syncthreads();
            float r[kSubB];
            dot_rows<D, kSubB>(r, krow, Qr);
            float dp[kSubB];
            if (WHICH == 1) dot_rows<D, kSubB>(dp, vrow, dOr);
#pragma unroll
            for (int ii = 0; ii < kSubB; ++ii) {
                const int irow = i0 + ii;
                const bool ok = key_valid && irow < N && (!a.causal || j <= irow);
                const float u = __fmaf_rn(cx, r[ii], -tau_s[ii]);
                float w;
                const float* src;
                if (WHICH == 0) { w = ok ? entmax_p<GM>(u, gamma) : 0.f; src = dOr + ii * D; }
                else { w = ok ? entmax_g<GM>(u, gamma) * (dp[ii] - delta_s[ii]) : 0.f; src = Qr + ii * D; }
#pragma unroll
                for (int c = 0; c < D; c += 4) {
                    const float4 sv = *reinterpret_cast<const float4*>(src + c);
                    acc[c] = fmaf(w, sv.x, acc[c]);
                    acc[c + 1] = fmaf(w, sv.y, acc[c + 1]);
                    acc[c + 2] = fmaf(w, sv.z, acc[c + 2]);
                    acc[c + 3] = fmaf(w, sv.w, acc[c + 3]);
                }
            }
        }
    }
    if (key_valid) {
        TIn* out = static_cast<TIn*>(WHICH == 0 ? a.dv : a.dk) + head + (size_t)j * D;
        const float sc = (WHICH == 0) ? 1.f : a.scale;
#pragma unroll
        for (int c = 0; c < D; ++c) store_f(out, c, acc[c] * sc);
    }
    // block GEMMs: dV needs S and P^T dO (2); dK needs S, dP and dS^T Q (3)
    if (tid == 0)
        atomicAdd(&a.hdr->counters[kCtrBwdBlocks], (unsigned long long)nvis * (WHICH == 0 ? 2 : 3));
}

// ------------------------------------------------------------------ launchers
template <typename TIn, int D, int GM>
cudaError_t simt_launch_fwd(const FwdArgs& a, cudaStream_t s) {
    const size_t sm = simt_fwd_smem<D>(a.T);
    auto kern = simt_fwd_kernel<TIn, D, GM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.T, a.BH), 128, sm, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn, int D, int GM>
cudaError_t simt_launch_bwd(const BwdArgs& a, cudaStream_t s) {
    {
        const size_t sm = simt_bwd_dq_smem<D>();
        auto kern = simt_bwd_dq_kernel<TIn, D, GM>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        kern<<<dim3(a.T, a.BH), 128, sm, s>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t sm = simt_bwd_dkv_smem<D>();
    auto kv = simt_bwd_dkv_kernel<TIn, D, GM, 0>;
    auto kk = simt_bwd_dkv_kernel<TIn, D, GM, 1>;
    cudaError_t e = cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kv<<<dim3(a.T, a.BH), 128, sm, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kk<<<dim3(a.T, a.BH), 128, sm, s>>>(a);
    return cudaGetLastError();
}

// gamma modes compiled for this path: exact 1 (alpha 2), 2 (alpha 1.5),
// 4 (alpha 1.25); everything else (including gamma 3) runs the general form.
template <typename TIn, int D>
cudaError_t simt_fwd_d(const FwdArgs& a, int gm, cudaStream_t s) {
    switch (gm) {
        case 1: return simt_launch_fwd<TIn, D, 1>(a, s);
        case 2: return simt_launch_fwd<TIn, D, 2>(a, s);
        case 4: return simt_launch_fwd<TIn, D, 4>(a, s);
        default: return simt_launch_fwd<TIn, D, 0>(a, s);
    }
}

template <typename TIn, int D>
cudaError_t simt_bwd_d(const BwdArgs& a, int gm, cudaStream_t s) {
    switch (gm) {
        case 1: return simt_launch_bwd<TIn, D, 1>(a, s);
        case 2: return simt_launch_bwd<TIn, D, 2>(a, s);
        case 4: return simt_launch_bwd<TIn, D, 4>(a, s);
        default: return simt_launch_bwd<TIn, D, 0>(a, s);
    }
}

}  // namespace ent
