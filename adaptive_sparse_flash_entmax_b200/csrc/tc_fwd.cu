// tc_fwd.cu -- the bf16 forward on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA per 128-row query tile ("AdaSplash: Adaptive Sparse Flash Attention",
// Technical Deep Dive / AdaSplash: Fused GPU Kernel for Attention: the Q tile is
// loaded once and stays on chip; K tiles stream for the tau passes; a final pass
// streams K and V and accumulates O = P V).  Warp roles:
//   warp 0   TMA producer: Q once, then K (and V in the P.V pass) blocks into a
//            two-stage ring;
//   warp 1   MMA issuer: S = Q K^T into a double-buffered TMEM accumulator
//            (128 x 128 fp32), and O += P V (P from shared memory, V MN-major);
//   warps 2-9 elementwise: two threads per query row (= TMEM lane), 64 columns
//            each.  Pass 0 builds the
//            row max and the sliding 64-bin histogram ("AdaSplash-2: ...",
//            Sparse Attention Makes Waves); solver passes accumulate
//            F0, F1, F2 and take a Halley-bisection step (Accelerated Alpha-Entmax
//            Transformation); the last solver pass marks live key blocks
//            (Exploiting Sparsity); the P.V pass writes P (bf16) for live blocks.
// After each score pass the elementwise group publishes a decision (another
// solver pass, or the P.V pass with its live-block list) that the producer and
// the MMA issuer wait on.  Every wait is bounded (2 s); a wait that gives up
// sets the workspace status and makes the whole CTA leave its loops, drain its
// in-flight copies and free its TMEM.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace ent {
using namespace tc;

namespace {

constexpr int kNst = 2;            // K/V ring stages
constexpr int kThreads = 320;      // 10 warps
constexpr int kEw = 256;           // elementwise threads (warps 2-9): two per query row
constexpr int kEwWarps = 8;
constexpr int kAtom = 128 * 128;   // bytes of a [128 rows x 64 bf16] swizzled atom
constexpr int kTmemCols = 512;     // S0 [0,128), S1 [128,256), O [256, 256+D)
constexpr int kDecSolve = 1, kDecPv = 2;

template <int D>
struct Layout {
    static constexpr int kTile = D / 64 * kAtom;          // [128 x D] bf16
    static constexpr int kQ = 0;
    static constexpr int kStage0 = kQ + kTile;
    static constexpr int kStageBytes = 2 * kTile;         // K, then V
    static constexpr int kP = kStage0 + kNst * kStageBytes;
    static constexpr int kPBytes = 2 * kAtom;             // P [128 x 128] bf16
    // Row histograms ([64 slots][128 rows] u32 per column half) live in memory that
    // is idle during the score passes: the V halves of the two stages when they
    // are 32 KB (D = 128), else P and a region of their own.
    static constexpr int kHist0 = (D == 128) ? kStage0 + kTile : kP;
    static constexpr int kHist1 = (D == 128) ? kStage0 + kStageBytes + kTile : kP + kPBytes;
    static constexpr int kXch = (D == 128) ? kP + kPBytes : kP + 2 * kPBytes;   // [4][2][128] f32
    static constexpr int kBars = kXch + 4 * 2 * 128 * 4;
    static constexpr int kNumBars = 16;
    static constexpr int kMisc = kBars + 8 * kNumBars;    // tmem base, decision, nlive, abort
    static constexpr int kPtab = kMisc + 16;              // 68 floats
    static constexpr int kLive = kPtab + 68 * 4;          // T bytes
    static size_t bytes(int T) { return (size_t)kLive + (size_t)((T + 15) / 16) * 16 + 4 * (size_t)T + 1024; }
};

struct Misc {
    uint32_t tmem_base;
    int decision;
    int nlive;
    int abort;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
}

}  // namespace

template <int D, int GM>
__global__ void __launch_bounds__(kThreads, 1)
tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* full = bars;                 // [kNst]  TMA -> MMA
    uint64_t* empty = bars + kNst;         // [kNst]  MMA -> TMA
    uint64_t* s_full = bars + 2 * kNst;    // [2]     MMA -> elementwise
    uint64_t* s_empty = s_full + 2;        // [2]     elementwise -> MMA
    uint64_t* p_full = s_empty + 2;        //         elementwise -> MMA
    uint64_t* p_empty = p_full + 1;        //         MMA -> elementwise
    uint64_t* o_full = p_empty + 1;        //         MMA -> elementwise
    uint64_t* q_full = o_full + 1;         //         TMA -> MMA
    uint64_t* dec_bar = q_full + 1;        //         elementwise -> TMA, MMA
    uint64_t* mma_done = dec_bar + 1;      //         MMA -> MMA (all issued MMAs retired)
    Misc* misc = reinterpret_cast<Misc*>(smem + L::kMisc);
    float* ptab = reinterpret_cast<float*>(smem + L::kPtab);
    uint8_t* live = smem + L::kLive;
    int* live_list = reinterpret_cast<int*>(smem + L::kLive + ((a.T + 15) / 16) * 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, N = a.N;
    const int t = a.causal ? (T - 1 - (int)blockIdx.x) : (int)blockIdx.x;   // long tiles first
    const int bh = blockIdx.y;
    const int nblk = a.causal ? t + 1 : T;
    const Abort ab{&misc->abort, a.hdr};

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&s_full[s], 1); mbar_init(&s_empty[s], kEwWarps); }
        mbar_init(p_full, kEwWarps);
        mbar_init(p_empty, 1);
        mbar_init(o_full, 1);
        mbar_init(q_full, 1);
        mbar_init(dec_bar, 1);
        mbar_init(mma_done, 1);
        misc->decision = 0;
        misc->nlive = 0;
        misc->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    for (int b = threadIdx.x; b < T; b += kThreads) live[b] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(q_full, L::kTile);
            for (int at = 0; at < D / 64; ++at)
                tma_load_3d(smem + L::kQ + at * kAtom, &tm_q, at * 64, t * kBlk, bh, q_full);
            int job = 0, kind = kDecSolve;
            uint32_t dec_phase = 0;
            bool ok = true;
            while (ok) {
                const bool pv = kind == kDecPv;
                const int njobs = pv ? misc->nlive : nblk;
                for (int i = 0; i < njobs && ok; ++i, ++job) {
                    const int b = pv ? live_list[i] : i;
                    const int st = job % kNst;
                    if (!(ok = mbar_wait(&empty[st], ((job / kNst) & 1) ^ 1, ab, 1))) break;
                    uint8_t* kb = smem + L::kStage0 + st * L::kStageBytes;
                    mbar_arrive_expect_tx(&full[st], pv ? 2 * L::kTile : L::kTile);
                    for (int at = 0; at < D / 64; ++at)
                        tma_load_3d(kb + at * kAtom, &tm_k, at * 64, b * kBlk, bh, &full[st]);
                    if (pv)
                        for (int at = 0; at < D / 64; ++at)
                            tma_load_3d(kb + L::kTile + at * kAtom, &tm_v, at * 64, b * kBlk, bh,
                                        &full[st]);
                }
                if (!ok || pv) break;
                if (!(ok = mbar_wait(dec_bar, dec_phase, ab, 2))) break;
                dec_phase ^= 1;
                kind = misc->decision;
            }
            // Copies issued but possibly not consumed land before the CTA ends.
            drain_wait(q_full, 0);
            for (int j = job - 1; j >= 0 && j >= job - kNst; --j)
                drain_wait(&full[j % kNst], (j / kNst) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, 0, 1);
            const uint32_t qb = smem_u32(smem + L::kQ);
            const uint32_t pb = smem_u32(smem + L::kP);
            bool ok = mbar_wait(q_full, 0, ab, 3);
            tc_fence_after();
            int job = 0, pvjob = 0, kind = kDecSolve;
            uint32_t dec_phase = 0;
            while (ok) {
                const bool pv = kind == kDecPv;
                const int njobs = pv ? misc->nlive : nblk;
                for (int i = 0; i < njobs && ok; ++i, ++job) {
                    const int st = job % kNst, sb = job & 1;
                    if (!(ok = mbar_wait(&full[st], (job / kNst) & 1, ab, 4))) break;
                    if (!(ok = mbar_wait(&s_empty[sb], ((job >> 1) & 1) ^ 1, ab, 5))) break;
                    tc_fence_after();
                    const uint32_t kb = smem_u32(smem + L::kStage0 + st * L::kStageBytes);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                        umma_bf16(tmem + sb * 128, sdesc_sw128(qb + off, 16, 1024),
                                  sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0);
                    }
                    umma_commit(&s_full[sb]);
                    if (!pv) {
                        umma_commit(&empty[st]);
                        continue;
                    }
                    if (!(ok = mbar_wait(p_full, pvjob & 1, ab, 6))) break;
                    tc_fence_after();
                    const uint32_t vb = kb + L::kTile;
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const uint32_t aoff = (kk >> 2) * kAtom + (kk & 3) * 32;
                        umma_bf16(tmem + 256, sdesc_sw128(pb + aoff, 16, 1024),
                                  sdesc_sw128(vb + kk * 16 * 128, kAtom, 1024), idesc_pv,
                                  (pvjob > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(p_empty);
                    umma_commit(&empty[st]);
                    ++pvjob;
                }
                if (!ok) break;
                if (pv) {
                    umma_commit(o_full);
                    break;
                }
                if (!(ok = mbar_wait(dec_bar, dec_phase, ab, 7))) break;
                dec_phase ^= 1;
                kind = misc->decision;
            }
            // every issued MMA retires before TMEM is freed
            umma_commit(mma_done);
            drain_wait(mma_done, 0);
        }
    } else {
        // ------------------------------------------------------------ elementwise
        // Two threads per query row: `half` selects columns [64*half, 64*half + 64)
        // of every 128-key block.  Row state (tau, bracket) is kept identically in
        // both; per-pass partial sums are combined through shared memory.
        const int ew = threadIdx.x - 64;          // 0..255
        const int half = ew >> 7;
        const int quarter = warp & 3;             // TMEM lane quarter of this warp
        const int row = quarter * 32 + lane;      // tile row == TMEM lane
        const int c0 = half * 64;                 // first column of this thread
        const int i = t * kBlk + row;
        const bool row_valid = i < N;
        const int key_end = !row_valid ? 0 : (a.causal ? i + 1 : N);
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float gamma = a.gamma, cx = a.cx;
        unsigned int* hist = reinterpret_cast<unsigned int*>(smem + (half ? L::kHist1 : L::kHist0)) + row;
        float* xch = reinterpret_cast<float*>(smem + L::kXch);   // [k][half][row]
        auto X = [&](int k, int h) -> float& { return xch[(k * 2 + h) * 128 + row]; };
        if (ew < 65) ptab[ew] = entmax_p<GM>((float)ew / kBinsPerUnit, gamma);
        for (int sl = 0; sl < kBins; ++sl) hist[sl * 128] = 0u;
        named_bar(1, kEw);

        float m = -INFINITY;
        int A = kNoBin;
        RowSolver sv;
        sv.tau = 0.f; sv.lo = 0.f; sv.hi = 0.f;
        sv.done = row_valid ? 0 : 1;
        sv.iters = 0;
        int job = 0, pass = 0, nlive = 0;
        bool ok = true;
        for (;; ++pass) {
            float F0 = 0.f, F1 = 0.f, F2 = 0.f;
            if (pass > 0) {
                for (int bb = ew; bb < nblk; bb += kEw) live[bb] = 0;
                named_bar(1, kEw);
            }
            for (int b = 0; b < nblk; ++b, ++job) {
                const int sb = job & 1;
                if (!(ok = mbar_wait(&s_full[sb], (job >> 1) & 1, ab, 8))) break;
                tc_fence_after();
                float s[64];
                tmem_ld32(lane_base + sb * 128 + c0, &s[0]);
                tmem_ld32(lane_base + sb * 128 + c0 + 32, &s[32]);
                tmem_wait_ld();
                reg_fence<64>(s);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[sb]);
                const int nv = key_end - b * kBlk - c0;   // valid columns of this thread: c < nv
                const bool full_blk = __all_sync(0xffffffffu, nv >= 64);
                if (!full_blk) {
#pragma unroll
                    for (int c = 0; c < 64; ++c) s[c] = (c < nv) ? s[c] : -INFINITY;
                }
                if (pass == 0) {
                    float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
                    for (int c = 4; c < 64; c += 4) {
                        m0 = fmaxf(m0, s[c]); m1 = fmaxf(m1, s[c + 1]);
                        m2 = fmaxf(m2, s[c + 2]); m3 = fmaxf(m3, s[c + 3]);
                    }
                    const float xm = __fmul_rn(cx, fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)));
                    if (xm > m) {
                        m = xm;
                        const int An = abs_bin(m);
                        hist_slide(hist, 128, A, An);
                        A = An;
                    }
                    // candidates: x >= (A-63)/63 (an exact integer test follows)
                    const float thr = (float)(A - (kBins - 1)) / kBinsPerUnit - 1e-3f;
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        const float x = __fmul_rn(cx, s[c]);
                        if (x >= thr) {
                            const int ab2 = abs_bin(x);
                            if (ab2 >= A - (kBins - 1)) hist[(ab2 & (kBins - 1)) * 128] += 1u;
                        }
                    }
                } else {
                    float f0a = 0.f, f0b = 0.f, f1a = 0.f, f1b = 0.f, f2a = 0.f, f2b = 0.f;
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        float t0, t1, t2, q0, q1, q2;
                        entmax_terms_bf<GM>(__fmaf_rn(cx, s[c], -sv.tau), gamma, t0, t1, t2);
                        entmax_terms_bf<GM>(__fmaf_rn(cx, s[c + 1], -sv.tau), gamma, q0, q1, q2);
                        f0a += t0; f1a += t1; f2a += t2;
                        f0b += q0; f1b += q1; f2b += q2;
                    }
                    const float f1 = f1a + f1b;
                    F0 += f0a + f0b; F1 += f1; F2 += f2a + f2b;
                    // liveness: t1 = u^(gamma-1) > 0 exactly where u > 0 (up to underflow,
                    // where p = u^gamma is 0 as well)
                    if (__any_sync(0xffffffffu, f1 > 0.f) && lane == 0) live[b] = 1;
                }
            }
            if (!ok) break;
            if (pass == 0) {
                // merge the two half-row histograms; the half-0 thread computes the start
                X(3, half) = m;
                named_bar(1, kEw);
                const float m_other = X(3, half ^ 1);
                if (half == 0 && row_valid) {
                    const int A0 = A;
                    const int A1 = (m_other == -INFINITY) ? kNoBin : abs_bin(m_other);
                    const unsigned int* h0 = hist;
                    const unsigned int* h1 = reinterpret_cast<const unsigned int*>(smem + L::kHist1) + row;
                    const float mr = fmaxf(m, m_other);
                    const int Ar = abs_bin(mr);
                    auto count = [&](int ab2) -> unsigned int {
                        unsigned int c = 0;
                        if (ab2 <= A0 && ab2 >= A0 - (kBins - 1)) c += h0[(ab2 & (kBins - 1)) * 128];
                        if (ab2 <= A1 && ab2 >= A1 - (kBins - 1)) c += h1[(ab2 & (kBins - 1)) * 128];
                        return c;
                    };
                    hist_start_fn<GM>(count, Ar, mr, key_end, a.alpha, gamma, ptab, sv.lo, sv.hi, sv.tau);
                    X(0, 0) = sv.lo; X(1, 0) = sv.hi; X(2, 0) = sv.tau;
                }
                named_bar(1, kEw);
                if (half == 1 && row_valid) { sv.lo = X(0, 0); sv.hi = X(1, 0); sv.tau = X(2, 0); }
            } else {
                X(0, half) = F0; X(1, half) = F1; X(2, half) = F2;
                named_bar(1, kEw);
                const float G0 = F0 + X(0, half ^ 1), G1 = F1 + X(1, half ^ 1), G2 = F2 + X(2, half ^ 1);
                solver_update(sv, G0, G1, G2, gamma, gamma == 1.f, pass, a.ftol, a.stol);
            }
            const int all = named_bar_and(1, kEw, sv.done) && pass > 0;
            if (ew == 0) {
                if (all) {
                    int n = 0;
                    for (int bb = 0; bb < nblk; ++bb)
                        if (live[bb]) live_list[n++] = bb;
                    misc->nlive = n;
                }
                misc->decision = all ? kDecPv : kDecSolve;
                mbar_arrive(dec_bar);
            }
            if (all) break;
        }
        const int npass = pass;
        if (ok) {
            named_bar(1, kEw);   // live_list / nlive visible to the group
            nlive = misc->nlive;
            int pvjob = 0;
            for (int li = 0; li < nlive; ++li, ++job, ++pvjob) {
                const int b = live_list[li];
                const int sb = job & 1;
                if (!(ok = mbar_wait(&s_full[sb], (job >> 1) & 1, ab, 9))) break;
                tc_fence_after();
                float s[64];
                tmem_ld32(lane_base + sb * 128 + c0, &s[0]);
                tmem_ld32(lane_base + sb * 128 + c0 + 32, &s[32]);
                tmem_wait_ld();
                reg_fence<64>(s);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[sb]);
                const int nv = key_end - b * kBlk - c0;
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float u0 = (c < nv) ? __fmaf_rn(cx, s[c], -sv.tau) : -1.f;
                    const float u1 = (c + 1 < nv) ? __fmaf_rn(cx, s[c + 1], -sv.tau) : -1.f;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(entmax_p_bf<GM>(u0, gamma),
                                                                    entmax_p_bf<GM>(u1, gamma));
                    pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                if (!(ok = mbar_wait(p_empty, (pvjob & 1) ^ 1, ab, 10))) break;
                uint8_t* prow = smem + L::kP + half * kAtom + row * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)   // 16-byte chunk = 8 keys
                    *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) =
                        make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
            }
        }
        // epilogue: this thread's half of the O row, tau, iters, mask row, counters
        constexpr int DH = D / 2;
        float o[DH];
        if (ok && nlive > 0) {
            ok = mbar_wait(o_full, 0, ab, 11);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < DH / 32; ++c)
                tmem_ld32(lane_base + 256 + half * DH + c * 32, &o[c * 32]);
            tmem_wait_ld();
            reg_fence<DH>(o);
        } else {
#pragma unroll
            for (int c = 0; c < DH; ++c) o[c] = 0.f;
        }
        if (row_valid) {
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + ((size_t)bh * N + i) * D + half * DH;
#pragma unroll
            for (int c = 0; c < DH; c += 8) {
                uint4 val;
                __nv_bfloat162 h;
                h = __floats2bfloat162_rn(o[c], o[c + 1]); val.x = *reinterpret_cast<uint32_t*>(&h);
                h = __floats2bfloat162_rn(o[c + 2], o[c + 3]); val.y = *reinterpret_cast<uint32_t*>(&h);
                h = __floats2bfloat162_rn(o[c + 4], o[c + 5]); val.z = *reinterpret_cast<uint32_t*>(&h);
                h = __floats2bfloat162_rn(o[c + 6], o[c + 7]); val.w = *reinterpret_cast<uint32_t*>(&h);
                *reinterpret_cast<uint4*>(orow + c) = val;
            }
            if (half == 0) {
                a.tau[(size_t)bh * N + i] = sv.tau;
                if (a.iters) a.iters[(size_t)bh * N + i] = (uint8_t)sv.iters;
            }
        }
        uint8_t* mrow = a.mask + ((size_t)bh * T + t) * T;
        for (int bb = ew; bb < T; bb += kEw) mrow[bb] = (bb < nblk) ? live[bb] : 0;
        if (ew == 0) {
            atomicAdd(&a.hdr->counters[kCtrQkBlocks], (unsigned long long)nblk * (npass + 1));
            atomicAdd(&a.hdr->counters[kCtrPvBlocks], (unsigned long long)nlive);
            atomicAdd(&a.hdr->counters[kCtrPasses], (unsigned long long)npass);
            atomicAdd(&a.hdr->counters[kCtrTiles], 1ull);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

// [BH][N][D] bf16 tensor, box {64, box_rows, 1}, 128-byte swizzle, zero fill out of bounds.
bool make_tmap_bf16_rows(CUtensorMap* map, const void* base, int BH, int N, int D, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, int BH, int N, int D) {
    return make_tmap_bf16_rows(map, base, BH, N, D, 128);
}

template <int D, int GM>
static cudaError_t launch_tc_fwd(const CUtensorMap& mq, const CUtensorMap& mk,
                                 const CUtensorMap& mv, const FwdArgs& a, cudaStream_t s) {
    const size_t sm = Layout<D>::bytes(a.T);
    auto kern = tc_fwd_kernel<D, GM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.T, a.BH), kThreads, sm, s>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t tc_fwd_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const FwdArgs& a, int gm, cudaStream_t s) {
    switch (gm) {
        case 1: return launch_tc_fwd<D, 1>(mq, mk, mv, a, s);
        case 2: return launch_tc_fwd<D, 2>(mq, mk, mv, a, s);
        case 4: return launch_tc_fwd<D, 4>(mq, mk, mv, a, s);
        default: return launch_tc_fwd<D, 0>(mq, mk, mv, a, s);
    }
}

cudaError_t tc_fwd(const FwdArgs& a, int d, int gm, cudaStream_t s, const char** why) {
    CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16(&mq, a.q, a.BH, a.N, d) || !make_tmap_bf16(&mk, a.k, a.BH, a.N, d) ||
        !make_tmap_bf16(&mv, a.v, a.BH, a.N, d)) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    return d == 64 ? tc_fwd_d<64>(mq, mk, mv, a, gm, s) : tc_fwd_d<128>(mq, mk, mv, a, gm, s);
}

}  // namespace ent
