// tc_bwd.cu -- the bf16 backward on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Entmax Jacobian (derived from the definition; the pages state that the
// backward skips the zero tiles, "AdaSplash: Adaptive Sparse Flash Attention",
// Experimental Setup & Results / Backward Pass, and Technical Deep Dive /
// Exploiting Sparsity): with u = x - tau, g = u^(gamma-1) on u > 0,
//     delta_i = sum_j g_ij dP_ij / sum_j g_ij,   dS = g (dP - delta),   dP = dO V^T,
//     dQ = dS K / sqrt(d),   dK = dS^T Q / sqrt(d),   dV = P^T dO.
// Only the 128 x 128 blocks marked live by the forward's block mask are visited.
//
// Two kernels, both with warp roles (warp 0 TMA, warp 1 MMA issuer, warps 2-9
// elementwise, two threads per TMEM lane) and 64-wide sub-tiles so that three
// stages and several TMEM accumulator pairs fit on chip.  The bf16 operand the
// elementwise warps produce (dS, P^T, dS^T) is written into TMEM over the S
// columns it came from, and the MMA reads it from there as its A operand:
//   dq kernel   one CTA per 128-row query tile, K/V in 64-key sub-blocks of
//               the live blocks.  Phase A: S = Q K^T, dP = dO V^T -> delta per
//               row (also written to the workspace).  Phase B: again S and dP,
//               dS as a pair of bf16 parts (hi + lo) and dQ += dS K (K read
//               MN-major).
//   dkv kernel  one CTA per 128-key block, Q/dO in 64-row sub-tiles of the
//               live query tiles.  S^T = K Q^T, dP^T = V dO^T, then P^T and
//               dS^T (bf16) and dV += P^T dO, dK += dS^T Q (dO and Q read
//               MN-major from the same tiles that fed S^T and dP^T).
// All waits are bounded as in the forward.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "tc_common.cuh"

namespace ent {
using namespace tc;

bool make_tmap_bf16_rows(CUtensorMap* map, const void* base, int BH, int N, int D, int box_rows);

namespace {

constexpr int kThreads = 320;                  // warp 0 TMA, warp 1 MMA, warps 2-9 elementwise
constexpr int kEw = 256;                       // two threads per TMEM lane, 32 columns each
constexpr int kEwWarps = 8;
constexpr int kNst = 3;                        // K/V (dq) or Q/dO (dkv) sub-tile stages
constexpr int kTmemCols = 512;
constexpr int kSub = 64;                       // sub-tile width (keys or query rows)
constexpr int kAtom128 = 128 * 128;            // [128 rows x 64 bf16] atom
constexpr int kAtom64 = 64 * 128;              // [64 rows x 64 bf16] atom
constexpr int kSbufDq = 3;                     // S/dP accumulator pairs of the dq kernel
// TMEM column of S/dP pair `sb` in the dq kernel (dQ lives at columns 256..383)
__host__ __device__ constexpr uint32_t dq_sbuf_col(int sb) { return sb < 2 ? sb * 128 : 384; }

struct Misc {
    uint32_t tmem_base;
    int njobs;      // sub-tile jobs per phase
    int abort;
    int pad;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void store_out_row(void* out, size_t off, const float* v, int D, float sc) {
    __nv_bfloat16* p = static_cast<__nv_bfloat16*>(out) + off;
    for (int c = 0; c < D; c += 8) {
        uint4 val = make_uint4(pack_bf16(v[c] * sc, v[c + 1] * sc), pack_bf16(v[c + 2] * sc, v[c + 3] * sc),
                               pack_bf16(v[c + 4] * sc, v[c + 5] * sc), pack_bf16(v[c + 6] * sc, v[c + 7] * sc));
        *reinterpret_cast<uint4*>(p + c) = val;
    }
}

}  // namespace

// =========================================================================
// dq kernel: delta and dQ for one 128-row query tile.
// =========================================================================
template <int D>
struct DqLayout {
    static constexpr int kTile = D / 64 * kAtom128;     // Q or dO [128 x D]
    static constexpr int kSubT = D / 64 * kAtom64;      // K or V sub-block [64 x D]
    static constexpr int kQ = 0;
    static constexpr int kDO = kQ + kTile;
    static constexpr int kStage0 = kDO + kTile;
    static constexpr int kStageBytes = 2 * kSubT;       // K_sub, V_sub
    static constexpr int kXch = kStage0 + kNst * kStageBytes;  // [2][2][128] f32
    static constexpr int kBars = kXch + 2 * 2 * 128 * 4;
    static constexpr int kMisc = kBars + 8 * 24;   // up to 24 mbarriers
    static constexpr int kList = kMisc + 16;            // int job list [2*T]
    static size_t bytes(int T) { return (size_t)kList + 8 * (size_t)T + 1024; }
};

template <int D, int GM>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_k64, const __grid_constant__ CUtensorMap tm_v64,
                 const BwdArgs a) {
    using L = DqLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* full = bars;                     // [kNst]
    uint64_t* empty = full + kNst;             // [kNst]
    uint64_t* s_full = empty + kNst;           // [kSbufDq]  MMA -> elementwise
    uint64_t* s_empty = s_full + kSbufDq;      // [kSbufDq]  elementwise -> MMA (phase A jobs)
    uint64_t* ds_full = s_empty + kSbufDq;     // [kSbufDq]  elementwise -> MMA (dS in TMEM)
    uint64_t* ds_free = ds_full + kSbufDq;     // [kSbufDq]  MMA -> MMA (dQ of a phase B job done)
    uint64_t* acc_full = ds_free + kSbufDq;
    uint64_t* in_full = acc_full + 1;          // Q and dO tiles
    uint64_t* mma_done = in_full + 1;
    Misc* misc = reinterpret_cast<Misc*>(smem + L::kMisc);
    int* jobs = reinterpret_cast<int*>(smem + L::kList);   // key offsets of the 64-key sub-blocks

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, N = a.N;
    const int t = a.causal ? (T - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int bh = blockIdx.y;
    const int nblk = a.causal ? t + 1 : T;
    const int last_row = min(t * kBlk + kBlk - 1, N - 1);
    const Abort ab{&misc->abort, a.hdr};

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < kSbufDq; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], kEwWarps);
            mbar_init(&ds_full[s], kEwWarps);
            mbar_init(&ds_free[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(in_full, 1);
        mbar_init(mma_done, 1);
        misc->abort = 0;
        // sub-block list of the live key blocks of this tile
        const uint8_t* mrow = a.mask + ((size_t)bh * T + t) * T;
        int n = 0;
        for (int b = 0; b < nblk; ++b) {
            if (!mrow[b]) continue;
            for (int h = 0; h < 2; ++h) {
                const int j0 = b * kBlk + h * kSub;
                if (j0 >= N || (a.causal && j0 > last_row)) continue;
                jobs[n++] = j0;
            }
        }
        misc->njobs = n;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int njobs = misc->njobs;
    const int total = 2 * njobs;     // phase A then phase B

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_q); prefetch_tmap(&tm_do); prefetch_tmap(&tm_k64); prefetch_tmap(&tm_v64);
            mbar_arrive_expect_tx(in_full, 2 * L::kTile);
            for (int at = 0; at < D / 64; ++at) {
                tma_load_3d(smem + L::kQ + at * kAtom128, &tm_q, at * 64, t * kBlk, bh, in_full);
                tma_load_3d(smem + L::kDO + at * kAtom128, &tm_do, at * 64, t * kBlk, bh, in_full);
            }
            int job = 0;
            bool ok = true;
            for (; job < total && ok; ++job) {
                const int j0 = jobs[job % njobs];
                const int st = job % kNst;
                if (!(ok = mbar_wait(&empty[st], ((job / kNst) & 1) ^ 1, ab, 21))) break;
                uint8_t* sb = smem + L::kStage0 + st * L::kStageBytes;
                mbar_arrive_expect_tx(&full[st], 2 * L::kSubT);
                for (int at = 0; at < D / 64; ++at) {
                    tma_load_3d(sb + at * kAtom64, &tm_k64, at * 64, j0, bh, &full[st]);
                    tma_load_3d(sb + L::kSubT + at * kAtom64, &tm_v64, at * 64, j0, bh, &full[st]);
                }
            }
            drain_wait(in_full, 0);
            for (int j = job - 1; j >= 0 && j >= job - kNst; --j) drain_wait(&full[j % kNst], (j / kNst) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(128, kSub, 0, 0);   // [128 x 64], K = d
            constexpr uint32_t idesc_dq = idesc_bf16(128, D, 0, 1);     // dQ += dS K, K MN-major
            // base descriptors; operands differ only by start-address offsets
            const uint64_t dq_ = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
            const uint64_t ddo = sdesc_sw128(smem_u32(smem + L::kDO), 16, 1024);
            const uint64_t dst = sdesc_sw128(smem_u32(smem + L::kStage0), 16, 1024);
            const uint64_t dst_mn = sdesc_sw128(smem_u32(smem + L::kStage0), kAtom64, 1024);
            bool ok = mbar_wait(in_full, 0, ab, 22);
            tc_fence_after();
            // issue S and dP of job j into TMEM pair j % kSbufDq.  The pair is free once
            // the previous job on it is done with it: a phase A job when the elementwise
            // warps have read S and dP, a phase B job when the dQ MMA has read its dS.
            auto issue_sdp = [&](int j) -> bool {
                const int st = j % kNst, sbuf = j % kSbufDq;
                if (!mbar_wait(&full[st], (j / kNst) & 1, ab, 23)) return false;
                const int jp = j - kSbufDq;
                const bool fr = (jp < njobs)
                                    ? mbar_wait(&s_empty[sbuf], ((j / kSbufDq) & 1) ^ 1, ab, 24)
                                    : mbar_wait(&ds_free[sbuf], ((jp - njobs) / kSbufDq) & 1, ab, 24);
                if (!fr) return false;
                tc_fence_after();
                const uint64_t dk = dst + ((st * L::kStageBytes) >> 4);
                const uint64_t dv = dk + (L::kSubT >> 4);
                const uint32_t dS = tmem + dq_sbuf_col(sbuf), dPc = dS + 64;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = ((kk >> 2) * kAtom128 + (kk & 3) * 32) >> 4;
                    const uint32_t ob = ((kk >> 2) * kAtom64 + (kk & 3) * 32) >> 4;
                    umma_bf16(dS, dq_ + oa, dk + ob, idesc_s, kk > 0);
                    umma_bf16(dPc, ddo + oa, dv + ob, idesc_s, kk > 0);
                }
                umma_commit(&s_full[sbuf]);
                return true;
            };
            if (ok && total > 0) ok = issue_sdp(0);
            for (int j = 0; j < total && ok; ++j) {
                if (j + 1 < total && !(ok = issue_sdp(j + 1))) break;
                const int st = j % kNst;
                if (j < njobs) {                 // phase A: K/V stage only fed S and dP
                    umma_commit(&empty[st]);
                    continue;
                }
                const int bj = j - njobs;        // phase B job: dQ += dS K
                const int sbuf = j % kSbufDq;
                // one ds_full per pair: dS(j+3) cannot complete before dQ(j) frees the pair
                if (!(ok = mbar_wait(&ds_full[sbuf], (bj / kSbufDq) & 1, ab, 25))) break;
                tc_fence_after();
                const uint64_t dkmn = dst_mn + ((st * L::kStageBytes) >> 4);
                // dQ += (dS_hi + dS_lo) K: the two bf16 parts carry dS to ~16 bits, which
                // the cancellation in sum_j dS_ij k_j (rows of dS sum to 0) needs.  The
                // half (kk >> 1) that owns keys 16kk .. 16kk+15 wrote their dS_hi into its
                // first 16 S columns and dS_lo into the next 16, two keys per column.
#pragma unroll
                for (int kk = 0; kk < kSub / 16; ++kk) {
                    const uint64_t bdesc = dkmn + ((kk * 16 * 128) >> 4);
                    const uint32_t hcol = tmem + dq_sbuf_col(sbuf) + 32 * (kk >> 1) + 8 * (kk & 1);
                    umma_bf16_ts(tmem + 256, hcol, bdesc, idesc_dq, (bj > 0 || kk > 0) ? 1u : 0u);
                    umma_bf16_ts(tmem + 256, hcol + 16, bdesc, idesc_dq, 1u);
                }
                umma_commit(&ds_free[sbuf]);
                umma_commit(&empty[st]);
            }
            if (ok) umma_commit(acc_full);
            umma_commit(mma_done);
            drain_wait(mma_done, 0);
        }
    } else {
        // two threads per query row: `half` takes columns [32*half, 32*half + 32)
        // of each 64-key sub-block; delta's partial sums meet in shared memory
        const int ew = threadIdx.x - 64;
        const int half = ew >> 7;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int i = t * kBlk + row;
        const bool row_valid = i < N;
        const int key_end = !row_valid ? 0 : (a.causal ? i + 1 : N);
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + half * 32;
        const float gamma = a.gamma, cx = a.cx;
        const float tau = row_valid ? a.tau[(size_t)bh * N + i] : 0.f;
        float* xch = reinterpret_cast<float*>(smem + L::kXch);   // [2][2][128]
        float sg = 0.f, sgdp = 0.f, delta = 0.f;
        const float2 cx2 = make_float2(cx, cx), nt2 = make_float2(-tau, -tau);
        bool ok = true;
        for (int j = 0; j < total && ok; ++j) {
            const int sbuf = j % kSbufDq;
            if (!(ok = mbar_wait(&s_full[sbuf], (j / kSbufDq) & 1, ab, 26))) break;
            tc_fence_after();
            float s[32], dp[32];
            tmem_ld32(lane_base + dq_sbuf_col(sbuf), &s[0]);
            tmem_ld32(lane_base + dq_sbuf_col(sbuf) + 64, &dp[0]);
            tmem_wait_ld();
            reg_fence<32>(s);
            reg_fence<32>(dp);
            if (j < njobs) {   // phase A: the pair is free again (phase B overwrites S with dS)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[sbuf]);
            }
            const int nv = key_end - jobs[j < njobs ? j : j - njobs] - half * 32;
            if (!__all_sync(0xffffffffu, nv >= 32)) {   // diagonal or ragged sub-block
#pragma unroll
                for (int c = 0; c < 32; ++c) s[c] = (c < nv) ? s[c] : -INFINITY;
            }
            if (j < njobs) {
                float2 a0 = make_float2(0.f, 0.f), b0 = a0, a1 = a0, b1 = a0;
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float2 g0 = entmax_g_x2<GM>(__ffma2_rn(make_float2(s[c], s[c + 1]), cx2, nt2), gamma);
                    const float2 g1 = entmax_g_x2<GM>(__ffma2_rn(make_float2(s[c + 2], s[c + 3]), cx2, nt2), gamma);
                    a0 = __fadd2_rn(a0, g0); b0 = __ffma2_rn(g0, make_float2(dp[c], dp[c + 1]), b0);
                    a1 = __fadd2_rn(a1, g1); b1 = __ffma2_rn(g1, make_float2(dp[c + 2], dp[c + 3]), b1);
                }
                a0 = __fadd2_rn(a0, a1); b0 = __fadd2_rn(b0, b1);
                sg += a0.x + a0.y;
                sgdp += b0.x + b0.y;
                if (j == njobs - 1) {
                    xch[(0 * 2 + half) * 128 + row] = sg;
                    xch[(1 * 2 + half) * 128 + row] = sgdp;
                    named_bar(1, kEw);
                    const float SG = sg + xch[(0 * 2 + (half ^ 1)) * 128 + row];
                    const float SGDP = sgdp + xch[(1 * 2 + (half ^ 1)) * 128 + row];
                    delta = (SG > 0.f) ? SGDP / SG : 0.f;
                    if (row_valid && half == 0) a.delta[(size_t)bh * N + i] = delta;
                }
            } else {
                uint32_t whi[16], wlo[16];
                const float2 nd2 = make_float2(-delta, -delta), m1 = make_float2(-1.f, -1.f);
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 g = entmax_g_x2<GM>(__ffma2_rn(make_float2(s[c], s[c + 1]), cx2, nt2), gamma);
                    const float2 d = __fmul2_rn(g, __fadd2_rn(make_float2(dp[c], dp[c + 1]), nd2));
                    const __nv_bfloat162 h = __floats2bfloat162_rn(d.x, d.y);
                    const float2 lo = __ffma2_rn(__bfloat1622float2(h), m1, d);   // d - bf16(d), exact
                    whi[c >> 1] = *reinterpret_cast<const uint32_t*>(&h);
                    wlo[c >> 1] = pack_bf16(lo.x, lo.y);
                }
                // dS over this thread's own S columns: hi in the first 16, lo in the next 16
                tmem_st16(lane_base + dq_sbuf_col(sbuf), whi);
                tmem_st16(lane_base + dq_sbuf_col(sbuf) + 16, wlo);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ds_full[sbuf]);
            }
        }
        if (njobs == 0 && row_valid && half == 0) a.delta[(size_t)bh * N + i] = 0.f;
        constexpr int DH = D / 2;
        float acc[DH];
        if (ok && njobs > 0) {
            ok = mbar_wait(acc_full, 0, ab, 28);
            tc_fence_after();
            const uint32_t ob = tmem + ((uint32_t)(quarter * 32) << 16) + 256 + half * DH;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) tmem_ld32(ob + c * 32, &acc[c * 32]);
            tmem_wait_ld();
            reg_fence<DH>(acc);
        } else {
#pragma unroll
            for (int c = 0; c < DH; ++c) acc[c] = 0.f;
        }
        if (row_valid) store_out_row(a.dq, ((size_t)bh * N + i) * D + half * DH, acc, DH, a.scale);
        if (threadIdx.x == 64)   // block products: phase A S,dP (2) + phase B S,dP,dQ hi,lo (4), per 64-key half
            atomicAdd(&a.hdr->counters[kCtrBwdBlocks], (unsigned long long)(3 * njobs));
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// =========================================================================
// dkv kernel: dK and dV for one 128-key block.
// =========================================================================
template <int D>
struct DkvLayout {
    static constexpr int kTile = D / 64 * kAtom128;     // K or V block [128 x D]
    static constexpr int kSubT = D / 64 * kAtom64;      // Q or dO sub-tile [64 x D]
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTile;
    static constexpr int kStage0 = kV + kTile;
    static constexpr int kStageBytes = 2 * kSubT;       // Q_sub, dO_sub
    static constexpr int kTauDelta = kStage0 + kNst * kStageBytes;   // [2][2][64] floats
    static constexpr int kBars = kTauDelta + 4 * 64 * 4;
    static constexpr int kMisc = kBars + 8 * 24;   // up to 24 mbarriers
    static constexpr int kList = kMisc + 16;
    static size_t bytes(int T) { return (size_t)kList + 8 * (size_t)T + 1024; }
};

template <int D, int GM>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_do64,
                  const BwdArgs a) {
    using L = DkvLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* full = bars;                     // [kNst]
    uint64_t* empty = full + kNst;             // [kNst]
    uint64_t* s_full = empty + kNst;           // [2]  MMA -> elementwise
    uint64_t* s_free = s_full + 2;             // [2]  MMA -> MMA (dV, dK of the pair's job done)
    uint64_t* p_full = s_free + 2;             // [2]  elementwise -> MMA (P^T, dS^T in TMEM)
    uint64_t* acc_full = p_full + 2;
    uint64_t* in_full = acc_full + 1;
    uint64_t* mma_done = in_full + 1;
    Misc* misc = reinterpret_cast<Misc*>(smem + L::kMisc);
    int* jobs = reinterpret_cast<int*>(smem + L::kList);   // row offsets of the 64-row sub-tiles
    float* td = reinterpret_cast<float*>(smem + L::kTauDelta);   // [buf][tau|delta][64]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, N = a.N;
    const int b = blockIdx.x;
    const int bh = blockIdx.y;
    const Abort ab{&misc->abort, a.hdr};

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 1);
            mbar_init(&p_full[s], kEwWarps);
        }
        mbar_init(acc_full, 1);
        mbar_init(in_full, 1);
        mbar_init(mma_done, 1);
        misc->abort = 0;
        int n = 0;
        for (int t = a.causal ? b : 0; t < T; ++t) {
            if (!a.mask[((size_t)bh * T + t) * T + b]) continue;
            for (int h = 0; h < 2; ++h) {
                const int i0 = t * kBlk + h * kSub;
                if (i0 >= N || (a.causal && i0 + kSub - 1 < b * kBlk)) continue;
                jobs[n++] = i0;
            }
        }
        misc->njobs = n;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int njobs = misc->njobs;
    const uint32_t tm_dv = tmem + 256, tm_dk = tmem + 256 + D;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_q64); prefetch_tmap(&tm_do64);
            mbar_arrive_expect_tx(in_full, 2 * L::kTile);
            for (int at = 0; at < D / 64; ++at) {
                tma_load_3d(smem + L::kK + at * kAtom128, &tm_k, at * 64, b * kBlk, bh, in_full);
                tma_load_3d(smem + L::kV + at * kAtom128, &tm_v, at * 64, b * kBlk, bh, in_full);
            }
            int job = 0;
            bool ok = true;
            for (; job < njobs && ok; ++job) {
                const int i0 = jobs[job];
                const int st = job % kNst;
                if (!(ok = mbar_wait(&empty[st], ((job / kNst) & 1) ^ 1, ab, 31))) break;
                uint8_t* sb = smem + L::kStage0 + st * L::kStageBytes;
                mbar_arrive_expect_tx(&full[st], 2 * L::kSubT);
                for (int at = 0; at < D / 64; ++at) {
                    tma_load_3d(sb + at * kAtom64, &tm_q64, at * 64, i0, bh, &full[st]);
                    tma_load_3d(sb + L::kSubT + at * kAtom64, &tm_do64, at * 64, i0, bh, &full[st]);
                }
            }
            drain_wait(in_full, 0);
            for (int j = job - 1; j >= 0 && j >= job - kNst; --j) drain_wait(&full[j % kNst], (j / kNst) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(128, kSub, 0, 0);   // S^T, dP^T [128 keys x 64]
            constexpr uint32_t idesc_acc = idesc_bf16(128, D, 0, 1);    // dV, dK: B (dO, Q) MN-major
            const uint64_t dkk = sdesc_sw128(smem_u32(smem + L::kK), 16, 1024);
            const uint64_t dvv = sdesc_sw128(smem_u32(smem + L::kV), 16, 1024);
            const uint64_t dst = sdesc_sw128(smem_u32(smem + L::kStage0), 16, 1024);
            const uint64_t dst_mn = sdesc_sw128(smem_u32(smem + L::kStage0), kAtom64, 1024);
            bool ok = mbar_wait(in_full, 0, ab, 32);
            tc_fence_after();
            auto issue_sdp = [&](int j) -> bool {
                const int st = j % kNst, sbuf = j & 1;
                if (!mbar_wait(&full[st], (j / kNst) & 1, ab, 33)) return false;
                // the pair holds P^T, dS^T of job j-2 until its dV, dK MMAs are done
                if (!mbar_wait(&s_free[sbuf], ((j >> 1) & 1) ^ 1, ab, 34)) return false;
                tc_fence_after();
                const uint64_t dqs = dst + ((st * L::kStageBytes) >> 4);
                const uint64_t dos = dqs + (L::kSubT >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = ((kk >> 2) * kAtom128 + (kk & 3) * 32) >> 4;
                    const uint32_t ob = ((kk >> 2) * kAtom64 + (kk & 3) * 32) >> 4;
                    umma_bf16(tmem + sbuf * 128, dkk + oa, dqs + ob, idesc_s, kk > 0);
                    umma_bf16(tmem + sbuf * 128 + 64, dvv + oa, dos + ob, idesc_s, kk > 0);
                }
                umma_commit(&s_full[sbuf]);
                return true;
            };
            if (ok && njobs > 0) ok = issue_sdp(0);
            for (int j = 0; j < njobs && ok; ++j) {
                if (j + 1 < njobs && !(ok = issue_sdp(j + 1))) break;
                const int sbuf = j & 1;
                if (!(ok = mbar_wait(&p_full[sbuf], (j >> 1) & 1, ab, 35))) break;
                tc_fence_after();
                const int st = j % kNst;
                const uint64_t qmn = dst_mn + ((st * L::kStageBytes) >> 4);
                const uint64_t domn = qmn + (L::kSubT >> 4);
#pragma unroll
                for (int kk = 0; kk < kSub / 16; ++kk) {
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    const uint32_t ok_ = (kk * 16 * 128) >> 4;
                    // queries 16kk .. 16kk+15 belong to half (kk >> 1), which wrote their P^T
                    // (dS^T) into its first 16 S^T (dP^T) columns, two queries per column
                    const uint32_t pcol = tmem + sbuf * 128 + 32 * (kk >> 1) + 8 * (kk & 1);
                    umma_bf16_ts(tm_dv, pcol, domn + ok_, idesc_acc, acc);
                    umma_bf16_ts(tm_dk, pcol + 64, qmn + ok_, idesc_acc, acc);
                }
                umma_commit(&s_free[sbuf]);
                umma_commit(&empty[st]);
            }
            if (ok) umma_commit(acc_full);
            umma_commit(mma_done);
            drain_wait(mma_done, 0);
        }
    } else {
        // two threads per key row: `half` takes query columns [32*half, 32*half + 32)
        const int ew = threadIdx.x - 64;
        const int half = ew >> 7;
        const int quarter = warp & 3;
        const int krow = quarter * 32 + lane;         // key row == TMEM lane
        const int jkey = b * kBlk + krow;
        const bool key_valid = jkey < N;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + half * 32;
        const float gamma = a.gamma, cx = a.cx;
        bool ok = true;
        // -tau, -delta of the sub-tile's 64 query rows, loaded one job ahead
        float ntau_n = 0.f, ndel_n = 0.f;
        auto load_td = [&](int jj) {
            const int ii = jobs[jj] + ew;
            ntau_n = ii < N ? -a.tau[(size_t)bh * N + ii] : 0.f;
            ndel_n = ii < N ? -a.delta[(size_t)bh * N + ii] : 0.f;
        };
        if (ew < 64 && njobs > 0) load_td(0);
        for (int j = 0; j < njobs && ok; ++j) {
            const int i0 = jobs[j];
            float* tdb = td + (j & 1) * 128;
            if (ew < 64) {
                tdb[ew] = ntau_n;
                tdb[64 + ew] = ndel_n;
                if (j + 1 < njobs) load_td(j + 1);
            }
            named_bar(1, kEw);
            const int sbuf = j & 1;
            if (!(ok = mbar_wait(&s_full[sbuf], (j >> 1) & 1, ab, 36))) break;
            tc_fence_after();
            float s[32], dp[32];
            tmem_ld32(lane_base + sbuf * 128, &s[0]);
            tmem_ld32(lane_base + sbuf * 128 + 64, &dp[0]);
            tmem_wait_ld();
            reg_fence<32>(s);
            reg_fence<32>(dp);
            // column c is query i0 + 32*half + c: admissible iff i < N, key valid, key <= i if causal
            const int ib = i0 + half * 32;
            const int cmin = a.causal ? jkey - ib : 0;       // c >= cmin
            const int cmax = min(32, N - ib);                // c < cmax
            const float* tcol = tdb + half * 32;
            if (!__all_sync(0xffffffffu, key_valid && cmin <= 0 && cmax >= 32)) {
                // diagonal or ragged sub-tile: inadmissible columns get s = -inf (u < 0)
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    s[c] = (key_valid && c >= cmin && c < cmax) ? s[c] : -INFINITY;
            }
            uint32_t wp[16], wd[16];
            const float2 cx2 = make_float2(cx, cx);
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 ntq = *reinterpret_cast<const float4*>(tcol + c);        // -tau
                const float4 ndl = *reinterpret_cast<const float4*>(tcol + 64 + c);   // -delta
                float2 p0, g0, p1, g1;
                entmax_pg_x2<GM>(__ffma2_rn(make_float2(s[c], s[c + 1]), cx2, make_float2(ntq.x, ntq.y)),
                                 gamma, p0, g0);
                entmax_pg_x2<GM>(__ffma2_rn(make_float2(s[c + 2], s[c + 3]), cx2, make_float2(ntq.z, ntq.w)),
                                 gamma, p1, g1);
                const float2 d0 = __fmul2_rn(g0, __fadd2_rn(make_float2(dp[c], dp[c + 1]), make_float2(ndl.x, ndl.y)));
                const float2 d1 = __fmul2_rn(g1, __fadd2_rn(make_float2(dp[c + 2], dp[c + 3]), make_float2(ndl.z, ndl.w)));
                wp[c >> 1] = pack_bf16(p0.x, p0.y);
                wp[(c >> 1) + 1] = pack_bf16(p1.x, p1.y);
                wd[c >> 1] = pack_bf16(d0.x, d0.y);
                wd[(c >> 1) + 1] = pack_bf16(d1.x, d1.y);
            }
            // P^T over this thread's own S^T columns, dS^T over its own dP^T columns
            tmem_st16(lane_base + sbuf * 128, wp);
            tmem_st16(lane_base + sbuf * 128 + 64, wd);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sbuf]);
        }
        constexpr int DH = D / 2;
        float acc[DH];
        const uint32_t qoff = ((uint32_t)(quarter * 32) << 16) + half * DH;
        if (ok && njobs > 0) {
            ok = mbar_wait(acc_full, 0, ab, 38);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) tmem_ld32(tm_dv + qoff + c * 32, &acc[c * 32]);
            tmem_wait_ld();
            reg_fence<DH>(acc);
        } else {
#pragma unroll
            for (int c = 0; c < DH; ++c) acc[c] = 0.f;
        }
        if (key_valid) store_out_row(a.dv, ((size_t)bh * N + jkey) * D + half * DH, acc, DH, 1.f);
        if (ok && njobs > 0) {
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) tmem_ld32(tm_dk + qoff + c * 32, &acc[c * 32]);
            tmem_wait_ld();
            reg_fence<DH>(acc);
        }
        if (key_valid) store_out_row(a.dk, ((size_t)bh * N + jkey) * D + half * DH, acc, DH, a.scale);
        if (ew == 0)   // block products: S^T, dP^T, dV, dK (4) per 64-row half
            atomicAdd(&a.hdr->counters[kCtrBwdBlocks], (unsigned long long)(2 * njobs));
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
template <int D, int GM>
static cudaError_t launch_tc_bwd(const BwdArgs& a, cudaStream_t s, const CUtensorMap* m) {
    // m: q128, do128, k64, v64, k128, v128, q64, do64
    {
        const size_t sm = DqLayout<D>::bytes(a.T);
        auto kern = tc_bwd_dq_kernel<D, GM>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        kern<<<dim3(a.T, a.BH), kThreads, sm, s>>>(m[0], m[1], m[2], m[3], a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t sm = DkvLayout<D>::bytes(a.T);
    auto kern = tc_bwd_dkv_kernel<D, GM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.T, a.BH), kThreads, sm, s>>>(m[4], m[5], m[6], m[7], a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t tc_bwd_d(const BwdArgs& a, int gm, cudaStream_t s, const CUtensorMap* m) {
    switch (gm) {
        case 1: return launch_tc_bwd<D, 1>(a, s, m);
        case 2: return launch_tc_bwd<D, 2>(a, s, m);
        case 4: return launch_tc_bwd<D, 4>(a, s, m);
        default: return launch_tc_bwd<D, 0>(a, s, m);
    }
}

cudaError_t tc_bwd(const BwdArgs& a, int d, int gm, cudaStream_t s, const char** why) {
    CUtensorMap m[8];
    const bool ok = make_tmap_bf16_rows(&m[0], a.q, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[1], a.dout, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[2], a.k, a.BH, a.N, d, 64) &&
                    make_tmap_bf16_rows(&m[3], a.v, a.BH, a.N, d, 64) &&
                    make_tmap_bf16_rows(&m[4], a.k, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[5], a.v, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[6], a.q, a.BH, a.N, d, 64) &&
                    make_tmap_bf16_rows(&m[7], a.dout, a.BH, a.N, d, 64);
    if (!ok) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    return d == 64 ? tc_bwd_d<64>(a, gm, s, m) : tc_bwd_d<128>(a, gm, s, m);
}

}  // namespace ent
