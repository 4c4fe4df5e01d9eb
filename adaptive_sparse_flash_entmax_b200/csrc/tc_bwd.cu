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
// elementwise, two threads per TMEM lane).  The bf16 operand the elementwise
// warps produce (dS, P^T, dS^T) is written into TMEM and the MMA reads it from
// there as its A operand:
//   dq kernel   one CTA per 128-row query tile, one live 128-key block per job.
//               Phase A: S = Q K^T, dP = dO V^T -> delta per row (also written
//               to the workspace).  Phase B: again S and dP, dS rounded to
//               bf16 and dQ += dS K (K read MN-major), then a rank-1 correction
//               for the rounding residual of dS's rows (which sum to 0).  Given
//               the forward's otilde = sum_j g_ij v_j / sum_j g_ij, delta_i =
//               dO_i . otilde_i (since dP = dO V^T) and phase A is skipped.
//   dkv kernel  one CTA per 128-key block, Q/dO in 64-row sub-tiles of the
//               live query tiles (so that two S^T/dP^T pairs fit in TMEM
//               beside dV and dK), P^T and dS^T over their own S^T and dP^T
//               columns.  S^T = K Q^T, dP^T = V dO^T, then P^T and
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

// 4-byte asynchronous copy global -> shared, and an arrive on `bar` once every earlier
// cp.async of this thread has landed (the arrival counts toward the barrier's expected
// count, which includes it).
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// The same with an fp32 row added after scaling: out = v * sc + add (the support-list
// kernel's dK / dV contributions).
__device__ __forceinline__ void store_out_row_add(void* out, size_t off, const float* v, int D, float sc,
                                                  const float* add) {
    __nv_bfloat16* p = static_cast<__nv_bfloat16*>(out) + off;
    for (int c = 0; c < D; c += 8) {
        const float4 a0 = *reinterpret_cast<const float4*>(add + off + c);
        const float4 a1 = *reinterpret_cast<const float4*>(add + off + c + 4);
        uint4 val = make_uint4(pack_bf16(fmaf(v[c], sc, a0.x), fmaf(v[c + 1], sc, a0.y)),
                               pack_bf16(fmaf(v[c + 2], sc, a0.z), fmaf(v[c + 3], sc, a0.w)),
                               pack_bf16(fmaf(v[c + 4], sc, a1.x), fmaf(v[c + 5], sc, a1.y)),
                               pack_bf16(fmaf(v[c + 6], sc, a1.z), fmaf(v[c + 7], sc, a1.w)));
        *reinterpret_cast<uint4*>(p + c) = val;
    }
}

}  // namespace

// =========================================================================
// dq kernel: delta and dQ for one 128-row query tile, one 128-key live block
// per job (128-wide MMAs run at the tensor rate; 64-wide ones do not).
// TMEM: phase A keeps two S/dP pairs (S at 256p, dP at 256p + 128); phase B
// one pair at 0, dQ at 256 and dS (bf16 at 384, two keys per column).  K blocks stay three jobs in shared memory (S, then dQ reads them
// MN-major one job later); V blocks feed dP only.
// =========================================================================
template <int D>
struct DqLayout {
    static constexpr int kTile = D / 64 * kAtom128;     // [128 x D] bf16: Q, dO, a K or a V block
    static constexpr int kKSlots = 3;
    static constexpr int kVSlots = (D == 64) ? 2 : 1;
    static constexpr int kQ = 0;
    static constexpr int kDO = kQ + kTile;
    static constexpr int kK0 = kDO + kTile;
    static constexpr int kV0 = kK0 + kKSlots * kTile;
    static constexpr int kXch = kV0 + kVSlots * kTile;  // [5][2][128] f32
    static constexpr int kBars = kXch + 5 * 2 * 128 * 4;
    static constexpr int kMisc = kBars + 8 * 24;        // up to 24 mbarriers
    static constexpr int kList = kMisc + 16;            // live key blocks, uint16 [T]
    static size_t bytes(int T) { return (size_t)kList + 2 * (size_t)T + 16 + 1024; }
};

template <int D, int GM>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const BwdArgs a) {
    using L = DqLayout<D>;
    constexpr int KS = L::kKSlots, VS = L::kVSlots;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* kfull = bars;                    // [KS]  TMA -> MMA
    uint64_t* kempty = kfull + KS;             // [KS]  MMA -> TMA (after S in phase A, after dQ in B)
    uint64_t* vfull = kempty + KS;             // [VS]
    uint64_t* vempty = vfull + VS;             // [VS]  MMA -> TMA (after dP)
    uint64_t* s_full = vempty + VS;            // [2]   MMA -> elementwise (S and dP of a pair)
    uint64_t* s_empty = s_full + 2;            // [2]   elementwise -> MMA (pair read)
    uint64_t* ds_full = s_empty + 2;           //       elementwise -> MMA (dS in TMEM)
    uint64_t* ds_free = ds_full + 1;           //       MMA -> elementwise (dQ read dS)
    uint64_t* acc_full = ds_free + 1;
    uint64_t* in_full = acc_full + 1;          // Q and dO tiles
    uint64_t* mma_done = in_full + 1;
    Misc* misc = reinterpret_cast<Misc*>(smem + L::kMisc);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + L::kList);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, N = a.N;
    // grid (BH, T): every head's longest causal tile first
    const int t = a.causal ? (T - 1 - (int)blockIdx.y) : (int)blockIdx.y;
    const int bh = blockIdx.x;
    const int nblk = a.causal ? t + 1 : T;
    const Abort ab{&misc->abort, a.hdr};
    // a tile every row of which has a support list is the list kernel's (it writes that
    // dQ); the decision is the list kernel's own rule, taken here from the same list
    // counts, so the two kernels can run at the same time
    if (a.list_n) {
        bool has = true;
        if (threadIdx.x < kBlk && t * kBlk + (int)threadIdx.x < N)
            has = a.list_n[(size_t)bh * N + t * kBlk + threadIdx.x] != kListOver;
        if (__syncthreads_and(has)) return;
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < KS; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
        for (int i = 0; i < VS; ++i) { mbar_init(&vfull[i], 1); mbar_init(&vempty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], kEwWarps); }
        mbar_init(ds_full, kEwWarps);
        mbar_init(ds_free, 1);
        mbar_init(acc_full, 1);
        mbar_init(in_full, 1);
        mbar_init(mma_done, 1);
        misc->abort = 0;
        fence_barrier_init();
        // Q and dO of the tile do not depend on the job list: start them first
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_do); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(in_full, 2 * L::kTile);
        for (int at = 0; at < D / 64; ++at) {
            tma_load_3d(smem + L::kQ + at * kAtom128, &tm_q, at * 64, t * kBlk, bh, in_full);
            tma_load_3d(smem + L::kDO + at * kAtom128, &tm_do, at * 64, t * kBlk, bh, in_full);
        }
    }
    if (warp == 2) {
        // live key blocks of this tile, in order: 32 mask bytes per step, compacted by ballot
        const uint8_t* mrow = a.mask + ((size_t)bh * T + t) * T;
        int n = 0;
        for (int base = 0; base < nblk; base += 32) {
            const int b = base + lane;
            const bool f = b < nblk && mrow[b] != 0;
            const unsigned int msk = __ballot_sync(0xffffffffu, f);
            if (f) list[n + __popc(msk & ((1u << lane) - 1u))] = (uint16_t)b;
            n += __popc(msk);
        }
        if (lane == 0) misc->njobs = n;
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    // phase A jobs 0..nA-1 (none when delta comes from otilde), phase B jobs nA..nA+nB-1,
    // both over the same live blocks
    const int nB = misc->njobs;
    const int nA = a.otilde ? 0 : nB;
    const int total = nA + nB;
    // pair of job j and the number of earlier jobs on that pair
    auto pair_of = [&](int j) { return j < nA ? (j & 1) : 0; };
    auto use_of = [&](int j) { return j < nA ? (j >> 1) : ((nA + 1) >> 1) + (j - nA); };

    if (warp == 0) {
        if (lane == 0) {
            int nk = 0, nv = 0;   // K and V blocks issued
            bool ok = true;
            for (int j = 0; j < total && ok; ++j) {
                const int b = list[j < nA ? j : j - nA];
                const int ks = j % KS, vs = j % VS;
                if (!(ok = mbar_wait(&kempty[ks], ((j / KS) & 1) ^ 1, ab, 21))) break;
                mbar_arrive_expect_tx(&kfull[ks], L::kTile);
                for (int at = 0; at < D / 64; ++at)
                    tma_load_3d(smem + L::kK0 + ks * L::kTile + at * kAtom128, &tm_k, at * 64, b * kBlk, bh,
                                &kfull[ks]);
                ++nk;
                if (!(ok = mbar_wait(&vempty[vs], ((j / VS) & 1) ^ 1, ab, 21))) break;
                mbar_arrive_expect_tx(&vfull[vs], L::kTile);
                for (int at = 0; at < D / 64; ++at)
                    tma_load_3d(smem + L::kV0 + vs * L::kTile + at * kAtom128, &tm_v, at * 64, b * kBlk, bh,
                                &vfull[vs]);
                ++nv;
            }
            drain_wait(in_full, 0);
            for (int j = nk - 1; j >= 0 && j >= nk - KS; --j) drain_wait(&kfull[j % KS], (j / KS) & 1);
            for (int j = nv - 1; j >= 0 && j >= nv - VS; --j) drain_wait(&vfull[j % VS], (j / VS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);   // [128 x 128], K = d
            constexpr uint32_t idesc_dq = idesc_bf16(128, D, 0, 1);    // dQ += dS K, K MN-major
            const uint64_t dq_ = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
            const uint64_t ddo = sdesc_sw128(smem_u32(smem + L::kDO), 16, 1024);
            const uint64_t dk = sdesc_sw128(smem_u32(smem + L::kK0), 16, 1024);
            const uint64_t dkmn = sdesc_sw128(smem_u32(smem + L::kK0), kAtom128, 1024);
            const uint64_t dv = sdesc_sw128(smem_u32(smem + L::kV0), 16, 1024);
            bool ok = mbar_wait(in_full, 0, ab, 22);
            tc_fence_after();
            auto issue_128 = [&](uint32_t dcol, uint64_t da, uint64_t db) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kAtom128 + (kk & 3) * 32) >> 4;
                    umma_bf16(tmem + dcol, da + off, db + off, idesc_s, kk > 0);
                }
            };
            // S and dP of job j into its pair; phase A releases the K block after S,
            // phase B keeps it for dQ
            auto issue_sdp = [&](int j) -> bool {
                const int p = pair_of(j), ks = j % KS, vs = j % VS;
                if (!mbar_wait(&s_empty[p], (use_of(j) & 1) ^ 1, ab, 24)) return false;
                if (!mbar_wait(&kfull[ks], (j / KS) & 1, ab, 23)) return false;
                tc_fence_after();
                issue_128(p * 256, dq_, dk + ((uint32_t)(ks * L::kTile) >> 4));
                if (j < nA) umma_commit(&kempty[ks]);
                if (!mbar_wait(&vfull[vs], (j / VS) & 1, ab, 23)) return false;
                tc_fence_after();
                issue_128(p * 256 + 128, ddo, dv + ((uint32_t)(vs * L::kTile) >> 4));
                umma_commit(&vempty[vs]);
                umma_commit(&s_full[p]);
                return true;
            };
            // dQ += bf16(dS) K for phase B job i (the rounding residual of dS, whose rows
            // sum to 0, is corrected in the epilogue)
            auto issue_dq = [&](int i) -> bool {
                const int ks = (nA + i) % KS;
                if (!mbar_wait(ds_full, i & 1, ab, 25)) return false;
                tc_fence_after();
                const uint64_t bk = dkmn + ((uint32_t)(ks * L::kTile) >> 4);
#pragma unroll
                for (int kk = 0; kk < kBlk / 16; ++kk) {
                    const uint64_t bdesc = bk + ((kk * 16 * 128) >> 4);
                    umma_bf16_ts(tmem + 256, tmem + 384 + kk * 8, bdesc, idesc_dq, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(ds_free);
                umma_commit(&kempty[ks]);
                return true;
            };
            for (int j = 0; j < nA && ok; ++j) ok = issue_sdp(j);
            // phase B: S and dP of job i go in ahead of dQ of job i-1, so the tensor
            // pipe has work while the elementwise warps turn job i-1 into dS
            for (int i = 0; i < nB && ok; ++i) {
                ok = issue_sdp(nA + i);
                if (ok && i > 0) ok = issue_dq(i - 1);
            }
            if (ok && nB > 0) ok = issue_dq(nB - 1);
            if (ok) umma_commit(acc_full);
            umma_commit(mma_done);
            drain_wait(mma_done, 0);
        }
    } else {
        // two threads per query row: `half` takes keys [64*half, 64*half + 64) of each
        // block, in two rounds of 32; delta's partial sums meet in shared memory
        const int ew = threadIdx.x - 64;
        const int half = ew >> 7;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int i = t * kBlk + row;
        const bool row_valid = i < N;
        const int key_end = !row_valid ? 0 : (a.causal ? i + 1 : N);
        const uint32_t lane0 = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t lane_base = lane0 + half * 64;
        const float gamma = a.gamma, cx = a.cx;
        const float tau = row_valid ? a.tau[(size_t)bh * N + i] : 0.f;
        float* xch = reinterpret_cast<float*>(smem + L::kXch);   // [5][2][128]
        const float2 cx2 = make_float2(cx, cx), nt2 = make_float2(-tau, -tau);
        bool ok = true;
        // phase A: sum_j g and sum_j g dP
        float sg = 0.f, sgdp = 0.f;
        for (int j = 0; j < nA && ok; ++j) {
            if (!(ok = mbar_wait(&s_full[pair_of(j)], use_of(j) & 1, ab, 26))) break;
            tc_fence_after();
            // both rounds in one go (the pair is free again after a single load latency)
            float sa[64], dpa[64];
            const int p = pair_of(j);
            tmem_ld32(lane_base + p * 256, &sa[0]);
            tmem_ld32(lane_base + p * 256 + 32, &sa[32]);
            tmem_ld32(lane_base + p * 256 + 128, &dpa[0]);
            tmem_ld32(lane_base + p * 256 + 128 + 32, &dpa[32]);
            tmem_wait_ld();
            reg_fence<64>(sa);
            reg_fence<64>(dpa);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[p]);
            const int nv = key_end - list[j] * kBlk - half * 64;
            if (!__all_sync(0xffffffffu, nv >= 64)) {   // diagonal or ragged block
#pragma unroll
                for (int c = 0; c < 64; ++c) sa[c] = (c < nv) ? sa[c] : -INFINITY;
            }
            float2 a0 = make_float2(0.f, 0.f), b0 = a0, a1 = a0, b1 = a0;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                const float2 g0 = entmax_g_x2<GM>(__ffma2_rn(make_float2(sa[c], sa[c + 1]), cx2, nt2), gamma);
                const float2 g1 = entmax_g_x2<GM>(__ffma2_rn(make_float2(sa[c + 2], sa[c + 3]), cx2, nt2), gamma);
                a0 = __fadd2_rn(a0, g0); b0 = __ffma2_rn(g0, make_float2(dpa[c], dpa[c + 1]), b0);
                a1 = __fadd2_rn(a1, g1); b1 = __ffma2_rn(g1, make_float2(dpa[c + 2], dpa[c + 3]), b1);
            }
            a0 = __fadd2_rn(a0, a1); b0 = __fadd2_rn(b0, b1);
            sg += a0.x + a0.y;
            sgdp += b0.x + b0.y;
        }
        constexpr int DH = D / 2;
        float dpart = 0.f;   // with otilde: this half's share of dO_i . otilde_i
        // d = 32 runs as D = 64 (zero upper columns): the half holding columns 32..63 reads
        // and stores nothing
        const bool own_half = half * DH < a.dr;
        if (a.otilde && row_valid && own_half) {
            const __nv_bfloat16* dor = static_cast<const __nv_bfloat16*>(a.dout) + ((size_t)bh * N + i) * a.dr + half * DH;
            const float* otr = a.otilde + ((size_t)bh * N + i) * a.dr + half * DH;
            float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll 4
            for (int c = 0; c < DH; c += 8) {
                const uint4 g8 = *reinterpret_cast<const uint4*>(dor + c);
                const float4 o0 = *reinterpret_cast<const float4*>(otr + c);
                const float4 o1 = *reinterpret_cast<const float4*>(otr + c + 4);
                const uint32_t w[4] = {g8.x, g8.y, g8.z, g8.w};
                const float2 ov[4] = {make_float2(o0.x, o0.y), make_float2(o0.z, o0.w),
                                      make_float2(o1.x, o1.y), make_float2(o1.z, o1.w)};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc2 = __ffma2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e])), ov[e], acc2);
            }
            dpart = acc2.x + acc2.y;
        }
        // every elementwise thread reaches this barrier once, also after an abort
        xch[(0 * 2 + half) * 128 + row] = a.otilde ? dpart : sg;
        xch[(1 * 2 + half) * 128 + row] = sgdp;
        named_bar(1, kEw);
        float delta;
        if (a.otilde) {
            delta = dpart + xch[(0 * 2 + (half ^ 1)) * 128 + row];
        } else {
            const float SG = sg + xch[(0 * 2 + (half ^ 1)) * 128 + row];
            const float SGDP = sgdp + xch[(1 * 2 + (half ^ 1)) * 128 + row];
            delta = (SG > 0.f) ? SGDP / SG : 0.f;
        }
        if (row_valid && half == 0) a.delta[(size_t)bh * N + i] = delta;
        // phase B: dS = g (dP - delta) rounded to bf16 into TMEM.  With dS rounded once,
        // the rows' residuals eps_i = sum_j (bf16(dS_ij) - dS_ij) would reach dQ as
        // eps_i times the common part of the support's keys (large on clustered keys,
        // where sum_j dS_ij k_j cancels); the epilogue subtracts eps_i k_{j*}, j* the
        // row's arg-max key, which leaves only eps-sized errors times k_j - k_{j*}.
        const float2 nd2 = make_float2(-delta, -delta), m1 = make_float2(-1.f, -1.f);
        float best = -INFINITY;   // this thread's largest score and its key
        int jbest = 0;
        float2 eps2 = make_float2(0.f, 0.f);
        for (int ib = 0; ib < nB && ok; ++ib) {
            const int j = nA + ib;
            if (!(ok = mbar_wait(&s_full[0], use_of(j) & 1, ab, 26))) break;
            tc_fence_after();
            const int key0 = list[ib] * kBlk + half * 64;   // key of this thread's first column
            // both rounds' S and dP in one go, so the pair is free for S(i+1), dP(i+1) after a
            // single TMEM load latency
            float sa[64], dpa[64];
            {
                const int p = pair_of(j);
                tmem_ld32(lane_base + p * 256, &sa[0]);
                tmem_ld32(lane_base + p * 256 + 32, &sa[32]);
                tmem_ld32(lane_base + p * 256 + 128, &dpa[0]);
                tmem_ld32(lane_base + p * 256 + 128 + 32, &dpa[32]);
                tmem_wait_ld();
                reg_fence<64>(sa);
                reg_fence<64>(dpa);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[p]);
                const int nv = key_end - key0;   // valid columns of this thread: c < nv
                if (!__all_sync(0xffffffffu, nv >= 64)) {   // diagonal or ragged block
#pragma unroll
                    for (int c = 0; c < 64; ++c) sa[c] = (c < nv) ? sa[c] : -INFINITY;
                }
            }
            uint32_t whi[32];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float* s = sa + 32 * r;
                const float* dp = dpa + 32 * r;
                float rmax = s[0];
#pragma unroll
                for (int c = 1; c < 32; ++c) rmax = fmaxf(rmax, s[c]);
                if (rmax > best) {   // rare after the first blocks: find the column
                    best = rmax;
                    int cc = 0;
#pragma unroll
                    for (int c = 31; c >= 0; --c) cc = (s[c] == rmax) ? c : cc;
                    jbest = key0 + r * 32 + cc;
                }
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 g = entmax_g_x2<GM>(__ffma2_rn(make_float2(s[c], s[c + 1]), cx2, nt2), gamma);
                    const float2 d = __fmul2_rn(g, __fadd2_rn(make_float2(dp[c], dp[c + 1]), nd2));
                    const __nv_bfloat162 h = __floats2bfloat162_rn(d.x, d.y);
                    eps2 = __fadd2_rn(eps2, __ffma2_rn(d, m1, __bfloat1622float2(h)));   // bf16(d) - d
                    whi[r * 16 + (c >> 1)] = *reinterpret_cast<const uint32_t*>(&h);
                }
            }
            // the dS region is free once dQ of the previous job has read it
            if (!(ok = mbar_wait(ds_free, (ib & 1) ^ 1, ab, 27))) break;
            tmem_st32(lane0 + 384 + half * 32, whi);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full);
        }
        float acc[DH];
        if (ok && nB > 0) {
            ok = mbar_wait(acc_full, 0, ab, 28);
            tc_fence_after();
            const uint32_t ob = lane0 + 256 + half * DH;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) tmem_ld32(ob + c * 32, &acc[c * 32]);
            tmem_wait_ld();
            reg_fence<DH>(acc);
        } else {
#pragma unroll
            for (int c = 0; c < DH; ++c) acc[c] = 0.f;
        }
        // the row's arg-max key and residual: the halves meet in shared memory (slots of
        // their own, so no reader of the delta exchange is overtaken; every elementwise
        // thread reaches this barrier once, also after an abort)
        xch[(2 * 2 + half) * 128 + row] = best;
        xch[(3 * 2 + half) * 128 + row] = __int_as_float(jbest);
        xch[(4 * 2 + half) * 128 + row] = eps2.x + eps2.y;
        named_bar(1, kEw);
        const float obest = xch[(2 * 2 + (half ^ 1)) * 128 + row];
        const int ojbest = __float_as_int(xch[(3 * 2 + (half ^ 1)) * 128 + row]);
        const float eps = eps2.x + eps2.y + xch[(4 * 2 + (half ^ 1)) * 128 + row];
        const int js = (obest > best || (obest == best && ojbest < jbest)) ? ojbest : jbest;
        if (row_valid && own_half && ok && nB > 0 && fmaxf(best, obest) > -INFINITY) {
            const __nv_bfloat16* kr = static_cast<const __nv_bfloat16*>(a.k) + ((size_t)bh * N + js) * a.dr + half * DH;
#pragma unroll
            for (int c = 0; c < DH; c += 8) {
                const uint4 k8 = *reinterpret_cast<const uint4*>(kr + c);
                const uint32_t w[4] = {k8.x, k8.y, k8.z, k8.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                    acc[c + 2 * e] = fmaf(-eps, kv.x, acc[c + 2 * e]);
                    acc[c + 2 * e + 1] = fmaf(-eps, kv.y, acc[c + 2 * e + 1]);
                }
            }
        }
        if (row_valid && own_half) store_out_row(a.dq, ((size_t)bh * N + i) * a.dr + half * DH, acc, DH, a.scale);
        if (threadIdx.x == 64)   // block products: phase A S, dP (2) + phase B S, dP, dQ (3)
            atomicAdd(&a.hdr->counters[kCtrBwdBlocks], (unsigned long long)(2 * nA + 3 * nB));
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
    static constexpr int kTauDelta = kStage0 + kNst * kStageBytes;   // [kNst][tau|delta][64] floats
    static constexpr int kBars = kTauDelta + kNst * 2 * 64 * 4;
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
    float* td = reinterpret_cast<float*>(smem + L::kTauDelta);   // [stage][tau|delta][64]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, N = a.N;
    // grid (BH, T): every head's key block 0 (the most live query tiles when causal) first
    const int b = blockIdx.y;
    const int bh = blockIdx.x;
    const Abort ab{&misc->abort, a.hdr};

    if (threadIdx.x == 0) {
        // a stage is full once its Q/dO tiles (TMA, one arrival with the byte count) and
        // its tau/delta (cp.async by the 32 producer lanes, one arrival each) have landed
        for (int s = 0; s < kNst; ++s) { mbar_init(&full[s], 1 + 32); mbar_init(&empty[s], 1); }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 1);
            mbar_init(&p_full[s], kEwWarps);
        }
        mbar_init(acc_full, 1);
        mbar_init(in_full, 1);
        mbar_init(mma_done, 1);
        misc->abort = 0;
        fence_barrier_init();
        // K and V of the block do not depend on the job list: start them first
        prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_q64); prefetch_tmap(&tm_do64);
        mbar_arrive_expect_tx(in_full, 2 * L::kTile);
        for (int at = 0; at < D / 64; ++at) {
            tma_load_3d(smem + L::kK + at * kAtom128, &tm_k, at * 64, b * kBlk, bh, in_full);
            tma_load_3d(smem + L::kV + at * kAtom128, &tm_v, at * 64, b * kBlk, bh, in_full);
        }
    }
    if (warp == 2) {
        // 64-row sub-tiles of the live query tiles of this key block, in order: one query
        // tile per lane and step (the mask column is strided, so the loads go out in
        // parallel), up to two jobs each, placed by a warp prefix sum
        int n = 0;
        for (int base = a.causal ? b : 0; base < T; base += 32) {
            const int t = base + lane;
            int c = 0, i0a = 0, i0b = 0;
            // live query tiles of this key block, except those the support-list kernel covered
            if (t < T && a.mask[((size_t)bh * T + t) * T + b] &&
                !(a.tile_list && a.tile_list[(size_t)bh * T + t])) {
                for (int h = 0; h < 2; ++h) {
                    const int i0 = t * kBlk + h * kSub;
                    if (i0 >= N || (a.causal && i0 + kSub - 1 < b * kBlk)) continue;
                    if (c == 0) i0a = i0; else i0b = i0;
                    ++c;
                }
            }
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int pos = n + incl - c;
            if (c > 0) jobs[pos] = i0a;
            if (c > 1) jobs[pos + 1] = i0b;
            n += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) misc->njobs = n;
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
        // the whole warp: lane 0 waits for the stage and issues the Q/dO tiles, every lane
        // copies two of the sub-tile's 64 tau and delta values
        int job = 0;
        bool ok = true;
        for (; job < njobs && ok; ++job) {
            const int i0 = jobs[job];
            const int st = job % kNst;
            if (lane == 0) ok = mbar_wait(&empty[st], ((job / kNst) & 1) ^ 1, ab, 31);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                uint8_t* sb = smem + L::kStage0 + st * L::kStageBytes;
                mbar_arrive_expect_tx(&full[st], 2 * L::kSubT);
                for (int at = 0; at < D / 64; ++at) {
                    tma_load_3d(sb + at * kAtom64, &tm_q64, at * 64, i0, bh, &full[st]);
                    tma_load_3d(sb + L::kSubT + at * kAtom64, &tm_do64, at * 64, i0, bh, &full[st]);
                }
            }
            // rows past N copy row N-1 (finite values for columns the elementwise warps mask)
            float* tds = td + st * 128;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int ii = min(i0 + lane + 32 * r, N - 1);
                cp_async_4(tds + lane + 32 * r, a.tau + (size_t)bh * N + ii);
                cp_async_4(tds + 64 + lane + 32 * r, a.delta + (size_t)bh * N + ii);
            }
            cp_async_arrive_noinc(&full[st]);
        }
        if (lane == 0) {
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
        for (int j = 0; j < njobs; ++j) {
            const int i0 = jobs[j];
            const int st = j % kNst;
            const int sbuf = j & 1;
            // tau and delta of the sub-tile arrive with its stage (the MMA waited for the
            // same phase before S^T); this wait makes the copies visible here
            if (!(ok = mbar_wait(&full[st], (j / kNst) & 1, ab, 37))) break;
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
            const float* tcol = td + st * 128 + half * 32;   // tau, then delta 64 floats on
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
                const float4 tq = *reinterpret_cast<const float4*>(tcol + c);
                const float4 dl = *reinterpret_cast<const float4*>(tcol + 64 + c);
                const float4 ntq = make_float4(-tq.x, -tq.y, -tq.z, -tq.w);
                const float4 ndl = make_float4(-dl.x, -dl.y, -dl.z, -dl.w);
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
        const bool own_half = half * DH < a.dr;   // d = 32 as D = 64: columns 32..63 are not stored
        const size_t orow = ((size_t)bh * N + jkey) * a.dr + half * DH;
        if (key_valid && own_half) {
            if (a.dv_acc) store_out_row_add(a.dv, orow, acc, DH, 1.f, a.dv_acc);
            else store_out_row(a.dv, orow, acc, DH, 1.f);
        }
        if (ok && njobs > 0) {
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) tmem_ld32(tm_dk + qoff + c * 32, &acc[c * 32]);
            tmem_wait_ld();
            reg_fence<DH>(acc);
        }
        if (key_valid && own_half) {
            if (a.dk_acc) store_out_row_add(a.dk, orow, acc, DH, a.scale, a.dk_acc);
            else store_out_row(a.dk, orow, acc, DH, a.scale);
        }
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
static cudaError_t launch_tc_bwd(const BwdArgs& a, cudaStream_t s, const CUtensorMap* m,
                                 cudaEvent_t before_dkv) {
    // m: q128, do128, k128, v128, q64, do64
    {
        const size_t sm = DqLayout<D>::bytes(a.T);
        auto kern = tc_bwd_dq_kernel<D, GM>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        kern<<<dim3(a.BH, a.T), kThreads, sm, s>>>(m[0], m[1], m[2], m[3], a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // dkv adds the list kernel's accumulators: it waits for that kernel here
    if (before_dkv) {
        cudaError_t e = cudaStreamWaitEvent(s, before_dkv, 0);
        if (e != cudaSuccess) return e;
    }
    const size_t sm = DkvLayout<D>::bytes(a.T);
    auto kern = tc_bwd_dkv_kernel<D, GM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.BH, a.T), kThreads, sm, s>>>(m[2], m[3], m[4], m[5], a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t tc_bwd_d(const BwdArgs& a, int gm, cudaStream_t s, const CUtensorMap* m,
                            cudaEvent_t before_dkv) {
    switch (gm) {
        case 1: return launch_tc_bwd<D, 1>(a, s, m, before_dkv);
        case 2: return launch_tc_bwd<D, 2>(a, s, m, before_dkv);
        case 4: return launch_tc_bwd<D, 4>(a, s, m, before_dkv);
        default: return launch_tc_bwd<D, 0>(a, s, m, before_dkv);
    }
}

cudaError_t tc_bwd(const BwdArgs& a, int d, int gm, cudaStream_t s, const char** why,
                   cudaEvent_t before_dkv) {
    CUtensorMap m[6];
    const bool ok = make_tmap_bf16_rows(&m[0], a.q, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[1], a.dout, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[2], a.k, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[3], a.v, a.BH, a.N, d, 128) &&
                    make_tmap_bf16_rows(&m[4], a.q, a.BH, a.N, d, 64) &&
                    make_tmap_bf16_rows(&m[5], a.dout, a.BH, a.N, d, 64);
    if (!ok) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    // d = 32 runs on the d = 64 kernels (zero-filled upper columns, see tc_fwd)
    return d == 128 ? tc_bwd_d<128>(a, gm, s, m, before_dkv) : tc_bwd_d<64>(a, gm, s, m, before_dkv);
}

}  // namespace ent
