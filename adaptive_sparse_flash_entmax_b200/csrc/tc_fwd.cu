// tc_fwd.cu -- the bf16 forward on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA per 128-row query tile, grid (heads, tiles) ("AdaSplash: Adaptive Sparse Flash Attention",
// Technical Deep Dive / AdaSplash: Fused GPU Kernel for Attention: the Q tile is
// loaded once and stays on chip; K tiles stream for the tau passes; a final pass
// streams K and V and accumulates O = P V).  Warp roles:
//   warp 0   TMA producer: Q once, then K blocks two at a time into two double
//            slots of the ring in the score passes (stacked as [256 rows x 64]
//            atoms), or K and V of each live block into four single slots (the
//            same memory) in the P.V pass;
//   warp 1   MMA issuer: in the score passes S = Q [K_a; K_b]^T as one 128 x 256
//            MMA into two 256-column TMEM buffers (a 256-wide instruction does
//            twice the work of a 128-wide one in ~1.5x the time, and the
//            elementwise warps' arithmetic slows every instruction); in the P.V
//            pass S = Q K^T into three 128-column buffers and O += P V with P
//            read from TMEM (it replaces S in its buffer), V MN-major;
//   warps 2-9 elementwise: two threads per query row (= TMEM lane), 64 columns
//            each.  Pass 0 builds the
//            row max and the sliding 64-bin histogram ("AdaSplash-2: ...",
//            Sparse Attention Makes Waves); solver passes accumulate
//            F0, F1, F2 and take a Halley-bisection step (Accelerated Alpha-Entmax
//            Transformation); the last solver pass marks live key blocks
//            (Exploiting Sparsity); the P.V pass writes P (bf16) for live blocks
//            into TMEM.
// Solver passes visit only candidate blocks: pass 0 records each warp's block
// maximum of x, and a block is streamed again only if some warp's maximum
// exceeds that warp's smallest current tau (otherwise no row of the tile has
// u > 0 there, so the skipped block adds nothing to the sums or the mask).
// Before pass 0 a bound pass may rule out whole key blocks (Exploiting
// Sparsity, applied to the statistics pass itself): S_c = Q C^T against the
// centroids of the 64-key half-blocks gives, per row and half-block, an upper
// bound q.c + |q| R of every score and a lower bound q.c - |q| L of the
// largest one.  A block whose upper bound lies at or below (largest lower
// bound) - 1 <= m - 1 <= tau for every row of the tile has p = 0 throughout,
// cannot hold a row maximum, and is left out of pass 0 and of everything after.
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

constexpr int kSlots = 4;          // single tile slots of the P.V pass (K or V blocks)
constexpr int kDSlots = 2;         // double slots of the score passes (two K blocks), same memory
constexpr int kSbuf = 3;           // 128-column S accumulators in TMEM (P.V pass; two when
                                   // the G.V accumulator of a d = 128 forward takes the third)
constexpr int kThreads = 320;      // 10 warps
constexpr int kEw = 256;           // elementwise threads (warps 2-9): two per query row
constexpr int kEwWarps = 8;
constexpr int kAtom = 128 * 128;   // bytes of a [128 rows x 64 bf16] swizzled atom
constexpr int kTmemCols = 512;     // score passes: S [0,256), [256,512); P.V pass: S0 [0,128),
                                   // S1 [128,256), O [256, 256+D), then either S2 [384, 512)
                                   // or, with otilde, G.V [256+D, 256+2D) (and S2 when D = 64)
constexpr int kDecSolve = 1, kDecPv = 2;
constexpr uint8_t kPvLive = 255;   // cand[] of a block with a nonzero p in the P.V pass
constexpr float kCalMargin = 0.03f; // calibrated start: offset below the nearest sample's gap

__host__ __device__ constexpr uint32_t sbuf_col(int sb) { return sb < 2 ? sb * 128 : 384; }

template <int D>
struct Layout {
    static constexpr int kTile = D / 64 * kAtom;          // [128 x D] bf16
    static constexpr int kQ = 0;
    static constexpr int kRing = kQ + kTile;              // kSlots tiles (K or V blocks)
    static constexpr int kP = kRing + kSlots * kTile;     // pass 0: the two half-row
    static constexpr int kPBytes = 2 * kAtom;             // histograms [64][128] u16
    static constexpr int kXch = kP + kPBytes;             // [4][2][128] f32 exchange
    static constexpr int kBars = kXch + 4 * 2 * 128 * 4;
    static constexpr int kNumBars = 40;
    static constexpr int kMisc = kBars + 8 * kNumBars;    // tmem base, decision, njobs, abort
    static constexpr int kPtab = kMisc + 32;              // 68 floats
    static constexpr int kMw = kPtab + 68 * 4;            // 8 floats: per-warp bound thresholds
    static constexpr int kLive = kMw + 8 * 4;             // live[T], cand[T] (bytes), list[T] (int),
                                                          // per-warp block maxima [T][8] (bf16)
    __host__ __device__ static size_t r16(int T) { return (size_t)((T + 15) / 16) * 16; }
    static size_t bytes(int T) { return (size_t)kLive + 2 * r16(T) + 4 * (size_t)T + 16 * (size_t)T + 1024; }
};

struct Misc {
    uint32_t tmem_base;
    int decision;
    int njobs;      // blocks in job_list for the next pass
    int abort;
    int inserts;    // histogram inserts of the whole tile so far (pass 0)
    int next;       // the CTA's next tile (flat bh * T + t), or -1
    int pad[2];
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Column maxima over the 32 lanes of a warp for 32 values per lane: after five
// exchange steps lane l holds the maximum of column l in v[0].  Each step keeps
// half of the columns (the lane bit picks which half) and combines them with the
// partner lane's copy of the same columns.
__device__ __forceinline__ void warp_colmax_32(float* v, int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int w = 16 >> step, bit = 16 >> step;
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int c = 0; c < w; ++c) {
            const float send = up ? v[c] : v[c + w];
            const float keep = up ? v[c + w] : v[c];
            v[c] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, bit));
        }
    }
}

// The speculative first job of the next score pass.  The decision after a pass (another
// solver pass, with its candidate list, or the P.V pass) drains the tile's pipeline: its
// first K blocks are loaded and multiplied only after it.  Instead, the blocks of this
// pass's first job -- usually also the next pass's first candidates -- are loaded by the
// producer and multiplied by the MMA issuer while the elementwise warps finish the pass;
// if the next pass starts with the same job, its S is already in TMEM, otherwise the
// elementwise warps drop it.  Every role arms it under the same condition from the same
// list and checks it against the same published decision, so all agree on hit or miss.
struct SpecJob {
    int b0 = -1, b1 = -1;   // the guessed job's blocks (b1 < 0: a one-block job)
    int use = 0;            // producer: the double-slot use that holds it
    bool on = false, hit = false;
    __device__ __forceinline__ void arm(bool want, bool all_blocks, int njobs, const int* jl) {
        on = want;
        if (want) {
            b0 = all_blocks ? 0 : jl[0];
            b1 = njobs > 1 ? (all_blocks ? 1 : jl[1]) : -1;
        }
    }
    __device__ __forceinline__ bool matches(int njobs, const int* jl) const {
        return njobs > 0 && jl[0] == b0 && (njobs > 1 ? jl[1] == b1 : b1 < 0);
    }
    __device__ __forceinline__ void check(bool solve, int njobs, const int* jl) {
        hit = on && solve && matches(njobs, jl);
    }
};

// Bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
}

}  // namespace

// OT: also accumulate G.V (g = u^(gamma-1) as bf16 beside P in TMEM) and write
// otilde = G.V / sum_j g, from which the backward takes delta without a pass over the keys.
template <int D, int GM, bool OT>
__global__ void __launch_bounds__(kThreads, 1)
tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_c,
              const FwdArgs a) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    uint64_t* kfull = bars;                    // [kSlots]     TMA -> MMA (P.V pass)
    uint64_t* kempty = kfull + kSlots;         // [kSlots]     MMA -> TMA
    uint64_t* kfull2 = kempty + kSlots;        // [kDSlots]    TMA -> MMA (score passes)
    uint64_t* kempty2 = kfull2 + kDSlots;      // [kDSlots]    MMA -> TMA
    uint64_t* s_full2 = kempty2 + kDSlots;     // [2]          MMA -> elementwise (score passes)
    uint64_t* s_empty2 = s_full2 + 2;          // [2]          elementwise -> MMA
    uint64_t* s_full = s_empty2 + 2;           // [kSbuf]      MMA -> elementwise (P.V pass)
    uint64_t* s_empty = s_full + kSbuf;        // [kSbuf]      (first use of a P.V buffer: fresh)
    uint64_t* pv_sfree = s_empty + kSbuf;      // [kSbuf]      MMA -> MMA (P.V pass: P(i) consumed)
    uint64_t* p_full = pv_sfree + kSbuf;       // [kSbuf]      elementwise -> MMA (P(i) in TMEM)
    uint64_t* o_full = p_full + kSbuf;         //              MMA -> elementwise
    uint64_t* q_full = o_full + 1;             //              TMA -> MMA
    uint64_t* dec_bar = q_full + 1;            //              elementwise -> TMA, MMA
    uint64_t* mma_done = dec_bar + 1;          //              MMA -> MMA (all MMAs retired)
    Misc* misc = reinterpret_cast<Misc*>(smem + L::kMisc);
    float* ptab = reinterpret_cast<float*>(smem + L::kPtab);
    uint8_t* live = smem + L::kLive;                       // live blocks of the current pass
    uint8_t* cand = live + L::r16(a.T);                    // candidate blocks, tagged by pass
    int* job_list = reinterpret_cast<int*>(cand + L::r16(a.T));   // blocks of the next pass
    __nv_bfloat16* bmw = reinterpret_cast<__nv_bfloat16*>(job_list + a.T);   // [T][8]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, N = a.N;
    constexpr int SB = (OT && D == 128) ? 2 : kSbuf;   // S buffers of the P.V pass
    constexpr uint32_t kOtCol = 256 + D;                // G.V accumulator (OT)
    if (warp == 1) {   // TMEM for the CTA's whole life (it may solve more than one tile)
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // This CTA's tile, then tiles from the failure list that it claims.
    // grid (BH, T): the heads' longest causal tiles are dispatched first, all of them
    // before any shorter one, so the last wave holds the shortest tiles
    int cur_t = a.causal ? (T - 1 - (int)blockIdx.y) : (int)blockIdx.y;
    int cur_bh = blockIdx.x;
    bool fixing = false;
    for (int rep = 0;; ++rep) {
    const int t = cur_t;
    const int bh = cur_bh;
    const int nblk = a.causal ? t + 1 : T;
    const Abort ab{&misc->abort, a.hdr};
    // a tile solved again takes evaluated stops only
    const AcceptRule acc = fixing ? AcceptRule() : a.acc;
    // Bound pass for this tile: only where a centroid bound can rule a block out at all
    // (some half-block of the head has R < 2 max |c|: a bound q.c_b + |q| R_b below
    // q.c_b' - |q| L_b' - 1/cx needs R_b < |c_b' - c_b| <= 2 max |c|)
    // (and only in tiles of at least kBoundMinBlocks key blocks: the pass and its decision
    // cost a few microseconds per tile, which a shorter tile does not win back)
    bool use_bound = false;
    if (a.bstats != nullptr && nblk >= kBoundMinBlocks) {
        const float maxc = __uint_as_float(a.head_words[bh]);
        const float minr = __uint_as_float(a.head_words[a.BH + bh]);
        use_bound = minr < 2.f * maxc;
    }
    const int nbj = use_bound ? (2 * nblk + 127) >> 7 : 0;   // 128-centroid jobs of the bound pass

    if (threadIdx.x == 0) {
        if (rep > 0)   // every phase of the previous tile is complete and nothing is in flight
            for (uint64_t* bb = bars; bb <= mma_done; ++bb) mbar_inval(bb);
        for (int s = 0; s < kSlots; ++s) { mbar_init(&kfull[s], 1); mbar_init(&kempty[s], 1); }
        for (int s = 0; s < kDSlots; ++s) { mbar_init(&kfull2[s], 1); mbar_init(&kempty2[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&s_full2[s], 1); mbar_init(&s_empty2[s], kEwWarps); }
        for (int s = 0; s < kSbuf; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], kEwWarps);
            mbar_init(&pv_sfree[s], 1);
            mbar_init(&p_full[s], kEwWarps);
        }
        mbar_init(o_full, 1);
        mbar_init(q_full, 1);
        mbar_init(dec_bar, 1);
        mbar_init(mma_done, 1);
        misc->decision = 0;
        misc->njobs = 0;
        misc->abort = 0;
        misc->inserts = 0;
        fence_barrier_init();
        // the Q tile goes first, before the block-wide setup
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
        if (use_bound) prefetch_tmap(&tm_c);
        mbar_arrive_expect_tx(q_full, L::kTile);
        for (int at = 0; at < D / 64; ++at)
            tma_load_3d(smem + L::kQ + at * kAtom, &tm_q, at * 64, t * kBlk, bh, q_full);
    }
    for (int b = threadIdx.x; b < T; b += kThreads) { live[b] = 0; cand[b] = 0; }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int sj = 0, dj = 0, kind = kDecSolve;   // P.V-pass tiles, score-pass double slots loaded
            uint32_t dec_phase = 0;
            bool ok = true, first = !use_bound, bound = use_bound;
            SpecJob spec;   // the next pass's first job, loaded before the decision
            // a score-pass job: K blocks b0 and b1 (b1 < 0: none) stacked in one double slot,
            // block h at rows 128h of each [256 rows x 64] atom (the bound pass loads blocks
            // of 128 centroids from `map` the same way)
            auto load_pair = [&](const CUtensorMap* map, int b0, int b1) -> bool {
                const int ds = dj % kDSlots;
                if (!mbar_wait(&kempty2[ds], ((dj / kDSlots) & 1) ^ 1, ab, 1)) return false;
                mbar_arrive_expect_tx(&kfull2[ds], (b1 >= 0 ? 2 : 1) * L::kTile);
                uint8_t* base = smem + L::kRing + ds * 2 * L::kTile;
                for (int at = 0; at < D / 64; ++at) {
                    tma_load_3d(base + at * 2 * kAtom, map, at * 64, b0 * kBlk, bh, &kfull2[ds]);
                    if (b1 >= 0)
                        tma_load_3d(base + at * 2 * kAtom + kAtom, map, at * 64, b1 * kBlk, bh, &kfull2[ds]);
                }
                ++dj;
                return true;
            };
            auto load_tile = [&](const CUtensorMap* map, int b) -> bool {
                const int sl = sj % kSlots;
                if (!mbar_wait(&kempty[sl], ((sj / kSlots) & 1) ^ 1, ab, 1)) return false;
                mbar_arrive_expect_tx(&kfull[sl], L::kTile);
                uint8_t* kb = smem + L::kRing + sl * L::kTile;
                for (int at = 0; at < D / 64; ++at)
                    tma_load_3d(kb + at * kAtom, map, at * 64, b * kBlk, bh, &kfull[sl]);
                ++sj;
                return true;
            };
            while (ok) {
                const bool pv = kind == kDecPv;
                const int njobs = bound ? nbj : first ? nblk : misc->njobs;
                if (bound) {
                    for (int i = 0; i < njobs && ok; i += 2)
                        ok = load_pair(&tm_c, i, (i + 1 < njobs) ? i + 1 : -1);
                } else if (!pv) {
                    // a hit: the first job is in the slot the speculative load filled.  The
                    // guess for the next pass is read now, while this pass's list is stable
                    // (the next decision needs every job of this pass loaded first).
                    const int i0 = spec.hit ? 2 : 0;
                    spec.arm(a.spec && njobs > 0, first, njobs, job_list);
                    for (int i = i0; i < njobs && ok; i += 2) {
                        const int b0 = first ? i : job_list[i];
                        const int b1 = (i + 1 < njobs) ? (first ? i + 1 : job_list[i + 1]) : -1;
                        ok = load_pair(&tm_k, b0, b1);
                    }
                    if (ok && spec.on) {
                        ok = load_pair(&tm_k, spec.b0, spec.b1);
                        spec.use = dj - 1;
                    }
                } else {
                    // the P.V tiles reuse the ring's memory: the speculative job's K blocks
                    // must have been read by its MMA first
                    if (spec.on)
                        ok = mbar_wait(&kempty2[spec.use % kDSlots], (spec.use / kDSlots) & 1, ab, 1);
                    for (int i = 0; i < njobs && ok; ++i) {
                        const int b = job_list[i];
                        ok = load_tile(&tm_k, b);
                        if (ok) ok = load_tile(&tm_v, b);
                    }
                }
                first = bound = false;
                if (!ok || pv) break;
                if (!(ok = mbar_wait(dec_bar, dec_phase, ab, 2))) break;
                dec_phase ^= 1;
                kind = misc->decision;
                spec.check(kind == kDecSolve, misc->njobs, job_list);
            }
            // Copies issued but possibly not consumed land before the CTA ends.
            drain_wait(q_full, 0);
            for (int j = sj - 1; j >= 0 && j >= sj - kSlots; --j) drain_wait(&kfull[j % kSlots], (j / kSlots) & 1);
            for (int j = dj - 1; j >= 0 && j >= dj - kDSlots; --j) drain_wait(&kfull2[j % kDSlots], (j / kDSlots) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idesc_qk2 = idesc_bf16(128, 256, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16(128, D, 0, 1);
            // Descriptors differ only in the start-address field (bits 0-13, address >> 4),
            // so each operand's base descriptor is built once and offsets are added.
            const uint64_t dq = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
            const uint64_t dring = sdesc_sw128(smem_u32(smem + L::kRing), 16, 1024);
            const uint64_t dring_mn = sdesc_sw128(smem_u32(smem + L::kRing), kAtom, 1024);
            bool ok = mbar_wait(q_full, 0, ab, 3);
            tc_fence_after();
            int sjob = 0, kind = kDecSolve;   // score-pass jobs issued (= double slots consumed)
            uint32_t dec_phase = 0;
            bool first = !use_bound, bound = use_bound;
            SpecJob spec;   // the next pass's first job, issued before the decision
            auto wait_tile = [&](int tt) { return mbar_wait(&kfull[tt % kSlots], (tt / kSlots) & 1, ab, 4); };
            auto issue_s = [&](int sb, int tt) {
                const uint64_t dk = dring + ((uint32_t)((tt % kSlots) * L::kTile) >> 4);
                const uint32_t dS = tmem + sbuf_col(sb);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kAtom + (kk & 3) * 32) >> 4;
                    umma_bf16(dS, dq + off, dk + off, idesc_qk, kk > 0);
                }
                umma_commit(&s_full[sb]);
                umma_commit(&kempty[tt % kSlots]);
            };
            // one score-pass job: S of one or two K blocks (one double slot) into an S buffer
            auto issue_job = [&](bool two) -> bool {
                const int sb = sjob & 1, ds = sjob % kDSlots;
                if (!mbar_wait(&kfull2[ds], (sjob / kDSlots) & 1, ab, 4)) return false;
                if (!mbar_wait(&s_empty2[sb], ((sjob >> 1) & 1) ^ 1, ab, 5)) return false;
                tc_fence_after();
                const uint32_t idesc = two ? idesc_qk2 : idesc_qk;
                const uint64_t dk = dring + ((uint32_t)(ds * 2 * L::kTile) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = ((kk >> 2) * kAtom + (kk & 3) * 32) >> 4;
                    const uint32_t ob = ((kk >> 2) * 2 * kAtom + (kk & 3) * 32) >> 4;
                    umma_bf16(tmem + sb * 256, dq + oa, dk + ob, idesc, kk > 0);
                }
                umma_commit(&s_full2[sb]);
                umma_commit(&kempty2[ds]);
                ++sjob;
                return true;
            };
            while (ok) {
                const bool pv = kind == kDecPv;
                const int njobs = bound ? nbj : first ? nblk : misc->njobs;
                const bool was_bound = bound, was_first = first;
                first = bound = false;
                if (!pv) {
                    // a hit: the first job was issued before the decision
                    const int i0 = spec.hit ? 2 : 0;
                    spec.arm(a.spec && njobs > 0 && !was_bound, was_first, njobs, job_list);
                    for (int i = i0; i < njobs && ok; i += 2) ok = issue_job(i + 1 < njobs);
                    if (!ok) break;
                    if (spec.on && !(ok = issue_job(spec.b1 >= 0))) break;
                    if (!(ok = mbar_wait(dec_bar, dec_phase, ab, 7))) break;
                    dec_phase ^= 1;
                    kind = misc->decision;
                    spec.check(kind == kDecSolve, misc->njobs, job_list);
                    continue;
                }
                // P.V pass over the live blocks, with its own barriers and ring counters:
                // ring tiles K_i = 2i, V_i = 2i + 1.
                // S(i) is issued ahead of P.V(i-1), so the score MMA of the next block
                // runs while the elementwise warps turn S(i-1) into P(i-1).  P(i)
                // replaces S(i) in its TMEM buffer, which is free again once P.V(i)
                // is done (pv_sfree).  Every score-pass S buffer was read before the
                // decision that started this pass, so TMEM is free.
                const int job = 0, sj = 0;
                for (int i = 0; i <= njobs && ok; ++i) {
                    if (i < njobs) {
                        const int jb = job + i, sb = jb % SB;
                        if (!(ok = wait_tile(sj + 2 * i))) break;
                        ok = (i < SB) ? mbar_wait(&s_empty[sb], ((jb / SB) & 1) ^ 1, ab, 5)
                                      : mbar_wait(&pv_sfree[sb], ((i / SB) - 1) & 1, ab, 5);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(sb, sj + 2 * i);
                    }
                    if (i > 0) {
                        const int ip = i - 1, sb = (job + ip) % SB, tv = sj + 2 * ip + 1;
                        if (!(ok = wait_tile(tv))) break;
                        // one p_full per buffer: P(i+SB) cannot complete before P.V(i) frees
                        // the buffer, so the elementwise warps never lap this wait
                        if (!(ok = mbar_wait(&p_full[sb], (ip / SB) & 1, ab, 6))) break;
                        tc_fence_after();
                        const uint64_t dv = dring_mn + ((uint32_t)((tv % kSlots) * L::kTile) >> 4);
                        const uint32_t ap = tmem + sbuf_col(sb);
#pragma unroll
                        for (int kk = 0; kk < kBlk / 16; ++kk) {
                            // keys 16kk .. 16kk+15: the half (kk >> 2) that owns them wrote
                            // their P, two per column, at the start of the 32 columns of the
                            // round ((kk >> 1) & 1) that held their scores
                            const uint32_t acol = (kk >> 2) * 64 + ((kk >> 1) & 1) * 32 + (kk & 1) * 8;
                            umma_bf16_ts(tmem + 256, ap + acol, dv + ((kk * 16 * 128) >> 4), idesc_pv,
                                         (ip > 0 || kk > 0) ? 1u : 0u);
                        }
                        if constexpr (OT) {
                            // G (bf16 pairs) sits 16 columns after the P of the same keys
#pragma unroll
                            for (int kk = 0; kk < kBlk / 16; ++kk) {
                                const uint32_t acol = (kk >> 2) * 64 + ((kk >> 1) & 1) * 32 + 16 + (kk & 1) * 8;
                                umma_bf16_ts(tmem + kOtCol, ap + acol, dv + ((kk * 16 * 128) >> 4),
                                             idesc_pv, (ip > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        umma_commit(&pv_sfree[sb]);
                        umma_commit(&kempty[tv % kSlots]);
                    }
                }
                if (ok) umma_commit(o_full);
                break;
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
        // Row histograms in the (then idle) P region: [64 slots][128 rows] u32 words,
        // the low 16 bits counting half 0's columns and the high 16 bits half 1's.
        // Updates are shared-memory reductions (no load-use chain, no lost updates).
        uint32_t* histw = reinterpret_cast<uint32_t*>(smem + L::kP) + row;
        const uint32_t hist_saddr = smem_u32(histw);
        const uint32_t hinc = half ? 65536u : 1u;
        const uint32_t hkeep = half ? 0x0000FFFFu : 0xFFFF0000u;   // red.and mask clearing my half
        const float c63 = cx * kBinsPerUnit;
        // Histogram start (selected by a nonzero a.hist_budget; the default 0 starts
        // every row from the plain bracket, measured faster on B200).
        // Insert budget per tile: a tile whose windows keep filling with scores
        // (dense rows) stops building histograms once the tile has made
        // a.hist_budget inserts after its first block (the first block's window
        // hangs from that block's own maximum and takes in most of it whatever
        // the rows look like), and all its rows start from the plain bracket
        // [m-1, m - n^(1-alpha)].  The decision is tile-wide because the tile runs
        // as many solver passes as its slowest row needs: a histogram kept for some
        // rows only would cost the inserts without saving a pass.  On dense rows
        // the inserts (shared-memory reductions) cost more than the pass they save
        // (measured).  The window width `wbins` is general: counts are complete for
        // every bin inside it, so any bracket taken from it is rigorous.  A budget
        // of 0 builds no histogram (every row starts from the plain bracket), a
        // negative one never stops.
        const int budget = a.hist_budget;
        auto over_budget = [&]() {
            return budget >= 0 && *reinterpret_cast<volatile int*>(&misc->inserts) > budget;
        };
        int n_ins = 0;
        int wbins = budget == 0 ? 0 : kBins;      // window width in bins (0: stopped)
        auto clear_bin = [&](int ab2) { red_shared_and_b32(hist_saddr + (ab2 & (kBins - 1)) * 512, hkeep); };
        float* xch = reinterpret_cast<float*>(smem + L::kXch);   // [k][half][row]
        auto X = [&](int k, int h) -> float& { return xch[(k * 2 + h) * 128 + row]; };
        if (budget != 0) {   // the histogram start is selected
            if (ew < 65) ptab[ew] = entmax_p<GM>((float)ew / kBinsPerUnit, gamma);
            if (half == 0)
                for (int sl = 0; sl < kBins; ++sl) histw[sl * 128] = 0u;
        }
        named_bar(1, kEw);

        float m = -INFINITY;
        int A = kNoBin;
        RowSolver sv;
        sv.tau = 0.f; sv.lo = 0.f; sv.hi = 0.f;
        sv.done = row_valid ? 0 : 1;
        sv.iters = 0;
        const int wi = warp - 2;                  // elementwise warp index 0..7
        int sjob = 0, pass = 0, nlive = 0;
        long long qk_blocks = use_bound ? nbj : nblk, skipped = 0;
        bool ok = true;
        SpecJob spec;
        // a speculative job that is not used: wait for its S, then free the buffer unread
        auto drop_job = [&]() -> bool {
            const int sb = sjob & 1;
            if (!mbar_wait(&s_full2[sb], (sjob >> 1) & 1, ab, 14)) return false;
            tc_fence_after();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty2[sb]);
            ++sjob;
            return true;
        };
        if (use_bound) {
            // ---- bound pass: S_c = Q C^T over the tile's half-block centroids
            // |q| of this row from the swizzled Q tile (a sum of squares does not depend on
            // the order of the 16-byte chunks; lanes start at different chunks so that a
            // warp's loads spread over the banks)
            ok = mbar_wait(q_full, 0, ab, 12);
            float qq = 0.f;
            if (ok) {
                constexpr int kCh = (D == 128) ? 8 : 4;
                const uint8_t* qrow = smem + L::kQ + (D == 128 ? half * kAtom : half * 64) + row * 128;
#pragma unroll
                for (int cc = 0; cc < kCh; ++cc) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(qrow + ((cc + lane) & (kCh - 1)) * 16);
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
                        qq = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, qq));
                    }
                }
            }
            X(1, half) = qq;
            named_bar(1, kEw);
            // rounding of the 2 x 64 squares and the square root: far below 1e-5 relative
            const float qn = sqrtf(qq + X(1, half ^ 1)) * 1.00001f;
            float mlb = -INFINITY;                      // largest lower bound of this half-row
            const float2* bst = a.bstats + (size_t)bh * 2 * T;
            const int wq = (quarter - 2) & 3;           // warp slot of this quarter, key half 0 (+4: 1)
            for (int jj = 0; jj < nbj && ok; jj += 2, ++sjob) {
                const int sb = sjob & 1;
                if (!(ok = mbar_wait(&s_full2[sb], (sjob >> 1) & 1, ab, 13))) break;
                tc_fence_after();
                const int nb2 = (jj + 1 < nbj) ? 2 : 1;
#pragma unroll 1
                for (int h = 0; h < nb2; ++h) {
#pragma unroll 1
                    for (int r = 0; r < 2; ++r) {
                        float s[32];
                        tmem_ld32(lane_base + sb * 256 + h * 128 + c0 + 32 * r, s);
                        tmem_wait_ld();
                        reg_fence<32>(s);
                        if (h == nb2 - 1 && r == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&s_empty2[sb]);
                        }
                        const int cbase = (jj + h) * kBlk + c0 + 32 * r;   // centroid of column 0
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int cent = cbase + c;       // half-block: keys 64 cent .. 64 cent + 63
                            const float2 st = (cent < 2 * nblk) ? __ldg(bst + cent) : make_float2(-1.f, 0.f);
                            const bool has = row_valid && st.x >= 0.f;
                            const bool some = !a.causal || cent * 64 <= i;        // a key of it is admissible
                            const bool every = !a.causal || cent * 64 + 63 <= i;  // all of its keys are
                            const float ub = cx * fmaf(qn, st.x, s[c]);
                            const float lb = cx * fmaf(-qn, st.y, s[c]);
                            if (has && every) mlb = fmaxf(mlb, lb);
                            s[c] = (has && some) ? ub : -INFINITY;
                        }
                        warp_colmax_32(s, lane);
                        const int cent = cbase + lane;    // lane l: the warp's maximum of column l
                        if ((cent >> 1) < nblk) bmw[(cent >> 1) * 8 + wq + 4 * (cent & 1)] = __float2bfloat16_ru(s[0]);
                    }
                }
            }
            ok = named_bar_and(1, kEw, ok);
            if (ok) {
                X(0, half) = mlb;
                named_bar(1, kEw);
                mlb = fmaxf(mlb, X(0, half ^ 1));
                // a block is ruled out for this warp's rows when its upper bound lies at or
                // below the smallest (lower bound of the row max) - 1 <= m - 1 <= tau
                float th = row_valid ? mlb - 1.f : INFINITY;
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) th = fminf(th, __shfl_xor_sync(0xffffffffu, th, o2));
                float* mw = reinterpret_cast<float*>(smem + L::kMw);
                if (lane == 0) mw[wi] = th;
                named_bar(1, kEw);   // every warp's bounds and threshold are in
                for (int b = ew; b < nblk; b += kEw) {
                    bool need = false;
#pragma unroll
                    for (int w8 = 0; w8 < 8; ++w8) {
                        const float thw = mw[w8];
                        need |= __bfloat162float(bmw[b * 8 + w8]) > thw - 1e-4f * fmaxf(1.f, fabsf(thw));
                    }
                    // a block left out holds no u > 0 for any tau the solver visits (tau >= m - 1)
                    if (!need)
                        for (int w8 = 0; w8 < 8; ++w8) bmw[b * 8 + w8] = __float2bfloat16(-INFINITY);
                    live[b] = need ? 1 : 0;
                }
                named_bar(1, kEw);
                if (warp == 2) {
                    int n = 0;
                    for (int base = 0; base < nblk; base += 32) {
                        const int bb = base + lane;
                        const bool f = bb < nblk && live[bb] != 0;
                        const unsigned int msk = __ballot_sync(0xffffffffu, f);
                        if (f) job_list[n + __popc(msk & ((1u << lane) - 1u))] = bb;
                        n += __popc(msk);
                    }
                    if (lane == 0) {
                        misc->njobs = n;
                        misc->decision = kDecSolve;
                        mbar_arrive(dec_bar);
                    }
                }
            }
        }
        for (;; ++pass) {
            float F0 = 0.f, F1 = 0.f, F2 = 0.f;
            int npj = nblk;
            if (pass > 0 || use_bound) {
                if (pass > 0)
                    for (int bb = ew; bb < nblk; bb += kEw) live[bb] = 0;
                named_bar(1, kEw);   // also publishes job_list / njobs of this pass
                npj = misc->njobs;
                qk_blocks += npj;
                if (pass == 0) skipped = nblk - npj;
            }
            // the speculative job issued after the previous pass: on a hit it is this pass's
            // first job (the next S buffer in sequence); on a miss its S is dropped
            if (spec.on && !spec.matches(npj, job_list)) {
                ok = ok && drop_job();
                qk_blocks += spec.b1 >= 0 ? 2 : 1;
            }
            spec.arm(a.spec && npj > 0, pass == 0 && !use_bound, npj, job_list);
            // jobs of two blocks (one 256-column S buffer); the buffer is released after
            // the second block's load
            for (int jj = 0; jj < npj && ok; jj += 2, ++sjob) {
                const int sb = sjob & 1;
                if (!(ok = mbar_wait(&s_full2[sb], (sjob >> 1) & 1, ab, 8))) break;
                tc_fence_after();
                const int nb2 = (jj + 1 < npj) ? 2 : 1;
#pragma unroll 1
                for (int h = 0; h < nb2; ++h) {
                    const int bi = jj + h;      // block index within this pass
                    const int b = (pass == 0 && !use_bound) ? bi : job_list[bi];
                    float s[64];
                    tmem_ld32(lane_base + sb * 256 + h * 128 + c0, &s[0]);
                    tmem_ld32(lane_base + sb * 256 + h * 128 + c0 + 32, &s[32]);
                    tmem_wait_ld();
                    reg_fence<64>(s);
                    if (h == nb2 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&s_empty2[sb]);
                    }
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
                        // per-warp block maximum (rounded up) for skipping in the solver passes
                        float xw = xm;
#pragma unroll
                        for (int o2 = 16; o2 > 0; o2 >>= 1) xw = fmaxf(xw, __shfl_xor_sync(0xffffffffu, xw, o2));
                        if (lane == 0) bmw[b * 8 + wi] = __float2bfloat16_ru(xw);
                        if (xm > m) {
                            m = xm;
                            const int An = abs_bin(m);
                            // bins leaving the window [A-w+1, A]: clear this half's 16 bits
                            if (An > A && wbins > 0) {
                                const int moved = An - A;
                                if (moved >= wbins) {
                                    for (int sl = 0; sl < kBins; ++sl) clear_bin(sl);
                                } else {
                                    for (int k2 = 0; k2 < moved; ++k2) clear_bin(A - wbins + 1 + k2);
                                }
                            }
                            A = An;
                        }
                        // Elements below the window's lowest bin (A-63)/63 <= m-1 are never in the
                        // support; blocks whose maximum is below the window are skipped as a whole.
                        if (wbins > 0 && over_budget()) {
                            for (int sl = 0; sl < kBins; ++sl) clear_bin(sl);   // tile over budget: stop
                            wbins = 0;
                        }
                        const float thr_x = (float)(A - (wbins - 1)) / kBinsPerUnit - 1e-3f;
                        if (__any_sync(0xffffffffu, xm >= thr_x && wbins > 0)) {
                            // bin = floor(x*63) via the 1.5*2^23 rounding trick: rint(x*63 - 1/2)
                            // (an element exactly on an edge may land one bin low, which keeps
                            // the edge bounds valid)
                            const int lo_bin = (wbins > 0) ? A - (wbins - 1) : 0x7FFFFFFF;
#pragma unroll
                            for (int c = 0; c < 64; ++c) {
                                const float y = __fmaf_rn(s[c], c63, -0.5f) + 12582912.0f;
                                const int ab2 = __float_as_int(y) - 0x4B400000;
                                const bool q = ab2 >= lo_bin;
                                if (q) red_shared_add_u32(hist_saddr + (ab2 & (kBins - 1)) * 512, hinc);
                                n_ins += q;
                            }
                            const int wsum = __reduce_add_sync(0xffffffffu, n_ins);
                            if (lane == 0 && wsum && bi > 0) atomicAdd(&misc->inserts, wsum);
                            n_ins = 0;
                        }
                    } else {
                        // two packed accumulator sets (columns c mod 4 < 2 and >= 2)
                        float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, b0 = a0, b1 = a0, b2 = a0;
                        const float2 cx2 = make_float2(cx, cx), nt2 = make_float2(-sv.tau, -sv.tau);
                        if constexpr (GM == 2) {
                            // F2 = #{u > 0} as 64 minus the sign bits: an integer add per
                            // element instead of a compare and a float add (masked columns are
                            // -inf; an exact u = +0 counts, which adds nothing to F0, F1 and
                            // only makes the Halley step and the crossing bound more cautious)
                            unsigned int neg = 0u;
#pragma unroll
                            for (int c = 0; c < 64; c += 4) {
                                const float2 u0 = __ffma2_rn(make_float2(s[c], s[c + 1]), cx2, nt2);
                                const float2 u1 = __ffma2_rn(make_float2(s[c + 2], s[c + 3]), cx2, nt2);
                                neg += (__float_as_uint(u0.x) >> 31) + (__float_as_uint(u0.y) >> 31) +
                                       (__float_as_uint(u1.x) >> 31) + (__float_as_uint(u1.y) >> 31);
                                const float2 p0 = make_float2(fmaxf(u0.x, 0.f), fmaxf(u0.y, 0.f));
                                const float2 p1 = make_float2(fmaxf(u1.x, 0.f), fmaxf(u1.y, 0.f));
                                a0 = __ffma2_rn(p0, p0, a0); a1 = __fadd2_rn(a1, p0);
                                b0 = __ffma2_rn(p1, p1, b0); b1 = __fadd2_rn(b1, p1);
                            }
                            a2 = make_float2((float)(64u - neg), 0.f);
                        } else {
#pragma unroll
                            for (int c = 0; c < 64; c += 4) {
                                entmax_acc_x2<GM>(__ffma2_rn(make_float2(s[c], s[c + 1]), cx2, nt2), gamma, a0, a1, a2);
                                entmax_acc_x2<GM>(__ffma2_rn(make_float2(s[c + 2], s[c + 3]), cx2, nt2), gamma, b0, b1, b2);
                            }
                        }
                        a0 = __fadd2_rn(a0, b0); a1 = __fadd2_rn(a1, b1); a2 = __fadd2_rn(a2, b2);
                        const float f1 = a1.x + a1.y;
                        F0 += a0.x + a0.y; F1 += f1; F2 += a2.x + a2.y;
                        // liveness: t1 = u^(gamma-1) > 0 exactly where u > 0 (up to underflow,
                        // where p = u^gamma is 0 as well)
                        if (__any_sync(0xffffffffu, f1 > 0.f) && lane == 0) live[b] = 1;
                    }
                }
            }
            // A wait that gave up ends the pass for this thread only; the group agrees
            // here, so every thread leaves together and none is left at a barrier.
            ok = named_bar_and(1, kEw, ok);
            if (!ok) break;
            if (pass == 0) {
                // merge the two half-row histograms; the half-0 thread computes the start
                named_bar(1, kEw);   // the tile's insert count is final
                if (wbins > 0 && over_budget()) wbins = 0;
                X(3, half) = m;
                X(2, half) = (float)wbins;
                named_bar(1, kEw);
                const float m_other = X(3, half ^ 1);
                const int w_other = (int)X(2, half ^ 1);
                const bool over = (wbins == 0) || (w_other == 0);
                if (half == 0 && row_valid && over) {
                    // plain bracket [m-1, m - n^(1-alpha)], start at its midpoint, or at
                    // m - (the gap of the nearest sampled row) when the start is calibrated
                    const float mr = fmaxf(m, m_other);
                    sv.lo = mr - 1.f;
                    sv.hi = fmaxf(sv.lo, mr - exp2f((1.f - a.alpha) * __log2f((float)key_end)));
                    sv.tau = 0.5f * (sv.lo + sv.hi);
                    if (a.gap) {
                        const int sr = min(max((int)(((long long)(i + 1) * kCalRows + N / 2) / N) - 1, 0), kCalRows - 1);
                        const float g = a.gap[(size_t)bh * kCalRows + sr];
                        // kCalMargin below it: from below, Halley approaches the root with
                        // upward steps, whose unevaluated stops have the rigorous crossing
                        // bound (a start just above the root ends on a downward stop, which
                        // on clustered keys can miss the check)
                        if (g >= 0.f) sv.tau = fminf(fmaxf(mr - g - kCalMargin, sv.lo), sv.hi);
                    }
                }
                named_bar(1, kEw);
                if (half == 0 && row_valid && over) {
                    X(0, 0) = sv.lo; X(1, 0) = sv.hi; X(2, 0) = sv.tau;
                } else if (half == 0 && row_valid) {
                    const int A0 = A, w0 = wbins;
                    const int A1 = (m_other == -INFINITY) ? kNoBin : abs_bin(m_other), w1 = w_other;
                    const float mr = fmaxf(m, m_other);
                    const int Ar = abs_bin(mr);
                    // edges are usable only where both halves count every element above them
                    const int ebot = max(A0 == kNoBin ? kNoBin : A0 - w0 + 1,
                                         A1 == kNoBin ? kNoBin : A1 - w1 + 1);
                    auto count = [&](int ab2) -> unsigned int {
                        const uint32_t w = histw[(ab2 & (kBins - 1)) * 128];
                        unsigned int c = 0;
                        if (ab2 <= A0 && ab2 >= A0 - (w0 - 1)) c += w & 0xFFFFu;
                        if (ab2 <= A1 && ab2 >= A1 - (w1 - 1)) c += w >> 16;
                        return c;
                    };
                    hist_start_fn<GM>(count, Ar, max(ebot, Ar - (kBins - 1)), mr, key_end, a.alpha,
                                      gamma, ptab, sv.lo, sv.hi, sv.tau);
                    X(0, 0) = sv.lo; X(1, 0) = sv.hi; X(2, 0) = sv.tau;
                }
                named_bar(1, kEw);
                if (half == 1 && row_valid) { sv.lo = X(0, 0); sv.hi = X(1, 0); sv.tau = X(2, 0); }
            } else {
                X(0, half) = F0; X(1, half) = F1; X(2, half) = F2;
                named_bar(1, kEw);
                const float G0 = F0 + X(0, half ^ 1), G1 = F1 + X(1, half ^ 1), G2 = F2 + X(2, half ^ 1);
                solver_update(sv, G0, G1, G2, gamma, gamma == 1.f, pass, a.ftol, a.stol, acc);
            }
            const int all = named_bar_and(1, kEw, sv.done) && pass > 0;
            // after an unverified downward step the support may reach blocks that were not
            // live in this pass: the P.V pass then also visits the candidates at the final
            // tau (a uniform barrier, since `all` is)
            const bool any_down = all && !named_bar_and(1, kEw, !(row_valid && sv.down));
            const uint8_t tag = (uint8_t)(pass + 2);
            if (!all || any_down) {
                // Candidates for the next pass: a block can hold u > 0 for a row of this
                // warp only if the warp's block maximum exceeds the warp's smallest tau.
                float th = row_valid ? sv.tau : INFINITY;
#pragma unroll
                for (int o2 = 16; o2 > 0; o2 >>= 1) th = fminf(th, __shfl_xor_sync(0xffffffffu, th, o2));
                th -= 4e-7f * fmaxf(1.f, fabsf(th));
                for (int bb = lane; bb < nblk; bb += 32)
                    if (__bfloat162float(bmw[bb * 8 + wi]) > th) cand[bb] = tag;
                named_bar(1, kEw);
            }
            if (warp == 2) {
                // compact the next pass's blocks: live ones for P.V, else the candidates
                int n = 0;
                for (int base = 0; base < nblk; base += 32) {
                    const int bb = base + lane;
                    const bool f = bb < nblk && (all ? (live[bb] != 0 || (any_down && cand[bb] == tag))
                                                     : cand[bb] == tag);
                    const unsigned int msk = __ballot_sync(0xffffffffu, f);
                    if (f) job_list[n + __popc(msk & ((1u << lane) - 1u))] = bb;
                    n += __popc(msk);
                }
                if (lane == 0) {
                    misc->njobs = n;
                    misc->decision = all ? kDecPv : kDecSolve;
                    mbar_arrive(dec_bar);
                }
            }
            if (all) break;
        }
        // the P.V pass follows: a speculative job issued after the last pass is dropped
        if (spec.on) {
            ok = ok && drop_job();
            qk_blocks += spec.b1 >= 0 ? 2 : 1;
        }
        const int npass = pass;
        [[maybe_unused]] float2 sg2 = make_float2(0.f, 0.f);   // sum_j g of this half-row (OT)
        float2 fsum2 = make_float2(0.f, 0.f);                   // sum_j p of this half-row
        int lnum = 0;                                           // support-list entries of this half-row
        if (ok) {
            named_bar(1, kEw);   // job_list / njobs of the P.V pass visible to the group
            nlive = misc->njobs;
            for (int li = 0; li < nlive; ++li) {
                const int b = job_list[li];
                const int sb = li % SB;   // the P.V pass counts its own jobs
                if (!(ok = mbar_wait(&s_full[sb], (li / SB) & 1, ab, 9))) break;
                tc_fence_after();
                const int nv = key_end - b * kBlk - c0;   // valid columns of this thread: c < nv
                const bool full_blk = __all_sync(0xffffffffu, nv >= 64);
                const float2 cx2 = make_float2(cx, cx), nt2 = make_float2(-sv.tau, -sv.tau);
                uint32_t nzb = 0u;   // OR of this thread's bf16 p bits: nonzero iff some p > 0
                // two rounds of 32 keys, each loaded, turned into P (and G) and stored over its
                // own 32 S columns: P of keys c0 + 32 hc + 2k, +1 in column c0 + 32 hc + k
                // (k < 16), G with otilde 16 columns further on; one copy of the round's code
#pragma unroll 1
                for (int hc = 0; hc < 2; ++hc) {
                    float s[32];
                    tmem_ld32(lane_base + sbuf_col(sb) + c0 + 32 * hc, s);
                    tmem_wait_ld();
                    reg_fence<32>(s);
                    if (!full_blk) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) s[c] = (32 * hc + c < nv) ? s[c] : -INFINITY;
                    }
                    uint32_t pk[16];
                    [[maybe_unused]] uint32_t gk[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float2 u2 = __ffma2_rn(make_float2(s[c], s[c + 1]), cx2, nt2);
                        if constexpr (OT) {
                            float2 p2, g2;
                            entmax_pg_x2<GM>(u2, gamma, p2, g2);
                            fsum2 = __fadd2_rn(fsum2, p2);
                            const __nv_bfloat162 hp = __floats2bfloat162_rn(p2.x, p2.y);
                            const __nv_bfloat162 hg = __floats2bfloat162_rn(g2.x, g2.y);
                            pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
                            gk[c >> 1] = *reinterpret_cast<const uint32_t*>(&hg);
                            // sum the rounded weights the G.V product uses: otilde is then
                            // a weighted mean whose weights sum to one
                            sg2 = __fadd2_rn(sg2, __bfloat1622float2(hg));
                        } else {
                            const float2 p2 = entmax_p_x2<GM>(u2, gamma);
                            fsum2 = __fadd2_rn(fsum2, p2);
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p2.x, p2.y);
                            pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
                        }
                    }
                    uint32_t nzw = 0u;
#pragma unroll
                    for (int w = 0; w < 16; ++w) nzw |= pk[w];
                    nzb |= nzw;
                    if (a.list_n && __any_sync(0xffffffffu, nzw != 0u)) {
                        // support list of the row: (key, u) for every p > 0 of these keys (a
                        // packed pair is nonzero iff one of its p is).  Compact on purpose: the
                        // round's u go to this thread's column of the (by now idle) histogram
                        // area and a loop visits the nonzero words only.  Each half-row counts
                        // its own entries: half 0 fills the list from the front, half 1 from
                        // the back, and the epilogue closes the gap.
                        float* scr = reinterpret_cast<float*>(smem + L::kP) + ew;
#pragma unroll
                        for (int c = 0; c < 32; ++c) scr[c * kEw] = __fmaf_rn(s[c], cx, -sv.tau);
                        uint32_t wm = 0u;
#pragma unroll
                        for (int w = 0; w < 16; ++w) wm |= (pk[w] != 0u ? 1u : 0u) << w;
                        const size_t lbase = ((size_t)bh * N + i) * kListCap;
                        while (wm != 0u) {
                            const int w = __ffs(wm) - 1;
                            wm &= wm - 1u;
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float u = scr[(2 * w + e) * kEw];
                                if (u > 0.f) {
                                    if (lnum < kListCap) {
                                        const int slot = half ? kListCap - 1 - lnum : lnum;
                                        a.list_key[lbase + slot] = b * kBlk + c0 + 32 * hc + 2 * w + e;
                                        a.list_u[lbase + slot] = u;
                                    }
                                    ++lnum;
                                }
                            }
                        }
                    }
                    tmem_st16(lane_base + sbuf_col(sb) + c0 + 32 * hc, pk);
                    if constexpr (OT) tmem_st16(lane_base + sbuf_col(sb) + c0 + 32 * hc + 16, gk);
                }
                // the block mask: some p > 0 in the block at the final tau (a bf16 p is
                // nonzero exactly when its bits are)
                if (__any_sync(0xffffffffu, nzb != 0u) && lane == 0) cand[b] = kPvLive;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
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
        // d = 32 runs as D = 64 (zero upper columns): the half holding columns 32..63 stores nothing
        const bool store_half = half * DH < a.dr;
        if (row_valid && store_half) {
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + ((size_t)bh * N + i) * a.dr + half * DH;
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
        }
        if (row_valid) {
            if (half == 0) {
                a.tau[(size_t)bh * N + i] = sv.tau;
                if (a.iters) a.iters[(size_t)bh * N + i] = (uint8_t)sv.iters;
            }
        }
        if constexpr (OT) {
            // otilde = G.V / sum_j g; the halves' sums meet in shared memory (every
            // elementwise thread reaches this barrier once, also after an abort)
            X(0, half) = sg2.x + sg2.y;
            named_bar(1, kEw);
            const float sg = X(0, 0) + X(0, 1);
            if (ok && nlive > 0) {
#pragma unroll
                for (int c = 0; c < DH / 32; ++c)
                    tmem_ld32(lane_base + kOtCol + half * DH + c * 32, &o[c * 32]);
                tmem_wait_ld();
                reg_fence<DH>(o);
            } else {
#pragma unroll
                for (int c = 0; c < DH; ++c) o[c] = 0.f;
            }
            const float rs = sg > 0.f ? 1.f / sg : 0.f;
            if (row_valid && store_half) {
                float* orow = a.otilde + ((size_t)bh * N + i) * a.dr + half * DH;
#pragma unroll
                for (int c = 0; c < DH; c += 4)
                    *reinterpret_cast<float4*>(orow + c) =
                        make_float4(o[c] * rs, o[c + 1] * rs, o[c + 2] * rs, o[c + 3] * rs);
            }
        }
        if (a.list_n) {
            // the row's list: half 0's entries at the front, half 1's at the back; half 1
            // moves its entries to follow half 0's, in increasing order (each destination
            // n0 + e lies at or below its source 16 - n1 + e and below every later source)
            reinterpret_cast<int*>(xch)[(2 * 2 + half) * 128 + row] = lnum;
            named_bar(1, kEw);
            const int n0 = reinterpret_cast<int*>(xch)[(2 * 2 + 0) * 128 + row];
            const int n1 = reinterpret_cast<int*>(xch)[(2 * 2 + 1) * 128 + row];
            const bool fits = ok && n0 + n1 <= kListCap;
            if (row_valid && half == 1 && fits) {
                const size_t lbase = ((size_t)bh * N + i) * kListCap;
                for (int e = 0; e < n1; ++e) {
                    a.list_key[lbase + n0 + e] = a.list_key[lbase + kListCap - n1 + e];
                    a.list_u[lbase + n0 + e] = a.list_u[lbase + kListCap - n1 + e];
                }
            }
            if (row_valid && half == 0) a.list_n[(size_t)bh * N + i] = fits ? (uint8_t)(n0 + n1) : kListOver;
        }
        // verification of the rows that stopped on an unevaluated step: f at the final tau
        // is sum_j p_ij - 1, summed above over a superset of the support; a tile where one
        // such row misses the tolerance is solved again by the second launch
        X(3, half) = fsum2.x + fsum2.y;
        named_bar(1, kEw);   // also: every warp's P.V-pass mask flags are in
        const float f_end = X(3, 0) + X(3, 1) - 1.f;
        const bool bad = ok && row_valid && sv.unv && !(fabsf(f_end) <= a.verify_tol);
        const bool tile_bad = !named_bar_and(1, kEw, !bad);
        uint8_t* mrow = a.mask + ((size_t)bh * T + t) * T;
        for (int bb = ew; bb < T; bb += kEw) mrow[bb] = (bb < nblk && cand[bb] == kPvLive) ? 1 : 0;
        if (tile_bad) {
            // every output of this tile is written before the entry is: a CTA that claims
            // it writes them again, and its writes must land last
            named_bar(1, kEw);
            if (ew == 0) {
                __threadfence();
                a.fail_list[atomicAdd(&a.hdr->fail_count, 1u)] = bh * T + t + 1;   // 0: not written yet
                __threadfence();
            }
        }
        if (ew == 0) {
            atomicAdd(&a.hdr->counters[kCtrQkBlocks], (unsigned long long)qk_blocks);
            atomicAdd(&a.hdr->counters[kCtrPvBlocks], (unsigned long long)nlive);
            atomicAdd(&a.hdr->counters[kCtrPasses], (unsigned long long)npass);
            atomicAdd(&a.hdr->counters[kCtrTiles], 1ull);
            if (OT) atomicAdd(&a.hdr->counters[kCtrGvBlocks], (unsigned long long)nlive);
            if (skipped) atomicAdd(&a.hdr->counters[kCtrSkipped], (unsigned long long)skipped);
        }
    }

    tc_fence_before();
    __syncthreads();
    // next: a tile from the failure list, claimed by whichever CTA is free.  A CTA that
    // finishes its own tile takes the entries appended so far; the last CTA to finish
    // its own tile sees every entry (each failing tile appends before it counts itself
    // finished) and leaves only when all are claimed.  Re-solved tiles stop at evaluated
    // points only, so they never append.  An entry holds its tile + 1 (the host zeroes the
    // list), and a claimer waits (bounded) for its entry to be written.
    if (threadIdx.x == 0) {
        int next = -1;
        if (!misc->abort) {
            if (!fixing) {
                __threadfence();
                atomicAdd(&a.hdr->tile_counter, 1u);
                __threadfence();
            }
            volatile unsigned int* vcount = &a.hdr->fail_count;
            volatile unsigned int* vclaim = &a.hdr->claim;
            for (;;) {
                const unsigned int c = *vclaim;
                if (c >= *vcount) break;
                if (atomicCAS(&a.hdr->claim, c, c + 1u) != c) continue;
                const volatile int* entry = reinterpret_cast<volatile int*>(a.fail_list) + c;
                const uint64_t t0 = globaltimer_ns();
                int e = *entry;
                while (e == 0 && globaltimer_ns() - t0 <= kWaitLimitNs) e = *entry;
                if (e == 0) {   // never written: give up like any other bounded wait
                    atomicExch(&a.hdr->status, 1u);
                    atomicExch(&a.hdr->timeout_site, 15u);
                }
                next = e - 1;
                break;
            }
        }
        misc->next = next;
    }
    __syncthreads();
    const int next = misc->next;
    if (next < 0) break;
    fixing = true;
    cur_bh = next / T;
    cur_t = next - cur_bh * T;
    tc_fence_after();
    }   // tiles of this CTA

    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(misc->tmem_base, kTmemCols);
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

// [BH][N][D] bf16 tensor, box {64, box_rows, 1}, 128-byte swizzle, zero fill out of bounds
// (D = 32: the box's columns 32..63 lie outside the tensor and arrive as zeros).
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

// ------------------------------------------------------------------ key-block bounds
// One warp per 64-key half-block hb of head bh (keys 64 hb .. 64 hb + 63 below N):
//   c   = the mean of its keys, rounded to bf16 (stored: the bound pass multiplies it
//         with Q on the tensor cores),
//   r   = max_j |k_j - c|, so q.k_j <= q.c + |q| r (Cauchy-Schwarz),
//   dc  = |mean - c|, so max_j q.k_j >= q.mean >= q.c - |q| dc.
// The computed scores differ from the exact ones by the fp32 accumulation of the
// tensor-core products, at most d 2^-23 |q| |k| each; with e = 2 d 2^-23 (twice that
// bound) and |k_j| <= |c| + r the stored terms R = r + e (2|c| + r) and
// L = dc + e (2|c| + r) + 1e-4 (|c| + r) (the last term for the fp32 mean) cover both
// the score and the centroid product.  R < 0 marks a half-block with no key.  The
// head's max |c| and min R go to head_words by atomic max / min on the float bits
// (non-negative floats order like their bit patterns): head_words[bh] and
// head_words[BH + bh], BH = gridDim.y.
template <int D>
__global__ void __launch_bounds__(128) block_stats_kernel(const __nv_bfloat16* __restrict__ k, int N, int T2,
                                                          __nv_bfloat16* __restrict__ cent,
                                                          float2* __restrict__ bstats,
                                                          unsigned int* __restrict__ head_words) {
    constexpr int PL = D / 32;                 // dimensions per lane
    const int lane = threadIdx.x & 31;
    const int hb = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int bh = blockIdx.y;
    if (hb >= T2) return;
    const int j0 = hb * 64;
    const int nk = min(64, N - j0);
    const __nv_bfloat16* kr = k + ((size_t)bh * N + max(j0, 0)) * D + lane * PL;
    __nv_bfloat16* cr = cent + ((size_t)bh * T2 + hb) * D + lane * PL;
    auto load = [&](int j, float* x) {
        if (PL == 1) {
            x[0] = __bfloat162float(kr[(size_t)j * D]);
        } else if (PL == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(kr + (size_t)j * D);
            const float2 a2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
            const float2 b2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
            x[0] = a2.x; x[1] = a2.y; x[2] = b2.x; x[3] = b2.y;
        } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(kr + (size_t)j * D);
            const float2 a2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
            x[0] = a2.x; x[1] = a2.y;
        }
    };
    auto wsum = [](float x) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        return x;
    };
    if (nk <= 0) {
#pragma unroll
        for (int e = 0; e < PL; ++e) cr[e] = __float2bfloat16(0.f);
        if (lane == 0) bstats[(size_t)bh * T2 + hb] = make_float2(-1.f, 0.f);
        return;
    }
    float sum[PL];
#pragma unroll
    for (int e = 0; e < PL; ++e) sum[e] = 0.f;
    for (int j = 0; j < nk; ++j) {
        float x[PL];
        load(j, x);
#pragma unroll
        for (int e = 0; e < PL; ++e) sum[e] += x[e];
    }
    float c[PL], dc2 = 0.f, c2 = 0.f;
#pragma unroll
    for (int e = 0; e < PL; ++e) {
        const float mean = sum[e] / (float)nk;
        const __nv_bfloat16 cb = __float2bfloat16_rn(mean);
        cr[e] = cb;
        c[e] = __bfloat162float(cb);
        dc2 = fmaf(mean - c[e], mean - c[e], dc2);
        c2 = fmaf(c[e], c[e], c2);
    }
    dc2 = wsum(dc2);
    c2 = wsum(c2);
    float r2 = 0.f;
    for (int j = 0; j < nk; ++j) {
        float x[PL], d2 = 0.f;
        load(j, x);
#pragma unroll
        for (int e = 0; e < PL; ++e) d2 = fmaf(x[e] - c[e], x[e] - c[e], d2);
        r2 = fmaxf(r2, wsum(d2));
    }
    // fp32 sums of at most d squares: relative error below d 2^-24, halved by the root
    const float slack = 1.f + 4e-5f;
    const float r = sqrtf(r2) * slack, nc = sqrtf(c2) * slack, dc = sqrtf(dc2) * slack;
    const float e = 2.f * (float)D * 1.1920929e-7f;   // 2 d 2^-23
    const float R = (r + e * (2.f * nc + r)) * slack;
    const float Lm = (dc + e * (2.f * nc + r) + 1e-4f * (nc + r)) * slack;
    if (lane == 0) {
        bstats[(size_t)bh * T2 + hb] = make_float2(R, Lm);
        atomicMax(&head_words[bh], __float_as_uint(nc));
        atomicMin(&head_words[gridDim.y + bh], __float_as_uint(R));
    }
}

// ---------------------------------------------------------------- calibrated start
// Not on the pages.  A tile runs as many solver passes as its slowest row, and the plain
// bracket's midpoint m - (1 + n^(1-alpha))/2 sits far from the root where the gap m - tau
// is small (clustered keys: ~0.27 against ~0.5).  Before the forward, kCalRows query rows
// per head are solved exactly; each row of the forward then starts at m - (the gap of the
// nearest sampled row), inside its own bracket.  The result is a deterministic function of
// the inputs; only the path of the solver changes, not its stop rule.
//
// calib_scores_kernel: grid (ceil(N / 256), BH), one key per thread: x = cx q_s . k_j for
// every sampled row s with j in its (causal) range, q_s staged in shared memory as floats.
constexpr int kCalThreads = 256;

__global__ void __launch_bounds__(kCalThreads) calib_scores_kernel(const FwdArgs a) {
    extern __shared__ float qs[];   // [kCalRows][dr]
    const int bh = blockIdx.y, N = a.N, dr = a.dr;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + (size_t)bh * N * dr;
    for (int i = threadIdx.x; i < kCalRows * dr; i += kCalThreads) {
        const int sidx = i / dr, c = i - sidx * dr;
        const int p = (sidx + 1) * N / kCalRows - 1;
        qs[i] = __bfloat162float(q[(size_t)p * dr + c]);
    }
    __syncthreads();
    const int j = blockIdx.x * kCalThreads + threadIdx.x;
    if (j >= N) return;
    // causal: the sampled rows before this CTA's first key take none of its keys (the
    // rows are in increasing order, so those are the first r0 of them)
    int r0 = 0;
    if (a.causal)
        while (r0 < kCalRows && (r0 + 1) * N / kCalRows - 1 < (int)(blockIdx.x * kCalThreads)) ++r0;
    const __nv_bfloat16* kr = static_cast<const __nv_bfloat16*>(a.k) + ((size_t)bh * N + j) * dr;
    float acc[kCalRows];
#pragma unroll
    for (int r = 0; r < kCalRows; ++r) acc[r] = 0.f;
    for (int c = 0; c < dr; c += 8) {
        const uint4 w = *reinterpret_cast<const uint4*>(kr + c);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        float kv[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
            kv[2 * e] = f.x;
            kv[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int r = 0; r < kCalRows; ++r) {
            if (r < r0) continue;
            const float4 qa = *reinterpret_cast<const float4*>(qs + r * dr + c);
            const float4 qb = *reinterpret_cast<const float4*>(qs + r * dr + c + 4);
            acc[r] = fmaf(qa.x, kv[0], acc[r]); acc[r] = fmaf(qa.y, kv[1], acc[r]);
            acc[r] = fmaf(qa.z, kv[2], acc[r]); acc[r] = fmaf(qa.w, kv[3], acc[r]);
            acc[r] = fmaf(qb.x, kv[4], acc[r]); acc[r] = fmaf(qb.y, kv[5], acc[r]);
            acc[r] = fmaf(qb.z, kv[6], acc[r]); acc[r] = fmaf(qb.w, kv[7], acc[r]);
        }
    }
    float* out = a.calib + (size_t)bh * kCalRows * N;
#pragma unroll
    for (int r = 0; r < kCalRows; ++r) {
        const int p = (r + 1) * N / kCalRows - 1;
        if (!a.causal || j <= p) out[(size_t)r * N + j] = a.cx * acc[r];
    }
}

// calib_solve_kernel: grid (kCalRows, BH), one CTA per sampled row: the row maximum, then
// Halley-bisection passes from the plain bracket with evaluated stops only (the forward's
// stop rule), the sums reduced over the CTA; writes gap = m - tau.
template <int GM>
__global__ void __launch_bounds__(kCalThreads) calib_solve_kernel(const FwdArgs a) {
    __shared__ float red[3][kCalThreads / 32];
    __shared__ float bc[2];
    const int r = blockIdx.x, bh = blockIdx.y, N = a.N;
    const int p = (r + 1) * N / kCalRows - 1;
    const int n = a.causal ? p + 1 : N;
    const float* x = a.calib + ((size_t)bh * kCalRows + r) * N;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    auto reduce3 = [&](float& u, float& v, float& w, bool is_max) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            if (is_max) {
                u = fmaxf(u, __shfl_xor_sync(0xffffffffu, u, o));
            } else {
                u += __shfl_xor_sync(0xffffffffu, u, o);
                v += __shfl_xor_sync(0xffffffffu, v, o);
                w += __shfl_xor_sync(0xffffffffu, w, o);
            }
        }
        __syncthreads();   // the previous use of red is finished
        if (lane == 0) { red[0][warp] = u; red[1][warp] = v; red[2][warp] = w; }
        __syncthreads();
        u = red[0][0]; v = red[1][0]; w = red[2][0];
#pragma unroll
        for (int i = 1; i < kCalThreads / 32; ++i) {
            if (is_max) u = fmaxf(u, red[0][i]);
            else { u += red[0][i]; v += red[1][i]; w += red[2][i]; }
        }
    };
    float m = -INFINITY, d1 = 0.f, d2 = 0.f;
    for (int j = threadIdx.x; j < n; j += kCalThreads) m = fmaxf(m, x[j]);
    reduce3(m, d1, d2, true);
    RowSolver sv;
    sv.done = 0;
    sv.iters = 0;
    sv.lo = m - 1.f;
    sv.hi = fmaxf(sv.lo, m - exp2f((1.f - a.alpha) * __log2f((float)n)));
    sv.tau = 0.5f * (sv.lo + sv.hi);
    const float gamma = a.gamma;
    for (int pass = 1;; ++pass) {
        float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0;
        const float2 nt2 = make_float2(-sv.tau, -sv.tau);
        for (int j = 2 * threadIdx.x; j < n; j += 2 * kCalThreads) {
            const float2 xx = make_float2(x[j], j + 1 < n ? x[j + 1] : -INFINITY);
            entmax_acc_x2<GM>(__fadd2_rn(xx, nt2), gamma, s0, s1, s2);
        }
        float F0 = s0.x + s0.y, F1 = s1.x + s1.y, F2 = s2.x + s2.y;
        reduce3(F0, F1, F2, false);
        if (threadIdx.x == 0) {
            solver_update(sv, F0, F1, F2, gamma, gamma == 1.f, pass, a.ftol, a.stol);
            bc[0] = sv.tau;
            bc[1] = sv.done ? 1.f : 0.f;
        }
        __syncthreads();
        sv.tau = bc[0];
        if (bc[1] != 0.f) break;
    }
    if (threadIdx.x == 0) a.gap[(size_t)bh * kCalRows + r] = m - sv.tau;
}

template <int D, int GM>
static cudaError_t launch_tc_fwd(const CUtensorMap& mq, const CUtensorMap& mk,
                                 const CUtensorMap& mv, const CUtensorMap& mc, const FwdArgs& a,
                                 cudaStream_t s) {
    // the calibrated start's two kernels run beside the block statistics (both only read
    // the inputs), on a stream forked from `s` and joined before the forward
    cudaStream_t side = (a.gap && a.bstats) ? side_stream() : nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    if (side && (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
                 cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess ||
                 cudaEventRecord(fork, s) != cudaSuccess || cudaStreamWaitEvent(side, fork, 0) != cudaSuccess))
        side = nullptr;   // then on `s`, one after the other
    if (!side) {
        if (fork) cudaEventDestroy(fork);
        if (join) cudaEventDestroy(join);
    }
    if (a.gap) {
        cudaStream_t cs = side ? side : s;
        const size_t qsm = (size_t)kCalRows * a.dr * sizeof(float);
        calib_scores_kernel<<<dim3((a.N + kCalThreads - 1) / kCalThreads, a.BH), kCalThreads, qsm, cs>>>(a);
        calib_solve_kernel<GM><<<dim3(kCalRows, a.BH), kCalThreads, 0, cs>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess && side) e = cudaEventRecord(join, side);
        if (e != cudaSuccess) return e;
    }
    if (a.bstats) {
        const int T2 = 2 * a.T;
        const dim3 grid((T2 + 3) / 4, a.BH);
        const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(a.k);
        __nv_bfloat16* cc = static_cast<__nv_bfloat16*>(a.cent);
        if (a.dr == 32)
            block_stats_kernel<32><<<grid, 128, 0, s>>>(kk, a.N, T2, cc, a.bstats, a.head_words);
        else
            block_stats_kernel<D><<<grid, 128, 0, s>>>(kk, a.N, T2, cc, a.bstats, a.head_words);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (side) {
        cudaError_t e = cudaStreamWaitEvent(s, join, 0);
        cudaEventDestroy(fork);
        cudaEventDestroy(join);
        if (e != cudaSuccess) return e;
    }
    const size_t sm = Layout<D>::bytes(a.T);
    auto kern = a.otilde ? tc_fwd_kernel<D, GM, true> : tc_fwd_kernel<D, GM, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.BH, a.T), kThreads, sm, s>>>(mq, mk, mv, mc, a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t tc_fwd_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mc, const FwdArgs& a, int gm, cudaStream_t s) {
    switch (gm) {
        case 1: return launch_tc_fwd<D, 1>(mq, mk, mv, mc, a, s);
        case 2: return launch_tc_fwd<D, 2>(mq, mk, mv, mc, a, s);
        case 4: return launch_tc_fwd<D, 4>(mq, mk, mv, mc, a, s);
        default: return launch_tc_fwd<D, 0>(mq, mk, mv, mc, a, s);
    }
}

cudaError_t tc_fwd(const FwdArgs& a, int d, int gm, cudaStream_t s, const char** why) {
    CUtensorMap mq, mk, mv, mc;
    // the centroids [BH][2T][d] load like K blocks (128 of them per box); without the
    // bound pass the map is never used and points at K
    const bool okc = a.cent ? make_tmap_bf16(&mc, a.cent, a.BH, 2 * a.T, d) : make_tmap_bf16(&mc, a.k, a.BH, a.N, d);
    if (!make_tmap_bf16(&mq, a.q, a.BH, a.N, d) || !make_tmap_bf16(&mk, a.k, a.BH, a.N, d) ||
        !make_tmap_bf16(&mv, a.v, a.BH, a.N, d) || !okc) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    // d = 32 runs on the d = 64 kernel: its tiles hold zeros in columns 32..63, which add
    // nothing to q.k, make O's upper columns 0 and are not stored
    return d == 128 ? tc_fwd_d<128>(mq, mk, mv, mc, a, gm, s) : tc_fwd_d<64>(mq, mk, mv, mc, a, gm, s);
}

}  // namespace ent
