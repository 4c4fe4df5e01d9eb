// tc_lists.cu -- the support-list backward for query tiles whose rows have few
// nonzeros ("AdaSplash: Adaptive Sparse Flash Attention", Technical Deep Dive /
// Exploiting Sparsity, at a finer grain than 128 x 128 blocks).
//
// The forward's P.V pass can record, per query row, the keys j with p_ij > 0 and
// their u_ij = x_ij - tau_i (ent_attn_fwd_lists, up to kListCap per row).  Where
// every row of a query tile has such a list, the backward of that tile needs no
// score recomputation at all: with g = u^(gamma-1), p = u^gamma,
//     dP_ij = dO_i . v_j,   delta_i = sum_j g_ij dP_ij / sum_j g_ij,
//     dS_ij = g_ij (dP_ij - delta_i),
//     dQ_i = scale sum_j dS_ij k_j,  dK_j += scale dS_ij q_i,  dV_j += p_ij dO_i,
// summed over the listed keys only (the same formulas as the block kernels, which
// sum over every key of the live blocks; the unlisted keys have g = p = 0).  One warp
// per row: the lanes hold the row's list entries for the scalars and the head
// dimension for the vectors; dK and dV contributions go to fp32 accumulators by
// vector atomics (another tile's rows may list the same key), which the dkv kernel
// adds when it stores dK and dV.
#include "kernels.h"

namespace ent {

namespace {

template <int PL>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float* x) {
    if (PL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else if (PL == 2) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        x[0] = a.x; x[1] = a.y;
    } else {
        x[0] = __bfloat162float(*p);
    }
}

template <int PL>
__device__ __forceinline__ void atomic_add_row(float* dst, const float* x) {
    if (PL == 4) atomicAdd(reinterpret_cast<float4*>(dst), make_float4(x[0], x[1], x[2], x[3]));
    else if (PL == 2) atomicAdd(reinterpret_cast<float2*>(dst), make_float2(x[0], x[1]));
    else atomicAdd(dst, x[0]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace

template <int DR, int GM>
__global__ void __launch_bounds__(256) list_bwd_kernel(const BwdArgs a) {
    constexpr int PL = DR / 32;    // head-dimension elements per lane
    const int t = blockIdx.x, bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.N, r0 = t * kBlk;
    // the tile is the list kernel's only if every one of its rows has a list
    bool has = true;
    if (threadIdx.x < kBlk && r0 + threadIdx.x < N)
        has = a.list_n[(size_t)bh * N + r0 + threadIdx.x] != kListOver;
    const int all = __syncthreads_and(has);
    if (threadIdx.x == 0) a.tile_list[(size_t)bh * a.T + t] = all ? 1 : 0;
    if (!all) return;
    const float gamma = a.gamma, scale = a.scale;
    const __nv_bfloat16* Kp = static_cast<const __nv_bfloat16*>(a.k);
    const __nv_bfloat16* Vp = static_cast<const __nv_bfloat16*>(a.v);
    int entries = 0;   // list entries this warp handled
    for (int rr = warp; rr < kBlk; rr += 8) {
        const int i = r0 + rr;
        if (i >= N) break;
        const size_t row = (size_t)bh * N + i;
        const int n = a.list_n[row];
        entries += n;
        int j = 0;
        float g = 0.f, p = 0.f;
        if (lane < n) {
            j = a.list_key[row * kListCap + lane];
            const float u = a.list_u[row * kListCap + lane];
            float t2;
            entmax_terms<GM>(u, gamma, p, g, t2);
        }
        float dov[PL], qv[PL];
        load_row<PL>(static_cast<const __nv_bfloat16*>(a.dout) + row * DR + lane * PL, dov);
        load_row<PL>(static_cast<const __nv_bfloat16*>(a.q) + row * DR + lane * PL, qv);
        // dP of every entry (lane e keeps entry e's); dV_j += p dO_i
        float dp = 0.f;
        for (int e = 0; e < n; ++e) {
            const int je = __shfl_sync(0xffffffffu, j, e);
            const float pe = __shfl_sync(0xffffffffu, p, e);
            const size_t jrow = (size_t)bh * N + je;
            float vv[PL], part = 0.f;
            load_row<PL>(Vp + jrow * DR + lane * PL, vv);
#pragma unroll
            for (int c = 0; c < PL; ++c) part = fmaf(dov[c], vv[c], part);
            part = warp_sum(part);
            if (lane == e) dp = part;
            float add[PL];
#pragma unroll
            for (int c = 0; c < PL; ++c) add[c] = pe * dov[c];
            atomic_add_row<PL>(a.dv_acc + jrow * DR + lane * PL, add);
        }
        const float sg = warp_sum(lane < n ? g : 0.f);
        const float sgdp = warp_sum(lane < n ? g * dp : 0.f);
        const float delta = sg > 0.f ? sgdp / sg : 0.f;
        const float ds = lane < n ? g * (dp - delta) : 0.f;
        // dQ_i = scale sum dS k_j; dK_j += scale dS q_i
        float dq[PL];
#pragma unroll
        for (int c = 0; c < PL; ++c) dq[c] = 0.f;
        for (int e = 0; e < n; ++e) {
            const int je = __shfl_sync(0xffffffffu, j, e);
            const float dse = __shfl_sync(0xffffffffu, ds, e);
            const size_t jrow = (size_t)bh * N + je;
            float kv[PL], add[PL];
            load_row<PL>(Kp + jrow * DR + lane * PL, kv);
#pragma unroll
            for (int c = 0; c < PL; ++c) {
                dq[c] = fmaf(dse, kv[c], dq[c]);
                add[c] = scale * dse * qv[c];
            }
            atomic_add_row<PL>(a.dk_acc + jrow * DR + lane * PL, add);
        }
        __nv_bfloat16* dqr = static_cast<__nv_bfloat16*>(a.dq) + row * DR + lane * PL;
#pragma unroll
        for (int c = 0; c < PL; ++c) dqr[c] = __float2bfloat16_rn(dq[c] * scale);
    }
    if (lane == 0 && entries) atomicAdd(&a.hdr->counters[kCtrListEntries], (unsigned long long)entries);
}

template <int DR>
static cudaError_t list_bwd_d(const BwdArgs& a, int gm, cudaStream_t s) {
    const dim3 grid(a.T, a.BH);
    switch (gm) {
        case 1: list_bwd_kernel<DR, 1><<<grid, 256, 0, s>>>(a); break;
        case 2: list_bwd_kernel<DR, 2><<<grid, 256, 0, s>>>(a); break;
        case 4: list_bwd_kernel<DR, 4><<<grid, 256, 0, s>>>(a); break;
        default: list_bwd_kernel<DR, 0><<<grid, 256, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

cudaError_t list_bwd(const BwdArgs& a, int d, int gm, cudaStream_t s) {
    return d == 32 ? list_bwd_d<32>(a, gm, s) : d == 64 ? list_bwd_d<64>(a, gm, s) : list_bwd_d<128>(a, gm, s);
}

}  // namespace ent
