// entattn_api.cu -- the C ABI (include/entattn.h): argument validation,
// workspace layout, and dispatch to the kernels.  No exception crosses it.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/entattn.h"
#include "kernels.h"

namespace ent {

// A non-blocking stream per device for work forked from the caller's stream (created on
// first use, kept for the life of the process); null if it cannot be created.
cudaStream_t side_stream() {
    static cudaStream_t streams[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[dev] && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
        streams[dev] = nullptr;
    return streams[dev];
}

}  // namespace ent

namespace {

thread_local std::string g_err;

ent_status fail(ent_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

ent_status cuda_fail(cudaError_t e, const char* where) {
    return fail(ENT_ECUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr size_t kHdr = sizeof(ent::WsHeader);

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int n_tiles(int N) { return (N + ent::kBlk - 1) / ent::kBlk; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Exact integer gamma = 1/(alpha-1) in {1,2,3,4} gets a specialised kernel
// (alpha = 2, 1.5, 4/3, 1.25); any other alpha in (1, 2] uses exp2/log2.
int gamma_mode(float alpha, float* gamma_out) {
    const float gamma = 1.f / (alpha - 1.f);
    const float r = nearbyintf(gamma);
    if (r >= 1.f && r <= 4.f && fabsf(gamma - r) <= 1e-5f * r) {
        *gamma_out = r;
        return (int)r;
    }
    *gamma_out = gamma;
    return 0;
}

// Histogram insert budget of a bf16 forward tile (after its first block).  The
// default 0 starts every row from the plain bracket [m-1, m - n^(1-alpha)]: on B200
// the histogram's inserts and per-row bracket cost more than the ~2 solver passes
// they save, on every workload measured (the tiles then run ~4 cheap passes).
// ENTATTN_HIST_BUDGET selects the histogram start instead: a positive budget builds
// it until the tile has made that many inserts, a negative one always.
int hist_budget() {
    const char* v = getenv("ENTATTN_HIST_BUDGET");
    if (v && *v) return atoi(v);
    return 0;
}

// Forward workspace layout: the 256-byte header, then (bf16 path) the key-block bounds
// of the statistics pass: per head max |c| and min R (float bits), per 64-key
// half-block {R, L} and the bf16 centroid.
struct FwdLayout {
    size_t maxc, minr, stats, cent, fix, gap, calib, total;
};

FwdLayout fwd_layout(int B, int H, int N, int d) {
    const size_t BH = (size_t)B * H, T2 = 2 * (size_t)n_tiles(N);
    FwdLayout L;
    L.fix = kHdr;                        // failure list, one int per tile (zeroed with the header)
    L.maxc = L.fix + round_up(BH * T2 / 2 * 4, 256);   // [BH] words, then min R [BH]
    L.minr = L.maxc + BH * 4;
    L.stats = L.maxc + round_up(BH * 8, 256);
    L.cent = L.stats + round_up(BH * T2 * 8, 256);
    L.gap = L.cent + round_up(BH * T2 * (size_t)d * 2, 256);
    // calibrated start (sequences of >= kBoundMinBlocks query tiles): the sampled rows'
    // gaps and scores
    const bool cal = n_tiles(N) >= ent::kBoundMinBlocks;
    L.calib = L.gap + (cal ? round_up(BH * ent::kCalRows * 4, 256) : 0);
    L.total = L.calib + (cal ? round_up(BH * ent::kCalRows * (size_t)N * 4, 256) : 0);
    return L;
}

// Calibrated solver start (bf16 path, sequences of >= kBoundMinBlocks query tiles), on by
// default.  ENTATTN_CALIB=0 (environment, read per call) starts every row at the plain
// bracket's midpoint instead, for ablations; the outputs meet the same stop rule either way.
bool calib_enabled() {
    const char* v = getenv("ENTATTN_CALIB");
    return !(v && *v && atoi(v) == 0);
}

// Statistics-pass skipping by key-block bounds (bf16 path), on by default.
// ENTATTN_BOUND=0 (environment, read per call) turns it off, for ablations; the
// outputs are the same either way (a block it rules out holds no u > 0 and no row
// maximum, so every later pass sees the same blocks and sums).
bool bound_enabled() {
    const char* v = getenv("ENTATTN_BOUND");
    return !(v && *v && atoi(v) == 0);
}

// Unverified Halley steps of the bf16 forward (each checked in the P.V pass, see
// solver_update): steps up to 1e-2 either way whose boundary crossings can change f by
// at most 5e-5 upward (a bound on all leaving elements together, from the sums: half
// the check's 1e-4) or 3e-5 per entering element downward (at least four would have to
// enter within the step to miss the check).  ENTATTN_ACCEPT=0
// (environment, read per call) stops every row at an evaluated tau instead, for
// ablations.  ENTATTN_VERIFY_TOL sets the check's tolerance on |sum_j p - 1| (default
// 1e-4; a negative value makes every tile with such a row be solved again, which
// tests that path).
ent::AcceptRule accept_rule() {
    ent::AcceptRule r;
    const char* v = getenv("ENTATTN_ACCEPT");
    if (v && *v && atoi(v) == 0) return r;
    r.step = 1e-2f;
    r.cert_up = 5e-5f;
    r.cert_down = 3e-5f;
    return r;
}

// Speculative first job of each score pass in the bf16 forward (on by default);
// ENTATTN_SPEC=0 (environment, read per call) waits for each decision instead, for ablations.
int spec_enabled() {
    const char* v = getenv("ENTATTN_SPEC");
    return (v && *v && atoi(v) == 0) ? 0 : 1;
}

float verify_tol() {
    const char* v = getenv("ENTATTN_VERIFY_TOL");
    return (v && *v) ? (float)atof(v) : 1e-4f;
}

// Backward workspace layout: the 256-byte header, then delta (one float per query row).
struct BwdLayout {
    size_t delta, total;
};

BwdLayout bwd_layout(int B, int H, int N) {
    const size_t BH = (size_t)B * H;
    BwdLayout L;
    L.delta = kHdr;
    L.total = L.delta + round_up(BH * N * sizeof(float), 256);
    return L;
}

ent_status check_common(int B, int H, int N, int d, int dtype, float alpha, int causal) {
    if (B < 0 || H < 0 || N < 0) return fail(ENT_EINVAL, "negative size (B=%d H=%d N=%d)", B, H, N);
    if (dtype != ENT_F32 && dtype != ENT_BF16) return fail(ENT_EINVAL, "unknown dtype %d", dtype);
    if (!(alpha > 1.f && alpha <= 2.f)) return fail(ENT_EINVAL, "alpha=%g outside (1, 2]", (double)alpha);
    if (causal != 0 && causal != 1) return fail(ENT_EINVAL, "causal must be 0 or 1 (got %d)", causal);
    if (d != 32 && d != 64 && d != 128)
        return fail(ENT_EUNSUPPORTED, "head dim d=%d (supported: 32, 64, 128)", d);
    if ((long long)B * H > 65535) return fail(ENT_EUNSUPPORTED, "B*H=%lld exceeds 65535", (long long)B * H);
    if (N > 130944) return fail(ENT_EUNSUPPORTED, "N=%d exceeds 130944", N);
    return ENT_OK;
}

// Copies a workspace header (status word and counters) to the host after the
// work queued on `stream` is done.
ent_status read_header(const void* ws, long long* counters, void* stream) {
    ent::WsHeader h;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading the workspace header");
    if (counters)
        for (int i = 0; i < 8; ++i) counters[i] = (long long)h.counters[i];
    if (h.status != 0)
        return fail(ENT_ETIMEOUT, "a bounded device wait gave up (site %u)", h.timeout_site);
    return ENT_OK;
}

}  // namespace

extern "C" {

int ent_attn_block_size(void) { return ent::kBlk; }

size_t ent_attn_fwd_workspace_size(int B, int H, int N, int d, int dtype) {
    (void)dtype;
    if (B < 0 || H < 0 || N < 0 || d < 0) return 0;
    return fwd_layout(B, H, N, d).total;
}

size_t ent_attn_bwd_workspace_size(int B, int H, int N, int d, int dtype) {
    (void)dtype;
    if (B < 0 || H < 0 || N < 0 || d < 0) return 0;
    return bwd_layout(B, H, N).total;
}

const char* ent_attn_last_error(void) { return g_err.c_str(); }

}  // extern "C"

namespace {

// Support lists of ent_attn_fwd_lists / ent_attn_bwd_lists (all null otherwise).
struct Lists {
    int32_t* key = nullptr;
    float* u = nullptr;
    uint8_t* n = nullptr;
    bool want = false;
};

// Backward workspace of ent_attn_bwd_lists: the plain layout, then the per-tile flags
// and the fp32 dK, dV accumulators of the list kernel.
struct ListLayout {
    size_t tiles, dk, dv, total;
};

ListLayout list_layout(int B, int H, int N, int d) {
    const size_t BH = (size_t)B * H;
    ListLayout L;
    L.tiles = bwd_layout(B, H, N).total;
    L.dk = L.tiles + round_up(BH * (size_t)n_tiles(N), 256);
    L.dv = L.dk + round_up(BH * N * (size_t)d * 4, 256);
    L.total = L.dv + round_up(BH * N * (size_t)d * 4, 256);
    return L;
}

// Forward of ent_attn_fwd and, with a non-null otilde, of ent_attn_fwd_otilde.
ent_status fwd_impl(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                    int dtype, float alpha, int causal, void* o, float* tau, uint8_t* block_mask,
                    uint8_t* iters, float* otilde, bool want_otilde, void* ws, size_t ws_bytes,
                    void* stream, const Lists& lists = Lists()) {
    ent_status st = check_common(B, H, N, d, dtype, alpha, causal);
    if (st != ENT_OK) return st;
    if (lists.want && dtype != ENT_BF16)
        return fail(ENT_EUNSUPPORTED, "support lists are built by the bf16 forward only");
    if (!ws) return fail(ENT_EINVAL, "null workspace");
    if (ws_bytes < ent_attn_fwd_workspace_size(B, H, N, d, dtype))
        return fail(ENT_EINVAL, "workspace of %zu bytes is below the required %zu", ws_bytes,
                    ent_attn_fwd_workspace_size(B, H, N, d, dtype));
    if (!aligned16(ws)) return fail(ENT_EINVAL, "workspace pointer not 16-byte aligned");
    const bool empty = (long long)B * H == 0 || N == 0;
    if (!empty && (!q || !k || !v || !o || !tau || !block_mask))
        return fail(ENT_EINVAL, "null q/k/v/o/tau/block_mask pointer");
    if (!empty && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)))
        return fail(ENT_EINVAL, "q/k/v/o must be 16-byte aligned");
    if (!empty && want_otilde && (!otilde || !aligned16(otilde)))
        return fail(ENT_EINVAL, "otilde must be a non-null 16-byte aligned pointer");
    if (!empty && lists.want && (!lists.key || !lists.u || !lists.n))
        return fail(ENT_EINVAL, "null list_key/list_u/list_n pointer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const FwdLayout FL = fwd_layout(B, H, N, d);
    // (no tile of a shorter sequence runs the bound pass, so its statistics are not computed)
    const bool bound = dtype == ENT_BF16 && hist_budget() == 0 && bound_enabled() && !empty &&
                       n_tiles(N) >= ent::kBoundMinBlocks;
    // header, failure list (entries are tile + 1, 0 until written) and the per-head max |c|
    // start at 0, the per-head min R at all ones
    cudaError_t e = cudaMemsetAsync(ws, 0, bound ? FL.minr : (dtype == ENT_BF16 ? FL.maxc : kHdr), s);
    if (e == cudaSuccess && bound) e = cudaMemsetAsync(static_cast<char*>(ws) + FL.minr, 0xFF, (size_t)B * H * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace header");
    if (empty) return ENT_OK;

    ent::FwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.o = o; a.tau = tau; a.mask = block_mask; a.iters = iters;
    a.otilde = want_otilde ? otilde : nullptr;
    a.list_key = lists.key; a.list_u = lists.u; a.list_n = lists.n;
    a.hdr = static_cast<ent::WsHeader*>(ws);
    a.BH = B * H; a.N = N; a.T = n_tiles(N); a.causal = causal; a.dr = d;
    a.alpha = alpha;
    const int gm = gamma_mode(alpha, &a.gamma);
    a.scale = 1.f / sqrtf((float)d);
    a.cx = (alpha - 1.f) * a.scale;
    // Stop rule: bf16 outputs resolve ~4e-3 relative, so |sum p - 1| <= 1e-5 is
    // far below their rounding; float32 outputs get 1e-6.
    a.ftol = dtype == ENT_F32 ? 1e-6f : 1e-5f;
    a.stol = dtype == ENT_F32 ? 4e-7f : 1e-6f;
    a.hist_budget = hist_budget();
    if (dtype == ENT_BF16) {
        a.acc = accept_rule();
        a.verify_tol = verify_tol();
        a.spec = spec_enabled();
        a.fail_list = reinterpret_cast<int*>(static_cast<char*>(ws) + FL.fix);
    }
    if (dtype == ENT_BF16 && hist_budget() == 0 && calib_enabled() && n_tiles(N) >= ent::kBoundMinBlocks) {
        char* base = static_cast<char*>(ws);
        a.gap = reinterpret_cast<float*>(base + FL.gap);
        a.calib = reinterpret_cast<float*>(base + FL.calib);
    }
    if (bound) {
        // statistics-pass skipping by key-block bounds; off with the histogram start, whose
        // windows must count every score down to their lowest bin
        char* base = static_cast<char*>(ws);
        a.head_words = reinterpret_cast<unsigned int*>(base + FL.maxc);
        a.bstats = reinterpret_cast<float2*>(base + FL.stats);
        a.cent = base + FL.cent;
    }
    if (dtype == ENT_F32) {
        e = ent::simt_fwd_f32(a, d, gm, s);
    } else {
        const char* why = nullptr;
        e = ent::tc_fwd(a, d, gm, s, &why);
        if (e != cudaSuccess && why) return fail(ENT_ECUDA, "forward launch: %s", why);
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return ENT_OK;
}

// Backward of ent_attn_bwd and, with a non-null otilde, of ent_attn_bwd_otilde.
ent_status bwd_impl(const void* q, const void* k, const void* v, const float* otilde,
                    bool want_otilde, const void* dout, const float* tau,
                    const uint8_t* block_mask, int B, int H, int N, int d, int dtype, float alpha,
                    int causal, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                    void* stream, const Lists& lists = Lists()) {
    ent_status st = check_common(B, H, N, d, dtype, alpha, causal);
    if (st != ENT_OK) return st;
    if (lists.want && dtype != ENT_BF16)
        return fail(ENT_EUNSUPPORTED, "support lists are built by the bf16 forward only");
    if (!ws) return fail(ENT_EINVAL, "null workspace");
    const BwdLayout L = bwd_layout(B, H, N);
    const ListLayout LL = list_layout(B, H, N, d);
    const size_t need = lists.want ? LL.total : L.total;
    if (ws_bytes < need)
        return fail(ENT_EINVAL, "workspace of %zu bytes is below the required %zu", ws_bytes, need);
    if (!aligned16(ws)) return fail(ENT_EINVAL, "workspace pointer not 16-byte aligned");
    const bool empty = (long long)B * H == 0 || N == 0;
    if (!empty && (!q || !k || !v || !dout || !tau || !block_mask || !dq || !dk || !dv))
        return fail(ENT_EINVAL, "null q/k/v/dout/tau/block_mask/dq/dk/dv pointer");
    if (!empty && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) ||
                   !aligned16(dq) || !aligned16(dk) || !aligned16(dv)))
        return fail(ENT_EINVAL, "q/k/v/dout/dq/dk/dv must be 16-byte aligned");
    if (!empty && want_otilde && (!otilde || !aligned16(otilde)))
        return fail(ENT_EINVAL, "otilde must be a non-null 16-byte aligned pointer");
    if (!empty && lists.want && (!lists.key || !lists.u || !lists.n))
        return fail(ENT_EINVAL, "null list_key/list_u/list_n pointer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(ws, 0, kHdr, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace header");
    if (empty) return ENT_OK;
    if (lists.want) {   // the list kernel's dK, dV accumulators start at zero
        e = cudaMemsetAsync(static_cast<char*>(ws) + LL.dk, 0, LL.total - LL.dk, s);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the list accumulators");
    }

    ent::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.dout = dout; a.tau = tau; a.mask = block_mask;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.otilde = want_otilde ? otilde : nullptr;
    char* base = static_cast<char*>(ws);
    a.hdr = reinterpret_cast<ent::WsHeader*>(base);
    a.delta = reinterpret_cast<float*>(base + L.delta);
    a.BH = B * H; a.N = N; a.T = n_tiles(N); a.causal = causal; a.dr = d;
    a.alpha = alpha;
    const int gm = gamma_mode(alpha, &a.gamma);
    a.scale = 1.f / sqrtf((float)d);
    a.cx = (alpha - 1.f) * a.scale;
    if (lists.want) {
        a.list_key = lists.key; a.list_u = lists.u; a.list_n = lists.n;
        a.tile_list = reinterpret_cast<uint8_t*>(base + LL.tiles);
        a.dk_acc = reinterpret_cast<float*>(base + LL.dk);
        a.dv_acc = reinterpret_cast<float*>(base + LL.dv);
    }
    if (dtype == ENT_F32) {
        e = ent::simt_bwd_f32(a, d, gm, s);
    } else {
        const char* why = nullptr;
        if (lists.want) {
            // the list kernel and dq take disjoint query tiles (both decide from the list
            // counts) and run at the same time, the list kernel on a side stream forked
            // from `s`; dkv, which adds the list kernel's accumulators, joins it
            cudaStream_t side = ent::side_stream();
            cudaEvent_t fork = nullptr, join = nullptr;
            if (!side) side = s;   // no side stream: the two run one after the other
            e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventRecord(fork, s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
            if (e == cudaSuccess) e = ent::list_bwd(a, d, gm, side);
            if (e == cudaSuccess) e = cudaEventRecord(join, side);
            if (e == cudaSuccess) e = ent::tc_bwd(a, d, gm, s, &why, join);
            if (fork) cudaEventDestroy(fork);   // released once the recorded work is done
            if (join) cudaEventDestroy(join);
        } else {
            e = ent::tc_bwd(a, d, gm, s, &why);
        }
        if (e != cudaSuccess && why) return fail(ENT_ECUDA, "backward launch: %s", why);
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return ENT_OK;
}

}  // namespace

extern "C" {

ent_status ent_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                        int dtype, float alpha, int causal, void* o, float* tau,
                        uint8_t* block_mask, uint8_t* iters, void* ws, size_t ws_bytes,
                        void* stream) {
    return fwd_impl(q, k, v, B, H, N, d, dtype, alpha, causal, o, tau, block_mask, iters, nullptr,
                    false, ws, ws_bytes, stream);
}

ent_status ent_attn_fwd_otilde(const void* q, const void* k, const void* v, int B, int H, int N,
                               int d, int dtype, float alpha, int causal, void* o, float* tau,
                               uint8_t* block_mask, uint8_t* iters, float* otilde, void* ws,
                               size_t ws_bytes, void* stream) {
    return fwd_impl(q, k, v, B, H, N, d, dtype, alpha, causal, o, tau, block_mask, iters, otilde,
                    true, ws, ws_bytes, stream);
}

ent_status ent_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* tau, const uint8_t* block_mask, int B,
                        int H, int N, int d, int dtype, float alpha, int causal, void* dq,
                        void* dk, void* dv, void* ws, size_t ws_bytes, void* stream) {
    (void)o;
    return bwd_impl(q, k, v, nullptr, false, dout, tau, block_mask, B, H, N, d, dtype, alpha,
                    causal, dq, dk, dv, ws, ws_bytes, stream);
}

ent_status ent_attn_bwd_otilde(const void* q, const void* k, const void* v, const float* otilde,
                               const void* dout, const float* tau, const uint8_t* block_mask,
                               int B, int H, int N, int d, int dtype, float alpha, int causal,
                               void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                               void* stream) {
    return bwd_impl(q, k, v, otilde, true, dout, tau, block_mask, B, H, N, d, dtype, alpha, causal,
                    dq, dk, dv, ws, ws_bytes, stream);
}

int ent_attn_list_cap(void) { return ent::kListCap; }

size_t ent_attn_bwd_lists_workspace_size(int B, int H, int N, int d, int dtype) {
    (void)dtype;
    if (B < 0 || H < 0 || N < 0 || d < 0) return 0;
    return list_layout(B, H, N, d).total;
}

ent_status ent_attn_fwd_lists(const void* q, const void* k, const void* v, int B, int H, int N,
                              int d, int dtype, float alpha, int causal, void* o, float* tau,
                              uint8_t* block_mask, uint8_t* iters, int32_t* list_key,
                              float* list_u, uint8_t* list_n, void* ws, size_t ws_bytes,
                              void* stream) {
    Lists l;
    l.key = list_key; l.u = list_u; l.n = list_n; l.want = true;
    return fwd_impl(q, k, v, B, H, N, d, dtype, alpha, causal, o, tau, block_mask, iters, nullptr,
                    false, ws, ws_bytes, stream, l);
}

ent_status ent_attn_bwd_lists(const void* q, const void* k, const void* v, const int32_t* list_key,
                              const float* list_u, const uint8_t* list_n, const void* dout,
                              const float* tau, const uint8_t* block_mask, int B, int H, int N,
                              int d, int dtype, float alpha, int causal, void* dq, void* dk,
                              void* dv, void* ws, size_t ws_bytes, void* stream) {
    Lists l;
    l.key = const_cast<int32_t*>(list_key); l.u = const_cast<float*>(list_u);
    l.n = const_cast<uint8_t*>(list_n); l.want = true;
    return bwd_impl(q, k, v, nullptr, false, dout, tau, block_mask, B, H, N, d, dtype, alpha,
                    causal, dq, dk, dv, ws, ws_bytes, stream, l);
}

int ent_entmax_rows_max_n(void) { return 16384; }

}  // extern "C"

namespace {

static_assert(ENT_SOLVE_HIST == ent::kSolveHist && ENT_SOLVE_HALLEY == ent::kSolveHalley &&
                  ENT_SOLVE_BISECT == ent::kSolveBisect,
              "solver codes of the header and the kernels agree");

ent_status check_rows(int rows, int n, int dtype, float alpha) {
    if (rows < 0 || n < 0) return fail(ENT_EINVAL, "negative size (rows=%d n=%d)", rows, n);
    if (dtype != ENT_F32 && dtype != ENT_BF16) return fail(ENT_EINVAL, "unknown dtype %d", dtype);
    if (!(alpha > 1.f && alpha <= 2.f)) return fail(ENT_EINVAL, "alpha=%g outside (1, 2]", (double)alpha);
    if (n > ent_entmax_rows_max_n())
        return fail(ENT_EUNSUPPORTED, "n=%d exceeds %d", n, ent_entmax_rows_max_n());
    return ENT_OK;
}

ent::RowArgs row_args(int rows, int n, int dtype, float alpha) {
    ent::RowArgs a{};
    a.rows = rows; a.n = n; a.alpha = alpha;
    a.cx = alpha - 1.f;
    a.ftol = dtype == ENT_F32 ? 1e-6f : 1e-5f;
    a.stol = dtype == ENT_F32 ? 4e-7f : 1e-6f;
    return a;
}

}  // namespace

extern "C" {

ent_status ent_entmax_rows_fwd(const void* z, int rows, int n, int dtype, float alpha, int method,
                               void* p, float* tau, uint8_t* iters, void* stream) {
    ent_status st = check_rows(rows, n, dtype, alpha);
    if (st != ENT_OK) return st;
    if (method != ENT_SOLVE_HIST && method != ENT_SOLVE_HALLEY && method != ENT_SOLVE_BISECT)
        return fail(ENT_EINVAL, "unknown method %d", method);
    if (rows == 0 || n == 0) return ENT_OK;
    if (!z || !p || !tau) return fail(ENT_EINVAL, "null z/p/tau pointer");
    ent::RowArgs a = row_args(rows, n, dtype, alpha);
    a.z = z; a.p = p; a.tau = tau; a.iters = iters; a.method = method;
    const int gm = gamma_mode(alpha, &a.gamma);
    cudaError_t e = ent::rows_entmax(a, dtype == ENT_BF16, gm, false, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "row entmax launch");
    return ENT_OK;
}

ent_status ent_entmax_rows_bwd(const void* z, const float* tau, const void* dp, int rows, int n,
                               int dtype, float alpha, void* dz, void* stream) {
    ent_status st = check_rows(rows, n, dtype, alpha);
    if (st != ENT_OK) return st;
    if (rows == 0 || n == 0) return ENT_OK;
    if (!z || !tau || !dp || !dz) return fail(ENT_EINVAL, "null z/tau/dp/dz pointer");
    ent::RowArgs a = row_args(rows, n, dtype, alpha);
    a.z = z; a.tau_in = tau; a.dp = dp; a.dz = dz;
    const int gm = gamma_mode(alpha, &a.gamma);
    cudaError_t e = ent::rows_entmax(a, dtype == ENT_BF16, gm, true, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "row entmax backward launch");
    return ENT_OK;
}

ent_status ent_attn_read_status(const void* ws, long long* counters, void* stream) {
    if (!ws) return fail(ENT_EINVAL, "null workspace");
    return read_header(ws, counters, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward with library-owned scratch (no workspace argument).
//
// Some callers cannot call cudaMalloc at the point where they run the
// backward: serving and training stacks that plan all device memory up front
// and treat any later allocation as an error (a cudaMalloc may synchronise the
// device and fragments a pre-sized pool), and plain-C callers with no device
// allocator of their own.  For them the backward's scratch (a 256-byte status
// and counter header plus delta, one float per query row) lives in the
// fixed-size array below, compiled into the library.  Every GPU that loads the
// library holds this array until the process exits.
namespace {

constexpr size_t kFixedScratchBytes = size_t(4) << 20;   // 4 MiB: header + 1,048,512 rows of delta
constexpr int kMaxScratchDevices = 64;

static __device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

std::mutex g_fixed_scratch_mu;
void* g_fixed_scratch_addr[kMaxScratchDevices] = {};

// Device address of g_fixed_scratch on the current device.  The first call on
// a device looks it up with cudaGetSymbolAddress (the host-side name is only a
// stand-in, never a device address) and caches it.
cudaError_t fixed_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_fixed_scratch_mu);
    if (!g_fixed_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_fixed_scratch);
        if (e != cudaSuccess) return e;
        g_fixed_scratch_addr[dev] = p;
    }
    *out = g_fixed_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ent_status ent_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                           const void* o, const void* dout, const float* tau,
                                           const uint8_t* block_mask, int B, int H, int N, int d,
                                           int dtype, float alpha, int causal, void* dq, void* dk,
                                           void* dv, void* stream) {
    (void)o;
    ent_status st = check_common(B, H, N, d, dtype, alpha, causal);
    if (st != ENT_OK) return st;
    const bool empty = (long long)B * H == 0 || N == 0;
    const size_t need = kHdr + round_up((size_t)B * H * N * sizeof(float), 256);
    if (need > kFixedScratchBytes)
        return fail(ENT_EUNSUPPORTED,
                    "ent_attn_bwd_noalloc: B*H*N = %lld rows exceed the %zu rows its fixed "
                    "scratch holds; use ent_attn_bwd with a workspace",
                    (long long)B * H * N, (kFixedScratchBytes - kHdr) / sizeof(float));
    if (!empty && (!q || !k || !v || !dout || !tau || !block_mask || !dq || !dk || !dv))
        return fail(ENT_EINVAL, "null q/k/v/dout/tau/block_mask/dq/dk/dv pointer");
    if (!empty && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) ||
                   !aligned16(dq) || !aligned16(dk) || !aligned16(dv)))
        return fail(ENT_EINVAL, "q/k/v/dout/dq/dk/dv must be 16-byte aligned");
    void* base = nullptr;
    cudaError_t e = fixed_scratch_address(&base);
    if (e != cudaSuccess) return cuda_fail(e, "looking up the fixed scratch address");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The scratch keeps the previous call's contents: the header (status and
    // counters) must start at zero; delta is fully rewritten before it is read.
    e = cudaMemsetAsync(base, 0, kHdr, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the fixed scratch header");
    if (empty) return ENT_OK;

    ent::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.dout = dout; a.tau = tau; a.mask = block_mask;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.otilde = nullptr;
    char* b = static_cast<char*>(base);
    a.hdr = reinterpret_cast<ent::WsHeader*>(b);
    a.delta = reinterpret_cast<float*>(b + kHdr);
    a.BH = B * H; a.N = N; a.T = n_tiles(N); a.causal = causal; a.dr = d;
    a.alpha = alpha;
    const int gm = gamma_mode(alpha, &a.gamma);
    a.scale = 1.f / sqrtf((float)d);
    a.cx = (alpha - 1.f) * a.scale;
    if (dtype == ENT_F32) {
        e = ent::simt_bwd_f32(a, d, gm, s);
    } else {
        const char* why = nullptr;
        e = ent::tc_bwd(a, d, gm, s, &why);
        if (e != cudaSuccess && why) return fail(ENT_ECUDA, "backward launch: %s", why);
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return ENT_OK;
}

extern "C" ent_status ent_attn_noalloc_read_status(long long* counters, void* stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    void* base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_fixed_scratch_mu);
        if (dev >= 0 && dev < kMaxScratchDevices) base = g_fixed_scratch_addr[dev];
    }
    if (!base)
        return fail(ENT_EINVAL,
                    "ent_attn_noalloc_read_status: no ent_attn_bwd_noalloc call on device %d yet", dev);
    return read_header(base, counters, stream);
}
