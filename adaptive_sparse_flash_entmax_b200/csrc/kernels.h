// kernels.h -- host-side launch interface between the C ABI (entattn_api.cu)
// and the kernel files.  Internal to the library.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include "common.cuh"

namespace ent {

constexpr int kListCap = 16;        // entries per row in the support lists
constexpr int kBoundMinBlocks = 64;  // shortest query tile (key blocks) that runs the bound pass
constexpr int kCalRows = 8;          // sampled rows per head of the calibrated start
constexpr uint8_t kListOver = 255;  // list_n of a row with more than kListCap nonzeros

struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* tau;
    uint8_t* mask;
    uint8_t* iters;        // nullable
    WsHeader* hdr;         // workspace header (status, counters)
    int BH, N, T, causal;
    int dr;                // head dimension of the tensors (row stride); the tensor-core
                           // kernels run d = 32 as d = 64 with zero-filled upper columns
    float alpha, gamma;    // gamma = 1/(alpha-1)
    float cx;              // (alpha-1)/sqrt(d): x = cx * (q . k)
    float scale;           // 1/sqrt(d)
    float ftol, stol;      // solver stop rule: |f| <= ftol, or a step <= stol*max(1,|tau|)
    int hist_budget;       // tensor-core path: histogram inserts a tile may make after its
                           // first block (0: no histogram, < 0: no limit)
    // Unverified Halley steps (tensor-core path): the rule, and the check in the P.V pass
    // (|sum_j p_ij - 1| <= verify_tol for every row that stopped on one).  A tile that
    // fails it goes on the failure list fail_list [BH*T] (tile + 1; count and claim counter
    // in the workspace header); CTAs that finished their own tile claim the entries and
    // solve those tiles again with evaluated stops.
    AcceptRule acc;
    float verify_tol;
    int* fail_list;
    int spec;              // tensor-core path: load and multiply the next score pass's likely
                           // first job before the decision after a pass (0: wait for it)
    float* otilde;         // nullable [BH][N][d] fp32: sum_j g_ij v_j / sum_j g_ij
    // Key-block bounds for skipping statistics-pass blocks (tensor-core path; all null:
    // no bound pass).  Per 64-key half-block hb of head bh (T2 = 2T of them):
    //   cent[bh][hb][d]  bf16 centroid c (mean of its valid keys, rounded),
    //   bstats[bh][hb]   {R, L}: every computed score q.k_j of the half-block is
    //                    <= q.c + |q| R, and the largest is >= q.c - |q| L (R < 0: no
    //                    valid key),
    //   head_words       [BH] max |c| then [BH] min R, as float bits (a bound can rule out
    //                    a block only where R < 2 max |c|, so heads without such a block
    //                    skip the pass).
    void* cent;
    float2* bstats;
    unsigned int* head_words;
    // Calibrated start (tensor-core path; null: every row starts at the plain bracket's
    // midpoint).  Per head, kCalRows sampled query rows p_s = (s+1) N / kCalRows - 1 are
    // solved exactly before the forward: calib [BH][kCalRows][N] holds their scores x,
    // gap [BH][kCalRows] their m - tau; a row then starts at m - gap of the nearest
    // sample, clamped into its bracket.
    float* calib;
    float* gap;
    // Per-row support lists (nullable; tensor-core path): for each query row the keys j
    // with p_ij > 0 and their u_ij = x_ij - tau_i, up to kListCap of them, in list_key /
    // list_u [BH][N][kListCap]; list_n [BH][N] the count, kListOver when the row has more.
    int* list_key;
    float* list_u;
    uint8_t* list_n;
};

struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* dout;
    const float* tau;
    const uint8_t* mask;
    void* dq;
    void* dk;
    void* dv;
    const float* otilde;   // nullable: the forward's otilde; then delta_i = dO_i . otilde_i
                           // and the delta pass over the keys is skipped
    float* delta;          // workspace [BH*N]
    // Support-list backward (nullable): the forward's lists, a per-tile flag (1: every row
    // of the query tile has a list, so the list kernel covers the tile and the block
    // kernels skip it) and fp32 accumulators of the list kernel's dK, dV contributions
    // that the dkv kernel adds before it stores.
    const int* list_key;
    const float* list_u;
    const uint8_t* list_n;
    uint8_t* tile_list;    // workspace [BH][T]
    float* dk_acc;         // workspace [BH][N][d]
    float* dv_acc;         // workspace [BH][N][d]
    WsHeader* hdr;
    int BH, N, T, causal;
    int dr;                // head dimension of the tensors, as in FwdArgs
    float alpha, gamma, cx, scale;
};

// Row-wise alpha-entmax of a [rows][n] score matrix (rows.cu).  Solver codes match
// the public ENT_SOLVE_* values.
enum RowSolve { kSolveHist = 0, kSolveHalley = 1, kSolveBisect = 2 };

struct RowArgs {
    const void* z;         // scores [rows][n]
    void* p;               // forward: probabilities [rows][n]
    float* tau;            // forward: tau per row (x units)
    uint8_t* iters;        // forward, nullable: solver passes per row
    const float* tau_in;   // backward: tau per row
    const void* dp;        // backward: upstream gradient [rows][n]
    void* dz;              // backward: gradient w.r.t. z [rows][n]
    int rows, n, method;
    float alpha, gamma;    // gamma = 1/(alpha-1)
    float cx;              // alpha - 1: x = cx * z
    float ftol, stol;      // stop rule, as in FwdArgs
};
cudaError_t rows_entmax(const RowArgs& a, int dtype_bf16, int gm, bool bwd, cudaStream_t s);

// FP32 CUDA-core path: float32 inputs (scores by FFMA, no TF32 rounding).
cudaError_t simt_fwd_f32(const FwdArgs& a, int d, int gm, cudaStream_t s);
cudaError_t simt_bwd_f32(const BwdArgs& a, int d, int gm, cudaStream_t s);

// bf16 tensor-core path (tcgen05 + TMEM + TMA).  `why` names a host-side failure.
cudaError_t tc_fwd(const FwdArgs& a, int d, int gm, cudaStream_t s, const char** why);
// A non-blocking stream per device for work forked from the caller's stream (null if it
// cannot be created); defined with the ABI.
cudaStream_t side_stream();

// before_dkv (nullable): an event the dkv kernel waits for (the list kernel's end).
cudaError_t tc_bwd(const BwdArgs& a, int d, int gm, cudaStream_t s, const char** why,
                   cudaEvent_t before_dkv = nullptr);

// Support-list backward of the query tiles whose rows all have lists (tc_lists.cu): dQ of
// those rows, their dK / dV contributions added into dk_acc / dv_acc, and tile_list.
cudaError_t list_bwd(const BwdArgs& a, int d, int gm, cudaStream_t s);

}  // namespace ent
