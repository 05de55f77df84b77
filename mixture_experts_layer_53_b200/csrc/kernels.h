// kernels.h -- host-side launchers of the MoE kernels (internal to libmoe).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// dtype / router / activation codes are those of moe.h.
enum { kF32 = 0, kBF16 = 1 };
enum { kSoftmaxTopk = 0, kTopkSoftmax = 1, kSigmoid = 2 };
enum { kGelu = 0, kSwiglu = 1 };

inline int64_t num_chunks(int64_t N) { return (N + 31) / 32; }

struct RouterArgs {
    const void *x;       // [N, d]
    const void *Wg;      // [E, d]
    const float *b_sel;  // [E] or null (sigmoid router only)
    int32_t *ids;        // [N, k]
    float *w;            // [N, k]
    float *probs;        // [N, E] or null
    int32_t *hist;       // [chunks, E] or null
    float *psum;         // [chunks, E] or null
    float *zpart;        // [chunks] sum of the chunk's (lse z_n)^2, or null
    int64_t N;
    int d, E, k, router, norm_topk;
    float scaling;
    float *lse;          // [N] per-token log-sum-exp of the logits, or null
};
// CUDA-core router (fp32 path).
cudaError_t launch_router(int dtype, const RouterArgs &a, cudaStream_t s);
// tcgen05 router logits (bf16 path): router_splits(N, d) partial sums over
// d, logits [splits, N, logits_ld(E)] fp32; `status` receives device wait
// timeouts.
int logits_ld(int E);
int router_splits(int64_t N, int d);
// clear_status: the kernel zeroes *status before anything else (used as the
// first kernel of a forward instead of a memset).
cudaError_t launch_router_logits_sm100(const void *x, const void *W_g, float *logits, int64_t N, int d, int E,
                                       int32_t *status, bool clear_status, cudaStream_t s);
// E <= 32: logits, scores, top-k, gates and the per-chunk statistics of
// RouterArgs in one streaming kernel, one CTA per 32-token chunk, warps over
// column ranges of d, warp-level MMAs (router_mma.cu).
cudaError_t launch_router_stream(const RouterArgs &r, int32_t *status, bool clear_status, cudaStream_t s);

// Scores, top-k, gates and per-chunk statistics from fp32 logits (E > 32;
// smaller E selects inside launch_router_stream).
struct SelectKernelArgs {
    const float *logits;  // [splits, N, ld] partial logits, summed in split order
    const float *b_sel;   // [E] or null (sigmoid router only)
    int32_t *ids;
    float *w;
    float *probs;         // [N, E] or null
    int32_t *hist;        // [chunks, E] or null
    float *psum;          // [chunks, E] or null
    float *zpart;         // [chunks] sum of the chunk's (lse z_n)^2, or null
    int64_t N;
    int ld, E, k, router, norm_topk;
    float scaling;
    int splits;
    float *lse;           // [N] or null
};
cudaError_t launch_select(const SelectKernelArgs &a, cudaStream_t s);

// Per-chunk histograms of expert ids (with range check) and, optionally,
// per-chunk sums of probs.
struct HistArgs {
    const int32_t *ids;  // [N, k] or null (then hist is not written)
    const float *probs;  // [N, E] or null
    int32_t *hist;       // [chunks, E]
    float *psum;         // [chunks, E] or null
    int32_t *status;
    int64_t N;
    int E, k;
};
cudaError_t launch_hist(const HistArgs &a, cudaStream_t s);

// Counts, offsets, per-chunk bases inside each expert's slice (in place over
// hist), the GEMM tile table, the Switch loss and the sign-rule bias step:
// one CTA per expert, then one finalizing CTA.
struct ScanArgs {
    int32_t *hist;        // in: [chunks, E] counts; out: chunk bases within the expert's slice
    const float *psum;    // [chunks, E] or null (no loss then)
    int64_t chunks, N;
    int E, k;
    int32_t *counts;      // [E] or null
    int32_t *offsets;     // [E+1]
    int32_t *mt_prefix;   // [E+1] or null
    float *aux_out;       // scalar or null
    float gamma;
    float *b_e;           // [E] or null
    double *pe;           // [E] P_e * N = sum_n p_{n,e} in fp64 (needed when psum is given; written)
    int tile_m;           // rows per m-tile of the tile table (when mt_prefix is given)
    const float *zpart;   // [chunks] per-chunk z-loss sums, or null
    float *z_out;         // router z-loss (scalar) or null; needs zpart
    int32_t *dense_offsets;  // [2] or null: {0, N}, the one-slice table of the shared expert
    int32_t *dense_mt;       // [2] or null: {0, ceil(N / dense_tile_m)}
    int dense_tile_m;
};
cudaError_t launch_scan(const ScanArgs &a, cudaStream_t s);

// The Switch loss and the sign-rule step from assignment counts and
// probability sums added up over several forwards (the ranks of a
// data-parallel layer): N = sum_e counts[e] / k, L = E sum_e counts[e]
// psum[e] / N^2, b_e += gamma sign(sum counts - E counts[e]).
struct AuxPartialsArgs {
    const int32_t *counts;  // [E]
    const double *psum;     // [E] sum over tokens of p_{n,e}
    float *aux_out;         // scalar or null
    float gamma;
    float *b_e;             // [E] or null
    int E, k;
};
cudaError_t launch_aux_partials(const AuxPartialsArgs &a, cudaStream_t s);

// Router z-loss from per-chunk sums: *z_out = (sum of zpart) / N in fp64.
cudaError_t launch_z_loss(const float *zpart, int64_t N, float *z_out, cudaStream_t s);

// One-slice tile table over all N rows (the shared expert's GEMMs):
// offsets = {0, N}, mt = {0, ceil(N / tile_m)}.
cudaError_t launch_dense_table(int32_t *offsets, int32_t *mt, int64_t N, int tile_m, cudaStream_t s);

// Sorted position of assignment a: offsets[e] + chunk base + rank in chunk.
struct ScatterArgs {
    const int32_t *ids;
    const int32_t *chunk_base;  // [chunks, E], relative to the slice start
    int32_t *perm;              // [N k] or null
    int32_t *inv_perm;          // [N k]
    int64_t N;
    int E, k;
    const int32_t *offsets;     // [E+1]
};
cudaError_t launch_scatter(const ScatterArgs &a, cudaStream_t s);

struct GatherArgs {
    const void *x;
    const int32_t *inv_perm;
    void *x_sorted;
    int64_t N;
    int d, k;
};
cudaError_t launch_gather(int dtype, const GatherArgs &a, int num_sms, cudaStream_t s);

// Scatter and gather in one pass (positions as in ScatterArgs, rows as in
// GatherArgs); invalid expert ids get inv_perm = -1.
struct DispatchRowsArgs {
    const int32_t *ids;         // [N k]
    const int32_t *chunk_base;  // [chunks, E], relative to the slice start
    const int32_t *offsets;     // [E+1]
    int32_t *perm;              // [N k] or null
    int32_t *inv_perm;          // [N k]
    const void *x;              // [N, d]
    void *x_sorted;             // [N k, d]
    int64_t N;
    int d, E, k;
};
cudaError_t launch_dispatch_rows(int dtype, const DispatchRowsArgs &a, int num_sms, cudaStream_t s);

struct CombineArgs {
    const void *y_sorted;
    const float *w;
    const int32_t *inv_perm;
    void *y;
    int64_t N;
    int d, k;
    const void *y_add;  // [N, d] or null: added after the weighted sum (shared expert)
};
cudaError_t launch_combine(int dtype, const CombineArgs &a, int num_sms, cudaStream_t s);

// mt_prefix[e+1] = mt_prefix[e] + ceil((offsets[e+1] - offsets[e]) / tile_m).
cudaError_t launch_tile_table(const int32_t *offsets, int32_t *mt_prefix, int E, int tile_m, cudaStream_t s);

// Strided grouped GEMM on the CUDA cores, fp32 out (backward products):
// C_g(m, n) (+)= sum_k A(m, k) B_g(k, n), A(m, k) = A[m sam + k sak],
// B_g(k, n) = B[g sbg + k sbk + n sbn], C_g(m, n) = C[g scg + m scm + n scn].
// ragged_k = 0: group g owns rows offsets[g] .. offsets[g+1]-1 of A and C
// (mt_prefix: the per-group 64-row tile prefix, launch with an upper bound
// on the tiles); ragged_k = 1: group g sums k over offsets[g] ..
// offsets[g+1]-1.
struct GenericGemmArgs {
    const void *A;
    int64_t sam, sak;
    const void *B;
    int64_t sbk, sbn, sbg;
    float *C;
    int64_t scm, scn, scg;
    const int32_t *offsets;
    const int32_t *mt_prefix;
    int G;
    int ragged_k;
    int64_t M, N, K;
    int accumulate, a_bf16, b_bf16;
    // ragged_k only: split each reduction ksplit ways (> 1: dense partials
    // [G * ksplit][M][N] in `partial`, then summed in split order)
    int ksplit;
    float *partial;
};
constexpr int kGenericTileM = 64;
constexpr int64_t kGenericPartialFloats = 4 << 20;  // workspace floats for split partials
cudaError_t launch_gemm_generic(const GenericGemmArgs &g, int64_t max_tiles_m, cudaStream_t s);

// ---- backward (backward.cu)
struct BwdRowsArgs {
    const int32_t *perm, *ids;  // sorted position -> assignment; [N k]
    const float *w;             // [N k] gate weights
    int64_t rows;
    int k;
    int32_t *row_tok, *row_e;   // [rows]
    float *row_w;               // [rows]
    float *one;                 // receives 1.0f
};
cudaError_t launch_rows_prep(const BwdRowsArgs &a, int num_sms, cudaStream_t s);

struct BwdActArgs {
    int64_t rows;
    int F, d, act, bf16;   // bf16: the layer dtype of b1, b2, dy_s
    float *pre, *up, *h;   // [rows, F]: pre-activations, SwiGLU up, h
    const float *dh;       // [rows, F]: dy_s W2[e]
    const void *b1, *b2;   // [E, F], [E, d] or null
    const int32_t *row_e;  // [rows] or null (expert 0)
    const float *row_w;    // [rows] or null (weight 1)
    float *dw;             // [N k] or null: <dy_n, Expert(x_n)> per assignment
    const int32_t *perm;   // [rows] (with dw)
    const void *dy_s;      // [rows, d] (with dw and b2)
    __nv_bfloat16 *dcat;   // [rows, m F] or null: bf16 copies [da | du] (the tensor-core dgrad operand)
    __nv_bfloat16 *hw_bf;  // [rows, F] or null: bf16 copy of w h (the tensor-core dW2 operand)
    int skip_f32;          // row_backward: fp32 results not written back (kSkip* bits)
};
constexpr int kSkipPre = 1, kSkipUp = 2, kSkipH = 4;
cudaError_t launch_act_forward(const BwdActArgs &a, int num_sms, cudaStream_t s);
cudaError_t launch_row_backward(const BwdActArgs &a, int num_sms, cudaStream_t s);

struct BwdGatherSumArgs {
    const float *dxs;          // [N k, d]
    const int32_t *inv_perm;   // [N k]
    float *dx;                 // [N, d]
    int64_t N;
    int d, k;
    // with dz (E <= 32): also dx_n += sum_e dz[n, e] W_g[e, :], the router's
    // input gradient (W_g [E, d] in the layer dtype)
    const float *dz;
    const void *W_g;
    int E, bf16;
};
cudaError_t launch_gather_sum(const BwdGatherSumArgs &a, int num_sms, cudaStream_t s);

struct BwdRouterArgs {
    const float *probs, *lse;  // [N, E], [N]
    const int32_t *ids;        // [N k]
    const float *dw;           // [N k]
    const int32_t *counts;     // [E]
    float *dz;                 // [N, E]
    int64_t N;
    int E, k, router, norm_topk;
    float scaling, aux_coef, z_coef;
};
cudaError_t launch_router_backward(const BwdRouterArgs &a, int num_sms, cudaStream_t s);

struct FfnArgs {
    const void *x_sorted;      // [rows, d]
    const int32_t *offsets;    // [E+1]
    const int32_t *mt_prefix;  // [E+1]
    const void *W1, *b1, *W3, *W2, *b2;
    void *h;                   // [rows, F] scratch
    void *y_sorted;            // [rows, d]
    int32_t *status;
    int64_t rows;              // N k
    int d, F, E, act;
    int tile_m;                // m-tile rows of mt_prefix: 128 (single CTA) or 256 (CTA pair)
};
}  // namespace moe

#include <cuda.h>

namespace moe {

// TMA descriptor of a bf16 matrix [outer, inner] (inner contiguous) with a
// box of [box_outer, 64] elements, 128-byte swizzle, zero fill outside.
bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_outer);
bool make_tmap_bf16_mn(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t groups);
bool make_tmap_bf16_mn_rows(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t ld);
bool make_tmap_f32_store(CUtensorMap *m, void *base, uint64_t inner, uint64_t rows, uint64_t groups);
bool make_tmap_bf16_store(CUtensorMap *m, void *base, uint64_t inner, uint64_t rows);

// C (fp32) from bf16 operands on tcgen05 (the backward's products on the
// tensor cores), 128 x 256 tiles:
//   ragged M (ragged_k = 0): rows offsets[e] .. offsets[e+1]-1 of A
//     [a_rows, K] (K-major) and of C belong to group e (mt_prefix: its
//     128-row tile prefix); B is K-major [E * n_out, K] (C = A B^T), or with
//     b_mn the MN-major weights below (C = A B);
//   ragged K (ragged_k = rows_mn = 1): group e's result (m_total x n_out at
//     C + e * c_stride) sums over rows offsets[e] .. offsets[e+1]-1 of the
//     two row-major activations below, both read MN-major.
struct TcGemmArgs {
    const void *A;
    uint64_t a_rows, a_cols;
    const void *B;
    uint64_t b_rows, b_cols;
    float *C;
    int64_t ldc, c_stride;
    const int32_t *offsets, *mt_prefix;
    int E, ragged_k, K, n_out;
    int64_t m_total;
    int32_t *status;
    int accumulate;  // add to C instead of overwriting it
    // b_mn (ragged M only): B is E matrices [k1 rows][n_out] with n_out
    // contiguous, read as an MN-major operand (no transposed copy); A's
    // columns 0..k1-1 pair with B, columns k1..k1+k2-1 with B2 (same layout,
    // k2 rows; k2 = 0 and B2 = null without it)
    int b_mn;
    const void *B2;
    int64_t k1, k2;
    // rows_mn (ragged K only): A and B are row-major [a_rows][lda] and
    // [a_rows][ldb] whose columns 0..m_total-1 and 0..n_out-1 are the result
    // rows and columns; expert e sums rows offsets[e] .. offsets[e+1]-1 (no
    // padding; the result of an expert without rows is zero)
    int rows_mn;
    int64_t lda, ldb;
};
cudaError_t launch_gemm_tc_f32(const TcGemmArgs &t, int num_sms, cudaStream_t s);
// The same on CTA pairs (256 x 256 tiles) for ragged-M products; mt_prefix
// must count 256-row tiles.
cudaError_t launch_gemm_tc_f32_pair(const TcGemmArgs &t, int num_sms, cudaStream_t s);

// Both expert GEMMs; `mid` (may be null) is recorded between them.
// CTA pairs, 256-row m-tiles:
cudaError_t launch_ffn_bf16_sm100(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s);
// single CTAs, 128-row m-tiles:
cudaError_t launch_ffn_bf16_sm100_single(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s);
cudaError_t launch_ffn_f32_simt(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s);

}  // namespace moe
