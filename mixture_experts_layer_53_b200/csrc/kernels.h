// kernels.h -- host-side launchers of the MoE kernels (internal to libmoe).
#pragma once

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
// RouterArgs in one tcgen05 kernel (clusters of router_splits CTAs).
cudaError_t launch_router_fused_sm100(const RouterArgs &r, int32_t *status, bool clear_status, cudaStream_t s);

// Scores, top-k, gates and per-chunk statistics from fp32 logits (E > 32;
// smaller E selects inside launch_router_fused_sm100).
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
    double *pe;           // [E] scratch for P_e * N (needed when psum is given)
    int tile_m;           // rows per m-tile of the tile table (when mt_prefix is given)
    const float *zpart;   // [chunks] per-chunk z-loss sums, or null
    float *z_out;         // router z-loss (scalar) or null; needs zpart
    int32_t *dense_offsets;  // [2] or null: {0, N}, the one-slice table of the shared expert
    int32_t *dense_mt;       // [2] or null: {0, ceil(N / dense_tile_m)}
    int dense_tile_m;
};
cudaError_t launch_scan(const ScanArgs &a, cudaStream_t s);

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

// Both expert GEMMs; `mid` (may be null) is recorded between them.
// CTA pairs, 256-row m-tiles:
cudaError_t launch_ffn_bf16_sm100(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s);
// single CTAs, 128-row m-tiles:
cudaError_t launch_ffn_bf16_sm100_single(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s);
cudaError_t launch_ffn_f32_simt(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s);

}  // namespace moe
