// moe_api.cu -- the extern "C" entry points of libmoe.so (declared in
// include/moe.h): argument validation, workspace carving and the launch
// sequence of each operation.  No allocation, no host synchronisation.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using namespace moe;

thread_local std::string g_last_error;

moe_status cuda_fail(cudaError_t err)
{
    g_last_error = cudaGetErrorString(err);
    return MOE_ERR_CUDA;
}

int num_sms()
{
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

size_t elem_size(const moe_config *c) { return c->dtype == MOE_F32 ? 4 : 2; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status validate(const moe_config *c)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->N < 0 || c->d_model <= 0 || c->d_ff <= 0 || c->E <= 0 || c->k <= 0) return MOE_ERR_INVALID_ARG;
    if (c->k > c->E) return MOE_ERR_INVALID_ARG;
    if (c->router < MOE_ROUTER_SOFTMAX_TOPK || c->router > MOE_ROUTER_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (c->act < MOE_ACT_GELU || c->act > MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
    if (c->dtype < MOE_F32 || c->dtype > MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (c->norm_topk != 0 && c->norm_topk != 1) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(c->routed_scaling)) return MOE_ERR_INVALID_ARG;
    if (c->E > kMaxE || c->k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (c->d_ff_shared < 0) return MOE_ERR_INVALID_ARG;
    if (c->d_model % 8 != 0 || c->d_ff % 8 != 0 || c->d_ff_shared % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (c->N * static_cast<int64_t>(c->k) >= (static_cast<int64_t>(1) << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

struct Layout {
    size_t hist, psum, zpart, logits, pe, offsets, mt, shoff, shmt, counts, ids, w, perm, inv, xs, h, ys, ysh,
        total;
};

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

Layout layout(const moe_config *c)
{
    Layout L{};
    size_t o = 0;
    auto take = [&o](size_t bytes) {
        const size_t at = o;
        o += align256(bytes > 0 ? bytes : 1);
        return at;
    };
    const size_t C = static_cast<size_t>(num_chunks(c->N));
    const size_t E = static_cast<size_t>(c->E);
    const size_t A = static_cast<size_t>(c->N) * static_cast<size_t>(c->k);
    const size_t es = elem_size(c);
    L.hist = take(C * E * 4);
    L.logits = take(static_cast<size_t>(router_splits(c->N, c->d_model)) * static_cast<size_t>(c->N) *
                    static_cast<size_t>(logits_ld(c->E)) * 4);
    L.psum = take(C * E * 4);
    L.zpart = take(C * 4);
    L.pe = take(E * 8);
    L.offsets = take((E + 1) * 4);
    L.mt = take((E + 1) * 4);
    L.shoff = take(2 * 4);
    L.shmt = take(2 * 4);
    L.counts = take(E * 4);
    L.ids = take(A * 4);
    L.w = take(A * 4);
    L.perm = take(A * 4);
    L.inv = take(A * 4);
    L.xs = take(A * c->d_model * es);
    // h holds the routed experts' hidden rows, then (reused) the shared expert's
    const size_t Nn = static_cast<size_t>(c->N);
    const size_t h_rows_cols = A * c->d_ff > Nn * c->d_ff_shared ? A * c->d_ff : Nn * c->d_ff_shared;
    L.h = take(h_rows_cols * es);
    L.ys = take(A * c->d_model * es);
    L.ysh = take(c->d_ff_shared > 0 ? Nn * c->d_model * es : 0);
    L.total = o;
    return L;
}

template <typename T> T *at(void *ws, size_t off) { return reinterpret_cast<T *>(static_cast<char *>(ws) + off); }

moe_status check_ws(const moe_config *c, const void *ws, size_t ws_bytes)
{
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (ws_bytes < layout(c).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

RouterArgs router_args(const moe_config *c, const void *x, const void *W_g, const float *b_e, int32_t *ids,
                       float *w, float *probs, int32_t *hist, float *psum, float *zpart = nullptr)
{
    RouterArgs r{};
    r.x = x;
    r.Wg = W_g;
    r.b_sel = c->router == MOE_ROUTER_SIGMOID ? b_e : nullptr;
    r.ids = ids;
    r.w = w;
    r.probs = probs;
    r.hist = hist;
    r.psum = psum;
    r.zpart = zpart;
    r.N = c->N;
    r.d = c->d_model;
    r.E = c->E;
    r.k = c->k;
    r.router = c->router;
    r.norm_topk = c->norm_topk;
    r.scaling = c->routed_scaling;
    return r;
}

// Rows per m-tile of the expert GEMMs.  bf16: CTA pairs (256 rows) when the
// experts hold many rows on average, single CTAs (128 rows) for fine-grained
// experts, where 256-row tiles would mostly compute rows of the next expert.
int ffn_tile_m(const moe_config *c)
{
    if (c->dtype != MOE_BF16) return 128;
    const int64_t rows_per_expert = c->N * c->k / c->E;
    return rows_per_expert > 192 ? 256 : 128;
}

// The same rule for the shared expert, whose one slice holds all N rows.
int shared_tile_m(const moe_config *c)
{
    if (c->dtype != MOE_BF16) return 128;
    return c->N > 192 ? 256 : 128;
}

FfnArgs ffn_args(const moe_config *c, const void *x_sorted, const int32_t *offsets, const int32_t *mt,
                 const void *W1, const void *b1, const void *W3, const void *W2, const void *b2, void *h,
                 void *y_sorted, int32_t *status)
{
    FfnArgs f{};
    f.x_sorted = x_sorted;
    f.offsets = offsets;
    f.mt_prefix = mt;
    f.W1 = W1;
    f.b1 = c->act == MOE_ACT_GELU ? b1 : nullptr;
    f.W3 = W3;
    f.W2 = W2;
    f.b2 = b2;
    f.h = h;
    f.y_sorted = y_sorted;
    f.status = status;
    f.rows = c->N * c->k;
    f.d = c->d_model;
    f.F = c->d_ff;
    f.E = c->E;
    f.act = c->act;
    f.tile_m = ffn_tile_m(c);
    return f;
}

moe_status check_ffn_ptrs(const moe_config *c, const void *W1, const void *b1, const void *W3, const void *W2,
                          const void *b2)
{
    if (!W1 || !W2) return MOE_ERR_INVALID_ARG;
    if (c->act == MOE_ACT_SWIGLU && !W3) return MOE_ERR_INVALID_ARG;
    if (c->act == MOE_ACT_SWIGLU && b1) return MOE_ERR_INVALID_ARG;  // SwiGLU experts carry no hidden bias
    if (!aligned16(W1) || !aligned16(W2) || (W3 && !aligned16(W3)) || (b1 && !aligned16(b1)) ||
        (b2 && !aligned16(b2)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// bf16 routes on the tensor cores; fp32 keeps the CUDA-core router (tf32
// products would not meet the fp32 tolerance).
cudaError_t launch_route(const moe_config *c, const RouterArgs &r, int32_t *status, float *logits, cudaStream_t s,
                         bool clear_status = false)
{
    if (c->dtype != MOE_BF16) return launch_router(c->dtype, r, s);
    if (c->E <= 32) return launch_router_fused_sm100(r, status, clear_status, s);
    cudaError_t err = launch_router_logits_sm100(r.x, r.Wg, logits, r.N, r.d, r.E, status, clear_status, s);
    if (err != cudaSuccess) return err;
    SelectKernelArgs sk{logits, r.b_sel, r.ids, r.w, r.probs, r.hist, r.psum, r.zpart, r.N, logits_ld(r.E),
                        r.E, r.k, r.router, r.norm_topk, r.scaling, router_splits(r.N, r.d)};
    return launch_select(sk, s);
}

cudaError_t launch_ffn(const moe_config *c, const FfnArgs &f, cudaEvent_t mid, cudaStream_t s)
{
    if (c->dtype != MOE_BF16) return launch_ffn_f32_simt(f, num_sms(), mid, s);
    return f.tile_m == 256 ? launch_ffn_bf16_sm100(f, num_sms(), mid, s)
                           : launch_ffn_bf16_sm100_single(f, num_sms(), mid, s);
}

// The shared expert: cfg->d_ff_shared > 0 exactly when its weights are given.
moe_status check_shared(const moe_config *c, const moe_shared_expert *sh)
{
    if ((c->d_ff_shared > 0) != (sh != nullptr)) return MOE_ERR_INVALID_ARG;
    if (!sh) return MOE_OK;
    return check_ffn_ptrs(c, sh->W1, sh->b1, sh->W3, sh->W2, sh->b2);
}

// Both GEMMs of the shared expert over the N rows of x into y_shared, with
// the one-slice tile table at (offsets, mt) already written.
cudaError_t launch_shared(const moe_config *c, const moe_shared_expert *sh, const void *x, const int32_t *offsets,
                          const int32_t *mt, void *h, void *y_shared, int32_t *status, cudaStream_t s)
{
    FfnArgs f{};
    f.x_sorted = x;
    f.offsets = offsets;
    f.mt_prefix = mt;
    f.W1 = sh->W1;
    f.b1 = c->act == MOE_ACT_GELU ? sh->b1 : nullptr;
    f.W3 = sh->W3;
    f.W2 = sh->W2;
    f.b2 = sh->b2;
    f.h = h;
    f.y_sorted = y_shared;
    f.status = status;
    f.rows = c->N;
    f.d = c->d_model;
    f.F = c->d_ff_shared;
    f.E = 1;
    f.act = c->act;
    f.tile_m = shared_tile_m(c);
    return launch_ffn(c, f, nullptr, s);
}

}  // namespace

extern "C" {

const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_BAD_EXPERT_ID: return "expert id out of range";
    }
    return "unknown status";
}

const char *moe_last_error(void) { return g_last_error.c_str(); }

int32_t moe_version(void) { return 100; }

size_t moe_workspace_size(const moe_config *cfg)
{
    if (validate(cfg) != MOE_OK) return 0;
    return layout(cfg).total;
}

moe_status moe_route(const moe_config *cfg, const void *x, const void *W_g, const float *b_e, int32_t *topk_ids,
                     float *topk_w, float *probs, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    const bool empty = cfg->N == 0;  // token-sized buffers may then be NULL
    if (!W_g || (!empty && (!x || !topk_ids || !topk_w))) return MOE_ERR_INVALID_ARG;
    if (b_e && cfg->router != MOE_ROUTER_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_g)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    if (cfg->N == 0) return MOE_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const RouterArgs r = router_args(cfg, x, W_g, b_e, topk_ids, topk_w, probs, nullptr, nullptr);
    cudaError_t err = launch_route(cfg, r, nullptr, at<float>(ws, layout(cfg).logits), s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
}

moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *topk_ids, void *x_sorted,
                        int32_t *perm, int32_t *inv_perm, int32_t *offsets, int32_t *counts, int32_t *dev_status,
                        void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    const bool empty = cfg->N == 0;
    if (!offsets || !counts || (!empty && (!topk_ids || !inv_perm))) return MOE_ERR_INVALID_ARG;
    if ((x == nullptr) != (x_sorted == nullptr)) return MOE_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || (x_sorted && !aligned16(x_sorted))) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(cfg);
    int32_t *hist = at<int32_t>(ws, L.hist);
    cudaError_t err;
    HistArgs h{topk_ids, nullptr, hist, nullptr, dev_status, cfg->N, cfg->E, cfg->k};
    if ((err = launch_hist(h, s)) != cudaSuccess) return cuda_fail(err);
    ScanArgs sc{};
    sc.hist = hist;
    sc.chunks = num_chunks(cfg->N);
    sc.N = cfg->N;
    sc.E = cfg->E;
    sc.k = cfg->k;
    sc.counts = counts;
    sc.offsets = offsets;
    if ((err = launch_scan(sc, s)) != cudaSuccess) return cuda_fail(err);
    if (x) {  // positions and rows in one pass
        DispatchRowsArgs da{topk_ids, hist, offsets, perm, inv_perm, x, x_sorted, cfg->N, cfg->d_model, cfg->E,
                            cfg->k};
        if ((err = launch_dispatch_rows(cfg->dtype, da, num_sms(), s)) != cudaSuccess) return cuda_fail(err);
    } else {
        ScatterArgs sa{topk_ids, hist, perm, inv_perm, cfg->N, cfg->E, cfg->k, offsets};
        if ((err = launch_scatter(sa, s)) != cudaSuccess) return cuda_fail(err);
    }
    return MOE_OK;
}

moe_status moe_expert_ffn(const moe_config *cfg, const void *x_sorted, const int32_t *offsets, const void *W1,
                          const void *b1, const void *W3, const void *W2, const void *b2, void *y_sorted,
                          int32_t *dev_status, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    const bool empty = cfg->N == 0;
    if (!offsets || (!empty && (!x_sorted || !y_sorted))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_sorted) || !aligned16(y_sorted)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ffn_ptrs(cfg, W1, b1, W3, W2, b2)) != MOE_OK) return st;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(cfg);
    int32_t *mt = at<int32_t>(ws, L.mt);
    cudaError_t err;
    if ((err = launch_tile_table(offsets, mt, cfg->E, ffn_tile_m(cfg), s)) != cudaSuccess) return cuda_fail(err);
    const FfnArgs f = ffn_args(cfg, x_sorted, offsets, mt, W1, b1, W3, W2, b2, at<void>(ws, L.h), y_sorted,
                               dev_status);
    if ((err = launch_ffn(cfg, f, nullptr, s)) != cudaSuccess) return cuda_fail(err);
    return MOE_OK;
}

moe_status moe_combine_shared(const moe_config *cfg, const void *y_sorted, const float *topk_w,
                              const int32_t *inv_perm, const void *y_shared, void *y, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->N > 0 && (!y_sorted || !topk_w || !inv_perm || !y)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_sorted) || !aligned16(y) || !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    CombineArgs ca{y_sorted, topk_w, inv_perm, y, cfg->N, cfg->d_model, cfg->k, y_shared};
    cudaError_t err = launch_combine(cfg->dtype, ca, num_sms(), s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
}

moe_status moe_combine(const moe_config *cfg, const void *y_sorted, const float *topk_w, const int32_t *inv_perm,
                       void *y, moe_stream_t stream)
{
    return moe_combine_shared(cfg, y_sorted, topk_w, inv_perm, nullptr, y, stream);
}

moe_status moe_shared_ffn(const moe_config *cfg, const void *x, const moe_shared_expert *shared, void *y_shared,
                          int32_t *dev_status, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    if (cfg->d_ff_shared == 0 || !shared) return MOE_ERR_INVALID_ARG;
    if (cfg->N > 0 && (!x || !y_shared)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
    if ((st = check_shared(cfg, shared)) != MOE_OK) return st;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(cfg);
    int32_t *off = at<int32_t>(ws, L.shoff), *mt = at<int32_t>(ws, L.shmt);
    cudaError_t err;
    if ((err = launch_dense_table(off, mt, cfg->N, shared_tile_m(cfg), s)) != cudaSuccess) return cuda_fail(err);
    err = launch_shared(cfg, shared, x, off, mt, at<void>(ws, L.h), y_shared, dev_status, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
}

moe_status moe_router_z_loss(const moe_config *cfg, const void *x, const void *W_g, float *z_loss_out,
                             int32_t *dev_status, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!W_g || !z_loss_out || (cfg->N > 0 && !x)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_g)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(cfg);
    float *zpart = at<float>(ws, L.zpart);
    cudaError_t err;
    if (cfg->N > 0) {
        // the routing itself lands in the workspace; only the z-loss is kept
        const RouterArgs r = router_args(cfg, x, W_g, nullptr, at<int32_t>(ws, L.ids), at<float>(ws, L.w),
                                         nullptr, nullptr, nullptr, zpart);
        if ((err = launch_route(cfg, r, dev_status, at<float>(ws, L.logits), s)) != cudaSuccess)
            return cuda_fail(err);
    }
    err = launch_z_loss(zpart, cfg->N, z_loss_out, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
}

moe_status moe_aux_loss(const moe_config *cfg, const float *probs, const int32_t *topk_ids, float *aux_out,
                        int32_t *counts_out, float gamma, float *b_e_inout, int32_t *dev_status, void *ws,
                        size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!aux_out || (cfg->N > 0 && (!probs || !topk_ids))) return MOE_ERR_INVALID_ARG;
    if (!(gamma >= 0.f) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(cfg);
    int32_t *hist = at<int32_t>(ws, L.hist);
    float *psum = at<float>(ws, L.psum);
    cudaError_t err;
    HistArgs h{topk_ids, probs, hist, psum, dev_status, cfg->N, cfg->E, cfg->k};
    if ((err = launch_hist(h, s)) != cudaSuccess) return cuda_fail(err);
    ScanArgs sc{};
    sc.hist = hist;
    sc.psum = psum;
    sc.pe = at<double>(ws, L.pe);
    sc.chunks = num_chunks(cfg->N);
    sc.N = cfg->N;
    sc.E = cfg->E;
    sc.k = cfg->k;
    sc.counts = counts_out;
    sc.offsets = at<int32_t>(ws, L.offsets);
    sc.aux_out = aux_out;
    sc.gamma = gamma;
    sc.b_e = b_e_inout;
    if ((err = launch_scan(sc, s)) != cudaSuccess) return cuda_fail(err);
    return MOE_OK;
}

moe_status moe_forward(const moe_config *cfg, const void *x, const void *W_g, float *b_e_inout, float gamma,
                       const void *W1, const void *b1, const void *W3, const void *W2, const void *b2, void *y,
                       int32_t *topk_ids, float *topk_w, int32_t *counts, float *aux_out, int32_t *dev_status,
                       void *ws, size_t ws_bytes, void *const *stage_events, moe_stream_t stream)
{
    return moe_forward_ex(cfg, x, W_g, b_e_inout, gamma, W1, b1, W3, W2, b2, nullptr, y, topk_ids, topk_w, counts,
                          aux_out, nullptr, dev_status, ws, ws_bytes, stage_events, stream);
}

moe_status moe_forward_ex(const moe_config *cfg, const void *x, const void *W_g, float *b_e_inout, float gamma,
                          const void *W1, const void *b1, const void *W3, const void *W2, const void *b2,
                          const moe_shared_expert *shared, void *y, int32_t *topk_ids, float *topk_w,
                          int32_t *counts, float *aux_out, float *z_loss_out, int32_t *dev_status, void *ws,
                          size_t ws_bytes, void *const *stage_events, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!W_g || (cfg->N > 0 && (!x || !y))) return MOE_ERR_INVALID_ARG;  // N = 0: x, y may be NULL
    if (!aligned16(x) || !aligned16(W_g) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    if (b_e_inout && cfg->router != MOE_ROUTER_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (!(gamma >= 0.f) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ffn_ptrs(cfg, W1, b1, W3, W2, b2)) != MOE_OK) return st;
    if ((st = check_shared(cfg, shared)) != MOE_OK) return st;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Layout L = layout(cfg);
    cudaEvent_t ev[MOE_NUM_STAGES + 1] = {};
    if (stage_events)
        for (int i = 0; i <= MOE_NUM_STAGES; ++i) ev[i] = static_cast<cudaEvent_t>(stage_events[i]);
    auto mark = [&](int i) { return ev[i] ? cudaEventRecord(ev[i], s) : cudaSuccess; };

    int32_t *hist = at<int32_t>(ws, L.hist);
    float *psum = at<float>(ws, L.psum);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *mt = at<int32_t>(ws, L.mt);
    int32_t *ids = topk_ids ? topk_ids : at<int32_t>(ws, L.ids);
    float *w = topk_w ? topk_w : at<float>(ws, L.w);
    int32_t *inv = at<int32_t>(ws, L.inv);
    void *ys = at<void>(ws, L.ys);

    cudaError_t err;
    if ((err = mark(0)) != cudaSuccess) return cuda_fail(err);
    // dev_status is cleared by the bf16 router's first CTA (no memset between
    // this forward's kernels and the previous ones); the fp32 path and N = 0
    // clear it with a memset
    const bool router_clears = cfg->dtype == MOE_BF16 && cfg->N > 0;
    if (dev_status && !router_clears && (err = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s)) != cudaSuccess)
        return cuda_fail(err);
    // route: logits, scores, top-k, gates, per-chunk histograms and P sums
    float *zpart = at<float>(ws, L.zpart);
    const RouterArgs r = router_args(cfg, x, W_g, b_e_inout, ids, w, nullptr, hist, psum,
                                     z_loss_out ? zpart : nullptr);
    if (cfg->N > 0 && (err = launch_route(cfg, r, dev_status, at<float>(ws, L.logits), s, router_clears)) !=
                          cudaSuccess)
        return cuda_fail(err);
    if ((err = mark(1)) != cudaSuccess) return cuda_fail(err);
    // dispatch: counts, offsets, tile table, Switch loss, bias step; scatter; gather
    ScanArgs sc{};
    sc.hist = hist;
    sc.psum = psum;
    sc.pe = at<double>(ws, L.pe);
    sc.chunks = num_chunks(cfg->N);
    sc.N = cfg->N;
    sc.E = cfg->E;
    sc.k = cfg->k;
    sc.counts = counts;
    sc.offsets = offsets;
    sc.mt_prefix = mt;
    sc.aux_out = aux_out;
    sc.gamma = gamma;
    sc.tile_m = ffn_tile_m(cfg);
    sc.b_e = b_e_inout;
    sc.zpart = zpart;
    sc.z_out = z_loss_out;
    int32_t *shoff = at<int32_t>(ws, L.shoff), *shmt = at<int32_t>(ws, L.shmt);
    if (shared) {
        sc.dense_offsets = shoff;
        sc.dense_mt = shmt;
        sc.dense_tile_m = shared_tile_m(cfg);
    }
    if ((err = launch_scan(sc, s)) != cudaSuccess) return cuda_fail(err);
    // positions and rows in one pass
    void *xs = at<void>(ws, L.xs);
    DispatchRowsArgs da{ids, hist, offsets, nullptr, inv, x, xs, cfg->N, cfg->d_model, cfg->E, cfg->k};
    if ((err = launch_dispatch_rows(cfg->dtype, da, num_sms(), s)) != cudaSuccess) return cuda_fail(err);
    if ((err = mark(2)) != cudaSuccess) return cuda_fail(err);
    // expert FFNs over the ragged slices
    const FfnArgs f = ffn_args(cfg, xs, offsets, mt, W1, b1, W3, W2, b2, at<void>(ws, L.h), ys, dev_status);
    if ((err = launch_ffn(cfg, f, ev[3], s)) != cudaSuccess) return cuda_fail(err);
    // the shared expert over all N rows (its hidden rows reuse h)
    void *ysh = shared ? at<void>(ws, L.ysh) : nullptr;
    if (shared && (err = launch_shared(cfg, shared, x, shoff, shmt, at<void>(ws, L.h), ysh, dev_status, s)) !=
                      cudaSuccess)
        return cuda_fail(err);
    if ((err = mark(4)) != cudaSuccess) return cuda_fail(err);
    // combine back in token order (+ the shared expert's rows)
    CombineArgs ca{ys, w, inv, y, cfg->N, cfg->d_model, cfg->k, ysh};
    if ((err = launch_combine(cfg->dtype, ca, num_sms(), s)) != cudaSuccess) return cuda_fail(err);
    if ((err = mark(5)) != cudaSuccess) return cuda_fail(err);
    return MOE_OK;
}

}  // extern "C"
