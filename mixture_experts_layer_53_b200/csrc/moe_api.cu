// moe_api.cu -- the extern "C" entry points of libmoe.so (declared in
// include/moe.h): argument validation, workspace carving and the launch
// sequence of each operation.  No allocation, no host synchronisation.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "api_internal.h"
#include "common.cuh"
#include "kernels.h"

namespace {
thread_local std::string g_last_error;
}  // namespace

namespace moe {

moe_status record_cuda_error(cudaError_t err)
{
    g_last_error = cudaGetErrorString(err);
    return MOE_ERR_CUDA;
}

int device_sms()
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

moe_status validate_config(const moe_config *c)
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

namespace {
bool aligned16_(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

moe_status check_dispatch_args(const moe_config *c, const void *x, const int32_t *topk_ids, const void *x_sorted,
                               const int32_t *inv_perm, const int32_t *offsets, const int32_t *counts)
{
    const bool empty = c->N == 0;
    if (!offsets || !counts || (!empty && (!topk_ids || !inv_perm))) return MOE_ERR_INVALID_ARG;
    if ((x == nullptr) != (x_sorted == nullptr)) return MOE_ERR_INVALID_ARG;
    if (!aligned16_(x) || !aligned16_(x_sorted)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

cudaError_t enqueue_dispatch(const moe_config *c, const void *x, const int32_t *topk_ids, void *x_sorted,
                             int32_t *perm, int32_t *inv_perm, int32_t *offsets, int32_t *counts,
                             int32_t *dev_status, int32_t *hist, cudaStream_t s)
{
    cudaError_t err;
    HistArgs h{topk_ids, nullptr, hist, nullptr, dev_status, c->N, c->E, c->k};
    if ((err = launch_hist(h, s)) != cudaSuccess) return err;
    ScanArgs sc{};
    sc.hist = hist;
    sc.chunks = num_chunks(c->N);
    sc.N = c->N;
    sc.E = c->E;
    sc.k = c->k;
    sc.counts = counts;
    sc.offsets = offsets;
    if ((err = launch_scan(sc, s)) != cudaSuccess) return err;
    if (x) {  // positions and rows in one pass
        DispatchRowsArgs da{topk_ids, hist, offsets, perm, inv_perm, x, x_sorted, c->N, c->d_model, c->E, c->k};
        return launch_dispatch_rows(c->dtype, da, device_sms(), s);
    }
    ScatterArgs sa{topk_ids, hist, perm, inv_perm, c->N, c->E, c->k, offsets};
    return launch_scatter(sa, s);
}

}  // namespace moe

namespace {

using namespace moe;

moe_status cuda_fail(cudaError_t err) { return record_cuda_error(err); }
int num_sms() { return device_sms(); }
moe_status validate(const moe_config *c) { return validate_config(c); }
size_t elem_size(const moe_config *c) { return c->dtype == MOE_F32 ? 4 : 2; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
    if (c->E <= 32) return launch_router_stream(r, status, clear_status, s);
    cudaError_t err = launch_router_logits_sm100(r.x, r.Wg, logits, r.N, r.d, r.E, status, clear_status, s);
    if (err != cudaSuccess) return err;
    SelectKernelArgs sk{logits, r.b_sel, r.ids, r.w, r.probs, r.hist, r.psum, r.zpart, r.N, logits_ld(r.E),
                        r.E, r.k, r.router, r.norm_topk, r.scaling, router_splits(r.N, r.d), r.lse};
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

// ------------------------------------------------------------- backward

struct BwdLayout {
    size_t hist, logits, offsets, mt64, counts, ids, w, perm, inv, probs, lse, xs, dys, row_tok, row_e, row_w,
        pre, up, h, dh, dxs, dw, dz, doff, dmt, one, spre, sup, sh, sdh;
    // bf16 path (tensor cores): 128- or 256-row tile prefix, the bf16
    // [da | du] and w h operands
    size_t mtc, dacat, hwb, partial;
    // bf16 shared expert on the tensor cores: the same over one group of N rows
    size_t smtc, sdcat, shb, total;
};

BwdLayout bwd_layout(const moe_config *c)
{
    BwdLayout L{};
    size_t o = 0;
    auto take = [&o](size_t bytes) {
        const size_t at = o;
        o += align256(bytes > 0 ? bytes : 1);
        return at;
    };
    const size_t C = static_cast<size_t>(num_chunks(c->N));
    const size_t E = static_cast<size_t>(c->E);
    const size_t Nn = static_cast<size_t>(c->N);
    const size_t A = Nn * static_cast<size_t>(c->k);
    const size_t es = elem_size(c);
    const size_t d = static_cast<size_t>(c->d_model), F = static_cast<size_t>(c->d_ff);
    const size_t Fs = static_cast<size_t>(c->d_ff_shared);
    const bool swiglu = c->act == MOE_ACT_SWIGLU;
    L.hist = take(C * E * 4);
    L.logits = take(static_cast<size_t>(router_splits(c->N, c->d_model)) * Nn * logits_ld(c->E) * 4);
    L.offsets = take((E + 1) * 4);
    L.mt64 = take((E + 1) * 4);
    L.counts = take(E * 4);
    L.ids = take(A * 4);
    L.w = take(A * 4);
    L.perm = take(A * 4);
    L.inv = take(A * 4);
    L.probs = take(Nn * E * 4);
    L.lse = take(Nn * 4);
    L.xs = take(A * d * es);
    L.dys = take(A * d * es);
    L.row_tok = take(A * 4);
    L.row_e = take(A * 4);
    L.row_w = take(A * 4);
    L.pre = take(A * F * 4);
    L.up = take(swiglu ? A * F * 4 : 0);
    L.h = take(A * F * 4);
    L.dh = take(A * F * 4);
    L.dxs = take(A * d * 4);
    L.dw = take(A * 4);
    L.dz = take(Nn * E * 4);
    L.doff = take(2 * 4);
    L.dmt = take(2 * 4);
    L.one = take(4);
    L.spre = take(Nn * Fs * 4);
    L.sup = take(swiglu ? Nn * Fs * 4 : 0);
    L.sh = take(Nn * Fs * 4);
    L.sdh = take(Nn * Fs * 4);
    const bool tc = c->dtype == MOE_BF16;
    const size_t m = swiglu ? 2 : 1;
    L.mtc = take((E + 1) * 4);
    L.dacat = take(tc ? A * m * F * 2 : 0);
    L.hwb = take(tc ? A * F * 2 : 0);
    L.partial = take(static_cast<size_t>(kGenericPartialFloats) * 4);
    const bool stc = tc && Fs > 0;
    L.smtc = take(2 * 4);
    L.sdcat = take(stc ? Nn * m * Fs * 2 : 0);
    L.shb = take(stc ? Nn * Fs * 2 : 0);
    L.total = o;
    return L;
}

// One strided product on gemm_generic_kernel (see kernels.h).
struct GG {
    GenericGemmArgs g{};
    float *partial = nullptr;  // workspace for split reductions (sum_rows)
    GG &a(const void *p, int64_t sm, int64_t sk, bool bf16)
    {
        g.A = p; g.sam = sm; g.sak = sk; g.a_bf16 = bf16 ? 1 : 0;
        return *this;
    }
    GG &b(const void *p, int64_t sk, int64_t sn, int64_t sg, bool bf16)
    {
        g.B = p; g.sbk = sk; g.sbn = sn; g.sbg = sg; g.b_bf16 = bf16 ? 1 : 0;
        return *this;
    }
    GG &c(float *p, int64_t sm, int64_t sn, int64_t sg, bool acc = false)
    {
        g.C = p; g.scm = sm; g.scn = sn; g.scg = sg; g.accumulate = acc ? 1 : 0;
        return *this;
    }
    // rows offsets[gi] .. offsets[gi+1]-1 of A and C per group; N columns, K depth
    cudaError_t rows(const int32_t *off, const int32_t *mt, int G, int64_t rows_total, int64_t N, int64_t K,
                     cudaStream_t s)
    {
        g.offsets = off; g.mt_prefix = mt; g.G = G; g.ragged_k = 0; g.N = N; g.K = K;
        return launch_gemm_generic(g, (rows_total + kGenericTileM - 1) / kGenericTileM + G, s);
    }
    // per group an M x N result summed over rows offsets[gi] .. offsets[gi+1]-1
    // Few output tiles (the router's dW_g, the shared expert): the sums are
    // split so that about four CTAs per SM run, partials fixed-order reduced.
    cudaError_t sum_rows(const int32_t *off, int G, int64_t M, int64_t N, cudaStream_t s)
    {
        g.offsets = off; g.mt_prefix = nullptr; g.G = G; g.ragged_k = 1; g.M = M; g.N = N;
        const int64_t tiles = ((M + 63) / 64) * ((N + 63) / 64) * G;
        int64_t ks = tiles > 0 ? (148 * 4) / tiles : 1;
        ks = ks > 32 ? 32 : (ks < 1 ? 1 : ks);
        while (ks > 1 && ks * G * M * N > kGenericPartialFloats) --ks;
        g.ksplit = partial ? static_cast<int>(ks) : 1;
        g.partial = partial;
        return launch_gemm_generic(g, 0, s);
    }
    GG &split(float *p)
    {
        partial = p;
        return *this;
    }
};

moe_status check_grads(const moe_config *c, const moe_grads *gr, bool shared)
{
    if (!gr || (c->N > 0 && !gr->dx) || !gr->dW_g || !gr->dW1 || !gr->dW2) return MOE_ERR_INVALID_ARG;
    if (c->act == MOE_ACT_SWIGLU && !gr->dW3) return MOE_ERR_INVALID_ARG;
    if (shared && (!gr->dWs1 || !gr->dWs2 || (c->act == MOE_ACT_SWIGLU && !gr->dWs3))) return MOE_ERR_INVALID_ARG;
    // the gradient kernels store 16-byte vectors (and the tensor-core
    // weight gradients go out through TMA stores)
    for (const float *p : {gr->dx, gr->dW_g, gr->dW1, gr->db1, gr->dW3, gr->dW2, gr->db2, gr->dWs1, gr->dbs1,
                           gr->dWs3, gr->dWs2, gr->dbs2})
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
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
    if ((st = check_dispatch_args(cfg, x, topk_ids, x_sorted, inv_perm, offsets, counts)) != MOE_OK) return st;
    if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
    const cudaError_t err = enqueue_dispatch(cfg, x, topk_ids, x_sorted, perm, inv_perm, offsets, counts, dev_status,
                                             at<int32_t>(ws, layout(cfg).hist), reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
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

}  // extern "C"

namespace {

// The layer forward behind moe_forward, moe_forward_ex and
// moe_forward_partials; psum_out (may be NULL) receives sum_n p_{n,e}.
moe_status forward_impl(const moe_config *cfg, const void *x, const void *W_g, float *b_e_inout, float gamma,
                        const void *W1, const void *b1, const void *W3, const void *W2, const void *b2,
                        const moe_shared_expert *shared, void *y, int32_t *topk_ids, float *topk_w,
                        int32_t *counts, float *aux_out, float *z_loss_out, double *psum_out, int32_t *dev_status,
                        void *ws, size_t ws_bytes, void *const *stage_events, moe_stream_t stream)
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
    sc.pe = psum_out ? psum_out : at<double>(ws, L.pe);
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

}  // namespace

extern "C" {

moe_status moe_forward_ex(const moe_config *cfg, const void *x, const void *W_g, float *b_e_inout, float gamma,
                          const void *W1, const void *b1, const void *W3, const void *W2, const void *b2,
                          const moe_shared_expert *shared, void *y, int32_t *topk_ids, float *topk_w,
                          int32_t *counts, float *aux_out, float *z_loss_out, int32_t *dev_status, void *ws,
                          size_t ws_bytes, void *const *stage_events, moe_stream_t stream)
{
    return forward_impl(cfg, x, W_g, b_e_inout, gamma, W1, b1, W3, W2, b2, shared, y, topk_ids, topk_w, counts,
                        aux_out, z_loss_out, nullptr, dev_status, ws, ws_bytes, stage_events, stream);
}

moe_status moe_forward_partials(const moe_config *cfg, const void *x, const void *W_g, const float *b_e,
                                const void *W1, const void *b1, const void *W3, const void *W2, const void *b2,
                                const moe_shared_expert *shared, void *y, int32_t *topk_ids, float *topk_w,
                                int32_t *counts, double *psum_out, float *z_loss_out, int32_t *dev_status,
                                void *ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!counts || !psum_out) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(psum_out) & 7u) return MOE_ERR_INVALID_ARG;
    // the selection bias is read, never moved: its step needs the global load
    return forward_impl(cfg, x, W_g, const_cast<float *>(b_e), 0.0f, W1, b1, W3, W2, b2, shared, y, topk_ids,
                        topk_w, counts, nullptr, z_loss_out, psum_out, dev_status, ws, ws_bytes, nullptr, stream);
}

moe_status moe_aux_from_partials(int32_t E, int32_t k, const int32_t *counts, const double *psum, float *aux_out,
                                 float gamma, float *b_e_inout, moe_stream_t stream)
{
    if (E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (!counts || !psum || (!aux_out && !b_e_inout)) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(psum) & 7u) return MOE_ERR_INVALID_ARG;
    if (!(gamma >= 0.f) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
    AuxPartialsArgs a{counts, psum, aux_out, gamma, b_e_inout, E, k};
    const cudaError_t err = launch_aux_partials(a, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
}

moe_status moe_permute_rows(int32_t dtype, const void *src, const int32_t *dst_row, void *dst, int64_t rows,
                            int32_t d, moe_stream_t stream)
{
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (rows < 0 || d <= 0 || d % 8 != 0 || rows >= (static_cast<int64_t>(1) << 31)) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!src || !dst_row || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
    // the dispatch's row copy with one slot per row: dst[dst_row[i]] = src[i]
    GatherArgs ga{src, dst_row, dst, rows, d, 1};
    const cudaError_t err = launch_gather(dtype, ga, num_sms(), reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : cuda_fail(err);
}

size_t moe_backward_workspace_size(const moe_config *cfg)
{
    if (validate(cfg) != MOE_OK) return 0;
    return bwd_layout(cfg).total;
}

moe_status moe_backward(const moe_config *cfg, const void *x, const void *W_g, const float *b_e, const void *W1,
                        const void *b1, const void *W3, const void *W2, const void *b2,
                        const moe_shared_expert *shared, const void *dy, float aux_coef, float z_coef,
                        const moe_grads *grads, int32_t *dev_status, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    moe_status st = validate(cfg);
    if (st != MOE_OK) return st;
    if (!W_g || (cfg->N > 0 && (!x || !dy))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W_g) || !aligned16(dy)) return MOE_ERR_INVALID_ARG;
    if (b_e && cfg->router != MOE_ROUTER_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(aux_coef) || !std::isfinite(z_coef)) return MOE_ERR_INVALID_ARG;
    if ((st = check_ffn_ptrs(cfg, W1, b1, W3, W2, b2)) != MOE_OK) return st;
    if ((st = check_shared(cfg, shared)) != MOE_OK) return st;
    if ((st = check_grads(cfg, grads, shared != nullptr)) != MOE_OK) return st;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < bwd_layout(cfg).total)
        return MOE_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const BwdLayout L = bwd_layout(cfg);
    const int64_t N = cfg->N, rows = N * cfg->k;
    const int E = cfg->E, k = cfg->k, d = cfg->d_model, F = cfg->d_ff, Fs = cfg->d_ff_shared;
    const bool bf = cfg->dtype == MOE_BF16, swiglu = cfg->act == MOE_ACT_SWIGLU;
    const moe_grads &gr = *grads;
    cudaError_t err;
#define MOE_TRY(call)                                   \
    do {                                                \
        if ((err = (call)) != cudaSuccess) return cuda_fail(err); \
    } while (0)
    if (dev_status) MOE_TRY(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s));
    if (N == 0) {  // empty sums: every parameter gradient is zero
        MOE_TRY(cudaMemsetAsync(gr.dW_g, 0, sizeof(float) * E * d, s));
        MOE_TRY(cudaMemsetAsync(gr.dW1, 0, sizeof(float) * E * F * d, s));
        MOE_TRY(cudaMemsetAsync(gr.dW2, 0, sizeof(float) * E * d * F, s));
        if (swiglu) MOE_TRY(cudaMemsetAsync(gr.dW3, 0, sizeof(float) * E * F * d, s));
        if (b1 && gr.db1) MOE_TRY(cudaMemsetAsync(gr.db1, 0, sizeof(float) * E * F, s));
        if (b2 && gr.db2) MOE_TRY(cudaMemsetAsync(gr.db2, 0, sizeof(float) * E * d, s));
        if (shared) {
            MOE_TRY(cudaMemsetAsync(gr.dWs1, 0, sizeof(float) * Fs * d, s));
            MOE_TRY(cudaMemsetAsync(gr.dWs2, 0, sizeof(float) * d * Fs, s));
            if (swiglu) MOE_TRY(cudaMemsetAsync(gr.dWs3, 0, sizeof(float) * Fs * d, s));
            if (shared->b1 && gr.dbs1) MOE_TRY(cudaMemsetAsync(gr.dbs1, 0, sizeof(float) * Fs, s));
            if (shared->b2 && gr.dbs2) MOE_TRY(cudaMemsetAsync(gr.dbs2, 0, sizeof(float) * d, s));
        }
        return MOE_OK;
    }
    const int sms = num_sms();
    int32_t *hist = at<int32_t>(ws, L.hist), *offsets = at<int32_t>(ws, L.offsets), *mt = at<int32_t>(ws, L.mt64);
    int32_t *counts = at<int32_t>(ws, L.counts), *ids = at<int32_t>(ws, L.ids), *perm = at<int32_t>(ws, L.perm);
    int32_t *inv = at<int32_t>(ws, L.inv), *doff = at<int32_t>(ws, L.doff), *dmt = at<int32_t>(ws, L.dmt);
    float *w = at<float>(ws, L.w), *probs = at<float>(ws, L.probs), *lse = at<float>(ws, L.lse);
    void *xs = at<void>(ws, L.xs), *dys = at<void>(ws, L.dys);
    float *row_w = at<float>(ws, L.row_w), *pre = at<float>(ws, L.pre), *up = swiglu ? at<float>(ws, L.up) : nullptr;
    float *h = at<float>(ws, L.h), *dh = at<float>(ws, L.dh), *dxs = at<float>(ws, L.dxs), *dw = at<float>(ws, L.dw);
    float *dz = at<float>(ws, L.dz), *one = at<float>(ws, L.one), *partial = at<float>(ws, L.partial);

    // ---- recompute: routing (with p and lse), counts, slices, x_sorted
    RouterArgs r = router_args(cfg, x, W_g, b_e, ids, w, probs, hist, nullptr);
    r.lse = lse;
    MOE_TRY(launch_route(cfg, r, dev_status, at<float>(ws, L.logits), s));
    ScanArgs sc{};
    sc.hist = hist;
    sc.chunks = num_chunks(N);
    sc.N = N;
    sc.E = E;
    sc.k = k;
    sc.counts = counts;
    sc.offsets = offsets;
    sc.mt_prefix = mt;
    sc.tile_m = kGenericTileM;
    sc.dense_offsets = doff;  // {0, N}: one group of all tokens
    sc.dense_mt = dmt;
    sc.dense_tile_m = kGenericTileM;
    MOE_TRY(launch_scan(sc, s));
    DispatchRowsArgs da{ids, hist, offsets, perm, inv, x, xs, N, d, E, k};
    MOE_TRY(launch_dispatch_rows(cfg->dtype, da, sms, s));
    BwdRowsArgs ra{perm, ids, w, rows, k, at<int32_t>(ws, L.row_tok), at<int32_t>(ws, L.row_e), row_w, one};
    MOE_TRY(launch_rows_prep(ra, sms, s));
    GatherArgs gd{dy, inv, dys, N, d, k};  // dy_s[r] = dy[token of r]
    MOE_TRY(launch_gather(cfg->dtype, gd, sms, s));

    // tensor-core products: rows offsets[g] .. of A and C per group (B per
    // group n_out rows of K), or (tc_sum_rows) per group a sum over the
    // group's padded columns of A [m_total, cols] and B [n_out, cols]
    // (ragged M: CTA pairs with 256-row tiles where the groups average more
    // than 192 rows, as in the forward; the tile prefix mt_ counts tile_m rows)
    auto tc_launch = [&](const TcGemmArgs &t, int tile_m) {
        return tile_m == 256 ? launch_gemm_tc_f32_pair(t, sms, s) : launch_gemm_tc_f32(t, sms, s);
    };
    auto tc_rows = [&](const void *A, int64_t nrows, int64_t K, const void *B, int n_out, float *C,
                       const int32_t *off, const int32_t *mt_, int tile_m, int G, bool accumulate) {
        TcGemmArgs t{};
        t.A = A; t.a_rows = static_cast<uint64_t>(nrows); t.a_cols = static_cast<uint64_t>(K);
        t.B = B; t.b_rows = static_cast<uint64_t>(G) * n_out; t.b_cols = static_cast<uint64_t>(K);
        t.C = C; t.ldc = n_out; t.offsets = off; t.mt_prefix = mt_; t.E = G; t.K = static_cast<int>(K);
        t.n_out = n_out; t.status = dev_status; t.accumulate = accumulate ? 1 : 0;
        return tc_launch(t, tile_m);
    };
    // C_g [m_total, n_out] = sum over rows off[g] .. off[g+1]-1 of A[r, :m_total]^T B[r, :n_out]
    // (row-major A [nrows][lda], B [nrows][ldb], both read MN-major in place)
    // (CTA pairs under the same rule as the ragged-M products)
    auto tc_sum_rows = [&](const void *A, int64_t lda, int64_t m_total, const void *B, int64_t ldb, int n_out, float *C,
                           const int32_t *off, int tile_m, int G, int64_t nrows) {
        TcGemmArgs t{};
        t.A = A; t.a_rows = static_cast<uint64_t>(nrows); t.lda = lda; t.B = B; t.ldb = ldb; t.rows_mn = 1;
        t.C = C; t.ldc = n_out; t.c_stride = m_total * n_out; t.offsets = off; t.E = G; t.ragged_k = 1;
        t.n_out = n_out; t.m_total = m_total; t.status = dev_status;
        return tile_m == 256 ? launch_gemm_tc_f32_pair(t, sms, s) : launch_gemm_tc_f32(t, sms, s);
    };
    // the same with B = G matrices [K rows][n_out] read MN-major in place:
    // A's columns 0..k1-1 against B1, k1..k1+k2-1 against B2
    auto tc_rows_mn = [&](const void *A, int64_t nrows, const void *B1, int64_t k1, const void *B2, int64_t k2,
                          int n_out, float *C, const int32_t *off, const int32_t *mt_, int tile_m, int G,
                          bool accumulate) {
        TcGemmArgs t{};
        t.A = A; t.a_rows = static_cast<uint64_t>(nrows); t.a_cols = static_cast<uint64_t>(k1 + k2);
        t.B = B1; t.B2 = B2; t.k1 = k1; t.k2 = k2; t.b_mn = 1;
        t.C = C; t.ldc = n_out; t.offsets = off; t.mt_prefix = mt_; t.E = G; t.K = static_cast<int>(k1 + k2);
        t.n_out = n_out; t.status = dev_status; t.accumulate = accumulate ? 1 : 0;
        return tc_launch(t, tile_m);
    };
    BwdActArgs act{rows, F, d, cfg->act, bf ? 1 : 0, pre, up, h, dh, swiglu ? nullptr : b1, b2,
                   at<int32_t>(ws, L.row_e), row_w, dw, perm, dys, nullptr};
    const int m = swiglu ? 2 : 1;
    if (bf) {
        // ---- bf16: every expert product on the tensor cores (fp32 results),
        // every operand read in place: dgrad with the weights MN-major, wgrad
        // over each expert's token rows of the activations (MN-major)
        const int tm = ffn_tile_m(cfg);
        int32_t *mtc = at<int32_t>(ws, L.mtc);
        auto *dacat = at<__nv_bfloat16>(ws, L.dacat), *hwb = at<__nv_bfloat16>(ws, L.hwb);
        auto ragged_m = [&](const void *A, int64_t K, const void *B, int n_out, float *C) {
            return tc_rows(A, rows, K, B, n_out, C, offsets, mtc, tm, E, false);
        };
        MOE_TRY(launch_tile_table(offsets, mtc, E, tm, s));
        MOE_TRY(ragged_m(xs, d, W1, F, pre));
        if (swiglu) MOE_TRY(ragged_m(xs, d, W3, F, up));
        MOE_TRY(launch_act_forward(act, sms, s));
        MOE_TRY(tc_rows_mn(dys, rows, W2, d, nullptr, 0, F, dh, offsets, mtc, tm, E, false));  // dh = dy_s W2[e]
        act.dcat = dacat;  // [da | du] and w h in bf16; fp32 da only for db1
        act.hw_bf = hwb;
        act.skip_f32 = kSkipUp | kSkipH | ((!swiglu && b1 && gr.db1) ? 0 : kSkipPre);
        MOE_TRY(launch_row_backward(act, sms, s));
        // dx_s = [da | du] [W1[e] ; W3[e]]: one product with K = m F
        MOE_TRY(tc_rows_mn(dacat, rows, W1, F, swiglu ? W3 : nullptr, swiglu ? F : 0, d, dxs, offsets, mtc, tm, E,
                           false));
        // weight gradients, each expert over its own rows
        const int64_t ldcat = static_cast<int64_t>(m) * F;
        MOE_TRY(tc_sum_rows(dys, d, d, hwb, F, F, gr.dW2, offsets, tm, E, rows));          // dW2[e] = dy_s^T (w h)
        MOE_TRY(tc_sum_rows(dacat, ldcat, F, xs, d, d, gr.dW1, offsets, tm, E, rows));     // dW1[e] = da^T x_s
        if (swiglu) MOE_TRY(tc_sum_rows(dacat + F, ldcat, F, xs, d, d, gr.dW3, offsets, tm, E, rows));
    } else {
        // ---- fp32: the same products on the CUDA cores
        MOE_TRY(GG().a(xs, d, 1, bf).b(W1, 1, d, static_cast<int64_t>(F) * d, bf).c(pre, F, 1, 0)
                    .rows(offsets, mt, E, rows, F, d, s));
        if (swiglu)
            MOE_TRY(GG().a(xs, d, 1, bf).b(W3, 1, d, static_cast<int64_t>(F) * d, bf).c(up, F, 1, 0)
                        .rows(offsets, mt, E, rows, F, d, s));
        MOE_TRY(launch_act_forward(act, sms, s));
        // output side: dh = dy_s W2[e]; gates, activation backward
        MOE_TRY(GG().a(dys, d, 1, bf).b(W2, F, 1, static_cast<int64_t>(d) * F, bf).c(dh, F, 1, 0)
                    .rows(offsets, mt, E, rows, F, d, s));
        MOE_TRY(launch_row_backward(act, sms, s));
        // dW2[e] = dy_s^T (w h)
        MOE_TRY(GG().a(dys, 1, d, bf).b(h, F, 1, 0, false).c(gr.dW2, F, 1, static_cast<int64_t>(d) * F)
                    .sum_rows(offsets, E, d, F, s));
        // input side: dx_s = da W1[e] (+ du W3[e]); dW1, dW3
        MOE_TRY(GG().a(pre, F, 1, false).b(W1, d, 1, static_cast<int64_t>(F) * d, bf).c(dxs, d, 1, 0)
                    .rows(offsets, mt, E, rows, d, F, s));
        if (swiglu)
            MOE_TRY(GG().a(up, F, 1, false).b(W3, d, 1, static_cast<int64_t>(F) * d, bf).c(dxs, d, 1, 0, true)
                        .rows(offsets, mt, E, rows, d, F, s));
        MOE_TRY(GG().a(pre, 1, F, false).b(xs, d, 1, 0, bf).c(gr.dW1, d, 1, static_cast<int64_t>(F) * d)
                    .sum_rows(offsets, E, F, d, s));
        if (swiglu)
            MOE_TRY(GG().a(up, 1, F, false).b(xs, d, 1, 0, bf).c(gr.dW3, d, 1, static_cast<int64_t>(F) * d)
                        .sum_rows(offsets, E, F, d, s));
    }
    // bias gradients: db2[e] = sum_r w_r dy_s r, db1[e] = sum_r da_r
    if (b2 && gr.db2)
        MOE_TRY(GG().a(dys, 1, d, bf).b(row_w, 1, 0, 0, false).c(gr.db2, 1, 0, d).sum_rows(offsets, E, d, 1, s));
    if (!swiglu && b1 && gr.db1)
        MOE_TRY(GG().a(pre, 1, F, false).b(one, 0, 0, 0, false).c(gr.db1, 1, 0, F).sum_rows(offsets, E, F, 1, s));
    // ---- router: dz; dx = sum_j dx_s (+ dz W_g, folded in for E <= 32); dW_g = dz^T x
    BwdRouterArgs rb{probs, lse, ids, dw, counts, dz, N, E, k, cfg->router, cfg->norm_topk, cfg->routed_scaling,
                     aux_coef, z_coef};
    MOE_TRY(launch_router_backward(rb, sms, s));
    const bool fold_router_dx = E <= 32;
    BwdGatherSumArgs gs{dxs, inv, gr.dx, N, d, k, fold_router_dx ? dz : nullptr, W_g, E, bf ? 1 : 0};
    MOE_TRY(launch_gather_sum(gs, sms, s));
    MOE_TRY(GG().split(partial).a(dz, 1, E, false).b(x, d, 1, 0, bf).c(gr.dW_g, d, 1, 0).sum_rows(doff, 1, E, d, s));
    if (!fold_router_dx)
        MOE_TRY(GG().a(dz, E, 1, false).b(W_g, d, 1, 0, bf).c(gr.dx, d, 1, 0, true).rows(doff, dmt, 1, N, d, E, s));

    // ---- shared expert: the same with weight 1 over all N rows of x
    if (shared) {
        float *spre = at<float>(ws, L.spre), *sup = swiglu ? at<float>(ws, L.sup) : nullptr;
        float *sh = at<float>(ws, L.sh), *sdh = at<float>(ws, L.sdh);
        BwdActArgs sa{N, Fs, d, cfg->act, bf ? 1 : 0, spre, sup, sh, sdh, swiglu ? nullptr : shared->b1, nullptr,
                      nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
        if (bf) {  // tensor cores, one group of N rows
            const int stm = shared_tile_m(cfg);
            int32_t *smt = at<int32_t>(ws, L.smtc);
            auto *sdcat = at<__nv_bfloat16>(ws, L.sdcat), *shb = at<__nv_bfloat16>(ws, L.shb);
            MOE_TRY(launch_tile_table(doff, smt, 1, stm, s));
            MOE_TRY(tc_rows(x, N, d, shared->W1, Fs, spre, doff, smt, stm, 1, false));
            if (swiglu) MOE_TRY(tc_rows(x, N, d, shared->W3, Fs, sup, doff, smt, stm, 1, false));
            MOE_TRY(launch_act_forward(sa, sms, s));
            MOE_TRY(tc_rows_mn(dy, N, shared->W2, d, nullptr, 0, Fs, sdh, doff, smt, stm, 1, false));
            sa.dcat = sdcat;
            sa.hw_bf = shb;
            sa.skip_f32 = kSkipUp | kSkipH | ((!swiglu && shared->b1 && gr.dbs1) ? 0 : kSkipPre);
            MOE_TRY(launch_row_backward(sa, sms, s));
            MOE_TRY(tc_rows_mn(sdcat, N, shared->W1, Fs, swiglu ? shared->W3 : nullptr, swiglu ? Fs : 0, d, gr.dx,
                               doff, smt, stm, 1, true));
            const int64_t ldcat = static_cast<int64_t>(m) * Fs;
            MOE_TRY(tc_sum_rows(dy, d, d, shb, Fs, Fs, gr.dWs2, doff, stm, 1, N));
            MOE_TRY(tc_sum_rows(sdcat, ldcat, Fs, x, d, d, gr.dWs1, doff, stm, 1, N));
            if (swiglu) MOE_TRY(tc_sum_rows(sdcat + Fs, ldcat, Fs, x, d, d, gr.dWs3, doff, stm, 1, N));
        } else {
            MOE_TRY(GG().a(x, d, 1, bf).b(shared->W1, 1, d, 0, bf).c(spre, Fs, 1, 0).rows(doff, dmt, 1, N, Fs, d, s));
            if (swiglu)
                MOE_TRY(GG().a(x, d, 1, bf).b(shared->W3, 1, d, 0, bf).c(sup, Fs, 1, 0).rows(doff, dmt, 1, N, Fs, d, s));
            MOE_TRY(launch_act_forward(sa, sms, s));
            MOE_TRY(GG().a(dy, d, 1, bf).b(shared->W2, Fs, 1, 0, bf).c(sdh, Fs, 1, 0).rows(doff, dmt, 1, N, Fs, d, s));
            MOE_TRY(launch_row_backward(sa, sms, s));
            MOE_TRY(GG().split(partial).a(dy, 1, d, bf).b(sh, Fs, 1, 0, false).c(gr.dWs2, Fs, 1, 0)
                        .sum_rows(doff, 1, d, Fs, s));
            MOE_TRY(GG().split(partial).a(spre, 1, Fs, false).b(x, d, 1, 0, bf).c(gr.dWs1, d, 1, 0)
                        .sum_rows(doff, 1, Fs, d, s));
            if (swiglu)
                MOE_TRY(GG().split(partial).a(sup, 1, Fs, false).b(x, d, 1, 0, bf).c(gr.dWs3, d, 1, 0)
                            .sum_rows(doff, 1, Fs, d, s));
            MOE_TRY(GG().a(spre, Fs, 1, false).b(shared->W1, d, 1, 0, bf).c(gr.dx, d, 1, 0, true)
                        .rows(doff, dmt, 1, N, d, Fs, s));
            if (swiglu)
                MOE_TRY(GG().a(sup, Fs, 1, false).b(shared->W3, d, 1, 0, bf).c(gr.dx, d, 1, 0, true)
                            .rows(doff, dmt, 1, N, d, Fs, s));
        }
        if (shared->b2 && gr.dbs2)
            MOE_TRY(GG().split(partial).a(dy, 1, d, bf).b(one, 0, 0, 0, false).c(gr.dbs2, 1, 0, 0)
                        .sum_rows(doff, 1, d, 1, s));
        if (!swiglu && shared->b1 && gr.dbs1)
            MOE_TRY(GG().split(partial).a(spre, 1, Fs, false).b(one, 0, 0, 0, false).c(gr.dbs1, 1, 0, 0)
                        .sum_rows(doff, 1, Fs, 1, s));
    }
#undef MOE_TRY
    return MOE_OK;
}

}  // extern "C"
