// router.cu -- fused MoE router: logits z = W_g x, softmax (or sigmoid),
// warp-shuffle top-k with the lowest-id tie rule, gate weights, and the
// per-chunk statistics the dispatch and the Switch loss need.
//
// Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
// loss, aux-free bias": sec. 2 symbol table (z_n = W_g x_n, p_n =
// softmax(z_n)), sec. 2.1 router table (softmax_topk / topk_softmax /
// sigmoid, ties to the lowest id, routed_scaling), sec. 2.5 (the bias b_e
// enters the selection score only).
//
// One CTA of 256 threads handles 32 tokens (a dispatch chunk).  Warp w owns
// tokens w, w+8, w+16, w+24; lane l owns experts l, l+32, ... so every
// logit of a token lives in one warp's registers and the top-k runs on
// shuffles without touching shared memory.  Selection for the softmax
// routers compares logits (softmax is increasing, so the chosen set equals
// that of p, without exp rounding).
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"
#include "router_select.cuh"

namespace moe {
namespace {

constexpr int kRT = 32;       // tokens per CTA
constexpr int kKC = 32;       // reduction chunk
constexpr int kKP = kKC + 1;  // padded smem row (conflict-free column reads)
constexpr int kThreads = 256;

template <typename T> struct Load4;
template <> struct Load4<float> {
    __device__ static void run(const float *p, float *f)
    {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
};
template <> struct Load4<__nv_bfloat16> {
    __device__ static void run(const __nv_bfloat16 *p, float *f)
    {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        f[0] = __uint_as_float(v.x << 16);
        f[1] = __uint_as_float(v.x & 0xFFFF0000u);
        f[2] = __uint_as_float(v.y << 16);
        f[3] = __uint_as_float(v.y & 0xFFFF0000u);
    }
};

// Sum of the chunk's per-token z-loss terms, in token order.
__device__ __forceinline__ float chunk_sum(const float *zl, int ntok)
{
    float s = 0.f;
    for (int t = 0; t < ntok; ++t) s += zl[t];
    return s;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) router_kernel(RouterArgs a)
{
    pdl_enter();
    extern __shared__ float smem[];
    const int E = a.E, d = a.d, k = a.k;
    const int EJ = (E + 31) >> 5;
    const int ZS = E + 1;
    float *xs = smem;                 // [kRT][kKP]
    float *ws = xs + kRT * kKP;       // [E][kKP]
    float *zt = ws + E * kKP;         // [kRT][E+1]   probabilities p
    int *ids_s = reinterpret_cast<int *>(zt + kRT * ZS);  // [kRT][k]
    float *zl = reinterpret_cast<float *>(ids_s + kRT * k);  // [kRT] lse^2

    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRT;
    const int ntok = static_cast<int>(min64(kRT, a.N - tok0));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const T *x = static_cast<const T *>(a.x);
    const T *Wg = static_cast<const T *>(a.Wg);

    // ---- logits: z[t][e] for t = warp + 8i, e = lane + 32j
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kKC) {
        for (int q = tid; q < kRT * (kKC / 4); q += kThreads) {
            const int t = q / (kKC / 4), c = (q % (kKC / 4)) * 4;
            float f[4] = {0.f, 0.f, 0.f, 0.f};
            if (t < ntok && k0 + c < d) Load4<T>::run(x + (tok0 + t) * d + k0 + c, f);
#pragma unroll
            for (int u = 0; u < 4; ++u) xs[t * kKP + c + u] = f[u];
        }
        for (int q = tid; q < E * (kKC / 4); q += kThreads) {
            const int e = q / (kKC / 4), c = (q % (kKC / 4)) * 4;
            float f[4] = {0.f, 0.f, 0.f, 0.f};
            if (k0 + c < d) Load4<T>::run(Wg + static_cast<int64_t>(e) * d + k0 + c, f);
#pragma unroll
            for (int u = 0; u < 4; ++u) ws[e * kKP + c + u] = f[u];
        }
        __syncthreads();
#pragma unroll 4
        for (int c = 0; c < kKC; ++c) {
            float xv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[(warp + 8 * i) * kKP + c];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < EJ) {
                    const int e = lane + 32 * j;
                    const float wv = (e < E) ? ws[e * kKP + c] : 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(xv[i], wv, acc[i][j]);
                }
            }
        }
        __syncthreads();
    }

    // ---- scores, top-k and gates, one token at a time per warp
    SelectArgs sa{a.b_sel, a.ids, a.w, a.probs, E, k, a.router, a.norm_topk, a.scaling, a.lse};
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
        const int t = warp + 8 * i;
        if (t >= ntok) break;  // warp-uniform
        float z[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) z[j] = acc[i][j];
        int sel_ids[kMaxK];
        const float lse = select_token(z, sa, tok0 + t, true, sel_ids);
        if (lane == 0) zl[t] = lse * lse;
#pragma unroll
        for (int r = 0; r < kMaxK; ++r)
            if (r < k && lane == r) ids_s[t * k + r] = sel_ids[r];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < EJ && lane + 32 * j < E) zt[t * ZS + lane + 32 * j] = z[j];
    }
    __syncthreads();

    // ---- per-chunk statistics in a fixed order (deterministic)
    if (a.zpart && tid == 0) a.zpart[blockIdx.x] = chunk_sum(zl, ntok);
    if (a.psum || a.hist) {
        for (int e = tid; e < E; e += kThreads) {
            if (a.psum) {
                float s = 0.f;
                for (int t = 0; t < ntok; ++t) s += zt[t * ZS + e];
                a.psum[static_cast<int64_t>(blockIdx.x) * E + e] = s;
            }
            if (a.hist) {
                int c = 0;
                for (int q = 0; q < ntok * k; ++q) c += (ids_s[q] == e);
                a.hist[static_cast<int64_t>(blockIdx.x) * E + e] = c;
            }
        }
    }
}

// Logit z_{n,e}: the tcgen05 router's partial sums over d, added in split
// order.
__device__ __forceinline__ float logit_of(const SelectKernelArgs &a, int64_t n, int e)
{
    const float *p = a.logits + n * a.ld + e;
    const int64_t stride = a.N * a.ld;
    float z = p[0];
    for (int s = 1; s < a.splits; ++s) z += p[s * stride];
    return z;
}

// Scores, top-k and gates from precomputed fp32 logits (the tcgen05 router
// of the bf16 path writes them), for E > 32.  One CTA per 32-token dispatch
// chunk, one warp per token (16 warps, 2 tokens each): the selection is a
// serial shuffle chain per token, so many independent warps hide its
// latency.  Each token's k choices go into a shared histogram (integer
// atomics: order-free); the chunk's sum of p is then taken per expert in
// token order.
constexpr int kSelWarps = 16;

template <int EJ>
__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(SelectKernelArgs a)
{
    pdl_enter();
    extern __shared__ float smem[];
    const int E = a.E, k = a.k;
    const int ZS = E + 1;
    float *pt = smem;                                          // [32][E+1] p
    int *hist_s = reinterpret_cast<int *>(pt + kRT * ZS);      // [E]
    float *zl = reinterpret_cast<float *>(hist_s + kMaxE);     // [32] lse^2
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRT;
    const int ntok = static_cast<int>(min64(kRT, a.N - tok0));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += kSelWarps * 32) hist_s[e] = 0;
    __syncthreads();
    const SelectArgs sa{a.b_sel, a.ids, a.w, a.probs, E, k, a.router, a.norm_topk, a.scaling, a.lse};
    // software pipeline: the next token's row is loaded while this one is
    // selected
    float znext[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
        const int e = lane + 32 * j;
        znext[j] = (warp < ntok && e < E) ? logit_of(a, tok0 + warp, e) : 0.f;
    }
#pragma unroll 1
    for (int t = warp; t < ntok; t += kSelWarps) {
        float z[EJ];
#pragma unroll
        for (int j = 0; j < EJ; ++j) z[j] = znext[j];
        const int tn = t + kSelWarps;
#pragma unroll
        for (int j = 0; j < EJ; ++j) {
            const int e = lane + 32 * j;
            znext[j] = (tn < ntok && e < E) ? logit_of(a, tok0 + tn, e) : 0.f;
        }
        int sel_id;
        const float lse = select_token_keys<EJ>(z, sa, tok0 + t, true, &sel_id);
        if (lane == 0) zl[t] = lse * lse;
        if (lane < k) atomicAdd(&hist_s[sel_id], 1);
#pragma unroll
        for (int j = 0; j < EJ; ++j)
            if (lane + 32 * j < E) pt[t * ZS + lane + 32 * j] = z[j];
    }
    __syncthreads();
    if (a.zpart && threadIdx.x == 0) a.zpart[blockIdx.x] = chunk_sum(zl, ntok);
    for (int e = threadIdx.x; e < E; e += kSelWarps * 32) {
        if (a.psum) {
            float s = 0.f;
            for (int t = 0; t < ntok; ++t) s += pt[t * ZS + e];
            a.psum[static_cast<int64_t>(blockIdx.x) * E + e] = s;
        }
        if (a.hist) a.hist[static_cast<int64_t>(blockIdx.x) * E + e] = hist_s[e];
    }
}

size_t router_smem_bytes(int E, int k)
{
    return sizeof(float) * (kRT * kKP + E * kKP + kRT * (E + 1) + kRT) + sizeof(int) * kRT * k;
}

template <typename T> cudaError_t launch_router_t(const RouterArgs &a, cudaStream_t s)
{
    const size_t smem = router_smem_bytes(a.E, a.k);
    // the largest need (E = 256, k = 16) once per device
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void *>(&router_kernel<T>),
                                       static_cast<int>(router_smem_bytes(kMaxE, kMaxK)));
    if (err != cudaSuccess) return err;
    const int64_t grid = num_chunks(a.N);
    if (grid == 0) return cudaSuccess;
    return launch_k(router_kernel<T>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, s, a);
}

}  // namespace

cudaError_t launch_select(const SelectKernelArgs &a, cudaStream_t s)
{
    const int64_t grid = num_chunks(a.N);
    if (grid == 0) return cudaSuccess;
    const size_t smem = sizeof(float) * (kRT * (a.E + 1) + kRT) + sizeof(int) * kMaxE;
    const dim3 g(static_cast<unsigned>(grid)), b(kSelWarps * 32);
    if (a.E <= 64) return launch_k(select_kernel<2>, g, b, smem, s, a);
    if (a.E <= 128) return launch_k(select_kernel<4>, g, b, smem, s, a);
    return launch_k(select_kernel<8>, g, b, smem, s, a);
}

cudaError_t launch_router(int dtype, const RouterArgs &a, cudaStream_t s)
{
    return dtype == kF32 ? launch_router_t<float>(a, s) : launch_router_t<__nv_bfloat16>(a, s);
}

}  // namespace moe
