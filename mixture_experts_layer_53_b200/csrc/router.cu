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

// (value desc, id asc): does candidate (v, e) rank ahead of (bv, be)?
__device__ __forceinline__ bool ahead(float v, int e, float bv, int be)
{
    return v > bv || (v == bv && e < be);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) router_kernel(RouterArgs a)
{
    extern __shared__ float smem[];
    const int E = a.E, d = a.d, k = a.k;
    const int EJ = (E + 31) >> 5;
    const int ZS = E + 1;
    float *xs = smem;                 // [kRT][kKP]
    float *ws = xs + kRT * kKP;       // [E][kKP]
    float *zt = ws + E * kKP;         // [kRT][E+1]   probabilities p
    int *ids_s = reinterpret_cast<int *>(zt + kRT * ZS);  // [kRT][k]

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
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
        const int t = warp + 8 * i;
        if (t >= ntok) break;  // warp-uniform
        const int64_t n = tok0 + t;

        float zmax = -FLT_MAX;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < EJ && lane + 32 * j < E) zmax = fmaxf(zmax, acc[i][j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));

        float ex[8], sel[8], graw[8];
        float esum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            ex[j] = 0.f; sel[j] = -FLT_MAX; graw[j] = 0.f;
            if (j < EJ && e < E) {
                ex[j] = expf(acc[i][j] - zmax);
                esum += ex[j];
                if (a.router == kSigmoid) {
                    const float sg = 1.0f / (1.0f + expf(-acc[i][j]));
                    sel[j] = sg + (a.b_sel ? a.b_sel[e] : 0.f);
                    graw[j] = sg;
                } else {
                    sel[j] = acc[i][j];
                    graw[j] = ex[j];
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) esum += __shfl_xor_sync(0xffffffffu, esum, o);
        const float inv_esum = 1.0f / esum;

        uint32_t taken = 0;
        int idsel[kMaxK];
        float gsel[kMaxK];
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            idsel[r] = 0;
            gsel[r] = 0.f;
            if (r < k) {
                float bv = -FLT_MAX, bg = 0.f;
                int be = INT_MAX;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = lane + 32 * j;
                    if (j < EJ && e < E && !((taken >> j) & 1u) && ahead(sel[j], e, bv, be)) {
                        bv = sel[j]; be = e; bg = graw[j];
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                    const float og = __shfl_xor_sync(0xffffffffu, bg, o);
                    if (ahead(ov, oe, bv, be)) { bv = ov; be = oe; bg = og; }
                }
                if ((be & 31) == lane) taken |= 1u << (be >> 5);
                idsel[r] = be;
                gsel[r] = bg;
            }
        }

        float gs = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxK; ++r)
            if (r < k) gs += gsel[r];
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            if (r < k && lane == r) {
                float wr;
                if (a.router == kSoftmaxTopk) wr = a.norm_topk ? gsel[r] / gs : gsel[r] * inv_esum;
                else if (a.router == kTopkSoftmax) wr = gsel[r] / gs;
                else wr = a.norm_topk ? gsel[r] / gs : gsel[r];
                a.ids[n * k + r] = idsel[r];
                a.w[n * k + r] = wr * a.scaling;
                ids_s[t * k + r] = idsel[r];
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            if (j < EJ && e < E) {
                const float p = ex[j] * inv_esum;
                zt[t * ZS + e] = p;
                if (a.probs) a.probs[n * E + e] = p;
            }
        }
    }
    __syncthreads();

    // ---- per-chunk statistics in a fixed order (deterministic)
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

size_t router_smem_bytes(int E, int k)
{
    return sizeof(float) * (kRT * kKP + E * kKP + kRT * (E + 1)) + sizeof(int) * kRT * k;
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
    router_kernel<T><<<static_cast<unsigned>(grid), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(int dtype, const RouterArgs &a, cudaStream_t s)
{
    return dtype == kF32 ? launch_router_t<float>(a, s) : launch_router_t<__nv_bfloat16>(a, s);
}

}  // namespace moe
