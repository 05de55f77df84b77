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

// Scores, top-k and gates from precomputed fp32 logits (the tcgen05 router
// of the bf16 path writes them), for E > 32.  One CTA per 32-token dispatch
// chunk; a group of G lanes (up to a whole warp) owns one token, and lane q
// of the group holds a contiguous block of EJ = E_pad / G of its experts.  Each expert gets the
// 64-bit rank key of (selection score desc, id asc) (rank_key); every lane
// first sorts its EJ keys, descending, with a bitonic network.  Each of the
// k rounds is then a group max of the lanes' first keys (xor butterfly over
// the G lanes) after which the lane holding the winner drops it (its list
// moves up by one): k short rounds instead of k scans of all EJ keys.  The
// winner's logit is read back from shared memory, where the group left its
// logits; the gates' sum is formed round by round in choice order.  The
// chunk's histogram uses integer shared-memory atomics (order-free); its
// sum of p is taken per expert in token order.
//
// Before that, a shorter exact path is tried.  Let T be the k-th largest of
// the G lanes' largest keys.  Those k lanes hold k keys at or above T, so
// each of the token's k choices is at or above T: the choices are the k
// largest of the keys >= T, about ten of them for random logits at E = 128
// or 256.  When they fit one per lane (at most G of them, and k <= G), they
// are gathered through shared memory and one bitonic sort across the group
// ranks them; lane r then holds the r-th choice.  A warp in which any token
// has more candidates (ties, or k > G) takes the rounds above.  Both paths
// choose the same experts in the same order and form the gates' sum in the
// same order, so their outputs are bitwise equal.
template <int N> __device__ __forceinline__ void bitonic_sort_desc(uint64_t (&v)[N])
{
#pragma unroll
    for (int blk = 2; blk <= N; blk <<= 1)
#pragma unroll
        for (int j = blk >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const uint64_t a = v[i], b = v[l];
                    const bool sw = (i & blk) == 0 ? a < b : a > b;  // this block descending, or ascending
                    v[i] = sw ? b : a;
                    v[l] = sw ? a : b;
                }
            }
}

// Sorts one 64-bit key per lane descending across each group of G lanes
// (lane q of the group ends with the q-th largest), q = lane % G.
template <int G> __device__ __forceinline__ uint64_t group_sort_desc(uint64_t v, int q)
{
#pragma unroll
    for (int blk = 2; blk <= G; blk <<= 1)
#pragma unroll
        for (int j = blk >> 1; j > 0; j >>= 1) {
            const uint64_t o = __shfl_xor_sync(0xffffffffu, v, j);
            const bool keep_max = ((q & blk) == 0) == ((q & j) == 0);
            v = keep_max ? (o > v ? o : v) : (o < v ? o : v);
        }
    return v;
}

template <int EJ, int G>
__global__ void __launch_bounds__(kRT * G) select_kernel(SelectKernelArgs a)
{
    pdl_enter();
    extern __shared__ float smem[];
    const int E = a.E, k = a.k;
    const int ZS = E + 1;
    float *pt = smem;                                          // [32][E+1] z, then p
    int *hist_s = reinterpret_cast<int *>(pt + kRT * ZS);      // [E]
    float *zl = reinterpret_cast<float *>(hist_s + kMaxE);     // [32] lse^2
    uint64_t *cand = reinterpret_cast<uint64_t *>(               // [32][G] candidate keys (8-byte aligned)
        reinterpret_cast<uintptr_t>(zl + kRT + 1) & ~static_cast<uintptr_t>(7));
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRT;
    const int ntok = static_cast<int>(min64(kRT, a.N - tok0));
    const int lane = threadIdx.x & 31, q = lane & (G - 1);
    const int t = threadIdx.x / G;  // token of this lane's group, 0..31
    const bool live = t < ntok;
    const int64_t n = tok0 + t;
    const int e0 = q * EJ;  // this lane's experts e0 .. e0 + EJ - 1
    float *zrow = pt + t * ZS;
    for (int e = threadIdx.x; e < E; e += kRT * G) hist_s[e] = 0;

    // logits: the splits' partial sums in split order
    float z[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) z[j] = 0.f;
    if (live) {
        const float *row = a.logits + n * a.ld;
        const int64_t stride = a.N * a.ld;
        for (int sp = 0; sp < a.splits; ++sp) {
#pragma unroll
            for (int j = 0; j < EJ; j += 4) {
                if (e0 + j < a.ld) {  // ld and EJ are multiples of 4: whole float4s in or out
                    const float4 v = *reinterpret_cast<const float4 *>(row + sp * stride + e0 + j);
                    z[j] += v.x;
                    z[j + 1] += v.y;
                    z[j + 2] += v.z;
                    z[j + 3] += v.w;
                }
            }
        }
    }
    // softmax over all E (p = exp(z - max) / sum), in the group
    float zmax = -FLT_MAX;
#pragma unroll
    for (int j = 0; j < EJ; ++j)
        if (e0 + j < E) zmax = fmaxf(zmax, z[j]);
#pragma unroll
    for (int o = 1; o < G; o <<= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
    float ex[EJ], esum = 0.f;
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
        ex[j] = e0 + j < E ? expf(z[j] - zmax) : 0.f;
        esum += ex[j];
    }
#pragma unroll
    for (int o = 1; o < G; o <<= 1) esum += __shfl_xor_sync(0xffffffffu, esum, o);
    const float inv_esum = 1.0f / esum;
    const float lse = zmax + logf(esum);
    // selection keys (0: below every real key), sorted; the logits to shared
    // memory for the gates
    uint64_t key[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
        const int e = e0 + j;
        key[j] = 0ull;
        if (e < E) {
            float sc = z[j];
            if (a.router == kSigmoid) sc = 1.0f / (1.0f + expf(-z[j])) + (a.b_sel ? a.b_sel[e] : 0.f);
            key[j] = rank_key(sc, e);
            zrow[e] = z[j];
        }
    }
    auto raw_gate = [&](float zr) {
        return a.router == kSigmoid ? 1.0f / (1.0f + expf(-zr)) : expf(zr - zmax);
    };
    int my_id = -1, my_id2 = -1;  // lane q < k (and q + G < k): the q-th (q + G-th) choice
    float my_z = 0.f, my_z2 = 0.f, gs = 0.f;
    // the candidates: keys at or above T, the k-th largest lane maximum
    uint64_t lane_max = 0ull;
#pragma unroll
    for (int j = 0; j < EJ; ++j) lane_max = key[j] > lane_max ? key[j] : lane_max;
    const uint64_t T = __shfl_sync(0xffffffffu, group_sort_desc<G>(lane_max, q), k <= G ? k - 1 : 0, G);
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < EJ; ++j) cnt += (key[j] != 0ull && key[j] >= T) ? 1 : 0;
    int before = cnt;  // inclusive prefix of cnt over the group's lanes
#pragma unroll
    for (int o = 1; o < G; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, before, o, G);
        if (q >= o) before += u;
    }
    const int C = __shfl_sync(0xffffffffu, before, G - 1, G);
    before -= cnt;
    const bool fits = k <= G && T != 0ull && C <= G;
    __syncwarp();  // the group's logits are in shared memory
    if (__all_sync(0xffffffffu, fits)) {
        // this lane's candidates to slots before .. before + cnt - 1 of its
        // token's G slots (C <= G of them in all)
        uint64_t *slots = cand + t * G;
#pragma unroll
        for (int j = 0; j < EJ; ++j)
            if (key[j] != 0ull && key[j] >= T) slots[before++] = key[j];
        __syncwarp();
        const uint64_t mine = group_sort_desc<G>(q < C ? slots[q] : 0ull, q);
        // lane r < k: the r-th choice (every one of them a real key: C >= k)
        const int e = 0xFFFF - static_cast<int>(mine & 0xFFFFu);
        const float ez = q < k ? zrow[e] : 0.f;
        const float g = raw_gate(ez);
        for (int r = 0; r < k; ++r) gs += __shfl_sync(0xffffffffu, g, r, G);
        if (q < k) {
            my_id = e;
            my_z = ez;
        }
    } else {
    bitonic_sort_desc(key);
    // k rounds: the group's largest remaining key
#pragma unroll 1
    for (int r = 0; r < k; ++r) {
        uint64_t best = key[0];
#pragma unroll
        for (int o = 1; o < G; o <<= 1) {
            const uint64_t ob = __shfl_xor_sync(0xffffffffu, best, o);
            best = ob > best ? ob : best;
        }
        if (key[0] == best) {  // the winner's lane (keys are unique)
#pragma unroll
            for (int j = 0; j + 1 < EJ; ++j) key[j] = key[j + 1];
            key[EJ - 1] = 0ull;
        }
        const int e = 0xFFFF - static_cast<int>(best & 0xFFFFu);
        const float ez = zrow[e];
        gs += raw_gate(ez);
        if (q == r) {
            my_id = e;
            my_z = ez;
        }
        if (q + G == r) {
            my_id2 = e;
            my_z2 = ez;
        }
    }
    }
    // gates: raw gate of each choice over their sum (in choice order), then
    // this lane's one or two outputs
    auto weight = [&](float zr) {
        const float g = raw_gate(zr);
        float wr;
        if (a.router == kSoftmaxTopk) wr = a.norm_topk ? g / gs : g * inv_esum;
        else if (a.router == kTopkSoftmax) wr = g / gs;
        else wr = a.norm_topk ? g / gs : g;
        return wr * a.scaling;
    };
    if (live) {
        if (q < k) {
            a.ids[n * k + q] = my_id;
            a.w[n * k + q] = weight(my_z);
            atomicAdd(&hist_s[my_id], 1);
        }
        if (q + G < k) {
            a.ids[n * k + q + G] = my_id2;
            a.w[n * k + q + G] = weight(my_z2);
            atomicAdd(&hist_s[my_id2], 1);
        }
        if (q == 0) {
            zl[t] = lse * lse;
            if (a.lse) a.lse[n] = lse;
        }
    }
    __syncwarp();  // the group's logits have been read: p replaces them
    // p for the chunk's sums (and probs if asked for)
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
        const int e = e0 + j;
        if (e < E) {
            const float p = live ? ex[j] * inv_esum : 0.f;
            zrow[e] = p;
            if (live && a.probs) a.probs[n * E + e] = p;
        }
    }
    __syncthreads();
    if (a.zpart && threadIdx.x == 0) a.zpart[blockIdx.x] = chunk_sum(zl, ntok);
    for (int e = threadIdx.x; e < E; e += kRT * G) {
        if (a.psum) {
            float s = 0.f;
            for (int tt = 0; tt < ntok; ++tt) s += pt[tt * ZS + e];
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
    // logits rows of ld >= E columns, a multiple of 4 (columns E .. ld-1 are
    // read as whole float4s and ignored)
    if (a.ld % 4 != 0 || a.ld < a.E || a.E > kMaxE) return cudaErrorInvalidValue;
    // logits / p rows, histogram, z-loss terms, then (8-byte aligned, at
    // most 4 bytes of padding) G candidate keys per token
    auto smem = [&](int G) {
        return sizeof(float) * (kRT * (a.E + 1) + kRT) + sizeof(int) * kMaxE + 8 + sizeof(uint64_t) * kRT * G;
    };
    // experts per lane x lanes per token: 8 x 8, 8 x 16 or 8 x 32 (eight keys
    // per lane keep the registers low enough for 32 warps per SM)
    const dim3 g(static_cast<unsigned>(grid));
    if (a.E <= 64) return launch_k(select_kernel<8, 8>, g, dim3(kRT * 8), smem(8), s, a);
    if (a.E <= 128) return launch_k(select_kernel<8, 16>, g, dim3(kRT * 16), smem(16), s, a);
    return launch_k(select_kernel<8, 32>, g, dim3(kRT * 32), smem(32), s, a);
}

cudaError_t launch_router(int dtype, const RouterArgs &a, cudaStream_t s)
{
    return dtype == kF32 ? launch_router_t<float>(a, s) : launch_router_t<__nv_bfloat16>(a, s);
}

}  // namespace moe
