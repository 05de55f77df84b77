// backward.cu -- element-wise and per-token kernels of the layer backward.
//
// The scalar differentiated is loss = <dy, y> + aux_coef L_aux + z_coef L_z
// for the forward of the course module (sec. 2.1 with the sec. 2.3 Switch
// loss) and the "nano-moe" router z-loss.  The expert choice and f_e are
// piecewise constant; the selection bias only selects.  Everything here is
// fp32; the products between these kernels run on the tensor-core GEMM
// (bf16 layers) or gemm_generic_kernel (fp32 layers).
#include <float.h>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace moe {
namespace {

__device__ __forceinline__ float sigmoidf_(float v) { return 1.0f / (1.0f + expf(-v)); }

// Element i of a layer-dtype array (bf16 or fp32).
__device__ __forceinline__ float ldv(const void *p, int64_t i, int bf16)
{
    return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]) : static_cast<const float *>(p)[i];
}

// Per sorted row r: its token, gate weight and expert (from perm and the
// routing); thread 0 of block 0 also stores the constant 1.0 that the bias
// gradients use as a one-element B operand.
__global__ void rows_prep_kernel(BwdRowsArgs a)
{
    pdl_enter();
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.one = 1.0f;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < a.rows;
         r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t asg = a.perm[r];
        a.row_tok[r] = asg / a.k;
        a.row_w[r] = a.w[asg];
        a.row_e[r] = a.ids[asg];
    }
}

// Pre-activations a (+ b1 for GELU) and the hidden activations h, four
// elements per thread (F is a multiple of 8).
__global__ void act_forward_kernel(BwdActArgs a)
{
    pdl_enter();
    const int64_t total4 = a.rows * a.F / 4;
    const bool swiglu = a.act == kSwiglu;
    for (int64_t i4 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i4 < total4;
         i4 += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = i4 * 4;
        float4 p = *reinterpret_cast<const float4 *>(a.pre + i);
        float v[4] = {p.x, p.y, p.z, p.w}, h[4];
        if (swiglu) {
            const float4 u = *reinterpret_cast<const float4 *>(a.up + i);
            const float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) h[q] = silu(v[q]) * uv[q];
        } else {
            if (a.b1) {
                const int64_t r = i / a.F;
                const int f = static_cast<int>(i - r * a.F);
                const int e = a.row_e ? a.row_e[r] : 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) v[q] += ldv(a.b1, static_cast<int64_t>(e) * a.F + f + q, a.bf16);
                *reinterpret_cast<float4 *>(a.pre + i) = make_float4(v[0], v[1], v[2], v[3]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) h[q] = gelu_erf(v[q]);
        }
        *reinterpret_cast<float4 *>(a.h + i) = make_float4(h[0], h[1], h[2], h[3]);
    }
}

// One warp per sorted row r, given dh_raw = dy_s W2[e] (the output gradient
// before the gate weight), in one pass over the row with 4-float vectors:
//   dw_r = <dh_raw_r, h_r> + <dy_s r, b2[e]>     (= <dy_n, Expert_e(x_n)>)
//   dh = w_r dh_raw_r through the activation: pre <- da, up <- du, and
//   h <- w_r h (the right operand of dW2 = dy_s^T (w h)); with dcat and
//   hw_bf also the bf16 copies [da | du] and w h that the tensor-core
//   products read (fp32 results in skip_f32 are then not written back).
// Without a weight array (the shared expert) w_r = 1 and dw is not kept.
__global__ void __launch_bounds__(256) row_backward_kernel(BwdActArgs a)
{
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const bool swiglu = a.act == kSwiglu;
    const int64_t wcat = swiglu ? 2LL * a.F : a.F;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < a.rows;
         r += warps) {
        const float wr = a.row_w ? a.row_w[r] : 1.0f;
        const int e = a.row_e ? a.row_e[r] : 0;
        float *pre = a.pre + r * a.F;
        float *up = swiglu ? a.up + r * a.F : nullptr;
        float *h = a.h + r * a.F;
        const float *dh = a.dh + r * a.F;
        float s = 0.f;
        for (int f = lane * 4; f < a.F; f += 128) {  // F is a multiple of 8
            const float4 dh4 = *reinterpret_cast<const float4 *>(dh + f);
            float4 h4 = *reinterpret_cast<const float4 *>(h + f);
            float4 p4 = *reinterpret_cast<const float4 *>(pre + f);
            float4 u4 = swiglu ? *reinterpret_cast<const float4 *>(up + f) : make_float4(0.f, 0.f, 0.f, 0.f);
            float dhv[4] = {dh4.x, dh4.y, dh4.z, dh4.w}, hv[4] = {h4.x, h4.y, h4.z, h4.w};
            float pv[4] = {p4.x, p4.y, p4.z, p4.w}, uv[4] = {u4.x, u4.y, u4.z, u4.w};
            float da[4], du[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                s += dhv[q] * hv[q];
                const float g = wr * dhv[q];
                const float v = pv[q];
                if (swiglu) {
                    const float sg = sigmoidf_(v);
                    da[q] = g * uv[q] * sg * (1.0f + v * (1.0f - sg));
                    du[q] = g * v * sg;
                } else {
                    const float Phi = 0.5f * (1.0f + erff(v * 0.70710678118654752f));
                    const float phi = 0.39894228040143268f * expf(-0.5f * v * v);
                    da[q] = g * (Phi + v * phi);
                    du[q] = 0.f;
                }
                hv[q] *= wr;
            }
            if (!(a.skip_f32 & kSkipPre)) *reinterpret_cast<float4 *>(pre + f) = make_float4(da[0], da[1], da[2], da[3]);
            if (swiglu && !(a.skip_f32 & kSkipUp))
                *reinterpret_cast<float4 *>(up + f) = make_float4(du[0], du[1], du[2], du[3]);
            if (!(a.skip_f32 & kSkipH)) *reinterpret_cast<float4 *>(h + f) = make_float4(hv[0], hv[1], hv[2], hv[3]);
            if (a.hw_bf) {
                __nv_bfloat16 b4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) b4[q] = __float2bfloat16_rn(hv[q]);
                *reinterpret_cast<uint2 *>(a.hw_bf + r * a.F + f) = *reinterpret_cast<const uint2 *>(b4);
            }
            if (a.dcat) {
                __nv_bfloat16 b4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) b4[q] = __float2bfloat16_rn(da[q]);
                *reinterpret_cast<uint2 *>(a.dcat + r * wcat + f) = *reinterpret_cast<const uint2 *>(b4);
                if (swiglu) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) b4[q] = __float2bfloat16_rn(du[q]);
                    *reinterpret_cast<uint2 *>(a.dcat + r * wcat + a.F + f) = *reinterpret_cast<const uint2 *>(b4);
                }
            }
        }
        if (a.dw) {
            if (a.b2) {
                for (int c = lane; c < a.d; c += 32)
                    s += ldv(a.dy_s, r * a.d + c, a.bf16) * ldv(a.b2, static_cast<int64_t>(e) * a.d + c, a.bf16);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) a.dw[a.perm[r]] = s;
        }
    }
}

// dx_n = sum_j dx_s[inv_perm[n k + j]] (+ sum_e dz[n, e] W_g[e, :]) (fp32),
// one warp per token.
__global__ void __launch_bounds__(256) gather_sum_kernel(BwdGatherSumArgs a)
{
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.N;
         n += warps) {
        const int src_l = lane < a.k ? a.inv_perm[n * a.k + lane] : 0;
        const float dz_l = (a.dz && lane < a.E) ? a.dz[n * a.E + lane] : 0.f;
        for (int c0 = 0; c0 < a.d; c0 += 128) {  // warp-uniform; 4 columns per lane (d is a multiple of 8)
            const int c = c0 + lane * 4;
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < a.k; ++j) {  // fixed order over the token's k rows
                const int src = __shfl_sync(0xffffffffu, src_l, j);
                if (c < a.d) {
                    const float4 v = *reinterpret_cast<const float4 *>(a.dxs + static_cast<int64_t>(src) * a.d + c);
                    s.x += v.x;
                    s.y += v.y;
                    s.z += v.z;
                    s.w += v.w;
                }
            }
            if (a.dz) {
                for (int e = 0; e < a.E; ++e) {  // fixed order over the experts
                    const float z = __shfl_sync(0xffffffffu, dz_l, e);
                    if (c < a.d) {
                        const int64_t o = static_cast<int64_t>(e) * a.d + c;
                        float4 wv;
                        if (a.bf16) {
                            const uint2 q = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(a.W_g) + o);
                            const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&q.x);
                            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&q.y);
                            wv = make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
                        } else {
                            wv = *reinterpret_cast<const float4 *>(static_cast<const float *>(a.W_g) + o);
                        }
                        s.x = fmaf(z, wv.x, s.x);
                        s.y = fmaf(z, wv.y, s.y);
                        s.z = fmaf(z, wv.z, s.z);
                        s.w = fmaf(z, wv.w, s.w);
                    }
                }
            }
            if (c < a.d) *reinterpret_cast<float4 *>(a.dx + n * a.d + c) = s;
        }
    }
}

// Router backward, one warp per token (lane l holds experts l + 32 j).
// dg_e = routed_scaling dw_j for the chosen experts; then per router
//   softmax_topk: dp = dg (/ S - <dg, p>_T / S^2 with norm_topk)
//   topk_softmax: dz_T = g (dg - <g, dg>_T), g = p / S over the chosen
//   sigmoid:      ds = dg (/ S - <dg, s>_T / S^2), dz = ds s (1 - s),
//                 s = sigmoid(z), z = log p + lse
// plus dp_e += aux_coef E f_e / N (Switch loss through P_e), dz += p (dp -
// <p, dp>) (softmax), dz += z_coef 2 lse p / N (z-loss).
__global__ void __launch_bounds__(256) router_backward_kernel(BwdRouterArgs a)
{
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int E = a.E, k = a.k;
    const float invN = 1.0f / static_cast<float>(a.N);
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.N;
         n += warps) {
        const float *p = a.probs + n * E;
        const float lse = a.lse[n];
        // the k choices: lane j < k holds id, p, dg and (sigmoid) s
        const int id_l = lane < k ? a.ids[n * k + lane] : 0;
        const float p_l = lane < k ? p[id_l] : 0.f;
        const float dg_l = lane < k ? a.scaling * a.dw[n * k + lane] : 0.f;
        const float s_l = (lane < k && a.router == kSigmoid) ? sigmoidf_(logf(p_l) + lse) : 0.f;
        float S = 0.f, gdot = 0.f;
        if (a.router == kSigmoid) {
            S = s_l;
            gdot = dg_l * s_l;
        } else {
            S = p_l;
            gdot = dg_l * p_l;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            S += __shfl_xor_sync(0xffffffffu, S, o);
            gdot += __shfl_xor_sync(0xffffffffu, gdot, o);
        }
        // per chosen expert: its dp (softmax path) or its direct dz
        float dp_l = 0.f, dzd_l = 0.f;
        if (lane < k) {
            if (a.router == kSoftmaxTopk) {
                dp_l = a.norm_topk ? dg_l / S - gdot / (S * S) : dg_l;
            } else if (a.router == kTopkSoftmax) {
                const float g = p_l / S;
                dzd_l = g * (dg_l - gdot / S);
            } else {
                const float ds = a.norm_topk ? dg_l / S - gdot / (S * S) : dg_l;
                dzd_l = ds * s_l * (1.0f - s_l);
            }
        }
        // expert e's dp and direct dz, <p, dp>; the shuffles run in every
        // lane (warp-uniform loops), only the accumulation is per lane
        float dp[8], dzd[8], pdp = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            dp[j] = 0.f;
            dzd[j] = 0.f;
        }
        for (int q = 0; q < k; ++q) {
            const int idq = __shfl_sync(0xffffffffu, id_l, q);
            const float dpq = __shfl_sync(0xffffffffu, dp_l, q);
            const float dzq = __shfl_sync(0xffffffffu, dzd_l, q);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (idq == lane + 32 * j) {
                    dp[j] += dpq;
                    dzd[j] += dzq;
                }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            if (e < E) {
                dp[j] += a.aux_coef * static_cast<float>(E) * (static_cast<float>(a.counts[e]) * invN) * invN;
                pdp += p[e] * dp[j];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            if (e < E) {
                float dz = dzd[j] + p[e] * (dp[j] - pdp);
                if (a.z_coef != 0.f) dz += a.z_coef * 2.0f * lse * p[e] * invN;
                a.dz[n * E + e] = dz;
            }
        }
    }
}

int grid_for(int64_t work, int per_block, int num_sms)
{
    const int64_t want = (work + per_block - 1) / per_block;
    return static_cast<int>(max64(1, min64(want, static_cast<int64_t>(num_sms) * 16)));
}

}  // namespace

cudaError_t launch_rows_prep(const BwdRowsArgs &a, int num_sms, cudaStream_t s)
{
    return launch_k(rows_prep_kernel, dim3(grid_for(max64(a.rows, 1), 256, num_sms)), dim3(256), 0, s, a);
}

cudaError_t launch_act_forward(const BwdActArgs &a, int num_sms, cudaStream_t s)
{
    if (a.rows == 0) return cudaSuccess;
    return launch_k(act_forward_kernel, dim3(grid_for(a.rows * a.F / 4, 256, num_sms)), dim3(256), 0, s, a);
}

cudaError_t launch_row_backward(const BwdActArgs &a, int num_sms, cudaStream_t s)
{
    if (a.rows == 0) return cudaSuccess;
    return launch_k(row_backward_kernel, dim3(grid_for(a.rows, 8, num_sms)), dim3(256), 0, s, a);
}

cudaError_t launch_gather_sum(const BwdGatherSumArgs &a, int num_sms, cudaStream_t s)
{
    if (a.N == 0) return cudaSuccess;
    return launch_k(gather_sum_kernel, dim3(grid_for(a.N, 8, num_sms)), dim3(256), 0, s, a);
}

cudaError_t launch_router_backward(const BwdRouterArgs &a, int num_sms, cudaStream_t s)
{
    if (a.N == 0) return cudaSuccess;
    return launch_k(router_backward_kernel, dim3(grid_for(a.N, 8, num_sms)), dim3(256), 0, s, a);
}

}  // namespace moe
