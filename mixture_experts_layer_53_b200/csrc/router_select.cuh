// router_select.cuh -- scores, top-k and gates of one token, computed by one
// warp with the token's E logits spread over the lanes (lane l holds experts
// l, l+32, ...).  Shared by the CUDA-core router and the tcgen05 router.
//
// Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
// loss, aux-free bias": sec. 2 symbol table (p_n = softmax(z_n)), sec. 2.1
// router table (softmax_topk / topk_softmax / sigmoid, ties to the lowest id,
// routed_scaling), sec. 2.5 (b_e enters the selection score only).
// Selection for the softmax routers compares logits: softmax is increasing,
// so the chosen set and slot order are those of p, without exp rounding.
#pragma once

#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

struct SelectArgs {
    const float *b_sel;  // [E] or null
    int32_t *ids;        // [N, k]
    float *w;            // [N, k]
    float *probs;        // [N, E] or null
    int E, k, router, norm_topk;
    float scaling;
    float *lse;          // [N] log-sum-exp of each token's logits, or null
};

// (value desc, id asc): does (v, e) rank ahead of (bv, be)?
__device__ __forceinline__ bool rank_ahead(float v, int e, float bv, int be)
{
    return v > bv || (v == bv && e < be);
}

// z[j] = logit of expert lane + 32 j (j < ceil(E/32) <= 8).  Writes the
// token's ids / weights / probs rows (if `write`), returns p in z[] and the
// chosen ids in sel_ids[0..k) (valid in every lane).  The return value is
// log sum_e exp z_e (every lane), the token's term of the router z-loss
// ("nano-moe", "Router z-loss").
__device__ __forceinline__ float select_token(float (&z)[8], const SelectArgs &a, int64_t n, bool write,
                                             int (&sel_ids)[kMaxK])
{
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    const int EJ = (E + 31) >> 5;
    float zmax = -FLT_MAX;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < EJ && lane + 32 * j < E) zmax = fmaxf(zmax, z[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));

    float ex[8], sel[8], graw[8];
    float esum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        ex[j] = 0.f;
        sel[j] = -FLT_MAX;
        graw[j] = 0.f;
        if (j < EJ && e < E) {
            ex[j] = expf(z[j] - zmax);
            esum += ex[j];
            if (a.router == kSigmoid) {
                const float sg = 1.0f / (1.0f + expf(-z[j]));
                sel[j] = sg + (a.b_sel ? a.b_sel[e] : 0.f);
                graw[j] = sg;
            } else {
                sel[j] = z[j];
                graw[j] = ex[j];
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) esum += __shfl_xor_sync(0xffffffffu, esum, o);
    const float inv_esum = 1.0f / esum;

    // k rounds of a warp argmax under the (score desc, id asc) order.  The
    // round loop stays rolled (small code); results land in the register
    // arrays through static-index selects.
    uint32_t taken = 0;
    float gsel[kMaxK];
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
        sel_ids[r] = 0;
        gsel[r] = 0.f;
    }
#pragma unroll 1
    for (int r = 0; r < k; ++r) {
        float bv = -FLT_MAX, bg = 0.f;
        int be = INT_MAX;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane + 32 * j;
            if (j < EJ && e < E && !((taken >> j) & 1u) && rank_ahead(sel[j], e, bv, be)) {
                bv = sel[j];
                be = e;
                bg = graw[j];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float og = __shfl_xor_sync(0xffffffffu, bg, o);
            if (rank_ahead(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
                bg = og;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j == r) {
                sel_ids[j] = be;
                gsel[j] = bg;
            }
    }

    float gs = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxK; ++r)
        if (r < k) gs += gsel[r];
    if (write && a.lse && lane == 0) a.lse[n] = zmax + logf(esum);
    if (write) {
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            if (r < k && lane == r) {
                float wr;
                if (a.router == kSoftmaxTopk) wr = a.norm_topk ? gsel[r] / gs : gsel[r] * inv_esum;
                else if (a.router == kTopkSoftmax) wr = gsel[r] / gs;
                else wr = a.norm_topk ? gsel[r] / gs : gsel[r];
                a.ids[n * k + r] = sel_ids[r];
                a.w[n * k + r] = wr * a.scaling;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        z[j] = (j < EJ && e < E) ? ex[j] * inv_esum : 0.f;
        if (write && a.probs && j < EJ && e < E) a.probs[n * E + e] = z[j];
    }
    return zmax + logf(esum);
}

// Order-preserving 64-bit key of (selection score desc, expert id asc):
// larger key = ranks ahead.  -0 is folded into +0 so that equal scores tie.
__device__ __forceinline__ uint64_t rank_key(float score, int e)
{
    uint32_t u = __float_as_uint(score + 0.0f);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(0xFFFF - e);
}

// Sums v[e] over the 32 lanes of a warp for all EB (8, 16 or 32) values at
// once, in a fixed order: at each step the lanes with bit o set keep the upper
// half of their values and add their partner's copy of it, the others the
// lower half.  After log2(EB) steps each lane holds one expert's partial,
// expert lane / (32 / EB); a butterfly over the remaining lane bits completes
// it.  EB + log2(32 / EB) - 1 shuffles instead of 5 EB.
template <int EB>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[EB], int lane)
{
    static_assert(EB == 8 || EB == 16 || EB == 32, "EB");
#pragma unroll
    for (int h = EB / 2, o = 16; h >= 1; h /= 2, o /= 2) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = up ? v[i] : v[i + h];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = (up ? v[i + h] : v[i]) + recv;
        }
    }
#pragma unroll
    for (int o = 16 * 2 / EB / 2; o >= 1; o /= 2) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    return v[0];
}

// One token per thread for E <= EB <= 32, called by all 32 lanes of a warp
// that holds one 32-token chunk (lane = token; `live` is false past N).  z[e]
// = logit of expert e.  Softmax, the k argmax rounds (score desc, id asc) and
// the gates run in the thread's registers, without shuffles; the chunk's
// sum of p, histogram and sum of (lse z_n)^2 are warp reductions in a fixed
// butterfly order, written for `chunk` (each may be null).
template <int EB>
__device__ __forceinline__ void select_thread_chunk(float (&z)[EB], const SelectArgs &a, float *psum,
                                                    int32_t *hist, float *zpart, int64_t n, bool live,
                                                    int64_t chunk)
{
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    float zmax = -FLT_MAX;
#pragma unroll
    for (int e = 0; e < EB; ++e)
        if (e < E) zmax = fmaxf(zmax, z[e]);
    float ex[EB], sel[EB], graw[EB];
    float esum = 0.f;
#pragma unroll
    for (int e = 0; e < EB; ++e) {
        ex[e] = 0.f;
        sel[e] = -FLT_MAX;
        graw[e] = 0.f;
        if (e < E) {
            ex[e] = expf(z[e] - zmax);
            esum += ex[e];
            if (a.router == kSigmoid) {
                const float sg = 1.0f / (1.0f + expf(-z[e]));
                sel[e] = sg + (a.b_sel ? a.b_sel[e] : 0.f);
                graw[e] = sg;
            } else {
                sel[e] = z[e];
                graw[e] = ex[e];
            }
        }
    }
    const float inv_esum = 1.0f / esum;
    const float lse = zmax + logf(esum);

    // k argmax rounds; the choices go to small per-thread arrays (indexed by
    // the round, so they live in local memory: a few loads and stores)
    uint32_t taken = 0;
    int ids[kMaxK];
    float gsel[kMaxK];
    float gs = 0.f;
    int cnt[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) cnt[e] = 0;
#pragma unroll 1
    for (int r = 0; r < k; ++r) {
        float bv = -FLT_MAX, bg = 0.f;
        int be = 0;
        bool found = false;
#pragma unroll
        for (int e = 0; e < EB; ++e) {
            if (e < E && !((taken >> e) & 1u) && (!found || sel[e] > bv)) {  // ascending e: ties keep the lower id
                bv = sel[e];
                be = e;
                bg = graw[e];
                found = true;
            }
        }
        taken |= 1u << be;
        ids[r] = be;
        gsel[r] = bg;
        gs += bg;
#pragma unroll
        for (int e = 0; e < EB; ++e) cnt[e] += (live && be == e) ? 1 : 0;
    }
    if (live) {
        if (a.lse) a.lse[n] = lse;
#pragma unroll 1
        for (int r = 0; r < k; ++r) {
            float wr;
            if (a.router == kSoftmaxTopk) wr = a.norm_topk ? gsel[r] / gs : gsel[r] * inv_esum;
            else if (a.router == kTopkSoftmax) wr = gsel[r] / gs;
            else wr = a.norm_topk ? gsel[r] / gs : gsel[r];
            a.ids[n * k + r] = ids[r];
            a.w[n * k + r] = wr * a.scaling;
        }
        if (a.probs) {
#pragma unroll
            for (int e = 0; e < EB; ++e)
                if (e < E) a.probs[n * E + e] = ex[e] * inv_esum;
        }
    }

    // chunk statistics; tokens past N contribute nothing.  Sums over the
    // warp's 32 tokens for all EB experts at once: a reduce-scatter leaves
    // expert e's total in lanes e * 32 / EB .. (e + 1) * 32 / EB - 1.
    if (psum) {
        float v[EB];
#pragma unroll
        for (int e = 0; e < EB; ++e) v[e] = live ? ex[e] * inv_esum : 0.f;
        const float tot = warp_reduce_scatter<EB>(v, lane);
        const int e = lane / (32 / EB);
        if (lane % (32 / EB) == 0 && e < E) psum[chunk * E + e] = tot;
    }
    if (hist) {
#pragma unroll
        for (int e = 0; e < EB; ++e) {
            if (e >= E) break;
            const int c = __reduce_add_sync(0xffffffffu, cnt[e]);
            if (lane == e) hist[chunk * E + e] = c;
        }
    }
    if (zpart) {
        float v = live ? lse * lse : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) zpart[chunk] = v;
    }
}

}  // namespace moe
