// common.cuh -- small device helpers shared by the MoE kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device-side status codes (same values as moe_status in moe.h).
enum : int32_t { kDevOk = 0, kDevTimeout = 5, kDevBadExpertId = 6 };

// Tokens handled by one router CTA; also the dispatch chunk (chunk c holds
// tokens [c*kChunkTokens, (c+1)*kChunkTokens) and their assignments).
constexpr int kChunkTokens = 32;
constexpr int kMaxE = 256;
constexpr int kMaxK = 16;

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Programmatic dependent launch.  Every kernel of this library starts with
// pdl_enter(): griddepcontrol.wait returns once the previous grid on the
// stream has completed and its memory is visible (immediately if there is no
// programmatic dependency), so nothing below it can race with the
// predecessor; launch_dependents then lets the next kernel's CTAs be
// scheduled while this grid runs, hiding the launch latency between the
// kernels of one forward.
__device__ __forceinline__ void pdl_enter()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// First error wins; later errors leave the word alone.
__device__ __forceinline__ void set_status(int32_t *status, int32_t code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// A 16-byte vector holds 8 bf16 or 4 fp32 values.
template <typename T> struct Vec16 { static constexpr int n = 16 / sizeof(T); };

__device__ __forceinline__ void unpack16(const uint4 &v, float *f, const float *)
{
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ void unpack16(const uint4 &v, float *f, const __nv_bfloat16 *)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 pack16(const float *f, const float *)
{
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

__device__ __forceinline__ uint4 pack16(const float *f, const __nv_bfloat16 *)
{
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st16(void *p, const uint4 &v)
{
    *reinterpret_cast<uint4 *>(p) = v;
}

// 2^x and 1/x by the special-function unit (PTX ex2.approx.ftz /
// rcp.approx.ftz: about 2 ulp, subnormal results flushed to zero).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// GELU (erf form), fp32: gelu(v) = v Phi(v) with Phi the standard normal
// distribution function, taken from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 26.2.17: for x >= 0, 1 - Phi(x) =
// Z(x) t (b1 + t (b2 + t (b3 + t (b4 + t b5)))), t = 1 / (1 + p x), Z the
// normal density, |error| < 7.5e-8; Phi(-x) = 1 - Phi(x).  The b_i below
// carry Z's factor 1/sqrt(2 pi), and Z's exponential is 2^(-x^2 log2(e) / 2):
// eleven multiply-adds, a select and two special-function operations per
// value.  This is the same approximation as formula 7.1.26 for erf (whose
// |error| 1.5e-7 halves on Phi).  The GELU epilogues of the expert GEMMs
// (results rounded to bf16) are bound by this function when the k-loop is
// short.  Large |v|: the exponential flushes to 0 and Phi to 0 or 1.
__device__ __forceinline__ float gelu_erf(float v)
{
    const float t = rcp_approx(fmaf(0.2316419f, fabsf(v), 1.0f));
    const float poly =
        t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 0.530702710f, -0.726576030f), 0.710706890f), -0.142248362f), 0.127414793f);
    const float q = poly * ex2_approx(v * (v * -0.72134752f));  // 1 - Phi(|v|)
    return v * (v >= 0.0f ? 1.0f - q : q);
}
__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }
// The same on the special-function unit, for results rounded to bf16:
// v / (1 + 2^(-v log2 e)) with ex2.approx and rcp.approx (relative error a
// few 1e-7; large negative v: the exponential overflows to +inf and the
// reciprocal to 0, so silu -> -0).
__device__ __forceinline__ float silu_approx(float v)
{
    return v * rcp_approx(1.0f + ex2_approx(v * -1.44269504f));
}

}  // namespace moe
