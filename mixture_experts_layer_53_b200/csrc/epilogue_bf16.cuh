// epilogue_bf16.cuh -- bf16 result rows of a tcgen05 accumulator tile for
// the forward's expert GEMMs, shared by the single-CTA and CTA-pair kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace sm100 {

enum { EPIB_SWIGLU = 0, EPIB_GELU = 1, EPIB_LINEAR = 2 };

// Bytes of shared memory one epilogue warp stages through: 32 rows of 32
// bf16 (64 B) padded to 80 B, so that both the row-per-lane writes and the
// row-segment reads below are free of bank conflicts.
constexpr int kBf16StageRowBytes = 80;
constexpr int kBf16StageBytes = 32 * kBf16StageRowBytes;

// 32 accumulator columns of this lane's row -> 16 packed bf16 pairs.
// SwiGLU: h = silu(gate) * up (gate at columns c.., up at 128 + c..); GELU:
// gelu_erf(acc + b); linear: acc + b (b = bias[col], absent if bias null).
template <int EPI>
__device__ __forceinline__ void epi_bf16_math(const uint32_t (&acc)[32], const uint32_t (&up)[32],
                                              const __nv_bfloat16 *bias, int col0, int n_out, uint32_t (&p)[16])
{
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        float o[8];
        if constexpr (EPI == EPIB_SWIGLU) {
#pragma unroll
            for (int u = 0; u < 8; ++u) o[u] = silu(__uint_as_float(acc[v * 8 + u])) * __uint_as_float(up[v * 8 + u]);
        } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) o[u] = __uint_as_float(acc[v * 8 + u]);
            if (bias && col0 + v * 8 < n_out) {
                float b[8];
                unpack16(*reinterpret_cast<const uint4 *>(bias + col0 + v * 8), b,
                         static_cast<const __nv_bfloat16 *>(nullptr));
#pragma unroll
                for (int u = 0; u < 8; ++u) o[u] += b[u];
            }
            if constexpr (EPI == EPIB_GELU) {
#pragma unroll
                for (int u = 0; u < 8; ++u) o[u] = gelu_erf(o[u]);
            }
        }
        const uint4 q = pack16(o, static_cast<const __nv_bfloat16 *>(nullptr));
        p[v * 4 + 0] = q.x;
        p[v * 4 + 1] = q.y;
        p[v * 4 + 2] = q.z;
        p[v * 4 + 3] = q.w;
    }
}

// One 32-column chunk of the warp's 32 rows: lane l writes row l's 64 B
// into `stage`, then each store instruction writes 8 whole 64-B row
// segments (lanes 4r .. 4r+3: 16 B each of row r).  Rows from row_end on
// and columns from n_out on are not stored (n_out is a multiple of 8).
__device__ __forceinline__ void epi_bf16_store_chunk(const uint32_t (&p)[16], uint8_t *stage, __nv_bfloat16 *out,
                                                     int64_t ldo, int64_t row_first, int64_t row_end, int col0,
                                                     int n_out)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(stage + lane * kBf16StageRowBytes + j * 16) =
            make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
    __syncwarp();
    const int piece = lane & 3;
    const int col = col0 + piece * 8;
    if (col < n_out) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = (lane >> 2) + 8 * i;
            const int64_t row = row_first + r;
            if (row < row_end)
                st16(out + row * ldo + col,
                     *reinterpret_cast<const uint4 *>(stage + r * kBf16StageRowBytes + piece * 16));
        }
    }
    __syncwarp();
}

// The warp's rows row_first .. row_first + 31 (TMEM lane quarter at tbase:
// lane l holds row row_first + l), accumulator columns [c_begin, c_end) of
// the tile, a multiple of 64 wide; result column n0 + c.  The TMEM loads of
// the next 32-column chunk are in flight while the current one is computed
// and stored.  `stage`: the warp's kBf16StageBytes, 16-byte aligned.
template <int EPI>
__device__ __forceinline__ void epilogue_bf16_rows(__nv_bfloat16 *out, int64_t ldo, int n_out,
                                                   const __nv_bfloat16 *bias_row, uint32_t tbase, int64_t row_first,
                                                   int64_t row_end, int n0, int c_begin, int c_end, uint8_t *stage)
{
    uint32_t a0[32], a1[32], u0[32], u1[32];
    auto load = [&](uint32_t (&acc)[32], uint32_t (&up)[32], int c) {
        tmem_ld32(tbase + c, acc);
        if constexpr (EPI == EPIB_SWIGLU) tmem_ld32(tbase + 128 + c, up);
    };
    load(a0, u0, c_begin);
    tmem_ld_wait();
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 64) {
        uint32_t p[16];
        load(a1, u1, c + 32);
        epi_bf16_math<EPI>(a0, u0, bias_row, n0 + c, n_out, p);
        epi_bf16_store_chunk(p, stage, out, ldo, row_first, row_end, n0 + c, n_out);
        tmem_ld_wait();
        if (c + 64 < c_end) load(a0, u0, c + 64);
        epi_bf16_math<EPI>(a1, u1, bias_row, n0 + c + 32, n_out, p);
        epi_bf16_store_chunk(p, stage, out, ldo, row_first, row_end, n0 + c + 32, n_out);
        tmem_ld_wait();
    }
}

}  // namespace sm100
}  // namespace moe
