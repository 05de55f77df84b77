// epilogue_f32.cuh -- fp32 result rows of a tcgen05 accumulator tile, shared
// by the single-CTA and CTA-pair GEMM kernels (the backward's products).
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace moe {
namespace sm100 {

// One epilogue warp's 32 accumulator rows (TMEM lane quarter at tbase; lane
// l holds result row row_first + l) and 256 columns from n0: rows from
// row_end on and columns from n_out on are not stored; `accumulate` adds to
// the existing result, `zero` stores zeros (no MMA wrote the accumulator).
// Each 32-column chunk goes through `stage` (32 rows padded to 36 floats, no
// bank conflicts): lane l writes its row, then lanes 8j .. 8j+7 store 128 B
// of row 4q + j (q = 0..7), so every store instruction writes four whole
// 128-byte rows.  out + row * ldo + col must be 16-byte aligned for every
// stored (row, col) (ldo and n_out multiples of 4).
__device__ __forceinline__ void epilogue_f32_rows(float *out, int64_t ldo, int n_out, uint32_t tbase,
                                                  int64_t row_first, int64_t row_end, int n0, float (*stage)[36],
                                                  bool zero, bool accumulate)
{
    const int lane = threadIdx.x & 31;
    const int sub = lane >> 3, cq = (lane & 7) * 4;
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
        uint32_t acc[32];
        tmem_ld32(tbase + c, acc);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 8; ++v)
            *reinterpret_cast<float4 *>(&stage[lane][4 * v]) =
                zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                     : make_float4(__uint_as_float(acc[4 * v]), __uint_as_float(acc[4 * v + 1]),
                                   __uint_as_float(acc[4 * v + 2]), __uint_as_float(acc[4 * v + 3]));
        __syncwarp();
        const int col = n0 + c + cq;
        if (col < n_out) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int r = 4 * q + sub;
                const int64_t row = row_first + r;
                if (row < row_end) {
                    float4 v4 = *reinterpret_cast<const float4 *>(&stage[r][cq]);
                    float *dst = out + row * ldo + col;
                    if (accumulate) {
                        const float4 o = *reinterpret_cast<const float4 *>(dst);
                        v4.x += o.x; v4.y += o.y; v4.z += o.z; v4.w += o.w;
                    }
                    *reinterpret_cast<float4 *>(dst) = v4;
                }
            }
        }
        __syncwarp();
    }
}

}  // namespace sm100
}  // namespace moe
