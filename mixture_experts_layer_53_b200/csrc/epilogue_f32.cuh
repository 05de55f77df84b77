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

// The same warp's rows written by TMA stores instead (the weight gradients,
// whose short per-expert reductions would otherwise wait on thread stores):
// the result is [E][m_total][n_out] behind tm_out ({n_out, m_total, E},
// 32 x 32 boxes, 128-byte swizzle, clipped at the edges); this is group e,
// rows row_first .. row_first + 31.  buf: the warp's 4 KB, 1024-byte aligned,
// written in the box's swizzled layout (16-byte piece j of row r at piece
// j ^ (r & 7)), which is also free of bank conflicts.  Lane 0 owns the
// stores: it waits for the previous one to have read buf before buf is
// rewritten, and the caller waits for all of them (bulk_wait_all) before
// the CTA exits.
__device__ __forceinline__ void epilogue_f32_tma(const CUtensorMap *tm_out, uint32_t tbase, int e, int row_first,
                                                 int64_t m_total, int n0, int n_out, uint8_t *buf, bool zero)
{
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
        uint32_t acc[32];
        tmem_ld32(tbase + c, acc);
        tmem_ld_wait();
        const int col = n0 + c;
        if (row_first >= m_total || col >= n_out) continue;  // warp-uniform: nothing to store
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4 *>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                     : make_float4(__uint_as_float(acc[4 * j]), __uint_as_float(acc[4 * j + 1]),
                                   __uint_as_float(acc[4 * j + 2]), __uint_as_float(acc[4 * j + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(tm_out, buf, col, row_first, e);
            bulk_commit();
        }
    }
}

}  // namespace sm100
}  // namespace moe
