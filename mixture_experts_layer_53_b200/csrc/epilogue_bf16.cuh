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

// Shared memory one epilogue warp stages a 32 x 32 bf16 chunk through: 32
// rows of 64 B in the layout of a 64-byte-swizzled TMA box (16-byte piece j
// of row r at piece j ^ ((r >> 1) & 3)).  Both the row-per-lane writes and
// the row-segment reads below are free of bank conflicts in this layout, and
// a TMA store can take the chunk from it as it is (buffer 512-byte aligned).
constexpr int kBf16StageBytes = 32 * 64;

__device__ __forceinline__ int stage_piece(int r, int j) { return r * 64 + ((j ^ ((r >> 1) & 3)) << 4); }

// The bias values of result columns col0 .. col0 + 31 (zero past n_out).
__device__ __forceinline__ void load_bias_chunk(const __nv_bfloat16 *bias, int col0, int n_out, uint4 (&bv)[4])
{
#pragma unroll
    for (int v = 0; v < 4; ++v)
        bv[v] = (bias && col0 + v * 8 < n_out) ? __ldg(reinterpret_cast<const uint4 *>(bias + col0 + v * 8))
                                               : make_uint4(0u, 0u, 0u, 0u);
}

// 32 accumulator columns of this lane's row -> 16 packed bf16 pairs.
// SwiGLU: h = silu(gate) * up (gate at columns c.., up at 128 + c..); GELU:
// gelu_erf(acc + b); linear: acc + b (added only if has_bias; bias(v, b)
// gives the 8 values of columns 8v .. 8v+7 of the chunk).
template <int EPI, typename Bias>
__device__ __forceinline__ void epi_bf16_math(const uint32_t (&acc)[32], const uint32_t (&up)[32], Bias &&bias,
                                              bool has_bias, uint32_t (&p)[16])
{
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        float o[8];
        if constexpr (EPI == EPIB_SWIGLU) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
                o[u] = silu_approx(__uint_as_float(acc[v * 8 + u])) * __uint_as_float(up[v * 8 + u]);
        } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) o[u] = __uint_as_float(acc[v * 8 + u]);
            if (has_bias) {
                float b[8];
                bias(v, b);
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

// Lane l puts row l's 64 B of the chunk into `stage`.
__device__ __forceinline__ void epi_bf16_stage(const uint32_t (&p)[16], uint8_t *stage)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(stage + stage_piece(lane, j)) =
            make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
}

// The staged chunk to rows row_first .. row_first + 31 of `out`, columns
// col0 .. col0 + 31: each store instruction writes 8 whole 64-B row
// segments (lanes 4r .. 4r+3: 16 B each of row r).  Rows from row_end on
// and columns from n_out on are not stored (n_out is a multiple of 8).
__device__ __forceinline__ void epi_bf16_store_rows(const uint8_t *stage, __nv_bfloat16 *out, int64_t ldo,
                                                    int64_t row_first, int64_t row_end, int col0, int n_out)
{
    const int lane = threadIdx.x & 31;
    const int piece = lane & 3;
    const int col = col0 + piece * 8;
    if (col < n_out) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = (lane >> 2) + 8 * i;
            const int64_t row = row_first + r;
            if (row < row_end)
                st16(out + row * ldo + col, *reinterpret_cast<const uint4 *>(stage + stage_piece(r, piece)));
        }
    }
}

// The warp's rows row_first .. row_first + 31 (TMEM lane quarter at tbase:
// lane l holds row row_first + l), accumulator columns [c_begin, c_end) of
// the tile, a multiple of 64 wide; result column n0 + c.  The TMEM loads
// (and bias values) of the next 32-column chunk are in flight while the
// current one is computed and stored.  `stage`: the warp's kBf16StageBytes.
//
// With a store tensor map `tm` (bf16 [rows][n_out], 32 x 32 boxes, 64-byte
// swizzle; stage 512-byte aligned) a chunk whose 32 rows all lie before
// row_end leaves through one TMA store; lane 0 waits until the previous
// store has read the buffer before it is rewritten, and the caller waits
// for all of them (bulk_wait_all) before the kernel ends.  A chunk that
// straddles row_end (the next expert's rows follow) is stored row by row.
// Without a map (tm null) every chunk is stored row by row.  `release()`
// runs once (warp-uniform) as soon as the warp's last TMEM load of the tile
// has completed, before the last chunk is computed and stored.  LEAN: one
// chunk in registers at a time (for kernels with enough epilogue warps per
// scheduler to hide the TMEM load latency, and registers for no more); the
// warp's bias values are first converted to fp32 into bias_s (c_end -
// c_begin floats, 16-byte aligned) and read from there as broadcasts.
template <int EPI, bool LEAN = false, typename Release>
__device__ __forceinline__ void epilogue_bf16_rows(const CUtensorMap *tm, __nv_bfloat16 *out, int64_t ldo, int n_out,
                                                   const __nv_bfloat16 *bias_row, uint32_t tbase, int64_t row_first,
                                                   int64_t row_end, int n0, int c_begin, int c_end, uint8_t *stage,
                                                   Release &&release, float *bias_s = nullptr)
{
    if (row_first >= row_end || n0 + c_begin >= n_out) {  // warp-uniform: nothing of this warp's to store
        release();
        return;
    }
    const int lane = threadIdx.x & 31;
    const bool whole = tm != nullptr && row_first + 32 <= row_end;
    const bool has_bias = EPI != EPIB_SWIGLU && bias_row != nullptr;
    uint32_t a0[32], a1[32], u0[32], u1[32];
    uint4 b0[4], b1[4];
    auto load = [&](uint32_t (&acc)[32], uint32_t (&up)[32], uint4 (&bv)[4], int c) {
        tmem_ld32(tbase + c, acc);
        if constexpr (EPI == EPIB_SWIGLU) tmem_ld32(tbase + 128 + c, up);
        if (has_bias) load_bias_chunk(bias_row, n0 + c, n_out, bv);
    };
    auto put = [&](const uint32_t (&p)[16], int col0) {
        if (col0 >= n_out) return;  // warp-uniform
        if (lane == 0) bulk_wait_read_all();  // an earlier TMA store has read the buffer
        __syncwarp();
        epi_bf16_stage(p, stage);
        if (whole) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(tm, stage, col0, static_cast<int32_t>(row_first));
                bulk_commit();
            }
        } else {
            __syncwarp();
            epi_bf16_store_rows(stage, out, ldo, row_first, row_end, col0, n_out);
            __syncwarp();
        }
    };
    if constexpr (LEAN) {
        const int c_stop = min(c_end, c_begin + ((n_out - n0 - c_begin + 31) & ~31));
        if (has_bias) {
            for (int j = lane; j < c_stop - c_begin; j += 32) {
                const int col = n0 + c_begin + j;
                bias_s[j] = col < n_out ? __bfloat162float(bias_row[col]) : 0.0f;
            }
            __syncwarp();
        }
#pragma unroll 1
        for (int c = c_begin; c < c_stop; c += 32) {
            uint32_t p[16];
            tmem_ld32(tbase + c, a0);
            if constexpr (EPI == EPIB_SWIGLU) tmem_ld32(tbase + 128 + c, u0);
            tmem_ld_wait();
            if (c + 32 >= c_stop) release();
            const float4 *bs = reinterpret_cast<const float4 *>(bias_s + (c - c_begin));
            epi_bf16_math<EPI>(
                a0, u0,
                [&](int v, float (&b)[8]) {
                    const float4 lo = bs[2 * v], hi = bs[2 * v + 1];
                    b[0] = lo.x, b[1] = lo.y, b[2] = lo.z, b[3] = lo.w;
                    b[4] = hi.x, b[5] = hi.y, b[6] = hi.z, b[7] = hi.w;
                },
                has_bias, p);
            put(p, n0 + c);
        }
        if (has_bias) __syncwarp();  // bias_s is read before the next tile rewrites it
        return;
    }
    auto from_regs = [](const uint4 (&bv)[4]) {
        return [&bv](int v, float (&b)[8]) { unpack16(bv[v], b, static_cast<const __nv_bfloat16 *>(nullptr)); };
    };
    const int c_stop = min(c_end, c_begin + ((n_out - n0 - c_begin + 63) & ~63));
    load(a0, u0, b0, c_begin);
    tmem_ld_wait();
#pragma unroll 1
    for (int c = c_begin; c < c_stop; c += 64) {
        uint32_t p[16];
        load(a1, u1, b1, c + 32);
        epi_bf16_math<EPI>(a0, u0, from_regs(b0), has_bias, p);
        put(p, n0 + c);
        tmem_ld_wait();
        if (c + 64 < c_stop) load(a0, u0, b0, c + 64);
        else release();
        epi_bf16_math<EPI>(a1, u1, from_regs(b1), has_bias, p);
        put(p, n0 + c + 32);
        tmem_ld_wait();
    }
}

}  // namespace sm100
}  // namespace moe
