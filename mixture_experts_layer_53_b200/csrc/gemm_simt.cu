// gemm_simt.cu -- fp32 ragged grouped GEMM for the expert FFNs (CUDA cores).
//
// The fp32 workload must match an fp64 oracle to 1e-5 relative, which the
// tf32 tensor-core path cannot guarantee, so fp32 runs the same ragged tile
// walk as the tcgen05 kernel (course module sec. 2.2: one product per expert
// over its slice of x_sorted) with FFMA: each table tile of tile_m rows is
// computed 128 rows x 64 columns at a time, 256 threads, 8x4 outputs per
// thread, k-chunks of 16 staged in shared memory.
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace moe {
namespace {

constexpr int TM = 128, TN = 64, TK = 16, THREADS = 256;

enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_LINEAR = 2 };

struct SimtArgs {
    const float *A;         // [rows, K]
    const float *B;         // [E * b_rows, K]
    const float *B3;        // SwiGLU up projection, same layout
    const float *bias;      // [E, n_out] or null
    float *out;             // [rows, n_out]
    const int32_t *offsets;
    const int32_t *mt_prefix;
    int64_t rows;
    int E, K, n_out, n_tiles, b_rows, tile_m;
};

template <int EPI>
__global__ void __launch_bounds__(THREADS) simt_gemm_kernel(SimtArgs g)
{
    pdl_enter();
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    __shared__ float B3s[EPI == EPI_SWIGLU ? TK : 1][TN + 4];
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;  // rows ty*8.., cols tx*4..
    const int total = g.mt_prefix[g.E] * g.n_tiles;

    for (int t = blockIdx.x; t < total; t += gridDim.x) {
        // tile -> (expert, n-tile, m-tile), m-tile innermost
        const int q = t / g.n_tiles;
        int lo = 0, hi = g.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (g.mt_prefix[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo;
        const int mt_e = g.mt_prefix[e + 1] - g.mt_prefix[e];
        const int local = t - g.mt_prefix[e] * g.n_tiles;
        const int m_tile = local % mt_e, n_tile = local / mt_e;
        const int64_t row_end = g.offsets[e + 1];
        const int n0 = n_tile * TN;
        // a tile of the table spans tile_m rows: walk it TM rows at a time
        for (int part = 0; part * TM < g.tile_m; ++part) {
        const int64_t row0 = g.offsets[e] + static_cast<int64_t>(m_tile) * g.tile_m + part * TM;
        if (row0 >= row_end) break;  // uniform across the block

        float acc[8][4], acc3[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = acc3[i][j] = 0.f;

        for (int k0 = 0; k0 < g.K; k0 += TK) {
            for (int idx = tid; idx < TM * TK; idx += THREADS) {
                const int r = idx / TK, c = idx % TK;
                const int64_t row = row0 + r;
                As[c][r] = (row < row_end && k0 + c < g.K) ? g.A[row * g.K + k0 + c] : 0.f;
            }
            for (int idx = tid; idx < TN * TK; idx += THREADS) {
                const int r = idx / TK, c = idx % TK;
                const bool ok = n0 + r < g.n_out && k0 + c < g.K;
                const int64_t brow = static_cast<int64_t>(e) * g.b_rows + n0 + r;
                Bs[c][r] = ok ? g.B[brow * g.K + k0 + c] : 0.f;
                if (EPI == EPI_SWIGLU) B3s[c][r] = ok ? g.B3[brow * g.K + k0 + c] : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int c = 0; c < TK; ++c) {
                float a[8], b[4], b3[4];
#pragma unroll
                for (int i = 0; i < 8; ++i) a[i] = As[c][ty * 8 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    b[j] = Bs[c][tx * 4 + j];
                    if (EPI == EPI_SWIGLU) b3[j] = B3s[c][tx * 4 + j];
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
                        if (EPI == EPI_SWIGLU) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
                    }
            }
            __syncthreads();
        }

#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t row = row0 + ty * 8 + i;
            if (row >= row_end) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = n0 + tx * 4 + j;
                if (col >= g.n_out) continue;
                float v = acc[i][j];
                if (EPI == EPI_SWIGLU) {
                    v = silu(v) * acc3[i][j];
                } else {
                    if (g.bias) v += g.bias[static_cast<int64_t>(e) * g.n_out + col];
                    if (EPI == EPI_GELU) v = gelu_erf(v);
                }
                g.out[row * g.n_out + col] = v;
            }
        }
        }
    }
}

template <int EPI> cudaError_t launch_simt(const SimtArgs &g, int num_sms, cudaStream_t s)
{
    return launch_k(simt_gemm_kernel<EPI>, dim3(num_sms * 4), dim3(THREADS), 0, s, g);
}

}  // namespace

cudaError_t launch_ffn_f32_simt(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s)
{
    cudaError_t err = cudaSuccess;
    const bool swiglu = a.act == kSwiglu;
    if (a.rows > 0) {
        SimtArgs g1{};
        g1.A = static_cast<const float *>(a.x_sorted);
        g1.B = static_cast<const float *>(a.W1);
        g1.B3 = static_cast<const float *>(a.W3);
        g1.bias = swiglu ? nullptr : static_cast<const float *>(a.b1);
        g1.out = static_cast<float *>(a.h);
        g1.offsets = a.offsets;
        g1.mt_prefix = a.mt_prefix;
        g1.rows = a.rows;
        g1.E = a.E;
        g1.K = a.d;
        g1.n_out = a.F;
        g1.n_tiles = (a.F + TN - 1) / TN;
        g1.b_rows = a.F;
        g1.tile_m = a.tile_m;
        err = swiglu ? launch_simt<EPI_SWIGLU>(g1, num_sms, s) : launch_simt<EPI_GELU>(g1, num_sms, s);
        if (err != cudaSuccess) return err;
    }
    if (mid && (err = cudaEventRecord(mid, s)) != cudaSuccess) return err;
    if (a.rows > 0) {
        SimtArgs g2{};
        g2.A = static_cast<const float *>(a.h);
        g2.B = static_cast<const float *>(a.W2);
        g2.bias = static_cast<const float *>(a.b2);
        g2.out = static_cast<float *>(a.y_sorted);
        g2.offsets = a.offsets;
        g2.mt_prefix = a.mt_prefix;
        g2.rows = a.rows;
        g2.E = a.E;
        g2.K = a.F;
        g2.n_out = a.d;
        g2.n_tiles = (a.d + TN - 1) / TN;
        g2.b_rows = a.d;
        g2.tile_m = a.tile_m;
        err = launch_simt<EPI_LINEAR>(g2, num_sms, s);
    }
    return err;
}

}  // namespace moe
