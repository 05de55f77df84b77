// gemm_generic.cu -- strided grouped GEMM on the CUDA cores (fp32
// accumulation and output) for the backward pass.
//
// C_g(m, n) (+)= sum_k A(m, k) B_g(k, n) over groups g, with every operand
// given by element strides, so one kernel covers the transposed products of
// the backward:
//   ragged M (rows offsets[g] .. offsets[g+1]-1 of A and C belong to group
//   g; B_g = B + g * sbg): the dgrad products dh = dy_s W2[e],
//   dx_s = da W1[e] (+ du W3[e]) and the recomputed pre-activations
//   x_s W1[e]^T;
//   ragged K (the reduction runs over rows offsets[g] .. offsets[g+1]-1;
//   C_g = C + g * scg): the weight gradients dW2[e] = dy_s^T (w h),
//   dW1[e] = da^T x_s and the bias gradients (B a single 1.0 with stride 0).
// 64 x 64 tiles, k-chunks of 16 staged in shared memory, 256 threads with
// 4 x 4 outputs each.  Correct for any strides; not tuned: the tensor-core
// version of the backward products needs MN-major tcgen05 operands.
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16, THREADS = 256;

template <bool BF16> __device__ __forceinline__ float ld_el(const void *p, int64_t i)
{
    if constexpr (BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    else return static_cast<const float *>(p)[i];
}

template <bool ABF, bool BBF>
__global__ void __launch_bounds__(THREADS) gemm_generic_kernel(GenericGemmArgs g)
{
    pdl_enter();
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;  // rows ty*4.., cols tx*4..
    int grp;
    int64_t m0, m_end, k_lo, k_hi;
    int split = 0;
    if (g.ragged_k) {
        grp = blockIdx.z / g.ksplit;
        split = blockIdx.z - grp * g.ksplit;
        m0 = static_cast<int64_t>(blockIdx.x) * TM;
        m_end = g.M;
        k_lo = g.offsets[grp];
        k_hi = g.offsets[grp + 1];
        if (g.ksplit > 1) {  // this CTA's share of the reduction, whole k-chunks
            const int64_t chunk = ((k_hi - k_lo + g.ksplit - 1) / g.ksplit + TK - 1) / TK * TK;
            k_lo = min64(k_hi, k_lo + split * chunk);
            k_hi = min64(k_hi, k_lo + chunk);
        }
    } else {
        // tile -> (group, m-tile) through the per-group tile prefix
        const int t = blockIdx.x;
        if (t >= g.mt_prefix[g.G]) return;  // block-uniform
        int lo = 0, hi = g.G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (g.mt_prefix[mid] <= t) lo = mid;
            else hi = mid - 1;
        }
        grp = lo;
        m0 = g.offsets[grp] + static_cast<int64_t>(t - g.mt_prefix[grp]) * TM;
        m_end = g.offsets[grp + 1];
        k_lo = 0;
        k_hi = g.K;
    }
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * TN;
    const int64_t boff = static_cast<int64_t>(grp) * g.sbg;
    // split reductions write dense partials [G * ksplit][M][N], summed in
    // split order by split_reduce_kernel
    const bool partial = g.ragged_k && g.ksplit > 1;
    float *C = partial ? g.partial + (static_cast<int64_t>(grp) * g.ksplit + split) * g.M * g.N
                       : g.C + static_cast<int64_t>(grp) * g.scg;
    const int64_t scm = partial ? g.N : g.scm, scn = partial ? 1 : g.scn;

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int64_t k0 = k_lo; k0 < k_hi; k0 += TK) {
        for (int idx = tid; idx < TM * TK; idx += THREADS) {
            const int r = idx / TK, c = idx % TK;
            const int64_t m = m0 + r, kk = k0 + c;
            As[c][r] = (m < m_end && kk < k_hi) ? ld_el<ABF>(g.A, m * g.sam + kk * g.sak) : 0.f;
        }
        for (int idx = tid; idx < TN * TK; idx += THREADS) {
            const int c = idx / TN, r = idx % TN;
            const int64_t n = n0 + r, kk = k0 + c;
            Bs[c][r] = (n < g.N && kk < k_hi) ? ld_el<BBF>(g.B, boff + kk * g.sbk + n * g.sbn) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < TK; ++c) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[c][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[c][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= m_end) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t n = n0 + tx * 4 + j;
            if (n >= g.N) continue;
            float *cp = C + m * scm + n * scn;
            *cp = (g.accumulate && !partial) ? *cp + acc[i][j] : acc[i][j];
        }
    }
}

// C_g(m, n) (+)= sum over splits, in split order.
__global__ void __launch_bounds__(256) split_reduce_kernel(GenericGemmArgs g)
{
    pdl_enter();
    const int64_t total = static_cast<int64_t>(g.G) * g.M * g.N;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t grp = i / (g.M * g.N), mn = i - grp * g.M * g.N;
        const int64_t m = mn / g.N, n = mn - m * g.N;
        float s = 0.f;
        for (int sp = 0; sp < g.ksplit; ++sp) s += g.partial[(grp * g.ksplit + sp) * g.M * g.N + mn];
        float *cp = g.C + grp * g.scg + m * g.scm + n * g.scn;
        *cp = g.accumulate ? *cp + s : s;
    }
}

}  // namespace

cudaError_t launch_gemm_generic(const GenericGemmArgs &g, int64_t max_tiles_m, cudaStream_t s)
{
    dim3 grid;
    if (g.ragged_k) grid = dim3(static_cast<unsigned>((g.M + TM - 1) / TM), static_cast<unsigned>((g.N + TN - 1) / TN),
                                static_cast<unsigned>(g.G * max(g.ksplit, 1)));
    else grid = dim3(static_cast<unsigned>(max_tiles_m), static_cast<unsigned>((g.N + TN - 1) / TN), 1);
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
    cudaError_t err;
    if (g.a_bf16 && g.b_bf16) err = launch_k(gemm_generic_kernel<true, true>, grid, dim3(THREADS), 0, s, g);
    else if (g.a_bf16) err = launch_k(gemm_generic_kernel<true, false>, grid, dim3(THREADS), 0, s, g);
    else if (g.b_bf16) err = launch_k(gemm_generic_kernel<false, true>, grid, dim3(THREADS), 0, s, g);
    else err = launch_k(gemm_generic_kernel<false, false>, grid, dim3(THREADS), 0, s, g);
    if (err != cudaSuccess || !g.ragged_k || g.ksplit <= 1) return err;
    const int64_t total = static_cast<int64_t>(g.G) * g.M * g.N;
    const int rgrid = static_cast<int>(min64((total + 255) / 256, 148 * 8));
    return launch_k(split_reduce_kernel, dim3(rgrid), dim3(256), 0, s, g);
}

}  // namespace moe
