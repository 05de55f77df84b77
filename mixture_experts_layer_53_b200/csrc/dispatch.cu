// dispatch.cu -- sorted dispatch (course module "Mixture of Experts: routing,
// sorted dispatch, Switch aux loss, aux-free bias", sec. 2.2), the Switch
// loss (sec. 2.3) and the sign-rule bias step (sec. 2.5), plus the combine.
//
// The stable sort of assignments a = n k + j by expert is a counting sort
// over fixed chunks of 32 tokens:
//   1. per-chunk expert histograms (from the router, or from the ids),
//   2. one CTA scans them: counts, offsets = exclusive prefix of counts,
//      and for every (chunk, expert) the first sorted position the chunk
//      owns inside that expert's slice,
//   3. each chunk ranks its own assignments in assignment order, so
//      position = chunk base + rank is the stable order,
//   4. rows are copied x -> x_sorted with 16-byte vectors, one warp per token
//      (the token row is read once and written k times).
// Every reduction runs in a fixed order, so results are bitwise repeatable.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kCT = kChunkTokens;

// ---------------------------------------------------------------- histogram

__global__ void __launch_bounds__(256) hist_kernel(HistArgs a)
{
    __shared__ int ids_s[kCT * kMaxK];
    const int64_t c = blockIdx.x;
    const int64_t tok0 = c * kCT;
    const int ntok = static_cast<int>(min64(kCT, a.N - tok0));
    const int nas = ntok * a.k;
    if (a.ids) {
        for (int q = threadIdx.x; q < nas; q += blockDim.x) {
            const int e = a.ids[tok0 * a.k + q];
            ids_s[q] = e;
            if (e < 0 || e >= a.E) set_status(a.status, kDevBadExpertId);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        if (a.ids) {
            int cnt = 0;
            for (int q = 0; q < nas; ++q) cnt += (ids_s[q] == e);
            a.hist[c * a.E + e] = cnt;
        }
        if (a.psum) {
            float s = 0.f;
            for (int t = 0; t < ntok; ++t) s += a.probs[(tok0 + t) * a.E + e];
            a.psum[c * a.E + e] = s;
        }
    }
}

// ------------------------------------------------------------------- scan

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) scan_kernel(ScanArgs a)
{
    __shared__ int part[kScanThreads];       // [seg][e]
    __shared__ int segbase[kScanThreads];    // [seg][e]
    __shared__ double ppart[kScanThreads];   // [seg][e]
    __shared__ int off_s[kMaxE + 1];
    __shared__ int cnt_s[kMaxE];
    __shared__ double P_s[kMaxE];

    const int E = a.E;
    const int nseg = kScanThreads / E;  // >= 4 because E <= 256
    const int64_t seglen = (a.chunks + nseg - 1) / nseg;
    const int tid = threadIdx.x;
    const int e = tid % E, s = tid / E;
    const bool active = s < nseg;
    const int64_t c_begin = active ? min64(a.chunks, s * seglen) : 0;
    const int64_t c_end = active ? min64(a.chunks, (s + 1) * seglen) : 0;

    if (active) {
        int sum = 0;
        double psum = 0.0;
        for (int64_t c = c_begin; c < c_end; ++c) {
            sum += a.hist[c * E + e];
            if (a.psum) psum += static_cast<double>(a.psum[c * E + e]);
        }
        part[s * E + e] = sum;
        ppart[s * E + e] = psum;
    }
    __syncthreads();
    if (tid < E) {
        int run = 0;
        double P = 0.0;
        for (int q = 0; q < nseg; ++q) {
            segbase[q * E + tid] = run;
            run += part[q * E + tid];
            P += ppart[q * E + tid];
        }
        cnt_s[tid] = run;
        P_s[tid] = P;
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int q = 0; q < E; ++q) {
            off_s[q] = run;
            run += cnt_s[q];
        }
        off_s[E] = run;
        if (a.mt_prefix) {
            int mt = 0;
            a.mt_prefix[0] = 0;
            for (int q = 0; q < E; ++q) {
                mt += (cnt_s[q] + kTileM - 1) / kTileM;
                a.mt_prefix[q + 1] = mt;
            }
        }
        if (a.aux_out && a.psum && a.N == 0) {
            *a.aux_out = 0.0f;  // no tokens: every sum is empty
        } else if (a.aux_out && a.psum) {
            // L = E * sum_e (count_e / N) * (P_e / N), in fp64 (sec. 2.3)
            const double Nd = static_cast<double>(a.N);
            double L = 0.0;
            for (int q = 0; q < E; ++q)
                L += (static_cast<double>(cnt_s[q]) / Nd) * (P_s[q] / Nd);
            *a.aux_out = static_cast<float>(L * static_cast<double>(E));
        }
    }
    __syncthreads();
    for (int q = tid; q <= E; q += kScanThreads) a.offsets[q] = off_s[q];
    if (tid < E) {
        if (a.counts) a.counts[tid] = cnt_s[tid];
        if (a.b_e && a.gamma > 0.f) {
            // b_e += gamma * sign(mean load - load_e), mean load = N k / E (sec. 2.5)
            const long long diff = static_cast<long long>(a.N) * a.k - static_cast<long long>(E) * cnt_s[tid];
            const float sg = static_cast<float>((diff > 0) - (diff < 0));
            a.b_e[tid] += a.gamma * sg;
        }
    }
    if (active) {
        int run = off_s[e] + segbase[s * E + e];
        for (int64_t c = c_begin; c < c_end; ++c) {
            const int v = a.hist[c * E + e];
            a.hist[c * E + e] = run;
            run += v;
        }
    }
}

// ---------------------------------------------------------------- scatter

__global__ void __launch_bounds__(256) scatter_kernel(ScatterArgs a)
{
    __shared__ int ids_s[kCT * kMaxK];
    const int64_t c = blockIdx.x;
    const int64_t a0 = c * kCT * a.k;
    const int ntok = static_cast<int>(min64(kCT, a.N - c * kCT));
    const int nas = ntok * a.k;
    for (int q = threadIdx.x; q < nas; q += blockDim.x) ids_s[q] = a.ids[a0 + q];
    __syncthreads();
    for (int q = threadIdx.x; q < nas; q += blockDim.x) {
        const int e = ids_s[q];
        if (e < 0 || e >= a.E) continue;  // reported by the histogram pass
        int rank = 0;
        for (int r = 0; r < q; ++r) rank += (ids_s[r] == e);
        const int pos = a.chunk_base[c * a.E + e] + rank;
        if (a.perm) a.perm[pos] = static_cast<int32_t>(a0 + q);
        a.inv_perm[a0 + q] = pos;
    }
}

// ----------------------------------------------------------------- gather

template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t row_bytes = static_cast<int64_t>(a.d) * sizeof(T);
    const char *x = static_cast<const char *>(a.x);
    char *xs = static_cast<char *>(a.x_sorted);
    const int64_t rows = a.N * a.k;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.N;
         n += warps) {
        const int dst_l = lane < a.k ? a.inv_perm[n * a.k + lane] : 0;
        const char *src = x + n * row_bytes;
        // warp-uniform trip count: every lane reaches every shuffle
        for (int64_t ob = 0; ob < row_bytes; ob += 512) {
            const int64_t o = ob + static_cast<int64_t>(lane) * 16;
            const bool in_row = o < row_bytes;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (in_row) v = ld_stream16(src + o);
            for (int j = 0; j < a.k; ++j) {
                const int dst = __shfl_sync(0xffffffffu, dst_l, j);
                // positions of assignments with an invalid expert id were
                // never written; never let them address outside x_sorted
                if (in_row && static_cast<uint32_t>(dst) < static_cast<uint32_t>(rows))
                    st16(xs + static_cast<int64_t>(dst) * row_bytes + o, v);
            }
        }
    }
}

// ---------------------------------------------------------------- combine

// y_n = sum_{j<k} w[n,j] * y_sorted[inv_perm[n k + j]], fp32 accumulation in
// slot order (sec. 2.2); one warp per token, 16-byte vectors.
template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a)
{
    constexpr int V = Vec16<T>::n;
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t row_bytes = static_cast<int64_t>(a.d) * sizeof(T);
    const char *ys = static_cast<const char *>(a.y_sorted);
    char *y = static_cast<char *>(a.y);
    const int64_t rows = a.N * a.k;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.N;
         n += warps) {
        const int src_l = lane < a.k ? a.inv_perm[n * a.k + lane] : 0;
        const float w_l = lane < a.k ? a.w[n * a.k + lane] : 0.f;
        // warp-uniform trip count: every lane reaches every shuffle
        for (int64_t ob = 0; ob < row_bytes; ob += 512) {
            const int64_t o = ob + static_cast<int64_t>(lane) * 16;
            const bool in_row = o < row_bytes;
            float acc[V];
#pragma unroll
            for (int u = 0; u < V; ++u) acc[u] = 0.f;
            for (int j = 0; j < a.k; ++j) {
                const int src = __shfl_sync(0xffffffffu, src_l, j);
                const float wj = __shfl_sync(0xffffffffu, w_l, j);
                if (!in_row || static_cast<uint32_t>(src) >= static_cast<uint32_t>(rows)) continue;
                float f[V];
                unpack16(ld_stream16(ys + static_cast<int64_t>(src) * row_bytes + o), f,
                         static_cast<const T *>(nullptr));
#pragma unroll
                for (int u = 0; u < V; ++u) acc[u] = fmaf(wj, f[u], acc[u]);
            }
            if (in_row) st16(y + n * row_bytes + o, pack16(acc, static_cast<const T *>(nullptr)));
        }
    }
}

// ------------------------------------------------------------- tile table

__global__ void tile_table_kernel(const int32_t *offsets, int32_t *mt_prefix, int E)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        int mt = 0;
        mt_prefix[0] = 0;
        for (int e = 0; e < E; ++e) {
            mt += (offsets[e + 1] - offsets[e] + kTileM - 1) / kTileM;
            mt_prefix[e + 1] = mt;
        }
    }
}

int warp_grid(int64_t N, int num_sms)
{
    const int64_t want = (N + 7) / 8;  // 8 warps per CTA, one token per warp
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    return static_cast<int>(max64(1, min64(want, cap)));
}

}  // namespace

cudaError_t launch_hist(const HistArgs &a, cudaStream_t s)
{
    const int64_t grid = num_chunks(a.N);
    if (grid == 0) return cudaSuccess;
    hist_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scan(const ScanArgs &a, cudaStream_t s)
{
    scan_kernel<<<1, kScanThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterArgs &a, cudaStream_t s)
{
    const int64_t grid = num_chunks(a.N);
    if (grid == 0) return cudaSuccess;
    scatter_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gather(int dtype, const GatherArgs &a, int num_sms, cudaStream_t s)
{
    if (a.N == 0) return cudaSuccess;
    const int grid = warp_grid(a.N, num_sms);
    if (dtype == kF32) gather_kernel<float><<<grid, 256, 0, s>>>(a);
    else gather_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_combine(int dtype, const CombineArgs &a, int num_sms, cudaStream_t s)
{
    if (a.N == 0) return cudaSuccess;
    const int grid = warp_grid(a.N, num_sms);
    if (dtype == kF32) combine_kernel<float><<<grid, 256, 0, s>>>(a);
    else combine_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_tile_table(const int32_t *offsets, int32_t *mt_prefix, int E, cudaStream_t s)
{
    tile_table_kernel<<<1, 32, 0, s>>>(offsets, mt_prefix, E);
    return cudaGetLastError();
}

}  // namespace moe
