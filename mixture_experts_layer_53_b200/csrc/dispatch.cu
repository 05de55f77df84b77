// dispatch.cu -- sorted dispatch (course module "Mixture of Experts: routing,
// sorted dispatch, Switch aux loss, aux-free bias", sec. 2.2), the Switch
// loss (sec. 2.3) and the sign-rule bias step (sec. 2.5), plus the combine.
//
// The stable sort of assignments a = n k + j by expert is a counting sort
// over fixed chunks of 32 tokens:
//   1. per-chunk expert histograms (from the router, or from the ids),
//   2. one CTA per expert scans its column over the chunks: for every
//      (chunk, expert) the first position the chunk owns inside the expert's
//      slice, and the expert's count; one more CTA turns the counts into
//      offsets = exclusive prefix (slice starts),
//   3. each chunk ranks its own assignments in assignment order, so
//      position = offsets[e] + chunk base + rank is the stable order,
//   4. rows are copied x -> x_sorted with 16-byte vectors, one warp per token
//      (the token row is read once and written k times).
// Every reduction runs in a fixed order, so results are bitwise repeatable.
#include <map>
#include <mutex>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kCT = kChunkTokens;

// ---------------------------------------------------------------- histogram

__global__ void __launch_bounds__(256) hist_kernel(HistArgs a)
{
    pdl_enter();
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

constexpr int kScanThreads = 256;

// Exclusive prefix of v over the block (kScanThreads threads, fixed order).
__device__ __forceinline__ int block_exclusive_scan(int v, int *total)
{
    __shared__ int warp_sums[kScanThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int base = 0, tot = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) {
        if (w < warp) base += warp_sums[w];
        tot += warp_sums[w];
    }
    __syncthreads();
    *total = tot;
    return base + incl - v;
}

// One CTA per expert e: the chunk bases inside e's slice (prefix over chunks
// of hist[c][e], in place), count_e (into offsets[e+1]) and, if psum is given,
// P_e * N = sum over chunks of psum[c][e] in fp64 (fixed tree order).
__global__ void __launch_bounds__(kScanThreads) scan_cols_kernel(ScanArgs a)
{
    pdl_enter();
    const int e = blockIdx.x, E = a.E;
    const int64_t C = a.chunks;
    const int64_t per = (C + kScanThreads - 1) / kScanThreads;
    const int64_t c0 = min64(C, threadIdx.x * per), c1 = min64(C, c0 + per);
    int s = 0;
    double p = 0.0;
    for (int64_t c = c0; c < c1; ++c) {
        s += a.hist[c * E + e];
        if (a.psum) p += static_cast<double>(a.psum[c * E + e]);
    }
    int total;
    int run = block_exclusive_scan(s, &total);
    for (int64_t c = c0; c < c1; ++c) {
        const int v = a.hist[c * E + e];
        a.hist[c * E + e] = run;
        run += v;
    }
    if (a.psum && a.pe) {
        __shared__ double wsum[kScanThreads / 32];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = p;
        __syncthreads();
        if (threadIdx.x == 0) {
            double P = 0.0;
            for (int w = 0; w < kScanThreads / 32; ++w) P += wsum[w];
            a.pe[e] = P;
        }
    }
    if (threadIdx.x == 0) a.offsets[e + 1] = total;
}

// Router z-loss ("nano-moe", "Router z-loss"): (1/N) sum_n (lse z_n)^2 from
// the per-chunk sums, reduced in fp64 in a fixed order (strided per-thread
// sums, warp butterflies, then the warp sums in order).  Called by every
// thread of a kScanThreads block.
__device__ __forceinline__ void reduce_z_loss(const float *zpart, int64_t chunks, int64_t N, float *z_out)
{
    __shared__ double zsum[kScanThreads / 32];
    double s = 0.0;
    for (int64_t c = threadIdx.x; c < chunks; c += kScanThreads) s += static_cast<double>(zpart[c]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) zsum[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < kScanThreads / 32; ++w) t += zsum[w];
        *z_out = N > 0 ? static_cast<float>(t / static_cast<double>(N)) : 0.0f;
    }
}

__device__ __forceinline__ void write_dense_table(int32_t *offsets, int32_t *mt, int64_t N, int tile_m)
{
    offsets[0] = 0;
    offsets[1] = static_cast<int32_t>(N);
    if (mt) {
        mt[0] = 0;
        mt[1] = static_cast<int32_t>((N + tile_m - 1) / tile_m);
    }
}

__global__ void __launch_bounds__(kScanThreads) z_loss_kernel(const float *zpart, int64_t N, float *z_out)
{
    pdl_enter();
    reduce_z_loss(zpart, (N + kCT - 1) / kCT, N, z_out);
}

__global__ void dense_table_kernel(int32_t *offsets, int32_t *mt, int64_t N, int tile_m)
{
    pdl_enter();
    if (threadIdx.x == 0 && blockIdx.x == 0) write_dense_table(offsets, mt, N, tile_m);
}

// One CTA (E <= 256 threads' worth): offsets = exclusive prefix of counts,
// the GEMM tile table, the Switch loss L = E sum_e (count_e/N)(P_e/N) in fp64
// (course module sec. 2.3) and the sign-rule step b_e += gamma *
// sign(N k - E count_e) (sec. 2.5).
__global__ void __launch_bounds__(kScanThreads) scan_finalize_kernel(ScanArgs a)
{
    pdl_enter();
    const int E = a.E, t = threadIdx.x;
    const int cnt = t < E ? a.offsets[t + 1] : 0;
    int total, mt_total;
    const int off = block_exclusive_scan(cnt, &total);
    const int mt = (t < E && a.mt_prefix) ? (cnt + a.tile_m - 1) / a.tile_m : 0;
    const int mt_off = block_exclusive_scan(mt, &mt_total);
    if (t < E) {
        a.offsets[t] = off;
        if (a.counts) a.counts[t] = cnt;
        if (a.mt_prefix) a.mt_prefix[t] = mt_off;
        if (a.b_e && a.gamma > 0.f) {
            const long long diff = static_cast<long long>(a.N) * a.k - static_cast<long long>(E) * cnt;
            a.b_e[t] += a.gamma * static_cast<float>((diff > 0) - (diff < 0));
        }
    }
    if (t == 0) {
        a.offsets[E] = total;
        if (a.mt_prefix) a.mt_prefix[E] = mt_total;
        if (a.dense_offsets) write_dense_table(a.dense_offsets, a.dense_mt, a.N, a.dense_tile_m);
    }
    if (a.z_out && a.zpart) reduce_z_loss(a.zpart, a.chunks, a.N, a.z_out);  // block-uniform
    if (a.aux_out && a.psum && a.pe) {
        // L = E / N^2 * sum_e count_e (N P_e): one term per thread, summed in a
        // fixed tree (warp butterflies, then the 8 warp sums in order)
        __shared__ double wsum[kScanThreads / 32];
        double term = t < E ? static_cast<double>(cnt) * a.pe[t] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o);
        if ((t & 31) == 0) wsum[t >> 5] = term;
        __syncthreads();
        if (t == 0) {
            if (a.N == 0) {
                *a.aux_out = 0.0f;  // no tokens: every sum is empty
            } else {
                double s = 0.0;
                for (int w = 0; w < kScanThreads / 32; ++w) s += wsum[w];
                const double Nd = static_cast<double>(a.N);
                *a.aux_out = static_cast<float>(s * static_cast<double>(E) / (Nd * Nd));
            }
        }
    }
}

// For E <= 32 the whole of the above in one CTA: warp w scans the columns of
// experts w, w+8, ... (chunk bases in place, count_e, P_e * N in fp64 with
// fixed-order sums), then warp 0 does the finalizing step with lane e for
// expert e.  One launch instead of two.  STAGED (chunks * E <= kScanStage,
// chunks <= kScanStageZ): the histograms, probability sums and z-loss sums
// are first copied into shared memory with coalesced loads (one round trip
// instead of a chain of strided ones per lane), scanned there, and the
// chunk bases copied back; the sums are taken in the same order either way.
constexpr int kScanStage = 4096;
constexpr int kScanStageZ = 1024;

template <bool STAGED>
__global__ void __launch_bounds__(kScanThreads) scan_small_kernel(ScanArgs a)
{
    pdl_enter();
    __shared__ int cnt_s[32];
    __shared__ double pe_s[32];
    __shared__ int h_s[STAGED ? kScanStage : 1];
    __shared__ float p_s[STAGED ? kScanStage : 1];
    __shared__ float z_s[STAGED ? kScanStageZ : 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E;
    const int64_t C = a.chunks;
    int *hist = a.hist;
    const float *psum = a.psum;
    const float *zpart = a.zpart;
    if constexpr (STAGED) {
        for (int i = threadIdx.x; i < C * E; i += kScanThreads) {
            h_s[i] = a.hist[i];
            if (a.psum) p_s[i] = a.psum[i];
        }
        if (a.z_out && a.zpart)
            for (int i = threadIdx.x; i < C; i += kScanThreads) z_s[i] = a.zpart[i];
        __syncthreads();
        hist = h_s;
        psum = a.psum ? p_s : nullptr;
        zpart = z_s;
    }
    const int64_t per = (C + 31) / 32;
    const int64_t c0 = min64(C, lane * per), c1 = min64(C, c0 + per);
    for (int e = warp; e < E; e += kScanThreads / 32) {  // warp-uniform
        int s = 0;
        double p = 0.0;
#pragma unroll 8
        for (int64_t c = c0; c < c1; ++c) s += hist[c * E + e];
        if (psum) {
#pragma unroll 8
            for (int64_t c = c0; c < c1; ++c) p += static_cast<double>(psum[c * E + e]);
        }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        int run = incl - s;
        for (int64_t c = c0; c < c1; ++c) {
            const int v = hist[c * E + e];
            hist[c * E + e] = run;
            run += v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if (lane == 0) {
            cnt_s[e] = total;
            pe_s[e] = p;
        }
    }
    __syncthreads();
    if (warp == 0) {
        const int cnt = lane < E ? cnt_s[lane] : 0;
        const int mt = (lane < E && a.mt_prefix) ? (cnt + a.tile_m - 1) / a.tile_m : 0;
        int incl = cnt, mincl = mt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            const int v = __shfl_up_sync(0xffffffffu, mincl, o);
            if (lane >= o) {
                incl += u;
                mincl += v;
            }
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const int mt_total = __shfl_sync(0xffffffffu, mincl, 31);
        if (lane < E) {
            a.offsets[lane] = incl - cnt;
            if (a.counts) a.counts[lane] = cnt;
            if (a.psum && a.pe) a.pe[lane] = pe_s[lane];
            if (a.mt_prefix) a.mt_prefix[lane] = mincl - mt;
            if (a.b_e && a.gamma > 0.f) {
                const long long diff = static_cast<long long>(a.N) * a.k - static_cast<long long>(E) * cnt;
                a.b_e[lane] += a.gamma * static_cast<float>((diff > 0) - (diff < 0));
            }
        }
        if (lane == 0) {
            a.offsets[E] = total;
            if (a.mt_prefix) a.mt_prefix[E] = mt_total;
            if (a.dense_offsets) write_dense_table(a.dense_offsets, a.dense_mt, a.N, a.dense_tile_m);
        }
        if (a.aux_out && a.psum) {
            // L = E / N^2 * sum_e count_e (N P_e), summed in a fixed butterfly
            double term = lane < E ? static_cast<double>(cnt) * pe_s[lane] : 0.0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o);
            if (lane == 0) {
                const double Nd = static_cast<double>(a.N);
                *a.aux_out = a.N == 0 ? 0.0f : static_cast<float>(term * static_cast<double>(E) / (Nd * Nd));
            }
        }
    }
    if (a.z_out && a.zpart) reduce_z_loss(zpart, a.chunks, a.N, a.z_out);  // block-uniform
    if constexpr (STAGED)  // the chunk bases back to the workspace (after the barrier above)
        for (int i = threadIdx.x; i < C * E; i += kScanThreads) a.hist[i] = h_s[i];
}

// Switch loss and sign-rule step from partials summed over several forwards
// (course module sec. 2.3: L = E sum_e f_e P_e over the whole batch; sec.
// 2.5: the sign rule on the whole batch's load).  One CTA; the same fixed
// reduction order as scan_finalize_kernel.
__global__ void __launch_bounds__(kScanThreads) aux_partials_kernel(AuxPartialsArgs a)
{
    pdl_enter();
    const int E = a.E, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cnt = t < E ? a.counts[t] : 0;
    __shared__ long long csum[kScanThreads / 32];
    __shared__ double wsum[kScanThreads / 32];
    long long c = cnt;
    double term = t < E ? static_cast<double>(cnt) * a.psum[t] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        c += __shfl_xor_sync(0xffffffffu, c, o);
        term += __shfl_xor_sync(0xffffffffu, term, o);
    }
    if (lane == 0) {
        csum[warp] = c;
        wsum[warp] = term;
    }
    __syncthreads();
    long long total = 0;  // N k assignments
    double s = 0.0;
    for (int w = 0; w < kScanThreads / 32; ++w) {
        total += csum[w];
        s += wsum[w];
    }
    if (t < E && a.b_e && a.gamma > 0.f) {
        const long long diff = total - static_cast<long long>(E) * cnt;
        a.b_e[t] += a.gamma * static_cast<float>((diff > 0) - (diff < 0));
    }
    if (t == 0 && a.aux_out) {
        const double Nd = static_cast<double>(total) / static_cast<double>(a.k);
        *a.aux_out = total == 0 ? 0.0f : static_cast<float>(s * static_cast<double>(E) / (Nd * Nd));
    }
}

// ---------------------------------------------------------------- scatter

__global__ void __launch_bounds__(256) scatter_kernel(ScatterArgs a)
{
    pdl_enter();
    __shared__ int ids_s[kCT * kMaxK];
    const int64_t c = blockIdx.x;
    const int64_t a0 = c * kCT * a.k;
    const int ntok = static_cast<int>(min64(kCT, a.N - c * kCT));
    const int nas = ntok * a.k;
    for (int q = threadIdx.x; q < nas; q += blockDim.x) ids_s[q] = a.ids[a0 + q];
    __syncthreads();
    for (int q = threadIdx.x; q < nas; q += blockDim.x) {
        const int e = ids_s[q];
        if (e < 0 || e >= a.E) {  // reported by the histogram pass; no position
            a.inv_perm[a0 + q] = -1;
            continue;
        }
        int rank = 0;
        for (int r = 0; r < q; ++r) rank += (ids_s[r] == e);
        const int pos = a.offsets[e] + a.chunk_base[c * a.E + e] + rank;
        if (a.perm) a.perm[pos] = static_cast<int32_t>(a0 + q);
        a.inv_perm[a0 + q] = pos;
    }
}

// ----------------------------------------------------------------- gather

template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a)
{
    pdl_enter();
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

// ------------------------------------------------- scatter fused with gather

// Positions and row copies in one pass, one warp per token n of chunk c:
// the warp reads the chunk's ids (a few coalesced loads, shared through L1 by
// the chunk's 32 warps), ranks each of its k assignments among the chunk's
// earlier assignments to the same expert with ballots, so that
// position = offsets[e] + chunk base + rank exactly as in scatter_kernel,
// writes inv_perm (and perm), then stores the token's row at its k
// positions.  An assignment with an invalid expert id gets inv_perm = -1 and
// no row.
// The row kernels walk their work with a warp stride over a grid of exactly
// the CTAs that fit at once, so no partial wave trails.  Each lane moves kRowU
// 16-byte vectors of a kRowBlock-byte block, loading all of them before
// storing or accumulating.  dispatch_rows_kernel: one token per warp (its
// ranks are computed once); combine_kernel: (token, block) items.
constexpr int kRowU = 4;
constexpr int kRowBlock = 512 * kRowU;

template <typename T>
__global__ void __launch_bounds__(256) dispatch_rows_kernel(DispatchRowsArgs a)
{
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t row_bytes = static_cast<int64_t>(a.d) * sizeof(T);
    const int64_t nblk = (row_bytes + kRowBlock - 1) / kRowBlock;
    const char *x = static_cast<const char *>(a.x);
    char *xs = static_cast<char *>(a.x_sorted);
    const int k = a.k;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < a.N;
         n += warps) {
        const int64_t c = n / kCT;
        const int64_t a0 = c * kCT * k;                                   // chunk's first assignment
        const int nas = static_cast<int>(min64(kCT, a.N - c * kCT)) * k;  // chunk's assignments
        const int e_l = lane < k ? a.ids[n * k + lane] : -1;
        const int q_l = static_cast<int>(n * k + lane - a0);              // this slot inside the chunk
        const bool valid_l = lane < k && e_l >= 0 && e_l < a.E;
        int rank_l = 0;
        for (int base = 0; base < nas; base += 32) {  // warp-uniform
            const int q = base + lane;
            const int idq = q < nas ? a.ids[a0 + q] : -1;
            for (int j = 0; j < k; ++j) {
                const int ej = __shfl_sync(0xffffffffu, e_l, j);
                const int qj = __shfl_sync(0xffffffffu, q_l, j);
                const unsigned m = __ballot_sync(0xffffffffu, idq == ej && q < qj);
                if (lane == j) rank_l += __popc(m);
            }
        }
        int dst_l = -1;
        if (valid_l) dst_l = a.offsets[e_l] + a.chunk_base[c * a.E + e_l] + rank_l;
        if (lane < k) {
            a.inv_perm[n * k + lane] = dst_l;
            if (valid_l && a.perm) a.perm[dst_l] = static_cast<int32_t>(n * k + lane);
        }
        const char *src = x + n * row_bytes;
        for (int64_t ob = 0; ob < nblk * kRowBlock; ob += kRowBlock) {
            uint4 v[kRowU];
#pragma unroll
            for (int u = 0; u < kRowU; ++u) {
                const int64_t o = ob + u * 512 + static_cast<int64_t>(lane) * 16;
                v[u] = o < row_bytes ? ld_stream16(src + o) : make_uint4(0, 0, 0, 0);
            }
            for (int j = 0; j < k; ++j) {
                const int dst = __shfl_sync(0xffffffffu, dst_l, j);
                if (dst < 0) continue;  // warp-uniform
                char *drow = xs + static_cast<int64_t>(dst) * row_bytes;
#pragma unroll
                for (int u = 0; u < kRowU; ++u) {
                    const int64_t o = ob + u * 512 + static_cast<int64_t>(lane) * 16;
                    if (o < row_bytes) st16(drow + o, v[u]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- combine

// y_n = sum_{j<k} w[n,j] * y_sorted[inv_perm[n k + j]], fp32 accumulation in
// slot order (sec. 2.2), plus y_add[n] (the shared expert's output, sec. 2.1)
// when given; work items as in dispatch_rows_kernel, 16-byte vectors.
template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a)
{
    pdl_enter();
    constexpr int V = Vec16<T>::n;
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t row_bytes = static_cast<int64_t>(a.d) * sizeof(T);
    const int64_t nblk = (row_bytes + kRowBlock - 1) / kRowBlock;
    const char *ys = static_cast<const char *>(a.y_sorted);
    char *y = static_cast<char *>(a.y);
    const int64_t rows = a.N * a.k;
    for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         it < a.N * nblk; it += warps) {
        const int64_t n = it / nblk;
        const int64_t ob = (it - n * nblk) * kRowBlock;
        const int src_l = lane < a.k ? a.inv_perm[n * a.k + lane] : 0;
        const float w_l = lane < a.k ? a.w[n * a.k + lane] : 0.f;
        float acc[kRowU][V];
#pragma unroll
        for (int u = 0; u < kRowU; ++u)
#pragma unroll
            for (int i = 0; i < V; ++i) acc[u][i] = 0.f;
        for (int j = 0; j < a.k; ++j) {  // warp-uniform: every lane reaches every shuffle
            const int src = __shfl_sync(0xffffffffu, src_l, j);
            const float wj = __shfl_sync(0xffffffffu, w_l, j);
            // positions of assignments with an invalid expert id were never
            // written; never let them address outside y_sorted
            const bool ok = static_cast<uint32_t>(src) < static_cast<uint32_t>(rows);
            const char *row = ys + static_cast<int64_t>(ok ? src : 0) * row_bytes;
            uint4 v[kRowU];
#pragma unroll
            for (int u = 0; u < kRowU; ++u) {
                const int64_t o = ob + u * 512 + static_cast<int64_t>(lane) * 16;
                v[u] = (ok && o < row_bytes) ? ld_stream16(row + o) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kRowU; ++u) {
                const int64_t o = ob + u * 512 + static_cast<int64_t>(lane) * 16;
                if (!ok || o >= row_bytes) continue;
                float f[V];
                unpack16(v[u], f, static_cast<const T *>(nullptr));
#pragma unroll
                for (int i = 0; i < V; ++i) acc[u][i] = fmaf(wj, f[i], acc[u][i]);
            }
        }
#pragma unroll
        for (int u = 0; u < kRowU; ++u) {
            const int64_t o = ob + u * 512 + static_cast<int64_t>(lane) * 16;
            if (o >= row_bytes) continue;
            if (a.y_add) {  // + Shared(x_n), after the routed sum
                float f[V];
                unpack16(ld_stream16(static_cast<const char *>(a.y_add) + n * row_bytes + o), f,
                         static_cast<const T *>(nullptr));
#pragma unroll
                for (int i = 0; i < V; ++i) acc[u][i] += f[i];
            }
            st16(y + n * row_bytes + o, pack16(acc[u], static_cast<const T *>(nullptr)));
        }
    }
}

// ------------------------------------------------------------- tile table

__global__ void tile_table_kernel(const int32_t *offsets, int32_t *mt_prefix, int E, int tile_m)
{
    pdl_enter();
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        int mt = 0;
        mt_prefix[0] = 0;
        for (int e = 0; e < E; ++e) {
            mt += (offsets[e + 1] - offsets[e] + tile_m - 1) / tile_m;
            mt_prefix[e + 1] = mt;
        }
    }
}

// CTAs of `kernel` (256 threads) that fit on the device at once, capped by
// the work: items / 8 (one item per warp).
int row_grid(const void *kernel, int64_t items, int num_sms)
{
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> occ;
    int dev = 0, per_sm = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = occ.find({kernel, dev});
        if (it != occ.end()) per_sm = it->second;
    }
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        std::lock_guard<std::mutex> lock(mu);
        occ[{kernel, dev}] = per_sm;
    }
    const int64_t want = (items + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
    return static_cast<int>(max64(1, min64(want, cap)));
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
    return launch_k(hist_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, s, a);
}

cudaError_t launch_scan(const ScanArgs &a, cudaStream_t s)
{
    if (a.E > kScanThreads) return cudaErrorInvalidValue;
    if (a.E <= 32) {
        if (a.chunks * a.E <= kScanStage && a.chunks <= kScanStageZ)
            return launch_k(scan_small_kernel<true>, dim3(1), dim3(kScanThreads), 0, s, a);
        return launch_k(scan_small_kernel<false>, dim3(1), dim3(kScanThreads), 0, s, a);
    }
    cudaError_t err = launch_k(scan_cols_kernel, dim3(a.E), dim3(kScanThreads), 0, s, a);
    if (err != cudaSuccess) return err;
    return launch_k(scan_finalize_kernel, dim3(1), dim3(kScanThreads), 0, s, a);
}

cudaError_t launch_aux_partials(const AuxPartialsArgs &a, cudaStream_t s)
{
    if (a.E > kScanThreads) return cudaErrorInvalidValue;
    return launch_k(aux_partials_kernel, dim3(1), dim3(kScanThreads), 0, s, a);
}

cudaError_t launch_scatter(const ScatterArgs &a, cudaStream_t s)
{
    const int64_t grid = num_chunks(a.N);
    if (grid == 0) return cudaSuccess;
    return launch_k(scatter_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, s, a);
}

cudaError_t launch_gather(int dtype, const GatherArgs &a, int num_sms, cudaStream_t s)
{
    if (a.N == 0) return cudaSuccess;
    const int grid = warp_grid(a.N, num_sms);
    if (dtype == kF32) return launch_k(gather_kernel<float>, dim3(grid), dim3(256), 0, s, a);
    return launch_k(gather_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, a);
}

template <typename T>
cudaError_t launch_rows(void (*kernel)(T), const T &a, int64_t items, int num_sms, cudaStream_t s)
{
    if (items == 0) return cudaSuccess;
    const int grid = row_grid(reinterpret_cast<const void *>(kernel), items, num_sms);
    return launch_k(kernel, dim3(grid), dim3(256), 0, s, a);
}

int64_t row_blocks(int dtype, int d) { return (static_cast<int64_t>(d) * (dtype == kF32 ? 4 : 2) + kRowBlock - 1) / kRowBlock; }

cudaError_t launch_dispatch_rows(int dtype, const DispatchRowsArgs &a, int num_sms, cudaStream_t s)
{
    if (dtype == kF32) return launch_rows(dispatch_rows_kernel<float>, a, a.N, num_sms, s);
    return launch_rows(dispatch_rows_kernel<__nv_bfloat16>, a, a.N, num_sms, s);
}

cudaError_t launch_combine(int dtype, const CombineArgs &a, int num_sms, cudaStream_t s)
{
    const int64_t items = a.N * row_blocks(dtype, a.d);
    if (dtype == kF32) return launch_rows(combine_kernel<float>, a, items, num_sms, s);
    return launch_rows(combine_kernel<__nv_bfloat16>, a, items, num_sms, s);
}

cudaError_t launch_z_loss(const float *zpart, int64_t N, float *z_out, cudaStream_t s)
{
    return launch_k(z_loss_kernel, dim3(1), dim3(kScanThreads), 0, s, zpart, N, z_out);
}

cudaError_t launch_dense_table(int32_t *offsets, int32_t *mt, int64_t N, int tile_m, cudaStream_t s)
{
    return launch_k(dense_table_kernel, dim3(1), dim3(32), 0, s, offsets, mt, N, tile_m);
}

cudaError_t launch_tile_table(const int32_t *offsets, int32_t *mt_prefix, int E, int tile_m, cudaStream_t s)
{
    return launch_k(tile_table_kernel, dim3(1), dim3(32), 0, s, offsets, mt_prefix, E, tile_m);
}

}  // namespace moe
