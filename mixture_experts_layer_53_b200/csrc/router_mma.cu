// router_mma.cu -- the whole router for E <= 32 on the bf16 path: logits
// z = W_g x, softmax / sigmoid, top-k, gates and the per-chunk statistics,
// in one kernel that streams x from HBM once.
//
// Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
// loss, aux-free bias", sec. 2 symbol table (z_n = W_g x_n, p_n =
// softmax(z_n)) and sec. 2.1 router table.
//
// With E <= 32 the product [N, d] x [d, E] is a few hundred MFLOP against
// N d bf16 bytes of x: the kernel is bound by reading x, and what matters is
// that every SM keeps many 16-byte loads of x in flight from its first cycle
// to its last.  So there is no shared-memory pipeline, no TMEM and no
// cluster: CTA c owns the 32 tokens of dispatch chunk c, and its warps split
// d into column ranges.  Each warp reads its range of the 32 rows straight
// from global memory into registers and multiplies on the warp-level tensor
// core instruction (mma.sync m16n8k16, bf16 in, fp32 out; 8 experts per n
// tile) -- the math is a small fraction of the load time.
//
// Fragment mapping.  The dot product sums over the reduction index, so A
// and B may use any one permutation of it.  Thread (g = lane / 4, t = lane %
// 4) loads CW consecutive columns (CW = 8 or 16: one 16- or 32-byte load) of
// token rows g and g + 8 and of W_g row (expert) g; for MMA m of the step
// its k slots {2t, 2t+1} hold its columns 4m, 4m+1 and {2t+8, 2t+9} hold
// 4m+2, 4m+3.  So one load per row and per expert feeds CW / 4 MMAs with no
// shuffles, and a load instruction of a warp reads 8 rows x 4 CW * 2
// contiguous bytes (64 or 128).
//
// Each step starts a fresh accumulator (CW / 4 MMAs deep) that is added to
// the warp's running sums in fp32, so the tensor core's own accumulation
// stays short.  The warps' partial logits are added in shared
// memory in warp (column) order, and one thread per token selects
// (select_thread_chunk): the result is bitwise repeatable.
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"
#include "router_select.cuh"

namespace moe {
namespace {

constexpr int kRows = kChunkTokens;     // tokens per CTA: one dispatch chunk
constexpr int kTargetWarps = 148 * 16;  // warps over the whole grid that keep HBM busy
// Steps in flight per warp (each step: 4 rows x CW columns of x and NT x CW
// of W_g per thread, in registers)
constexpr int kDepth = 2;

// Registers per thread, roughly: the buffered loads ((4 + NT) CW / 2 per
// step), the accumulators (8 NT), the row pointers and some 30 more.
__host__ __device__ constexpr int est_regs(int NT, int CW, int depth)
{
    return depth * (4 + NT) * CW / 2 + 8 * NT + 2 * (4 + NT) + 30;
}
// Warps per CTA at most: 16 while that fits 128 registers per thread (512
// threads), else 8 (255 registers).
__host__ __device__ constexpr int max_warps(int NT, int CW, int depth)
{
    return est_regs(NT, CW, depth) <= 110 ? 16 : 8;
}

struct StreamArgs {
    const __nv_bfloat16 *x;   // [N, d]
    const __nv_bfloat16 *Wg;  // [E, d]
    int64_t N;
    int d, E;
    int warps;       // column ranges per CTA (= warps per CTA)
    int range_cols;  // columns per range, a multiple of the step width
    int32_t *status;
    int clear_status;  // CTA 0 zeroes *status first (the forward's first kernel)
    SelectArgs sel;
    float *psum;
    int32_t *hist;
    float *zpart;
};

// CW consecutive bf16 (16 or 32 bytes, aligned to that size), not allocated
// in L1 (x is read once here; L2 keeps it for the dispatch's row copy that
// follows).  Not volatile: the loads of later steps may be issued before the
// MMAs of earlier ones.
template <int CW> __device__ __forceinline__ void ld_cols(const __nv_bfloat16 *p, uint32_t (&r)[CW / 2]);
template <> __device__ __forceinline__ void ld_cols<8>(const __nv_bfloat16 *p, uint32_t (&r)[4])
{
    asm("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "l"(p));
}
template <> __device__ __forceinline__ void ld_cols<16>(const __nv_bfloat16 *p, uint32_t (&r)[8])
{
    asm("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "l"(p));
}

// D += A B, m16n8k16, bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT: 8-expert n tiles (E <= 8 NT).  CW: columns of one row each thread
// loads per step (8: 16-byte loads; 16: 32-byte loads, when d is a multiple
// of 16 and x and W_g are 32-byte aligned), so a step is 4 CW columns and
// CW / 4 MMAs per row group and n tile.  DEPTH: steps in flight per warp.
template <int NT, int CW, int DEPTH>
__global__ void __launch_bounds__(max_warps(NT, CW, DEPTH) * 32) router_stream_kernel(const StreamArgs a)
{
    pdl_enter();
    if (a.clear_status && a.status && blockIdx.x == 0 && threadIdx.x == 0) *a.status = 0;
    constexpr int EB = 8 * NT;
    constexpr int LD = EB + 1;  // partial-row stride in floats (conflict-free per-token reads)
    constexpr int SW = 4 * CW;  // columns per step
    constexpr int V = CW / 2;   // 32-bit registers per row and step
    extern __shared__ float part[];  // [warps][kRows][LD]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRows;
    const int d = a.d;

    // this thread's token rows g, g + 8, g + 16, g + 24 of the chunk and
    // W_g rows (experts) nt * 8 + g
    const __nv_bfloat16 *xr[4];
    bool rv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t row = tok0 + g + 8 * r;
        rv[r] = row < a.N;
        xr[r] = a.x + (rv[r] ? row : 0) * static_cast<int64_t>(d);
    }
    const __nv_bfloat16 *wr[NT];
    bool ev[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int e = nt * 8 + g;
        ev[nt] = e < a.E;
        wr[nt] = a.Wg + static_cast<int64_t>(ev[nt] ? e : 0) * d;
    }

    float acc[2][NT][4];
#pragma unroll
    for (int rg = 0; rg < 2; ++rg)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[rg][nt][i] = 0.f;

    const int c_begin = warp * a.range_cols;
    const int c_end = min(d, c_begin + a.range_cols);
    // one step: columns c + CW t .. c + CW t + CW - 1 of the thread's 4 token
    // rows and NT expert rows (zeros past c_end, past N and past E; d is a
    // multiple of CW here, so the CW columns are all in or all out)
    auto load_step = [&](int c, uint32_t (&xv)[4][V], uint32_t (&wv)[NT][V]) {
        const int col = c + CW * t;
        const bool cv = col < c_end;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (rv[r] && cv) {
                ld_cols<CW>(xr[r] + col, xv[r]);
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) xv[r][i] = 0u;
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            if (ev[nt] && cv) {
                ld_cols<CW>(wr[nt] + col, wv[nt]);
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) wv[nt][i] = 0u;
            }
        }
    };
    // MMA m of a step: k slots {2t, 2t+1} hold the thread's columns 4m, 4m+1
    // and {2t+8, 2t+9} its columns 4m+2, 4m+3, for A and B alike
    auto mma_step = [&](const uint32_t (&xv)[4][V], const uint32_t (&wv)[NT][V]) {
#pragma unroll
        for (int rg = 0; rg < 2; ++rg) {
            const uint32_t(&lo)[V] = xv[2 * rg];      // row g of the row group
            const uint32_t(&hi)[V] = xv[2 * rg + 1];  // row g + 8
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < CW / 4; ++m)
                    mma16816(s4, lo[2 * m], hi[2 * m], lo[2 * m + 1], hi[2 * m + 1], wv[nt][2 * m], wv[nt][2 * m + 1]);
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[rg][nt][i] += s4[i];
            }
        }
    };
    // DEPTH steps in flight: step i's buffer is refilled with step i + DEPTH
    // right after its MMAs (steps past c_end load zeros)
    uint32_t xb[DEPTH][4][V], wb[DEPTH][NT][V];
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) load_step(c_begin + SW * j, xb[j], wb[j]);
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += SW * DEPTH) {
#pragma unroll
        for (int j = 0; j < DEPTH; ++j) {
            mma_step(xb[j], wb[j]);
            load_step(c + SW * (j + DEPTH), xb[j], wb[j]);
        }
    }

    // partial logits: fragment (rows g / g + 8 of each row group, experts
    // 2t, 2t + 1 of each n tile)
    float *mine = part + warp * kRows * LD;
#pragma unroll
    for (int rg = 0; rg < 2; ++rg)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int e = nt * 8 + 2 * t, r0 = rg * 16 + g;
            mine[r0 * LD + e] = acc[rg][nt][0];
            mine[r0 * LD + e + 1] = acc[rg][nt][1];
            mine[(r0 + 8) * LD + e] = acc[rg][nt][2];
            mine[(r0 + 8) * LD + e + 1] = acc[rg][nt][3];
        }
    __syncthreads();
    if (warp == 0) {  // one thread per token: the warps' partials in column order, then selection
        float z[EB];
#pragma unroll
        for (int e = 0; e < EB; ++e) z[e] = 0.f;
        for (int w = 0; w < a.warps; ++w) {
#pragma unroll
            for (int e = 0; e < EB; ++e) z[e] += part[(w * kRows + lane) * LD + e];
        }
        const int64_t n = tok0 + lane;
        select_thread_chunk<EB>(z, a.sel, a.psum, a.hist, a.zpart, n, n < a.N, static_cast<int64_t>(blockIdx.x));
    }
}

template <int NT, int CW>
cudaError_t launch_stream(StreamArgs a, int64_t ctas, cudaStream_t s)
{
    constexpr int LD = 8 * NT + 1;
    constexpr int MW = max_warps(NT, CW, kDepth);
    // column ranges: enough warps over the grid to keep HBM busy, at most MW
    // per CTA and at least one step per warp
    const int steps = (a.d + 4 * CW - 1) / (4 * CW);
    int64_t want = (kTargetWarps + ctas - 1) / ctas;
    want = want < 1 ? 1 : (want > MW ? MW : want);
    want = want > steps ? steps : want;
    const int per = (steps + static_cast<int>(want) - 1) / static_cast<int>(want);  // steps per warp
    a.range_cols = per * 4 * CW;
    a.warps = (steps + per - 1) / per;
    const size_t smem = static_cast<size_t>(a.warps) * kRows * LD * sizeof(float);
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void *>(&router_stream_kernel<NT, CW, kDepth>),
                                       MW * kRows * LD * static_cast<int>(sizeof(float)));
    if (err != cudaSuccess) return err;
    return launch_k(router_stream_kernel<NT, CW, kDepth>, dim3(static_cast<unsigned>(ctas)), dim3(a.warps * 32), smem,
                    s, a);
}

// 32-byte loads need twice the registers per step: used up to 16 experts.
template <int NT>
cudaError_t launch_stream_nt(const StreamArgs &a, int64_t ctas, bool wide, cudaStream_t s)
{
    if constexpr (NT <= 2) {
        if (wide) return launch_stream<NT, 16>(a, ctas, s);
    }
    return launch_stream<NT, 8>(a, ctas, s);
}

}  // namespace

cudaError_t launch_router_stream(const RouterArgs &r, int32_t *status, bool clear_status, cudaStream_t s)
{
    if (r.N == 0) return cudaSuccess;
    if (r.E > 32 || r.d % 8 != 0) return cudaErrorInvalidValue;
    StreamArgs a{};
    a.x = static_cast<const __nv_bfloat16 *>(r.x);
    a.Wg = static_cast<const __nv_bfloat16 *>(r.Wg);
    a.N = r.N;
    a.d = r.d;
    a.E = r.E;
    a.status = status;
    a.clear_status = clear_status ? 1 : 0;
    a.sel = SelectArgs{r.b_sel, r.ids, r.w, r.probs, r.E, r.k, r.router, r.norm_topk, r.scaling, r.lse};
    a.psum = r.psum;
    a.hist = r.hist;
    a.zpart = r.zpart;
    // 32-byte loads when every row starts on a 32-byte boundary
    const bool wide = r.d % 16 == 0 && (reinterpret_cast<uintptr_t>(r.x) & 31u) == 0 &&
                      (reinterpret_cast<uintptr_t>(r.Wg) & 31u) == 0;
    const int64_t ctas = num_chunks(r.N);
    if (r.E <= 8) return launch_stream_nt<1>(a, ctas, wide, s);
    if (r.E <= 16) return launch_stream_nt<2>(a, ctas, wide, s);
    return launch_stream_nt<4>(a, ctas, wide, s);
}

}  // namespace moe
