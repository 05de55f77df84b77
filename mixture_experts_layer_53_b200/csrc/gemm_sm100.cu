// gemm_sm100.cu -- ragged grouped GEMM for the expert FFNs on CTA pairs
// (tcgen05 cta_group::2): each pair computes a 256 x 256 tile.
//
// Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
// loss, aux-free bias", sec. 2.2: each expert runs once on its slice --
// rows offsets[e] .. offsets[e+1]-1 of x_sorted, no padding to a capacity.
//
// GEMM1: h = act(x_sorted W1[e]^T (, x_sorted W3[e]^T))  [rows, d_ff]
// GEMM2: y_sorted = h W2[e]^T (+ b2[e])                   [rows, d_model]
//
// A cluster of two CTAs (one SM pair) owns a tile of 256 rows x 256
// accumulator columns.  Each CTA loads its own 128 rows of A and one half of
// the B tile (128 of its 256 rows) with TMA into its own shared memory; the
// even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), which
// reads A from each CTA and B from both, and accumulates each CTA's 128 rows
// in that CTA's TMEM.  Per k-block each SM so moves 32 KB instead of the 48 KB
// of a one-SM 128 x 256 tile, and a weight tile crosses L2 once per pair.
// No TMA load uses multicast: each CTA fetches its own tiles.
//
// Tiles are (expert, n-tile, m-tile of 256 rows), m-tile innermost, walked
// by a persistent grid of one pair per two SMs.  Warp roles per CTA:
//   warp 0     TMA producer (both CTAs; completion is counted on the even
//              CTA's `full` barrier, which expects both CTAs' bytes)
//   warp 1     TMEM allocation for the pair (both CTAs); in the even CTA one
//              lane issues the MMAs and commits to both CTAs' barriers
//   warps 2-   epilogue on the CTA's own 128 rows (tcgen05.ld), one or
//              (GELU) two warps per TMEM lane quarter, the latter each on
//              half of the tile's output columns; fused activation / bias,
//              bf16 stores
// SwiGLU: the even CTA's B half holds 128 rows of W1 and the odd CTA's the
// same 128 rows of W3, so accumulator columns 0..127 are the gate and
// 128..255 the up projection of 128 hidden units.
//
// The backward's products use the same kernel with fp32 results (EPI_F32):
// the recomputed pre-activations x_s W1[e]^T (K-major B); the dgrad
// products dy_s W2[e], [da | du] [W1[e]; W3[e]] (OPS_K_MN: each CTA loads
// its 128 result columns of the [E][K][n_out] weights as two 64 x 64
// MN-major boxes, so no transposed copy of the weights is made); and the
// weight gradients (OPS_MN_MN, ragged K): tile (expert, m-tile of 256,
// n-tile) sums its expert's own rows of two row-major activations, each CTA
// loading its 128 columns of both as MN-major boxes.  Only an expert's last
// k-block, which also holds rows of the next expert, needs more than the
// forward's protocol: there each CTA loads onto its own `tail_full`
// barrier, zeroes those rows in its own shared memory, fences, and arrives
// on the even CTA's `ready` barrier, which the even CTA waits on (cluster
// scope) before the MMA; the even CTA's `full` barrier gets a 0-byte arrival
// so that its phases stay in step.  The results leave through TMA stores.
#include <cuda.h>

#include "common.cuh"
#include "epilogue_bf16.cuh"
#include "epilogue_f32.cuh"
#include "host_util.h"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;        // rows per CTA
constexpr int PAIR_M = 256;    // rows per pair tile
constexpr int BN = 256;        // accumulator columns
constexpr int BK = 64;
constexpr int STAGES = 6;  // the most k-block stages a kernel uses
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES = (BN / 2) * BK * 2;  // 16 KB: this CTA's half of B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// Epilogue warps: one per TMEM lane quarter, or (GELU, whose erf epilogue
// outlasts a short k-loop) four per quarter, each on a quarter of the
// columns, one 32-column chunk at a time; that kernel keeps five k-block
// stages so that its staging buffers fit.  More epilogue warps let the pairs
// run further apart, which costs L2 reuse of the weight tiles: SwiGLU and
// the linear GEMM keep four.
template <int EPI> __host__ __device__ constexpr int epi_warps();
template <int EPI> __host__ __device__ constexpr int threads_of() { return 64 + 32 * epi_warps<EPI>(); }
constexpr uint32_t TMEM_COLS = 512;


enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_LINEAR = 2, EPI_F32 = 3 };
// B K-major / B MN-major (A K-major in both) / A and B MN-major, ragged K
enum { OPS_KK = 0, OPS_K_MN = 1, OPS_MN_MN = 2 };
constexpr int BOX_BYTES = 64 * 64 * 2;  // one 64 x 64 MN-major box
template <int EPI> __host__ __device__ constexpr int epi_warps() { return EPI == EPI_GELU ? 16 : 4; }
template <int EPI> __host__ __device__ constexpr int stages_of() { return epi_warps<EPI>() > 8 ? 5 : STAGES; }
template <int EPI> __host__ __device__ constexpr int bias_floats() { return 4 * BN / epi_warps<EPI>(); }

struct GemmArgs {
    const int32_t *offsets;
    const int32_t *mt_prefix;
    __nv_bfloat16 *out;
    int64_t ldo;
    const __nv_bfloat16 *bias;  // [E, n_out] or null
    int32_t *status;
    int E, K, n_out, n_tiles, b_rows;
    float *out_f32;  // EPI_F32: the result, ldo floats per row
    int accumulate;  // EPI_F32: add to the existing result
    // OPS_K_MN: k-blocks 0..kb1-1 read tmB rows kb * BK of expert e with A
    // columns kb * BK; k-blocks kb1..kb_total-1 read tmB3 with A columns
    // a_col2 + (kb - kb1) * BK
    int kb1, kb_total, a_col2;
    // OPS_MN_MN: expert e sums rows offsets[e] .. offsets[e+1]-1; the result
    // [E][m_total][n_out] has m_tiles tiles of 256 rows
    int m_tiles;
    int64_t m_total;
};

// Staging for the epilogue warps, after the k-block stages: EPI_F32, a
// 32 x 32 fp32 chunk per warp (rows padded to 36 floats, or 4 KB in the TMA
// store box's layout); bf16, kBf16StageBytes per warp (each buffer 2 KB-aligned).
// Lean epilogues (more than 8 warps) add each warp's fp32 bias values for
// its share of the columns.
template <int EPI> __host__ __device__ constexpr int stage_bytes_of()
{
    return EPI == EPI_F32 ? 4 * 32 * 36 * 4
                          : epi_warps<EPI>() * (kBf16StageBytes + (epi_warps<EPI>() > 8 ? bias_floats<EPI>() * 4 : 0));
}

struct Ctl {
    uint64_t full[STAGES];   // used in the even CTA: both CTAs' bytes
    uint64_t empty[STAGES];  // each CTA: arrived by the even CTA's commit
    uint64_t tfull[2];       // each CTA: arrived by the even CTA's commit
    uint64_t tempty[2];      // even CTA: 4 epilogue warps x 2 CTAs
    uint64_t drain;
    uint64_t tail_full[STAGES];  // OPS_MN_MN, each CTA: its own copies of an expert's last k-block
    uint64_t ready[STAGES];      // OPS_MN_MN, even CTA: both CTAs zeroed that k-block's extra rows
    uint32_t tmem_base;
    int abort;
    int off[kMaxE + 1];
    int mt[kMaxE + 1];
};

template <int EPI> constexpr size_t smem_bytes_of()
{
    return 1024 + stages_of<EPI>() * STAGE_BYTES + stage_bytes_of<EPI>() + sizeof(Ctl);
}
static_assert(smem_bytes_of<EPI_SWIGLU>() <= 232448 && smem_bytes_of<EPI_GELU>() <= 232448 &&
                  smem_bytes_of<EPI_LINEAR>() <= 232448 && smem_bytes_of<EPI_F32>() <= 232448,
              "shared memory per CTA");

struct Tile {
    int e, m_tile, n_tile;
};

__device__ __forceinline__ Tile decode_tile(int t, const Ctl *c, int E, int n_tiles)
{
    const int q = t / n_tiles;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (c->mt[mid] <= q) lo = mid;
        else hi = mid - 1;
    }
    const int mt_e = c->mt[lo + 1] - c->mt[lo];
    const int local = t - c->mt[lo] * n_tiles;
    return Tile{lo, local % mt_e, local / mt_e};
}

template <int EPI> __host__ __device__ constexpr int out_cols() { return EPI == EPI_SWIGLU ? 128 : 256; }

// Tile t: the ragged-M tile table, or (OPS_MN_MN) experts x n-tiles x
// m-tiles with m innermost.
template <int OPS> __device__ __forceinline__ Tile tile_at(int t, const Ctl *c, const GemmArgs &g)
{
    if constexpr (OPS != OPS_MN_MN) {
        return decode_tile(t, c, g.E, g.n_tiles);
    } else {
        const int per = g.m_tiles * g.n_tiles;
        const int e = t / per, local = t - e * per;
        return Tile{e, local % g.m_tiles, local / g.m_tiles};
    }
}

// OPS_MN_MN: 64-column boxes CTA r of the pair loads for a 256-wide range
// starting at `base` of an extent (0 past the end).
__device__ __forceinline__ int half_boxes(int r, int64_t extent, int base)
{
    const int64_t left = extent - (base + r * 128);
    return left <= 0 ? 0 : static_cast<int>(min64(2, (left + 63) / 64));
}

template <int EPI, int OPS = OPS_KK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_of<EPI>(), 1)
    ffn_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmOut,
                         const GemmArgs g)
{
    pdl_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
    constexpr int NST = stages_of<EPI>();
    uint8_t *stage_base = tiles + NST * STAGE_BYTES;
    Ctl *ctl = reinterpret_cast<Ctl *>(stage_base + stage_bytes_of<EPI>());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    volatile int *abort_flag = &ctl->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 2 * epi_warps<EPI>());  // every epilogue warp of both CTAs
        }
        mbar_init(&ctl->drain, 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&ctl->tail_full[s], 1);
            mbar_init(&ctl->ready[s], 2);
        }
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (EPI == EPI_SWIGLU || OPS != OPS_KK) prefetch_tmap(&tmB3);
        if (EPI != EPI_F32) prefetch_tmap(&tmOut);
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    for (int i = threadIdx.x; i <= g.E; i += threads_of<EPI>()) {
        ctl->off[i] = g.offsets[i];
        ctl->mt[i] = OPS == OPS_MN_MN ? 0 : g.mt_prefix[i];
    }
    tc_fence_before();
    // barriers of both CTAs are initialised before either CTA signals the other
    cluster_sync();
    tc_fence_after();

    const uint32_t tmem_base = ctl->tmem_base;
    const int total = OPS == OPS_MN_MN ? g.E * g.m_tiles * g.n_tiles : ctl->mt[g.E] * g.n_tiles;
    const int num_kb = OPS == OPS_K_MN ? g.kb_total : (g.K + BK - 1) / BK;
    // OPS_MN_MN: an expert's rows in k-blocks of BK
    auto mn_kblocks = [&](int e) { return (ctl->off[e + 1] - ctl->off[e] + BK - 1) / BK; };
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_parity = 0;
            uint32_t tpar = 0, tarmed = 0, tarmed_parity = 0;  // OPS_MN_MN tail_full phases per stage
            bool ok = true;
            for (int t = pair; t < total && ok; t += npairs) {
                const Tile ti = tile_at<OPS>(t, ctl, g);
                if constexpr (OPS == OPS_MN_MN) {
                    const int mrow = ti.m_tile * PAIR_M, ncol = ti.n_tile * BN;
                    const int ab0 = half_boxes(0, g.m_total, mrow), ab1 = half_boxes(1, g.m_total, mrow);
                    const int bb0 = half_boxes(0, g.n_out, ncol), bb1 = half_boxes(1, g.n_out, ncol);
                    const int ab = rank ? ab1 : ab0, bb = rank ? bb1 : bb0;
                    const uint32_t both_bytes = static_cast<uint32_t>(ab0 + bb0 + ab1 + bb1) * BOX_BYTES;
                    const uint32_t my_bytes = static_cast<uint32_t>(ab + bb) * BOX_BYTES;
                    const int m0 = mrow + static_cast<int>(rank) * BM, n0 = ncol + static_cast<int>(rank) * (BN / 2);
                    const int cnt = ctl->off[ti.e + 1] - ctl->off[ti.e], nkb = mn_kblocks(ti.e);
                    for (int kb = 0; kb < nkb; ++kb) {
                        if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag, g.status)) {
                            ok = false;
                            break;
                        }
                        uint8_t *sA = tiles + stage * STAGE_BYTES;
                        const int r = ctl->off[ti.e] + kb * BK;
                        const bool tail = cnt - kb * BK < BK;
                        if (leader) {  // a tail k-block only completes the phase
                            mbar_arrive_expect_tx(&ctl->full[stage], tail ? 0u : both_bytes);
                            armed |= 1u << stage;
                            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                        }
                        if (!tail) {
                            const uint32_t full_leader = mapa_shared(smem_u32(&ctl->full[stage]), 0);
                            for (int c = 0; c < ab; ++c)
                                tma_load_2d_pair(sA + c * BOX_BYTES, &tmA, full_leader, m0 + c * 64, r);
                            for (int c = 0; c < bb; ++c)
                                tma_load_2d_pair(sA + A_BYTES + c * BOX_BYTES, &tmB, full_leader, n0 + c * 64, r);
                        } else {
                            const uint32_t tp = (tpar >> stage) & 1u;
                            mbar_arrive_expect_tx(&ctl->tail_full[stage], my_bytes);
                            tarmed |= 1u << stage;
                            tarmed_parity = (tarmed_parity & ~(1u << stage)) | (tp << stage);
                            for (int c = 0; c < ab; ++c)
                                tma_load_2d(sA + c * BOX_BYTES, &tmA, &ctl->tail_full[stage], m0 + c * 64, r);
                            for (int c = 0; c < bb; ++c)
                                tma_load_2d(sA + A_BYTES + c * BOX_BYTES, &tmB, &ctl->tail_full[stage], n0 + c * 64,
                                            r);
                            tpar ^= 1u << stage;
                        }
                        if (++stage == NST) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    continue;
                }
                const int row0 = ctl->off[ti.e] + ti.m_tile * PAIR_M + static_cast<int>(rank) * BM;
                int brow;
                const CUtensorMap *tb;
                if (EPI == EPI_SWIGLU) {  // even CTA: W1 rows, odd CTA: the same rows of W3
                    brow = ti.e * g.b_rows + ti.n_tile * 128;
                    tb = rank ? &tmB3 : &tmB;
                } else {
                    brow = ti.e * g.b_rows + ti.n_tile * BN + static_cast<int>(rank) * (BN / 2);
                    tb = &tmB;
                }
                // OPS_K_MN: this CTA's 128 result columns as two boxes; boxes
                // wholly past n_out are not loaded (their columns are never
                // stored), and the even CTA expects both CTAs' bytes
                const int nc0 = ti.n_tile * BN + static_cast<int>(rank) * (BN / 2);
                auto boxes_of = [&](int r) {
                    const int left = g.n_out - (ti.n_tile * BN + r * (BN / 2));
                    return left <= 0 ? 0 : min(2, (left + 63) / 64);
                };
                const int my_boxes = boxes_of(static_cast<int>(rank));
                const uint32_t pair_bytes = OPS == OPS_K_MN
                                                ? 2u * A_BYTES + static_cast<uint32_t>(boxes_of(0) + boxes_of(1)) * BOX_BYTES
                                                : 2u * STAGE_BYTES;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag, g.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sA = tiles + stage * STAGE_BYTES;
                    const uint32_t full_leader = mapa_shared(smem_u32(&ctl->full[stage]), 0);
                    if constexpr (OPS == OPS_K_MN) {
                        if (leader) {
                            mbar_arrive_expect_tx(&ctl->full[stage], pair_bytes);
                            armed |= 1u << stage;
                            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                        }
                        const bool second = kb >= g.kb1;
                        const int kk0 = (second ? kb - g.kb1 : kb) * BK;
                        tma_load_2d_pair(sA, &tmA, full_leader, (second ? g.a_col2 : 0) + kk0, row0);
                        const CUtensorMap *mb = second ? &tmB3 : &tmB;
                        for (int c = 0; c < my_boxes; ++c)
                            tma_load_3d_pair(sA + A_BYTES + c * BOX_BYTES, mb, full_leader, nc0 + c * 64, kk0, ti.e);
                        if (++stage == NST) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    if (leader) {
                        mbar_arrive_expect_tx(&ctl->full[stage], 2 * STAGE_BYTES);
                        armed |= 1u << stage;
                        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    }
                    tma_load_2d_pair(sA, &tmA, full_leader, kb * BK, row0);
                    tma_load_2d_pair(sA + A_BYTES, tb, full_leader, kb * BK, brow);
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag && leader) {
                // both CTAs' copies land on these barriers: wait for them
                for (int s = 0; s < NST; ++s)
                    if ((armed >> s) & 1u)
                        mbar_wait(&ctl->full[s], (armed_parity >> s) & 1u, abort_flag, g.status, false);
            }
            if (*abort_flag) {
                // OPS_MN_MN: this CTA's own copies of tail k-blocks
                for (int s = 0; s < NST; ++s)
                    if ((tarmed >> s) & 1u)
                        mbar_wait(&ctl->tail_full[s], (tarmed_parity >> s) & 1u, abort_flag, g.status, false);
            }
        }
    } else if (warp == 1 && OPS == OPS_MN_MN) {
        // ------------------------ OPS_MN_MN: MMA issuer (even CTA) and the
        // tail k-blocks' zeroing (both CTAs, the whole warp)
        constexpr uint32_t idesc = idesc_bf16_f32_mn(PAIR_M, BN);
        auto wait_all = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, g.status));
        };
        int stage = 0, buf = 0;
        uint32_t phase = 0, tphase = 0, tpar = 0;
        bool ok = true, issued = false;
        for (int t = pair; t < total && ok; t += npairs) {
            const int e = tile_at<OPS>(t, ctl, g).e;
            const int nkb = mn_kblocks(e), cnt = ctl->off[e + 1] - ctl->off[e];
            if (leader) {
                if (!wait_all(&ctl->tempty[buf], tphase ^ 1u)) break;
                tc_fence_after();
            }
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
            for (int kb = 0; kb < nkb; ++kb) {
                uint8_t *st = tiles + stage * STAGE_BYTES;
                const int v = cnt - kb * BK;  // rows of the expert in this k-block
                const bool tail = v < BK;
                const uint32_t tp = (tpar >> stage) & 1u;
                if (tail) {
                    if (!wait_all(&ctl->tail_full[stage], tp)) {
                        ok = false;
                        break;
                    }
                    // rows v..63 of the four boxes (whole 128-B rows)
                    const int per_box = (BK - v) * 8;  // 16-B pieces
                    for (int i = lane; i < 4 * per_box; i += 32) {
                        const int box = i / per_box, j = i - box * per_box;
                        *reinterpret_cast<uint4 *>(st + box * BOX_BYTES + v * 128 + j * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->ready[stage]), 0));
                    tpar ^= 1u << stage;
                }
                if (leader) {
                    const bool w = tail ? __all_sync(0xffffffffu, mbar_wait<true>(&ctl->ready[stage], tp, abort_flag,
                                                                                 g.status))
                                        : wait_all(&ctl->full[stage], phase);
                    if (!w) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a_addr = smem_u32(st);
                        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_bf16_pair(d_tmem, desc_sw128_mn(a_addr + kk * 2048, BOX_BYTES),
                                           desc_sw128_mn(b_addr + kk * 2048, BOX_BYTES), idesc,
                                           (kb | kk) != 0 ? 1u : 0u);
                        issued = true;
                        umma_commit_pair(&ctl->empty[stage], 0x3);
                    }
                    __syncwarp();
                }
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (leader && lane == 0) umma_commit_pair(&ctl->tfull[buf], 0x3);
            if (++buf == 2) {
                buf = 0;
                tphase ^= 1u;
            }
        }
        if (leader && lane == 0 && *abort_flag && issued) {
            umma_commit_pair(&ctl->drain, 0x1);
            mbar_wait(&ctl->drain, 0, abort_flag, g.status, false);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = OPS == OPS_K_MN ? idesc_bf16_f32_bmn(PAIR_M, BN) : idesc_bf16_f32(PAIR_M, BN);
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true, issued = false;
            for (int t = pair; t < total && ok; t += npairs) {
                if (!mbar_wait(&ctl->tempty[buf], tphase ^ 1u, abort_flag, g.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&ctl->full[stage], phase, abort_flag, g.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(tiles + stage * STAGE_BYTES);
                    const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // MN-major B: 16 K rows are two whole swizzle atoms;
                        // each CTA's 128 columns are two chunks BOX_BYTES apart
                        const uint64_t bd = OPS == OPS_K_MN ? desc_sw128_mn(b_addr + kk * 2048, BOX_BYTES)
                                                            : desc_sw128(b_addr + kk * 32);
                        umma_bf16_pair(d_tmem, desc_sw128(a_addr + kk * 32), bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    umma_commit_pair(&ctl->empty[stage], 0x3);
                    if (++stage == NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair(&ctl->tfull[buf], 0x3);
                if (++buf == 2) {
                    buf = 0;
                    tphase ^= 1u;
                }
            }
            if (*abort_flag && issued) {
                umma_commit_pair(&ctl->drain, 0x1);
                mbar_wait(&ctl->drain, 0, abort_flag, g.status, false);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        constexpr int parts = epi_warps<EPI>() / 4;  // warps per TMEM lane quarter
        const int part = (warp - 2) / 4;            // which part of the output columns
        const int row_in_cta = quarter * 32 + lane;
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&ctl->tempty[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&ctl->tempty[1]), 0);
        int buf = 0;
        uint32_t tphase = 0;
        for (int t = pair; t < total; t += npairs) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&ctl->tfull[buf], tphase, abort_flag, g.status));
            if (!ok) break;
            tc_fence_after();
            const Tile ti = tile_at<OPS>(t, ctl, g);
            const int row = ctl->off[ti.e] + ti.m_tile * PAIR_M + static_cast<int>(rank) * BM + row_in_cta;
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(buf * BN);
            // the MMA warp may refill this accumulator once every epilogue
            // warp of both CTAs has read its part of it (the loads have
            // completed, tcgen05.wait::ld, before this runs)
            auto release = [&] {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_cta(buf ? tempty_leader1 : tempty_leader0);
            };
            if constexpr (EPI == EPI_F32 && OPS == OPS_MN_MN) {
                epilogue_f32_tma(&tmB3, tbase, ti.e, ti.m_tile * PAIR_M + static_cast<int>(rank) * BM + quarter * 32,
                                 g.m_total, ti.n_tile * BN, g.n_out, stage_base + quarter * 4096,
                                 mn_kblocks(ti.e) == 0);
                release();
            } else if constexpr (EPI == EPI_F32) {
                epilogue_f32_rows(g.out_f32, g.ldo, g.n_out, tbase, row - lane, ctl->off[ti.e + 1], ti.n_tile * BN,
                                  reinterpret_cast<float(*)[36]>(stage_base + quarter * (32 * 36 * 4)), false,
                                  g.accumulate != 0);
                release();
            } else {
                epilogue_bf16_rows<EPI, (epi_warps<EPI>() > 8)>(&tmOut, g.out, g.ldo, g.n_out,
                                        g.bias ? g.bias + static_cast<int64_t>(ti.e) * g.n_out : nullptr, tbase,
                                        row - lane, ctl->off[ti.e + 1], ti.n_tile * out_cols<EPI>(),
                                        part * out_cols<EPI>() / parts, (part + 1) * out_cols<EPI>() / parts,
                                        stage_base + (warp - 2) * kBf16StageBytes, release,
                                        reinterpret_cast<float *>(stage_base + epi_warps<EPI>() * kBf16StageBytes) +
                                            (warp - 2) * bias_floats<EPI>());
            }
            if (++buf == 2) {
                buf = 0;
                tphase ^= 1u;
            }
        }
        // the staging buffers stay valid until this warp's stores are done
        if ((EPI != EPI_F32 || OPS == OPS_MN_MN) && lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA frees TMEM or leaves while its pair partner may still use it
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <int EPI, int OPS = OPS_KK>
cudaError_t launch_pair(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &b3, const CUtensorMap &out,
                        const GemmArgs &g, int num_sms, cudaStream_t s)
{
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void *>(&ffn_gemm_pair_kernel<EPI, OPS>),
                                       static_cast<int>(smem_bytes_of<EPI>()));
    if (err != cudaSuccess) return err;
    const int grid = (num_sms / 2) * 2;
    return launch_k(ffn_gemm_pair_kernel<EPI, OPS>, dim3(grid), dim3(threads_of<EPI>()), smem_bytes_of<EPI>(), s, a, b, b3,
                    out, g);
}

}  // namespace

cudaError_t launch_gemm_tc_f32_pair(const TcGemmArgs &t, int num_sms, cudaStream_t s)
{
    if (t.rows_mn) {
        // weight gradients: ragged K over each group's rows, A and B read
        // MN-major in place, the result out through TMA stores
        if (!t.ragged_k || t.b_mn || t.lda % 8 != 0 || t.ldb % 8 != 0 || t.m_total % 8 != 0 || t.n_out % 8 != 0 ||
            t.m_total > t.lda || t.n_out > t.ldb || t.ldc != t.n_out || t.c_stride != t.m_total * t.n_out ||
            (reinterpret_cast<uintptr_t>(t.C) & 15u) != 0)
            return cudaErrorInvalidValue;
        if (t.m_total == 0 || t.n_out == 0) return cudaSuccess;
        CUtensorMap tA, tB, tOut;
        if (!make_tmap_bf16_mn_rows(&tA, t.A, static_cast<uint64_t>(t.m_total), t.a_rows,
                                    static_cast<uint64_t>(t.lda)) ||
            !make_tmap_bf16_mn_rows(&tB, t.B, static_cast<uint64_t>(t.n_out), t.a_rows,
                                    static_cast<uint64_t>(t.ldb)) ||
            !make_tmap_f32_store(&tOut, t.C, static_cast<uint64_t>(t.n_out), static_cast<uint64_t>(t.m_total),
                                 static_cast<uint64_t>(t.E)))
            return cudaErrorInvalidValue;
        GemmArgs g{};
        g.offsets = t.offsets;
        g.status = t.status;
        g.E = t.E;
        g.n_out = t.n_out;
        g.n_tiles = (t.n_out + BN - 1) / BN;
        g.m_tiles = static_cast<int>((t.m_total + PAIR_M - 1) / PAIR_M);
        g.m_total = t.m_total;
        return launch_pair<EPI_F32, OPS_MN_MN>(tA, tB, tOut, tOut, g, num_sms, s);
    }
    if (t.ragged_k) return cudaErrorInvalidValue;  // ragged K only with rows_mn
    if (t.a_rows == 0 || t.n_out == 0) return cudaSuccess;
    if (t.b_mn && (t.k1 <= 0 || t.k2 < 0 || (t.k2 > 0) != (t.B2 != nullptr) ||
                   static_cast<uint64_t>(t.k1 + t.k2) != t.a_cols || t.k1 % 8 != 0 || t.n_out % 8 != 0))
        return cudaErrorInvalidValue;  // A's second column block must start on a 16-byte boundary
    CUtensorMap tA, tB, tB3;
    if (!make_tmap_bf16(&tA, t.A, t.a_cols, t.a_rows, BM)) return cudaErrorInvalidValue;
    if (t.b_mn) {
        const uint64_t n = static_cast<uint64_t>(t.n_out), G = static_cast<uint64_t>(t.E);
        if (!make_tmap_bf16_mn(&tB, t.B, n, static_cast<uint64_t>(t.k1), G) ||
            !make_tmap_bf16_mn(&tB3, t.B2 ? t.B2 : t.B, n, static_cast<uint64_t>(t.B2 ? t.k2 : t.k1), G))
            return cudaErrorInvalidValue;
    } else if (!make_tmap_bf16(&tB, t.B, t.b_cols, t.b_rows, 128)) {
        return cudaErrorInvalidValue;
    }
    GemmArgs g{};
    g.offsets = t.offsets;
    g.mt_prefix = t.mt_prefix;
    g.out_f32 = t.C;
    g.ldo = t.ldc;
    g.status = t.status;
    g.E = t.E;
    g.K = t.K;
    g.n_out = t.n_out;
    g.n_tiles = (t.n_out + BN - 1) / BN;
    g.b_rows = t.n_out;
    g.accumulate = t.accumulate;
    if (t.b_mn) {
        g.kb1 = static_cast<int>((t.k1 + BK - 1) / BK);
        g.kb_total = g.kb1 + static_cast<int>((t.k2 + BK - 1) / BK);
        g.a_col2 = static_cast<int>(t.k1);
        return launch_pair<EPI_F32, OPS_K_MN>(tA, tB, tB3, tB3, g, num_sms, s);
    }
    return launch_pair<EPI_F32>(tA, tB, tB, tB, g, num_sms, s);
}

cudaError_t launch_ffn_bf16_sm100(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s)
{
    if (a.tile_m != PAIR_M) return cudaErrorInvalidValue;  // the tile table must count 256-row tiles
    if (a.rows == 0) {
        if (mid) return cudaEventRecord(mid, s);
        return cudaSuccess;
    }
    const bool swiglu = a.act == kSwiglu;
    const uint64_t rows = static_cast<uint64_t>(a.rows);
    const uint64_t E = static_cast<uint64_t>(a.E);
    CUtensorMap tA, tB, tB3, tH, tW2, tHout, tYout;
    // each CTA loads 128 rows of A and 128 rows of B per k-block; h and
    // y_sorted are written through 32 x 32 store boxes
    if (!make_tmap_bf16(&tA, a.x_sorted, a.d, rows, BM) || !make_tmap_bf16(&tB, a.W1, a.d, E * a.F, 128) ||
        !make_tmap_bf16(&tB3, swiglu ? a.W3 : a.W1, a.d, E * a.F, 128) ||
        !make_tmap_bf16(&tH, a.h, a.F, rows, BM) || !make_tmap_bf16(&tW2, a.W2, a.F, E * a.d, 128) ||
        !make_tmap_bf16_store(&tHout, a.h, a.F, rows) || !make_tmap_bf16_store(&tYout, a.y_sorted, a.d, rows))
        return cudaErrorInvalidValue;

    GemmArgs g1{};
    g1.offsets = a.offsets;
    g1.mt_prefix = a.mt_prefix;
    g1.out = static_cast<__nv_bfloat16 *>(a.h);
    g1.ldo = a.F;
    g1.bias = swiglu ? nullptr : static_cast<const __nv_bfloat16 *>(a.b1);
    g1.status = a.status;
    g1.E = a.E;
    g1.K = a.d;
    g1.n_out = a.F;
    g1.n_tiles = (a.F + (swiglu ? 127 : 255)) / (swiglu ? 128 : 256);
    g1.b_rows = a.F;
    cudaError_t err = swiglu ? launch_pair<EPI_SWIGLU>(tA, tB, tB3, tHout, g1, num_sms, s)
                             : launch_pair<EPI_GELU>(tA, tB, tB3, tHout, g1, num_sms, s);
    if (err != cudaSuccess) return err;
    if (mid && (err = cudaEventRecord(mid, s)) != cudaSuccess) return err;

    GemmArgs g2{};
    g2.offsets = a.offsets;
    g2.mt_prefix = a.mt_prefix;
    g2.out = static_cast<__nv_bfloat16 *>(a.y_sorted);
    g2.ldo = a.d;
    g2.bias = static_cast<const __nv_bfloat16 *>(a.b2);
    g2.status = a.status;
    g2.E = a.E;
    g2.K = a.F;
    g2.n_out = a.d;
    g2.n_tiles = (a.d + 255) / 256;
    g2.b_rows = a.d;
    return launch_pair<EPI_LINEAR>(tH, tW2, tW2, tYout, g2, num_sms, s);
}

}  // namespace moe
