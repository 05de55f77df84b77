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
// The backward's ragged-M products use the same kernel with fp32 results
// (EPI_F32): the recomputed pre-activations x_s W1[e]^T (K-major B) and the
// dgrad products dy_s W2[e], [da | du] [W1[e]; W3[e]] (OPS_K_MN: each CTA
// loads its 128 result columns of the [E][K][n_out] weights as two 64 x 64
// MN-major boxes, so no transposed copy of the weights is made).
#include <cuda.h>

#include "common.cuh"
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
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES = (BN / 2) * BK * 2;  // 16 KB: this CTA's half of B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// Epilogue warps: one per TMEM lane quarter, or (GELU, whose erf epilogue
// outlasts a short k-loop) two per quarter, each on half of the columns.
// More epilogue warps let the pairs run further apart, which costs L2 reuse
// of the weight tiles: SwiGLU and the linear GEMM keep four.
template <int EPI> __host__ __device__ constexpr int epi_warps();
template <int EPI> __host__ __device__ constexpr int threads_of() { return 64 + 32 * epi_warps<EPI>(); }
constexpr uint32_t TMEM_COLS = 512;


enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_LINEAR = 2, EPI_F32 = 3 };
enum { OPS_KK = 0, OPS_K_MN = 1 };  // B K-major / MN-major (A K-major in both)
constexpr int BOX_BYTES = 64 * 64 * 2;  // one 64 x 64 MN-major box
template <int EPI> __host__ __device__ constexpr int epi_warps() { return EPI == EPI_GELU ? 8 : 4; }

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
};

struct Ctl {
    // EPI_F32: per epilogue warp, a 32 x 32 chunk on its way to global memory
    alignas(1024) float stage[4][32][36];
    uint64_t full[STAGES];   // used in the even CTA: both CTAs' bytes
    uint64_t empty[STAGES];  // each CTA: arrived by the even CTA's commit
    uint64_t tfull[2];       // each CTA: arrived by the even CTA's commit
    uint64_t tempty[2];      // even CTA: 4 epilogue warps x 2 CTAs
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int off[kMaxE + 1];
    int mt[kMaxE + 1];
};

constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + sizeof(Ctl);
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

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

// Output columns [c_begin, c_end) of one accumulator row (this thread's row).
template <int EPI>
__device__ __forceinline__ void epilogue_rows(const GemmArgs &g, uint32_t tbase, int e, int row, bool row_ok,
                                              int n0, int c_begin, int c_end)
{
    __nv_bfloat16 *orow = g.out + static_cast<int64_t>(row) * g.ldo;
    const __nv_bfloat16 *brow = g.bias ? g.bias + static_cast<int64_t>(e) * g.n_out : nullptr;
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
        uint32_t acc[32];
        tmem_ld32(tbase + c, acc);
        if constexpr (EPI == EPI_SWIGLU) {
            uint32_t up[32];
            tmem_ld32(tbase + 128 + c, up);
            tmem_ld_wait();
            if (row_ok) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int col = n0 + c + v * 8;
                    if (col < g.n_out) {
                        float h[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            h[u] = silu(__uint_as_float(acc[v * 8 + u])) * __uint_as_float(up[v * 8 + u]);
                        st16(orow + col, pack16(h, static_cast<const __nv_bfloat16 *>(nullptr)));
                    }
                }
            }
        } else {
            tmem_ld_wait();
            if (row_ok) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int col = n0 + c + v * 8;
                    if (col < g.n_out) {
                        float o[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) o[u] = __uint_as_float(acc[v * 8 + u]);
                        if (brow) {
                            float b[8];
                            unpack16(*reinterpret_cast<const uint4 *>(brow + col), b,
                                     static_cast<const __nv_bfloat16 *>(nullptr));
#pragma unroll
                            for (int u = 0; u < 8; ++u) o[u] += b[u];
                        }
                        if constexpr (EPI == EPI_GELU) {
#pragma unroll
                            for (int u = 0; u < 8; ++u) o[u] = gelu_erf(o[u]);
                        }
                        st16(orow + col, pack16(o, static_cast<const __nv_bfloat16 *>(nullptr)));
                    }
                }
            }
        }
    }
}

template <int EPI, int OPS = OPS_KK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_of<EPI>(), 1)
    ffn_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmB3, const GemmArgs g)
{
    pdl_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(tiles + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    volatile int *abort_flag = &ctl->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 2 * epi_warps<EPI>());  // every epilogue warp of both CTAs
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (EPI == EPI_SWIGLU || OPS == OPS_K_MN) prefetch_tmap(&tmB3);
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    for (int i = threadIdx.x; i <= g.E; i += threads_of<EPI>()) {
        ctl->off[i] = g.offsets[i];
        ctl->mt[i] = g.mt_prefix[i];
    }
    tc_fence_before();
    // barriers of both CTAs are initialised before either CTA signals the other
    cluster_sync();
    tc_fence_after();

    const uint32_t tmem_base = ctl->tmem_base;
    const int total = ctl->mt[g.E] * g.n_tiles;
    const int num_kb = OPS == OPS_K_MN ? g.kb_total : (g.K + BK - 1) / BK;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_parity = 0;
            bool ok = true;
            for (int t = pair; t < total && ok; t += npairs) {
                const Tile ti = decode_tile(t, ctl, g.E, g.n_tiles);
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
                        if (++stage == STAGES) {
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
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag && leader) {
                // both CTAs' copies land on these barriers: wait for them
                for (int s = 0; s < STAGES; ++s)
                    if ((armed >> s) & 1u)
                        mbar_wait(&ctl->full[s], (armed_parity >> s) & 1u, abort_flag, g.status, false);
            }
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
                    if (++stage == STAGES) {
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
            const Tile ti = decode_tile(t, ctl, g.E, g.n_tiles);
            const int row = ctl->off[ti.e] + ti.m_tile * PAIR_M + static_cast<int>(rank) * BM + row_in_cta;
            const bool row_ok = row < ctl->off[ti.e + 1];
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(buf * BN);
            if constexpr (EPI == EPI_F32)
                epilogue_f32_rows(g.out_f32, g.ldo, g.n_out, tbase, row - lane, ctl->off[ti.e + 1], ti.n_tile * BN,
                                  ctl->stage[quarter], false, g.accumulate != 0);
            else
                epilogue_rows<EPI>(g, tbase, ti.e, row, row_ok, ti.n_tile * out_cols<EPI>(),
                                   part * out_cols<EPI>() / parts, (part + 1) * out_cols<EPI>() / parts);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
            if (++buf == 2) {
                buf = 0;
                tphase ^= 1u;
            }
        }
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
cudaError_t launch_pair(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &b3, const GemmArgs &g,
                        int num_sms, cudaStream_t s)
{
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void *>(&ffn_gemm_pair_kernel<EPI, OPS>),
                                       static_cast<int>(kSmemBytes));
    if (err != cudaSuccess) return err;
    const int grid = (num_sms / 2) * 2;
    return launch_k(ffn_gemm_pair_kernel<EPI, OPS>, dim3(grid), dim3(threads_of<EPI>()), kSmemBytes, s, a, b, b3,
                    g);
}

}  // namespace

cudaError_t launch_gemm_tc_f32_pair(const TcGemmArgs &t, int num_sms, cudaStream_t s)
{
    if (t.ragged_k || t.rows_mn) return cudaErrorInvalidValue;  // ragged M only
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
        return launch_pair<EPI_F32, OPS_K_MN>(tA, tB, tB3, g, num_sms, s);
    }
    return launch_pair<EPI_F32>(tA, tB, tB, g, num_sms, s);
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
    CUtensorMap tA, tB, tB3, tH, tW2;
    // each CTA loads 128 rows of A and 128 rows of B per k-block
    if (!make_tmap_bf16(&tA, a.x_sorted, a.d, rows, BM) || !make_tmap_bf16(&tB, a.W1, a.d, E * a.F, 128) ||
        !make_tmap_bf16(&tB3, swiglu ? a.W3 : a.W1, a.d, E * a.F, 128) ||
        !make_tmap_bf16(&tH, a.h, a.F, rows, BM) || !make_tmap_bf16(&tW2, a.W2, a.F, E * a.d, 128))
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
    cudaError_t err = swiglu ? launch_pair<EPI_SWIGLU>(tA, tB, tB3, g1, num_sms, s)
                             : launch_pair<EPI_GELU>(tA, tB, tB3, g1, num_sms, s);
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
    return launch_pair<EPI_LINEAR>(tH, tW2, tW2, g2, num_sms, s);
}

}  // namespace moe
