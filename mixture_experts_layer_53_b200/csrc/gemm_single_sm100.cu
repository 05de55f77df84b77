// gemm_single_sm100.cu -- ragged grouped GEMM for the expert FFNs on single
// CTAs (tcgen05 cta_group::1, 128 x 256 tiles), for experts with few rows.
// The tile table it walks counts 128-row m-tiles; the CTA-pair kernel in
// gemm_sm100.cu takes the experts with many rows.
//
// Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
// loss, aux-free bias", sec. 2.2: after the sorted dispatch "each expert runs
// once on its slice" -- one matrix product per expert over rows
// offsets[e] .. offsets[e+1]-1 of x_sorted, no padding to a capacity.
//
// GEMM1: h = act(x_sorted W1[e]^T (, x_sorted W3[e]^T))  [rows, d_ff]
// GEMM2: y_sorted = h W2[e]^T (+ b2[e])                   [rows, d_model]
//
// When experts hold about 128 rows or fewer (fine-grained MoE such as the
// DeepSeek-V3 shape), 256-row pair tiles would compute mostly rows of the next
// expert; 128-row tiles waste less tensor work, which matters under the
// power cap.  Tiles are 128 rows x 256 accumulator columns, k-blocks of 64.  The tile
// list is (expert, n-tile, m-tile) with the m-tile innermost, so CTAs that run
// at the same time share one expert's weight tile through L2.  The tile
// count lives on the device (from the dispatch scan), so a persistent grid
// of one CTA per SM walks it with no host synchronisation.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A and B tiles into a 4-stage shared-memory ring
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (M=128, N=256, K=16, bf16 -> fp32) and tcgen05.commit
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (one row per
//               thread), fused activation / bias, bf16 stores
// Accumulators are double-buffered in TMEM (2 x 256 columns) so the
// epilogue of one tile overlaps the MMAs of the next.
//
// SwiGLU: the B tile holds 128 rows of W1 and the same 128 rows of W3, so
// accumulator columns 0..127 are the gate and 128..255 the up projection of
// 128 hidden units; the epilogue writes silu(gate) * up.
#include <cuda.h>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"
#include "epilogue_bf16.cuh"
#include "epilogue_f32.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;

enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_LINEAR = 2, EPI_F32 = 3 };
// Operand layouts (kernel template OPS):
//   OPS_KK    A and B K-major (the forward, the recomputed pre-activations)
//   OPS_K_MN  B MN-major: [E][K][n_out] weights read in place by 64 x 64
//             boxes (the dgrad products against W^T); ragged M
//   OPS_MN_MN A and B MN-major: row-major activations [rows][M] and
//             [rows][n_out]; expert e sums its own rows offsets[e] ..
//             offsets[e+1]-1 (the weight gradients); ragged K
enum { OPS_KK = 0, OPS_K_MN = 1, OPS_MN_MN = 2 };
constexpr int BOX_BYTES = 64 * 64 * 2;  // one 64 x 64 MN-major box

struct GemmArgs {
    const int32_t *offsets;
    const int32_t *mt_prefix;
    __nv_bfloat16 *out;
    int64_t ldo;
    const __nv_bfloat16 *bias;  // [E, n_out] or null
    int32_t *status;
    int E, K, n_out, n_tiles, b_rows;
    // EPI_F32: plain fp32 stores to out_f32 (the backward's products)
    float *out_f32;
    // ragged_k (OPS_MN_MN): the reduction of expert e runs over rows
    // offsets[e] .. offsets[e+1]-1 of the activations; A's columns are the
    // m_total result rows (m_tiles tiles of BM), B's the n_out result
    // columns; expert e's result starts at out_f32 + e * c_stride
    int ragged_k, m_tiles;
    int64_t m_total, c_stride;
    int accumulate;  // EPI_F32: add to the existing result instead of overwriting
    // OPS_K_MN: k-blocks 0..kb1-1 read tmB rows kb * BK of expert e with A
    // columns kb * BK; k-blocks kb1..kb_total-1 read tmB3 with A columns
    // a_col2 + (kb - kb1) * BK
    int kb1, kb_total, a_col2;
};

struct Ctl {
    // EPI_F32: per epilogue warp, a 32 x 32 fp32 chunk of its rows on the
    // way from TMEM (one row per lane) to global memory.  Ragged M: rows
    // padded to 36 floats (no bank conflicts) and stored back by the lanes in
    // whole 128-B rows; OPS_MN_MN: 4 KB per warp in the 128-byte swizzled
    // layout of a TMA store box (also free of bank conflicts).
    alignas(1024) float stage[4][32][36];  // bf16 results: kBf16StageBytes per warp at its start
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int off[kMaxE + 1];
    int mt[kMaxE + 1];
};
static_assert(sizeof(float) * 4 * 32 * 36 >= 4 * 4096, "TMA store staging fits");
static_assert(1024 + STAGES * STAGE_BYTES + sizeof(Ctl) <= 232448, "shared memory per CTA");

constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + sizeof(Ctl);

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

// Tile t of either schedule: the forward's ragged-M table, or (ragged_k)
// experts x m-tiles x n-tiles with m innermost.
__device__ __forceinline__ Tile tile_of(int t, const Ctl *c, const GemmArgs &g)
{
    if (!g.ragged_k) return decode_tile(t, c, g.E, g.n_tiles);
    const int per = g.m_tiles * g.n_tiles;
    const int e = t / per, local = t - e * per;
    return Tile{e, local % g.m_tiles, local / g.m_tiles};
}

// The warp's rows are row_first .. row_first + 31 (lane l holds TMEM lane
// row_first + l); rows from row_end on are not stored.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs &g, uint32_t tbase, int e, int row_first,
                                              int64_t row_end, int n0, float (*stage)[36], bool zero = false)
{
    if constexpr (EPI == EPI_F32) {
        float *out = g.out_f32 + (g.ragged_k ? static_cast<int64_t>(e) * g.c_stride : 0);
        epilogue_f32_rows(out, g.ldo, g.n_out, tbase, row_first, row_end, n0, stage, zero, g.accumulate != 0);
        return;
    }
    epilogue_bf16_rows<EPI>(nullptr, g.out, g.ldo, g.n_out, g.bias ? g.bias + static_cast<int64_t>(e) * g.n_out : nullptr,
                            tbase, row_first, row_end, n0, 0, out_cols<EPI>(), reinterpret_cast<uint8_t *>(stage),
                            [] {});
}

// MN-major operand tiles (OPS_K_MN, OPS_MN_MN; EPI_F32 only) are 64-column
// x 64-row boxes 8 KB apart, so the backward's products against W^T and
// over token rows need no transposed copies.  In OPS_MN_MN the last k-block
// of an expert can hold rows of the next one: the MMA warp zeroes those rows
// of both tiles in shared memory before the MMA reads them.
// The third tensor map is W3 (SwiGLU), the second B (OPS_K_MN) or the fp32
// result (OPS_MN_MN).
template <int EPI, int OPS = OPS_KK>
__global__ void __launch_bounds__(THREADS, 1)
    ffn_gemm_single_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB3, const GemmArgs g)
{
    pdl_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
    Ctl *ctl = reinterpret_cast<Ctl *>(tiles + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &ctl->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 128);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (EPI == EPI_SWIGLU || OPS != OPS_KK) prefetch_tmap(&tmB3);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i <= g.E; i += THREADS) {
        ctl->off[i] = g.offsets[i];
        ctl->mt[i] = g.mt_prefix ? g.mt_prefix[i] : 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = ctl->tmem_base;
    const int total = g.ragged_k ? g.E * g.m_tiles * g.n_tiles : ctl->mt[g.E] * g.n_tiles;
    const int num_kb = OPS == OPS_K_MN ? g.kb_total : (g.K + BK - 1) / BK;
    // k-blocks of a tile and the column (OPS_MN_MN: row) they start at
    auto kblocks = [&](int e) { return OPS == OPS_MN_MN ? (ctl->off[e + 1] - ctl->off[e] + BK - 1) / BK : num_kb; };
    auto kstart = [&](int e) { return OPS == OPS_MN_MN ? ctl->off[e] : 0; };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_parity = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile ti = tile_of(t, ctl, g);
                // ragged M (the OPS_MN_MN branch below places its own boxes)
                const int row0 = ctl->off[ti.e] + ti.m_tile * BM;
                const int brow = ti.e * g.b_rows + ti.n_tile * out_cols<EPI>();
                const int nkb = kblocks(ti.e), k0 = kstart(ti.e);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag, g.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sA = tiles + stage * STAGE_BYTES;
                    uint8_t *sB = sA + A_BYTES;
                    if constexpr (OPS == OPS_MN_MN) {
                        // boxes wholly past m_total / n_out are not loaded:
                        // their accumulator rows / columns are never stored
                        const int m0 = ti.m_tile * BM, n0 = ti.n_tile * BN;
                        const int aboxes = min(BM / 64, static_cast<int>((g.m_total - m0 + 63) / 64));
                        const int bboxes = min(BN / 64, (g.n_out - n0 + 63) / 64);
                        mbar_arrive_expect_tx(&ctl->full[stage], (aboxes + bboxes) * BOX_BYTES);
                        armed |= 1u << stage;
                        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                        const int r = k0 + kb * BK;
                        for (int c = 0; c < aboxes; ++c)
                            tma_load_2d(sA + c * BOX_BYTES, &tmA, &ctl->full[stage], m0 + c * 64, r);
                        for (int c = 0; c < bboxes; ++c)
                            tma_load_2d(sB + c * BOX_BYTES, &tmB, &ctl->full[stage], n0 + c * 64, r);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    if constexpr (OPS == OPS_K_MN) {
                        // boxes wholly past n_out are not loaded: their
                        // accumulator columns are never stored
                        const int n0 = ti.n_tile * BN;
                        const int boxes = min(BN / 64, (g.n_out - n0 + 63) / 64);
                        mbar_arrive_expect_tx(&ctl->full[stage], A_BYTES + boxes * BOX_BYTES);
                        armed |= 1u << stage;
                        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                        const bool second = kb >= g.kb1;
                        const int kk0 = (second ? kb - g.kb1 : kb) * BK;
                        tma_load_2d(sA, &tmA, &ctl->full[stage], (second ? g.a_col2 : 0) + kk0, row0);
                        const CUtensorMap *mb = second ? &tmB3 : &tmB;
                        for (int c = 0; c < boxes; ++c)
                            tma_load_3d(sB + c * BOX_BYTES, mb, &ctl->full[stage], n0 + c * 64, kk0, ti.e);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    mbar_arrive_expect_tx(&ctl->full[stage], STAGE_BYTES);
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    tma_load_2d(sA, &tmA, &ctl->full[stage], k0 + kb * BK, row0);
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(sB, &tmB, &ctl->full[stage], kb * BK, brow);
                        tma_load_2d(sB + B_BYTES / 2, &tmB3, &ctl->full[stage], kb * BK, brow);
                    } else {
                        tma_load_2d(sB, &tmB, &ctl->full[stage], k0 + kb * BK, brow);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag) {
                // let every copy this thread started land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if ((armed >> s) & 1u)
                        mbar_wait(&ctl->full[s], (armed_parity >> s) & 1u, abort_flag, g.status, false);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        // One lane issues; with OPS_MN_MN the whole warp runs the loop and
        // zeroes the rows past an expert's end before the MMA reads them.
        constexpr bool kWarp = OPS == OPS_MN_MN;
        if (kWarp || lane == 0) {
            constexpr uint32_t idesc = OPS == OPS_MN_MN   ? idesc_bf16_f32_mn(BM, BN)
                                       : OPS == OPS_K_MN ? idesc_bf16_f32_bmn(BM, BN)
                                                         : idesc_bf16_f32(BM, BN);
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                const bool w = mbar_wait(bar, parity, abort_flag, g.status);
                return kWarp ? __all_sync(0xffffffffu, w) : w;
            };
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true, issued = false;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                if (!wait(&ctl->tempty[buf], tphase ^ 1u)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                const int e = tile_of(t, ctl, g).e;
                const int nkb = kblocks(e);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait(&ctl->full[stage], phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = tiles + stage * STAGE_BYTES;
                    if constexpr (kWarp) {
                        // rows v..63 of every box (2 of A, 4 of B) belong to
                        // the next expert; whole 128-B rows, so the swizzle
                        // does not matter
                        const int v = ctl->off[e + 1] - ctl->off[e] - kb * BK;
                        if (v < BK) {
                            const int per_box = (BK - v) * 8;  // 16-B chunks
                            for (int i = lane; i < 6 * per_box; i += 32) {
                                const int box = i / per_box, j = i - box * per_box;
                                *reinterpret_cast<uint4 *>(st + box * BOX_BYTES + v * 128 + j * 16) =
                                    make_uint4(0u, 0u, 0u, 0u);
                            }
                            fence_proxy_async_smem();
                        }
                        __syncwarp();
                    }
                    if (!kWarp || lane == 0) {
                        const uint32_t a_addr = smem_u32(st);
                        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            // K-major: 16 columns are 32 B inside each 128-B
                            // row; MN-major: 16 K rows are two whole swizzle atoms
                            const uint64_t ad = OPS == OPS_MN_MN ? desc_sw128_mn(a_addr + kk * 2048, BOX_BYTES)
                                                                 : desc_sw128(a_addr + kk * 32);
                            const uint64_t bd = OPS != OPS_KK ? desc_sw128_mn(b_addr + kk * 2048, BOX_BYTES)
                                                              : desc_sw128(b_addr + kk * 32);
                            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        issued = true;
                        umma_commit(&ctl->empty[stage]);
                    }
                    if (kWarp) __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (!kWarp || lane == 0) umma_commit(&ctl->tfull[buf]);
                if (++buf == 2) {
                    buf = 0;
                    tphase ^= 1u;
                }
            }
            if ((!kWarp || lane == 0) && *abort_flag && issued) {
                // wait for every MMA issued so far before TMEM is freed
                umma_commit(&ctl->drain);
                mbar_wait(&ctl->drain, 0, abort_flag, g.status, false);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        int buf = 0;
        uint32_t tphase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&ctl->tfull[buf], tphase, abort_flag, g.status));
            if (!ok) break;
            tc_fence_after();
            const Tile ti = tile_of(t, ctl, g);
            int row_first;  // the warp's first row
            int64_t row_end;
            if (g.ragged_k) {  // result row m of expert e
                row_first = ti.m_tile * BM + quarter * 32;
                row_end = g.m_total;
            } else {
                row_first = ctl->off[ti.e] + ti.m_tile * BM + quarter * 32;
                row_end = ctl->off[ti.e + 1];
            }
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(buf * BN);
            if constexpr (EPI == EPI_F32 && OPS == OPS_MN_MN)
                epilogue_f32_tma(&tmB3, tbase, ti.e, row_first, g.m_total, ti.n_tile * BN, g.n_out,
                                 reinterpret_cast<uint8_t *>(ctl->stage) + quarter * 4096, kblocks(ti.e) == 0);
            else
                epilogue_tile<EPI>(g, tbase, ti.e, row_first, row_end, ti.n_tile * out_cols<EPI>(),
                                   ctl->stage[quarter], kblocks(ti.e) == 0);
            tc_fence_before();
            mbar_arrive(&ctl->tempty[buf]);
            if (++buf == 2) {
                buf = 0;
                tphase ^= 1u;
            }
        }
        // the staging buffers stay valid until this warp's stores are done
        if (EPI == EPI_F32 && OPS == OPS_MN_MN && lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// --------------------------------------------------------------- host side

template <int EPI, int OPS = OPS_KK>
cudaError_t launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &b3, const GemmArgs &g,
                        int num_sms, cudaStream_t s)
{
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void *>(&ffn_gemm_single_kernel<EPI, OPS>),
                                       static_cast<int>(kSmemBytes));
    if (err != cudaSuccess) return err;
    return launch_k(ffn_gemm_single_kernel<EPI, OPS>, dim3(num_sms), dim3(THREADS), kSmemBytes, s, a, b, b3, g);
}

}  // namespace

cudaError_t launch_gemm_tc_f32(const TcGemmArgs &t, int num_sms, cudaStream_t s)
{
    if (t.ragged_k != t.rows_mn) return cudaErrorInvalidValue;  // ragged K always reads the rows MN-major
    if (t.ragged_k ? (t.m_total == 0 || t.n_out == 0) : (t.a_rows == 0 || t.n_out == 0)) return cudaSuccess;
    if (t.b_mn && (t.ragged_k || t.k1 <= 0 || t.k2 < 0 || (t.k2 > 0) != (t.B2 != nullptr) ||
                   static_cast<uint64_t>(t.k1 + t.k2) != t.a_cols || t.k1 % 8 != 0 || t.n_out % 8 != 0))
        return cudaErrorInvalidValue;  // A's second column block must start on a 16-byte boundary
    if (t.rows_mn) {
        // row strides and inner extents in whole 16-byte units (tensor map rules)
        if (!t.ragged_k || t.b_mn || t.lda % 8 != 0 || t.ldb % 8 != 0 || t.m_total % 8 != 0 || t.n_out % 8 != 0 ||
            t.m_total > t.lda || t.n_out > t.ldb)
            return cudaErrorInvalidValue;
        // the result goes out through TMA stores: [E][m_total][n_out], 16-byte aligned
        if (t.ldc != t.n_out || t.c_stride != t.m_total * t.n_out || (reinterpret_cast<uintptr_t>(t.C) & 15u) != 0)
            return cudaErrorInvalidValue;
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
        g.out_f32 = t.C;
        g.ldo = t.ldc;
        g.status = t.status;
        g.E = t.E;
        g.n_out = t.n_out;
        g.n_tiles = (t.n_out + 255) / 256;
        g.ragged_k = 1;
        g.m_tiles = static_cast<int>((t.m_total + BM - 1) / BM);
        g.m_total = t.m_total;
        g.c_stride = t.c_stride;
        g.accumulate = t.accumulate;
        return launch_gemm<EPI_F32, OPS_MN_MN>(tA, tB, tOut, g, num_sms, s);
    }
    CUtensorMap tA, tB, tB3;
    if (!make_tmap_bf16(&tA, t.A, t.a_cols, t.a_rows, BM)) return cudaErrorInvalidValue;
    if (t.b_mn) {
        const uint64_t n = static_cast<uint64_t>(t.n_out), G = static_cast<uint64_t>(t.E);
        if (!make_tmap_bf16_mn(&tB, t.B, n, static_cast<uint64_t>(t.k1), G) ||
            !make_tmap_bf16_mn(&tB3, t.B2 ? t.B2 : t.B, n, static_cast<uint64_t>(t.B2 ? t.k2 : t.k1), G))
            return cudaErrorInvalidValue;
    } else if (!make_tmap_bf16(&tB, t.B, t.b_cols, t.b_rows, 256)) {
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
    g.n_tiles = (t.n_out + 255) / 256;
    g.b_rows = t.n_out;
    g.accumulate = t.accumulate;
    if (t.b_mn) {
        g.kb1 = static_cast<int>((t.k1 + BK - 1) / BK);
        g.kb_total = g.kb1 + static_cast<int>((t.k2 + BK - 1) / BK);
        g.a_col2 = static_cast<int>(t.k1);
        return launch_gemm<EPI_F32, OPS_K_MN>(tA, tB, tB3, g, num_sms, s);
    }
    return launch_gemm<EPI_F32>(tA, tB, tB, g, num_sms, s);
}

cudaError_t launch_ffn_bf16_sm100_single(const FfnArgs &a, int num_sms, cudaEvent_t mid, cudaStream_t s)
{
    if (a.tile_m != BM) return cudaErrorInvalidValue;  // the tile table must count 128-row tiles
    if (a.rows == 0) {
        if (mid) return cudaEventRecord(mid, s);
        return cudaSuccess;
    }
    const bool swiglu = a.act == kSwiglu;
    const uint64_t rows = static_cast<uint64_t>(a.rows);
    const uint64_t E = static_cast<uint64_t>(a.E);
    CUtensorMap tA, tB, tB3, tH, tW2;
    if (!make_tmap_bf16(&tA, a.x_sorted, a.d, rows, BM) ||
        !make_tmap_bf16(&tB, a.W1, a.d, E * a.F, swiglu ? 128 : 256) ||
        !make_tmap_bf16(&tB3, swiglu ? a.W3 : a.W1, a.d, E * a.F, swiglu ? 128 : 256) ||
        !make_tmap_bf16(&tH, a.h, a.F, rows, BM) || !make_tmap_bf16(&tW2, a.W2, a.F, E * a.d, 256))
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
    cudaError_t err = swiglu ? launch_gemm<EPI_SWIGLU>(tA, tB, tB3, g1, num_sms, s)
                             : launch_gemm<EPI_GELU>(tA, tB, tB3, g1, num_sms, s);
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
    return launch_gemm<EPI_LINEAR>(tH, tW2, tW2, g2, num_sms, s);
}

}  // namespace moe
