// router_sm100.cu -- router logits z = x W_g^T on the Blackwell tensor cores
// (bf16 inputs, fp32 accumulation), for the bf16 path.
//
// Course module "Mixture of Experts: routing, sorted dispatch, Switch aux
// loss, aux-free bias", sec. 2 symbol table: z_n = W_g x_n.  The scores,
// top-k and gates follow in select_kernel (router.cu); E <= 32 uses the
// streaming router of router_mma.cu instead.
//
// The product is [N, d] x [d, E] with small E, so the kernel is bound by
// reading x.  To keep every SM streaming x even when N / 128 is small, the
// reduction over d is split S ways (router_splits): CTA (tile, s) sums the
// k-blocks of split s of a tile of 128 tokens and writes its own partial
// logits [N, ld] at logits + s * N * ld; the selection kernel adds the S
// partials in split order.  One CTA:
//   warp 0      TMA: x tile (128 x 64) and W_g tile (E_pad x 64) per k-block
//               into a shared-memory ring (up to 8 stages)
//   warp 1      allocates TMEM, one lane issues tcgen05.mma M=128, N=E_pad
//               (E rounded up to 16; the W_g rows past E are TMA zero fill)
//   warps 2-5   one thread per token row: tcgen05.ld, fp32 stores of the row
// k-blocks are spread round-robin over several TMEM accumulators, which the
// epilogue then adds in fp32 round-to-nearest: the tensor core's own running
// sums are only num_kb / nacc steps deep, which keeps the logits close enough
// to an fp32 dot product for the 1e-5 tolerance of the Switch loss.
//
#include <cuda.h>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;
#ifndef MOE_ROUTER_MAX_STAGES
#define MOE_ROUTER_MAX_STAGES 8
#endif
#ifndef MOE_ROUTER_CTA_TARGET
#define MOE_ROUTER_CTA_TARGET 148
#endif
constexpr int MAX_STAGES = MOE_ROUTER_MAX_STAGES;
constexpr int THREADS = 192;
constexpr int A_BYTES = BM * BK * 2;
constexpr int SMEM_TILE_BUDGET = 196608;

struct Ctl {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tfull;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct LArgs {
    float *logits;  // [splits, N, ld] (unfused)
    int32_t *status;
    int clear_status;  // CTA 0 zeroes *status first (the forward's first kernel)
    int64_t N;
    int d, E, E_pad, ld, stages, splits;
    int nacc;            // TMEM accumulators, k-block kb -> kb % nacc
    uint32_t acc_cols;   // TMEM columns between accumulators (power of 2 >= max(E_pad, 32))
    uint32_t tmem_cols;  // nacc * acc_cols rounded up to a power of 2
};

__global__ void __launch_bounds__(THREADS, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                         const LArgs a)
{
    pdl_enter();
    // Clearing here instead of with a memset keeps the forward a chain of
    // kernels.  Any other writer of *status in this grid is a wait that ran
    // out after seconds, long after CTA 0 started.
    if (a.clear_status && a.status && blockIdx.x == 0 && threadIdx.x == 0) *a.status = 0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
    const int stage_bytes = A_BYTES + a.E_pad * BK * 2;
    Ctl *ctl = reinterpret_cast<Ctl *>(tiles + a.stages * stage_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &ctl->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->tfull, 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = ctl->tmem_base;
    // this CTA: token tile blockIdx.x / splits, k-blocks [kb0, kb0 + num_kb)
    const int all_kb = (a.d + BK - 1) / BK;
    const int split = static_cast<int>(blockIdx.x % a.splits);
    const int kb0 = split * all_kb / a.splits;
    const int num_kb = (split + 1) * all_kb / a.splits - kb0;
    const int row0 = static_cast<int>(blockIdx.x / a.splits) * BM;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_parity = 0;
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag, a.status)) break;
                uint8_t *sA = tiles + stage * stage_bytes;
                mbar_arrive_expect_tx(&ctl->full[stage], static_cast<uint32_t>(stage_bytes));
                armed |= 1u << stage;
                armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                tma_load_2d(sA, &tmX, &ctl->full[stage], (kb0 + kb) * BK, row0);
                tma_load_2d(sA + A_BYTES, &tmW, &ctl->full[stage], (kb0 + kb) * BK, 0);
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (*abort_flag) {
                for (int s = 0; s < a.stages; ++s)
                    if ((armed >> s) & 1u)
                        mbar_wait(&ctl->full[s], (armed_parity >> s) & 1u, abort_flag, a.status, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            const uint32_t idesc = idesc_bf16_f32(BM, a.E_pad);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&ctl->full[stage], phase, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(tiles + stage * stage_bytes);
                const uint32_t b_addr = a_addr + A_BYTES;
                // k-block kb accumulates into accumulator kb % nacc; the first
                // k-block of each accumulator overwrites it
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(kb % a.nacc) * a.acc_cols;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_bf16(d_tmem, desc_sw128(a_addr + kk * 32), desc_sw128(b_addr + kk * 32), idesc,
                              (kb >= a.nacc || kk != 0) ? 1u : 0u);
                issued = true;
                umma_commit(&ctl->empty[stage]);
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok && issued) umma_commit(&ctl->tfull);
            if (*abort_flag && issued) {
                umma_commit(&ctl->drain);
                mbar_wait(&ctl->drain, 0, abort_flag, a.status, false);
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int64_t n = static_cast<int64_t>(row0) + q * 32 + lane;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&ctl->tfull, 0, abort_flag, a.status));
        if (ok && num_kb > 0) {
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            const int used = min(a.nacc, num_kb);
            float *zrow = a.logits + (static_cast<int64_t>(split) * a.N + n) * a.ld;
            for (int c0 = 0; c0 < a.E_pad; c0 += 32) {
                uint32_t r[32];
                for (int s0 = 0; s0 < used; s0 += 2) {
                    // two accumulators' loads in flight, added in order
                    uint32_t t[32];
                    if (s0 == 0) tmem_ld32(taddr + c0, r);
                    else tmem_ld32(taddr + static_cast<uint32_t>(s0) * a.acc_cols + c0, t);
                    uint32_t t2[32];
                    const bool two = s0 + 1 < used;
                    if (two) tmem_ld32(taddr + static_cast<uint32_t>(s0 + 1) * a.acc_cols + c0, t2);
                    tmem_ld_wait();
                    if (s0 != 0) {
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            r[u] = __float_as_uint(__uint_as_float(r[u]) + __uint_as_float(t[u]));
                    }
                    if (two) {
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            r[u] = __float_as_uint(__uint_as_float(r[u]) + __uint_as_float(t2[u]));
                    }
                }
                if (n < a.N) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const int c = c0 + 4 * v;
                        if (c < a.ld)  // ld is a multiple of 4
                            st16(zrow + c, make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, a.tmem_cols);
    }
}

}  // namespace

int logits_ld(int E) { return (E + 3) / 4 * 4; }

// Splits of the d reduction: enough (tile, split) CTAs to cover the 148 SMs
// of a B200 once, at most one per k-block and at most 8.  A fixed function of
// the shape, so the workspace size does not depend on the device.
int router_splits(int64_t N, int d)
{
    const int64_t tiles = (N + BM - 1) / BM;
    const int64_t kbs = (d + BK - 1) / BK;
    int64_t sp = tiles > 0 ? MOE_ROUTER_CTA_TARGET / tiles : 1;
    sp = sp < 1 ? 1 : sp;
    sp = sp > 8 ? 8 : sp;
    sp = sp > kbs ? kbs : sp;
    return static_cast<int>(sp);
}

namespace {

// Fills the shape-dependent fields of LArgs; false if the tensor maps fail.
bool setup(LArgs &a, CUtensorMap &tX, CUtensorMap &tW, const void *x, const void *W_g, int64_t N, int d, int E,
           int32_t *status, bool clear_status)
{
    a.status = status;
    a.clear_status = clear_status ? 1 : 0;
    a.N = N;
    a.d = d;
    a.E = E;
    a.E_pad = ((E + 15) / 16) * 16;
    a.ld = logits_ld(E);
    a.splits = router_splits(N, d);
    // accumulators 32-column aligned (a power of 2 >= E_pad, >= 32), k-blocks
    // dealt round-robin so that each sums at most 4 of the CTA's k-blocks
    // (the tensor core's own running sums stay short), at most 8 and as many
    // as fit in 512 columns
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(a.E_pad)) cols <<= 1;
    a.acc_cols = cols;
    const int kb_per_cta = ((d + BK - 1) / BK + a.splits - 1) / a.splits;
    a.nacc = (kb_per_cta + 3) / 4;
    if (a.nacc > 8) a.nacc = 8;
    if (a.nacc > static_cast<int>(512 / cols)) a.nacc = static_cast<int>(512 / cols);
    if (a.nacc < 1) a.nacc = 1;
    uint32_t tcols = 32;
    while (tcols < cols * static_cast<uint32_t>(a.nacc)) tcols <<= 1;
    a.tmem_cols = tcols;
    const int stage_bytes = A_BYTES + a.E_pad * BK * 2;
    a.stages = SMEM_TILE_BUDGET / stage_bytes;
    if (a.stages > MAX_STAGES) a.stages = MAX_STAGES;
    return make_tmap_bf16(&tX, x, d, static_cast<uint64_t>(N), BM) &&
           make_tmap_bf16(&tW, W_g, d, static_cast<uint64_t>(E), static_cast<uint32_t>(a.E_pad));
}

constexpr int kSmemMax = 1024 + SMEM_TILE_BUDGET + static_cast<int>(sizeof(Ctl));

size_t smem_bytes(const LArgs &a)
{
    const int stage_bytes = A_BYTES + a.E_pad * BK * 2;
    return 1024 + static_cast<size_t>(a.stages) * stage_bytes + sizeof(Ctl);
}

}  // namespace

cudaError_t launch_router_logits_sm100(const void *x, const void *W_g, float *logits, int64_t N, int d, int E,
                                       int32_t *status, bool clear_status, cudaStream_t s)
{
    if (N == 0) return cudaSuccess;
    LArgs a{};
    CUtensorMap tX, tW;
    if (!setup(a, tX, tW, x, W_g, N, d, E, status, clear_status)) return cudaErrorInvalidValue;
    a.logits = logits;
    cudaError_t err = ensure_smem_attr(reinterpret_cast<const void *>(&router_logits_kernel), kSmemMax);
    if (err != cudaSuccess) return err;
    const int64_t grid = (N + BM - 1) / BM * a.splits;
    return launch_k(router_logits_kernel, dim3(static_cast<unsigned>(grid)), dim3(THREADS), smem_bytes(a), s, tX,
                    tW, a);
}

}  // namespace moe
