// dispatch_noalloc.cu -- moe_dispatch_noalloc: the sorted dispatch with its
// scratch in a fixed device array of this library instead of a workspace the
// caller allocates.
//
// The dispatch needs one int32 per (chunk of 32 tokens, expert): the chunk's
// expert histogram, which the scan rewrites in place into the chunk's first
// position inside each expert slice.  Here that scratch is the file-scope
// array below, MOE_NOALLOC_DISPATCH_MAX_SLOTS int32 (2 MiB), which every GPU
// that loads the library keeps until the process exits.
//
// Host code must not use the array's name as a device address (in host code
// it names a host-side shadow), so the first call on each device looks up the
// real device address with cudaGetSymbolAddress, with that device current,
// and caches it; later calls on that device reuse it.
//
// The histogram pass writes every scratch slot the scan then reads, so
// nothing left over from an earlier call is ever read and no clearing is
// needed.  All calls share the one array: two calls whose kernels overlap on
// the GPU (for example on two streams) race on it and must be ordered by the
// caller.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using namespace moe;

static __device__ __align__(256) int32_t g_dispatch_scratch[MOE_NOALLOC_DISPATCH_MAX_SLOTS];

// Device address of g_dispatch_scratch on the current device (looked up once
// per device).
cudaError_t scratch_address(int32_t **out)
{
    static std::mutex mu;
    static int32_t *addr[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (err != cudaSuccess) return err;
        addr[dev] = static_cast<int32_t *>(p);
    }
    *out = addr[dev];
    return cudaSuccess;
}

moe_status check_config(const moe_config *c)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->N < 0 || c->d_model <= 0 || c->d_ff <= 0 || c->E <= 0 || c->k <= 0 || c->k > c->E)
        return MOE_ERR_INVALID_ARG;
    if (c->router < MOE_ROUTER_SOFTMAX_TOPK || c->router > MOE_ROUTER_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (c->act < MOE_ACT_GELU || c->act > MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
    if (c->dtype < MOE_F32 || c->dtype > MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (c->E > kMaxE || c->k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (c->d_model % 8 != 0 || c->d_ff % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (c->N * static_cast<int64_t>(c->k) >= (static_cast<int64_t>(1) << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status fail(cudaError_t) { return MOE_ERR_CUDA; }

}  // namespace

extern "C" {

moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x, const int32_t *topk_ids, void *x_sorted,
                                int32_t *perm, int32_t *inv_perm, int32_t *offsets, int32_t *counts,
                                int32_t *dev_status, moe_stream_t stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    const bool empty = cfg->N == 0;
    if (!offsets || !counts || (!empty && (!topk_ids || !inv_perm))) return MOE_ERR_INVALID_ARG;
    if ((x == nullptr) != (x_sorted == nullptr)) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_sorted) & 15u))
        return MOE_ERR_INVALID_ARG;
    const int64_t slots = num_chunks(cfg->N) * static_cast<int64_t>(cfg->E);
    // too large for the fixed scratch: refuse before touching the device
    if (slots > MOE_NOALLOC_DISPATCH_MAX_SLOTS) return MOE_ERR_WORKSPACE;
    int32_t *scratch = nullptr;
    cudaError_t err = scratch_address(&scratch);
    if (err != cudaSuccess) return fail(err);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    HistArgs h{topk_ids, nullptr, scratch, nullptr, dev_status, cfg->N, cfg->E, cfg->k};
    if ((err = launch_hist(h, s)) != cudaSuccess) return fail(err);
    ScanArgs sc{};
    sc.hist = scratch;
    sc.chunks = num_chunks(cfg->N);
    sc.N = cfg->N;
    sc.E = cfg->E;
    sc.k = cfg->k;
    sc.counts = counts;
    sc.offsets = offsets;
    if ((err = launch_scan(sc, s)) != cudaSuccess) return fail(err);
    ScatterArgs sa{topk_ids, scratch, perm, inv_perm, cfg->N, cfg->E, cfg->k, offsets};
    if ((err = launch_scatter(sa, s)) != cudaSuccess) return fail(err);
    if (x) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        GatherArgs ga{x, inv_perm, x_sorted, cfg->N, cfg->d_model, cfg->k};
        if ((err = launch_gather(cfg->dtype, ga, sms > 0 ? sms : 148, s)) != cudaSuccess) return fail(err);
    }
    return MOE_OK;
}

}  // extern "C"
