// dispatch_noalloc.cu -- moe_dispatch_noalloc: the sorted dispatch with its
// scratch in a fixed device array of this library instead of a workspace the
// caller allocates.
//
// The dispatch needs one int32 per (chunk of 32 tokens, expert): the chunk's
// expert histogram, which the scan rewrites in place into the chunk's first
// position inside each expert slice.  Here that scratch is the file-scope
// array below, MOE_NOALLOC_DISPATCH_MAX_SLOTS int32 (2 MiB), which every GPU
// that loads the library keeps until the process exits.  Everything else --
// the checks, the kernels and their order -- is moe_dispatch's own
// (enqueue_dispatch), so both entry points give the same outputs and errors.
//
// Host code must not use the array's name as a device address (in host code
// it names a host-side shadow), so the first call on each device looks up the
// real device address with cudaGetSymbolAddress, with that device current,
// and caches it together with the id of the device's context; a call that
// finds another context current (after cudaDeviceReset the module is loaded
// again, possibly elsewhere) looks the address up again.
//
// The histogram pass writes every scratch slot the scan then reads, so
// nothing left over from an earlier call is ever read and no clearing is
// needed.  All calls share the one array: two calls whose kernels overlap on
// the GPU (for example on two streams) race on it and must be ordered by the
// caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "api_internal.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using namespace moe;

static __device__ __align__(256) int32_t g_dispatch_scratch[MOE_NOALLOC_DISPATCH_MAX_SLOTS];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Id of the current context (unique for the life of the process), or 0 if
// the driver cannot tell.
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_dispatch_scratch on the current device, looked up once
// per (device, context).
cudaError_t scratch_address(int32_t **out)
{
    static std::mutex mu;
    static int32_t *addr[64] = {};
    static unsigned long long ctx_of[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    // 0 while no context is current on this thread yet: then look up (which
    // makes the device's primary context current) and record the id after
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (err != cudaSuccess) return err;
        addr[dev] = static_cast<int32_t *>(p);
        ctx_of[dev] = current_context_id();
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x, const int32_t *topk_ids, void *x_sorted,
                                int32_t *perm, int32_t *inv_perm, int32_t *offsets, int32_t *counts,
                                int32_t *dev_status, moe_stream_t stream)
{
    moe_status st = validate_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_dispatch_args(cfg, x, topk_ids, x_sorted, inv_perm, offsets, counts)) != MOE_OK) return st;
    const int64_t slots = num_chunks(cfg->N) * static_cast<int64_t>(cfg->E);
    // too large for the fixed scratch: refuse before touching the device
    if (slots > MOE_NOALLOC_DISPATCH_MAX_SLOTS) return MOE_ERR_WORKSPACE;
    int32_t *scratch = nullptr;
    cudaError_t err = scratch_address(&scratch);
    if (err != cudaSuccess) return record_cuda_error(err);
    err = enqueue_dispatch(cfg, x, topk_ids, x_sorted, perm, inv_perm, offsets, counts, dev_status, scratch,
                           reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MOE_OK : record_cuda_error(err);
}

}  // extern "C"
