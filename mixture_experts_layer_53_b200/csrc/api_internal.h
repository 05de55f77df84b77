// api_internal.h -- host pieces shared by the entry points of libmoe.so that
// live in different source files (internal; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// Argument checks on a moe_config that every entry point applies first.
moe_status validate_config(const moe_config *c);

// Records err's message for moe_last_error() and returns MOE_ERR_CUDA.
moe_status record_cuda_error(cudaError_t err);

// Multiprocessors of the current device (cached per device).
int device_sms();

// The sorted dispatch's launches (histogram, scan, then positions and rows
// in one pass when x is given, positions only otherwise) with its per-chunk
// scratch at `hist` (num_chunks(N) * E int32).  The caller has validated
// every argument.  Returns the first launch error.
cudaError_t enqueue_dispatch(const moe_config *c, const void *x, const int32_t *topk_ids, void *x_sorted,
                             int32_t *perm, int32_t *inv_perm, int32_t *offsets, int32_t *counts,
                             int32_t *dev_status, int32_t *hist, cudaStream_t s);

// Pointer checks of moe_dispatch (everything but the workspace).
moe_status check_dispatch_args(const moe_config *c, const void *x, const int32_t *topk_ids, const void *x_sorted,
                               const int32_t *inv_perm, const int32_t *offsets, const int32_t *counts);

}  // namespace moe
