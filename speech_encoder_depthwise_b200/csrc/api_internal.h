// Host-side argument handling shared by the translation units of the C ABI (api.cu and
// dw_noalloc.cu): status mapping and the checks of the weight/bias gradient.
#pragma once

#include "dw_internal.h"
#include "dwconv.h"

namespace dwapi {

// DW_OK for cudaSuccess; otherwise records the error for dw_last_cuda_error and returns DW_ERR_CUDA.
dw_status_t cuda_status(cudaError_t e);

// Checks and argument set-up of the depthwise conv1d weight/bias gradient, everything except
// the memory of the partial rows: on DW_OK, *a holds every field but `partials` and `G`, and
// *n = B * T * C (0: nothing to read, dW and dbias are only zeroed).
dw_status_t bwd_dw_prepare(const void *x, const void *dy, float *dw, float *dbias, const int32_t *lengths,
                           int64_t B, int64_t T, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                           dwk::DwArgs *a, int64_t *n);

}  // namespace dwapi
