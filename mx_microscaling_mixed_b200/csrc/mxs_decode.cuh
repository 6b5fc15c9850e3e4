// mxs_decode.cuh -- the GEMM's decode path (a handful of activation rows),
// called by mxs_gemm.
#pragma once

#include "mxs_internal.cuh"

namespace mxs {

// True when the decode path takes this call: up to 16 activation rows whose
// packed rows fit in shared memory.  The path needs no workspace.
bool small_fits(const mxs_mxtensor *A, const mxs_mxtensor *W);

// Y = dequant(A) dequant(W)^T on the decode path (one launch).
mxs_status gemm_small(const mxs_mxtensor *A, const mxs_mxtensor *W, void *Y, int64_t ldy, cudaStream_t cs);

}  // namespace mxs
