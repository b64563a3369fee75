// Host launchers of the quantize-side kernels (one translation unit each).
#pragma once

#include "common.cuh"

namespace gptq {

// Columns [j0, j0+bw) of the float32 working copy Wp (m×n, processing order):
// quantize column by column with in-block error propagation.  Writes codes
// (m×n u8, processing order), scale/zero (m×ngroups), the scaled errors
// Err (m×bw, leading dimension ldE) and adds Σe² to loss_row (may be NULL).
gptq_status launch_sweep(const float* Wp, int64_t m, int64_t n, int64_t j0,
                         int bw, const float* U, int bits, int group,
                         int64_t ngroups, uint8_t* codes, float* scale,
                         uint8_t* zero, float* Err, int ldE, float* loss_row,
                         cudaStream_t s);

// Wp[:, c0:n] −= Err[:, 0:kw]·U[k0:k0+kw, c0:n]   (lazy-batch update).
gptq_status launch_trailing(float* Wp, int64_t m, int64_t n, int64_t c0,
                            const float* Err, int ldE, int64_t k0, int kw,
                            const float* U, cudaStream_t s);

}  // namespace gptq
