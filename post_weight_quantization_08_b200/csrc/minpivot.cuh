// The min-pivot processing order (minpivot.cu), used by gptq_prepare.
#pragma once

#include "common.cuh"

namespace gptq {

constexpr int MP_PANEL = 32;   // elimination steps between two trailing updates
constexpr int MP_MAX_N = 16384;  // the Schur diagonal of a panel sits in shared memory

// Doubles of scratch launch_min_pivot_order needs beside S.
size_t min_pivot_scratch_doubles(int64_t n);

// perm[p] = original column processed at position p under the min-pivot rule
// on H_d = H (dead diagonals → 1) + damp·mean·I.  S: n×n float64 scratch with
// leading dimension ld ≥ n; scratch: min_pivot_scratch_doubles(n) doubles.  A
// pivot that is not a positive normal float64 reports GPTQ_ERR_NOT_PD at its
// processing position.  n > MP_MAX_N returns GPTQ_ERR_UNSUPPORTED.
gptq_status launch_min_pivot_order(const float* H, int64_t n, const double* mean, double damp,
                                   double* S, int64_t ld, double* scratch, int32_t* perm,
                                   int32_t* info, cudaStream_t s);

}  // namespace gptq
