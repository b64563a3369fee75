// K4: lazy-batch trailing update  W[:, c0:] −= Err·U[k0:k0+kw, c0:].
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: every
// quantized column's error is subtracted from the columns not yet quantized.
// Applied per block instead of per column this is one product with K = block
// width; the result is the same up to float32 rounding order.
//
// float32 SIMT tile product: 128×128 output tile per CTA, 256 threads with an
// 8×8 register tile each, K staged 16 at a time through shared memory.
#include "kernels.cuh"

namespace gptq {
namespace {

constexpr int TM = 128, TN = 128, TK = 16;

__global__ void __launch_bounds__(256)
trailing_simt_kernel(float* __restrict__ Wp, int64_t m, int64_t n, int64_t c0,
                     const float* __restrict__ Err, int ldE, int64_t k0, int kw,
                     const float* __restrict__ U) {
  __shared__ __align__(16) float as[TK][TM];
  __shared__ __align__(16) float bs[TK][TN];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t rb = (int64_t)blockIdx.y * TM;
  const int64_t cb = c0 + (int64_t)blockIdx.x * TN;
  float acc[8][8] = {};
  for (int kb = 0; kb < kw; kb += TK) {
    for (int e = tid; e < TM * TK; e += 256) {
      const int r = e / TK, kk = e % TK;
      as[kk][r] = (rb + r < m && kb + kk < kw) ? Err[(rb + r) * ldE + kb + kk] : 0.f;
    }
    for (int e = tid; e < TK * TN; e += 256) {
      const int kk = e / TN, c = e % TN;
      bs[kk][c] = (kb + kk < kw && cb + c < n) ? U[(k0 + kb + kk) * n + cb + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = as[kk][ty * 4 + i];
        a[4 + i] = as[kk][64 + ty * 4 + i];
        b[i] = bs[kk][tx * 4 + i];
        b[4 + i] = bs[kk][64 + tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = rb + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (r >= m) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t c = cb + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (c < n) Wp[r * n + c] -= acc[i][j];
    }
  }
}

}  // namespace

gptq_status launch_trailing(float* Wp, int64_t m, int64_t n, int64_t c0,
                            const float* Err, int ldE, int64_t k0, int kw,
                            const float* U, cudaStream_t s) {
  if (c0 >= n || kw <= 0 || m <= 0) return GPTQ_OK;
  const dim3 grid((unsigned)ceil_div(n - c0, TN), (unsigned)ceil_div(m, TM));
  GPTQ_LAUNCH(KK_TRAIL, s, trailing_simt_kernel, grid, 256, 0, Wp, m, n, c0,
              Err, ldE, k0, kw, U);
  return GPTQ_OK;
}

}  // namespace gptq
