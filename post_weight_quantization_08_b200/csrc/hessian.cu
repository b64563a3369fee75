// K1: Hessian accumulation H += 2·XᵀX.
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: the
// Hessian of a layer comes from its calibration activations X (XᵀX/n there;
// 2·XᵀX here, which leaves the codes unchanged because the damping is
// relative).  "GPTQ as Babai's Nearest Plane Algorithm", §2.1: XᵀX is the
// Gram matrix of the lattice basis.
//
// X is T×n bfloat16, token-major.  Products of two bf16 values are exact in
// float32, so the only rounding is the float32 accumulation over T.
// Only tiles on or above the diagonal are computed; each off-diagonal tile is
// also written mirrored, so H stays exactly symmetric.
#include <cuda_bf16.h>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int HT = 64;   // output tile edge
constexpr int HK = 32;   // tokens per shared-memory stage

__global__ void __launch_bounds__(256)
hessian_simt_kernel(const __nv_bfloat16* __restrict__ X, int64_t T, int64_t n,
                    int nt, float* __restrict__ H) {
  // Decode the upper-triangular tile pair (bi <= bj) from the linear index.
  int lin = blockIdx.x, bi = 0;
  while (lin >= nt - bi) { lin -= nt - bi; ++bi; }
  const int bj = bi + lin;
  const int64_t i0 = (int64_t)bi * HT, j0 = (int64_t)bj * HT;

  __shared__ __align__(16) float xa[HK][HT];
  __shared__ __align__(16) float xb[HK][HT];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};

  for (int64_t t0 = 0; t0 < T; t0 += HK) {
    for (int e = tid; e < HK * HT; e += 256) {
      const int kk = e / HT, c = e % HT;
      const int64_t t = t0 + kk;
      float va = 0.f, vb = 0.f;
      if (t < T) {
        if (i0 + c < n) va = __bfloat162float(X[t * n + i0 + c]);
        if (j0 + c < n) vb = __bfloat162float(X[t * n + j0 + c]);
      }
      xa[kk][c] = va;
      xb[kk][c] = vb;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < HK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xa[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&xb[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = i0 + ty * 4 + r;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t j = j0 + tx * 4 + c;
      if (i < n && j < n) {
        const float v = 2.0f * acc[r][c];
        H[i * n + j] += v;
        if (bi != bj) H[j * n + i] += v;
      }
    }
  }
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_hessian_accumulate(const void* X, int64_t T,
                                               int64_t n, float* H,
                                               void* stream) {
  if (H == nullptr || (X == nullptr && T > 0))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hessian_accumulate: null pointer");
  if (T < 0 || n < 1)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hessian_accumulate: T=%lld n=%lld",
                (long long)T, (long long)n);
  if (T == 0) return GPTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nt = (int)ceil_div(n, HT);
  const int tiles = nt * (nt + 1) / 2;
  GPTQ_LAUNCH(KK_HESSIAN, s, hessian_simt_kernel, tiles, 256, 0,
              static_cast<const __nv_bfloat16*>(X), T, n, nt, H);
  return GPTQ_OK;
}
