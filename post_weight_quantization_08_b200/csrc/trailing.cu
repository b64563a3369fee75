// K4: lazy-batch trailing update  W[:, c0:] −= Err·U[k0:k0+kw, c0:].
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: every
// quantized column's error is subtracted from the columns not yet quantized.
// Applied once per block instead of once per column this is one product with
// K = block width; the result is the same up to float32 rounding order.
//
// The tensor-core update (n a multiple of 4) is trailing_tc.cuh's CTA body,
// run by the CTAs that ride in each sweep's launch; this file holds the
// transposed TF32 split of U it reads, its tensor maps, and the float32 SIMT
// tiles that take over when n % 4 ≠ 0.

#include "kernels.cuh"
#include "sm100.cuh"
#include "trailing_tc.cuh"

namespace gptq {
namespace {

// ---------------------------------------------------------------- SIMT path

constexpr int TM = 128, TN = 128, TK = 16;

__global__ void __launch_bounds__(256)
trailing_simt_kernel(float* __restrict__ Wp, int64_t m, int64_t n, int64_t c0, int64_t c1,
                     const float* __restrict__ Ehi, const float* __restrict__ Elo,
                     int64_t k0, int kw, const float* __restrict__ U) {
  __shared__ __align__(16) float as[TK][TM];
  __shared__ __align__(16) float bs[TK][TN];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t rb = (int64_t)blockIdx.y * TM;
  const int64_t cb = c0 + (int64_t)blockIdx.x * TN;
  float acc[8][8] = {};
  for (int kb = 0; kb < kw; kb += TK) {
    for (int e = tid; e < TM * TK; e += 256) {
      const int r = e / TK, kk = e % TK;
      const int64_t o = (rb + r) * SWEEP_BLOCK_MAX + kb + kk;
      as[kk][r] = (rb + r < m && kb + kk < kw) ? Ehi[o] + Elo[o] : 0.f;
    }
    for (int e = tid; e < TK * TN; e += 256) {
      const int kk = e / TN, c = e % TN;
      bs[kk][c] = (kb + kk < kw && cb + c < c1) ? U[(k0 + kb + kk) * n + cb + c] : 0.f;
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
      if (c < c1) Wp[r * n + c] -= acc[i][j];
    }
  }
}

// ---------------------------------------------------------------- split

// hi = TF32(x), lo = x − hi, written transposed: hiT[c][r] = TF32(x[r][c]).
// 32×32 tiles through shared memory (coalesced reads and writes).
__global__ void __launch_bounds__(256)
split_tf32_t_kernel(const float* __restrict__ x, int64_t n, float* __restrict__ hiT,
                    float* __restrict__ loT) {
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t r = r0 + ty + 8 * k, c = c0 + tx;
    tile[ty + 8 * k][tx] = (r < n && c < n) ? x[r * n + c] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t c = c0 + ty + 8 * k, r = r0 + tx;
    if (r < n && c < n) {
      const float v = tile[tx][ty + 8 * k];
      const float h = to_tf32(v);
      hiT[c * n + r] = h;
      loT[c * n + r] = v - h;
    }
  }
}

// ---------------------------------------------------------------- tcgen05 path

bool encode_f32(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  return encode_tiled_2d(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, inner, outer, row_bytes,
                         box_inner, box_outer);
}

}  // namespace

bool make_trail_maps(TrailMaps* maps, float* Wp, int64_t m, int64_t n, const float* Ehi,
                     const float* Elo, int64_t kw, int64_t epitch, const float* UhiT,
                     const float* UloT) {
  const int64_t mr = error_rows(m);
  return encode_f32(&maps->ahi, Ehi, kw, mr, epitch * 4, QK, QM) &&
         encode_f32(&maps->alo, Elo, kw, mr, epitch * 4, QK, QM) &&
         encode_f32(&maps->bhi, UhiT, n, n, n * 4, QK, QN) &&
         encode_f32(&maps->blo, UloT, n, n, n * 4, QK, QN) &&
         encode_f32(&maps->c, Wp, n, mr, n * 4, 32, QM);
}

bool trailing_uses_tensor_cores(int64_t n, int block) {
  return (n % 4 == 0) && (block % QK == 0) && n <= (1 << 30);
}

gptq_status launch_split_tf32_t(const float* x, int64_t n, float* hiT, float* loT,
                                cudaStream_t s) {
  const dim3 grid((unsigned)ceil_div(n, 32), (unsigned)ceil_div(n, 32));
  GPTQ_LAUNCH(KK_TRAIL, s, split_tf32_t_kernel, grid, 256, 0, x, n, hiT, loT);
  return GPTQ_OK;
}

gptq_status launch_trailing(float* Wp, int64_t m, int64_t n, int64_t c0, int64_t c1,
                            const float* Ehi, const float* Elo, int64_t k0, int kw,
                            const float* U, cudaStream_t s) {
  if (c1 > n) c1 = n;
  if (c0 >= c1 || kw <= 0 || m <= 0) return GPTQ_OK;
  const dim3 grid((unsigned)ceil_div(c1 - c0, TN), (unsigned)ceil_div(m, TM));
  GPTQ_LAUNCH(KK_TRAIL, s, trailing_simt_kernel, grid, 256, 0, Wp, m, n, c0, c1, Ehi, Elo, k0,
              kw, U);
  return GPTQ_OK;
}

}  // namespace gptq
