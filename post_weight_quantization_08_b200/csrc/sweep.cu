// K3: the column sweep of one lazy-batch block.
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: for
// column j, quantize with the group's scale, err_j = (col_j − q_j)/H⁻¹[j,j]
// and subtract err_j·H⁻¹[j, j+1:] from the columns not yet quantized.  With
// U the upper inverse-Cholesky factor: e_j = (w_j − q̂_j)/U_jj and
// w[j+1:] −= e_j·U[j, j+1:].  Inside the block every column updates the
// block's later columns; the columns after the block receive the block's
// errors in one product afterwards (trailing.cu).
//
// Rows are independent (U is shared), so one thread owns one row.  The CTA
// stages its rows' block values (transposed, conflict-free) and the block's
// U panel (transposed, so the values a later column needs from one sub-block
// are contiguous) in shared memory.  The block is walked in sub-blocks of 32
// columns held in registers: the 32 dependent column steps run fully
// unrolled on registers, then the sub-block's 32 errors update the block's
// later columns in shared memory with vectorised U reads.
//
// Scale and zero: min-max over the group's current values at the group's
// first column, the range always containing 0; decisions in IEEE float32
// (division and rint are correctly rounded, no fast-math).
#include "kernels.cuh"

namespace gptq {
namespace {

constexpr int SB = 128;      // largest block width
constexpr int SS = 32;       // register sub-block
constexpr int LDU = SB + 4;  // transposed-U row stride (floats; 16-byte rows)
constexpr int SWEEP_RT = 64; // rows (threads) per CTA

template <int RT>
struct SweepSmem {
  static constexpr int LDV = RT + 1;   // values: [SB][LDV] floats
  static constexpr int LDC = RT + 4;   // codes:  [SB][LDC] bytes
  static constexpr size_t bytes =
      sizeof(float) * (SB * LDU + SB * LDV + SB) + SB * LDC;
};

template <int RT>
__global__ void __launch_bounds__(RT)
sweep_kernel(const float* __restrict__ Wp, int64_t m, int64_t n, int64_t j0,
             int bw, const float* __restrict__ U, int bits, int group,
             int64_t ngroups, uint8_t* __restrict__ codes,
             float* __restrict__ scale, uint8_t* __restrict__ zero,
             float* __restrict__ Err, int ldE, float* __restrict__ loss_row) {
  constexpr int LDV = SweepSmem<RT>::LDV;
  constexpr int LDC = SweepSmem<RT>::LDC;
  extern __shared__ __align__(16) unsigned char smraw[];
  float* UT = reinterpret_cast<float*>(smraw);     // UT[c][i] = U[j0+i][j0+c]
  float* vals = UT + SB * LDU;                     // vals[c][r]
  float* rdiag = vals + SB * LDV;                  // 1/U_jj
  uint8_t* cs = reinterpret_cast<uint8_t*>(rdiag + SB);

  const int t = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * RT;
  const int64_t row = r0 + t;

  for (int e = t; e < SB * SB; e += RT) {
    const int i = e / SB, c = e % SB;
    UT[c * LDU + i] = (i < bw && c < bw) ? U[(j0 + i) * n + j0 + c] : 0.f;
  }
  for (int e = t; e < RT * SB; e += RT) {
    const int r = e / SB, c = e % SB;
    vals[c * LDV + r] = (r0 + r < m && c < bw) ? Wp[(r0 + r) * n + j0 + c] : 0.f;
  }
  __syncthreads();
  for (int c = t; c < SB; c += RT) rdiag[c] = (c < bw) ? 1.0f / UT[c * LDU + c] : 0.f;
  __syncthreads();

  const float maxq = (float)((1 << bits) - 1);
  float s = 1.f, z = 0.f, loss = 0.f;
  const int nsb = (bw + SS - 1) / SS;
  for (int sb = 0; sb < nsb; ++sb) {
    const int c0 = sb * SS;
    if (c0 % group == 0) {
      const int cend = min(c0 + group, bw);
      float xmin = 0.f, xmax = 0.f;
      for (int c = c0; c < cend; ++c) {
        const float x = vals[c * LDV + t];
        xmin = fminf(xmin, x);
        xmax = fmaxf(xmax, x);
      }
      if (xmin == 0.f && xmax == 0.f) { xmin = -1.f; xmax = 1.f; }
      s = __fdiv_rn(xmax - xmin, maxq);
      z = rintf(__fdiv_rn(-xmin, s));
      if (row < m) {
        const int64_t g = (j0 + c0) / group;
        scale[row * ngroups + g] = s;
        zero[row * ngroups + g] = (uint8_t)z;
      }
    }
    float v[SS], e[SS];
#pragma unroll
    for (int k = 0; k < SS; ++k) v[k] = vals[(c0 + k) * LDV + t];
#pragma unroll
    for (int i = 0; i < SS; ++i) {
      const int c = c0 + i;
      float q = rintf(__fdiv_rn(v[i], s)) + z;
      q = fminf(fmaxf(q, 0.f), maxq);
      const float d = v[i] - s * (q - z);
      const float ei = d * rdiag[c];
      e[i] = ei;
      loss = fmaf(ei, ei, loss);
      cs[c * LDC + t] = (uint8_t)q;
#pragma unroll
      for (int k = i + 1; k < SS; ++k) v[k] = fmaf(-ei, UT[(c0 + k) * LDU + c], v[k]);
    }
#pragma unroll
    for (int k = 0; k < SS; ++k) vals[(c0 + k) * LDV + t] = e[k];
    for (int c = c0 + SS; c < bw; ++c) {
      float acc = vals[c * LDV + t];
      const float4* u4 = reinterpret_cast<const float4*>(UT + c * LDU + c0);
#pragma unroll
      for (int q4 = 0; q4 < SS / 4; ++q4) {
        const float4 u = u4[q4];
        acc = fmaf(-e[4 * q4 + 0], u.x, acc);
        acc = fmaf(-e[4 * q4 + 1], u.y, acc);
        acc = fmaf(-e[4 * q4 + 2], u.z, acc);
        acc = fmaf(-e[4 * q4 + 3], u.w, acc);
      }
      vals[c * LDV + t] = acc;
    }
  }
  if (row < m && loss_row != nullptr) loss_row[row] += loss;
  __syncthreads();
  for (int e2 = t; e2 < RT * SB; e2 += RT) {
    const int r = e2 / SB, c = e2 % SB;
    if (r0 + r < m && c < bw) {
      Err[(r0 + r) * ldE + c] = vals[c * LDV + r];
      codes[(r0 + r) * n + j0 + c] = cs[c * LDC + r];
    }
  }
}

bool g_attr_set = false;

}  // namespace

gptq_status launch_sweep(const float* Wp, int64_t m, int64_t n, int64_t j0,
                         int bw, const float* U, int bits, int group,
                         int64_t ngroups, uint8_t* codes, float* scale,
                         uint8_t* zero, float* Err, int ldE, float* loss_row,
                         cudaStream_t s) {
  constexpr size_t smem = SweepSmem<SWEEP_RT>::bytes;
  if (!g_attr_set) {
    GPTQ_CUDA(cudaFuncSetAttribute(sweep_kernel<SWEEP_RT>,
              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    g_attr_set = true;
  }
  const unsigned grid = (unsigned)ceil_div(m, SWEEP_RT);
  GPTQ_LAUNCH(KK_SWEEP, s, sweep_kernel<SWEEP_RT>, grid, SWEEP_RT, smem, Wp, m,
              n, j0, bw, U, bits, group, ngroups, codes, scale, zero, Err, ldE,
              loss_row);
  return GPTQ_OK;
}

}  // namespace gptq
