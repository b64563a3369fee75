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
// Rows are independent (U is shared), so one thread owns one row and a CTA
// owns 128 rows.  The block's U panel is pre-transposed once per call
// (panel_kernel: UT[c][i] = U[j0+i][j0+c] plus 1/U_jj) so that each CTA
// fetches it with a single bulk (TMA) copy into shared memory while its
// threads load their rows.  The block is walked in sub-blocks of 32 columns
// held in registers: the 32 dependent column steps run fully unrolled, then
// the sub-block's 32 errors update the block's later columns (four columns
// at a time for instruction-level parallelism) with vectorised panel reads.
//
// Scale and zero: min-max over the group's current values at the group's
// first column, the range always containing 0; decisions in IEEE float32
// (correctly rounded division and rint, no fast-math).
//
// The block's errors leave as a TF32 split (Ehi = TF32(e), Elo = e − Ehi) for
// the tensor-core trailing update.
#include "kernels.cuh"
#include "sm100.cuh"

namespace gptq {
namespace {

constexpr int SB = 128;       // largest block width
constexpr int SS = 32;        // register sub-block
constexpr int LDU = SB + 4;   // transposed-panel row stride (floats; 16-byte rows)
constexpr int RT = 128;       // rows (threads) per CTA
constexpr int LDV = SB + 1;   // row-major values, odd stride: conflict-free columns
constexpr int LDB = SB + 4;   // bytes per staged code row
constexpr size_t PANEL_FLOATS = (size_t)SB * LDU + SB;
constexpr size_t SMEM_BYTES = PANEL_BYTES + sizeof(float) * RT * LDV + (size_t)RT * LDB + 16;
static_assert(PANEL_BYTES == PANEL_FLOATS * sizeof(float), "panel layout");
static_assert(PANEL_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");

// Panel of block b: UT[c][i] = U[j0+i][j0+c] (zero outside the block), and
// rdiag[c] = 1/U[j0+c][j0+c].  32×32 tiles through shared memory.
__global__ void __launch_bounds__(256)
panel_kernel(const float* __restrict__ U, int64_t n, int block,
             float* __restrict__ panels) {
  __shared__ float tile[32][33];
  const int b = blockIdx.x, ci = blockIdx.y, ii = blockIdx.z;
  const int64_t j0 = (int64_t)b * block;
  const int bw = (int)((n - j0 < block) ? (n - j0) : block);
  float* P = panels + (size_t)b * PANEL_FLOATS;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = ii * 32 + ty + 8 * k, c = ci * 32 + tx;
    tile[ty + 8 * k][tx] = (i < bw && c < bw) ? U[(j0 + i) * n + j0 + c] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = ci * 32 + ty + 8 * k, i = ii * 32 + tx;
    P[c * LDU + i] = tile[tx][ty + 8 * k];
  }
  if (ii == 3 && threadIdx.x < 32 * (LDU - SB)) {       // zero the row padding
    const int c = ci * 32 + (threadIdx.x >> 2), p = SB + (threadIdx.x & 3);
    P[c * LDU + p] = 0.f;
  }
  if (ii == ci && ty == 0) {
    const int c = ci * 32 + tx;
    P[SB * LDU + c] = (c < bw) ? 1.0f / U[(j0 + c) * n + j0 + c] : 0.f;
  }
}

__global__ void __launch_bounds__(RT)
sweep_kernel(const float* __restrict__ Wp, int64_t m, int64_t n, int64_t j0, int bw,
             const float* __restrict__ panel, int bits, int group, int64_t ngroups,
             uint8_t* __restrict__ codes, float* __restrict__ scale,
             uint8_t* __restrict__ zero, float* __restrict__ Ehi,
             float* __restrict__ Elo, float* __restrict__ loss_row, int32_t* info) {
  extern __shared__ __align__(128) unsigned char smraw[];
  float* UT = reinterpret_cast<float*>(smraw);
  const float* rdiag = UT + SB * LDU;
  float* vals = reinterpret_cast<float*>(smraw + PANEL_BYTES);
  uint8_t* cs = reinterpret_cast<uint8_t*>(vals + RT * LDV);
  uint64_t* bar = reinterpret_cast<uint64_t*>(cs + RT * LDB);

  const int t = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * RT;
  const int64_t row = r0 + t;

  if (t == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (t == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)PANEL_BYTES);
    bulk_g2s(UT, panel, (uint32_t)PANEL_BYTES, bar);
  }

  // this thread's row of the block → vals (row-major, odd stride)
  float* vr = vals + t * LDV;
  if (row < m) {
    const float* src = Wp + row * n + j0;
    if ((n & 3) == 0 && bw == SB) {
      const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
      for (int b4 = 0; b4 < SB / 4; b4 += 8) {
        float4 buf[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) buf[k] = s4[b4 + k];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          vr[4 * (b4 + k) + 0] = buf[k].x;
          vr[4 * (b4 + k) + 1] = buf[k].y;
          vr[4 * (b4 + k) + 2] = buf[k].z;
          vr[4 * (b4 + k) + 3] = buf[k].w;
        }
      }
    } else {
      for (int c = 0; c < SB; ++c) vr[c] = (c < bw) ? src[c] : 0.f;
    }
  } else {
    for (int c = 0; c < SB; ++c) vr[c] = 0.f;
  }

  if (!mbar_wait_bounded(bar, 0)) {
    report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
    if (t == 0) mbar_wait_bounded(bar, 0);   // let our own copy land first
    return;
  }

  const float maxq = (float)((1 << bits) - 1);
  float s = 1.f, z = 0.f, loss = 0.f;
  uint8_t* cr = cs + t * LDB;
  const int nsb = (bw + SS - 1) / SS;
  for (int sb = 0; sb < nsb; ++sb) {
    const int c0 = sb * SS;
    if (c0 % group == 0) {
      const int cend = min(c0 + group, bw);
      float xmin = 0.f, xmax = 0.f;
      for (int c = c0; c < cend; ++c) {
        const float x = vr[c];
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
    for (int k = 0; k < SS; ++k) v[k] = vr[c0 + k];
#pragma unroll
    for (int i = 0; i < SS; ++i) {
      const int c = c0 + i;
      float q = rintf(__fdiv_rn(v[i], s)) + z;
      q = fminf(fmaxf(q, 0.f), maxq);
      const float ei = (v[i] - s * (q - z)) * rdiag[c];
      e[i] = ei;
      loss = fmaf(ei, ei, loss);
      cr[c] = (uint8_t)q;
#pragma unroll
      for (int k = i + 1; k < SS; ++k) v[k] = fmaf(-ei, UT[(c0 + k) * LDU + c], v[k]);
    }
#pragma unroll
    for (int k = 0; k < SS; ++k) vr[c0 + k] = e[k];
    for (int c = c0 + SS; c < bw; c += 4) {
      float a0 = vr[c], a1 = vr[c + 1], a2 = vr[c + 2], a3 = vr[c + 3];
      const float4* u0 = reinterpret_cast<const float4*>(UT + (c + 0) * LDU + c0);
      const float4* u1 = reinterpret_cast<const float4*>(UT + (c + 1) * LDU + c0);
      const float4* u2 = reinterpret_cast<const float4*>(UT + (c + 2) * LDU + c0);
      const float4* u3 = reinterpret_cast<const float4*>(UT + (c + 3) * LDU + c0);
#pragma unroll
      for (int q4 = 0; q4 < SS / 4; ++q4) {
        const float4 x0 = u0[q4], x1 = u1[q4], x2 = u2[q4], x3 = u3[q4];
        const float e0 = e[4 * q4], e1 = e[4 * q4 + 1], e2 = e[4 * q4 + 2], e3 = e[4 * q4 + 3];
        a0 = fmaf(-e0, x0.x, a0); a1 = fmaf(-e0, x1.x, a1);
        a2 = fmaf(-e0, x2.x, a2); a3 = fmaf(-e0, x3.x, a3);
        a0 = fmaf(-e1, x0.y, a0); a1 = fmaf(-e1, x1.y, a1);
        a2 = fmaf(-e1, x2.y, a2); a3 = fmaf(-e1, x3.y, a3);
        a0 = fmaf(-e2, x0.z, a0); a1 = fmaf(-e2, x1.z, a1);
        a2 = fmaf(-e2, x2.z, a2); a3 = fmaf(-e2, x3.z, a3);
        a0 = fmaf(-e3, x0.w, a0); a1 = fmaf(-e3, x1.w, a1);
        a2 = fmaf(-e3, x2.w, a2); a3 = fmaf(-e3, x3.w, a3);
      }
      vr[c] = a0; vr[c + 1] = a1; vr[c + 2] = a2; vr[c + 3] = a3;
    }
  }
  if (row < m && loss_row != nullptr) loss_row[row] += loss;
  __syncthreads();

  // errors and codes out, one warp per row, coalesced
  const int lane = t & 31, warp = t >> 5;
  for (int rr = warp; rr < RT; rr += RT / 32) {
    const int64_t r = r0 + rr;
    if (r >= m) break;
#pragma unroll
    for (int it = 0; it < SB / 32; ++it) {
      const int c = lane + 32 * it;
      if (c < bw) {
        const float e = vals[rr * LDV + c];
        const float h = to_tf32(e);
        Ehi[r * SB + c] = h;
        Elo[r * SB + c] = e - h;
        codes[r * n + j0 + c] = cs[rr * LDB + c];
      }
    }
  }
}

bool g_attr_set = false;

}  // namespace

size_t panel_workspace_bytes(int64_t n, int block) {
  return (size_t)ceil_div(n, block) * PANEL_BYTES;
}

gptq_status launch_panels(const float* U, int64_t n, int block, float* panels,
                          cudaStream_t s) {
  const dim3 grid((unsigned)ceil_div(n, block), SB / 32, SB / 32);
  GPTQ_LAUNCH(KK_INGEST, s, panel_kernel, grid, 256, 0, U, n, block, panels);
  return GPTQ_OK;
}

gptq_status launch_sweep(const float* Wp, int64_t m, int64_t n, int64_t j0, int bw,
                         const float* panel, int bits, int group, int64_t ngroups,
                         uint8_t* codes, float* scale, uint8_t* zero, float* Ehi,
                         float* Elo, float* loss_row, int32_t* info, cudaStream_t s) {
  if (!g_attr_set) {
    GPTQ_CUDA(cudaFuncSetAttribute(sweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)SMEM_BYTES));
    g_attr_set = true;
  }
  const unsigned grid = (unsigned)ceil_div(m, RT);
  GPTQ_LAUNCH(KK_SWEEP, s, sweep_kernel, grid, RT, SMEM_BYTES, Wp, m, n, j0, bw, panel,
              bits, group, ngroups, codes, scale, zero, Ehi, Elo, loss_row, info);
  return GPTQ_OK;
}

}  // namespace gptq
