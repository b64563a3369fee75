// CHMC frontend, step 1: the low-rank part along the activation cone.
//
// "Warum Geometrie Gewichte nicht komprimiert", section "Methodik. Was ist
// CHMC", Schritt 1: damped activation energies c_j = (1/n)·Σ_t x²_tj +
// λ·mean(c); W̃ = W·diag(√c); a randomized SVD of W̃ with rank r and a few
// power iterations; W_lr = (U·S)·Vᵀ·diag(1/√c).  Schritt 2 quantizes the
// residual R = W − W_lr (gptq_quantize_rowgroups).
//
// The randomized SVD is the randomized subspace iteration (Halko, Martinsson,
// Tropp 2011, Algorithm 4.4): Q = orth(W̃·Ω), then per power iteration
// Q = orth(W̃ᵀ·Q), Q = orth(W̃·Q).  Since the sketch has exactly r columns,
// (U·S)·Vᵀ·diag(1/√c) = Q·Qᵀ·W, so the library returns the factors Q (o × r,
// orthonormal) and P = Qᵀ·W (r × i) with W_lr = Q·P, and the residual.
//
// Everything runs in float64 on the CUDA cores: every product is a thin one
// (r ≤ 32 columns), bound by reading W, and the answer has to match a float64
// oracle to well below the quantizer's resolution.
//   * row products   Y = W̃·X   one warp per row of W, lanes along the row;
//   * column products Z = W̃ᵀ·Q  one thread per column of W and CTAs over
//                     128-row chunks; the chunks' partial sums are added in a
//                     fixed order (results are deterministic);
//   * orth           CholeskyQR2: the Gram matrix (partial Grams per 128-row
//                     chunk, added in a fixed order), its Cholesky factor by one
//                     warp, Q = Y·R⁻¹, twice.  A pivot that is not positive
//                     (a direction the sketch does not reach, e.g. rank(W) < r)
//                     drops its column, which leaves Q·Qᵀ a projector onto the
//                     span found.

#include <cmath>
#include <cuda_bf16.h>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int CHMC_MAX_RANK = GPTQ_CHMC_MAX_RANK;
constexpr int CHUNK = 128;            // rows per partial sum

template <typename T> __device__ __forceinline__ double to_f64(T x);
template <> __device__ __forceinline__ double to_f64<float>(float x) { return (double)x; }
template <> __device__ __forceinline__ double to_f64<__nv_bfloat16>(__nv_bfloat16 x) {
  return (double)__bfloat162float(x);
}

// √c_j with c_j = H_jj/(2·tokens) + λ·mean_j'(H_j'j'/(2·tokens)); one CTA.
__global__ void __launch_bounds__(1024)
chmc_energy_kernel(const float* __restrict__ H, int64_t n, int64_t tokens, double lam,
                   double* __restrict__ sq, int32_t* info) {
  __shared__ double red[1024];
  const int t = threadIdx.x;
  const double inv2t = 1.0 / (2.0 * (double)tokens);
  double acc = 0.0;
  for (int64_t j = t; j < n; j += 1024) acc += (double)H[j * n + j] * inv2t;
  red[t] = acc;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if (t < s) red[t] += red[t + s];
    __syncthreads();
  }
  const double mean = red[0] / (double)n;
  for (int64_t j = t; j < n; j += 1024) {
    const double c = (double)H[j * n + j] * inv2t + lam * mean;
    if (!(c > 0.0) || !isfinite(c)) {
      report(info, GPTQ_ERR_INVALID_ARG, j);
      sq[j] = 1.0;
    } else {
      sq[j] = sqrt(c);
    }
  }
}

__global__ void chmc_to_f64_kernel(const float* __restrict__ x, int64_t count,
                                   double* __restrict__ y) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e < count) y[e] = (double)x[e];
}

// Y[row][k] = Σ_j W[row][j]·(sq ? sq[j] : 1)·X[j][k]: one warp per row, lanes
// along the row (coalesced), then a fixed shuffle tree per k.
template <typename T>
__global__ void __launch_bounds__(256)
chmc_rowprod_kernel(const T* __restrict__ W, int64_t o, int64_t i,
                    const double* __restrict__ sq, const double* __restrict__ X, int r,
                    double* __restrict__ Y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= o) return;
  double acc[CHMC_MAX_RANK];
#pragma unroll
  for (int k = 0; k < CHMC_MAX_RANK; ++k) acc[k] = 0.0;
  for (int64_t j = lane; j < i; j += 32) {
    double w = to_f64(W[row * i + j]);
    if (sq) w *= sq[j];
    const double* x = X + j * r;
#pragma unroll
    for (int k = 0; k < CHMC_MAX_RANK; ++k)
      if (k < r) acc[k] = fma(w, x[k], acc[k]);
  }
#pragma unroll
  for (int k = 0; k < CHMC_MAX_RANK; ++k) {
    if (k < r) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < CHMC_MAX_RANK; ++k)
      if (k < r) Y[row * r + k] = acc[k];
  }
}

// Zp[chunk][j][k] = Σ_{row in chunk} W[row][j]·Qo[row][k]: one thread per
// column of W, one CTA per (128 columns, 128-row chunk).
template <typename T>
__global__ void __launch_bounds__(128)
chmc_colprod_kernel(const T* __restrict__ W, int64_t o, int64_t i,
                    const double* __restrict__ Qo, int r, double* __restrict__ Zp) {
  __shared__ double qs[CHUNK * CHMC_MAX_RANK];
  const int64_t j = (int64_t)blockIdx.x * 128 + threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * CHUNK;
  const int rows = (int)((o - r0 < CHUNK) ? (o - r0) : CHUNK);
  for (int e = threadIdx.x; e < rows * r; e += 128) qs[e] = Qo[r0 * r + e];
  __syncthreads();
  if (j >= i) return;
  double acc[CHMC_MAX_RANK];
#pragma unroll
  for (int k = 0; k < CHMC_MAX_RANK; ++k) acc[k] = 0.0;
  for (int rr = 0; rr < rows; ++rr) {
    const double w = to_f64(W[(r0 + rr) * i + j]);
    const double* q = qs + rr * r;
#pragma unroll
    for (int k = 0; k < CHMC_MAX_RANK; ++k)
      if (k < r) acc[k] = fma(w, q[k], acc[k]);
  }
  double* out = Zp + ((int64_t)blockIdx.y * i + j) * r;
#pragma unroll
  for (int k = 0; k < CHMC_MAX_RANK; ++k)
    if (k < r) out[k] = acc[k];
}

// Z[j][k] = (sq ? sq[j] : 1)·Σ_chunk Zp[chunk][j][k], chunks in order.
__global__ void chmc_colreduce_kernel(const double* __restrict__ Zp, int nchunk, int64_t i,
                                      int r, const double* __restrict__ sq,
                                      double* __restrict__ Z) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= i * r) return;
  double acc = 0.0;
  for (int c = 0; c < nchunk; ++c) acc += Zp[(int64_t)c * i * r + e];
  Z[e] = sq ? acc * sq[e / r] : acc;
}

// Gp[chunk][a][b] = Σ_{row in chunk} Y[row][a]·Y[row][b], a ≤ b (upper half).
__global__ void __launch_bounds__(1024)
chmc_gram_kernel(const double* __restrict__ Y, int64_t rows, int r, double* __restrict__ Gp) {
  __shared__ double ys[CHUNK * CHMC_MAX_RANK];
  const int64_t r0 = (int64_t)blockIdx.x * CHUNK;
  const int nr = (int)((rows - r0 < CHUNK) ? (rows - r0) : CHUNK);
  for (int e = threadIdx.x; e < nr * r; e += 1024) ys[e] = Y[r0 * r + e];
  __syncthreads();
  const int a = threadIdx.x / CHMC_MAX_RANK, b = threadIdx.x % CHMC_MAX_RANK;
  if (a >= r || b >= r || b < a) return;
  double acc = 0.0;
  for (int rr = 0; rr < nr; ++rr) acc = fma(ys[rr * r + a], ys[rr * r + b], acc);
  Gp[((int64_t)blockIdx.x * r + a) * r + b] = acc;
}

// G = Σ_chunk Gp (in order); G = LLᵀ by one warp (lane j owns row j of L),
// dropping a column whose pivot is not positive; Rinv = (L⁻¹)ᵀ, upper.
__global__ void __launch_bounds__(32)
chmc_chol_kernel(const double* __restrict__ Gp, int nchunk, int r, double* __restrict__ Rinv) {
  __shared__ double G[CHMC_MAX_RANK][CHMC_MAX_RANK + 1];
  __shared__ double L[CHMC_MAX_RANK][CHMC_MAX_RANK + 1];
  const int lane = threadIdx.x;
  if (lane < r) {
    for (int b = 0; b < r; ++b) {
      double acc = 0.0;
      const int a0 = lane < b ? lane : b, b0 = lane < b ? b : lane;
      for (int c = 0; c < nchunk; ++c) acc += Gp[((int64_t)c * r + a0) * r + b0];
      G[lane][b] = acc;
      L[lane][b] = 0.0;
    }
  }
  __syncwarp();
  double tr = 0.0;
  for (int k = 0; k < r; ++k) tr += G[k][k];
  const double floor_piv = 1e-28 * (tr > 0.0 ? tr : 1.0);
  // right-looking Cholesky: lane j updates row j
  for (int k = 0; k < r; ++k) {
    const double piv = G[k][k];
    const bool keep = piv > floor_piv;
    const double d = keep ? sqrt(piv) : 0.0;
    __syncwarp();
    if (lane >= k && lane < r) L[lane][k] = keep ? G[lane][k] / d : 0.0;
    __syncwarp();
    // trailing update of the lower triangle, row by row (only it is read)
    if (lane > k && lane < r) {
      for (int l = k + 1; l <= lane; ++l) G[lane][l] -= L[lane][k] * L[l][k];
    }
    __syncwarp();
  }
  // column j of L⁻¹ by forward substitution (lane j); dropped pivots give 0
  if (lane < r) {
    double x[CHMC_MAX_RANK];
#pragma unroll
    for (int i = 0; i < CHMC_MAX_RANK; ++i) x[i] = 0.0;
    for (int i = lane; i < r; ++i) {
      double s = (i == lane) ? 1.0 : 0.0;
      for (int m = lane; m < i; ++m) s -= L[i][m] * x[m];
      x[i] = (L[i][i] != 0.0) ? s / L[i][i] : 0.0;
    }
    // Rinv[a][b] = (L⁻¹)[b][a]: row `lane` of Rinv is column `lane` of L⁻¹
    for (int i = 0; i < r; ++i) Rinv[lane * r + i] = (i >= lane) ? x[i] : 0.0;
  }
}

// Q[row][k] = Σ_{l ≤ k} Y[row][l]·Rinv[l][k]  (Y·R⁻¹, R = Lᵀ upper).
__global__ void chmc_apply_kernel(const double* __restrict__ Y, int64_t rows, int r,
                                  const double* __restrict__ Rinv, double* __restrict__ Q) {
  __shared__ double R[CHMC_MAX_RANK * CHMC_MAX_RANK];
  for (int e = threadIdx.x; e < r * r; e += 256) R[e] = Rinv[e];
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (row >= rows) return;
  double y[CHMC_MAX_RANK];
#pragma unroll
  for (int k = 0; k < CHMC_MAX_RANK; ++k) y[k] = (k < r) ? Y[row * r + k] : 0.0;
#pragma unroll
  for (int k = 0; k < CHMC_MAX_RANK; ++k) {
    if (k < r) {
      double acc = 0.0;
#pragma unroll
      for (int l = 0; l < CHMC_MAX_RANK; ++l)
        if (l <= k) acc = fma(y[l], R[l * r + k], acc);
      Q[row * r + k] = acc;
    }
  }
}

// Outputs: Qf = Q (o × r), Pf = Pᵀ stored r × i, Res = W − Q·P (o × i); all float32.
template <typename T>
__global__ void __launch_bounds__(256)
chmc_residual_kernel(const T* __restrict__ W, int64_t o, int64_t i,
                     const double* __restrict__ Q, const double* __restrict__ P, int r,
                     float* __restrict__ Res) {
  const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const int64_t row = blockIdx.y;
  if (j >= i) return;
  double acc = to_f64(W[row * i + j]);
  for (int k = 0; k < r; ++k) acc = fma(-Q[row * r + k], P[j * r + k], acc);
  Res[row * i + j] = (float)acc;
}

__global__ void chmc_factors_kernel(const double* __restrict__ Q, const double* __restrict__ P,
                                    int64_t o, int64_t i, int r, float* __restrict__ Qf,
                                    float* __restrict__ Pf) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (Qf && e < o * r) Qf[e] = (float)Q[e];
  if (Pf && e < i * r) {
    const int64_t j = e / r, k = e % r;
    Pf[k * i + j] = (float)P[e];
  }
}

template <typename T>
__global__ void chmc_copy_kernel(const T* __restrict__ W, int64_t count, float* __restrict__ Res) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e < count) Res[e] = (float)to_f64(W[e]);
}

size_t chmc_layout(int64_t o, int64_t i, int r, char* base, double** sq, double** om,
                   double** Y, double** Q, double** Z, double** Qi, double** Zp, double** Gp,
                   double** Rinv, double** P) {
  const int64_t nco = ceil_div(o, CHUNK), nci = ceil_div(i, CHUNK);
  const int64_t nch = nco > nci ? nco : nci;
  size_t off = 0;
  auto take = [&](size_t bytes, double** p) {
    off = (off + 255) / 256 * 256;
    if (base && p) *p = reinterpret_cast<double*>(base + off);
    off += bytes;
  };
  take(sizeof(double) * i, sq);
  take(sizeof(double) * i * r, om);
  take(sizeof(double) * o * r, Y);
  take(sizeof(double) * o * r, Q);
  take(sizeof(double) * i * r, Z);
  take(sizeof(double) * i * r, Qi);
  take(sizeof(double) * nco * i * r, Zp);
  take(sizeof(double) * nch * r * r, Gp);
  take(sizeof(double) * r * r, Rinv);
  take(sizeof(double) * i * r, P);
  return (off + 255) / 256 * 256;
}

// CholeskyQR2 of the rows × r matrix Y into Q: Y ← Y·R₁⁻¹ in place (each
// thread reads its whole row before writing it), then Q = Y·R₂⁻¹.
gptq_status orth_rows(double* Y, int64_t rows, int r, double* Q, double* Gp, double* Rinv,
                      cudaStream_t s) {
  const unsigned nch = (unsigned)ceil_div(rows, CHUNK);
  const unsigned ga = (unsigned)ceil_div(rows, 256);
  for (int pass = 0; pass < 2; ++pass) {
    GPTQ_LAUNCH(KK_CHMC, s, chmc_gram_kernel, nch, 1024, 0, Y, rows, r, Gp);
    GPTQ_LAUNCH(KK_CHMC, s, chmc_chol_kernel, 1, 32, 0, Gp, (int)nch, r, Rinv);
    GPTQ_LAUNCH(KK_CHMC, s, chmc_apply_kernel, ga, 256, 0, Y, rows, r, Rinv,
                pass == 0 ? Y : Q);
  }
  return GPTQ_OK;
}

template <typename T>
gptq_status lowrank_impl(const T* W, int64_t o, int64_t i, const float* H, int64_t tokens,
                         double lam, const float* Omega, int r, int niter, float* Qf,
                         float* Pf, float* Res, int32_t* info, char* ws, cudaStream_t s) {
  double *sq, *om, *Y, *Q, *Z, *Qi, *Zp, *Gp, *Rinv, *P;
  chmc_layout(o, i, r, ws, &sq, &om, &Y, &Q, &Z, &Qi, &Zp, &Gp, &Rinv, &P);
  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  if (r == 0) {
    GPTQ_LAUNCH(KK_CHMC, s, chmc_copy_kernel<T>, (unsigned)ceil_div(o * i, 256), 256, 0, W,
                o * i, Res);
    return GPTQ_OK;
  }
  GPTQ_LAUNCH(KK_CHMC, s, chmc_energy_kernel, 1, 1024, 0, H, i, tokens, lam, sq, info);
  GPTQ_LAUNCH(KK_CHMC, s, chmc_to_f64_kernel, (unsigned)ceil_div(i * r, 256), 256, 0, Omega,
              i * r, om);
  const unsigned grow = (unsigned)ceil_div(o, 8);
  const dim3 gcol((unsigned)ceil_div(i, 128), (unsigned)ceil_div(o, CHUNK));
  const int nco = (int)ceil_div(o, CHUNK);
  const unsigned gred = (unsigned)ceil_div(i * r, 256);
  // Y = W̃·Ω, Q = orth(Y)
  GPTQ_LAUNCH(KK_CHMC, s, chmc_rowprod_kernel<T>, grow, 256, 0, W, o, i, sq, om, r, Y);
  gptq_status st = orth_rows(Y, o, r, Q, Gp, Rinv, s);
  if (st != GPTQ_OK) return st;
  for (int it = 0; it < niter; ++it) {
    // Qi = orth(W̃ᵀ·Q) with W̃ᵀ·Q = diag(√c)·Wᵀ·Q
    GPTQ_LAUNCH(KK_CHMC, s, chmc_colprod_kernel<T>, gcol, 128, 0, W, o, i, Q, r, Zp);
    GPTQ_LAUNCH(KK_CHMC, s, chmc_colreduce_kernel, gred, 256, 0, Zp, nco, i, r, sq, Z);
    st = orth_rows(Z, i, r, Qi, Gp, Rinv, s);
    if (st != GPTQ_OK) return st;
    // Q = orth(W̃·Qi)
    GPTQ_LAUNCH(KK_CHMC, s, chmc_rowprod_kernel<T>, grow, 256, 0, W, o, i, sq, Qi, r, Y);
    st = orth_rows(Y, o, r, Q, Gp, Rinv, s);
    if (st != GPTQ_OK) return st;
  }
  // P = Qᵀ·W (stored i × r), then the residual W − Q·P and the factors
  GPTQ_LAUNCH(KK_CHMC, s, chmc_colprod_kernel<T>, gcol, 128, 0, W, o, i, Q, r, Zp);
  GPTQ_LAUNCH(KK_CHMC, s, chmc_colreduce_kernel, gred, 256, 0, Zp, nco, i, r,
              (const double*)nullptr, P);
  const dim3 gres((unsigned)ceil_div(i, 256), (unsigned)o);
  GPTQ_LAUNCH(KK_CHMC, s, chmc_residual_kernel<T>, gres, 256, 0, W, o, i, Q, P, r, Res);
  const int64_t nf = (o > i ? o : i) * r;
  if (Qf || Pf)
    GPTQ_LAUNCH(KK_CHMC, s, chmc_factors_kernel, (unsigned)ceil_div(nf, 256), 256, 0, Q, P, o,
                i, r, Qf, Pf);
  return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_chmc_rank(int64_t o, int64_t i, int bits, int gs, double bpw_target) {
  if (o < 1 || i < 1 || bits < 1 || gs < 1) return 0;
  const double num = bpw_target * (double)o * (double)i - (double)bits * (double)o * (double)i -
                     16.0 * (double)ceil_div(o, gs) * (double)i;
  const double r = std::floor(num / (16.0 * (double)(o + i)));
  if (!(r > 0.0)) return 0;
  const double cap = (double)(o < i ? o : i);
  return (int)(r < cap ? r : cap);
}

extern "C" size_t gptq_chmc_workspace_bytes(int64_t o, int64_t i, int r) {
  if (o < 1 || i < 1 || r < 0 || r > CHMC_MAX_RANK) return 0;
  return chmc_layout(o, i, r > 0 ? r : 1, nullptr, nullptr, nullptr, nullptr, nullptr,
                     nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
}

extern "C" gptq_status gptq_chmc_lowrank(const void* W, int w_dtype, int64_t o, int64_t i,
                                         const float* H, int64_t tokens, double lam,
                                         const float* Omega, int r, int niter, float* Q,
                                         float* P, float* R, int32_t* info, void* ws,
                                         size_t ws_bytes, void* stream) {
  if (!W || !R || !info || !ws || (r > 0 && (!H || !Omega)))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_chmc_lowrank: null pointer");
  if (o < 1 || i < 1 || o > 65535 || i > ((int64_t)1 << 20) || tokens < 1)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_chmc_lowrank: o=%lld i=%lld tokens=%lld",
                (long long)o, (long long)i, (long long)tokens);
  if (r < 0 || r > CHMC_MAX_RANK || r > o || r > i || niter < 0 || niter > 64)
    return fail(GPTQ_ERR_UNSUPPORTED, "gptq_chmc_lowrank: rank %d (0..%d, at most min(o, i)), "
                "niter %d (0..64)", r, CHMC_MAX_RANK, niter);
  if (!(lam >= 0.0) || !std::isfinite(lam))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_chmc_lowrank: lambda");
  if (w_dtype != GPTQ_DTYPE_F32 && w_dtype != GPTQ_DTYPE_BF16)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_chmc_lowrank: w_dtype=%d", w_dtype);
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_chmc_lowrank: workspace not 256-byte aligned");
  const size_t need = gptq_chmc_workspace_bytes(o, i, r);
  if (ws_bytes < need)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_chmc_lowrank: workspace %zu < %zu bytes", ws_bytes,
                need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  if (w_dtype == GPTQ_DTYPE_BF16)
    return lowrank_impl(static_cast<const __nv_bfloat16*>(W), o, i, H, tokens, lam, Omega, r,
                        niter, Q, P, R, info, base, s);
  return lowrank_impl(static_cast<const float*>(W), o, i, H, tokens, lam, Omega, r, niter, Q,
                      P, R, info, base, s);
}
