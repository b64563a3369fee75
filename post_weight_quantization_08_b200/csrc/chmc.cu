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
template <typename T, int RMAX>
__global__ void __launch_bounds__(256)
chmc_rowprod_kernel(const T* __restrict__ W, int64_t o, int64_t i,
                    const double* __restrict__ sq, const double* __restrict__ X, int r,
                    double* __restrict__ Y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= o) return;
  double acc[RMAX];
#pragma unroll
  for (int k = 0; k < RMAX; ++k) acc[k] = 0.0;
  for (int64_t j0 = lane; j0 < i; j0 += 128) {
    double w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + 32 * u;
      w[u] = (j < i) ? to_f64(W[row * i + j]) * (sq ? sq[j] : 1.0) : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = j0 + 32 * u;
      if (j < i) {
        const double* x = X + j * r;
#pragma unroll
        for (int k = 0; k < RMAX; ++k)
          if (k < r) acc[k] = fma(w[u], x[k], acc[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < RMAX; ++k) {
    if (k < r) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < RMAX; ++k)
      if (k < r) Y[row * r + k] = acc[k];
  }
}

// Zp[chunk][j][k] = Σ_{row in chunk} W[row][j]·Qo[row][k]: one CTA per (64
// columns, 128-row chunk); thread (column, slice) sums 32 rows with eight
// loads in flight, and the four slices are added in a fixed order.
constexpr int CP_COLS = 64, CP_SLICES = 4;
template <typename T, int RMAX>
__global__ void __launch_bounds__(256)
chmc_colprod_kernel(const T* __restrict__ W, int64_t o, int64_t i,
                    const double* __restrict__ Qo, int r, double* __restrict__ Zp) {
  __shared__ double qs[CHUNK * CHMC_MAX_RANK];   // Q rows, then the slices' sums
  static_assert(2 * CP_COLS * CHMC_MAX_RANK <= CHUNK * CHMC_MAX_RANK, "reduction space");
  const int tid = threadIdx.x, jc = tid % CP_COLS, sl = tid / CP_COLS;
  const int64_t j = (int64_t)blockIdx.x * CP_COLS + jc;
  const int64_t r0 = (int64_t)blockIdx.y * CHUNK;
  const int rows = (int)((o - r0 < CHUNK) ? (o - r0) : CHUNK);
  for (int e = tid; e < rows * r; e += 256) qs[e] = Qo[r0 * r + e];
  __syncthreads();
  double acc[RMAX];
#pragma unroll
  for (int k = 0; k < RMAX; ++k) acc[k] = 0.0;
  const int rs = sl * (CHUNK / CP_SLICES);
  const int re = (rs + CHUNK / CP_SLICES < rows) ? rs + CHUNK / CP_SLICES : rows;
  if (j < i) {
    for (int rr0 = rs; rr0 < re; rr0 += 8) {
      double w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        w[u] = (rr0 + u < re) ? to_f64(W[(r0 + rr0 + u) * i + j]) : 0.0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (rr0 + u < re) {
          const double* q = qs + (rr0 + u) * r;
#pragma unroll
          for (int k = 0; k < RMAX; ++k)
            if (k < r) acc[k] = fma(w[u], q[k], acc[k]);
        }
      }
    }
  }
  // ((slice 0 + slice 2) + (slice 1 + slice 3)) through the Q staging space
  double* red = qs;                                  // [2][CP_COLS][r]
  __syncthreads();
  if (sl >= 2) {
#pragma unroll
    for (int k = 0; k < RMAX; ++k)
      if (k < r) red[((sl - 2) * CP_COLS + jc) * r + k] = acc[k];
  }
  __syncthreads();
  if (sl < 2) {
#pragma unroll
    for (int k = 0; k < RMAX; ++k)
      if (k < r) acc[k] += red[(sl * CP_COLS + jc) * r + k];
  }
  __syncthreads();
  if (sl == 1) {
#pragma unroll
    for (int k = 0; k < RMAX; ++k)
      if (k < r) red[jc * r + k] = acc[k];
  }
  __syncthreads();
  if (sl == 0 && j < i) {
    double* out = Zp + ((int64_t)blockIdx.y * i + j) * r;
#pragma unroll
    for (int k = 0; k < RMAX; ++k)
      if (k < r) out[k] = acc[k] + red[jc * r + k];
  }
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

// CholeskyQR2 of a rows × r matrix that fits in shared memory, in one CTA:
// Y is staged once; each pass forms the Gram matrix (a warp per (a, b) pair,
// lanes over the rows, a fixed shuffle tree), factors it with warp 0 as
// chmc_chol_kernel does (dropping non-positive pivots), and multiplies in
// place by R⁻¹.  Q receives the result.
constexpr int ORTH_SMALL_MAX = 12288;          // rows·r doubles staged (96 KB)
constexpr int ORTH_T = 256;
__global__ void __launch_bounds__(ORTH_T)
chmc_orth_small_kernel(const double* __restrict__ Yin, int rows, int r, double* __restrict__ Q) {
  extern __shared__ double osm[];
  double* Y = osm;                                  // rows × r
  __shared__ double G[CHMC_MAX_RANK][CHMC_MAX_RANK + 1];
  __shared__ double L[CHMC_MAX_RANK][CHMC_MAX_RANK + 1];
  __shared__ double Ri[CHMC_MAX_RANK * CHMC_MAX_RANK];
  const int t = threadIdx.x, lane = t & 31;
#pragma unroll 8
  for (int e = t; e < rows * r; e += ORTH_T) Y[e] = Yin[e];
  const int npair = r * (r + 1) / 2;
  const int warp = t >> 5;
  auto pair_ab = [&](int pidx, int& a, int& b) {
    int rem = pidx;
    a = 0;
    while (rem >= r - a) { rem -= r - a; ++a; }
    b = a + rem;
  };
  for (int pass = 0; pass < 2; ++pass) {
    __syncthreads();
    // Gram entries: warp w takes pairs w, w + 8, ...; its lanes stride the
    // rows four at a time, then a fixed shuffle tree adds the lanes
    for (int pidx = warp; pidx < npair; pidx += ORTH_T / 32) {
      int a, b;
      pair_ab(pidx, a, b);
      double acc0 = 0.0, acc1 = 0.0;
      int rr = lane;
      for (; rr + 96 < rows; rr += 128) {
        const double y0 = Y[rr * r + a], z0 = Y[rr * r + b];
        const double y1 = Y[(rr + 32) * r + a], z1 = Y[(rr + 32) * r + b];
        const double y2 = Y[(rr + 64) * r + a], z2 = Y[(rr + 64) * r + b];
        const double y3 = Y[(rr + 96) * r + a], z3 = Y[(rr + 96) * r + b];
        acc0 = fma(y0, z0, acc0);
        acc1 = fma(y1, z1, acc1);
        acc0 = fma(y2, z2, acc0);
        acc1 = fma(y3, z3, acc1);
      }
      for (; rr < rows; rr += 32) acc0 = fma(Y[rr * r + a], Y[rr * r + b], acc0);
      double acc = acc0 + acc1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) {
        G[a][b] = acc;
        G[b][a] = acc;
      }
    }
    __syncthreads();
    if (t < 32) {
      for (int b = 0; b < r; ++b)
        if (lane < r) L[lane][b] = 0.0;
      double tr = 0.0;
      for (int k = 0; k < r; ++k) tr += G[k][k];
      const double floor_piv = 1e-28 * (tr > 0.0 ? tr : 1.0);
      __syncwarp();
      for (int k = 0; k < r; ++k) {
        const double piv = G[k][k];
        const bool keep = piv > floor_piv;
        const double d = keep ? sqrt(piv) : 0.0;
        __syncwarp();
        if (lane >= k && lane < r) L[lane][k] = keep ? G[lane][k] / d : 0.0;
        __syncwarp();
        if (lane > k && lane < r)
          for (int l = k + 1; l <= lane; ++l) G[lane][l] -= L[lane][k] * L[l][k];
        __syncwarp();
      }
      if (lane < r) {
        double x[CHMC_MAX_RANK];
#pragma unroll
        for (int i = 0; i < CHMC_MAX_RANK; ++i) x[i] = 0.0;
        for (int i = lane; i < r; ++i) {
          double sacc = (i == lane) ? 1.0 : 0.0;
          for (int m2 = lane; m2 < i; ++m2) sacc -= L[i][m2] * x[m2];
          x[i] = (L[i][i] != 0.0) ? sacc / L[i][i] : 0.0;
        }
        for (int i = 0; i < r; ++i) Ri[lane * r + i] = (i >= lane) ? x[i] : 0.0;
      }
    }
    __syncthreads();
    // Y ← Y·R⁻¹ in place, a row per thread: column k needs columns l ≤ k, so
    // the columns are formed from the last to the first
    for (int row = t; row < rows; row += ORTH_T) {
      double* y = Y + row * r;
      for (int k = r - 1; k >= 0; --k) {
        double acc = 0.0;
        for (int l = 0; l <= k; ++l) acc = fma(y[l], Ri[l * r + k], acc);
        y[k] = acc;
      }
    }
  }
  __syncthreads();
  for (int e = t; e < rows * r; e += ORTH_T) Q[e] = Y[e];
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
  if (rows * r <= ORTH_SMALL_MAX) {               // one CTA, Y in shared memory
    const size_t smem = sizeof(double) * (size_t)rows * r;
    GPTQ_LAUNCH(KK_CHMC, s, chmc_orth_small_kernel, 1, ORTH_T, smem, Y, (int)rows, r, Q);
    return GPTQ_OK;
  }
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

// The thin products at the smallest compiled rank bound that holds r.
template <typename T, int RM>
gptq_status rowprod_at(unsigned grid, const T* W, int64_t o, int64_t i, const double* sq,
                       const double* X, int r, double* Y, cudaStream_t s) {
  const auto kfn = &chmc_rowprod_kernel<T, RM>;
  GPTQ_LAUNCH(KK_CHMC, s, kfn, grid, 256, 0, W, o, i, sq, X, r, Y);
  return GPTQ_OK;
}
template <typename T>
gptq_status launch_rowprod(unsigned grid, const T* W, int64_t o, int64_t i, const double* sq,
                           const double* X, int r, double* Y, cudaStream_t s) {
  if (r <= 4) return rowprod_at<T, 4>(grid, W, o, i, sq, X, r, Y, s);
  if (r <= 8) return rowprod_at<T, 8>(grid, W, o, i, sq, X, r, Y, s);
  if (r <= 16) return rowprod_at<T, 16>(grid, W, o, i, sq, X, r, Y, s);
  return rowprod_at<T, 32>(grid, W, o, i, sq, X, r, Y, s);
}
template <typename T, int RM>
gptq_status colprod_at(dim3 grid, const T* W, int64_t o, int64_t i, const double* Q, int r,
                       double* Zp, cudaStream_t s) {
  const auto kfn = &chmc_colprod_kernel<T, RM>;
  GPTQ_LAUNCH(KK_CHMC, s, kfn, grid, 256, 0, W, o, i, Q, r, Zp);
  return GPTQ_OK;
}
template <typename T>
gptq_status launch_colprod(dim3 grid, const T* W, int64_t o, int64_t i, const double* Q, int r,
                           double* Zp, cudaStream_t s) {
  if (r <= 4) return colprod_at<T, 4>(grid, W, o, i, Q, r, Zp, s);
  if (r <= 8) return colprod_at<T, 8>(grid, W, o, i, Q, r, Zp, s);
  if (r <= 16) return colprod_at<T, 16>(grid, W, o, i, Q, r, Zp, s);
  return colprod_at<T, 32>(grid, W, o, i, Q, r, Zp, s);
}


template <typename T>
gptq_status lowrank_impl(const T* W, int64_t o, int64_t i, const float* H, int64_t tokens,
                         double lam, const float* Omega, int r, int niter, float* Qf,
                         float* Pf, float* Res, int32_t* info, char* ws, cudaStream_t s) {
  double *sq, *om, *Y, *Q, *Z, *Qi, *Zp, *Gp, *Rinv, *P;
  chmc_layout(o, i, r, ws, &sq, &om, &Y, &Q, &Z, &Qi, &Zp, &Gp, &Rinv, &P);
  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  {
    const gptq_status st = ensure_smem_limit((const void*)chmc_orth_small_kernel,
                                             (int)(sizeof(double) * ORTH_SMALL_MAX),
                                             "chmc_orth_small_kernel");
    if (st != GPTQ_OK) return st;
  }
  if (r == 0) {
    GPTQ_LAUNCH(KK_CHMC, s, chmc_copy_kernel<T>, (unsigned)ceil_div(o * i, 256), 256, 0, W,
                o * i, Res);
    return GPTQ_OK;
  }
  GPTQ_LAUNCH(KK_CHMC, s, chmc_energy_kernel, 1, 1024, 0, H, i, tokens, lam, sq, info);
  GPTQ_LAUNCH(KK_CHMC, s, chmc_to_f64_kernel, (unsigned)ceil_div(i * r, 256), 256, 0, Omega,
              i * r, om);
  const unsigned grow = (unsigned)ceil_div(o, 8);
  const dim3 gcol((unsigned)ceil_div(i, CP_COLS), (unsigned)ceil_div(o, CHUNK));
  const int nco = (int)ceil_div(o, CHUNK);
  const unsigned gred = (unsigned)ceil_div(i * r, 256);
  // Y = W̃·Ω, Q = orth(Y)
  gptq_status st = launch_rowprod(grow, W, o, i, sq, om, r, Y, s);
  if (st != GPTQ_OK) return st;
  st = orth_rows(Y, o, r, Q, Gp, Rinv, s);
  if (st != GPTQ_OK) return st;
  for (int it = 0; it < niter; ++it) {
    // Qi = orth(W̃ᵀ·Q) with W̃ᵀ·Q = diag(√c)·Wᵀ·Q
    st = launch_colprod(gcol, W, o, i, Q, r, Zp, s);
    if (st != GPTQ_OK) return st;
    GPTQ_LAUNCH(KK_CHMC, s, chmc_colreduce_kernel, gred, 256, 0, Zp, nco, i, r, sq, Z);
    st = orth_rows(Z, i, r, Qi, Gp, Rinv, s);
    if (st != GPTQ_OK) return st;
    // Q = orth(W̃·Qi)
    st = launch_rowprod(grow, W, o, i, sq, Qi, r, Y, s);
    if (st != GPTQ_OK) return st;
    st = orth_rows(Y, o, r, Q, Gp, Rinv, s);
    if (st != GPTQ_OK) return st;
  }
  // P = Qᵀ·W (stored i × r), then the residual W − Q·P and the factors
  st = launch_colprod(gcol, W, o, i, Q, r, Zp, s);
  if (st != GPTQ_OK) return st;
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
