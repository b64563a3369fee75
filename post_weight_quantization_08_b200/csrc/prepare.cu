// K2: damping, dead columns, processing order and the inverse-Cholesky
// factor U (upper, UᵀU = (P·H_d·Pᵀ)⁻¹), all in float64.
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: relative
// damping λ·mean(diag H)·I, act-order, and H⁻¹ "über die Cholesky-Zerlegung";
// GPTQ reads, for column j, the inverse over the columns not yet quantized,
// which is row j of U (up to its diagonal).  "GPTQ as Babai's Nearest Plane
// Algorithm", §2.3: act-order sorts the Hessian diagonal.
//
// Route (no explicit inverse of H): with J the index reversal and
// A = J·H_p·J = L·Lᵀ (lower Cholesky), R̃ = J·L·J is upper with H_p = R̃·R̃ᵀ,
// and U = R̃⁻¹ = J·L⁻¹·J.  UᵀU = R̃⁻ᵀR̃⁻¹ = H_p⁻¹, and U is upper with a
// positive diagonal, so it is THE upper Cholesky factor of H_p⁻¹.  This costs
// n³/3 (Cholesky) + n³/3 (triangular inverse), both fused into one blocked,
// right-looking sweep over 64×64 float64 tiles:
//   diag(k):  L_kk = chol(A_kk) and D_k = L_kk⁻¹ (one CTA)
//   panel(k): L_ik = A_ik·D_kᵀ (i > k);  M_kc = D_k·M_kc (c < k): finished
//             block row k of L⁻¹
//   trail(k): A_ij −= L_ik·L_jkᵀ (k < j ≤ i);  M_ic −= L_ik·M_kc (i > k, c ≤ k)
// A is padded with an identity block to a multiple of 64.
#include <cmath>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int NB = 64;          // float64 tile edge
constexpr int LDT = NB + 1;     // padded shared-memory row (doubles)

struct PrepWs {
  double* mean;   // 1
  int32_t* seen;  // n (custom-order check)
  double* A;      // np × np
  double* M;      // np × np
  double* D;      // NB × NB (L_kk⁻¹ of the current step)
};

size_t prep_ws_layout(int64_t n, PrepWs* w, char* base) {
  const int64_t np = ceil_div(n, NB) * NB;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  size_t o_mean = take(sizeof(double));
  size_t o_seen = take(sizeof(int32_t) * (size_t)n);
  size_t o_A = take(sizeof(double) * (size_t)np * (size_t)np);
  size_t o_M = take(sizeof(double) * (size_t)np * (size_t)np);
  size_t o_D = take(sizeof(double) * NB * NB);
  if (w && base) {
    w->mean = reinterpret_cast<double*>(base + o_mean);
    w->seen = reinterpret_cast<int32_t*>(base + o_seen);
    w->A = reinterpret_cast<double*>(base + o_A);
    w->M = reinterpret_cast<double*>(base + o_M);
    w->D = reinterpret_cast<double*>(base + o_D);
  }
  return off;
}

// mean(diag H) in a fixed summation order (deterministic), dead mask,
// finiteness of the diagonal.
__global__ void __launch_bounds__(1024)
prep_stats_kernel(const float* __restrict__ H, int64_t n, uint8_t* __restrict__ dead,
                  double* __restrict__ mean, int32_t* info) {
  __shared__ double part[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += 1024) {
    const float h = H[i * n + i];
    if (!isfinite(h)) report(info, GPTQ_ERR_NONFINITE, i * n + i);
    dead[i] = (h == 0.0f) ? 1 : 0;
    s += (double)h;
  }
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *mean = part[0] / (double)n;
}

// Processing permutation.  act: rank of each column under "larger diagonal
// first, then smaller index"; dead diagonals count as 1.
__global__ void __launch_bounds__(256)
prep_order_kernel(const float* __restrict__ H, int64_t n, int order,
                  int32_t* __restrict__ perm, int32_t* __restrict__ seen,
                  int32_t* info) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (order == GPTQ_ORDER_NATURAL) {
    if (i < n) perm[i] = (int32_t)i;
    return;
  }
  if (order == GPTQ_ORDER_REVERSE) {
    if (i < n) perm[i] = (int32_t)(n - 1 - i);
    return;
  }
  if (order == GPTQ_ORDER_CUSTOM) {
    if (i < n) {
      const int32_t v = perm[i];
      if (v < 0 || v >= n) report(info, GPTQ_ERR_INVALID_ARG, i);
      else atomicAdd(&seen[v], 1);
    }
    return;
  }
  // act-order
  __shared__ float keys[2048];
  float ki = 0.f;
  if (i < n) {
    ki = H[i * n + i];
    if (ki == 0.0f) ki = 1.0f;
  }
  int64_t rank = 0;
  for (int64_t c0 = 0; c0 < n; c0 += 2048) {
    __syncthreads();
    for (int e = threadIdx.x; e < 2048; e += 256) {
      const int64_t j = c0 + e;
      float kj = 0.f;
      if (j < n) {
        kj = H[j * n + j];
        if (kj == 0.0f) kj = 1.0f;
      }
      keys[e] = kj;
    }
    __syncthreads();
    if (i < n) {
      const int64_t lim = (n - c0 < 2048) ? (n - c0) : 2048;
      for (int64_t e = 0; e < lim; ++e) {
        const float kj = keys[e];
        const int64_t j = c0 + e;
        rank += (kj > ki) || (kj == ki && j < i);
      }
    }
  }
  if (i < n) perm[rank] = (int32_t)i;
}

// A[a][b] = H_d[perm[n−1−a]][perm[n−1−b]] (lower triangle), identity padding;
// M := 0 (lower triangle).
__global__ void __launch_bounds__(256)
prep_gather_kernel(const float* __restrict__ H, int64_t n, int64_t np,
                   const int32_t* __restrict__ perm,
                   const int32_t* __restrict__ seen, int check_seen,
                   const double* __restrict__ mean, double damp,
                   double* __restrict__ A, double* __restrict__ M, int32_t* info) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= np * np) return;
  const int64_t a = e / np, b = e % np;
  if (b > a) return;
  M[e] = 0.0;
  double v;
  if (a >= n) {
    v = (a == b) ? 1.0 : 0.0;
  } else {
    const int32_t pa = perm[n - 1 - a], pb = perm[n - 1 - b];
    if (pa < 0 || pa >= n || pb < 0 || pb >= n) {   // bad custom order
      report(info, GPTQ_ERR_INVALID_ARG, n - 1 - a);
      A[e] = (a == b) ? 1.0 : 0.0;
      return;
    }
    if (check_seen && a == b && seen[pa] != 1) report(info, GPTQ_ERR_INVALID_ARG, n - 1 - a);
    const float h = H[(int64_t)pa * n + pb];
    if (!isfinite(h)) report(info, GPTQ_ERR_NONFINITE, (int64_t)pa * n + pb);
    v = (double)h;
    if (a == b) {
      if (h == 0.0f) v = 1.0;          // dead column
      v += damp * (*mean);
    }
  }
  A[e] = v;
}

// Diagonal tile: L_kk = chol(A_kk) and D = L_kk⁻¹, fused right-looking, one
// barrier per column.  Column c's scaled entries are written one step late,
// when nothing reads them any more.
__global__ void __launch_bounds__(256)
chol_diag_kernel(double* __restrict__ A, double* __restrict__ M,
                 double* __restrict__ D, int64_t n, int64_t np, int k,
                 int32_t* info) {
  if (info[0] != 0) return;
  extern __shared__ double sm[];
  double (*a)[LDT] = reinterpret_cast<double (*)[LDT]>(sm);
  double (*b)[LDT] = reinterpret_cast<double (*)[LDT]>(sm + NB * LDT);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t base = (int64_t)k * NB;
  for (int e = tid; e < NB * NB; e += 256) {
    const int r = e / NB, c = e % NB;
    a[r][c] = (c <= r) ? A[(base + r) * np + base + c] : 0.0;
    b[r][c] = (r == c) ? 1.0 : 0.0;
  }
  __syncthreads();
  double prev_piv = 0.0, prev_rp = 0.0;
  bool bad = false;
  for (int c = 0; c < NB; ++c) {
    const double d = a[c][c];
    if (!(d > 0.0) || !isfinite(d)) {
      if (tid == 0) {
        const int64_t apos = base + c;                // index in A
        report(info, isfinite(d) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE,
               n - 1 - apos);                         // processing position
      }
      bad = true;
      break;
    }
    const double piv = sqrt(d);
    const double rp = 1.0 / piv;
    // deferred scaling of column c−1 of a and row c−1 of b
    if (c > 0) {
      for (int r = c + tid; r < NB; r += 256) a[r][c - 1] *= prev_rp;
      for (int x = tid; x < c; x += 256) b[c - 1][x] *= prev_rp;
      if (tid == 0) a[c - 1][c - 1] = prev_piv;
    }
    // rank-1 updates with l = column c scaled by 1/piv
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = ty * 4 + rr;
      if (r <= c) continue;
      const double lr = a[r][c] * rp;
#pragma unroll
      for (int xx = 0; xx < 4; ++xx) {
        const int x = tx * 4 + xx;
        if (x > c) {
          if (x <= r) a[r][x] -= lr * (a[x][c] * rp);
        } else {
          b[r][x] -= lr * (b[c][x] * rp);
        }
      }
    }
    prev_piv = piv;
    prev_rp = rp;
    __syncthreads();
  }
  if (bad) return;
  // last column's deferred scaling
  for (int x = tid; x < NB - 1; x += 256) b[NB - 1][x] *= prev_rp;
  if (tid == 0) {
    a[NB - 1][NB - 1] = prev_piv;
    b[NB - 1][NB - 1] *= prev_rp;
  }
  __syncthreads();
  for (int e = tid; e < NB * NB; e += 256) {
    const int r = e / NB, c = e % NB;
    if (c <= r) A[(base + r) * np + base + c] = a[r][c];
    M[(base + r) * np + base + c] = b[r][c];
    D[e] = b[r][c];
  }
}

// 64×64 float64 tile product C = X·Y on shared-memory tiles; each of the 256
// threads owns a 4×4 block of C.
__device__ __forceinline__ void tile_mm(const double (*x)[LDT], const double (*y)[LDT],
                                        double acc[4][4], int tx, int ty) {
#pragma unroll 4
  for (int q = 0; q < NB; ++q) {
    double xv[4], yv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xv[i] = x[ty * 4 + i][q];
      yv[i] = y[q][tx * 4 + i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv[i], yv[j], acc[i][j]);
  }
}

__device__ __forceinline__ void load_tile(double (*dst)[LDT], const double* src,
                                          int64_t ld, bool transpose, int tid) {
  for (int e = tid; e < NB * NB; e += 256) {
    const int r = e / NB, c = e % NB;
    const double v = src[(int64_t)r * ld + c];
    if (transpose) dst[c][r] = v; else dst[r][c] = v;
  }
}

// panel(k): blocks [0, N−k−1): L_ik = A_ik·Dᵀ; blocks [N−k−1, N−1): M_kc = D·M_kc.
__global__ void __launch_bounds__(256)
chol_panel_kernel(double* __restrict__ A, double* __restrict__ M,
                  const double* __restrict__ D, int64_t np, int N, int k,
                  int32_t* info) {
  if (info[0] != 0) return;
  extern __shared__ double sm[];
  double (*x)[LDT] = reinterpret_cast<double (*)[LDT]>(sm);
  double (*y)[LDT] = reinterpret_cast<double (*)[LDT]>(sm + NB * LDT);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int nlow = N - k - 1;
  double* out;
  if ((int)blockIdx.x < nlow) {
    const int i = k + 1 + blockIdx.x;
    out = A + (int64_t)i * NB * np + (int64_t)k * NB;
    load_tile(x, out, np, false, tid);
    load_tile(y, D, NB, true, tid);
  } else {
    const int c = blockIdx.x - nlow;
    out = M + (int64_t)k * NB * np + (int64_t)c * NB;
    load_tile(x, D, NB, false, tid);
    load_tile(y, out, np, false, tid);
  }
  __syncthreads();
  double acc[4][4] = {};
  tile_mm(x, y, acc, tx, ty);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) out[(int64_t)(ty * 4 + i) * np + tx * 4 + j] = acc[i][j];
}

// trail(k): first r(r+1)/2 blocks are (i, j), k < j ≤ i: A_ij −= L_ik·L_jkᵀ;
// the next r·(k+1) are (i, c), i > k, c ≤ k: M_ic −= L_ik·M_kc.
__global__ void __launch_bounds__(256)
chol_trail_kernel(double* __restrict__ A, double* __restrict__ M, int64_t np,
                  int N, int k, int32_t* info) {
  if (info[0] != 0) return;
  extern __shared__ double sm[];
  double (*x)[LDT] = reinterpret_cast<double (*)[LDT]>(sm);
  double (*y)[LDT] = reinterpret_cast<double (*)[LDT]>(sm + NB * LDT);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r = N - k - 1;
  const int ntri = r * (r + 1) / 2;
  int lin = blockIdx.x;
  double* out;
  if (lin < ntri) {
    // decode (ii, jj) with 0 <= jj <= ii < r
    int ii = 0;
    while (lin >= ii + 1) { lin -= ii + 1; ++ii; }
    const int i = k + 1 + ii, j = k + 1 + lin;
    out = A + (int64_t)i * NB * np + (int64_t)j * NB;
    load_tile(x, A + (int64_t)i * NB * np + (int64_t)k * NB, np, false, tid);
    load_tile(y, A + (int64_t)j * NB * np + (int64_t)k * NB, np, true, tid);
  } else {
    lin -= ntri;
    const int i = k + 1 + lin / (k + 1), c = lin % (k + 1);
    out = M + (int64_t)i * NB * np + (int64_t)c * NB;
    load_tile(x, A + (int64_t)i * NB * np + (int64_t)k * NB, np, false, tid);
    load_tile(y, M + (int64_t)k * NB * np + (int64_t)c * NB, np, false, tid);
  }
  __syncthreads();
  double acc[4][4] = {};
  tile_mm(x, y, acc, tx, ty);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) out[(int64_t)(ty * 4 + i) * np + tx * 4 + j] -= acc[i][j];
}

// U[i][j] = L⁻¹[n−1−i][n−1−j] for j ≥ i, 0 below the diagonal.
__global__ void __launch_bounds__(256)
prep_out_kernel(const double* __restrict__ M, int64_t n, int64_t np,
                float* __restrict__ U) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= n * n) return;
  const int64_t i = e / n, j = e % n;
  U[e] = (j >= i) ? (float)M[(n - 1 - i) * np + (n - 1 - j)] : 0.0f;
}

bool g_smem_set = false;

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" size_t gptq_prepare_workspace_bytes(int64_t n) {
  if (n < 1) return 0;
  return prep_ws_layout(n, nullptr, nullptr);
}

extern "C" gptq_status gptq_prepare(const float* H, int64_t n, double damp,
                                    int order, int32_t* perm, float* U,
                                    uint8_t* dead, int32_t* info, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (!H || !perm || !U || !dead || !info || !ws)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: null pointer");
  if (n < 1 || n > (int64_t)1 << 20)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: n=%lld", (long long)n);
  if (!(damp >= 0.0) || !std::isfinite(damp))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: damp must be finite and >= 0");
  if (order < GPTQ_ORDER_NATURAL || order > GPTQ_ORDER_CUSTOM)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: order=%d", order);
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: workspace not 256-byte aligned");
  const size_t need = prep_ws_layout(n, nullptr, nullptr);
  if (ws_bytes < need)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: workspace %zu < %zu bytes",
                ws_bytes, need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PrepWs w;
  prep_ws_layout(n, &w, static_cast<char*>(ws));
  const int64_t np = ceil_div(n, NB) * NB;
  const int N = (int)(np / NB);
  const size_t tile_smem = 2 * NB * LDT * sizeof(double);
  if (!g_smem_set) {
    GPTQ_CUDA(cudaFuncSetAttribute(chol_diag_kernel,
              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem));
    GPTQ_CUDA(cudaFuncSetAttribute(chol_panel_kernel,
              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem));
    GPTQ_CUDA(cudaFuncSetAttribute(chol_trail_kernel,
              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem));
    g_smem_set = true;
  }

  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  if (order == GPTQ_ORDER_CUSTOM)
    GPTQ_CUDA(cudaMemsetAsync(w.seen, 0, sizeof(int32_t) * n, s));
  GPTQ_LAUNCH(KK_PREP_STATS, s, prep_stats_kernel, 1, 1024, 0, H, n, dead, w.mean, info);
  GPTQ_LAUNCH(KK_PREP_ORDER, s, prep_order_kernel, (int)ceil_div(n, 256), 256, 0,
              H, n, order, perm, w.seen, info);
  GPTQ_LAUNCH(KK_PREP_GATHER, s, prep_gather_kernel, (unsigned)ceil_div(np * np, 256),
              256, 0, H, n, np, perm, w.seen, order == GPTQ_ORDER_CUSTOM ? 1 : 0,
              w.mean, damp, w.A, w.M, info);
  for (int k = 0; k < N; ++k) {
    GPTQ_LAUNCH(KK_CHOL_DIAG, s, chol_diag_kernel, 1, 256, tile_smem, w.A, w.M, w.D, n, np, k, info);
    const int r = N - k - 1;
    if (r + k > 0)
      GPTQ_LAUNCH(KK_CHOL_PANEL, s, chol_panel_kernel, r + k, 256, tile_smem,
                  w.A, w.M, w.D, np, N, k, info);
    const int tiles = r * (r + 1) / 2 + r * (k + 1);
    if (tiles > 0)
      GPTQ_LAUNCH(KK_CHOL_TRAIL, s, chol_trail_kernel, tiles, 256, tile_smem,
                  w.A, w.M, np, N, k, info);
  }
  GPTQ_LAUNCH(KK_PREP_OUT, s, prep_out_kernel, (unsigned)ceil_div(n * n, 256), 256, 0,
              w.M, n, np, U);
  return GPTQ_OK;
}
