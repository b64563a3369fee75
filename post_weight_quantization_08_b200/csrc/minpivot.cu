// The min-pivot processing order ("The Geometry of LLM Quantization: GPTQ as
// Babai's Nearest Plane Algorithm", §2.3, "Rolle der Reihenfolge"): the LDL
// factorisation of Satz 5 takes, at every step, the smallest diagonal entry
// of the current Schur complement.  That LDL eliminates the last processed
// column first, so the column eliminated at step t is processed at position
// n−1−t.  Equal diagonals go to the larger column index (a diagonal H then
// gives act-order, H = I the natural order).
//
// Float64, on the damped and dead-fixed H_d, without moving rows: S stays in
// the original column order, eliminated columns are marked by an infinite
// diagonal, and the factor columns of the current panel (32, 16 or 8 steps,
// the most that fit in shared memory) are kept by original row index.
//   mp_init:   S = H_d (both triangles), d = diag S, panel columns zero
//   mp_panel:  one CTA, 32 dependent steps: argmin of d (ties → larger
//              index), pivot d_j, the column c = S[j, :] − Σ_panel Lp[:, s]·Lp[j, s],
//              L = c/√d_j, d −= L², d_j = ∞
//   mp_trail:  S −= Lp·Lpᵀ after each panel (float64 tiles)
//   mp_finish: perm[n−1−t] = column eliminated at step t
// The order then feeds the regular factorisation as a custom order.
#include <cmath>

#include "common.cuh"
#include "minpivot.cuh"

namespace gptq {
namespace {

constexpr int MP_THREADS = 512;
constexpr int MP_TILE = 64;          // trailing update tile edge

__global__ void __launch_bounds__(256)
mp_init_kernel(const float* __restrict__ H, int64_t n, int64_t ld, const double* __restrict__ mean,
               double damp, double* __restrict__ S, double* __restrict__ d,
               double* __restrict__ Lp, int32_t* info) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e < n * MP_PANEL) Lp[e] = 0.0;      // the grid covers max(n², n·MP_PANEL)
  if (e >= n * n) return;
  const int64_t a = e / n, b = e % n;
  const float h = H[e];
  if (!isfinite(h)) report(info, GPTQ_ERR_NONFINITE, e);
  double v = (double)h;
  if (a == b) {
    if (h == 0.0f) v = 1.0;          // dead column
    v += damp * (*mean);
    d[a] = v;
  }
  S[a * ld + b] = v;
}

// (value, index) order of the pivot search: the smaller value, ties to the
// larger index.  A total order, so any reduction order gives the same pivot.
__device__ __forceinline__ bool mp_better(double ov, int oi, double v, int i) {
  return ov < v || (ov == v && oi > i);
}

// One panel of pw ≤ MP_PANEL dependent steps in one CTA.  The Schur diagonal
// d and, when they fit (lp_smem), the panel's factor columns live in shared
// memory for the panel; d goes back to global memory at the end and the
// columns are written to Lp (row i at i·MP_PANEL) for the trailing update.
//
// Thread t owns rows t, t + MP_THREADS, …: it alone updates their d and
// panel columns, and while it does so it keeps the running pivot candidate
// of its rows.  One barrier a step: each warp's best candidate goes to a
// shared slot (two sets, alternating by step), and after the barrier every
// thread reduces the slots itself.  The pivot value comes with the candidate
// (the owner of row j sets d_j = ∞ during the same step); row j's panel
// columns (written in earlier steps, before this step's barrier) are read in
// place.  The only global reads per step are row j of S (and, without
// lp_smem, the rows' panel columns), all issued before use.
__global__ void __launch_bounds__(MP_THREADS, 1)
mp_panel_kernel(const double* __restrict__ S, int64_t n, int64_t ld, double* __restrict__ dg,
                double* __restrict__ Lp, int32_t* __restrict__ elim, int64_t t0, int pw,
                int lp_smem, int32_t* info) {
  extern __shared__ double smem[];
  double* d = smem;                                  // n
  double* lps = smem + ((n + 1) & ~int64_t(1));      // n rows of pw + 1 when lp_smem
  const int lds = pw + 1;                            // odd stride: no bank conflicts
  constexpr int NW = MP_THREADS / 32;
  __shared__ double sv[2][NW];
  __shared__ int si[2][NW];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (*reinterpret_cast<volatile int32_t*>(info) != 0) return;
  for (int64_t i = tid; i < n; i += MP_THREADS) d[i] = dg[i];
  if (lp_smem)
    for (int64_t e = tid; e < n * lds; e += MP_THREADS) lps[e] = 0.0;
  __syncthreads();
  // the first candidate of this thread's rows
  double bv = INFINITY;
  int bi = -1;
  for (int64_t i = tid; i < n; i += MP_THREADS) {
    const double v = d[i];
    if (v < INFINITY && mp_better(v, (int)i, bv, bi)) { bv = v; bi = (int)i; }
  }
  const int steps = (int)((n - t0 < pw) ? (n - t0) : pw);
  for (int k = 0; k < steps; ++k) {
    const int b = k & 1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_down_sync(0xffffffffu, bv, o);
      const int oi = __shfl_down_sync(0xffffffffu, bi, o);
      if (mp_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) { sv[b][warp] = bv; si[b][warp] = bi; }
    __syncthreads();
    double piv = sv[b][0];
    int j = si[b][0];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      const double ov = sv[b][w];
      const int oi = si[b][w];
      if (mp_better(ov, oi, piv, j)) { piv = ov; j = oi; }
    }
    if (!(piv < INFINITY)) j = -1;
    if (j < 0 || !(piv >= 2.2250738585072014e-308 && piv <= 1.7976931348623157e308)) {
      if (tid == 0) report(info, GPTQ_ERR_NOT_PD, n - 1 - (t0 + k));   // uniform exit
      break;
    }
    if (tid == 0) elim[t0 + k] = j;
    const double rp = 1.0 / sqrt(piv);
    bv = INFINITY;
    bi = -1;
    if (lp_smem) {
      const double* lj = lps + (int64_t)j * lds;    // row j's panel columns, q < k
      // row j of S for all of this thread's rows first, then the sums
      constexpr int R = 8;                           // rows per thread per pass
      for (int64_t i0 = tid; i0 < n; i0 += (int64_t)R * MP_THREADS) {
        double sj[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int64_t i = i0 + (int64_t)r * MP_THREADS;
          sj[r] = (i < n) ? S[(int64_t)j * ld + i] : 0.0;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int64_t i = i0 + (int64_t)r * MP_THREADS;
          if (i >= n) continue;
          if (i == j) {                              // this thread owns the pivot row
            d[i] = INFINITY;
            lps[i * lds + k] = 0.0;
            continue;
          }
          const double di = d[i];
          if (!(di < INFINITY)) continue;
          const double* li = lps + i * lds;
          double c0 = sj[r], c1 = 0.0;
          int q = 0;
          for (; q + 1 < k; q += 2) {
            c0 -= li[q] * lj[q];
            c1 -= li[q + 1] * lj[q + 1];
          }
          if (q < k) c0 -= li[q] * lj[q];
          const double l = (c0 + c1) * rp;
          lps[i * lds + k] = l;
          const double dn = di - l * l;
          d[i] = dn;
          if (dn < INFINITY && mp_better(dn, (int)i, bv, bi)) { bv = dn; bi = (int)i; }
        }
      }
    } else {
      const double* lj = Lp + (int64_t)j * MP_PANEL;
      for (int64_t i = tid; i < n; i += MP_THREADS) {
        if (i == j) {
          d[i] = INFINITY;
          Lp[i * MP_PANEL + k] = 0.0;
          continue;
        }
        const double di = d[i];
        if (!(di < INFINITY)) continue;
        double c = S[(int64_t)j * ld + i];            // S is symmetric: row j
        const double2* li = reinterpret_cast<const double2*>(Lp + i * MP_PANEL);
#pragma unroll
        for (int h = 0; h < 2; ++h) {                 // two halves of 16 columns
          if (16 * h >= k) break;
          double2 lv[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int s0 = 16 * h + 2 * q;
            lv[q] = (s0 < k) ? li[8 * h + q] : make_double2(0.0, 0.0);
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int s0 = 16 * h + 2 * q;
            c -= ((s0 < k) ? lv[q].x : 0.0) * ((s0 < k) ? lj[s0] : 0.0);
            c -= ((s0 + 1 < k) ? lv[q].y : 0.0) * ((s0 + 1 < k) ? lj[s0 + 1] : 0.0);
          }
        }
        const double l = c * rp;
        Lp[i * MP_PANEL + k] = l;
        const double dn = di - l * l;
        d[i] = dn;
        if (dn < INFINITY && mp_better(dn, (int)i, bv, bi)) { bv = dn; bi = (int)i; }
      }
    }
  }
  __syncthreads();
  for (int64_t i = tid; i < n; i += MP_THREADS) dg[i] = d[i];
  if (lp_smem) {
    // the panel's columns out for the trailing update (zeros past pw)
    for (int64_t e = tid; e < n * MP_PANEL; e += MP_THREADS) {
      const int64_t i = e / MP_PANEL;
      const int q = (int)(e % MP_PANEL);
      Lp[e] = (q < pw) ? lps[i * lds + q] : 0.0;
    }
  }
}

// S −= Lp·Lpᵀ over the whole n×n matrix, K = the panel width pw (rows of
// eliminated columns are never read again, so they need no mask).  64×64
// tiles, 256 threads, 4×4 each.
__global__ void __launch_bounds__(256)
mp_trail_kernel(double* __restrict__ S, int64_t n, int64_t ld, const double* __restrict__ Lp,
                int pw) {
  __shared__ double a[MP_PANEL][MP_TILE + 1];
  __shared__ double b[MP_PANEL][MP_TILE + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t r0 = (int64_t)blockIdx.y * MP_TILE, c0 = (int64_t)blockIdx.x * MP_TILE;
  for (int e = tid; e < MP_TILE * pw; e += 256) {
    const int r = e / pw, s = e % pw;
    a[s][r] = (r0 + r < n) ? Lp[(r0 + r) * MP_PANEL + s] : 0.0;
    b[s][r] = (c0 + r < n) ? Lp[(c0 + r) * MP_PANEL + s] : 0.0;
  }
  __syncthreads();
  double acc[4][4] = {};
#pragma unroll 8
  for (int s = 0; s < pw; ++s) {
    double x[4], y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[i] = a[s][ty + 16 * i];
      y[i] = b[s][tx + 16 * i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = fma(x[i], y[q], acc[i][q]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty + 16 * i;
    if (r >= n) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t c = c0 + tx + 16 * q;
      if (c < n) S[r * ld + c] -= acc[i][q];
    }
  }
}

__global__ void __launch_bounds__(256)
mp_finish_kernel(const int32_t* __restrict__ elim, int64_t n, int32_t* __restrict__ perm) {
  const int64_t t = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (t < n) perm[n - 1 - t] = elim[t];
}

}  // namespace

size_t min_pivot_scratch_doubles(int64_t n) {
  // d (n), the panel columns (n × MP_PANEL), the elimination order (n int32)
  return (size_t)n + (size_t)n * MP_PANEL + ((size_t)n + 1) / 2 + 64;
}

gptq_status launch_min_pivot_order(const float* H, int64_t n, const double* mean, double damp,
                                   double* S, int64_t ld, double* scratch, int32_t* perm,
                                   int32_t* info, cudaStream_t s) {
  if (n > MP_MAX_N)
    return fail(GPTQ_ERR_UNSUPPORTED, "min-pivot order: n=%lld > %d", (long long)n, MP_MAX_N);
  double* d = scratch;
  double* Lp = scratch + align_up((size_t)n, 2);
  int32_t* elim = reinterpret_cast<int32_t*>(Lp + (size_t)n * MP_PANEL);
  const int64_t init = (n * n > n * MP_PANEL) ? n * n : n * MP_PANEL;
  GPTQ_LAUNCH(KK_PREP_ORDER, s, mp_init_kernel, (unsigned)ceil_div(init, 256), 256, 0, H, n,
              ld, mean, damp, S, d, Lp, info);
  const int64_t tiles = ceil_div(n, MP_TILE);
  // panel width: the widest of 32, 16, 8 whose columns fit in shared memory
  // beside d; past that, 32 columns kept in global memory
  const size_t dbytes = sizeof(double) * (size_t)((n + 1) & ~int64_t(1));
  const size_t budget = 224 * 1024;    // of the 227 KB a CTA may have
  int pw = MP_PANEL, lp_smem = 0;
  for (int w = MP_PANEL; w >= 8; w /= 2) {
    if (dbytes + sizeof(double) * (size_t)n * (w + 1) <= budget) { pw = w; lp_smem = 1; break; }
  }
  const size_t panel_smem = dbytes + (lp_smem ? sizeof(double) * (size_t)n * (pw + 1) : 0);
  if (panel_smem > 48 * 1024) {
    const gptq_status st = ensure_smem_limit((const void*)mp_panel_kernel, (int)panel_smem,
                                             "mp_panel_kernel");
    if (st != GPTQ_OK) return st;
  }
  for (int64_t t0 = 0; t0 < n; t0 += pw) {
    GPTQ_LAUNCH(KK_PREP_ORDER, s, mp_panel_kernel, 1, MP_THREADS, panel_smem, S, n, ld, d, Lp,
                elim, t0, pw, lp_smem, info);
    if (t0 + pw < n)
      GPTQ_LAUNCH(KK_PREP_ORDER, s, mp_trail_kernel, dim3((unsigned)tiles, (unsigned)tiles),
                  256, 0, S, n, ld, Lp, pw);
  }
  GPTQ_LAUNCH(KK_PREP_ORDER, s, mp_finish_kernel, (unsigned)ceil_div(n, 256), 256, 0, elim, n,
              perm);
  return GPTQ_OK;
}

}  // namespace gptq
