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
  double* D;      // N × NB × NB: L_kk⁻¹ of every diagonal tile
  int* sync;      // flags and counters of the dataflow factorisation
  size_t sync_bytes;
};

inline size_t sync_ints(int64_t N) { return 4 + (size_t)N + 4 * (size_t)N * (size_t)N; }

size_t prep_ws_layout(int64_t n, PrepWs* w, char* base) {
  const int64_t np = ceil_div(n, NB) * NB;
  const int64_t N = np / NB;
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
  size_t o_D = take(sizeof(double) * NB * NB * (size_t)N);
  size_t o_S = take(sizeof(int) * sync_ints(N));
  if (w && base) {
    w->mean = reinterpret_cast<double*>(base + o_mean);
    w->seen = reinterpret_cast<int32_t*>(base + o_seen);
    w->A = reinterpret_cast<double*>(base + o_A);
    w->M = reinterpret_cast<double*>(base + o_M);
    w->D = reinterpret_cast<double*>(base + o_D);
    w->sync = reinterpret_cast<int*>(base + o_S);
    w->sync_bytes = sizeof(int) * sync_ints(N);
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

// Diagonal tile: L_kk = chol(A_kk) and D = L_kk⁻¹, blocked by panels of 8
// columns so that the 64 dependent pivots cost 16 barriers instead of 64:
//   phase 1 (warp 0): factor the 8-column panel in registers (lane l owns rows
//            l and l + 32), pivots and multipliers exchanged by shuffles, and
//            finish the panel's 8 rows of D by forward substitution (lanes
//            over columns);
//   phase 2 (8 warps): rank-8 update of the trailing block of A and of the
//            rows of D below the panel.
// Pivots use rsqrt_pivot (Newton steps from the float32 estimate).
constexpr int DIAG_THREADS = 256;
constexpr int PW = 8;                         // panel width

// 1/sqrt(d) for a pivot d > 0 by Newton–Raphson on f(y) = y⁻² − d,
// y ← y·(3 − d·y²)/2, started from the float32 reciprocal-square-root estimate
// (≈ 2⁻²² relative); quadratic convergence gives float64 precision after two
// steps.  Much shorter on the critical path than a correctly rounded float64
// sqrt followed by a division.  Pivots outside the float32 range take the
// exact route.
__device__ __forceinline__ double rsqrt_pivot(double d) {
  if (d < 1e-30 || d > 1e30) return 1.0 / sqrt(d);
  double y = (double)rsqrtf((float)d);
  y = y * (1.5 - 0.5 * d * y * y);
  y = y * (1.5 - 0.5 * d * y * y);
  return y;
}

// Returns false (after reporting through info) when a pivot is not positive.
// Called by a whole CTA of DIAG_THREADS threads; sm holds 2·NB·LDT doubles.
__device__ bool diag_tile(double* __restrict__ A, double* __restrict__ M,
                          double* __restrict__ D, int64_t n, int64_t np, int k,
                          int32_t* info, double* sm) {
  double (*a)[LDT] = reinterpret_cast<double (*)[LDT]>(sm);
  double (*b)[LDT] = reinterpret_cast<double (*)[LDT]>(sm + NB * LDT);
  __shared__ int bad_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t base = (int64_t)k * NB;
  for (int e = tid; e < NB * NB; e += DIAG_THREADS) {
    const int r = e / NB, c = e % NB;
    a[r][c] = (c <= r) ? __ldcg(A + (base + r) * np + base + c) : 0.0;
    b[r][c] = (r == c) ? 1.0 : 0.0;
  }
  if (tid == 0) bad_s = 0;
  __syncthreads();

  for (int c0 = 0; c0 < NB; c0 += PW) {
    if (warp == 0) {
      // ---- phase 1: the panel, rows c0..63, columns c0..c0+7
      double v0[PW], v1[PW];                 // rows lane and lane + 32
#pragma unroll
      for (int c = 0; c < PW; ++c) {
        v0[c] = a[lane][c0 + c];
        v1[c] = a[lane + 32][c0 + c];
      }
      double ys[PW];
      bool bad = false;
#pragma unroll
      for (int c = 0; c < PW; ++c) {
        const int pr = c0 + c;
        const double mine = (pr < 32) ? v0[c] : v1[c];
        const double d = __shfl_sync(0xffffffffu, mine, pr & 31);
        if (!(d > 0.0) || !isfinite(d)) bad = true;
        const double y = (d > 0.0) ? rsqrt_pivot(d) : 0.0;
        ys[c] = y;
        // scale column c below the pivot; the pivot becomes sqrt(d)
        if (lane > pr) v0[c] *= y;
        else if (lane == pr) v0[c] = d * y;
        if (lane + 32 > pr) v1[c] *= y;
        else if (lane + 32 == pr) v1[c] = d * y;
        // update the panel's later columns
#pragma unroll
        for (int cc = c + 1; cc < PW; ++cc) {
          const int rr = c0 + cc;                     // row whose multiplier we need
          const double own = (rr < 32) ? v0[c] : v1[c];
          const double lk = __shfl_sync(0xffffffffu, own, rr & 31);
          if (lane >= rr) v0[cc] -= v0[c] * lk;
          if (lane + 32 >= rr) v1[cc] -= v1[c] * lk;
        }
      }
      if (bad) {
        if (lane == 0) {
          bad_s = 1;
          report(info, GPTQ_ERR_NOT_PD, n - 1 - (base + c0));
        }
      }
#pragma unroll
      for (int c = 0; c < PW; ++c) {
        if (lane >= c0) a[lane][c0 + c] = v0[c];
        if (lane + 32 >= c0) a[lane + 32][c0 + c] = v1[c];
      }
      __syncwarp();
      // panel rows of D: forward substitution over the panel, lanes over x
#pragma unroll
      for (int c = 0; c < PW; ++c) {
        const int pr = c0 + c;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int x = lane + 32 * h;
          if (x <= pr) {
            double acc = b[pr][x];
#pragma unroll
            for (int cp = 0; cp < c; ++cp) acc -= a[pr][c0 + cp] * b[c0 + cp][x];
            b[pr][x] = acc * ys[c];
          }
        }
        __syncwarp();
      }
    }
    __syncthreads();
    if (bad_s) return false;
    // ---- phase 2: rank-8 update of rows below the panel
    const int rs = c0 + PW;
    for (int r = rs + warp; r < NB; r += DIAG_THREADS / 32) {
      double lr[PW];
#pragma unroll
      for (int c = 0; c < PW; ++c) lr[c] = a[r][c0 + c];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int x = lane + 32 * h;
        if (x >= rs) {
          if (x <= r) {
            double acc = a[r][x];
#pragma unroll
            for (int c = 0; c < PW; ++c) acc -= lr[c] * a[x][c0 + c];
            a[r][x] = acc;
          }
        } else {
          double acc = b[r][x];
#pragma unroll
          for (int c = 0; c < PW; ++c) acc -= lr[c] * b[c0 + c][x];
          b[r][x] = acc;
        }
      }
    }
    __syncthreads();
  }

  for (int e = tid; e < NB * NB; e += DIAG_THREADS) {
    const int r = e / NB, c = e % NB;
    if (c <= r) A[(base + r) * np + base + c] = a[r][c];
    M[(base + r) * np + base + c] = b[r][c];
    D[e] = b[r][c];
  }
  return true;
}

// 64×64 float64 tile products on the float64 tensor cores (DMMA,
// mma.sync m8n8k4).  Tiles sit in shared memory with a row stride of 68
// doubles, which spreads the fragment reads over all banks.  Warp w owns rows
// 16·(w/2) .. +16 and columns 32·(w%2) .. +32 of C: 2 × 4 accumulator tiles
// of 8×8, two doubles per thread each (row g = lane/4, columns 2·(lane%4)+{0,1}).
constexpr int LDM = 68;

__device__ __forceinline__ void dmma_884(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

__device__ __forceinline__ void tile_mm(const double (*x)[LDM], const double (*y)[LDM],
                                        double acc[2][4][2], int warp, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int rb = 16 * (warp >> 1), cb = 32 * (warp & 1);
#pragma unroll 4
  for (int q = 0; q < NB; q += 4) {
    double a[2], b[4];
#pragma unroll
    for (int i = 0; i < 2; ++i) a[i] = x[rb + 8 * i + g][q + t];
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = y[q + t][cb + 8 * j + g];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dmma_884(acc[i][j], a[i], b[j]);
  }
}

// out ±= C (sign = +1 stores C, −1 subtracts it), leading dimension ld.
template <bool SUBTRACT>
__device__ __forceinline__ void tile_store(double* out, int64_t ld, const double acc[2][4][2],
                                           int warp, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int rb = 16 * (warp >> 1), cb = 32 * (warp & 1);
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double2* p = reinterpret_cast<double2*>(out + (int64_t)(rb + 8 * i + g) * ld + cb + 8 * j + 2 * t);
      double2 v;
      if (SUBTRACT) {
        v = __ldcg(p);
        v.x -= acc[i][j][0];
        v.y -= acc[i][j][1];
      } else {
        v = make_double2(acc[i][j][0], acc[i][j][1]);
      }
      *p = v;
    }
}

// 64×64 float64 tile from global (leading dimension ld) into shared memory,
// optionally transposed; 16-byte loads (L2 only: tiles are rewritten by other
// CTAs of the same launch), all issued before the stores.
__device__ __forceinline__ void load_tile(double (*dst)[LDM], const double* src,
                                          int64_t ld, bool transpose, int tid) {
  double2 buf[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = tid + 256 * k;            // 2048 pairs
    const int r = e >> 5, c2 = (e & 31) * 2;
    buf[k] = __ldcg(reinterpret_cast<const double2*>(src + (int64_t)r * ld + c2));
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = tid + 256 * k;
    const int r = e >> 5, c2 = (e & 31) * 2;
    if (transpose) {
      dst[c2][r] = buf[k].x;
      dst[c2 + 1][r] = buf[k].y;
    } else {
      dst[r][c2] = buf[k].x;
      dst[r][c2 + 1] = buf[k].y;
    }
  }
}

// ---------------------------------------------------------------------------
// The factorisation as one persistent, dataflow launch.
//
// Tasks of step k (64-column block k), in the fixed global order in which the
// workers take them (critical ones first, so step k+1 can start while step k
// is still updating far tiles):
//   PANEL(k,k+1), TRAIL(k,k+1,k+1), PANEL(k,i) i > k+1, TRAIL(k,i,k+1),
//   MROW(k,c) c < k, MTRAIL(k,k+1,c), TRAIL(k,i,j) k+1 < j ≤ i, MTRAIL(k,i,c)
// with PANEL:  L_ik = A_ik·D_kᵀ          (needs D_k and tile (i,k) updated k times)
//      MROW:   M_kc = D_k·M_kc           (needs D_k and M_kc updated k−c times)
//      TRAIL:  A_ij −= L_ik·L_jkᵀ         (needs L_ik, L_jk, tile (i,j) updated k times)
//      MTRAIL: M_ic −= L_ik·M_kc          (needs L_ik, final M_kc, M_ic updated k−c times)
// and DIAG(k) — L_kk = chol(A_kk), D_k = L_kk⁻¹ — run by the first CTA to
// arrive (its instruction cache stays warm across the chain of diagonal
// tiles) once tile (k,k) has received its k updates.  Every dependency of a
// task is an earlier task, and tasks are taken in order only by running
// CTAs, so the launch needs no co-residency guarantee.  Flags are set with
// release stores after a fence and polled with acquire loads; every wait is
// bounded and a time-out (or a bad pivot) raises a shared abort flag.
// ---------------------------------------------------------------------------
constexpr uint32_t kSpinLimit = 1u << 22;   // ≈ a few seconds with the back-off below

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct CholSync {
  int* ctrl;        // [0] next task, [1] arrivals, [2] abort
  int* diag_done;   // N
  int* pdone;       // N·N: pdone[k·N + i], L_ik final
  int* mdone;       // N·N: mdone[k·N + c], M_kc final
  int* upd;         // N·N: updates applied to A tile (i, j)
  int* mupd;        // N·N: updates applied to M tile (i, c)
};

__device__ CholSync sync_view(int* base, int N) {
  CholSync s;
  s.ctrl = base;
  s.diag_done = base + 4;
  s.pdone = s.diag_done + N;
  s.mdone = s.pdone + N * N;
  s.upd = s.mdone + N * N;
  s.mupd = s.upd + N * N;
  return s;
}

// Whole-CTA bounded wait for *flag ≥ target; false on abort or time-out.
__device__ bool cta_wait(const int* flag, int target, int* abortp, int32_t* info, int* s_ok) {
  if (threadIdx.x == 0) {
    bool ok = false;
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
      if (ld_acquire(flag) >= target) { ok = true; break; }
      if (*reinterpret_cast<volatile int*>(abortp)) break;
      if (it > 32) __nanosleep(64);
    }
    if (!ok && !*reinterpret_cast<volatile int*>(abortp)) {
      report(info, GPTQ_ERR_TIMEOUT, target);
      atomicExch(abortp, 1);
    }
    *s_ok = ok ? 1 : 0;
  }
  __syncthreads();
  const bool ok = *s_ok != 0;
  __syncthreads();
  return ok;
}

__device__ __forceinline__ void cta_signal(int* flag, int value) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    st_release(flag, value);
  }
}

__host__ __device__ inline int step_tasks(int N, int k) {
  const int r = N - k - 1;
  if (r <= 0) return k;                              // MROW only
  return 2 + 2 * (r - 1) + k + (k + 1) + (r - 1) * r / 2 + (r - 1) * (k + 1);
}

int total_tasks(int N) {
  int t = 0;
  for (int k = 0; k < N; ++k) t += step_tasks(N, k);
  return t;
}

enum TaskKind { T_PANEL = 0, T_MROW, T_TRAIL, T_MTRAIL };

__device__ void decode_task(int task, int N, int& kind, int& k, int& i, int& j) {
  k = 0;
  while (task >= step_tasks(N, k)) { task -= step_tasks(N, k); ++k; }
  const int r = N - k - 1;
  if (r <= 0) { kind = T_MROW; i = k; j = task; return; }
  if (task < 1) { kind = T_PANEL; i = k + 1; j = k; return; }
  task -= 1;
  if (task < 1) { kind = T_TRAIL; i = k + 1; j = k + 1; return; }
  task -= 1;
  if (task < r - 1) { kind = T_PANEL; i = k + 2 + task; j = k; return; }
  task -= r - 1;
  if (task < r - 1) { kind = T_TRAIL; i = k + 2 + task; j = k + 1; return; }
  task -= r - 1;
  if (task < k) { kind = T_MROW; i = k; j = task; return; }
  task -= k;
  if (task < k + 1) { kind = T_MTRAIL; i = k + 1; j = task; return; }
  task -= k + 1;
  if (task < (r - 1) * r / 2) {
    int ii = 0;
    while (task >= ii + 1) { task -= ii + 1; ++ii; }
    kind = T_TRAIL; i = k + 2 + ii; j = k + 2 + task; return;
  }
  task -= (r - 1) * r / 2;
  kind = T_MTRAIL; i = k + 2 + task / (k + 1); j = task % (k + 1);
}

__global__ void __launch_bounds__(256)
chol_persistent_kernel(double* __restrict__ A, double* __restrict__ M,
                       double* __restrict__ Dall, int64_t n, int64_t np, int N,
                       int ntasks, int* sync_base, int32_t* info) {
  extern __shared__ double sm[];
  __shared__ int s_role, s_task, s_ok;
  const CholSync S = sync_view(sync_base, N);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) s_role = atomicAdd(&S.ctrl[1], 1);
  __syncthreads();
  if (*reinterpret_cast<volatile int32_t*>(info) != 0) return;

  if (s_role == 0) {
    // ---- the chain of diagonal tiles
    for (int k = 0; k < N; ++k) {
      if (!cta_wait(&S.upd[k * N + k], k, &S.ctrl[2], info, &s_ok)) return;
      if (!diag_tile(A, M, Dall + (size_t)k * NB * NB, n, np, k, info, sm)) {
        if (tid == 0) atomicExch(&S.ctrl[2], 1);
        return;
      }
      cta_signal(&S.diag_done[k], 1);
    }
    return;
  }

  double (*x)[LDM] = reinterpret_cast<double (*)[LDM]>(sm);
  double (*y)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + NB * LDM);
  for (;;) {
    if (tid == 0) s_task = atomicAdd(&S.ctrl[0], 1);
    __syncthreads();
    const int task = s_task;
    __syncthreads();
    if (task >= ntasks || *reinterpret_cast<volatile int*>(&S.ctrl[2])) return;
    int kind, k, i, j;
    decode_task(task, N, kind, k, i, j);
    double acc[2][4][2] = {};
    if (kind == T_PANEL) {
      if (!cta_wait(&S.diag_done[k], 1, &S.ctrl[2], info, &s_ok)) return;
      if (!cta_wait(&S.upd[i * N + k], k, &S.ctrl[2], info, &s_ok)) return;
      double* out = A + (int64_t)i * NB * np + (int64_t)k * NB;
      load_tile(x, out, np, false, tid);
      load_tile(y, Dall + (size_t)k * NB * NB, NB, true, tid);
      __syncthreads();
      tile_mm(x, y, acc, warp, lane);
      tile_store<false>(out, np, acc, warp, lane);
      cta_signal(&S.pdone[k * N + i], 1);
    } else if (kind == T_MROW) {
      const int c = j;
      if (!cta_wait(&S.diag_done[k], 1, &S.ctrl[2], info, &s_ok)) return;
      if (!cta_wait(&S.mupd[k * N + c], k - c, &S.ctrl[2], info, &s_ok)) return;
      double* out = M + (int64_t)k * NB * np + (int64_t)c * NB;
      load_tile(x, Dall + (size_t)k * NB * NB, NB, false, tid);
      load_tile(y, out, np, false, tid);
      __syncthreads();
      tile_mm(x, y, acc, warp, lane);
      tile_store<false>(out, np, acc, warp, lane);
      cta_signal(&S.mdone[k * N + c], 1);
    } else if (kind == T_TRAIL) {
      if (!cta_wait(&S.pdone[k * N + i], 1, &S.ctrl[2], info, &s_ok)) return;
      if (j != i && !cta_wait(&S.pdone[k * N + j], 1, &S.ctrl[2], info, &s_ok)) return;
      if (!cta_wait(&S.upd[i * N + j], k, &S.ctrl[2], info, &s_ok)) return;
      double* out = A + (int64_t)i * NB * np + (int64_t)j * NB;
      load_tile(x, A + (int64_t)i * NB * np + (int64_t)k * NB, np, false, tid);
      load_tile(y, A + (int64_t)j * NB * np + (int64_t)k * NB, np, true, tid);
      __syncthreads();
      tile_mm(x, y, acc, warp, lane);
      tile_store<true>(out, np, acc, warp, lane);
      cta_signal(&S.upd[i * N + j], k + 1);
    } else {   // T_MTRAIL
      const int c = j;
      if (!cta_wait(&S.pdone[k * N + i], 1, &S.ctrl[2], info, &s_ok)) return;
      if (c < k) {
        if (!cta_wait(&S.mdone[k * N + c], 1, &S.ctrl[2], info, &s_ok)) return;
      } else if (!cta_wait(&S.diag_done[k], 1, &S.ctrl[2], info, &s_ok)) {
        return;
      }
      if (!cta_wait(&S.mupd[i * N + c], k - c, &S.ctrl[2], info, &s_ok)) return;
      double* out = M + (int64_t)i * NB * np + (int64_t)c * NB;
      load_tile(x, A + (int64_t)i * NB * np + (int64_t)k * NB, np, false, tid);
      load_tile(y, M + (int64_t)k * NB * np + (int64_t)c * NB, np, false, tid);
      __syncthreads();
      tile_mm(x, y, acc, warp, lane);
      tile_store<true>(out, np, acc, warp, lane);
      cta_signal(&S.mupd[i * N + c], k - c + 1);
    }
  }
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
int g_num_sms = 148;

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
  const size_t tile_smem = 2 * NB * LDM * sizeof(double);   // ≥ the diagonal tile's 2·NB·LDT
  if (!g_smem_set) {
    GPTQ_CUDA(cudaFuncSetAttribute(chol_persistent_kernel,
              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem));
    int dev = 0;
    GPTQ_CUDA(cudaGetDevice(&dev));
    GPTQ_CUDA(cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev));
    g_smem_set = true;
  }

  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  GPTQ_CUDA(cudaMemsetAsync(w.sync, 0, w.sync_bytes, s));
  if (order == GPTQ_ORDER_CUSTOM)
    GPTQ_CUDA(cudaMemsetAsync(w.seen, 0, sizeof(int32_t) * n, s));
  GPTQ_LAUNCH(KK_PREP_STATS, s, prep_stats_kernel, 1, 1024, 0, H, n, dead, w.mean, info);
  GPTQ_LAUNCH(KK_PREP_ORDER, s, prep_order_kernel, (int)ceil_div(n, 256), 256, 0,
              H, n, order, perm, w.seen, info);
  GPTQ_LAUNCH(KK_PREP_GATHER, s, prep_gather_kernel, (unsigned)ceil_div(np * np, 256),
              256, 0, H, n, np, perm, w.seen, order == GPTQ_ORDER_CUSTOM ? 1 : 0,
              w.mean, damp, w.A, w.M, info);
  const int ntasks = total_tasks(N);
  const int grid = (ntasks + 1 < 2 * g_num_sms) ? ntasks + 1 : 2 * g_num_sms;
  GPTQ_LAUNCH(KK_CHOL, s, chol_persistent_kernel, grid, 256, tile_smem, w.A, w.M, w.D, n, np,
              N, ntasks, w.sync, info);
  GPTQ_LAUNCH(KK_PREP_OUT, s, prep_out_kernel, (unsigned)ceil_div(n * n, 256), 256, 0,
              w.M, n, np, U);
  return GPTQ_OK;
}

// ---------------------------------------------------------------------------
// gptq_prepare_noalloc: gptq_prepare on a scratch area that lives in the
// library itself, for callers that cannot hand over device memory.
// ---------------------------------------------------------------------------
#include <mutex>

namespace gptq {
namespace {

constexpr int64_t kNoAllocMaxN = GPTQ_NOALLOC_MAX_N;
constexpr size_t up256(size_t x) { return (x + 255) / 256 * 256; }
// Same arithmetic as prep_ws_layout() for n = kNoAllocMaxN (a multiple of 64).
constexpr int64_t kNoAllocN = kNoAllocMaxN / NB;
constexpr size_t kNoAllocBytes =
    up256(sizeof(double)) + up256(sizeof(int32_t) * kNoAllocMaxN) +
    2 * up256(sizeof(double) * kNoAllocMaxN * kNoAllocMaxN) +
    up256(sizeof(double) * NB * NB * kNoAllocN) +
    up256(sizeof(int) * (4 + kNoAllocN + 4 * kNoAllocN * kNoAllocN));
static_assert(kNoAllocMaxN % NB == 0, "the fixed limit is a whole number of tiles");

// The scratch itself: every GPU that loads this library holds it until the
// process exits.  All calls on one device share it.
static __device__ __align__(256) unsigned char g_prepare_scratch[kNoAllocBytes];

std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 128;
void* g_noalloc_ptr[kMaxDevices] = {};

}  // namespace
}  // namespace gptq

extern "C" gptq_status gptq_prepare_noalloc(const float* H, int64_t n, double damp, int order,
                                            int32_t* perm, float* U, uint8_t* dead,
                                            int32_t* info, void* stream) {
  if (n < 1 || n > kNoAllocMaxN)
    return fail(GPTQ_ERR_INVALID_ARG,
                "gptq_prepare_noalloc: n=%lld is outside 1..%lld, the size of the library's "
                "fixed scratch; use gptq_prepare with a caller workspace",
                (long long)n, (long long)kNoAllocMaxN);
  if (prep_ws_layout(n, nullptr, nullptr) > sizeof(g_prepare_scratch))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare_noalloc: scratch layout exceeds the array");
  int dev = 0;
  GPTQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare_noalloc: device ordinal %d", dev);
  void* scratch = nullptr;
  {
    // Once per device, with that device current: the device address of the
    // array (host code only sees a stand-in symbol, not a device pointer).
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    scratch = g_noalloc_ptr[dev];
    if (scratch == nullptr) {
      cudaError_t e = cudaGetSymbolAddress(&scratch, g_prepare_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_prepare_scratch)");
      g_noalloc_ptr[dev] = scratch;
    }
  }
  return gptq_prepare(H, n, damp, order, perm, U, dead, info, scratch,
                      sizeof(g_prepare_scratch), stream);
}
