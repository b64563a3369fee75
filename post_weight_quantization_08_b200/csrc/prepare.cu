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
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "chol_tasks.cuh"
#include "minpivot.cuh"

namespace gptq {
namespace {

constexpr int NB = 64;          // float64 tile edge

struct PrepWs {
  double* mean;   // 1
  int32_t* seen;  // n (custom-order check)
  double* A;      // np × np
  double* M;      // np × np
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
  size_t o_S = take(sizeof(int) * sync_ints(N));
  if (w && base) {
    w->mean = reinterpret_cast<double*>(base + o_mean);
    w->seen = reinterpret_cast<int32_t*>(base + o_seen);
    w->A = reinterpret_cast<double*>(base + o_A);
    w->M = reinterpret_cast<double*>(base + o_M);
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

// Float64 tensor-core products (DMMA, mma.sync m8n8k4).  Shared-memory tiles
// have a row stride of 68 doubles, which spreads the fragment reads of a warp
// over all banks and keeps every row 16-byte aligned.  Fragment layout of an
// 8×8×4 product: lane = 4·g + t holds A[g][t], B[t][g] and C[g][2t], C[g][2t+1].
constexpr int LDM = 68;
// Worker groups of 4 warps per CTA, the launch's threads, and the shared
// memory before the slot prefix: the chain's five tiles and 192 doubles, or
// two tiles per worker group.
constexpr int kGroups = 3;
constexpr int kCholThreads = 128 * kGroups;
constexpr int kTileDoubles = (5 * NB * LDM + 192 > 2 * kGroups * NB * LDM) ? 5 * NB * LDM + 192
                                                                            : 2 * kGroups * NB * LDM;

__device__ __forceinline__ void dmma_884(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// Lower-triangle 8×8 blocks (I, J), J ≤ I < 8, row by row (e = I·(I+1)/2 + J).
__constant__ unsigned char kTri8I[36] = {0, 1, 1, 2, 2, 2, 3, 3, 3, 3, 4, 4, 4, 4, 4, 5, 5, 5,
                                         5, 5, 5, 6, 6, 6, 6, 6, 6, 6, 7, 7, 7, 7, 7, 7, 7, 7};
__constant__ unsigned char kTri8J[36] = {0, 0, 1, 0, 1, 2, 0, 1, 2, 3, 0, 1, 2, 3, 4, 0, 1, 2,
                                         3, 4, 5, 0, 1, 2, 3, 4, 5, 6, 0, 1, 2, 3, 4, 5, 6, 7};

// Polls a bounded wait makes before it reports GPTQ_ERR_TIMEOUT (≈ a few
// seconds with the back-off below); gptq_set_wait_limit() may lower it.
constexpr uint32_t kSpinLimit = 1u << 22;

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Tiles the otherwise idle warp 4 of the diagonal tile fetches ahead: a tile
// is final once *flag ≥ target; up to two 64×64 float64 tiles (leading
// dimension ld) into shared memory.
struct TilePrefetch {
  const int* flag[2];
  int target[2];
  const double* src[2];
  double (*dst[2])[LDM];
  int64_t ld;
  int count;
  uint32_t spin;     // polls before the prefetcher leaves the tiles to the panel phase
};

// The panel of the step before, still in shared memory (src), goes to global
// memory (dst, leading dimension ld) at the start of the diagonal tile, and
// *flag is released once it is there; dst = nullptr: none.
struct PanelOut {
  const double (*src)[LDM];
  double* dst;
  int* flag;
};

// Named barriers of the diagonal tile (0 is the chain's CTA-wide barrier): 1 joins the six
// working warps (1–3, 5–7); 2 hands X and the next panel block from warp 0 to
// them; 3 hands their finished trailing updates back to warp 0; 4 tells warp 4
// that they have stored the panel of the step before; 5 joins warps 0–3 and
// 5–7 in the panel phase after the diagonal tile (warp 4 publishes the tile
// meanwhile); 6 tells them there that warp 4's prefetched tiles have landed.
// Warp 4 shares warp 0's scheduler and stays out of 1–3 and 5.
constexpr int kBarRest = 1, kBarX = 2, kBarDone = 3, kBarPanel = 4, kBarChain = 5, kBarFetch = 6;
constexpr int kRest = 192, kHand = 224;     // 6 working warps; + warp 0

__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// The chain runs on the first 256 threads of its CTA (the launch has
// kCholThreads; the rest of the chain CTA leaves at once): barrier 0 with
// that count stands for __syncthreads on the chain's path.
constexpr int kChainThreads = 256;
__device__ __forceinline__ void chain_sync() {
  asm volatile("bar.sync 0, %0;" ::"n"(kChainThreads) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id, int count) {
  __threadfence_block();
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// C (8×8 at c, row stride LDM) ±= X·Yᵀ for 8×8 blocks X, Y at x, y (row stride
// ldx, ldy): two k-steps of the float64 tensor-core product.  Operands are
// loaded before the products, so C may alias X.
template <bool SUBTRACT, bool ACCUMULATE>
__device__ __forceinline__ void block8_nt(double* c, const double* x, int ldx,
                                          const double* y, int ldy, int lane) {
  const int g = lane >> 2, t = lane & 3;
  double2* cp = reinterpret_cast<double2*>(c + g * LDM + 2 * t);
  double acc[2] = {0.0, 0.0};
  if (ACCUMULATE) {
    const double2 cv = *cp;
    acc[0] = cv.x;
    acc[1] = cv.y;
  }
  const double x0 = x[g * ldx + t], x1 = x[g * ldx + 4 + t];
  const double y0 = y[g * ldy + t], y1 = y[g * ldy + 4 + t];
  dmma_884(acc, SUBTRACT ? -x0 : x0, y0);
  dmma_884(acc, SUBTRACT ? -x1 : x1, y1);
  *cp = make_double2(acc[0], acc[1]);
}

// C (8×8 at c) = X·B for X 8×8 row-major with stride 8 and B 8×8 at b (row
// stride LDM); C may alias B.
__device__ __forceinline__ void block8_xb(double* c, const double* X, const double* b, int lane) {
  const int g = lane >> 2, t = lane & 3;
  double acc[2] = {0.0, 0.0};
  const double b0 = b[t * LDM + g], b1 = b[(4 + t) * LDM + g];
  dmma_884(acc, X[g * 8 + t], b0);
  dmma_884(acc, X[g * 8 + 4 + t], b1);
  *reinterpret_cast<double2*>(c + g * LDM + 2 * t) = make_double2(acc[0], acc[1]);
}

constexpr double kMinNormal = 2.2250738585072014e-308;
constexpr double kMaxFinite = 1.7976931348623157e308;

// Cholesky of an 8×8 block held (lower triangle, packed row by row) in the
// registers of every lane of one warp, two pivots at a time: for the leading
// 2×2 block [[d, b], [b, c]] with det = d·c − b², the two reciprocal square
// roots 1/√d and 1/√det are independent, and 1/L₁₁ = √d/√det.  Lane j also
// builds column j (j = lane mod 8) of X = L⁻¹ by forward substitution as the
// pivots appear, X[i][j] = −(1/L_ii)·Σ_{j≤m<i} L[i][m]·X[m][j].  Returns the
// first pivot position whose pivot (or 2×2 determinant) is not a positive
// normal float64, else 8.
__device__ __forceinline__ int chol8_pairs(double (&l)[36], double (&x)[8], int lane) {
  const int jc = lane & 7;
  int badp = 8;
#pragma unroll
  for (int p = 0; p < 8; p += 2) {
    const int P0 = p * (p + 1) / 2, P1 = (p + 1) * (p + 2) / 2;
    const double d1 = l[P0 + p], bb = l[P1 + p], cc = l[P1 + p + 1];
    const double det = fma(d1, cc, -bb * bb);
    const bool ok1 = d1 >= kMinNormal && d1 <= kMaxFinite;
    const bool ok2 = det >= kMinNormal && det <= kMaxFinite;
    badp = (badp == 8 && !ok1) ? p : ((badp == 8 && !ok2) ? p + 1 : badp);
    const double y1 = ok1 ? rsqrt(d1) : 0.0;
    const double z = ok2 ? rsqrt(det) : 0.0;
    const double s1 = d1 * y1;
    const double lb = bb * y1;
    const double y2 = s1 * z;
    double s = 0.0;
#pragma unroll
    for (int m = 0; m < p; ++m) s = fma(l[P0 + m], x[m], s);
    x[p] = (p == jc) ? y1 : ((p < jc) ? 0.0 : -y1 * s);
    double s2 = lb * x[p];
#pragma unroll
    for (int m = 0; m < p; ++m) s2 = fma(l[P1 + m], x[m], s2);
    x[p + 1] = (p + 1 == jc) ? y2 : ((p + 1 < jc) ? 0.0 : -y2 * s2);
    l[P0 + p] = s1;
    l[P1 + p] = lb;
    l[P1 + p + 1] = (det * z) * y1;
#pragma unroll
    for (int i = p + 2; i < 8; ++i) {
      const int I = i * (i + 1) / 2;
      const double li0 = l[I + p] * y1;
      l[I + p] = li0;
      l[I + p + 1] = fma(-li0, lb, l[I + p + 1]) * y2;
    }
#pragma unroll
    for (int i = p + 2; i < 8; ++i)
#pragma unroll
      for (int j = p + 2; j <= i; ++j) {
        const int I = i * (i + 1) / 2, J = j * (j + 1) / 2;
        l[I + j] = fma(-l[I + p], l[J + p], fma(-l[I + p + 1], l[J + p + 1], l[I + j]));
      }
  }
  return badp;
}

// Diagonal tile: D = L⁻¹ with L = chol(A) for a 64×64 tile in shared memory
// (a: lower triangle of A on entry, overwritten; b: zero on entry, D on
// exit; xs: 3 × 64 doubles), blocked by 8 columns and software-pipelined:
//   warp 0, step kb: Cholesky of the diagonal block kb (registers), X_kb =
//     its inverse; then, once the working warps have applied step kb−1 to block row
//     kb+1, the panel block L_{kb+1,kb} = A_{kb+1,kb}·X_kbᵀ and the diagonal
//     block A_{kb+1,kb+1} −= L_{kb+1,kb}·L_{kb+1,kb}ᵀ, so that step kb+1 can
//     start at once;
//   warps 1–3 and 5–7, step kb: the other panel blocks L_{I,kb} (I ≥ kb+2), the
//     other trailing blocks A_{IJ} −= L_{I,kb}·L_{J,kb}ᵀ, and block row kb of
//     D: D_{kb,J} = X_kb·D_{kb,J} (J < kb), D_{kb,kb} = X_kb, then
//     D_{IJ} −= L_{I,kb}·D_{kb,J} for I > kb, J ≤ kb (the elimination applied
//     to an identity matrix).
// Warp 4 shares warp 0's scheduler and float64 pipe, so it takes none of this
// work: it publishes the panel of the step before once the working warps have
// stored it (po, while warp 0 factors the first block), clears the blocks
// below the diagonal of bz (the D buffer of the step before, zero above the
// diagonal already), and fetches the tiles in pf.  Each block row of D goes
// out to dout (leading dimension ld) as soon as it is final.  All products
// are 8×8 blocks on the float64 tensor cores.  A bad pivot is
// reported through info (the factorisation runs to the end on zeros, so that
// every barrier is met) and makes the function return false.  Called by a
// whole CTA of 256 threads.
__device__ __forceinline__ bool diag_tile_smem(double (*a)[LDM], double (*b)[LDM], double (*bz)[LDM],
                               double* xs, double* __restrict__ dout, int64_t ld, int64_t n,
                               int64_t base, int32_t* info, int* bad_s, const TilePrefetch& pf,
                               const PanelOut& po, volatile int* s_stop, int* s_got) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  if (tid == 0) {
    *s_stop = 0;
    *s_got = 0;
  }
  chain_sync();
  if (warp == 0) {
    double l[36];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j <= i; ++j) l[i * (i + 1) / 2 + j] = a[i][j];
    int bad = 8 * 8;
    for (int kb = 0; kb < 8; ++kb) {
      const int c0 = 8 * kb;
      double x[8];
      const int badp = chol8_pairs(l, x, lane);
      bad = (bad == 64 && badp < 8) ? c0 + badp : bad;
      double* X = xs + 64 * (kb % 3);   // warp 0 runs up to two steps ahead of the readers
      if (lane < 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) X[i * 8 + lane] = x[i];
      }
      __syncwarp();
      // warps 1–7 have applied step kb−1 (and so have all passed barrier X
      // of step kb−1: no arrival below can fall into an older generation)
      if (kb > 0) bar_sync(kBarDone, kHand);
      if (kb < 7) {
        const int r1 = c0 + 8;
        block8_nt<false, false>(&a[r1][c0], &a[r1][c0], LDM, X, 8, lane);
        __syncwarp();
        block8_nt<true, true>(&a[r1][r1], &a[r1][c0], LDM, &a[r1][c0], LDM, lane);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j <= i; ++j) l[i * (i + 1) / 2 + j] = a[r1 + i][r1 + j];
      }
      bar_arrive(kBarX, kHand);                        // X_kb and L_{kb+1,kb} ready
    }
    if (lane == 0) *s_stop = 1;                        // the prefetcher may give up now
    if (lane == 0 && bad < 64) {
      *bad_s = 1;
      report(info, GPTQ_ERR_NOT_PD, n - 1 - (base + bad));
    }
  } else if (warp == 4) {
    // The prefetcher: each tile of pf as soon as its flag says it is final
    // (lane 0 polls with acquire loads; the copies are cp.async through L2),
    // until both are issued or warp 0 is done.  s_got says which were issued:
    // the master copies the others itself.
    if (po.dst) {
      bar_sync(kBarPanel, kHand);       // the working warps have stored it
      if (lane == 0) {
        __threadfence();
        st_release(po.flag, 1);
      }
      __syncwarp();
    }
    if (bz) {
#pragma unroll 4
      for (int r = 8; r < NB; ++r)
        if (lane < 4 * (r >> 3))
          *reinterpret_cast<double2*>(&bz[r][2 * lane]) = make_double2(0.0, 0.0);
    }
    int got = 0;
    const int all = (1 << pf.count) - 1;
    for (uint32_t it = 0; it < pf.spin && got != all; ++it) {
      int ready = 0;
      if (lane == 0) {
        for (int t2 = 0; t2 < pf.count; ++t2)
          if (!((got >> t2) & 1) && ld_acquire(pf.flag[t2]) >= pf.target[t2]) ready |= 1 << t2;
      }
      ready = __shfl_sync(0xffffffffu, ready, 0);
      __syncwarp();
      for (int t2 = 0; t2 < pf.count; ++t2) {
        if (!((ready >> t2) & 1)) continue;
        for (int r = 0; r < NB; ++r) {
          const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(&pf.dst[t2][r][2 * lane]));
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d),
                       "l"(pf.src[t2] + (int64_t)r * pf.ld + 2 * lane)
                       : "memory");
        }
        got |= 1 << t2;
      }
      if (got == all || *s_stop) break;
      __nanosleep(128);
    }
    // the copies land while the panel phase starts: warp 4 waits for them
    // there and announces them on barrier kBarFetch
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (lane == 0) *s_got = got;
  } else {
    // v numbers the six working warps (warp 4 prefetches)
    const int v = (warp < 4) ? warp - 1 : warp - 2;
    if (po.dst) {
      for (int e = 32 * v + lane; e < NB * NB / 2; e += 192) {
        const int r = e >> 5, c = (e & 31) * 2;
        *reinterpret_cast<double2*>(po.dst + (int64_t)r * ld + c) =
            *reinterpret_cast<const double2*>(&po.src[r][c]);
      }
      bar_arrive(kBarPanel, kHand);
    }
    for (int kb = 0; kb < 8; ++kb) {
      const int c0 = 8 * kb;
      const double* X = xs + 64 * (kb % 3);
      bar_sync(kBarX, kHand);
      // panel blocks I ≥ kb + 2
      if (v >= 0 && kb + 2 + v < 8) {
        const int r = 8 * (kb + 2 + v);
        block8_nt<false, false>(&a[r][c0], &a[r][c0], LDM, X, 8, lane);
      }
      bar_sync(kBarRest, kRest);
      // trailing blocks kb+1 ≤ J ≤ I ≤ 7 except (kb+1, kb+1); operands first
      const int rem = 7 - kb;
      const int nblk = rem * (rem + 1) / 2;
      double2 cv[5];
      double f[5][4];
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int e = 1 + v + 6 * s;
        if (v >= 0 && e < nblk) {
          const int bi = kb + 1 + kTri8I[e], bj = kb + 1 + kTri8J[e];
          cv[s] = *reinterpret_cast<const double2*>(&a[8 * bi + g][8 * bj + 2 * q]);
          f[s][0] = a[8 * bi + g][c0 + q];
          f[s][1] = a[8 * bi + g][c0 + 4 + q];
          f[s][2] = a[8 * bj + g][c0 + q];
          f[s][3] = a[8 * bj + g][c0 + 4 + q];
        }
      }
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int e = 1 + v + 6 * s;
        if (v >= 0 && e < nblk) {
          const int bi = kb + 1 + kTri8I[e], bj = kb + 1 + kTri8J[e];
          double acc[2] = {cv[s].x, cv[s].y};
          dmma_884(acc, -f[s][0], f[s][2]);
          dmma_884(acc, -f[s][1], f[s][3]);
          *reinterpret_cast<double2*>(&a[8 * bi + g][8 * bj + 2 * q]) = make_double2(acc[0], acc[1]);
        }
      }
      if (kb < 7) bar_arrive(kBarDone, kHand);         // warp 0 waits for steps 0..6
      // block row kb of D
      if (v >= 0) {
        for (int J = v; J < kb; J += 6) block8_xb(&b[c0][8 * J], X, &b[c0][8 * J], lane);
      }
      if (v == 5) {
        for (int e = lane; e < 64; e += 32) b[c0 + (e >> 3)][c0 + (e & 7)] = X[e];
      }
      bar_sync(kBarRest, kRest);
      // block row kb of D is final: out to global memory now, so that little
      // is left in flight when the tile is published
      if (v >= 0) {
        for (int e = 32 * v + lane; e < 256; e += 192) {
          const int r = c0 + (e >> 5), c = (e & 31) * 2;
          *reinterpret_cast<double2*>(dout + (int64_t)r * ld + c) =
              *reinterpret_cast<const double2*>(&b[r][c]);
        }
      }
      // D_{IJ} −= L_{I,kb}·D_{kb,J}, I > kb, J ≤ kb
      const int ncol = kb + 1;
      for (int e = (v >= 0 ? v : rem * ncol); e < rem * ncol; e += 6) {
        const int I = kb + 1 + e / ncol, J = e % ncol;
        double2* cp = reinterpret_cast<double2*>(&b[8 * I + g][8 * J + 2 * q]);
        const double2 c2 = *cp;
        double acc[2] = {c2.x, c2.y};
        dmma_884(acc, -a[8 * I + g][c0 + q], b[c0 + q][8 * J + g]);
        dmma_884(acc, -a[8 * I + g][c0 + 4 + q], b[c0 + 4 + q][8 * J + g]);
        *cp = make_double2(acc[0], acc[1]);
      }
    }
  }
  chain_sync();
  return *bad_s == 0;
}

// 64×64 tile loads into shared memory: the lower triangle (zeros above), and
// zeros.  16-byte loads through L2 only (tiles are rewritten by other CTAs of
// the same launch).
__device__ __forceinline__ void load_lower(double (*dst)[LDM], const double* src, int64_t ld,
                                           int tid) {
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int e = tid + 256 * s;              // 2048 pairs
    const int r = e >> 5, c = (e & 31) * 2;
    const double2 v = __ldcg(reinterpret_cast<const double2*>(src + (int64_t)r * ld + c));
    *reinterpret_cast<double2*>(&dst[r][c]) = make_double2(c <= r ? v.x : 0.0, c + 1 <= r ? v.y : 0.0);
  }
}
__device__ __forceinline__ void zero_tile(double (*dst)[LDM], int tid) {
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int e = tid + 256 * s;
    *reinterpret_cast<double2*>(&dst[e >> 5][(e & 31) * 2]) = make_double2(0.0, 0.0);
  }
}
// Asynchronous 64×64 tile copies global → shared memory are 16-byte cp.async
// through L2 only (tiles are rewritten by other CTAs of the same launch).
__device__ __forceinline__ void copy_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// One tile, copied by the 224 threads of warps 0–3 and 5–7 (gt numbers them).
__device__ __forceinline__ void copy_tile_async_group(double (*dst)[LDM], const double* src,
                                                      int64_t ld, int gt) {
  for (int e = gt; e < NB * NB / 2; e += kHand) {
    const int r = e >> 5, c = (e & 31) * 2;
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(&dst[r][c]));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src + (int64_t)r * ld + c)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// L = A·Dᵀ for 64×64 shared-memory tiles with D lower triangular, so block
// column J of L needs only q < 8·(J+1).  Warp w owns row blocks 4·(w/4) .. +4
// and block columns J = w mod 4 and 7 − J, which gives every warp the same
// number of products (and every scheduler the same load).  acc[i][c] is
// block (4·(w/4) + i, c ? 7 − J : J).  The k-loops have compile-time bounds
// (one instance per J) and are unrolled, so that the fragment loads run ahead
// of the products and the float64 pipe stays busy.
template <int J, int NH>
__device__ __forceinline__ void panel_mm_j(const double (*x)[LDM], const double (*d)[LDM],
                                           double acc[2][4][2][2], int rb, int g, int t) {
  constexpr int J1 = 7 - J, qlo = 8 * (J + 1), qhi = 8 * (J1 + 1);
#pragma unroll
  for (int q = 0; q < qlo; q += 4) {
    double a[NH][4];
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) a[h][i] = x[rb + 32 * h + 8 * i + g][q + t];
    const double b0 = d[8 * J + g][q + t], b1 = d[8 * J1 + g][q + t];
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dmma_884(acc[h][i][0], a[h][i], b0);
        dmma_884(acc[h][i][1], a[h][i], b1);
      }
  }
#pragma unroll
  for (int q = qlo; q < qhi; q += 4) {
    double a[NH][4];
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) a[h][i] = x[rb + 32 * h + 8 * i + g][q + t];
    const double b1 = d[8 * J1 + g][q + t];
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) dmma_884(acc[h][i][1], a[h][i], b1);
  }
}
// The panel over warps 0–3 and 5–7: warp w ≠ 0 owns row blocks 4·(w/4) .. +4
// and block columns J = w mod 4 and 7 − J; warp 0 owns both row halves of
// J = 0 (what warps 0 and 4 would own), so that every scheduler keeps the
// same share.  acc[h] is row half h (warp 0) or the warp's only half (h = 0).
__device__ __forceinline__ void panel_mm(const double (*x)[LDM], const double (*d)[LDM],
                                         double acc[2][4][2][2], int warp, int lane) {
  const int g = lane >> 2, t = lane & 3, rb = 32 * (warp >> 2);
  switch (warp & 3) {
    case 0: panel_mm_j<0, 2>(x, d, acc, 0, g, t); break;      // warp 0: both halves
    case 1: panel_mm_j<1, 1>(x, d, acc, rb, g, t); break;
    case 2: panel_mm_j<2, 1>(x, d, acc, rb, g, t); break;
    default: panel_mm_j<3, 1>(x, d, acc, rb, g, t); break;
  }
}

// Writes the panel accumulators to a shared-memory tile (it goes to global
// memory from there later, off the chain).
__device__ __forceinline__ void panel_to_smem(double (*xs_)[LDM], const double acc[2][4][2][2],
                                              int warp, int lane) {
  const int g = lane >> 2, t = lane & 3, J = warp & 3;
  const int nh = (warp == 0) ? 2 : 1;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h >= nh) break;
    const int rb = (warp == 0) ? 32 * h : 32 * (warp >> 2);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int r = rb + 8 * i + g, col = 8 * (c ? 7 - J : J) + 2 * t;
        *reinterpret_cast<double2*>(&xs_[r][col]) = make_double2(acc[h][i][c][0], acc[h][i][c][1]);
      }
  }
}

// T −= L·Lᵀ on the lower triangle of a 64×64 shared-memory tile, in groups of
// 2×2 blocks of 8×8 that share their fragment loads.  Group G < 6 is one of
// the six 16×16 groups below the diagonal, (I, J) = (1,0), (2,0), (2,1),
// (3,0), (3,1), (3,2) (four products from four loads per k-step); groups 6
// and 7 are two diagonal groups each (three products from two loads per
// group; blocks above the diagonal are neither computed nor read).
__device__ __forceinline__ void lower_syrk_group(double (*tt)[LDM], const double (*l)[LDM],
                                                 int G, int lane) {
  const int g = lane >> 2, t = lane & 3;
  if (G < 6) {
    const int I = (G < 1) ? 1 : ((G < 3) ? 2 : 3);
    const int J = G - I * (I - 1) / 2;
    const int ra = 16 * I + g, rb = 16 * J + g;
    double acc[2][2][2] = {};
#pragma unroll 4
    for (int q = 0; q < NB; q += 4) {
      const double a0 = l[ra][q + t], a1 = l[ra + 8][q + t];
      const double b0 = l[rb][q + t], b1 = l[rb + 8][q + t];
      dmma_884(acc[0][0], a0, b0);
      dmma_884(acc[0][1], a0, b1);
      dmma_884(acc[1][0], a1, b0);
      dmma_884(acc[1][1], a1, b1);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        double2* p = reinterpret_cast<double2*>(&tt[ra + 8 * i][16 * J + 8 * j + 2 * t]);
        const double2 o = *p;
        *p = make_double2(o.x - acc[i][j][0], o.y - acc[i][j][1]);
      }
  } else {
    // diagonal groups 2·(G − 6) and the next: blocks (0,0), (1,0), (1,1) of each
    const int r0 = 32 * (G - 6) + g;
    double acc[2][3][2] = {};
#pragma unroll 4
    for (int q = 0; q < NB; q += 4) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const double u0 = l[r0 + 16 * h][q + t], u1 = l[r0 + 16 * h + 8][q + t];
        dmma_884(acc[h][0], u0, u0);
        dmma_884(acc[h][1], u1, u0);
        dmma_884(acc[h][2], u1, u1);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + 16 * h, c = 32 * (G - 6) + 16 * h + 2 * t;
      double2* p0 = reinterpret_cast<double2*>(&tt[r][c]);
      double2* p1 = reinterpret_cast<double2*>(&tt[r + 8][c]);
      double2* p2 = reinterpret_cast<double2*>(&tt[r + 8][c + 8]);
      const double2 o0 = *p0, o1 = *p1, o2 = *p2;
      *p0 = make_double2(o0.x - acc[h][0][0], o0.y - acc[h][0][1]);
      *p1 = make_double2(o1.x - acc[h][1][0], o1.y - acc[h][1][1]);
      *p2 = make_double2(o2.x - acc[h][2][0], o2.y - acc[h][2][1]);
    }
  }
}
// Over warps 0–3 and 5–7: warp w takes group w, and warp 0 also group 4.
__device__ __forceinline__ void lower_syrk(double (*tt)[LDM], const double (*l)[LDM], int warp,
                                           int lane) {
  lower_syrk_group(tt, l, warp, lane);
  if (warp == 0) lower_syrk_group(tt, l, 4, lane);
}

// 64×64 float64 tile products C = X·B of a worker group (4 warps).  Warp w
// owns rows 32·(w/2) .. +32 and columns 32·(w%2) .. +32 of C: 4 × 4
// accumulator blocks of 8×8.  X is held row-major (row r of C, column q of
// the sum).  B comes in one of two layouts, both copied from global memory
// as they are:
//   NT: y holds Bᵀ (row n of C, column q): C = X·Yᵀ;
//   NN: y holds B (row q, column n):       C = X·Y.
// With the row pitch LDM ≡ 4 (mod 16) doubles, every fragment load of either
// layout touches each bank pair exactly twice (two wavefronts, no conflict).
// With NEG the products are subtracted (acc −= X·B): the accumulators start
// from the tile being updated.
template <bool NT, bool NEG>
__device__ __forceinline__ void group_mm(const double (*x)[LDM], const double (*y)[LDM],
                                        double acc[4][4][2], int hw, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int rb = 32 * (hw >> 1), cb = 32 * (hw & 1);
#pragma unroll 2
  for (int q = 0; q < NB; q += 4) {
    double a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = NEG ? -x[rb + 8 * i + g][q + t] : x[rb + 8 * i + g][q + t];
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = NT ? y[cb + 8 * j + g][q + t] : y[q + t][cb + 8 * j + g];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dmma_884(acc[i][j], a[i], b[j]);
  }
}

// The part of a 64×64 output tile (leading dimension ld) that a lane's
// accumulators cover: into the accumulators (the start of C −= X·B), and
// back out.
__device__ __forceinline__ void group_load_acc(const double* out, int64_t ld, double acc[4][4][2],
                                              int hw, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int rb = 32 * (hw >> 1), cb = 32 * (hw & 1);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double2 v = __ldcg(reinterpret_cast<const double2*>(out + (int64_t)(rb + 8 * i + g) * ld +
                                                                cb + 8 * j + 2 * t));
      acc[i][j][0] = v.x;
      acc[i][j][1] = v.y;
    }
}

__device__ __forceinline__ void group_store(double* out, int64_t ld, const double acc[4][4][2],
                                           int hw, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int rb = 32 * (hw >> 1), cb = 32 * (hw & 1);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<double2*>(out + (int64_t)(rb + 8 * i + g) * ld + cb + 8 * j + 2 * t) =
          make_double2(acc[i][j][0], acc[i][j][1]);
}

// Two 64×64 float64 tiles (leading dimension ld) into shared memory as they
// are, by the 96 threads of a group's last three warps (w = 0..95): 16-byte
// cp.async through L2 only (tiles are rewritten by other CTAs of the same
// launch).  The group's first warp meanwhile loads its part of the output
// tile and its thread 0 decodes the next task.  The caller commits.
__device__ __forceinline__ void group_copy2(double (*dx)[LDM], const double* sx,
                                            double (*dy)[LDM], const double* sy, int64_t ld,
                                            int w) {
#pragma unroll 4
  for (int k = 0; k < 43; ++k) {
    const int e = w + 96 * k;               // 4096 chunks of 16 bytes
    if (e < 4096) {
      const int q = e & 2047, r = q >> 5, c = (q & 31) * 2;
      double (*dst)[LDM] = (e < 2048) ? dx : dy;
      const double* src = (e < 2048) ? sx : sy;
      const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(&dst[r][c]));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d),
                   "l"(src + (int64_t)r * ld + c) : "memory");
    }
  }
}

// ---------------------------------------------------------------------------
// The factorisation as one persistent, dataflow launch.
//
// The first CTA to arrive runs the critical chain, keeping the diagonal tile
// in shared memory from one step to the next (and its instruction cache
// warm): DIAG(k) — D_k = L_kk⁻¹ —, then PANEL(k,k+1) — L_{k+1,k} =
// A_{k+1,k}·D_kᵀ — and the last update of tile (k+1,k+1), once those two
// tiles have received their first k updates from the workers.
// The other CTAs take the remaining tasks in a fixed global order of slots.
// Slot s holds the factor tasks of step s (64-column block s), those the
// next steps wait for first,
//   PANEL(s,i) i > s+1, TRAIL(s,i,s+1) i > s+1, TRAIL(s,i,j) s+1 < j ≤ i,
// and then the inverse tasks of step s − kMLag,
//   MROW(k,c) c < k, MTRAIL(k,k+1,c), MTRAIL(k,i,c) i > k+1   (k = s − kMLag),
// with PANEL:  L_ik = A_ik·D_kᵀ          (needs D_k and tile (i,k) updated k times)
//      MROW:   M_kc = D_k·M_kc           (needs D_k and M_kc updated k−c times)
//      TRAIL:  A_ij −= L_ik·L_jkᵀ         (needs L_ik, L_jk, tile (i,j) updated k times)
//      MTRAIL: M_ic −= L_ik·M_kc          (needs L_ik, final M_kc, M_ic updated k−c times)
// The chain never reads M, so its tasks trail the factor by kMLag steps and
// leave the workers to the tiles the chain waits for when a step has many
// tasks.  Every dependency of a task is an earlier task or a step of the
// chain, the chain at step k waits only for factor tasks of step k−1, and
// tasks are taken in order only by running CTAs, so the launch needs no
// co-residency guarantee.
// Flags are set with release stores after a fence and polled with acquire
// loads; every wait is bounded and a time-out (or a bad pivot) raises a
// shared abort flag.
// ---------------------------------------------------------------------------


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

// The same wait for warps 0–3 and 5–7 (thread 0 polls), joined by barrier
// kBarChain.
__device__ bool group_wait(const int* flag, int target, int* abortp, int32_t* info, int* s_ok,
                           uint32_t limit) {
  if (threadIdx.x == 0) {
    bool ok = false;
    for (uint32_t it = 0; it < limit; ++it) {
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
  bar_sync(kBarChain, kHand);
  const bool ok = *s_ok != 0;
  bar_sync(kBarChain, kHand);
  return ok;
}


// A worker task as operands, output and dependencies:
//   PANEL  (k,i):   L_ik = A_ik·D_kᵀ     x = A_ik, y = D_k (NT)
//   MROW   (k,c):   M_kc = D_k·M_kc      x = D_k,  y = M_kc (NN)
//   TRAIL  (k,i,j): A_ij −= L_ik·L_jkᵀ   x = L_ik, y = L_jk (NT)
//   MTRAIL (k,i,c): M_ic −= L_ik·M_kc    x = L_ik, y = M_kc (NN)
// (D_k = L_kk⁻¹ is stored in tile (k,k) of M.)  The task may start once
// every dep[d] flag is ≥ its target; it then sets *flag = value.
struct WorkTask {
  const double* x;
  const double* y;
  double* out;
  bool nt, subtract;
  int* flag;
  int value;
  int ndep;
  const int* dep[3];
  int target[3];
};

__device__ WorkTask work_task(int task, int N, const int* prefix, int64_t np, double* A,
                              double* M, const CholSync& S) {
  int kind, k, i, j;
  decode_task(task, N, prefix, kind, k, i, j);
  auto tile = [np](double* base, int r, int c) { return base + (int64_t)r * NB * np + (int64_t)c * NB; };
  WorkTask t = {};
  if (kind == T_PANEL) {
    t.x = tile(A, i, k); t.y = tile(M, k, k); t.out = tile(A, i, k);
    t.nt = true; t.subtract = false;
    t.flag = &S.pdone[k * N + i]; t.value = 1;
    t.dep[0] = &S.diag_done[k]; t.target[0] = 1;
    t.dep[1] = &S.upd[i * N + k]; t.target[1] = k;
    t.ndep = 2;
  } else if (kind == T_MROW) {
    const int c = j;
    t.x = tile(M, k, k); t.y = tile(M, k, c); t.out = tile(M, k, c);
    t.nt = false; t.subtract = false;
    t.flag = &S.mdone[k * N + c]; t.value = 1;
    t.dep[0] = &S.diag_done[k]; t.target[0] = 1;
    t.dep[1] = &S.mupd[k * N + c]; t.target[1] = k - c;
    t.ndep = 2;
  } else if (kind == T_TRAIL) {
    t.x = tile(A, i, k); t.y = tile(A, j, k); t.out = tile(A, i, j);
    t.nt = true; t.subtract = true;
    t.flag = &S.upd[i * N + j]; t.value = k + 1;
    t.dep[0] = &S.pdone[k * N + i]; t.target[0] = 1;
    t.dep[1] = &S.pdone[k * N + j]; t.target[1] = 1;
    t.dep[2] = &S.upd[i * N + j]; t.target[2] = k;
    t.ndep = 3;
  } else {   // T_MTRAIL
    const int c = j;
    t.x = tile(A, i, k); t.y = tile(M, k, c); t.out = tile(M, i, c);
    t.nt = false; t.subtract = true;
    t.flag = &S.mupd[i * N + c]; t.value = k - c + 1;
    t.dep[0] = &S.pdone[k * N + i]; t.target[0] = 1;
    t.dep[1] = (c < k) ? &S.mdone[k * N + c] : &S.diag_done[k]; t.target[1] = 1;
    t.dep[2] = &S.mupd[i * N + c]; t.target[2] = k - c;
    t.ndep = 3;
  }
  return t;
}

__device__ __forceinline__ int ld_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One look at every dependency of t (relaxed loads, all in flight at once).
__device__ __forceinline__ bool deps_final(const WorkTask& t) {
  int v[3];
#pragma unroll
  for (int d = 0; d < 3; ++d) v[d] = d < t.ndep ? ld_relaxed(t.dep[d]) : 0;
  bool ok = true;
#pragma unroll
  for (int d = 0; d < 3; ++d) ok = ok && (d >= t.ndep || v[d] >= t.target[d]);
  return ok;
}

// A worker group's bounded wait for every dependency of t (thread 0 of the
// group polls; a fence after the final look gives the acquire the group's
// tile loads need); false on abort or time-out (reported).  One barrier:
// thread 0 writes *s_ok again only in the group's next wait, after two more
// group barriers that every reader has passed.
__device__ bool group_wait_deps(const WorkTask& t, int* abortp, int32_t* info, int* s_ok, uint32_t spin,
                          int ht, int hbar) {
  if (ht == 0) {
    bool ok = false;
    for (uint32_t it = 0; it < spin; ++it) {
      if (deps_final(t)) {
        ok = true;
        break;
      }
      if (*reinterpret_cast<volatile int*>(abortp)) break;
      if (it > 32) __nanosleep(64);
    }
    if (ok) {
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
    } else if (!*reinterpret_cast<volatile int*>(abortp)) {
      report(info, GPTQ_ERR_TIMEOUT, t.target[0]);
      atomicExch(abortp, 1);
    }
    *s_ok = ok ? 1 : 0;
  }
  bar_sync(hbar, 128);
  return *s_ok != 0;
}

__global__ void __launch_bounds__(kCholThreads, 1)
chol_persistent_kernel(double* __restrict__ A, double* __restrict__ M,
                       int64_t n, int64_t np, int N,
                       int ntasks, int* sync_base, int32_t* info, uint32_t spin) {
  extern __shared__ double sm[];
  __shared__ int s_role, s_ok, s_bad, s_got, s_fail;
  __shared__ int s_htask[kGroups][2], s_hok[kGroups], s_hready[kGroups];
  __shared__ WorkTask s_hwt[kGroups][2];
  // the task numbering's slot prefix, after the tiles
  int* prefix = reinterpret_cast<int*>(sm + kTileDoubles);
  __shared__ volatile int s_stop;
  const CholSync S = sync_view(sync_base, N);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    s_role = atomicAdd(&S.ctrl[1], 1);
    build_slot_prefix(N, prefix);
  }
  __syncthreads();
  if (*reinterpret_cast<volatile int32_t*>(info) != 0) return;

  if (s_role == 0) {
    if (warp >= kChainThreads / 32) return;
    // ---- the critical chain: DIAG(k), then PANEL(k, k+1) and the last
    // update of tile (k+1, k+1), which stays in shared memory for DIAG(k+1).
    // Two buffers alternate as the diagonal tile and two as D (warp 4 clears
    // the one of the step before during the diagonal tile).  D_k leaves block
    // row by block row during DIAG(k); L_{k+1,k} stays in shared memory and
    // leaves (and is published) during the first block of DIAG(k+1), so that
    // no store stands in the way of the chain's shared-memory loads.
    double (*t0)[LDM] = reinterpret_cast<double (*)[LDM]>(sm);
    double (*t1)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + NB * LDM);
    double (*b0)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + 2 * NB * LDM);
    double (*x)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + 3 * NB * LDM);
    double (*b1)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + 4 * NB * LDM);
    double* xs = sm + 5 * NB * LDM;
    load_lower(t0, A, np, tid);
    zero_tile(b0, tid);
    zero_tile(b1, tid);
    if (tid == 0) {
      s_bad = 0;
      s_fail = 0;
    }
    chain_sync();
    for (int k = 0; k < N; ++k) {
      const int64_t base = (int64_t)k * NB;
      double (*a)[LDM] = (k & 1) ? t1 : t0;
      double (*an)[LDM] = (k & 1) ? t0 : t1;
      double (*b)[LDM] = (k & 1) ? b1 : b0;
      double (*bz)[LDM] = (k > 0) ? ((k & 1) ? b0 : b1) : nullptr;
      const bool more = k + 1 < N;
      double* Lp = A + (base + NB) * np + base;          // tile (k+1, k)
      const double* An = A + (base + NB) * np + base + NB;   // tile (k+1, k+1)
      // L_{k,k−1}, computed in the step before, still in x
      PanelOut po = {};
      if (k > 0) {
        po.src = x;
        po.dst = A + base * np + base - NB;
        po.flag = &S.pdone[(k - 1) * N + k];
      }
      // warp 4 fetches the next step's two input tiles during the diagonal
      // tile, as soon as the workers have finished them
      TilePrefetch pf = {};
      pf.spin = spin;
      if (more) {
        pf.count = 2;
        pf.flag[0] = &S.upd[(k + 1) * N + k];
        pf.flag[1] = &S.upd[(k + 1) * N + k + 1];
        pf.target[0] = pf.target[1] = k;
        pf.src[0] = Lp;
        pf.src[1] = An;
        pf.dst[0] = x;
        pf.dst[1] = an;
        pf.ld = np;
      }
      if (!diag_tile_smem(a, b, bz, xs, M + base * np + base, np, n, base, info, &s_bad, pf, po,
                          &s_stop, &s_got)) {
        if (tid == 0) atomicExch(&S.ctrl[2], 1);
        return;
      }
      if (!more) {
        if (tid == 0) {               // D_k is out (the diagonal tile ended with a barrier)
          __threadfence();
          st_release(&S.diag_done[k], 1);
        }
        break;
      }
      const int got = s_got;                        // read after the tile's last barrier
      if (warp == 4) {
        if (got) {                    // the prefetched tiles have landed
          asm volatile("cp.async.wait_all;" ::: "memory");
          __syncwarp();
          bar_arrive(kBarFetch, kHand + 32);
        }
        // D_k is out (the diagonal tile ended with a barrier); the fence waits
        // for its last stores while the other warps compute the panel
        if (lane == 0) {
          __threadfence();
          st_release(&S.diag_done[k], 1);
        }
      } else {
        const int gt = (warp < 4) ? tid : tid - 32;   // 0..223 over warps 0–3, 5–7
        bool ok = true;
        if (got) bar_sync(kBarFetch, kHand + 32);
        // L_{k+1,k} = A_{k+1,k}·D_kᵀ
        if (!(got & 1)) {
          ok = group_wait(&S.upd[(k + 1) * N + k], k, &S.ctrl[2], info, &s_ok, spin);
          if (ok) {
            copy_tile_async_group(x, Lp, np, gt);
            copy_wait_all();
          }
        }
        if (ok) {
          bar_sync(kBarChain, kHand);
          double acc[2][4][2][2] = {};
          panel_mm(x, b, acc, warp, lane);
          bar_sync(kBarChain, kHand);
          panel_to_smem(x, acc, warp, lane);
          // A_{k+1,k+1} −= L_{k+1,k}·L_{k+1,k}ᵀ, in shared memory
          if (!(got & 2)) {
            ok = group_wait(&S.upd[(k + 1) * N + k + 1], k, &S.ctrl[2], info, &s_ok, spin);
            if (ok) {
              copy_tile_async_group(an, An, np, gt);
              copy_wait_all();
            }
          }
          if (ok) {
            bar_sync(kBarChain, kHand);
            lower_syrk(an, x, warp, lane);
          }
        }
        if (!ok && tid == 0) s_fail = 1;
      }
      chain_sync();
      if (s_fail) return;
    }
    return;
  }

  // ---- the workers: kGroups independent groups of 4 warps (h = warp / 4),
  // each claiming and computing its own tasks in numbering order, as that
  // many workers would.  One group's waits (its claim, its dependency poll,
  // its tile copies and the release of its result) then run under the other
  // groups' float64 products.  Group h synchronises on named barrier 1 + h
  // (128 threads) and uses tiles 2h (x) and 2h + 1 (y).
  const int h = warp >> 2, hw = warp & 3, ht = tid & 127, hbar = 1 + h;
  double (*x)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + 2 * h * NB * LDM);
  double (*y)[LDM] = reinterpret_cast<double (*)[LDM]>(sm + (2 * h + 1) * NB * LDM);
  // thread 0 of the group claims and decodes the next task while the current
  // one's tiles land; during the current products the group then pulls the
  // next output tile towards L2 (the trailing matrix does not fit there, so
  // an update tile would otherwise come from DRAM on the critical path)
  if (ht == 0) {
    const int c = atomicAdd(&S.ctrl[0], 1);
    s_htask[h][0] = c;
    if (c < ntasks) s_hwt[h][0] = work_task(c, N, prefix, np, A, M, S);
  }
  if (ht == 0) s_hready[h] = 0;
  bar_sync(hbar, 128);
  // Per task two or three group barriers: in the wait (the dependencies are
  // final; skipped when thread 0 saw them final during the task before),
  // after the copies (the tiles have landed; the next task is decoded), after
  // the stores.  Task records alternate between two slots: round r reads slot
  // r & 1 at its top and thread 0 writes the next one into the other slot
  // before the second barrier; that slot's last readers (round r − 1) passed
  // the second barrier of round r − 1 before.  The readiness flag is written
  // before the third barrier and read after it.
  for (int rd = 0;; rd ^= 1) {
    if (s_htask[h][rd] >= ntasks) return;
    const WorkTask t = s_hwt[h][rd];
    if (!s_hready[h] && !group_wait_deps(t, &S.ctrl[2], info, &s_hok[h], spin, ht, hbar)) return;
    // the next task's number, claimed once this one can start: the atomic's
    // round trip runs under the copies (it is decoded once they are issued)
    int claimed = 0;
    if (ht == 0) claimed = atomicAdd(&S.ctrl[0], 1);
    if (hw > 0) {
      group_copy2(x, t.x, y, t.y, np, ht - 32);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // C −= X·B starts from C; out = X·B from zero
    double acc[4][4][2];
    if (t.subtract) {
      group_load_acc(t.out, np, acc, hw, lane);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    }
    if (ht == 0) {
      int c = claimed;
      if (*reinterpret_cast<volatile int*>(&S.ctrl[2])) c = ntasks;
      s_htask[h][rd ^ 1] = c;                 // read at the top of the next round
      if (c < ntasks) s_hwt[h][rd ^ 1] = work_task(c, N, prefix, np, A, M, S);
    }
    copy_wait_all();
    bar_sync(hbar, 128);
    const bool more = s_htask[h][rd ^ 1] < ntasks;
    const WorkTask& nx = s_hwt[h][rd ^ 1];
    // thread 0 takes one look at the next task's dependencies, the loads in
    // flight under the products
    int nv[3] = {0, 0, 0};
    if (ht == 0 && more) {
#pragma unroll
      for (int d = 0; d < 3; ++d)
        if (d < nx.ndep) nv[d] = ld_relaxed(nx.dep[d]);
    }
    if (more && ht >= 64 && nx.subtract) {
      // 64 rows × four 128-byte lines, by the group's last two warps (so that
      // thread 0's fence below does not wait for them)
      const double* o = nx.out + (int64_t)(ht - 64) * np;
#pragma unroll
      for (int l = 0; l < 4; ++l) asm volatile("prefetch.global.L2 [%0];" ::"l"(o + 16 * l));
    }
    if (t.nt) {
      if (t.subtract) group_mm<true, true>(x, y, acc, hw, lane);
      else group_mm<true, false>(x, y, acc, hw, lane);
    } else {
      if (t.subtract) group_mm<false, true>(x, y, acc, hw, lane);
      else group_mm<false, false>(x, y, acc, hw, lane);
    }
    if (ht == 0) {
      // every dependency already final: the acquire now (before this thread's
      // stores, so the fence waits for nothing), and no wait next round
      bool ready = more;
#pragma unroll
      for (int d = 0; d < 3; ++d) ready = ready && (d >= nx.ndep || nv[d] >= nx.target[d]);
      if (ready) asm volatile("fence.acq_rel.gpu;" ::: "memory");
      s_hready[h] = ready ? 1 : 0;
    }
    group_store(t.out, np, acc, hw, lane);
    bar_sync(hbar, 128);                          // the group's stores are issued
    // a thread of the second warp publishes the result (the release orders the
    // group's stores, through the barrier, before the flag) while thread 0
    // polls the next task's dependencies
    if (ht == 32) st_release(t.flag, t.value);
  }
}

// Host side: the poll limit of the factorisation's waits (0: kSpinLimit), and
// the most worker CTAs one factorisation launch may use (0: every SM but one).
std::atomic<uint32_t> g_wait_limit{0};
std::atomic<int> g_max_workers{0};

// U[i][j] = L⁻¹[n−1−i][n−1−j] for j ≥ i, 0 below the diagonal.
__global__ void __launch_bounds__(256)
prep_out_kernel(const double* __restrict__ M, int64_t n, int64_t np,
                float* __restrict__ U) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= n * n) return;
  const int64_t i = e / n, j = e % n;
  U[e] = (j >= i) ? (float)M[(n - 1 - i) * np + (n - 1 - j)] : 0.0f;
}


}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" void gptq_set_wait_limit(uint32_t polls) {
  g_wait_limit.store(polls, std::memory_order_relaxed);
}

extern "C" void gptq_set_factor_workers(int max_ctas) {
  g_max_workers.store(max_ctas > 0 ? max_ctas : 0, std::memory_order_relaxed);
}

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
  if (order < GPTQ_ORDER_NATURAL || order > GPTQ_ORDER_MINPIVOT)
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
  // the tiles (the chain's five and its 8×8 pivot blocks, or two per worker
  // group), then the task numbering's slot prefix (N + kMLag + 1 ints)
  const size_t tile_smem = kTileDoubles * sizeof(double) +
                           sizeof(int) * (size_t)(task_slots(N) + 1);
  if (total_tasks(N) >= ((int64_t)1 << 31) || tile_smem > 227 * 1024)
    return fail(GPTQ_ERR_UNSUPPORTED, "gptq_prepare: n=%lld is too large for the factorisation",
                (long long)n);
  int num_sms = 0;
  {
    gptq_status st = ensure_smem_limit((const void*)chol_persistent_kernel, (int)tile_smem,
                                       "chol_persistent_kernel");
    if (st == GPTQ_OK) st = device_sm_count(&num_sms);
    if (st != GPTQ_OK) return st;
  }

  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  GPTQ_CUDA(cudaMemsetAsync(w.sync, 0, w.sync_bytes, s));
  if (order == GPTQ_ORDER_CUSTOM)
    GPTQ_CUDA(cudaMemsetAsync(w.seen, 0, sizeof(int32_t) * n, s));
  GPTQ_LAUNCH(KK_PREP_STATS, s, prep_stats_kernel, 1, 1024, 0, H, n, dead, w.mean, info);
  if (order == GPTQ_ORDER_MINPIVOT) {
    // the order comes from a pivoted factorisation of its own, on the
    // workspace's two float64 arrays (both rewritten by the gather below)
    if (min_pivot_scratch_doubles(n) > (size_t)(np * np))
      return fail(GPTQ_ERR_INVALID_ARG, "gptq_prepare: min-pivot scratch does not fit");
    gptq_status st = launch_min_pivot_order(H, n, w.mean, damp, w.M, np, w.A, perm, info, s);
    if (st != GPTQ_OK) return st;
  } else {
    GPTQ_LAUNCH(KK_PREP_ORDER, s, prep_order_kernel, (int)ceil_div(n, 256), 256, 0,
                H, n, order, perm, w.seen, info);
  }
  GPTQ_LAUNCH(KK_PREP_GATHER, s, prep_gather_kernel, (unsigned)ceil_div(np * np, 256),
              256, 0, H, n, np, perm, w.seen, order == GPTQ_ORDER_CUSTOM ? 1 : 0,
              w.mean, damp, w.A, w.M, info);
  const int ntasks = (int)total_tasks(N);
  // Workers: enough that the two tiles the chain needs next are never queued
  // behind other ready tasks (a step offers ≈ N²/2 tile tasks, each ≈ a third
  // of the chain's step; N²/6 workers left the chain waiting ≈ 6.8 K cycles a
  // step for its panel input, N²/3 ≈ 0.5 K), never more than one CTA per SM
  // besides the chain's, so that work on other streams finds SMs.
  int workers = N * N / 3 + 2;
  if (workers > num_sms - 1) workers = num_sms - 1;
  const int cap = g_max_workers.load(std::memory_order_relaxed);
  if (cap > 0 && workers > cap) workers = cap;
  if (workers > ntasks) workers = ntasks;
  const int grid = 1 + workers;
  const uint32_t lim = g_wait_limit.load(std::memory_order_relaxed);
  GPTQ_LAUNCH(KK_CHOL, s, chol_persistent_kernel, grid, kCholThreads, tile_smem, w.A, w.M, n, np,
              N, ntasks, w.sync, info, lim != 0 ? lim : kSpinLimit);
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
