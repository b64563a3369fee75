// K4: lazy-batch trailing update  W[:, c0:] −= Err·U[k0:k0+kw, c0:].
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: every
// quantized column's error is subtracted from the columns not yet quantized.
// Applied once per block instead of once per column this is one product with
// K = block width; the result is the same up to float32 rounding order.
//
// Tensor-core path (n a multiple of 4): tcgen05.mma kind::tf32 with a
// three-term split.  Every float32 operand is written as hi + lo with
// hi = TF32(x) (round to nearest) and lo = x − hi (exact), and
//   Err·U ≈ Err_hi·U_hi + Err_hi·U_lo + Err_lo·U_hi
// (the dropped lo·lo term and the TF32 truncation of lo are ≈ 2⁻²¹ relative,
// float32-grade; a single TF32 product would be 2⁻¹¹ and move pre-rounding
// values by far more than the 1e-4 code units the parity criterion allows).
// The sweep writes Err_hi/Err_lo; the split of U is written once per call,
// transposed (UT[c][k] = U[k][c]), so that both tf32 operands are K-major:
// MN-major tf32 operands would need the 32-byte-atom variant of the 128-byte
// swizzle, K-major ones take the plain 128-byte swizzle.
//
// One CTA per 128-row × 256-column tile of W:
//   warp 0 lane 0  TMA: Err_hi/lo boxes 128 rows × 32 K and Uᵀ_hi/lo boxes
//                  256 columns × 32 K (both K-major), 128-byte swizzle,
//                  2-stage ring over K in chunks of 32;
//   warp 1 lane 0  3 × tcgen05.mma (M=128, N=256, K=8) per 8 K, A negated so
//                  the 256 TMEM columns hold −Err·U;
//   4 warps        drain TMEM into swizzled shared boxes, then one TMA
//                  reduce-add per 32-column box adds them into W.
// Fallback: float32 SIMT tiles.

#include "kernels.cuh"
#include "sm100.cuh"

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

constexpr int QM = 128, QN = 256, QK = 32, QSTAGES = 2;
constexpr uint32_t A_BOX = QK * QM * 4;          // 32 K × 128 rows, 16 KB
constexpr uint32_t B_OPER = QK * QN * 4;         // 32 K × 256 columns, 32 KB
constexpr uint32_t STAGE = 2 * A_BOX + 2 * B_OPER;          // 96 KB
constexpr uint32_t C_BOX = 32 * QM * 4;                     // 32 columns × 128 rows
constexpr uint32_t QIDESC = idesc_f32acc(2, 2, 0, 0, QM, QN) | (1u << 13);  // tf32 K-major, −A
constexpr size_t QSMEM = 1024 + QSTAGES * STAGE + 256;
static_assert(QSTAGES * STAGE >= (QN / 32) * C_BOX, "epilogue boxes reuse the ring");

struct TrailMaps {
  CUtensorMap ahi, alo, bhi, blo, c;
};

__global__ void __launch_bounds__(128, 1)
trailing_tc_kernel(const __grid_constant__ TrailMaps maps, int64_t m, int64_t n, int64_t c0,
                   int64_t c1, int64_t k0, int kw, int32_t* info) {
  extern __shared__ unsigned char smraw[];
  const uint32_t raw = smem_addr(smraw);
  unsigned char* ring = smraw + ((1024 - (raw & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + QSTAGES * STAGE);
  uint64_t* empty = full + QSTAGES;
  uint64_t* done = empty + QSTAGES;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = blockIdx.y * QM;
  const int cb = (int)(c0 + (int64_t)blockIdx.x * QN);
  const int nk = kw / QK;

  if (tid == 0) {
    for (int s = 0; s < QSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, QN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();                           // the errors come from the previous kernel
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    for (int c = 0; c < nk; ++c) {
      const int s = c % QSTAGES;
      if (c >= QSTAGES && !mbar_wait_bounded(&empty[s], ((c / QSTAGES) - 1) & 1)) {
        report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
        *abort_flag = 1;
        break;
      }
      unsigned char* st = ring + s * STAGE;
      const int kq = c * QK;
      mbar_arrive_expect_tx(&full[s], STAGE);
      tma_load_2d(st, &maps.ahi, kq, r0, &full[s]);
      tma_load_2d(st + A_BOX, &maps.alo, kq, r0, &full[s]);
      tma_load_2d(st + 2 * A_BOX, &maps.bhi, (int)k0 + kq, cb, &full[s]);
      tma_load_2d(st + 2 * A_BOX + B_OPER, &maps.blo, (int)k0 + kq, cb, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    for (int c = 0; c < nk; ++c) {
      const int s = c % QSTAGES;
      if (!mbar_wait_bounded(&full[s], (c / QSTAGES) & 1)) {
        report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
        *abort_flag = 1;
        break;
      }
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t st = smem_addr(ring + s * STAGE);
      const uint32_t ahi = st, alo = st + A_BOX;
      const uint32_t bhi = st + 2 * A_BOX, blo = bhi + B_OPER;
#pragma unroll
      for (int ks = 0; ks < QK / 8; ++ks) {
        // both K-major: 8 TF32 = 32 bytes further inside each 128-byte row;
        // 8-row groups 1024 bytes apart.
        const uint64_t dah = sdesc_sw128(ahi + ks * 32, SW128_KMAJOR_LBO, 1024);
        const uint64_t dal = sdesc_sw128(alo + ks * 32, SW128_KMAJOR_LBO, 1024);
        const uint64_t dbh = sdesc_sw128(bhi + ks * 32, SW128_KMAJOR_LBO, 1024);
        const uint64_t dbl = sdesc_sw128(blo + ks * 32, SW128_KMAJOR_LBO, 1024);
        umma_tf32_ss(tmem, dah, dbh, QIDESC, (c > 0 || ks > 0) ? 1u : 0u);
        umma_tf32_ss(tmem, dah, dbl, QIDESC, 1u);
        umma_tf32_ss(tmem, dal, dbh, QIDESC, 1u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);
  }
  __syncwarp();

  const bool ok = mbar_wait_bounded(done, 0);
  if (!ok) report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
  tc_fence_after();
  const bool write = ok && !*abort_flag;
  if (write) {
    // −Err·U rows into 128-byte-swizzled boxes (row r at r·128 B, 16-byte
    // chunk q stored at chunk q ^ (r mod 8)), which the TMA reduce reads.
    const int r = warp * 32 + lane;
#pragma unroll 1
    for (int b = 0; b < QN / 32; ++b) {
      float v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + b * 32, v);
      unsigned char* box = ring + b * C_BOX + r * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 w = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        *reinterpret_cast<float4*>(box + ((q ^ (r & 7)) * 16)) = w;
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (write && tid == 0) {
#pragma unroll 1
    for (int b = 0; b < QN / 32; ++b)
      if ((int64_t)cb + 32 * b < c1) tma_reduce_add_2d(&maps.c, cb + 32 * b, r0, ring + b * C_BOX);
    bulk_commit();
    bulk_wait_all();
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, QN);
}

bool encode_f32(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  return encode_tiled_2d(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, inner, outer, row_bytes,
                         box_inner, box_outer);
}

bool g_attr = false;

}  // namespace

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
                            const float* U, const float* Uhi, const float* Ulo, int32_t* info,
                            cudaStream_t s) {
  if (c1 > n) c1 = n;
  if (c0 >= c1 || kw <= 0 || m <= 0) return GPTQ_OK;
  if (Uhi != nullptr && trailing_uses_tensor_cores(n, kw)) {
    TrailMaps maps;
    const int64_t mr = error_rows(m);
    bool ok = encode_f32(&maps.ahi, Ehi, SWEEP_BLOCK_MAX, mr, SWEEP_BLOCK_MAX * 4, QK, QM) &&
              encode_f32(&maps.alo, Elo, SWEEP_BLOCK_MAX, mr, SWEEP_BLOCK_MAX * 4, QK, QM) &&
              encode_f32(&maps.bhi, Uhi, n, n, n * 4, QK, QN) &&
              encode_f32(&maps.blo, Ulo, n, n, n * 4, QK, QN) &&
              encode_f32(&maps.c, Wp, n, mr, n * 4, 32, QM);
    if (!ok) return fail(GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the trailing update");
    if (!g_attr) {
      GPTQ_CUDA(cudaFuncSetAttribute(trailing_tc_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QSMEM));
      g_attr = true;
    }
    const dim3 grid((unsigned)ceil_div(c1 - c0, QN), (unsigned)ceil_div(m, QM));
    GPTQ_LAUNCH_PDL(KK_TRAIL, s, trailing_tc_kernel, grid, 128, QSMEM, maps, m, n, c0, c1, k0,
                    kw, info);
    return GPTQ_OK;
  }
  const dim3 grid((unsigned)ceil_div(c1 - c0, TN), (unsigned)ceil_div(m, TM));
  GPTQ_LAUNCH(KK_TRAIL, s, trailing_simt_kernel, grid, 256, 0, Wp, m, n, c0, c1, Ehi, Elo, k0,
              kw, U);
  return GPTQ_OK;
}

}  // namespace gptq
