// K4 on the tensor cores: the lazy-batch trailing update
// W[:, c0:c1] −= Err·U[k0:k0+kw, c0:c1] as a CTA body, run by the CTAs that
// ride in each sweep's launch (the far columns of the block before).
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
// Fallback (n % 4 ≠ 0): float32 SIMT tiles, trailing.cu.
#pragma once

#include "kernels.cuh"
#include "sm100.cuh"

namespace gptq {

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

// Tensor maps of the update Wp[:, c0:] −= (Ehi+Elo)·U (errors error_rows(m) ×
// 128, UhiT/UloT the transposed TF32 split of U, Wp error_rows(m) × n).
bool make_trail_maps(TrailMaps* maps, float* Wp, int64_t m, int64_t n, const float* Ehi,
                     const float* Elo, int64_t kw, int64_t epitch, const float* UhiT,
                     const float* UloT);

namespace {

// One CTA's tile (bx: 256-column tile from c0, by: 128-row tile) of
// Wp[:, c0:c1] −= Err·U[k0:k0+kw, c0:c1]; smraw: at least QSMEM bytes of
// dynamic shared memory.  Called by 128 threads.
__device__ __forceinline__ void trailing_tc_body(const TrailMaps& maps, int64_t m, int64_t n,
                                                 int64_t c0, int64_t c1, int64_t k0, int kw,
                                                 int32_t* info, int bx, int by,
                                                 unsigned char* smraw) {
  const uint32_t raw = smem_addr(smraw);
  unsigned char* ring = smraw + ((1024 - (raw & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + QSTAGES * STAGE);
  uint64_t* empty = full + QSTAGES;
  uint64_t* done = empty + QSTAGES;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = by * QM;
  const int cb = (int)(c0 + (int64_t)bx * QN);
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
        report(info, GPTQ_ERR_TIMEOUT, bx);
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
        report(info, GPTQ_ERR_TIMEOUT, bx);
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
  if (!ok) report(info, GPTQ_ERR_TIMEOUT, bx);
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


}  // namespace
}  // namespace gptq
