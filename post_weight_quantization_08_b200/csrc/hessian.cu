// K1: Hessian accumulation H += 2·XᵀX.
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: the
// Hessian of a layer comes from its calibration activations X (XᵀX/n there;
// 2·XᵀX here, which leaves the codes unchanged because the damping is
// relative).  "GPTQ as Babai's Nearest Plane Algorithm", §2.1: XᵀX is the
// Gram matrix of the lattice basis.
//
// X is T×n bfloat16, token-major.  bf16×bf16 products are exact in float32,
// so the only rounding is the float32 accumulation over T.  Only 128×128
// tiles on or above the diagonal are computed; each off-diagonal tile is also
// written mirrored, so H stays exactly symmetric.
//
// Main path (n a multiple of 8, so that TMA row strides are 16-byte
// multiples): one CTA per tile, a 4-stage TMA → tcgen05 pipeline.
//   warp 0 lane 0   TMA producer: boxes of 64 columns × 64 tokens with
//                   128-byte swizzle (two boxes per 128-column operand);
//   warp 1 lane 0   MMA issuer: tcgen05.mma kind::f16 (bf16 in, f32 in TMEM),
//                   M = N = 128, K = 16 per instruction, both operands
//                   MN-major (X is token-major, so columns of H are contiguous);
//   all 4 warps     epilogue: tcgen05.ld of the 128×128 accumulator into
//                   128-byte-swizzled shared boxes (2·D, and for off-diagonal
//                   tiles also 2·Dᵀ), then TMA reduce-adds into H — no
//                   read-modify-write round trips from the threads.
// Every wait is bounded; a time-out is reported through `info`.
// Fallback (n not a multiple of 8): a float32 SIMT tile kernel.
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gptq {
namespace {

// ---------------------------------------------------------------- SIMT path

constexpr int HT = 64;   // output tile edge
constexpr int HK = 32;   // tokens per shared-memory stage

__device__ __forceinline__ void upper_tile(int lin, int nt, int& bi, int& bj) {
  bi = 0;
  while (lin >= nt - bi) { lin -= nt - bi; ++bi; }
  bj = bi + lin;
}

__global__ void __launch_bounds__(256)
hessian_simt_kernel(const __nv_bfloat16* __restrict__ X, int64_t T, int64_t n,
                    int nt, float* __restrict__ H) {
  int bi, bj;
  upper_tile(blockIdx.x, nt, bi, bj);
  const int64_t i0 = (int64_t)bi * HT, j0 = (int64_t)bj * HT;

  __shared__ __align__(16) float xa[HK][HT];
  __shared__ __align__(16) float xb[HK][HT];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};

  for (int64_t t0 = 0; t0 < T; t0 += HK) {
    for (int e = tid; e < HK * HT; e += 256) {
      const int kk = e / HT, c = e % HT;
      const int64_t t = t0 + kk;
      float va = 0.f, vb = 0.f;
      if (t < T) {
        if (i0 + c < n) va = __bfloat162float(X[t * n + i0 + c]);
        if (j0 + c < n) vb = __bfloat162float(X[t * n + j0 + c]);
      }
      xa[kk][c] = va;
      xb[kk][c] = vb;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < HK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xa[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&xb[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = i0 + ty * 4 + r;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t j = j0 + tx * 4 + c;
      if (i < n && j < n) {
        const float v = 2.0f * acc[r][c];
        H[i * n + j] += v;
        if (bi != bj) H[j * n + i] += v;
      }
    }
  }
}

// ---------------------------------------------------------------- tcgen05 path

constexpr int TC_TILE = 128;                 // M = N = 128
constexpr int TC_KT = 64;                    // tokens per stage
constexpr int TC_STAGES = 4;
constexpr uint32_t TC_BOX_BYTES = 64 * TC_KT * 2;           // 64 columns × 64 tokens bf16
constexpr uint32_t TC_OPER_BYTES = 2 * TC_BOX_BYTES;        // 128 columns
constexpr uint32_t TC_STAGE_BYTES = 2 * TC_OPER_BYTES;      // A and B
constexpr uint32_t TC_IDESC = idesc_f32acc(1, 1, 1, 1, TC_TILE, TC_TILE);   // bf16, MN-major
constexpr size_t TC_SMEM = 1024 + TC_STAGES * TC_STAGE_BYTES + 256;
constexpr uint32_t EP_BOX = 32 * TC_TILE * 4;               // 32 columns × 128 rows f32
static_assert(8 * EP_BOX <= TC_STAGES * TC_STAGE_BYTES, "epilogue boxes reuse the ring");

__global__ void __launch_bounds__(128, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmH,
                  int64_t T, int64_t n, int nt, int32_t* info) {
  extern __shared__ unsigned char smraw[];
  // 1024-byte aligned operand ring (128-byte swizzle atoms are 1 KB)
  const uint32_t raw = smem_addr(smraw);
  unsigned char* ring = smraw + ((1024 - (raw & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + TC_STAGES * TC_STAGE_BYTES);
  uint64_t* empty = full + TC_STAGES;
  uint64_t* done = empty + TC_STAGES;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  int bi, bj;
  upper_tile(blockIdx.x, nt, bi, bj);
  const bool diag = bi == bj;
  const int i0 = bi * TC_TILE, j0 = bj * TC_TILE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = (int)((T + TC_KT - 1) / TC_KT);

  if (tid == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, TC_TILE);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0 && lane == 0) {
    // ---- TMA producer
    for (int c = 0; c < nk; ++c) {
      const int s = c % TC_STAGES;
      if (c >= TC_STAGES && !mbar_wait_bounded(&empty[s], ((c / TC_STAGES) - 1) & 1)) {
        report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
        *abort_flag = 1;
        break;
      }
      if (*abort_flag) break;
      unsigned char* a = ring + s * TC_STAGE_BYTES;
      unsigned char* b = a + TC_OPER_BYTES;
      const int t0 = c * TC_KT;
      mbar_arrive_expect_tx(&full[s], diag ? TC_OPER_BYTES : TC_STAGE_BYTES);
      tma_load_2d(a, &tmX, i0, t0, &full[s]);
      tma_load_2d(a + TC_BOX_BYTES, &tmX, i0 + 64, t0, &full[s]);
      if (!diag) {
        tma_load_2d(b, &tmX, j0, t0, &full[s]);
        tma_load_2d(b + TC_BOX_BYTES, &tmX, j0 + 64, t0, &full[s]);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer
    for (int c = 0; c < nk; ++c) {
      const int s = c % TC_STAGES;
      if (!mbar_wait_bounded(&full[s], (c / TC_STAGES) & 1)) {
        report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
        *abort_flag = 1;
        break;
      }
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t a = smem_addr(ring + s * TC_STAGE_BYTES);
      const uint32_t b = diag ? a : a + TC_OPER_BYTES;
#pragma unroll
      for (int ks = 0; ks < TC_KT / 16; ++ks) {
        // 16 tokens = two 8-row swizzle atoms (2 × 1024 B) further along K;
        // the second 64-column half of the operand sits one box further.
        const uint64_t ad = sdesc_sw128(a + ks * 2048, TC_BOX_BYTES, 1024);
        const uint64_t bd = sdesc_sw128(b + ks * 2048, TC_BOX_BYTES, 1024);
        umma_f16_ss(tmem, ad, bd, TC_IDESC, (c > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);   // also after an abort: retires the MMAs in flight
  }
  __syncwarp();

  // ---- epilogue: all four warps, one accumulator row per thread.  The ring
  // is free again (every load was consumed, every MMA has retired): boxes
  // 0..3 take 2·D (row r, columns 32b..32b+31), boxes 4..7 take 2·Dᵀ.
  const bool ok = mbar_wait_bounded(done, 0);
  if (!ok) report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
  tc_fence_after();
  const bool write = ok && !*abort_flag;
  if (write) {
    const int r = warp * 32 + lane;
#pragma unroll 1
    for (int ch = 0; ch < TC_TILE / 32; ++ch) {
      float v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, v);
      unsigned char* box = ring + ch * EP_BOX + r * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(box + ((q ^ (r & 7)) << 4)) =
            make_float4(2.f * v[4 * q], 2.f * v[4 * q + 1], 2.f * v[4 * q + 2], 2.f * v[4 * q + 3]);
      if (!diag) {
        // Dᵀ: row c = 32·ch + k of the mirrored tile, column r
        unsigned char* mbox = ring + (4 + warp) * EP_BOX;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int c = 32 * ch + k;
          *reinterpret_cast<float*>(mbox + c * 128 + (((lane >> 2) ^ (c & 7)) << 4) + (lane & 3) * 4) =
              2.f * v[k];
        }
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (write && tid == 0) {
#pragma unroll 1
    for (int b = 0; b < TC_TILE / 32; ++b) {
      if (j0 + 32 * b < n) tma_reduce_add_2d(&tmH, j0 + 32 * b, i0, ring + b * EP_BOX);
      if (!diag && i0 + 32 * b < n) tma_reduce_add_2d(&tmH, i0 + 32 * b, j0, ring + (4 + b) * EP_BOX);
    }
    bulk_commit();
    bulk_wait_all();
  }
  // ---- teardown: no copy or MMA may still be in flight when TMEM goes
  if (tid == 0) {
    for (int s = 0; s < TC_STAGES && s < nk; ++s) {
      const int last = s + ((nk - 1 - s) / TC_STAGES) * TC_STAGES;   // last chunk on stage s
      mbar_wait_bounded(&full[s], (last / TC_STAGES) & 1, 1u << 16);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TC_TILE);
}


}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_hessian_accumulate(const void* X, int64_t T, int64_t n,
                                               float* H, int32_t* info, void* stream) {
  if (H == nullptr || (X == nullptr && T > 0))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hessian_accumulate: null pointer");
  if (T < 0 || n < 1 || n > (1 << 20) || T > ((int64_t)1 << 31) - TC_KT)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hessian_accumulate: T=%lld n=%lld",
                (long long)T, (long long)n);
  if (T == 0) return GPTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tma_ok = (n % 8 == 0) && (reinterpret_cast<uintptr_t>(X) % 16 == 0) &&
                      (reinterpret_cast<uintptr_t>(H) % 16 == 0);
  if (tma_ok) {
    CUtensorMap tm, th;
    if (!encode_tiled_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, n, T, n * 2, 64, TC_KT) ||
        !encode_tiled_2d(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, H, n, n, n * 4, 32, TC_TILE))
      return fail(GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the Hessian");
    {
      const gptq_status st = ensure_smem_limit((const void*)hessian_tc_kernel, (int)TC_SMEM,
                                               "hessian_tc_kernel");
      if (st != GPTQ_OK) return st;
    }
    const int nt = (int)ceil_div(n, TC_TILE);
    GPTQ_LAUNCH(KK_HESSIAN, s, hessian_tc_kernel, nt * (nt + 1) / 2, 128, TC_SMEM, tm, th, T, n,
                nt, info);
    return GPTQ_OK;
  }
  const int nt = (int)ceil_div(n, HT);
  GPTQ_LAUNCH(KK_HESSIAN, s, hessian_simt_kernel, nt * (nt + 1) / 2, 256, 0,
              static_cast<const __nv_bfloat16*>(X), T, n, nt, H);
  return GPTQ_OK;
}
