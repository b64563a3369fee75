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
// multiples): a persistent CTA per SM walks its tiles through a 3-stage TMA →
// tcgen05 pipeline, with two TMEM accumulators so that a tile's epilogue runs
// under the next tile's products.
//   warp 0 lane 0   TMA producer: boxes of 64 columns × 64 tokens with
//                   128-byte swizzle (two boxes per 128-column operand);
//   warp 1 lane 0   MMA issuer: tcgen05.mma kind::f16 (bf16 in, f32 in TMEM),
//                   M = N = 128, K = 16 per instruction, both operands
//                   MN-major (X is token-major, so columns of H are contiguous);
//   warps 2–5       epilogue: tcgen05.ld of the 128×128 accumulator into
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
constexpr int TC_STAGES = 3;
constexpr int TC_THREADS = 192;              // 6 warps: TMA, MMA, 4 × epilogue
constexpr uint32_t TC_BOX_BYTES = 64 * TC_KT * 2;           // 64 columns × 64 tokens bf16
constexpr uint32_t TC_OPER_BYTES = 2 * TC_BOX_BYTES;        // 128 columns
constexpr uint32_t TC_STAGE_BYTES = 2 * TC_OPER_BYTES;      // A and B
constexpr uint32_t TC_IDESC = idesc_f32acc(1, 1, 1, 1, TC_TILE, TC_TILE);   // bf16, MN-major
constexpr uint32_t EP_BOX = 32 * TC_TILE * 4;               // 32 columns × 128 rows f32
constexpr uint32_t TC_RING = TC_STAGES * TC_STAGE_BYTES;
constexpr uint32_t TC_STAGING = 8 * EP_BOX;                 // 2·D and 2·Dᵀ boxes
constexpr size_t TC_SMEM = 1024 + TC_RING + TC_STAGING + 256;
static_assert(TC_SMEM <= 227 * 1024, "shared memory");

// Persistent: CTA x takes the upper tiles x, x + grid, x + 2·grid, ...
// Warp 0 lane 0 streams every tile's stages through the ring; warp 1 lane 0
// accumulates tile i into one of two TMEM accumulators (i & 1), so that the
// epilogue of tile i overlaps the products of tile i + 1; warps 2–5 drain
// an accumulator into 128-byte-swizzled staging boxes (TMEM lanes 32·(w mod
// 4) for warp w) and add them into H with TMA reduce-adds.  Barriers: full /
// empty per ring stage, acc_full / acc_empty per accumulator.
__global__ void __launch_bounds__(TC_THREADS, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmH,
                  int64_t T, int64_t n, int nt, int ntiles, int32_t* info) {
  extern __shared__ unsigned char smraw[];
  // 1024-byte aligned ring and staging (128-byte swizzle atoms are 1 KB)
  const uint32_t raw = smem_addr(smraw);
  unsigned char* ring = smraw + ((1024 - (raw & 1023)) & 1023);
  unsigned char* stag = ring + TC_RING;
  uint64_t* full = reinterpret_cast<uint64_t*>(stag + TC_STAGING);
  uint64_t* empty = full + TC_STAGES;
  uint64_t* accf = empty + TC_STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  int* issued = const_cast<int*>(abort_flag + 1);
  volatile int* ep_ok = abort_flag + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = (int)((T + TC_KT - 1) / TC_KT);
  const int ntl = (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4 * 32);
    }
    *abort_flag = 0;
    *issued = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 2 * TC_TILE);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer
      uint32_t g = 0;
      for (int it = 0; it < ntl && !*abort_flag; ++it) {
        int bi, bj;
        upper_tile((int)blockIdx.x + it * (int)gridDim.x, nt, bi, bj);
        const bool diag = bi == bj;
        const int i0 = bi * TC_TILE, j0 = bj * TC_TILE;
        for (int c = 0; c < nk; ++c, ++g) {
          const int s = (int)(g % TC_STAGES);
          if (g >= TC_STAGES && !mbar_wait_bounded(&empty[s], ((g / TC_STAGES) - 1) & 1)) {
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
      }
      *issued = (int)g;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer
      uint32_t g = 0;
      bool stop = false;
      for (int it = 0; it < ntl && !stop; ++it) {
        int bi, bj;
        upper_tile((int)blockIdx.x + it * (int)gridDim.x, nt, bi, bj);
        const bool diag = bi == bj;
        const int ac = it & 1;
        if (it >= 2 && !mbar_wait_bounded(&acce[ac], ((it - 2) >> 1) & 1)) {
          report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
          *abort_flag = 1;
          stop = true;
        }
        tc_fence_after();
        const uint32_t td = tmem + (uint32_t)(ac * TC_TILE);
        for (int c = 0; c < nk && !stop; ++c, ++g) {
          const int s = (int)(g % TC_STAGES);
          if (!mbar_wait_bounded(&full[s], (g / TC_STAGES) & 1)) {
            report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
            *abort_flag = 1;
            stop = true;
            break;
          }
          if (*abort_flag) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_addr(ring + s * TC_STAGE_BYTES);
          const uint32_t b = diag ? a : a + TC_OPER_BYTES;
#pragma unroll
          for (int ks = 0; ks < TC_KT / 16; ++ks) {
            // 16 tokens = two 8-row swizzle atoms (2 × 1024 B) further along K;
            // the second 64-column half of the operand sits one box further.
            const uint64_t ad = sdesc_sw128(a + ks * 2048, TC_BOX_BYTES, 1024);
            const uint64_t bd = sdesc_sw128(b + ks * 2048, TC_BOX_BYTES, 1024);
            umma_f16_ss(td, ad, bd, TC_IDESC, (c > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&accf[ac]);   // also after a stop: retires the products in flight
      }
    }
  } else {
    // ---- epilogue: warps 2–5, one accumulator row per thread
    const int et = tid - 64, qw = warp & 3, r = 32 * qw + lane;
    for (int it = 0; it < ntl; ++it) {
      int bi, bj;
      upper_tile((int)blockIdx.x + it * (int)gridDim.x, nt, bi, bj);
      const bool diag = bi == bj;
      const int i0 = bi * TC_TILE, j0 = bj * TC_TILE;
      const int ac = it & 1;
      // one thread waits for the accumulator (and, the staging being reused,
      // for the previous tile's reduce-adds to have read it); the barrier
      // hands the outcome to the other epilogue threads
      if (et == 0) {
        *ep_ok = mbar_wait_bounded(&accf[ac], (it >> 1) & 1) ? 1 : 0;
        if (!*ep_ok) {
          report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
          *abort_flag = 1;
        }
        bulk_wait_read_all();
      }
      named_bar_sync(1, 128);
      if (!*ep_ok) break;
      tc_fence_after();
      const bool write = !*abort_flag;
      if (write) {
#pragma unroll 1
        for (int ch = 0; ch < TC_TILE / 32; ++ch) {
          float v[32];
          tmem_ld_32x32b_x32(tmem + (uint32_t)(ac * TC_TILE) + ((uint32_t)(32 * qw) << 16) + ch * 32, v);
          unsigned char* box = stag + ch * EP_BOX + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(box + ((q ^ (r & 7)) << 4)) =
                make_float4(2.f * v[4 * q], 2.f * v[4 * q + 1], 2.f * v[4 * q + 2], 2.f * v[4 * q + 3]);
          if (!diag) {
            // Dᵀ: row c = 32·ch + k of the mirrored tile, column r
            unsigned char* mbox = stag + (4 + qw) * EP_BOX;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int cc = 32 * ch + k;
              *reinterpret_cast<float*>(mbox + cc * 128 + (((lane >> 2) ^ (cc & 7)) << 4) + (lane & 3) * 4) =
                  2.f * v[k];
            }
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(&acce[ac]);          // this thread is done with the accumulator
      named_bar_sync(1, 128);          // every staging box is written, ep_ok read
      if (write && et == 0) {
#pragma unroll 1
        for (int b = 0; b < TC_TILE / 32; ++b) {
          if (j0 + 32 * b < n) tma_reduce_add_2d(&tmH, j0 + 32 * b, i0, stag + b * EP_BOX);
          if (!diag && i0 + 32 * b < n)
            tma_reduce_add_2d(&tmH, i0 + 32 * b, j0, stag + (4 + b) * EP_BOX);
        }
        bulk_commit();
      }
    }
    if (et == 0) bulk_wait_all();      // H holds every sum before the CTA leaves
  }

  // ---- teardown: no copy or product may still be in flight when TMEM goes
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    const int g = *issued;
    for (int k = g - TC_STAGES; k < g; ++k)
      if (k >= 0) mbar_wait_bounded(&full[k % TC_STAGES], (k / TC_STAGES) & 1, 1u << 16);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 2 * TC_TILE);
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
    int sms = 0;
    {
      const gptq_status st = device_sm_count(&sms);
      if (st != GPTQ_OK) return st;
    }
    const int nt = (int)ceil_div(n, TC_TILE);
    const int ntiles = nt * (nt + 1) / 2;
    const int grid = ntiles < sms ? ntiles : sms;
    GPTQ_LAUNCH(KK_HESSIAN, s, hessian_tc_kernel, grid, TC_THREADS, TC_SMEM, tm, th, T, n, nt,
                ntiles, info);
    return GPTQ_OK;
  }
  const int nt = (int)ceil_div(n, HT);
  GPTQ_LAUNCH(KK_HESSIAN, s, hessian_simt_kernel, nt * (nt + 1) / 2, 256, 0,
              static_cast<const __nv_bfloat16*>(X), T, n, nt, H);
  return GPTQ_OK;
}
