// Peak probes: kernels that keep one arithmetic pipe busy and nothing else,
// so that a caller timing them with CUDA events measures the pipe's rate on
// this GPU (the denominators of the float64 and TF32 rooflines).
//
//   kind 0  float64 tensor-core products (mma.sync m8n8k4 .f64), eight
//           independent accumulators per warp, 8 warps per CTA, 4 CTAs per SM
//   kind 1  tcgen05.mma kind::tf32, M = 128, N = 256, K = 8, operands in
//           shared memory (zeros), accumulator in tensor memory, one issuing
//           thread per CTA, one CTA per SM
//   kind 2  the same with kind::f16 (bf16 operands, K = 16)
//   kind 3  kind 0 with one CTA of 8 warps per SM (two warps per scheduler,
//           the occupancy of the float64 factorisation's CTAs)
//
// The operands' values do not matter for the rate; nothing is read from or
// written to global memory except one sink word that is never written in
// practice (it keeps the products alive).
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace gptq {
namespace {

__device__ __forceinline__ void dmma884(double (&d)[2], double a, double b) {
  asm volatile(
      "mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
      : "+d"(d[0]), "+d"(d[1])
      : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(256) probe_dmma_kernel(int64_t iters, double* sink,
                                                         double never) {
  double a = 1.0 + threadIdx.x * 1e-9, b = 1.0 - blockIdx.x * 1e-9;
  double acc[8][2] = {};
  for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
    for (int k = 0; k < 8; ++k) dmma884(acc[k], a, b);
  }
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) s += acc[k][0] + acc[k][1];
  if (s == never) sink[0] = s;
}

constexpr int PA_BYTES = 128 * 128;   // A: 128 rows × 128 bytes (K-major, 128-byte swizzle)
constexpr int PB_BYTES = 256 * 128;   // B: 256 rows × 128 bytes
constexpr int PROBE_SMEM = PA_BYTES + PB_BYTES + 1024;

template <int KIND>
__global__ void __launch_bounds__(128, 1) probe_umma_kernel(int64_t iters, int32_t* info) {
  extern __shared__ unsigned char smraw[];
  __shared__ uint64_t done;
  __shared__ uint32_t tslot;
  const uint32_t raw = smem_addr(smraw);
  unsigned char* base = smraw + ((1024 - (raw & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < (PA_BYTES + PB_BYTES) / 16; i += 128)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tslot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  if (tid == 0) {
    const uint32_t a = smem_addr(base), b = a + PA_BYTES;
    constexpr uint32_t fmt = KIND == 1 ? 2u : 1u;     // tf32 or bf16
    constexpr uint32_t idesc = idesc_f32acc(fmt, fmt, 0, 0, 128, 256);
    for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {                 // 32 bytes of K per product
        const uint64_t ad = sdesc_sw128(a + ks * 32, SW128_KMAJOR_LBO, 1024);
        const uint64_t bd = sdesc_sw128(b + ks * 32, SW128_KMAJOR_LBO, 1024);
        if (KIND == 1)
          umma_tf32_ss(tmem, ad, bd, idesc, (i > 0 || ks > 0) ? 1u : 0u);
        else
          umma_f16_ss(tmem, ad, bd, idesc, (i > 0 || ks > 0) ? 1u : 0u);
      }
    }
    umma_commit(&done);
  }
  __syncwarp();
  bool ok = true;
  if (tid == 0) ok = mbar_wait_bounded(&done, 0);
  if (!ok) report(info, GPTQ_ERR_TIMEOUT, blockIdx.x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_peak_probe(int kind, int64_t iters, double* flops, int32_t* info,
                                       void* sink, void* stream) {
  if (kind < 0 || kind > 3 || iters < 1 || !flops || !info || !sink)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_peak_probe: kind=%d iters=%lld", kind,
                (long long)iters);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int sms = 0;
  {
    const gptq_status st = device_sm_count(&sms);
    if (st != GPTQ_OK) return st;
  }
  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  if (kind == 0 || kind == 3) {
    const int grid = (kind == 0 ? 4 : 1) * sms;
    GPTQ_LAUNCH(KK_PROBE, s, probe_dmma_kernel, grid, 256, 0, iters,
                static_cast<double*>(sink), -1.2345e300);
    *flops = (double)grid * 8 * 8 * (double)iters * 2.0 * 8 * 8 * 4;
    return GPTQ_OK;
  }
  const void* fn = kind == 1 ? (const void*)probe_umma_kernel<1> : (const void*)probe_umma_kernel<2>;
  {
    const gptq_status st = ensure_smem_limit(fn, PROBE_SMEM, "probe_umma_kernel");
    if (st != GPTQ_OK) return st;
  }
  if (kind == 1)
    GPTQ_LAUNCH(KK_PROBE, s, probe_umma_kernel<1>, sms, 128, PROBE_SMEM, iters, info);
  else
    GPTQ_LAUNCH(KK_PROBE, s, probe_umma_kernel<2>, sms, 128, PROBE_SMEM, iters, info);
  const double k = kind == 1 ? 8.0 : 16.0;
  *flops = (double)sms * (double)iters * 4.0 * 2.0 * 128 * 256 * k;
  return GPTQ_OK;
}
