// Shared plumbing of the GPTQ kernels: kernel kinds, launch bookkeeping,
// error reporting through the caller's device `info` words.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>
#include <cstddef>

#include "../../include/gptq_b200.h"

namespace gptq {

// Kernel kinds, for the launch counter and the event profiler.
enum KernelKind : int {
  KK_HESSIAN = 0,     // H += 2·XᵀX
  KK_PREP_STATS,      // mean(diag H), dead columns, order keys
  KK_PREP_ORDER,      // processing permutation
  KK_PREP_GATHER,     // reversed, permuted, damped float64 copy of H
  KK_CHOL,            // blocked Cholesky + triangular inverse (one dataflow launch)
  KK_PREP_OUT,        // U = reversed L⁻¹, rounded to float32
  KK_INGEST,          // W → float32 working copy in processing order
  KK_SWEEP,           // one block of the column sweep (+ the far update of the block before)
  KK_TRAIL,           // TF32 split of U, or the SIMT lazy-batch trailing update
  KK_PACK,            // codes → packed words, g_idx, dequantized copy
  KK_CHMC,            // CHMC frontend: activation energies, randomized subspace iteration, residual
  KK_SSQR,            // SSQR: the binary search's state, the outlier list
  KK_HPTQ,            // HPTQ: histogram, Huffman code and search step, encoder
  KK_PROBE,           // peak probes (float64, TF32, bf16 tensor pipes)
  KK_COUNT
};

const char* kernel_kind_name(int k);

// Launch bookkeeping (counter always; CUDA events when profiling is on).
void launch_begin(int kind, cudaStream_t s);
void launch_end(int kind, cudaStream_t s);

// Record a failure message for gptq_last_error() and return `st`.
gptq_status fail(gptq_status st, const char* fmt, ...);
gptq_status cuda_fail(cudaError_t e, const char* what);

// Per-device set-up.  A kernel's dynamic shared-memory limit is an attribute
// held by the device's context, and the SM count is a property of the device,
// so both are kept per device ordinal, under a lock (one process may drive
// several GPUs, from several host threads).  Each is set or read once per
// device, with that device current; a device reset between calls is not
// supported (the cached set-up would not be redone).
gptq_status ensure_smem_limit(const void* kernel, int bytes, const char* name);
gptq_status device_sm_count(int* sms);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Device-side error report: first error wins (status word goes 0 → st).
__device__ __forceinline__ void report(int32_t* info, int32_t st, int64_t index) {
  if (info == nullptr) return;
  if (atomicCAS(info, 0, st) == 0) info[1] = (int32_t)(index + 1);
}

}  // namespace gptq

#define GPTQ_LAUNCH(kind, stream, kernel, grid, block, smem, ...)              \
  do {                                                                         \
    gptq::launch_begin((kind), (stream));                                      \
    kernel<<<(grid), (block), (smem), (stream)>>>(__VA_ARGS__);                \
    gptq::launch_end((kind), (stream));                                        \
    cudaError_t e__ = cudaGetLastError();                                      \
    if (e__ != cudaSuccess) return gptq::cuda_fail(e__, #kernel);              \
  } while (0)

// The same with programmatic dependent launch: the kernel may start (and run
// its prologue) while the previous kernel of the stream finishes; it must
// execute pdl_wait() (sm100.cuh) before touching anything that kernel writes.
#define GPTQ_LAUNCH_PDL(kind, strm, kernel, grid, block, smem, ...)          \
  do {                                                                         \
    gptq::launch_begin((kind), (strm));                                        \
    cudaLaunchConfig_t cfg__ = {};                                             \
    cfg__.gridDim = dim3(grid);                                                \
    cfg__.blockDim = dim3(block);                                              \
    cfg__.dynamicSmemBytes = (smem);                                           \
    cfg__.stream = (strm);                                                     \
    cudaLaunchAttribute at__[1];                                               \
    at__[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;           \
    at__[0].val.programmaticStreamSerializationAllowed = 1;                    \
    cfg__.attrs = at__;                                                        \
    cfg__.numAttrs = 1;                                                        \
    cudaError_t e__ = cudaLaunchKernelEx(&cfg__, kernel, __VA_ARGS__);         \
    gptq::launch_end((kind), (strm));                                          \
    if (e__ != cudaSuccess) return gptq::cuda_fail(e__, #kernel);              \
  } while (0)

#define GPTQ_CUDA(call)                                                        \
  do {                                                                         \
    cudaError_t e__ = (call);                                                  \
    if (e__ != cudaSuccess) return gptq::cuda_fail(e__, #call);                \
  } while (0)
