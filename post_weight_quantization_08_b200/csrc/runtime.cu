// Host runtime of the library: error strings, the launch counter, the
// CUDA-event kernel profiler and gptq_check().
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gptq {

namespace {

thread_local char g_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};

const char* const kKindNames[KK_COUNT] = {
    "hessian",  "prep_stats", "prep_order", "prep_gather", "cholesky",
    "prep_out", "ingest",     "sweep",      "trailing",    "pack",
    "chmc",     "ssqr",       "hptq",        "probe"};

struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> ev;   // 2 per slot
  std::vector<int> kind;
  size_t used = 0;
  double total_ms[KK_COUNT] = {};
  int64_t count[KK_COUNT] = {};
  bool pending = false;          // an event was recorded between begin/end
};

Profiler& prof() {
  static Profiler p;
  return p;
}

}  // namespace

const char* kernel_kind_name(int k) {
  return (k >= 0 && k < KK_COUNT) ? kKindNames[k] : "?";
}

gptq_status fail(gptq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

gptq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(GPTQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

void launch_begin(int kind, cudaStream_t s) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  Profiler& p = prof();
  if (!p.on) return;
  std::lock_guard<std::mutex> lk(p.mu);
  p.pending = false;
  if (!p.on || p.used >= p.kind.size()) return;
  if (cudaEventRecord(p.ev[2 * p.used], s) == cudaSuccess) p.pending = true;
}

void launch_end(int kind, cudaStream_t s) {
  Profiler& p = prof();
  if (!p.on) return;
  std::lock_guard<std::mutex> lk(p.mu);
  if (!p.pending || p.used >= p.kind.size()) return;
  if (cudaEventRecord(p.ev[2 * p.used + 1], s) == cudaSuccess) {
    p.kind[p.used] = kind;
    ++p.used;
  }
  p.pending = false;
}

namespace {

constexpr int kMaxDev = 128;

struct DeviceSetup {
  std::mutex mu;
  // (device, kernel) pairs whose limit is set, with the limit
  std::vector<std::pair<std::pair<int, const void*>, int>> smem;
  int sms[kMaxDev] = {};
};

DeviceSetup& setup() {
  static DeviceSetup d;
  return d;
}

}  // namespace

gptq_status ensure_smem_limit(const void* kernel, int bytes, const char* name) {
  int dev = 0;
  GPTQ_CUDA(cudaGetDevice(&dev));
  DeviceSetup& d = setup();
  std::lock_guard<std::mutex> lk(d.mu);
  for (auto& e : d.smem)
    if (e.first.first == dev && e.first.second == kernel) {
      if (e.second >= bytes) return GPTQ_OK;
      cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           bytes);
      if (r != cudaSuccess) return cuda_fail(r, name);
      e.second = bytes;
      return GPTQ_OK;
    }
  cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes);
  if (r != cudaSuccess) return cuda_fail(r, name);
  d.smem.push_back({{dev, kernel}, bytes});
  return GPTQ_OK;
}

gptq_status device_sm_count(int* sms) {
  int dev = 0;
  GPTQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDev) return fail(GPTQ_ERR_INVALID_ARG, "device ordinal %d", dev);
  DeviceSetup& d = setup();
  std::lock_guard<std::mutex> lk(d.mu);
  if (d.sms[dev] == 0) {
    int v = 0;
    GPTQ_CUDA(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev));
    d.sms[dev] = v;
  }
  *sms = d.sms[dev];
  return GPTQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_tiled_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner,
                     uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(tm, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gptq

using namespace gptq;

extern "C" {

const char* gptq_last_error(void) { return g_last_error; }

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "GPTQ_OK";
    case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
    case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD";
    case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
    case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
    case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
    case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
    case GPTQ_ERR_CAPACITY: return "GPTQ_ERR_CAPACITY";
    default: return "GPTQ_ERR_UNKNOWN";
  }
}

uint64_t gptq_launch_count(void) { return g_launches.load(); }

int gptq_kernel_kinds(void) { return KK_COUNT; }

const char* gptq_kernel_name(int kind) { return kernel_kind_name(kind); }

gptq_status gptq_check(const int32_t* info, int32_t* index, void* stream) {
  if (info == nullptr) return fail(GPTQ_ERR_INVALID_ARG, "gptq_check: info is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GPTQ_CUDA(cudaStreamSynchronize(s));
  int32_t h[2] = {0, 0};
  GPTQ_CUDA(cudaMemcpy(h, info, sizeof(h), cudaMemcpyDeviceToHost));
  if (index) *index = h[1];
  if (h[0] < 0 || h[0] > GPTQ_ERR_CAPACITY)
    return fail(GPTQ_ERR_CUDA, "gptq_check: corrupt info word %d", h[0]);
  return static_cast<gptq_status>(h[0]);
}

gptq_status gptq_profile_start(int capacity) {
  if (capacity < 1) return fail(GPTQ_ERR_INVALID_ARG, "profile capacity < 1");
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  for (cudaEvent_t e : p.ev) cudaEventDestroy(e);
  p.ev.assign(2 * (size_t)capacity, nullptr);
  for (auto& e : p.ev) GPTQ_CUDA(cudaEventCreate(&e));
  p.kind.assign((size_t)capacity, -1);
  p.used = 0;
  for (int k = 0; k < KK_COUNT; ++k) { p.total_ms[k] = 0; p.count[k] = 0; }
  p.on = true;
  return GPTQ_OK;
}

gptq_status gptq_profile_stop(void) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  p.on = false;
  for (size_t i = 0; i < p.used; ++i) {
    GPTQ_CUDA(cudaEventSynchronize(p.ev[2 * i + 1]));
    float ms = 0.f;
    GPTQ_CUDA(cudaEventElapsedTime(&ms, p.ev[2 * i], p.ev[2 * i + 1]));
    int k = p.kind[i];
    if (k >= 0 && k < KK_COUNT) { p.total_ms[k] += ms; p.count[k] += 1; }
  }
  for (cudaEvent_t e : p.ev) cudaEventDestroy(e);
  p.ev.clear();
  p.kind.clear();
  p.used = 0;
  return GPTQ_OK;
}

gptq_status gptq_profile_get(int kind, double* total_ms, int64_t* launches) {
  if (kind < 0 || kind >= KK_COUNT)
    return fail(GPTQ_ERR_INVALID_ARG, "profile kind %d out of range", kind);
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (total_ms) *total_ms = p.total_ms[kind];
  if (launches) *launches = p.count[kind];
  return GPTQ_OK;
}

}  // extern "C"
