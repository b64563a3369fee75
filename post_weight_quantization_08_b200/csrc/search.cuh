// The device-side binary search on a layer-wide scale factor α, shared by
// SSQR and HPTQ ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest
// Plane Algorithm", §3: both adjust the scales by a binary search, SSQR to an
// outlier density, HPTQ to a compression budget), and the row-pointer scan
// both use for their per-row outputs.
#pragma once

#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace gptq {
namespace {

struct SearchState {
  float lo, hi;             // the bracket: hi admissible (or α_hi), lo not
  float a;                  // the α of the next pass
  int32_t done;             // the search has ended: later passes run at hi
  unsigned long long count; // the running pass's measure (outliers, coded bits)
  // two bisection levels per round: the midpoint and both quarter points of
  // the level after it, evaluated side by side
  float cand[3];            // mid, lower quarter, upper quarter
  int32_t steps;            // bisection steps taken (pass 0 excluded)
  unsigned long long ccount[3];
};

__global__ void search_init_kernel(SearchState* st, float lo, float hi) {
  st->lo = lo;
  st->hi = hi;
  st->a = hi;
  st->done = 0;
  st->count = 0ull;
  st->steps = 0;
}

// (lo + hi)/2 rounded once to float32 (exact in double for float operands).
__host__ __device__ __forceinline__ float bisect_mid(float lo, float hi) {
#ifdef __CUDA_ARCH__
  return __double2float_rn(((double)lo + (double)hi) * 0.5);
#else
  return (float)(((double)lo + (double)hi) * 0.5);   // round to nearest even
#endif
}

// After pass k (run at st->a, whose measure is st->count): pass 0 evaluates
// α_hi, and a measure over `limit` there ends the search.  Later passes
// evaluate the bracket's midpoint and keep it as hi when admissible (measure
// ≤ limit), else as lo.  The next midpoint is (lo + hi)/2 rounded once to
// float32; one equal to an end of the bracket ends the search.  The trace
// records (α, measure) per pass, −1 for a pass run after the end.
__host__ __device__ __forceinline__ void search_step(SearchState* st, int k, long long limit,
                                                     float* trace_alpha, int64_t* trace_count) {
  const unsigned long long c = st->count;
  const float a = st->a;
  const bool was_done = st->done != 0;
  if (trace_alpha != nullptr) trace_alpha[k] = a;
  if (trace_count != nullptr) trace_count[k] = was_done ? -1 : (int64_t)c;
  if (!was_done) {
    bool done = false;
    if (k == 0) {
      done = c > (unsigned long long)limit;
    } else if (c <= (unsigned long long)limit) {
      st->hi = a;
    } else {
      st->lo = a;
    }
    if (!done) {
      const float mid = bisect_mid(st->lo, st->hi);
      if (mid <= st->lo || mid >= st->hi) done = true;
      else st->a = mid;
    }
    if (done) {
      st->done = 1;
      st->a = st->hi;
    }
  }
  st->count = 0ull;
}

// Before a round: the candidates are the next midpoint (st->a, set by the
// step before) and the midpoints of its two halves, each rounded as a
// bisection step would round it.  After the search has ended all three are hi.
__host__ __device__ __forceinline__ void search_plan(SearchState* st) {
  if (st->done) {
    st->cand[0] = st->cand[1] = st->cand[2] = st->hi;
  } else {
    const float mid = st->a;
    st->cand[0] = mid;
    st->cand[1] = bisect_mid(st->lo, mid);
    st->cand[2] = bisect_mid(mid, st->hi);
  }
  st->ccount[0] = st->ccount[1] = st->ccount[2] = 0ull;
}

__global__ void search_plan_kernel(SearchState* st) { search_plan(st); }

// After a round (its first trace entry k0): the midpoint's measure decides
// the first level exactly as a bisection step; the second level's midpoint is
// then the quarter on the side kept, whose measure decides it.  A midpoint
// equal to an end of the bracket, or `iters` steps, ends the search; trace
// entries of steps not taken read (hi, −1).
__host__ __device__ __forceinline__ void search_decide(SearchState* st, int k0, int iters,
                                                       long long limit, float* trace_alpha,
                                                       int64_t* trace_count) {
  bool lower = false;                 // the first level kept the lower half
  for (int lev = 0; lev < 2; ++lev) {
    const int k = k0 + lev;
    if (k > iters) break;
    if (st->done) {
      if (trace_alpha != nullptr) trace_alpha[k] = st->hi;
      if (trace_count != nullptr) trace_count[k] = -1;
      continue;
    }
    const float a = st->a;
    const int slot = lev == 0 ? 0 : (lower ? 1 : 2);
    const unsigned long long c = st->ccount[slot];
    if (trace_alpha != nullptr) trace_alpha[k] = a;
    if (trace_count != nullptr) trace_count[k] = (int64_t)c;
    if (c <= (unsigned long long)limit) {
      st->hi = a;
      lower = true;
    } else {
      st->lo = a;
      lower = false;
    }
    st->steps += 1;
    const float mid = bisect_mid(st->lo, st->hi);
    if (mid <= st->lo || mid >= st->hi || st->steps >= iters) {
      st->done = 1;
      st->a = st->hi;
    } else {
      st->a = mid;
    }
  }
}

__global__ void search_decide_kernel(SearchState* st, int k0, int iters, long long limit,
                                     float* trace_alpha, int64_t* trace_count) {
  search_decide(st, k0, iters, limit, trace_alpha, trace_count);
}

// Two streams forked from a caller's stream for the round's side passes, and
// the events that fork and join them; one set per (device, caller stream),
// created on first use and kept for the life of the process.
struct ForkStreams {
  cudaStream_t side[2] = {nullptr, nullptr};
  cudaEvent_t fork = nullptr;
  cudaEvent_t join[2] = {nullptr, nullptr};
};

inline gptq_status fork_streams_for(cudaStream_t s, ForkStreams** out) {
  static std::mutex mu;
  static std::map<std::pair<int, cudaStream_t>, ForkStreams> reg;
  int dev = 0;
  GPTQ_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(mu);
  ForkStreams& f = reg[{dev, s}];
  if (f.side[0] == nullptr) {
    for (int i = 0; i < 2; ++i) {
      GPTQ_CUDA(cudaStreamCreateWithFlags(&f.side[i], cudaStreamNonBlocking));
      GPTQ_CUDA(cudaEventCreateWithFlags(&f.join[i], cudaEventDisableTiming));
    }
    GPTQ_CUDA(cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming));
  }
  *out = &f;
  return GPTQ_OK;
}

// One round: plan the three candidates, run `pass(slot, stream)` for the
// midpoint on the caller's stream and for the two quarter points on forked
// streams, join, and decide two levels (trace entries k0 and k0 + 1).
template <typename Pass>
gptq_status search_round(SearchState* st, int k0, int iters, long long limit, float* trace_alpha,
                         int64_t* trace_count, int kind, cudaStream_t s, Pass&& pass) {
  ForkStreams* f = nullptr;
  gptq_status r = fork_streams_for(s, &f);
  if (r != GPTQ_OK) return r;
  GPTQ_LAUNCH(kind, s, search_plan_kernel, 1, 1, 0, st);
  GPTQ_CUDA(cudaEventRecord(f->fork, s));
  for (int i = 0; i < 2; ++i) GPTQ_CUDA(cudaStreamWaitEvent(f->side[i], f->fork, 0));
  r = pass(0, s);
  if (r != GPTQ_OK) return r;
  for (int i = 0; i < 2; ++i) {
    r = pass(i + 1, f->side[i]);
    if (r != GPTQ_OK) return r;
    GPTQ_CUDA(cudaEventRecord(f->join[i], f->side[i]));
    GPTQ_CUDA(cudaStreamWaitEvent(s, f->join[i], 0));
  }
  GPTQ_LAUNCH(kind, s, search_decide_kernel, 1, 1, 0, st, k0, iters, limit, trace_alpha,
              trace_count);
  return GPTQ_OK;
}

// ptr[0] = 0, ptr[r+1] = Σ_{i≤r} cnt[i] (one CTA of 1024 threads: a
// contiguous run of rows per thread, a block-wide scan of the runs' sums).
// Reports CAPACITY when the total exceeds `cap`, and writes st->hi to
// alpha_out.
__global__ void __launch_bounds__(1024)
row_scan_kernel(const int32_t* __restrict__ cnt, int64_t m, int64_t* __restrict__ ptr,
                int64_t cap, const SearchState* st, float* alpha_out, int32_t* info) {
  __shared__ long long wsum[32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t per = (m + 1023) / 1024;
  const int64_t r0 = min(m, (int64_t)t * per), r1 = min(m, r0 + per);
  long long mine = 0;
  for (int64_t r = r0; r < r1; ++r) mine += cnt[r];
  long long x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  long long base = x - mine + (warp > 0 ? wsum[warp - 1] : 0ll);
  if (t == 0) ptr[0] = 0;
  for (int64_t r = r0; r < r1; ++r) {
    base += cnt[r];
    ptr[r + 1] = base;
  }
  if (t == 0) {
    const long long total = wsum[31];
    if (total > cap) report(info, GPTQ_ERR_CAPACITY, total < 0x7ffffffe ? total : 0x7ffffffe);
    if (alpha_out != nullptr) *alpha_out = st->hi;
  }
}

}  // namespace
}  // namespace gptq
