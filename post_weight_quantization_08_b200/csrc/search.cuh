// The device-side binary search on a layer-wide scale factor α, shared by
// SSQR and HPTQ ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest
// Plane Algorithm", §3: both adjust the scales by a binary search, SSQR to an
// outlier density, HPTQ to a compression budget), and the row-pointer scan
// both use for their per-row outputs.
#pragma once

#include "common.cuh"

namespace gptq {
namespace {

struct SearchState {
  float lo, hi;             // the bracket: hi admissible (or α_hi), lo not
  float a;                  // the α of the next pass
  int32_t done;             // the search has ended: later passes run at hi
  unsigned long long count; // the running pass's measure (outliers, coded bits)
};

__global__ void search_init_kernel(SearchState* st, float lo, float hi) {
  st->lo = lo;
  st->hi = hi;
  st->a = hi;
  st->done = 0;
  st->count = 0ull;
}

// After pass k (run at st->a, whose measure is st->count): pass 0 evaluates
// α_hi, and a measure over `limit` there ends the search.  Later passes
// evaluate the bracket's midpoint and keep it as hi when admissible (measure
// ≤ limit), else as lo.  The next midpoint is (lo + hi)/2 rounded once to
// float32; one equal to an end of the bracket ends the search.  The trace
// records (α, measure) per pass, −1 for a pass run after the end.
__device__ __forceinline__ void search_step(SearchState* st, int k, long long limit,
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
      const float mid = __double2float_rn(((double)st->lo + (double)st->hi) * 0.5);
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
