// SSQR: GPTQ that keeps its overflowing weights instead of clipping them.
//
// "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
// Algorithm", §3: a small share of the weights (the outliers) stays in full
// precision as a sparse part, the inliers are quantized to a low bit width,
// and a binary search adjusts the scales until the outlier density meets a
// target.  §2.3 (Satz 5): clipping an overflowing weight breaks the error
// bound, which keeping it does not.
//
// The search runs on the device: one sweep of the whole layer per candidate
// scale factor α (the sweep kernel's outlier variant reads α from the state
// below and counts its outliers there), and a one-thread step kernel between
// the passes updates the bracket.  No host round trip, so the whole call can
// be captured in a CUDA graph.  A last pass at the chosen α produces the
// outputs; the outlier list is then compacted into CSR (one warp per row,
// original column order) and the codes are packed.
#include <cmath>

#include "kernels.cuh"

namespace gptq {
namespace {

struct SsqrState {
  float lo, hi;            // the bracket: hi admissible (or α_hi), lo not
  float a;                 // the α of the next pass
  int32_t done;            // the search has ended: later passes run at hi
  unsigned long long count;// outliers of the running pass
};

size_t ssqr_ws_layout(int64_t m, int64_t n, int block, QuantWs* w, SsqrState** st,
                      int32_t** row_cnt, char* base) {
  const size_t q = quant_ws_layout(m, n, block, w, base);
  const size_t o_st = q;
  const size_t o_cnt = align_up(o_st + sizeof(SsqrState), 256);
  const size_t end = align_up(o_cnt + sizeof(int32_t) * (size_t)m, 256);
  if (base) {
    *st = reinterpret_cast<SsqrState*>(base + o_st);
    *row_cnt = reinterpret_cast<int32_t*>(base + o_cnt);
  }
  return end;
}

__global__ void ssqr_init_kernel(SsqrState* st, float lo, float hi) {
  st->lo = lo;
  st->hi = hi;
  st->a = hi;
  st->done = 0;
  st->count = 0ull;
}

// After pass k (run at st->a with st->count outliers).  Pass 0 evaluates α_hi:
// over the budget ends the search there.  Later passes evaluate the bracket's
// midpoint and keep it as hi when admissible, else as lo.  The next midpoint
// is (lo + hi)/2 rounded once to float32; one equal to an end of the bracket
// ends the search.
__global__ void ssqr_step_kernel(SsqrState* st, int k, long long n_max, float* trace_alpha,
                                 int64_t* trace_count) {
  const unsigned long long c = st->count;
  const float a = st->a;
  const bool was_done = st->done != 0;
  if (trace_alpha != nullptr) trace_alpha[k] = a;
  if (trace_count != nullptr) trace_count[k] = was_done ? -1 : (int64_t)c;
  if (!was_done) {
    bool done = false;
    if (k == 0) {
      done = c > (unsigned long long)n_max;
    } else if (c <= (unsigned long long)n_max) {
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

// row_ptr[0] = 0, row_ptr[r+1] = Σ_{i≤r} cnt[i] (one CTA: a contiguous run of
// rows per thread, a block-wide scan of the runs' sums).  Reports CAPACITY
// when the total exceeds the caller's capacity, and writes the chosen α.
__global__ void __launch_bounds__(1024)
ssqr_scan_kernel(const int32_t* __restrict__ cnt, int64_t m, int64_t* __restrict__ row_ptr,
                 int64_t cap, const SsqrState* st, float* alpha_out, int32_t* info) {
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
  if (t == 0) row_ptr[0] = 0;
  for (int64_t r = r0; r < r1; ++r) {
    base += cnt[r];
    row_ptr[r + 1] = base;
  }
  if (t == 0) {
    const long long total = wsum[31];
    if (total > cap) report(info, GPTQ_ERR_CAPACITY, total < 0x7ffffffe ? total : 0x7ffffffe);
    if (alpha_out != nullptr) *alpha_out = st->hi;
  }
}

// One warp per row: the row's flagged codes in original column order (32
// columns per step, a ballot and a prefix count place them), column index and
// kept value into the CSR arrays (entries at or beyond cap are dropped).
__global__ void __launch_bounds__(256)
ssqr_fill_kernel(const uint8_t* __restrict__ codes, const int32_t* __restrict__ pinv,
                 const float* __restrict__ Wp, int64_t m, int64_t n,
                 const int64_t* __restrict__ row_ptr, int64_t cap, int32_t* __restrict__ col_idx,
                 float* __restrict__ val) {
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= m) return;
  int64_t base = row_ptr[r];
  if (row_ptr[r + 1] == base) return;
  const uint8_t* cr = codes + r * n;
  for (int64_t c0 = 0; c0 < n; c0 += 32) {
    const int64_t c = c0 + lane;
    int32_t p = 0;
    bool f = false;
    if (c < n) {
      p = pinv[c];
      f = p >= 0 && p < n && (cr[p] & OUTLIER_FLAG) != 0;
    }
    const unsigned b = __ballot_sync(0xffffffffu, f);
    if (f) {
      const int64_t i = base + __popc(b & ((1u << lane) - 1u));
      if (i < cap) {
        col_idx[i] = (int32_t)c;
        val[i] = Wp[r * n + p];
      }
    }
    base += __popc(b);
  }
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" size_t gptq_ssqr_workspace_bytes(int64_t m, int64_t n, int block) {
  if (m < 1 || n < 1 || block < 1) return 0;
  return ssqr_ws_layout(m, n, block, nullptr, nullptr, nullptr, nullptr);
}

extern "C" gptq_status gptq_ssqr_quantize(
    const void* W, int w_dtype, int64_t m, int64_t n, const float* U, const int32_t* perm,
    const uint8_t* dead, int bits, int group, int block, double target, int iters,
    float alpha_lo, float alpha_hi, uint32_t* qweight, float* scale, uint8_t* zero,
    int32_t* g_idx, int64_t* row_ptr, int32_t* col_idx, float* val, int64_t nnz_cap,
    float* alpha, float* trace_alpha, int64_t* trace_count, float* loss_row, float* Qdq,
    int32_t* info, void* ws, size_t ws_bytes, void* stream) {
  if (!W || !U || !perm || !dead || !qweight || !scale || !zero || !g_idx || !row_ptr ||
      !info || !ws || (nnz_cap > 0 && (!col_idx || !val)))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_ssqr_quantize: null pointer");
  if (bits != 2 && bits != 3 && bits != 4)
    return fail(GPTQ_ERR_UNSUPPORTED, "gptq_ssqr_quantize: bits=%d (2, 3, 4)", bits);
  if (!(target >= 0.0 && target <= 1.0))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_ssqr_quantize: target=%g (0..1)", target);
  if (iters < 0 || iters > 64)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_ssqr_quantize: iters=%d (0..64)", iters);
  if (!(alpha_lo > 0.f && alpha_lo <= alpha_hi && alpha_hi <= 16.f))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_ssqr_quantize: alpha bracket [%g, %g]",
                (double)alpha_lo, (double)alpha_hi);
  if (nnz_cap < 0)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_ssqr_quantize: nnz_cap=%lld", (long long)nnz_cap);
  const size_t need = (m >= 1 && n >= 1 && block >= 1)
                          ? ssqr_ws_layout(m, n, block, nullptr, nullptr, nullptr, nullptr)
                          : 0;
  gptq_status st = quant_check_args(w_dtype, m, n, bits, group, block, ws, ws_bytes, need);
  if (st != GPTQ_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  QuantWs w;
  SsqrState* state = nullptr;
  int32_t* row_cnt = nullptr;
  ssqr_ws_layout(m, n, block, &w, &state, &row_cnt, static_cast<char*>(ws));
  const long long n_max = (long long)std::floor(target * (double)m * (double)n);

  st = quant_setup(w, m, n, U, perm, group, block, g_idx, info, s);
  if (st != GPTQ_OK) return st;
  GPTQ_LAUNCH(KK_SSQR, s, ssqr_init_kernel, 1, 1, 0, state, alpha_lo, alpha_hi);
  OutlierArgs search;
  search.alpha = &state->a;
  search.row_cnt = row_cnt;
  search.total = &state->count;
  for (int k = 0; k <= iters; ++k) {
    GPTQ_CUDA(cudaMemsetAsync(row_cnt, 0, sizeof(int32_t) * (size_t)m, s));
    st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, scale, zero,
                    loss_row, &search, info, s);
    if (st != GPTQ_OK) return st;
    GPTQ_LAUNCH(KK_SSQR, s, ssqr_step_kernel, 1, 1, 0, state, k, n_max, trace_alpha,
                trace_count);
  }
  // the outputs: one more pass at the chosen α (the bracket's hi)
  OutlierArgs fin = search;
  fin.alpha = &state->hi;
  GPTQ_CUDA(cudaMemsetAsync(row_cnt, 0, sizeof(int32_t) * (size_t)m, s));
  st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, scale, zero,
                  loss_row, &fin, info, s);
  if (st != GPTQ_OK) return st;
  GPTQ_LAUNCH(KK_SSQR, s, ssqr_scan_kernel, 1, 1024, 0, row_cnt, m, row_ptr, nnz_cap, state,
              alpha, info);
  GPTQ_LAUNCH(KK_SSQR, s, ssqr_fill_kernel, (unsigned)ceil_div(m, 8), 256, 0, w.codes, w.pinv,
              w.Wp, m, n, row_ptr, nnz_cap, col_idx, val);
  return quant_pack(w, m, n, bits, group, 0, scale, zero, qweight, Qdq, w.Wp, info, s);
}
