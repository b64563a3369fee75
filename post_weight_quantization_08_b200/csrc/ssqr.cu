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
// scale factor α (the sweep kernel's outlier variant reads α from the search
// state and counts its outliers there).  After the pass at α_hi, each round
// runs the bracket's midpoint and both quarter points of the next level side
// by side on three streams, and a one-thread kernel takes the two bisection
// steps they decide (search.cuh): the same steps as one pass at a time, in
// half the passes on the critical path.  No host round trip, so the whole
// call can be captured in a CUDA graph.  A last pass at the chosen α produces the
// outputs; the outlier list is then compacted into CSR (one warp per row,
// original column order) and the codes are packed.
#include <cmath>

#include "kernels.cuh"
#include "search.cuh"

namespace gptq {
namespace {

// The workspace: the call's working set (slot 0, which also holds the
// U-derived parts), two more for the quarter-point passes of a round, the
// search state, and per slot the row counts and the scale and zero of its
// pass (slot 0 uses the caller's).
struct SsqrWs {
  QuantWs w[3];
  SearchState* st;
  int32_t* row_cnt[3];
  float* scale[3];
  uint8_t* zero[3];
};

size_t ssqr_ws_layout(int64_t m, int64_t n, int block, SsqrWs* o, char* base) {
  size_t off = quant_ws_layout(m, n, block, o ? &o->w[0] : nullptr, base);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t ngmax = (size_t)ceil_div(n, 32);        // group ≥ 32
  const size_t o_st = take(sizeof(SearchState));
  size_t o_cnt[3], o_sc[3], o_z[3], o_slot[3];
  for (int k = 0; k < 3; ++k) o_cnt[k] = take(sizeof(int32_t) * (size_t)m);
  for (int k = 1; k < 3; ++k) {
    o_sc[k] = take(sizeof(float) * (size_t)m * ngmax);
    o_z[k] = take((size_t)m * ngmax);
    o_slot[k] = take(quant_slot_layout(m, n, block, nullptr, nullptr, nullptr));
  }
  if (base && o) {
    o->st = reinterpret_cast<SearchState*>(base + o_st);
    for (int k = 0; k < 3; ++k) o->row_cnt[k] = reinterpret_cast<int32_t*>(base + o_cnt[k]);
    o->scale[0] = nullptr;
    o->zero[0] = nullptr;
    for (int k = 1; k < 3; ++k) {
      o->scale[k] = reinterpret_cast<float*>(base + o_sc[k]);
      o->zero[k] = reinterpret_cast<uint8_t*>(base + o_z[k]);
      quant_slot_layout(m, n, block, &o->w[0], &o->w[k], base + o_slot[k]);
    }
  }
  return off;
}

// Between passes: the outlier count against the budget (search.cuh).
__global__ void ssqr_step_kernel(SearchState* st, int k, long long n_max, float* trace_alpha,
                                 int64_t* trace_count) {
  search_step(st, k, n_max, trace_alpha, trace_count);
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
  return ssqr_ws_layout(m, n, block, nullptr, nullptr);
}

extern "C" gptq_status gptq_ssqr_quantize(
    const void* W, int w_dtype, int64_t m, int64_t n, const float* U, const int32_t* perm,
    const uint8_t* dead, int bits, int group, int block, double target, int iters,
    float alpha_lo, float alpha_hi, int lookahead, uint32_t* qweight, float* scale, uint8_t* zero,
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
                          ? ssqr_ws_layout(m, n, block, nullptr, nullptr)
                          : 0;
  gptq_status st = quant_check_args(w_dtype, m, n, bits, group, block, ws, ws_bytes, need);
  if (st != GPTQ_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SsqrWs o;
  ssqr_ws_layout(m, n, block, &o, static_cast<char*>(ws));
  const QuantWs& w = o.w[0];
  SearchState* state = o.st;
  const long long n_max = (long long)std::floor(target * (double)m * (double)n);

  st = quant_setup(w, m, n, U, perm, group, block, g_idx, info, s);
  if (st != GPTQ_OK) return st;
  GPTQ_LAUNCH(KK_SSQR, s, search_init_kernel, 1, 1, 0, state, alpha_lo, alpha_hi);
  // pass 0 at α_hi
  OutlierArgs first;
  first.alpha = &state->a;
  first.row_cnt = o.row_cnt[0];
  first.total = &state->count;
  GPTQ_CUDA(cudaMemsetAsync(o.row_cnt[0], 0, sizeof(int32_t) * (size_t)m, s));
  st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, scale, zero,
                  nullptr, &first, info, s);
  if (st != GPTQ_OK) return st;
  GPTQ_LAUNCH(KK_SSQR, s, ssqr_step_kernel, 1, 1, 0, state, 0, n_max, trace_alpha,
              trace_count);
  // the bisection: one pass a step, or (lookahead) two levels a round, slot 0
  // the midpoint and slots 1 and 2 the quarter points side by side
  for (int k = 1; k <= iters && !lookahead; ++k) {
    GPTQ_CUDA(cudaMemsetAsync(o.row_cnt[0], 0, sizeof(int32_t) * (size_t)m, s));
    st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, scale, zero,
                    nullptr, &first, info, s);
    if (st != GPTQ_OK) return st;
    GPTQ_LAUNCH(KK_SSQR, s, ssqr_step_kernel, 1, 1, 0, state, k, n_max, trace_alpha,
                trace_count);
  }
  for (int k0 = 1; k0 <= iters && lookahead; k0 += 2) {
    st = search_round(state, k0, iters, n_max, trace_alpha, trace_count, KK_SSQR, s,
                      [&](int slot, cudaStream_t ss) -> gptq_status {
                        OutlierArgs a;
                        a.alpha = &state->cand[slot];
                        a.row_cnt = o.row_cnt[slot];
                        a.total = &state->ccount[slot];
                        GPTQ_CUDA(cudaMemsetAsync(o.row_cnt[slot], 0,
                                                  sizeof(int32_t) * (size_t)m, ss));
                        return quant_pass(o.w[slot], W, w_dtype, m, n, U, perm, dead, bits,
                                          group, block, 0, slot ? o.scale[slot] : scale,
                                          slot ? o.zero[slot] : zero, nullptr, &a, info, ss);
                      });
    if (st != GPTQ_OK) return st;
  }
  // the outputs: one more pass at the chosen α (the bracket's hi)
  OutlierArgs fin = first;
  fin.alpha = &state->hi;
  GPTQ_CUDA(cudaMemsetAsync(o.row_cnt[0], 0, sizeof(int32_t) * (size_t)m, s));
  st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, scale, zero,
                  loss_row, &fin, info, s);
  if (st != GPTQ_OK) return st;
  GPTQ_LAUNCH(KK_SSQR, s, row_scan_kernel, 1, 1024, 0, o.row_cnt[0], m, row_ptr, nnz_cap, state,
              alpha, info);
  GPTQ_LAUNCH(KK_SSQR, s, ssqr_fill_kernel, (unsigned)ceil_div(m, 8), 256, 0, w.codes, w.pinv,
              w.Wp, m, n, row_ptr, nnz_cap, col_idx, val);
  return quant_pack(w, m, n, bits, group, 0, scale, zero, qweight, Qdq, w.Wp, info, s);
}
