// HPTQ: GPTQ on one unbounded integer grid, Huffman-coded to a bit budget.
//
// "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
// Algorithm", §3: Huffman-encoded PTQ puts inliers and outliers on one
// integer grid without clipping and Huffman-codes the integers, so that the
// bit width follows the weight distribution while a compression budget is
// met; §4 names 3.125 bits per weight; §2.3 (Satz 5): without clipping the
// error bound holds.
//
// The grid is the lattice s·ℤ of each group (s = α·min-max step): with no
// clamp a zero point has no role, and a weight's integer is its coordinate
// k = rint(w/s), centred on 0, one code for every group.
//
// Every pass of the device-side search (search.cuh) is: the sweep's
// unclipped variant at α (int16 coordinates), a histogram of the codes over a
// window of GPTQ_HPTQ_SYMBOLS symbols, and a one-CTA Huffman construction
// whose optimal cost (coded bits) drives the bisection; after the pass at
// α_hi, a round runs the midpoint and both quarter points of the next level
// side by side and takes two steps.  A last pass at
// the chosen α is encoded: canonical codes, per-row bit counts, their scan,
// and one warp per row writing its codes most significant bit first.
#include <algorithm>
#include <cmath>

#include "kernels.cuh"
#include "search.cuh"

namespace gptq {
namespace {

constexpr int NSYM = GPTQ_HPTQ_SYMBOLS;
constexpr int SYM0 = GPTQ_HPTQ_SYMBOL_OFFSET;
constexpr int MAXLEN = 64;

// The workspace: three working sets (slot 0 the call's, with the U-derived
// parts; slots 1 and 2 for the quarter-point passes of a round), and per slot
// the lattice coordinates, histogram, scales and zero points of its pass
// (slot 0's scales are the caller's; the zero points of the min-max steps are
// written by the sweep and unused by the unbounded grid).
struct HptqWs {
  QuantWs w[3];
  SearchState* st;
  int16_t* codes16[3];          // m × n lattice coordinates, processing order
  unsigned long long* hist[3];  // NSYM counts of the slot's pass
  float* scale[3];
  uint8_t* zero[3];
  unsigned char* lens;          // NSYM code lengths (0: unused symbol)
  unsigned long long* canon;    // NSYM canonical code words (right-aligned)
  int32_t* rowbits;             // m coded bits per row
};

size_t hptq_ws_layout(int64_t m, int64_t n, int block, HptqWs* h, char* base) {
  size_t off = quant_ws_layout(m, n, block, h ? &h->w[0] : nullptr, base);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t ngmax = (size_t)ceil_div(n, 32);        // group ≥ 32
  const size_t o_st = take(sizeof(SearchState));
  size_t o_c[3], o_h[3], o_s[3], o_z[3], o_slot[3];
  for (int k = 0; k < 3; ++k) {
    o_c[k] = take(sizeof(int16_t) * (size_t)m * (size_t)n);
    o_h[k] = take(sizeof(unsigned long long) * NSYM);
    o_s[k] = take(sizeof(float) * (size_t)m * ngmax);
    o_z[k] = take((size_t)m * ngmax);
    o_slot[k] = k ? take(quant_slot_layout(m, n, block, nullptr, nullptr, nullptr)) : 0;
  }
  const size_t o_l = take(NSYM);
  const size_t o_k = take(sizeof(unsigned long long) * NSYM);
  const size_t o_r = take(sizeof(int32_t) * (size_t)m);
  if (base && h) {
    h->st = reinterpret_cast<SearchState*>(base + o_st);
    for (int k = 0; k < 3; ++k) {
      h->codes16[k] = reinterpret_cast<int16_t*>(base + o_c[k]);
      h->hist[k] = reinterpret_cast<unsigned long long*>(base + o_h[k]);
      h->scale[k] = reinterpret_cast<float*>(base + o_s[k]);
      h->zero[k] = reinterpret_cast<uint8_t*>(base + o_z[k]);
      if (k) quant_slot_layout(m, n, block, &h->w[0], &h->w[k], base + o_slot[k]);
    }
    h->lens = reinterpret_cast<unsigned char*>(base + o_l);
    h->canon = reinterpret_cast<unsigned long long*>(base + o_k);
    h->rowbits = reinterpret_cast<int32_t*>(base + o_r);
  }
  return off;
}

// Histogram of the codes over the symbol window (symbol = q + SYM0): a
// shared-memory histogram per CTA, lanes holding the same symbol adding
// once (match.any), then the CTA's non-zero bins into the global counts.  A
// code outside the window is reported (UNSUPPORTED, its flat index) and not
// counted.
__global__ void __launch_bounds__(512)
hptq_hist_kernel(const int16_t* __restrict__ codes, int64_t total,
                 unsigned long long* __restrict__ hist, int32_t* info) {
  __shared__ unsigned int h[NSYM];
  for (int i = threadIdx.x; i < NSYM; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e0 = (int64_t)blockIdx.x * blockDim.x; e0 < total; e0 += stride) {
    const int64_t e = e0 + threadIdx.x;
    int sym = -1;
    if (e < total) {
      sym = (int)codes[e] + SYM0;
      if (sym < 0 || sym >= NSYM) {
        report(info, GPTQ_ERR_UNSUPPORTED, e);
        sym = -1;
      }
    }
    const unsigned same = __match_any_sync(0xffffffffu, sym);
    if (sym >= 0 && lane == __ffs(same) - 1) atomicAdd(&h[sym], (unsigned)__popc(same));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NSYM; i += blockDim.x)
    if (h[i] != 0u) atomicAdd(&hist[i], (unsigned long long)h[i]);
}

// One CTA: the optimal prefix code of the pass's histogram, its cost, and
// (k ≥ 0) the bisection step on that cost, else the cost into *cost_out; with
// `final`, the code lengths and canonical code words for the encoder.
//  1. the used symbols, compacted in symbol order (a block scan);
//  2. sorted by (count, symbol) by rank counting;
//  3. Huffman's construction with two queues (sorted leaves, internal nodes
//     in creation order, whose weights never decrease), then depths from
//     the root down; one symbol alone gets length 1;
//  4. cost = Σ count·length;
//  5. canonical words: lengths counted per length, first word per length as
//     (previous first word + previous count) << 1, symbols in increasing
//     order taking consecutive words within their length.
constexpr size_t HUF_SMEM = (size_t)NSYM * 8 * 3 + (size_t)NSYM * 2 * 2 + (size_t)2 * NSYM * 4 +
                            (size_t)2 * NSYM + (MAXLEN + 1) * 8;
static_assert(HUF_SMEM <= 227 * 1024, "shared memory per CTA");
__global__ void __launch_bounds__(1024)
hptq_huffman_kernel(const unsigned long long* __restrict__ hist, SearchState* st, int k,
                    unsigned long long* cost_out,
                    long long limit, float* trace_alpha, int64_t* trace_count, int final_pass,
                    unsigned char* __restrict__ lens_out, unsigned long long* __restrict__ canon_out,
                    int32_t* info) {
  extern __shared__ unsigned long long hsm[];
  unsigned long long* cnt = hsm;                       // compacted counts, symbol order
  unsigned long long* scnt = cnt + NSYM;               // sorted counts
  unsigned long long* iw = scnt + NSYM;                // internal node weights
  unsigned short* sym = reinterpret_cast<unsigned short*>(iw + NSYM);   // compacted symbols
  unsigned short* ssym = sym + NSYM;                   // sorted symbols
  int* par = reinterpret_cast<int*>(ssym + NSYM);      // 2·NSYM parents
  unsigned char* dep = reinterpret_cast<unsigned char*>(par + 2 * NSYM);  // 2·NSYM depths
  unsigned long long* blc = reinterpret_cast<unsigned long long*>(dep + 2 * NSYM);  // MAXLEN+1
  __shared__ int wsum[32];
  __shared__ int K_s;
  __shared__ unsigned long long red[32];
  __shared__ int bad_len;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  // 1. compaction: thread t owns symbols 4t .. 4t+3
  int mine = 0;
  unsigned long long c4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c4[i] = hist[4 * t + i];
    mine += c4[i] != 0ull ? 1 : 0;
  }
  int x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  if (t == 0) bad_len = 0;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  int pos = x - mine + (warp > 0 ? wsum[warp - 1] : 0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (c4[i] != 0ull) {
      cnt[pos] = c4[i];
      sym[pos] = (unsigned short)(4 * t + i);
      ++pos;
    }
  }
  if (t == 0) K_s = wsum[31];
  __syncthreads();
  const int K = K_s;

  // 2. sort by (count, symbol): the rank of an entry is the number of smaller keys
  for (int i = t; i < K; i += blockDim.x) {
    const unsigned long long ci = cnt[i];
    const unsigned short si = sym[i];
    int r = 0;
    for (int j = 0; j < K; ++j) {
      const unsigned long long cj = cnt[j];
      r += (cj < ci || (cj == ci && sym[j] < si)) ? 1 : 0;
    }
    scnt[r] = ci;
    ssym[r] = si;
  }
  __syncthreads();

  // 3. the two-queue construction (leaves 0..K−1, internal nodes K..2K−2)
  if (t == 0 && K > 1) {
    int li = 0, ii = 0, ni = 0;
    for (int s = 0; s < K - 1; ++s) {
      int nd[2];
      unsigned long long wsum2 = 0ull;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (li < K && (ii >= ni || scnt[li] <= iw[ii])) {
          nd[q] = li;
          wsum2 += scnt[li];
          ++li;
        } else {
          nd[q] = K + ii;
          wsum2 += iw[ii];
          ++ii;
        }
      }
      iw[ni] = wsum2;
      par[nd[0]] = K + ni;
      par[nd[1]] = K + ni;
      ++ni;
    }
    dep[2 * K - 2] = 0;
    for (int j = K - 3; j >= 0; --j) {
      const int d = dep[par[K + j]] + 1;
      dep[K + j] = (unsigned char)(d > 255 ? 255 : d);
    }
  }
  __syncthreads();
  unsigned long long part = 0ull;
  for (int i = t; i < K; i += blockDim.x) {
    int d = K > 1 ? dep[par[i]] + 1 : 1;
    if (d > MAXLEN) {
      bad_len = 1;
      d = MAXLEN;
    }
    dep[i] = (unsigned char)d;
    part += scnt[i] * (unsigned long long)d;
  }
  // 4. cost
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_down_sync(0xffffffffu, part, o);
  if (lane == 0) red[warp] = part;
  __syncthreads();
  if (t == 0) {
    unsigned long long c = 0ull;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) c += red[w];
    if (bad_len) report(info, GPTQ_ERR_UNSUPPORTED, 0);
    if (k >= 0) {
      st->count = c;
      search_step(st, k, limit, trace_alpha, trace_count);
    } else if (cost_out != nullptr) {
      *cost_out = c;
    }
  }
  if (!final_pass) return;

  // 5. lengths per symbol and canonical words
  for (int i = t; i < NSYM; i += blockDim.x) {
    lens_out[i] = 0;
    canon_out[i] = 0ull;
  }
  __syncthreads();
  for (int i = t; i < K; i += blockDim.x) lens_out[ssym[i]] = dep[i];
  __syncthreads();
  if (t == 0) {
    for (int l = 0; l <= MAXLEN; ++l) blc[l] = 0ull;
    for (int i = 0; i < K; ++i) blc[dep[i]] += 1ull;
    unsigned long long next[MAXLEN + 1];
    unsigned long long code = 0ull;
    next[0] = 0ull;
    for (int l = 1; l <= MAXLEN; ++l) {                // blc[0] = 0: no code is empty
      code = (code + blc[l - 1]) << 1;
      next[l] = code;
    }
    for (int i = 0; i < K; ++i) {                      // increasing symbol order
      const int s = sym[i];
      const int l = lens_out[s];
      canon_out[s] = next[l]++;
    }
  }
}

// Coded bits per row: the sum of the code lengths of its codes.
__global__ void __launch_bounds__(256)
hptq_rowbits_kernel(const int16_t* __restrict__ codes, int64_t m, int64_t n,
                    const unsigned char* __restrict__ lens, int32_t* __restrict__ rowbits) {
  __shared__ unsigned char L[NSYM];
  for (int i = threadIdx.x; i < NSYM; i += blockDim.x) L[i] = lens[i];
  __syncthreads();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= m) return;
  const int16_t* cr = codes + r * n;
  int acc = 0;
  for (int64_t c = lane; c < n; c += 32) {
    const int s = (int)cr[c] + SYM0;
    acc += (s >= 0 && s < NSYM) ? (int)L[s] : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_down_sync(0xffffffffu, acc, o);
  if (lane == 0) rowbits[r] = acc;
}

// One warp per row, original column order, 32 columns a step: each lane's
// code word, a warp prefix sum of the lengths for its bit position, and the
// word's bits OR-ed into the stream (most significant bit first; a word of up
// to 64 bits touches at most three 32-bit stream words).  Words at or past
// `cap_words` are not written.
__global__ void __launch_bounds__(256)
hptq_encode_kernel(const int16_t* __restrict__ codes, const int32_t* __restrict__ pinv,
                   int64_t m, int64_t n, const unsigned char* __restrict__ lens,
                   const unsigned long long* __restrict__ canon,
                   const int64_t* __restrict__ row_off, unsigned int* __restrict__ out,
                   int64_t cap_words) {
  __shared__ unsigned char L[NSYM];
  __shared__ unsigned long long Cw[NSYM];
  for (int i = threadIdx.x; i < NSYM; i += blockDim.x) {
    L[i] = lens[i];
    Cw[i] = canon[i];
  }
  __syncthreads();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= m) return;
  int64_t base = row_off[r];
  const int16_t* cr = codes + r * n;
  for (int64_t c0 = 0; c0 < n; c0 += 32) {
    const int64_t c = c0 + lane;
    int len = 0;
    unsigned long long word = 0ull;
    if (c < n) {
      const int32_t p = pinv[c];
      if (p >= 0 && p < n) {
        const int s = (int)cr[p] + SYM0;
        if (s >= 0 && s < NSYM) {
          len = L[s];
          word = Cw[s];
        }
      }
    }
    int x = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int64_t pos = base + (x - len);
    if (len > 0) {
      const unsigned long long v = word << (64 - len);   // left-aligned
      const int64_t w0 = pos >> 5;
      const int off = (int)(pos & 31);
      const int64_t wl = (pos + len - 1) >> 5;           // last stream word touched
      const unsigned int p0 = (unsigned int)(v >> (32 + off));
      const unsigned int p1 = (unsigned int)((v << (32 - off)) >> 32);
      const unsigned int p2 = off > 0 ? (unsigned int)((v << (64 - off)) >> 32) : 0u;
      if (w0 < cap_words && p0) atomicOr(out + w0, p0);
      if (w0 + 1 <= wl && w0 + 1 < cap_words && p1) atomicOr(out + w0 + 1, p1);
      if (w0 + 2 <= wl && w0 + 2 < cap_words && p2) atomicOr(out + w0 + 2, p2);
    }
    base += __shfl_sync(0xffffffffu, x, 31);
  }
}

// The codes in original column order, and the dequantized copy s·k.
__global__ void __launch_bounds__(256)
hptq_out_kernel(const int16_t* __restrict__ codes16, const int32_t* __restrict__ pinv, int64_t m,
                int64_t n, int group, int64_t ngroups, const float* __restrict__ scale,
                int16_t* __restrict__ codes_out, float* __restrict__ Qdq) {
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= m * n) return;
  const int64_t r = e / n, c = e % n;
  const int32_t p = pinv[c];
  if (p < 0 || p >= n) return;
  const int16_t q = codes16[r * n + p];
  if (codes_out != nullptr) codes_out[e] = q;
  if (Qdq != nullptr) Qdq[e] = scale[r * ngroups + p / group] * (float)q;
}


// One pass of slot `slot` at *alpha: sweep (unclipped), histogram, Huffman;
// k ≥ 0: the bisection step on its cost; k < 0: the cost into *cost_out.
gptq_status hptq_pass(const HptqWs& h, int slot, const void* W, int w_dtype, int64_t m,
                      int64_t n, const float* U, const int32_t* perm, const uint8_t* dead,
                      int bits, int group, int block, float* scale, float* loss_row,
                      const float* alpha, int k, unsigned long long* cost_out, long long limit,
                      float* trace_alpha, int64_t* trace_count, int final_pass, int32_t* info,
                      cudaStream_t s) {
  OutlierArgs oa;
  oa.alpha = alpha;
  oa.unclipped = true;
  oa.codes16 = h.codes16[slot];
  GPTQ_CUDA(cudaMemsetAsync(h.hist[slot], 0, sizeof(unsigned long long) * NSYM, s));
  gptq_status st = quant_pass(h.w[slot], W, w_dtype, m, n, U, perm, dead, bits, group, block, 0,
                              scale, h.zero[slot], loss_row, &oa, info, s);
  if (st != GPTQ_OK) return st;
  const int64_t total = m * n;
  const unsigned gh = (unsigned)std::min<int64_t>(ceil_div(total, 512 * 8), 148 * 4);
  GPTQ_LAUNCH(KK_HPTQ, s, hptq_hist_kernel, gh > 0 ? gh : 1, 512, 0, h.codes16[slot], total,
              h.hist[slot], info);
  {
    const gptq_status st = ensure_smem_limit((const void*)hptq_huffman_kernel, (int)HUF_SMEM,
                                             "hptq_huffman_kernel");
    if (st != GPTQ_OK) return st;
  }
  GPTQ_LAUNCH(KK_HPTQ, s, hptq_huffman_kernel, 1, 1024, HUF_SMEM, h.hist[slot], h.st, k,
              cost_out, limit, trace_alpha, trace_count, final_pass, h.lens, h.canon, info);
  return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" size_t gptq_hptq_workspace_bytes(int64_t m, int64_t n, int block) {
  if (m < 1 || n < 1 || block < 1) return 0;
  return hptq_ws_layout(m, n, block, nullptr, nullptr);
}

extern "C" gptq_status gptq_hptq_quantize(
    const void* W, int w_dtype, int64_t m, int64_t n, const float* U, const int32_t* perm,
    const uint8_t* dead, int bits, int group, int block, double budget, int iters,
    float alpha_lo, float alpha_hi, int lookahead, int16_t* codes, float* scale,
    int32_t* g_idx, uint8_t* code_len, uint64_t* code_word, int64_t* row_off,
    uint32_t* stream_words, int64_t stream_cap, float* alpha, float* trace_alpha,
    int64_t* trace_bits, float* loss_row, float* Qdq, int32_t* info, void* ws,
    size_t ws_bytes, void* stream) {
  if (!W || !U || !perm || !dead || !scale || !g_idx || !code_len || !row_off ||
      !alpha || !info || !ws || (stream_cap > 0 && !stream_words))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hptq_quantize: null pointer");
  if (!(budget > 0.0 && budget <= 64.0))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hptq_quantize: budget=%g (0..64 bits)", budget);
  if (iters < 0 || iters > 64)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hptq_quantize: iters=%d (0..64)", iters);
  if (!(alpha_lo > 0.f && alpha_lo <= alpha_hi && alpha_hi <= 256.f))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hptq_quantize: alpha bracket [%g, %g]",
                (double)alpha_lo, (double)alpha_hi);
  if (stream_cap < 0)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_hptq_quantize: stream_cap=%lld",
                (long long)stream_cap);
  const size_t need = (m >= 1 && n >= 1 && block >= 1)
                          ? hptq_ws_layout(m, n, block, nullptr, nullptr)
                          : 0;
  gptq_status st = quant_check_args(w_dtype, m, n, bits, group, block, ws, ws_bytes, need);
  if (st != GPTQ_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  HptqWs h;
  hptq_ws_layout(m, n, block, &h, static_cast<char*>(ws));
  const QuantWs& w = h.w[0];
  const long long b_max = (long long)std::floor(budget * (double)m * (double)n);

  st = quant_setup(w, m, n, U, perm, group, block, g_idx, info, s);
  if (st != GPTQ_OK) return st;
  GPTQ_LAUNCH(KK_HPTQ, s, search_init_kernel, 1, 1, 0, h.st, alpha_lo, alpha_hi);
  // pass 0 at α_hi, then one pass a bisection step, or (lookahead) two levels
  // a round (slot 0 the midpoint, slots 1 and 2 the quarter points side by side)
  st = hptq_pass(h, 0, W, w_dtype, m, n, U, perm, dead, bits, group, block, scale, nullptr,
                 &h.st->a, 0, nullptr, b_max, trace_alpha, trace_bits, 0, info, s);
  if (st != GPTQ_OK) return st;
  for (int k = 1; k <= iters && !lookahead; ++k) {
    st = hptq_pass(h, 0, W, w_dtype, m, n, U, perm, dead, bits, group, block, scale, nullptr,
                   &h.st->a, k, nullptr, b_max, trace_alpha, trace_bits, 0, info, s);
    if (st != GPTQ_OK) return st;
  }
  for (int k0 = 1; k0 <= iters && lookahead; k0 += 2) {
    st = search_round(h.st, k0, iters, b_max, trace_alpha, trace_bits, KK_HPTQ, s,
                      [&](int slot, cudaStream_t ss) -> gptq_status {
                        return hptq_pass(h, slot, W, w_dtype, m, n, U, perm, dead, bits, group,
                                         block, slot ? h.scale[slot] : scale, nullptr,
                                         &h.st->cand[slot], -1, &h.st->ccount[slot], b_max,
                                         nullptr, nullptr, 0, info, ss);
                      });
    if (st != GPTQ_OK) return st;
  }
  // the outputs: one more pass at the chosen α (the bracket's hi), encoded
  st = hptq_pass(h, 0, W, w_dtype, m, n, U, perm, dead, bits, group, block, scale, loss_row,
                 &h.st->hi, -1, nullptr, b_max, nullptr, nullptr, 1, info, s);
  if (st != GPTQ_OK) return st;
  const unsigned g8 = (unsigned)ceil_div(m, 8);
  GPTQ_LAUNCH(KK_HPTQ, s, hptq_rowbits_kernel, g8, 256, 0, h.codes16[0], m, n, h.lens,
              h.rowbits);
  GPTQ_LAUNCH(KK_HPTQ, s, row_scan_kernel, 1, 1024, 0, h.rowbits, m, row_off, stream_cap * 32,
              h.st, alpha, info);
  if (stream_cap > 0) {
    GPTQ_CUDA(cudaMemsetAsync(stream_words, 0, sizeof(uint32_t) * (size_t)stream_cap, s));
    GPTQ_LAUNCH(KK_HPTQ, s, hptq_encode_kernel, g8, 256, 0, h.codes16[0], w.pinv, m, n,
                h.lens, h.canon, row_off, stream_words, stream_cap);
  }
  GPTQ_CUDA(cudaMemcpyAsync(code_len, h.lens, NSYM, cudaMemcpyDeviceToDevice, s));
  if (code_word != nullptr)
    GPTQ_CUDA(cudaMemcpyAsync(code_word, h.canon, sizeof(uint64_t) * NSYM,
                              cudaMemcpyDeviceToDevice, s));
  if (codes != nullptr || Qdq != nullptr)
    GPTQ_LAUNCH(KK_HPTQ, s, hptq_out_kernel, (unsigned)ceil_div(m * n, 256), 256, 0,
                h.codes16[0], w.pinv, m, n, group, ceil_div(n, group), scale, codes, Qdq);
  return GPTQ_OK;
}
