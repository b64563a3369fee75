// gptq_quantize: ingest (W → float32, processing order), the block loop of
// sweep (K3) and trailing update (K4), and K5: packing the codes back into the
// original column order, g_idx and the optional dequantized copy.
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2 (the
// column loop) and Table 1 (GPTQ stores integer indices plus group scales);
// Schritt 3 (GPTQ's groups run along the input channels).
#include <algorithm>
#include <cuda_bf16.h>

#include <map>
#include <mutex>
#include <utility>

#include "kernels.cuh"

namespace gptq {

int error_width(int64_t n, int block) {
  return (trailing_uses_tensor_cores(n, block) && block == SWEEP_BLOCK_MAX)
             ? kSuperBlocks * SWEEP_BLOCK_MAX
             : SWEEP_BLOCK_MAX;
}

size_t quant_ws_layout(int64_t m, int64_t n, int block, QuantWs* w, char* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  // Wp and the error buffers hold whole 128-row boxes, so that no box store
  // or reduction is clipped (rows ≥ m are never read back)
  const size_t mrows = (size_t)error_rows(m);
  size_t o_wp = take(sizeof(float) * mrows * (size_t)n);
  size_t o_codes = take((size_t)m * (size_t)n);
  const int ew = error_width(n, block);
  size_t o_e[4];
  for (int k = 0; k < 4; ++k) o_e[k] = take(sizeof(float) * mrows * (size_t)ew);
  size_t o_pinv = take(sizeof(int32_t) * (size_t)(n + 1));
  size_t o_pan = take(panel_workspace_bytes(n, block));
  const bool tc = trailing_uses_tensor_cores(n, block);
  size_t o_uhi = tc ? take(sizeof(float) * (size_t)n * (size_t)n) : 0;
  size_t o_ulo = tc ? take(sizeof(float) * (size_t)n * (size_t)n) : 0;
  if (w && base) {
    w->Wp = reinterpret_cast<float*>(base + o_wp);
    w->codes = reinterpret_cast<uint8_t*>(base + o_codes);
    for (int k = 0; k < 2; ++k) {
      w->Ehi[k] = reinterpret_cast<float*>(base + o_e[2 * k]);
      w->Elo[k] = reinterpret_cast<float*>(base + o_e[2 * k + 1]);
    }
    w->ew = ew;
    w->pinv = reinterpret_cast<int32_t*>(base + o_pinv);
    w->panels = reinterpret_cast<float*>(base + o_pan);
    w->Uhi = tc ? reinterpret_cast<float*>(base + o_uhi) : nullptr;
    w->Ulo = tc ? reinterpret_cast<float*>(base + o_ulo) : nullptr;
  }
  return off;
}

size_t quant_slot_layout(int64_t m, int64_t n, int block, const QuantWs* shared, QuantWs* w,
                         char* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t mrows = (size_t)error_rows(m);
  const size_t o_wp = take(sizeof(float) * mrows * (size_t)n);
  const size_t o_codes = take((size_t)m * (size_t)n);
  const int ew = error_width(n, block);
  size_t o_e[4];
  for (int k = 0; k < 4; ++k) o_e[k] = take(sizeof(float) * mrows * (size_t)ew);
  if (w && base && shared) {
    *w = *shared;
    w->Wp = reinterpret_cast<float*>(base + o_wp);
    w->codes = reinterpret_cast<uint8_t*>(base + o_codes);
    for (int k = 0; k < 2; ++k) {
      w->Ehi[k] = reinterpret_cast<float*>(base + o_e[2 * k]);
      w->Elo[k] = reinterpret_cast<float*>(base + o_e[2 * k + 1]);
    }
  }
  return off;
}

namespace {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// The far part of each trailing update runs on a side stream of the caller's
// stream, so that it overlaps the next block's sweep; one side stream and two
// events per (device, caller stream), created on first use and kept for the
// life of the process.
struct SideStream {
  cudaStream_t s2 = nullptr;
  cudaEvent_t swept = nullptr;    // recorded on the caller's stream after a sweep
  cudaEvent_t far[2] = {};        // recorded on the side stream after the far update
                                  // of an even / odd block
};

gptq_status side_stream_for(cudaStream_t s, SideStream** out) {
  static std::mutex mu;
  static std::map<std::pair<int, cudaStream_t>, SideStream> reg;
  int dev = 0;
  GPTQ_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(mu);
  SideStream& e = reg[{dev, s}];
  if (e.s2 == nullptr) {
    GPTQ_CUDA(cudaStreamCreateWithFlags(&e.s2, cudaStreamNonBlocking));
    GPTQ_CUDA(cudaEventCreateWithFlags(&e.swept, cudaEventDisableTiming));
    GPTQ_CUDA(cudaEventCreateWithFlags(&e.far[0], cudaEventDisableTiming));
    GPTQ_CUDA(cudaEventCreateWithFlags(&e.far[1], cudaEventDisableTiming));
  }
  *out = &e;
  return GPTQ_OK;
}

// pinv[perm[p]] = p and g_idx[perm[p]] = p / group (static groups: c / group);
// pinv[n] (−1 before the launch) becomes 0 unless perm is the identity.
__global__ void __launch_bounds__(256)
pinv_kernel(const int32_t* __restrict__ perm, int64_t n, int group,
            int32_t* __restrict__ pinv, int32_t* __restrict__ g_idx, int static_groups,
            int32_t* info) {
  const int64_t p = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (p >= n) return;
  const int32_t c = perm[p];
  if (c != p) pinv[n] = 0;
  if (c < 0 || c >= n) { report(info, GPTQ_ERR_INVALID_ARG, p); return; }
  pinv[c] = (int32_t)p;
  if (g_idx) g_idx[c] = (int32_t)((static_groups ? c : p) / group);
}

// Static groups: a warp per (row, group) takes the min-max parameters of the
// group's original columns [g·group, (g+1)·group) of W (dead columns read 0),
// with the hot path's quantizer: 0 inside the range, an all-zero group → [−1,
// 1], s = (xmax − xmin)/maxq and z = rint(−xmin/s) correctly rounded in
// float32.
template <typename T>
__global__ void __launch_bounds__(256)
static_params_kernel(const T* __restrict__ W, int64_t m, int64_t n,
                     const uint8_t* __restrict__ dead, int group, int64_t ngroups, int bits,
                     float* __restrict__ scale, uint8_t* __restrict__ zero) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= m * ngroups) return;
  const int64_t r = wid / ngroups, g = wid % ngroups;
  const int64_t c0 = g * group, c1 = min(n, c0 + group);
  float xmin = 0.f, xmax = 0.f;
  for (int64_t c = c0 + lane; c < c1; c += 32) {
    const float v = dead[c] ? 0.f : to_f32(W[r * n + c]);
    xmin = fminf(xmin, v);
    xmax = fmaxf(xmax, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    xmin = fminf(xmin, __shfl_xor_sync(0xffffffffu, xmin, o));
    xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
  }
  if (lane != 0) return;
  if (xmin == 0.f && xmax == 0.f) {
    xmin = -1.f;
    xmax = 1.f;
  }
  const float maxq = (float)((1 << bits) - 1);
  const float s = __fdiv_rn(xmax - xmin, maxq);
  scale[r * ngroups + g] = s;
  zero[r * ngroups + g] = (uint8_t)rintf(__fdiv_rn(-xmin, s));
}

// Eight consecutive elements of W as float32 (16- or 32-byte loads).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Wp[r][p] = W[r][perm[p]] as float32; dead columns read as 0.  A CTA takes
// `rpb` consecutive rows.
//  * The processing order is the identity (*ident = −1) and `vec` (n a
//    multiple of 8, W 16-byte and dead 8-byte aligned): a stream, eight consecutive elements
//    a thread (one or two 16-byte loads, the eight dead flags in one 8-byte
//    load, two 16-byte stores).
//  * Otherwise the rows come into shared memory as they are (coalesced
//    16-byte loads; rows of W are contiguous), and each thread then writes
//    consecutive processing positions of a row (coalesced stores), gathering
//    through perm from shared memory.  Rows longer than the staging area are
//    gathered from global memory instead (staged = 0).
template <typename T>
__global__ void __launch_bounds__(256)
ingest_kernel(const T* __restrict__ W, int64_t m, int64_t n,
              const int32_t* __restrict__ perm, const uint8_t* __restrict__ dead,
              float* __restrict__ Wp, int rpb, int staged, const int32_t* __restrict__ ident,
              int vec, int32_t* info) {
  extern __shared__ __align__(16) unsigned char ig[];
  T* sw = reinterpret_cast<T*>(ig);
  const int64_t r0 = (int64_t)blockIdx.x * rpb;
  const int rows = (int)(m - r0 < rpb ? m - r0 : (int64_t)rpb);
  const int tid = threadIdx.x;
  if (vec && *ident == -1) {
    const int n8 = (int)(n >> 3);
    for (int rl = 0; rl < rows; ++rl) {
      const int64_t r = r0 + rl;
      for (int k = tid; k < n8; k += 256) {
        const int64_t c = (int64_t)k * 8;
        float v[8];
        load8(W + r * n + c, v);
        const uint2 d = __ldg(reinterpret_cast<const uint2*>(dead + c));
        const uint32_t dw[2] = {d.x, d.y};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (!isfinite(v[e])) { report(info, GPTQ_ERR_NONFINITE, r * n + c + e); v[e] = 0.f; }
          if ((dw[e >> 2] >> (8 * (e & 3))) & 0xFFu) v[e] = 0.f;
        }
        float4* o = reinterpret_cast<float4*>(Wp + r * n + c);
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
      }
    }
    return;
  }
  const T* src = W + r0 * n;
  const int64_t elems = (int64_t)rows * n;
  if (staged) {
    const int64_t bytes = elems * (int64_t)sizeof(T);
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
      const int64_t v16 = bytes >> 4;
      for (int64_t e = tid; e < v16; e += 256)
        reinterpret_cast<uint4*>(ig)[e] = __ldg(reinterpret_cast<const uint4*>(src) + e);
      for (int64_t e = (v16 << 4) / (int64_t)sizeof(T) + tid; e < elems; e += 256) sw[e] = src[e];
    } else {
      for (int64_t e = tid; e < elems; e += 256) sw[e] = src[e];
    }
    __syncthreads();
  }
  const T* rowsrc = staged ? sw : src;
  for (int rl = 0; rl < rows; ++rl) {
    const int64_t r = r0 + rl;
    for (int p = tid; p < n; p += 256) {
      const int32_t c = perm[p];
      float v = 0.f;
      if (c >= 0 && c < n) {
        v = to_f32(rowsrc[(int64_t)rl * n + c]);
        if (!isfinite(v)) { report(info, GPTQ_ERR_NONFINITE, r * n + c); v = 0.f; }
        if (dead[c]) v = 0.f;
      }
      Wp[r * n + p] = v;
    }
  }
}

// Rows per ingest CTA: up to 32 KB of W in shared memory (one row, read from
// global memory, when a row is longer than 48 KB).
inline int ingest_rows_per_block(int64_t n, size_t elem) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(16, 32768 / (n * (int64_t)elem)));
}

// What the packer needs to fetch one code (and write its dequantized value).
struct PackRow {
  const uint8_t* codes;       // the CTA's rows of codes (shared or global memory)
  int64_t n;
  const int32_t* pinv;
  const float* outv;
  float* Qdq;
  const float* scale;
  const uint8_t* zero;
  int group;
  int64_t ngroups;
  int rowgs;
  int static_groups;
  int32_t* info;
};

// Code of original column c of local row rl (row r), and its dequantized
// value into Qdq when asked for.
__device__ __forceinline__ uint32_t pack_code(const PackRow& a, int rl, int64_t r, int64_t c) {
  const int64_t n = a.n;
  if (c >= n) return 0u;
  const int32_t p = a.pinv[c];
  if (p < 0 || p >= n) {
    report(a.info, GPTQ_ERR_INVALID_ARG, c);
    return 0u;
  }
  uint32_t q = a.codes[(int64_t)rl * n + p];
  bool kept = false;                 // an SSQR outlier: its value, not its code
  if (a.outv != nullptr) {
    kept = (q & OUTLIER_FLAG) != 0;
    q &= ~(uint32_t)OUTLIER_FLAG;
  }
  if (a.Qdq != nullptr) {
    // input-channel groups: [row][group of processing position p];
    // output-channel groups (rowgs rows): [row group][original column c]
    // (32-bit quotients: rows < 2^31, columns < 2^20)
    const int64_t sx = a.rowgs > 0 ? (int64_t)((int)r / a.rowgs) * n + c
                                   : r * a.ngroups + (a.static_groups ? (int)c : p) / a.group;
    a.Qdq[r * n + c] = kept ? a.outv[r * n + p] : a.scale[sx] * ((float)q - (float)a.zero[sx]);
  }
  return q;
}

// Words of 32 consecutive codes (in processing order = original order) at
// BITS bits each, LSB first: BITS words from 32 code bytes (each < 2^BITS).
template <int BITS>
__device__ __forceinline__ void pack32(const uint4 (&c)[2], uint32_t (&out)[BITS]) {
  const uint32_t b[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[1].x, c[1].y, c[1].z, c[1].w};
  if constexpr (BITS == 8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) out[k] = b[k];
  } else if constexpr (BITS == 4) {
    // four bytes → 16 bits: byte pairs merged, then the two halves
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t lo = b[2 * k], hi = b[2 * k + 1];
      lo |= lo >> 4;
      hi |= hi >> 4;
      out[k] = (lo & 0xFFu) | ((lo >> 8) & 0xFF00u) | ((hi & 0xFFu) << 16) | ((hi << 8) & 0xFF000000u);
    }
  } else if constexpr (BITS == 2) {
    // four bytes → 8 bits
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t w = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t x = b[4 * k + q];
        x |= x >> 6;
        w |= ((x & 0xFu) | ((x >> 12) & 0xF0u)) << (8 * q);
      }
      out[k] = w;
    }
  } else {
    // 3 bits: code j at bit 3j of a 96-bit string
    uint64_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint64_t q = (b[j >> 2] >> (8 * (j & 3))) & 0xFFu;
      const int pos = 3 * j;
      if (pos < 64) lo |= q << pos;
      if (pos + 3 > 64) hi |= pos >= 64 ? q << (pos - 64) : q >> (64 - pos);
    }
    out[0] = (uint32_t)lo;
    out[1] = (uint32_t)(lo >> 32);
    out[2] = (uint32_t)hi;
  }
}

// Packing.  With the identity as processing order, plain codes (no outlier
// values, no dequantized copy) and `flat` (n a multiple of 32, qweight
// 16-byte aligned), the codes of the CTA's rows and their words are two
// contiguous streams: a thread turns 32 code bytes (two 16-byte loads) into
// BITS words.  Otherwise a CTA takes `rpb` consecutive rows: their codes (processing
// order, contiguous in the code array) come into shared memory with coalesced
// 16-byte loads.  Then a warp walks a row's original columns in chunks: each
// column's processing position pinv[c] (a coalesced load), its code from
// shared memory, its dequantized value (a coalesced store).  The chunk's
// words are formed in registers: for widths that divide 32 by shuffles over
// groups of lanes, for 3 bits by a transpose through ballots.
template <int BITS>
__global__ void __launch_bounds__(256, 4)
pack_kernel(const uint8_t* __restrict__ codes, int64_t m, int64_t n,
            const int32_t* __restrict__ pinv, int group, int64_t ngroups, int rowgs,
            const float* __restrict__ scale, const uint8_t* __restrict__ zero,
            uint32_t* __restrict__ qweight, int64_t nwords,
            float* __restrict__ Qdq, const float* __restrict__ outv, int static_groups,
            int rpb, int staged, int flat, int32_t* info) {
  extern __shared__ __align__(16) uint8_t sc[];
  const int64_t r0 = (int64_t)blockIdx.x * rpb;
  const int rows = (int)(m - r0 < rpb ? m - r0 : (int64_t)rpb);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (flat && pinv[n] == -1) {
    // 32 codes → BITS words; the CTA's rows are contiguous in both arrays
    const int chunks = (int)(((int64_t)rows * n) >> 5);
    const uint4* in = reinterpret_cast<const uint4*>(codes + r0 * n);
    uint32_t* out = qweight + r0 * nwords;
    for (int k = tid; k < chunks; k += 256) {
      const uint4 c[2] = {__ldg(in + 2 * k), __ldg(in + 2 * k + 1)};
      uint32_t w[BITS];
      pack32<BITS>(c, w);
      if constexpr (BITS % 4 == 0) {
#pragma unroll
        for (int q = 0; q < BITS; q += 4)
          *reinterpret_cast<uint4*>(out + (int64_t)k * BITS + q) = make_uint4(w[q], w[q + 1], w[q + 2], w[q + 3]);
      } else if constexpr (BITS == 2) {
        *reinterpret_cast<uint2*>(out + (int64_t)k * 2) = make_uint2(w[0], w[1]);
      } else {
#pragma unroll
        for (int q = 0; q < BITS; ++q) out[(int64_t)k * BITS + q] = w[q];
      }
    }
    return;
  }
  const uint8_t* src = codes + r0 * n;
  const int64_t bytes = (int64_t)rows * n;
  if (!staged) {
    // a row too long for shared memory: codes gathered from global memory
  } else if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    const int64_t v16 = bytes >> 4;
    for (int64_t e = tid; e < v16; e += 256)
      reinterpret_cast<uint4*>(sc)[e] = __ldg(reinterpret_cast<const uint4*>(src) + e);
    for (int64_t e = (v16 << 4) + tid; e < bytes; e += 256) sc[e] = src[e];
  } else {
    for (int64_t e = tid; e < bytes; e += 256) sc[e] = src[e];
  }
  __syncthreads();
  const PackRow pr = {staged ? sc : src, n, pinv, outv, Qdq, scale, zero, group, ngroups, rowgs,
                      static_groups, info};
  if constexpr (32 % BITS == 0) {
    // widths that divide 32: a warp takes 128 columns at a time, lane l the
    // four columns 4l .. 4l+3 (a 4·BITS-bit piece at bit 4l·BITS of the
    // chunk); G = 8/BITS lanes fill a word, OR-ed together by shuffles, and
    // the first lane of each group stores it (4·BITS consecutive words)
    constexpr int G = 8 / BITS;
    const int chunks = (int)((n + 127) / 128);
    for (int rl = 0; rl < rows; ++rl)
    for (int ch = warp; ch < chunks; ch += 8) {
      const int64_t r = r0 + rl;
      const int64_t c0 = (int64_t)ch * 128 + 4 * lane;
      uint32_t v = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) v |= pack_code(pr, rl, r, c0 + i) << (BITS * i);
      v <<= 4 * BITS * (lane % G);
#pragma unroll
      for (int o = 1; o < G; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
      const int64_t wi = (int64_t)ch * 4 * BITS + lane / G;
      if (lane % G == 0 && wi < nwords) qweight[r * nwords + wi] = v;
    }
  } else {
    // codes straddle words: a warp takes 32 columns at a time, lane l column
    // 32·chunk + l; one ballot per code bit (plane b: bit b of every lane's
    // code), then one ballot per word, lane t supplying bit t
    const int chunks = (int)((n + 31) / 32);
    for (int rl = 0; rl < rows; ++rl)
    for (int ch = warp; ch < chunks; ch += 8) {
      const int64_t r = r0 + rl;
      const uint32_t q = pack_code(pr, rl, r, (int64_t)ch * 32 + lane);
      uint32_t plane[BITS];
#pragma unroll
      for (int b = 0; b < BITS; ++b) plane[b] = __ballot_sync(0xffffffffu, (q >> b) & 1u);
      uint32_t mine = 0;                   // lane j < BITS: word j of the chunk
#pragma unroll
      for (int j = 0; j < BITS; ++j) {
        const int idx = 32 * j + lane, code = idx / BITS, b = idx % BITS;
        uint32_t pb = plane[0];
#pragma unroll
        for (int bb = 1; bb < BITS; ++bb) pb = (b == bb) ? plane[bb] : pb;
        const uint32_t word = __ballot_sync(0xffffffffu, (pb >> code) & 1u);
        if (lane == j) mine = word;
      }
      const int64_t wi = (int64_t)ch * BITS + lane;
      if (lane < BITS && wi < nwords) qweight[r * nwords + wi] = mine;
    }
  }
}

// Rows per packing CTA: up to 16 KB of codes in shared memory (one row, read
// from global memory, when a row is longer than 48 KB).
inline int pack_rows_per_block(int64_t n) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(16, 16384 / n));
}
constexpr int64_t kPackStageMax = 48 * 1024;

}  // namespace

gptq_status quant_check_args(int w_dtype, int64_t m, int64_t n, int bits, int group,
                             int block, const void* ws, size_t ws_bytes, size_t need) {
  if (m < 1 || n < 1 || m > ((int64_t)1 << 31) || n > ((int64_t)1 << 20))
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_quantize: m=%lld n=%lld", (long long)m,
                (long long)n);
  if (w_dtype != GPTQ_DTYPE_F32 && w_dtype != GPTQ_DTYPE_BF16)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_quantize: w_dtype=%d", w_dtype);
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8)
    return fail(GPTQ_ERR_UNSUPPORTED, "gptq_quantize: bits=%d (2, 3, 4, 8)", bits);
  if (group < 32 || group % 32 != 0 || block < group || block > 128 || block % group != 0)
    return fail(GPTQ_ERR_UNSUPPORTED,
                "gptq_quantize: group=%d block=%d (group a multiple of 32, block a "
                "multiple of group, block <= 128)", group, block);
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_quantize: workspace not 256-byte aligned");
  if (ws_bytes < need)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_quantize: workspace %zu < %zu bytes", ws_bytes,
                need);
  return GPTQ_OK;
}

gptq_status quant_setup(const QuantWs& w, int64_t m, int64_t n, const float* U,
                        const int32_t* perm, int group, int block, int32_t* g_idx,
                        int32_t* info, cudaStream_t s, bool static_groups) {
  (void)m;
  GPTQ_CUDA(cudaMemsetAsync(info, 0, 2 * sizeof(int32_t), s));
  GPTQ_CUDA(cudaMemsetAsync(w.pinv, 0xFF, sizeof(int32_t) * (n + 1), s));
  GPTQ_LAUNCH(KK_INGEST, s, pinv_kernel, (unsigned)ceil_div(n, 256), 256, 0, perm, n,
              group, w.pinv, g_idx, static_groups ? 1 : 0, info);
  gptq_status st = launch_panels(U, n, block, w.panels, s);
  if (st != GPTQ_OK) return st;
  if (w.Uhi != nullptr && n > block) {
    st = launch_split_tf32_t(U, n, w.Uhi, w.Ulo, s);
    if (st != GPTQ_OK) return st;
  }
  return GPTQ_OK;
}

gptq_status quant_pass(const QuantWs& w, const void* W, int w_dtype, int64_t m, int64_t n,
                       const float* U, const int32_t* perm, const uint8_t* dead, int bits,
                       int group, int block, int rowgs, float* scale, uint8_t* zero,
                       float* loss_row, const OutlierArgs* outl, int32_t* info,
                       cudaStream_t s) {
  const int64_t ngroups = rowgs > 0 ? ceil_div(m, rowgs) : ceil_div(n, group);
  if (loss_row) GPTQ_CUDA(cudaMemsetAsync(loss_row, 0, sizeof(float) * m, s));
  {
    const size_t es = w_dtype == GPTQ_DTYPE_BF16 ? 2 : 4;
    const int rpb = ingest_rows_per_block(n, es);
    const int staged = (int64_t)rpb * n * (int64_t)es <= 48 * 1024 ? 1 : 0;
    const size_t ism = staged ? align_up((size_t)rpb * (size_t)n * es, 16) : 0;
    const unsigned gin = (unsigned)ceil_div(m, rpb);
    const int vec = (n % 8 == 0 && (reinterpret_cast<uintptr_t>(W) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(dead) & 7) == 0) ? 1 : 0;
    if (w_dtype == GPTQ_DTYPE_BF16)
      GPTQ_LAUNCH(KK_INGEST, s, ingest_kernel<__nv_bfloat16>, gin, 256, ism,
                  static_cast<const __nv_bfloat16*>(W), m, n, perm, dead, w.Wp, rpb, staged,
                  w.pinv + n, vec, info);
    else
      GPTQ_LAUNCH(KK_INGEST, s, ingest_kernel<float>, gin, 256, ism,
                  static_cast<const float*>(W), m, n, perm, dead, w.Wp, rpb, staged,
                  w.pinv + n, vec, info);
  }

  // padding rows of the working copy: zero, so that the last row box of
  // every sweep and trailing update reads defined values
  if (error_rows(m) > m)
    GPTQ_CUDA(cudaMemsetAsync(w.Wp + m * n, 0, sizeof(float) * (size_t)(error_rows(m) - m) * n, s));
  // Block b's errors reach the later columns in parts:
  //  * block b+1's columns: on the tensor-core path, sweep b+1 applies them
  //    itself in its prologue (in TMEM, before its first column); otherwise a
  //    trailing update on the caller's stream;
  //  * the columns from block b+2 on: on the tensor-core path, CTAs of sweep
  //    b+1's own launch (those columns are not sweep b+1's, and the errors
  //    come from the launch before), so that the sweeps follow each other on
  //    one stream; otherwise a trailing update on the side stream,
  //    overlapping sweep b+1.  On the tensor-core path with super-blocks of
  //    S blocks, those CTAs cover only the rest of b's super-block and the
  //    block after it; the columns past that receive the whole super-block's
  //    errors at once, from the CTAs of the next super-block's first sweep.
  // Every column still receives the contributions in block order: the
  // launches follow each other on one stream (or whatever touches block b's
  // columns first waits for the far update of block b−2), and the error
  // buffers alternate by super-block, so a far update's input is not
  // overwritten before it is read.
  const bool fused = w.Uhi != nullptr && trailing_uses_tensor_cores(n, block);
  SideStream* side = nullptr;
  if (!fused) {
    gptq_status st = side_stream_for(s, &side);
    if (st != GPTQ_OK) return st;
  }
  bool pending[2] = {false, false};
  // errors: block b's slot of its super-block's buffer (S blocks a buffer,
  // the two buffers alternate by super-block; S = 1 off the tensor-core path)
  const int S = w.ew / SWEEP_BLOCK_MAX;
  auto eslot = [&](int64_t bb, int hi) -> float* {
    float* const* e = hi ? w.Ehi : w.Elo;
    return e[(bb / S) & 1] + (bb % S) * SWEEP_BLOCK_MAX;
  };
  for (int64_t j0 = 0, b = 0; j0 < n; j0 += block, ++b) {
    const int bw = (int)((n - j0 < block) ? (n - j0) : block);
    float* ehi = eslot(b, 1);
    float* elo = eslot(b, 0);
    if (pending[b & 1]) {                      // the far update of block b−2
      GPTQ_CUDA(cudaStreamWaitEvent(s, side->far[b & 1], 0));
      pending[b & 1] = false;
    }
    SweepPrologue pre;
    SweepFar far;
    if (fused && b > 0) {
      // block b−1's errors on this block's columns: the sweep's prologue
      pre.Ehi = eslot(b - 1, 1);
      pre.Elo = eslot(b - 1, 0);
      pre.epitch = far.epitch = w.ew;
      pre.Uhi = far.Uhi = w.Uhi;
      pre.Ulo = far.Ulo = w.Ulo;
      pre.k0 = j0 - block;
      pre.kw = block;
      // the far columns: block b−1's errors inside a super-block, the whole
      // previous super-block's at the first block of the next (far_range)
      const FarRange fr = far_range(n, block, S, b);
      far.c0 = fr.c0;
      far.c1 = fr.c1;
      far.k0 = fr.k0;
      far.kw = fr.kw;
      far.Ehi = fr.whole ? w.Ehi[(b / S - 1) & 1] : pre.Ehi;
      far.Elo = fr.whole ? w.Elo[(b / S - 1) & 1] : pre.Elo;
    }
    const float* panel = w.panels + (size_t)(j0 / block) * (PANEL_BYTES / sizeof(float));
    gptq_status st = launch_sweep(w.Wp, m, n, j0, bw, panel, bits, group, ngroups, w.codes,
                                  scale, zero, ehi, elo, w.ew, pre, far, loss_row, info,
                                  rowgs > 0 ? perm : nullptr, outl, s);
    if (st != GPTQ_OK) return st;
    const int64_t c0 = j0 + bw, c1 = c0 + block;
    if (c0 >= n || fused) continue;
    if (b > 0 && pending[(b - 1) & 1]) {       // the far update of block b−1
      GPTQ_CUDA(cudaStreamWaitEvent(s, side->far[(b - 1) & 1], 0));
      pending[(b - 1) & 1] = false;
    }
    st = launch_trailing(w.Wp, m, n, c0, c1, ehi, elo, j0, bw, U, s);
    if (st != GPTQ_OK) return st;
    if (c1 < n) {
      GPTQ_CUDA(cudaEventRecord(side->swept, s));
      GPTQ_CUDA(cudaStreamWaitEvent(side->s2, side->swept, 0));
      st = launch_trailing(w.Wp, m, n, c1, n, ehi, elo, j0, bw, U, side->s2);
      if (st != GPTQ_OK) return st;
      GPTQ_CUDA(cudaEventRecord(side->far[b & 1], side->s2));
      pending[b & 1] = true;
    }
  }
  for (int p = 0; p < 2; ++p)
    if (pending[p]) GPTQ_CUDA(cudaStreamWaitEvent(s, side->far[p], 0));
  return GPTQ_OK;
}

gptq_status quant_pack(const QuantWs& w, int64_t m, int64_t n, int bits, int group, int rowgs,
                       const float* scale, const uint8_t* zero, uint32_t* qweight,
                       float* Qdq, const float* outl_vals, int32_t* info, cudaStream_t s,
                       bool static_groups) {
  const int sg = static_groups ? 1 : 0;
  const int64_t ngroups = rowgs > 0 ? ceil_div(m, rowgs) : ceil_div(n, group);
  const int64_t nwords = ceil_div(n * bits, 32);
  const int rpb = pack_rows_per_block(n);
  const unsigned gpk = (unsigned)ceil_div(m, rpb);
  const int staged = (int64_t)rpb * n <= kPackStageMax ? 1 : 0;
  const size_t psm = staged ? align_up((size_t)rpb * (size_t)n, 16) : 0;
  const int flat = (n % 32 == 0 && (reinterpret_cast<uintptr_t>(qweight) & 15) == 0 &&
                    Qdq == nullptr && outl_vals == nullptr) ? 1 : 0;
  switch (bits) {
    case 2:
      GPTQ_LAUNCH(KK_PACK, s, pack_kernel<2>, gpk, 256, psm, w.codes, m, n, w.pinv, group,
                  ngroups, rowgs, scale, zero, qweight, nwords, Qdq, outl_vals, sg, rpb, staged, flat, info);
      break;
    case 3:
      GPTQ_LAUNCH(KK_PACK, s, pack_kernel<3>, gpk, 256, psm, w.codes, m, n, w.pinv, group,
                  ngroups, rowgs, scale, zero, qweight, nwords, Qdq, outl_vals, sg, rpb, staged, flat, info);
      break;
    case 4:
      GPTQ_LAUNCH(KK_PACK, s, pack_kernel<4>, gpk, 256, psm, w.codes, m, n, w.pinv, group,
                  ngroups, rowgs, scale, zero, qweight, nwords, Qdq, outl_vals, sg, rpb, staged, flat, info);
      break;
    default:
      GPTQ_LAUNCH(KK_PACK, s, pack_kernel<8>, gpk, 256, psm, w.codes, m, n, w.pinv, group,
                  ngroups, rowgs, scale, zero, qweight, nwords, Qdq, outl_vals, sg, rpb, staged, flat, info);
      break;
  }
  return GPTQ_OK;
}

}  // namespace gptq

using namespace gptq;

extern "C" size_t gptq_quantize_workspace_bytes(int64_t m, int64_t n, int block) {
  if (m < 1 || n < 1 || block < 1) return 0;
  return quant_ws_layout(m, n, block, nullptr, nullptr);
}

namespace gptq {
namespace {

// The quantize path of gptq_quantize (rowgs = 0: scale groups of `group`
// columns) and gptq_quantize_rowgroups (rowgs = 128: scale groups of the
// rows, per column).
gptq_status quantize_impl(const void* W, int w_dtype, int64_t m, int64_t n, const float* U,
                          const int32_t* perm, const uint8_t* dead, int bits, int group,
                          int block, int rowgs, uint32_t* qweight, float* scale, uint8_t* zero,
                          int32_t* g_idx, float* loss_row, float* Qdq, int32_t* info, void* ws,
                          size_t ws_bytes, void* stream) {
  if (!W || !U || !perm || !dead || !qweight || !scale || !zero || (!g_idx && rowgs == 0) ||
      !info || !ws)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_quantize: null pointer");
  const size_t need = (m >= 1 && n >= 1 && block >= 1) ? quant_ws_layout(m, n, block, nullptr, nullptr) : 0;
  gptq_status st = quant_check_args(w_dtype, m, n, bits, group, block, ws, ws_bytes, need);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  QuantWs w;
  quant_ws_layout(m, n, block, &w, static_cast<char*>(ws));
  st = quant_setup(w, m, n, U, perm, group, block, g_idx, info, s);
  if (st != GPTQ_OK) return st;
  st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, rowgs, scale, zero,
                  loss_row, nullptr, info, s);
  if (st != GPTQ_OK) return st;
  return quant_pack(w, m, n, bits, group, rowgs, scale, zero, qweight, Qdq, nullptr, info, s);
}

}  // namespace
}  // namespace gptq

extern "C" gptq_status gptq_quantize(const void* W, int w_dtype, int64_t m,
                                     int64_t n, const float* U,
                                     const int32_t* perm, const uint8_t* dead,
                                     int bits, int group, int block,
                                     uint32_t* qweight, float* scale,
                                     uint8_t* zero, int32_t* g_idx,
                                     float* loss_row, float* Qdq, int32_t* info,
                                     void* ws, size_t ws_bytes, void* stream) {
  return quantize_impl(W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, qweight, scale,
                       zero, g_idx, loss_row, Qdq, info, ws, ws_bytes, stream);
}

extern "C" gptq_status gptq_quantize_static(const void* W, int w_dtype, int64_t m, int64_t n,
                                            const float* U, const int32_t* perm,
                                            const uint8_t* dead, int bits, int group, int block,
                                            uint32_t* qweight, float* scale, uint8_t* zero,
                                            int32_t* g_idx, float* loss_row, float* Qdq,
                                            int32_t* info, void* ws, size_t ws_bytes,
                                            void* stream) {
  if (!W || !U || !perm || !dead || !qweight || !scale || !zero || !g_idx || !info || !ws)
    return fail(GPTQ_ERR_INVALID_ARG, "gptq_quantize_static: null pointer");
  if (group < 1 || block < 32 || block > 128 || block % 32 != 0)
    return fail(GPTQ_ERR_UNSUPPORTED,
                "gptq_quantize_static: group=%d block=%d (group >= 1, block a multiple of 32, "
                "at most 128)", group, block);
  const size_t need =
      (m >= 1 && n >= 1) ? quant_ws_layout(m, n, block, nullptr, nullptr) : 0;
  // the hot path's checks with the block standing in for the group (any
  // static group width goes with any block)
  gptq_status st = quant_check_args(w_dtype, m, n, bits, block, block, ws, ws_bytes, need);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  QuantWs w;
  quant_ws_layout(m, n, block, &w, static_cast<char*>(ws));
  const int64_t ng = ceil_div(n, group);
  st = quant_setup(w, m, n, U, perm, group, block, g_idx, info, s, true);
  if (st != GPTQ_OK) return st;
  const unsigned gsp = (unsigned)ceil_div(m * ng, 8);
  if (w_dtype == GPTQ_DTYPE_BF16)
    GPTQ_LAUNCH(KK_INGEST, s, static_params_kernel<__nv_bfloat16>, gsp, 256, 0,
                static_cast<const __nv_bfloat16*>(W), m, n, dead, group, ng, bits, scale, zero);
  else
    GPTQ_LAUNCH(KK_INGEST, s, static_params_kernel<float>, gsp, 256, 0,
                static_cast<const float*>(W), m, n, dead, group, ng, bits, scale, zero);
  OutlierArgs sa;
  sa.static_groups = true;
  sa.st_scale = scale;
  sa.st_zero = zero;
  sa.perm = perm;
  sa.st_ng = ng;
  st = quant_pass(w, W, w_dtype, m, n, U, perm, dead, bits, group, block, 0, scale, zero,
                  loss_row, &sa, info, s);
  if (st != GPTQ_OK) return st;
  return quant_pack(w, m, n, bits, group, 0, scale, zero, qweight, Qdq, nullptr, info, s, true);
}

extern "C" gptq_status gptq_quantize_rowgroups(const void* W, int w_dtype, int64_t m,
                                               int64_t n, const float* U,
                                               const int32_t* perm, const uint8_t* dead,
                                               int bits, int gs, int block,
                                               uint32_t* qweight, float* scale,
                                               uint8_t* zero, float* loss_row, float* Qdq,
                                               int32_t* info, void* ws, size_t ws_bytes,
                                               void* stream) {
  if (gs != GPTQ_ROWGROUP_SIZE)
    return fail(GPTQ_ERR_UNSUPPORTED, "gptq_quantize_rowgroups: gs=%d (only %d)", gs,
                GPTQ_ROWGROUP_SIZE);
  return quantize_impl(W, w_dtype, m, n, U, perm, dead, bits, block, block, gs, qweight, scale,
                       zero, nullptr, loss_row, Qdq, info, ws, ws_bytes, stream);
}
