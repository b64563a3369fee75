// K3: the column sweep of one lazy-batch block.
//
// "Warum Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2: for
// column j, quantize with the group's scale, err_j = (col_j − q_j)/H⁻¹[j,j]
// and subtract err_j·H⁻¹[j, j+1:] from the columns not yet quantized.  With
// U the upper inverse-Cholesky factor: e_j = (w_j − q̂_j)/U_jj and
// w[j+1:] −= e_j·U[j, j+1:].  Inside the block every column updates the
// block's later columns; the columns after the block receive the block's
// errors in one product afterwards (trailing.cu).
//
// One thread owns one row; a CTA owns 128 rows and walks the block in
// sub-blocks of 32 columns:
//   * the 32 dependent column steps of a sub-block run unrolled in registers,
//     each step updating the sub-block's later columns in float32 with the
//     sub-block's diagonal 32×32 piece of U (row-major, vector reads);
//   * the sub-block's errors E (128 rows × 32) then update the block's later
//     columns on the tensor core: D[rows, later] += E·U[sub-block rows, later]
//     with tcgen05.mma kind::tf32 and the same three-term TF32 split as the
//     trailing update (E = E_hi + E_lo, U = U_hi + U_lo, lo·lo dropped).  D
//     lives in tensor memory (TMEM lane = row = thread) and accumulates over
//     the sub-blocks; a sub-block's current values are its loaded values
//     minus D, read back with tcgen05.ld.
// Everything U-derived a CTA needs (the B operands in K-major, 128-byte
// swizzled boxes, the diagonal pieces and 1/U_jj) is packed once per call by
// package_kernel and fetched with one bulk (TMA) copy per CTA.
//
// Scale and zero: min-max over the group's current values at the group's
// first column, the range always containing 0; decisions in IEEE float32
// (correctly rounded division and rint, no fast-math).  The block's errors
// also leave as a TF32 split (Ehi, Elo) for the trailing update.
#include <cstring>

#include "kernels.cuh"
#include "sm100.cuh"
#include "trailing_tc.cuh"

namespace gptq {
namespace {

constexpr int SB = 128;       // largest block width
constexpr int SS = 32;        // sub-block
constexpr int RT = 128;       // rows (threads) per CTA
constexpr int LDB = SB + 4;   // bytes per staged code row

// package layout (bytes)
constexpr uint32_t BOX = 32 * 128;                 // 32 rows × 32 TF32 (K-major, swizzled)
constexpr uint32_t PK_BHI = 0;                     // 6 boxes: (s,t) for s < t ≤ 3
constexpr uint32_t PK_BLO = 6 * BOX;
constexpr uint32_t PK_UD = 12 * BOX;               // 4 diagonal 32×32 pieces, row-major
constexpr uint32_t PK_RD = PK_UD + 4 * 32 * 32 * 4;// 128 reciprocal diagonals
constexpr uint32_t PK_BYTES = PK_RD + SB * 4;
static_assert(PK_BYTES == PANEL_BYTES, "package size");
static_assert(PK_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");

__host__ __device__ constexpr int box_index(int s, int t) {   // s < t
  return s == 0 ? t - 1 : (s == 1 ? t + 1 : 5);
}

// smem layout (bytes from a 1024-aligned base)
constexpr uint32_t SM_PKG = 0;
constexpr uint32_t SM_AHI = 66560;                 // 65 KB, 1024-aligned
constexpr uint32_t SM_ALO = SM_AHI + RT * 128;
constexpr uint32_t SM_VALS = SM_ALO + RT * 128;
constexpr uint32_t VBOX = RT * 128;                // 128 rows × 32 floats, swizzled
constexpr uint32_t SM_CODES = SM_VALS + 4 * VBOX;
// the prologue's U chunk: TF32 hi part in its own box, lo part in the code
// rows' space (1024-aligned, unused until the column steps)
constexpr uint32_t SM_BPHI = (SM_CODES + RT * LDB + 1023) / 1024 * 1024;
constexpr uint32_t SM_BPLO = SM_CODES;
constexpr uint32_t SM_BARS = SM_BPHI + 32 * RT * 4;
constexpr uint32_t SM_RGRED = SM_BARS + 128;        // 2 × 8 floats: row-group min/max
constexpr uint32_t SM_SGRP = SM_BARS + 192;         // 128 ints: static group of each column
static_assert(GPTQ_ROWGROUP_SIZE == RT, "an output-channel group is one CTA's rows");
constexpr size_t SMEM_BYTES = 1024 + SM_BARS + 192 + SB * 4;
static_assert(SM_AHI >= PK_BYTES && SM_AHI % 1024 == 0, "A operand placement");
static_assert(SM_VALS % 1024 == 0, "the strip's boxes use the 128-byte swizzle");
static_assert(SM_CODES % 1024 == 0 && RT * LDB >= 32 * RT * 4, "U chunk lo part placement");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

// The block's strip of Wp in shared memory: four boxes of 32 columns × 128
// rows with the TMA 128-byte swizzle, the 16-byte chunk j of row r at
// r·128 + ((j ^ (r mod 8))·16).  Chunk j of row r, box q:
__device__ __forceinline__ float4 strip_chunk(const unsigned char* vals, int q, int r, int j) {
  return *reinterpret_cast<const float4*>(vals + q * VBOX + r * 128 + ((j ^ (r & 7)) << 4));
}

// Package of block b.  blockIdx.y: 0..5 a B box (hi and lo), 6..9 a diagonal
// piece, 10 the reciprocal diagonals.  Box (s,t) holds, in K-major 128-byte
// swizzled layout, row nn = column j0+32t+nn of U and, along K, kk = rows
// j0+32s+kk: element at byte nn·128 + ((kk/4) ^ (nn mod 8))·16 + (kk mod 4)·4.
__global__ void __launch_bounds__(256)
package_kernel(const float* __restrict__ U, int64_t n, int block,
               unsigned char* __restrict__ pkgs) {
  __shared__ float tile[32][33];
  const int b = blockIdx.x, part = blockIdx.y;
  const int64_t j0 = (int64_t)b * block;
  const int bw = (int)((n - j0 < block) ? (n - j0) : block);
  unsigned char* P = pkgs + (size_t)b * PK_BYTES;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  if (part < 6) {
    const int s = part < 3 ? 0 : (part < 5 ? 1 : 2);
    const int t = part < 3 ? part + 1 : (part < 5 ? part - 1 : 3);
    // tile[kk][nn] = U[j0+32s+kk][j0+32t+nn]
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int kk = ty + 8 * q, nn = tx;
      const int r = 32 * s + kk, c = 32 * t + nn;
      tile[kk][nn] = (r < bw && c < bw) ? U[(j0 + r) * n + j0 + c] : 0.f;
    }
    __syncthreads();
    float* hi = reinterpret_cast<float*>(P + PK_BHI + box_index(s, t) * BOX);
    float* lo = reinterpret_cast<float*>(P + PK_BLO + box_index(s, t) * BOX);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int nn = ty + 8 * q, kk = tx;
      const float v = tile[kk][nn];
      const float h = to_tf32(v);
      const int off = nn * 32 + (((kk >> 2) ^ (nn & 7)) << 2) + (kk & 3);   // floats
      hi[off] = h;
      lo[off] = v - h;
    }
  } else if (part < 10) {
    const int s = part - 6;
    float* ud = reinterpret_cast<float*>(P + PK_UD) + s * 32 * 32;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = ty + 8 * q, kk = tx;
      const int r = 32 * s + i, c = 32 * s + kk;
      ud[i * 32 + kk] = (r < bw && c < bw) ? U[(j0 + r) * n + j0 + c] : 0.f;
    }
  } else if (threadIdx.x < SB) {
    const int c = threadIdx.x;
    float* rd = reinterpret_cast<float*>(P + PK_RD);
    rd[c] = (c < bw) ? 1.0f / U[(j0 + c) * n + j0 + c] : 0.f;
  }
}

// x/s correctly rounded, for s > 0.  A zero numerator is answered directly
// (the quotient is that same signed zero): the division's general route is
// many times slower for it, and zero rows (padding, dead columns) are common.
__device__ __forceinline__ float div_rn(float x, float s) {
  const float q = __fdiv_rn(x == 0.f ? 1.f : x, s);
  return x == 0.f ? x : q;
}

// x/s correctly rounded from rs = RN(1/s) by Markstein's FMA correction
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", 1990): q0 = RN(x·rs), r = x − q0·s (exact by FMA),
// RN(q0 + r·rs) = RN(x/s) when the reciprocal is correctly rounded and nothing
// under- or overflows.  Three dependent operations and no branch, where the
// column chain needs it most.  rs is capped at the largest float, so a zero x
// still gives a zero quotient for a pathologically small s.
__device__ __forceinline__ float div_fma(float x, float s, float rs) {
  const float q0 = x * rs;
  const float r = fmaf(-q0, s, x);
  return fmaf(r, rs, q0);
}

// Signed-integer image of a float that orders like the float (finite values).
__device__ __forceinline__ int ord_key(float f) {
  const int b = __float_as_int(f);
  return b ^ ((b >> 31) & 0x7fffffff);
}
__device__ __forceinline__ int ord_key_inv(int k) { return k ^ ((k >> 31) & 0x7fffffff); }

// One CTA (bx: the 128-row tile) of the sweep; smraw: SMEM_BYTES of dynamic
// shared memory.  ROWG: scales along the output channels (CHMC page, Schritt
// 2 and 3: ⌈o/gs⌉·i scales, gs = 128 rows, the CTA's own rows): each column's
// scale and zero come from the column's current values over the CTA's rows,
// and are stored at [bx][perm[j0 + c]] (row group × original column).
// OUTL (SSQR, "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
// Algorithm", §3): the group's step is α·s₀ with the zero point of s₀; a
// weight whose unclipped code leaves the grid is an outlier: it keeps its
// current value (written to Wp at its own position, the strip being loaded
// already), contributes no error, and its code byte carries OUTLIER_FLAG.
// QM selects the quantizer: 0 the hot path's clamp, 1 SSQR's outliers, 2
// HPTQ's unbounded lattice s·ℤ (same α-scaled step, k = rint(v/s) with no
// clamp; each int16 coordinate goes to the thread's own row of the strip box
// it was loaded from, which nothing reads again, and leaves with the block),
// 3 static groups (the clamp, with the scale and zero of each column's
// original group fixed beforehand and read per column).
template <bool ROWG, int QM>
__device__ __forceinline__ void sweep_body(
    const CUtensorMap& tmEhi, const CUtensorMap& tmElo, const CUtensorMap& tmW, int strip_tma,
    const CUtensorMap& tmPhi, const CUtensorMap& tmPlo, const CUtensorMap& tmUhi,
    const CUtensorMap& tmUlo, int64_t k0p, int kwp, float* Wp, int64_t m,
    int64_t n, int64_t j0, int bw, const unsigned char* __restrict__ pkg, int bits, int group,
    int64_t ngroups, uint8_t* __restrict__ codes, float* __restrict__ scale,
    uint8_t* __restrict__ zero, float* __restrict__ loss_row, int32_t* info,
    const int32_t* __restrict__ perm, const OutlierArgs& oa, int bx, unsigned char* smraw) {
  const uint32_t raw = smem_addr(smraw);
  unsigned char* sm = smraw + ((1024 - (raw & 1023)) & 1023);
  const float* Ud = reinterpret_cast<const float*>(sm + SM_PKG + PK_UD);
  const float* rdiag = reinterpret_cast<const float*>(sm + SM_PKG + PK_RD);
  unsigned char* ahi = sm + SM_AHI;
  unsigned char* alo = sm + SM_ALO;
  unsigned char* vals = sm + SM_VALS;
  uint8_t* cs = sm + SM_CODES;
  uint64_t* pkg_bar = reinterpret_cast<uint64_t*>(sm + SM_BARS);
  uint64_t* mma_bar = pkg_bar + 1;
  uint64_t* pro_bar = mma_bar + 1;      // prologue chunk loads, one per buffer set
  uint64_t* pro_mma = pro_bar + 2;      // prologue products but the last, one per set
  uint64_t* pro_done = pro_mma + 2;     // the last prologue product
  uint64_t* strip_bar = pro_done + 1;   // the strip's four boxes
  uint32_t* tslot = reinterpret_cast<uint32_t*>(strip_bar + 1);
  const bool pro = kwp > 0;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t r0 = (int64_t)bx * RT;
  const int64_t row = r0 + t;

  if (t == 0) {
    mbar_init(pkg_bar, 1);
    mbar_init(mma_bar, 1);
    mbar_init(&pro_bar[0], 1);
    mbar_init(&pro_bar[1], 1);
    mbar_init(&pro_mma[0], 1);
    mbar_init(&pro_mma[1], 1);
    mbar_init(pro_done, 1);
    mbar_init(strip_bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, SB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  pdl_wait();                           // the strip was written by the previous kernel
  pdl_trigger();
  float alpha = 1.f;
  if constexpr (QM != 0) alpha = *oa.alpha;
  // row groups: column j0 + t's original index, so that thread c stores column
  // c's scale and zero without a load in the column chain
  int32_t perm_t = 0;
  if constexpr (ROWG) perm_t = (t < bw) ? perm[j0 + t] : 0;
  int* sgrp = reinterpret_cast<int*>(sm + SM_SGRP);
  if constexpr (QM == 3) sgrp[t] = (t < bw) ? oa.perm[j0 + t] / group : 0;   // read after a barrier
  if (t == 0) {
    // the strip, when the rows allow a tensor map: four boxes at (j0 + 32q,
    // r0); columns past n read as zero, and Wp holds whole 128-row boxes
    if (strip_tma) {
      mbar_arrive_expect_tx(strip_bar, 4 * VBOX);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tma_load_2d(vals + q * VBOX, &tmW, (int)j0 + 32 * q, (int)r0, strip_bar);
    }
    if (!pro) {
      mbar_arrive_expect_tx(pkg_bar, PK_BYTES);
      bulk_g2s(sm + SM_PKG, pkg, PK_BYTES, pkg_bar);
    } else {
      // Prologue: D = E_prev·U[prev block, this block] in TMEM, the previous
      // block's contribution to this block's columns (the part of the
      // lazy-batch update the next sweep needs first), 3xTF32 like the
      // trailing update, in K-chunks of 32.  The chunks alternate between two
      // buffer sets, the A/B buffers and the package's region, so that the
      // next chunk's copies run under this chunk's products; the package
      // follows the last product (all threads wait for pro_done before they
      // read D, and for the package before the first column step).
      const int nk = kwp / SS;
      const uint32_t idesc = idesc_f32acc(2, 2, 0, 0, RT, SB);
      auto opnd = [&](int st, int w) -> unsigned char* {      // w: A hi, A lo, B hi, B lo
        if (st) return sm + SM_PKG + w * VBOX;
        return w == 0 ? ahi : (w == 1 ? alo : (w == 2 ? sm + SM_BPHI : sm + SM_BPLO));
      };
      auto load = [&](int c) {
        const int st = c & 1;
        mbar_arrive_expect_tx(&pro_bar[st], 4 * VBOX);
        tma_load_2d(opnd(st, 0), &tmPhi, SS * c, (int)r0, &pro_bar[st]);
        tma_load_2d(opnd(st, 1), &tmPlo, SS * c, (int)r0, &pro_bar[st]);
        tma_load_2d(opnd(st, 2), &tmUhi, (int)k0p + SS * c, (int)j0, &pro_bar[st]);
        tma_load_2d(opnd(st, 3), &tmUlo, (int)k0p + SS * c, (int)j0, &pro_bar[st]);
      };
      load(0);
      if (nk > 1) load(1);
      int landed = 0;                   // chunks whose copies are known to have landed
      const int loaded = nk;            // every chunk is loaded unless a wait fails
      bool fail = false;
      for (int c = 0; c < nk && !fail; ++c) {
        const int st = c & 1;
        if (!mbar_wait_bounded(&pro_bar[st], (c >> 1) & 1)) {
          fail = true;
          break;
        }
        landed = c + 1;
        tc_fence_after();
        const uint32_t ah = smem_addr(opnd(st, 0)), al = smem_addr(opnd(st, 1));
        const uint32_t bh = smem_addr(opnd(st, 2)), bl = smem_addr(opnd(st, 3));
#pragma unroll
        for (int ks = 0; ks < SS / 8; ++ks) {
          const uint64_t dah = sdesc_sw128(ah + ks * 32, SW128_KMAJOR_LBO, 1024);
          const uint64_t dal = sdesc_sw128(al + ks * 32, SW128_KMAJOR_LBO, 1024);
          const uint64_t dbh = sdesc_sw128(bh + ks * 32, SW128_KMAJOR_LBO, 1024);
          const uint64_t dbl = sdesc_sw128(bl + ks * 32, SW128_KMAJOR_LBO, 1024);
          umma_tf32_ss(tmem, dah, dbh, idesc, (c > 0 || ks > 0) ? 1u : 0u);
          umma_tf32_ss(tmem, dah, dbl, idesc, 1u);
          umma_tf32_ss(tmem, dal, dbh, idesc, 1u);
        }
        umma_commit(c + 1 < nk ? &pro_mma[st] : pro_done);
        // the set of chunk c − 1 is free once its products are: chunk c + 1
        if (c >= 1 && c + 1 < nk) {
          if (!mbar_wait_bounded(&pro_mma[(c - 1) & 1], ((c - 1) >> 1) & 1)) {
            fail = true;
            break;
          }
          load(c + 1);
        }
      }
      if (fail) {
        report(info, GPTQ_ERR_TIMEOUT, bx);
        // let our own copies land before the CTA gives up (at most two sets
        // are in flight: chunks landed and landed + 1)
        for (int c = landed; c < loaded && c < landed + 2; ++c)
          mbar_wait_bounded(&pro_bar[c & 1], (c >> 1) & 1);
      } else if (mbar_wait_bounded(pro_done, 0)) {
        mbar_arrive_expect_tx(pkg_bar, PK_BYTES);  // the package's region is free again
        bulk_g2s(sm + SM_PKG, pkg, PK_BYTES, pkg_bar);
      }
    }
  }

  if (!strip_tma) {
    // rows of n % 4 ≠ 0 floats: warp w reads rows 32w .. 32w+31 with lanes
    // along the columns (coalesced) into the same swizzled layout; rows past
    // m and columns past the block are zero
#pragma unroll 1
    for (int i0 = 0; i0 < 32; i0 += 8) {
      float buf[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t r = r0 + 32 * warp + i0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = lane + 32 * j;
          buf[i][j] = (r < m && c < bw) ? __ldg(Wp + r * n + j0 + c) : 0.f;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = 32 * warp + i0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int cc = lane;       // column 32j + lane: box j, chunk lane/4
          *reinterpret_cast<float*>(vals + j * VBOX + rr * 128 + (((cc >> 2) ^ (rr & 7)) << 4) +
                                    (cc & 3) * 4) = buf[i][j];
        }
      }
    }
    __syncthreads();
  }

  // the strip (and, without a prologue, the package); with a prologue the
  // package is waited for after the group statistics, before the first step
  bool ok0 = !strip_tma || mbar_wait_bounded(strip_bar, 0);
  if (!pro) ok0 = mbar_wait_bounded(pkg_bar, 0) && ok0;
  bool abort = __syncthreads_or(!ok0) != 0;
  if (abort) {
    report(info, GPTQ_ERR_TIMEOUT, bx);
    if (t == 0) {                       // let our own copies land first
      if (strip_tma) mbar_wait_bounded(strip_bar, 0);
      if (!pro) mbar_wait_bounded(pkg_bar, 0);
    }
  }

  const float maxq = (float)((1 << bits) - 1);
  const float rmaxq = __frcp_rn(maxq);
  float s = 1.f, z = 0.f, loss = 0.f, rs = 1.f, klo = 0.f, khi = maxq;
  uint8_t* cr = cs + t * LDB;
  int ocnt = 0;                         // this row's outliers in the block
  const int nsb = (bw + SS - 1) / SS;
  int issued = 0;                       // MMA groups committed to mma_bar
  for (int sb = 0; sb < nsb && !abort; ++sb) {
    const int c0 = sb * SS;
    float v[SS], e[SS];
    if (sb == 0) {
      float d[32];
      if (pro) {
        const bool ok = mbar_wait_bounded(pro_done, 0);
        if (__syncthreads_or(!ok)) {
          report(info, GPTQ_ERR_TIMEOUT, bx);
          abort = true;
          break;
        }
        tc_fence_after();
        tmem_ld_32x32b_x32(trow, d);
      }
#pragma unroll
      for (int j = 0; j < SS / 4; ++j) {
        const float4 f = strip_chunk(vals, 0, t, j);
        v[4 * j] = f.x - (pro ? d[4 * j] : 0.f);
        v[4 * j + 1] = f.y - (pro ? d[4 * j + 1] : 0.f);
        v[4 * j + 2] = f.z - (pro ? d[4 * j + 2] : 0.f);
        v[4 * j + 3] = f.w - (pro ? d[4 * j + 3] : 0.f);
      }
    } else {
      const bool ok = mbar_wait_bounded(mma_bar, (sb - 1) & 1);
      if (t == 0) bulk_wait_read_all();   // the previous errors have left the A buffers
      if (__syncthreads_or(!ok)) {
        report(info, GPTQ_ERR_TIMEOUT, bx);
        abort = true;
        break;
      }
      tc_fence_after();
      float d[32];
      tmem_ld_32x32b_x32(trow + c0, d);
#pragma unroll
      for (int j = 0; j < SS / 4; ++j) {
        const float4 f = strip_chunk(vals, sb, t, j);
        v[4 * j] = f.x - d[4 * j];
        v[4 * j + 1] = f.y - d[4 * j + 1];
        v[4 * j + 2] = f.z - d[4 * j + 2];
        v[4 * j + 3] = f.w - d[4 * j + 3];
      }
    }
    if (!ROWG && QM != 3 && c0 % group == 0) {
      // the group's current values: this sub-block, then later ones in the group
      float xmin = 0.f, xmax = 0.f;
#pragma unroll
      for (int k = 0; k < SS; ++k) {
        const float x = (c0 + k < bw) ? v[k] : 0.f;
        xmin = fminf(xmin, x);
        xmax = fmaxf(xmax, x);
      }
      const int gend = min(c0 + group, bw);
      for (int cs0 = c0 + SS; cs0 < gend; cs0 += SS) {
        float d[32];
        const bool upd = sb > 0 || pro;            // D holds updates for these columns
        if (upd) tmem_ld_32x32b_x32(trow + cs0, d);
#pragma unroll
        for (int j = 0; j < SS / 4; ++j) {
          const float4 f = strip_chunk(vals, cs0 / SS, t, j);
          const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int k = 4 * j + k4;
            const float x = (cs0 + k < gend) ? fv[k4] - (upd ? d[k] : 0.f) : 0.f;
            xmin = fminf(xmin, x);
            xmax = fmaxf(xmax, x);
          }
        }
      }
      if (xmin == 0.f && xmax == 0.f) { xmin = -1.f; xmax = 1.f; }
      s = __fdiv_rn(xmax - xmin, maxq);
      z = rintf(div_rn(-xmin, s));
      if constexpr (QM != 0) s = __fmul_rn(s, alpha);
      rs = fminf(__frcp_rn(s), 3.4028234663852886e38f);
      klo = -z;
      khi = maxq - z;
      if (row < m) {
        const int64_t g = (j0 + c0) / group;
        scale[row * ngroups + g] = s;
        zero[row * ngroups + g] = (uint8_t)z;
      }
    }
    if (sb == 0 && pro) {               // the package, loaded after the prologue
      const bool okp = mbar_wait_bounded(pkg_bar, 0);
      if (__syncthreads_or(!okp)) {
        report(info, GPTQ_ERR_TIMEOUT, bx);
        if (t == 0) mbar_wait_bounded(pkg_bar, 0);   // let our own copy land first
        abort = true;
        break;
      }
    }
    // ---- the 32 dependent column steps
    const float* ud = Ud + sb * SS * SS;
#pragma unroll
    for (int i = 0; i < SS; ++i) {
      const int c = c0 + i;
      if constexpr (ROWG) {
        // the column's min and max over the CTA's rows (0 inside the range):
        // warp shuffles, then the four warps through shared memory (two
        // buffers by column parity, so one barrier per column suffices)
        // warp min and max in one instruction each, on an integer image of
        // the floats that orders like them (negative values get their
        // magnitude bits flipped; the map is its own inverse)
        const int kn = ord_key(fminf(v[i], 0.f)), kx = ord_key(fmaxf(v[i], 0.f));
        int wn, wx;
        asm volatile("redux.sync.min.s32 %0, %1, 0xffffffff;" : "=r"(wn) : "r"(kn));
        asm volatile("redux.sync.max.s32 %0, %1, 0xffffffff;" : "=r"(wx) : "r"(kx));
        const float mn = __int_as_float(ord_key_inv(wn)), mx = __int_as_float(ord_key_inv(wx));
        float* red = reinterpret_cast<float*>(sm + SM_RGRED) + (i & 1) * 8;
        if (lane == 0) {
          red[warp] = mn;
          red[4 + warp] = mx;
        }
        __syncthreads();
        float xmin = fminf(fminf(red[0], red[1]), fminf(red[2], red[3]));
        float xmax = fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]));
        if (xmin == 0.f && xmax == 0.f) {
          xmin = -1.f;
          xmax = 1.f;
        }
        // range/maxq correctly rounded: Markstein's correction from RN(1/maxq)
        // for a normal range, the division itself for a tiny one
        const float range = xmax - xmin;
        s = range >= 1e-30f ? div_fma(range, maxq, rmaxq) : __fdiv_rn(range, maxq);
        rs = fminf(__frcp_rn(s), 3.4028234663852886e38f);
        z = rintf(div_rn(-xmin, s));
        klo = -z;
        khi = maxq - z;
        if (t == c && c < bw) {
          scale[(int64_t)bx * n + perm_t] = s;
          zero[(int64_t)bx * n + perm_t] = (uint8_t)z;
        }
      }
      if constexpr (QM == 3) {
        const int64_t gx = row * oa.st_ng + sgrp[c];
        s = row < m ? oa.st_scale[gx] : 1.f;
        z = row < m ? (float)oa.st_zero[gx] : 0.f;
        rs = fminf(__frcp_rn(s), 3.4028234663852886e38f);
        klo = -z;
        khi = maxq - z;
      }
      // q − z = clamp(rint(v/s), −z, maxq − z) exactly (small integers), so
      // the clamp works on k = q − z and the error takes one FMA
      const float raw = rintf(div_fma(v[i], s, rs));
      const float k = QM == 2 ? raw : fminf(fmaxf(raw, klo), khi);
      float ei = fmaf(-s, k, v[i]) * rdiag[c];
      if constexpr (QM == 2) {
        const int qi = __float2int_rn(k);          // the lattice coordinate; saturating
        const int q16 = max(-32768, min(32767, qi));
        *reinterpret_cast<int16_t*>(vals + sb * VBOX + t * 128 + i * 2) = (int16_t)q16;
      } else if constexpr (QM == 1) {
        const bool o = raw != k;        // the unclipped code leaves the grid
        ei = o ? 0.f : ei;
        ocnt += o ? 1 : 0;
        if (o && row < m && c < bw) Wp[row * n + j0 + c] = v[i];
        cr[c] = (uint8_t)(k + z) | (o ? OUTLIER_FLAG : (uint8_t)0);
      } else {
        cr[c] = (uint8_t)(k + z);
      }
      e[i] = ei;
      loss = fmaf(ei, ei, loss);
      const float4* ur = reinterpret_cast<const float4*>(ud + i * SS);
#pragma unroll
      for (int q4 = (i + 1) / 4; q4 < SS / 4; ++q4) {
        const float4 u = ur[q4];
        if (4 * q4 + 0 > i) v[4 * q4 + 0] = fmaf(-ei, u.x, v[4 * q4 + 0]);
        if (4 * q4 + 1 > i) v[4 * q4 + 1] = fmaf(-ei, u.y, v[4 * q4 + 1]);
        if (4 * q4 + 2 > i) v[4 * q4 + 2] = fmaf(-ei, u.z, v[4 * q4 + 2]);
        if (4 * q4 + 3 > i) v[4 * q4 + 3] = fmaf(-ei, u.w, v[4 * q4 + 3]);
      }
    }
    // ---- errors out: TF32 split into the K-major swizzled A operand in
    // shared memory, which feeds the in-block far update (tensor cores) and
    // leaves for the trailing update as two TMA box stores
    float eh[SS], el[SS];
#pragma unroll
    for (int k = 0; k < SS; ++k) {
      eh[k] = to_tf32(e[k]);
      el[k] = e[k] - eh[k];
    }
#pragma unroll
    for (int q = 0; q < SS / 4; ++q) {
      const uint32_t off = t * 128 + ((q ^ (t & 7)) << 4);
      *reinterpret_cast<float4*>(ahi + off) =
          make_float4(eh[4 * q], eh[4 * q + 1], eh[4 * q + 2], eh[4 * q + 3]);
      *reinterpret_cast<float4*>(alo + off) =
          make_float4(el[4 * q], el[4 * q + 1], el[4 * q + 2], el[4 * q + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      if (sb + 1 < nsb) {
        tc_fence_after();
        // D[:, 32(sb+1) : 128] += E·U[c0:c0+32, 32(sb+1):128]
        const uint32_t N = (uint32_t)(SB - SS * (sb + 1));
        const uint32_t idesc = idesc_f32acc(2, 2, 0, 0, RT, N);
        const uint32_t bhi = smem_addr(sm + SM_PKG + PK_BHI + box_index(sb, sb + 1) * BOX);
        const uint32_t blo = smem_addr(sm + SM_PKG + PK_BLO + box_index(sb, sb + 1) * BOX);
        const uint32_t ah = smem_addr(ahi), al = smem_addr(alo);
        const uint32_t dcol = tmem + (uint32_t)(SS * (sb + 1));
#pragma unroll
        for (int ks = 0; ks < SS / 8; ++ks) {
          const uint64_t dah = sdesc_sw128(ah + ks * 32, SW128_KMAJOR_LBO, 1024);
          const uint64_t dal = sdesc_sw128(al + ks * 32, SW128_KMAJOR_LBO, 1024);
          const uint64_t dbh = sdesc_sw128(bhi + ks * 32, SW128_KMAJOR_LBO, 1024);
          const uint64_t dbl = sdesc_sw128(blo + ks * 32, SW128_KMAJOR_LBO, 1024);
          umma_tf32_ss(dcol, dah, dbh, idesc, (pro || sb > 0 || ks > 0) ? 1u : 0u);
          umma_tf32_ss(dcol, dah, dbl, idesc, 1u);
          umma_tf32_ss(dcol, dal, dbh, idesc, 1u);
        }
        umma_commit(mma_bar);
      }
      // the error buffers hold whole 128-row boxes (rows past m are zeros)
      tma_store_2d(&tmEhi, c0, (int)r0, ahi);
      tma_store_2d(&tmElo, c0, (int)r0, alo);
      bulk_commit();
    }
    if (sb + 1 < nsb) ++issued;
  }
  if (!abort && row < m && loss_row != nullptr) loss_row[row] += loss;
  if constexpr (QM == 1) {
    if (!abort && row < m) oa.row_cnt[row] += ocnt;
    const int wc = __reduce_add_sync(0xffffffffu, ocnt);
    if (lane == 0 && wc != 0 && !abort) atomicAdd(oa.total, (unsigned long long)wc);
  }
  tc_fence_before();
  __syncthreads();

  // codes out, one warp per row, coalesced (four codes per lane and store
  // when rows and the block width allow it; j0 is a multiple of 32)
  if (QM == 2 && !abort) {
    // int16 codes from the strip boxes: column c of row rr at box c/32,
    // byte rr·128 + (c mod 32)·2
    const bool wide = ((n & 3) == 0);
    for (int rr = warp; rr < RT; rr += RT / 32) {
      const int64_t r = r0 + rr;
      if (r >= m) break;
      const int c = 4 * lane;
      if (c >= bw) continue;
      const unsigned char* src = vals + (c >> 5) * VBOX + rr * 128 + (c & 31) * 2;
      int16_t* dst = oa.codes16 + r * n + j0 + c;
      if (wide && c + 3 < bw) {
        *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
      } else {
        for (int k = 0; k < 4 && c + k < bw; ++k)
          dst[k] = reinterpret_cast<const int16_t*>(src)[k];
      }
    }
  } else if (!abort) {
    const bool wide = ((n & 3) == 0) && ((bw & 3) == 0);
    for (int rr = warp; rr < RT; rr += RT / 32) {
      const int64_t r = r0 + rr;
      if (r >= m) break;
      if (wide) {
        const int c = 4 * lane;
        if (c < bw)
          *reinterpret_cast<uint32_t*>(codes + r * n + j0 + c) =
              *reinterpret_cast<const uint32_t*>(cs + rr * LDB + c);
      } else {
#pragma unroll
        for (int it = 0; it < SB / 32; ++it) {
          const int c = lane + 32 * it;
          if (c < bw) codes[r * n + j0 + c] = cs[rr * LDB + c];
        }
      }
    }
  }
  if (t == 0) bulk_wait_all();          // the error boxes are in global memory
  if (abort && t == 0 && issued > 0)            // no MMA may still write TMEM
    mbar_wait_bounded(mma_bar, (issued - 1) & 1, 1u << 16);
  if (abort && t == 0 && pro) mbar_wait_bounded(pro_done, 0, 1u << 16);
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, SB);
}

// The sweep of one block (CTAs 0 .. nsweep−1) and, in the same launch, the
// far-column update of the block before (the CTAs after them, fx tiles of
// 256 columns per 128-row tile): the two touch different columns, and both
// take their inputs from earlier launches, so that consecutive sweeps follow
// each other with nothing between them but the programmatic launch edge.
template <bool ROWG, int QM>
__global__ void __launch_bounds__(RT, 1)
sweep_kernel(const __grid_constant__ CUtensorMap tmEhi, const __grid_constant__ CUtensorMap tmElo,
             const __grid_constant__ CUtensorMap tmW, int strip_tma,
             const __grid_constant__ CUtensorMap tmPhi, const __grid_constant__ CUtensorMap tmPlo,
             const __grid_constant__ CUtensorMap tmUhi, const __grid_constant__ CUtensorMap tmUlo,
             int64_t k0p, int kwp,
             float* Wp, int64_t m, int64_t n, int64_t j0, int bw,
             const unsigned char* __restrict__ pkg, int bits, int group, int64_t ngroups,
             uint8_t* __restrict__ codes, float* __restrict__ scale,
             uint8_t* __restrict__ zero, float* __restrict__ loss_row, int32_t* info,
             const int32_t* __restrict__ perm, const OutlierArgs oa, int nsweep,
             const __grid_constant__ TrailMaps far, int64_t fc0, int64_t fc1, int64_t fk0,
             int fkw, int fx) {
  extern __shared__ unsigned char smraw[];
  const int b = (int)blockIdx.x;
  if (b < nsweep) {
    sweep_body<ROWG, QM>(tmEhi, tmElo, tmW, strip_tma, tmPhi, tmPlo, tmUhi, tmUlo, k0p, kwp,
                           Wp, m, n, j0, bw, pkg, bits, group, ngroups, codes, scale, zero,
                           loss_row, info, perm, oa, b, smraw);
  } else {
    const int f = b - nsweep;
    trailing_tc_body(far, m, n, fc0, fc1, fk0, fkw, info, f % fx, f / fx, smraw);
  }
}

}  // namespace

size_t panel_workspace_bytes(int64_t n, int block) {
  return (size_t)ceil_div(n, block) * PANEL_BYTES;
}

gptq_status launch_panels(const float* U, int64_t n, int block, float* panels,
                          cudaStream_t s) {
  const dim3 grid((unsigned)ceil_div(n, block), 11);
  GPTQ_LAUNCH(KK_INGEST, s, package_kernel, grid, 256, 0, U, n, block,
              reinterpret_cast<unsigned char*>(panels));
  return GPTQ_OK;
}

gptq_status launch_sweep(float* Wp, int64_t m, int64_t n, int64_t j0, int bw,
                         const float* panel, int bits, int group, int64_t ngroups,
                         uint8_t* codes, float* scale, uint8_t* zero, float* Ehi,
                         float* Elo, int64_t epitch, const SweepPrologue& pre, const SweepFar& far,
                         float* loss_row, int32_t* info, const int32_t* rowgroup_perm,
                         const OutlierArgs* outl, cudaStream_t s) {
  constexpr size_t kSmem = SMEM_BYTES > QSMEM ? SMEM_BYTES : QSMEM;
  const bool rowg = rowgroup_perm != nullptr;
  if (rowg && outl != nullptr)
    return fail(GPTQ_ERR_UNSUPPORTED, "sweep: outliers with output-channel groups");
  if (outl != nullptr && outl->static_groups &&
      (!outl->st_scale || !outl->st_zero || !outl->perm || outl->st_ng < 1))
    return fail(GPTQ_ERR_INVALID_ARG, "sweep: static-group arguments");
  if (outl != nullptr && !outl->unclipped && !outl->static_groups &&
      (!outl->alpha || !outl->row_cnt || !outl->total || bits > 7))
    return fail(GPTQ_ERR_INVALID_ARG, "sweep: outlier arguments");
  if (outl != nullptr && outl->unclipped && (!outl->alpha || !outl->codes16))
    return fail(GPTQ_ERR_INVALID_ARG, "sweep: unclipped-grid arguments");
  const int variant = rowg ? 1
                      : (outl == nullptr ? 0
                                         : (outl->static_groups ? 4 : (outl->unclipped ? 3 : 2)));
  {
    const void* fn = variant == 1 ? (const void*)sweep_kernel<true, 0>
                     : variant == 2 ? (const void*)sweep_kernel<false, 1>
                     : variant == 3 ? (const void*)sweep_kernel<false, 2>
                     : variant == 4 ? (const void*)sweep_kernel<false, 3>
                                    : (const void*)sweep_kernel<false, 0>;
    const gptq_status st = ensure_smem_limit(fn, (int)kSmem, "sweep_kernel");
    if (st != GPTQ_OK) return st;
  }
  const OutlierArgs oa = outl != nullptr ? *outl : OutlierArgs();
  // the far-column update riding along: fx 256-column tiles per 128-row tile
  TrailMaps fm;
  memset(&fm, 0, sizeof(fm));
  const int64_t fc1 = far.c1 < n ? far.c1 : n;
  int fx = 0, nfar = 0;
  if (far.kw > 0 && far.c0 < fc1 && far.Ehi && far.Elo && far.Uhi && far.Ulo) {
    if (far.kw % QK != 0 || far.kw > kSuperBlocks * SB || far.kw > far.epitch || (n % 4) != 0)
      return fail(GPTQ_ERR_INVALID_ARG, "sweep far update: width %d", far.kw);
    if (!make_trail_maps(&fm, Wp, m, n, far.Ehi, far.Elo, far.kw, far.epitch, far.Uhi, far.Ulo))
      return fail(GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the sweep's far update");
    fx = (int)ceil_div(fc1 - far.c0, QN);
    nfar = fx * (int)ceil_div(m, QM);
  }
  CUtensorMap th, tl;
  const int64_t mr = error_rows(m);     // whole boxes: a clipped box store is slow
  CUtensorMap tw;
  const int strip_tma = ((n & 3) == 0) ? 1 : 0;   // row pitch a multiple of 16 bytes
  if (strip_tma &&
      !encode_tiled_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Wp, n, mr, n * 4, SS, RT))
    return fail(GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the sweep's strip");
  if (!strip_tma) memset(&tw, 0, sizeof(tw));
  CUtensorMap tph, tpl, tuh, tul;
  const int kwp = (pre.kw > 0 && pre.Ehi && pre.Elo && pre.Uhi && pre.Ulo) ? pre.kw : 0;
  if (kwp > 0) {
    if (kwp % SS != 0 || pre.kw > SB)
      return fail(GPTQ_ERR_INVALID_ARG, "sweep prologue: width %d", pre.kw);
    if (!encode_tiled_2d(&tph, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pre.Ehi, SB, mr, pre.epitch * 4,
                         SS, RT) ||
        !encode_tiled_2d(&tpl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pre.Elo, SB, mr, pre.epitch * 4,
                         SS, RT) ||
        !encode_tiled_2d(&tuh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pre.Uhi, n, n, n * 4, SS, RT) ||
        !encode_tiled_2d(&tul, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pre.Ulo, n, n, n * 4, SS, RT))
      return fail(GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the sweep's prologue");
  } else {
    memset(&tph, 0, sizeof(tph));
    memset(&tpl, 0, sizeof(tpl));
    memset(&tuh, 0, sizeof(tuh));
    memset(&tul, 0, sizeof(tul));
  }
  if (!encode_tiled_2d(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Ehi, SB, mr, epitch * 4, SS, RT) ||
      !encode_tiled_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Elo, SB, mr, epitch * 4, SS, RT))
    return fail(GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the sweep's error output");
  const int nsweep = (int)ceil_div(m, RT);
  const unsigned grid = (unsigned)(nsweep + nfar);
  const unsigned char* pk = reinterpret_cast<const unsigned char*>(panel);
  const int fxx = fx > 0 ? fx : 1;
  if (variant == 1)
    GPTQ_LAUNCH_PDL(KK_SWEEP, s, (sweep_kernel<true, 0>), grid, RT, kSmem, th, tl, tw,
                    strip_tma, tph, tpl, tuh, tul, (int64_t)pre.k0, kwp, Wp, m, n, j0, bw, pk,
                    bits, group, ngroups, codes, scale, zero, loss_row, info, rowgroup_perm, oa,
                    nsweep, fm, far.c0, fc1, far.k0, far.kw, fxx);
  else if (variant == 2)
    GPTQ_LAUNCH_PDL(KK_SWEEP, s, (sweep_kernel<false, 1>), grid, RT, kSmem, th, tl, tw,
                    strip_tma, tph, tpl, tuh, tul, (int64_t)pre.k0, kwp, Wp, m, n, j0, bw, pk,
                    bits, group, ngroups, codes, scale, zero, loss_row, info,
                    (const int32_t*)nullptr, oa, nsweep, fm, far.c0, fc1, far.k0, far.kw, fxx);
  else if (variant == 4)
    GPTQ_LAUNCH_PDL(KK_SWEEP, s, (sweep_kernel<false, 3>), grid, RT, kSmem, th, tl, tw,
                    strip_tma, tph, tpl, tuh, tul, (int64_t)pre.k0, kwp, Wp, m, n, j0, bw, pk,
                    bits, group, ngroups, codes, scale, zero, loss_row, info,
                    (const int32_t*)nullptr, oa, nsweep, fm, far.c0, fc1, far.k0, far.kw, fxx);
  else if (variant == 3)
    GPTQ_LAUNCH_PDL(KK_SWEEP, s, (sweep_kernel<false, 2>), grid, RT, kSmem, th, tl, tw,
                    strip_tma, tph, tpl, tuh, tul, (int64_t)pre.k0, kwp, Wp, m, n, j0, bw, pk,
                    bits, group, ngroups, codes, scale, zero, loss_row, info,
                    (const int32_t*)nullptr, oa, nsweep, fm, far.c0, fc1, far.k0, far.kw, fxx);
  else
    GPTQ_LAUNCH_PDL(KK_SWEEP, s, (sweep_kernel<false, 0>), grid, RT, kSmem, th, tl, tw,
                    strip_tma, tph, tpl, tuh, tul, (int64_t)pre.k0, kwp, Wp, m, n, j0, bw, pk,
                    bits, group, ngroups, codes, scale, zero, loss_row, info,
                    (const int32_t*)nullptr, oa, nsweep, fm, far.c0, fc1, far.k0, far.kw, fxx);
  return GPTQ_OK;
}

}  // namespace gptq
