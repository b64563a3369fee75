// Host launchers of the quantize-side kernels (one translation unit each).
#pragma once

#include "common.cuh"

namespace gptq {

// Largest block width, and the bytes of the per-block package of U that the
// sweep fetches with one bulk copy: 12 swizzled 32×32 TF32 boxes (hi and lo
// of the 6 off-diagonal pieces), 4 diagonal 32×32 pieces, 128 reciprocal
// diagonals.
constexpr int SWEEP_BLOCK_MAX = 128;
constexpr size_t PANEL_BYTES = (size_t)16 * 4096 + 128 * sizeof(float);

size_t panel_workspace_bytes(int64_t n, int block);

// Rows of the working copy Wp and of the error buffers Ehi/Elo: m rounded up
// to whole 128-row boxes, so that no box store or reduction is clipped (a
// clipped one is several times slower).  Rows ≥ m are never read back.
inline int64_t error_rows(int64_t m) { return (m + 127) / 128 * 128; }

// One panel per block of U, laid out for the sweep's bulk copy.
gptq_status launch_panels(const float* U, int64_t n, int block, float* panels,
                          cudaStream_t s);

// Columns [j0, j0+bw) of the float32 working copy Wp (m×n, processing order):
// quantize column by column with in-block error propagation.  Writes codes
// (m×n u8, processing order), scale/zero (m×ngroups), the scaled errors as a
// TF32 split Ehi + Elo (each error_rows(m)×128, Ehi = TF32(e), Elo = e − Ehi
// exactly) and
// adds Σe² to loss_row (may be NULL).
//
// With pre.kw > 0 the sweep first applies the previous block's contribution to
// its own columns: D = (pre.Ehi + pre.Elo)[:, 0:pre.kw]·U[pre.k0 : pre.k0+pre.kw,
// j0 : j0+bw] on the tensor cores (pre.Uhi/Ulo: the transposed TF32 split of U,
// n % 4 == 0), so that no separate trailing update is needed for those columns.
struct SweepPrologue {
  const float* Ehi = nullptr;   // previous block's errors (error_rows(m) rows, pitch epitch)
  const float* Elo = nullptr;
  int64_t epitch = SWEEP_BLOCK_MAX;  // floats between rows of the error buffers
  const float* Uhi = nullptr;   // transposed TF32 split of U
  const float* Ulo = nullptr;
  int64_t k0 = 0;               // first column of the previous block
  int kw = 0;                   // its width (a multiple of 32), 0 for none
};
// rowgroup_perm != NULL: scales along the output channels instead (groups of
// the CTA's 128 rows, one scale and zero per row group and column, from the
// column's current values), stored as scale[g·n + rowgroup_perm[j]] for
// processing position j; `group` and `ngroups` are then unused.
//
// With far.kw > 0 and far.c0 < far.c1 the same launch also applies the
// block before's far-column update, Wp[:, c0:c1] −= (far.Ehi + far.Elo)[:, 0:kw]·
// U[far.k0 : far.k0+kw, c0:c1] (tensor cores, far.Uhi/Ulo as above): columns
// the sweep does not touch, from inputs of earlier launches.
struct SweepFar {
  const float* Ehi = nullptr;   // errors: kw columns from here on each row, pitch epitch
  const float* Elo = nullptr;
  int64_t epitch = SWEEP_BLOCK_MAX;
  const float* Uhi = nullptr;
  const float* Ulo = nullptr;
  int64_t c0 = 0, c1 = 0;       // columns (c1 is clipped to n)
  int64_t k0 = 0;               // first column of the blocks whose errors they are
  int kw = 0;                   // their width (one block, or a super-block), 0 for none
};
//
// outl != NULL (SSQR): every group's step is multiplied by *outl->alpha (a
// device float, read when the launch starts; the zero point stays that of the
// min-max step).  A weight whose unclipped code falls outside [0, 2^bits − 1]
// is an outlier: its error is 0, its code byte carries OUTLIER_FLAG on top of
// the clipped code, its current value is written to Wp at its own position,
// and it is counted in outl->row_cnt[row] and *outl->total.  bits ≤ 7.
//
// outl->unclipped (HPTQ): the same α-scaled step, no clamp and no outliers;
// every weight's lattice coordinate k = rint(v/s) is written as int16
// (saturated) to outl->codes16 (m × n, processing order) instead of `codes`,
// and its error is v − s·k.
constexpr uint8_t OUTLIER_FLAG = 0x80;
//
// outl->static_groups: the hot path's clamped quantizer with every group's
// scale and zero fixed beforehand (st_scale / st_zero, m × st_ng, group g =
// perm[j] / group of processing column j); nothing is taken from the current
// values and the sweep writes no scale or zero.
struct OutlierArgs {
  const float* alpha = nullptr;
  int32_t* row_cnt = nullptr;          // m counts, accumulated over the blocks
  unsigned long long* total = nullptr; // all outliers of the pass
  bool unclipped = false;
  int16_t* codes16 = nullptr;
  bool static_groups = false;
  const float* st_scale = nullptr;
  const uint8_t* st_zero = nullptr;
  const int32_t* perm = nullptr;
  int64_t st_ng = 0;
};
gptq_status launch_sweep(float* Wp, int64_t m, int64_t n, int64_t j0, int bw,
                         const float* panel, int bits, int group, int64_t ngroups,
                         uint8_t* codes, float* scale, uint8_t* zero, float* Ehi,
                         float* Elo, int64_t epitch, const SweepPrologue& pre, const SweepFar& far,
                         float* loss_row, int32_t* info, const int32_t* rowgroup_perm,
                         const OutlierArgs* outl, cudaStream_t s);

// ---- the stages of gptq_quantize, shared with the SSQR entry point

// The two-level lazy batch: on the tensor-core path with 128-column blocks,
// the errors of kSuperBlocks consecutive blocks (a super-block) sit side by
// side, and the columns past the super-block (and the block after it)
// receive them in one K = kSuperBlocks·128 product instead of one product a
// block.
constexpr int kSuperBlocks = 4;
// Floats per row of the error buffers: a super-block, or one block elsewhere.
int error_width(int64_t n, int block);

// The far part of the trailing update carried by sweep b's launch (b ≥ 1) on
// the tensor-core path with super-blocks of S blocks (S = 1: none).  Block
// b−1's errors reach block b in sweep b's prologue; the far CTAs then apply
//  * inside a super-block (b mod S ≠ 0): block b−1's errors (K = block,
//    errors from column k0) to the rest of the super-block and the block
//    after it;
//  * at the first block of a super-block: the whole previous super-block's
//    errors (K = S·block) to every column past block b.
// Columns [c0, c1); empty when c0 ≥ c1.
struct FarRange {
  int64_t c0, c1, k0;
  int kw;
  bool whole;       // the previous super-block's errors
};
inline FarRange far_range(int64_t n, int block, int S, int64_t b) {
  const int64_t j0 = b * block;
  const int64_t bw = (n - j0 < block) ? (n - j0) : block;
  FarRange r;
  r.c0 = j0 + bw;
  if (b % S != 0) {
    const int64_t end = (b / S + 1) * S * (int64_t)block + block;
    r.c1 = end < n ? end : n;
    r.k0 = j0 - block;
    r.kw = block;
    r.whole = false;
  } else {
    r.c1 = n;
    r.k0 = j0 - (int64_t)S * block;
    r.kw = S * block;
    r.whole = true;
  }
  return r;
}

struct QuantWs {
  float* Wp;        // error_rows(m) × n working copy, processing order
  uint8_t* codes;   // m × n codes, processing order
  float* Ehi[2];    // error_rows(m) × ew scaled errors of a super-block, TF32 part
  float* Elo[2];    // remainder e − Ehi; two sets, alternating by super-block
  int ew;           // floats per row of the error buffers (error_width)
  int32_t* pinv;    // n + 1: processing position of each original column; pinv[n] = −1
                    // when the processing order is the identity, else 0
  float* panels;    // pre-transposed U panels, one per block
  float* Uhi;       // n × n TF32 part of Uᵀ (tensor-core trailing update only)
  float* Ulo;       // n × n remainder, transposed likewise
};
// Bytes of the layout (256-byte aligned parts); fills *w when both are given.
size_t quant_ws_layout(int64_t m, int64_t n, int block, QuantWs* w, char* base);

// A second working set for a pass that runs beside another: its own Wp,
// codes and error buffers at `base`, the U-derived parts (pinv, panels, the
// TF32 split) shared with `shared`.  Returns its bytes; fills *w when given.
size_t quant_slot_layout(int64_t m, int64_t n, int block, const QuantWs* shared, QuantWs* w,
                         char* base);

// Host checks shared by the quantize entry points (no device work).
gptq_status quant_check_args(int w_dtype, int64_t m, int64_t n, int bits, int group,
                             int block, const void* ws, size_t ws_bytes, size_t need);

// Once per call: info and pinv reset, pinv/g_idx, the panels and the TF32
// split of U.
gptq_status quant_setup(const QuantWs& w, int64_t m, int64_t n, const float* U,
                        const int32_t* perm, int group, int block, int32_t* g_idx,
                        int32_t* info, cudaStream_t s, bool static_groups = false);

// One pass of the column sweep over the whole layer: W → Wp (processing
// order, dead columns zeroed), then the block loop of sweeps and trailing
// updates.  rowgs > 0: output-channel groups (rowgroup mode).
gptq_status quant_pass(const QuantWs& w, const void* W, int w_dtype, int64_t m, int64_t n,
                       const float* U, const int32_t* perm, const uint8_t* dead, int bits,
                       int group, int block, int rowgs, float* scale, uint8_t* zero,
                       float* loss_row, const OutlierArgs* outl, int32_t* info,
                       cudaStream_t s);

// Codes → packed words in original column order, and the optional
// dequantized copy.  outl_vals != NULL: code bytes carry OUTLIER_FLAG, and the
// dequantized value of a flagged weight is outl_vals at its processing position.
gptq_status quant_pack(const QuantWs& w, int64_t m, int64_t n, int bits, int group, int rowgs,
                       const float* scale, const uint8_t* zero, uint32_t* qweight,
                       float* Qdq, const float* outl_vals, int32_t* info, cudaStream_t s,
                       bool static_groups = false);

// Whether the trailing update runs on the tensor cores for this shape.
bool trailing_uses_tensor_cores(int64_t n, int block);

// TF32 split of the n×n matrix x, transposed: hiT[c][r] = TF32(x[r][c]),
// loT[c][r] = x[r][c] − hiT[c][r].
gptq_status launch_split_tf32_t(const float* x, int64_t n, float* hiT, float* loT,
                                cudaStream_t s);

// Wp[:, c0:c1] −= (Ehi+Elo)[:, 0:kw]·U[k0:k0+kw, c0:c1]   (lazy-batch update;
// c1 is clipped to n) in float32 SIMT tiles: the path for n % 4 ≠ 0, where
// the tensor-core update (which rides in the sweep launches, SweepFar) cannot
// take its operands by tensor map.
gptq_status launch_trailing(float* Wp, int64_t m, int64_t n, int64_t c0, int64_t c1,
                            const float* Ehi, const float* Elo, int64_t k0, int kw,
                            const float* U, cudaStream_t s);

}  // namespace gptq
