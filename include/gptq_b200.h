/*
 * gptq_b200.h — C ABI of the B200 (sm_100a) GPTQ library.
 *
 * GPTQ quantizes a linear layer's weights column by column and pushes each
 * column's rounding error onto the columns not yet quantized, weighted by the
 * inverse Hessian of the layer inputs:
 *   "Warum Geometrie Gewichte nicht komprimiert" (nonndazone.ru), section
 *   "Methodik. Was ist CHMC", Schritt 2 — H = XᵀX/n + λ·mean(diag H)·I, the
 *   inverse through the Cholesky factorisation, act-order, and per column j:
 *   err_j = (col_j − q_j)/H⁻¹[j,j],  R[:, j+1:] −= err_j·H⁻¹[j, j+1:].
 *   "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
 *   Algorithm" (gist.science summary), §2.1–§2.3 — the same loop is Babai's
 *   nearest-plane algorithm on the lattice that the Hessian defines.
 *
 * Three calls follow that statement of the problem:
 *   gptq_hessian_accumulate(X)                 H += 2·XᵀX
 *   gptq_prepare(H, damp)                      U = upper Cholesky factor of
 *                                              (P·(H + damp·mean(diag H)·I)·Pᵀ)⁻¹
 *   gptq_quantize(W, U, bits, group, block)    packed codes + scale + zero
 *
 * Conventions shared by every call
 *   - Every array pointer is a DEVICE pointer unless stated otherwise; the
 *     caller owns all memory (outputs and workspaces).  The library never
 *     allocates device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it.
 *   - Arrays are dense and row-major (C order).
 *   - Host-detectable argument errors return before anything is enqueued.
 *     Errors found on the device (non-positive pivot, NaN/Inf input) are
 *     written to the caller's `info` array (two int32 on the device:
 *     info[0] = gptq_status, info[1] = index) and reported by gptq_check().
 *   - A CUDA launch error returns GPTQ_ERR_CUDA; gptq_last_error() gives the
 *     message of the last failure on the calling thread.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, workspace too small   */
  GPTQ_ERR_NOT_PD = 2,       /* damped, permuted H not positive definite     */
  GPTQ_ERR_NONFINITE = 3,    /* NaN or Inf in H or W                         */
  GPTQ_ERR_UNSUPPORTED = 4,  /* bits/group/block combination not implemented */
  GPTQ_ERR_TIMEOUT = 5,      /* a bounded device wait ran out                */
  GPTQ_ERR_CUDA = 6,         /* a CUDA runtime call failed                   */
  GPTQ_ERR_CAPACITY = 7      /* more results than the caller's buffer holds  */
} gptq_status;

typedef enum {
  GPTQ_ORDER_NATURAL = 0,  /* columns 0..n−1                                  */
  GPTQ_ORDER_ACT = 1,      /* descending diag(H); equal entries keep index order
                              ("act-order": Schritt 2 of the CHMC page; the
                              Babai page, §2.3, defines it by the diagonal)   */
  GPTQ_ORDER_REVERSE = 2,  /* columns n−1..0: back to front, the order in which
                              GPTQ is Babai's algorithm (Babai page, §2.2)    */
  GPTQ_ORDER_CUSTOM = 3,   /* caller's permutation, read from `perm`          */
  GPTQ_ORDER_MINPIVOT = 4  /* min-pivot: the LDL of Satz 5 takes the smallest
                              Schur-complement diagonal of H_d at every step
                              (Babai page, §2.3); that LDL eliminates the last
                              processed column first, so the column eliminated
                              at step t is processed at position n−1−t; equal
                              entries go to the larger column index;
                              n ≤ 16384, else UNSUPPORTED                     */
} gptq_order;

typedef enum {
  GPTQ_DTYPE_F32 = 0,
  GPTQ_DTYPE_BF16 = 1
} gptq_dtype;

/*
 * H += 2·XᵀX.
 *   X  T×n bfloat16, row-major (one row per calibration token), device.
 *   H  n×n float32, row-major, device; read and written (accumulates, so a
 *      calibration set may arrive in several calls).  The caller zeroes H
 *      before the first call.  Both triangles are written (H stays symmetric).
 *   T  may be 0 (no-op).  n ≥ 1.
 *   info  int32[2] on the device, or NULL: a bounded wait inside the kernel
 *      that runs out is reported there as GPTQ_ERR_TIMEOUT (it is not reset
 *      by this call, so several calls may share one info pair).
 * Kernel: for n a multiple of 8 (and X 16-byte aligned) a TMA → tcgen05
 * pipeline (bf16 operands, float32 accumulator in tensor memory, 128×128
 * tiles on or above the diagonal); otherwise a float32 SIMT tile kernel.
 * Source: CHMC page, Schritt 2 ("Hesse-Matrix aus den
 * Kalibrierungsaktivierungen", XᵀX/n); the factor 2 instead of 1/n leaves the
 * codes unchanged because the damping is relative.  Babai page, §2.1: XᵀX is
 * the Gram matrix of the lattice basis.
 * Errors: INVALID_ARG (null pointer, T < 0, n < 1), CUDA; TIMEOUT via info.
 */
gptq_status gptq_hessian_accumulate(const void* X, int64_t T, int64_t n,
                                    float* H, int32_t* info, void* stream);

/* Bytes of device workspace gptq_prepare needs for size n (256-byte aligned). */
size_t gptq_prepare_workspace_bytes(int64_t n);

/*
 * Damp, order and factor.
 *   H      n×n float32 from gptq_hessian_accumulate, device, read only.
 *   damp   relative damping λ ≥ 0 (float64): H_d = H + λ·mean(diag H)·I.  The mean is
 *          taken before the dead-column fix.  Dead columns (H_jj == 0) get
 *          H_jj := 1 (and gptq_quantize zeroes their weights).
 *   order  a gptq_order value.
 *   perm   int32[n], device.  Output (processing position p → original column
 *          perm[p]) unless order == CUSTOM, where it is the input.
 *   U      n×n float32, device, output: upper triangular, UᵀU = (P·H_d·Pᵀ)⁻¹
 *          with P the processing-order permutation; the strict lower triangle
 *          is written as 0.  Computed in float64 and rounded once.
 *   dead   uint8[n], device, output: 1 where H_jj == 0.
 *   info   int32[2], device, output: {status, index}; NOT_PD sets index to
 *          the failing pivot (processing position) + 1; NONFINITE to the
 *          flattened index + 1 of a NaN/Inf entry of H.  With MINPIVOT a pivot
 *          ≤ 0 met while choosing the order is reported the same way.
 *   ws     device workspace of at least gptq_prepare_workspace_bytes(n),
 *          256-byte aligned.
 * Source: CHMC page, Schritt 2 (damping, act-order, "H⁻¹ über die
 * Cholesky-Zerlegung"); Babai page, §2.3 (ordering by the Hessian diagonal,
 * the min-pivot order).
 * Errors: INVALID_ARG (null pointer, n < 1, damp < 0 or not finite, bad
 * order, workspace too small; a CUSTOM perm that is not a permutation is
 * reported through info), CUDA; NOT_PD / NONFINITE through info.
 */
gptq_status gptq_prepare(const float* H, int64_t n, double damp, int order,
                         int32_t* perm, float* U, uint8_t* dead, int32_t* info,
                         void* ws, size_t ws_bytes, void* stream);

/*
 * Peak probe (a measurement aid; the pages have no counterpart): one launch
 * that keeps a single arithmetic pipe busy, for the roofline denominators of
 * the kernels that use it.  The caller times the launch with CUDA events on
 * `stream` and divides *flops by the time.
 *   kind 0  float64 tensor-core products (mma.sync m8n8k4), 4 CTAs of 8 warps
 *           per SM, each warp 8 independent accumulators, `iters` rounds;
 *   kind 1  tcgen05.mma kind::tf32 128×256×8 from shared memory into tensor
 *           memory, one CTA per SM, 4·iters products each;
 *   kind 2  the same with kind::f16 on bf16 operands (K = 16);
 *   kind 3  kind 0 with one CTA of 8 warps per SM.
 *   flops  host, output: the floating-point operations of the launch
 *          (2 per multiply-add).
 *   info   int32[2] on the device: a bounded wait that runs out sets TIMEOUT.
 *   sink   ≥ 8 bytes of device memory (never written in practice; it keeps
 *          the products from being optimised away).
 * Errors: INVALID_ARG (kind outside 0..3, iters < 1, a null pointer), CUDA.
 */
gptq_status gptq_peak_probe(int kind, int64_t iters, double* flops, int32_t* info, void* sink,
                            void* stream);

/*
 * Polls each bounded wait of gptq_prepare's dataflow factorisation makes
 * (one launch whose CTAs wait on each other's tiles through flags in the
 * workspace) before it gives up, reports GPTQ_ERR_TIMEOUT through info,
 * raises the launch's abort flag so that every CTA returns, and leaves U
 * undefined.  0 restores the default, 2^22 polls with a back-off of 64 ns
 * after the first 32 (a few seconds).  Process-wide, read at each
 * gptq_prepare call.  A small limit makes the time-out path run on purpose
 * (tests of failure detection); normal use never needs to set it.
 */
void gptq_set_wait_limit(uint32_t polls);

/*
 * The most worker CTAs (one per SM, beside the one CTA that runs the
 * factorisation's critical chain) a gptq_prepare launch may use; 0 restores
 * the default, every SM but one.  Process-wide, read at each gptq_prepare
 * call.  A caller running several factorisations and sweeps side by side on
 * different streams may leave SMs to the other streams' kernels this way
 * (the factorisation's CTAs stay resident until its last task).  The result
 * does not depend on it.
 */
void gptq_set_factor_workers(int max_ctas);

/*
 * gptq_prepare without a workspace argument: the same operation, arguments
 * and results as gptq_prepare, for callers that cannot hand this library a
 * block of device memory — for example code that runs while another
 * framework owns every allocation on the device, a plugin with no allocator
 * of its own, or a caller that must not call cudaMalloc/cudaFree (which
 * synchronise the device) on a latency-sensitive path.  The pages have no
 * counterpart to this entry point.
 *   The scratch is a fixed array inside the library (about 16 MB for the
 *   limit below), reserved on every GPU that loads the library until the
 *   process exits.  This call allocates nothing: no cudaMalloc, no cudaFree,
 *   no allocating library routine.
 *   n must be at most GPTQ_NOALLOC_MAX_N; larger n returns
 *   GPTQ_ERR_INVALID_ARG with a message (use gptq_prepare instead).
 *   The first call on each device looks up the array's device address
 *   (with that device current); make that first call before any stream
 *   capture.  The address is kept for the life of the process, so a device
 *   reset (cudaDeviceReset) between calls is not supported.
 *   All calls on one device share the array and it keeps the last call's
 *   contents; the call initialises every part it reads.  Calls whose work
 *   overlaps on the GPU (different streams, or different host threads, on
 *   the same device) race on the array: serialise them.
 */
#define GPTQ_NOALLOC_MAX_N 1024
gptq_status gptq_prepare_noalloc(const float* H, int64_t n, double damp, int order,
                                 int32_t* perm, float* U, uint8_t* dead, int32_t* info,
                                 void* stream);

/* Bytes of device workspace gptq_quantize needs (256-byte aligned). */
size_t gptq_quantize_workspace_bytes(int64_t m, int64_t n, int block);

/*
 * Quantize W (m×n) column by column with error compensation.
 *   W        m×n, device, bfloat16 or float32 (w_dtype), row-major; not
 *            modified.  Rows are output channels, columns input channels.
 *   U, perm, dead   from gptq_prepare for this W's Hessian.
 *   bits     2, 3, 4 or 8.  Asymmetric min-max grid with an integer zero
 *            point; the range contains 0; all-zero group → [−1, 1].
 *   group    columns per scale group, along the input channels, counted in
 *            processing order (CHMC page, Schritt 3: GPTQ keeps o·⌈i/gs⌉
 *            scales).  A multiple of 32.
 *   block    lazy-batch width: a multiple of group, at most 128.  The block
 *            changes rounding order only, not the algorithm.
 *   qweight  m × ceil(n·bits/32) uint32, output: per row an LSB-first bit
 *            stream of the codes in ORIGINAL column order (column c in bits
 *            [c·bits, (c+1)·bits) of the row's stream).
 *   scale    m × ceil(n/group) float32, output; zero: same shape, uint8.
 *            Group g covers processing positions [g·group, (g+1)·group).
 *   g_idx    int32[n], output: group of each original column.
 *   loss_row float32[m] or NULL: Σ_j e_j² with e_j = (w_j − q̂_j)/U_jj, the
 *            damped layer loss of the row.
 *   Qdq      m×n float32 or NULL: dequantized weights s·(q − z), original
 *            column order.
 *   info     int32[2], device, output (NONFINITE: flattened index + 1 of the
 *            first NaN/Inf weight found).
 *   ws       device workspace of at least gptq_quantize_workspace_bytes().
 * Per column j (processing order):  q = clamp(rint(w/s) + z, 0, 2^bits − 1),
 *   e = (w − s·(q − z))/U_jj,  w[j+1:] −= e·U[j, j+1:]   (CHMC page, Schritt 2;
 *   scale and zero from the group's current values at its first column.)
 * Errors: INVALID_ARG, UNSUPPORTED (bits, group, block), CUDA; NONFINITE
 * through info.
 */
gptq_status gptq_quantize(const void* W, int w_dtype, int64_t m, int64_t n,
                          const float* U, const int32_t* perm,
                          const uint8_t* dead, int bits, int group, int block,
                          uint32_t* qweight, float* scale, uint8_t* zero,
                          int32_t* g_idx, float* loss_row, float* Qdq,
                          int32_t* info, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * Static groups: as gptq_quantize, except that every group's scale and zero
 * are fixed before the sweep from the ORIGINAL weights (dead columns read 0)
 * of `group` consecutive ORIGINAL columns [g·group, (g+1)·group), with the
 * same min-max quantizer; the sweep then quantizes processing column j with
 * the parameters of group perm[j] / group and recomputes nothing from the
 * current values.  The pages define only the groups met in processing order
 * (CHMC page, Schritt 2 and 3); this is the common variant that lets act-order
 * change the order of the columns but not which columns share a scale.
 *   group    any width ≥ 1 (groups need not align with blocks).
 *   block    a multiple of 32, at most 128.
 *   scale, zero   m × ceil(n/group), group g = original columns as above.
 *   g_idx    int32[n], output: c / group.
 * Workspace: gptq_quantize_workspace_bytes(m, n, block).
 */
gptq_status gptq_quantize_static(const void* W, int w_dtype, int64_t m, int64_t n,
                                 const float* U, const int32_t* perm, const uint8_t* dead,
                                 int bits, int group, int block, uint32_t* qweight,
                                 float* scale, uint8_t* zero, int32_t* g_idx,
                                 float* loss_row, float* Qdq, int32_t* info, void* ws,
                                 size_t ws_bytes, void* stream);

/* ---- CHMC frontend (next to the hot path) -------------------------------
 * "Warum Geometrie Gewichte nicht komprimiert", section "Methodik. Was ist
 * CHMC": every weight matrix W (o × i) is split into a low-rank part W_lr
 * along the activation cone (Schritt 1) and a residual R = W − W_lr quantized
 * by GPTQ with scales along the output channels (Schritt 2); the rank comes
 * from the bit budget (Schritt 3).
 */

/* Output-channel group size of gptq_quantize_rowgroups (the page's gs). */
#define GPTQ_ROWGROUP_SIZE 128
/* Largest rank gptq_chmc_lowrank accepts. */
#define GPTQ_CHMC_MAX_RANK 32

/*
 * Schritt 3, the rank rule (host arithmetic, no device work):
 *   r = floor((bpw_target·o·i − bits·o·i − 16·ceil(o/gs)·i) / (16·(o + i))),
 * clamped to [0, min(o, i)].  Returns 0 for invalid arguments.
 */
int gptq_chmc_rank(int64_t o, int64_t i, int bits, int gs, double bpw_target);

/* Bytes of device workspace gptq_chmc_lowrank needs (256-byte aligned);
 * 0 if r is outside [0, GPTQ_CHMC_MAX_RANK]. */
size_t gptq_chmc_workspace_bytes(int64_t o, int64_t i, int r);

/*
 * Schritt 1: the low-rank part and the residual.
 *   W        o × i, device, float32 or bfloat16 (w_dtype), row-major (rows are
 *            output channels).  Not modified.
 *   H        i × i float32, device: 2·XᵀX over `tokens` calibration rows (the
 *            Hessian of gptq_hessian_accumulate).  Only its diagonal is read:
 *            c_j = H_jj/(2·tokens) + lam·mean_j(H_jj/(2·tokens)), the page's
 *            damped activation energies (lam = 0.05 on the page).
 *   Omega    i × r float32, device, row-major: the randomized SVD's test
 *            matrix (standard normal entries, drawn by the caller).
 *   r        rank, 0..GPTQ_CHMC_MAX_RANK and at most min(o, i); r = 0 copies W
 *            to R (H and Omega may then be NULL).
 *   niter    power iterations (the page uses 5), 0..64.
 *   Q        o × r float32 or NULL, output: an orthonormal basis of the range
 *            found by the randomized subspace iteration on W·diag(√c).
 *   P        r × i float32 or NULL, output: Qᵀ·W, so that W_lr = Q·P
 *            (= (U·S)·Vᵀ·diag(1/√c) of the page: B = Qᵀ·W̃ has exactly r rows,
 *            so its SVD only rotates the factors).
 *   R        o × i float32, output: W − Q·P, computed in float64.
 *   info     int32[2], device, output (INVALID_ARG with the column index if an
 *            activation energy is not positive).
 * Computes in float64 throughout; deterministic.  Errors: INVALID_ARG,
 * UNSUPPORTED (rank, niter), CUDA.
 */
gptq_status gptq_chmc_lowrank(const void* W, int w_dtype, int64_t o, int64_t i,
                              const float* H, int64_t tokens, double lam,
                              const float* Omega, int r, int niter, float* Q, float* P,
                              float* R, int32_t* info, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * Schritt 2: GPTQ with scales along the output channels ("eine gemeinsame
 * Skala pro Gruppe von Ausgabekanälen", ceil(o/gs)·i scales).  As
 * gptq_quantize, except:
 *   gs       rows per scale group; must be GPTQ_ROWGROUP_SIZE.
 *   scale    ceil(m/gs) × n float32, output: scale[g][c] for rows
 *            [g·gs, (g+1)·gs) and ORIGINAL column c; zero: same shape, uint8.
 *            Each column's parameters come from the column's current
 *            (error-updated) values over the group's rows, when the column is
 *            processed (min-max, 0 inside the range, all-zero → [−1, 1]).
 *   block    lazy-batch width: a multiple of 32, at most 128.
 *   (no g_idx: every column has its own scale per row group.)
 * Workspace: gptq_quantize_workspace_bytes(m, n, block).
 */
gptq_status gptq_quantize_rowgroups(const void* W, int w_dtype, int64_t m, int64_t n,
                                    const float* U, const int32_t* perm,
                                    const uint8_t* dead, int bits, int gs, int block,
                                    uint32_t* qweight, float* scale, uint8_t* zero,
                                    float* loss_row, float* Qdq, int32_t* info, void* ws,
                                    size_t ws_bytes, void* stream);

/* ---- SSQR (next to the hot path) ----------------------------------------
 * "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
 * Algorithm" (gist.science summary), §3: scale-adjusted SpQR keeps the
 * weights that overflow the grid (the outliers) in full precision as a sparse
 * part and quantizes the rest (the inliers) with GPTQ; a binary search on the
 * scales meets a target outlier density.  §2.3: clipping those weights would
 * break Satz 5's error bound.
 */

/* Bytes of device workspace gptq_ssqr_quantize needs (256-byte aligned): three
 * working sets of gptq_quantize's (the second and third serve lookahead),
 * the search state and per-set row counts, scales and zero points. */
size_t gptq_ssqr_workspace_bytes(int64_t m, int64_t n, int block);

/*
 * As gptq_quantize (W, U, perm, dead, group, block, qweight, scale, zero,
 * g_idx, loss_row, Qdq, info have the same meaning), except:
 *   bits       2, 3 or 4.
 *   Scales     the min-max step s0 of each group (taken where gptq_quantize
 *              takes it) becomes s = alpha·s0 (float32); the zero point stays
 *              rint(−xmin/s0).  `scale` holds s.
 *   Outliers   a weight whose unclipped code rint(w/s) + z falls outside
 *              [0, 2^bits − 1] keeps its current (error-updated) value: its
 *              error is 0 and nothing propagates from it.  Its code in
 *              qweight is the clipped one; dequantization uses the value.
 *   Search     (all on the device, no host synchronisation):
 *              n_max = floor(target·m·n).  Pass 0 runs at alpha_hi; more than
 *              n_max outliers there ends the search with alpha = alpha_hi.
 *              Otherwise each of up to `iters` passes runs at
 *              mid = float32((lo + hi)/2) of the bracket [alpha_lo, alpha_hi]
 *              and makes mid the new hi when it has at most n_max outliers,
 *              else the new lo; a mid equal to lo or hi ends the search.  A
 *              last pass at hi writes the outputs.  Cost: iters + 2 sweeps of
 *              the layer, one after another.
 *   lookahead  0: one pass per bisection step.  1: each round runs the
 *              midpoint and both quarter points of the step after it side by
 *              side (on `stream` and two streams forked from it, joined before
 *              the call returns) and takes both steps: the same steps and
 *              result, about half the passes in sequence and 1.5 times the
 *              work; worth it when the GPU has SMs to spare beside the call.
 *   target     outlier density, 0..1.  iters 0..64.
 *   alpha_lo, alpha_hi   the bracket, 0 < alpha_lo ≤ alpha_hi ≤ 16.
 *   row_ptr    int64[m + 1], output: CSR row pointers of the outliers
 *              (row_ptr[m] = their number).
 *   col_idx, val  int32 / float32 [nnz_cap], output: ORIGINAL column and
 *              kept value of each outlier, row-major, columns ascending.
 *              Entries beyond nnz_cap are dropped and info reports
 *              GPTQ_ERR_CAPACITY (row_ptr stays complete).  May be NULL when
 *              nnz_cap == 0.
 *   alpha      float32[1], output: the chosen factor.
 *   trace_alpha, trace_count   float32 / int64 [iters + 1] or NULL: the α of
 *              each search pass and its outlier count (−1 for a pass run
 *              after the search had ended).
 *   ws         device workspace of at least gptq_ssqr_workspace_bytes().
 * Errors: INVALID_ARG (null pointer, target, iters, bracket, nnz_cap < 0,
 * workspace), UNSUPPORTED (bits, group, block), CUDA; NONFINITE and CAPACITY
 * through info.
 */
gptq_status gptq_ssqr_quantize(const void* W, int w_dtype, int64_t m, int64_t n,
                               const float* U, const int32_t* perm, const uint8_t* dead,
                               int bits, int group, int block, double target, int iters,
                               float alpha_lo, float alpha_hi, int lookahead, uint32_t* qweight,
                               float* scale, uint8_t* zero, int32_t* g_idx,
                               int64_t* row_ptr, int32_t* col_idx, float* val,
                               int64_t nnz_cap, float* alpha, float* trace_alpha,
                               int64_t* trace_count, float* loss_row, float* Qdq,
                               int32_t* info, void* ws, size_t ws_bytes, void* stream);

/* ---- HPTQ (next to the hot path) ----------------------------------------
 * "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
 * Algorithm", §3: Huffman-encoded PTQ quantizes inliers and outliers on one
 * unbounded integer grid (no clipping, so Satz 5's bound of §2.3 holds) and
 * Huffman-codes the integers to meet a compression budget; §4 names 3.125
 * bits per weight.
 */

/* Symbol window of the code: symbol = q + GPTQ_HPTQ_SYMBOL_OFFSET, in
 * [0, GPTQ_HPTQ_SYMBOLS).  Codes outside it are reported as UNSUPPORTED. */
#define GPTQ_HPTQ_SYMBOLS 4096
#define GPTQ_HPTQ_SYMBOL_OFFSET 2048

/* Bytes of device workspace gptq_hptq_quantize needs (256-byte aligned): as
 * gptq_ssqr_workspace_bytes, plus per set m×n int16 coordinates and a
 * histogram, and the code table. */
size_t gptq_hptq_workspace_bytes(int64_t m, int64_t n, int block);

/*
 * As gptq_quantize (W, U, perm, dead, group, block, scale, g_idx, loss_row,
 * Qdq, info have the same meaning), except:
 *   bits       nominal bits of the min-max step s0 = range/(2^bits − 1),
 *              2, 3, 4 or 8.
 *   Grid       the lattice s·Z of each group, s = alpha·s0 (float32): a
 *              weight's integer is q = rint(w/s), any integer (no clamp and
 *              no zero point, which an unbounded grid does not need); its
 *              error is w − s·q (|·| ≤ s/2).  Dequantized: s·q.
 *   Code       one Huffman code per call over the integers q; its cost (the
 *              payload bits Σ count(q)·len(q)) drives the search.  A single
 *              used symbol gets length 1.  Code words are canonical: in order
 *              of (length, symbol) each is the previous plus one, shifted
 *              left when the length grows.
 *   Search     as gptq_ssqr_quantize's, with "admissible" meaning coded bits
 *              ≤ floor(budget·m·n): alpha_hi (the coarsest grid) first, then up
 *              to `iters` bisection steps; a last pass at the chosen alpha is
 *              encoded.  Cost: iters + 2 sweeps of the layer.
 *   lookahead  as gptq_ssqr_quantize's.
 *   budget     payload bits per weight, (0, 64].  iters 0..64.
 *   alpha_lo, alpha_hi   0 < alpha_lo ≤ alpha_hi ≤ 256.
 *   codes      m×n int16 or NULL, output: q in ORIGINAL column order.
 *   code_len   uint8[GPTQ_HPTQ_SYMBOLS], output: length per symbol (0: unused).
 *   code_word  uint64[GPTQ_HPTQ_SYMBOLS] or NULL, output: canonical code
 *              words, right-aligned.
 *   row_off    int64[m + 1], output: bit offset of each row in the stream
 *              (row_off[m] = the coded bits).
 *   stream_words  uint32[stream_cap], output: rows one after another in
 *              original column order, each code most significant bit first,
 *              words filled from their most significant bit.  Bits past
 *              stream_cap·32 are dropped and info reports CAPACITY.  May be
 *              NULL when stream_cap == 0.
 *   alpha      float32[1], output: the chosen factor.
 *   trace_alpha, trace_bits   float32 / int64 [iters + 1] or NULL: the alpha and
 *              coded bits of each search pass (−1 after the search ended).
 *   ws         device workspace of at least gptq_hptq_workspace_bytes().
 * Errors: INVALID_ARG (null pointer, budget, iters, bracket, stream_cap < 0,
 * workspace), UNSUPPORTED (bits, group, block), CUDA; NONFINITE, CAPACITY and
 * UNSUPPORTED (a code outside the symbol window, a code longer than 64 bits)
 * through info.
 */
gptq_status gptq_hptq_quantize(const void* W, int w_dtype, int64_t m, int64_t n,
                               const float* U, const int32_t* perm, const uint8_t* dead,
                               int bits, int group, int block, double budget, int iters,
                               float alpha_lo, float alpha_hi, int lookahead, int16_t* codes,
                               float* scale,
                               int32_t* g_idx, uint8_t* code_len,
                               uint64_t* code_word, int64_t* row_off, uint32_t* stream_words,
                               int64_t stream_cap, float* alpha, float* trace_alpha,
                               int64_t* trace_bits, float* loss_row, float* Qdq,
                               int32_t* info, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronize `stream`, read info[0..1] and return info[0] (a gptq_status).
 * If `index` is not NULL it receives info[1].  `info` is a device pointer.
 */
gptq_status gptq_check(const int32_t* info, int32_t* index, void* stream);

/* Message of the last failure on the calling thread ("" if none). */
const char* gptq_last_error(void);

/* Name of a status code. */
const char* gptq_status_string(int status);

/* ---- instrumentation (host-side; no device memory) ---------------------- */

/* Number of kernels this library has launched in this process. */
uint64_t gptq_launch_count(void);

/* Number of kernel kinds, and the name of kind k (e.g. "hessian_tc"). */
int gptq_kernel_kinds(void);
const char* gptq_kernel_name(int kind);

/*
 * Kernel timing: after gptq_profile_start(capacity) every launch (up to
 * `capacity`) is bracketed by a pair of CUDA events recorded on the stream it
 * is launched on.  gptq_profile_stop() waits for those events and sums the
 * elapsed times per kernel kind; gptq_profile_get() returns the sum (ms) and
 * the number of timed launches of kind k.  Events are host objects; no device
 * memory is allocated.
 */
gptq_status gptq_profile_start(int capacity);
gptq_status gptq_profile_stop(void);
gptq_status gptq_profile_get(int kind, double* total_ms, int64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
