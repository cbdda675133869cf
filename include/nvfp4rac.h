/*
 * nvfp4rac.h -- C ABI of the NVFP4 W4A4 + Residual Activation Compensation
 * (RAC) rollout path and its trainer-side weight fake-quantization companion,
 * for NVIDIA B200 (sm_100a).
 *
 * What the operations compute comes from the QUADS pages:
 *   - "Technische Samenvatting: QUADS" (gist.science), section 2.2 B
 *     "Residual Activation Compensatie (Rollout-zijde)": high-residual
 *     channels get a second-pass quantization, a residual correction term is
 *     added to the quantized output, a binary channel mask keeps the top k%
 *     of channels by residual magnitude, native W4A4 GEMM throughput is kept
 *     for most of the work;
 *   - the same page, section 2.1 (weights) and 2.2 A "Asymmetrische
 *     Quantization-Aware Training": trainer and rollout share one QDQ path
 *     for the weights, the trainer fake-quantizes weights to NVFP4 (W4A16);
 *   - the same page, section 1 "Probleemstelling": NVFP4 is Blackwell's
 *     native W4A4 format on the coarse E2M1 grid (8 levels per sign).
 * The pages fix no formula.  The adopted reading is
 *     Y = DQ(Q(X)) DQ(Q(W))^T + DQ(Q(dX_sel)) DQ(Q(W_sel))^T
 * with dX = X - DQ(Q(X)), 16-element blocks along K with E4M3 block scales
 * and one fp32 tensor scale s_t = RN(amax / 2688) per tensor,
 *     sb = E4M3(RN(amax_b / RN(6 s_t))),  s_dec = RN(E4M3dec(sb) s_t),
 *     code = E2M1(RN(x / s_dec)),         DQ = RN(RN(E2M1dec E4M3dec) s_t),
 * channel scores score_j = sum_i |dX_ij| in fp64 (rows in chunks of 128
 * from row 0, each chunk summed row by row in row order, the chunk sums
 * added in chunk order; every addition rounded to nearest even),
 * n_sel = floor(k K / 100), ties to the lower channel, sel ascending, and
 * dX_sel / W_sel re-quantized with their own tensor scales.
 *
 * Conventions shared by every call
 *   - Memory: every pointer is a DEVICE pointer unless marked (host).  The
 *     caller allocates and owns every buffer, including the workspace; the
 *     library allocates nothing and keeps no pointer after a call returns.
 *   - bf16 tensors are passed as their bit patterns (uint16_t), row-major
 *     with a leading dimension in elements.
 *   - Streams: `stream` is a cudaStream_t passed as void*.  Every call only
 *     enqueues work on it and returns; none synchronizes the device.
 *   - Errors: argument errors are returned before anything is enqueued and
 *     nothing is written.  A CUDA launch error gives NVFP4_ERR_CUDA.  Errors
 *     found on the device (a bounded wait that gave up) are recorded in a
 *     device error word and reported by nvfp4_stream_status().
 *   - Alignment: every pointer 16-byte aligned; ldx, ldw a multiple of 8.
 *   - Shapes: K (in-features) a multiple of 64; M, N >= 1; N a multiple of
 *     16 for the GEMMs; inputs finite.
 *
 * NVFP4 tensor layout (nvfp4_tensor)
 *   codes:  rows x cols/2 bytes, row-major, element 2j in the low nibble of
 *           byte j and 2j+1 in the high nibble; E2M1 code = sign<<3 | magnitude.
 *   scales: one E4M3 byte per 16-element block.
 *           scale_layout 0 (canonical): [rows][cols/16], row-major.
 *           scale_layout 1 (MMA-tiled, required by the GEMMs): rows padded to
 *           128 and blocks to multiples of 4; the scale of (row r, block c)
 *           sits at byte ((r/128) * (cols_p/64) + c/4) * 512
 *                          + (r%32) * 16 + ((r%128)/32) * 4 + c%4,
 *           cols_p = cols rounded up to 64; padding bytes are written as 0.
 *           nvfp4_scale_bytes() gives the size of either layout.
 *   tensor_scale: device fp32 decode scale s_t (one per matrix).
 */
#ifndef NVFP4RAC_H_
#define NVFP4RAC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,      /* null pointer, bad enum, k outside [0,100] */
  NVFP4_ERR_MISALIGNED = 2,       /* pointer not 16-byte aligned or ld % 8 != 0 */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 3,/* K % 64, N % 16, sizes out of range */
  NVFP4_ERR_WORKSPACE = 4,        /* workspace smaller than nvfp4_workspace_size() */
  NVFP4_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed */
  NVFP4_ERR_TIMEOUT = 6,          /* a device-side bounded wait gave up */
  NVFP4_ERR_DEVICE = 7,           /* current device is not sm_100 */
  NVFP4_ERR_BOUNDS = 8            /* an index check of the checked build failed */
} nvfp4_status;

typedef struct {
  uint8_t* codes;         /* device, rows x cols/2 */
  uint8_t* scales;        /* device, see scale_layout */
  float* tensor_scale;    /* device, fp32 s_t (E of them for a stacked weight) */
  int64_t rows, cols;     /* logical shape (cols % 64 == 0) */
  int32_t scale_layout;   /* 0 canonical, 1 MMA-tiled */
} nvfp4_tensor;

/* Workspace ops for nvfp4_workspace_size(). */
enum {
  NVFP4_OP_QUANTIZE = 0,  /* nvfp4_quantize(M, K) */
  NVFP4_OP_RAC_SELECT = 1,/* rac_select(M, K) */
  NVFP4_OP_GEMM = 2,      /* w4a4_rac_gemm(N, K): N x K worst-case W_sel */
  NVFP4_OP_MOE = 3,       /* moe_grouped_w4a4_rac_gemm(T = M, N, K, E) */
  NVFP4_OP_WEIGHT_QDQ = 4 /* weight_qdq(batch = E) */
};

/* Bytes of the scale buffer of a rows x cols NVFP4 tensor in `layout`. */
size_t nvfp4_scale_bytes(int64_t rows, int64_t cols, int32_t layout);

/* Bytes of workspace a call needs (0 for none).  op: NVFP4_OP_*. */
size_t nvfp4_workspace_size(int32_t op, int64_t M, int64_t N, int64_t K, int32_t E);

/*
 * nvfp4_quantize -- Q(X) of bf16 activations plus the RAC channel statistics.
 * Pages: QUADS technical summary section 1 (E2M1 grid) and 2.2 B (residual).
 *   x [M, K] bf16, row stride ldx.  amax_or_null: device fp32 max|X|
 *   supplied by the caller (skips the amax pass), or NULL.
 *   qx: rows = M, cols = K, codes/scales/tensor_scale written (either layout).
 *   score_or_null: fp64 [K] channel scores sum_i |dX_ij| in the fixed order;
 *   res_colamax_or_null: fp32 [K] max_i |dX_ij|.  Both, neither, or the
 *   column maxima alone (a step that reuses an earlier channel mask needs
 *   them for the residual tensor scale but no scores); scores without the
 *   column maxima are refused.
 *   dX = RN(x - DQ(Q(x))) is formed in registers and never written.
 *   ws: nvfp4_workspace_size(NVFP4_OP_QUANTIZE, M, 0, K, 1) bytes.
 */
nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                            const float* amax_or_null, nvfp4_tensor* qx,
                            double* score_or_null, float* res_colamax_or_null,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * rac_select -- top-k% channel mask and second-pass quantization of the
 * gathered residual.  Pages: QUADS technical summary 2.2 B (binary channel
 * mask, top k%, second-pass quantization of the high-residual channels).
 *   score / res_colamax: outputs of nvfp4_quantize for the same x and qx.
 *   k_percent in [0, 100]; n_sel = floor(k K / 100) is computed on the host
 *   and returned in *n_sel_out (host pointer).
 *   mask: u8 [K] (1 = selected).  sel: i32 [n_sel], ascending channel index.
 *   q_res: rows = M, cols = nvfp4_rac_width(n_sel) (n_sel rounded up to 64),
 *   zero padded; its tensor scale is RN(max_{j in sel} res_colamax_j / 2688).
 *   q_res may be NULL when n_sel == 0.
 */
nvfp4_status rac_select(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                        const nvfp4_tensor* qx, const double* score, const float* res_colamax,
                        float k_percent, uint8_t* mask, int32_t* sel, int64_t* n_sel_out,
                        nvfp4_tensor* q_res, void* ws, size_t ws_bytes, void* stream);

/*
 * rac_select_channels -- the first half of rac_select: the top-k% channel
 * mask, sel and the residual tensor scale, without the residual gather, so
 * that the gathers of the residual and of the weight (rac_residual_quant,
 * rac_weight_quant) can run concurrently on two streams.  Pages: 2.2 B
 * (binary channel mask, top k%).
 *   score / res_colamax [K]: outputs of nvfp4_quantize.  mask u8 [K];
 *   sel i32 [n_sel] ascending (may be NULL when n_sel == 0); *n_sel_out
 *   (host) = floor(k K / 100).  res_tensor_scale (device fp32, required):
 *   RN(max_{j in sel} res_colamax_j / 2688), the residual's tensor scale
 *   (0 when n_sel == 0); pass q_res->tensor_scale to rac_residual_quant.
 */
nvfp4_status rac_select_channels(const double* score, const float* res_colamax, int64_t K, float k_percent,
                                 uint8_t* mask, int32_t* sel, int64_t* n_sel_out, float* res_tensor_scale,
                                 void* stream);

/*
 * rac_sel_tensor_scale -- tensor_scale (device fp32) = RN(max_{j in sel}
 * colamax_j / 2688): the tensor scale of a second-pass operand over a given
 * channel selection, e.g. the residual's for a step that reuses the channel
 * mask of an earlier step (sel kept, colamax = this step's residual column
 * maxima from nvfp4_quantize).  Pages: 2.2 B (second-pass quantization of
 * the selected channels); keeping the mask across steps is a variant the
 * pages do not describe.  sel: n_sel (>= 1) channel indices in [0, K).
 */
nvfp4_status rac_sel_tensor_scale(const float* colamax, int64_t K, const int32_t* sel, int64_t n_sel,
                                  float* tensor_scale, void* stream);

/*
 * rac_residual_quant -- the second half of rac_select: Q(dX_sel), the
 * second-pass quantization of the residual's selected channels, with the
 * tensor scale rac_select_channels wrote into q_res->tensor_scale (read on
 * the device, so it must be ordered after that call).  Pages: 2.2 B
 * (second-pass quantization of the high-residual channels).
 *   x, qx as for rac_select; sel [n_sel], n_sel >= 1; q_res: rows = M,
 *   cols = nvfp4_rac_width(n_sel), either scale layout.
 */
nvfp4_status rac_residual_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* qx,
                                const int32_t* sel, int64_t n_sel, nvfp4_tensor* q_res, void* stream);

/*
 * rac_quantize_select -- nvfp4_quantize (with scores and residual column
 * maxima) and rac_select_channels in one pass over X: the CTA that finishes
 * the last column strip of the quantize pass runs the top-k% selection on the
 * finished scores, so mask, sel and the residual tensor scale come out of the
 * same launch (plus the amax pass unless amax_or_null is given).  Pages:
 * 2.2 B (residual magnitude, binary channel mask of the top k%; the pages'
 * implementation fuses its kernels to keep the overhead low).  Arguments as
 * for the two calls; the outputs are identical to theirs.
 *   ws: nvfp4_workspace_size(NVFP4_OP_QUANTIZE, M, 0, K, 1) bytes.
 */
nvfp4_status rac_quantize_select(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                 const float* amax_or_null, nvfp4_tensor* qx, double* score,
                                 float* res_colamax, float k_percent, uint8_t* mask, int32_t* sel,
                                 int64_t* n_sel_out, float* res_tensor_scale, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * rac_second_pass -- both second-pass quantizations of a RAC linear in one
 * call: Q(dX_sel) exactly as rac_residual_quant (q_res->tensor_scale must
 * hold the residual tensor scale already) and Q(W_sel) exactly as
 * rac_weight_quant from bf16 w [N, K] (stride ldw), or, with w == NULL, as
 * rac_weight_quant_fp4 from qw (w_colamax then nvfp4_dq_colamax(qw, 1)).
 * One kernel launch runs both when the weight side uses the tile gather
 * (weights of up to about 9000 rows at K = 4096), two otherwise.  Pages: 2.2 B
 * (second-pass quantization of the selected channels).
 *   q_res: rows = M, cols = nvfp4_rac_width(n_sel); q_wsel: rows = N, same
 *   cols, scale_layout 1 for the GEMM.
 */
nvfp4_status rac_second_pass(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* qx,
                             const int32_t* sel, int64_t n_sel, nvfp4_tensor* q_res, const uint16_t* w,
                             int64_t N, int64_t ldw, const nvfp4_tensor* qw, const float* w_colamax,
                             nvfp4_tensor* q_wsel, void* stream);

/* n_sel for k_percent of K channels (exact floor), and the padded width of
 * the gathered residual / weight operands (n_sel rounded up to 64). */
int64_t nvfp4_rac_nsel(float k_percent, int64_t K);
int64_t nvfp4_rac_width(int64_t n_sel);

/*
 * rac_weight_quant -- second-pass quantization of the selected weight
 * columns W_sel = W[:, sel] from bf16 W, with tensor scale
 * RN(max_{j in sel} w_colamax_j / 2688).  Pages: 2.2 B (second pass on the
 * selected channels).  q_wsel: rows = N, cols = nvfp4_rac_width(n_sel),
 * scale_layout 1 for the GEMM.
 */
nvfp4_status rac_weight_quant(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                              const int32_t* sel, int64_t n_sel, const float* w_colamax,
                              nvfp4_tensor* q_wsel, void* stream);

/*
 * nvfp4_dq_colamax -- colamax [batch, cols] fp32, the column maxima
 * max_n |DQ(Q(W))_nj| of `batch` stacked NVFP4 matrices of q->rows / batch
 * rows each (tensor_scale[batch]).  The statistic rac_weight_quant_fp4 and
 * the w == NULL forms below take as their column maxima; it changes only
 * when the weights do.  Either scale layout.  colamax is overwritten.
 */
nvfp4_status nvfp4_dq_colamax(const nvfp4_tensor* q, int32_t batch, float* colamax, void* stream);

/*
 * rac_weight_quant_fp4 -- the second-pass quantization of the selected
 * weight columns taken from the NVFP4 weights alone, for rollout engines that
 * hold Q(W) but not the bf16 W: W_sel = DQ(Q(W))[:, sel] (exact fp32
 * values), re-quantized with tensor scale RN(max_{j in sel} dq_colamax_j /
 * 2688).  Pages: 2.2 B (second-pass quantization of the selected channels;
 * the pages do not say where the weight values come from) and 2.1 (rollout
 * and trainer share the weight QDQ path).  This is a variant beyond the
 * plainest reading: Y differs from the bf16-sourced form by the weight's
 * own quantization error in the correction term.
 *   qw: the single weight's Q(W) (rows = N, cols = K, either scale layout);
 *   dq_colamax: nvfp4_dq_colamax(qw, 1); q_wsel as for rac_weight_quant.
 */
nvfp4_status rac_weight_quant_fp4(const nvfp4_tensor* qw, const int32_t* sel, int64_t n_sel,
                                  const float* dq_colamax, nvfp4_tensor* q_wsel, void* stream);

/*
 * w4a4_rac_gemm -- Y = s_tX s_tW (A B^T) + s_tR s_tWs (R B_sel^T), one
 * block-scaled FP4 tensor-core GEMM over the K-concatenated operand
 * [Q(X) | Q(dX_sel)] x [Q(W) | Q(W_sel)] with two accumulators.
 * Pages: 2.2 B (correction added to the quantized output, W4A4 throughput
 * kept for the bulk), section 1 (native W4A4 GEMM).
 *   qx, qw: scale_layout 1; qx.cols == qw.cols == K; qw.rows == N.
 *   q_res_or_null / sel / n_sel: from rac_select; n_sel == 0 (or NULL q_res)
 *   gives plain W4A4.  w (bf16 [N, K], stride ldw) and w_colamax (fp32 [K])
 *   are used to quantize W_sel into the workspace when n_sel > 0.  With
 *   w == NULL, W_sel is taken from qw instead (rac_weight_quant_fp4) and
 *   w_colamax must be nvfp4_dq_colamax(qw, 1).
 *   y: [M, N] fp32 (y_dtype 0) or bf16 (y_dtype 1, RN of the fp32 value),
 *   row stride ldy elements.  ws: NVFP4_OP_GEMM bytes for (N, K).
 */
nvfp4_status w4a4_rac_gemm(const nvfp4_tensor* qx, const nvfp4_tensor* q_res_or_null,
                           const int32_t* sel, int64_t n_sel,
                           const uint16_t* w, int64_t N, int64_t ldw, const nvfp4_tensor* qw,
                           const float* w_colamax, void* y, int32_t y_dtype, int64_t ldy,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * w4a4_gemm_quantized -- the GEMM alone, with every operand already
 * quantized (scale_layout 1): Y = s_tA s_tB A B^T [+ s_tR s_tWs R Ws^T].
 * q_res_or_null and q_wsel_or_null are both given (same cols) or both NULL.
 * Each product of two tensor scales is applied as m 2^e (no fp32 underflow
 * of s_tA s_tB while Y is representable).  A tensor scale of 0 must come
 * with all-zero codes, as every quantizer of this library writes them (an
 * all-zero X or W has an all-zero residual and W_sel too, and Y = 0).
 */
nvfp4_status w4a4_gemm_quantized(const nvfp4_tensor* qa, const nvfp4_tensor* qb,
                                 const nvfp4_tensor* q_res_or_null,
                                 const nvfp4_tensor* q_wsel_or_null,
                                 void* y, int32_t y_dtype, int64_t ldy, void* stream);

/*
 * moe_grouped_w4a4_rac_gemm -- the RAC linear of every expert of an MoE
 * layer in one call: each expert is its own linear with its own amax, tensor
 * scales, scores, mask and residual scale.  Pages: section 4 (25B MoE with
 * 2.8B active parameters) and 2.2 B.
 *   x_perm [T, K] bf16: rows grouped by expert, expert e owning rows
 *   offsets_dev[e] .. offsets_dev[e+1] (device int64 [E+1], read on the
 *   device only; offsets_dev[0] == 0, offsets_dev[E] == T, non-decreasing).
 *   w [E, N, K] bf16 (row stride K), qw: the stacked Q(W) from weight_qdq
 *   with batch E (rows = E*N, cols = K, scale_layout 1, tensor_scale[E]),
 *   w_colamax [E, K].  w == NULL takes every W_sel from qw instead (as
 *   rac_weight_quant_fp4 does per expert) and then w_colamax must be
 *   nvfp4_dq_colamax(qw, E).
 *   y_perm [T, N] (dtype y_dtype), masks_or_null u8 [E, K].
 *   An empty expert writes no rows; its mask is the first n_sel channels.
 *   ws: nvfp4_workspace_size(NVFP4_OP_MOE, T, N, K, E) bytes.
 */
nvfp4_status moe_grouped_w4a4_rac_gemm(const uint16_t* x_perm, int64_t T, int64_t K,
                                       const int64_t* offsets_dev, int32_t E,
                                       const uint16_t* w, int64_t N, const nvfp4_tensor* qw,
                                       const float* w_colamax, float k_percent,
                                       void* y_perm, int32_t y_dtype, uint8_t* masks_or_null,
                                       void* ws, size_t ws_bytes, void* stream);

/*
 * weight_qdq -- trainer-side W4A16 fake quantization of `batch` stacked bf16
 * weights [batch, N, K]: W' = bf16_RNE(DQ(Q(W))) with one tensor scale per
 * matrix.  Pages: 2.1 (shared QDQ path removes the weight mismatch) and 2.2 A
 * (weights fake-quantized to NVFP4, activations stay BF16).
 *   w_out may alias w.  qw_or_null: also write Q(W) (rows = batch*N, cols = K,
 *   tensor_scale[batch]) for the rollout GEMM.  colamax_or_null: fp32
 *   [batch, K] max_n |W_nk|, used by rac_weight_quant.
 *   ws: nvfp4_workspace_size(NVFP4_OP_WEIGHT_QDQ, 0, N, K, batch) bytes.
 */
nvfp4_status weight_qdq(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t batch,
                        uint16_t* w_out, nvfp4_tensor* qw_or_null, float* colamax_or_null,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * nvfp4_quantize_static_ws -- nvfp4_quantize with the same arguments minus
 * the workspace, for callers that cannot allocate device memory (plugin hooks
 * whose interface passes only inputs and outputs, processes whose device
 * memory is entirely reserved by another runtime's allocator).  The pages
 * have no counterpart: this is a property of the library, not of the method.
 *   Scratch lives in one file-scope device array of 4 MiB that every GPU
 *   loading the library keeps until the process exits; shapes whose scratch
 *   exceeds it are refused with NVFP4_ERR_WORKSPACE before anything is
 *   queued.  The scratch is nvfp4_workspace_size(NVFP4_OP_QUANTIZE, M, 0, K,
 *   1) minus that function's 256-byte alignment allowance (the array itself
 *   is 256-byte aligned); with scores it is about 12 bytes per element of
 *   ceil(M / 128) * 128 x K, so M * K up to about 44.7 million elements fit.
 *   The call allocates nothing and calls no allocating routine; on a device
 *   that is not sm_100 it returns NVFP4_ERR_DEVICE before touching it.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress with that device current); make that first call
 *   before any stream capture.
 *   All calls share the one array: calls whose work overlaps on the GPU
 *   (different streams, no ordering between them) race on it and give wrong
 *   results.  Calls ordered on one stream are safe; the words that must
 *   start at zero are cleared on the stream by every call.
 */
nvfp4_status nvfp4_quantize_static_ws(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                      const float* amax_or_null, nvfp4_tensor* qx,
                                      double* score_or_null, float* res_colamax_or_null,
                                      void* stream);

/*
 * The FP8 comparator: MXFP8 operands and a W8A8 tensor-core GEMM, so that the
 * NVFP4 path can be timed beside FP8 on the same shapes.  Pages: QUADS
 * technical summary section 1 "Probleemstelling" (NVFP4 has about twice the
 * GEMM throughput of FP8) and section 4 (about 16% faster rollout than FP8);
 * the pages do not name the FP8 scheme.  The adopted one is the block-scaled
 * FP8 that sm_100 tensor cores run natively, OCP MXFP8: E4M3 elements and
 * one UE8M0 scale 2^E per 32 consecutive elements along K, with
 * E = floor(log2 max|x_b|) - 8 clamped to [-127, 127] (-127 for an all-zero
 * block) and code = E4M3(x / 2^E), nearest, ties to the even code,
 * saturating at 448, the sign bit of x kept (so -0 stays -0).
 */
typedef struct {
  uint8_t* codes;         /* device, rows x cols E4M3 bytes, row-major */
  uint8_t* scales;        /* device, UE8M0 (E + 127) per 32-element block */
  int64_t rows, cols;
  int32_t scale_layout;   /* 0 canonical [rows][cols/32]; 1 MMA-tiled: rows
                             padded to 128, the scale of (row r, block c) at
                             ((r/128) * (cols/128) + c/4) * 512 + (r%32) * 16
                             + ((r%128)/32) * 4 + c%4, padding written as 0 */
} mxfp8_tensor;

/* Bytes of the scale buffer of a rows x cols MXFP8 tensor in `layout`. */
size_t mxfp8_scale_bytes(int64_t rows, int64_t cols, int32_t layout);

/* mxfp8_quantize -- MXFP8 of bf16 x [M, K] (row stride ldx), K % 256 == 0;
 * q: rows = M, cols = K, either scale layout.  Needs no workspace. */
nvfp4_status mxfp8_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, mxfp8_tensor* q,
                            void* stream);

/* w8a8_gemm_quantized -- Y = A B^T with A [M, K] and B [N, K] MXFP8
 * (scale_layout 1), K % 128 == 0, N % 16 == 0: a block-scaled E4M3 tensor-core
 * GEMM (tcgen05 kind::mxf8f6f4) with fp32 accumulation; y fp32 (y_dtype 0)
 * or bf16 (1, RN of the fp32 value), row stride ldy. */
nvfp4_status w8a8_gemm_quantized(const mxfp8_tensor* qa, const mxfp8_tensor* qb, void* y, int32_t y_dtype,
                                 int64_t ldy, void* stream);

/*
 * Element converters used by the kernels, exposed for checking them:
 * nvfp4_encode_e2m1 writes one E2M1 code (0..15) per fp32 input,
 * nvfp4_encode_e4m3 one E4M3 code per fp32 input >= 0 (RN, saturating).
 */
nvfp4_status nvfp4_encode_e2m1(const float* in, uint8_t* out, int64_t n, void* stream);
nvfp4_status nvfp4_encode_e4m3(const float* in, uint8_t* out, int64_t n, void* stream);

/* Synchronize `stream`, then report (and clear) the device error word:
 * NVFP4_ERR_TIMEOUT if a bounded wait gave up since the last query, and in
 * the checked build NVFP4_ERR_BOUNDS if an index check failed (its source
 * line is printed to stderr). */
nvfp4_status nvfp4_stream_status(void* stream);

/* Test hook for the bounded waits: launch one CTA that waits on an mbarrier
 * nothing arrives at, giving up after about timeout_ms milliseconds (capped
 * at 2000) and recording NVFP4_ERR_TIMEOUT in the device error word. */
nvfp4_status nvfp4_check_bounded_wait(int32_t timeout_ms, void* stream);

/* Build flags: bit 0 set in the checked build (libnvfp4rac_checked.so,
 * compiled with NVFP4_CHECKS): every global-memory store and the gathered
 * loads of the kernels test their index against the shapes of the call; a
 * failing test skips the access, records the source line and makes
 * nvfp4_stream_status return NVFP4_ERR_BOUNDS.  Nothing traps. */
int32_t nvfp4_build_flags(void);

const char* nvfp4_status_string(nvfp4_status s);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4RAC_H_ */
