// Host-side launchers of the NVFP4 W4A4 + RAC kernels.  Internal to the
// library: the C ABI in api.cu validates arguments and calls these.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <utility>

#include "common.cuh"

namespace nvfp4 {

// Index-check flags of each translation unit's kernels (checked build; 0
// otherwise), read and reset; *line gets the largest failing source line.
unsigned bounds_flags_quant(unsigned* line);
unsigned bounds_flags_select(unsigned* line);
unsigned bounds_flags_gemm(unsigned* line);

// The current device is an sm_100 GPU: 0 yes, 1 another architecture, 2 the
// query failed (cached per device; defined with the C ABI).
int device_check();

// cuTensorMapEncodeTiled through the runtime's driver entry point (null if
// the driver does not provide it) and the current device's SM count.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
int sm_count();

// Kernel attributes (the dynamic shared-memory opt-in) belong to a device:
// set_max_smem raises `kernel`'s limit to `bytes` once on each device the
// library runs on (the flags of one kernel live in `done`, indexed by device).
constexpr int kMaxAttrDevices = 64;
template <typename... KArgs>
cudaError_t set_max_smem(void (*kernel)(KArgs...), int bytes, bool (&done)[kMaxAttrDevices]) {
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return ge;
  if (dev >= 0 && dev < kMaxAttrDevices && done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxAttrDevices) done[dev] = true;
  return e;
}

// Programmatic dependent launch is on unless NVFP4_NO_PDL=1.
inline bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("NVFP4_NO_PDL");
    v = (e != nullptr && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}

// Launch `kernel` on stream s allowing programmatic dependent launch: its
// CTAs may be scheduled while the previous kernel of the stream still runs
// (every kernel launched this way calls pdl_wait() before touching global
// memory).  Extra launch attributes (a cluster shape) can be passed in.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     const cudaLaunchAttribute* extra, int n_extra, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[4];
  int n = 0;
  for (int i = 0; i < n_extra && n < 3; ++i) attr[n++] = extra[i];
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(n);
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Upper bound of the number of 128-row tiles of `g` (exact for dense).
inline int64_t max_tiles(const RowGroups& g, int64_t rows) {
  return g.off ? (rows + kTileRows - 1) / kTileRows + g.E : (g.M + kTileRows - 1) / kTileRows;
}

// amax_bits[e] |= max |x| over group e (as fp32 bits); amax_bits zeroed by caller.
// With batch > 1, blockIdx.z walks `batch` dense matrices mat_stride elements
// apart and writes amax_bits[b].
cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                        const RowGroups& g, unsigned* amax_bits, cudaStream_t s,
                        int32_t batch = 1, int64_t mat_stride = 0);

// MoE only: tile_start[e] = sum_{e' < e} ceil(m_e' / 128), e = 0..E, and
// (right after it, tile_start[E + 1 + e]) the prefix of ceil(tiles_e / 2),
// the 256-row tiles of the CTA-pair GEMM.  tile_start holds 2 (E + 1) ints.
cudaError_t launch_group_tiles(const int64_t* off, int32_t E, int32_t* tile_start, cudaStream_t s);

// Q(X) plus score partials.  amax: fp32 per group.  codes [codes_rows, K/2]
// on padded rows; scales in `layout`; tensor_scale[e] written for non-empty
// groups; part_sum / part_max [tiles, K] (may be null).  With strip_count
// (E x K/64 counters, zero on entry and left zero) the last CTA of every
// column strip of a group also writes score[e, :] and colamax[e, :].
// Dense activations without a caller amax: per-CTA partial maxima (see
// amax_partial_kernel); n_parts from amax_parts_count.  zero_ptr[0 .. n_zero)
// is cleared on the way (counters that must start at zero).
int amax_parts_count(int64_t rows, int64_t K);
cudaError_t launch_amax_partial(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, int32_t batch,
                                int64_t mat_stride, unsigned* parts, int n_parts, unsigned* zero_ptr,
                                int n_zero, cudaStream_t s);

// The top-k% selection fused into the quantize pass (dense, with scores and
// strip counters): mask [K], sel [n_sel], residual tensor scale s_t; the
// counter strips_done must be zero on entry and is left zero.
struct FusedSelect {
  int64_t n_sel;
  uint8_t* mask;
  int32_t* sel;
  float* s_t;
  unsigned* strips_done;
};

// amax: fp32 per group, or (n_parts > 0) the max of amax_parts[0 .. n_parts).
cudaError_t launch_quant_score(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                               const RowGroups& g, const float* amax, const unsigned* amax_parts,
                               int n_parts, int64_t codes_rows,
                               uint8_t* codes, uint8_t* scales, int layout, float* tensor_scale,
                               double* part_sum, float* part_max, unsigned* strip_count,
                               double* score, float* colamax, cudaStream_t s,
                               const FusedSelect* fused = nullptr);

// score[e, j] = sum over the group's tiles of part_sum in tile order;
// colamax[e, j] = max of part_max.  For empty groups (MoE) also writes
// tensor_scale[e] = 0 and zero scores.
cudaError_t launch_score_reduce(const double* part_sum, const float* part_max, int64_t K,
                                const RowGroups& g, int64_t tiles, double* score, float* colamax,
                                float* tensor_scale_empty, cudaStream_t s);

// Per group: top-n_sel mask, ascending sel, s_tR = RN(max_sel colamax / 2688).
cudaError_t launch_topk(const double* score, const float* colamax, int64_t K, int32_t E,
                        int64_t n_sel, uint8_t* mask, int32_t* sel, float* s_t_out,
                        cudaStream_t s);

// Q(dX_sel) on padded rows (width = n_sel rounded to 64, zero padded).
cudaError_t launch_residual_gather(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                                   const RowGroups& g, int64_t prows,
                                   const uint8_t* qx_codes, const uint8_t* qx_scales, int qx_layout,
                                   const float* qx_st, const int32_t* sel, int64_t n_sel,
                                   int64_t width, const float* r_st, uint8_t* r_codes,
                                   uint8_t* r_scales, int r_layout, cudaStream_t s);

// Both second passes of a dense RAC linear: Q(dX_sel) into r_* (as
// launch_residual_gather) and Q(W_sel) into ws_* from bf16 w, or from the
// NVFP4 weight w_codes / w_scales / w_st when w is null (w_colamax then holds
// the DQ column maxima).  One launch when the weight side takes the tile
// gather, two when it takes the row-staged kernel.
cudaError_t launch_second_pass(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const uint8_t* qx_codes,
                               const uint8_t* qx_scales, int qx_layout, const float* qx_st, const int32_t* sel,
                               int64_t n_sel, int64_t width, const float* r_st, uint8_t* r_codes, uint8_t* r_scales,
                               int r_layout, const uint16_t* w, int64_t N, int64_t ldw, const uint8_t* w_codes,
                               const uint8_t* w_scales, int w_layout, const float* w_st, const float* w_colamax,
                               float* ws_st, uint8_t* ws_codes, uint8_t* ws_scales, int ws_layout, cudaStream_t s);

// s_t[e] = RN(max_{j < n_sel} colamax[e*K + sel[e*n_sel + j]] / 2688).
cudaError_t launch_sel_tensor_scale(const float* colamax, int64_t K, const int32_t* sel,
                                    int64_t n_sel, int32_t E, float* s_t, cudaStream_t s);

// Q(W_sel) for E stacked weights [E, N, K] (row stride ldw, matrix stride
// N*ldw): out rows E*N, width columns.  Also writes the W_sel tensor scales
// s_t[e] = RN(max_{j in sel_e} colamax[e*K + j] / 2688).
cudaError_t launch_weight_gather(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t E,
                                 const int32_t* sel, int64_t n_sel, int64_t width,
                                 const float* colamax, float* s_t, uint8_t* codes, uint8_t* scales,
                                 int layout, cudaStream_t s);

// W_sel re-quantized from the NVFP4 weight alone (codes, scales, tensor
// scales w_st[E] of E stacked N x K matrices): the values are DQ(Q(W)) and
// dq_colamax [E, K] holds max_n |DQ(Q(W))_nk| (launch_dq_colamax).
cudaError_t launch_weight_gather_fp4(const uint8_t* w_codes, const uint8_t* w_scales, int w_layout,
                                     const float* w_st, int64_t N, int64_t K, int32_t E,
                                     const int32_t* sel, int64_t n_sel, int64_t width,
                                     const float* dq_colamax, float* s_t, uint8_t* codes,
                                     uint8_t* scales, int layout, cudaStream_t s);
// colamax [batch, K] = max over the N rows of each stacked matrix of |DQ|.
cudaError_t launch_dq_colamax(const uint8_t* codes, const uint8_t* scales, int layout, const float* st,
                              int64_t N, int64_t K, int32_t batch, float* colamax, cudaStream_t s);

// W' = bf16(DQ(Q(W))) for `batch` matrices; optional Q(W) and colamax
// (colamax_bits zeroed beforehand, written as fp32 bits).  amax of matrix b:
// max of amax_parts[b * n_parts .. + n_parts).
cudaError_t launch_weight_qdq(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t batch,
                              const unsigned* amax_parts, int n_parts, uint16_t* w_out, uint8_t* codes,
                              uint8_t* scales, int layout, float* tensor_scale,
                              unsigned* colamax_bits, cudaStream_t s);

cudaError_t launch_encode(const float* in, uint8_t* out, int64_t n, int which, cudaStream_t s);

cudaError_t launch_wait_probe(uint64_t limit_ns, unsigned* err, cudaStream_t s);

// Block-scaled FP4 GEMM with an optional second (residual) K segment.
struct GemmOperand {
  const uint8_t* codes;   // [rows, cols/2]
  const uint8_t* scales;  // MMA-tiled
  const float* st;        // tensor scale(s), indexed by group
  int64_t rows, cols;
};

struct GemmArgs {
  GemmOperand a0, b0;     // plain segment: A [M(padded), K], B [E*N, K]
  GemmOperand a1, b1;     // residual segment (a1.codes == null: none)
  RowGroups g;            // rows of A / Y
  int64_t M;              // dense rows (or T for MoE)
  int64_t N;              // out-features per group
  int64_t m_tiles;        // dense: ceil(M/128); MoE: upper bound
  const int32_t* pair_start;  // MoE: prefix of 256-row tiles per group (E + 1)
  void* y;
  int32_t y_dtype;        // 0 fp32, 1 bf16
  int64_t ldy;
  unsigned* err;
};

cudaError_t launch_gemm(const GemmArgs& args, cudaStream_t s);

// MXFP8 x MXFP8 comparator GEMM (single K segment, single-CTA kernel):
// a0 / b0 codes are E4M3 bytes [rows, cols], scales UE8M0 in the MMA-tiled
// layout with 32-element blocks; st unused; cols % 128 == 0; dense rows.
cudaError_t launch_gemm_fp8(const GemmArgs& args, cudaStream_t s);

// MXFP8 quantization of bf16 x [rows, K] (K % 128 == 0): codes [rows, K]
// E4M3 bytes, scales UE8M0 per 32-element block in `layout` (0 canonical
// [rows][K/32], 1 MMA-tiled: per 128-row block one 512-byte atom per 128
// columns, row r at (r%32)*16 + ((r%128)/32)*4 + block%4).
cudaError_t launch_mxfp8_quant(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, uint8_t* codes,
                               uint8_t* scales, int layout, cudaStream_t s);

}  // namespace nvfp4
