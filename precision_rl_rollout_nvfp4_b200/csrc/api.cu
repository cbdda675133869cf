// C ABI of the NVFP4 W4A4 + RAC library (declared in include/nvfp4rac.h):
// argument validation, workspace carving and the launch sequence of each
// call.  No call allocates or synchronizes (except nvfp4_stream_status).
#include <cmath>
#include <cstdio>

#include "kernels.h"
#include "nvfp4rac.h"

using namespace nvfp4;

namespace {

__device__ unsigned g_device_error;   // device error word (bit set = kErr*)

constexpr int kMaxDevices = 64;

// Address of g_device_error on the current device (host code may not take
// the address of a __device__ variable directly).
unsigned* device_error_word() {
  static unsigned* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned*>(p);
  }
  return addr[dev];
}

nvfp4_status device_ok() {
  static int checked[kMaxDevices] = {};   // 0 unknown, 1 ok, 2 not sm_100
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  if (checked[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    checked[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return checked[dev] == 1 ? NVFP4_OK : NVFP4_ERR_DEVICE;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int nvfp4::device_check() {
  const nvfp4_status d = device_ok();
  return d == NVFP4_OK ? 0 : (d == NVFP4_ERR_DEVICE ? 1 : 2);
}

namespace {

nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

#define NV_TRY(expr)                                  \
  do {                                                \
    cudaError_t e_ = (expr);                          \
    if (e_ != cudaSuccess) return NVFP4_ERR_CUDA;     \
  } while (0)

#define NV_CHECK(cond, code)          \
  do {                                \
    if (!(cond)) return (code);       \
  } while (0)

// Carves 256-byte aligned pieces out of a workspace; with base == nullptr it
// only measures.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t scale_bytes(int64_t rows, int64_t cols, int layout) {
  if (layout == 0) return static_cast<size_t>(rows * (cols / kBlock));
  return static_cast<size_t>(ceil_div(rows, 128) * 128 * ceil_div(cols, 64) * 4);
}

bool tensor_ok(const nvfp4_tensor* t) {
  return t && t->codes && t->scales && t->tensor_scale && aligned16(t->codes) && aligned16(t->scales) &&
         (t->scale_layout == 0 || t->scale_layout == 1);
}

// Workspace pieces of nvfp4_quantize.
struct QuantWs {
  unsigned* counters;
  unsigned* amax;
  double* part_sum;
  float* part_max;
};
QuantWs carve_quant(Carver& c, int64_t M, int64_t K, bool scores) {
  QuantWs w{};
  const int64_t tiles = ceil_div(M, kTileRows);
  w.counters = c.take<unsigned>(K / 64 + 1);  // one counter per 64-column strip, then the strips-done count
  w.amax = c.take<unsigned>(amax_parts_count(M, K));   // partial maxima
  if (scores) {
    w.part_sum = c.take<double>(tiles * K);
    w.part_max = c.take<float>(tiles * K);
  }
  return w;
}

// Workspace pieces of the MoE call.
struct MoeWs {
  int32_t* tile_start;
  unsigned* amax;
  uint8_t *qx_codes, *qx_scales;
  float* qx_st;
  double* part_sum;
  float* part_max;
  double* score;
  float* colamax;
  uint8_t* mask;
  int32_t* sel;
  float* r_st;
  uint8_t *r_codes, *r_scales;
  float* ws_st;
  uint8_t *ws_codes, *ws_scales;
};
MoeWs carve_moe(Carver& c, int64_t T, int64_t N, int64_t K, int32_t E, int64_t n_sel, int64_t width) {
  MoeWs w{};
  const int64_t tiles = ceil_div(T, kTileRows) + E;
  const int64_t prows = tiles * kTileRows;
  w.tile_start = c.take<int32_t>(2 * (E + 1));     // 128-row then 256-row tile prefixes
  w.amax = c.take<unsigned>(E);
  w.qx_codes = c.take<uint8_t>(prows * K / 2);
  w.qx_scales = c.take<uint8_t>(scale_bytes(prows, K, 1));
  w.qx_st = c.take<float>(E);
  w.part_sum = c.take<double>(tiles * K);
  w.part_max = c.take<float>(tiles * K);
  w.score = c.take<double>(static_cast<int64_t>(E) * K);
  w.colamax = c.take<float>(static_cast<int64_t>(E) * K);
  w.mask = c.take<uint8_t>(static_cast<int64_t>(E) * K);
  w.sel = c.take<int32_t>(static_cast<int64_t>(E) * (n_sel > 0 ? n_sel : 1));
  w.r_st = c.take<float>(E);
  w.r_codes = c.take<uint8_t>(prows * width / 2 + 16);
  w.r_scales = c.take<uint8_t>(scale_bytes(prows, width, 1) + 16);
  w.ws_st = c.take<float>(E);
  w.ws_codes = c.take<uint8_t>(static_cast<int64_t>(E) * N * width / 2 + 16);
  w.ws_scales = c.take<uint8_t>(scale_bytes(static_cast<int64_t>(E) * N, width, 1) + 16);
  return w;
}

// Workspace of w4a4_rac_gemm: W_sel for the worst case width = K.
struct GemmWs {
  float* st;
  uint8_t *codes, *scales;
};
GemmWs carve_gemm(Carver& c, int64_t N, int64_t width) {
  GemmWs w{};
  w.st = c.take<float>(1);
  w.codes = c.take<uint8_t>(N * width / 2 + 16);
  w.scales = c.take<uint8_t>(scale_bytes(N, width, 1) + 16);
  return w;
}

RowGroups dense_groups(int64_t M) {
  RowGroups g{};
  g.off = nullptr;
  g.tile_start = nullptr;
  g.E = 1;
  g.M = M;
  return g;
}

}  // namespace

extern "C" {

size_t nvfp4_scale_bytes(int64_t rows, int64_t cols, int32_t layout) {
  if (rows < 0 || cols < 0 || (layout != 0 && layout != 1)) return 0;
  return scale_bytes(rows, cols, layout);
}

int64_t nvfp4_rac_nsel(float k_percent, int64_t K) {
  if (!(k_percent >= 0.0f && k_percent <= 100.0f) || K < 0) return -1;
  // floor(k K / 100) with k the exact value of the float: k K is exact in
  // double for K < 2^29; the quotient is corrected to the exact floor.
  const double v = static_cast<double>(k_percent) * static_cast<double>(K);
  int64_t n = static_cast<int64_t>(std::floor(v / 100.0));
  while (static_cast<double>(n + 1) * 100.0 <= v) ++n;
  while (n > 0 && static_cast<double>(n) * 100.0 > v) --n;
  return n;
}

int64_t nvfp4_rac_width(int64_t n_sel) { return n_sel <= 0 ? 0 : ceil_div(n_sel, 64) * 64; }

size_t nvfp4_workspace_size(int32_t op, int64_t M, int64_t N, int64_t K, int32_t E) {
  Carver c(nullptr);
  switch (op) {
    case NVFP4_OP_QUANTIZE: carve_quant(c, M, K, true); break;
    case NVFP4_OP_RAC_SELECT: c.take<float>(1); break;
    case NVFP4_OP_GEMM: carve_gemm(c, N, nvfp4_rac_width(K)); break;
    case NVFP4_OP_MOE: carve_moe(c, M, N, K, E, K, nvfp4_rac_width(K)); break;
    case NVFP4_OP_WEIGHT_QDQ: c.take<unsigned>(static_cast<size_t>(E > 0 ? E : 1) * amax_parts_count(N, K)); break;
    default: return 0;
  }
  return c.off + 256;
}

nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                            const float* amax_or_null, nvfp4_tensor* qx, double* score_or_null,
                            float* res_colamax_or_null, void* ws, size_t ws_bytes, void* stream) {
  NV_CHECK(x && tensor_ok(qx), NVFP4_ERR_INVALID_ARG);
  NV_CHECK(score_or_null == nullptr || res_colamax_or_null != nullptr, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(M >= 1 && K >= 64 && K % 64 == 0 && ldx >= K && qx->rows == M && qx->cols == K,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x) && ldx % 8 == 0, NVFP4_ERR_MISALIGNED);
  // stats: the residual column maxima (and with scores the channel sums)
  // go through per-tile partials and the last CTA of each column strip
  const bool scores = score_or_null != nullptr, stats = res_colamax_or_null != nullptr;
  Carver c(ws);
  const QuantWs w = carve_quant(c, M, K, stats);
  NV_CHECK(ws != nullptr && ws_bytes >= c.off, NVFP4_ERR_WORKSPACE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const RowGroups g = dense_groups(M);
  // the strip counters must start at zero: the amax pass clears them, or a
  // memset does when the caller supplies amax
  int n_parts = 0;
  if (amax_or_null == nullptr) {
    n_parts = amax_parts_count(M, K);
    NV_TRY(launch_amax_partial(x, M, K, ldx, 1, 0, w.amax, n_parts, w.counters,
                               stats ? static_cast<int>(K / 64 + 1) : 0, s));
  } else if (stats) {
    NV_TRY(cudaMemsetAsync(w.counters, 0, sizeof(unsigned) * (K / 64 + 1), s));
  }
  NV_TRY(launch_quant_score(x, M, K, ldx, g, amax_or_null, w.amax, n_parts, M, qx->codes, qx->scales,
                            qx->scale_layout, qx->tensor_scale, scores ? w.part_sum : nullptr,
                            stats ? w.part_max : nullptr, stats ? w.counters : nullptr, score_or_null,
                            res_colamax_or_null, s));
  return NVFP4_OK;
}

nvfp4_status rac_quantize_select(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const float* amax_or_null,
                                 nvfp4_tensor* qx, double* score, float* res_colamax, float k_percent, uint8_t* mask,
                                 int32_t* sel, int64_t* n_sel_out, float* res_tensor_scale, void* ws,
                                 size_t ws_bytes, void* stream) {
  NV_CHECK(x && tensor_ok(qx) && score && res_colamax && mask && n_sel_out && res_tensor_scale,
           NVFP4_ERR_INVALID_ARG);
  NV_CHECK(k_percent >= 0.0f && k_percent <= 100.0f, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(M >= 1 && K >= 64 && K % 64 == 0 && ldx >= K && qx->rows == M && qx->cols == K,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x) && ldx % 8 == 0, NVFP4_ERR_MISALIGNED);
  const int64_t n_sel = nvfp4_rac_nsel(k_percent, K);
  NV_CHECK(n_sel == 0 || sel, NVFP4_ERR_INVALID_ARG);
  Carver c(ws);
  const QuantWs w = carve_quant(c, M, K, true);
  NV_CHECK(ws != nullptr && ws_bytes >= c.off, NVFP4_ERR_WORKSPACE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int n_parts = 0;
  if (amax_or_null == nullptr) {
    n_parts = amax_parts_count(M, K);
    NV_TRY(launch_amax_partial(x, M, K, ldx, 1, 0, w.amax, n_parts, w.counters, static_cast<int>(K / 64 + 1), s));
  } else {
    NV_TRY(cudaMemsetAsync(w.counters, 0, sizeof(unsigned) * (K / 64 + 1), s));
  }
  const FusedSelect fs{n_sel, mask, sel, res_tensor_scale, w.counters + K / 64};
  *n_sel_out = n_sel;
  NV_TRY(launch_quant_score(x, M, K, ldx, dense_groups(M), amax_or_null, w.amax, n_parts, M, qx->codes, qx->scales,
                            qx->scale_layout, qx->tensor_scale, w.part_sum, w.part_max, w.counters, score,
                            res_colamax, s, &fs));
  return NVFP4_OK;
}

nvfp4_status rac_second_pass(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* qx,
                             const int32_t* sel, int64_t n_sel, nvfp4_tensor* q_res, const uint16_t* w, int64_t N,
                             int64_t ldw, const nvfp4_tensor* qw, const float* w_colamax, nvfp4_tensor* q_wsel,
                             void* stream) {
  NV_CHECK(x && tensor_ok(qx) && sel && tensor_ok(q_res) && tensor_ok(q_wsel) && w_colamax, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(w != nullptr || tensor_ok(qw), NVFP4_ERR_INVALID_ARG);
  const int64_t width = nvfp4_rac_width(n_sel);
  NV_CHECK(M >= 1 && K >= 64 && K % 64 == 0 && ldx >= K && qx->rows == M && qx->cols == K && n_sel >= 1 &&
               n_sel <= K && q_res->rows == M && q_res->cols == width && N >= 1 && q_wsel->rows == N &&
               q_wsel->cols == width && (w == nullptr ? (qw->rows == N && qw->cols == K) : ldw >= K),
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x) && ldx % 8 == 0 && (w == nullptr || (aligned16(w) && ldw % 8 == 0)), NVFP4_ERR_MISALIGNED);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q_wsel->scale_layout == 1 && N % 128 != 0)
    NV_TRY(cudaMemsetAsync(q_wsel->scales, 0, scale_bytes(N, width, 1), s));
  NV_TRY(launch_second_pass(x, M, K, ldx, qx->codes, qx->scales, qx->scale_layout, qx->tensor_scale, sel, n_sel,
                            width, q_res->tensor_scale, q_res->codes, q_res->scales, q_res->scale_layout, w, N,
                            w != nullptr ? ldw : K, w == nullptr ? qw->codes : nullptr,
                            w == nullptr ? qw->scales : nullptr, w == nullptr ? qw->scale_layout : 0,
                            w == nullptr ? qw->tensor_scale : nullptr, w_colamax, q_wsel->tensor_scale,
                            q_wsel->codes, q_wsel->scales, q_wsel->scale_layout, s));
  return NVFP4_OK;
}

nvfp4_status rac_select(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* qx,
                        const double* score, const float* res_colamax, float k_percent,
                        uint8_t* mask, int32_t* sel, int64_t* n_sel_out, nvfp4_tensor* q_res,
                        void* ws, size_t ws_bytes, void* stream) {
  NV_CHECK(x && tensor_ok(qx) && score && res_colamax && mask && n_sel_out, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(k_percent >= 0.0f && k_percent <= 100.0f, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(M >= 1 && K >= 64 && K % 64 == 0 && ldx >= K && qx->rows == M && qx->cols == K,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x) && ldx % 8 == 0, NVFP4_ERR_MISALIGNED);
  const int64_t n_sel = nvfp4_rac_nsel(k_percent, K);
  const int64_t width = nvfp4_rac_width(n_sel);
  if (n_sel > 0) {
    NV_CHECK(sel && tensor_ok(q_res), NVFP4_ERR_INVALID_ARG);
    NV_CHECK(q_res->rows == M && q_res->cols == width, NVFP4_ERR_UNSUPPORTED_SHAPE);
  }
  Carver c(ws);
  float* st_scratch = c.take<float>(1);
  NV_CHECK(ws != nullptr && ws_bytes >= c.off, NVFP4_ERR_WORKSPACE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  *n_sel_out = n_sel;
  float* r_st = n_sel > 0 ? q_res->tensor_scale : st_scratch;
  NV_TRY(launch_topk(score, res_colamax, K, 1, n_sel, mask, sel, r_st, s));
  if (n_sel > 0)
    NV_TRY(launch_residual_gather(x, M, K, ldx, dense_groups(M), M, qx->codes, qx->scales,
                                  qx->scale_layout, qx->tensor_scale, sel, n_sel, width, r_st,
                                  q_res->codes, q_res->scales, q_res->scale_layout, s));
  return NVFP4_OK;
}

nvfp4_status rac_select_channels(const double* score, const float* res_colamax, int64_t K, float k_percent,
                                 uint8_t* mask, int32_t* sel, int64_t* n_sel_out, float* res_tensor_scale,
                                 void* stream) {
  NV_CHECK(score && res_colamax && mask && n_sel_out && res_tensor_scale, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(k_percent >= 0.0f && k_percent <= 100.0f, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(K >= 64 && K % 64 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE);
  const int64_t n_sel = nvfp4_rac_nsel(k_percent, K);
  NV_CHECK(n_sel == 0 || sel, NVFP4_ERR_INVALID_ARG);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  *n_sel_out = n_sel;
  NV_TRY(launch_topk(score, res_colamax, K, 1, n_sel, mask, sel, res_tensor_scale,
                     static_cast<cudaStream_t>(stream)));
  return NVFP4_OK;
}

nvfp4_status rac_residual_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* qx,
                                const int32_t* sel, int64_t n_sel, nvfp4_tensor* q_res, void* stream) {
  NV_CHECK(x && tensor_ok(qx) && sel && tensor_ok(q_res), NVFP4_ERR_INVALID_ARG);
  NV_CHECK(M >= 1 && K >= 64 && K % 64 == 0 && ldx >= K && qx->rows == M && qx->cols == K && n_sel >= 1 &&
               n_sel <= K && q_res->rows == M && q_res->cols == nvfp4_rac_width(n_sel),
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x) && ldx % 8 == 0, NVFP4_ERR_MISALIGNED);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  NV_TRY(launch_residual_gather(x, M, K, ldx, dense_groups(M), M, qx->codes, qx->scales, qx->scale_layout,
                                qx->tensor_scale, sel, n_sel, q_res->cols, q_res->tensor_scale, q_res->codes,
                                q_res->scales, q_res->scale_layout, static_cast<cudaStream_t>(stream)));
  return NVFP4_OK;
}

nvfp4_status rac_sel_tensor_scale(const float* colamax, int64_t K, const int32_t* sel, int64_t n_sel,
                                  float* tensor_scale, void* stream) {
  NV_CHECK(colamax && sel && tensor_scale, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(K >= 1 && n_sel >= 1 && n_sel <= K, NVFP4_ERR_UNSUPPORTED_SHAPE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  NV_TRY(launch_sel_tensor_scale(colamax, K, sel, n_sel, 1, tensor_scale, static_cast<cudaStream_t>(stream)));
  return NVFP4_OK;
}

nvfp4_status rac_weight_quant(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, const int32_t* sel,
                              int64_t n_sel, const float* w_colamax, nvfp4_tensor* q_wsel,
                              void* stream) {
  NV_CHECK(w && sel && w_colamax && tensor_ok(q_wsel), NVFP4_ERR_INVALID_ARG);
  NV_CHECK(N >= 1 && K >= 64 && K % 64 == 0 && ldw >= K && n_sel >= 1 && n_sel <= K,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  const int64_t width = nvfp4_rac_width(n_sel);
  NV_CHECK(q_wsel->rows == N && q_wsel->cols == width, NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(w) && ldw % 8 == 0, NVFP4_ERR_MISALIGNED);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q_wsel->scale_layout == 1 && N % 128 != 0)
    NV_TRY(cudaMemsetAsync(q_wsel->scales, 0, scale_bytes(N, width, 1), s));
  NV_TRY(launch_weight_gather(w, N, K, ldw, 1, sel, n_sel, width, w_colamax, q_wsel->tensor_scale,
                              q_wsel->codes, q_wsel->scales, q_wsel->scale_layout, s));
  return NVFP4_OK;
}

nvfp4_status nvfp4_dq_colamax(const nvfp4_tensor* q, int32_t batch, float* colamax, void* stream) {
  NV_CHECK(tensor_ok(q) && colamax, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(batch >= 1 && q->rows >= batch && q->rows % batch == 0 && q->cols >= 64 && q->cols % 64 == 0,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(colamax), NVFP4_ERR_MISALIGNED);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  NV_TRY(launch_dq_colamax(q->codes, q->scales, q->scale_layout, q->tensor_scale, q->rows / batch, q->cols,
                           batch, colamax, static_cast<cudaStream_t>(stream)));
  return NVFP4_OK;
}

nvfp4_status rac_weight_quant_fp4(const nvfp4_tensor* qw, const int32_t* sel, int64_t n_sel,
                                  const float* dq_colamax, nvfp4_tensor* q_wsel, void* stream) {
  NV_CHECK(tensor_ok(qw) && sel && dq_colamax && tensor_ok(q_wsel), NVFP4_ERR_INVALID_ARG);
  const int64_t N = qw->rows, K = qw->cols;
  NV_CHECK(N >= 1 && K >= 64 && K % 64 == 0 && n_sel >= 1 && n_sel <= K, NVFP4_ERR_UNSUPPORTED_SHAPE);
  const int64_t width = nvfp4_rac_width(n_sel);
  NV_CHECK(q_wsel->rows == N && q_wsel->cols == width, NVFP4_ERR_UNSUPPORTED_SHAPE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q_wsel->scale_layout == 1 && N % 128 != 0)
    NV_TRY(cudaMemsetAsync(q_wsel->scales, 0, scale_bytes(N, width, 1), s));
  NV_TRY(launch_weight_gather_fp4(qw->codes, qw->scales, qw->scale_layout, qw->tensor_scale, N, K, 1, sel,
                                  n_sel, width, dq_colamax, q_wsel->tensor_scale, q_wsel->codes,
                                  q_wsel->scales, q_wsel->scale_layout, s));
  return NVFP4_OK;
}

static nvfp4_status gemm_checked(const nvfp4_tensor* qa, const nvfp4_tensor* qb, const nvfp4_tensor* qr,
                                 const nvfp4_tensor* qws, void* y, int32_t y_dtype, int64_t ldy,
                                 cudaStream_t s) {
  NV_CHECK(tensor_ok(qa) && tensor_ok(qb) && y, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(qa->scale_layout == 1 && qb->scale_layout == 1, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(y_dtype == 0 || y_dtype == 1, NVFP4_ERR_INVALID_ARG);
  NV_CHECK((qr == nullptr) == (qws == nullptr), NVFP4_ERR_INVALID_ARG);
  const int64_t M = qa->rows, N = qb->rows, K = qa->cols;
  NV_CHECK(M >= 1 && N >= 16 && N % 16 == 0 && K >= 64 && K % 64 == 0 && qb->cols == K && ldy >= N,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(y) && ldy % 8 == 0, NVFP4_ERR_MISALIGNED);
  GemmArgs a{};
  a.a0 = {qa->codes, qa->scales, qa->tensor_scale, M, K};
  a.b0 = {qb->codes, qb->scales, qb->tensor_scale, N, K};
  if (qr) {
    NV_CHECK(tensor_ok(qr) && tensor_ok(qws) && qr->scale_layout == 1 && qws->scale_layout == 1,
             NVFP4_ERR_INVALID_ARG);
    NV_CHECK(qr->rows == M && qws->rows == N && qr->cols == qws->cols && qr->cols % 64 == 0 && qr->cols > 0,
             NVFP4_ERR_UNSUPPORTED_SHAPE);
    a.a1 = {qr->codes, qr->scales, qr->tensor_scale, M, qr->cols};
    a.b1 = {qws->codes, qws->scales, qws->tensor_scale, N, qws->cols};
  }
  a.g = dense_groups(M);
  a.M = M;
  a.N = N;
  a.m_tiles = ceil_div(M, 128);
  a.y = y;
  a.y_dtype = y_dtype;
  a.ldy = ldy;
  a.err = device_error_word();
  NV_CHECK(a.err != nullptr, NVFP4_ERR_CUDA);
  return cuda_status(launch_gemm(a, s));
}

nvfp4_status w4a4_gemm_quantized(const nvfp4_tensor* qa, const nvfp4_tensor* qb,
                                 const nvfp4_tensor* q_res_or_null, const nvfp4_tensor* q_wsel_or_null,
                                 void* y, int32_t y_dtype, int64_t ldy, void* stream) {
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  return gemm_checked(qa, qb, q_res_or_null, q_wsel_or_null, y, y_dtype, ldy,
                      static_cast<cudaStream_t>(stream));
}

nvfp4_status w4a4_rac_gemm(const nvfp4_tensor* qx, const nvfp4_tensor* q_res_or_null, const int32_t* sel,
                           int64_t n_sel, const uint16_t* w, int64_t N, int64_t ldw,
                           const nvfp4_tensor* qw, const float* w_colamax, void* y, int32_t y_dtype,
                           int64_t ldy, void* ws, size_t ws_bytes, void* stream) {
  NV_CHECK(tensor_ok(qx) && tensor_ok(qw), NVFP4_ERR_INVALID_ARG);
  NV_CHECK(qw->rows == N, NVFP4_ERR_UNSUPPORTED_SHAPE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_sel <= 0 || q_res_or_null == nullptr)
    return gemm_checked(qx, qw, nullptr, nullptr, y, y_dtype, ldy, s);
  const int64_t K = qx->cols;
  const int64_t width = nvfp4_rac_width(n_sel);
  NV_CHECK(sel && w_colamax, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(n_sel <= K && q_res_or_null->cols == width && qw->cols == K, NVFP4_ERR_UNSUPPORTED_SHAPE);
  Carver c(ws);
  const GemmWs gw = carve_gemm(c, N, width);
  NV_CHECK(ws != nullptr && ws_bytes >= c.off, NVFP4_ERR_WORKSPACE);
  nvfp4_tensor wsel{gw.codes, gw.scales, gw.st, N, width, 1};
  // W_sel from the bf16 weight, or (w == NULL) from Q(W) itself
  const nvfp4_status r = w ? rac_weight_quant(w, N, K, ldw, sel, n_sel, w_colamax, &wsel, stream)
                           : rac_weight_quant_fp4(qw, sel, n_sel, w_colamax, &wsel, stream);
  if (r != NVFP4_OK) return r;
  return gemm_checked(qx, qw, q_res_or_null, &wsel, y, y_dtype, ldy, s);
}

nvfp4_status moe_grouped_w4a4_rac_gemm(const uint16_t* x_perm, int64_t T, int64_t K,
                                       const int64_t* offsets_dev, int32_t E, const uint16_t* w,
                                       int64_t N, const nvfp4_tensor* qw, const float* w_colamax,
                                       float k_percent, void* y_perm, int32_t y_dtype,
                                       uint8_t* masks_or_null, void* ws, size_t ws_bytes,
                                       void* stream) {
  NV_CHECK(x_perm && offsets_dev && tensor_ok(qw) && w_colamax && y_perm, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(k_percent >= 0.0f && k_percent <= 100.0f && (y_dtype == 0 || y_dtype == 1),
           NVFP4_ERR_INVALID_ARG);
  NV_CHECK(E >= 1 && E <= 4096 && T >= 1 && K >= 64 && K % 64 == 0 && N >= 128 && N % 128 == 0,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(qw->scale_layout == 1 && qw->rows == static_cast<int64_t>(E) * N && qw->cols == K,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x_perm) && aligned16(w) && aligned16(y_perm), NVFP4_ERR_MISALIGNED);   // w may be NULL
  const int64_t n_sel = nvfp4_rac_nsel(k_percent, K);
  const int64_t width = nvfp4_rac_width(n_sel);
  Carver c(ws);
  const MoeWs m = carve_moe(c, T, N, K, E, n_sel, width);
  NV_CHECK(ws != nullptr && ws_bytes >= c.off, NVFP4_ERR_WORKSPACE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t tiles = ceil_div(T, kTileRows) + E;
  const int64_t prows = tiles * kTileRows;
  RowGroups g{};
  g.off = offsets_dev;
  g.tile_start = m.tile_start;
  g.E = E;
  g.M = T;
  uint8_t* mask = masks_or_null ? masks_or_null : m.mask;
  NV_TRY(launch_group_tiles(offsets_dev, E, m.tile_start, s));
  NV_TRY(cudaMemsetAsync(m.amax, 0, sizeof(unsigned) * E, s));
  NV_TRY(launch_amax(x_perm, T, K, K, g, m.amax, s));
  NV_TRY(launch_quant_score(x_perm, T, K, K, g, reinterpret_cast<const float*>(m.amax), nullptr, 0, prows,
                            m.qx_codes, m.qx_scales, 1, m.qx_st, m.part_sum, m.part_max, nullptr,
                            nullptr, nullptr, s));
  NV_TRY(launch_score_reduce(m.part_sum, m.part_max, K, g, tiles, m.score, m.colamax, m.qx_st, s));
  NV_TRY(launch_topk(m.score, m.colamax, K, E, n_sel, mask, m.sel, m.r_st, s));
  GemmArgs a{};
  a.a0 = {m.qx_codes, m.qx_scales, m.qx_st, prows, K};
  a.b0 = {qw->codes, qw->scales, qw->tensor_scale, static_cast<int64_t>(E) * N, K};
  if (n_sel > 0) {
    NV_TRY(launch_residual_gather(x_perm, T, K, K, g, prows, m.qx_codes, m.qx_scales, 1, m.qx_st, m.sel,
                                  n_sel, width, m.r_st, m.r_codes, m.r_scales, 1, s));
    if (w)
      NV_TRY(launch_weight_gather(w, N, K, K, E, m.sel, n_sel, width, w_colamax, m.ws_st, m.ws_codes,
                                  m.ws_scales, 1, s));
    else
      NV_TRY(launch_weight_gather_fp4(qw->codes, qw->scales, 1, qw->tensor_scale, N, K, E, m.sel, n_sel,
                                      width, w_colamax, m.ws_st, m.ws_codes, m.ws_scales, 1, s));
    a.a1 = {m.r_codes, m.r_scales, m.r_st, prows, width};
    a.b1 = {m.ws_codes, m.ws_scales, m.ws_st, static_cast<int64_t>(E) * N, width};
  }
  a.g = g;
  a.M = T;
  a.N = N;
  a.m_tiles = tiles;
  a.pair_start = m.tile_start + E + 1;
  a.y = y_perm;
  a.y_dtype = y_dtype;
  a.ldy = N;
  a.err = device_error_word();
  NV_CHECK(a.err != nullptr, NVFP4_ERR_CUDA);
  return cuda_status(launch_gemm(a, s));
}

nvfp4_status weight_qdq(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t batch,
                        uint16_t* w_out, nvfp4_tensor* qw_or_null, float* colamax_or_null, void* ws,
                        size_t ws_bytes, void* stream) {
  NV_CHECK(w && w_out, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(batch >= 1 && N >= 1 && K >= 64 && K % 64 == 0 && ldw >= K, NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(w) && aligned16(w_out) && ldw % 8 == 0, NVFP4_ERR_MISALIGNED);
  if (qw_or_null) {
    NV_CHECK(tensor_ok(qw_or_null), NVFP4_ERR_INVALID_ARG);
    NV_CHECK(qw_or_null->rows == static_cast<int64_t>(batch) * N && qw_or_null->cols == K,
             NVFP4_ERR_UNSUPPORTED_SHAPE);
  }
  Carver c(ws);
  const int n_parts = amax_parts_count(N, K);
  unsigned* amax = c.take<unsigned>(static_cast<size_t>(batch) * n_parts);
  NV_CHECK(ws != nullptr && ws_bytes >= c.off, NVFP4_ERR_WORKSPACE);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (qw_or_null && qw_or_null->scale_layout == 1 && (static_cast<int64_t>(batch) * N) % 128 != 0)
    NV_TRY(cudaMemsetAsync(qw_or_null->scales, 0, scale_bytes(static_cast<int64_t>(batch) * N, K, 1), s));
  // the amax pass also clears colamax (accumulated with atomic max)
  NV_TRY(launch_amax_partial(w, N, K, ldw, batch, N * ldw, amax, n_parts,
                             reinterpret_cast<unsigned*>(colamax_or_null),
                             colamax_or_null ? static_cast<int>(batch * K) : 0, s));
  NV_TRY(launch_weight_qdq(w, N, K, ldw, batch, amax, n_parts, w_out, qw_or_null ? qw_or_null->codes : nullptr,
                           qw_or_null ? qw_or_null->scales : nullptr,
                           qw_or_null ? qw_or_null->scale_layout : 0,
                           qw_or_null ? qw_or_null->tensor_scale : nullptr,
                           reinterpret_cast<unsigned*>(colamax_or_null), s));
  return NVFP4_OK;
}

size_t mxfp8_scale_bytes(int64_t rows, int64_t cols, int32_t layout) {
  if (rows < 0 || cols < 0 || (layout != 0 && layout != 1)) return 0;
  if (layout == 0) return static_cast<size_t>(rows * (cols / 32));
  return static_cast<size_t>(ceil_div(rows, 128) * 128 * ceil_div(cols, 128) * 4);
}

static bool mx_tensor_ok(const mxfp8_tensor* t) {
  return t && t->codes && t->scales && aligned16(t->codes) && aligned16(t->scales) &&
         (t->scale_layout == 0 || t->scale_layout == 1);
}

nvfp4_status mxfp8_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, mxfp8_tensor* q, void* stream) {
  NV_CHECK(x && mx_tensor_ok(q), NVFP4_ERR_INVALID_ARG);
  NV_CHECK(M >= 1 && K >= 256 && K % 256 == 0 && ldx >= K && q->rows == M && q->cols == K,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(x) && ldx % 8 == 0, NVFP4_ERR_MISALIGNED);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q->scale_layout == 1 && M % 128 != 0)
    NV_TRY(cudaMemsetAsync(q->scales, 0, mxfp8_scale_bytes(M, K, 1), s));
  NV_TRY(launch_mxfp8_quant(x, M, K, ldx, q->codes, q->scales, q->scale_layout, s));
  return NVFP4_OK;
}

nvfp4_status w8a8_gemm_quantized(const mxfp8_tensor* qa, const mxfp8_tensor* qb, void* y, int32_t y_dtype,
                                 int64_t ldy, void* stream) {
  NV_CHECK(mx_tensor_ok(qa) && mx_tensor_ok(qb) && y, NVFP4_ERR_INVALID_ARG);
  NV_CHECK(qa->scale_layout == 1 && qb->scale_layout == 1 && (y_dtype == 0 || y_dtype == 1),
           NVFP4_ERR_INVALID_ARG);
  const int64_t M = qa->rows, N = qb->rows, K = qa->cols;
  NV_CHECK(M >= 1 && N >= 16 && N % 16 == 0 && K >= 128 && K % 128 == 0 && qb->cols == K && ldy >= N,
           NVFP4_ERR_UNSUPPORTED_SHAPE);
  NV_CHECK(aligned16(y) && ldy % 8 == 0, NVFP4_ERR_MISALIGNED);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  GemmArgs a{};
  a.a0 = {qa->codes, qa->scales, nullptr, M, K};
  a.b0 = {qb->codes, qb->scales, nullptr, N, K};
  a.g = dense_groups(M);
  a.M = M;
  a.N = N;
  a.m_tiles = ceil_div(M, 128);
  a.y = y;
  a.y_dtype = y_dtype;
  a.ldy = ldy;
  a.err = device_error_word();
  NV_CHECK(a.err != nullptr, NVFP4_ERR_CUDA);
  return cuda_status(launch_gemm_fp8(a, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_encode_e2m1(const float* in, uint8_t* out, int64_t n, void* stream) {
  NV_CHECK(in && out && n >= 0, NVFP4_ERR_INVALID_ARG);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  return cuda_status(launch_encode(in, out, n, 0, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_encode_e4m3(const float* in, uint8_t* out, int64_t n, void* stream) {
  NV_CHECK(in && out && n >= 0, NVFP4_ERR_INVALID_ARG);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  return cuda_status(launch_encode(in, out, n, 1, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_stream_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
  {
    // index checks of the checked build (always 0 in the normal build)
    unsigned l0 = 0, l1 = 0, l2 = 0;
    const unsigned f = bounds_flags_quant(&l0) | bounds_flags_select(&l1) | bounds_flags_gemm(&l2);
    if (f != 0) {
      fprintf(stderr, "nvfp4: index check failed (quant.cu line %u, select.cu line %u, gemm.cu line %u)\n", l0,
              l1, l2);
      return NVFP4_ERR_BOUNDS;
    }
  }
  unsigned* word = device_error_word();
  if (word == nullptr) return NVFP4_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v & kErrTimeout) return NVFP4_ERR_TIMEOUT;
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_check_bounded_wait(int32_t timeout_ms, void* stream) {
  NV_CHECK(timeout_ms >= 1, NVFP4_ERR_INVALID_ARG);
  const nvfp4_status d = device_ok();
  if (d != NVFP4_OK) return d;
  unsigned* word = device_error_word();
  NV_CHECK(word != nullptr, NVFP4_ERR_CUDA);
  const uint64_t ms = timeout_ms > 2000 ? 2000 : static_cast<uint64_t>(timeout_ms);
  return cuda_status(launch_wait_probe(ms * 1000000ull, word, static_cast<cudaStream_t>(stream)));
}

int32_t nvfp4_build_flags(void) {
#ifdef NVFP4_CHECKS
  return 1;
#else
  return 0;
#endif
}

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_MISALIGNED: return "pointer or leading dimension misaligned";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_WORKSPACE: return "workspace too small";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device-side wait timed out";
    case NVFP4_ERR_DEVICE: return "device is not sm_100 (B200)";
    case NVFP4_ERR_BOUNDS: return "index check failed (checked build)";
  }
  return "unknown status";
}

}  // extern "C"
