// Memory-bound kernels of the NVFP4 W4A4 + RAC path: tensor amax, the fused
// quantize + residual + channel-score pass, the score reduction, the
// second-pass gather-quantize of the residual and of the weight columns, and
// the trainer-side weight fake quantization.
//
// Operations (QUADS technical summary, gist.science): the coarse E2M1 grid
// (section 1), the shared weight QDQ path (2.1), W4A16 fake quantization of
// the weights (2.2 A), high-residual channel selection and second-pass
// quantization (2.2 B).  The formulas are the reading in include/nvfp4rac.h.
//
// Layout of the quantize pass: a CTA of 256 threads owns a 128-row x 64-column
// tile.  Thread t handles 8 consecutive columns (one 16-byte load) of rows
// t/8 + 32 i, i = 0..3; the two halves of a 16-element block sit in threads
// t and t^1 and meet through one shfl.xor.  |dX| goes to shared memory and 64
// threads then sum their column over the 128 rows in row order in fp64.
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kQThreads = 256;
constexpr int kQCols = 64;
constexpr int kDxStride = kQCols + 4;

// ---------------------------------------------------------------------------
// amax
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQThreads)
amax_kernel(const uint16_t* __restrict__ x, int64_t K, int64_t ldx, RowGroups g,
            int64_t mat_stride, unsigned* __restrict__ amax_bits) {
  // blockIdx.z: matrix of a stack of dense matrices (mat_stride elements apart)
  x += blockIdx.z * mat_stride;
  amax_bits += blockIdx.z;
  const TileInfo ti = tile_info(g, blockIdx.y);
  if (!ti.valid) return;
  const int t = threadIdx.x, cg = t & 7, rr = t >> 3;
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kQCols + 8 * cg;
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = ti.row0 + rr + 32 * i;
    if (row < ti.row_end) {
      const uint4 v = ld_nc_v4(x + row * ldx + col);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m = max(m, w[j] & 0x7FFFu);
        m = max(m, (w[j] >> 16) & 0x7FFFu);
      }
    }
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t wmax[kQThreads / 32];
  if ((t & 31) == 0) wmax[t >> 5] = m;
  __syncthreads();
  if (t == 0) {
    uint32_t r = 0;
    for (int i = 0; i < kQThreads / 32; ++i) r = max(r, wmax[i]);
    if (r) atomicMax(amax_bits + ti.e, r << 16);   // |bf16| bits order like their values
  }
}

__global__ void group_tiles_kernel(const int64_t* __restrict__ off, int32_t E,
                                   int32_t* __restrict__ tile_start) {
  if (threadIdx.x != 0) return;
  int32_t acc = 0;
  for (int e = 0; e < E; ++e) {
    tile_start[e] = acc;
    const int64_t m = off[e + 1] - off[e];
    acc += static_cast<int32_t>((m + kTileRows - 1) / kTileRows);
  }
  tile_start[E] = acc;
}

// ---------------------------------------------------------------------------
// quantize + residual + score partials
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQThreads)
quant_score_kernel(const uint16_t* __restrict__ x, int64_t K, int64_t ldx, RowGroups g,
                   const float* __restrict__ amax, int64_t codes_rows,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int layout,
                   float* __restrict__ tensor_scale, double* __restrict__ part_sum,
                   float* __restrict__ part_max) {
  const int64_t tile = blockIdx.y;
  const TileInfo ti = tile_info(g, tile);
  if (!ti.valid) return;
  __shared__ float dxs[kTileRows][kDxStride];
  const int t = threadIdx.x, cg = t & 7, rr = t >> 3;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kQCols;
  const int64_t col = col0 + 8 * cg;
  const float s_t = __fdiv_rn(amax[ti.e], kTensorScaleDiv);
  if (blockIdx.x == 0 && t == 0 && (g.off == nullptr ? tile == 0 : tile == g.tile_start[ti.e]))
    tensor_scale[ti.e] = s_t;

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rr + 32 * i;
    const int64_t row = ti.row0 + r;
    const int64_t prow = tile * kTileRows + r;
    float f[8];
    if (row < ti.row_end) {
      unpack_bf16x8(ld_nc_v4(x + row * ldx + col), f);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = 0.0f;
    }
    float am = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(f[j]));
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
    const BlockScale bs = block_scale(am, s_t);
    const uint32_t q = encode8(f, bs.s_dec);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float dq = dequant((q >> (4 * j)) & 15u, bs.sbv, s_t);
      dxs[r][8 * cg + j] = fabsf(__fsub_rn(f[j], dq));
    }
    if (prow < codes_rows)
      *reinterpret_cast<uint32_t*>(codes + prow * (K / 2) + col / 2) = q;
    if ((cg & 1) == 0 && (layout == 1 || prow < codes_rows))
      scales[scale_offset(prow, col / kBlock, K, layout)] = static_cast<uint8_t>(bs.sb);
  }
  if (part_sum == nullptr) return;
  __syncthreads();
  if (t < kQCols) {
    double acc = 0.0;
    float mx = 0.0f;
    for (int r = 0; r < kTileRows; ++r) {       // row order within the chunk
      const float v = dxs[r][t];
      acc += static_cast<double>(v);
      mx = fmaxf(mx, v);
    }
    part_sum[tile * K + col0 + t] = acc;
    part_max[tile * K + col0 + t] = mx;
  }
}

__global__ void score_reduce_kernel(const double* __restrict__ part_sum,
                                    const float* __restrict__ part_max, int64_t K, RowGroups g,
                                    int64_t tiles, double* __restrict__ score,
                                    float* __restrict__ colamax, float* __restrict__ st_empty) {
  const int e = blockIdx.y;
  int64_t t0 = 0, t1 = tiles;
  if (g.off != nullptr) { t0 = g.tile_start[e]; t1 = g.tile_start[e + 1]; }
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (st_empty != nullptr && t0 == t1 && blockIdx.x == 0 && threadIdx.x == 0) st_empty[e] = 0.0f;
  if (j >= K) return;
  double acc = 0.0;
  float mx = 0.0f;
  for (int64_t t = t0; t < t1; ++t) {          // chunk order
    acc += part_sum[t * K + j];
    mx = fmaxf(mx, part_max[t * K + j]);
  }
  score[e * K + j] = acc;
  colamax[e * K + j] = mx;
}

// ---------------------------------------------------------------------------
// second-pass gather + quantize
// ---------------------------------------------------------------------------
constexpr int kGThreads = 128;

// One thread per (padded row, 16-block of the gathered width).  grid.x = rows,
// grid.y = ceil(width/16 / 128).
__global__ void __launch_bounds__(kGThreads)
residual_gather_kernel(const uint16_t* __restrict__ x, int64_t K, int64_t ldx, RowGroups g,
                       const uint8_t* __restrict__ qx_codes, const uint8_t* __restrict__ qx_scales,
                       int qx_layout, const float* __restrict__ qx_st,
                       const int32_t* __restrict__ sel, int64_t n_sel, int64_t width,
                       const float* __restrict__ r_st, uint8_t* __restrict__ r_codes,
                       uint8_t* __restrict__ r_scales, int r_layout, int64_t r_rows) {
  const int64_t prow = blockIdx.x;
  const int64_t blk = static_cast<int64_t>(blockIdx.y) * kGThreads + threadIdx.x;
  if (blk * kBlock >= width) return;
  const TileInfo ti = tile_info(g, prow / kTileRows);
  const int64_t row = ti.row0 + (prow % kTileRows);
  const bool live = ti.valid && row < ti.row_end;
  const int e = ti.e;
  const float st_x = live ? qx_st[e] : 0.0f;
  const float st_r = live ? r_st[e] : 0.0f;
  const int32_t* s = sel + static_cast<int64_t>(e) * n_sel;
  float v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int64_t j = blk * kBlock + u;
    v[u] = 0.0f;
    if (live && j < n_sel) {
      const int64_t c = s[j];
      if (c < 0 || c >= K) continue;            // never taken for a valid sel list
      const float xv = bf16_bits_to_f32(x[row * ldx + c]);
      const uint32_t code = (qx_codes[prow * (K / 2) + (c >> 1)] >> (4 * (c & 1))) & 15u;
      const uint32_t sb = qx_scales[scale_offset(prow, c / kBlock, K, qx_layout)];
      v[u] = __fsub_rn(xv, dequant(code, e4m3_to_f32(sb), st_x));
    }
  }
  float am = 0.0f;
#pragma unroll
  for (int u = 0; u < 16; ++u) am = fmaxf(am, fabsf(v[u]));
  const BlockScale bs = block_scale(am, st_r);
  const uint32_t lo = encode8(v, bs.s_dec), hi = encode8(v + 8, bs.s_dec);
  if (prow < r_rows)
    *reinterpret_cast<uint2*>(r_codes + prow * (width / 2) + blk * 8) = make_uint2(lo, hi);
  if (r_layout == 1 || prow < r_rows)
    r_scales[scale_offset(prow, blk, width, r_layout)] = static_cast<uint8_t>(bs.sb);
}

__global__ void sel_tensor_scale_kernel(const float* __restrict__ colamax, int64_t K,
                                        const int32_t* __restrict__ sel, int64_t n_sel,
                                        float* __restrict__ s_t) {
  const int e = blockIdx.x;
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < n_sel; j += blockDim.x) {
    const int64_t c = sel[e * n_sel + j];
    if (c >= 0 && c < K) m = fmaxf(m, colamax[e * K + c]);
  }
  m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));
  __shared__ float wm[32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r = fmaxf(r, wm[i]);
    s_t[e] = __fdiv_rn(r, kTensorScaleDiv);
  }
}

// One thread per (weight row, 16-block of the gathered width).
// grid.x = E*N rows, grid.y = ceil(width/16 / 128).
__global__ void __launch_bounds__(kGThreads)
weight_gather_kernel(const uint16_t* __restrict__ w, int64_t N, int64_t K, int64_t ldw,
                     const int32_t* __restrict__ sel, int64_t n_sel, int64_t width,
                     const float* __restrict__ s_t, uint8_t* __restrict__ codes,
                     uint8_t* __restrict__ scales, int layout) {
  const int64_t row = blockIdx.x;                 // e * N + n
  const int64_t blk = static_cast<int64_t>(blockIdx.y) * kGThreads + threadIdx.x;
  if (blk * kBlock >= width) return;
  const int64_t e = row / N;
  const int32_t* s = sel + e * n_sel;
  const uint16_t* wr = w + e * N * ldw + (row - e * N) * ldw;
  float v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int64_t j = blk * kBlock + u;
    const int64_t c = j < n_sel ? s[j] : -1;
    v[u] = (c >= 0 && c < K) ? bf16_bits_to_f32(wr[c]) : 0.0f;
  }
  float am = 0.0f;
#pragma unroll
  for (int u = 0; u < 16; ++u) am = fmaxf(am, fabsf(v[u]));
  const BlockScale bs = block_scale(am, s_t[e]);
  const uint32_t lo = encode8(v, bs.s_dec), hi = encode8(v + 8, bs.s_dec);
  *reinterpret_cast<uint2*>(codes + row * (width / 2) + blk * 8) = make_uint2(lo, hi);
  scales[scale_offset(row, blk, width, layout)] = static_cast<uint8_t>(bs.sb);
}

// ---------------------------------------------------------------------------
// weight fake quantization (W4A16 trainer side)
// ---------------------------------------------------------------------------
// CTA: 64 rows x 64 columns of one matrix; thread t: columns 8 (t & 7), rows
// t/8 and t/8 + 32.  grid = (K/64, ceil(N/64), batch).
__global__ void __launch_bounds__(kQThreads)
weight_qdq_kernel(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                  const unsigned* __restrict__ amax_bits, uint16_t* w_out,   // w_out may alias w
                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int layout,
                  float* __restrict__ tensor_scale, unsigned* __restrict__ colamax_bits) {
  const int64_t b = blockIdx.z;
  const int t = threadIdx.x, cg = t & 7, rr = t >> 3;
  const int64_t col = static_cast<int64_t>(blockIdx.x) * 64 + 8 * cg;
  const float s_t = __fdiv_rn(__uint_as_float(amax_bits[b]), kTensorScaleDiv);
  if (tensor_scale && blockIdx.x == 0 && blockIdx.y == 0 && t == 0) tensor_scale[b] = s_t;
  uint32_t cmax[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t n = static_cast<int64_t>(blockIdx.y) * 64 + rr + 32 * i;
    const bool live = n < N;
    const int64_t off = (b * N + n) * ldw + col;
    float f[8];
    if (live) {
      unpack_bf16x8(*reinterpret_cast<const uint4*>(w + off), f);   // coherent load: w may alias w_out
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = 0.0f;
    }
    float am = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      am = fmaxf(am, fabsf(f[j]));
      cmax[j] = max(cmax[j], __float_as_uint(fabsf(f[j])));
    }
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
    const BlockScale bs = block_scale(am, s_t);
    const uint32_t q = encode8(f, bs.s_dec);
    const int64_t qrow = b * N + n;
    if (live) {
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float d0 = dequant((q >> (8 * j)) & 15u, bs.sbv, s_t);
        const float d1 = dequant((q >> (8 * j + 4)) & 15u, bs.sbv, s_t);
        const uint32_t b0 = __bfloat16_as_ushort(__float2bfloat16_rn(d0));
        const uint32_t b1 = __bfloat16_as_ushort(__float2bfloat16_rn(d1));
        o[j] = b0 | (b1 << 16);
      }
      *reinterpret_cast<uint4*>(w_out + off) = make_uint4(o[0], o[1], o[2], o[3]);
      if (codes) *reinterpret_cast<uint32_t*>(codes + qrow * (K / 2) + col / 2) = q;
    }
    // rows past N belong to the next matrix: only live rows write (the caller
    // zero-fills the padding of a tiled scale buffer beforehand)
    if (scales && (cg & 1) == 0 && live)
      scales[scale_offset(qrow, col / kBlock, K, layout)] = static_cast<uint8_t>(bs.sb);
  }
  if (colamax_bits == nullptr) return;
  __shared__ uint32_t cm[32][65];
#pragma unroll
  for (int j = 0; j < 8; ++j) cm[rr][8 * cg + j] = cmax[j];
  __syncthreads();
  if (t < 64) {
    uint32_t m = 0;
    for (int r = 0; r < 32; ++r) m = max(m, cm[r][t]);
    if (m) atomicMax(colamax_bits + b * K + blockIdx.x * 64 + t, m);
  }
}

// ---------------------------------------------------------------------------
// element converters and the bounded-wait probe
// ---------------------------------------------------------------------------
__global__ void encode_kernel(const float* __restrict__ in, uint8_t* __restrict__ out, int64_t n,
                              int which) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = in[i];
  if (which == 0) {
    float q[8] = {v, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    out[i] = static_cast<uint8_t>(e2m1x8(q) & 15u);
  } else {
    out[i] = static_cast<uint8_t>(f32_to_e4m3(v));
  }
}

__global__ void wait_probe_kernel(uint64_t limit_ns, unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) mbar_init(&bar, 1);
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, limit_ns);   // nothing ever arrives
  __syncthreads();
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                        const RowGroups& g, unsigned* amax_bits, cudaStream_t s,
                        int32_t batch, int64_t mat_stride) {
  const int64_t tiles = max_tiles(g, rows);
  if (tiles == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(K / kQCols), static_cast<unsigned>(tiles), static_cast<unsigned>(batch));
  amax_kernel<<<grid, kQThreads, 0, s>>>(x, K, ldx, g, mat_stride, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_group_tiles(const int64_t* off, int32_t E, int32_t* tile_start, cudaStream_t s) {
  group_tiles_kernel<<<1, 32, 0, s>>>(off, E, tile_start);
  return cudaGetLastError();
}

cudaError_t launch_quant_score(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                               const RowGroups& g, const float* amax, int64_t codes_rows,
                               uint8_t* codes, uint8_t* scales, int layout, float* tensor_scale,
                               double* part_sum, float* part_max, cudaStream_t s) {
  const int64_t tiles = max_tiles(g, rows);
  if (tiles == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(K / kQCols), static_cast<unsigned>(tiles));
  quant_score_kernel<<<grid, kQThreads, 0, s>>>(x, K, ldx, g, amax, codes_rows, codes, scales,
                                                layout, tensor_scale, part_sum, part_max);
  return cudaGetLastError();
}

cudaError_t launch_score_reduce(const double* part_sum, const float* part_max, int64_t K,
                                const RowGroups& g, int64_t tiles, double* score, float* colamax,
                                float* tensor_scale_empty, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((K + 255) / 256), static_cast<unsigned>(g.E));
  score_reduce_kernel<<<grid, 256, 0, s>>>(part_sum, part_max, K, g, tiles, score, colamax,
                                           tensor_scale_empty);
  return cudaGetLastError();
}

cudaError_t launch_residual_gather(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                                   const RowGroups& g, int64_t prows,
                                   const uint8_t* qx_codes, const uint8_t* qx_scales, int qx_layout,
                                   const float* qx_st, const int32_t* sel, int64_t n_sel,
                                   int64_t width, const float* r_st, uint8_t* r_codes,
                                   uint8_t* r_scales, int r_layout, cudaStream_t s) {
  (void)rows;
  if (width == 0 || prows == 0) return cudaSuccess;
  const int64_t nblk = width / kBlock;
  // rows of the scale buffer are padded to 128 for the tiled layout
  const int64_t grid_rows = r_layout == 1 ? (prows + kTileRows - 1) / kTileRows * kTileRows : prows;
  dim3 grid(static_cast<unsigned>(grid_rows), static_cast<unsigned>((nblk + kGThreads - 1) / kGThreads));
  residual_gather_kernel<<<grid, kGThreads, 0, s>>>(x, K, ldx, g, qx_codes, qx_scales, qx_layout,
                                                    qx_st, sel, n_sel, width, r_st, r_codes,
                                                    r_scales, r_layout, prows);
  return cudaGetLastError();
}

cudaError_t launch_sel_tensor_scale(const float* colamax, int64_t K, const int32_t* sel,
                                    int64_t n_sel, int32_t E, float* s_t, cudaStream_t s) {
  sel_tensor_scale_kernel<<<E, 512, 0, s>>>(colamax, K, sel, n_sel, s_t);
  return cudaGetLastError();
}

cudaError_t launch_weight_gather(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t E,
                                 const int32_t* sel, int64_t n_sel, int64_t width,
                                 const float* s_t, uint8_t* codes, uint8_t* scales, int layout,
                                 cudaStream_t s) {
  if (width == 0) return cudaSuccess;
  const int64_t nblk = width / kBlock;
  dim3 grid(static_cast<unsigned>(E * N), static_cast<unsigned>((nblk + kGThreads - 1) / kGThreads));
  weight_gather_kernel<<<grid, kGThreads, 0, s>>>(w, N, K, ldw, sel, n_sel, width, s_t, codes,
                                                  scales, layout);
  return cudaGetLastError();
}

cudaError_t launch_weight_qdq(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t batch,
                              const unsigned* amax_bits, uint16_t* w_out, uint8_t* codes,
                              uint8_t* scales, int layout, float* tensor_scale,
                              unsigned* colamax_bits, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(K / 64), static_cast<unsigned>((N + 63) / 64),
            static_cast<unsigned>(batch));
  weight_qdq_kernel<<<grid, kQThreads, 0, s>>>(w, N, K, ldw, amax_bits, w_out, codes, scales,
                                               layout, tensor_scale, colamax_bits);
  return cudaGetLastError();
}

cudaError_t launch_encode(const float* in, uint8_t* out, int64_t n, int which, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  encode_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(in, out, n, which);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint64_t limit_ns, unsigned* err, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace nvfp4
