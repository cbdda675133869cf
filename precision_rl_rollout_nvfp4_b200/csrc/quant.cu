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
// tile.  Thread t handles 8 consecutive columns (one 16-byte load) of 4
// consecutive rows; the two halves of a 16-element block sit in threads t and
// t^1 and meet through one shfl.xor.  The channel score of the tile's 128 rows
// is their fp64 sum in row order (see quant_score2_kernel).
#include "kernels.h"
#include "topk.cuh"

namespace nvfp4 {
namespace {

constexpr int kQThreads = 256;
constexpr int kQCols = 64;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------------------
// amax
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQThreads)
amax_kernel(const uint16_t* __restrict__ x, int64_t K, int64_t ldx, RowGroups g,
            int64_t mat_stride, unsigned* __restrict__ amax_bits) {
  pdl_wait();
  pdl_launch_dependents();
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
    if (row < ti.row_end && NV_IDX(col + 8 <= K)) {
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
    if (r && NV_IDX(ti.e < g.E)) atomicMax(amax_bits + ti.e, r << 16);   // |bf16| bits order like their values
  }
}

__global__ void group_tiles_kernel(const int64_t* __restrict__ off, int32_t E,
                                   int32_t* __restrict__ tile_start) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x != 0) return;
  int32_t acc = 0, pacc = 0;
  int32_t* pair_start = tile_start + E + 1;
  for (int e = 0; e < E; ++e) {
    tile_start[e] = acc;
    pair_start[e] = pacc;
    const int64_t m = off[e + 1] - off[e];
    const int32_t t = static_cast<int32_t>((m + kTileRows - 1) / kTileRows);
    acc += t;
    pacc += (t + 1) / 2;                           // 256-row tiles of the CTA-pair GEMM
  }
  tile_start[E] = acc;
  pair_start[E] = pacc;
}

// Per-CTA partial maxima of |x| for `batch` dense matrices (blockIdx.y), no
// atomics and nothing to clear beforehand: CTA i of matrix b writes
// parts[b * gridDim.x + i] (fp32 bits); the consumer takes the max of the
// partials (exact in any order).  Grid-stride over 16-byte vectors with eight
// loads in flight per thread.  The grid also clears zero_ptr[0 .. n_zero).
__global__ void __launch_bounds__(kQThreads)
amax_partial_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ldx,
                    int64_t mat_stride, unsigned* __restrict__ parts, unsigned* __restrict__ zero_ptr,
                    int n_zero) {
  pdl_wait();
  pdl_launch_dependents();
  x += blockIdx.y * mat_stride;
  {
    const int cta = blockIdx.y * gridDim.x + blockIdx.x;
    const int nthreads = gridDim.x * gridDim.y * kQThreads;
    for (int i = cta * kQThreads + threadIdx.x; i < n_zero; i += nthreads) zero_ptr[i] = 0u;
  }
  const int64_t kv = K / 8;                       // 16-byte vectors per row
  const int64_t nvec = rows * kv;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kQThreads;
  const bool flat = ldx == K;
  uint32_t m = 0;
  // vectors are visited from the end of the matrix backwards, so that its
  // first rows are the ones still in L2 when the next pass starts there
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kQThreads + threadIdx.x; v0 < nvec; v0 += 8 * stride) {
    uint4 r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t v = nvec - 1 - (v0 + u * stride);
      r[u] = make_uint4(0, 0, 0, 0);
      if (v >= 0 && NV_IDX(v < nvec)) {
        const int64_t off = flat ? v * 8 : (v / kv) * ldx + (v % kv) * 8;
        r[u] = ld_nc_v4(x + off);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t w[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t wmax[kQThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int i = 0; i < kQThreads / 32; ++i) r = max(r, wmax[i]);
    parts[blockIdx.y * gridDim.x + blockIdx.x] = r << 16;   // |bf16| bits order like their values
  }
}

// Block-wide max of n partial maxima (fp32 bits); every thread gets it.
__device__ __forceinline__ float reduce_parts(const unsigned* parts, int n, uint32_t* wscratch) {
  uint32_t m = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = max(m, __ldcg(parts + i));
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0) wscratch[threadIdx.x >> 5] = m;
  __syncthreads();
  uint32_t r = 0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r = max(r, wscratch[i]);
  __syncthreads();
  return __uint_as_float(r);
}

// ---------------------------------------------------------------------------
// quantize + residual + score partials (+ the ordered reduction of the
// partials by the last CTA of each 64-column strip of a row group)
//
// Thread t of the 256 owns 8 consecutive columns (one 16-byte load) of the 4
// consecutive rows 4 (t/8) .. 4 (t/8) + 3 of the tile; the two halves of a
// 16-element block sit in threads t and t^1.
//
// The tile's rows are one 128-row chunk of the channel score, whose chunk sum
// is defined as the fp64 sum of the chunk's |dX_ij| added one by one in row
// order.  The threads write the tile's |dX| (fp32) to shared memory; then
// four threads per column each take 32 rows.  When the nonzero values of a
// column span at most 22 binades (largest biased exponent minus smallest, a
// subnormal counted as exponent 1), every partial sum of them is a multiple
// of the last bit of the smallest and stays below 2^53 of those units, so
// every fp64 addition is exact and any order of addition gives the row-order
// result: the four 32-row sums are added.  A column whose values span more
// (a value far below the others; rare) is summed again by one thread over
// the 128 rows in order.
// ---------------------------------------------------------------------------
constexpr int kSpanExact = 22;
// strips one CTA may complete: the in-kernel strip totals serve dense X
// (one group), whose strips all complete in the last row tile, where a CTA
// takes at most ceil(K/64 / grid) <= 3 tiles (K <= 65472, grid >= min(work,
// 3 SMs)); a completion beyond the list would be dropped, never written
// out of bounds
constexpr int kMaxDone = 64;
// tensor scales from 2^-55 up: every nonzero block decode scale
// RN(E4M3dec(sb) s_t) >= 2^-9 2^-55 = 2^-64, so its reciprocal table entry
// serves the quotient (Markstein) and no division fallback is needed
constexpr float kFastScale = 2.7755575615628914e-17f;   // 2^-55

// E2M1 codes of 16 values with block amax am under a table of tensor scale
// >= kFastScale: the block scale by Markstein's correction of am / d, then
// the element quotients formed negated from the reciprocal table (c = -q,
// see the quantize pass) and every code's sign bit flipped back.  Returns
// the E4M3 block scale byte.
__device__ __forceinline__ uint32_t encode16_fast(const float* v, float am, const ScaleTable& T, uint32_t& lo,
                                                  uint32_t& hi) {
  const float q0 = __fmul_rn(am, T.rcp_d);
  const float rr = __fmaf_rn(-q0, T.d, am);
  const uint32_t sb = f32_to_e4m3(__fmaf_rn(rr, T.rcp_d, q0));
  const float ny = -T.rcp[sb], sd = T.sdec[sb];
  const uint64_t ny2 = f2_pack(ny, ny), sd2 = f2_pack(sd, sd);
  uint64_t c2[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint64_t x2 = f2_pack(v[2 * j], v[2 * j + 1]);
    const uint64_t a = f2_mul(x2, ny2);
    c2[j] = f2_fma(f2_fma(a, sd2, x2), ny2, a);
  }
  lo = e2m1x8_f2(c2) ^ 0x88888888u;
  hi = e2m1x8_f2(c2 + 4) ^ 0x88888888u;
  return sb;
}

// Optional top-k% selection fused into the quantize pass's tail.
struct SelectOut {
  int64_t n_sel;            // < 0: no selection
  uint8_t* mask;
  int32_t* sel;
  float* s_t;               // residual tensor scale
  unsigned* strips_done;    // zero on entry, left zero
};

// ---------------------------------------------------------------------------
// The quantize + residual + score pass (persistent).  The grid is a few
// CTAs per SM; CTA b takes the (row tile, 64-column strip) pairs b, b + grid,
// ... in row-tile-major order, so the whole grid sweeps X from its first rows
// to its last (the amax pass walks X backwards, so the first rows are still
// in L2 here).  Each thread copies the 4 rows x 16 bytes it will quantize in
// the next tile into a shared double buffer with cp.async while it works on
// the current one, so the loads of one tile overlap the arithmetic of the
// other and need no barrier (every thread reads only its own copies).  The
// tensor amax, s_t and the block-scale table are formed once per CTA (again
// only when an MoE row group changes).  The tile's channel score is the exact
// two-level reduction or the row-order sum described above.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

// The last CTA to finish a column strip of a row group: the chunk-order
// totals of the strip's partial sums and maxima (staged through the idle
// partial buffers ps / pm, 32 chunks at a time), and, when a selection is
// fused, the top-k% selection by the last strip overall.  Kept out of line:
// it runs once per strip and should not weigh on the registers of the
// tile loop.
template <bool SCORES>
static __device__ __noinline__ void finish_strip(int64_t t0, int64_t t1, unsigned* counter, double* ps, float* pm,
                                                 const double* part_sum, const float* part_max, int64_t K,
                                                 int64_t col0, double* score, float* colamax, int e, int E,
                                                 SelectOut sel_out, int64_t n_strips, uint8_t* keys, bool* s_last) {
  constexpr int kGroups = kTileRows / 4;
  const int t = threadIdx.x;
  __threadfence();
  double total_s = 0.0;
  float tmax = 0.0f;
  for (int64_t c0 = t0; c0 < t1; c0 += kGroups) {
    const int nt = static_cast<int>(t1 - c0 < kGroups ? t1 - c0 : kGroups);
    __syncthreads();
    for (int k = t; k < nt * kQCols; k += kQThreads) {
      const int tt = k / kQCols, cc = k % kQCols;
      if (SCORES) ps[k] = __ldcg(part_sum + (c0 + tt) * K + col0 + cc);
      pm[k] = __ldcg(part_max + (c0 + tt) * K + col0 + cc);
    }
    __syncthreads();
    if (t < kQCols) {
      for (int tt = 0; tt < nt; ++tt) {          // chunk order
        if (SCORES) total_s += ps[tt * kQCols + t];
        tmax = fmaxf(tmax, pm[tt * kQCols + t]);
      }
    }
  }
  if (t < kQCols && NV_IDX(e < E && col0 + t < K)) {
    if (SCORES) score[static_cast<int64_t>(e) * K + col0 + t] = total_s;
    colamax[static_cast<int64_t>(e) * K + col0 + t] = tmax;
  }
  if (t == 0) *counter = 0;                      // ready for the next call
  __syncthreads();                               // staging buffers free before the next tile
  if (SCORES && sel_out.n_sel >= 0) {
    // the last strip to finish selects the channels; its scores were
    // published like the partials (barrier, then one thread's fence before
    // the counter moves)
    if (t == 0) {
      __threadfence();
      *s_last = atomicAdd(sel_out.strips_done, 1u) == static_cast<unsigned>(n_strips - 1);
    }
    __syncthreads();
    if (*s_last) {
      __threadfence();
      // the (now idle) tile buffers and partial-sum buffer are its scratch
      static_assert(2 * kTileRows * kQCols * 2 == kSelScratchBytes && kTileRows * kQCols * 4 == kSelScratchBytes,
                    "selection scratch: two 32 KB buffers");
      topk_select(score, colamax, K, sel_out.n_sel, sel_out.mask, sel_out.sel, sel_out.s_t, 0, keys,
                  reinterpret_cast<uint8_t*>(ps));
      if (t == 0) *sel_out.strips_done = 0;
    }
  }
}

// With sel_out.n_sel >= 0 (dense only) the CTA that completes the last
// column strip also runs the top-k% selection over the finished scores.
template <bool SCORES>
__global__ void __launch_bounds__(kQThreads, 3)
quant_score2_kernel(const uint16_t* __restrict__ x, int64_t K, int64_t ldx, RowGroups g,
                    const float* __restrict__ amax, const unsigned* __restrict__ amax_parts,
                    int n_parts, int64_t codes_rows,
                    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int layout,
                    float* __restrict__ tensor_scale, double* __restrict__ part_sum,
                    float* __restrict__ part_max, unsigned* __restrict__ strip_count,
                    double* __restrict__ score, float* __restrict__ colamax, SelectOut sel_out) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int kGroups = kTileRows / 4;
  extern __shared__ __align__(16) uint8_t q2_dyn[];                // 2 x 16 KB tile buffers
  uint16_t (*xbuf)[kTileRows][kQCols] = reinterpret_cast<uint16_t (*)[kTileRows][kQCols]>(q2_dyn);
  // 32 KB: with scores the tile's |dX| (fp32 [128][64]); without, the
  // per-thread column maxima [32][64]; after a strip the staging of its
  // partials (finish_strip)
  __shared__ __align__(16) uint8_t red[kTileRows * kQCols * 4];
  float (*dxs)[kQCols] = reinterpret_cast<float (*)[kQCols]>(red);
  float (*gmax)[kQCols] = reinterpret_cast<float (*)[kQCols]>(red);
  __shared__ __align__(16) double qsum[4][kQCols];
  __shared__ __align__(16) float qmax[4][kQCols];
  __shared__ __align__(16) uint32_t qmin[4][kQCols];
  __shared__ __align__(16) uint8_t s_sb[2][kTileRows][kQCols / kBlock];
  __shared__ uint32_t wscratch[kQThreads / 32];
  __shared__ bool s_last;
  // (group, strip) of the strips this CTA completed: their chunk-order
  // totals are formed after the tile loop (a call inside it would make the
  // loop spill its live values around the call)
  __shared__ int2 s_done[kMaxDone];
  __shared__ int s_ndone;
  __shared__ ScaleTable T;
  __shared__ float4 T4[128];                       // {sbv, sdec, -rcp} per scale code
  const int t = threadIdx.x, cg = t & 7, grp = t >> 3;
  const int64_t n_strips = K / kQCols;
  const int64_t row_tiles = g.off == nullptr ? (g.M + kTileRows - 1) / kTileRows : g.tile_start[g.E];
  const int64_t total = row_tiles * n_strips;
  // the tensor amax once per CTA (dense: the max of the partial maxima)
  const float a_dense = (g.off == nullptr && n_parts > 0) ? reduce_parts(amax_parts, n_parts, wscratch) : 0.0f;
  int cur_e = -1;
  float s_t = 0.0f, dd = 0.0f, rcpd = 0.0f;
  bool fast = false;

  // tile and strip counts fit in 32 bits: 32-bit division per tile
  const uint32_t ns32 = static_cast<uint32_t>(n_strips);
  auto prefetch = [&](int64_t idx, int b) {
    const uint32_t i32 = static_cast<uint32_t>(idx);
    const int64_t rt = i32 / ns32, strip = i32 % ns32;
    const TileInfo ti = tile_info(g, rt);
    const int64_t col = strip * kQCols + 8 * cg;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * grp + i;
      const int64_t row = ti.row0 + r;
      const bool ok = ti.valid && row < ti.row_end && NV_IDX(col + 8 <= K);
      cp_async16_zfill(smem_u32(&xbuf[b][r][8 * cg]), ok ? static_cast<const void*>(x + row * ldx + col)
                                                           : static_cast<const void*>(x), ok);
    }
    cp_async_commit();
  };

  int64_t idx = blockIdx.x;
  if (idx < total) prefetch(idx, 0);
  if (t == 0) s_ndone = 0;                         // first read after the table build's barriers
  for (int it = 0; idx < total; ++it, idx += gridDim.x) {
    const int b = it & 1;
    const int64_t nidx = idx + gridDim.x;
    if (nidx < total) {
      prefetch(nidx, b ^ 1);
      cp_async_wait<1>();                          // this thread's copies of the current tile landed
    } else {
      cp_async_wait<0>();
    }
    const int64_t tile = static_cast<uint32_t>(idx) / ns32, strip = static_cast<uint32_t>(idx) % ns32;
    const TileInfo ti = tile_info(g, tile);
    if (ti.e != cur_e) {                           // uniform over the CTA
      const float a = g.off == nullptr ? (n_parts > 0 ? a_dense : amax[0]) : amax[ti.e];
      s_t = __fdiv_rn(a, kTensorScaleDiv);
      __syncthreads();                             // nobody reads the previous group's table any more
      build_scale_table(T, s_t, t);
      if (t < 128) T4[t] = make_float4(T.sbv[t], T.sdec[t], -T.rcp[t], 0.0f);   // this thread's own entries
      __syncthreads();
      cur_e = ti.e;
      fast = s_t >= kFastScale;
      dd = T.d;
      rcpd = T.rcp_d;
    }
    const int64_t col0 = strip * kQCols;
    const int64_t col = col0 + 8 * cg;
    if (strip == 0 && t == 0 && (g.off == nullptr ? tile == 0 : tile == g.tile_start[ti.e]))
      tensor_scale[ti.e] = s_t;
    uint8_t* code_base = codes + tile * kTileRows * (K / 2) + col / 2;
    float mx[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) mx[j] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * grp + i;
      const int64_t prow = tile * kTileRows + r;
      const uint4 rv = *reinterpret_cast<const uint4*>(&xbuf[b][r][8 * cg]);
      const uint32_t wv[4] = {rv.x, rv.y, rv.z, rv.w};
      uint64_t x2[4];
      uint32_t mbits = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x2[j] = bf16x2_to_f2(wv[j]);
        mbits = __vmaxu2(mbits, wv[j] & 0x7FFF7FFFu);
      }
      float am = __uint_as_float(max(mbits & 0xFFFFu, mbits >> 16) << 16);
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
      uint32_t packed, sb;
      float sbv;
      if (fast) {
        // every block decode scale is 0 or >= 2^-64: the quotients need no
        // division fallback.  sb = E4M3(RN(am / d)) by Markstein's
        // correction; the element quotients are formed negated, c = -q with
        // q = RN(x / sdec) (a = RN(-x y) = -q0, the remainder x - q0 sdec
        // is exact, c = RN(-(r y + q0))), which also gives signed zeros the
        // right sign: E2M1(c) with every sign bit flipped is E2M1(q).
        const float q0 = __fmul_rn(am, rcpd);
        const float rr = __fmaf_rn(-q0, dd, am);
        sb = f32_to_e4m3(__fmaf_rn(rr, rcpd, q0));
        const float4 tv = T4[sb];
        const uint64_t ny2 = f2_pack(tv.z, tv.z), sd2 = f2_pack(tv.y, tv.y);
        uint64_t c2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t a = f2_mul(x2[j], ny2);
          c2[j] = f2_fma(f2_fma(a, sd2, x2[j]), ny2, a);
        }
        packed = e2m1x8_f2(c2) ^ 0x88888888u;
        sbv = tv.x;
      } else {
        const BlockQ bq = block_q(am, T);
        uint64_t q2[4];
        block_quotients(x2, bq, q2);
        packed = e2m1x8_f2(q2);
        sb = bq.sb;
        sbv = bq.sbv;
      }
      const uint64_t sbv2 = f2_pack(sbv, sbv);
      float dv[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // dX = RN(x - RN(p s_t)) with p = E2M1dec E4M3dec exact (scalar
        // product and difference: two roundings)
        float p0, p1, x0, x1;
        f2_unpack(f2_mul(e2m1x2_to_f2((packed >> (8 * j)) & 0xFFu), sbv2), p0, p1);
        f2_unpack(x2[j], x0, x1);
        const float d0 = fabsf(__fsub_rn(x0, __fmul_rn(p0, s_t)));
        const float d1 = fabsf(__fsub_rn(x1, __fmul_rn(p1, s_t)));
        dv[2 * j] = d0;
        dv[2 * j + 1] = d1;
        if (!SCORES) {
          mx[2 * j] = fmaxf(mx[2 * j], d0);
          mx[2 * j + 1] = fmaxf(mx[2 * j + 1], d1);
        }
      }
      if (SCORES) {
        // columns 8 cg + 4 h + e sit at position 32 h + 4 cg + e of the row:
        // each 16-byte store of 8 threads covers 128 contiguous bytes
        *reinterpret_cast<float4*>(&dxs[r][4 * cg]) = make_float4(dv[0], dv[1], dv[2], dv[3]);
        *reinterpret_cast<float4*>(&dxs[r][32 + 4 * cg]) = make_float4(dv[4], dv[5], dv[6], dv[7]);
      }
      if (prow < codes_rows && NV_IDX(col + 8 <= K))
        *reinterpret_cast<uint32_t*>(code_base + static_cast<uint32_t>(r) * static_cast<uint32_t>(K / 2)) = packed;
      if ((cg & 1) == 0) s_sb[b][r][cg >> 1] = static_cast<uint8_t>(sb);
    }
    if (!SCORES && part_max != nullptr) {
      *reinterpret_cast<float4*>(&gmax[grp][8 * cg]) = make_float4(mx[0], mx[1], mx[2], mx[3]);
      *reinterpret_cast<float4*>(&gmax[grp][8 * cg + 4]) = make_float4(mx[4], mx[5], mx[6], mx[7]);
    }
    __syncthreads();
    // the tile's block scales leave from shared memory: one 512-byte atom
    // (tiled layout: 32 threads x 16 bytes) or one 4-byte word per row
    if (layout == 1) {
      if (t < 32) {
        const int64_t off = (tile * ((K + 63) / 64) + (col0 >> 6)) * 512 + 16 * t;
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(&s_sb[b][0][0]);
        if (NV_IDX(off + 16 <= scale_extent(codes_rows, K, layout, kBlock)))
          *reinterpret_cast<uint4*>(scales + off) = make_uint4(sw[t], sw[t + 32], sw[t + 64], sw[t + 96]);
      }
    } else if (t < kTileRows) {
      const int64_t prow = tile * kTileRows + t;
      const int64_t off = prow * (K / kBlock) + (col0 >> 4);
      if (prow < codes_rows && NV_IDX(off + 4 <= scale_extent(codes_rows, K, layout, kBlock)))
        *reinterpret_cast<uint32_t*>(scales + off) = *reinterpret_cast<const uint32_t*>(&s_sb[b][t][0]);
    }
    if (part_max == nullptr) continue;
    {
      // column c, rows 32 q4 .. 32 q4 + 31 (scores: the fp64 sum, the
      // smallest nonzero |dX| as bits - 1 and the maximum; else the maximum
      // of the per-thread maxima)
      int c = t & (kQCols - 1);
      const int q4 = t >> 6;
      double sum = 0.0;
      float m = 0.0f;
      uint32_t lo = 0xFFFFFFFFu;
      if (SCORES) {
        const int pos = c;                         // this thread reads position pos of the rows
        c = 8 * ((pos & 31) >> 2) + 4 * (pos >> 5) + (pos & 3);   // ... which holds column c
#pragma unroll 8
        for (int r = 32 * q4; r < 32 * q4 + 32; ++r) {
          const float v = dxs[r][pos];
          sum += static_cast<double>(v);
          lo = min(lo, __float_as_uint(v) - 1u);
          m = fmaxf(m, v);
        }
      } else {
#pragma unroll
        for (int gi = 8 * q4; gi < 8 * q4 + 8; ++gi) m = fmaxf(m, gmax[gi][c]);
      }
      if (SCORES) {
        qsum[q4][c] = sum;
        qmin[q4][c] = lo;
      }
      qmax[q4][c] = m;
    }
    __syncthreads();
    int wide = 0;
    if (t < kQCols) {
      double part = 0.0;
      float m = 0.0f;
      uint32_t lo = 0xFFFFFFFFu;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        if (SCORES) {
          part += qsum[q4][t];
          lo = min(lo, qmin[q4][t]);
        }
        m = fmaxf(m, qmax[q4][t]);
      }
      if (SCORES && lo != 0xFFFFFFFFu) {
        const int e_hi = static_cast<int>(__float_as_uint(m) >> 23);
        const int e_lo = max(static_cast<int>((lo + 1u) >> 23), 1);
        wide = e_hi - e_lo > kSpanExact;
      }
      if (NV_IDX(tile < row_tiles && col0 + t < K)) {
        if (SCORES && !wide) part_sum[tile * K + col0 + t] = part;
        part_max[tile * K + col0 + t] = m;
      }
    }
    // columns whose values span more than kSpanExact binades: the row-order
    // sum itself, by the column's own thread from the |dX| tile (rows past
    // the end hold 0), then a barrier before the next tile overwrites it
    if (SCORES && __syncthreads_or(wide)) {
      if (wide) {
        const int pos = 32 * ((t >> 2) & 1) + 4 * (t >> 3) + (t & 3);   // column t's position
        double chain = 0.0;
        for (int r = 0; r < kTileRows; ++r) chain += static_cast<double>(dxs[r][pos]);
        if (NV_IDX(tile < row_tiles && col0 + t < K)) part_sum[tile * K + col0 + t] = chain;
      }
      __syncthreads();
    }
    if (strip_count == nullptr) continue;
    __syncthreads();
    const int64_t t0 = g.off == nullptr ? 0 : g.tile_start[ti.e];
    const int64_t t1 = g.off == nullptr ? row_tiles : g.tile_start[ti.e + 1];
    unsigned* counter = strip_count + static_cast<int64_t>(ti.e) * n_strips + strip;
    if (t == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(counter, 1u);
      if (prev == static_cast<unsigned>(t1 - t0 - 1) && s_ndone < kMaxDone)
        s_done[s_ndone++] = make_int2(ti.e, static_cast<int>(strip));
    }
  }
  // the strips this CTA completed, after its last tile (with a selection
  // fused, the CTA that completes the last strip overall also selects)
  __syncthreads();
  const int nd = strip_count != nullptr ? s_ndone : 0;
  for (int i = 0; i < nd; ++i) {
    const int e = s_done[i].x;
    const int64_t strip = s_done[i].y;
    const int64_t t0 = g.off == nullptr ? 0 : g.tile_start[e];
    const int64_t t1 = g.off == nullptr ? row_tiles : g.tile_start[e + 1];
    finish_strip<SCORES>(t0, t1, strip_count + static_cast<int64_t>(e) * n_strips + strip,
                         reinterpret_cast<double*>(red),
                         reinterpret_cast<float*>(red + kGroups * kQCols * sizeof(double)), part_sum, part_max, K,
                         strip * kQCols, score, colamax, e, g.E, sel_out, n_strips, q2_dyn, &s_last);
  }
  cp_async_wait<0>();
}

__global__ void score_reduce_kernel(const double* __restrict__ part_sum,
                                    const float* __restrict__ part_max, int64_t K, RowGroups g,
                                    int64_t tiles, double* __restrict__ score,
                                    float* __restrict__ colamax, float* __restrict__ st_empty) {
  pdl_wait();
  pdl_launch_dependents();
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
constexpr int kGThreads = 256;

// Second-pass gather + quantize, shared by the residual and the weight side.
// A CTA (256 threads) takes tiles of 16 rows x 256 gathered channels:
//   phase 1: every thread reads the 8 channels it gathers straight from
//            sel[j0 + lane + 32 u] and then gathers 16 values (rows 2w and
//            2w+1, those channels), all loads in flight at once; the residual
//            side recomputes dX = x - DQ(Q(x)) from X, the code nibble and
//            the block scale byte of Q(X) (decoded through small shared
//            tables); values go to shared memory;
//   phase 2: thread = one 16-block (row, block): block scale, codes, stores.
// Tiles are visited grid-stride.  With fuse_scale (one weight) the W_sel
// tensor scale max_{j in sel} colamax_j / 2688 is reduced during the first
// tile, its loads issued beside that tile's gather loads; CTA 0 publishes it.
//
// MODE 0: W_sel from the bf16 weight `src`;
// MODE 1: the residual dX_sel from X (`src`) and Q(X) (`qx_*`);
// MODE 2: W_sel from the NVFP4 weight alone: the gathered values are
//         DQ(Q(W)) decoded from its codes and scales (`qx_*`, tensor scale
//         qx_st[e]); `src` is unused and colamax holds max_n |DQ(Q(W))_nj|.
constexpr int kGRows = 16, kGCols = 256;

// Arguments of one second-pass gather (see gather_quant_body).
struct GatherArgs {
  const uint16_t* src;
  int64_t K, ld;
  RowGroups g;
  int64_t N_per_group;
  const uint8_t* qx_codes;
  const uint8_t* qx_scales;
  int qx_layout;
  const float* qx_st;
  const int32_t* sel;
  int64_t n_sel, width;
  const float* colamax;
  int fuse_scale;
  float* out_st;
  uint8_t* out_codes;
  uint8_t* out_scales;
  int out_layout;
  int64_t out_rows, grid_rows;
};

struct GatherSmem {
  __align__(16) float s_val[kGRows][kGCols + 4];
  float s_e2m1[16];                                // E2M1 value of every code
  float s_e4m3[128];                               // E4M3 value of every scale byte
  float s_wm[kGThreads / 32];
  ScaleTable T;
};

// The residual's tiles run from the last rows of X to the first (the
// quantize pass that precedes them ends on the last rows, which are then
// still in L2); the weight's in order.
template <int MODE>
__device__ __forceinline__ void gather_quant_body(const GatherArgs& A, GatherSmem& sm, int cta, int ncta) {
  constexpr bool RESIDUAL = MODE == 1, FP4 = MODE == 2, CODES = MODE != 0;
  const uint16_t* __restrict__ src = A.src;
  const int64_t K = A.K, ld = A.ld, N_per_group = A.N_per_group, n_sel = A.n_sel, width = A.width;
  const RowGroups& g = A.g;
  const uint8_t* __restrict__ qx_codes = A.qx_codes;
  const uint8_t* __restrict__ qx_scales = A.qx_scales;
  const int qx_layout = A.qx_layout, fuse_scale = A.fuse_scale, out_layout = A.out_layout;
  const float* __restrict__ qx_st = A.qx_st;
  const int32_t* __restrict__ sel = A.sel;
  const float* __restrict__ colamax = A.colamax;
  float* __restrict__ out_st = A.out_st;
  uint8_t* __restrict__ out_codes = A.out_codes;
  uint8_t* __restrict__ out_scales = A.out_scales;
  const int64_t out_rows = A.out_rows, grid_rows = A.grid_rows;
  float (&s_val)[kGRows][kGCols + 4] = sm.s_val;
  float* s_e2m1 = sm.s_e2m1;
  float* s_e4m3 = sm.s_e4m3;
  float* s_wm = sm.s_wm;
  ScaleTable& T = sm.T;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (CODES) {
    if (t < 16) s_e2m1[t] = e2m1_to_f32(static_cast<uint32_t>(t));
    if (t < 128) s_e4m3[t] = t < 127 ? e4m3_to_f32(static_cast<uint32_t>(t)) : 0.0f;
  }
  const bool fuse = !RESIDUAL && fuse_scale != 0;
  bool first = true;
  float fused_st = 0.0f;
  const uint32_t K32 = static_cast<uint32_t>(K);
  const int64_t row_tiles = (grid_rows + kGRows - 1) / kGRows;
  const int64_t col_tiles = (width + kGCols - 1) / kGCols;
  for (int64_t tile = cta; tile < row_tiles * col_tiles; tile += ncta) {
    const int64_t rt = RESIDUAL ? row_tiles - 1 - tile / col_tiles : tile / col_tiles;
    const int64_t r0 = rt * kGRows, j0 = (tile % col_tiles) * kGCols;
    // rows of this tile belong to one group: 16 divides 128 and N % 16 == 0
    int e;
    int64_t row_base, row_end;     // source row of r0, end of the group's rows
    bool valid;
    if (RESIDUAL) {
      const TileInfo ti = tile_info(g, r0 / kTileRows);
      e = ti.e;
      valid = ti.valid;
      row_base = ti.row0 + (r0 % kTileRows);
      row_end = ti.row_end;
    } else {
      e = static_cast<int>(r0 / N_per_group);
      valid = true;
      row_base = r0;                               // stacked weight row e*N + n
      row_end = static_cast<int64_t>(e + 1) * N_per_group;
    }
    __syncthreads();                               // previous tile done with shared memory
    // level 1: the channels this thread gathers (and the fused scale's sel share)
    const int32_t* sel_e = sel + static_cast<int64_t>(e) * n_sel;
    int32_t c[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t j = j0 + lane + 32 * u;
      c[u] = (valid && j < n_sel) ? __ldg(sel_e + j) : -1;
      if (valid && j < n_sel && !NV_IDX(c[u] >= 0 && c[u] < K)) c[u] = -1;
    }
    const bool do_fuse = fuse && first;
    int32_t fc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t jf = t + kGThreads * u;
      fc[u] = (do_fuse && jf < n_sel) ? __ldg(sel + jf) : -1;
    }
    // level 2: the values (and the fused scale's colamax share)
    const float st_x = (CODES && valid) ? qx_st[e] : 0.0f;
    const int64_t k4 = (K + 63) / 64;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = 2 * warp + rr;
      const int64_t srow = row_base + r;
      const int64_t prow = r0 + r;
      const bool live = valid && srow < row_end;
      const uint16_t* xrow = FP4 ? nullptr : src + srow * ld;
      const uint8_t* crow = CODES ? qx_codes + prow * (K / 2) : nullptr;
      const uint8_t* srow_sc = nullptr;
      if (CODES)
        srow_sc = qx_layout == 1
                      ? qx_scales + ((prow >> 7) * k4) * 512 + (prow & 31) * 16 + ((prow & 127) >> 5) * 4
                      : qx_scales + prow * (K / kBlock);
      uint32_t xb[8], cb[8], sb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool ok = live && static_cast<uint32_t>(c[u]) < K32;   // never false for a valid sel list
        const uint32_t cc = ok ? static_cast<uint32_t>(c[u]) : 0u;
        xb[u] = (ok && !FP4) ? __ldg(xrow + cc) : 0u;
        if (CODES) {
          cb[u] = ok ? __ldg(crow + (cc >> 1)) : 0u;
          const uint32_t so = qx_layout == 1 ? (cc >> 6) * 512u + ((cc >> 4) & 3u) : (cc >> 4);
          sb[u] = ok ? __ldg(srow_sc + so) : 0u;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float v = 0.0f;
        if (live && static_cast<uint32_t>(c[u]) < K32) {
          if (CODES) {
            const float q = s_e2m1[(cb[u] >> ((c[u] & 1) << 2)) & 15u];
            const float dq = __fmul_rn(__fmul_rn(q, s_e4m3[sb[u] & 127u]), st_x);
            v = FP4 ? dq : __fsub_rn(bf16_bits_to_f32(xb[u]), dq);
          } else {
            v = bf16_bits_to_f32(xb[u]);
          }
        }
        s_val[r][lane + 32 * u] = v;
      }
    }
    if (do_fuse) {
      float fm = 0.0f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (static_cast<uint32_t>(fc[u]) < K32) fm = fmaxf(fm, __ldg(colamax + fc[u]));
      for (int64_t base = t + 8 * kGThreads; base < n_sel; base += 8 * kGThreads) {   // n_sel > 2048
        int32_t cf[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t jf = base + kGThreads * u;
          cf[u] = jf < n_sel ? __ldg(sel + jf) : -1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (static_cast<uint32_t>(cf[u]) < K32) fm = fmaxf(fm, __ldg(colamax + cf[u]));
      }
      fm = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fm)));
      if (lane == 0) s_wm[warp] = fm;
      __syncthreads();
      float r = 0.0f;
#pragma unroll
      for (int k = 0; k < kGThreads / 32; ++k) r = fmaxf(r, s_wm[k]);
      fused_st = __fdiv_rn(r, kTensorScaleDiv);
      if (cta == 0 && t == 0) out_st[0] = fused_st;
    }
    first = false;
    float st = 0.0f;
    if (valid) st = RESIDUAL ? out_st[e] : (fuse ? fused_st : out_st[e]);
    build_scale_table(T, st, t);
    __syncthreads();
    // phase 2: thread = (row t/16, block t%16)
    {
      const int r = t >> 4, b = t & 15;
      const int64_t prow = r0 + r;
      const int64_t blk = j0 / kBlock + b;
      const bool in_rows = prow < out_rows;
      if (blk * kBlock < width && prow < grid_rows && (in_rows || out_layout == 1)) {
        float v[16];
        const float4* vp = reinterpret_cast<const float4*>(&s_val[r][16 * b]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 f = vp[q];
          v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
        }
        float am = 0.0f;
#pragma unroll
        for (int u = 0; u < 16; ++u) am = fmaxf(am, fabsf(v[u]));
        uint32_t lo, hi, sb;
        if (st >= kFastScale) {
          sb = encode16_fast(v, am, T, lo, hi);
        } else {
          const BlockQ bq = block_q(am, T);
          lo = encode8_q(v, bq);
          hi = encode8_q(v + 8, bq);
          sb = bq.sb;
        }
        if (in_rows && NV_IDX(blk * kBlock + 16 <= width))
          *reinterpret_cast<uint2*>(out_codes + prow * (width / 2) + blk * 8) = make_uint2(lo, hi);
        if (NV_IDX(scale_offset(prow, blk, width, out_layout) < scale_extent(grid_rows, width, out_layout, kBlock)))
          out_scales[scale_offset(prow, blk, width, out_layout)] = static_cast<uint8_t>(sb);
      }
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(kGThreads, 4) gather_quant_kernel(GatherArgs A) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ GatherSmem sm;
  gather_quant_body<MODE>(A, sm, blockIdx.x, gridDim.x);
}

// Both second passes of a RAC linear in one launch: CTAs [0, n_res) run the
// residual's tiles (MODE 1), the others the weight's (MODE 0, or 2 from the
// NVFP4 weight).
template <int WMODE>
__global__ void __launch_bounds__(kGThreads, 4) gather_pair_kernel(GatherArgs R, GatherArgs W, int n_res) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ GatherSmem sm;
  if (static_cast<int>(blockIdx.x) < n_res)
    gather_quant_body<1>(R, sm, blockIdx.x, n_res);
  else
    gather_quant_body<WMODE>(W, sm, blockIdx.x - n_res, gridDim.x - n_res);
}

// s_t[e] = RN(max_{j < n_sel} colamax[e*K + sel[e*n_sel + j]] / 2688), one CTA per group.


// W_sel, staged by rows: the gather + second quantization of the selected
// weight columns, from the bf16 weight (FP4 = false) or from its NVFP4 codes
// and scales (FP4 = true: the values are DQ(Q(W)) = RN(RN(e sbv) s_t)).
//
// A thread owns output 16-blocks and keeps their 16 channel indices in
// registers for every row of the matrix (a padded channel reads element K of
// the staged row, which is zero), so per element and row a gather is one
// shared-memory load.  With nblk = width / 16 output blocks per row:
//   nblk <= blockDim: P = blockDim / nblk threads share a block, each taking
//                     the rows slot = phase + P k (k < RPT) of a pass;
//   nblk >  blockDim: one thread per block and row (blocks t + blockDim i;
//                     blockDim = nblk rounded up to 32, at most 512).
// A pass is R = P RPT consecutive rows of one matrix (R | N when E > 1); a
// CTA takes a contiguous range of passes and double-buffers them: the next
// pass's rows are copied with cp.async (16-byte copies, 4-byte copies for
// the NVFP4 scale words) while the current pass computes.  NVFP4 rows are
// then expanded once per pass, cooperatively and coalesced, into the exact
// products E2M1dec(code) E4M3dec(scale) as f16 (at most 6 significant bits
// in [2^-10, 2688], so exact), through the hardware e2m1x2 / e4m3x2 -> f16x2
// conversions; the gather reads those and applies RN(p s_t) in fp32.
// With fuse_scale (one matrix) each CTA reduces the W_sel tensor scale
// max_{j in sel} colamax_j / 2688 from its own blocks' channels.
struct WselGeom {
  int P, RPT, R, nob;          // threads per block, rows per thread, rows per pass, blocks per thread
  uint32_t rowbytes, rawbytes; // staged row (2K + 16) and raw NVFP4 row (K/2 + K/16, to 16 bytes)
};

// Both halves of an f16 pair = E4M3dec(sb) of one scale byte (sign ignored).
__device__ __forceinline__ uint32_t dup_e4m3_to_h2(uint32_t sb) { return e4m3x2_to_h2((sb & 0x7Fu) * 0x0101u); }

// MODE 0: W_sel from bf16 rows w; MODE 1: W_sel from the NVFP4 weight
// (codes / scales / w_st); MODE 2: the residual dX_sel of dense activations:
// rows of X (w, stride ldw) and of Q(X) (codes / scales / w_st = its tensor
// scale) are staged side by side, the Q(X) rows are expanded once into the
// exact f16 products p = E2M1dec E4M3dec, and each gathered element is
// RN(x - RN(p s_t)) in fp32 (as the quantize pass forms dX); the passes of
// each CTA run from its last rows to its first.
struct RowsArgs {
  const uint16_t* w;
  int64_t ldw;
  const uint8_t* codes;
  const uint8_t* scales;
  int layout;
  const float* w_st;
  int64_t N, K;
  int32_t E;
  const int32_t* sel;
  int64_t n_sel, width;
  const float* colamax;
  int fuse_scale;
  float* out_st;
  uint8_t* out_codes;
  uint8_t* out_scales;
  int out_layout;
  WselGeom g;
  // residual of grouped rows (MoE): grp.off != nullptr; x rows are the
  // tokens of the groups, Q(X) and the output live on the groups' padded
  // 128-row tiles (prows rows)
  RowGroups grp;
  int64_t prows;
};

template <int MODE>
__device__ __forceinline__ void wsel_rows_body(const RowsArgs& A, uint8_t* ws_smem, ScaleTable& T, float* s_wm,
                                               int cta, int ncta) {
  constexpr bool FP4 = MODE == 1, RES = MODE == 2;
  const uint16_t* __restrict__ w = A.w;
  const int64_t ldw = A.ldw, N = A.N, K = A.K, n_sel = A.n_sel, width = A.width;
  const uint8_t* __restrict__ codes = A.codes;
  const uint8_t* __restrict__ scales = A.scales;
  const int layout = A.layout, fuse_scale = A.fuse_scale, out_layout = A.out_layout;
  const float* __restrict__ w_st = A.w_st;
  const int32_t E = A.E;
  const int32_t* __restrict__ sel = A.sel;
  const float* __restrict__ colamax = A.colamax;
  float* __restrict__ out_st = A.out_st;
  uint8_t* __restrict__ out_codes = A.out_codes;
  uint8_t* __restrict__ out_scales = A.out_scales;
  const WselGeom& g = A.g;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, nthr = blockDim.x;
  const uint32_t Ku = static_cast<uint32_t>(K), half = Ku / 2u;
  const int nblk = static_cast<int>(width / kBlock);
  const uint32_t R = static_cast<uint32_t>(g.R);
  // shared memory: [staged rows, 2 buffers (bf16) or 1 (NVFP4)][raw NVFP4 rows, 2 buffers]
  // (residual: bf16 rows of X, 2 buffers, then the raw Q(X) rows, 1 buffer,
  // then their expansion into exact f16 products E2M1dec E4M3dec, 1 buffer)
  const uint32_t nbuf_rows = FP4 ? 1u : 2u;
  const uint32_t raw0 = nbuf_rows * R * g.rowbytes;
  const uint32_t exp0 = raw0 + R * g.rawbytes;     // (residual only)
  // zero the tails (element K onwards) of every staged row once: copies and
  // the expansions write only elements 0 .. K-1
  for (uint32_t r = t; r < (RES ? 3u : nbuf_rows) * R; r += nthr) {
    const uint32_t ro = RES && r >= 2u * R ? exp0 + (r - 2u * R) * g.rowbytes : r * g.rowbytes;
    *reinterpret_cast<uint4*>(ws_smem + ro + 2u * Ku) = make_uint4(0u, 0u, 0u, 0u);
  }
  // this thread's blocks and row phase
  const bool shared_blocks = nblk <= nthr;
  const int phase = shared_blocks ? t / nblk : 0;
  const bool active = phase < g.P;
  const int ob0 = shared_blocks ? t % nblk : t;
  const bool grouped = RES && A.grp.off != nullptr;
  const int64_t rows = grouped ? A.prows : static_cast<int64_t>(E) * N;
  const int64_t passes = (rows + R - 1) / R;
  const int64_t p0 = static_cast<int64_t>(cta) * passes / ncta;
  const int64_t p1 = static_cast<int64_t>(cta + 1) * passes / ncta;
  // the rows of pass p (output rows R p .. R p + R - 1): its matrix or row
  // group e, the first source row and the number of real rows.  Grouped
  // passes lie inside one padded 128-row tile (R divides 128); its rows
  // past the group's end are padding (zero output).
  struct PassRows {
    int e;
    int64_t src0;
    uint32_t n;
  };
  auto pass_rows = [&](int64_t p) {
    PassRows q;
    const int64_t r0 = p * R;
    if (grouped) {
      const TileInfo ti = tile_info(A.grp, r0 >> 7);
      q.e = ti.e;
      q.src0 = ti.row0 + (r0 & 127);
      const int64_t left = ti.valid ? ti.row_end - q.src0 : 0;
      q.n = static_cast<uint32_t>(left <= 0 ? 0 : (left < R ? left : R));
    } else {
      q.e = static_cast<int>(r0 / N);
      q.src0 = r0;
      q.n = static_cast<uint32_t>(rows - r0 < R ? rows - r0 : R);
    }
    return q;
  };
  // the i-th pass of this CTA (the residual walks its range backwards)
  auto pass_of = [&](int64_t i) { return RES ? p1 - 1 - (i - p0) : i; };
  auto stage = [&](int64_t p, uint32_t b) {
    const int64_t r0 = p * R;
    const PassRows pr = pass_rows(p);
    const uint32_t nrows = pr.n;
    for (uint32_t r = 0; r < nrows; ++r) {
      if (FP4) {
        const uint32_t ro = raw0 + (b * R + r) * g.rawbytes;
        const uint8_t* src = codes + (r0 + r) * static_cast<int64_t>(half);
        for (uint32_t q = t; q < half / 16u; q += nthr) cp_async16(ws_smem + ro + 16u * q, src + 16u * q);
        for (uint32_t q = t; q < Ku / 64u; q += nthr)
          cp_async4(ws_smem + ro + half + 4u * q, scales + scale_offset(r0 + r, 4 * q, K, layout));
      }
      if (!FP4) {
        const uint32_t ro = (b * R + r) * g.rowbytes;
        const uint16_t* src = w + (pr.src0 + r) * ldw;
        for (uint32_t q = t; q < Ku / 8u; q += nthr) cp_async16(ws_smem + ro + 16u * q, src + 8u * q);
      }
    }
    cp_async_commit();
  };
  // the raw Q(X) rows of a residual pass (one buffer: filled once the
  // previous pass has expanded its rows)
  auto stage_raw = [&](int64_t p) {
    const int64_t r0 = p * R;
    const uint32_t nrows = pass_rows(p).n;
    for (uint32_t r = 0; r < nrows; ++r) {
      const uint32_t ro = raw0 + r * g.rawbytes;
      const uint8_t* src = codes + (r0 + r) * static_cast<int64_t>(half);
      for (uint32_t q = t; q < half / 16u; q += nthr) cp_async16(ws_smem + ro + 16u * q, src + 16u * q);
      for (uint32_t q = t; q < Ku / 64u; q += nthr)
        cp_async4(ws_smem + ro + half + 4u * q, scales + scale_offset(r0 + r, 4 * q, K, layout));
    }
    cp_async_commit();
  };
  // channel indices of the thread's block ob (K for padding)
  auto load_idx = [&](int e, int ob, uint32_t* c) {
    const int32_t* sel_e = sel + static_cast<int64_t>(e) * n_sel;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int64_t j = static_cast<int64_t>(ob) * kBlock + u;
      const int32_t v = j < n_sel ? __ldg(sel_e + j) : -1;
      c[u] = (v >= 0 && v < K) ? static_cast<uint32_t>(v) : Ku;
      if (j < n_sel && !NV_IDX(v >= 0 && v < K)) c[u] = Ku;
    }
  };
  uint32_t cidx[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) cidx[u] = Ku;
  if (p0 < p1) {
    stage(pass_of(p0), 0u);
    if (RES) stage_raw(pass_of(p0));
  }
  int cur_e = -1;
  float st_w = 0.0f;
  bool fastq = false;
  for (int64_t pi = p0; pi < p1; ++pi) {
    const int64_t p = pass_of(pi);
    const uint32_t b = static_cast<uint32_t>((pi - p0) & 1);
    if (pi + 1 < p1) stage(pass_of(pi + 1), b ^ 1u);
    const int64_t r0 = p * R;
    const PassRows prow = pass_rows(p);
    const int e = prow.e;
    const uint32_t nrows = prow.n;                 // real (staged) rows
    const uint32_t nout = grouped ? R : nrows;     // output rows (grouped: padding rows too)
    if (e != cur_e) {                              // uniform over the CTA; overlaps the copies in flight
      if (g.nob == 1 && active && ob0 < nblk) load_idx(e, ob0, cidx);
      float st;
      if (fuse_scale) {
        float m = 0.0f;
        for (int i = 0; i < g.nob; ++i) {
          const int ob = ob0 + i * nthr;
          if (!active || phase != 0 || ob >= nblk) continue;
          if (g.nob > 1) load_idx(e, ob, cidx);
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (cidx[u] < Ku) m = fmaxf(m, __ldg(colamax + cidx[u]));
        }
        m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));
        if (lane == 0) s_wm[warp] = m;
        __syncthreads();
        float r = 0.0f;
        for (int k = 0; k < (nthr >> 5); ++k) r = fmaxf(r, s_wm[k]);
        st = __fdiv_rn(r, kTensorScaleDiv);
        if (cta == 0 && t == 0) out_st[0] = st;
      } else {
        st = out_st[e];
      }
      __syncthreads();                             // the previous matrix's table is no longer read
      build_scale_table(T, st, t);
      fastq = st >= kFastScale;
      if (FP4 || RES) st_w = w_st[e];
      cur_e = e;
    }
    if (pi + 1 < p1) {
      cp_async_wait<1>();                          // this thread's copies of pass p are done
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();                               // copies (and the scale table) are visible
    const uint32_t rows0 = FP4 ? 0u : b * R * g.rowbytes;
    if (FP4) {
      // expand the raw rows into exact f16 products, 8 elements per step
      const uint32_t steps = half / 4u;            // 32-bit code words per row
      for (uint32_t r = 0; r < nrows; ++r) {
        const uint32_t ro = raw0 + (b * R + r) * g.rawbytes;
        uint8_t* dst = ws_smem + r * g.rowbytes;
        for (uint32_t q = t; q < steps; q += nthr) {
          const uint32_t wd = *reinterpret_cast<const uint32_t*>(ws_smem + ro + 4u * q);
          const uint32_t sv = dup_e4m3_to_h2(ws_smem[ro + half + (q >> 1)]);
          uint4 o;
          o.x = h2_mul(e2m1x2_to_h2(wd & 0xFFu), sv);
          o.y = h2_mul(e2m1x2_to_h2((wd >> 8) & 0xFFu), sv);
          o.z = h2_mul(e2m1x2_to_h2((wd >> 16) & 0xFFu), sv);
          o.w = h2_mul(e2m1x2_to_h2(wd >> 24), sv);
          *reinterpret_cast<uint4*>(dst + 16u * q) = o;
        }
      }
      __syncthreads();
    }
    if (RES) {
      // expand the raw Q(X) rows into exact f16 products (as above), then
      // the raw buffer takes the next pass's rows
      const uint32_t steps = half / 4u;
      for (uint32_t r = 0; r < nrows; ++r) {
        const uint32_t ro = raw0 + r * g.rawbytes;
        uint8_t* dst = ws_smem + exp0 + r * g.rowbytes;
        for (uint32_t q = t; q < steps; q += nthr) {
          const uint32_t wd = *reinterpret_cast<const uint32_t*>(ws_smem + ro + 4u * q);
          const uint32_t sv = dup_e4m3_to_h2(ws_smem[ro + half + (q >> 1)]);
          uint4 o;
          o.x = h2_mul(e2m1x2_to_h2(wd & 0xFFu), sv);
          o.y = h2_mul(e2m1x2_to_h2((wd >> 8) & 0xFFu), sv);
          o.z = h2_mul(e2m1x2_to_h2((wd >> 16) & 0xFFu), sv);
          o.w = h2_mul(e2m1x2_to_h2(wd >> 24), sv);
          *reinterpret_cast<uint4*>(dst + 16u * q) = o;
        }
      }
      __syncthreads();
      if (pi + 1 < p1) stage_raw(pass_of(pi + 1));
    }
    if (active) {
      for (int i = 0; i < g.nob; ++i) {
        const int ob = ob0 + i * nthr;
        if (ob >= nblk) break;
        if (g.nob > 1) load_idx(e, ob, cidx);
        for (int k = 0; k < g.RPT; ++k) {
          const uint32_t slot = static_cast<uint32_t>(phase + g.P * k);
          if (slot >= nout) break;
          if (slot >= nrows) {                     // a padding row of a group: zero codes and scale
            const int64_t row = r0 + slot;
            if (NV_IDX(row < rows && (ob + 1) * kBlock <= width)) {
              *reinterpret_cast<uint2*>(out_codes + row * (width / 2) + static_cast<int64_t>(ob) * 8) =
                  make_uint2(0u, 0u);
              out_scales[scale_offset(row, ob, width, out_layout)] = 0;
            }
            continue;
          }
          const uint8_t* rb = ws_smem + rows0 + slot * g.rowbytes;
          const uint8_t* eb = ws_smem + exp0 + slot * g.rowbytes;   // (residual)
          float v[16];
          float am = 0.0f;
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const uint32_t h = *reinterpret_cast<const uint16_t*>(rb + 2u * cidx[u]);
            float x;
            if (FP4) {
              x = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h))), st_w);
            } else if (RES) {
              // padded channels read element K of both rows (zero): dX = 0
              const uint32_t ph = *reinterpret_cast<const uint16_t*>(eb + 2u * cidx[u]);
              const float dq = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(ph))), st_w);
              x = __fsub_rn(__uint_as_float(h << 16), dq);
            } else {
              x = __uint_as_float(h << 16);
            }
            v[u] = x;
            am = fmaxf(am, fabsf(x));
          }
          const int64_t row = r0 + slot;
          uint32_t lo, hi, sb;
          if (fastq) {                             // output tensor scale >= 2^-55
            sb = encode16_fast(v, am, T, lo, hi);
          } else {
            const BlockQ bq = block_q(am, T);
            lo = encode8_q(v, bq);
            hi = encode8_q(v + 8, bq);
            sb = bq.sb;
          }
          if (NV_IDX(row < rows && (ob + 1) * kBlock <= width)) {
            *reinterpret_cast<uint2*>(out_codes + row * (width / 2) + static_cast<int64_t>(ob) * 8) =
                make_uint2(lo, hi);
            out_scales[scale_offset(row, ob, width, out_layout)] = static_cast<uint8_t>(sb);
          }
        }
      }
    }
    __syncthreads();                               // staged rows and buffer b are free again
  }
}

template <int MODE>
__global__ void __launch_bounds__(512, MODE == 2 ? 1 : 2) wsel_rows_kernel(RowsArgs A) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t ws_smem[];
  __shared__ ScaleTable T;
  __shared__ float s_wm[32];
  wsel_rows_body<MODE>(A, ws_smem, T, s_wm, blockIdx.x, gridDim.x);
}

// Both second passes of a dense RAC linear, row-staged, in one launch: CTAs
// [0, n_res) run the residual (MODE 2), the others W_sel (WMODE 0 from the
// bf16 weight, 1 from the NVFP4 weight).
template <int WMODE>
__global__ void __launch_bounds__(512, 1) rows_pair_kernel(RowsArgs Rr, RowsArgs Wr, int n_res) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t ws_smem[];
  __shared__ ScaleTable T;
  __shared__ float s_wm[32];
  if (static_cast<int>(blockIdx.x) < n_res)
    wsel_rows_body<2>(Rr, ws_smem, T, s_wm, blockIdx.x, n_res);
  else
    wsel_rows_body<WMODE>(Wr, ws_smem, T, s_wm, blockIdx.x - n_res, gridDim.x - n_res);
}

// Column maxima of |DQ(Q(W))| for `batch` stacked NVFP4 matrices of N rows
// each: colamax[e][j] = max_n |DQ_{e,n,j}|.  |E2M1dec(code)| E4M3dec(scale)
// has at most 6 significant bits and lies in [2^-10, 2688] (or is 0), so it
// is exact in f16 and the products and their maxima run on f16 pairs; RN(p
// s_t) does not decrease as p grows, so the maximum over the exact products
// is scaled once, in fp32.  A CTA covers 128 columns x 256 rows: thread =
// (32-column slice t%4, rows t/4 + 64 i), one 16-byte code load and one
// 2-byte scale load per row; rows reduce by shuffles within the warp, warps
// through shared memory, CTAs by an integer atomicMax on the bits of the
// non-negative results (colamax zeroed beforehand).
constexpr int kCmRows = 256;

__global__ void __launch_bounds__(256)
dq_colamax_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int layout,
                  const float* __restrict__ st, int64_t N, int64_t K, unsigned* __restrict__ colamax) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ uint32_t s_part[8][64];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, cg = t & 3;
  const int e = blockIdx.z;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 128 + 32 * cg;   // first column of the slice
  const bool cols_ok = c0 < K;
  uint32_t m[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) m[u] = 0u;
  if (cols_ok) {
#pragma unroll
    for (int i = 0; i < kCmRows / 64; ++i) {
      const int64_t n = static_cast<int64_t>(blockIdx.y) * kCmRows + (t >> 2) + 64 * i;
      if (n < N) {
        const int64_t row = static_cast<int64_t>(e) * N + n;
        const uint4 w = ld_nc_v4(codes + row * (K / 2) + c0 / 2);
        const uint32_t sb2 = __ldg(reinterpret_cast<const uint16_t*>(scales + scale_offset(row, c0 / kBlock, K, layout)));
        const uint32_t sv = e4m3x2_to_h2(sb2 & 0x7F7Fu);
        const uint32_t sv0 = __byte_perm(sv, 0, 0x1010), sv1 = __byte_perm(sv, 0, 0x3232);
        const uint32_t wd[4] = {w.x & 0x77777777u, w.y & 0x77777777u, w.z & 0x77777777u, w.w & 0x77777777u};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t pr = h2_mul(e2m1x2_to_h2((wd[q] >> (8 * b)) & 0xFFu), q < 2 ? sv0 : sv1);
            m[4 * q + b] = h2_max(m[4 * q + b], pr);
          }
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    m[u] = h2_max(m[u], __shfl_xor_sync(0xFFFFFFFFu, m[u], 4));
    m[u] = h2_max(m[u], __shfl_xor_sync(0xFFFFFFFFu, m[u], 8));
    m[u] = h2_max(m[u], __shfl_xor_sync(0xFFFFFFFFu, m[u], 16));
  }
  if (lane < 4) {
#pragma unroll
    for (int u = 0; u < 16; ++u) s_part[warp][16 * lane + u] = m[u];
  }
  __syncthreads();
  if (t < 64) {
    uint32_t r = 0u;
#pragma unroll
    for (int w = 0; w < 8; ++w) r = h2_max(r, s_part[w][t]);
    const int64_t c = static_cast<int64_t>(blockIdx.x) * 128 + 2 * t;   // columns c, c + 1
    if (c < K) {
      const float s = st[e];
      const float lo = __half2float(__ushort_as_half(static_cast<unsigned short>(r & 0xFFFFu)));
      const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(r >> 16)));
      atomicMax(colamax + static_cast<int64_t>(e) * K + c, __float_as_uint(__fmul_rn(lo, s)));
      atomicMax(colamax + static_cast<int64_t>(e) * K + c + 1, __float_as_uint(__fmul_rn(hi, s)));
    }
  }
}

__global__ void sel_tensor_scale_kernel(const float* __restrict__ colamax, int64_t K,
                                        const int32_t* __restrict__ sel, int64_t n_sel,
                                        float* __restrict__ s_t) {
  pdl_wait();
  pdl_launch_dependents();
  const int e = blockIdx.x;
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < n_sel; j += blockDim.x) {
    const int64_t c = sel[e * n_sel + j];
    if (NV_IDX(c >= 0 && c < K)) m = fmaxf(m, colamax[e * K + c]);
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

// ---------------------------------------------------------------------------
// weight fake quantization (W4A16 trainer side)
// ---------------------------------------------------------------------------
// A tile is 128 rows x 64 columns of one matrix; thread t: columns 8 (t & 7),
// rows t/8 + 32 i, i = 0..3.

// The tile's four 16-byte rows of this thread (zero past row N).
__device__ __forceinline__ void qdq_tile_load(const uint16_t* w, int64_t N, int64_t ldw, int64_t b, int64_t ty,
                                              int64_t col, int rr, uint4* raw) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = ty * 128 + rr + 32 * i;
    // coherent load: w may alias w_out
    raw[i] = n < N ? *reinterpret_cast<const uint4*>(w + (b * N + n) * ldw + col) : make_uint4(0, 0, 0, 0);
  }
}

// W' = DQ(Q(W)) of the tile (and, with WQ, its codes and scales; with WCM,
// its column maxima) from the loaded rows; every thread of the CTA calls it
// (one barrier inside with WCM).
template <bool WQ, bool WCM>
__device__ __forceinline__ void qdq_tile_store(const uint4* raw, int64_t N, int64_t K, int64_t ldw, int64_t b,
                                               int64_t ty, int64_t tx, float s_t, const ScaleTable& T,
                                               uint16_t* w_out, uint8_t* codes, uint8_t* scales, int layout,
                                               unsigned* colamax_bits, uint32_t (*cm)[65]) {
  const int t = threadIdx.x, cg = t & 7, rr = t >> 3;
  const int64_t col = tx * 64 + 8 * cg;
  uint32_t cmax[4] = {0, 0, 0, 0};               // |bf16| bits of columns 2j, 2j+1
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = ty * 128 + rr + 32 * i;
    const bool live = n < N;
    const int64_t off = (b * N + n) * ldw + col;
    const uint32_t wv[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
    uint64_t x2[4];
    uint32_t mbits = 0;                          // max |bf16| bits, two lanes
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x2[j] = bf16x2_to_f2(wv[j]);
      const uint32_t a = wv[j] & 0x7FFF7FFFu;
      mbits = __vmaxu2(mbits, a);
      if (WCM) cmax[j] = __vmaxu2(cmax[j], a);   // columns 2j (low) and 2j+1 (high)
    }
    float am = __uint_as_float(max(mbits & 0xFFFFu, mbits >> 16) << 16);
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
    uint32_t q, sb;
    float sbv;
    if (s_t >= kFastScale) {
      // negated quotients, as in the quantize pass: every nonzero block
      // decode scale is >= 2^-64, so its reciprocal table entry serves
      const float q0 = __fmul_rn(am, T.rcp_d);
      const float rr = __fmaf_rn(-q0, T.d, am);
      sb = f32_to_e4m3(__fmaf_rn(rr, T.rcp_d, q0));
      sbv = T.sbv[sb];
      const float ny = -T.rcp[sb], sd = T.sdec[sb];
      const uint64_t ny2 = f2_pack(ny, ny), sd2 = f2_pack(sd, sd);
      uint64_t c2[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t a = f2_mul(x2[j], ny2);
        c2[j] = f2_fma(f2_fma(a, sd2, x2[j]), ny2, a);
      }
      q = e2m1x8_f2(c2) ^ 0x88888888u;
    } else {
      const BlockQ bs = block_q(am, T);
      uint64_t q2[4];
      block_quotients(x2, bs, q2);
      q = e2m1x8_f2(q2);
      sb = bs.sb;
      sbv = bs.sbv;
    }
    const int64_t qrow = b * N + n;
    if (live) {
      const uint64_t sbv2 = f2_pack(sbv, sbv), st2 = f2_pack(s_t, s_t);
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float d0, d1;
        f2_unpack(f2_mul(f2_mul(e2m1x2_to_f2((q >> (8 * j)) & 0xFFu), sbv2), st2), d0, d1);
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o[j]) : "f"(d1), "f"(d0));   // d0 in the low half
      }
      if (NV_IDX(col + 8 <= K)) {
        *reinterpret_cast<uint4*>(w_out + off) = make_uint4(o[0], o[1], o[2], o[3]);
        if (WQ) *reinterpret_cast<uint32_t*>(codes + qrow * (K / 2) + col / 2) = q;
      }
    }
    // rows past N belong to the next matrix: only live rows write (the caller
    // zero-fills the padding of a tiled scale buffer beforehand)
    if (WQ && (cg & 1) == 0 && live)
      scales[scale_offset(qrow, col / kBlock, K, layout)] = static_cast<uint8_t>(sb);
  }
  if (!WCM) return;
#pragma unroll
  for (int j = 0; j < 4; ++j) {                  // |bf16| bits -> fp32 bits
    cm[rr][8 * cg + 2 * j] = (cmax[j] & 0xFFFFu) << 16;
    cm[rr][8 * cg + 2 * j + 1] = cmax[j] & 0xFFFF0000u;
  }
  __syncthreads();
  if (t < 64) {
    uint32_t m = 0;
    for (int r = 0; r < 32; ++r) m = max(m, cm[r][t]);
    if (m) atomicMax(colamax_bits + b * K + tx * 64 + t, m);
  }
  __syncthreads();                               // cm is free again
}

// One tile per CTA, the tensor amax from amax_partial's partial maxima.
// grid = (K/64, ceil(N/128), batch).  WQ: codes and scales wanted; WCM:
// column maxima wanted.
template <bool WQ, bool WCM>
__global__ void __launch_bounds__(kQThreads)
weight_qdq_kernel(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                  const unsigned* __restrict__ amax_parts, int n_parts,
                  uint16_t* w_out,   // w_out may alias w
                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int layout,
                  float* __restrict__ tensor_scale, unsigned* __restrict__ colamax_bits) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t b = blockIdx.z;
  const int t = threadIdx.x;
  uint4 raw[4];
  qdq_tile_load(w, N, ldw, b, blockIdx.y, static_cast<int64_t>(blockIdx.x) * 64 + 8 * (t & 7), t >> 3, raw);
  __shared__ uint32_t wscratch[kQThreads / 32];
  const float s_t = __fdiv_rn(reduce_parts(amax_parts + b * n_parts, n_parts, wscratch), kTensorScaleDiv);
  if (tensor_scale && blockIdx.x == 0 && blockIdx.y == 0 && t == 0) tensor_scale[b] = s_t;
  __shared__ ScaleTable T;
  __shared__ uint32_t cm[32][65];
  build_scale_table(T, s_t, t);
  __syncthreads();                               // table ready
  qdq_tile_store<WQ, WCM>(raw, N, K, ldw, b, blockIdx.y, blockIdx.x, s_t, T, w_out, codes, scales, layout,
                          colamax_bits, cm);
}

// ---------------------------------------------------------------------------
// MXFP8 quantization (the FP8 comparator's operands): E4M3 elements, one
// UE8M0 scale per 32 elements, E = floor(log2 amax_b) - 8 clamped to
// [-127, 127] (-127 for an all-zero block), code = E4M3(x / 2^E) nearest-even
// saturating, sign from x.  A warp covers 256 consecutive elements of a row
// (8 blocks, 4 threads and one 16-byte load per thread and block quarter).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
mxfp8_quant_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ldx,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int layout) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t segs = K / 256;
  const int64_t units = rows * segs;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units;
       u += warps) {
    const int64_t row = u / segs;
    const int64_t col = (u % segs) * 256 + 8 * lane;
    const uint4 v = ld_nc_v4(x + row * ldx + col);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    // floor(log2 amax) of the block (amax = bf16 bits m, as fp32 bits m << 16)
    const uint32_t ab = m << 16;
    const int eb = static_cast<int>(ab >> 23);
    int E;
    if (ab == 0) {
      E = -127;
    } else {
      const int fl = eb != 0 ? eb - 127 : (31 - __clz(static_cast<int>(ab & 0x7FFFFFu))) - 149;
      E = min(max(fl - 8, -127), 127);
    }
    const float inv = pow2f(-E);                   // exact power of two
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t packed = 0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t wd = w[2 * h + j];
        const float lo = __fmul_rn(__uint_as_float(wd << 16), inv);
        const float hi = __fmul_rn(__uint_as_float(wd & 0xFFFF0000u), inv);
        uint16_t r;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
        const uint32_t c2 = static_cast<uint32_t>(r) | ((wd >> 8) & 0x80u) | ((wd >> 16) & 0x8000u);
        packed |= c2 << (16 * j);
      }
      out[h] = packed;
    }
    if (NV_IDX(row < rows && col + 8 <= K))
      *reinterpret_cast<uint2*>(codes + row * K + col) = make_uint2(out[0], out[1]);
    if ((lane & 3) == 0) {
      const int64_t blk = col / 32;
      const int64_t off = layout == 0 ? row * (K / 32) + blk
                                      : ((row >> 7) * (K / 128) + (blk >> 2)) * 512 + (row & 31) * 16 +
                                            ((row & 127) >> 5) * 4 + (blk & 3);
      if (NV_IDX(off < scale_extent(rows, K, layout, 32))) scales[off] = static_cast<uint8_t>(E + 127);
    }
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
  {
    const cudaError_t le = launch_k(amax_kernel, dim3(grid), dim3(kQThreads), 0, s, nullptr, 0,
                                   x, K, ldx, g, mat_stride, amax_bits);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_group_tiles(const int64_t* off, int32_t E, int32_t* tile_start, cudaStream_t s) {
  {
    const cudaError_t le = launch_k(group_tiles_kernel, dim3(1), dim3(32), 0, s, nullptr, 0,
                                   off, E, tile_start);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_score(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                               const RowGroups& g, const float* amax, const unsigned* amax_parts,
                               int n_parts, int64_t codes_rows,
                               uint8_t* codes, uint8_t* scales, int layout, float* tensor_scale,
                               double* part_sum, float* part_max, unsigned* strip_count,
                               double* score, float* colamax, cudaStream_t s, const FusedSelect* fused) {
  const int64_t tiles = max_tiles(g, rows);
  if (tiles == 0) return cudaSuccess;
  // persistent: a few CTAs per SM over every (row tile, strip) pair
  constexpr int kDyn = 2 * kTileRows * kQCols * 2;
  {
    static bool done1[kMaxAttrDevices] = {}, done0[kMaxAttrDevices] = {};
    const cudaError_t ae = part_sum != nullptr ? set_max_smem(quant_score2_kernel<true>, kDyn, done1)
                                               : set_max_smem(quant_score2_kernel<false>, kDyn, done0);
    if (ae != cudaSuccess) return ae;
  }
  const int64_t work = tiles * (K / kQCols);
  if (work >= (int64_t(1) << 31)) return cudaErrorInvalidValue;   // tile indices are 32-bit in the kernel
  const int64_t cap = static_cast<int64_t>(sm_count()) * 3;
  SelectOut so{-1, nullptr, nullptr, nullptr, nullptr};
  if (fused != nullptr) so = SelectOut{fused->n_sel, fused->mask, fused->sel, fused->s_t, fused->strips_done};
  const cudaError_t le = launch_k(part_sum != nullptr ? quant_score2_kernel<true> : quant_score2_kernel<false>,
                                  dim3(static_cast<unsigned>(work < cap ? work : cap)), dim3(kQThreads), kDyn, s,
                                  nullptr, 0, x, K, ldx, g, amax, amax_parts, n_parts, codes_rows, codes, scales,
                                  layout, tensor_scale, part_sum, part_max, strip_count, score, colamax, so);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int amax_parts_count(int64_t rows, int64_t K) {
  const int64_t nvec = rows * (K / 8);
  const int64_t want = (nvec + 8 * kQThreads - 1) / (8 * kQThreads);
  return static_cast<int>(want < 4 * 148 ? (want > 0 ? want : 1) : 4 * 148);
}

cudaError_t launch_amax_partial(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, int32_t batch,
                                int64_t mat_stride, unsigned* parts, int n_parts, unsigned* zero_ptr,
                                int n_zero, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(n_parts), static_cast<unsigned>(batch));
  {
    const cudaError_t le = launch_k(amax_partial_kernel, dim3(grid), dim3(kQThreads), 0, s, nullptr, 0,
                                   x, rows, K, ldx, mat_stride, parts, zero_ptr, n_zero);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_score_reduce(const double* part_sum, const float* part_max, int64_t K,
                                const RowGroups& g, int64_t tiles, double* score, float* colamax,
                                float* tensor_scale_empty, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((K + 255) / 256), static_cast<unsigned>(g.E));
  {
    const cudaError_t le = launch_k(score_reduce_kernel, dim3(grid), dim3(256), 0, s, nullptr, 0,
                                   part_sum, part_max, K, g, tiles, score, colamax, tensor_scale_empty);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

int gather_grid(int64_t rows, int64_t width) {
  const int64_t tiles = (rows + kGRows - 1) / kGRows * ((width + kGCols - 1) / kGCols);
  return static_cast<int>(tiles < 8 * 148 ? tiles : 8 * 148);
}

cudaError_t launch_sel_tensor_scale(const float* colamax, int64_t K, const int32_t* sel,
                                    int64_t n_sel, int32_t E, float* s_t, cudaStream_t s) {
  {
    const cudaError_t le = launch_k(sel_tensor_scale_kernel, dim3(E), dim3(512), 0, s, nullptr, 0,
                                   colamax, K, sel, n_sel, s_t);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

namespace {
// Launch shape of wsel_rows_kernel; ok == false when its shared memory would
// not fit or K is past 16-bit channel offsets (the generic gather runs
// instead).
struct WselPlan {
  WselGeom g;
  int threads;
  size_t smem;
  bool ok;
};
// mode 0: bf16 weight rows; 1: NVFP4 weight rows; 2: the residual (bf16 X
// rows double-buffered, raw Q(X) rows and their f16 expansion one buffer
// each).
WselPlan wsel_plan(int64_t N, int64_t K, int32_t E, int64_t width, int mode) {
  const bool fp4 = mode == 1;
  // at most 54 KB of rows keeps four CTAs (the register limit) on an SM; the
  // residual's rows are larger: up to 110 KB (two CTAs of 256 threads)
  const size_t kBudget = mode == 2 ? 110 * 1024 : 54 * 1024, kMax = 200 * 1024;
  WselPlan w{};
  const int64_t nblk = width / kBlock;
  w.threads = nblk <= 256 ? 256 : static_cast<int>(nblk < 512 ? (nblk + 31) / 32 * 32 : 512);
  int P = nblk <= w.threads ? static_cast<int>(w.threads / nblk) : 1;
  if (E > 1)
    while (P & (P - 1)) P &= P - 1;                // a power of two, so passes never straddle matrices
  int RPT = 4;
  w.g.rowbytes = static_cast<uint32_t>(2 * K + 16);
  w.g.rawbytes = static_cast<uint32_t>((K / 2 + K / kBlock + 15) / 16 * 16);
  auto bytes = [&](int r) {
    if (mode == 2) return static_cast<size_t>(r) * (3 * w.g.rowbytes + w.g.rawbytes);
    return fp4 ? static_cast<size_t>(r) * (w.g.rowbytes + 2 * w.g.rawbytes)
               : static_cast<size_t>(2 * r) * w.g.rowbytes;
  };
  while (bytes(P * RPT) > kBudget || (E > 1 && N % (P * RPT) != 0)) {
    if (RPT > 1) RPT /= 2;
    else if (P > 1) P /= 2;
    else break;
  }
  w.g.P = P;
  w.g.RPT = RPT;
  w.g.R = P * RPT;
  w.g.nob = static_cast<int>((nblk + w.threads - 1) / w.threads);
  w.smem = bytes(w.g.R);
  w.ok = K <= 65472 && w.smem <= kMax && (E == 1 || N % w.g.R == 0);
  return w;
}

template <int MODE>
cudaError_t launch_wsel_rows(const WselPlan& wp, const uint16_t* w, int64_t ldw, const uint8_t* w_codes,
                             const uint8_t* w_scales, int w_layout, const float* w_st, int64_t N, int64_t K,
                             int32_t E, const int32_t* sel, int64_t n_sel, int64_t width,
                             const float* colamax, int fuse, float* s_t, uint8_t* codes, uint8_t* scales,
                             int layout, cudaStream_t s) {
  static bool done[kMaxAttrDevices] = {};
  {
    const cudaError_t ae = set_max_smem(wsel_rows_kernel<MODE>, 200 * 1024, done);
    if (ae != cudaSuccess) return ae;
  }
  int per_sm = 0;
  const cudaError_t oe =
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wsel_rows_kernel<MODE>, wp.threads, wp.smem);
  if (oe != cudaSuccess) return oe;
  const int64_t rows = static_cast<int64_t>(E) * N;
  const int64_t passes = (rows + wp.g.R - 1) / wp.g.R;
  const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = static_cast<unsigned>(passes < cap ? passes : cap);
  const RowsArgs A{w, ldw, w_codes, w_scales, w_layout, w_st, N, K, E, sel, n_sel, width, colamax,
                   fuse, s_t, codes, scales, layout, wp.g};
  const cudaError_t le = launch_k(wsel_rows_kernel<MODE>, dim3(grid), dim3(wp.threads), wp.smem, s, nullptr, 0, A);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_residual_gather(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx,
                                   const RowGroups& g, int64_t prows,
                                   const uint8_t* qx_codes, const uint8_t* qx_scales, int qx_layout,
                                   const float* qx_st, const int32_t* sel, int64_t n_sel,
                                   int64_t width, const float* r_st, uint8_t* r_codes,
                                   uint8_t* r_scales, int r_layout, cudaStream_t s) {
  (void)rows;
  if (width == 0 || prows == 0) return cudaSuccess;
  // grouped rows (MoE) of 2048 channels or more: the row-staged residual
  // (whole rows of X and Q(X) read once, coalesced), passes inside the
  // groups' padded 128-row tiles (shorter rows: measured slower than the
  // tile gather, 1024 channels 731 -> 744 us per MoE call)
  if (g.off != nullptr && prows % kTileRows == 0 && K >= 2048) {
    const WselPlan wp = wsel_plan(kTileRows, K, 2, width, 2);   // R a power of two dividing 128
    if (wp.ok && kTileRows % wp.g.R == 0) {
      static bool done[kMaxAttrDevices] = {};
      const cudaError_t ae = set_max_smem(wsel_rows_kernel<2>, 200 * 1024, done);
      if (ae != cudaSuccess) return ae;
      int per_sm = 0;
      const cudaError_t oe =
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wsel_rows_kernel<2>, wp.threads, wp.smem);
      if (oe != cudaSuccess) return oe;
      const int64_t passes = prows / wp.g.R;
      const int64_t cap = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
      const unsigned grid = static_cast<unsigned>(passes < cap ? passes : cap);
      RowsArgs A{x, ldx, qx_codes, qx_scales, qx_layout, qx_st, prows, K, g.E, sel, n_sel, width, nullptr, 0,
                 const_cast<float*>(r_st), r_codes, r_scales, r_layout, wp.g};
      A.grp = g;
      A.prows = prows;
      const cudaError_t le = launch_k(wsel_rows_kernel<2>, dim3(grid), dim3(wp.threads), wp.smem, s, nullptr, 0, A);
      if (le != cudaSuccess) return le;
      return cudaGetLastError();
    }
  }
  // dense activations with at least two passes per SM: the row-staged
  // residual as in the fused second pass (it writes real rows only, so with
  // a tiled scale layout the rows must fill whole 128-row blocks)
  if (g.off == nullptr && (r_layout == 0 || prows % kTileRows == 0)) {
    const WselPlan rp = wsel_plan(prows, K, 1, width, 2);
    const int64_t sms = sm_count();
    if (rp.ok && (prows + rp.g.R - 1) / rp.g.R >= 2 * sms) {
      static bool done[kMaxAttrDevices] = {};
      const cudaError_t ae = set_max_smem(wsel_rows_kernel<2>, 200 * 1024, done);
      if (ae != cudaSuccess) return ae;
      int per_sm = 0;
      const cudaError_t oe =
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wsel_rows_kernel<2>, rp.threads, rp.smem);
      if (oe != cudaSuccess) return oe;
      const int64_t passes = (prows + rp.g.R - 1) / rp.g.R;
      const int64_t cap = sms * (per_sm > 0 ? per_sm : 1);
      const RowsArgs A{x, ldx, qx_codes, qx_scales, qx_layout, qx_st, prows, K, 1, sel, n_sel, width, nullptr, 0,
                       const_cast<float*>(r_st), r_codes, r_scales, r_layout, rp.g};
      const cudaError_t le = launch_k(wsel_rows_kernel<2>, dim3(static_cast<unsigned>(passes < cap ? passes : cap)),
                                      dim3(rp.threads), rp.smem, s, nullptr, 0, A);
      if (le != cudaSuccess) return le;
      return cudaGetLastError();
    }
  }
  // rows of the scale buffer are padded to 128 for the tiled layout
  const int64_t grid_rows = r_layout == 1 ? (prows + kTileRows - 1) / kTileRows * kTileRows : prows;
  {
    const GatherArgs A{x, K, ldx, g, 0, qx_codes, qx_scales, qx_layout, qx_st, sel, n_sel,
                       width, nullptr, 0, const_cast<float*>(r_st), r_codes, r_scales, r_layout, prows, grid_rows};
    const cudaError_t le = launch_k(gather_quant_kernel<1>, dim3(gather_grid(grid_rows, width)), dim3(kGThreads), 0, s,
                                    nullptr, 0, A);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_weight_gather(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t E,
                                 const int32_t* sel, int64_t n_sel, int64_t width,
                                 const float* colamax, float* s_t, uint8_t* codes, uint8_t* scales,
                                 int layout, cudaStream_t s) {
  if (width == 0) return cudaSuccess;
  const int fuse = E == 1 ? 1 : 0;
  if (!fuse) {
    cudaError_t e = launch_sel_tensor_scale(colamax, K, sel, n_sel, E, s_t, s);
    if (e != cudaSuccess) return e;
  }
  // the row-staged kernel pays off once every CTA runs several passes; a
  // weight with fewer rows than about two passes per resident CTA takes the
  // tile gather (its fixed cost per CTA is lower)
  const WselPlan ws = wsel_plan(N, K, E, width, 0);
  const int64_t passes_w = (static_cast<int64_t>(E) * N + ws.g.R - 1) / (ws.g.R > 0 ? ws.g.R : 1);
  if (ws.ok && passes_w >= 2 * 4 * static_cast<int64_t>(sm_count()))
    return launch_wsel_rows<0>(ws, w, ldw, nullptr, nullptr, 0, nullptr, N, K, E, sel, n_sel, width, colamax,
                                   fuse, s_t, codes, scales, layout, s);
  const int64_t rows = static_cast<int64_t>(E) * N;
  RowGroups none{};
  {
    const GatherArgs A{w, K, ldw, none, N, nullptr, nullptr, 0, nullptr, sel, n_sel, width,
                       colamax, fuse, s_t, codes, scales, layout, rows, rows};
    const cudaError_t le = launch_k(gather_quant_kernel<0>, dim3(gather_grid(rows, width)), dim3(kGThreads), 0, s,
                                    nullptr, 0, A);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_weight_gather_fp4(const uint8_t* w_codes, const uint8_t* w_scales, int w_layout,
                                     const float* w_st, int64_t N, int64_t K, int32_t E,
                                     const int32_t* sel, int64_t n_sel, int64_t width,
                                     const float* dq_colamax, float* s_t, uint8_t* codes,
                                     uint8_t* scales, int layout, cudaStream_t s) {
  if (width == 0) return cudaSuccess;
  const int fuse = E == 1 ? 1 : 0;
  if (!fuse) {
    cudaError_t e = launch_sel_tensor_scale(dq_colamax, K, sel, n_sel, E, s_t, s);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = static_cast<int64_t>(E) * N;
  const WselPlan ws = wsel_plan(N, K, E, width, 1);
  if (ws.ok)
    return launch_wsel_rows<1>(ws, nullptr, 0, w_codes, w_scales, w_layout, w_st, N, K, E, sel, n_sel, width,
                                  dq_colamax, fuse, s_t, codes, scales, layout, s);
  RowGroups none{};
  {
    const GatherArgs A{nullptr, K, K, none, N, w_codes, w_scales, w_layout, w_st, sel, n_sel,
                       width, dq_colamax, fuse, s_t, codes, scales, layout, rows, rows};
    const cudaError_t le = launch_k(gather_quant_kernel<2>, dim3(gather_grid(rows, width)), dim3(kGThreads), 0, s,
                                    nullptr, 0, A);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_dq_colamax(const uint8_t* codes, const uint8_t* scales, int layout, const float* st,
                              int64_t N, int64_t K, int32_t batch, float* colamax, cudaStream_t s) {
  {
    const cudaError_t me = cudaMemsetAsync(colamax, 0, sizeof(float) * K * batch, s);
    if (me != cudaSuccess) return me;
  }
  dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>((N + kCmRows - 1) / kCmRows),
            static_cast<unsigned>(batch));
  {
    const cudaError_t le = launch_k(dq_colamax_kernel, dim3(grid), dim3(256), 0, s, nullptr, 0,
                                   codes, scales, layout, st, N, K, reinterpret_cast<unsigned*>(colamax));
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_weight_qdq(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, int32_t batch,
                              const unsigned* amax_parts, int n_parts, uint16_t* w_out, uint8_t* codes,
                              uint8_t* scales, int layout, float* tensor_scale,
                              unsigned* colamax_bits, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(K / 64), static_cast<unsigned>((N + 127) / 128),
            static_cast<unsigned>(batch));
  {
    auto kern = codes != nullptr ? (colamax_bits != nullptr ? weight_qdq_kernel<true, true> : weight_qdq_kernel<true, false>)
                                 : (colamax_bits != nullptr ? weight_qdq_kernel<false, true> : weight_qdq_kernel<false, false>);
    const cudaError_t le = launch_k(kern, dim3(grid), dim3(kQThreads), 0, s, nullptr, 0,
                                   w, N, K, ldw, amax_parts, n_parts, w_out, codes, scales, layout,
                                   tensor_scale, colamax_bits);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

cudaError_t launch_mxfp8_quant(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, uint8_t* codes,
                               uint8_t* scales, int layout, cudaStream_t s) {
  const int64_t warps = rows * (K / 256);
  if (warps == 0) return cudaSuccess;
  const int64_t ctas = (warps + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const cudaError_t le = launch_k(mxfp8_quant_kernel, dim3(static_cast<unsigned>(ctas < cap ? ctas : cap)), dim3(256), 0,
                                  s, nullptr, 0, x, rows, K, ldx, codes, scales, layout);
  if (le != cudaSuccess) return le;
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

cudaError_t launch_second_pass(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const uint8_t* qx_codes,
                               const uint8_t* qx_scales, int qx_layout, const float* qx_st, const int32_t* sel,
                               int64_t n_sel, int64_t width, const float* r_st, uint8_t* r_codes, uint8_t* r_scales,
                               int r_layout, const uint16_t* w, int64_t N, int64_t ldw, const uint8_t* w_codes,
                               const uint8_t* w_scales, int w_layout, const float* w_st, const float* w_colamax,
                               float* ws_st, uint8_t* ws_codes, uint8_t* ws_scales, int ws_layout, cudaStream_t s) {
  if (width == 0) return cudaSuccess;
  const RowGroups dense{nullptr, nullptr, 1, M};
  const int64_t grid_rows = r_layout == 1 ? (M + kTileRows - 1) / kTileRows * kTileRows : M;
  const int wmode = w != nullptr ? 0 : 1;
  const int64_t sms = sm_count();
  // large activations: the residual row-staged (whole rows of X and Q(X)
  // read once, coalesced); with it the weight row-staged in the same launch
  const WselPlan rp = wsel_plan(M, K, 1, width, 2);
  const WselPlan wq = wsel_plan(N, K, 1, width, wmode);
  const int64_t passes_r = (M + rp.g.R - 1) / (rp.g.R > 0 ? rp.g.R : 1);
  const int64_t passes_w = (N + wq.g.R - 1) / (wq.g.R > 0 ? wq.g.R : 1);
  // (the row-staged residual writes real rows only: with a tiled layout the
  // padding rows of the scale buffer would stay unwritten unless M % 128 == 0)
  if (rp.ok && wq.ok && rp.threads == wq.threads && passes_r >= 2 * sms &&
      (r_layout == 0 || M % kTileRows == 0)) {
    const size_t smem = rp.smem > wq.smem ? rp.smem : wq.smem;
    static bool done0[kMaxAttrDevices] = {}, done1[kMaxAttrDevices] = {};
    {
      const cudaError_t ae = wmode == 0 ? set_max_smem(rows_pair_kernel<0>, 200 * 1024, done0)
                                        : set_max_smem(rows_pair_kernel<1>, 200 * 1024, done1);
      if (ae != cudaSuccess) return ae;
    }
    int per_sm = 0;
    const cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, wmode == 0 ? rows_pair_kernel<0> : rows_pair_kernel<1>, rp.threads, smem);
    if (oe != cudaSuccess) return oe;
    const int64_t total = sms * (per_sm > 0 ? per_sm : 1);
    // CTAs in proportion to the bytes each side reads
    const double rb = static_cast<double>(M) * 2.5625 * K;
    const double wb = static_cast<double>(N) * (wmode == 0 ? 2.0 : 0.5625) * K;
    int64_t n_res = static_cast<int64_t>(static_cast<double>(total) * rb / (rb + wb) + 0.5);
    n_res = n_res < 1 ? 1 : (n_res > total - 1 ? total - 1 : n_res);
    if (n_res > passes_r) n_res = passes_r;
    int64_t n_w = total - n_res;
    if (n_w > passes_w) n_w = passes_w;
    if (n_w < 1) n_w = 1;
    const RowsArgs Rr{x, ldx, qx_codes, qx_scales, qx_layout, qx_st, M, K, 1, sel, n_sel, width, nullptr, 0,
                      const_cast<float*>(r_st), r_codes, r_scales, r_layout, rp.g};
    const RowsArgs Wr{w, ldw, w_codes, w_scales, w_layout, w_st, N, K, 1, sel, n_sel, width, w_colamax, 1,
                      ws_st, ws_codes, ws_scales, ws_layout, wq.g};
    const cudaError_t le =
        wmode == 0 ? launch_k(rows_pair_kernel<0>, dim3(static_cast<unsigned>(n_res + n_w)), dim3(rp.threads), smem, s,
                              nullptr, 0, Rr, Wr, static_cast<int>(n_res))
                   : launch_k(rows_pair_kernel<1>, dim3(static_cast<unsigned>(n_res + n_w)), dim3(rp.threads), smem, s,
                              nullptr, 0, Rr, Wr, static_cast<int>(n_res));
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
  }
  // the weight side takes the row-staged kernel when it pays (see
  // launch_weight_gather): then the two passes are two launches
  const WselPlan wp = wsel_plan(N, K, 1, width, wmode);
  const int64_t passes_wt = (N + wp.g.R - 1) / (wp.g.R > 0 ? wp.g.R : 1);
  const bool rows_kernel = w != nullptr ? (wp.ok && passes_wt >= 2 * 4 * sms) : wp.ok;
  if (rows_kernel) {
    cudaError_t e = launch_residual_gather(x, M, K, ldx, dense, M, qx_codes, qx_scales, qx_layout, qx_st, sel, n_sel,
                                           width, r_st, r_codes, r_scales, r_layout, s);
    if (e != cudaSuccess) return e;
    return w != nullptr ? launch_weight_gather(w, N, K, ldw, 1, sel, n_sel, width, w_colamax, ws_st, ws_codes,
                                               ws_scales, ws_layout, s)
                        : launch_weight_gather_fp4(w_codes, w_scales, w_layout, w_st, N, K, 1, sel, n_sel, width,
                                                   w_colamax, ws_st, ws_codes, ws_scales, ws_layout, s);
  }
  const RowGroups none{};
  const GatherArgs R{x, K, ldx, dense, 0, qx_codes, qx_scales, qx_layout, qx_st, sel, n_sel,
                     width, nullptr, 0, const_cast<float*>(r_st), r_codes, r_scales, r_layout, M, grid_rows};
  const GatherArgs W{w, K, ldw, none, N, w_codes, w_scales, w_layout, w_st, sel, n_sel,
                     width, w_colamax, 1, ws_st, ws_codes, ws_scales, ws_layout, N, N};
  const int64_t ct = (width + kGCols - 1) / kGCols;
  const int64_t rt = (grid_rows + kGRows - 1) / kGRows * ct, wt = (N + kGRows - 1) / kGRows * ct;
  const int64_t cap = 8 * static_cast<int64_t>(sm_count());
  const int64_t grid = rt + wt < cap ? rt + wt : cap;
  int64_t n_res = (grid * rt + (rt + wt) / 2) / (rt + wt);
  n_res = n_res < 1 ? 1 : (n_res > grid - 1 ? grid - 1 : n_res);
  const cudaError_t le =
      w != nullptr ? launch_k(gather_pair_kernel<0>, dim3(static_cast<unsigned>(grid)), dim3(kGThreads), 0, s, nullptr,
                              0, R, W, static_cast<int>(n_res))
                   : launch_k(gather_pair_kernel<2>, dim3(static_cast<unsigned>(grid)), dim3(kGThreads), 0, s, nullptr,
                              0, R, W, static_cast<int>(n_res));
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

NV_DEFINE_BOUNDS_READER(bounds_flags_quant)

}  // namespace nvfp4
