// Shared device helpers of the NVFP4 W4A4 + RAC kernels (sm_100a).
//
// Arithmetic of the quantizer follows the NVFP4 reading stated in
// include/nvfp4rac.h: every step is an fp32 operation rounded to nearest
// even, written with the explicit __f*_rn intrinsics so that no multiply-add
// is fused and codes match a plain CPU restatement bit for bit.  The library
// is built without fast-math and without flush-to-zero.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace nvfp4 {

constexpr int kBlock = 16;          // elements per block scale
constexpr int kTileRows = 128;      // rows per quantizer / GEMM tile and per score chunk
constexpr float kTensorScaleDiv = 2688.0f;   // 6 (E2M1 max) x 448 (E4M3 max)

// Device error word bits (read by nvfp4_stream_status).
constexpr unsigned kErrTimeout = 1u;

// ---------------------------------------------------------------------------
// Element formats.
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
  return __uint_as_float((b & 0xFFFFu) << 16);
}

// E2M1 value of a code (sign in bit 3): exponent field e = (c >> 1) & 3 with
// bias 1, mantissa bit m = c & 1, e == 0 subnormal (m * 0.5).
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const uint32_t mag = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
  return __uint_as_float(mag | ((c & 8u) << 28));
}

// E4M3 value of a non-negative code 0..0x7E: exponent bias 7, 3 mantissa
// bits, exponent 0 subnormal (m * 2^-9).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;   // exact
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// E4M3 code of s >= 0: hardware conversion, round to nearest even,
// saturating to 448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}

// E2M1 magnitude codes of |v[0..7]| packed 2 per byte, element 2j in the
// low nibble of byte j (hardware conversion, round to nearest even,
// saturating at 6).  The sign bits are added from the inputs' own sign bits,
// so a negative value that rounds to zero keeps its sign (code 0x8).
__device__ __forceinline__ uint32_t e2m1x8(const float* v) {
  uint32_t mags;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(mags)
      : "f"(fabsf(v[0])), "f"(fabsf(v[1])), "f"(fabsf(v[2])), "f"(fabsf(v[3])),
        "f"(fabsf(v[4])), "f"(fabsf(v[5])), "f"(fabsf(v[6])), "f"(fabsf(v[7])));
  uint32_t signs = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) signs |= (__float_as_uint(v[j]) >> 31) << (4 * j + 3);
  return mags | signs;
}

// Per-block quantization parameters for a tensor with decode scale s_t:
// sb = E4M3(RN(amax_b / RN(6 s_t))), s_dec = RN(E4M3dec(sb) s_t).
struct BlockScale {
  uint32_t sb;
  float sbv;
  float s_dec;
};

__device__ __forceinline__ BlockScale block_scale(float amax_b, float s_t) {
  BlockScale r;
  const float d = __fmul_rn(6.0f, s_t);
  if (d > 0.0f) {
    r.sb = f32_to_e4m3(__fdiv_rn(amax_b, d));
  } else {
    r.sb = 0;
  }
  r.sbv = e4m3_to_f32(r.sb);
  r.s_dec = __fmul_rn(r.sbv, s_t);
  return r;
}

// RN(x / b) for a whole block that shares the divisor b = s_dec > 0, with
// y = RN(1/b) computed once per block (__frcp_rn).  Markstein's correction
// (P. Markstein, IBM J. Res. Dev. 1990; Muller et al., Handbook of
// Floating-Point Arithmetic, division with an FMA): q = RN(x y) is within one
// ulp of x/b, the remainder r = x - b q is exact with an FMA, and
// RN(q + r y) = RN(x / b) when y is within half an ulp of 1/b and nothing
// under- or overflows.  Blocks whose divisor is below 2^-100 use the full
// division instead.  The sign of the result is that of x (x = -0 gives -0).
struct BlockDivisor {
  float b, y;
  bool fast;
};

__device__ __forceinline__ BlockDivisor block_divisor(float s_dec) {
  BlockDivisor d;
  d.b = s_dec;
  d.fast = s_dec >= 7.888609052210118e-31f;   // 2^-100
  d.y = d.fast ? __frcp_rn(s_dec) : 0.0f;
  return d;
}

__device__ __forceinline__ float div_block(float x, const BlockDivisor& d) {
  float q;
  if (d.b <= 0.0f) {
    q = 0.0f;
  } else if (d.fast) {
    const float q0 = __fmul_rn(x, d.y);
    const float r = __fmaf_rn(-q0, d.b, x);
    q = __fmaf_rn(r, d.y, q0);
  } else {
    q = __fdiv_rn(x, d.b);
  }
  return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
}

// Codes of 8 consecutive elements (one half of a block) -> 4 bytes, element
// 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t encode8(const float* v, const BlockDivisor& d) {
  float q[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) q[j] = div_block(v[j], d);
  return e2m1x8(q);
}

// Per-tensor-scale lookup of everything a block needs, built once per CTA
// (and per tensor scale): for every non-negative E4M3 code sb,
//   sbv[sb]  = E4M3dec(sb)                 (exact),
//   sdec[sb] = RN(sbv[sb] * s_t)           (the block decode scale),
//   rcp[sb]  = RN(1 / sdec[sb])            (0 when sdec < 2^-64: full division),
// plus d = RN(6 s_t) and its reciprocal for the block-scale quotient.  The
// quotients then cost one multiply and two FMAs (Markstein's correction, see
// div_block) instead of a full IEEE division per block and per element.
struct ScaleTable {
  float sbv[128], sdec[128], rcp[128];
  float s_t, d, rcp_d;
};

// Threads [0, nthreads) fill the table; the caller synchronizes afterwards.
__device__ __forceinline__ void build_scale_table(ScaleTable& T, float s_t, int tid) {
  if (tid < 128) {
    const float v = tid < 127 ? e4m3_to_f32(static_cast<uint32_t>(tid)) : 0.0f;
    const float sd = __fmul_rn(v, s_t);
    T.sbv[tid] = v;
    T.sdec[tid] = sd;
    T.rcp[tid] = sd >= 5.421010862427522e-20f ? __frcp_rn(sd) : 0.0f;   // 2^-64
  }
  if (tid == 0) {
    const float d = __fmul_rn(6.0f, s_t);
    T.s_t = s_t;
    T.d = d;
    T.rcp_d = d >= 5.421010862427522e-20f ? __frcp_rn(d) : 0.0f;
  }
}

static __device__ __noinline__ float div_slow(float a, float b) { return __fdiv_rn(a, b); }

// RN(a / b) for a >= 0, b > 0, with y = RN(1/b) (or y == 0: full division).
// With b >= 2^-64 the remainder a - b q0 is exact for every quotient that can
// change an E2M1 or E4M3 code (>= 2^-10), so Markstein's correction holds.
__device__ __forceinline__ float div_rn_pos(float a, float b, float y) {
  if (y == 0.0f) return div_slow(a, b);
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-q0, b, a);
  return __fmaf_rn(r, y, q0);
}

// Block parameters from the table: sb = E4M3(RN(amax_b / d)).
struct BlockQ {
  uint32_t sb;
  float sbv, sdec, rcp;
};

__device__ __forceinline__ BlockQ block_q(float amax_b, const ScaleTable& T) {
  BlockQ q;
  q.sb = T.d > 0.0f ? f32_to_e4m3(div_rn_pos(amax_b, T.d, T.rcp_d)) : 0u;
  q.sbv = T.sbv[q.sb];
  q.sdec = T.sdec[q.sb];
  q.rcp = T.rcp[q.sb];
  return q;
}

// E2M1 codes of 8 values with block parameters q: magnitudes of RN(|v|/sdec)
// through the hardware conversion, sign bits from v (so -0 keeps code 0x8).
__device__ __forceinline__ uint32_t encode8_q(const float* v, const BlockQ& q) {
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = q.sdec > 0.0f ? div_rn_pos(fabsf(v[j]), q.sdec, q.rcp) : 0.0f;
  uint32_t mags;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(mags)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
  uint32_t signs = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) signs |= (__float_as_uint(v[j]) >> 31) << (4 * j + 3);
  return mags | signs;
}

// Exact E4M3 value of a non-negative code through the hardware e4m3 -> f16
// conversion (every E4M3 value is an f16 value).
__device__ __forceinline__ float e4m3_to_f32_hw(uint32_t code) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(code & 0xFFu));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Exact E2M1 values of the two codes of a packed byte (low nibble first),
// through the hardware e2m1x2 -> f16x2 conversion.
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"(byte));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// DQ = RN(RN(E2M1dec(code) * E4M3dec(sb)) * s_t).
__device__ __forceinline__ float dequant(uint32_t code, float sbv, float s_t) {
  return __fmul_rn(__fmul_rn(e2m1_to_f32(code), sbv), s_t);
}

// Byte offset of the scale of (row, block) in an NVFP4 scale buffer.
__device__ __host__ __forceinline__ int64_t scale_offset(int64_t row, int64_t blk, int64_t cols,
                                                         int layout) {
  if (layout == 0) return row * (cols / kBlock) + blk;
  const int64_t k4 = (cols + 63) / 64;   // 512-byte atoms per 128-row block
  return ((row >> 7) * k4 + (blk >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (blk & 3);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// Row groups: a dense tensor (one group of M rows) or the experts of an MoE
// layer (group e owns rows off[e] .. off[e+1]).  Each group is cut into
// 128-row tiles; tile_start[e] is the first tile of group e, so every
// quantized operand and every score chunk is laid out on "padded rows"
// prow = tile * 128 + (row - first row of the tile), and no tile spans two
// groups.  For a dense tensor prow == row.
// ---------------------------------------------------------------------------
struct RowGroups {
  const int64_t* off;        // device [E+1], null for a dense tensor
  const int32_t* tile_start; // device [E+1], null for a dense tensor
  int32_t E;
  int64_t M;                 // dense rows (ignored for MoE)
};

struct TileInfo {
  int e;            // group
  int64_t row0;     // first real row of the tile
  int64_t row_end;  // one past the last real row of the group
  bool valid;
};

__device__ __forceinline__ TileInfo tile_info(const RowGroups& g, int64_t tile) {
  TileInfo t;
  if (g.off == nullptr) {
    t.e = 0;
    t.row0 = tile * kTileRows;
    t.row_end = g.M;
    t.valid = t.row0 < g.M;
    return t;
  }
  const int total = g.tile_start[g.E];
  t.valid = tile < total;
  if (!t.valid) { t.e = 0; t.row0 = 0; t.row_end = 0; return t; }
  int lo = 0, hi = g.E - 1;               // last e with tile_start[e] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (g.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  t.e = lo;
  t.row0 = g.off[lo] + (tile - g.tile_start[lo]) * kTileRows;
  t.row_end = g.off[lo + 1];
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier helpers with bounded waits.  A wait that does not complete within
// the time limit sets kErrTimeout in the device error word and returns false;
// callers then leave their loops so the kernel always terminates.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

// One poll; the thread may be parked by the hardware until the phase
// completes or the suspend-time hint (10 ms) expires, whichever is first.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(bar), "r"(parity), "r"(10000000u) : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
constexpr uint32_t kWaitMaxPolls = 1u << 26;        // hard cap on polls as well

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* err,
                                          uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1; i < kWaitMaxPolls; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if ((i & 15u) == 0 && global_timer_ns() - t0 > limit_ns) break;
  }
  if (err) atomicOr(err, kErrTimeout);
  return false;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
               :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

}  // namespace nvfp4
