// Shared device helpers of the NVFP4 W4A4 + RAC kernels (sm_100a).
//
// Arithmetic of the quantizer follows the NVFP4 reading stated in
// include/nvfp4rac.h: every step is an fp32 operation rounded to nearest
// even, written with the explicit __f*_rn intrinsics so that no multiply-add
// is fused and codes match a plain CPU restatement bit for bit.  The library
// is built without fast-math and without flush-to-zero.
#pragma once

#include <cuda.h>
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
// Index checks of the checked build (compiled with -DNVFP4_CHECKS; the
// library's memory-safety evidence where no sanitizer can run).  NV_IDX(c)
// states the in-bounds condition of one global or shared memory access: in
// the checked build a false condition sets this translation unit's flag word
// and records the source line (the largest one seen), and the caller skips the
// access; nothing traps.  nvfp4_stream_status reports it as
// NVFP4_ERR_BOUNDS.  In the normal build NV_IDX(c) is the constant true.
// ---------------------------------------------------------------------------
#ifdef NVFP4_CHECKS
static __device__ unsigned g_bounds_flag;
static __device__ unsigned g_bounds_line;
__device__ __forceinline__ bool idx_ok(bool ok, unsigned line) {
  if (!ok) {
    atomicOr(&g_bounds_flag, 1u);
    atomicMax(&g_bounds_line, line);
  }
  return ok;
}
#define NV_IDX(cond) (::nvfp4::idx_ok(static_cast<bool>(cond), __LINE__))
// host reader of this translation unit's flag word (and reset)
#define NV_DEFINE_BOUNDS_READER(fname)                                                   \
  unsigned fname(unsigned* line) {                                                       \
    unsigned v = 0, l = 0, z = 0;                                                        \
    if (cudaMemcpyFromSymbol(&v, g_bounds_flag, sizeof(v)) != cudaSuccess) return 0;     \
    cudaMemcpyFromSymbol(&l, g_bounds_line, sizeof(l));                                  \
    if (v) {                                                                             \
      cudaMemcpyToSymbol(g_bounds_flag, &z, sizeof(z));                                  \
      cudaMemcpyToSymbol(g_bounds_line, &z, sizeof(z));                                  \
    }                                                                                    \
    if (line) *line = l;                                                                 \
    return v;                                                                            \
  }
#else
#define NV_IDX(cond) (true)
#define NV_DEFINE_BOUNDS_READER(fname) \
  unsigned fname(unsigned* line) {     \
    if (line) *line = 0;               \
    return 0;                          \
  }
#endif

// Bytes of a scale buffer of rows x cols with blocks of `blk` elements in
// `layout` (0 canonical, 1 MMA-tiled with 128-row blocks of 4-block atoms).
__device__ __host__ __forceinline__ int64_t scale_extent(int64_t rows, int64_t cols, int layout, int blk) {
  if (layout == 0) return rows * (cols / blk);
  return (rows + 127) / 128 * 128 * ((cols + 4 * blk - 1) / (4 * blk)) * 4;
}

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

// E2M1 codes of v[0..7] packed 2 per byte, element 2j in the low nibble of
// byte j (hardware conversion of the signed value: round to nearest even,
// saturating at 6, the sign kept even when the value rounds to zero, so that
// a negative input gives code 0x8 there).
__device__ __forceinline__ uint32_t e2m1x8(const float* v) {
  uint32_t codes;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(codes)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return codes;
}

// ---- fp32 pairs ------------------------------------------------------------
// sm_100a executes mul / fma (and add / sub) on two fp32 lanes in one
// instruction (.f32x2, each lane rounded to nearest even like the scalar
// form).  A pair lives in one 64-bit register: element 2j in the low half.
// A packed product that feeds a packed sum or difference is fused into one
// rounding by the code generator (measured: a mul.rn.f32x2 feeding an
// add.rn.f32x2 changed the residual's last bits), so only products whose
// result is consumed by something other than an addition use the packed
// form, and there is no packed add here.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_abs(uint64_t a) { return a & 0x7FFFFFFF7FFFFFFFull; }

// The two bf16 of a 32-bit word as an fp32 pair (exact).
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Exact values of the two E2M1 codes of a byte (low nibble first) as an fp32
// pair, through the hardware e2m1x2 -> f16x2 conversion.
__device__ __forceinline__ uint64_t e2m1x2_to_f2(uint32_t byte) {
  uint64_t r;
  asm("{\n\t.reg .b8 t;\n\t.reg .b32 h;\n\t.reg .b16 l, u;\n\t.reg .f32 fl, fu;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 h, t;\n\t"
      "mov.b32 {l, u}, h;\n\t"
      "cvt.f32.f16 fl, l;\n\t"
      "cvt.f32.f16 fu, u;\n\t"
      "mov.b64 %0, {fl, fu};\n\t}"
      : "=l"(r) : "r"(byte));
  return r;
}

// f16 pairs (one 32-bit register, element 2j in the low half).  The exact
// values of the two E2M1 codes of a byte (low nibble in the low half) and of
// two E4M3 scale bytes (low byte in the low half), through the hardware
// conversions; both formats are exact in f16, and so is a product of an
// E2M1 and an E4M3 value (at most 6 significant bits, in [2^-10, 2688]).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(byte));
  return h;
}
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(two));
  return h;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// E2M1 codes of four fp32 pairs (8 elements) -> 4 bytes, element 2j in the
// low nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8_f2(const uint64_t* p) {
  float v[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) f2_unpack(p[j], v[2 * j], v[2 * j + 1]);
  return e2m1x8(v);
}

// Per-tensor-scale lookup of everything a block needs, built once per CTA
// (and per tensor scale): for every non-negative E4M3 code sb,
//   sbv[sb]  = E4M3dec(sb)                 (exact),
//   sdec[sb] = RN(sbv[sb] * s_t)           (the block decode scale),
//   rcp[sb]  = RN(1 / sdec[sb])            (0 when sdec < 2^-64: full division),
// plus d = RN(6 s_t) and its reciprocal for the block-scale quotient.  The
// quotients then cost one multiply and two FMAs (Markstein's correction, see
// div_rn_pos) instead of a full IEEE division per block and per element.
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

// RN(a / b) for a >= 0, b > 0, with y = RN(1/b) (or y == 0: full division),
// by Markstein's correction (P. Markstein, IBM J. Res. Dev. 1990; Muller et
// al., Handbook of Floating-Point Arithmetic, division with an FMA):
// q0 = RN(a y) is within one ulp of a/b, the remainder r = a - b q0 is exact
// with an FMA, and RN(q0 + r y) = RN(a / b).  With b >= 2^-64 the remainder
// is exact for every quotient that can change an E2M1 or E4M3 code
// (>= 2^-10).
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

// Quotients of one block for four fp32 pairs: RN(v / sdec) with the sign
// bit of v (signed zeros when sdec == 0), through div_rn_pos's steps on both
// lanes at once.  Round-to-nearest-even and the FMA are symmetric under
// negation, so the correction gives RN(v / sdec) for negative v as well; the
// final OR only restores the sign of a zero quotient of v = -0 (whose
// correction sum is +0).
__device__ __forceinline__ void block_quotients(const uint64_t* x2, const BlockQ& q, uint64_t* out) {
  constexpr uint64_t kSign = 0x8000000080000000ull;
  if (q.sdec > 0.0f && q.rcp != 0.0f) {
    const uint64_t y2 = f2_pack(q.rcp, q.rcp), nb2 = f2_pack(-q.sdec, -q.sdec);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint64_t q0 = f2_mul(x2[j], y2);
      const uint64_t r = f2_fma(q0, nb2, x2[j]);      // v - q0 sdec, exact
      out[j] = f2_fma(r, y2, q0) | (x2[j] & kSign);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float lo, hi;
      f2_unpack(f2_abs(x2[j]), lo, hi);
      const float ql = q.sdec > 0.0f ? div_slow(lo, q.sdec) : 0.0f;
      const float qh = q.sdec > 0.0f ? div_slow(hi, q.sdec) : 0.0f;
      out[j] = f2_pack(ql, qh) | (x2[j] & kSign);
    }
  }
}

// E2M1 codes of 8 values with block parameters q: the signed quotients of
// block_quotients through the hardware conversion (so -0 keeps code 0x8).
__device__ __forceinline__ uint32_t encode8_q(const float* v, const BlockQ& q) {
  uint64_t x2[4], o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) x2[j] = f2_pack(v[2 * j], v[2 * j + 1]);
  block_quotients(x2, q, o);
  return e2m1x8_f2(o);
}

// ---- output scale of a block-scaled product --------------------------------
// The product of two tensor scales s_a s_b is kept as m 2^e (m = RN(ma mb) in
// [0.25, 1) from the frexp significands, e exact), so that it does not
// underflow fp32 when both scales are tiny while Y itself is representable.
struct ScaleProduct {
  float m;
  int e;
};

__device__ __forceinline__ ScaleProduct scale_product(float sa, float sb) {
  int ea = 0, eb = 0;
  const float ma = frexpf(sa, &ea), mb = frexpf(sb, &eb);
  ScaleProduct r;
  r.m = __fmul_rn(ma, mb);
  r.e = r.m != 0.0f ? ea + eb : 0;
  return r;
}

// 2^e as an fp32, e in [-149, 127] (a subnormal below -126).
__device__ __forceinline__ float pow2f(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23)
                   : __uint_as_float(1u << (e + 149));
}

// RN(t 2^e) as RN(RN(t p1) p2): p1 is 1 or an exact power-of-two pre-scale
// (2^-64 / 2^64 when 2^e is outside fp32) that leaves every accumulator
// value in range exact, and p2 carries the single rounding.
struct Pow2Apply {
  float p1, p2;
  __device__ __forceinline__ float operator()(float t) const { return __fmul_rn(__fmul_rn(t, p1), p2); }
};

// True when m 2^e (m in [0.25, 1)) is a normal fp32: then RN(t (m 2^e)) =
// RN(RN(t m) 2^e) for every t whose result is normal (the power-of-two step
// is exact there), so the output scale is one multiply.
__device__ __forceinline__ bool scale_is_normal(int e) { return e >= -124 && e <= 127; }

__device__ __forceinline__ Pow2Apply pow2_apply(int e) {
  Pow2Apply a;
  if (e > 127) {
    a.p1 = pow2f(64);
    a.p2 = pow2f(e - 64 < 127 ? e - 64 : 127);
  } else if (e >= -149) {
    a.p1 = 1.0f;
    a.p2 = pow2f(e);
  } else {
    a.p1 = pow2f(-64);
    a.p2 = pow2f(e + 64 > -149 ? e + 64 : -149);
  }
  return a;
}

// Byte offset of the scale of (row, block) in an NVFP4 scale buffer.
__device__ __host__ __forceinline__ int64_t scale_offset(int64_t row, int64_t blk, int64_t cols,
                                                         int layout) {
  if (layout == 0) return row * (cols / kBlock) + blk;
  const int64_t k4 = (cols + 63) / 64;   // 512-byte atoms per 128-row block
  return ((row >> 7) * k4 + (blk >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (blk & 3);
}

// Programmatic dependent launch (kernels started by launch_k): pdl_wait()
// returns once the previous kernel of the stream has completed and its
// writes are visible; every thread calls it before its first global memory
// access.  pdl_launch_dependents() lets the next kernel of the stream be
// scheduled (it then waits in its own pdl_wait()).  Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// 2-D tensor load (TMA) of one box into this CTA's shared memory; its bytes
// complete on the mbarrier at shared address `bar`.  The innermost
// coordinate times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar) : "memory");
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
