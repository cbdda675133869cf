// Block-scaled FP4 (NVFP4) GEMM on the 5th-generation tensor cores of sm_100a
// with the RAC residual folded in as a second K segment:
//
//     Y = s_tA s_tB (A B^T) + s_tR s_tWs (R Ws^T)
//
// A / R: quantized activations / gathered residual [M, K] / [M, width],
// B / Ws: quantized weights / gathered weight columns [N, K] / [N, width],
// all K-major packed E2M1 with E4M3 scales per 16 elements (MMA-tiled layout).
// QUADS technical summary (gist.science): native W4A4 GEMM on Blackwell
// (section 1), the residual correction added to the quantized output while the
// bulk keeps native W4A4 throughput (section 2.2 B).
//
// Design (one CTA per SM, persistent over 128 x 128 output tiles):
//   warp 0      TMA producer: per 256-element K step, two 2-D tensor copies
//               (A and B tiles, 128 B rows, 128 B swizzle) and two bulk
//               copies of the matching 128 x 16 scale atoms into a 4/5-stage
//               shared-memory ring guarded by full / empty mbarriers.
//   warp 6      scale copier: copies each stage's scales into that stage's
//               own TMEM columns (tcgen05.cp 32x128b.warpx4) and commits
//               them to a per-stage barrier.  The copies are issued by their
//               own thread: from the MMA thread they throttled its issue.
//   warp 1      MMA issuer: waits for the stage's data and scales, issues four
//               tcgen05.mma kind::mxf4nvf4 (128 x 128 x 64, ue4m3 scales per
//               16 elements) into accumulator 0 for the plain K segment and
//               accumulator 1 for the residual segment; tcgen05.commit frees
//               the stage and, after the last step, signals the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of both accumulators (TMEM lane = output
//               row), Y = alpha0 acc0 + alpha1 acc1 into a shared staging tile,
//               TMEM released, then coalesced fp32 / bf16 row stores.
// The two tensor scales differ, so the segments accumulate separately.  Every
// CTA loads its own tiles (no load is shared between CTAs).  Every mbarrier
// wait is bounded (see common.cuh).
//
// For dense activations with at least 256 rows (where its waves of tiles
// take no longer; see dense_pair_pays) a second kernel runs the same
// product on CTA pairs (tcgen05 cta_group::2): a pair computes a 256 x 256
// tile, each CTA loading its own 128 rows of A and of B, so a pair fetches
// half the operand bytes per FLOP of two 128 x 128 tiles; the leader's copier
// warp copies both CTAs' scales (12 copies per K step).  Its TMEM holds one
// 256-column accumulator; the residual segment is computed first and scaled
// in place by s_R s_Ws / (s_X s_W) (tcgen05.ld, multiply, tcgen05.st), then
// the plain segment accumulates on top and Y = s_X s_W acc.
//
// Dense products with few 128 x 128 tiles (decode shapes) run the single-CTA
// body split over K: a cluster of S = 2 or 4 CTAs per tile, CTA s taking the
// K steps [T s / S, T (s + 1) / S) of the two segments.  Each CTA writes its
// scaled fp32 partial over its idle pipeline stages; after a cluster
// barrier, CTA s sums rows s 128/S .. of all S partials in CTA order through
// distributed shared memory (ld.shared::cluster) and stores them; a second
// barrier keeps every CTA until its partial has been read.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstdlib>

#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int BM = 128, BN = 128;
constexpr int BK_BYTES = 128;                    // 256 FP4 elements per K step
constexpr int A_STAGE = BM * BK_BYTES;           // 16 KB
constexpr int B_STAGE = BN * BK_BYTES;           // 16 KB
constexpr int SF_ATOM = 512;                     // 128 rows x 4 scales
constexpr int SF_STAGE = 4 * SF_ATOM;            // 4 MMA K blocks per step

// Per output type: pipeline depth and the epilogue staging tile (128 rows,
// row stride padded by 16 bytes so 16-byte shared stores of 8 consecutive
// rows hit distinct banks).
template <int YBYTES, bool SPLIT = false>
struct Cfg {
  // the split-K form keeps no epilogue staging tile (its partials go over
  // the idle stages): one more stage
  static constexpr int STAGES = SPLIT ? 6 : (YBYTES == 2 ? 5 : 4);
  static constexpr int STG_STRIDE = BN * YBYTES + 16;
  static constexpr int STG_BYTES = SPLIT ? 0 : BM * STG_STRIDE;
  static constexpr int SMEM_BYTES = 1024 + STAGES * (A_STAGE + B_STAGE + 2 * SF_STAGE) + STG_BYTES + 256;
};constexpr uint32_t TMEM_COLS = 512;
// split-K partial tile: 128 fp32 rows of 128 columns, row stride padded by
// 16 bytes (528 B), over the idle pipeline stages of A and B
constexpr int kSplitStride = BN + 4;
constexpr uint32_t ACC0_COL = 0, ACC1_COL = 128;   // two 128-column fp32 accumulators
// block scales: per pipeline stage 32 columns (16 for A, 16 for B)
constexpr uint32_t SF1_COL = 256, SF1_STAGE_COLS = 32;
// warps of the single-CTA kernel: 0 TMA producer, 1 MMA issuer, 2..5
// epilogue, 6 scale-factor copier
constexpr int THREADS1 = 224;

// kind::mxf4nvf4 instruction descriptor: E2M1 x E2M1, ue4m3 scales, both
// K-major, N = 128, M = 128.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct KParams {
  RowGroups g;
  int64_t N;
  int64_t m_tiles_dense;
  int n_tiles;
  int kt[2], kb_last[2];
  const uint8_t* sfa[2];
  const uint8_t* sfb[2];
  int64_t sfa_rb[2], sfb_rb[2];   // bytes per 128-row block of the scale buffers
  int64_t sfa_bytes[2], sfb_bytes[2];   // sizes of the scale buffers (index checks)
  const float* sta[2];
  const float* stb[2];
  void* y;
  int y_dtype;
  int64_t ldy, M;
  unsigned* err;
  int split;                      // split-K kernel: CTAs (a cluster) per output tile
};

// ---- PTX wrappers ---------------------------------------------------------
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused (1).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (1ull << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Descriptor of a 512-byte scale atom (32 rows x 16 bytes, no swizzle):
// 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (1ull << 46);
}

__device__ __forceinline__ void utccp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_fp4(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(d), "l"(a), "l"(b), "r"(IDESC), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
}

// kind::mxf8f6f4 instruction descriptor: E4M3 x E4M3 (format 0), UE8M0
// scales (bit 23), both K-major, N = 128, M = 128.  Bits 29-30 / 4-5 select
// which byte of a row's 32-bit scale word in TMEM the MMA reads (the j-th
// 32-element block of a 128-element K step).
constexpr uint32_t IDESC8 = (1u << 23) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

__device__ __forceinline__ void mma_fp8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                        uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Shared::cluster address of shared-window address saddr in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr_u32(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Distributed shared memory: a 16-byte load from the shared::cluster
// address of another CTA of the cluster.
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}

// ---- the kernel -----------------------------------------------------------
// The single-CTA kernel's body, for NVFP4 operands (FP8 = false: 256
// elements per 128-byte K step, four kind::mxf4nvf4 MMAs of K = 64, one
// 512-byte scale atom per MMA) or MXFP8 operands (FP8 = true: 128 elements
// per K step, four kind::mxf8f6f4 MMAs of K = 32 reading the four bytes of
// one scale atom, no residual segment).
template <int YBYTES, bool FP8, bool SPLIT = false>
__device__ __forceinline__ void gemm1_body(const CUtensorMap& tmA0, const CUtensorMap& tmB0,
                                           const CUtensorMap& tmA1, const CUtensorMap& tmB1,
                                           const KParams& p) {
  constexpr int STAGES = Cfg<YBYTES, SPLIT>::STAGES;
  constexpr int SF_STEP = FP8 ? SF_ATOM : SF_STAGE;        // scale bytes per K step and operand
  constexpr int STG_STRIDE = Cfg<YBYTES, SPLIT>::STG_STRIDE;
  static_assert(!SPLIT || BM * kSplitStride * 4 <= STAGES * (A_STAGE + B_STAGE),
                "split-K partial tile fits over the A and B stages");
  static_assert(Cfg<YBYTES, SPLIT>::SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled tiles need 1024-byte aligned shared addresses
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE;
  uint8_t* sSFA = sB + STAGES * B_STAGE;
  uint8_t* sSFB = sSFA + STAGES * SF_STAGE;
  uint8_t* sOut = sSFB + STAGES * SF_STAGE;                     // epilogue staging
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + Cfg<YBYTES, SPLIT>::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_ready = empty + STAGES;       // the stage's scales are in TMEM
  uint64_t* tmem_full = sf_ready + STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint64_t* drain_cp = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_cp + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 128);
    mbar_init(drain, 1);
    mbar_init(drain_cp, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // barriers and TMEM are set up: wait for the previous kernel's writes
  pdl_wait();
  pdl_launch_dependents();

  const int64_t m_tiles = p.g.off ? p.g.tile_start[p.g.E] : p.m_tiles_dense;
  const int64_t total = m_tiles * p.n_tiles;
  const int nseg = p.kt[1] > 0 ? 2 : 1;
  // split-K (dense only): the S CTAs of a cluster share one tile, CTA s
  // taking K steps [T s / S, T (s + 1) / S) of the two segments in order;
  // otherwise persistent over the tiles with the whole of K
  const int S = SPLIT ? p.split : 1;
  const int sidx = SPLIT ? static_cast<int>(blockIdx.x % static_cast<unsigned>(S)) : 0;
  const int64_t tile_first = SPLIT ? blockIdx.x / S : blockIdx.x;
  const int64_t tile_step = SPLIT ? total : gridDim.x;
  const int T = p.kt[0] + (nseg > 1 ? p.kt[1] : 0);
  const int k_lo = T * sidx / S, k_hi = T * (sidx + 1) / S;
  auto kbeg = [&](int seg) { const int b = k_lo - (seg ? p.kt[0] : 0); return b > 0 ? b : 0; };
  auto kend = [&](int seg) {
    const int e = k_hi - (seg ? p.kt[0] : 0);
    return e < p.kt[seg] ? e : p.kt[seg];
  };
  const bool has0 = kend(0) > kbeg(0), has1 = nseg > 1 && kend(1) > kbeg(1);
  // the output scale factors depend on the row group only (dense: one
  // group); formed by the epilogue warps, used again by the split-K reduction
  int cur_e = -1;
  float c0 = 0.0f, c1 = 0.0f, c0n = 0.0f, c1n = 0.0f;
  Pow2Apply out{1.0f, 1.0f};
  bool one = true;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;     // per-stage: filled at least once / its parity
      bool ok = true;
      for (int64_t tile = tile_first; tile < total && ok; tile += tile_step) {
        const int64_t mt = tile / p.n_tiles, nt = tile % p.n_tiles;
        const TileInfo ti = tile_info(p.g, mt);
        const int64_t b_row = static_cast<int64_t>(ti.e) * p.N + nt * BN;
        for (int seg = 0; seg < nseg && ok; ++seg) {
          const CUtensorMap* tA = seg ? &tmA1 : &tmA0;
          const CUtensorMap* tB = seg ? &tmB1 : &tmB0;
          for (int kt = kbeg(seg); kt < kend(seg); ++kt) {
            if (!mbar_wait(&empty[stage], phase ^ 1, p.err)) { ok = false; break; }
            const int nkb = kt == p.kt[seg] - 1 ? p.kb_last[seg] : 4;
            const uint32_t sf_bytes = FP8 ? SF_ATOM : nkb * SF_ATOM;
            const uint32_t fb = smem_u32(&full[stage]);
            const int64_t sfa_off = mt * p.sfa_rb[seg] + kt * SF_STEP;
            const int64_t sfb_off = (b_row / BN) * p.sfb_rb[seg] + kt * SF_STEP;
            if (!NV_IDX(sfa_off + sf_bytes <= p.sfa_bytes[seg] && sfb_off + sf_bytes <= p.sfb_bytes[seg])) {
              ok = false;                          // (checked build) never issue the out-of-range copy
              break;
            }
            mbar_arrive_expect_tx(&full[stage], A_STAGE + B_STAGE + 2 * sf_bytes);
            tma_load_2d(smem_u32(sA + stage * A_STAGE), tA, kt * BK_BYTES, static_cast<int>(mt * BM), fb);
            tma_load_2d(smem_u32(sB + stage * B_STAGE), tB, kt * BK_BYTES, static_cast<int>(b_row), fb);
            bulk_load(smem_u32(sSFA + stage * SF_STAGE), p.sfa[seg] + sfa_off, sf_bytes, fb);
            bulk_load(smem_u32(sSFB + stage * SF_STAGE), p.sfb[seg] + sfb_off, sf_bytes, fb);
            armed |= 1u << stage;
            armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      // let every copy in flight land before the CTA can exit
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_phase >> s) & 1u, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t tile = tile_first; tile < total && ok; tile += tile_step) {
        if (!mbar_wait(tmem_empty, acc_phase ^ 1, p.err)) break;
        tc_fence_after();
        for (int seg = 0; seg < nseg && ok; ++seg) {
          const uint32_t d = tmem + (seg ? ACC1_COL : ACC0_COL);
          for (int kt = kbeg(seg); kt < kend(seg); ++kt) {
            if (!mbar_wait(&full[stage], phase, p.err) || !mbar_wait(&sf_ready[stage], phase, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int nkb = kt == p.kt[seg] - 1 ? p.kb_last[seg] : 4;
            const uint32_t a0 = smem_u32(sA + stage * A_STAGE), b0 = smem_u32(sB + stage * B_STAGE);
            const uint32_t sfa = tmem + SF1_COL + SF1_STAGE_COLS * stage, sfb = sfa + 16;
            for (int j = 0; j < nkb; ++j) {
              if (FP8)
                mma_fp8(d, desc_sw128(a0 + 32 * j), desc_sw128(b0 + 32 * j),
                        IDESC8 | (static_cast<uint32_t>(j) << 29) | (static_cast<uint32_t>(j) << 4), sfa, sfb,
                        (kt > kbeg(seg) || j > 0) ? 1u : 0u);
              else
                mma_fp4(d, desc_sw128(a0 + 32 * j), desc_sw128(b0 + 32 * j), sfa + 4 * j, sfb + 4 * j,
                        (kt > kbeg(seg) || j > 0) ? 1u : 0u);
            }
            umma_commit(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
        umma_commit(tmem_full);
        acc_phase ^= 1;
      }
      umma_commit(drain);                 // all issued tensor-core work done
      mbar_wait(drain, 0, p.err);
    }
  } else if (warp == 6) {
    if (lane == 0) {
      // ------------------------------ scale-factor copier: smem -> TMEM
      // copies of the stage's block scales; completion arrives on
      // sf_ready[stage], which the MMA issuer waits for
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t tile = tile_first; tile < total && ok; tile += tile_step) {
        for (int seg = 0; seg < nseg && ok; ++seg) {
          for (int kt = kbeg(seg); kt < kend(seg); ++kt) {
            if (!mbar_wait(&full[stage], phase, p.err)) { ok = false; break; }
            tc_fence_after();
            const int nkb = kt == p.kt[seg] - 1 ? p.kb_last[seg] : 4;
            const uint32_t fa = smem_u32(sSFA + stage * SF_STAGE), fb = smem_u32(sSFB + stage * SF_STAGE);
            const uint32_t sfa = tmem + SF1_COL + SF1_STAGE_COLS * stage, sfb = sfa + 16;
            for (int j = 0; j < (FP8 ? 1 : nkb); ++j) {
              utccp_sf(sfa + 4 * j, desc_sf(fa + j * SF_ATOM));
              utccp_sf(sfb + 4 * j, desc_sf(fb + j * SF_ATOM));
            }
            umma_commit(&sf_ready[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      umma_commit(drain_cp);
      mbar_wait(drain_cp, 0, p.err);
    }
  } else {
    // ------------------------------ epilogue (warps 2..5)
    // TMEM -> registers -> Y = a0 acc0 + a1 acc1 -> shared staging (this
    // warp's 32 rows); TMEM is released before the global stores so the next
    // tile's MMAs overlap them; rows then leave as coalesced 256/512 B stores.
    const int q = warp & 3;                        // TMEM lane quadrant of this warp
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    uint8_t* stg_warp = sOut + (32 * q) * STG_STRIDE;
    uint8_t* stg_row = stg_warp + lane * STG_STRIDE;
    uint32_t acc_phase = 0;
    for (int64_t tile = tile_first; tile < total; tile += tile_step) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(tmem_full, acc_phase, p.err);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int64_t mt = tile / p.n_tiles, nt = tile % p.n_tiles;
      const TileInfo ti = tile_info(p.g, mt);
      if (ti.e != cur_e) {
        // Y = a0 acc0 + a1 acc1 with a_s = s_tA,s s_tB,s = m_s 2^e_s: both
        // segments in the units 2^E of the first nonzero one, then one
        // power-of-two step (see Pow2Apply)
        // (MXFP8 operands carry no tensor scale: the scale product is 1)
        const ScaleProduct a0 = FP8 ? ScaleProduct{0.5f, 1} : scale_product(p.sta[0][ti.e], p.stb[0][ti.e]);
        const ScaleProduct a1 = nseg > 1 ? scale_product(p.sta[1][ti.e], p.stb[1][ti.e]) : ScaleProduct{0.0f, 0};
        const int E = a0.m != 0.0f ? a0.e : a1.e;
        c0 = a0.m;
        c1 = a1.m != 0.0f ? ldexpf(a1.m, a1.e - E) : 0.0f;
        out = pow2_apply(E);
        // with both segment scales normal the power-of-two step folds into
        // them (exact scaling, the same roundings for normal results)
        one = scale_is_normal(E) && (a1.m == 0.0f || scale_is_normal(a1.e));
        c0n = one ? ldexpf(c0, E) : 0.0f;
        c1n = one ? ldexpf(c1, E) : 0.0f;
        cur_e = ti.e;
      }
      if (SPLIT) {
        // this CTA's part of the tile, c0 acc0 + c1 acc1 over its K steps
        // (with `one`, the power-of-two step folded in), as fp32 rows of the
        // partial buffer over the idle pipeline stages
        float* part = reinterpret_cast<float*>(sA);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32], u[32];
          if (has0) tmem_ld32(trow + ACC0_COL + 32 * c, v);
          if (has1) tmem_ld32(trow + ACC1_COL + 32 * c, u);
          tmem_ld_wait();
          const float a0 = one ? c0n : c0, a1 = one ? c1n : c1;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x0 = has0 ? __fmul_rn(a0, v[i]) : 0.0f, x1 = has1 ? __fmul_rn(a1, u[i]) : 0.0f;
            v[i] = __fadd_rn(x0, x1);
          }
          float* dst = part + (32 * q + lane) * kSplitStride + 32 * c;
#pragma unroll
          for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
        tc_fence_before();
        acc_phase ^= 1;
        continue;
      }
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float v[32], u[32];
        tmem_ld32(trow + ACC0_COL + 32 * c, v);
        if (nseg > 1) tmem_ld32(trow + ACC1_COL + 32 * c, u);
        tmem_ld_wait();
        if (nseg > 1 && one) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __fadd_rn(__fmul_rn(c0n, v[i]), __fmul_rn(c1n, u[i]));
        } else if (nseg > 1) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = out(__fadd_rn(__fmul_rn(c0, v[i]), __fmul_rn(c1, u[i])));
        } else if (one) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(c0n, v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = out(__fmul_rn(c0, v[i]));
        }
        if (YBYTES == 4) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(stg_row + (32 * c + i) * 4) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        } else {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i]))) |
                   (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1]))) << 16);
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<uint4*>(stg_row + (32 * c + 2 * i) * 2) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(tmem_empty);                     // accumulators free for the next tile
      __syncwarp();
      const int64_t col = nt * BN + 4 * lane;      // this lane's 4 columns of every row
      const bool col_ok = col + 4 <= p.N;
#pragma unroll 4
      for (int r = 0; r < 32; ++r) {
        const int64_t row = ti.row0 + 32 * q + r;
        if (!ti.valid || row >= ti.row_end || !col_ok || !NV_IDX(row < p.M)) continue;
        const uint8_t* src = stg_warp + r * STG_STRIDE + lane * 4 * YBYTES;
        if (YBYTES == 4)
          *reinterpret_cast<float4*>(static_cast<float*>(p.y) + row * p.ldy + col) = *reinterpret_cast<const float4*>(src);
        else
          *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.y) + row * p.ldy + col) = *reinterpret_cast<const uint2*>(src);
      }
      __syncwarp();
      acc_phase ^= 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (SPLIT) {
    // the tile's rows r0 .. r0 + 128/S - 1 of this CTA: the S partials in
    // CTA order through distributed shared memory, then Y (the cluster
    // barriers: every partial written before any is read, and no CTA leaves
    // while its partial may still be read)
    cluster_sync_all();
    if (warp >= 2 && warp <= 5 && tile_first < total) {
      const int64_t mt = tile_first / p.n_tiles, nt = tile_first % p.n_tiles;
      const int rows = BM / S, r0 = sidx * rows;
      const uint32_t pbase = smem_u32(sA);
      for (int idx = threadIdx.x - 64; idx < rows * (BN / 4); idx += 128) {
        const int row = r0 + idx / (BN / 4), c4 = idx % (BN / 4);
        const uint32_t off = static_cast<uint32_t>((row * kSplitStride + 4 * c4) * 4);
        float4 acc = ld_cluster_f4(peer_addr_u32(pbase + off, 0));
        for (int sp = 1; sp < S; ++sp) {
          const float4 t = ld_cluster_f4(peer_addr_u32(pbase + off, static_cast<uint32_t>(sp)));
          acc.x = __fadd_rn(acc.x, t.x);
          acc.y = __fadd_rn(acc.y, t.y);
          acc.z = __fadd_rn(acc.z, t.z);
          acc.w = __fadd_rn(acc.w, t.w);
        }
        if (!one) {
          acc.x = out(acc.x);
          acc.y = out(acc.y);
          acc.z = out(acc.z);
          acc.w = out(acc.w);
        }
        const int64_t grow = mt * BM + row, gcol = nt * BN + 4 * c4;
        if (grow >= p.M || gcol + 4 > p.N || !NV_IDX(grow < p.M)) continue;
        if (YBYTES == 4) {
          *reinterpret_cast<float4*>(static_cast<float*>(p.y) + grow * p.ldy + gcol) = acc;
        } else {
          const uint32_t lo = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc.x))) |
                              (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc.y))) << 16);
          const uint32_t hi = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc.z))) |
                              (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc.w))) << 16);
          *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.y) + grow * p.ldy + gcol) = make_uint2(lo, hi);
        }
      }
    }
    cluster_sync_all();
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

template <int YBYTES>
__global__ void __launch_bounds__(THREADS1, 1)
w4a4_rac_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                     const KParams p) {
  gemm1_body<YBYTES, false>(tmA0, tmB0, tmA1, tmB1, p);
}

// Split-K form (dense products with few tiles): a cluster of p.split CTAs
// per output tile, the partials reduced through distributed shared memory.
template <int YBYTES>
__global__ void __launch_bounds__(THREADS1, 1)
w4a4_rac_gemm_split_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                           const KParams p) {
  gemm1_body<YBYTES, false, true>(tmA0, tmB0, tmA1, tmB1, p);
}

// MXFP8 x MXFP8 (the FP8 comparator): one K segment.
template <int YBYTES>
__global__ void __launch_bounds__(THREADS1, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                 const KParams p) {
  gemm1_body<YBYTES, true>(tmA0, tmB0, tmA0, tmB0, p);
}

// ---- host side -------------------------------------------------------------
// 2-D map over packed FP4 codes [rows, cols/2] bytes (or, with row_bytes,
// any byte matrix [rows, row_bytes]), box 128 B x box_rows.
bool make_code_map(CUtensorMap* tm, const uint8_t* codes, int64_t rows, int64_t cols, int box_rows,
                   int64_t row_bytes = -1) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const int64_t rb = row_bytes >= 0 ? row_bytes : cols / 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(rb)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK_BYTES), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// NVFP4_GEMM_SINGLE_CTA=1 in the environment keeps every GEMM on the
// single-CTA kernel (used to compare the two kernels).
bool gemm_force_single_cta() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("NVFP4_GEMM_SINGLE_CTA");
    v = (e != nullptr && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

// NVFP4_GEMM_NO_SPLIT=1 in the environment keeps the single-CTA kernel
// persistent over whole tiles (no split over K; used to compare the two).
bool gemm_no_split() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("NVFP4_GEMM_NO_SPLIT");
    v = (e != nullptr && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

template <int YBYTES>
cudaError_t prepare_kernel() {
  static bool done[kMaxAttrDevices] = {};
  return set_max_smem(w4a4_rac_gemm_kernel<YBYTES>, Cfg<YBYTES>::SMEM_BYTES, done);
}

template <int YBYTES>
cudaError_t prepare_split_kernel() {
  static bool done[kMaxAttrDevices] = {};
  return set_max_smem(w4a4_rac_gemm_split_kernel<YBYTES>, Cfg<YBYTES, true>::SMEM_BYTES, done);
}

template <int YBYTES>
cudaError_t prepare_kernel8() {
  static bool done[kMaxAttrDevices] = {};
  return set_max_smem(w8a8_gemm_kernel<YBYTES>, Cfg<YBYTES>::SMEM_BYTES, done);
}

// ===========================================================================
// CTA-pair kernel (tcgen05 cta_group::2), dense activations.
// ===========================================================================
// FP8 = true: MXFP8 operands (the FP8 comparator): one scale atom per 128
// rows and K step (4 blocks of 32), four kind::mxf8f6f4 MMAs reading its bytes.
template <int YBYTES, bool FP8 = false>
struct Cfg2 {
  static constexpr int STAGES = YBYTES == 2 ? 5 : 4;
  static constexpr int A_ST = 128 * BK_BYTES;          // own 128 rows of A
  static constexpr int B_ST = 128 * BK_BYTES;          // own 128 rows (N half) of B
  static constexpr int SFA_ST = (FP8 ? 1 : 4) * SF_ATOM;   // own 128 rows x 4 K blocks
  static constexpr int SFB_ST = (FP8 ? 2 : 8) * SF_ATOM;   // all 256 N rows x 4 K blocks
  static constexpr int STAGE = A_ST + B_ST + SFA_ST + SFB_ST;
  static constexpr int STG_STRIDE = 128 * YBYTES + 16; // staging: 128 columns per half tile
  static constexpr int STG_BYTES = 128 * STG_STRIDE;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + STG_BYTES + 512;
  static constexpr uint32_t TX = 2 * STAGE;            // bytes landing per stage (both CTAs)
};

// Warps of the pair kernel: 0 TMA producer, 1 MMA issuer, 2..5 epilogue,
// 6 scale-factor copier (leader CTA).
constexpr int THREADS2 = 224;
// TMEM columns: the 256-column accumulator, then per pipeline stage 48
// columns of block scales (16 for A, 32 for B), so the copies for later
// stages run while the MMAs of earlier ones read theirs.
constexpr uint32_t ACC2_COL = 0, SF2_COL = 256, SF2_STAGE_COLS = 48;
// kind::mxf4nvf4, M = 256 (pair), N = 256, both K-major, ue4m3 scales.
constexpr uint32_t IDESC2 = (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) | (uint32_t(256 >> 4) << 24);
// kind::mxf8f6f4, M = 256, N = 256: E4M3 x E4M3, UE8M0 scales (bit 23); bits
// 29-30 / 4-5 pick the byte of the scale word (see IDESC8).
constexpr uint32_t IDESC2_8 = (1u << 23) | (uint32_t(256 >> 3) << 17) | (uint32_t(256 >> 4) << 24);

struct KParams2 {
  int64_t M, N;
  int m_tiles, n_tiles;        // 256-row (dense) / 256-column tiles
  int kt[2];                   // K steps of the residual (0) and plain (1) segments
  const float* sta[2];         // tensor scales, one per group
  const float* stb[2];
  RowGroups g;                 // row groups of A and Y (g.off null: dense)
  const int32_t* pair_start;   // groups: prefix of each group's 256-row tiles
  void* y;
  int64_t ldy;
  unsigned* err;
};

// Rows of a 256-row pair tile.  Dense: tile mt covers rows 256 mt .. +255.
// Groups: pair tile pt belongs to the group e with pair_start[e] <= pt <
// pair_start[e + 1]; its two 128-row halves are the group's 128-row tiles
// 2 lp and 2 lp + 1 (lp = pt - pair_start[e]) on the padded rows; a half past
// the group's last tile computes rows that are never stored.
struct PairRows {
  int e;
  int64_t a_tile;              // this CTA's 128-row tile (padded rows / 128)
  int64_t local0;              // first row of this CTA's half within the group
  int64_t out0;                // output row of local row 0 of the group
  int64_t m;                   // rows of the group
};

__device__ __forceinline__ PairRows pair_rows(const KParams2& p, int64_t pt, uint32_t rank) {
  PairRows r;
  if (p.g.off == nullptr) {
    r.e = 0;
    r.a_tile = 2 * pt + rank;
    r.local0 = r.a_tile * 128;
    r.out0 = 0;
    r.m = p.M;
    return r;
  }
  int lo = 0, hi = p.g.E - 1;                      // last e with pair_start[e] <= pt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.pair_start[mid] <= pt) lo = mid; else hi = mid - 1;
  }
  const int64_t local_tile = 2 * (pt - p.pair_start[lo]) + rank;
  r.e = lo;
  r.a_tile = p.g.tile_start[lo] + local_tile;
  r.local0 = local_tile * 128;
  r.out0 = p.g.off[lo];
  r.m = p.g.off[lo + 1] - p.g.off[lo];
  return r;
}

// 2-D tensor load into this CTA's shared memory that completes its bytes on
// an mbarrier of the CTA pair (here: the leader's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void utccp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_fp8_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                             uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
}

__device__ __forceinline__ void mma_fp4_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa, uint32_t sfb,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(d), "l"(a), "l"(b), "r"(IDESC2), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
}

// Completion of this thread's tcgen05 work arrives on the mbarrier at the
// same shared offset in both CTAs of the pair.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               :: "r"(smem_u32(bar)), "h"(static_cast<uint16_t>(3)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      :: "r"(taddr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
         "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
         "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
         "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
         "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

template <int YBYTES, bool FP8>
__device__ __forceinline__ void gemm2_body(const CUtensorMap& tmA0, const CUtensorMap& tmB0, const CUtensorMap& tmSA0,
                                           const CUtensorMap& tmSB0, const CUtensorMap& tmA1, const CUtensorMap& tmB1,
                                           const CUtensorMap& tmSA1, const CUtensorMap& tmSB1, const KParams2& p) {
  using C = Cfg2<YBYTES, FP8>;
  constexpr int SF_X = FP8 ? 64 : 256;          // scale-map x extent of one K step (int64 units)
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sStage = smem;                                       // [STAGES][A | B | SFA | SFB]
  uint8_t* sOut = smem + STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + C::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_ready = empty + STAGES;   // the stage's scales are in TMEM
  uint64_t* tmem_full = sf_ready + STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* res_full = tmem_empty + 1;
  uint64_t* res_done = res_full + 1;
  uint64_t* drain = res_done + 1;
  uint64_t* drain_cp = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_cp + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 8);          // one arrival per epilogue warp of both CTAs
    mbar_init(res_full, 1);
    mbar_init(res_done, 8);
    mbar_init(drain, 1);
    mbar_init(drain_cp, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  cluster_sync_all();                  // barriers of both CTAs initialised
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // barriers and TMEM are set up: wait for the previous kernel's writes
  pdl_wait();
  pdl_launch_dependents();

  const int total = (p.g.off == nullptr ? p.m_tiles : p.pair_start[p.g.E]) * p.n_tiles;
  const bool has_res = p.kt[0] > 0;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
        const PairRows pr = pair_rows(p, mt, rank);
        const int a_row = static_cast<int>(pr.a_tile * 128);
        const int b_row0 = static_cast<int>(pr.e * p.N) + nt * 256;      // this group's B rows
        const int b_row = b_row0 + static_cast<int>(rank) * 128;
        for (int seg = has_res ? 0 : 1; seg < 2 && ok; ++seg) {
          const CUtensorMap* tA = seg ? &tmA1 : &tmA0;
          const CUtensorMap* tB = seg ? &tmB1 : &tmB0;
          const CUtensorMap* tSA = seg ? &tmSA1 : &tmSA0;
          const CUtensorMap* tSB = seg ? &tmSB1 : &tmSB0;
          for (int kt = 0; kt < p.kt[seg]; ++kt) {
            if (!mbar_wait(&empty[stage], phase ^ 1, p.err)) { ok = false; break; }
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], C::TX);
            const uint32_t lead_full = peer_addr(&full[stage], 0);
            uint8_t* st = sStage + stage * C::STAGE;
            tma_load_2d_pair(smem_u32(st), tA, kt * BK_BYTES, a_row, lead_full);
            tma_load_2d_pair(smem_u32(st + C::A_ST), tB, kt * BK_BYTES, b_row, lead_full);
            tma_load_2d_pair(smem_u32(st + C::A_ST + C::B_ST), tSA, kt * SF_X, a_row / 128, lead_full);
            tma_load_2d_pair(smem_u32(st + C::A_ST + C::B_ST + C::SFA_ST), tSB, kt * SF_X, b_row0 / 128, lead_full);
            armed |= 1u << stage;
            armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      // let this CTA's copies land before it can exit: the stages it filled
      // are freed (empty) once the leader's MMAs consumed them
      if (rank == 0) {
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (armed_phase >> s) & 1u, p.err);
      } else {
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&empty[s], (armed_phase >> s) & 1u, p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------ MMA issuer (leader CTA only)
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0, res_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        if (!mbar_wait(tmem_empty, acc_phase ^ 1, p.err)) break;
        tc_fence_after();
        for (int seg = has_res ? 0 : 1; seg < 2 && ok; ++seg) {
          for (int kt = 0; kt < p.kt[seg]; ++kt) {
            if (!mbar_wait(&full[stage], phase, p.err) || !mbar_wait(&sf_ready[stage], phase, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(sStage + stage * C::STAGE);
            const uint32_t a0 = st, b0 = st + C::A_ST;
            const uint32_t sfa = tmem + SF2_COL + SF2_STAGE_COLS * stage, sfb = sfa + 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t accum = (seg == 1 && has_res) ? 1u : ((kt > 0 || j > 0) ? 1u : 0u);
              if (FP8)
                mma_fp8_pair(tmem + ACC2_COL, desc_sw128(a0 + 32 * j), desc_sw128(b0 + 32 * j),
                             IDESC2_8 | (static_cast<uint32_t>(j) << 29) | (static_cast<uint32_t>(j) << 4), sfa, sfb,
                             accum);
              else
                mma_fp4_pair(tmem + ACC2_COL, desc_sw128(a0 + 32 * j), desc_sw128(b0 + 32 * j),
                             sfa + 4 * j, sfb + 8 * j, accum);
            }
            umma_commit_pair(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          if (seg == 0 && ok) {
            // residual product ready: let the epilogue scale it in place
            umma_commit_pair(res_full);
            if (!mbar_wait(res_done, res_phase, p.err)) { ok = false; break; }
            tc_fence_after();
            res_phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(tmem_full);
        acc_phase ^= 1;
      }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                   :: "r"(smem_u32(drain)) : "memory");
      mbar_wait(drain, 0, p.err);
    }
  } else if (warp == 6) {
    if (lane == 0 && rank == 0) {
      // ------------------------------ scale-factor copier (leader CTA only)
      // smem -> TMEM copies of both CTAs' block scales for each stage; their
      // completion arrives on sf_ready[stage], which the MMA issuer waits for
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        for (int seg = has_res ? 0 : 1; seg < 2 && ok; ++seg) {
          for (int kt = 0; kt < p.kt[seg]; ++kt) {
            if (!mbar_wait(&full[stage], phase, p.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t fa = smem_u32(sStage + stage * C::STAGE) + C::A_ST + C::B_ST, fb = fa + C::SFA_ST;
            const uint32_t sfa = tmem + SF2_COL + SF2_STAGE_COLS * stage, sfb = sfa + 16;
            if (FP8) {
              // one atom of A, the two 128-row atoms of B; every MMA of the
              // step reads these columns (its own byte of each word)
              utccp_sf_pair(sfa, desc_sf(fa));
              utccp_sf_pair(sfb, desc_sf(fb));
              utccp_sf_pair(sfb + 4, desc_sf(fb + SF_ATOM));
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                utccp_sf_pair(sfa + 4 * j, desc_sf(fa + j * SF_ATOM));
                utccp_sf_pair(sfb + 8 * j, desc_sf(fb + j * SF_ATOM));
                utccp_sf_pair(sfb + 8 * j + 4, desc_sf(fb + 4 * SF_ATOM + j * SF_ATOM));
              }
            }
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         :: "r"(smem_u32(&sf_ready[stage])) : "memory");
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                   :: "r"(smem_u32(drain_cp)) : "memory");
      mbar_wait(drain_cp, 0, p.err);
    }
  } else {
    // ------------------------------ epilogue (warps 2..5 of both CTAs)
    const int q = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    uint8_t* stg_warp = sOut + (32 * q) * C::STG_STRIDE;
    uint8_t* stg_row = stg_warp + lane * C::STG_STRIDE;
    const uint32_t lead_tmem_empty = peer_addr(tmem_empty, 0);
    const uint32_t lead_res_done = peer_addr(res_done, 0);
    uint32_t acc_phase = 0, res_phase = 0;
    // the output scale factors depend on the row group only: formed when it
    // changes (once for a dense product), not per tile
    int cur_e = -1;
    float ratio = 0.0f, fin = 0.0f, fin1 = 0.0f;
    Pow2Apply out{1.0f, 1.0f};
    bool one = true;
    for (int tile = pair; tile < total; tile += npairs) {
      const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
      const PairRows pr = pair_rows(p, mt, rank);
      if (pr.e != cur_e) {
        // the residual is scaled to the plain segment's units (ratio =
        // a_res / a_plain with a = s_tA s_tB = m 2^e), then Y = a_plain acc,
        // applied as RN(acc m) and one power-of-two step (see Pow2Apply).  A
        // zero plain scale means an all-zero X or W, whose residual and
        // W_sel are zero as well: Y = 0.
        const ScaleProduct ap = FP8 ? ScaleProduct{0.5f, 1} : scale_product(p.sta[1][pr.e], p.stb[1][pr.e]);
        const ScaleProduct ar = has_res ? scale_product(p.sta[0][pr.e], p.stb[0][pr.e]) : ScaleProduct{0.0f, 0};
        ratio = (ap.m != 0.0f && ar.m != 0.0f) ? ldexpf(__fdiv_rn(ar.m, ap.m), ar.e - ap.e) : 0.0f;
        fin = ap.m;
        out = pow2_apply(ap.e);
        // m 2^e as one fp32 multiplier when it is normal (see scale_is_normal)
        one = scale_is_normal(ap.e);
        fin1 = one ? ldexpf(fin, ap.e) : 0.0f;
        cur_e = pr.e;
      }
      // Y of 32 accumulator values in place
      auto scale32 = [&](float* v) {
        if (one) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(fin1, v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = out(__fmul_rn(fin, v[i]));
        }
      };
      bool ok = true;
      if (has_res) {
        if (lane == 0) ok = mbar_wait(res_full, res_phase, p.err);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; c += 2) {             // two loads in flight
          float v[32], u[32];
          tmem_ld32(trow + ACC2_COL + 32 * c, v);
          tmem_ld32(trow + ACC2_COL + 32 * (c + 1), u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v[i] = __fmul_rn(v[i], ratio);
            u[i] = __fmul_rn(u[i], ratio);
          }
          tmem_st32(trow + ACC2_COL + 32 * c, v);
          tmem_st32(trow + ACC2_COL + 32 * (c + 1), u);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_res_done);
        res_phase ^= 1;
      }
      if (lane == 0) ok = mbar_wait(tmem_full, acc_phase, p.err);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int64_t lrow0 = pr.local0 + 32 * q;     // first row of this warp within the group
      // rows of this warp (32 x 128 columns in the staging buffer) leave as
      // coalesced row stores
      auto store_rows = [&](int h) {
        const int64_t col = static_cast<int64_t>(nt) * 256 + 128 * h + 4 * lane;
        const bool col_ok = col + 4 <= p.N;
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
          if (lrow0 + r >= pr.m || !col_ok) continue;
          const int64_t row = pr.out0 + lrow0 + r;
          if (!NV_IDX(row < p.M)) continue;
          const uint8_t* src = stg_warp + r * C::STG_STRIDE + lane * 4 * YBYTES;
          if (YBYTES == 4)
            *reinterpret_cast<float4*>(static_cast<float*>(p.y) + row * p.ldy + col) = *reinterpret_cast<const float4*>(src);
          else
            *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.y) + row * p.ldy + col) = *reinterpret_cast<const uint2*>(src);
        }
      };
      if constexpr (YBYTES == 2) {
        // bf16: both halves leave TMEM first (the second one packed in
        // registers), so the accumulator is released before any global store
        // and the next tile's MMAs overlap the stores
        uint32_t hold[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32(trow + ACC2_COL + 128 * h + 32 * c, v);
            tmem_ld_wait();
            scale32(v);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[i]) : "f"(v[2 * i + 1]), "f"(v[2 * i]));
            if (h == 0) {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<uint4*>(stg_row + (32 * c + 2 * i) * 2) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) hold[16 * c + i] = w[i];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_tmem_empty);     // accumulator free
        store_rows(0);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 64; i += 4)
          *reinterpret_cast<uint4*>(stg_row + 4 * i) = make_uint4(hold[i], hold[i + 1], hold[i + 2], hold[i + 3]);
        __syncwarp();
        store_rows(1);
        __syncwarp();
      } else {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32(trow + ACC2_COL + 128 * h + 32 * c, v);
            tmem_ld_wait();
            scale32(v);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(stg_row + (32 * c + i) * 4) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          }
          if (h == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_tmem_empty);   // accumulator free
          }
          __syncwarp();
          store_rows(h);
          __syncwarp();
        }
      }
      acc_phase ^= 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                  // neither CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

template <int YBYTES>
__global__ void __launch_bounds__(THREADS2, 1)
w4a4_rac_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                          const __grid_constant__ CUtensorMap tmSA0, const __grid_constant__ CUtensorMap tmSB0,
                          const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                          const __grid_constant__ CUtensorMap tmSA1, const __grid_constant__ CUtensorMap tmSB1,
                          const KParams2 p) {
  gemm2_body<YBYTES, false>(tmA0, tmB0, tmSA0, tmSB0, tmA1, tmB1, tmSA1, tmSB1, p);
}

// MXFP8 x MXFP8 on CTA pairs (the FP8 comparator): one K segment.
template <int YBYTES>
__global__ void __launch_bounds__(THREADS2, 1)
w8a8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                      const __grid_constant__ CUtensorMap tmSA0, const __grid_constant__ CUtensorMap tmSB0,
                      const KParams2 p) {
  gemm2_body<YBYTES, true>(tmA0, tmB0, tmSA0, tmSB0, tmA0, tmB0, tmSA0, tmSB0, p);
}

// 2-D map over a tiled scale buffer seen as int64 elements: one row per
// 128-row block (all its 512-byte atoms), box = 4 atoms x box_rows blocks.
// atom_cols: K elements one atom covers (64 for NVFP4, 128 for MXFP8);
// box_x: int64 elements of one K step's scales (4 atoms, or 1).
bool make_scale_map(CUtensorMap* tm, const uint8_t* scales, int64_t rows, int64_t cols, int box_rows,
                    int64_t atom_cols = 64, uint32_t box_x = 256u) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const int64_t atoms = (cols + atom_cols - 1) / atom_cols;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(atoms * 64), static_cast<cuuint64_t>((rows + 127) / 128)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(atoms * 512)};
  cuuint32_t box[2] = {box_x, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_INT64, 2, const_cast<uint8_t*>(scales), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int YBYTES>
cudaError_t launch_pair(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg2<YBYTES>;
  static bool done[kMaxAttrDevices] = {};
  {
    const cudaError_t e = set_max_smem(w4a4_rac_gemm_pair_kernel<YBYTES>, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
  }
  KParams2 p{};
  p.M = a.M;
  p.N = a.N;
  p.g = a.g;
  p.pair_start = a.pair_start;
  // dense: 256-row tiles; groups: an upper bound of sum_e ceil(tiles_e / 2)
  // (the kernel reads the exact count from pair_start)
  p.m_tiles = static_cast<int>(a.g.off == nullptr ? (a.M + 255) / 256 : (a.m_tiles + a.g.E) / 2 + 1);
  p.n_tiles = static_cast<int>((a.N + 255) / 256);
  const bool res = a.a1.codes != nullptr;
  // segment 0: residual (may be absent), segment 1: plain
  const GemmOperand* A[2] = {res ? &a.a1 : &a.a0, &a.a0};
  const GemmOperand* B[2] = {res ? &a.b1 : &a.b0, &a.b0};
  CUtensorMap maps[8];
  for (int seg = 0; seg < 2; ++seg) {
    p.kt[seg] = (seg == 0 && !res) ? 0 : static_cast<int>((A[seg]->cols + 255) / 256);
    p.sta[seg] = A[seg]->st;
    p.stb[seg] = B[seg]->st;
    if (!make_code_map(&maps[4 * seg + 0], A[seg]->codes, A[seg]->rows, A[seg]->cols, 128) ||
        !make_code_map(&maps[4 * seg + 1], B[seg]->codes, B[seg]->rows, B[seg]->cols, 128) ||
        !make_scale_map(&maps[4 * seg + 2], A[seg]->scales, A[seg]->rows, A[seg]->cols, 1) ||
        !make_scale_map(&maps[4 * seg + 3], B[seg]->scales, B[seg]->rows, B[seg]->cols, 2))
      return cudaErrorInvalidValue;
  }
  p.y = a.y;
  p.ldy = a.ldy;
  p.err = a.err;
  const int tiles = p.m_tiles * p.n_tiles;
  const int pairs = tiles < sm_count() / 2 ? tiles : sm_count() / 2;
  if (pairs == 0) return cudaSuccess;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  return launch_k(w4a4_rac_gemm_pair_kernel<YBYTES>, dim3(static_cast<unsigned>(2 * pairs)), dim3(THREADS2),
                  C::SMEM_BYTES, s, attr, 1, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6],
                  maps[7], p);
}

}  // namespace

// Dense: the CTA-pair kernel when its waves of 256 x 256 tiles over the SM
// pairs take no longer than the single-CTA kernel's waves of 128 x 128
// tiles over the SMs (a pair tile is twice a single tile's time on half as
// many units), e.g. not for a 256-row product with few output columns.
bool dense_pair_pays(int64_t M, int64_t N) {
  if (M < 256) return false;
  const int64_t sms = sm_count(), pairs = sms / 2;
  const int64_t pt = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t st = ((M + 127) / 128) * ((N + 127) / 128);
  return 2 * ((pt + pairs - 1) / pairs) <= (st + sms - 1) / sms;
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s) {
  // row groups (256-row tiles per group) and dense products where it pays:
  // the CTA-pair kernel
  const bool pair_ok = a.g.off == nullptr ? dense_pair_pays(a.M, a.N) : a.pair_start != nullptr;
  if (pair_ok && !gemm_force_single_cta())
    return a.y_dtype == 0 ? launch_pair<4>(a, s) : launch_pair<2>(a, s);
  cudaError_t e = a.y_dtype == 0 ? prepare_kernel<4>() : prepare_kernel<2>();
  if (e != cudaSuccess) return e;
  KParams p{};
  p.g = a.g;
  p.N = a.N;
  p.m_tiles_dense = (a.M + BM - 1) / BM;
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.M = a.M;
  const GemmOperand* A[2] = {&a.a0, &a.a1};
  const GemmOperand* B[2] = {&a.b0, &a.b1};
  CUtensorMap maps[4];
  const int nseg = a.a1.codes ? 2 : 1;
  for (int seg = 0; seg < 2; ++seg) {
    const int sg = seg < nseg ? seg : 0;      // unused segment: harmless copy of segment 0
    const int64_t cols = A[sg]->cols;
    p.kt[seg] = seg < nseg ? static_cast<int>((cols + 255) / 256) : 0;
    p.kb_last[seg] = static_cast<int>(((cols + 63) / 64 - 1) % 4 + 1);
    p.sfa[seg] = A[sg]->scales;
    p.sfb[seg] = B[sg]->scales;
    p.sfa_rb[seg] = (cols + 63) / 64 * SF_ATOM;
    p.sfb_rb[seg] = (B[sg]->cols + 63) / 64 * SF_ATOM;
    p.sfa_bytes[seg] = scale_extent(A[sg]->rows, cols, 1, kBlock);
    p.sfb_bytes[seg] = scale_extent(B[sg]->rows, B[sg]->cols, 1, kBlock);
    p.sta[seg] = A[sg]->st;
    p.stb[seg] = B[sg]->st;
    if (!make_code_map(&maps[2 * seg], A[sg]->codes, A[sg]->rows, cols, BM)) return cudaErrorInvalidValue;
    if (!make_code_map(&maps[2 * seg + 1], B[sg]->codes, B[sg]->rows, B[sg]->cols, BN))
      return cudaErrorInvalidValue;
  }
  p.y = a.y;
  p.y_dtype = a.y_dtype;
  p.ldy = a.ldy;
  p.err = a.err;
  const int64_t tiles_bound = a.m_tiles * p.n_tiles;
  if (tiles_bound == 0) return cudaSuccess;
  // dense products with few tiles and a long K: S CTAs per tile over K
  // (S = 4 or 2, all tiles in one wave, at least 16 K steps in all and 3 per
  // CTA), the partials reduced in a cluster of S.  The split costs about
  // 2 us (cluster barriers, partial stores, reduction): at 8 K steps of a
  // 512 x 512 product it lost (10.4 -> 12.5 us), at 65 (decode down) it
  // gains 34.6 -> 26 us.
  p.split = 1;
  if (a.g.off == nullptr && !gemm_no_split()) {
    const int64_t tiles = p.m_tiles_dense * p.n_tiles;
    const int T = p.kt[0] + p.kt[1];
    for (int c = 4; c >= 2; c /= 2)
      if (tiles * c <= sm_count() && T >= 16 && T >= 3 * c) {
        p.split = c;
        break;
      }
  }
  if (p.split > 1) {
    e = a.y_dtype == 0 ? prepare_split_kernel<4>() : prepare_split_kernel<2>();
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(p.split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    const dim3 g(static_cast<unsigned>(p.m_tiles_dense * p.n_tiles * p.split));
    const cudaError_t le =
        a.y_dtype == 0 ? launch_k(w4a4_rac_gemm_split_kernel<4>, g, dim3(THREADS1), Cfg<4, true>::SMEM_BYTES, s, attr, 1,
                                  maps[0], maps[1], maps[2], maps[3], p)
                       : launch_k(w4a4_rac_gemm_split_kernel<2>, g, dim3(THREADS1), Cfg<2, true>::SMEM_BYTES, s, attr, 1,
                                  maps[0], maps[1], maps[2], maps[3], p);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
  }
  const int grid = static_cast<int>(tiles_bound < sm_count() ? tiles_bound : sm_count());
  if (a.y_dtype == 0)
    {
      const cudaError_t le = launch_k(w4a4_rac_gemm_kernel<4>, dim3(grid), dim3(THREADS1), Cfg<4>::SMEM_BYTES, s, nullptr, 0,
                                     maps[0], maps[1], maps[2], maps[3], p);
      if (le != cudaSuccess) return le;
    }
  else
    {
      const cudaError_t le = launch_k(w4a4_rac_gemm_kernel<2>, dim3(grid), dim3(THREADS1), Cfg<2>::SMEM_BYTES, s, nullptr, 0,
                                     maps[0], maps[1], maps[2], maps[3], p);
      if (le != cudaSuccess) return le;
    }
  return cudaGetLastError();
}

template <int YBYTES>
cudaError_t launch_pair_fp8(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg2<YBYTES, true>;
  static bool done[kMaxAttrDevices] = {};
  {
    const cudaError_t e = set_max_smem(w8a8_gemm_pair_kernel<YBYTES>, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
  }
  const int64_t K = a.a0.cols;
  KParams2 p{};
  p.M = a.M;
  p.N = a.N;
  p.g = a.g;
  p.m_tiles = static_cast<int>((a.M + 255) / 256);
  p.n_tiles = static_cast<int>((a.N + 255) / 256);
  p.kt[0] = 0;
  p.kt[1] = static_cast<int>(K / 128);
  CUtensorMap maps[4];
  if (!make_code_map(&maps[0], a.a0.codes, a.a0.rows, K, 128, K) ||
      !make_code_map(&maps[1], a.b0.codes, a.b0.rows, K, 128, K) ||
      !make_scale_map(&maps[2], a.a0.scales, a.a0.rows, K, 1, 128, 64u) ||
      !make_scale_map(&maps[3], a.b0.scales, a.b0.rows, K, 2, 128, 64u))
    return cudaErrorInvalidValue;
  p.y = a.y;
  p.ldy = a.ldy;
  p.err = a.err;
  const int tiles = p.m_tiles * p.n_tiles;
  const int pairs = tiles < sm_count() / 2 ? tiles : sm_count() / 2;
  if (pairs == 0) return cudaSuccess;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  return launch_k(w8a8_gemm_pair_kernel<YBYTES>, dim3(static_cast<unsigned>(2 * pairs)), dim3(THREADS2),
                  C::SMEM_BYTES, s, attr, 1, maps[0], maps[1], maps[2], maps[3], p);
}

cudaError_t launch_gemm_fp8(const GemmArgs& a, cudaStream_t s) {
  // CTA pairs where their waves pay, as for NVFP4 (NVFP4_GEMM_SINGLE_CTA=1 keeps the single-CTA form)
  if (dense_pair_pays(a.M, a.N) && !gemm_force_single_cta())
    return a.y_dtype == 0 ? launch_pair_fp8<4>(a, s) : launch_pair_fp8<2>(a, s);
  cudaError_t e = a.y_dtype == 0 ? prepare_kernel8<4>() : prepare_kernel8<2>();
  if (e != cudaSuccess) return e;
  KParams p{};
  p.g = a.g;
  p.N = a.N;
  p.m_tiles_dense = (a.M + BM - 1) / BM;
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.M = a.M;
  const int64_t K = a.a0.cols;                   // multiple of 128: 4 MMAs of K = 32 per step
  p.kt[0] = static_cast<int>(K / 128);
  p.kt[1] = 0;
  p.kb_last[0] = 4;
  p.kb_last[1] = 4;
  p.sfa[0] = p.sfa[1] = a.a0.scales;
  p.sfb[0] = p.sfb[1] = a.b0.scales;
  p.sfa_rb[0] = p.sfa_rb[1] = (K / 128) * SF_ATOM;   // one atom (128 rows x 4 blocks of 32) per step
  p.sfb_rb[0] = p.sfb_rb[1] = (K / 128) * SF_ATOM;
  p.sfa_bytes[0] = p.sfa_bytes[1] = scale_extent(a.a0.rows, K, 1, 32);
  p.sfb_bytes[0] = p.sfb_bytes[1] = scale_extent(a.b0.rows, K, 1, 32);
  CUtensorMap maps[2];
  if (!make_code_map(&maps[0], a.a0.codes, a.a0.rows, K, BM, K) ||
      !make_code_map(&maps[1], a.b0.codes, a.b0.rows, K, BN, K))
    return cudaErrorInvalidValue;
  p.y = a.y;
  p.y_dtype = a.y_dtype;
  p.ldy = a.ldy;
  p.err = a.err;
  const int64_t tiles = p.m_tiles_dense * p.n_tiles;
  if (tiles == 0) return cudaSuccess;
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  const cudaError_t le =
      a.y_dtype == 0
          ? launch_k(w8a8_gemm_kernel<4>, dim3(grid), dim3(THREADS1), Cfg<4>::SMEM_BYTES, s, nullptr, 0, maps[0],
                     maps[1], p)
          : launch_k(w8a8_gemm_kernel<2>, dim3(grid), dim3(THREADS1), Cfg<2>::SMEM_BYTES, s, nullptr, 0, maps[0],
                     maps[1], p);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

NV_DEFINE_BOUNDS_READER(bounds_flags_gemm)

}  // namespace nvfp4
