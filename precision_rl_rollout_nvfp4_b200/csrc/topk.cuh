// Top-k% channel selection of RAC as a CTA-wide device function, shared by
// the stand-alone selection kernel and the tail of the quantize pass (the
// CTA that finishes the last column strip selects the channels).  QUADS
// technical summary (gist.science), section 2.2 B "Implementatie": the binary
// channel mask keeps the k% of channels with the largest residual magnitude.
//
// The fp64 scores are non-negative, so their bit patterns order like their
// values.  A radix select over the 64-bit keys finds the n_sel-th largest key
// T exactly: it starts below the leading bits that all keys share, searches
// the bins of an 8-bit digit by a parallel scan and stops early once a whole
// bin is taken.  Every key > T is selected, and keys == T are taken in
// ascending channel order until n_sel are selected (ties go to the lower
// channel).  Each thread then classifies a contiguous run of channels; two
// block-wide scans place the ties and the ascending sel[] entries, and the
// same pass reduces the residual tensor scale
// s_tR = RN(max_{j in sel} colamax_j / 2688).
#pragma once

#include "common.cuh"

namespace nvfp4 {

// Exclusive prefix sum of v over the CTA in thread order; `total` receives
// the CTA-wide sum.  Every thread of the CTA must call it.
static __device__ __forceinline__ long long block_excl_scan(long long v, long long& total, long long* wsum) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nw = blockDim.x >> 5;
  long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  if (w == 0) {
    long long x = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long n = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += n;
    }
    if (lane < nw) wsum[lane] = x;                 // inclusive over warps
  }
  __syncthreads();
  const long long before = (w == 0 ? 0 : wsum[w - 1]) + incl - v;
  total = wsum[nw - 1];
  __syncthreads();
  return before;
}

// Selection of group e over K keys.  skeys / scm: shared memory for the K
// keys and the K column maxima, or null to read them from global memory.
// coherent: the scores were written by the same kernel (read through L2, not
// the read-only path).  Every thread of the CTA calls it.
static __device__ __noinline__ void topk_select(const double* __restrict__ score, const float* __restrict__ colamax,
                                         int64_t K, int64_t n_sel, uint8_t* __restrict__ mask,
                                         int32_t* __restrict__ sel, float* __restrict__ s_t_out, int64_t e,
                                         uint64_t* skeys, float* scm, bool coherent) {
  const uint64_t* gkeys = reinterpret_cast<const uint64_t*>(score + e * K);
  const float* gcm = colamax + e * K;
  const bool in_smem = skeys != nullptr;
  const bool cm_smem = scm != nullptr;
  if (in_smem || cm_smem) {
    // eight loads in flight per thread, then the stores
    for (int64_t j0 = threadIdx.x; j0 < K; j0 += 8 * static_cast<int64_t>(blockDim.x)) {
      uint64_t kv[8];
      float cv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t j = j0 + u * static_cast<int64_t>(blockDim.x);
        if (j < K) {
          if (in_smem) kv[u] = coherent ? __ldcg(gkeys + j) : __ldg(gkeys + j);
          if (cm_smem) cv[u] = coherent ? __ldcg(gcm + j) : __ldg(gcm + j);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t j = j0 + u * static_cast<int64_t>(blockDim.x);
        if (j < K) {
          if (in_smem) skeys[j] = kv[u];
          if (cm_smem) scm[j] = cv[u];
        }
      }
    }
    __syncthreads();
  }
  const uint64_t* keys = in_smem ? skeys : gkeys;
  const float* cm = cm_smem ? scm : gcm;
  uint8_t* mk = mask + e * K;
  int32_t* sl = sel + e * n_sel;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

  __shared__ unsigned hist[256];
  __shared__ long long wsum[32];
  __shared__ unsigned long long s_and, s_or, s_prefix;
  __shared__ long long s_remaining;
  __shared__ bool s_ge;
  __shared__ float s_max[32];

  // After each pass `prefix` holds the leading bits of the n_sel-th largest
  // key and `remaining` how many keys with that prefix are still to be
  // taken.  If every key of the chosen bin is taken, the selection is simply
  // key >= (prefix, zeros) (ge_mode); otherwise, once every bit is fixed, T
  // is the exact n_sel-th largest key and ties at T go to the lower channels.
  uint64_t prefix = 0;
  long long remaining = n_sel;
  bool ge_mode = n_sel >= K;                     // all selected: key >= 0
  if (n_sel > 0 && n_sel < K) {
    if (tid == 0) {
      s_and = ~0ull;
      s_or = 0ull;
    }
    __syncthreads();
    uint64_t a = ~0ull, o = 0ull;
#pragma unroll 8
    for (int64_t j = tid; j < K; j += blockDim.x) {
      const uint64_t k = in_smem ? keys[j] : __ldcg(keys + j);
      a &= k;
      o |= k;
    }
    const uint32_t ahi = __reduce_and_sync(0xFFFFFFFFu, static_cast<uint32_t>(a >> 32));
    const uint32_t alo = __reduce_and_sync(0xFFFFFFFFu, static_cast<uint32_t>(a));
    const uint32_t ohi = __reduce_or_sync(0xFFFFFFFFu, static_cast<uint32_t>(o >> 32));
    const uint32_t olo = __reduce_or_sync(0xFFFFFFFFu, static_cast<uint32_t>(o));
    if (lane == 0) {
      atomicAnd(&s_and, (static_cast<unsigned long long>(ahi) << 32) | alo);
      atomicOr(&s_or, (static_cast<unsigned long long>(ohi) << 32) | olo);
    }
    __syncthreads();
    const uint64_t diff = s_and ^ s_or;
    int pos = diff == 0 ? 0 : 64 - __clzll(static_cast<long long>(diff));   // free low bits
    uint64_t pmask = pos == 64 ? 0ull : ~((1ull << pos) - 1ull);
    prefix = s_and & pmask;
    while (pos > 0 && !ge_mode) {
      const int D = pos < 8 ? pos : 8;
      const int shift = pos - D;
      const int nb = 1 << D;
      if (tid < 256) hist[tid] = 0;
      __syncthreads();
#pragma unroll 8
      for (int64_t j = tid; j < K; j += blockDim.x) {
        const uint64_t k = in_smem ? keys[j] : __ldcg(keys + j);
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & static_cast<uint64_t>(nb - 1)], 1u);
      }
      __syncthreads();
      // threads 0..nb-1 own bins nb-1-tid (largest first); an inclusive scan
      // over them finds the bin that holds the remaining-th largest key
      unsigned h = 0, incl = 0;
      if (tid < 256) {
        h = tid < nb ? hist[nb - 1 - tid] : 0u;
        incl = h;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const unsigned n = __shfl_up_sync(0xFFFFFFFFu, incl, off);
          if (lane >= off) incl += n;
        }
        if (lane == 31) wsum[w] = incl;
      }
      __syncthreads();
      if (tid < nb) {
        long long before_warp = 0;
        for (int i = 0; i < w; ++i) before_warp += wsum[i];
        const long long upto = before_warp + incl;     // inclusive
        const long long before = upto - h;
        if (before < remaining && remaining <= upto) {
          s_prefix = prefix | (static_cast<uint64_t>(nb - 1 - tid) << shift);
          s_remaining = remaining - before;
          s_ge = (remaining - before) == static_cast<long long>(h);
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      ge_mode = s_ge;
      pmask |= static_cast<uint64_t>(nb - 1) << shift;
      pos = shift;
      __syncthreads();
    }
  }
  const uint64_t T = prefix;
  const long long need_eq = ge_mode ? 0 : remaining;   // keys == T still to take

  // classification: thread tid owns channels [jb, je)
  const int64_t per = (K + blockDim.x - 1) / blockDim.x;
  const int64_t jb = tid * per < K ? tid * per : K;
  const int64_t je = jb + per < K ? jb + per : K;
  const bool none = n_sel == 0;
  long long n_gt = 0, n_eq = 0;
  if (!none) {
#pragma unroll 8
    for (int64_t j = jb; j < je; ++j) {
      const uint64_t k = in_smem ? keys[j] : __ldcg(keys + j);
      if (ge_mode ? k >= T : k > T) ++n_gt;
      else if (!ge_mode && k == T) ++n_eq;
    }
  }
  long long tot;
  const long long eq_before = ge_mode || none ? 0 : block_excl_scan(n_eq, tot, wsum);
  long long take_eq = need_eq - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > n_eq ? n_eq : take_eq);
  long long p = block_excl_scan(n_gt + take_eq, tot, wsum);
  float mx = 0.0f;
  long long eq_seen = 0;
  for (int64_t j = jb; j < je; ++j) {
    bool m = false;
    if (!none) {
      const uint64_t k = in_smem ? keys[j] : __ldcg(keys + j);
      if (ge_mode ? k >= T : k > T) {
        m = true;
      } else if (!ge_mode && k == T) {
        m = eq_seen < take_eq;
        ++eq_seen;
      }
    }
    mk[j] = m ? 1 : 0;
    if (m) {
      if (NV_IDX(p < n_sel)) sl[p] = static_cast<int32_t>(j);
      ++p;
      mx = fmaxf(mx, cm_smem ? cm[j] : __ldcg(cm + j));
    }
  }
  mx = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mx)));
  if (lane == 0) s_max[w] = mx;
  __syncthreads();
  if (tid == 0) {
    float r = 0.0f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r = fmaxf(r, s_max[i]);
    s_t_out[e] = __fdiv_rn(r, kTensorScaleDiv);
  }
  __syncthreads();
}

}  // namespace nvfp4
