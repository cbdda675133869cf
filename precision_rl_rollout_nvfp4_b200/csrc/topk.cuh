// Top-k% channel selection of RAC as a CTA-wide device function, shared by
// the stand-alone selection kernel and the tail of the quantize pass (the
// CTA that finishes the last column strip selects the channels).  QUADS
// technical summary (gist.science), section 2.2 B "Implementatie": the binary
// channel mask keeps the k% of channels with the largest residual magnitude.
//
// The fp64 scores are non-negative, so their bit patterns order like their
// values.  Channel j is selected when its key is among the n_sel largest,
// equal keys ordered by ascending channel (ties go to the lower channel).
//
// topk_select (K <= 16384, K % 8 == 0):
//   1. one pass over the keys: their range [kmin, kmax];
//   2. one pass: each channel's 12-bit digit, (key - kmin) >> shift with
//      4096 equal bins over the range, kept in shared memory, and the
//      digits' histogram;
//   3. a scan of the histogram from the top finds the bin b holding the
//      n_sel-th largest key: every key of a higher bin is selected, and
//      `remaining` keys of bin b are still to take.  While bin b holds more
//      than 1024 keys that are not all equal, the next 12 bits of its keys
//      split it again (channels outside it are marked above / below);
//   4. unless bin b is taken whole, its keys are listed with their channels
//      and each gets its exact rank in the order (key descending, channel
//      ascending); ranks below `remaining` are marked in a channel bitmap
//      (a bin of more than 1024 equal keys: its lowest channels);
//   5. each warp classifies a contiguous run of channels from the digits and
//      the bitmap, lanes on consecutive channels; warp counts and a scan
//      over the warps place the ascending sel[] entries, and the same pass
//      reduces s_tR = RN(max_{j in sel} colamax_j / 2688).
// Every full pass over the keys keeps eight 16-byte loads in flight per
// thread.
//
// topk_select_radix (other K):
// radix select over the 64-bit keys starting below the shared leading bits,
// 8-bit digits, the bins searched by a parallel scan, stopping early once a
// whole bin is taken; then the same classification reading the keys.
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

// Radix selection of group e over K keys.  skeys / scm: shared memory for
// the K keys and the K column maxima, or null to read them from global
// memory.  coherent: the scores were written by the same kernel (read through
// L2, not the read-only path).  Every thread of the CTA calls it.
static __device__ __noinline__ void topk_select_radix(const double* __restrict__ score, const float* __restrict__ colamax,
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


constexpr int kSelDigitBits = 12;
constexpr int kSelBins = 1 << kSelDigitBits;            // 4096 x 4 B histogram
constexpr int kSelCandCap = 1024;                       // keys of the boundary bin ranked
constexpr int64_t kSelDigitKeys = 16384;                // u16 digits of 16384 channels = 32 KB
constexpr int kSelScratchBytes = 32768;                 // each of the two scratch buffers
constexpr uint16_t kSelAbove = 0xFFFF, kSelBelow = 0xFFFE;   // channels decided at an earlier level

// The bin of the target-th largest key (1-based) of a 4096-bin histogram:
// thread t sums the bins of descending rank t C .. t C + C - 1, a block scan
// orders the sums, and the thread whose range holds the target walks its
// bins.  Returns the bin; `before` receives the keys of higher bins.
static __device__ __forceinline__ int sel_boundary(const unsigned* hist, long long target, long long* wsum,
                                                   int* s_bin, long long* s_before, long long& before) {
  const int tid = threadIdx.x, C = (kSelBins + blockDim.x - 1) / blockDim.x;
  long long hs = 0;
  for (int i = 0; i < C; ++i) {
    const int r = tid * C + i;
    if (r < kSelBins) hs += hist[kSelBins - 1 - r];
  }
  long long tot;
  const long long before_t = block_excl_scan(hs, tot, wsum);
  if (hs > 0 && before_t < target && target <= before_t + hs) {
    long long acc = before_t;
    for (int i = 0; i < C; ++i) {
      const int r = tid * C + i;
      if (r >= kSelBins) break;
      const long long h = hist[kSelBins - 1 - r];
      if (acc + h >= target) {
        *s_bin = kSelBins - 1 - r;
        *s_before = acc;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
  before = *s_before;
  return *s_bin;
}

// Selection of group e over K keys (see the top of this file).  scr0 / scr1:
// two 32 KB shared buffers of the calling CTA (scr0: histogram, then the
// channel bitmap, the boundary bin's list and the scan words; scr1: the
// per-channel digits).  The scores and colamax are read through L2 (they
// may have been written by the same kernel).  Every thread of the CTA calls it.
static __device__ __noinline__ void topk_select(const double* __restrict__ score, const float* __restrict__ colamax,
                                                int64_t K, int64_t n_sel, uint8_t* __restrict__ mask,
                                                int32_t* __restrict__ sel, float* __restrict__ s_t_out, int64_t e,
                                                uint8_t* scr0, uint8_t* scr1) {
  const bool none = n_sel <= 0, all = n_sel >= K;
  // (the classification below takes whole groups of 8 channels, so K % 8
  // must be 0 for every n_sel; the 16-byte key loads also need 16-byte
  // aligned scores.  K is a multiple of 64 in every caller.)
  const bool keys16 = (reinterpret_cast<uintptr_t>(score + e * K) & 15u) == 0;
  if ((K & 7) != 0 || ((K > kSelDigitKeys || !keys16) && !none && !all)) {
    topk_select_radix(score, colamax, K, n_sel, mask, sel, s_t_out, e, nullptr, nullptr, true);
    return;
  }
  const uint64_t* keys = reinterpret_cast<const uint64_t*>(score + e * K);
  const float* cm = colamax + e * K;
  uint8_t* mk = mask + e * K;
  int32_t* sl = sel + e * n_sel;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nthr = blockDim.x;
  // scr0 layout
  unsigned* hist = reinterpret_cast<unsigned*>(scr0);                  // [kSelBins], later the bitmap
  uint64_t* ckey = reinterpret_cast<uint64_t*>(scr0 + 16384);          // [kSelCandCap]
  uint32_t* cidx = reinterpret_cast<uint32_t*>(scr0 + 24576);          // [kSelCandCap]
  long long* wsum = reinterpret_cast<long long*>(scr0 + 28672);        // [32]
  float* s_max = reinterpret_cast<float*>(scr0 + 28928);               // [32]
  unsigned long long* s_kmin = reinterpret_cast<unsigned long long*>(scr0 + 29056);
  unsigned long long* s_kmax = s_kmin + 1;
  long long* s_before = reinterpret_cast<long long*>(s_kmin + 2);
  int* s_bin = reinterpret_cast<int*>(s_kmin + 3);
  unsigned* s_ncand = reinterpret_cast<unsigned*>(s_bin + 1);
  uint16_t* digit = reinterpret_cast<uint16_t*>(scr1);                 // [K]

  int bin = 0;                   // boundary bin of the last level
  bool ge = true;                // boundary bin taken whole
  if (!none && !all) {
    // 1. the range of the keys
    if (tid == 0) {
      *s_kmin = ~0ull;
      *s_kmax = 0ull;
    }
    __syncthreads();
    // K is even and the keys 16-byte aligned: two keys per load
    const ulonglong2* keys2 = reinterpret_cast<const ulonglong2*>(keys);
    const int64_t K2 = K / 2;
    uint64_t kmn = ~0ull, kmx = 0ull;
    for (int64_t i0 = tid; i0 < K2; i0 += 8 * static_cast<int64_t>(nthr)) {
      ulonglong2 kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + u * static_cast<int64_t>(nthr);
        kv[u] = i < K2 ? __ldcg(keys2 + i) : make_ulonglong2(0ull, 0ull);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (i0 + u * static_cast<int64_t>(nthr) < K2) {
          const uint64_t lo = kv[u].x < kv[u].y ? kv[u].x : kv[u].y, hi = kv[u].x < kv[u].y ? kv[u].y : kv[u].x;
          kmn = lo < kmn ? lo : kmn;
          kmx = hi > kmx ? hi : kmx;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t a = __shfl_xor_sync(0xFFFFFFFFu, kmn, o), b = __shfl_xor_sync(0xFFFFFFFFu, kmx, o);
      kmn = a < kmn ? a : kmn;
      kmx = b > kmx ? b : kmx;
    }
    if (lane == 0) {
      atomicMin(s_kmin, static_cast<unsigned long long>(kmn));
      atomicMax(s_kmax, static_cast<unsigned long long>(kmx));
    }
    for (int b = tid; b < kSelBins; b += nthr) hist[b] = 0u;
    __syncthreads();
    // 2. digits of the first level: 4096 equal bins over [kmin, kmax]
    uint64_t base = *s_kmin;
    const uint64_t span = *s_kmax - base;
    int shift = span == 0 ? 0 : max(0, 64 - __clzll(static_cast<long long>(span)) - kSelDigitBits);
    for (int64_t i0 = tid; i0 < K2; i0 += 8 * static_cast<int64_t>(nthr)) {
      ulonglong2 kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + u * static_cast<int64_t>(nthr);
        kv[u] = i < K2 ? __ldcg(keys2 + i) : make_ulonglong2(0ull, 0ull);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + u * static_cast<int64_t>(nthr);
        if (i < K2) {
          const uint32_t d0 = static_cast<uint32_t>((kv[u].x - base) >> shift);
          const uint32_t d1 = static_cast<uint32_t>((kv[u].y - base) >> shift);
          atomicAdd(&hist[d0], 1u);
          atomicAdd(&hist[d1], 1u);
          reinterpret_cast<uint32_t*>(digit)[i] = d0 | (d1 << 16);
        }
      }
    }
    __syncthreads();
    // 3. the boundary bin; while it holds more than kSelCandCap keys that
    // are not all equal, the next 12 bits of its keys split it again (the
    // other channels are marked above / below once and for all)
    long long before;
    bin = sel_boundary(hist, n_sel, wsum, s_bin, s_before, before);
    long long count = hist[bin];
    long long remaining = n_sel - before;              // 1 .. count keys of the bin to take
    ge = remaining == count;
    while (!ge && count > kSelCandCap && shift > 0) {
      base += static_cast<uint64_t>(bin) << shift;
      const int nshift = shift > kSelDigitBits ? shift - kSelDigitBits : 0;
      __syncthreads();                                 // everyone has read hist[bin]
      for (int b = tid; b < kSelBins; b += nthr) hist[b] = 0u;
      __syncthreads();
      for (int64_t j0 = tid; j0 < K; j0 += 8 * static_cast<int64_t>(nthr)) {
        uint64_t kv[8];
        uint16_t dv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t j = j0 + u * static_cast<int64_t>(nthr);
          dv[u] = j < K ? digit[j] : kSelBelow;
          kv[u] = dv[u] == bin ? __ldcg(keys + j) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t j = j0 + u * static_cast<int64_t>(nthr);
          if (dv[u] >= kSelBelow) continue;            // decided (or past the end)
          if (dv[u] == bin) {
            const uint32_t d = static_cast<uint32_t>((kv[u] - base) >> nshift);
            atomicAdd(&hist[d], 1u);
            digit[j] = static_cast<uint16_t>(d);
          } else {
            digit[j] = dv[u] > bin ? kSelAbove : kSelBelow;
          }
        }
      }
      __syncthreads();
      shift = nshift;
      long long b2;
      bin = sel_boundary(hist, remaining, wsum, s_bin, s_before, b2);
      count = hist[bin];
      remaining -= b2;
      ge = remaining == count;
    }
    __syncthreads();                                   // hist read: scr0 reused below
    if (!ge) {
      // 4. the selected keys of the boundary bin as a channel bitmap
      if (tid == 0) *s_ncand = 0u;
      for (int64_t i = tid; i < (K + 31) / 32; i += nthr) hist[i] = 0u;
      __syncthreads();
      if (count <= kSelCandCap) {
        // exact ranks in the order (key descending, channel ascending)
        for (int64_t g = tid; g < K / 8; g += nthr) {       // 8 channels per 16-byte digit load
          const uint4 dv = reinterpret_cast<const uint4*>(digit)[g];
          const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (((dw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu) == static_cast<uint32_t>(bin)) {
              const int64_t j = 8 * g + i;
              const unsigned slot = atomicAdd(s_ncand, 1u);
              if (NV_IDX(slot < static_cast<unsigned>(kSelCandCap))) {
                ckey[slot] = __ldcg(keys + j);
                cidx[slot] = static_cast<uint32_t>(j);
              }
            }
          }
        }
        __syncthreads();
        const int n = static_cast<int>(count);
        for (int i = tid; i < n; i += nthr) {
          const uint64_t ki = ckey[i];
          const uint32_t ii = cidx[i];
          int r = 0;
          for (int m = 0; m < n; ++m) {
            const uint64_t km = ckey[m];
            r += (km > ki || (km == ki && cidx[m] < ii)) ? 1 : 0;
          }
          if (r < remaining) atomicOr(&hist[ii >> 5], 1u << (ii & 31));
        }
      } else {
        // the bin's keys are all equal (width one key): the lowest channels
        const int64_t per = (K + nthr - 1) / nthr;
        const int64_t jb = tid * per < K ? tid * per : K;
        const int64_t je = jb + per < K ? jb + per : K;
        long long n_eq = 0;
        for (int64_t j = jb; j < je; ++j) n_eq += digit[j] == bin ? 1 : 0;
        long long tot;
        const long long eq_before = block_excl_scan(n_eq, tot, wsum);
        long long take = remaining - eq_before;
        for (int64_t j = jb; j < je && take > 0; ++j) {
          if (digit[j] == bin) {
            atomicOr(&hist[j >> 5], 1u << (j & 31));
            --take;
          }
        }
      }
      __syncthreads();
    }
  }
  // selection bits of the 8 channels 8g .. 8g + 7 (one 16-byte digit load,
  // one byte of the bitmap)
  auto group_bits = [&](int64_t g) -> uint32_t {
    if (none) return 0u;
    if (all) return 0xFFu;
    const uint4 dv = reinterpret_cast<const uint4*>(digit)[g];
    const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
    const uint32_t bm = ge ? 0xFFu : (hist[g >> 2] >> (8 * (g & 3))) & 0xFFu;
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t d = (dw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
      const bool s = d >= kSelBelow ? d == kSelAbove
                                    : (d > static_cast<uint32_t>(bin) ||
                                       (d == static_cast<uint32_t>(bin) && ((bm >> i) & 1u)));
      r |= static_cast<uint32_t>(s) << i;
    }
    return r;
  };
  // 5. classification in rounds of 8 nthr channels: thread t takes the
  // 8-channel group t of the round, so mask bytes, sel entries and colamax
  // loads are coalesced; a block scan of the groups' counts places the
  // ascending sel[] entries
  const int64_t G = K / 8;
  const float4* cm4 = reinterpret_cast<const float4*>(cm);
  const bool cm16 = (reinterpret_cast<uintptr_t>(cm) & 15u) == 0;     // else scalar colamax loads
  const bool mk8 = (reinterpret_cast<uintptr_t>(mk) & 7u) == 0;       // else byte stores of the mask
  long long pbase = 0;
  float mx = 0.0f;
  for (int64_t g0 = 0; g0 < G; g0 += nthr) {
    const int64_t g = g0 + tid;
    const uint32_t b8 = g < G ? group_bits(g) : 0u;
    float4 c0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), c1 = c0;
    if (b8 != 0u) {                                    // colamax loads in flight across the scan
      if (cm16) {
        c0 = __ldcg(cm4 + 2 * g);
        c1 = __ldcg(cm4 + 2 * g + 1);
      } else {
        c0 = make_float4(__ldcg(cm + 8 * g), __ldcg(cm + 8 * g + 1), __ldcg(cm + 8 * g + 2), __ldcg(cm + 8 * g + 3));
        c1 = make_float4(__ldcg(cm + 8 * g + 4), __ldcg(cm + 8 * g + 5), __ldcg(cm + 8 * g + 6),
                         __ldcg(cm + 8 * g + 7));
      }
    }
    long long tot;
    long long p = pbase + block_excl_scan(__popc(b8), tot, wsum);
    if (g < G) {
      uint2 mb;                                        // one byte per channel
      mb.x = (b8 & 1u) | ((b8 >> 1) & 1u) << 8 | ((b8 >> 2) & 1u) << 16 | ((b8 >> 3) & 1u) << 24;
      mb.y = ((b8 >> 4) & 1u) | ((b8 >> 5) & 1u) << 8 | ((b8 >> 6) & 1u) << 16 | ((b8 >> 7) & 1u) << 24;
      if (mk8) {
        *reinterpret_cast<uint2*>(mk + 8 * g) = mb;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) mk[8 * g + i] = static_cast<uint8_t>((b8 >> i) & 1u);
      }
      const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((b8 >> i) & 1u) {
          if (NV_IDX(p < n_sel)) sl[p] = static_cast<int32_t>(8 * g + i);
          ++p;
          mx = fmaxf(mx, cv[i]);
        }
      }
    }
    pbase += tot;
  }
  mx = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mx)));
  if (lane == 0) s_max[w] = mx;
  __syncthreads();
  if (tid == 0) {
    float r = 0.0f;
    for (int i = 0; i < (nthr >> 5); ++i) r = fmaxf(r, s_max[i]);
    s_t_out[e] = __fdiv_rn(r, kTensorScaleDiv);
  }
  __syncthreads();
}

}  // namespace nvfp4
