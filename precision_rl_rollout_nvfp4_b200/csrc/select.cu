// Top-k% channel selection of RAC: the binary channel mask that keeps the
// k% of channels with the largest residual magnitude (QUADS technical
// summary, gist.science, section 2.2 B, "Implementatie").
//
// One CTA per row group (one for a dense linear, one per MoE expert).  The
// fp64 scores are non-negative, so their bit patterns order like their
// values; a radix select over the 64-bit keys (8-bit digits, bins searched by
// a parallel scan, early exit once a whole bin is taken) finds the n_sel-th
// largest key T exactly.  Every key > T is selected, and keys == T are taken
// in ascending channel order until n_sel are selected (ties go to the lower
// channel).  A block-wide scan in channel order then writes the ascending
// sel[] list, and the same pass reduces the residual tensor scale
// s_tR = RN(max_{j in sel} colamax_j / 2688).
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kSelThreads = 512;

// Exclusive prefix count of `flag` over the CTA in thread order; `total`
// receives the CTA-wide count.  Every thread of the CTA must call it.
__device__ int block_scan_flag(bool flag, int& total, int* wsum) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nw = blockDim.x >> 5;
  const unsigned b = __ballot_sync(0xFFFFFFFFu, flag);
  const int in_warp = __popc(b & ((1u << lane) - 1u));
  if (lane == 0) wsum[w] = __popc(b);
  __syncthreads();
  if (w == 0) {
    int v = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, v, o);
      if (lane >= o) v += n;
    }
    wsum[lane] = v;                      // inclusive
  }
  __syncthreads();
  const int before = w == 0 ? 0 : wsum[w - 1];
  total = wsum[nw - 1];
  __syncthreads();
  return before + in_warp;
}

__global__ void __launch_bounds__(kSelThreads)
topk_kernel(const double* __restrict__ score, const float* __restrict__ colamax, int64_t K,
            int64_t n_sel, uint8_t* __restrict__ mask, int32_t* __restrict__ sel,
            float* __restrict__ s_t_out, int keys_in_smem) {
  const int64_t e = blockIdx.x;
  const uint64_t* gkeys = reinterpret_cast<const uint64_t*>(score + e * K);
  // the keys are read once per radix pass and once more to classify: keep
  // them in shared memory when they fit (dynamic size K * 8 bytes)
  extern __shared__ uint64_t skeys[];
  const bool in_smem = keys_in_smem != 0;
  if (in_smem) {
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x) skeys[j] = __ldg(gkeys + j);
    __syncthreads();
  }
  const uint64_t* keys = in_smem ? skeys : gkeys;
  const float* cm = colamax + e * K;
  uint8_t* mk = mask + e * K;
  int32_t* sl = sel + e * n_sel;
  const int tid = threadIdx.x;

  __shared__ unsigned hist[256];
  __shared__ int wsum[32];
  __shared__ uint64_t s_prefix;
  __shared__ long long s_remaining;
  __shared__ bool s_ge;
  __shared__ float s_max[32];

  // Radix select, most significant byte first.  After each pass `prefix`
  // holds the leading bytes of the n_sel-th largest key and `remaining` how
  // many keys with that prefix are still to be taken.  If every key of the
  // chosen bin is taken, the selection is simply key >= (prefix, zeros) and
  // the search stops early (ge_mode); otherwise after 8 passes T is the exact
  // n_sel-th largest key and ties at T go to the lower channels.
  uint64_t prefix = 0, pmask = 0;
  long long remaining = n_sel;
  bool ge_mode = false;
  if (n_sel > 0 && n_sel < K) {
    for (int pass = 0; pass < 8 && !ge_mode; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      for (int64_t j = tid; j < K; j += blockDim.x) {
        const uint64_t k = keys[j];
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      // threads 0..255 own bins 255 - tid (largest first); an inclusive scan
      // over them finds the bin that holds the remaining-th largest key
      const int lane = tid & 31, w = tid >> 5;
      unsigned h = 0, incl = 0;
      if (tid < 256) {
        h = hist[255 - tid];
        incl = h;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += n;
        }
        if (lane == 31) wsum[w] = static_cast<int>(incl);
      }
      __syncthreads();
      if (tid < 256) {
        unsigned before_warp = 0;
        for (int i = 0; i < w; ++i) before_warp += static_cast<unsigned>(wsum[i]);
        const long long upto = static_cast<long long>(before_warp) + incl;     // inclusive
        const long long before = upto - h;
        if (before < remaining && remaining <= upto) {
          const unsigned b = 255u - static_cast<unsigned>(tid);
          s_prefix = prefix | (static_cast<uint64_t>(b) << shift);
          s_remaining = remaining - before;
          s_ge = (remaining - before) == static_cast<long long>(h);
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      ge_mode = s_ge;
      pmask |= 0xFFull << shift;
      __syncthreads();
    }
  }
  const uint64_t T = prefix;
  const long long need_eq = ge_mode ? 0 : remaining;   // keys == T still to take

  long long carry_eq = 0, carry_sel = 0;
  float mx = 0.0f;
  for (int64_t base = 0; base < K; base += blockDim.x) {
    const int64_t j = base + tid;
    const bool in = j < K;
    const uint64_t k = in ? keys[j] : 0;
    bool m;
    if (n_sel == 0) {
      m = false;
    } else if (n_sel >= K) {
      m = in;
    } else {
      const bool gt = in && (ge_mode ? k >= T : k > T), eq = in && !ge_mode && k == T;
      if (ge_mode) {
        m = gt;
      } else {
        int tot_eq;
        const int r_eq = block_scan_flag(eq, tot_eq, wsum);
        m = gt || (eq && carry_eq + r_eq < need_eq);
        carry_eq += tot_eq;
      }
    }
    int tot_m;
    const int pos = block_scan_flag(m, tot_m, wsum);
    if (in) mk[j] = m ? 1 : 0;
    if (m && carry_sel + pos < n_sel) {
      sl[carry_sel + pos] = static_cast<int32_t>(j);
      mx = fmaxf(mx, cm[j]);
    }
    carry_sel += tot_m;
  }
  mx = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mx)));
  if ((tid & 31) == 0) s_max[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    float r = 0.0f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r = fmaxf(r, s_max[i]);
    s_t_out[e] = __fdiv_rn(r, kTensorScaleDiv);
  }
}

}  // namespace

cudaError_t launch_topk(const double* score, const float* colamax, int64_t K, int32_t E,
                        int64_t n_sel, uint8_t* mask, int32_t* sel, float* s_t_out,
                        cudaStream_t s) {
  constexpr int64_t kMaxSmemKeys = 24576;          // 192 KB of keys
  const bool smem = K <= kMaxSmemKeys;
  const size_t bytes = smem ? static_cast<size_t>(K) * sizeof(uint64_t) : 0;
  static size_t attr = 48 * 1024;
  if (bytes > attr) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kMaxSmemKeys * sizeof(uint64_t)));
    if (e != cudaSuccess) return e;
    attr = kMaxSmemKeys * sizeof(uint64_t);
  }
  topk_kernel<<<E, kSelThreads, bytes, s>>>(score, colamax, K, n_sel, mask, sel, s_t_out, smem ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace nvfp4
