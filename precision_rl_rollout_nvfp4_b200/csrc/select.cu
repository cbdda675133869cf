// Top-k% channel selection of RAC: the binary channel mask that keeps the
// k% of channels with the largest residual magnitude (QUADS technical
// summary, gist.science, section 2.2 B, "Implementatie").
//
// One CTA per row group (one for a dense linear, one per MoE expert).  The
// fp64 scores are non-negative, so their bit patterns order like their
// values; an 8-pass radix select over the 64-bit keys finds the n_sel-th
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
            float* __restrict__ s_t_out) {
  const int64_t e = blockIdx.x;
  const uint64_t* keys = reinterpret_cast<const uint64_t*>(score + e * K);
  const float* cm = colamax + e * K;
  uint8_t* mk = mask + e * K;
  int32_t* sl = sel + e * n_sel;
  const int tid = threadIdx.x;

  __shared__ unsigned hist[256];
  __shared__ int wsum[32];
  __shared__ uint64_t s_prefix;
  __shared__ long long s_remaining;
  __shared__ float s_max[32];

  uint64_t prefix = 0, pmask = 0;
  long long remaining = n_sel;
  if (n_sel > 0 && n_sel < K) {
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      for (int64_t j = tid; j < K; j += blockDim.x) {
        const uint64_t k = keys[j];
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        long long acc = 0;
        int b = 255;
        for (; b > 0; --b) {                       // largest bins first
          if (acc + static_cast<long long>(hist[b]) >= remaining) break;
          acc += hist[b];
        }
        s_prefix = prefix | (static_cast<uint64_t>(b) << shift);
        s_remaining = remaining - acc;
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      pmask |= 0xFFull << shift;
    }
  }
  const uint64_t T = prefix;
  const long long need_eq = remaining;       // keys == T still to take

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
      const bool gt = in && k > T, eq = in && k == T;
      int tot_eq;
      const int r_eq = block_scan_flag(eq, tot_eq, wsum);
      m = gt || (eq && carry_eq + r_eq < need_eq);
      carry_eq += tot_eq;
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
  topk_kernel<<<E, kSelThreads, 0, s>>>(score, colamax, K, n_sel, mask, sel, s_t_out);
  return cudaGetLastError();
}

}  // namespace nvfp4
