// Top-k% channel selection of RAC: the binary channel mask that keeps the
// k% of channels with the largest residual magnitude (QUADS technical
// summary, gist.science, section 2.2 B, "Implementatie").
//
// One CTA per row group (one for a dense linear, one per MoE expert).  The
// fp64 scores are non-negative, so their bit patterns order like their
// values.  A radix select over the 64-bit keys finds the n_sel-th largest key
// T exactly: it starts below the leading bits that all keys share (the
// scores of one tensor have close exponents, so the first 8-bit digit
// already spreads them over the bins), searches the bins by a parallel scan
// and stops early once a whole bin is taken.  Every key > T is selected, and
// keys == T are taken in ascending channel order until n_sel are selected
// (ties go to the lower channel).  Each thread then classifies a contiguous
// run of channels; two block-wide scans place the ties and the ascending
// sel[] entries, and the same pass reduces the residual tensor scale
// s_tR = RN(max_{j in sel} colamax_j / 2688).  Keys and colamax sit in shared
// memory when they fit.
#include "kernels.h"
#include "topk.cuh"

namespace nvfp4 {
namespace {

constexpr int kSelThreads = 512;
constexpr int64_t kMaxSmemKeys = 16384;          // 16384 x (8 + 4) bytes = 192 KB

__global__ void __launch_bounds__(kSelThreads)
topk_kernel(const double* __restrict__ score, const float* __restrict__ colamax, int64_t K,
            int64_t n_sel, uint8_t* __restrict__ mask, int32_t* __restrict__ sel,
            float* __restrict__ s_t_out, int in_smem) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ uint64_t skeys[];            // [K] keys, then [K] colamax
  topk_select(score, colamax, K, n_sel, mask, sel, s_t_out, blockIdx.x, in_smem ? skeys : nullptr,
              in_smem ? reinterpret_cast<float*>(skeys + K) : nullptr, false);
}

}  // namespace

cudaError_t launch_topk(const double* score, const float* colamax, int64_t K, int32_t E,
                        int64_t n_sel, uint8_t* mask, int32_t* sel, float* s_t_out,
                        cudaStream_t s) {
  const bool smem = K <= kMaxSmemKeys;
  const size_t bytes = smem ? static_cast<size_t>(K) * (sizeof(uint64_t) + sizeof(float)) : 0;
  // static plus dynamic shared memory can pass the 48 KB default: opt in
  // once per device for the largest key buffer
  static bool done[kMaxAttrDevices] = {};
  {
    const cudaError_t e =
        set_max_smem(topk_kernel, static_cast<int>(kMaxSmemKeys * (sizeof(uint64_t) + sizeof(float))), done);
    if (e != cudaSuccess) return e;
  }
  {
    const cudaError_t le = launch_k(topk_kernel, dim3(E), dim3(kSelThreads), bytes, s, nullptr, 0,
                                   score, colamax, K, n_sel, mask, sel, s_t_out, smem ? 1 : 0);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

NV_DEFINE_BOUNDS_READER(bounds_flags_select)

}  // namespace nvfp4
