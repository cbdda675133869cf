// Top-k% channel selection of RAC: the binary channel mask that keeps the
// k% of channels with the largest residual magnitude (QUADS technical
// summary, gist.science, section 2.2 B, "Implementatie").
//
// One CTA per row group (one for a dense linear, one per MoE expert); the
// selection itself (topk.cuh) finds the boundary bin of a 12-bit digit of
// the fp64 keys, ranks that bin's keys exactly, and writes the mask, the
// ascending sel[] list and s_tR = RN(max_{j in sel} colamax_j / 2688).
#include "kernels.h"
#include "topk.cuh"

namespace nvfp4 {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelDyn = 2 * kSelScratchBytes;       // the selection's two scratch buffers

__global__ void __launch_bounds__(kSelThreads)
topk_kernel(const double* __restrict__ score, const float* __restrict__ colamax, int64_t K,
            int64_t n_sel, uint8_t* __restrict__ mask, int32_t* __restrict__ sel,
            float* __restrict__ s_t_out) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t sel_dyn[];
  topk_select(score, colamax, K, n_sel, mask, sel, s_t_out, blockIdx.x, sel_dyn, sel_dyn + kSelScratchBytes);
}

}  // namespace

cudaError_t launch_topk(const double* score, const float* colamax, int64_t K, int32_t E,
                        int64_t n_sel, uint8_t* mask, int32_t* sel, float* s_t_out,
                        cudaStream_t s) {
  // static plus dynamic shared memory passes the 48 KB default: opt in once
  // per device
  static bool done[kMaxAttrDevices] = {};
  {
    const cudaError_t e = set_max_smem(topk_kernel, kSelDyn, done);
    if (e != cudaSuccess) return e;
  }
  {
    const cudaError_t le = launch_k(topk_kernel, dim3(E), dim3(kSelThreads), kSelDyn, s, nullptr, 0,
                                   score, colamax, K, n_sel, mask, sel, s_t_out);
    if (le != cudaSuccess) return le;
  }
  return cudaGetLastError();
}

NV_DEFINE_BOUNDS_READER(bounds_flags_select)

}  // namespace nvfp4
