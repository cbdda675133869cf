// nvfp4_quantize_static_ws: nvfp4_quantize without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: plugin hooks of
// an inference engine whose interface passes only input and output pointers,
// or a process whose device memory is already fully reserved by another
// runtime's allocator (an engine that claims nearly all HBM for its caches at
// start-up).  For them this entry point keeps its scratch (the tensor amax,
// the per-strip counters and the channel-score partials) in one file-scope
// device array of kStaticScratchBytes, which every GPU that loads the library
// holds until the process exits.  The call itself allocates nothing.
#include "kernels.h"
#include "nvfp4rac.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB

static __device__ __align__(256) unsigned char g_quantize_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_quantize_scratch on the current device.  In host code
// the array's name only stands in for the symbol, so the address has to be
// asked for once per device (with that device current) and then cached.
void* scratch_address() {
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_quantize_scratch) != cudaSuccess) {
      cudaGetLastError();              // leave no pending error behind for later calls to report
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_static_ws(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                                 const float* amax_or_null, nvfp4_tensor* qx,
                                                 double* score_or_null, float* res_colamax_or_null,
                                                 void* stream) {
  // the device first: on another architecture the symbol lookup itself would fail
  const int dc = nvfp4::device_check();
  if (dc != 0) return dc == 1 ? NVFP4_ERR_DEVICE : NVFP4_ERR_CUDA;
  void* ws = scratch_address();
  if (ws == nullptr) return NVFP4_ERR_CUDA;
  // nvfp4_quantize refuses (NVFP4_ERR_WORKSPACE, before anything is queued)
  // any shape whose scratch exceeds the array, and writes every scratch word
  // it reads (partial maxima, cleared counters) on the stream before use, so
  // whatever an earlier call left in the array does not matter.
  return nvfp4_quantize(x, M, K, ldx, amax_or_null, qx, score_or_null, res_colamax_or_null, ws,
                        kStaticScratchBytes, stream);
}
