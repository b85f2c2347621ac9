// tcf4_noalloc.cu -- trellis_gemv_noalloc: the fused decode GEMV with its scratch in a fixed
// device array of this library instead of a caller-provided workspace.
//
// The array is a file-scope __device__ variable, so every device that loads the library has its own
// copy. Its address on the current device is looked up on every call (cudaGetSymbolAddress, a host
// side lookup once the module is loaded on the device) and never cached: a cached address would
// outlive a cudaDeviceReset, after which the array lives at a new address, and a cache shared by
// host threads would need its own synchronization. The call then forwards to trellis_gemv.
#include <cuda_runtime.h>

#include "tcf4.h"

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;  // 2 MiB: the largest GEMV workspace for cols <= 16384 is 1.63 MiB

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

}  // namespace

extern "C" tcf4_status trellis_gemv_noalloc(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *stream) {
  const size_t need = trellis_gemv_workspace(w, T);
  if (need > kScratchBytes) return TCF4_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (need > 0) {
    // the array's address on the current device, with that device current
    if (cudaGetSymbolAddress(&scratch, g_gemv_scratch) != cudaSuccess || scratch == nullptr) {
      (void)cudaGetLastError();
      return TCF4_ERR_CUDA;
    }
  }
  return trellis_gemv(w, x, T, y, scratch, need > 0 ? kScratchBytes : 0, stream);
}
