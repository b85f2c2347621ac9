// tcf4_noalloc.cu -- trellis_gemv_noalloc: the fused decode GEMV with its scratch in a fixed
// device array of this library instead of a caller-provided workspace.
//
// The array is a file-scope __device__ variable, so every device that loads the library has its own
// copy. Its address on the current device is looked up once (cudaGetSymbolAddress, with that device
// current) and cached per device ordinal; after that the call only forwards to trellis_gemv.
#include <cuda_runtime.h>

#include "tcf4.h"

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;  // 1 MiB: the largest GEMV workspace for cols <= 16384
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];
static void *g_scratch_addr[kMaxDevices];  // per device ordinal; written on its first call

}  // namespace

extern "C" tcf4_status trellis_gemv_noalloc(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return TCF4_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return TCF4_ERR_UNSUPPORTED;
  if (g_scratch_addr[dev] == nullptr) {  // one-time setup on this device
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return TCF4_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  const size_t need = trellis_gemv_workspace(w, T);
  if (need > kScratchBytes) return TCF4_ERR_WORKSPACE;
  return trellis_gemv(w, x, T, y, need > 0 ? g_scratch_addr[dev] : nullptr, need > 0 ? kScratchBytes : 0, stream);
}
