// df11_device_check.h -- the check every entry point of the library makes
// before it queues work: the device buffers it is given must be memory of
// the current device, since its kernels run there.  A pointer into another
// GPU's memory would make them read a peer's memory (an illegal access
// without peer access).  Internal to the library.
#pragma once
#include <cuda_runtime.h>

#include "df11.h"

namespace df11_internal {

// DF11_OK when every non-null pointer of `ptrs` is device memory of the
// current device or managed memory; DF11_ERR_DEVICE otherwise (host memory,
// another device's memory, an unknown address); DF11_ERR_CUDA when there is
// no current device.
inline df11_status check_device_pointers(const void *const *ptrs, int count) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
  for (int i = 0; i < count; ++i) {
    if (!ptrs[i]) continue;
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, ptrs[i]) != cudaSuccess) {
      (void)cudaGetLastError();  // clear this call's (non-sticky) error
      return DF11_ERR_DEVICE;
    }
    if (a.type == cudaMemoryTypeManaged) continue;
    if (a.type != cudaMemoryTypeDevice || a.device != dev) return DF11_ERR_DEVICE;
  }
  return DF11_OK;
}

}  // namespace df11_internal
