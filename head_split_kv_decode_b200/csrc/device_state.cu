// The device-side error word that bounded in-kernel waits set when they give
// up (see DeviceError in kernels.h); read and cleared by duo_poll_device_error.
#include "common.cuh"

namespace duo {

__device__ int g_error_word = 0;

int *device_error_word() {
  static int *addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int *>(p);
  }
  return addr[dev];
}

}  // namespace duo
