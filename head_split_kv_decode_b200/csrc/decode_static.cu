// Fixed scratch for duo_decode_attn_static: the split-K decode's partial
// outputs, log-sum-exp values and merge tickets live in one statically sized
// device array that the library owns, so that call allocates nothing.
//
// The array is a module global: every GPU that loads libduo.so holds
// kDecodeStaticScratchBytes of it until the process exits.  In host code the
// array's name is only a host-side stand-in, never a device address; its
// device address is looked up here with cudaGetSymbolAddress, once per
// device, with that device current.
#include "common.cuh"

namespace duo {

constexpr size_t kDecodeStaticScratchBytes = 8u << 20;  // 8 MiB

static __device__ __align__(256) uint8_t g_decode_scratch[kDecodeStaticScratchBytes];

size_t decode_static_scratch_bytes() { return kDecodeStaticScratchBytes; }

// Device address of the scratch array on the current device.  The first call
// on a device performs the symbol lookup (a runtime call that must not be
// made while a stream is being captured); later calls return the cached value.
cudaError_t decode_static_scratch(void **ptr) {
  static void *addr[kMaxDevices] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace duo
