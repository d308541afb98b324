// host_static.cu -- device memory owned by the library for
// wan_dit_attn_host_static: the staging area through which the host-buffer
// step runs when its caller cannot allocate device memory.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds one copy of it until the process exits. Host code cannot use
// the array's name as a device address (on the host it names a stand-in), so
// the address is looked up with cudaGetSymbolAddress, once per device, with
// that device current, on the first call that needs it.
#include <cuda_runtime.h>

#include <cstdint>

#include "wan_attn.h"  // include/ is on the include path
#include "wan_kernels.h"

namespace wan {
namespace {

// Packed QKV of the step in the first 3/4, its output in the last 1/4, at
// fixed offsets so that the pipeline's per-buffer ordering applies call to
// call.
constexpr size_t kStaticBytes = static_cast<size_t>(WAN_HOST_STATIC_MAX_ELEMENTS) * 8;
constexpr size_t kStaticOutOffset = static_cast<size_t>(WAN_HOST_STATIC_MAX_ELEMENTS) * 6;

static __device__ __align__(256) unsigned char g_host_static[kStaticBytes];

void* g_static_addr[kMaxDevices];

}  // namespace

cudaError_t host_static_buffers(void** qkv_dev, void** out_dev) {
  static PerDeviceOnce setup;
  int dev = 0;
  const cudaError_t e = setup.run(
      [](int d) { return cudaGetSymbolAddress(&g_static_addr[d], g_host_static); }, &dev);
  if (e != cudaSuccess) return e;
  *qkv_dev = g_static_addr[dev];
  *out_dev = static_cast<unsigned char*>(g_static_addr[dev]) + kStaticOutOffset;
  return cudaSuccess;
}

}  // namespace wan
