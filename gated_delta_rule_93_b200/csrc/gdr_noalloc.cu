// Fixed scratch for gdr_chunk_fwd_segmented_noalloc: the segment path's
// three fp32 states per segment and head, in a device array that is part of
// the library itself, so that the entry point allocates nothing.
//
// The array is reserved on every GPU that loads this module and stays there
// until the process exits.  Host code must not pass the array's name to a
// kernel (on the host that name is only a stand-in, not a device address):
// the device address is looked up once per device with
// cudaGetSymbolAddress and cached.
#include <mutex>

#include "gdr_internal.cuh"

namespace gdr {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void *g_addr[kMaxDevices] = {};

}  // namespace

cudaError_t noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_addr[dev]) {
    // the current device is `dev`, so this is its copy of the array
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace gdr
