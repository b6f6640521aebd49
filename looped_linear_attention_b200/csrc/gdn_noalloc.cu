// gdn_chunk_fwd_noalloc: the prefill entry point for callers that cannot
// allocate device memory, such as a plugin whose host engine owns every device
// allocation through its own pool, or a path that must not call cudaMalloc
// because it can synchronise the device.  The segmented prefill schedule needs
// scratch memory; here that scratch is one fixed array compiled into the
// library instead of a workspace the caller allocates.
#include <atomic>

#include "common.cuh"

namespace {

// Scratch of the segmented prefill schedule.  Every GPU that loads the library
// holds these bytes until the process exits.
constexpr size_t kNoallocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

using gdn::kMaxDevices;

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
gdn_status scratch_address(void** out) {
  static std::atomic<void*> cache[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
  void* ptr = cache[dev].load(std::memory_order_acquire);
  if (!ptr) {
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return GDN_ERR_CUDA;
    cache[dev].store(ptr, std::memory_order_release);
  }
  *out = ptr;
  return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_params* p, cudaStream_t stream) {
  const size_t need = gdn_chunk_fwd_workspace(p);
  if (need == (size_t)-1) return GDN_ERR_INVALID;
  if (need > kNoallocScratchBytes) {
    // the per-channel gate prefill has a one-launch kernel that needs none
    if (p->flags & GDN_CHANNEL_GATE) return gdn_chunk_fwd(p, nullptr, 0, stream);
    return GDN_ERR_WORKSPACE;
  }
  if (need == 0) return gdn_chunk_fwd(p, nullptr, 0, stream);
  void* scratch = nullptr;
  const gdn_status st = scratch_address(&scratch);
  if (st != GDN_OK) return st;
  // every word of the scratch that the call reads is written earlier in the
  // same call, so nothing needs clearing between calls
  return gdn_chunk_fwd(p, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
