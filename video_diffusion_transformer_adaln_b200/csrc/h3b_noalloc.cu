// h3b_block_forward_noalloc: the block forward with its scratch in a fixed
// device array of this library instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the moment they
// run the block. Examples are code running where the device allocator belongs
// to a host framework that forbids side allocations, plugin or callback code
// that only receives input/output pointers, and latency-critical loops where
// a cudaMalloc could synchronize the device or fail under fragmentation. This
// entry point calls no cudaMalloc, cudaFree or allocating library routine.
//
// The scratch is one file-scope device array of kStaticScratchBytes. Every GPU
// that loads this library holds it until the process exits, and every call on
// a device shares it: calls that overlap on the GPU (other streams, other host
// threads) race on it and must be serialized by the caller. Nothing in it has
// to start at zero: the block's kernels zero the one region that accumulates
// (the per-token absmax) on every call.
//
// Host code cannot use the array's name as a device address: the name is a
// host-side stand-in. The device address is taken with cudaGetSymbolAddress,
// once per device with that device current, on the first call on that device.
// That first call therefore performs setup work and should happen before any
// stream capture. The address is cached per device index, so it assumes one
// CUDA context per device and no cudaDeviceReset between calls.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "h3b.h"
#include "h3b_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once).
h3b_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    h3b::set_error_detail(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    return H3B_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    h3b::set_error_detail("device index out of range");
    return H3B_ERR_ARG;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      h3b::set_error_detail(std::string("cudaGetSymbolAddress(static scratch): ") + cudaGetErrorString(e));
      return H3B_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return H3B_OK;
}

}  // namespace

extern "C" h3b_status h3b_block_forward_noalloc(const h3b_dims* dims, const h3b_block_weights* w,
                                                const float* c, void* x, h3b_stream stream) {
  size_t need = 0;
  h3b_status s = h3b_workspace_size(dims, &need);
  if (s != H3B_OK) return s;
  if (need > kStaticScratchBytes) {
    h3b::set_error_detail("these dimensions need " + std::to_string(need) +
                          " bytes of scratch; the allocation-free entry point holds " +
                          std::to_string(kStaticScratchBytes) + " (use h3b_block_forward with a workspace)");
    return H3B_ERR_WORKSPACE;
  }
  // The device check comes first: on a device without an sm_100a image the symbol
  // lookup would fail with a CUDA error instead of the architecture status.
  if ((s = static_cast<h3b_status>(h3b::check_current_device())) != H3B_OK) return s;
  void* scratch = nullptr;
  if ((s = scratch_address(&scratch)) != H3B_OK) return s;
  return h3b_block_forward(dims, w, c, x, scratch, kStaticScratchBytes, stream);
}
