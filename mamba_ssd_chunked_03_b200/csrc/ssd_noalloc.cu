// ssd_fwd_noalloc: the SSD forward for callers that cannot allocate device
// memory at call time.
//
// Who needs this: code that runs where no device allocator is reachable or
// allowed once work has started -- for example a plugin inside a host runtime
// that owns all device memory and exposes no allocation hook to C, or a
// latency-critical loop that must not pay for (or risk the failure of) a
// cudaMalloc after start-up.  ssd_fwd asks such callers for a workspace they
// cannot provide; this entry point brings its own.
//
// How: the scratch lives in one file-scope __device__ array of fixed size,
// created when this module is loaded on a device and kept until the process
// exits.  The host never names the array directly (in host code its name is
// only a stand-in, not a device address); its address is looked up with
// cudaGetSymbolAddress while the device is current -- on the first call on a
// device and again on every call made outside stream capture, so that a
// device reset, which reloads the module, cannot leave a stale address -- and
// passed to ssd_fwd as its workspace.  The call takes ssd_fwd's own kernel
// path when that path's workspace fits the array, else the generic kernels.
// Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cuda_runtime.h>

#include <mutex>

#include "ssd.h"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device: looked up on the
// first call on a device and on every call outside stream capture (a lookup is
// not allowed while capturing; the address found before is used then).
// Returns nullptr if the lookup fails.
void* scratch_on_current_device(cudaStream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev] || cap == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_fwd_noalloc(const ssd_fwd_args* args, void* stream) {
  if (!args) return SSD_ERR_INVALID_ARG;
  // Same argument rules as ssd_fwd; the workspace fields are ignored.  The
  // kernel path is ssd_fwd's own if its workspace fits the array, else the
  // generic one.  The seq_idx check, if asked for, uses host memory only.
  ssd_fwd_args a = *args;
  a.flags = args->flags & (SSD_FLAG_GENERIC | SSD_FLAG_CHECK_SEQ);
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  size_t need = ssd_fwd_workspace_size(&a);
  if (need > ssd::kNoAllocScratchBytes && !(a.flags & SSD_FLAG_GENERIC)) {
    a.flags |= SSD_FLAG_GENERIC;
    need = ssd_fwd_workspace_size(&a);
  }
  if (need == 0) return ssd_fwd(&a, stream);  // invalid sizes: ssd_fwd names the error
  if (need > ssd::kNoAllocScratchBytes) return SSD_ERR_WORKSPACE;
  if (!a.x || !a.dt || !a.A || !a.B || !a.C || !a.y) return SSD_ERR_INVALID_ARG;
  void* scratch = ssd::scratch_on_current_device(static_cast<cudaStream_t>(stream));
  if (!scratch) return SSD_ERR_CUDA;
  a.workspace = scratch;
  a.workspace_bytes = ssd::kNoAllocScratchBytes;
  return ssd_fwd(&a, stream);
}
