// ssd_conv1d_silu_bwd and its workspace query: the kernels of
// ssd_conv_bwd.cuh, launched on the caller's stream.
#include <cuda_bf16.h>
#include <cuda_pipeline.h>
#include <cuda_runtime.h>

#include "ssd.h"
#include "ssd_conv_bwd.cuh"

namespace {

struct CudaLaunch {
  cudaStream_t stream;
  bool operator()(void (*kern)(ssd::convbwd::KArgs), unsigned grid, size_t smem, const ssd::convbwd::KArgs& k) const {
    if (grid == 0) return true;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return false;
    kern<<<grid, ssd::convbwd::kThreads, smem, stream>>>(k);
    return cudaGetLastError() == cudaSuccess;
  }
};

}  // namespace

extern "C" SSD_API size_t ssd_conv1d_silu_bwd_workspace_size(const ssd_conv_bwd_args* a) {
  ssd::convbwd::KArgs k;
  size_t ws = 0;
  return ssd::convbwd::plan(a, &k, &ws) == SSD_OK ? ws : 0;
}

extern "C" SSD_API ssd_status ssd_conv1d_silu_bwd(const ssd_conv_bwd_args* a, void* stream) {
  CudaLaunch launch{static_cast<cudaStream_t>(stream)};
  return ssd::convbwd::run(a, launch);
}
