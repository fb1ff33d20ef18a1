// ssd_bwd and ssd_bwd_workspace_size: the backward kernels of ssd_bwd.cuh and
// ssd_bwd_tc.cuh, launched on the caller's stream.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd.h"
#include "ssd_bwd.cuh"
#include "ssd_bwd_tc.cuh"

namespace {

struct CudaLaunch {
  cudaStream_t stream;
  bool operator()(void (*kern)(ssd::bwd::KArgs), unsigned grid, size_t smem, const ssd::bwd::KArgs& k) const {
    if (grid == 0) return true;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute((const void*)kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return false;
    kern<<<grid, ssd::bwd::kThreads, smem, stream>>>(k);
    return cudaGetLastError() == cudaSuccess;
  }
  bool record(void* event) const { return cudaEventRecord(static_cast<cudaEvent_t>(event), stream) == cudaSuccess; }
  bool chunk_tc_ok(const ssd::bwd::KArgs& k) const { return ssd::bwd::chunk_tc_supported(k); }
  bool chunk_tc(const ssd::bwd::KArgs& k) const { return ssd::bwd::chunk_tc_launch(k, stream) == cudaSuccess; }
  bool state_walk_tc(const ssd::bwd::KArgs& k, bool only_dh0) const {
    return ssd::bwd::state_walk_tc_launch(k, only_dh0, stream) == cudaSuccess;
  }
};

}  // namespace

extern "C" SSD_API size_t ssd_bwd_workspace_size(const ssd_bwd_args* a) {
  ssd::bwd::Plan pl;
  return ssd::bwd::plan(a, &pl) == SSD_OK ? pl.total : 0;
}

extern "C" SSD_API int64_t ssd_bwd_chunk_size(const ssd_bwd_args* a) {
  ssd::bwd::Plan pl;
  return ssd::bwd::plan(a, &pl) == SSD_OK ? pl.d.Q : 0;
}

extern "C" SSD_API const char* ssd_bwd_path(const ssd_bwd_args* a) {
  ssd::bwd::Plan pl;
  if (ssd::bwd::plan(a, &pl) != SSD_OK) return "invalid";
  return a->dtype == SSD_BF16 && ssd::bwd::chunk_tc_supported(ssd::bwd::make_kargs(a, pl)) ? "tcgen05" : "generic";
}

extern "C" SSD_API ssd_status ssd_bwd(const ssd_bwd_args* a, void* stream) {
  CudaLaunch launch{static_cast<cudaStream_t>(stream)};
  return ssd::bwd::run(a, launch);
}
