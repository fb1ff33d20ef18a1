// Internal declarations shared by the libssd translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// Resolved problem description (validated sizes, typed pointers).
struct Problem {
  int64_t b, L, H, P, N, G, Q, nc;  // nc = ceil(L / Q) chunks per row
  int64_t hpg;                      // heads per group, H / G
  ssd_dtype dtype;
  const void* x;
  const float* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  const float* h0;
  const int32_t* seq;
  int64_t num_seqs;
  void* y;
  float* final_states;
  const void* z;  // gate: y * SiLU(z), or null
  bool stall;     // SSD_FLAG_TEST_STALL: the two-head kernel's hand-over waits never succeed
};

constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---- generic (CUDA-core, fp32) path: ssd_generic.cu ----
size_t generic_workspace_bytes(const Problem& p);
cudaError_t generic_forward(const Problem& p, void* ws, cudaStream_t stream);
int generic_launch_count(const Problem& p);

// ---- fused tensor-core path: ssd_tc.cu ----
bool tc_supported(const Problem& p, uint32_t flags);
size_t tc_workspace_bytes(const Problem& p);
int tc_launch_count(const Problem& p);
// device address of the tensor-core path's error word inside the workspace
const int* tc_error_word(const Problem& p, const void* ws);
// name of the fused kernel the tensor-core path launches for p
const char* tc_main_kernel(const Problem& p);
cudaError_t tc_forward(const Problem& p, void* ws, cudaStream_t stream, cudaEvent_t ev0, cudaEvent_t ev1);

}  // namespace ssd
