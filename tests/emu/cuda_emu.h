// Test-only host emulation of the few CUDA built-ins the backward kernels
// use, so that their source runs on the CPU under AddressSanitizer or
// ThreadSanitizer.  It checks indexing, barriers and arithmetic before a GPU
// sees the code; it is not a CPU implementation of anything and nothing
// outside tests/ includes it.
//
// A block's threads run either as fibers in one host thread (the default:
// __syncthreads yields, and every fiber runs up to its next barrier in turn,
// in forward or reverse thread order) or, with SSD_EMU_THREADS, as host
// threads meeting at a std::barrier (for ThreadSanitizer).
#ifndef SSD_CUDA_EMU_H_
#define SSD_CUDA_EMU_H_

#include <cmath>
#include <cstdint>
#include <cstring>

#ifdef SSD_EMU_THREADS
#include <barrier>
#else
#include <ucontext.h>
#endif

#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)

struct dim3 {
  unsigned x = 1, y = 1, z = 1;
};

#ifdef SSD_EMU_THREADS
inline thread_local dim3 threadIdx;
inline thread_local dim3 blockIdx;
#else
inline dim3 threadIdx;  // the running fiber's
inline dim3 blockIdx;
#endif
inline dim3 blockDim;
inline dim3 gridDim;

namespace emu {
inline float* g_smem = nullptr;  // the running block's dynamic shared memory
#ifdef SSD_EMU_THREADS
inline std::barrier<>* g_barrier = nullptr;
#else
inline ucontext_t g_sched;       // the block scheduler's context
inline ucontext_t* g_self = nullptr;  // the running fiber's context
#endif
}  // namespace emu

#ifdef SSD_EMU_THREADS
inline void __syncthreads() { emu::g_barrier->arrive_and_wait(); }
#else
inline void __syncthreads() { swapcontext(emu::g_self, &emu::g_sched); }
#endif

#define SSD_DYN_SMEM(name) float* name = emu::g_smem

// The 16-byte vector type of 4 floats.
struct float4 {
  float x, y, z, w;
};
inline float4 make_float4(float x, float y, float z, float w) { return float4{x, y, z, w}; }

// The fast-math intrinsics, at host precision.
inline float __expf(float v) { return std::exp(v); }
inline float __fdividef(float a, float b) { return a / b; }

// The cuda_pipeline primitives: an asynchronous copy to shared memory lands
// at once here; the wait and the CTA barrier after it order it as on a GPU.
inline void __pipeline_memcpy_async(void* dst, const void* src, size_t n) { std::memcpy(dst, src, n); }
inline void __pipeline_commit() {}
inline void __pipeline_wait_prior(size_t) {}

// bf16 is the upper half of an IEEE binary32: widening is a shift.
struct __nv_bfloat16 {
  uint16_t bits;
};
inline float __bfloat162float(__nv_bfloat16 v) {
  const uint32_t u = (uint32_t)v.bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

#endif  // SSD_CUDA_EMU_H_
