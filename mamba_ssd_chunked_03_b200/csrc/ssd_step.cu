// One recurrent step of the SSD (decode): a single new token per batch row
// against a running state the caller keeps,
//     state[b,h] <- exp(dt A_h) state[b,h] + dt x[b,h] B[b,g]^T
//     y[b,h]      = state[b,h] C[b,g] + D_h x[b,h]
// the sequential (recurrent) form of the same model: "22 · Mamba 2 —
// Transformers are SSMs" section 3.1 (the scalar-A recurrence), with the D
// feed-through of "从Transformer的二次复杂度困境到Mamba的线性突围" (continuous
// SSM equations).  It equals ssd_fwd over one token with initial_states =
// state and final_states written back to state.
//
// The step is bound by HBM on the state (read and written once,
// 8 b H P N bytes); x, B, C, y are small.  One CTA per (row, head): its 8
// warps take the state rows p, each lane four consecutive states n (float4
// loads and stores, coalesced along the row), B and C held in registers, and
// y_p reduced across the warp.  A warp loads the state of kRowsInFlight of its
// rows before it updates any of them, so that many loads are in flight at
// once (one row at a time left the step bound by load latency).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {
namespace {

constexpr int kStepThreads = 256;
constexpr int kStepMaxN = 256;  // states per row a lane group covers: 4 per lane, twice
constexpr int kRowsInFlight = 8;  // rows a warp loads before updating them

struct StepArgs {
  int64_t H, P, N, hpg, G;
  const void* x;
  const float* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  float* state;
  void* y;
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f(float* d, float v) { *d = v; }
__device__ __forceinline__ void from_f(__nv_bfloat16* d, float v) { *d = __float2bfloat16_rn(v); }

// four consecutive values of B or C as fp32 (8- or 16-byte aligned loads)
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}

// NK: 128-state halves of a row a lane covers (1 for N <= 128, 2 up to 256)
template <typename T, int NK>
__global__ void __launch_bounds__(kStepThreads) k_ssd_step(const StepArgs a) {
  const int64_t bh = blockIdx.x;  // b * H + h
  const int64_t b = bh / a.H, h = bh % a.H, g = h / a.hpg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float dtv = a.dt[bh];
  const float decay = expf(dtv * a.A[h]);
  const float dsk = a.D ? a.D[h] : 0.f;
  const T* Bp = static_cast<const T*>(a.B) + (b * a.G + g) * a.N;
  const T* Cp = static_cast<const T*>(a.C) + (b * a.G + g) * a.N;
  const T* xp = static_cast<const T*>(a.x) + bh * a.P;
  T* yp = static_cast<T*>(a.y) + bh * a.P;
  float* __restrict__ S = a.state + bh * a.P * a.N;
  // this lane's states: n = 4 lane + 128 k, k < NK
  float4 bv[NK], cv[NK];
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const int n = 4 * lane + 128 * k;
    bv[k] = n < a.N ? load4(Bp + n) : make_float4(0.f, 0.f, 0.f, 0.f);
    cv[k] = n < a.N ? load4(Cp + n) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  constexpr int kWarps = kStepThreads / 32;
  for (int64_t p0 = warp; p0 < a.P; p0 += kRowsInFlight * kWarps) {
    float4 sv[kRowsInFlight][NK];
    float xv[kRowsInFlight];
#pragma unroll
    for (int r = 0; r < kRowsInFlight; ++r) {
      const int64_t p = p0 + (int64_t)r * kWarps;
      if (p < a.P) {
        xv[r] = to_f(xp[p]);
#pragma unroll
        for (int k = 0; k < NK; ++k) {
          const int n = 4 * lane + 128 * k;
          if (n < a.N) sv[r][k] = *reinterpret_cast<const float4*>(S + p * a.N + n);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsInFlight; ++r) {
      const int64_t p = p0 + (int64_t)r * kWarps;
      if (p >= a.P) break;  // (uniform across the warp)
      const float u = dtv * xv[r];
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        const int n = 4 * lane + 128 * k;
        if (n < a.N) {
          float4 st = sv[r][k];
          st.x = fmaf(decay, st.x, u * bv[k].x);
          st.y = fmaf(decay, st.y, u * bv[k].y);
          st.z = fmaf(decay, st.z, u * bv[k].z);
          st.w = fmaf(decay, st.w, u * bv[k].w);
          *reinterpret_cast<float4*>(S + p * a.N + n) = st;
          acc = fmaf(st.x, cv[k].x, fmaf(st.y, cv[k].y, fmaf(st.z, cv[k].z, fmaf(st.w, cv[k].w, acc))));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) from_f(yp + p, fmaf(dsk, xv[r], acc));
    }
  }
}

bool aligned(const void* p, size_t n) { return reinterpret_cast<uintptr_t>(p) % n == 0; }

}  // namespace
}  // namespace ssd

extern "C" SSD_API ssd_status ssd_step(const ssd_step_args* a, void* stream) {
  using namespace ssd;
  if (!a) return SSD_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->nheads <= 0 || a->headdim <= 0 || a->dstate <= 0 || a->ngroups <= 0)
    return SSD_ERR_INVALID_ARG;
  if (a->nheads % a->ngroups != 0) return SSD_ERR_INVALID_ARG;
  if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (!a->x || !a->dt || !a->A || !a->B || !a->C || !a->state || !a->y) return SSD_ERR_INVALID_ARG;
  const size_t esz = a->dtype == SSD_BF16 ? 2 : 4;
  if (!aligned(a->state, 16) || !aligned(a->B, 4 * esz) || !aligned(a->C, 4 * esz)) return SSD_ERR_INVALID_ARG;
  if (a->dstate % 4 != 0 || a->dstate > kStepMaxN) return SSD_ERR_UNSUPPORTED;
  if ((double)a->batch * (double)a->nheads >= 2147483647.0) return SSD_ERR_UNSUPPORTED;
  StepArgs s;
  s.H = a->nheads;
  s.P = a->headdim;
  s.N = a->dstate;
  s.G = a->ngroups;
  s.hpg = a->nheads / a->ngroups;
  s.x = a->x;
  s.dt = a->dt;
  s.A = a->A;
  s.B = a->B;
  s.C = a->C;
  s.D = a->D;
  s.state = a->state;
  s.y = a->y;
  const unsigned grid = (unsigned)(a->batch * a->nheads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool two = a->dstate > 128;
  if (a->dtype == SSD_BF16) {
    if (two) k_ssd_step<__nv_bfloat16, 2><<<grid, kStepThreads, 0, st>>>(s);
    else k_ssd_step<__nv_bfloat16, 1><<<grid, kStepThreads, 0, st>>>(s);
  } else {
    if (two) k_ssd_step<float, 2><<<grid, kStepThreads, 0, st>>>(s);
    else k_ssd_step<float, 1><<<grid, kStepThreads, 0, st>>>(s);
  }
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
