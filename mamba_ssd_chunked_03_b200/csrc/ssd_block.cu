// The Mamba-2 block pieces around the SSD that need no trained weights
// ("SSM 家族全景图（下）：Mamba-2 与 Jamba", section 5, the block's data
// flow): the main path's one-dimensional causal convolution followed by SiLU,
// depthwise (one filter of width K per channel):
//     out[b,t,c] = SiLU(bias_c + sum_k w[c,k] u[b, t-(K-1)+k, c])
// with zeros before the first token and, for packed sequences, no tap that
// reaches into an earlier sequence (the same cut as the SSD's decay).
//
// Bound by HBM: u read once (plus a K-1 token halo per strip, from L2) and
// out written once.  A thread owns one vector of 4 channels (8 bytes of bf16,
// 16 of fp32) over a strip of kStrip tokens; its filter taps, bias and the K-1
// previous inputs (with their sequence ids) stay in registers while it walks
// the strip.  Consecutive threads take consecutive channel vectors, so every
// load and store of a warp is contiguous.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {
namespace {

constexpr int kStrip = 32;        // tokens per thread
constexpr int kConvThreads = 128;
constexpr int kMaxWidth = 4;

struct ConvArgs {
  int64_t L, C;
  const void* u;
  const float* w;     // (C, K)
  const float* bias;  // (C) or null
  const int32_t* seq;  // (b, L) or null
  void* out;
};

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 4;  // 8-byte vectors: half the registers of 16-byte ones, twice the resident warps
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162*>(&q.x);
    const __nv_bfloat162 h1 = *reinterpret_cast<const __nv_bfloat162*>(&q.y);
    v[0] = __low2float(h0);
    v[1] = __high2float(h0);
    v[2] = __low2float(h1);
    v[3] = __high2float(h1);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[4]) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&h0),
                                              *reinterpret_cast<const uint32_t*>(&h1));
  }
};
template <>
struct Vec<float> {
  static constexpr int n = 4;
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x, v[1] = q.y, v[2] = q.z, v[3] = q.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

__device__ __forceinline__ float silu(float v) { return v / (1.f + expf(-v)); }

// grid: (channel vectors / kConvThreads, token strips, batch rows)
template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads) k_conv1d_silu(const ConvArgs a) {
  constexpr int V = Vec<T>::n;
  const int64_t c0 = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) * V;
  if (c0 >= a.C) return;
  const int64_t b = blockIdx.z;
  const int64_t t0 = (int64_t)blockIdx.y * kStrip;
  const T* u = static_cast<const T*>(a.u) + b * a.L * a.C + c0;
  T* out = static_cast<T*>(a.out) + b * a.L * a.C + c0;
  const int32_t* seq = a.seq ? a.seq + b * a.L : nullptr;
  float w[V][K], bias[V];
#pragma unroll
  for (int v = 0; v < V; ++v) {
    bias[v] = a.bias ? a.bias[c0 + v] : 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) w[v][k] = a.w[(c0 + v) * K + k];
  }
  // win[j]: the input at token t-(K-1)+j for j < K-1 (zero before token 0),
  // with its sequence id (-1 there)
  float win[K > 1 ? K - 1 : 1][V];
  int wseq[K > 1 ? K - 1 : 1];
#pragma unroll
  for (int j = 0; j < K - 1; ++j) {
    const int64_t s = t0 - (K - 1) + j;
    if (s >= 0) {
      Vec<T>::load(u + s * a.C, win[j]);
      wseq[j] = seq ? seq[s] : 0;
    } else {
#pragma unroll
      for (int v = 0; v < V; ++v) win[j][v] = 0.f;
      wseq[j] = -1;
    }
  }
  const int64_t t_end = t0 + kStrip < a.L ? t0 + kStrip : a.L;
  for (int64_t t = t0; t < t_end; ++t) {
    float cur[V];
    Vec<T>::load(u + t * a.C, cur);
    const int st = seq ? seq[t] : 0;
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = fmaf(w[v][K - 1], cur[v], bias[v]);
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
      if (wseq[j] == st) {  // same sequence (ids are >= 0; a tap before token 0 carries -1)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = fmaf(w[v][j], win[j][v], acc[v]);
      }
    }
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = silu(acc[v]);
    Vec<T>::store(out + t * a.C, acc);
#pragma unroll
    for (int j = 0; j + 1 < K - 1; ++j) {
#pragma unroll
      for (int v = 0; v < V; ++v) win[j][v] = win[j + 1][v];
      wseq[j] = wseq[j + 1];
    }
    if (K > 1) {
#pragma unroll
      for (int v = 0; v < V; ++v) win[K > 1 ? K - 2 : 0][v] = cur[v];
      wseq[K > 1 ? K - 2 : 0] = st;
    }
  }
}

template <typename T>
cudaError_t launch_conv(const ssd_conv_args* p, cudaStream_t st) {
  constexpr int V = Vec<T>::n;
  ConvArgs a;
  a.L = p->seqlen;
  a.C = p->channels;
  a.u = p->u;
  a.w = p->weight;
  a.bias = p->bias;
  a.seq = p->seq_idx;
  a.out = p->out;
  const dim3 grid((unsigned)((p->channels / V + kConvThreads - 1) / kConvThreads),
                  (unsigned)((p->seqlen + kStrip - 1) / kStrip), (unsigned)p->batch);
  switch (p->width) {
    case 1: k_conv1d_silu<T, 1><<<grid, kConvThreads, 0, st>>>(a); break;
    case 2: k_conv1d_silu<T, 2><<<grid, kConvThreads, 0, st>>>(a); break;
    case 3: k_conv1d_silu<T, 3><<<grid, kConvThreads, 0, st>>>(a); break;
    default: k_conv1d_silu<T, 4><<<grid, kConvThreads, 0, st>>>(a); break;
  }
  return cudaGetLastError();
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

}  // namespace
}  // namespace ssd

extern "C" SSD_API ssd_status ssd_conv1d_silu(const ssd_conv_args* a, void* stream) {
  using namespace ssd;
  if (!a || !a->u || !a->weight || !a->out) return SSD_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->seqlen <= 0 || a->channels <= 0 || a->width <= 0) return SSD_ERR_INVALID_ARG;
  if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (!aligned16(a->u) || !aligned16(a->out)) return SSD_ERR_INVALID_ARG;
  if (a->width > kMaxWidth || a->channels % 4 != 0) return SSD_ERR_UNSUPPORTED;
  if (a->batch > 65535 || (a->seqlen + kStrip - 1) / kStrip > 65535) return SSD_ERR_UNSUPPORTED;
  const cudaError_t e = a->dtype == SSD_BF16 ? launch_conv<__nv_bfloat16>(a, static_cast<cudaStream_t>(stream))
                                             : launch_conv<float>(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
