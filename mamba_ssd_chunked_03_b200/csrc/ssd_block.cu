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
// load and store of a warp is contiguous.  The strip is read kGroup tokens at
// a time, all of a group's loads issued before its first output is formed, so
// that each thread keeps several loads in flight; the channel pairs are
// computed in packed fp32x2 arithmetic, and SiLU takes the hardware exponential
// and an approximate divide: a relative error of a few millionths, far below
// the bf16 rounding of the output, for a third of the instructions of the
// correctly rounded forms (which left the kernel issue-bound).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {
namespace {

constexpr int kStrip = 32;        // tokens per thread
constexpr int kGroup = 4;         // tokens loaded before any of them is used
constexpr int kConvThreads = 128;
constexpr int kMaxWidth = 4;
constexpr int kVec = 4;           // channels per thread

struct ConvArgs {
  int64_t L, C;
  const void* u;
  const float* w;     // (C, K)
  const float* bias;  // (C) or null
  const int32_t* seq;  // (b, L) or null
  void* out;
};

// A thread's 4 channels as they sit in memory, and as two fp32 pairs.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  using Raw = uint2;  // 8 bytes: half the registers of 8-channel vectors, twice the resident warps
  static __device__ __forceinline__ float2 pair(uint32_t q) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q));
  }
  static __device__ __forceinline__ uint32_t pack(float2 v) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  static __device__ __forceinline__ void unpack(Raw q, float2 (&v)[2]) { v[0] = pair(q.x), v[1] = pair(q.y); }
  static __device__ __forceinline__ Raw pack(const float2 (&v)[2]) { return make_uint2(pack(v[0]), pack(v[1])); }
};
template <>
struct Vec<float> {
  using Raw = float4;
  static __device__ __forceinline__ void unpack(Raw q, float2 (&v)[2]) {
    v[0] = make_float2(q.x, q.y), v[1] = make_float2(q.z, q.w);
  }
  static __device__ __forceinline__ Raw pack(const float2 (&v)[2]) { return make_float4(v[0].x, v[0].y, v[1].x, v[1].y); }
};

__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// grid: (channel vectors / kConvThreads, token strips, batch rows).  SEQ: the
// row carries sequence ids (taps into an earlier sequence add nothing).
template <typename T, int K, bool SEQ>
__global__ void __launch_bounds__(kConvThreads) k_conv1d_silu(const ConvArgs a) {
  using Raw = typename Vec<T>::Raw;
  constexpr int NP = kVec / 2;  // channel pairs per thread
  const int64_t c0 = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) * kVec;
  if (c0 >= a.C) return;
  const int64_t b = blockIdx.z;
  const int64_t t0 = (int64_t)blockIdx.y * kStrip;
  const int64_t rs = a.C / kVec;  // a token row, in vectors
  const Raw* __restrict__ u = reinterpret_cast<const Raw*>(static_cast<const T*>(a.u) + b * a.L * a.C + c0);
  Raw* __restrict__ out = reinterpret_cast<Raw*>(static_cast<T*>(a.out) + b * a.L * a.C + c0);
  const int32_t* __restrict__ seq = SEQ ? a.seq + b * a.L : nullptr;
  float2 w[NP][K], bias[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int64_t c = c0 + 2 * p;
    bias[p] = a.bias ? make_float2(a.bias[c], a.bias[c + 1]) : make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < K; ++k) w[p][k] = make_float2(a.w[c * K + k], a.w[(c + 1) * K + k]);
  }
  // win[j]: the input at token t-(K-1)+j for j < K-1 (zero before token 0),
  // with its sequence id (-1 there)
  float2 win[K > 1 ? K - 1 : 1][NP];
  int wseq[K > 1 ? K - 1 : 1];
#pragma unroll
  for (int j = 0; j < K - 1; ++j) {
    const int64_t s = t0 - (K - 1) + j;
    if (s >= 0) {
      Vec<T>::unpack(__ldg(u + s * rs), win[j]);
      wseq[j] = SEQ ? seq[s] : 0;
    } else {
#pragma unroll
      for (int p = 0; p < NP; ++p) win[j][p] = make_float2(0.f, 0.f);
      wseq[j] = -1;
    }
  }
  const int64_t t_end = t0 + kStrip < a.L ? t0 + kStrip : a.L;
  for (int64_t tg = t0; tg < t_end; tg += kGroup) {
    Raw raw[kGroup];
    int sq[kGroup];
#pragma unroll
    for (int g = 0; g < kGroup; ++g) {
      if (tg + g < t_end) {
        raw[g] = __ldcs(u + (tg + g) * rs);
        sq[g] = SEQ ? seq[tg + g] : 0;
      }
    }
#pragma unroll
    for (int g = 0; g < kGroup; ++g) {
      if (tg + g < t_end) {
        float2 cur[NP], acc[NP];
        Vec<T>::unpack(raw[g], cur);
#pragma unroll
        for (int p = 0; p < NP; ++p) acc[p] = __ffma2_rn(w[p][K - 1], cur[p], bias[p]);
#pragma unroll
        for (int j = 0; j < K - 1; ++j) {
          // same sequence (ids are >= 0; a tap before token 0 carries -1 and a zero input)
          if (!SEQ || wseq[j] == sq[g]) {
#pragma unroll
            for (int p = 0; p < NP; ++p) acc[p] = __ffma2_rn(w[p][j], win[j][p], acc[p]);
          }
        }
#pragma unroll
        for (int p = 0; p < NP; ++p) acc[p] = make_float2(silu(acc[p].x), silu(acc[p].y));
        __stcs(out + (tg + g) * rs, Vec<T>::pack(acc));
#pragma unroll
        for (int j = 0; j + 1 < K - 1; ++j) {
#pragma unroll
          for (int p = 0; p < NP; ++p) win[j][p] = win[j + 1][p];
          wseq[j] = wseq[j + 1];
        }
        if (K > 1) {
#pragma unroll
          for (int p = 0; p < NP; ++p) win[K > 1 ? K - 2 : 0][p] = cur[p];
          wseq[K > 1 ? K - 2 : 0] = sq[g];
        }
      }
    }
  }
}

template <typename T, bool SEQ>
void launch_width(const ConvArgs& a, int width, dim3 grid, cudaStream_t st) {
  switch (width) {
    case 1: k_conv1d_silu<T, 1, SEQ><<<grid, kConvThreads, 0, st>>>(a); break;
    case 2: k_conv1d_silu<T, 2, SEQ><<<grid, kConvThreads, 0, st>>>(a); break;
    case 3: k_conv1d_silu<T, 3, SEQ><<<grid, kConvThreads, 0, st>>>(a); break;
    default: k_conv1d_silu<T, 4, SEQ><<<grid, kConvThreads, 0, st>>>(a); break;
  }
}

template <typename T>
cudaError_t launch_conv(const ssd_conv_args* p, cudaStream_t st) {
  ConvArgs a;
  a.L = p->seqlen;
  a.C = p->channels;
  a.u = p->u;
  a.w = p->weight;
  a.bias = p->bias;
  a.seq = p->seq_idx;
  a.out = p->out;
  const dim3 grid((unsigned)((p->channels / kVec + kConvThreads - 1) / kConvThreads),
                  (unsigned)((p->seqlen + kStrip - 1) / kStrip), (unsigned)p->batch);
  if (a.seq)
    launch_width<T, true>(a, (int)p->width, grid, st);
  else
    launch_width<T, false>(a, (int)p->width, grid, st);
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
