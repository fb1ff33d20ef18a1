// The backward of the Mamba-2 block's causal depthwise conv1d + SiLU ("SSM
// 家族全景图（下）：Mamba-2 与 Jamba", section 5, the block's data flow).  The
// forward is out[t] = SiLU(a[t]), a[t] = bias + sum_k w[k] u[t-(K-1)+k] over
// the taps inside t's sequence.  With g[t] = dout[t] SiLU'(a[t]):
//
//   du[s]   = sum_k w[k] g[s+(K-1)-k]   (taps from later tokens of s's sequence)
//   dw[k]   = sum_t g[t] u[t-(K-1)+k]    (the taps the forward takes)
//   dbias   = sum_t g[t]
//
// k_conv_bwd: one thread per channel over a strip of kConvStrip tokens.  It
// recomputes a[t] from a register window of the K-1 previous inputs (with
// their sequence ids), like the forward, and runs K-1 tokens past its strip,
// since du of the strip's last tokens takes g from the next ones.  du of a
// token gets its K contributions in K consecutive steps: a K-deep shift
// register of pending sums, flushed to HBM as each token completes.  dw and
// dbias are summed per (row, strip) and written as partials; k_conv_bwd_reduce
// adds the partials of each channel in fp64, in a fixed order.
//
// Bound by HBM: u and dout read once (plus a K-1 token halo from L2), du
// written once.  Consecutive threads take consecutive channels, so every
// load and store of a warp is contiguous.  Only standard CUDA built-ins are
// used, so the same source also runs under the tests' host emulation.
#ifndef SSD_CONV_BWD_CUH_
#define SSD_CONV_BWD_CUH_

#include <stddef.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {
namespace convbwd {

constexpr int kThreads = 256;
constexpr int kConvStrip = 32;  // tokens per thread
constexpr int kMaxWidth = 4;

struct KArgs {
  int64_t b, L, C, nstrips, cblocks;
  int K;
  const void* u;
  const float* w;     // (C, K)
  const float* bias;  // (C) or null
  const int32_t* seq;
  const void* dout;
  float* du;
  float* dw;
  float* dbias;
  float* part;        // (b * nstrips, C, K + 1): per-strip dw and dbias partials
};

__device__ __forceinline__ float cv_ld(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float cv_ld(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }

// SiLU'(v) = s (1 + v (1 - s)), s = 1 / (1 + e^-v)
__device__ __forceinline__ float silu_slope(float v) {
  const float s = 1.f / (1.f + expf(-v));
  return s * fmaf(v, 1.f - s, 1.f);
}

// blockIdx.x = (row, strip, channel block), channel block fastest
template <typename T, int K>
__global__ void __launch_bounds__(kThreads) k_conv_bwd(const KArgs a) {
  const int64_t blk = blockIdx.x;
  const int64_t cb = blk % a.cblocks;
  const int64_t strip = (blk / a.cblocks) % a.nstrips;
  const int64_t b = blk / (a.cblocks * a.nstrips);
  const int64_t c = cb * kThreads + threadIdx.x;
  if (c >= a.C) return;
  const int64_t t0 = strip * kConvStrip;
  const int64_t t1 = t0 + kConvStrip < a.L ? t0 + kConvStrip : a.L;  // the strip's own tokens
  const int64_t te = t1 + (K - 1) < a.L ? t1 + (K - 1) : a.L;         // tokens whose g reaches them
  const T* u = static_cast<const T*>(a.u) + b * a.L * a.C + c;
  const T* dout = static_cast<const T*>(a.dout) + b * a.L * a.C + c;
  float* du = a.du + b * a.L * a.C + c;
  const int32_t* seq = a.seq ? a.seq + b * a.L : nullptr;
  float w[K];
#pragma unroll
  for (int k = 0; k < K; ++k) w[k] = a.w[c * K + k];
  const float bias = a.bias ? a.bias[c] : 0.f;
  // win[j]: u at token t-(K-1)+j for j < K-1 (0 before token 0), wseq[j] its id (-1 there)
  float win[K > 1 ? K - 1 : 1];
  int wseq[K > 1 ? K - 1 : 1];
#pragma unroll
  for (int j = 0; j < K - 1; ++j) {
    const int64_t s = t0 - (K - 1) + j;
    win[j] = s >= 0 ? cv_ld(u, s * a.C) : 0.f;
    wseq[j] = s >= 0 ? (seq ? seq[s] : 0) : -1;
  }
  // pend[j]: the du sum of token t-(K-1)+j so far
  float pend[K];
#pragma unroll
  for (int j = 0; j < K; ++j) pend[j] = 0.f;
  float dw[K], db = 0.f;
#pragma unroll
  for (int k = 0; k < K; ++k) dw[k] = 0.f;

  // the next token's inputs are loaded before this token's du store, which the
  // compiler cannot tell apart from them: two tokens' loads in flight
  float nu = t0 < te ? cv_ld(u, t0 * a.C) : 0.f;
  float nd = t0 < te ? cv_ld(dout, t0 * a.C) : 0.f;
  int ns = (t0 < te && seq) ? seq[t0] : 0;
  for (int64_t t = t0; t < te; ++t) {
    const float cur = nu, dcur = nd;
    const int st = ns;
    if (t + 1 < te) {
      nu = cv_ld(u, (t + 1) * a.C);
      nd = cv_ld(dout, (t + 1) * a.C);
      ns = seq ? seq[t + 1] : 0;
    }
    float pre = fmaf(w[K - 1], cur, bias);
#pragma unroll
    for (int j = 0; j < K - 1; ++j)
      if (wseq[j] == st) pre = fmaf(w[j], win[j], pre);
    const float g = dcur * silu_slope(pre);
    if (t < t1) {
      db += g;
      dw[K - 1] = fmaf(g, cur, dw[K - 1]);
#pragma unroll
      for (int j = 0; j < K - 1; ++j)
        if (wseq[j] == st) dw[j] = fmaf(g, win[j], dw[j]);
    }
    pend[K - 1] = fmaf(w[K - 1], g, pend[K - 1]);
#pragma unroll
    for (int j = 0; j < K - 1; ++j)
      if (wseq[j] == st) pend[j] = fmaf(w[j], g, pend[j]);
    // token t-(K-1) has all its contributions now
    const int64_t done = t - (K - 1);
    if (done >= t0 && done < t1) du[done * a.C] = pend[0];
#pragma unroll
    for (int j = 0; j + 1 < K; ++j) pend[j] = pend[j + 1];
    pend[K - 1] = 0.f;
#pragma unroll
    for (int j = 0; j + 1 < K - 1; ++j) {
      win[j] = win[j + 1];
      wseq[j] = wseq[j + 1];
    }
    if (K > 1) {
      win[K > 1 ? K - 2 : 0] = cur;
      wseq[K > 1 ? K - 2 : 0] = st;
    }
  }
  // at the end of the row the last tokens of the strip are complete too
#pragma unroll
  for (int j = 0; j < K - 1; ++j) {
    const int64_t s = te - (K - 1) + j;
    if (te == a.L && s >= t0 && s < t1) du[s * a.C] = pend[j];
  }
  float* part = a.part + ((b * a.nstrips + strip) * a.C + c) * (K + 1);
#pragma unroll
  for (int k = 0; k < K; ++k) part[k] = dw[k];
  part[K] = db;
}

// dw (C, K) and dbias (C): the partials of every (row, strip), added in fp64.
__global__ void __launch_bounds__(kThreads) k_conv_bwd_reduce(const KArgs a) {
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;  // c * (K + 1) + k
  if (i >= a.C * (a.K + 1)) return;
  const int64_t c = i / (a.K + 1), k = i % (a.K + 1);
  const int64_t n = a.b * a.nstrips;
  double s = 0.0;
  for (int64_t r = 0; r < n; ++r) s += a.part[(r * a.C + c) * (a.K + 1) + k];
  if (k < a.K)
    a.dw[c * a.K + k] = (float)s;
  else if (a.dbias)
    a.dbias[c] = (float)s;
}

// ---------------------------------------------------------------- host side

inline ssd_status plan(const ssd_conv_bwd_args* a, KArgs* k, size_t* ws) {
  if (!a) return SSD_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->seqlen <= 0 || a->channels <= 0 || a->width <= 0) return SSD_ERR_INVALID_ARG;
  if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (a->width > kMaxWidth) return SSD_ERR_UNSUPPORTED;
  k->b = a->batch;
  k->L = a->seqlen;
  k->C = a->channels;
  k->K = (int)a->width;
  k->nstrips = (a->seqlen + kConvStrip - 1) / kConvStrip;
  k->cblocks = (a->channels + kThreads - 1) / kThreads;
  const double blocks = (double)k->b * (double)k->nstrips * (double)k->cblocks;
  if (blocks >= 2147483647.0) return SSD_ERR_UNSUPPORTED;
  *ws = ((size_t)(k->b * k->nstrips) * (size_t)k->C * (size_t)(k->K + 1) * 4 + 255) & ~(size_t)255;
  return SSD_OK;
}

template <typename T, class Launch>
ssd_status enqueue_typed(const KArgs& k, Launch& launch) {
  const unsigned grid = (unsigned)(k.b * k.nstrips * k.cblocks);
  bool ok = false;
  switch (k.K) {
    case 1: ok = launch(&k_conv_bwd<T, 1>, grid, (size_t)0, k); break;
    case 2: ok = launch(&k_conv_bwd<T, 2>, grid, (size_t)0, k); break;
    case 3: ok = launch(&k_conv_bwd<T, 3>, grid, (size_t)0, k); break;
    default: ok = launch(&k_conv_bwd<T, 4>, grid, (size_t)0, k); break;
  }
  if (!ok) return SSD_ERR_CUDA;
  const unsigned rgrid = (unsigned)((k.C * (k.K + 1) + kThreads - 1) / kThreads);
  return launch(&k_conv_bwd_reduce, rgrid, (size_t)0, k) ? SSD_OK : SSD_ERR_CUDA;
}

template <class Launch>
ssd_status run(const ssd_conv_bwd_args* a, Launch& launch) {
  KArgs k;
  size_t ws = 0;
  ssd_status st = plan(a, &k, &ws);
  if (st != SSD_OK) return st;
  if (!a->u || !a->weight || !a->dout || !a->du || !a->dweight) return SSD_ERR_INVALID_ARG;
  if (!a->workspace || a->workspace_bytes < ws) return SSD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) % 256 != 0) return SSD_ERR_INVALID_ARG;
  k.u = a->u;
  k.w = a->weight;
  k.bias = a->bias;
  k.seq = a->seq_idx;
  k.dout = a->dout;
  k.du = a->du;
  k.dw = a->dweight;
  k.dbias = a->dbias;
  k.part = static_cast<float*>(a->workspace);
  return a->dtype == SSD_BF16 ? enqueue_typed<__nv_bfloat16>(k, launch) : enqueue_typed<float>(k, launch);
}

}  // namespace convbwd
}  // namespace ssd

#endif  // SSD_CONV_BWD_CUH_
