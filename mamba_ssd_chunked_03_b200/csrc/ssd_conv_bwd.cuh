// The backward of the Mamba-2 block's causal depthwise conv1d + SiLU ("SSM
// 家族全景图（下）：Mamba-2 与 Jamba", section 5, the block's data flow).  The
// forward is out[t] = SiLU(a[t]), a[t] = bias + sum_k w[k] u[t-(K-1)+k] over
// the taps inside t's sequence.  With g[t] = dout[t] SiLU'(a[t]):
//
//   du[s]   = sum_k w[k] g[s+(K-1)-k]   (taps from later tokens of s's sequence)
//   dw[k]   = sum_t g[t] u[t-(K-1)+k]    (the taps the forward takes)
//   dbias   = sum_t g[t]
//
// k_conv_bwd: a block takes 256 channels (one per thread) over a strip of
// tokens (64 for bf16 inputs, 32 for fp32, the same 16 KB of each row).  It
// first stages the strip's u (with the K-1 tokens before and after it) and
// dout (with the K-1 after it) in shared memory, with 16-byte asynchronous
// copies where the rows allow them: a block keeps its whole tile in flight
// without holding registers, so three blocks per SM keep HBM busy.  Each
// thread then walks its channel through the strip: it recomputes a[t] from a
// register window of the K-1 previous inputs (with their sequence ids), like
// the forward, and runs K-1 tokens past its strip, since du of the strip's
// last tokens takes g from the next ones.  du of a token gets its K
// contributions in K consecutive steps: a K-deep shift register of pending
// sums, flushed to HBM as each token completes.  dw and dbias are summed per
// (row, strip) and written as partials; k_conv_bwd_reduce adds the partials of
// each channel in fp64, in a fixed order.  SiLU' takes the hardware exponential
// and an approximate reciprocal (a relative error of a few millionths).
//
// Bound by HBM: u and dout read once (plus a K-1 token halo from L2), du
// written once.  Only CUDA built-ins are used (the asynchronous copies through
// the cuda_pipeline primitives), so the same source also runs under the tests'
// host emulation.
#ifndef SSD_CONV_BWD_CUH_
#define SSD_CONV_BWD_CUH_

#include <stddef.h>
#include <stdint.h>

#include <type_traits>

#include "ssd.h"

#ifndef SSD_DYN_SMEM
#define SSD_DYN_SMEM(name) extern __shared__ __align__(16) float name[]
#endif

namespace ssd {
namespace convbwd {

constexpr int kThreads = 256;  // channels per block
constexpr int kMaxWidth = 4;

// tokens per strip: the same 128 bytes of each channel's column for either input type
template <typename T>
constexpr int strip_len() {
  return sizeof(T) == 2 ? 64 : 32;
}
inline int64_t strip_len(ssd_dtype d) { return d == SSD_BF16 ? 64 : 32; }

// shared memory of k_conv_bwd: u rows for tokens t0-(K-1) .. t1+(K-1)-1, dout
// rows for tokens t0 .. t1+(K-1)-1, kThreads elements each
inline size_t tile_bytes(ssd_dtype d, int K) {
  const int64_t S = strip_len(d);
  return (size_t)((S + 2 * (K - 1)) + (S + K - 1)) * kThreads * (d == SSD_BF16 ? 2 : 4);
}

struct KArgs {
  int64_t b, L, C, nstrips, cblocks;
  int K;
  int async;          // rows staged with 16-byte asynchronous copies (aligned rows)
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
  const float s = __fdividef(1.f, 1.f + __expf(-v));
  return s * fmaf(v, 1.f - s, 1.f);
}

// blockIdx.x = (row, strip, channel block), channel block fastest.  SEQ: the
// rows carry sequence ids (a.seq), and taps into an earlier sequence add nothing.
template <typename T, int K, bool SEQ>
__global__ void __launch_bounds__(kThreads) k_conv_bwd(const KArgs a) {
  SSD_DYN_SMEM(smem);
  constexpr int S = strip_len<T>();
  constexpr int RU = S + 2 * (K - 1);  // u rows of the tile
  T* su = reinterpret_cast<T*>(smem);  // row r: token t0-(K-1)+r
  T* sd = su + (size_t)RU * kThreads;  // row r: token t0+r
  const int64_t blk = blockIdx.x;
  const int64_t cb = blk % a.cblocks;
  const int64_t strip = (blk / a.cblocks) % a.nstrips;
  const int64_t b = blk / (a.cblocks * a.nstrips);
  const int64_t cbase = cb * kThreads;
  const int nch = (int)(a.C - cbase < kThreads ? a.C - cbase : kThreads);  // the block's channels
  const int64_t t0 = strip * S;
  const int64_t t1 = t0 + S < a.L ? t0 + S : a.L;              // the strip's own tokens
  const int64_t te = t1 + (K - 1) < a.L ? t1 + (K - 1) : a.L;  // tokens whose g reaches them
  const int64_t su0 = t0 - (K - 1) > 0 ? t0 - (K - 1) : 0;     // the first u token staged
  const int nu = (int)(te - su0), nd = (int)(te - t0);
  const int ru0 = (int)(su0 - (t0 - (K - 1)));
  const T* u = static_cast<const T*>(a.u) + b * a.L * a.C + cbase;
  const T* dout = static_cast<const T*>(a.dout) + b * a.L * a.C + cbase;

  // stage u tokens [su0, te) and dout tokens [t0, te) of the block's channels
  if (a.async) {
    constexpr int E = 16 / (int)sizeof(T);  // elements per copy; nch is a multiple of E here
    const int per_row = nch / E;
    for (int i = threadIdx.x; i < (nu + nd) * per_row; i += kThreads) {
      const int r = i / per_row, q = (i - r * per_row) * E;
      if (r < nu)
        __pipeline_memcpy_async(su + (size_t)(ru0 + r) * kThreads + q, u + (su0 + r) * a.C + q, 16);
      else
        __pipeline_memcpy_async(sd + (size_t)(r - nu) * kThreads + q, dout + (t0 + r - nu) * a.C + q, 16);
    }
    __pipeline_commit();
    __pipeline_wait_prior(0);
  } else if ((int)threadIdx.x < nch) {
    for (int r = 0; r < nu; ++r) su[(size_t)(ru0 + r) * kThreads + threadIdx.x] = u[(su0 + r) * a.C + threadIdx.x];
    for (int r = 0; r < nd; ++r) sd[(size_t)r * kThreads + threadIdx.x] = dout[(t0 + r) * a.C + threadIdx.x];
  }
  __syncthreads();
  if ((int)threadIdx.x >= nch) return;

  const int64_t c = cbase + threadIdx.x;
  const T* tu = su + threadIdx.x;
  const T* td = sd + threadIdx.x;
  float* du = a.du + b * a.L * a.C + c;
  const int32_t* seq = SEQ ? a.seq + b * a.L : nullptr;
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
    win[j] = s >= 0 ? cv_ld(tu, (int64_t)j * kThreads) : 0.f;
    wseq[j] = s >= 0 ? (SEQ ? seq[s] : 0) : -1;
  }
  // pend[j]: the du sum of token t-(K-1)+j so far
  float pend[K];
#pragma unroll
  for (int j = 0; j < K; ++j) pend[j] = 0.f;
  float dw[K], db = 0.f;
#pragma unroll
  for (int k = 0; k < K; ++k) dw[k] = 0.f;

  // One token of the walk.  IN: the token is the strip's own (dw and dbias
  // take its terms); ST: 0 no du store (the first K-1 tokens), 1 store (token
  // t-(K-1) is in the strip), 2 store if it is.  The walk runs in these three
  // phases so that the checks leave its main loop, which is unrolled: the
  // window and pending-sum shifts then become register renames.
  auto token = [&](int64_t t, auto in_strip, auto store_mode) {
    constexpr bool IN = decltype(in_strip)::value;
    constexpr int ST = decltype(store_mode)::value;
    const float cur = cv_ld(tu, (t - t0 + (K - 1)) * kThreads);
    const float dcur = cv_ld(td, (t - t0) * kThreads);
    const int st = SEQ ? seq[t] : 0;
    // a tap before token 0 carries id -1 and a zero input: without ids every tap counts
    bool take[K > 1 ? K - 1 : 1];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) take[j] = !SEQ || wseq[j] == st;
    float pre = fmaf(w[K - 1], cur, bias);
#pragma unroll
    for (int j = 0; j < K - 1; ++j)
      if (take[j]) pre = fmaf(w[j], win[j], pre);
    const float g = dcur * silu_slope(pre);
    if constexpr (IN) {
      db += g;
      dw[K - 1] = fmaf(g, cur, dw[K - 1]);
#pragma unroll
      for (int j = 0; j < K - 1; ++j)
        if (take[j]) dw[j] = fmaf(g, win[j], dw[j]);
    }
    pend[K - 1] = fmaf(w[K - 1], g, pend[K - 1]);
#pragma unroll
    for (int j = 0; j < K - 1; ++j)
      if (take[j]) pend[j] = fmaf(w[j], g, pend[j]);
    // token t-(K-1) has all its contributions now
    const int64_t done = t - (K - 1);
    if constexpr (ST == 1) {
      du[done * a.C] = pend[0];
    } else if constexpr (ST == 2) {
      if (done >= t0 && done < t1) du[done * a.C] = pend[0];
    }
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
  };
  using yes = std::true_type;
  using no = std::false_type;
  const int64_t tw = t0 + (K - 1) < t1 ? t0 + (K - 1) : t1;  // the first token whose t-(K-1) is in the strip
  for (int64_t t = t0; t < tw; ++t) token(t, yes{}, std::integral_constant<int, 0>{});
#pragma unroll 4
  for (int64_t t = tw; t < t1; ++t) token(t, yes{}, std::integral_constant<int, 1>{});
  for (int64_t t = t1; t < te; ++t) token(t, no{}, std::integral_constant<int, 2>{});
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

// dw (C, K) and dbias (C): the partials of every (row, strip), added in fp64
// in a fixed order.  A block takes 32 consecutive outputs; its warp r adds
// partial rows r, r+8, r+16, ... and warp 0 then adds the 8 sums pairwise.
constexpr int kReduceLanes = kThreads / 32;
constexpr size_t kReduceSmem = (size_t)kReduceLanes * 32 * sizeof(double);

__global__ void __launch_bounds__(kThreads) k_conv_bwd_reduce(const KArgs a) {
  SSD_DYN_SMEM(smem);
  double* red = reinterpret_cast<double*>(smem);  // [kReduceLanes][32]
  const int lane = (int)threadIdx.x % 32, rl = (int)threadIdx.x / 32;
  const int64_t W = a.C * (a.K + 1);
  const int64_t i = (int64_t)blockIdx.x * 32 + lane;  // c * (K + 1) + k
  const int64_t n = a.b * a.nstrips;
  double s = 0.0;
  if (i < W)
    for (int64_t r = rl; r < n; r += kReduceLanes) s += a.part[r * W + i];
  red[rl * 32 + lane] = s;
  __syncthreads();
  if (rl != 0 || i >= W) return;
  const double* q = red + lane;
  const double t = ((q[0] + q[32]) + (q[64] + q[96])) + ((q[128] + q[160]) + (q[192] + q[224]));
  const int64_t c = i / (a.K + 1), k = i % (a.K + 1);
  if (k < a.K)
    a.dw[c * a.K + k] = (float)t;
  else if (a.dbias)
    a.dbias[c] = (float)t;
}
static_assert(kReduceLanes == 8, "the pairwise sum above adds 8 lanes");

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
  k->nstrips = (a->seqlen + strip_len(a->dtype) - 1) / strip_len(a->dtype);
  k->cblocks = (a->channels + kThreads - 1) / kThreads;
  const double blocks = (double)k->b * (double)k->nstrips * (double)k->cblocks;
  if (blocks >= 2147483647.0) return SSD_ERR_UNSUPPORTED;
  *ws = ((size_t)(k->b * k->nstrips) * (size_t)k->C * (size_t)(k->K + 1) * 4 + 255) & ~(size_t)255;
  return SSD_OK;
}

template <typename T, bool SEQ, class Launch>
bool launch_width(const KArgs& k, unsigned grid, size_t smem, Launch& launch) {
  switch (k.K) {
    case 1: return launch(&k_conv_bwd<T, 1, SEQ>, grid, smem, k);
    case 2: return launch(&k_conv_bwd<T, 2, SEQ>, grid, smem, k);
    case 3: return launch(&k_conv_bwd<T, 3, SEQ>, grid, smem, k);
    default: return launch(&k_conv_bwd<T, 4, SEQ>, grid, smem, k);
  }
}

template <typename T, class Launch>
ssd_status enqueue_typed(const KArgs& k, Launch& launch) {
  const unsigned grid = (unsigned)(k.b * k.nstrips * k.cblocks);
  const size_t smem = tile_bytes(sizeof(T) == 2 ? SSD_BF16 : SSD_F32, k.K);
  const bool ok = k.seq ? launch_width<T, true>(k, grid, smem, launch) : launch_width<T, false>(k, grid, smem, launch);
  if (!ok) return SSD_ERR_CUDA;
  const unsigned rgrid = (unsigned)((k.C * (k.K + 1) + 31) / 32);
  return launch(&k_conv_bwd_reduce, rgrid, kReduceSmem, k) ? SSD_OK : SSD_ERR_CUDA;
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
  // 16-byte copies need 16-byte aligned rows: the bases and every row's stride
  const size_t esz = a->dtype == SSD_BF16 ? 2 : 4;
  k.async = reinterpret_cast<uintptr_t>(a->u) % 16 == 0 && reinterpret_cast<uintptr_t>(a->dout) % 16 == 0 &&
            ((size_t)k.C * esz) % 16 == 0;
  return a->dtype == SSD_BF16 ? enqueue_typed<__nv_bfloat16>(k, launch) : enqueue_typed<float>(k, launch);
}

}  // namespace convbwd
}  // namespace ssd

#endif  // SSD_CONV_BWD_CUH_
