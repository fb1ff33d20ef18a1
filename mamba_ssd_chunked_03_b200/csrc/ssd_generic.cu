// Generic chunked SSD forward on CUDA cores, fp32 arithmetic throughout.
//
// This is the fp32 path (x, B, C, y in fp32) and, with bf16 tensors, the
// cross-check for the tensor-core kernels.  It follows the four chunked steps
// of "SSM 家族全景图（下）：Mamba-2 与 Jamba" section 三.4 as separate kernels
// with the per-chunk states kept in fp32 in the workspace:
//
//   k_chunk_cumsum   cs_t = sum_{k = chunk start .. t} dt_k A_h           (step 0)
//   k_chunk_state    S_c  = sum_s exp(cs_e - cs_s) dt_s x_s B_s^T          (step 2)
//   k_state_passing  H_{c+1} = keep_c exp(cs_e) H_c + S_c, in place       (step 3)
//   k_chunk_scan     y_t = sum_s (C_t.B_s) exp(cs_t - cs_s) dt_s x_s      (step 1)
//                          + keep_t exp(cs_t) C_t H_c^T + D_h x_t          (step 4)
//   k_seq_ends / k_packed_final   per-sequence final states when packed
//
// e is the chunk's last token; "keep" is 1 when no packed-sequence boundary
// lies between the chunk's start and the token in question (boundaries reset
// the transition to zero, "Transformers与SSMs的隐藏联系" section 4.2).  With
// non-decreasing ids that is an equality test of seq_idx values.  The decay
// between two tokens is always formed as exp of a difference of in-chunk
// cumulative sums with the later token first, so it never exceeds 1.
#include <cuda_bf16.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each -> 64 x 64 tiles
constexpr int kTile = 64;
constexpr int kK = 32;         // k-slab of the smem GEMMs
constexpr int kLdA = kK + 1;   // As[m][k], padded
constexpr int kLdB = kTile + 4;  // Bs[k][n], padded, keeps float4 alignment

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// acc[i][j] += sum_{k < kk} As[(ty*4+i)][k] * Bs[k][(tx*4+j)]
__device__ __forceinline__ void mma_tile(float acc[4][4], const float* As, int lda, const float* Bs,
                                         int ldb, int kk, int ty, int tx) {
#pragma unroll 4
  for (int k = 0; k < kk; ++k) {
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = As[(ty * 4 + i) * lda + k];
    const float4 bv = *reinterpret_cast<const float4*>(Bs + k * ldb + tx * 4);
    const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
  }
}

__device__ __forceinline__ int seq_at(const Problem& pr, int64_t b, int64_t t) {
  return pr.seq ? pr.seq[b * pr.L + t] : 0;
}

// ---------------------------------------------------------------- step 0
__global__ void k_chunk_cumsum(Problem pr, float* __restrict__ cs) {
  const int64_t c = blockIdx.x;
  const int64_t b = blockIdx.y;
  for (int64_t h = threadIdx.x; h < pr.H; h += blockDim.x) {
    const float a = pr.A[h];
    float acc = 0.f;
    float* out = cs + ((b * pr.H + h) * pr.nc + c) * pr.Q;
    for (int64_t i = 0; i < pr.Q; ++i) {
      const int64_t t = c * pr.Q + i;
      if (t < pr.L) acc = fmaf(pr.dt[(b * pr.L + t) * pr.H + h], a, acc);
      out[i] = acc;
    }
  }
}

// ---------------------------------------------------------------- step 2 tile
// acc[p][n] (64 x 64 tile at p0, n0) = sum over in-chunk s <= e with the same
// sequence as e of exp(cs_e - cs_s) dt_s x[s,p] B[s,n].
template <typename T>
__device__ void state_tile(const Problem& pr, const float* __restrict__ cs, int64_t b, int64_t c,
                           int64_t h, int e, int p0, int n0, float acc[4][4], float* smem) {
  float* As = smem;                  // [64 p][kLdA] : x[s][p] * w_s
  float* Bs = As + kTile * kLdA;     // [kK s][kLdB] : B[s][n]
  float* ws = Bs + kK * kLdB;        // [kK] weights
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t g = h / pr.hpg;
  const int64_t t0 = c * pr.Q;
  const float* csc = cs + ((b * pr.H + h) * pr.nc + c) * pr.Q;
  const float cs_e = csc[e];
  const int seq_e = seq_at(pr, b, t0 + e);
  const T* x = static_cast<const T*>(pr.x);
  const T* Bm = static_cast<const T*>(pr.B);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 <= e; k0 += kK) {
    if (tid < kK) {
      const int k = k0 + tid;
      float w = 0.f;
      if (k <= e && seq_at(pr, b, t0 + k) == seq_e)
        w = expf(cs_e - csc[k]) * pr.dt[(b * pr.L + t0 + k) * pr.H + h];
      ws[tid] = w;
    }
    __syncthreads();
    for (int idx = tid; idx < kK * kTile; idx += kThreads) {
      // As[p][k]: consecutive threads take consecutive p (coalesced x reads)
      const int p = idx % kTile, k = idx / kTile;
      float v = 0.f;
      if (k0 + k <= e && p0 + p < pr.P)
        v = to_f(x[((b * pr.L + t0 + k0 + k) * pr.H + h) * pr.P + p0 + p]) * ws[k];
      As[p * kLdA + k] = v;
      const int n = idx % kTile;
      float bv = 0.f;
      if (k0 + k <= e && n0 + n < pr.N)
        bv = to_f(Bm[((b * pr.L + t0 + k0 + k) * pr.G + g) * pr.N + n0 + n]);
      Bs[k * kLdB + n] = bv;
    }
    __syncthreads();
    mma_tile(acc, As, kLdA, Bs, kLdB, kK, ty, tx);
    __syncthreads();
  }
}

constexpr size_t kStateSmem = (kTile * kLdA + kK * kLdB + kK) * sizeof(float);

template <typename T>
__global__ void __launch_bounds__(kThreads) k_chunk_state(Problem pr, const float* __restrict__ cs,
                                                          float* __restrict__ states) {
  extern __shared__ float smem[];
  const int64_t tp = (pr.P + kTile - 1) / kTile, tn = (pr.N + kTile - 1) / kTile;
  int64_t r = blockIdx.x;
  const int64_t tile = r % (tp * tn);
  r /= (tp * tn);
  const int64_t h = r % pr.H;
  const int64_t c = r / pr.H;
  const int64_t b = blockIdx.y;
  const int p0 = (int)(tile / tn) * kTile, n0 = (int)(tile % tn) * kTile;
  const int e = (int)(((c + 1) * pr.Q <= pr.L ? pr.Q : pr.L - c * pr.Q) - 1);
  float acc[4][4];
  state_tile<T>(pr, cs, b, c, h, e, p0, n0, acc, smem);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float* out = states + ((b * pr.nc + c) * pr.H + h) * pr.P * pr.N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int p = p0 + ty * 4 + i;
    if (p >= pr.P) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < pr.N) out[(int64_t)p * pr.N + n] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------- step 3
// In place: states[c] holds S_c on entry and H_c (the state entering chunk c)
// on exit.  One thread per 4 consecutive state elements of one (b, h).
__global__ void k_state_passing(Problem pr, const float* __restrict__ cs, float* __restrict__ states) {
  const int64_t bh = blockIdx.y;
  const int64_t b = bh / pr.H, h = bh % pr.H;
  const int64_t PN = pr.P * pr.N;
  const int64_t i4 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i4 >= PN) return;
  float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
  if (pr.h0) hs = *reinterpret_cast<const float4*>(pr.h0 + (b * pr.H + h) * PN + i4);
  const float* csh = cs + (b * pr.H + h) * pr.nc * pr.Q;
  for (int64_t c = 0; c < pr.nc; ++c) {
    float4* slot = reinterpret_cast<float4*>(states + ((b * pr.nc + c) * pr.H + h) * PN + i4);
    const float4 s = *slot;
    *slot = hs;
    const int64_t t0 = c * pr.Q;
    const int64_t e = ((c + 1) * pr.Q <= pr.L ? pr.Q : pr.L - t0) - 1;
    const bool keep = seq_at(pr, b, t0 + e) == seq_at(pr, b, t0 > 0 ? t0 - 1 : 0);
    const float dec = keep ? expf(csh[c * pr.Q + e]) : 0.f;
    hs.x = fmaf(dec, hs.x, s.x);
    hs.y = fmaf(dec, hs.y, s.y);
    hs.z = fmaf(dec, hs.z, s.z);
    hs.w = fmaf(dec, hs.w, s.w);
  }
  if (!pr.seq && pr.final_states)
    *reinterpret_cast<float4*>(pr.final_states + (b * pr.H + h) * PN + i4) = hs;
}

// ---------------------------------------------------------------- steps 1 + 4
constexpr int kLdW = kTile + 1;  // As[t][s] for the W.X product
constexpr size_t kScanSmem =
    (kTile * kLdA + kK * kLdB + kTile * kLdW + kTile * kLdB) * sizeof(float) + 3 * 256 * sizeof(float);

template <typename T>
__global__ void __launch_bounds__(kThreads) k_chunk_scan(Problem pr, const float* __restrict__ cs,
                                                         const float* __restrict__ prev) {
  extern __shared__ float smem[];
  float* As = smem;                  // [64 t][kLdA] C slab
  float* Bs = As + kTile * kLdA;     // [kK][kLdB] H^T or B^T slab
  float* Ws = Bs + kK * kLdB;        // [64 t][kLdW] masked weights
  float* Xs = Ws + kTile * kLdW;     // [64 s][kLdB] x tile
  float* css = Xs + kTile * kLdB;    // [Q] cumulative sums
  float* dts = css + 256;            // [Q] dt
  int* sqs = reinterpret_cast<int*>(dts + 256);  // [Q] seq ids

  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t tp = (pr.P + kTile - 1) / kTile;
  const int64_t tt = (pr.Q + kTile - 1) / kTile;
  int64_t r = blockIdx.x;
  const int pp0 = (int)(r % tp) * kTile;
  r /= tp;
  const int tt0 = (int)(r % tt) * kTile;
  r /= tt;
  const int64_t h = r % pr.H;
  const int64_t c = r / pr.H;
  const int64_t b = blockIdx.y;
  const int64_t g = h / pr.hpg;
  const int64_t t0 = c * pr.Q;
  const int nvalid = (int)((c + 1) * pr.Q <= pr.L ? pr.Q : pr.L - t0);
  if (tt0 >= nvalid) return;  // whole tile past the ragged tail (uniform per block)
  const T* x = static_cast<const T*>(pr.x);
  const T* Bm = static_cast<const T*>(pr.B);
  const T* Cm = static_cast<const T*>(pr.C);
  T* y = static_cast<T*>(pr.y);

  for (int i = tid; i < pr.Q; i += kThreads) {
    css[i] = cs[((b * pr.H + h) * pr.nc + c) * pr.Q + i];
    const bool v = i < nvalid;
    dts[i] = v ? pr.dt[(b * pr.L + t0 + i) * pr.H + h] : 0.f;
    sqs[i] = v ? seq_at(pr, b, t0 + i) : -1;
  }
  const int seq_prev = seq_at(pr, b, t0 > 0 ? t0 - 1 : 0);
  __syncthreads();

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  // step 4: C_t . H_c^T for the state entering the chunk
  const float* Hc = prev + ((b * pr.nc + c) * pr.H + h) * pr.P * pr.N;
  for (int n0 = 0; n0 < pr.N; n0 += kK) {
    for (int idx = tid; idx < kTile * kK; idx += kThreads) {
      const int k = idx % kK, m = idx / kK;
      const int t = tt0 + m;
      float cv = 0.f;
      if (t < nvalid && n0 + k < pr.N) cv = to_f(Cm[((b * pr.L + t0 + t) * pr.G + g) * pr.N + n0 + k]);
      As[m * kLdA + k] = cv;
      const int p = pp0 + m;
      float hv = 0.f;
      if (p < pr.P && n0 + k < pr.N) hv = Hc[(int64_t)p * pr.N + n0 + k];
      Bs[k * kLdB + m] = hv;
    }
    __syncthreads();
    mma_tile(acc, As, kLdA, Bs, kLdB, kK, ty, tx);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = tt0 + ty * 4 + i;
    const float sc = (t < nvalid && sqs[t] == seq_prev) ? expf(css[t]) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] *= sc;
  }

  // step 1: masked decay-weighted C B^T applied to x, s-tiles up to the diagonal
  for (int st0 = 0; st0 <= tt0; st0 += kTile) {
    float w[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) w[i][j] = 0.f;
    for (int n0 = 0; n0 < pr.N; n0 += kK) {
      for (int idx = tid; idx < kTile * kK; idx += kThreads) {
        const int k = idx % kK, m = idx / kK;
        const int t = tt0 + m, s = st0 + m;
        float cv = 0.f, bv = 0.f;
        if (t < nvalid && n0 + k < pr.N) cv = to_f(Cm[((b * pr.L + t0 + t) * pr.G + g) * pr.N + n0 + k]);
        if (s < nvalid && n0 + k < pr.N) bv = to_f(Bm[((b * pr.L + t0 + s) * pr.G + g) * pr.N + n0 + k]);
        As[m * kLdA + k] = cv;
        Bs[k * kLdB + m] = bv;
      }
      __syncthreads();
      mma_tile(w, As, kLdA, Bs, kLdB, kK, ty, tx);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tt0 + ty * 4 + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = st0 + tx * 4 + j;
        float v = 0.f;
        if (s <= t && t < nvalid && s < nvalid && sqs[s] == sqs[t])
          v = w[i][j] * expf(css[t] - css[s]) * dts[s];
        Ws[(ty * 4 + i) * kLdW + tx * 4 + j] = v;
      }
    }
    for (int idx = tid; idx < kTile * kTile; idx += kThreads) {
      const int p = idx % kTile, s = idx / kTile;
      float xv = 0.f;
      if (st0 + s < nvalid && pp0 + p < pr.P)
        xv = to_f(x[((b * pr.L + t0 + st0 + s) * pr.H + h) * pr.P + pp0 + p]);
      Xs[s * kLdB + p] = xv;
    }
    __syncthreads();
    mma_tile(acc, Ws, kLdW, Xs, kLdB, kTile, ty, tx);
    __syncthreads();
  }

  const float d = pr.D ? pr.D[h] : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = tt0 + ty * 4 + i;
    if (t >= nvalid) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = pp0 + tx * 4 + j;
      if (p >= pr.P) continue;
      const int64_t off = ((b * pr.L + t0 + t) * pr.H + h) * pr.P + p;
      float v = fmaf(d, to_f(x[off]), acc[i][j]);
      if (pr.z) {  // the gate: y * SiLU(z)
        const float zv = to_f(static_cast<const T*>(pr.z)[off]);
        v *= zv / (1.f + expf(-zv));
      }
      y[off] = from_f<T>(v);
    }
  }
}

// ---------------------------------------------------------------- packed finals
__global__ void k_seq_ends(Problem pr, int64_t* __restrict__ ends) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= pr.b * pr.L) return;
  const int64_t t = i % pr.L;
  const int sid = pr.seq[i];
  if ((t == pr.L - 1 || pr.seq[i + 1] != sid) && sid >= 0 && sid < pr.num_seqs) ends[sid] = i;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_packed_final(Problem pr, const float* __restrict__ cs,
                                                           const float* __restrict__ prev,
                                                           const int64_t* __restrict__ ends) {
  extern __shared__ float smem[];
  const int64_t tp = (pr.P + kTile - 1) / kTile, tn = (pr.N + kTile - 1) / kTile;
  int64_t r = blockIdx.x;
  const int64_t tile = r % (tp * tn);
  r /= (tp * tn);
  const int64_t h = r % pr.H;
  const int64_t sid = r / pr.H;
  const int p0 = (int)(tile / tn) * kTile, n0 = (int)(tile % tn) * kTile;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float* out = pr.final_states + (sid * pr.H + h) * pr.P * pr.N;
  const int64_t end = ends[sid];
  float acc[4][4];
  if (end < 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  } else {
    const int64_t b = end / pr.L, t = end % pr.L;
    const int64_t c = t / pr.Q, t0 = c * pr.Q;
    const int e = (int)(t - t0);
    state_tile<T>(pr, cs, b, c, h, e, p0, n0, acc, smem);
    const bool keep = seq_at(pr, b, t) == seq_at(pr, b, t0 > 0 ? t0 - 1 : 0);
    const float dec = keep ? expf(cs[((b * pr.H + h) * pr.nc + c) * pr.Q + e]) : 0.f;
    const float* Hc = prev + ((b * pr.nc + c) * pr.H + h) * pr.P * pr.N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int p = p0 + ty * 4 + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (p < pr.P && n < pr.N) acc[i][j] = fmaf(dec, Hc[(int64_t)p * pr.N + n], acc[i][j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int p = p0 + ty * 4 + i;
    if (p >= pr.P) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < pr.N) out[(int64_t)p * pr.N + n] = acc[i][j];
    }
  }
}

struct GenericLayout {
  size_t cs, states, ends, total;
};

GenericLayout layout(const Problem& p) {
  GenericLayout l;
  size_t off = 0;
  l.cs = off;
  off = align_up(off + sizeof(float) * (size_t)(p.b * p.H * p.nc * p.Q), kWsAlign);
  l.states = off;
  off = align_up(off + sizeof(float) * (size_t)(p.b * p.nc * p.H * p.P * p.N), kWsAlign);
  l.ends = off;
  if (p.seq && p.final_states) off = align_up(off + sizeof(int64_t) * (size_t)p.num_seqs, kWsAlign);
  l.total = off;
  return l;
}

template <typename T>
cudaError_t run(const Problem& p, char* ws, cudaStream_t st) {
  const GenericLayout l = layout(p);
  float* cs = reinterpret_cast<float*>(ws + l.cs);
  float* states = reinterpret_cast<float*>(ws + l.states);
  const int64_t tp = (p.P + kTile - 1) / kTile, tn = (p.N + kTile - 1) / kTile;
  const int64_t tt = (p.Q + kTile - 1) / kTile;

  k_chunk_cumsum<<<dim3((unsigned)p.nc, (unsigned)p.b), 128, 0, st>>>(p, cs);

  cudaError_t err = cudaFuncSetAttribute(k_chunk_state<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kStateSmem);
  if (err != cudaSuccess) return err;
  k_chunk_state<T><<<dim3((unsigned)(p.nc * p.H * tp * tn), (unsigned)p.b), kThreads, kStateSmem, st>>>(
      p, cs, states);

  const int64_t pn4 = (p.P * p.N + 3) / 4;
  k_state_passing<<<dim3((unsigned)((pn4 + 255) / 256), (unsigned)(p.b * p.H)), 256, 0, st>>>(p, cs, states);

  err = cudaFuncSetAttribute(k_chunk_scan<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScanSmem);
  if (err != cudaSuccess) return err;
  k_chunk_scan<T><<<dim3((unsigned)(p.nc * p.H * tt * tp), (unsigned)p.b), kThreads, kScanSmem, st>>>(
      p, cs, states);

  if (p.seq && p.final_states) {
    int64_t* ends = reinterpret_cast<int64_t*>(ws + l.ends);
    err = cudaMemsetAsync(ends, 0xff, sizeof(int64_t) * (size_t)p.num_seqs, st);
    if (err != cudaSuccess) return err;
    const int64_t ntok = p.b * p.L;
    k_seq_ends<<<(unsigned)((ntok + 255) / 256), 256, 0, st>>>(p, ends);
    err = cudaFuncSetAttribute(k_packed_final<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kStateSmem);
    if (err != cudaSuccess) return err;
    k_packed_final<T><<<(unsigned)(p.num_seqs * p.H * tp * tn), kThreads, kStateSmem, st>>>(p, cs, states,
                                                                                             ends);
  }
  return cudaGetLastError();
}

}  // namespace

size_t generic_workspace_bytes(const Problem& p) { return layout(p).total; }

int generic_launch_count(const Problem& p) { return (p.seq && p.final_states) ? 6 : 4; }

cudaError_t generic_forward(const Problem& p, void* ws, cudaStream_t stream) {
  if (p.dtype == SSD_BF16) return run<__nv_bfloat16>(p, static_cast<char*>(ws), stream);
  return run<float>(p, static_cast<char*>(ws), stream);
}

}  // namespace ssd
