// The SSD backward: kernels and the host-side plan that launches them.
//
// The gradients are the adjoint of the recurrence of "22 · Mamba 2 —
// Transformers are SSMs" section 3.1 (with the D feed-through of "从
// Transformer的二次复杂度困境到Mamba的线性突围", continuous SSM equations,
// and the packed-sequence cut of "Transformers与SSMs的隐藏联系" section 4.2),
// taken in the chunked form of "SSM 家族全景图（下）：Mamba-2 与 Jamba"
// section 三.4 and recomputing the forward's states as the hardware-aware
// algorithm of the first page above does.  Per batch row b, head h (group g)
// and chunk c of Q tokens, with cs_t the in-chunk cumulative sum of dt A
// (restarted at a packed-sequence boundary), E(t,s) = exp(cs_t - cs_s) for
// s <= t in the same packed sequence (else 0), w_s = dt_s, h_in the state
// entering the chunk and Lam = dLoss/d(state leaving the chunk):
//
//   y_t   = sum_s E(t,s) (C_t.B_s) w_s x_s + e_t h_in C_t + D x_t
//   h_out = e_last h_in + sum_s E(last,s) w_s x_s B_s^T
//
// where e_t = exp(cs_t) while no boundary has occurred in the chunk up to t
// (else 0).  Differentiating sum_t dy_t.y_t + <Lam, h_out>:
//
//   dx_s  = w_s [sum_{t>=s} E(t,s) (C_t.B_s) dy_t + E(last,s) Lam B_s] + D dy_s
//   dB_s  = w_s [sum_{t>=s} E(t,s) (dy_t.x_s) C_t + E(last,s) Lam^T x_s]
//   dC_t  = sum_{s<=t} E(t,s) w_s (dy_t.x_s) B_s + e_t h_in^T dy_t
//   dw_s  = sum_{t>=s} E(t,s) (C_t.B_s)(dy_t.x_s) + E(last,s) x_s^T Lam B_s
//   dLam' = e_last Lam + sum_t e_t dy_t C_t^T     (= dLoss/dh_in)
//
// and, for the log-decays l_k = dt_k A (cs_t = sum of l_k over the segment
// up to t), with M(t,s) = E(t,s) w_s (C_t.B_s)(dy_t.x_s) and
// N_s = E(last,s) w_s x_s^T Lam B_s:
//
//   dl_k = sum_{s < k <= t} M(t,s) + sum_{t >= k} e_t dy_t.(h_in C_t)
//          + sum_{s < k} N_s + e_last <Lam, h_in>
//
// (every term whose decay spans token k), ddt_k = dw_k + A dl_k and
// dA = sum_k dt_k dl_k.  A token that starts a segment has no decay term.
// The pair sum is formed directly over the block s < k <= t; written as row
// sums minus column sums, the pairs after k would cancel only to rounding.
// With the block's gate (out = y SiLU(z)), k_bwd_chunk first recomputes the
// chunk's y from the same K and h_in, writes dz = dout y SiLU'(z), and all of
// the above then runs on dy = dout SiLU(z).
//
// Six kernels, in stream order:
//   k_bwd_chunk_states   per (b, c, h): the chunk's end state from a zero
//                        state, its adjoint input sum_t e_t dy_t C_t^T, and
//                        its decay e_last
//   k_bwd_state_passing  per state entry: h_in of every chunk (forward) and
//                        Lam of every chunk (backward), dinitial_states
//   k_bwd_chunk_cb       per (b, c, g): C_t.B_s of the chunk, which the
//                        group's heads share
//   k_bwd_chunk          per (b, c, h): the formulas above from the chunk's
//                        tokens, h_in and Lam; dB and dC per head
//   k_bwd_group_sum      dB, dC summed over each group's heads
//   k_bwd_param_sum      dA, dD summed over rows and chunks (fp64, one CTA
//                        a head, a fixed-order tree)
//   (k_bwd_chunk_states and k_bwd_state_passing give way to
//   k_bwd_state_walk_tc, k_bwd_chunk_cb and k_bwd_chunk to k_bwd_chunk_tc, of
//   ssd_bwd_tc.cuh: the same formulas on the tensor cores, where those take
//   the call)
//
// With SSD_BWD_DINITIAL_ONLY only the first two run.
//
// All fp32 on the CUDA cores; every loop is bounded by the chunk's own token
// count, and nothing waits on another CTA.  The kernels use only standard
// CUDA built-ins so that the same source also runs, for tests only, under a
// host emulation of a CTA's threads; dynamic shared memory is declared
// through SSD_DYN_SMEM for that reason.
#ifndef SSD_BWD_CUH_
#define SSD_BWD_CUH_

#include <stddef.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "ssd.h"

#ifndef SSD_DYN_SMEM
#define SSD_DYN_SMEM(name) extern __shared__ __align__(16) float name[]
#endif

namespace ssd {
namespace bwd {

constexpr int kThreads = 256;
constexpr int64_t kMaxChunk = 64;
constexpr int64_t kMaxDim = 256;          // headdim and dstate
constexpr size_t kSmemLimit = 232448;     // dynamic shared memory one CTA may opt into on sm_100

struct Dims {
  int64_t b, L, H, P, N, G, hpg, Q, nc;
};

struct KArgs {
  Dims d;
  const void* x;
  const float* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  const float* h0;
  const int32_t* seq;
  const void* dy;
  const float* dfinal;
  float* dx;
  float* ddt;
  float* dA;
  float* dB;
  float* dC;
  float* dD;
  float* dh0;
  const void* z;    // (b,L,H,P) gate or null
  float* dz;        // (b,L,H,P) with z
  // workspace
  float* S;         // (b,H,nc,P,N): chunk end states from zero, then each chunk's h_in
  float* T;         // (b,H,nc,P,N): each chunk's sum_t e_t dy_t C_t^T, then its Lam
  float* dec;       // (b,H,nc): e_last of each chunk
  float* CB;        // (b,nc,G,Q,Q): C_t.B_s of each chunk, shared by the group's heads
  float* dBh;       // (b,L,H,N): dB per head
  float* dCh;       // (b,L,H,N): dC per head
  double* dA_part;  // (H, b*nc)
  double* dD_part;  // (H, b*nc)
};

__device__ __forceinline__ float ld(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }

// The gate: SiLU(v) = v / (1 + e^-v) and its slope s (1 + v (1 - s)), s = 1 / (1 + e^-v).
__device__ __forceinline__ float gate_silu(float v) { return v / (1.f + expf(-v)); }
__device__ __forceinline__ float gate_slope(float v) {
  const float s = 1.f / (1.f + expf(-v));
  return s * fmaf(v, 1.f - s, 1.f);
}

// Chunk c's coordinates from a CTA index ordered (b, c, h), h fastest.
struct ChunkPos {
  int64_t b, c, h, g, t0;
  int Qc;
};

__device__ __forceinline__ ChunkPos chunk_pos(const Dims& d, int64_t bid) {
  ChunkPos q;
  q.h = bid % d.H;
  q.c = (bid / d.H) % d.nc;
  q.b = bid / (d.H * d.nc);
  q.g = q.h / d.hpg;
  q.t0 = q.c * d.Q;
  const int64_t left = d.L - q.t0;
  q.Qc = (int)(left < d.Q ? left : d.Q);
  return q;
}

// In-chunk cumulative log-decay cs[t] and seg[t], the in-chunk index of the
// first token of t's packed sequence, or -1 while that sequence began before
// the chunk (those tokens see h_in).  A token whose id differs from the
// previous token's starts a sequence: its own decay is not applied (a_t = 0),
// so the sum restarts at 0 there.  Every thread of the block calls it: the
// log-decays and the sequence starts are loaded in parallel into cs and seg,
// then one thread runs the scan over shared memory.  It ends with a barrier.
__device__ __forceinline__ void chunk_cumsum(const KArgs& a, const ChunkPos& q, float* cs, int* seg, int tid) {
  const float Ah = a.A[q.h];
  const int32_t* sq = a.seq ? a.seq + q.b * a.d.L : nullptr;
  for (int t = tid; t < q.Qc; t += kThreads) {
    const int64_t l = q.t0 + t;
    cs[t] = a.dt[(q.b * a.d.L + l) * a.d.H + q.h] * Ah;
    seg[t] = sq && l > 0 && sq[l] != sq[l - 1];  // a sequence starts at t
  }
  __syncthreads();
  if (tid == 0) {
    float acc = 0.f;
    int s0 = -1;
    for (int t = 0; t < q.Qc; ++t) {
      if (seg[t]) {
        s0 = t;
        acc = 0.f;
      } else {
        acc += cs[t];
      }
      cs[t] = acc;
      seg[t] = s0;
    }
  }
  __syncthreads();
}

// ---- register-tiled products of small matrices in shared memory
//
// A thread owns a TM x TN block of an M x Nn product: rows r_i = TM tr + i and
// columns c_j = tc + j TC (TC = ceil(Nn / TN)), with tile = tr TC + tc.  The
// threads of a warp take consecutive tc, so they read consecutive columns of
// one operand and the same few rows of the other (a broadcast); row strides
// are padded where a column walk would otherwise meet one bank.  Contiguous
// rows let a triangular product stop at the thread's own first or last row.
// Indices past the edge are clamped for loads, and their results are never
// stored.  Each block costs TM + TN shared loads per TM TN multiply-adds.
constexpr int kT = 4;   // 4 x 4 blocks by default
constexpr int kTN = 8;  // rows of the 8 x 4 blocks of the Q x dstate and headdim x dstate products

template <int TM, int TN>
struct TileT {
  int tc;               // column-block index (the partial-sum slot of a row)
  int r[TM], c[TN];     // clamped row and column indices
  bool rv[TM], cv[TN];  // inside the product?
};
using Tile = TileT<kT, kT>;

template <int TM = kT, int TN = kT>
__device__ __forceinline__ int tiles_of(int M, int Nn) {
  return ((M + TM - 1) / TM) * ((Nn + TN - 1) / TN);
}

template <int TM = kT, int TN = kT>
__device__ __forceinline__ TileT<TM, TN> make_tile(int tile, int M, int Nn) {
  const int TC = (Nn + TN - 1) / TN;
  const int tr = tile / TC;
  TileT<TM, TN> t;
  t.tc = tile % TC;
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int r = tr * TM + i;
    t.rv[i] = r < M;
    t.r[i] = r < M ? r : M - 1;
  }
#pragma unroll
  for (int j = 0; j < TN; ++j) {
    const int c = t.tc + j * TC;
    t.cv[j] = c < Nn;
    t.c[j] = c < Nn ? c : Nn - 1;
  }
  return t;
}

template <int TM, int TN>
__device__ __forceinline__ void tile_zero(float (&acc)[TM][TN]) {
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// acc[i][j] += sum_{k0 <= k < k1} A(r_i, k) B(k, c_j), with A(m, k) = a[m am + k ak]
// (times ks[k] when kScale) and B(k, n) = b[k bk + n bn].
template <bool kScale, int TM, int TN>
__device__ __forceinline__ void tile_mac(float (&acc)[TM][TN], const TileT<TM, TN>& t, const float* a, int am,
                                         int ak, const float* ks, const float* b, int bk, int bn, int k0, int k1) {
  for (int k = k0; k < k1; ++k) {
    float av[TM], bv[TN];
    const float sk = kScale ? ks[k] : 1.f;
#pragma unroll
    for (int i = 0; i < TM; ++i) av[i] = kScale ? a[t.r[i] * am + k * ak] * sk : a[t.r[i] * am + k * ak];
#pragma unroll
    for (int j = 0; j < TN; ++j) bv[j] = b[k * bk + t.c[j] * bn];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// Shared-memory floats of k_bwd_chunk_cb for chunk length Q.
inline size_t smem_cb_floats(int64_t Q, int64_t N) { return (size_t)(2 * Q * (N + 1)); }

// C_t.B_s (Q x Q, over dstate) of every chunk and group: the heads of a group
// share it.  One CTA per (b, c, g), g fastest.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_chunk_cb(const KArgs a) {
  const Dims& d = a.d;
  const int64_t bid = blockIdx.x;
  const int64_t g = bid % d.G, c = (bid / d.G) % d.nc, b = bid / (d.G * d.nc);
  const int64_t t0 = c * d.Q;
  const int Qc = (int)(d.L - t0 < d.Q ? d.L - t0 : d.Q);
  const int N = (int)d.N, Q = (int)d.Q, sN = N + 1;
  const int tid = threadIdx.x;
  SSD_DYN_SMEM(sm);
  float* Bs = sm;            // Q x sN
  float* Cs = Bs + Q * sN;   // Q x sN
  const T* B = static_cast<const T*>(a.B);
  const T* C = static_cast<const T*>(a.C);
  for (int i = tid; i < Qc * N; i += kThreads) {
    const int t = i / N, n = i % N;
    const int64_t gi = ((b * d.L + t0 + t) * d.G + g) * d.N + n;
    Bs[t * sN + n] = ld(B, gi);
    Cs[t * sN + n] = ld(C, gi);
  }
  __syncthreads();
  float* out = a.CB + ((b * d.nc + c) * d.G + g) * d.Q * d.Q;
  for (int tile = tid; tile < tiles_of(Qc, Qc); tile += kThreads) {
    const Tile tl = make_tile(tile, Qc, Qc);
    float cb[kT][kT];
    tile_zero(cb);
    tile_mac<false>(cb, tl, Cs, sN, 1, nullptr, Bs, 1, sN, 0, N);
#pragma unroll
    for (int i = 0; i < kT; ++i)
#pragma unroll
      for (int j = 0; j < kT; ++j)
        if (tl.rv[i] && tl.cv[j]) out[tl.r[i] * Q + tl.c[j]] = cb[i][j];
  }
}

// Shared-memory floats of k_bwd_chunk_states for chunk length Q.
inline size_t smem_states_floats(int64_t Q, int64_t P, int64_t N) { return (size_t)(2 * Q * P + 2 * Q * N + 4 * Q); }

// Two CTAs per SM (2 x 99 KB of shared memory at headdim 64, dstate 128): at
// most 128 registers a thread.
template <typename T>
__global__ void __launch_bounds__(kThreads, 2) k_bwd_chunk_states(const KArgs a) {
  const Dims& d = a.d;
  const ChunkPos q = chunk_pos(d, blockIdx.x);
  const int P = (int)d.P, N = (int)d.N, Q = (int)d.Q, Qc = q.Qc;
  const int tid = threadIdx.x;
  SSD_DYN_SMEM(sm);
  float* xs = sm;          // Q x P
  float* dys = xs + Q * P;  // Q x P
  float* Bs = dys + Q * P;  // Q x N
  float* Cs = Bs + Q * N;   // Q x N
  float* cs = Cs + Q * N;   // Q
  float* cS = cs + Q;       // Q: weight of x_t B_t^T in the end state
  float* cT = cS + Q;       // Q: weight of dy_t C_t^T in dLoss/dh_in
  int* seg = reinterpret_cast<int*>(cT + Q);

  const T* x = static_cast<const T*>(a.x);
  const T* dy = static_cast<const T*>(a.dy);
  const T* z = static_cast<const T*>(a.z);
  const T* B = static_cast<const T*>(a.B);
  const T* C = static_cast<const T*>(a.C);
  for (int i = tid; i < Qc * P; i += kThreads) {
    const int t = i / P, p = i % P;
    const int64_t gi = ((q.b * d.L + q.t0 + t) * d.H + q.h) * d.P + p;
    xs[i] = ld(x, gi);
    dys[i] = z ? ld(dy, gi) * gate_silu(ld(z, gi)) : ld(dy, gi);  // the gradient reaching y
  }
  for (int i = tid; i < Qc * N; i += kThreads) {
    const int t = i / N, n = i % N;
    const int64_t gi = ((q.b * d.L + q.t0 + t) * d.G + q.g) * d.N + n;
    Bs[i] = ld(B, gi);
    Cs[i] = ld(C, gi);
  }
  chunk_cumsum(a, q, cs, seg, tid);
  for (int t = tid; t < Qc; t += kThreads) {
    const float w = a.dt[(q.b * d.L + q.t0 + t) * d.H + q.h];
    cS[t] = seg[t] == seg[Qc - 1] ? w * expf(cs[Qc - 1] - cs[t]) : 0.f;
    cT[t] = seg[t] == -1 ? expf(cs[t]) : 0.f;
  }
  if (tid == 0) a.dec[(q.b * d.H + q.h) * d.nc + q.c] = seg[Qc - 1] == -1 ? expf(cs[Qc - 1]) : 0.f;
  __syncthreads();
  // S (P x N) = sum_t cS_t x_t B_t^T and T = sum_t cT_t dy_t C_t^T, over the chunk's tokens
  const int64_t off = ((q.b * d.H + q.h) * d.nc + q.c) * d.P * d.N;
  float* So = a.S + off;
  float* To = a.T + off;
  // 8 x 4 blocks: P x N = 8192 outputs at headdim 64, dstate 128 is one block per thread
  constexpr int TM = kTN, TN = kT;
  const int nt = tiles_of<TM, TN>(P, N);
  for (int tile = tid; tile < nt; tile += kThreads) {
    const TileT<TM, TN> tl = make_tile<TM, TN>(tile, P, N);
    float s[TM][TN], u[TM][TN];
    tile_zero(s);
    tile_zero(u);
    tile_mac<true>(s, tl, xs, 1, P, cS, Bs, N, 1, 0, Qc);
    tile_mac<true>(u, tl, dys, 1, P, cT, Cs, N, 1, 0, Qc);
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j)
        if (tl.rv[i] && tl.cv[j]) {
          So[tl.r[i] * N + tl.c[j]] = s[i][j];
          To[tl.r[i] * N + tl.c[j]] = u[i][j];
        }
  }
}

// V consecutive state entries (b, h, p, n..n+V-1) per thread: the forward
// scan turns S into the state entering each chunk, the backward scan turns T
// into the gradient with respect to the state leaving each chunk; what the
// backward scan carries out of chunk 0 is dLoss/dinitial_states.  V = 4 when
// P N is a multiple of 4 (S and T are 256-byte aligned workspace, so each
// chunk's row is then read and written as 16-byte vectors), else 1; h0,
// dfinal and dh0 are the caller's and are accessed one float at a time.
template <int V>
__device__ __forceinline__ void ld_v(const float* p, float (&o)[V]) {
  if constexpr (V == 4) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    o[0] = q.x, o[1] = q.y, o[2] = q.z, o[3] = q.w;
  } else {
#pragma unroll
    for (int k = 0; k < V; ++k) o[k] = p[k];
  }
}
template <int V>
__device__ __forceinline__ void st_v(float* p, const float (&o)[V]) {
  if constexpr (V == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
  } else {
#pragma unroll
    for (int k = 0; k < V; ++k) p[k] = o[k];
  }
}

template <int V>
__global__ void __launch_bounds__(kThreads) k_bwd_state_passing(const KArgs a) {
  const Dims& d = a.d;
  const int64_t PN = d.P * d.N;
  const int64_t i = ((int64_t)blockIdx.x * kThreads + threadIdx.x) * V;  // the thread's first entry
  if (i >= d.b * d.H * PN) return;
  const int64_t bh = i / PN, e = i % PN;
  float* S = a.S + bh * d.nc * PN + e;
  float* T = a.T + bh * d.nc * PN + e;
  const float* dec = a.dec + bh * d.nc;
  // The two scans run side by side, kBatch chunks at a time: a batch of S
  // (walking forward) and one of T (walking back) are loaded before either is
  // overwritten, so that 2 kBatch loads are in flight per thread (the
  // addresses differ, which the compiler cannot see).  The scans are each
  // thread's own, so a batch is a plain reordering of the loads.
  constexpr int kBatch = V == 4 ? 8 : 16;
  float run[V], lam[V];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    run[k] = a.h0 ? a.h0[i + k] : 0.f;
    lam[k] = a.dfinal ? a.dfinal[i + k] : 0.f;
  }
  const int64_t nc = d.nc;
  for (int64_t c = 0; c < nc; c += kBatch) {
    const int n = (int)(nc - c < kBatch ? nc - c : kBatch);
    const int64_t cb = nc - 1 - c;  // the backward scan's chunk for j = 0
    float vs[kBatch][V], vt[kBatch][V];
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (j < n) {
        ld_v<V>(S + (c + j) * PN, vs[j]);
        ld_v<V>(T + (cb - j) * PN, vt[j]);
      }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (j < n) {
        st_v<V>(S + (c + j) * PN, run);
        st_v<V>(T + (cb - j) * PN, lam);
        const float ds = dec[c + j], dl = dec[cb - j];
#pragma unroll
        for (int k = 0; k < V; ++k) {
          run[k] = fmaf(ds, run[k], vs[j][k]);
          lam[k] = fmaf(dl, lam[k], vt[j][k]);
        }
      }
  }
  if (a.dh0)
#pragma unroll
    for (int k = 0; k < V; ++k) a.dh0[i + k] = lam[k];
}

// Columns of k_bwd_chunk's partial-sum array: one per column block of a
// Q x P or Q x N product, and at least 8 (four row and four column quarters).
__host__ __device__ inline int64_t part_cols(int64_t P, int64_t N) {
  const int64_t m = ((P > N ? P : N) + kT - 1) / kT;
  return m > 8 ? m : 8;
}

// Shared-memory floats of k_bwd_chunk for chunk length Q (rows padded by one
// float so that column walks do not collide in a bank).
inline size_t smem_chunk_floats(int64_t Q, int64_t P, int64_t N) {
  return (size_t)(2 * Q * (P + 1) + 2 * Q * (N + 1) + P * (N + 1) + 3 * Q * (Q + 1) + Q * part_cols(P, N) +
                  10 * Q + kThreads);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_chunk(const KArgs a) {
  const Dims& d = a.d;
  const ChunkPos q = chunk_pos(d, blockIdx.x);
  const int P = (int)d.P, N = (int)d.N, Q = (int)d.Q, Qc = q.Qc;
  const int sP = P + 1, sN = N + 1, sQ = Q + 1, PC = (int)part_cols(d.P, d.N);
  const int tid = threadIdx.x;
  SSD_DYN_SMEM(sm);
  float* xs = sm;             // Q x sP: x_t
  float* dys = xs + Q * sP;   // Q x sP: dy_t (with a gate: first dout_t, then dout_t SiLU(z_t))
  float* Bs = dys + Q * sP;   // Q x sN
  float* Cs = Bs + Q * sN;    // Q x sN
  float* SB = Cs + Q * sN;    // P x sN: h_in, then Lam
  float* Km = SB + P * sN;    // Q x sQ: E(t,s) C_t.B_s
  float* Zm = Km + Q * sQ;    // Q x sQ: E(t,s) dy_t.x_s
  float* Mm = Zm + Q * sQ;    // Q x sQ: E(t,s) (C_t.B_s)(dy_t.x_s)
  float* part = Mm + Q * sQ;  // Q x PC: partial sums per row
  float* cs = part + Q * PC;  // Q
  float* w = cs + Q;          // Q: dt
  float* el = w + Q;          // Q: E(last, s)
  float* ein = el + Q;        // Q: e_t
  float* dg = ein + Q;        // Q: dy_t.x_t
  float* nv = dg + Q;         // Q: x_s^T Lam B_s
  float* dw = nv + Q;         // Q
  float* dcs = dw + Q;        // Q
  float* nn = dcs + Q;        // Q: N_s
  float* red = nn + Q;        // kThreads
  int* seg = reinterpret_cast<int*>(red + kThreads);  // Q

  const T* x = static_cast<const T*>(a.x);
  const T* dy = static_cast<const T*>(a.dy);
  const T* z = static_cast<const T*>(a.z);
  const T* B = static_cast<const T*>(a.B);
  const T* C = static_cast<const T*>(a.C);
  const int64_t soff = ((q.b * d.H + q.h) * d.nc + q.c) * d.P * d.N;
  const float* Hin = a.S + soff;  // P x N
  const float* Lam = a.T + soff;  // P x N
  const float Dh = a.D ? a.D[q.h] : 0.f;

  for (int i = tid; i < Qc * P; i += kThreads) {
    const int t = i / P, p = i % P;
    const int64_t gi = ((q.b * d.L + q.t0 + t) * d.H + q.h) * d.P + p;
    xs[t * sP + p] = ld(x, gi);
    dys[t * sP + p] = ld(dy, gi);
  }
  for (int i = tid; i < Qc * N; i += kThreads) {
    const int t = i / N, n = i % N;
    const int64_t gi = ((q.b * d.L + q.t0 + t) * d.G + q.g) * d.N + n;
    Bs[t * sN + n] = ld(B, gi);
    Cs[t * sN + n] = ld(C, gi);
  }
  {
    float part_lh = 0.f;  // <Lam, h_in>, this thread's share
    for (int e = tid; e < P * N; e += kThreads) {
      const float h = Hin[e];
      SB[(e / N) * sN + e % N] = h;
      part_lh = fmaf(Lam[e], h, part_lh);
    }
    red[tid] = part_lh;
  }
  for (int t = tid; t < Qc; t += kThreads) w[t] = a.dt[(q.b * d.L + q.t0 + t) * d.H + q.h];
  chunk_cumsum(a, q, cs, seg, tid);
  // <Lam, h_in>: the threads' shares summed pairwise (red[0] holds it)
  for (int off = kThreads / 2; off > 0; off >>= 1) {
    if (tid < off) red[tid] += red[tid + off];
    __syncthreads();
  }

  const int last = Qc - 1;
  // K = E o (C B^T) on the chunk's Q x Q triangle (C B^T from k_bwd_chunk_cb, once
  // per group), and the decays to the chunk's ends
  {
    const float* cb = a.CB + ((q.b * d.nc + q.c) * d.G + q.g) * d.Q * d.Q;
    for (int i = tid; i < Qc * Qc; i += kThreads) {
      const int t = i / Qc, s = i % Qc;
      const float e = (s <= t && seg[s] == seg[t]) ? expf(cs[t] - cs[s]) : 0.f;
      Km[t * sQ + s] = s <= t ? e * cb[t * Q + s] : 0.f;
    }
  }
  for (int t = tid; t < Qc; t += kThreads) {
    el[t] = seg[t] == seg[last] ? expf(cs[last] - cs[t]) : 0.f;
    ein[t] = seg[t] == -1 ? expf(cs[t]) : 0.f;
  }
  __syncthreads();

  if (z) {
    // the gate: recompute y_t = sum_s K(t,s) dt_s x_s + e_t h_in C_t + D x_t, write
    // dz = dout y SiLU'(z), and carry on with dy = dout SiLU(z)
    for (int tile = tid; tile < tiles_of(Qc, P); tile += kThreads) {
      const Tile tl = make_tile(tile, Qc, P);
      int kmax = 0;
#pragma unroll
      for (int i = 0; i < kT; ++i)
        if (tl.rv[i]) kmax = tl.r[i] + 1;
      float yi[kT][kT], yh[kT][kT];
      tile_zero(yi);
      tile_zero(yh);
      tile_mac<true>(yi, tl, Km, sQ, 1, w, xs, sP, 1, 0, kmax);
      tile_mac<false>(yh, tl, Cs, sN, 1, nullptr, SB, 1, sN, 0, N);
#pragma unroll
      for (int i = 0; i < kT; ++i)
#pragma unroll
        for (int j = 0; j < kT; ++j) {
          if (!tl.rv[i] || !tl.cv[j]) continue;
          const int t = tl.r[i], p = tl.c[j];
          const int64_t gi = ((q.b * d.L + q.t0 + t) * d.H + q.h) * d.P + p;
          const float y = fmaf(ein[t], yh[i][j], fmaf(Dh, xs[t * sP + p], yi[i][j]));
          const float zz = ld(z, gi), dout = dys[t * sP + p];
          a.dz[gi] = dout * y * gate_slope(zz);
          dys[t * sP + p] = dout * gate_silu(zz);
        }
    }
    __syncthreads();
  }

  // Z = E o (dy x^T) and M = K o (dy x^T); the diagonal dy_t.x_t
  for (int tile = tid; tile < tiles_of(Qc, Qc); tile += kThreads) {
    const Tile tl = make_tile(tile, Qc, Qc);
    float xy[kT][kT];
    tile_zero(xy);
    tile_mac<false>(xy, tl, dys, sP, 1, nullptr, xs, 1, sP, 0, P);
#pragma unroll
    for (int i = 0; i < kT; ++i)
#pragma unroll
      for (int j = 0; j < kT; ++j) {
        if (!tl.rv[i] || !tl.cv[j]) continue;
        const int t = tl.r[i], s = tl.c[j];
        const float e = (s <= t && seg[s] == seg[t]) ? expf(cs[t] - cs[s]) : 0.f;
        Zm[t * sQ + s] = e * xy[i][j];
        Mm[t * sQ + s] = Km[t * sQ + s] * xy[i][j];
        if (s == t) dg[t] = xy[i][j];
      }
  }
  __syncthreads();

  // dC of this head (Q x N, 8 x 4 blocks: one per thread at Q 64, dstate 128):
  // sum_s Z(t,s) w_s B_s + e_t h_in^T dy_t; with the row partials of C_t . (h_in^T dy_t)
  for (int tile = tid; tile < tiles_of<kTN, kT>(Qc, N); tile += kThreads) {
    const TileT<kTN, kT> tl = make_tile<kTN, kT>(tile, Qc, N);
    int kmax = 0;
#pragma unroll
    for (int i = 0; i < kTN; ++i)
      if (tl.rv[i]) kmax = tl.r[i] + 1;
    float ci[kTN][kT], ch[kTN][kT];
    tile_zero(ci);
    tile_zero(ch);
    tile_mac<true>(ci, tl, Zm, sQ, 1, w, Bs, sN, 1, 0, kmax);
    tile_mac<false>(ch, tl, dys, sP, 1, nullptr, SB, sN, 1, 0, P);
#pragma unroll
    for (int i = 0; i < kTN; ++i) {
      if (!tl.rv[i]) continue;
      const int t = tl.r[i];
      float cy = 0.f;
#pragma unroll
      for (int j = 0; j < kT; ++j) {
        if (!tl.cv[j]) continue;
        const int n = tl.c[j];
        a.dCh[((q.b * d.L + q.t0 + t) * d.H + q.h) * d.N + n] = fmaf(ein[t], ch[i][j], ci[i][j]);
        cy = fmaf(Cs[t * sN + n], ch[i][j], cy);
      }
      part[t * PC + tl.tc] = cy;
    }
  }
  __syncthreads();

  // the h_in term of dcs (kept in dcs for now); Lam replaces h_in
  const int tcn = (N + kT - 1) / kT;
  for (int t = tid; t < Qc; t += kThreads) {
    float v = 0.f;
    for (int k = 0; k < tcn; ++k) v += part[t * PC + k];
    dcs[t] = ein[t] * v;
  }
  for (int e = tid; e < P * N; e += kThreads) SB[(e / N) * sN + e % N] = Lam[e];
  __syncthreads();

  // dx (Q x P): w_s [sum_t K(t,s) dy_t + E(last,s) Lam B_s] + D dy_s; with the
  // row partials of x_s . (Lam B_s)
  for (int tile = tid; tile < tiles_of(Qc, P); tile += kThreads) {
    const Tile tl = make_tile(tile, Qc, P);
    float acc[kT][kT], lb[kT][kT];
    tile_zero(acc);
    tile_zero(lb);
    tile_mac<false>(acc, tl, Km, 1, sQ, nullptr, dys, sP, 1, tl.r[0], Qc);
    tile_mac<false>(lb, tl, Bs, sN, 1, nullptr, SB, 1, sN, 0, N);
#pragma unroll
    for (int i = 0; i < kT; ++i) {
      if (!tl.rv[i]) continue;
      const int s = tl.r[i];
      float nx = 0.f;
#pragma unroll
      for (int j = 0; j < kT; ++j) {
        if (!tl.cv[j]) continue;
        const int p = tl.c[j];
        a.dx[((q.b * d.L + q.t0 + s) * d.H + q.h) * d.P + p] =
            fmaf(w[s], fmaf(el[s], lb[i][j], acc[i][j]), Dh * dys[s * sP + p]);
        nx = fmaf(xs[s * sP + p], lb[i][j], nx);
      }
      part[s * PC + tl.tc] = nx;
    }
  }
  // dB of this head (Q x N, 8 x 4 blocks): w_s [sum_t Z(t,s) C_t + E(last,s) Lam^T x_s]
  for (int tile = tid; tile < tiles_of<kTN, kT>(Qc, N); tile += kThreads) {
    const TileT<kTN, kT> tl = make_tile<kTN, kT>(tile, Qc, N);
    float bi[kTN][kT], bl[kTN][kT];
    tile_zero(bi);
    tile_zero(bl);
    tile_mac<false>(bi, tl, Zm, 1, sQ, nullptr, Cs, sN, 1, tl.r[0], Qc);
    tile_mac<false>(bl, tl, xs, sP, 1, nullptr, SB, sN, 1, 0, P);
#pragma unroll
    for (int i = 0; i < kTN; ++i)
#pragma unroll
      for (int j = 0; j < kT; ++j)
        if (tl.rv[i] && tl.cv[j]) {
          const int s = tl.r[i];
          a.dBh[((q.b * d.L + q.t0 + s) * d.H + q.h) * d.N + tl.c[j]] = w[s] * fmaf(el[s], bl[i][j], bi[i][j]);
        }
  }
  __syncthreads();

  const int tcp = (P + kT - 1) / kT;
  for (int s = tid; s < Qc; s += kThreads) {
    float v = 0.f;
    for (int k = 0; k < tcp; ++k) v += part[s * PC + k];
    nv[s] = v;
  }
  __syncthreads();

  // per token k, four threads each: a quarter of the column sum of M below the
  // diagonal (for dw) and of the block sum S_k = sum_{u >= k, s < k} M(u,s) w_s,
  // the pairs whose decay spans k
  for (int i = tid; i < 4 * Qc; i += kThreads) {
    const int k = i >> 2, qq = i & 3;
    const int lo = k + (Qc - k) * qq / 4, hi = k + (Qc - k) * (qq + 1) / 4;
    float col = 0.f, blk = 0.f;
    for (int u = lo; u < hi; ++u) {
      if (u > k) col += Mm[u * sQ + k];
      for (int s2 = 0; s2 < k; ++s2) blk = fmaf(Mm[u * sQ + s2], w[s2], blk);
    }
    part[k * PC + qq] = col;
    part[k * PC + 4 + qq] = blk;
  }
  __syncthreads();
  for (int t = tid; t < Qc; t += kThreads) {
    const float col = part[t * PC] + part[t * PC + 1] + part[t * PC + 2] + part[t * PC + 3];
    const float blk = part[t * PC + 4] + part[t * PC + 5] + part[t * PC + 6] + part[t * PC + 7];
    dw[t] = fmaf(el[t], nv[t], col + Mm[t * sQ + t]);
    nn[t] = el[t] * w[t] * nv[t];
    part[t * PC] = blk;  // S_t
  }
  __syncthreads();

  if (tid == 0) {
    // dl_k = S_k + sum_{t >= k} (h_in term)_t + sum_{s < k} N_s + e_last <Lam, h_in>;
    // the h_in terms live in the first sequence only and N in the last, so
    // none of the sums crosses a boundary that matters
    const float lh = red[0];
    const float e_last = seg[last] == -1 ? expf(cs[last]) : 0.f;
    float before = 0.f;  // sum_{s < k} N_s, kept in nn as an exclusive prefix
    for (int k = 0; k <= last; ++k) {
      const float v = nn[k];
      nn[k] = before;
      before += v;
    }
    const float Ah = a.A[q.h];
    double dA = 0.0, dD = 0.0;
    float after = 0.f;  // sum_{t >= k} of the h_in term (kept in dcs)
    for (int k = last; k >= 0; --k) {
      after += dcs[k];
      const float dl = seg[k] == k ? 0.f : part[k * PC] + after + nn[k] + e_last * lh;  // none at a sequence start
      a.ddt[(q.b * d.L + q.t0 + k) * d.H + q.h] = fmaf(Ah, dl, dw[k]);
      dA += (double)w[k] * (double)dl;
      dD += (double)dg[k];
    }
    const int64_t pi = q.h * (d.b * d.nc) + q.b * d.nc + q.c;
    a.dA_part[pi] = dA;
    a.dD_part[pi] = dD;
  }
}

// dB, dC (b,L,G,N): the per-head gradients summed over each group's heads.
// V consecutive states n..n+V-1 per thread: 16-byte loads and stores when
// V = 4 (N a multiple of 4, dB and dC 16-byte aligned; dBh, dCh are 256-byte
// aligned workspace), the heads of the group added in order.
template <int V>
__global__ void __launch_bounds__(kThreads) k_bwd_group_sum(const KArgs a) {
  const Dims& d = a.d;
  const int64_t i = ((int64_t)blockIdx.x * kThreads + threadIdx.x) * V;  // the thread's first output
  if (i >= d.b * d.L * d.G * d.N) return;
  const int64_t n = i % d.N, r = i / d.N;
  const int64_t g = r % d.G, bl = r / d.G;
  const float* pb = a.dBh + (bl * d.H + g * d.hpg) * d.N + n;
  const float* pc = a.dCh + (bl * d.H + g * d.hpg) * d.N + n;
  float sb[V], sc[V];
#pragma unroll
  for (int k = 0; k < V; ++k) sb[k] = sc[k] = 0.f;
#pragma unroll 4
  for (int64_t j = 0; j < d.hpg; ++j) {
    float vb[V], vc[V];
    ld_v<V>(pb + j * d.N, vb);
    ld_v<V>(pc + j * d.N, vc);
#pragma unroll
    for (int k = 0; k < V; ++k) sb[k] += vb[k], sc[k] += vc[k];
  }
  st_v<V>(a.dB + i, sb);
  st_v<V>(a.dC + i, sc);
}

// dA, dD (H): the per-chunk partial sums added in fp64, in a fixed order.
// One CTA per head: each thread sums a fixed stride of the head's per-chunk
// partials in fp64, then a tree over the threads in a fixed order (2 kThreads
// doubles of dynamic shared memory), so the result does not vary run to run.
__global__ void __launch_bounds__(kThreads) k_bwd_param_sum(const KArgs a) {
  const Dims& d = a.d;
  const int64_t h = blockIdx.x;
  const int tid = threadIdx.x;
  SSD_DYN_SMEM(sm);
  double* ra = reinterpret_cast<double*>(sm);
  double* rd = ra + kThreads;
  const int64_t n = d.b * d.nc;
  double sa = 0.0, sd = 0.0;
  for (int64_t i = tid; i < n; i += kThreads) {
    sa += a.dA_part[h * n + i];
    sd += a.dD_part[h * n + i];
  }
  ra[tid] = sa;
  rd[tid] = sd;
  __syncthreads();
  for (int off = kThreads / 2; off > 0; off >>= 1) {
    if (tid < off) {
      ra[tid] += ra[tid + off];
      rd[tid] += rd[tid + off];
    }
    __syncthreads();
  }
  if (tid == 0) {
    a.dA[h] = (float)ra[0];
    if (a.dD) a.dD[h] = (float)rd[0];
  }
}

// ---------------------------------------------------------------- host side

struct Plan {
  Dims d;
  size_t smem_states, smem_chunk;  // bytes
  size_t smem_cb;                  // bytes
  size_t off_S, off_T, off_dec, off_CB, off_dBh, off_dCh, off_dA, off_dD, total;
};

inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Sizes, chunk length and workspace layout; reads no pointer.
inline ssd_status plan(const ssd_bwd_args* a, Plan* pl) {
  if (!a) return SSD_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->seqlen <= 0 || a->nheads <= 0 || a->headdim <= 0 || a->dstate <= 0 ||
      a->ngroups <= 0 || a->nheads % a->ngroups != 0)
    return SSD_ERR_INVALID_ARG;
  if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (a->chunk_size < 0) return SSD_ERR_INVALID_ARG;
  if (a->headdim > kMaxDim || a->dstate > kMaxDim || a->chunk_size > kMaxChunk) return SSD_ERR_UNSUPPORTED;
  Dims& d = pl->d;
  d.b = a->batch;
  d.L = a->seqlen;
  d.H = a->nheads;
  d.P = a->headdim;
  d.N = a->dstate;
  d.G = a->ngroups;
  d.hpg = d.H / d.G;
  int64_t Q = a->chunk_size;
  if (Q == 0) {
    Q = kMaxChunk;
    while (Q > 8 && smem_chunk_floats(Q, d.P, d.N) * 4 > kSmemLimit) Q /= 2;
  }
  if (smem_chunk_floats(Q, d.P, d.N) * 4 > kSmemLimit) return SSD_ERR_UNSUPPORTED;
  d.Q = Q;
  d.nc = (d.L + Q - 1) / Q;
  // grid sizes must fit gridDim.x
  const double chunk_ctas = (double)d.b * (double)d.nc * (double)d.H;
  const double state_ctas = (double)d.b * (double)d.H * (double)d.P * (double)d.N / kThreads;
  const double group_ctas = (double)d.b * (double)d.L * (double)d.G * (double)d.N / kThreads;
  if (chunk_ctas >= 2147483647.0 || state_ctas >= 2147483647.0 || group_ctas >= 2147483647.0)
    return SSD_ERR_UNSUPPORTED;
  pl->smem_states = smem_states_floats(Q, d.P, d.N) * 4;
  pl->smem_cb = smem_cb_floats(Q, d.N) * 4;
  pl->smem_chunk = smem_chunk_floats(Q, d.P, d.N) * 4;
  const size_t states = (size_t)(d.b * d.H * d.nc) * (size_t)(d.P * d.N) * 4;
  const size_t per_head = (size_t)(d.b * d.L * d.H) * (size_t)d.N * 4;
  const size_t parts = (size_t)(d.H * d.b * d.nc) * 8;
  size_t o = 0;
  pl->off_S = o;
  o = align256(o + states);
  pl->off_T = o;
  o = align256(o + states);
  pl->off_dec = o;
  o = align256(o + (size_t)(d.b * d.H * d.nc) * 4);
  pl->off_CB = o;
  o = align256(o + (size_t)(d.b * d.nc * d.G) * (size_t)(d.Q * d.Q) * 4);
  pl->off_dBh = o;
  o = align256(o + per_head);
  pl->off_dCh = o;
  o = align256(o + per_head);
  pl->off_dA = o;
  o = align256(o + parts);
  pl->off_dD = o;
  o = align256(o + parts);
  pl->total = o;
  return SSD_OK;
}

// Arguments and workspace for one call; the workspace is required.
inline ssd_status check_call(const ssd_bwd_args* a, const Plan& pl) {
  if (a->flags & ~SSD_BWD_DINITIAL_ONLY) return SSD_ERR_INVALID_ARG;
  const bool only_dh0 = (a->flags & SSD_BWD_DINITIAL_ONLY) != 0;
  if (!a->x || !a->dt || !a->A || !a->B || !a->C || !a->dy) return SSD_ERR_INVALID_ARG;
  if (only_dh0 ? !a->dinitial_states : (!a->dx || !a->ddt || !a->dA || !a->dB || !a->dC)) return SSD_ERR_INVALID_ARG;
  if (a->seq_idx && a->dfinal_states) return SSD_ERR_UNSUPPORTED;
  if (!a->workspace || a->workspace_bytes < pl.total) return SSD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) % 256 != 0) return SSD_ERR_INVALID_ARG;
  if ((a->timing_events[0] == nullptr) != (a->timing_events[1] == nullptr)) return SSD_ERR_INVALID_ARG;
  if (!only_dh0 && (a->z == nullptr) != (a->dz == nullptr)) return SSD_ERR_INVALID_ARG;
  if (a->dz && !a->z) return SSD_ERR_INVALID_ARG;
  return SSD_OK;
}

inline KArgs make_kargs(const ssd_bwd_args* a, const Plan& pl) {
  KArgs k;
  k.d = pl.d;
  k.x = a->x;
  k.dt = a->dt;
  k.A = a->A;
  k.B = a->B;
  k.C = a->C;
  k.D = a->D;
  k.h0 = a->initial_states;
  k.seq = a->seq_idx;
  k.dy = a->dy;
  k.dfinal = a->dfinal_states;
  k.dx = a->dx;
  k.ddt = a->ddt;
  k.dA = a->dA;
  k.dB = a->dB;
  k.dC = a->dC;
  k.dD = a->dD;
  k.dh0 = a->dinitial_states;
  k.z = a->z;
  k.dz = a->dz;
  char* ws = static_cast<char*>(a->workspace);
  k.S = reinterpret_cast<float*>(ws + pl.off_S);
  k.T = reinterpret_cast<float*>(ws + pl.off_T);
  k.dec = reinterpret_cast<float*>(ws + pl.off_dec);
  k.CB = reinterpret_cast<float*>(ws + pl.off_CB);
  k.dBh = reinterpret_cast<float*>(ws + pl.off_dBh);
  k.dCh = reinterpret_cast<float*>(ws + pl.off_dCh);
  k.dA_part = reinterpret_cast<double*>(ws + pl.off_dA);
  k.dD_part = reinterpret_cast<double*>(ws + pl.off_dD);
  return k;
}

inline unsigned blocks_for(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

// A launcher may offer the tensor-core kernels (ssd_bwd_tc.cuh, GPU builds):
// chunk_tc_ok(k) says whether they take the call, state_walk_tc(k, only_dh0)
// runs the chunk states and their scans in place of k_bwd_chunk_states and
// k_bwd_state_passing, and chunk_tc(k) runs in place of k_bwd_chunk.
// The host emulation of the kernels offers none and runs the CUDA-core ones.
template <class L, class = void>
struct has_chunk_tc : std::false_type {};
template <class L>
struct has_chunk_tc<L, std::void_t<decltype(std::declval<L&>().chunk_tc(std::declval<const KArgs&>()))>>
    : std::true_type {};

// Validate, then enqueue the six kernels through `launch(kernel, grid,
// shared bytes, args)`, which returns false when a launch fails;
// `launch.record(event)` records a caller's timing event (false on failure).
template <typename T, class Launch>
ssd_status enqueue_typed(const KArgs& k, const Plan& pl, void* const events[2], bool only_dh0, Launch& launch) {
  const Dims& d = pl.d;
  const unsigned chunk_ctas = (unsigned)(d.b * d.nc * d.H);
  bool tensor_cores = false;
  if constexpr (has_chunk_tc<Launch>::value && std::is_same<T, __nv_bfloat16>::value) tensor_cores = launch.chunk_tc_ok(k);
  if (tensor_cores) {  // the chunk states and their scans in one pass
    if constexpr (has_chunk_tc<Launch>::value)
      if (!launch.state_walk_tc(k, only_dh0)) return SSD_ERR_CUDA;
  } else {
    if (!launch(&k_bwd_chunk_states<T>, chunk_ctas, pl.smem_states, k)) return SSD_ERR_CUDA;
    const int64_t n_states = d.b * d.H * d.P * d.N;
    if (!((d.P * d.N) % 4 == 0 ? launch(&k_bwd_state_passing<4>, blocks_for(n_states / 4), (size_t)0, k)
                                : launch(&k_bwd_state_passing<1>, blocks_for(n_states), (size_t)0, k)))
      return SSD_ERR_CUDA;
  }
  if (only_dh0) {  // k_bwd_chunk is not run: its timing events mark the same point
    if (events[0] && !(launch.record(events[0]) && launch.record(events[1]))) return SSD_ERR_CUDA;
    return SSD_OK;
  }
  if (tensor_cores) {  // C B^T is formed inside the kernel
    if (events[0] && !launch.record(events[0])) return SSD_ERR_CUDA;
    if constexpr (has_chunk_tc<Launch>::value)
      if (!launch.chunk_tc(k)) return SSD_ERR_CUDA;
    if (events[1] && !launch.record(events[1])) return SSD_ERR_CUDA;
  } else {
    if (!launch(&k_bwd_chunk_cb<T>, (unsigned)(d.b * d.nc * d.G), pl.smem_cb, k)) return SSD_ERR_CUDA;
    if (events[0] && !launch.record(events[0])) return SSD_ERR_CUDA;
    if (!launch(&k_bwd_chunk<T>, chunk_ctas, pl.smem_chunk, k)) return SSD_ERR_CUDA;
    if (events[1] && !launch.record(events[1])) return SSD_ERR_CUDA;
  }
  // 16-byte vectors when N allows them and the caller's dB, dC are 16-byte aligned
  const int64_t n_bc = d.b * d.L * d.G * d.N;
  const bool vec = d.N % 4 == 0 && (reinterpret_cast<uintptr_t>(k.dB) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(k.dC) & 15) == 0;
  if (!(vec ? launch(&k_bwd_group_sum<4>, blocks_for(n_bc / 4), (size_t)0, k)
            : launch(&k_bwd_group_sum<1>, blocks_for(n_bc), (size_t)0, k)))
    return SSD_ERR_CUDA;
  if (!launch(&k_bwd_param_sum, (unsigned)d.H, (size_t)(2 * kThreads * sizeof(double)), k)) return SSD_ERR_CUDA;
  return SSD_OK;
}

template <class Launch>
ssd_status run(const ssd_bwd_args* a, Launch& launch) {
  Plan pl;
  ssd_status st = plan(a, &pl);
  if (st != SSD_OK) return st;
  st = check_call(a, pl);
  if (st != SSD_OK) return st;
  const KArgs k = make_kargs(a, pl);
  const bool only_dh0 = (a->flags & SSD_BWD_DINITIAL_ONLY) != 0;
  return a->dtype == SSD_BF16 ? enqueue_typed<__nv_bfloat16>(k, pl, a->timing_events, only_dh0, launch)
                               : enqueue_typed<float>(k, pl, a->timing_events, only_dh0, launch);
}

}  // namespace bwd
}  // namespace ssd

#endif  // SSD_BWD_CUH_
