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
// up to t), dcs_t = sum_{s<t} M(t,s) - sum_{u>t} M(u,t) + e_t dy_t.(h_in C_t)
// - N_t (+ e_last <Lam,h_in> + sum_s N_s at the last token), with
// M(t,s) = E(t,s) w_s (C_t.B_s)(dy_t.x_s) and N_s = E(last,s) w_s x_s^T Lam B_s;
// dl_k = sum of dcs_t over t >= k in k's segment, ddt_k = dw_k + A dl_k and
// dA = sum_k dt_k dl_k.  A token that starts a segment has no decay term.
//
// Five kernels, in stream order:
//   k_bwd_chunk_states   per (b, c, h): the chunk's end state from a zero
//                        state, its adjoint input sum_t e_t dy_t C_t^T, and
//                        its decay e_last
//   k_bwd_state_passing  per state entry: h_in of every chunk (forward) and
//                        Lam of every chunk (backward), dinitial_states
//   k_bwd_chunk          per (b, c, h): the formulas above from the chunk's
//                        tokens, h_in and Lam; dB and dC per head
//   k_bwd_group_sum      dB, dC summed over each group's heads
//   k_bwd_param_sum      dA, dD summed over rows and chunks (fp64)
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
  // workspace
  float* S;         // (b,H,nc,P,N): chunk end states from zero, then each chunk's h_in
  float* T;         // (b,H,nc,P,N): each chunk's sum_t e_t dy_t C_t^T, then its Lam
  float* dec;       // (b,H,nc): e_last of each chunk
  float* dBh;       // (b,L,H,N): dB per head
  float* dCh;       // (b,L,H,N): dC per head
  double* dA_part;  // (H, b*nc)
  double* dD_part;  // (H, b*nc)
};

__device__ __forceinline__ float ld(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }

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
// so the sum restarts at 0 there.  One thread runs this.
__device__ __forceinline__ void chunk_cumsum(const KArgs& a, const ChunkPos& q, float* cs, int* seg) {
  const float Ah = a.A[q.h];
  const int32_t* sq = a.seq ? a.seq + q.b * a.d.L : nullptr;
  float acc = 0.f;
  int s0 = -1;
  for (int t = 0; t < q.Qc; ++t) {
    const int64_t l = q.t0 + t;
    if (sq && l > 0 && sq[l] != sq[l - 1]) {
      s0 = t;
      acc = 0.f;
    } else {
      acc += a.dt[(q.b * a.d.L + l) * a.d.H + q.h] * Ah;
    }
    cs[t] = acc;
    seg[t] = s0;
  }
}

// Shared-memory floats of k_bwd_chunk_states for chunk length Q.
inline size_t smem_states_floats(int64_t Q, int64_t P, int64_t N) { return (size_t)(2 * Q * P + 2 * Q * N + 4 * Q); }

template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_chunk_states(const KArgs a) {
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
  const T* B = static_cast<const T*>(a.B);
  const T* C = static_cast<const T*>(a.C);
  for (int i = tid; i < Qc * P; i += kThreads) {
    const int t = i / P, p = i % P;
    const int64_t gi = ((q.b * d.L + q.t0 + t) * d.H + q.h) * d.P + p;
    xs[i] = ld(x, gi);
    dys[i] = ld(dy, gi);
  }
  for (int i = tid; i < Qc * N; i += kThreads) {
    const int t = i / N, n = i % N;
    const int64_t gi = ((q.b * d.L + q.t0 + t) * d.G + q.g) * d.N + n;
    Bs[i] = ld(B, gi);
    Cs[i] = ld(C, gi);
  }
  if (tid == 0) chunk_cumsum(a, q, cs, seg);
  __syncthreads();
  for (int t = tid; t < Qc; t += kThreads) {
    const float w = a.dt[(q.b * d.L + q.t0 + t) * d.H + q.h];
    cS[t] = seg[t] == seg[Qc - 1] ? w * expf(cs[Qc - 1] - cs[t]) : 0.f;
    cT[t] = seg[t] == -1 ? expf(cs[t]) : 0.f;
  }
  if (tid == 0) a.dec[(q.b * d.H + q.h) * d.nc + q.c] = seg[Qc - 1] == -1 ? expf(cs[Qc - 1]) : 0.f;
  __syncthreads();
  const int64_t off = ((q.b * d.H + q.h) * d.nc + q.c) * d.P * d.N;
  float* So = a.S + off;
  float* To = a.T + off;
  for (int e = tid; e < P * N; e += kThreads) {
    const int p = e / N, n = e % N;
    float s = 0.f, u = 0.f;
    for (int t = 0; t < Qc; ++t) {
      s = fmaf(cS[t] * xs[t * P + p], Bs[t * N + n], s);
      u = fmaf(cT[t] * dys[t * P + p], Cs[t * N + n], u);
    }
    So[e] = s;
    To[e] = u;
  }
}

// One thread per state entry (b, h, p, n): the forward scan turns S into the
// state entering each chunk, the backward scan turns T into the gradient with
// respect to the state leaving each chunk; what the backward scan carries out
// of chunk 0 is dLoss/dinitial_states.
__global__ void __launch_bounds__(kThreads) k_bwd_state_passing(const KArgs a) {
  const Dims& d = a.d;
  const int64_t PN = d.P * d.N;
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (i >= d.b * d.H * PN) return;
  const int64_t bh = i / PN, e = i % PN;
  float* S = a.S + bh * d.nc * PN + e;
  float* T = a.T + bh * d.nc * PN + e;
  const float* dec = a.dec + bh * d.nc;
  float run = a.h0 ? a.h0[i] : 0.f;
  for (int64_t c = 0; c < d.nc; ++c) {
    const float s = S[c * PN];
    S[c * PN] = run;
    run = fmaf(dec[c], run, s);
  }
  float lam = a.dfinal ? a.dfinal[i] : 0.f;
  for (int64_t c = d.nc - 1; c >= 0; --c) {
    const float u = T[c * PN];
    T[c * PN] = lam;
    lam = fmaf(dec[c], lam, u);
  }
  if (a.dh0) a.dh0[i] = lam;
}

// Shared-memory floats of k_bwd_chunk for chunk length Q (rows padded by one
// float so that column walks do not collide in a bank).
inline size_t smem_chunk_floats(int64_t Q, int64_t P, int64_t N) {
  return (size_t)(4 * Q * (P + 1) + 2 * Q * (N + 1) + 3 * Q * (Q + 1) + 6 * Q + kThreads);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_chunk(const KArgs a) {
  const Dims& d = a.d;
  const ChunkPos q = chunk_pos(d, blockIdx.x);
  const int P = (int)d.P, N = (int)d.N, Q = (int)d.Q, Qc = q.Qc;
  const int sP = P + 1, sN = N + 1, sQ = Q + 1;
  const int tid = threadIdx.x;
  SSD_DYN_SMEM(sm);
  float* xs = sm;             // Q x sP: x_t
  float* dys = xs + Q * sP;   // Q x sP: dy_t
  float* LB = dys + Q * sP;   // Q x sP: (Lam B_s)_p
  float* HC = LB + Q * sP;    // Q x sP: (h_in C_t)_p
  float* Bs = HC + Q * sP;    // Q x sN
  float* Cs = Bs + Q * sN;    // Q x sN
  float* Em = Cs + Q * sN;    // Q x sQ: E(t,s)
  float* CB = Em + Q * sQ;    // Q x sQ: C_t.B_s (s <= t)
  float* XY = CB + Q * sQ;    // Q x sQ: dy_t.x_s (s <= t)
  float* cs = XY + Q * sQ;    // Q
  float* w = cs + Q;          // Q: dt
  float* dw = w + Q;          // Q
  float* dcs = dw + Q;        // Q
  float* nn = dcs + Q;        // Q: N_s
  float* red = nn + Q;        // kThreads
  int* seg = reinterpret_cast<int*>(red + kThreads);  // Q

  const T* x = static_cast<const T*>(a.x);
  const T* dy = static_cast<const T*>(a.dy);
  const T* B = static_cast<const T*>(a.B);
  const T* C = static_cast<const T*>(a.C);
  const int64_t soff = ((q.b * d.H + q.h) * d.nc + q.c) * d.P * d.N;
  const float* Hin = a.S + soff;  // P x N
  const float* Lam = a.T + soff;  // P x N

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
  for (int t = tid; t < Qc; t += kThreads) w[t] = a.dt[(q.b * d.L + q.t0 + t) * d.H + q.h];
  if (tid == 0) chunk_cumsum(a, q, cs, seg);
  __syncthreads();

  // the chunk's Q x Q matrices, lower triangle
  for (int i = tid; i < Qc * Qc; i += kThreads) {
    const int t = i / Qc, s = i % Qc;
    float e = 0.f, cb = 0.f, xy = 0.f;
    if (s <= t) {
      if (seg[s] == seg[t]) e = expf(cs[t] - cs[s]);
      for (int n = 0; n < N; ++n) cb = fmaf(Cs[t * sN + n], Bs[s * sN + n], cb);
      for (int p = 0; p < P; ++p) xy = fmaf(dys[t * sP + p], xs[s * sP + p], xy);
    }
    Em[t * sQ + s] = e;
    CB[t * sQ + s] = cb;
    XY[t * sQ + s] = xy;
  }
  // Lam B_s and h_in C_t
  for (int i = tid; i < P * Qc; i += kThreads) {
    const int p = i / Qc, s = i % Qc;
    float lb = 0.f, hc = 0.f;
    for (int n = 0; n < N; ++n) {
      lb = fmaf(Lam[p * N + n], Bs[s * sN + n], lb);
      hc = fmaf(Hin[p * N + n], Cs[s * sN + n], hc);
    }
    LB[s * sP + p] = lb;
    HC[s * sP + p] = hc;
  }
  // <Lam, h_in>, this thread's share
  {
    float part = 0.f;
    for (int e = tid; e < P * N; e += kThreads) part = fmaf(Lam[e], Hin[e], part);
    red[tid] = part;
  }
  __syncthreads();

  const int last = Qc - 1;
  const float Dh = a.D ? a.D[q.h] : 0.f;
  // dx
  for (int i = tid; i < Qc * P; i += kThreads) {
    const int s = i / P, p = i % P;
    float acc = 0.f;
    for (int t = s; t < Qc; ++t) acc = fmaf(Em[t * sQ + s] * CB[t * sQ + s], dys[t * sP + p], acc);
    acc = fmaf(Em[last * sQ + s], LB[s * sP + p], acc);
    a.dx[((q.b * d.L + q.t0 + s) * d.H + q.h) * d.P + p] = fmaf(w[s], acc, Dh * dys[s * sP + p]);
  }
  // dB and dC of this head
  for (int i = tid; i < Qc * N; i += kThreads) {
    const int s = i / N, n = i % N;
    float accB = 0.f;
    for (int t = s; t < Qc; ++t) accB = fmaf(Em[t * sQ + s] * XY[t * sQ + s], Cs[t * sN + n], accB);
    float lx = 0.f;
    for (int p = 0; p < P; ++p) lx = fmaf(Lam[p * N + n], xs[s * sP + p], lx);
    accB = fmaf(Em[last * sQ + s], lx, accB);
    float accC = 0.f;
    for (int r = 0; r <= s; ++r) accC = fmaf(Em[s * sQ + r] * w[r] * XY[s * sQ + r], Bs[r * sN + n], accC);
    if (seg[s] == -1) {
      float hy = 0.f;
      for (int p = 0; p < P; ++p) hy = fmaf(Hin[p * N + n], dys[s * sP + p], hy);
      accC = fmaf(expf(cs[s]), hy, accC);
    }
    const int64_t gi = ((q.b * d.L + q.t0 + s) * d.H + q.h) * d.N + n;
    a.dBh[gi] = w[s] * accB;
    a.dCh[gi] = accC;
  }
  // per token: dw and dcs (before the last token's extra terms)
  for (int t = tid; t < Qc; t += kThreads) {
    float nx = 0.f;
    for (int p = 0; p < P; ++p) nx = fmaf(xs[t * sP + p], LB[t * sP + p], nx);
    float y0 = 0.f;
    if (seg[t] == -1) {
      for (int p = 0; p < P; ++p) y0 = fmaf(dys[t * sP + p], HC[t * sP + p], y0);
      y0 *= expf(cs[t]);
    }
    float dwt = 0.f, colm = 0.f;
    for (int u = t; u < Qc; ++u) {
      const float m = Em[u * sQ + t] * CB[u * sQ + t] * XY[u * sQ + t];
      dwt += m;
      if (u > t) colm += m;
    }
    float rowm = 0.f;
    for (int s = 0; s < t; ++s) rowm = fmaf(Em[t * sQ + s] * w[s], CB[t * sQ + s] * XY[t * sQ + s], rowm);
    const float el = Em[last * sQ + t];
    dw[t] = fmaf(el, nx, dwt);
    nn[t] = el * w[t] * nx;
    dcs[t] = rowm - w[t] * colm + y0 - nn[t];
  }
  __syncthreads();

  if (tid == 0) {
    float lh = 0.f;
    for (int i = 0; i < kThreads; ++i) lh += red[i];
    float sn = 0.f;
    for (int t = 0; t < Qc; ++t) sn += nn[t];
    const float e_last = seg[last] == -1 ? expf(cs[last]) : 0.f;
    dcs[last] += sn + e_last * lh;
    const float Ah = a.A[q.h];
    double dA = 0.0, dD = 0.0;
    float run = 0.f;
    for (int k = last; k >= 0; --k) {
      if (k == last || seg[k] != seg[k + 1]) run = 0.f;
      run += dcs[k];
      const float dl = seg[k] == k ? 0.f : run;  // a segment's first token has no decay
      a.ddt[(q.b * d.L + q.t0 + k) * d.H + q.h] = fmaf(Ah, dl, dw[k]);
      dA += (double)w[k] * (double)dl;
      dD += (double)XY[k * sQ + k];
    }
    const int64_t pi = q.h * (d.b * d.nc) + q.b * d.nc + q.c;
    a.dA_part[pi] = dA;
    a.dD_part[pi] = dD;
  }
}

// dB, dC (b,L,G,N): the per-head gradients summed over each group's heads.
__global__ void __launch_bounds__(kThreads) k_bwd_group_sum(const KArgs a) {
  const Dims& d = a.d;
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (i >= d.b * d.L * d.G * d.N) return;
  const int64_t n = i % d.N, r = i / d.N;
  const int64_t g = r % d.G, bl = r / d.G;
  float sb = 0.f, sc = 0.f;
  for (int64_t j = 0; j < d.hpg; ++j) {
    const int64_t gi = (bl * d.H + g * d.hpg + j) * d.N + n;
    sb += a.dBh[gi];
    sc += a.dCh[gi];
  }
  a.dB[i] = sb;
  a.dC[i] = sc;
}

// dA, dD (H): the per-chunk partial sums added in fp64, in a fixed order.
__global__ void __launch_bounds__(kThreads) k_bwd_param_sum(const KArgs a) {
  const Dims& d = a.d;
  const int64_t h = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (h >= d.H) return;
  const int64_t n = d.b * d.nc;
  double sa = 0.0, sd = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    sa += a.dA_part[h * n + i];
    sd += a.dD_part[h * n + i];
  }
  a.dA[h] = (float)sa;
  if (a.dD) a.dD[h] = (float)sd;
}

// ---------------------------------------------------------------- host side

struct Plan {
  Dims d;
  size_t smem_states, smem_chunk;  // bytes
  size_t off_S, off_T, off_dec, off_dBh, off_dCh, off_dA, off_dD, total;
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
  if (!a->x || !a->dt || !a->A || !a->B || !a->C || !a->dy || !a->dx || !a->ddt || !a->dA || !a->dB || !a->dC)
    return SSD_ERR_INVALID_ARG;
  if (a->seq_idx && a->dfinal_states) return SSD_ERR_UNSUPPORTED;
  if (!a->workspace || a->workspace_bytes < pl.total) return SSD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) % 256 != 0) return SSD_ERR_INVALID_ARG;
  if ((a->timing_events[0] == nullptr) != (a->timing_events[1] == nullptr)) return SSD_ERR_INVALID_ARG;
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
  char* ws = static_cast<char*>(a->workspace);
  k.S = reinterpret_cast<float*>(ws + pl.off_S);
  k.T = reinterpret_cast<float*>(ws + pl.off_T);
  k.dec = reinterpret_cast<float*>(ws + pl.off_dec);
  k.dBh = reinterpret_cast<float*>(ws + pl.off_dBh);
  k.dCh = reinterpret_cast<float*>(ws + pl.off_dCh);
  k.dA_part = reinterpret_cast<double*>(ws + pl.off_dA);
  k.dD_part = reinterpret_cast<double*>(ws + pl.off_dD);
  return k;
}

inline unsigned blocks_for(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

// Validate, then enqueue the five kernels through `launch(kernel, grid,
// shared bytes, args)`, which returns false when a launch fails;
// `launch.record(event)` records a caller's timing event (false on failure).
template <typename T, class Launch>
ssd_status enqueue_typed(const KArgs& k, const Plan& pl, void* const events[2], Launch& launch) {
  const Dims& d = pl.d;
  const unsigned chunk_ctas = (unsigned)(d.b * d.nc * d.H);
  if (!launch(&k_bwd_chunk_states<T>, chunk_ctas, pl.smem_states, k)) return SSD_ERR_CUDA;
  if (!launch(&k_bwd_state_passing, blocks_for(d.b * d.H * d.P * d.N), (size_t)0, k)) return SSD_ERR_CUDA;
  if (events[0] && !launch.record(events[0])) return SSD_ERR_CUDA;
  if (!launch(&k_bwd_chunk<T>, chunk_ctas, pl.smem_chunk, k)) return SSD_ERR_CUDA;
  if (events[1] && !launch.record(events[1])) return SSD_ERR_CUDA;
  if (!launch(&k_bwd_group_sum, blocks_for(d.b * d.L * d.G * d.N), (size_t)0, k)) return SSD_ERR_CUDA;
  if (!launch(&k_bwd_param_sum, blocks_for(d.H), (size_t)0, k)) return SSD_ERR_CUDA;
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
  return a->dtype == SSD_BF16 ? enqueue_typed<__nv_bfloat16>(k, pl, a->timing_events, launch)
                               : enqueue_typed<float>(k, pl, a->timing_events, launch);
}

}  // namespace bwd
}  // namespace ssd

#endif  // SSD_BWD_CUH_
