// The backward's per-chunk gradients on the tensor cores (tcgen05 MMAs with
// fp32 accumulators in tensor memory): the formulas of k_bwd_chunk in
// ssd_bwd.cuh, with every contraction an MMA.  One CTA per (batch row, chunk,
// head), for headdim 64, dstate 128, 64-token chunks, bf16 inputs and no gate;
// other calls take the CUDA-core kernels.
//
// Per chunk (E(t,s) = exp(cs_t - cs_s) inside one packed sequence, w = dt,
// e_t, el_s = E(last, s), h_in the state entering the chunk, Lam the
// gradient with respect to the state leaving it):
//
//   CB = C B^T,  G = dy x^T                              (bf16 operands as loaded)
//   K = E o CB,  Z = E o G,  Zw = Z diag(w),  M = K o G   (CUDA cores)
//   dx = diag(w) [K^T dy + diag(el) B Lam^T] + D dy
//   dB = diag(w) [Z^T C + diag(el) x Lam]
//   dC = Zw B + diag(e) dy h_in
//
// and the decay gradients from row sums of M and of the products, as in
// ssd_bwd.cuh.  The fp32 operands (K, Z, Zw, Lam, h_in) enter the MMAs as
// three bf16 terms, v = hi + mid + lo with hi = bf16(v), mid = bf16(v - hi),
// lo = bf16(v - hi - mid): the terms miss v by at most 2^-24 |v|, and each
// product of a term with a bf16 input is exact in fp32, so the contractions
// keep fp32 accuracy.
//
// A row-scaled term shares its accumulator with the unscaled one: the product
// with Lam is formed first, read out, scaled by el_s and written back, and
// the other product accumulates on top of it.  Tensor memory (the M = 64
// layout: row m at lane 32 (m / 16) + m % 16), 448 of 512 columns:
//   [0, 64)    dx        [64, 192)  dB
//   [192, 256) CB, then with [256, 320) (G) the product dy h_in
//   [320, 448) Zw B
// Shared memory holds x, dy, B and C as the TMA loads them (bf16, 128-byte
// rows, 128-byte swizzle), the chunk's Lam and h_in as two bulk copies leave
// them (fp32), the three-term split tiles written by the threads in the
// tiles' layout, and M in fp32 for the decay sums.  The MMAs run in five
// groups with a completion barrier each (C B^T and G; the Lam products; dx;
// dB; dC), so the threads start on each result while the next is formed.
// Every wait is bounded (1 s); a CTA whose wait gives up lets its copies and
// MMAs finish, frees its tensor memory and exits without writing gradients.
//
// Included by ssd_bwd.cu only (after ssd_bwd.cuh): the host emulation of the
// CUDA-core kernels includes ssd_bwd.cuh alone.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "sm100.cuh"
#include "ssd_bwd.cuh"
#include "ssd_internal.h"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace bwd {
namespace {

using namespace sm100;

struct TcCfg {
  static constexpr int Q = 64;
  static constexpr uint32_t kTile = 8192;          // 64 rows x 128 bytes
  static constexpr uint32_t oX = 0;                 // x  [s][p]
  static constexpr uint32_t oDY = oX + kTile;       // dy [t][p]
  static constexpr uint32_t oB = oDY + kTile;       // B  [s][n], n-blocks 0-63, 64-127
  static constexpr uint32_t oC = oB + 2 * kTile;    // C  [t][n]
  static constexpr uint32_t oK = oC + 2 * kTile;    // K  terms [3][t][s]
  static constexpr uint32_t oZ = oK + 3 * kTile;    // Z  terms [3][t][s]
  static constexpr uint32_t oZw = oZ + 3 * kTile;   // Zw terms [3][t][s]
  static constexpr uint32_t oS = oZw + 3 * kTile;   // Lam, then h_in: terms [3][n-block][p][n]
  static constexpr uint32_t oM = oS + 6 * kTile;    // M fp32 [t][s], rows of kMs
  static constexpr int kMs = Q + 1;
  // the chunk's states as their bulk loads leave them, fp32 [p][n]: h_in in a
  // region of its own (read again for its terms after the first MMAs), Lam over
  // the K and Z terms (split into its terms before those are written)
  static constexpr uint32_t kStateBytes = 64 * 128 * 4;
  static constexpr uint32_t oHin = (oM + Q * kMs * 4 + 1023) & ~1023u;
  static constexpr uint32_t oLam = oK;
  static_assert(oLam + kStateBytes <= oZw, "Lam staging");
  static constexpr uint32_t oEnd = oHin + kStateBytes;
  // The gradients staged for their bulk stores (32-column fp32 boxes, 64 rows
  // of 128 bytes, 128-byte swizzle), each where nothing still running reads:
  // dx over the K terms (read only by the dx MMAs), dB over the h_in copy
  // (dead once its terms are written), dC over the Z and Zw terms (all MMAs
  // done); the tail's R over the state terms.
  static constexpr uint32_t oStDx = oK, oStDB = oHin, oStDC = oZ, oR = oS;
  static_assert(oStDx + 2 * kTile <= oZ && oStDB + 4 * kTile <= oEnd && oStDC + 4 * kTile <= oS, "staging");
  static_assert(oR + Q * kMs * 4 <= oM, "R");
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  // tensor memory columns
  static constexpr uint32_t tDx = 0, tDB = 64, tCB = 192, tG = 256, tDC2 = 192, tDC1 = 320, kTmemCols = 512;
};

struct __align__(16) TcSmem {
  // MMA completions: p1a C B^T and G, p1 the Lam products; p2a dx, p2b dB, p2 dC
  uint64_t bar_in, bar_st, bar_p1a, bar_p1, bar_p2a, bar_p2b, bar_p2, bar_drain;
  uint32_t tmem_base;
  int abort_flag, never;
  // per-token arrays, one buffer per unit parity (warp 0 reads a unit's while the
  // other warps write the next one's); cs, w and seg are read as 16-byte vectors
  __align__(16) float cs[2][64];
  __align__(16) float w[2][64];
  __align__(16) int seg[2][64];
  float el[2][64], ein[2][64], dg[2][64];
  float nv[64], dw[64], dcs[64], nn[64];
  float nxp[64][4], cyp[64][4];  // row sums, four shares a row
  float pair[64][8];             // the decay pair sums, in quarters
  float red[2][kThreads / 32];  // <Lam, h_in>, a share per warp
};

// Byte offset of 16-byte chunk k16 of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw_chunk(int r, int k16) {
  return (uint32_t)r * 128 + ((uint32_t)(k16 ^ (r & 7)) << 4);
}

// 8 bf16 of row r, chunk k16 of a swizzled tile, as floats
__device__ __forceinline__ void load8(const unsigned char* tile, int r, int k16, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(tile + sw_chunk(r, k16));
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w4[i] << 16);
    f[2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
  }
}

// split3 of two values at once, as packed bf16 pairs (the first value in the
// low half): bf16x2 roundings and fp32x2 differences, each difference exact
// as in split3, so the terms are split3's.
__device__ __forceinline__ void split3x2(float a, float b, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  const float2 v = make_float2(a, b), neg = make_float2(-1.f, -1.f);
  const __nv_bfloat162 h = __float22bfloat162_rn(v);
  const float2 r1 = __ffma2_rn(__bfloat1622float2(h), neg, v);
  const __nv_bfloat162 m = __float22bfloat162_rn(r1);
  const float2 r2 = __ffma2_rn(__bfloat1622float2(m), neg, r1);
  const __nv_bfloat162 l = __float22bfloat162_rn(r2);
  hi = reinterpret_cast<const uint32_t&>(h);
  mid = reinterpret_cast<const uint32_t&>(m);
  lo = reinterpret_cast<const uint32_t&>(l);
}

// Three-term split of 8 consecutive values of row r (chunk k16) into three
// tiles `stride` bytes apart.
__device__ __forceinline__ void store_terms8(unsigned char* tile, uint32_t stride, int r, int k16, const float* v) {
  uint4 h, m, l;
  split3x2(v[0], v[1], h.x, m.x, l.x);
  split3x2(v[2], v[3], h.y, m.y, l.y);
  split3x2(v[4], v[5], h.z, m.z, l.z);
  split3x2(v[6], v[7], h.w, m.w, l.w);
  const uint32_t off = sw_chunk(r, k16);
  *reinterpret_cast<uint4*>(tile + off) = h;
  *reinterpret_cast<uint4*>(tile + stride + off) = m;
  *reinterpret_cast<uint4*>(tile + 2 * stride + off) = l;
}

// chunk_pos in 32-bit arithmetic: the tensor-core kernels' grids (one CTA per
// row, chunk and head) stay below 2^31 CTAs.
__device__ __forceinline__ ChunkPos chunk_pos_u32(const Dims& d, uint32_t bid) {
  const uint32_t H = (uint32_t)d.H, nc = (uint32_t)d.nc;
  const uint32_t bc = bid / H, bb = bc / nc;
  ChunkPos q;
  q.h = bid - bc * H;
  q.c = bc - bb * nc;
  q.b = bb;
  q.g = (uint32_t)q.h / (uint32_t)d.hpg;
  q.t0 = q.c * d.Q;
  const int64_t left = d.L - q.t0;
  q.Qc = (int)(left < d.Q ? left : d.Q);
  return q;
}

// The chunk's per-token scalars for tokens 2 lane and 2 lane + 1, by one warp:
// w = dt, the in-chunk cumulative log-decay cs and the in-chunk index seg of
// the token's sequence start (-1: it began before the chunk), as chunk_cumsum
// defines them, then el = E(last, t) and ein = e_t.  cs is a segmented scan
// (a start contributes 0 and restarts the sum) and seg a max scan of the
// starts, both over the warp's shuffles.  Tokens past the chunk's end get 0
// everywhere.
struct DtScan {
  float w[2], cs[2], el[2], ein[2];
  int seg[2];
};
// The loads behind a DtScan: dt of the two tokens and whether a sequence
// starts at each, so that a loop can issue them a few chunks ahead.
struct DtRaw {
  float w[2];
  bool v[2], f[2];
};
__device__ __forceinline__ DtRaw dt_load(const KArgs& a, const ChunkPos& q, int lane) {
  const Dims& d = a.d;
  const float* dtp = a.dt + (q.b * d.L + q.t0) * d.H + q.h;
  const int32_t* sq = a.seq ? a.seq + q.b * d.L + q.t0 : nullptr;
  DtRaw r;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int t = 2 * lane + e;
    r.v[e] = t < q.Qc;
    r.w[e] = r.v[e] ? dtp[(int64_t)t * d.H] : 0.f;
    r.f[e] = r.v[e] && sq && q.t0 + t > 0 && sq[t] != sq[t - 1];  // a sequence starts at t
  }
  return r;
}
__device__ __forceinline__ DtScan dt_scan_from(const DtRaw& raw, const ChunkPos& q, float Ah, int lane) {
  DtScan r;
  const bool* v = raw.v;
  const bool* f = raw.f;
  r.w[0] = raw.w[0], r.w[1] = raw.w[1];
  const float a0 = f[0] ? 0.f : r.w[0] * Ah;
  const float a1 = f[1] ? 0.f : a0 + r.w[1] * Ah;
  float sum = a1;                                         // the lane's sum since its last start
  int rs = f[0] || f[1];                                  // ... and whether it has one
  int st = f[1] ? 2 * lane + 1 : f[0] ? 2 * lane : -1;  // its last start
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float ps = __shfl_up_sync(0xffffffffu, sum, o);
    const int pr = __shfl_up_sync(0xffffffffu, rs, o);
    const int pst = __shfl_up_sync(0xffffffffu, st, o);
    if (lane >= o) {
      if (!rs) sum += ps;
      rs |= pr;
      st = max(st, pst);
    }
  }
  float pre = __shfl_up_sync(0xffffffffu, sum, 1);
  int pst = __shfl_up_sync(0xffffffffu, st, 1);
  if (lane == 0) pre = 0.f, pst = -1;
  r.cs[0] = f[0] ? 0.f : a0 + pre;
  r.cs[1] = f[1] ? 0.f : f[0] ? a1 : a1 + pre;
  r.seg[0] = f[0] ? 2 * lane : pst;
  r.seg[1] = f[1] ? 2 * lane + 1 : r.seg[0];
  const int last = q.Qc - 1;
  const float csl = __shfl_sync(0xffffffffu, (last & 1) ? r.cs[1] : r.cs[0], last >> 1);
  const int segl = __shfl_sync(0xffffffffu, (last & 1) ? r.seg[1] : r.seg[0], last >> 1);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    if (!v[e]) r.cs[e] = 0.f, r.seg[e] = 0;
    r.el[e] = v[e] && r.seg[e] == segl ? expf(csl - r.cs[e]) : 0.f;
    r.ein[e] = v[e] && r.seg[e] == -1 ? expf(r.cs[e]) : 0.f;
  }
  return r;
}
__device__ __forceinline__ DtScan dt_scan_warp(const KArgs& a, const ChunkPos& q, int lane) {
  return dt_scan_from(dt_load(a, q, lane), q, a.A[q.h], lane);
}

// The three-term split of a fp32 state [p][n] as its bulk load leaves it in
// shared memory, into the MN-major term tiles at `area` (two 64-column blocks
// a term): items i = first, first + stride, .. < 1024, item i being the
// 16-byte chunk k16 = i % 16 of row p = i / 16.  Returns the thread's share of
// <v, w> when `w` is given.
__device__ __forceinline__ float split_state(unsigned char* area, const float* v, const float* w, int first,
                                             int stride) {
  float dot = 0.f;
#pragma unroll 2
  for (int it = first; it < 64 * 16; it += stride) {
    const int p = it >> 4, k16 = it & 15;
    const float4* vr = reinterpret_cast<const float4*>(v + p * 128 + 8 * k16);
    const float4 x0 = vr[0], x1 = vr[1];
    const float e[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    if (w) {
      const float4* wr = reinterpret_cast<const float4*>(w + p * 128 + 8 * k16);
      const float4 y0 = wr[0], y1 = wr[1];
      const float f[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(e[i], f[i], dot);
    }
    store_terms8(area + (k16 >> 3) * TcCfg::kTile, 2 * TcCfg::kTile, p, k16 & 7, e);
  }
  return dot;
}

// Descriptor of K step kk of a K-major operand: 16 bf16 (32 bytes) along the
// row, the next 64-column tile after 4 steps.
__device__ __forceinline__ uint64_t kmaj(uint64_t d0, int kk) {
  return d0 + (uint64_t)(((kk >> 2) * TcCfg::kTile + (kk & 3) * 32) >> 4);
}
// ... of an MN-major operand: 16 rows (2048 bytes)
__device__ __forceinline__ uint64_t mnmaj(uint64_t d0, int kk) { return d0 + (uint64_t)((kk * 2048) >> 4); }

__global__ void __launch_bounds__(kThreads, 1)
    k_bwd_chunk_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dy,
                   const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                   const __grid_constant__ CUtensorMap tm_dx, const __grid_constant__ CUtensorMap tm_dbh,
                   const __grid_constant__ CUtensorMap tm_dch, const KArgs a) {
  using K = TcCfg;
  constexpr uint64_t kLimit = tc::kWaitLimitNs;
  const Dims& d = a.d;
  const uint32_t n_units = (uint32_t)(d.b * d.nc * d.H);
  constexpr int kStoreThread = kThreads - 1, kTileThread = kThreads - 33;  // lanes 31 of warps 7 and 6
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  float* Mm = reinterpret_cast<float*>(sm + K::oM);
  __shared__ TcSmem s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // TMEM reads: warp (qd, hf) reads rows 16 qd + (lane & 15) of its lane
  // quadrant; 64-column accumulators give it columns c0 + [0, 16), 128-column
  // ones columns c1 + [0, 32)
  const int qd = warp & 3, hf = warp >> 2;
  const int row = 16 * qd + (lane & 15);
  const int c0 = 16 * hf + 32 * (lane >> 4);
  const int c1 = 64 * hf + 32 * (lane >> 4);
  volatile int* abort_flag = &s.abort_flag;
  volatile int* never = &s.never;

  if (tid == 0) {
    mbar_init(&s.bar_in, 1);
    mbar_init(&s.bar_st, 1);
    mbar_init(&s.bar_p1a, 1);
    mbar_init(&s.bar_p1, 1);
    mbar_init(&s.bar_p2a, 1);
    mbar_init(&s.bar_p2b, 1);
    mbar_init(&s.bar_p2, 1);
    mbar_init(&s.bar_drain, 1);
    s.abort_flag = 0;
    s.never = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_dy);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_dx);
    tma_prefetch_desc(&tm_dbh);
    tma_prefetch_desc(&tm_dch);
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, K::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint32_t tq = tmem + ((uint32_t)(32 * qd) << 16);
  // A unit's loads: its tiles (x, dy, B, C) on bar_in, its states (Lam and
  // h_in, one contiguous P x N block each) on bar_st.
  auto issue_tiles = [&](const ChunkPos& u) {
    const int col = (int)(u.h * d.P), tok = (int)u.t0, bb = (int)u.b, grp = (int)u.g;
    mbar_arrive_expect_tx(&s.bar_in, 6 * K::kTile);
    tma_load_3d(sm + K::oX, &tm_x, &s.bar_in, col, tok, bb);
    tma_load_3d(sm + K::oDY, &tm_dy, &s.bar_in, col, tok, bb);
    for (int jb = 0; jb < 2; ++jb) {
      tma_load_4d(sm + K::oB + jb * K::kTile, &tm_b, &s.bar_in, 64 * jb, grp, tok, bb);
      tma_load_4d(sm + K::oC + jb * K::kTile, &tm_c, &s.bar_in, 64 * jb, grp, tok, bb);
    }
  };
  auto state_offset = [&](const ChunkPos& u) { return ((u.b * d.H + u.h) * d.nc + u.c) * d.P * d.N; };
  auto issue_states = [&](const ChunkPos& u) {
    const int64_t so = state_offset(u);
    mbar_arrive_expect_tx(&s.bar_st, 2 * K::kStateBytes);
    bulk_load(sm + K::oLam, a.T + so, K::kStateBytes, &s.bar_st);
    bulk_load(sm + K::oHin, a.S + so, K::kStateBytes, &s.bar_st);
  };
  if (tid == 0) {  // the first unit (the grid has at most one CTA per unit)
    const ChunkPos u0 = chunk_pos_u32(d, blockIdx.x);
    issue_states(u0);
    issue_tiles(u0);
  }
  // descriptors: K-major tiles (rows along K) and MN-major ones (rows along K,
  // the 64-element blocks of M or N one tile apart)
  const uint64_t dX = sw128_desc(smem_u32(sm + K::oX), 16, 1024);
  const uint64_t dDY = sw128_desc(smem_u32(sm + K::oDY), 16, 1024);
  const uint64_t dB = sw128_desc(smem_u32(sm + K::oB), 16, 1024);
  const uint64_t dC = sw128_desc(smem_u32(sm + K::oC), 16, 1024);
  const uint64_t dDYmn = sw128_desc(smem_u32(sm + K::oDY), K::kTile, 1024);
  const uint64_t dBmn = sw128_desc(smem_u32(sm + K::oB), K::kTile, 1024);
  const uint64_t dCmn = sw128_desc(smem_u32(sm + K::oC), K::kTile, 1024);
  constexpr uint32_t id_kk64 = idesc_bf16(64, 64, 0, 0);
  constexpr uint32_t id_km128 = idesc_bf16(64, 128, 0, 1);
  constexpr uint32_t id_mm64 = idesc_bf16(64, 64, 1, 1);
  constexpr uint32_t id_mm128 = idesc_bf16(64, 128, 1, 1);
  // term t3 of a split: the Q x Q ones one tile apart, the states two
  auto qq_term = [&](uint32_t base, int t3, bool mn) {
    return sw128_desc(smem_u32(sm + base + (uint32_t)t3 * K::kTile), mn ? K::kTile : 16, 1024);
  };
  auto st_term = [&](int t3, bool mn) {
    return sw128_desc(smem_u32(sm + K::oS + (uint32_t)t3 * 2 * K::kTile), mn ? K::kTile : 16, 1024);
  };

  // The CTA's units, one after the other: each unit's loads are issued during
  // the previous unit's tail, so its start finds them landed.
  bool ok = true;
  int it = 0;
  for (uint32_t unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
  const uint32_t par = (uint32_t)it & 1u;  // every barrier completes one phase a unit
  const int pb = (int)par;                 // the per-token arrays alternate between units
  const ChunkPos q = chunk_pos_u32(d, unit);
  const int Qc = q.Qc, last = Qc - 1;
  const uint32_t next = unit + gridDim.x;
  if (tid == 0 && next < n_units) {  // the next unit's states into L2 (its bulk loads come in the tail)
    const int64_t o = state_offset(chunk_pos_u32(d, next));
    const uint32_t bytes = (uint32_t)(d.P * d.N * 4);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.S + o), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.T + o), "r"(bytes) : "memory");
  }
  // Warp 0 forms C B^T and G as soon as their tiles land, warp 1 the per-token
  // scalars, warps 2-7 the Lam terms (the h_in ones come after the first MMAs)
  // and <Lam, h_in>.
  float lh = 0.f;
  if (warp == 0) {
    ok = mbar_wait(&s.bar_in, par, abort_flag, kLimit);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // CB = C B^T (K = n)
          mma_bf16_ss(tmem + K::tCB, kmaj(dC, kk), kmaj(dB, kk), id_kk64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // G = dy x^T (K = p)
          mma_bf16_ss(tmem + K::tG, kmaj(dDY, kk), kmaj(dX, kk), id_kk64, kk > 0);
        mma_commit(&s.bar_p1a);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    const DtScan r = dt_scan_warp(a, q, lane);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      s.w[pb][t] = r.w[e];
      s.cs[pb][t] = r.cs[e];
      s.seg[pb][t] = r.seg[e];
      s.el[pb][t] = r.el[e];
      s.ein[pb][t] = r.ein[e];
      s.dg[pb][t] = 0.f;
    }
  } else {
    ok = mbar_wait(&s.bar_st, par, abort_flag, kLimit);
    if (ok)
      lh = split_state(sm + K::oS, reinterpret_cast<const float*>(sm + K::oLam),
                       reinterpret_cast<const float*>(sm + K::oHin), tid - 64, kThreads - 64);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lh += __shfl_xor_sync(0xffffffffu, lh, o);
  if (lane == 0) s.red[pb][warp] = lh;
  fence_proxy_async_smem();  // the Lam terms are read by the MMAs
  ok = __syncthreads_and(ok);

  // ---- MMAs, first round, continued: B Lam^T, x Lam
  ok = ok && mbar_wait(&s.bar_in, par, abort_flag, kLimit);  // every thread reads the tiles later
  if (warp == 0 && __all_sync(0xffffffffu, ok)) {
    tc_fence_after();
    if (elect_one()) {
#pragma unroll
      for (int t3 = 0; t3 < 3; ++t3) {
        const uint64_t lk = st_term(t3, false), lm = st_term(t3, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dx <- B Lam^T (K = n)
          mma_bf16_ss(tmem + K::tDx, kmaj(dB, kk), kmaj(lk, kk), id_kk64, t3 > 0 || kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dB <- x Lam (K = p)
          mma_bf16_ss(tmem + K::tDB, kmaj(dX, kk), mnmaj(lm, kk), id_km128, t3 > 0 || kk > 0);
      }
      mma_commit(&s.bar_p1);
    }
    __syncwarp();
  }
  ok = ok && mbar_wait(&s.bar_p1a, par, abort_flag, kLimit);
  if (ok) {
    tc_fence_after();
    // ---- the Q x Q matrices: row t, columns s in [c0, c0 + 16)
    {
      uint32_t rcb[16], rg[16];
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tCB + 16 * hf, rcb);
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tG + 16 * hf, rg);
      SSD_TMEM_WAIT_LD_16(rcb);
      SSD_TMEM_WAIT_LD_16(rg);
      const int t = row;
      const float cst = s.cs[pb][t];
      const int segt = s.seg[pb][t];
      float csv[16], wv[16];
      int sgv[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 c4 = reinterpret_cast<const float4*>(s.cs[pb] + c0)[j];
        const float4 w4 = reinterpret_cast<const float4*>(s.w[pb] + c0)[j];
        const int4 g4 = reinterpret_cast<const int4*>(s.seg[pb] + c0)[j];
        csv[4 * j] = c4.x, csv[4 * j + 1] = c4.y, csv[4 * j + 2] = c4.z, csv[4 * j + 3] = c4.w;
        wv[4 * j] = w4.x, wv[4 * j + 1] = w4.y, wv[4 * j + 2] = w4.z, wv[4 * j + 3] = w4.w;
        sgv[4 * j] = g4.x, sgv[4 * j + 1] = g4.y, sgv[4 * j + 2] = g4.z, sgv[4 * j + 3] = g4.w;
      }
      float kv[16], zv[16], zwv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int sc = c0 + i;
        const float g = __uint_as_float(rg[i]);
        const bool in = t < Qc && sc <= t && sgv[i] == segt;
        const float e = in ? expf(cst - csv[i]) : 0.f;
        kv[i] = e * __uint_as_float(rcb[i]);
        zv[i] = e * g;
        zwv[i] = zv[i] * wv[i];
        Mm[t * K::kMs + sc] = kv[i] * g;
        if (sc == t && t < Qc) s.dg[pb][t] = g;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int k16 = (c0 >> 3) + c;
        store_terms8(sm + K::oK, K::kTile, t, k16, kv + 8 * c);
        store_terms8(sm + K::oZ, K::kTile, t, k16, zv + 8 * c);
        store_terms8(sm + K::oZw, K::kTile, t, k16, zwv + 8 * c);
      }
    }
  }
  ok = ok && mbar_wait(&s.bar_p1, par, abort_flag, kLimit);  // the Lam products
  if (ok) {
    tc_fence_after();
    // ---- B Lam^T: the row sums x_s . (Lam B_s), then scaled by el_s and written back
    {
      uint32_t r[16];
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDx + 16 * hf, r);
      SSD_TMEM_WAIT_LD_16(r);
      const int sr = row;
      float xv[16];
      load8(sm + K::oX, sr, c0 >> 3, xv);
      load8(sm + K::oX, sr, (c0 >> 3) + 1, xv + 8);
      float nx = 0.f;
      const float els = s.el[pb][sr];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v = __uint_as_float(r[i]);
        nx = fmaf(xv[i], v, nx);
        r[i] = __float_as_uint(els * v);
      }
      s.nxp[sr][2 * hf + (lane >> 4)] = nx;
      SSD_TMEM_ST_16x32bx2_X16_HALF32(tq + K::tDx + 16 * hf, r);
    }
    // ---- x Lam: scaled by el_s and written back
    {
      const float els = s.el[pb][row];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t r[16];
        SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDB + 64 * hf + 16 * half, r);
        SSD_TMEM_WAIT_LD_16(r);
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(els * __uint_as_float(r[i]));
        SSD_TMEM_ST_16x32bx2_X16_HALF32(tq + K::tDB + 64 * hf + 16 * half, r);
      }
    }
    tmem_wait_st();
  }
  tc_fence_before();
  fence_proxy_async_smem();  // the split tiles are read by the MMAs
  ok = __syncthreads_and(ok);

  // ---- MMAs, second round: K^T dy, Z^T C (accumulating on the scaled Lam
  // products), Zw B; then, once its terms are written, dy h_in.  dx, dB and dC
  // complete on barriers of their own, so the read-out of one overlaps the next.
  if (ok && warp == 0) {
    tc_fence_after();
    if (elect_one()) {
#pragma unroll
      for (int t3 = 0; t3 < 3; ++t3) {
        const uint64_t k_mn = qq_term(K::oK, t3, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = t
          mma_bf16_ss(tmem + K::tDx, mnmaj(k_mn, kk), mnmaj(dDYmn, kk), id_mm64, 1);
      }
      mma_commit(&s.bar_p2a);
#pragma unroll
      for (int t3 = 0; t3 < 3; ++t3) {
        const uint64_t z_mn = qq_term(K::oZ, t3, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = t
          mma_bf16_ss(tmem + K::tDB, mnmaj(z_mn, kk), mnmaj(dCmn, kk), id_mm128, 1);
      }
      mma_commit(&s.bar_p2b);
#pragma unroll
      for (int t3 = 0; t3 < 3; ++t3) {
        const uint64_t zw_k = qq_term(K::oZw, t3, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = s
          mma_bf16_ss(tmem + K::tDC1, kmaj(zw_k, kk), mnmaj(dBmn, kk), id_km128, t3 > 0 || kk > 0);
      }
    }
    __syncwarp();
  }
  // ---- h_in terms over the Lam terms (the MMAs that read those are done), by
  // warps 1-7 while warp 0 issues
  if (ok && warp > 0) split_state(sm + K::oS, reinterpret_cast<const float*>(sm + K::oHin), nullptr, tid - 32, kThreads - 32);
  fence_proxy_async_smem();  // the h_in terms are read by the MMAs
  ok = __syncthreads_and(ok);
  if (ok && warp == 0) {
    tc_fence_after();
    if (elect_one()) {
#pragma unroll
      for (int t3 = 0; t3 < 3; ++t3) {
        const uint64_t h_mn = st_term(t3, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = p
          mma_bf16_ss(tmem + K::tDC2, kmaj(dDY, kk), mnmaj(h_mn, kk), id_km128, t3 > 0 || kk > 0);
      }
      mma_commit(&s.bar_p2);
    }
    __syncwarp();
  }
  ok = ok && mbar_wait(&s.bar_p2a, par, abort_flag, kLimit);
  if (ok) {
    tc_fence_after();
    // this thread's token row is staged whole (rows past the chunk's last token are
    // beyond L and the bulk stores clip them)
    // ---- dx = w_s [K^T dy + el_s B Lam^T] + D dy_s (columns p in [c0, c0 + 16))
    {
      uint32_t r[16];
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDx + 16 * hf, r);
      SSD_TMEM_WAIT_LD_16(r);
      float dyv[16];
      load8(sm + K::oDY, row, c0 >> 3, dyv);
      load8(sm + K::oDY, row, (c0 >> 3) + 1, dyv + 8);
      const float ws = s.w[pb][row], Dh = a.D ? a.D[q.h] : 0.f;
      // columns c0 .. c0 + 15: box c0 / 32, 16-byte chunks 4 hf .. 4 hf + 3 of its row
      unsigned char* box = sm + K::oStDx + (uint32_t)(c0 >> 5) * K::kTile;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float4*>(box + sw_chunk(row, 4 * hf + i)) =
            make_float4(fmaf(ws, __uint_as_float(r[4 * i]), Dh * dyv[4 * i]),
                        fmaf(ws, __uint_as_float(r[4 * i + 1]), Dh * dyv[4 * i + 1]),
                        fmaf(ws, __uint_as_float(r[4 * i + 2]), Dh * dyv[4 * i + 2]),
                        fmaf(ws, __uint_as_float(r[4 * i + 3]), Dh * dyv[4 * i + 3]));
    }
  }
  ok = ok && mbar_wait(&s.bar_p2b, par, abort_flag, kLimit);
  if (ok) {
    tc_fence_after();
    // ---- dB of this head = w_s [Z^T C + el_s x Lam] (states n in [c1, c1 + 32))
    {
      uint32_t r[32];
      uint32_t* r_hi = r + 16;
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDB + 64 * hf, r);
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDB + 64 * hf + 16, r_hi);
      SSD_TMEM_WAIT_LD_32(r);
      const float ws = s.w[pb][row];
      unsigned char* box = sm + K::oStDB + (uint32_t)(c1 >> 5) * K::kTile;  // a whole 32-column row
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<float4*>(box + sw_chunk(row, i)) =
            make_float4(ws * __uint_as_float(r[4 * i]), ws * __uint_as_float(r[4 * i + 1]),
                        ws * __uint_as_float(r[4 * i + 2]), ws * __uint_as_float(r[4 * i + 3]));
    }
  }
  ok = ok && mbar_wait(&s.bar_p2, par, abort_flag, kLimit);
  if (ok) {
    tc_fence_after();
    // ---- dC of this head = Zw B + e_t dy h_in, and the row sums C_t . (h_in^T dy_t)
    {
      uint32_t r2[32], r1[32];
      uint32_t* r2_hi = r2 + 16;
      uint32_t* r1_hi = r1 + 16;
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDC2 + 64 * hf, r2);
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDC2 + 64 * hf + 16, r2_hi);
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDC1 + 64 * hf, r1);
      SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tDC1 + 64 * hf + 16, r1_hi);
      SSD_TMEM_WAIT_LD_32(r2);
      SSD_TMEM_WAIT_LD_32(r1);
      float cv[32];
      const unsigned char* ctile = sm + K::oC + hf * K::kTile;  // states 64 hf ..
#pragma unroll
      for (int c = 0; c < 4; ++c) load8(ctile, row, 4 * (lane >> 4) + c, cv + 8 * c);
      const float et = s.ein[pb][row];
      float cy = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) cy = fmaf(cv[i], __uint_as_float(r2[i]), cy);
      s.cyp[row][2 * hf + (lane >> 4)] = cy;
      unsigned char* box = sm + K::oStDC + (uint32_t)(c1 >> 5) * K::kTile;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<float4*>(box + sw_chunk(row, i)) =
            make_float4(fmaf(et, __uint_as_float(r2[4 * i]), __uint_as_float(r1[4 * i])),
                        fmaf(et, __uint_as_float(r2[4 * i + 1]), __uint_as_float(r1[4 * i + 1])),
                        fmaf(et, __uint_as_float(r2[4 * i + 2]), __uint_as_float(r1[4 * i + 2])),
                        fmaf(et, __uint_as_float(r2[4 * i + 3]), __uint_as_float(r1[4 * i + 3])));
    }
    fence_proxy_async_smem();  // the staged gradients are read by the bulk stores
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);

  if (ok) {
    // The bulk operations of the tail, each on the last lane of a warp with
    // little of the tail's work (the column sums of its tokens are the shortest)
    if (tid == kStoreThread) {
      // dx, dB and dC of this head and chunk: 32-column boxes, rows past L clipped
      const int h = (int)q.h, tk = (int)q.t0, bb = (int)q.b;
      for (int k = 0; k < 2; ++k) tma_store_4d(&tm_dx, sm + K::oStDx + k * K::kTile, 32 * k, h, tk, bb);
      for (int k = 0; k < 4; ++k) {
        tma_store_4d(&tm_dbh, sm + K::oStDB + k * K::kTile, 32 * k, h, tk, bb);
        tma_store_4d(&tm_dch, sm + K::oStDC + k * K::kTile, 32 * k, h, tk, bb);
      }
      bulk_commit_group();
    }
    if (tid == kTileThread && next < n_units) issue_tiles(chunk_pos_u32(d, next));  // the tiles are read no more
    // ---- the decay gradients (the tail of k_bwd_chunk, on the row sums above)
    for (int t = tid; t < Qc; t += kThreads) {
      s.nv[t] = s.nxp[t][0] + s.nxp[t][1] + s.nxp[t][2] + s.nxp[t][3];
      s.dcs[t] = s.ein[pb][t] * (s.cyp[t][0] + s.cyp[t][1] + s.cyp[t][2] + s.cyp[t][3]);
    }
    // The pairs whose decay spans token k: S_k = sum_{u >= k} R(u, k) with the
    // row prefix R(u, k) = sum_{s < k} M(u, s) w_s, and the column sum of M
    // below the diagonal (for dw).  R goes over the state terms (the MMAs
    // that read them are done).  Row u's prefix: four threads, 16 columns each.
    float* Rm = reinterpret_cast<float*>(sm + K::oR);  // [u][k], rows of kMs
    {
      const int u = tid >> 2, sg = tid & 3;
      float pre[16], run = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int sc = 16 * sg + j;
        pre[j] = run;
        run = fmaf(Mm[u * K::kMs + sc], s.w[pb][sc], run);
      }
      s.pair[u][sg] = run;  // this segment's total
      __syncwarp();
      float off = 0.f;  // the segments before this one (same warp: threads 4u .. 4u + 3)
      for (int g2 = 0; g2 < sg; ++g2) off += s.pair[u][g2];
#pragma unroll
      for (int j = 0; j < 16; ++j) Rm[u * K::kMs + 16 * sg + j] = off + pre[j];
    }
    // the next unit's states go over this unit's staging once the stores have
    // read it, early enough to land during the rest of this tail
    if (tid == kStoreThread && next < n_units) {
      bulk_wait_read<0>();
      issue_states(chunk_pos_u32(d, next));
    }
    __syncthreads();
    for (int i = tid; i < 4 * Qc; i += kThreads) {
      const int k = i >> 2, qq = i & 3;
      const int lo = k + (Qc - k) * qq / 4, hi = k + (Qc - k) * (qq + 1) / 4;
      float col = 0.f, blk = 0.f;
      for (int u = lo; u < hi; ++u) {
        if (u > k) col += Mm[u * K::kMs + k];
        blk += Rm[u * K::kMs + k];
      }
      s.pair[k][qq] = col;
      s.pair[k][4 + qq] = blk;
    }
    __syncthreads();
    for (int t = tid; t < Qc; t += kThreads) {
      const float col = s.pair[t][0] + s.pair[t][1] + s.pair[t][2] + s.pair[t][3];
      const float blk = s.pair[t][4] + s.pair[t][5] + s.pair[t][6] + s.pair[t][7];
      s.dw[t] = fmaf(s.el[pb][t], s.nv[t], col + Mm[t * K::kMs + t]);
      s.nn[t] = s.el[pb][t] * s.w[pb][t] * s.nv[t];
      s.pair[t][0] = blk;  // S_t
    }
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (!ok) break;
  // The per-token tail on warp 0 while warps 1-7 begin the next unit (its
  // per-token arrays are the other buffer).
    if (warp == 0) {
      // dl_k = S_k + sum_{t >= k} (h_in term)_t + sum_{s < k} N_s + e_last <Lam, h_in>,
      // tokens k = lane and lane + 32, the sums as warp scans
      float lh = 0.f;
#pragma unroll
      for (int i = 0; i < kThreads / 32; ++i) lh += s.red[pb][i];
      const float e_last = s.seg[pb][last] == -1 ? expf(s.cs[pb][last]) : 0.f;
      const int k0 = lane, k1 = lane + 32;
      const bool v0 = k0 <= last, v1 = k1 <= last;
      const float n0 = v0 ? s.nn[k0] : 0.f, n1 = v1 ? s.nn[k1] : 0.f;
      const float h0v = v0 ? s.dcs[k0] : 0.f, h1v = v1 ? s.dcs[k1] : 0.f;
      float pre0 = n0, pre1 = n1, suf0 = h0v, suf1 = h1v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float a0 = __shfl_up_sync(0xffffffffu, pre0, o), a1 = __shfl_up_sync(0xffffffffu, pre1, o);
        const float b0 = __shfl_down_sync(0xffffffffu, suf0, o), b1 = __shfl_down_sync(0xffffffffu, suf1, o);
        if (lane >= o) pre0 += a0, pre1 += a1;
        if (lane + o < 32) suf0 += b0, suf1 += b1;
      }
      pre1 += __shfl_sync(0xffffffffu, pre0, 31);  // the first 32 tokens' total
      suf0 += __shfl_sync(0xffffffffu, suf1, 0);   // the last 32 tokens' total
      const float Ah = a.A[q.h];
      double dA = 0.0, dD = 0.0;
      if (v0) {
        const float dl = s.seg[pb][k0] == k0 ? 0.f : s.pair[k0][0] + suf0 + (pre0 - n0) + e_last * lh;
        a.ddt[(q.b * d.L + q.t0 + k0) * d.H + q.h] = fmaf(Ah, dl, s.dw[k0]);
        dA += (double)s.w[pb][k0] * (double)dl;
        dD += (double)s.dg[pb][k0];
      }
      if (v1) {
        const float dl = s.seg[pb][k1] == k1 ? 0.f : s.pair[k1][0] + suf1 + (pre1 - n1) + e_last * lh;
        a.ddt[(q.b * d.L + q.t0 + k1) * d.H + q.h] = fmaf(Ah, dl, s.dw[k1]);
        dA += (double)s.w[pb][k1] * (double)dl;
        dD += (double)s.dg[pb][k1];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        dA += __shfl_xor_sync(0xffffffffu, dA, o);
        dD += __shfl_xor_sync(0xffffffffu, dD, o);
      }
      if (lane == 0) {
        const int64_t pi = q.h * (d.b * d.nc) + q.b * d.nc + q.c;
        a.dA_part[pi] = dA;
        a.dD_part[pi] = dD;
      }
    }
  }
  if (!ok && warp == 0) {
    // a wait gave up: let this CTA's copies (the current unit's: the next
    // unit's are issued only after a unit went through) and MMAs finish
    // before its memory goes
    mbar_wait(&s.bar_st, (uint32_t)it & 1u, never, kLimit);
    mbar_wait(&s.bar_in, (uint32_t)it & 1u, never, kLimit);
    if (elect_one()) {
      mma_commit(&s.bar_drain);
      mbar_wait(&s.bar_drain, 0, never, kLimit);
    }
    __syncwarp();
  }
  if (tid == kStoreThread) bulk_wait_read<0>();  // the gradient stores have read their staging before the CTA's memory goes
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, K::kTmemCols);
}

// The chunk states and their scan in one pass: one CTA walks the chunks of
// one (batch row, head), forward or backward,
//
//   forward:  h_in(0) = h0,        h_in(c+1) = dec_c h_in(c) + S_c
//   backward: Lam(nc-1) = dfinal,  Lam(c-1)   = dec_c Lam(c) + T_c,   dh0 = Lam(-1)
//
// with the chunk's products (the formulas of k_bwd_chunk_states)
//
//   S_c = (diag(cS) x_c)^T B_c,   cS_t = dt_t E(last, t)
//   T_c = (diag(cT) dy_c)^T C_c,  cT_t = e_t
//
// formed by tcgen05 MMAs (M = 64 rows p, N = 128 states, K = 64 tokens) with
// the scaled x or dy as three bf16 terms, and the scans of k_bwd_state_passing;
// h_in goes to S and Lam to T, and the per-chunk products never reach memory.
// Roles
// (384 threads):
//   warp 0      TMA loads (one thread): x or dy, and B or C, 3 chunks ahead
//   warp 1      MMAs (one elected lane) into two 128-column accumulators
//   warps 2, 7  per-chunk scalars (dt_scan_from), alternate chunks each, their
//               loads issued two of their chunks ahead: the token scales, dec_c
//   warps 3-6   the scaled tile's three-term split, two chunks' terms in flight
//   warps 8-11  the state: warp 8 + q owns rows 16 q .. 16 q + 15 (TMEM lane
//               quadrant q) and all 128 states, in fp32 registers; each chunk's
//               entering state is staged (128-byte swizzled 32-column boxes)
//               and sent by bulk tensor stores, two stagings in flight
// Every wait is bounded; a CTA that gives up drains its copies, MMAs and
// stores, frees its tensor memory and exits.
struct WalkCfg {
  static constexpr int kThreads = 384;
  static constexpr int kRing = 3;  // input slots
  static constexpr int kScan = 4;  // per-chunk scalar slots
  // warps: 0 TMA, 1 MMA, 2 and 7 the scalars (alternate chunks), 3-6 the split, 8-11 the state
  static constexpr int kScanWarpA = 2, kScanWarpB = 7;
  static constexpr int kSplitWarp0 = 3, kSplitWarps = 4, kStateWarp0 = 8, kStateWarps = 4;
  static constexpr uint32_t kTile = 8192;
  static constexpr uint32_t kInSlot = 3 * kTile;  // x or dy [t][p], then B or C [t][n] (two n-blocks)
  static constexpr uint32_t oIn = 0;
  static constexpr uint32_t kTermSlot = 3 * kTile;  // the three terms [t][p]
  static constexpr uint32_t oTerms = oIn + kRing * kInSlot;
  static constexpr uint32_t kStageSlot = 4 * kTile;  // a state: four 32-column fp32 boxes
  static constexpr uint32_t oStage = oTerms + 2 * kTermSlot;
  static constexpr uint32_t oEnd = oStage + 2 * kStageSlot;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static constexpr uint32_t kTmemCols = 256;
};

struct __align__(16) WalkSmem {
  uint64_t full_in[WalkCfg::kRing], in_free[WalkCfg::kRing];
  uint64_t scan_full[WalkCfg::kScan], scan_empty[WalkCfg::kScan];
  uint64_t terms_full[2], terms_free[2];
  uint64_t mma_done[2], acc_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag, never;
  float f[WalkCfg::kScan][64];  // token scales: dt_t E(last, t) forward, e_t backward
  float dec[WalkCfg::kScan];    // the chunk's decay
};

// Grid: both directions of every (row, head) (blockIdx.x = 2 unit + dir), or
// only the backward ones (blockIdx.x = unit) when `both` is 0.
__global__ void __launch_bounds__(WalkCfg::kThreads, 1)
    k_bwd_state_walk_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dy,
                        const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                        const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_t,
                        const KArgs a, int both) {
  using K = WalkCfg;
  constexpr uint64_t kLimit = tc::kWaitLimitNs;
  const Dims& d = a.d;
  const uint32_t unit = both ? blockIdx.x >> 1 : blockIdx.x;  // b H + h
  const int dir = both ? (int)(blockIdx.x & 1) : 1;           // 0 forward (h_in), 1 backward (Lam)
  const uint32_t H = (uint32_t)d.H;
  const int64_t bb = unit / H, hh = unit - (uint32_t)bb * H, gg = (uint32_t)hh / (uint32_t)d.hpg;
  const int nc = (int)d.nc;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  __shared__ WalkSmem s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &s.abort_flag;
  volatile int* never = &s.never;
  const CUtensorMap* mX = dir ? &tm_dy : &tm_x;
  const CUtensorMap* mY = dir ? &tm_c : &tm_b;
  const CUtensorMap* mO = dir ? &tm_t : &tm_s;
  auto chunk_of = [&](int k) { return dir ? nc - 1 - k : k; };

  if (tid == 0) {
    for (int i = 0; i < K::kRing; ++i) {
      mbar_init(&s.full_in[i], 1);
      mbar_init(&s.in_free[i], K::kSplitWarps + 1);  // the split warps (x or dy) and the MMAs' commit (B or C)
    }
    for (int i = 0; i < K::kScan; ++i) {
      mbar_init(&s.scan_full[i], 1);
      mbar_init(&s.scan_empty[i], K::kSplitWarps + K::kStateWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.terms_full[i], K::kSplitWarps);
      mbar_init(&s.terms_free[i], 1);
      mbar_init(&s.mma_done[i], 1);
      mbar_init(&s.acc_free[i], K::kStateWarps);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    s.never = 0;
    fence_mbar_init();
    tma_prefetch_desc(mX);
    tma_prefetch_desc(mY);
    tma_prefetch_desc(mO);
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, K::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ TMA loads
    if (lane == 0) {
      int last = -1;
      for (int k = 0; k < nc; ++k) {
        const int sl = k % K::kRing;
        if (k >= K::kRing && !mbar_wait(&s.in_free[sl], ((k / K::kRing) - 1) & 1, abort_flag, kLimit)) break;
        const int tok = chunk_of(k) * 64;
        unsigned char* base = sm + K::oIn + sl * K::kInSlot;
        mbar_arrive_expect_tx(&s.full_in[sl], K::kInSlot);
        tma_load_3d(base, mX, &s.full_in[sl], (int)(hh * d.P), tok, (int)bb);
        for (int jb = 0; jb < 2; ++jb)
          tma_load_4d(base + (1 + jb) * K::kTile, mY, &s.full_in[sl], 64 * jb, (int)gg, tok, (int)bb);
        last = k;
      }
      if (*abort_flag)  // let the copies in flight land before the CTA's memory goes
        for (int k = last - (K::kRing - 1) < 0 ? 0 : last - (K::kRing - 1); k <= last; ++k)
          mbar_wait(&s.full_in[k % K::kRing], (k / K::kRing) & 1, never, kLimit);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMAs: S or T of chunk k = terms^T (B or C)
    constexpr uint32_t id = idesc_bf16(64, 128, 1, 1);  // A = terms^T (MN-major), B MN-major
    for (int k = 0; k < nc; ++k) {
      const int sl = k % K::kRing, ts = k & 1;
      bool ok = mbar_wait_warp(&s.full_in[sl], (k / K::kRing) & 1, abort_flag, kLimit);
      ok = ok && mbar_wait_warp(&s.terms_full[ts], (k >> 1) & 1, abort_flag, kLimit);
      if (ok && k >= 2) ok = mbar_wait_warp(&s.acc_free[ts], ((k >> 1) - 1) & 1, abort_flag, kLimit);
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t dY = sw128_desc(smem_u32(sm + K::oIn + sl * K::kInSlot + K::kTile), K::kTile, 1024);
#pragma unroll
        for (int t3 = 0; t3 < 3; ++t3) {
          const uint64_t xs = sw128_desc(smem_u32(sm + K::oTerms + ts * K::kTermSlot + t3 * K::kTile), K::kTile, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // K = tokens
            mma_bf16_ss(tmem + 128 * ts, mnmaj(xs, kk), mnmaj(dY, kk), id, t3 > 0 || kk > 0);
        }
        mma_commit(&s.mma_done[ts]);
        mma_commit(&s.in_free[sl]);
        mma_commit(&s.terms_free[ts]);
      }
      __syncwarp();
    }
    if (elect_one()) {  // every MMA (and its commits) done before the CTA's memory goes
      mma_commit(&s.drain);
      mbar_wait(&s.drain, 0, never, kLimit);
    }
    __syncwarp();
  } else if (warp == K::kScanWarpA || warp == K::kScanWarpB) {
    // ------------------------------------------------ per-chunk scalars
    // (this warp's chunks k0, k0 + 2, ..; the loads of chunk k + 4 are issued
    // before chunk k is scanned)
    const int k0 = warp == K::kScanWarpA ? 0 : 1;
    auto pos = [&](int k) {
      ChunkPos q;
      q.b = bb, q.h = hh, q.g = gg, q.c = chunk_of(k), q.t0 = q.c * d.Q;
      const int64_t left = d.L - q.t0;
      q.Qc = (int)(left < d.Q ? left : d.Q);
      return q;
    };
    const float Ah = a.A[hh];
    DtRaw r0{}, r1{};
    if (k0 < nc) r0 = dt_load(a, pos(k0), lane);
    if (k0 + 2 < nc) r1 = dt_load(a, pos(k0 + 2), lane);
    for (int k = k0; k < nc; k += 2) {
      const int ss = k % K::kScan;
      DtRaw r2{};
      if (k + 4 < nc) r2 = dt_load(a, pos(k + 4), lane);
      if (k >= K::kScan && !mbar_wait_warp(&s.scan_empty[ss], ((k / K::kScan) - 1) & 1, abort_flag, kLimit)) break;
      const ChunkPos q = pos(k);
      const int last = q.Qc - 1;
      const DtScan r = dt_scan_from(r0, q, Ah, lane);
      r0 = r1;
      r1 = r2;
#pragma unroll
      for (int e = 0; e < 2; ++e) s.f[ss][2 * lane + e] = dir ? r.ein[e] : r.w[e] * r.el[e];
      if (lane == (last >> 1)) s.dec[ss] = (last & 1) ? r.ein[1] : r.ein[0];  // 0 when a sequence starts inside
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.scan_full[ss]);
    }
  } else if (warp < K::kStateWarp0) {
    // ------------------------------------------------ the scaled tile's terms
    const int st = tid - 32 * K::kSplitWarp0;
    for (int k = 0; k < nc; ++k) {
      const int sl = k % K::kRing, ss = k % K::kScan, ts = k & 1;
      bool ok = mbar_wait_warp(&s.full_in[sl], (k / K::kRing) & 1, abort_flag, kLimit);
      ok = ok && mbar_wait_warp(&s.scan_full[ss], (k / K::kScan) & 1, abort_flag, kLimit);
      if (ok && k >= 2) ok = mbar_wait_warp(&s.terms_free[ts], ((k >> 1) - 1) & 1, abort_flag, kLimit);
      if (!ok) break;
      const unsigned char* X = sm + K::oIn + sl * K::kInSlot;
      unsigned char* terms = sm + K::oTerms + ts * K::kTermSlot;
      static_assert(64 * 8 == 4 * 32 * K::kSplitWarps, "four items a thread");
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // row t, 16-byte chunk k16 of p
        const int it = st + 32 * K::kSplitWarps * j;
        const int t = it >> 3, k16 = it & 7;
        float v[8];
        load8(X, t, k16, v);
        const float ft = s.f[ss][t];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= ft;
        store_terms8(terms, K::kTile, t, k16, v);
      }
      fence_proxy_async_smem();  // the terms are read by the MMAs
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s.terms_full[ts]);
        mbar_arrive(&s.in_free[sl]);
        mbar_arrive(&s.scan_empty[ss]);
      }
    }
  } else {
    // ------------------------------------------------ the state
    const int qd = warp & 3;
    const int row = 16 * qd + (lane & 15);  // state row p
    const int cb = 32 * (lane >> 4);        // states n = 64 h2 + cb + [0, 32), h2 = 0, 1
    const uint32_t tq = tmem + ((uint32_t)(32 * qd) << 16);
    const bool issuer = warp == K::kStateWarp0 && lane == 0;
    const int64_t e0 = ((int64_t)unit * d.P + row) * d.N + cb;
    const float* init = dir ? a.dfinal : a.h0;
    float hv[64];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
      for (int i = 0; i < 32; ++i) hv[32 * h2 + i] = init ? init[e0 + 64 * h2 + i] : 0.f;
    bool done = true;
    for (int k = 0; k < nc; ++k) {
      const int ab = k & 1, ss = k % K::kScan;
      unsigned char* stage = sm + K::oStage + ab * K::kStageSlot;
      if (issuer && k >= 2) bulk_wait_read<1>();  // the stores of chunk k - 2 have read this staging
      named_barrier_sync(1, 32 * K::kStateWarps);
      // the state entering (forward) or leaving (backward) chunk k: row `row`, a
      // whole 32-column row of boxes 2 h2 + cb / 32
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        unsigned char* box = stage + (uint32_t)(2 * h2 + (cb >> 5)) * K::kTile;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(box + sw_chunk(row, i)) =
              make_float4(hv[32 * h2 + 4 * i], hv[32 * h2 + 4 * i + 1], hv[32 * h2 + 4 * i + 2], hv[32 * h2 + 4 * i + 3]);
      }
      bool ok = mbar_wait_warp(&s.mma_done[ab], (k >> 1) & 1, abort_flag, kLimit);
      ok = ok && mbar_wait_warp(&s.scan_full[ss], (k / K::kScan) & 1, abort_flag, kLimit);
      if (ok) {
        tc_fence_after();
        const float dc = s.dec[ss];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t r[32];
          uint32_t* r_hi = r + 16;
          // warp-uniform address: lanes 16-31 read 32 columns further (cb)
          SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + 128 * ab + 64 * h2, r);
          SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + 128 * ab + 64 * h2 + 16, r_hi);
          SSD_TMEM_WAIT_LD_32(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) hv[32 * h2 + i] = fmaf(dc, hv[32 * h2 + i], __uint_as_float(r[i]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.acc_free[ab]);
          mbar_arrive(&s.scan_empty[ss]);
        }
      }
      fence_proxy_async_smem();  // the staged state is read by the bulk stores
      if (named_barrier_any(2, 32 * K::kStateWarps, !ok)) {
        done = false;
        break;
      }
      if (issuer) {
        const int u = (int)((int64_t)unit * nc + chunk_of(k));
        for (int j = 0; j < 4; ++j) tma_store_3d(mO, stage + j * K::kTile, 32 * j, 0, u);
        bulk_commit_group();
      }
    }
    if (done && dir == 1 && a.dh0)
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int i = 0; i < 32; ++i) a.dh0[e0 + 64 * h2 + i] = hv[32 * h2 + i];
    if (issuer) bulk_wait_read<0>();  // the stores have read their staging before the CTA's memory goes
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, K::kTmemCols);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

// The tensor-core kernels take bf16 calls without a gate at headdim 64, dstate
// 128 and 64-token chunks (TMA needs 16-byte aligned x, dy, B, C; the
// gradient stores are 16-byte vectors).
inline bool chunk_tc_supported(const KArgs& k) {
  const Dims& d = k.d;
  return d.P == 64 && d.N == 128 && d.Q == 64 && !k.z && aligned16(k.x) && aligned16(k.dy) && aligned16(k.B) &&
         aligned16(k.C) && aligned16(k.dx) && d.L < ((int64_t)1 << 31) && d.H * d.P < ((int64_t)1 << 31);
}

// the four tensor maps of the tensor-core kernels (x, dy, B, C)
inline bool chunk_tc_maps(const KArgs& k, CUtensorMap* tx, CUtensorMap* tdy, CUtensorMap* tb, CUtensorMap* tc_) {
  const Dims& d = k.d;
  return tc::make_map_3d(tx, k.x, d.H * d.P, d.L, d.b) && tc::make_map_3d(tdy, k.dy, d.H * d.P, d.L, d.b) &&
         tc::make_map_bc(tb, k.B, d.N, d.G, d.L, d.b) && tc::make_map_bc(tc_, k.C, d.N, d.G, d.L, d.b);
}

// The forward and backward state walks (only the backward one when just
// dLoss/dh0 is wanted): one CTA per (row, head) and direction.
inline cudaError_t state_walk_tc_launch(const KArgs& k, bool only_dh0, cudaStream_t st) {
  const Dims& d = k.d;
  CUtensorMap tx, tdy, tb, tc_, ts, tt;
  if (!chunk_tc_maps(k, &tx, &tdy, &tb, &tc_)) return cudaErrorInvalidValue;
  if (!tc::make_map_f32_blocks(&ts, k.S, d.N, d.P, d.b * d.H * d.nc) ||
      !tc::make_map_f32_blocks(&tt, k.T, d.N, d.P, d.b * d.H * d.nc))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_bwd_state_walk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)WalkCfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(d.b * d.H * (only_dh0 ? 1 : 2));
  k_bwd_state_walk_tc<<<grid, WalkCfg::kThreads, WalkCfg::kSmemBytes, st>>>(tx, tdy, tb, tc_, ts, tt, k,
                                                                            only_dh0 ? 0 : 1);
  return cudaGetLastError();
}

inline cudaError_t chunk_tc_launch(const KArgs& k, cudaStream_t st) {
  const Dims& d = k.d;
  CUtensorMap tx, tdy, tb, tc_, tdx, tdb, tdc;
  if (!chunk_tc_maps(k, &tx, &tdy, &tb, &tc_)) return cudaErrorInvalidValue;
  // the gradient tiles' bulk stores: dx (b, L, H, P) and the per-head dB, dC (b, L, H, N), fp32
  if (!tc::make_map_f32_tiles(&tdx, k.dx, d.P, d.H, d.L, d.b) || !tc::make_map_f32_tiles(&tdb, k.dBh, d.N, d.H, d.L, d.b) ||
      !tc::make_map_f32_tiles(&tdc, k.dCh, d.N, d.H, d.L, d.b))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_bwd_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)TcCfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int64_t units = d.b * d.nc * d.H;  // a persistent grid, one CTA an SM, walking the units
  const unsigned grid = (unsigned)(units < sms ? units : sms);
  k_bwd_chunk_tc<<<grid, kThreads, TcCfg::kSmemBytes, st>>>(tx, tdy, tb, tc_, tdx, tdb, tdc, k);
  return cudaGetLastError();
}

}  // namespace bwd
}  // namespace ssd
