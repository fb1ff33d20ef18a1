// Fast fused chunked SSD forward on sm_100a (tcgen05 + TMEM + TMA), for the
// common case where every chunk's decay range is moderate.
//
// Two kernels:
//
// k_chunk_cb (one CTA per batch row, chunk, B/C group): the head-independent
//   part of the intra-chunk "attention",
//       W'[t][s] = C_t . B_s  if s <= t, both tokens valid and in the same
//                             packed sequence, else 0          (bf16, 64 x 64)
//   (the masked C B^T of the dual form, "22 · Mamba 2 — Transformers are
//   SSMs" section 3.2), computed once and shared by all heads of the group.
//   It also flags, per (chunk, head), whether the chunk's in-chunk cumulative
//   decay stays within +-kRangeLog2 of its midpoint value (see below).
//
// k_ssd_fwd_fast (one CTA per (batch row, head), chunks in order, the running
//   state kept on chip).  With cs_t the in-chunk cumulative sum of dt*A (log2
//   units) and m = cs at the chunk's midpoint, the decay between tokens s <= t
//   factorises as exp2(cs_t - cs_s) = u_t v_s / dt_s with
//       u_t = exp2(cs_t - m),   v_s = exp2(m - cs_s) dt_s,
//   both within 2^+-kRangeLog2 when the chunk is flagged in range.  Then
//       X'  = diag(v) X                                      (one scaling pass)
//       Yd  = W' X' + C (e^m H_c)^T                          (one accumulator)
//       y_t = u_t Yd_t + D_h x_t
//       S'  = B^T X',   H_{c+1} = exp2(cs_e) H_c + exp2(cs_e - m) S'
//   which are the four chunked steps of "SSM 家族全景图（下）：Mamba-2 与 Jamba"
//   section 三.4: the intra-chunk output (W' X' scaled by u), the chunk state
//   (S'), the state passing (H), and the correction from the chunk's true
//   initial state (the C H^T term, whose per-row factor exp2(cs_t) equals
//   u_t e^m).  A (batch row, head) unit with any chunk out of range is left to
//   the exact kernel (ssd_tc.cu), which forms every decay separately.
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 MMA issuer (one
// thread), warps 2-9 compute.  W'/x tiles, Yd, S and the bf16 state copy are
// double-buffered so chunk c's MMAs overlap chunk c-1's state update and
// epilogue.  Every wait is bounded; a CTA that times out records the error,
// drains its copies and MMAs, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "ssd_internal.h"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

using namespace sm100;
using namespace tc;

// ============================================================== k_chunk_cb
template <int NS>
struct CbCfg {
  static constexpr int NB = NS / 64;
  static constexpr uint32_t kTile = 8192;
  static constexpr uint32_t oC = 0, oB = NB * kTile, oEnd = 2 * NB * kTile;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
};

template <int NS>
__global__ void __launch_bounds__(128) k_chunk_cb(const __grid_constant__ CUtensorMap tm_b,
                                                 const __grid_constant__ CUtensorMap tm_c, const CbArgs a) {
  using K = CbCfg<NS>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  __shared__ uint64_t bar_full, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int never;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t r = blockIdx.x;
  const int64_t g = r % a.G;
  const int64_t c = (r / a.G) % a.nc;
  const int64_t b = r / (a.G * a.nc);
  const int t0 = (int)(c * 64);
  const int nvalid = (int)((c + 1) * 64 <= a.L ? 64 : a.L - t0);
  const int64_t rowbase = b * a.L;

  if (tid == 0) {
    mbar_init(&bar_full, 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    never = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  volatile int* abort_p = &abort_flag;

  if (tid == 0) {
    mbar_arrive_expect_tx(&bar_full, 2 * K::NB * K::kTile);
    for (int j = 0; j < K::NB; ++j) {
      tma_load_3d(sm + K::oC + j * K::kTile, &tm_c, &bar_full, (int)(g * NS + 64 * j), t0, (int)b);
      tma_load_3d(sm + K::oB + j * K::kTile, &tm_b, &bar_full, (int)(g * NS + 64 * j), t0, (int)b);
    }
    if (mbar_wait(&bar_full, 0, abort_p, kWaitLimitNs)) {
      tc_fence_after();
      const uint32_t aC = smem_u32(sm + K::oC), aB = smem_u32(sm + K::oB);
      constexpr uint32_t id = idesc_bf16(64, 64, 0, 0);
#pragma unroll
      for (int kk = 0; kk < NS / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * K::kTile + (kk & 3) * 32;
        mma_bf16_ss(tmem, sw128_desc(aC + koff, 16, 1024), sw128_desc(aB + koff, 16, 1024), id, kk > 0);
      }
    } else {
      mbar_wait(&bar_full, 0, (volatile int*)&never, kWaitLimitNs);  // let the copies land
    }
    mma_commit(&bar_mma);
  }
  __syncwarp();

  // per-(chunk, head) range flags: warp w handles heads w, w+4, ... of the group
  for (int64_t hh = warp; hh < a.hpg; hh += 4) {
    const int64_t h = g * a.hpg + hh;
    const float a2 = a.A[h] * kLog2e;
    float x0 = 0.f, x1 = 0.f;
    const int i0 = 2 * lane, i1 = 2 * lane + 1;
    if (i0 < nvalid) x0 = a.dt[(rowbase + t0 + i0) * a.H + h] * a2;
    if (i1 < nvalid) x1 = a.dt[(rowbase + t0 + i1) * a.H + h] * a2;
    float v = x0 + x1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    const float cs1 = v, cs0 = v - x1;  // inclusive sums at tokens 2l+1 and 2l
    const float mid = __shfl_sync(0xffffffffu, cs1, 15);  // token 31
    float dev = fmaxf(fabsf(cs0 - mid), fabsf(cs1 - mid));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
    if (lane == 0) a.ok[(b * a.nc + c) * a.H + h] = (dev <= kRangeLog2) ? 1 : 0;
  }

  // W' = masked C B^T -> bf16, row-major 64 x 64 per (b, c, g)
  const bool ok = mbar_wait(&bar_mma, 0, abort_p, kWaitLimitNs);
  tc_fence_after();
  if (ok) {
    const int q = warp;
    uint32_t rr[32];
    SSD_TMEM_LD_16x32bx2_X32_HALF32(tmem + ((uint32_t)(32 * q) << 16), rr);
    SSD_TMEM_WAIT_LD_32(rr);
    const int t = 16 * q + (lane & 15);
    const int s0 = 32 * (lane >> 4);
    const int seq_t = (a.seq && t < nvalid) ? a.seq[rowbase + t0 + t] : 0;
    uint32_t packed[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      float w2[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int sc = s0 + j + u;
        bool keep = t < nvalid && sc <= t;
        if (keep && a.seq) keep = a.seq[rowbase + t0 + sc] == seq_t;
        w2[u] = keep ? __uint_as_float(rr[j + u]) : 0.f;
      }
      packed[j >> 1] = pack_bf16x2(w2[0], w2[1]);
    }
    uint4* dst = reinterpret_cast<uint4*>(a.wp + (r * 64 + t) * 64 + s0);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_p && tid == 0) atomicExch(a.err, 1);
  if (warp == 0) tmem_dealloc(tmem, 64);
}

// ============================================================== k_ssd_fwd_fast
template <int NS>
struct FastCfg {
  static constexpr int NB = NS / 64, NH = NS / 128;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTile = 8192;
  static constexpr uint32_t oW = 0;                    // [2] W' tiles
  static constexpr uint32_t oX = oW + 2 * kTile;       // [2] x tiles
  static constexpr uint32_t oC = oX + 2 * kTile;       // C, NB tiles
  static constexpr uint32_t oB = oC + NB * kTile;      // B, NB tiles
  static constexpr uint32_t oXp = oB + NB * kTile;     // X' = diag(v) x
  static constexpr uint32_t oH = oXp + kTile;          // [2] bf16 e^m H, NB tiles each
  static constexpr uint32_t oEnd = oH + 2 * NB * kTile;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  // TMEM columns: Yd[2] (M = 64 layout) then S^T[2] (M = 128 rows per half)
  static constexpr uint32_t tYd0 = 0, tS0 = 128;
  static constexpr uint32_t kSCols = 64 * NH;
  static constexpr uint32_t kTmemCols = NS <= 128 ? 256 : 512;
  static constexpr int kMinBlocks = NS <= 128 ? 2 : 1;
};

struct __align__(8) FastSmem {
  uint64_t full_x[2], empty_x[2], full_cb, cb_free, xp_ready, xp_free;
  uint64_t s_full[2], s_free[2], h_ready[2], h_free[2], y_full[2], y_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int never;
  float cs2[64];
  float u[2][64];
  float v[64];
  float sc[2][4];  // per chunk parity: E = 2^m, f = 2^(cs_e - m), d = 2^cs_e
  float warp_tot;
};

template <int NS>
__global__ void __launch_bounds__(320, FastCfg<NS>::kMinBlocks)
    k_ssd_fwd_fast(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_w,
                   const FastArgs a) {
  using K = FastCfg<NS>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  __shared__ FastSmem s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t unit = blockIdx.x;
  const int64_t b = unit / a.H, h = unit % a.H;
  const int64_t g = h / a.hpg;
  const int nc = (int)a.nc;

  // units with any chunk out of the factorisable range belong to the exact kernel
  bool in_range = true;
  for (int c = tid; c < nc; c += blockDim.x) in_range &= a.ok[(b * a.nc + c) * a.H + h] != 0;
  if (!__syncthreads_and(in_range)) return;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full_x[i], 1);
      mbar_init(&s.empty_x[i], 1 + 256);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_free[i], 256);
      mbar_init(&s.h_ready[i], 256);
      mbar_init(&s.h_free[i], 1);
      mbar_init(&s.y_full[i], 1);
      mbar_init(&s.y_free[i], 256);
    }
    mbar_init(&s.full_cb, 1);
    mbar_init(&s.cb_free, 1);
    mbar_init(&s.xp_ready, 256);
    mbar_init(&s.xp_free, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = *reinterpret_cast<volatile int*>(a.err) != 0;
    s.never = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, K::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort_flag = &s.abort_flag;
  volatile int* never = &s.never;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_x = -1, last_cb = -1;
      for (int c = 0; c < nc; ++c) {
        const int i = c & 1;
        const int t0 = c * 64;
        if (c >= 2 && !mbar_wait(&s.empty_x[i], ((c - 2) >> 1) & 1, abort_flag, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&s.full_x[i], 2 * K::kTile);
        tma_load_3d(sm + K::oW + i * K::kTile, &tm_w, &s.full_x[i], 0, (int)(((b * a.nc + c) * a.G + g) * 64), 0);
        tma_load_3d(sm + K::oX + i * K::kTile, &tm_x, &s.full_x[i], (int)(h * 64), t0, (int)b);
        last_x = c;
        if (c >= 1 && !mbar_wait(&s.cb_free, (c - 1) & 1, abort_flag, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&s.full_cb, 2 * K::NB * K::kTile);
        for (int j = 0; j < K::NB; ++j) {
          tma_load_3d(sm + K::oC + j * K::kTile, &tm_c, &s.full_cb, (int)(g * NS + 64 * j), t0, (int)b);
          tma_load_3d(sm + K::oB + j * K::kTile, &tm_b, &s.full_cb, (int)(g * NS + 64 * j), t0, (int)b);
        }
        last_cb = c;
      }
      if (*abort_flag) {  // let this CTA's own copies land before its smem is released
        if (last_x >= 0) mbar_wait(&s.full_x[last_x & 1], (last_x >> 1) & 1, never, kWaitLimitNs);
        if (last_cb >= 0) mbar_wait(&s.full_cb, last_cb & 1, never, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t aW = smem_u32(sm + K::oW), aC = smem_u32(sm + K::oC), aB = smem_u32(sm + K::oB);
      const uint32_t aXp = smem_u32(sm + K::oXp), aH = smem_u32(sm + K::oH);
      constexpr uint32_t id_64 = idesc_bf16(64, 64, 0, 1);    // A K-major, B MN-major, M = 64
      constexpr uint32_t id_st = idesc_bf16(128, 64, 1, 1);   // both MN-major, M = 128
      for (int c = 0; c < nc; ++c) {
        const int i = c & 1;
        const uint32_t pb = (c >> 1) & 1, ps = c & 1, pp = ((c - 2) >> 1) & 1;
        bool ok = mbar_wait(&s.full_x[i], pb, abort_flag, kWaitLimitNs);
        ok = ok && mbar_wait(&s.xp_ready, ps, abort_flag, kWaitLimitNs);
        ok = ok && mbar_wait(&s.full_cb, ps, abort_flag, kWaitLimitNs);
        if (c >= 2) {
          ok = ok && mbar_wait(&s.y_free[i], pp, abort_flag, kWaitLimitNs);
          ok = ok && mbar_wait(&s.s_free[i], pp, abort_flag, kWaitLimitNs);
        }
        if (!ok) break;
        tc_fence_after();
        const uint32_t yd = tmem + K::tYd0 + 64 * i;
        const uint32_t st = tmem + K::tS0 + K::kSCols * i;
        // Yd = W' X'   (K = 64 tokens)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(yd, sw128_desc(aW + i * K::kTile + kk * 32, 16, 1024),
                      sw128_desc(aXp + kk * 2048, K::kTile, 1024), id_64, kk > 0);
        // S'^T = B^T X'   (M = 128 state rows per half, K = 64 tokens)
#pragma unroll
        for (int hf = 0; hf < K::NH; ++hf)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(st + 64 * hf, sw128_desc(aB + hf * 2 * K::kTile + kk * 2048, K::kTile, 1024),
                        sw128_desc(aXp + kk * 2048, K::kTile, 1024), id_st, kk > 0);
        mma_commit(&s.s_full[i]);
        mma_commit(&s.xp_free);
        // Yd += C (e^m H_c)^T   (K = N)
        if (!mbar_wait(&s.h_ready[i], pb, abort_flag, kWaitLimitNs)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * K::kTile + (kk & 3) * 32;
          mma_bf16_ss(yd, sw128_desc(aC + koff, 16, 1024),
                      sw128_desc(aH + i * K::NB * K::kTile + kk * 2048, K::kTile, 1024), id_64, 1);
        }
        mma_commit(&s.y_full[i]);
        mma_commit(&s.h_free[i]);
        mma_commit(&s.cb_free);
        mma_commit(&s.empty_x[i]);
      }
      mma_commit(&s.drain);
      mbar_wait(&s.drain, 0, never, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int wt = tid - 64;            // 0..255
    const int q = warp & 3;             // TMEM lane quadrant
    const int hq = (warp - 2) >> 2;     // which half of the 64 columns
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    const float a2 = a.A[h] * kLog2e;
    const float dskip = a.D ? a.D[h] : 0.f;
    const int64_t rowbase = b * a.L;
    const int n0 = 32 * q + lane;       // state row(s): n0 (+128)
    const int pc0 = 32 * hq;            // state columns [pc0, pc0 + 32)
    float H[K::NH][32];
#pragma unroll
    for (int hf = 0; hf < K::NH; ++hf)
#pragma unroll
      for (int j = 0; j < 32; ++j)
        H[hf][j] = a.h0 ? a.h0[((b * a.H + h) * 64 + pc0 + j) * NS + n0 + 128 * hf] : 0.f;

    float dt_next = 0.f;
    if (wt < 64 && wt < a.L) dt_next = a.dt[(rowbase + wt) * a.H + h];
    float d_prev = 0.f, f_prev = 0.f;  // chunk c-1 scalars
    bool failed = false;

    for (int c = 0; c <= nc; ++c) {
      if (named_barrier_any(2, 256, failed)) {
        failed = true;
        break;
      }
      float E_c = 0.f;
      if (c < nc) {
        const int i = c & 1;
        const int t0 = c * 64;
        const int nvalid = (int)((int64_t)(c + 1) * 64 <= a.L ? 64 : a.L - t0);
        // ---- in-chunk cumulative sum and the factor vectors u, v
        if (wt < 64) {
          const float dtv = wt < nvalid ? dt_next : 0.f;
          if ((int64_t)t0 + 64 + wt < a.L) dt_next = a.dt[(rowbase + t0 + 64 + wt) * a.H + h];
          float x = dtv * a2;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += u;
          }
          if (wt == 31) s.warp_tot = x;
          named_barrier_sync(1, 256);
          if (wt >= 32) x += s.warp_tot;
          s.cs2[wt] = x;
          named_barrier_sync(1, 256);
          const float m = s.cs2[31];
          const float cse = s.cs2[nvalid - 1];
          s.u[i][wt] = exp2f(x - m);
          s.v[wt] = exp2f(m - x) * dtv;
          if (wt == 0) {
            s.sc[i][0] = exp2f(m);
            s.sc[i][1] = exp2f(cse - m);
            s.sc[i][2] = exp2f(cse);
          }
        } else {
          named_barrier_sync(1, 256);
          named_barrier_sync(1, 256);
        }
        named_barrier_sync(1, 256);
        E_c = s.sc[i][0];
        // ---- X' = diag(v) x for chunk c
        if (!mbar_wait(&s.full_x[i], (c >> 1) & 1, abort_flag, kWaitLimitNs) ||
            (c >= 1 && !mbar_wait(&s.xp_free, (c - 1) & 1, abort_flag, kWaitLimitNs))) {
          failed = true;
          continue;
        }
        {
          const int srow = wt >> 2, j4 = wt & 3;
          const float w = s.v[srow];
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const uint32_t off = sw128((uint32_t)srow * 128 + (2 * j4 + jj) * 16);
            uint4 vv = *reinterpret_cast<const uint4*>(sm + K::oX + i * K::kTile + off);
            float f0, f1;
            unpack_bf16x2(vv.x, f0, f1);
            vv.x = pack_bf16x2(f0 * w, f1 * w);
            unpack_bf16x2(vv.y, f0, f1);
            vv.y = pack_bf16x2(f0 * w, f1 * w);
            unpack_bf16x2(vv.z, f0, f1);
            vv.z = pack_bf16x2(f0 * w, f1 * w);
            unpack_bf16x2(vv.w, f0, f1);
            vv.w = pack_bf16x2(f0 * w, f1 * w);
            *reinterpret_cast<uint4*>(sm + K::oXp + off) = vv;
          }
          fence_proxy_async_smem();
          mbar_arrive(&s.xp_ready);
        }
      }
      // ---- state update for chunk c-1, then publish e^m H_c for chunk c
      if (c >= 1) {
        const int ip = (c - 1) & 1;
        if (!mbar_wait(&s.s_full[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          continue;
        }
        tc_fence_after();
#pragma unroll
        for (int hf = 0; hf < K::NH; ++hf) {
          uint32_t r[32];
          SSD_TMEM_LD_32x32b_X32(tq + K::tS0 + K::kSCols * ip + 64 * hf + pc0, r);
          SSD_TMEM_WAIT_LD_32(r);
#pragma unroll
          for (int j = 0; j < 32; ++j) H[hf][j] = fmaf(d_prev, H[hf][j], f_prev * __uint_as_float(r[j]));
        }
        tc_fence_before();
        mbar_arrive(&s.s_free[ip]);
      }
      if (c < nc) {
        const int i = c & 1;
        if (c >= 2 && !mbar_wait(&s.h_free[i], ((c - 2) >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          continue;
        }
#pragma unroll
        for (int hf = 0; hf < K::NH; ++hf) {
          const uint32_t row = (uint32_t)(n0 + 128 * hf);
          unsigned char* base = sm + K::oH + i * K::NB * K::kTile + row * 128;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint4 vv;
            vv.x = pack_bf16x2(E_c * H[hf][8 * jj + 0], E_c * H[hf][8 * jj + 1]);
            vv.y = pack_bf16x2(E_c * H[hf][8 * jj + 2], E_c * H[hf][8 * jj + 3]);
            vv.z = pack_bf16x2(E_c * H[hf][8 * jj + 4], E_c * H[hf][8 * jj + 5]);
            vv.w = pack_bf16x2(E_c * H[hf][8 * jj + 6], E_c * H[hf][8 * jj + 7]);
            const uint32_t chunk = (uint32_t)(pc0 / 8 + jj);
            *reinterpret_cast<uint4*>(base + ((chunk ^ (row & 7)) << 4)) = vv;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&s.h_ready[i]);
      }
      // ---- epilogue for chunk c-1: y = u_t Yd + D x
      if (c >= 1) {
        const int ip = (c - 1) & 1;
        const int t0p = (c - 1) * 64;
        const int nvp = (int)((int64_t)c * 64 <= a.L ? 64 : a.L - t0p);
        if (!mbar_wait(&s.y_full[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          continue;
        }
        tc_fence_after();
        uint32_t r[16];
        SSD_TMEM_LD_16x32bx2_X16_HALF32(tq + K::tYd0 + 64 * ip + 16 * hq, r);
        SSD_TMEM_WAIT_LD_16(r);
        tc_fence_before();
        mbar_arrive(&s.y_free[ip]);
        const int t = 16 * q + (lane & 15);
        const int p0 = 16 * hq + 32 * (lane >> 4);
        if (t < nvp) {
          const float ut = s.u[ip][t];
          const unsigned char* xrow = sm + K::oX + ip * K::kTile + (uint32_t)t * 128;
          uint32_t packed[8];
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const uint32_t chunk = (uint32_t)(p0 / 8 + jj);
            const uint4 xv = *reinterpret_cast<const uint4*>(xrow + ((chunk ^ (t & 7)) << 4));
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float x0, x1;
              unpack_bf16x2(xw[k], x0, x1);
              const int j = 8 * jj + 2 * k;
              packed[4 * jj + k] = pack_bf16x2(fmaf(ut, __uint_as_float(r[j]), dskip * x0),
                                               fmaf(ut, __uint_as_float(r[j + 1]), dskip * x1));
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(a.y + ((rowbase + t0p + t) * a.H + h) * 64 + p0);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        mbar_arrive(&s.empty_x[ip]);
      }
      if (c < nc) {
        d_prev = s.sc[c & 1][2];
        f_prev = s.sc[c & 1][1];
      }
    }
    if (!failed && a.final_states) {
#pragma unroll
      for (int hf = 0; hf < K::NH; ++hf) {
        float* dst = a.final_states + ((b * a.H + h) * 64 + pc0) * NS + n0 + 128 * hf;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(int64_t)j * NS] = H[hf][j];
      }
    }
  }

  if (*abort_flag && tid == 0) atomicExch(a.err, 1);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, K::kTmemCols);
}

template <int NS>
cudaError_t launch_fast(const Problem& p, const TcWorkspace& w, cudaStream_t st) {
  CUtensorMap tx, tb, tc_, tw;
  if (!make_map_3d(&tx, p.x, p.H * p.P, p.L, p.b) || !make_map_3d(&tb, p.B, p.G * p.N, p.L, p.b) ||
      !make_map_3d(&tc_, p.C, p.G * p.N, p.L, p.b) || !make_map_3d(&tw, w.wp, 64, p.b * p.nc * p.G * 64, 1))
    return cudaErrorInvalidValue;
  CbArgs ca;
  ca.L = p.L;
  ca.H = p.H;
  ca.G = p.G;
  ca.hpg = p.hpg;
  ca.nc = p.nc;
  ca.dt = p.dt;
  ca.A = p.A;
  ca.seq = p.seq;
  ca.wp = w.wp;
  ca.ok = w.ok;
  ca.err = w.err;
  cudaError_t e = cudaFuncSetAttribute(k_chunk_cb<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)CbCfg<NS>::kSmemBytes);
  if (e != cudaSuccess) return e;
  k_chunk_cb<NS><<<(unsigned)(p.b * p.nc * p.G), 128, CbCfg<NS>::kSmemBytes, st>>>(tb, tc_, ca);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  FastArgs fa;
  fa.L = p.L;
  fa.H = p.H;
  fa.G = p.G;
  fa.hpg = p.hpg;
  fa.nc = p.nc;
  fa.dt = p.dt;
  fa.A = p.A;
  fa.D = p.D;
  fa.h0 = p.h0;
  fa.y = static_cast<__nv_bfloat16*>(p.y);
  fa.final_states = p.final_states;
  fa.ok = w.ok;
  fa.err = w.err;
  e = cudaFuncSetAttribute(k_ssd_fwd_fast<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)FastCfg<NS>::kSmemBytes);
  if (e != cudaSuccess) return e;
  k_ssd_fwd_fast<NS><<<(unsigned)(p.b * p.H), FastCfg<NS>::kThreads, FastCfg<NS>::kSmemBytes, st>>>(tx, tb, tc_,
                                                                                                      tw, fa);
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_fast_forward(const Problem& p, const TcWorkspace& w, cudaStream_t st) {
  return p.N == 128 ? launch_fast<128>(p, w, st) : launch_fast<256>(p, w, st);
}

}  // namespace ssd
