// Two-head variant of the fast fused SSD forward (see ssd_tc_fast.cu for the
// factorised-decay formulation): one CTA owns two heads (h, h+1) of the same
// batch row and B/C group and walks their chunks together.  The heads share
// the C, B and W' = masked C B^T tiles, and every MMA covers both heads at
// once with N = 128:
//
//   Yd   = W' [X'_h | X'_h+1]                     (M = 64 tokens,  K = 64 tokens)
//   S'^T = B^T [X'_h | X'_h+1]                    (M = 128 states, K = 64 tokens)
//   Yd  += C [e^m H_h | e^m H_h+1]^T              (M = 64 tokens,  K = N)
//   y_t  = u_t Yd_t + D x_t,   H <- exp2(cs_e) H + exp2(cs_e - m) S'
//
// (per head; u, v, m, cs as in ssd_tc_fast.cu).  The chunked steps are those
// of "SSM 家族全景图（下）：Mamba-2 与 Jamba" section 三.4; the D feed-through
// is from "从Transformer的二次复杂度困境到Mamba的线性突围" (continuous SSM).
//
// The D x_t feed-through is taken from the scaled tile: D x_t = (D / v_t) X'_t,
// so the epilogue needs no second read of x.  It writes y over X' in the
// same shared-memory slot (each thread overwrites exactly what it read) and
// one TMA store per head moves the tile out.
//
// Warp roles (448 threads): warp 0 scans both heads' cumulative sums two
// chunks ahead and issues the TMA loads; warp 1 issues the MMAs (one
// thread); warps 2-5 scale both heads' x tiles into X' in place; warps 6-9
// and 10-13 each own one head: state update (fp32 state in registers),
// publishing the bf16 e^m H tile, and the epilogue.  x tiles sit in a
// 4-deep ring, loaded 3 chunks ahead and freed once the y tile stored from
// the same slot has been read out; W', B, C, the e^m H tiles, Yd and S are
// double-buffered.  Every wait is bounded; a CTA that times out records the
// error, drains its copies, stores and MMAs, frees its TMEM and exits.
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

struct PairCfg {
  static constexpr int NS = 128, NB = 2;
  static constexpr int kThreads = 448;
  static constexpr uint32_t kTile = 8192;
  static constexpr int kXSlots = 4;
  static constexpr uint32_t oX = 0;                        // [4 slots][2 heads] x -> X' -> y, in place
  static constexpr uint32_t oW = oX + 2 * kXSlots * kTile; // [2] W' tiles
  static constexpr uint32_t oB = oW + 2 * kTile;           // [2] B, 2 n-blocks each
  static constexpr uint32_t oC = oB + 2 * NB * kTile;      // [2] C, 2 n-blocks each
  static constexpr uint32_t oH = oC + 2 * NB * kTile;      // [2 bufs][2 heads] e^m H, 16 KB each
  static constexpr uint32_t kHTile = NB * kTile;
  static constexpr uint32_t oEnd = oH + 4 * kHTile;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  // TMEM: Yd[2] at 0 / 128 (M = 64 layout, head j in columns 64j..64j+63),
  //       S[2]  at 256 / 384 (M = 128 layout, head j in columns 64j..)
  static constexpr uint32_t tYd0 = 0, tS0 = 256, kTmemCols = 512;
};

struct __align__(8) PairSmem {
  uint64_t full_x[4], x_empty[4], full_w[2], w_empty[2], full_b[2], b_free[2], full_c[2], c_free[2];
  // Ring barriers are indexed like the buffers they guard, so no barrier can
  // complete a second phase before every waiter has seen the first.
  uint64_t scan_full[4], scan_empty[4], xp_ready[4], h_ready[2];
  uint64_t h_free[2], s_full[2], s_free[2], y_full[2], y_free[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int never;
  int unit_bad;
  float u[4][2][64];
  float v[4][2][64];
  float g[4][2][64];  // D / v_t: D x_t = g_t X'_t
  float sc[4][2][4];  // E = 2^m, f = 2^(cs_e - m), d = 2^cs_e
};

__global__ void __launch_bounds__(448, 1)
    k_ssd_fwd_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_y, const FastArgs a) {
  using K = PairCfg;
  constexpr int NS = K::NS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  __shared__ PairSmem s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t pairs = a.H / 2;
  const int64_t b = blockIdx.x / pairs;
  const int64_t h0 = (blockIdx.x % pairs) * 2;  // heads h0, h0 + 1
  const int64_t g = h0 / a.hpg;
  const int nc = (int)a.nc;
  const int64_t rowbase = b * a.L;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s.scan_full[i], 32);
      mbar_init(&s.scan_empty[i], 256);
    }
    for (int i = 0; i < K::kXSlots; ++i) {
      mbar_init(&s.full_x[i], 1);
      mbar_init(&s.x_empty[i], 2);  // one store-issuing thread per head
      mbar_init(&s.xp_ready[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full_b[i], 1);
      mbar_init(&s.b_free[i], 1);
      mbar_init(&s.full_w[i], 1);
      mbar_init(&s.w_empty[i], 1);
      mbar_init(&s.full_c[i], 1);
      mbar_init(&s.c_free[i], 1);
      mbar_init(&s.h_free[i], 1);
      mbar_init(&s.h_ready[i], 256);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_free[i], 256);
      mbar_init(&s.y_full[i], 1);
      mbar_init(&s.y_free[i], 256);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = *reinterpret_cast<volatile int*>(a.err) != 0;
    s.never = 0;
    s.unit_bad = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_y);
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
    // ------------------------------------------------ scans + TMA producer warp
    float a2[2], p0[2], p1[2], dsk[2];
    for (int j = 0; j < 2; ++j) {
      a2[j] = a.A[h0 + j] * kLog2e;
      dsk[j] = a.D ? a.D[h0 + j] : 0.f;
    }
    auto load_dt = [&](int c) {
      const int64_t t = (int64_t)c * 64 + 2 * lane;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        p0[j] = (c < nc && t < a.L) ? a.dt[(rowbase + t) * a.H + h0 + j] : 0.f;
        p1[j] = (c < nc && t + 1 < a.L) ? a.dt[(rowbase + t + 1) * a.H + h0 + j] : 0.f;
      }
    };
    load_dt(0);
    int scanned = 0;
    auto scan_next = [&]() -> bool {
      const int c = scanned;
      const int slot = c & 3;
      if (c >= 4 && !mbar_wait(&s.scan_empty[slot], ((c - 4) >> 2) & 1, abort_flag, kWaitLimitNs)) return false;
      float d0[2], d1[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        d0[j] = p0[j];
        d1[j] = p1[j];
      }
      const int nvalid = (int)((int64_t)(c + 1) * 64 <= a.L ? 64 : a.L - (int64_t)c * 64);
      const int e = nvalid - 1;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float x0 = d0[j] * a2[j], x1 = d1[j] * a2[j];
        float v = x0 + x1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        const float cs1 = v, cs0 = v - x1;
        const float m = __shfl_sync(0xffffffffu, cs1, 15);  // token 31
        const float cse = __shfl_sync(0xffffffffu, (e & 1) ? cs1 : cs0, e >> 1);
        float dev = fmaxf(fabsf(cs0 - m), fabsf(cs1 - m));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
        const float v0 = exp2f(m - cs0) * d0[j], v1 = exp2f(m - cs1) * d1[j];
        const float g0 = dsk[j] != 0.f ? dsk[j] / v0 : 0.f, g1 = dsk[j] != 0.f ? dsk[j] / v1 : 0.f;
        // D x_t is recovered from X'_t = v_t x_t, so a valid token needs a finite D / v_t
        const bool gbad = (2 * lane < nvalid && !(fabsf(g0) < INFINITY)) ||
                          (2 * lane + 1 < nvalid && !(fabsf(g1) < INFINITY));
        if (!(dev <= kRangeLog2) || gbad) s.unit_bad = 1;
        s.u[slot][j][2 * lane] = exp2f(cs0 - m);
        s.u[slot][j][2 * lane + 1] = exp2f(cs1 - m);
        s.v[slot][j][2 * lane] = v0;
        s.v[slot][j][2 * lane + 1] = v1;
        s.g[slot][j][2 * lane] = g0;
        s.g[slot][j][2 * lane + 1] = g1;
        if (lane == 0) {
          s.sc[slot][j][0] = exp2f(m);
          s.sc[slot][j][1] = exp2f(cse - m);
          s.sc[slot][j][2] = exp2f(cse);
        }
      }
      mbar_arrive(&s.scan_full[slot]);
      // the next chunk's dt is fetched only now: a release arrive waits for this
      // thread's loads in flight, which would otherwise stall it for a full load
      load_dt(c + 1);
      ++scanned;
      return true;
    };
    int last_x = -1, last_w = -1, last_b = -1, last_c = -1;
    auto issue_x = [&](int c) {
      const int sl = c & 3;
      mbar_arrive_expect_tx(&s.full_x[sl], 2 * K::kTile);
      for (int j = 0; j < 2; ++j)
        tma_load_3d(sm + K::oX + (sl * 2 + j) * K::kTile, &tm_x, &s.full_x[sl], (int)((h0 + j) * 64), c * 64,
                    (int)b);
      last_x = c;
    };
    auto issue_w = [&](int c) {
      mbar_arrive_expect_tx(&s.full_w[c & 1], K::kTile);
      tma_load_3d(sm + K::oW + (c & 1) * K::kTile, &tm_w, &s.full_w[c & 1], 0,
                  (int)(((b * a.nc + c) * a.G + g) * 64), 0);
      last_w = c;
    };
    auto issue_b = [&](int c) {
      uint64_t* bar = &s.full_b[c & 1];
      mbar_arrive_expect_tx(bar, K::NB * K::kTile);
      for (int j = 0; j < K::NB; ++j)
        tma_load_3d(sm + K::oB + ((c & 1) * K::NB + j) * K::kTile, &tm_b, bar, (int)(g * NS + 64 * j), c * 64,
                    (int)b);
      last_b = c;
    };
    auto issue_c = [&](int c) {
      uint64_t* bar = &s.full_c[c & 1];
      mbar_arrive_expect_tx(bar, K::NB * K::kTile);
      for (int j = 0; j < K::NB; ++j)
        tma_load_3d(sm + K::oC + ((c & 1) * K::NB + j) * K::kTile, &tm_c, bar, (int)(g * NS + 64 * j), c * 64,
                    (int)b);
      last_c = c;
    };
    bool ok = true;
    for (int k = 0; k < 2 && k < nc && ok; ++k) ok = scan_next();
    if (lane == 0 && ok) {
      for (int c = 0; c < 3 && c < nc; ++c) issue_x(c);  // slot 3 starts free
      for (int c = 0; c < 2 && c < nc; ++c) {
        issue_w(c);
        issue_b(c);
        issue_c(c);
      }
    }
    // each tile of chunk c is refilled for a later chunk as soon as the MMAs
    // reading it complete, in the order they complete
    for (int c = 0; c < nc && ok; ++c) {
      if (scanned < nc) ok = scan_next();  // chunk c + 2
      if (lane == 0 && ok) {
        if (c + 2 < nc) {
          ok = mbar_wait(&s.w_empty[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_w(c + 2);
          ok = ok && mbar_wait(&s.b_free[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_b(c + 2);
        }
        if (ok && c + 2 < nc) {
          ok = mbar_wait(&s.c_free[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_c(c + 2);
        }
        // x of chunk c + 3 goes where chunk c - 1 was, once its y tile has been stored
        if (ok && c + 3 < nc) {
          ok = c < 1 || mbar_wait(&s.x_empty[(c - 1) & 3], ((c - 1) >> 2) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_x(c + 3);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
    }
    if (lane == 0 && *abort_flag) {  // let this CTA's own copies land before its smem is released
      if (last_x >= 0) mbar_wait(&s.full_x[last_x & 3], (last_x >> 2) & 1, never, kWaitLimitNs);
      if (last_w >= 0) mbar_wait(&s.full_w[last_w & 1], (last_w >> 1) & 1, never, kWaitLimitNs);
      if (last_b >= 0) mbar_wait(&s.full_b[last_b & 1], (last_b >> 1) & 1, never, kWaitLimitNs);
      if (last_c >= 0) mbar_wait(&s.full_c[last_c & 1], (last_c >> 1) & 1, never, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t aW = smem_u32(sm + K::oW), aC = smem_u32(sm + K::oC), aB = smem_u32(sm + K::oB);
      const uint32_t aX = smem_u32(sm + K::oX), aH = smem_u32(sm + K::oH);
      constexpr uint32_t id_y = idesc_bf16(64, 128, 0, 1);    // A K-major, B MN-major (2 heads)
      constexpr uint32_t id_s = idesc_bf16(128, 128, 1, 1);   // both MN-major
      for (int c = 0; c < nc; ++c) {
        const int i = c & 1;
        const uint32_t ph = (c >> 1) & 1, pp = ((c - 2) >> 1) & 1;
        bool ok = mbar_wait(&s.full_w[i], ph, abort_flag, kWaitLimitNs);
        ok = ok && mbar_wait(&s.xp_ready[c & 3], (c >> 2) & 1, abort_flag, kWaitLimitNs);
        if (c >= 2) {
          ok = ok && mbar_wait(&s.y_free[i], pp, abort_flag, kWaitLimitNs);
          ok = ok && mbar_wait(&s.s_free[i], pp, abort_flag, kWaitLimitNs);
        }
        if (!ok) break;
        tc_fence_after();
        const uint32_t yd = tmem + K::tYd0 + 128 * i;
        const uint32_t st = tmem + K::tS0 + 128 * i;
        const uint32_t aXp = aX + (c & 3) * 2 * K::kTile;  // X' of both heads, this chunk
        // Yd = W' [X'_0 | X'_1]   (K = 64 tokens)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(yd, sw128_desc(aW + i * K::kTile + kk * 32, 16, 1024),
                      sw128_desc(aXp + kk * 2048, K::kTile, 1024), id_y, kk > 0);
        mma_commit(&s.w_empty[i]);
        // S'^T = B^T [X'_0 | X'_1]   (M = 128 states, K = 64 tokens)
        if (!mbar_wait(&s.full_b[i], ph, abort_flag, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t aBi = aB + i * K::NB * K::kTile;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(st, sw128_desc(aBi + kk * 2048, K::kTile, 1024), sw128_desc(aXp + kk * 2048, K::kTile, 1024),
                      id_s, kk > 0);
        mma_commit(&s.s_full[i]);
        mma_commit(&s.b_free[i]);
        // Yd += C [e^m H_0 | e^m H_1]^T   (K = N)
        ok = mbar_wait(&s.h_ready[i], ph, abort_flag, kWaitLimitNs);
        ok = ok && mbar_wait(&s.full_c[i], ph, abort_flag, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t aCi = aC + i * K::NB * K::kTile;
        const uint32_t aHi = aH + i * 2 * K::kHTile;
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * K::kTile + (kk & 3) * 32;
          mma_bf16_ss(yd, sw128_desc(aCi + koff, 16, 1024), sw128_desc(aHi + kk * 2048, K::kHTile, 1024), id_y, 1);
        }
        mma_commit(&s.y_full[i]);
        mma_commit(&s.h_free[i]);
        mma_commit(&s.c_free[i]);
      }
      mma_commit(&s.drain);
      mbar_wait(&s.drain, 0, never, kWaitLimitNs);
    }
  } else if (warp < 6) {
    // ------------------------------------------------ x scaling warps (both heads)
    const int wt = tid - 64;             // 0..127
    const int j = wt >> 6, srow = wt & 63;
    bool failed = false;
    for (int c = 0; c < nc; ++c) {
      if (named_barrier_any(2, 128, failed)) break;
      const int sl = c & 3, ix = c & 3;
      if (!mbar_wait(&s.scan_full[sl], (c >> 2) & 1, abort_flag, kWaitLimitNs) ||
          !mbar_wait(&s.full_x[ix], (c >> 2) & 1, abort_flag, kWaitLimitNs)) {
        failed = true;
        continue;
      }
      const __nv_bfloat162 w2 = __float2bfloat162_rn(s.v[sl][j][srow]);
      unsigned char* row = sm + K::oX + (ix * 2 + j) * K::kTile + srow * 128;
      // the whole 128-byte row, scaled in place; neighbouring rows start at
      // different 16-byte columns so that a quarter warp hits distinct banks
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint4* px = reinterpret_cast<uint4*>(row + ((k ^ (srow & 7)) << 4));
        uint4 vv = *px;
        __nv_bfloat162* e2 = reinterpret_cast<__nv_bfloat162*>(&vv);
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) e2[q2] = __hmul2(e2[q2], w2);
        *px = vv;
      }
      fence_proxy_async_smem();
      mbar_arrive(&s.xp_ready[ix]);
    }
  } else {
    // ------------------------------------------------ per-head state / epilogue warps
    // Every thread of the group reaches both named barriers of an iteration
    // whether or not its waits succeeded, so a failure never splits the group.
    const int j = (warp - 6) >> 2;       // head h0 + j
    const int64_t h = h0 + j;
    const int q = warp & 3;              // TMEM lane quadrant
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    const int n = 32 * q + lane;         // state row
    const bool issuer = (warp == 6 + 4 * j) && lane == 0;  // issues this head's y stores
    float H[64];
#pragma unroll
    for (int p = 0; p < 64; ++p) H[p] = a.h0 ? a.h0[((b * a.H + h) * 64 + p) * NS + n] : 0.f;
    bool failed = false;
    const int te = 16 * q + (lane & 15);   // epilogue row (token) of this thread
    const int half = lane >> 4;            // epilogue columns p in [32 half, 32 half + 32)
    for (int c = 0; c <= nc; ++c) {
      if (named_barrier_any(3 + j, 128, failed)) {
        failed = true;
        break;
      }
      // ---- state update for chunk c-1
      if (c >= 1) {
        const int ip = (c - 1) & 1, slp = (c - 1) & 3;
        if (mbar_wait(&s.s_full[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) {
          tc_fence_after();
          const float dd = s.sc[slp][j][2], ff = s.sc[slp][j][1];
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            uint32_t r[32];
            SSD_TMEM_LD_32x32b_X32(tq + K::tS0 + 128 * ip + 64 * j + 32 * hlf, r);
            SSD_TMEM_WAIT_LD_32(r);
#pragma unroll
            for (int k = 0; k < 32; ++k) H[32 * hlf + k] = fmaf(dd, H[32 * hlf + k], ff * __uint_as_float(r[k]));
          }
          tc_fence_before();
          mbar_arrive(&s.s_free[ip]);
        } else {
          failed = true;
        }
      }
      // ---- publish e^m H (bf16) for chunk c's C H^T product
      if (c < nc && !failed) {
        const int i = c & 1;
        if (mbar_wait(&s.scan_full[c & 3], (c >> 2) & 1, abort_flag, kWaitLimitNs) &&
            (c < 2 || mbar_wait(&s.h_free[i], ((c - 2) >> 1) & 1, abort_flag, kWaitLimitNs))) {
          const float E = s.sc[c & 3][j][0];
          unsigned char* base = sm + K::oH + (i * 2 + j) * K::kHTile + (uint32_t)n * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint4 vv;
            vv.x = pack_bf16x2(E * H[8 * k + 0], E * H[8 * k + 1]);
            vv.y = pack_bf16x2(E * H[8 * k + 2], E * H[8 * k + 3]);
            vv.z = pack_bf16x2(E * H[8 * k + 4], E * H[8 * k + 5]);
            vv.w = pack_bf16x2(E * H[8 * k + 6], E * H[8 * k + 7]);
            *reinterpret_cast<uint4*>(base + ((k ^ (n & 7)) << 4)) = vv;
          }
          fence_proxy_async_smem();
          mbar_arrive(&s.h_ready[i]);
        } else {
          failed = true;
        }
      }
      // ---- epilogue for chunk c-1: y = u_t Yd + (D / v_t) X'_t, written over X'
      if (c >= 1) {
        const int ip = (c - 1) & 1, slp = (c - 1) & 3, xs = (c - 1) & 3;
        unsigned char* tile = sm + K::oX + (xs * 2 + j) * K::kTile;
        if (!failed && mbar_wait(&s.y_full[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) {
          tc_fence_after();
          uint32_t r[32];
          SSD_TMEM_LD_16x32bx2_X32_HALF32(tq + K::tYd0 + 128 * ip + 64 * j, r);
          SSD_TMEM_WAIT_LD_32(r);
          tc_fence_before();
          mbar_arrive(&s.y_free[ip]);
          const float ut = s.u[slp][j][te], gt = s.g[slp][j][te];
          unsigned char* row = tile + te * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // 16-byte column 4 half + k of row te, at its swizzled position
            uint4* px = reinterpret_cast<uint4*>(row + (((4 * half + k) ^ (te & 7)) << 4));
            const uint4 xv = *px;
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            uint32_t o[4];
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              float x0, x1;
              unpack_bf16x2(xw[k2], x0, x1);
              const int jj = 8 * k + 2 * k2;
              o[k2] = pack_bf16x2(fmaf(ut, __uint_as_float(r[jj]), gt * x0),
                                  fmaf(ut, __uint_as_float(r[jj + 1]), gt * x1));
            }
            *px = make_uint4(o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
        } else {
          failed = true;
        }
        if (named_barrier_any(5 + j, 128, failed)) {
          failed = true;
          continue;
        }
        if (issuer) {
          tma_store_3d(&tm_y, tile, (int)(h * 64), (c - 1) * 64, (int)b);
          bulk_commit_group();
          bulk_wait_read<0>();  // the tile has been read out: its slot may be refilled
          mbar_arrive(&s.x_empty[xs]);
        }
        mbar_arrive(&s.scan_empty[slp]);
      }
    }
    if (issuer) bulk_wait<0>();  // stores complete before the CTA's shared memory is released
    if (!failed && a.final_states) {
      float* dst = a.final_states + ((b * a.H + h) * 64) * NS + n;
#pragma unroll
      for (int p = 0; p < 64; ++p) dst[(int64_t)p * NS] = H[p];
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    if (*abort_flag) atomicExch(a.err, 1);
    // a chunk's decay range was too wide to factorise: the exact kernel redoes both heads
    if (s.unit_bad) {
      const int at = atomicAdd(a.failed_count, 2);
      a.failed_list[at] = (int)(b * a.H + h0);
      a.failed_list[at + 1] = (int)(b * a.H + h0 + 1);
    }
  }
  if (warp == 0) tmem_dealloc(tmem, K::kTmemCols);
}

}  // namespace

bool tc_pair_supported(const Problem& p) { return p.N == 128 && p.hpg % 2 == 0; }

cudaError_t tc_pair_launch(const Problem& p, const TcWorkspace& w, const CUtensorMap& tx, const CUtensorMap& tb,
                           const CUtensorMap& tc_, const CUtensorMap& tw, const CUtensorMap& ty,
                           const tc::FastArgs& fa, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(k_ssd_fwd_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PairCfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  (void)w;
  k_ssd_fwd_pair<<<(unsigned)(p.b * p.H / 2), PairCfg::kThreads, PairCfg::kSmemBytes, st>>>(tx, tb, tc_, tw, ty, fa);
  return cudaGetLastError();
}

}  // namespace ssd
