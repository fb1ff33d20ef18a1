// Two-head variant of the fast fused SSD forward (see ssd_tc_fast.cu for the
// factorised-decay formulation): one CTA owns two heads (h, h+1) of the same
// batch row and B/C group and walks their chunks together.  The heads share
// the C, B and W' = masked C B^T tiles, and every MMA covers both heads at
// once with N = 128:
//
//   Yd   = W' [X'_h | X'_h+1]                     (M = 64 tokens,  K = 64 tokens)
//   S'^T = B^T [X'_h | X'_h+1]                    (M = 128 states, K = 64 tokens)
//   Yd  += C [H_h | H_h+1]^T                      (M = 64 tokens,  K = N)
//   y_t  = u_t Yd_t + D x_t,   H <- 2^cs_e (H + S')
//
// per head, with cs_t the in-chunk cumulative sum of dt A (log2 units),
// u_t = 2^cs_t, v_s = 2^-cs_s dt_s and X' = diag(v) x: u_t v_s = exp of the
// decay from s to t times dt_s.  The factors are taken about the chunk's
// first token (ssd_tc_fast.cu takes them about its middle), so the state
// enters the C H^T product as it is, with no per-chunk rescaling; a chunk
// whose total decay exceeds 2^kRangeLog2 sends the pair to the exact kernel.
// The chunked steps are those
// of "SSM 家族全景图（下）：Mamba-2 与 Jamba" section 三.4; the D feed-through
// is from "从Transformer的二次复杂度困境到Mamba的线性突围" (continuous SSM).
//
// The D x_t feed-through is taken from the scaled tile: D x_t = (D / v_t) X'_t,
// so the epilogue needs no second read of x.  It writes y over X' in the
// same shared-memory slot (each thread overwrites exactly what it read) and
// a bulk tensor store per head moves the tile out.
//
// Warp roles (512 threads), each a loop over the chunks that only waits on
// the barriers it needs:
//   warp 0      TMA loads (one thread): x 3 chunks ahead (L2 prefetch 6 ahead),
//               W', B, C 2 ahead
//   warp 1      MMA issue (descriptors formed by the warp, one elected lane issues)
//   warp 2      dt scan of both heads: u, v, D / v and the chunk scalars; it
//               also loads dt by TMA into an 8-deep ring of its own
//   warp 3      y stores (one thread); frees an x slot once its tile is read out
//   warps 4-7   the epilogue of both heads
//   warps 8-11, 12-15   one head each: state update (fp32 state in registers),
//               publishing the bf16 e^m H tile, and scaling the head's next
//               x tile into X' in place
// x tiles sit in a 4-deep ring; W'+B, C, the e^m H tiles, Yd and S are
// double-buffered.  Every wait is bounded; a CTA that times out records the
// error, drains its copies, stores and MMAs, frees its TMEM and exits.
//
// The grid is persistent: with G CTAs, CTA i owns the contiguous range
// [i T / G, (i+1) T / G) of the T = pairs x chunks steps in pair-major order,
// so every CTA gets the same number of chunk steps.  A pair split between CTAs
// i and i+1 hands its fp32 state over through global memory (per state warp:
// data, then a release flag).  Each CTA runs the head of its last pair first
// and the tail of its first pair last, so a tail normally finds its hand-over
// long written.  Every warp role walks the CTA's segments as one sequence of
// chunks, so the pipelines run across segment boundaries without draining.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "sm100.cuh"
#include "ssd_internal.h"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

using namespace sm100;
using namespace tc;

struct PairCfg {
  static constexpr int NS = 128, NB = 2;
  static constexpr int kThreads = 512;
  static constexpr uint32_t kTile = 8192;
  static constexpr int kXSlots = 4;
  static constexpr uint32_t oX = 0;                        // [4 slots][2 heads] x -> X' -> y, in place
  static constexpr uint32_t oW = oX + 2 * kXSlots * kTile; // [2] W' tiles
  static constexpr uint32_t oB = oW + 2 * kTile;           // [2] B, 2 n-blocks each
  static constexpr uint32_t oC = oB + 2 * NB * kTile;      // [2] C, 2 n-blocks each
  static constexpr uint32_t oH = oC + 2 * NB * kTile;      // [2 bufs][2 heads] e^m H, 16 KB each
  static constexpr uint32_t kHTile = NB * kTile;
  static constexpr uint32_t oDt = oH + 4 * kHTile;          // [8] dt boxes: 64 tokens x 4 heads fp32
  static constexpr uint32_t kDtBox = 64 * 16;
  static constexpr uint32_t oEnd = oDt + 8 * kDtBox;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  // TMEM: Yd[2] at 0 / 128 (M = 64 layout, head j in columns 64j..64j+63),
  //       S[2]  at 256 / 384 (M = 128 layout, head j in columns 64j..)
  static constexpr uint32_t tYd0 = 0, tS0 = 256, kTmemCols = 512;
};

constexpr int kPairMaxSeg = 32;  // segments (pairs touched) per CTA, at most

// Ring barriers are indexed like the buffers they guard, so no barrier can
// complete a second phase before every waiter has seen the first.
struct __align__(16) PairSmem {
  uint64_t full_x[4], x_empty[4];        // x ring: TMA landed / y tile read out by the store
  uint64_t full_dt[8];                   // dt ring (the scan warp's own)
  uint64_t full_wb[2], full_c[2];        // W' + B, C of a chunk landed
  uint64_t scan_full[4], scan_empty[4];  // scan results of a chunk ready / consumed
  uint64_t xp_ready[4];                  // X' of a chunk scaled
  uint64_t s_full[2];                    // S of a chunk in TMEM (its W' and B reads are done)
  uint64_t mma_done[2];                  // every MMA of a chunk done: Yd final, C and e^m H free
  uint64_t h_ready[2];                   // e^m H of a chunk published
  uint64_t acc_free[2];                  // Yd (epilogue) and S (state) TMEM buffers read out
  uint64_t y_staged[4];                  // y of a chunk written over its x slot
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int never;
  int nseg, total;                       // segments of this CTA and their chunk count
  // per segment: pair, batch row, first head, group, first chunk, length, first step
  int seg_pair[kPairMaxSeg], seg_b[kPairMaxSeg], seg_h0[kPairMaxSeg], seg_grp[kPairMaxSeg];
  int seg_c0[kPairMaxSeg], seg_len[kPairMaxSeg], seg_g0[kPairMaxSeg];
  int seg_i0[kPairMaxSeg];  // split mode: the first CTA whose range holds the segment's pair start
  alignas(16) float u[4][2][64];  // written as float4
  alignas(16) float v[4][2][64];
  alignas(16) float g[4][2][64];  // D / v_t: D x_t = g_t X'_t
  float sc[4][2][4];  // [0]: d = 2^cs_e, the chunk's total decay
};

static_assert(offsetof(PairSmem, u) % 16 == 0 && offsetof(PairSmem, v) % 16 == 0 &&
                  offsetof(PairSmem, g) % 16 == 0,
              "scan results are stored as float4");

// Position of one of a CTA's step streams (each role walks its steps in
// order): segment k, chunk c.  next() moves to the following step.
struct PairCursor {
  int k, c;
  __device__ __forceinline__ void start(const PairSmem& s) {
    k = 0;
    c = s.seg_c0[0];
  }
  __device__ __forceinline__ void next(const PairSmem& s) {
    if (++c == s.seg_c0[k] + s.seg_len[k] && k + 1 < s.nseg) {
      ++k;
      c = s.seg_c0[k];
    }
  }
};

// kStateOnly: the state-only pass of split mode.  Each CTA takes only the
// segment of its range that ends inside a pair (there is at most one: the
// head of its last pair), runs it from a zero state with x and B alone (no
// W', C, y) and leaves the end state in handoff and the segment's total decay
// per head in seg_decay.
template <bool kStateOnly>
__global__ void __launch_bounds__(512, 1)
    k_ssd_fwd_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_dt,
                   const FastArgs a) {
  using K = PairCfg;
  constexpr int NS = K::NS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  __shared__ PairSmem s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_launch_dependents();  // the exact kernel may set up while this grid runs
  const int64_t pairs = a.H / 2;
  const int nc = (int)a.nc;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s.full_x[i], 1);
      mbar_init(&s.x_empty[i], 1);
      mbar_init(&s.scan_full[i], 32);
      mbar_init(&s.scan_empty[i], kStateOnly ? 256 : 384);  // epilogue warps and state warps
      mbar_init(&s.xp_ready[i], 256);  // both heads' state warps
      mbar_init(&s.y_staged[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full_wb[i], 1);
      mbar_init(&s.full_c[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.mma_done[i], 1);
      mbar_init(&s.h_ready[i], 256);
      mbar_init(&s.acc_free[i], kStateOnly ? 256 : 384);  // epilogue (Yd) and state (S) readers
    }
    for (int i = 0; i < 8; ++i) mbar_init(&s.full_dt[i], 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = *reinterpret_cast<volatile int*>(a.err) != 0;
    s.never = 0;
    // this CTA's range of (pair, chunk) steps, as segments in processing order:
    // the head of the last pair, the whole pairs, the tail of the first pair
    // (steps, pairs and chunks fit in 32 bits: the launch checks b * H * nc)
    const int64_t T = a.batch * pairs * a.nc;
    const int start = (int)((int64_t)blockIdx.x * T / gridDim.x);
    const int end = (int)(((int64_t)blockIdx.x + 1) * T / gridDim.x);
    const int ncs = nc, npr = (int)pairs, hpg = (int)a.hpg;
    int n = 0, tot = 0;
    auto add = [&](int pr, int c0, int len) {
      if (n < kPairMaxSeg && len > 0) {
        s.seg_pair[n] = pr;
        s.seg_b[n] = pr / npr;
        s.seg_h0[n] = (pr % npr) * 2;
        s.seg_grp[n] = (pr % npr) * 2 / hpg;
        s.seg_c0[n] = c0;
        s.seg_len[n] = len;
        s.seg_g0[n] = tot;
        tot += len;
        ++n;
      }
    };
    if (end > start) {
      const int p0 = start / ncs, c0 = start % ncs, q = (end - 1) / ncs, cq = (end - 1) % ncs + 1;
      if (q == p0) {
        add(p0, c0, cq - c0);
      } else {
        add(q, 0, cq);
        for (int pr = p0 + 1; pr < q; ++pr) add(pr, 0, ncs);
        add(p0, c0, ncs - c0);
      }
    }
    if (kStateOnly) {  // only a segment that ends inside its pair
      if (n > 0 && s.seg_c0[0] + s.seg_len[0] < ncs) {
        n = 1;
        tot = s.seg_len[0];
      } else {
        n = tot = 0;
      }
    } else if (a.split) {
      // the CTAs before this one that hold a part of the segment's pair
      for (int k = 0; k < n; ++k) {
        const int64_t s0 = (int64_t)s.seg_pair[k] * ncs;
        int i0 = (int)blockIdx.x;
        while (i0 > 0 && (int64_t)i0 * T / gridDim.x > s0) --i0;
        s.seg_i0[k] = i0;
      }
    }
    s.nseg = n;
    s.total = tot;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_c);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_y);
    tma_prefetch_desc(&tm_dt);
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
  const int total = s.total;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      int last_x = -1, last_wb = -1, last_c = -1;
      // (the argument is this CTA's step number; each stream has a cursor on
      // its pair and chunk, advanced as the stream issues its steps in order)
      PairCursor ux, uwb, uc, upf;
      ux.start(s);
      uwb.start(s);
      uc.start(s);
      upf.start(s);
      for (int k = 0; k < 3; ++k) upf.next(s);
      auto issue_x = [&](int gg) {
        const int sl = gg & 3, bb = s.seg_b[ux.k], hh = s.seg_h0[ux.k];
        mbar_arrive_expect_tx(&s.full_x[sl], 2 * K::kTile);
        for (int j = 0; j < 2; ++j)
          tma_load_3d(sm + K::oX + (sl * 2 + j) * K::kTile, &tm_x, &s.full_x[sl], (hh + j) * 64, ux.c * 64, bb);
        ux.next(s);
        last_x = gg;
      };
      auto issue_wb = [&](int gg) {
        const int i = gg & 1, bb = s.seg_b[uwb.k], grp = s.seg_grp[uwb.k];
        mbar_arrive_expect_tx(&s.full_wb[i], (kStateOnly ? K::NB : 1 + K::NB) * K::kTile);
        if (!kStateOnly)
          tma_load_3d(sm + K::oW + i * K::kTile, &tm_w, &s.full_wb[i], 0, ((bb * nc + uwb.c) * (int)a.G + grp) * 64,
                      0);
        for (int jb = 0; jb < K::NB; ++jb)
          tma_load_4d(sm + K::oB + (i * K::NB + jb) * K::kTile, &tm_b, &s.full_wb[i], 64 * jb, grp, uwb.c * 64,
                      bb);
        uwb.next(s);
        last_wb = gg;
      };
      auto issue_c = [&](int gg) {
        const int i = gg & 1, bb = s.seg_b[uc.k], grp = s.seg_grp[uc.k];
        mbar_arrive_expect_tx(&s.full_c[i], K::NB * K::kTile);
        for (int jb = 0; jb < K::NB; ++jb)
          tma_load_4d(sm + K::oC + (i * K::NB + jb) * K::kTile, &tm_c, &s.full_c[i], 64 * jb, grp, uc.c * 64, bb);
        uc.next(s);
        last_c = gg;
      };
      // x comes from HBM and takes several chunk periods to arrive; L2
      // prefetches run 6 chunks ahead of use, the loads into the ring 3
      auto prefetch_x = [&](int) {
        const int bb = s.seg_b[upf.k], hh = s.seg_h0[upf.k];
        for (int j = 0; j < 2; ++j) tma_prefetch_l2_3d(&tm_x, (hh + j) * 64, upf.c * 64, bb);
        upf.next(s);
      };
      if (!*abort_flag) {
        #pragma unroll 1
        for (int c = 3; c < 6 && c < total; ++c) prefetch_x(c);
        #pragma unroll 1
        for (int c = 0; c < 3 && c < total; ++c) issue_x(c);  // slot 3 starts free
        if (!kStateOnly) griddep_wait();  // W' comes from the C B^T kernel launched before this one
        #pragma unroll 1
        for (int c = 0; c < 2 && c < total; ++c) {
          issue_wb(c);
          if (!kStateOnly) issue_c(c);
        }
      }
      bool ok = !*abort_flag;
      // each tile is refilled for a later chunk as soon as its last reader is done
      #pragma unroll 1
      for (int c = 0; c < total && ok; ++c) {
        if (c + 2 < total) {
          ok = mbar_wait(&s.s_full[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_wb(c + 2);
          if (!kStateOnly) {
            ok = ok && mbar_wait(&s.mma_done[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
            if (ok) issue_c(c + 2);
          }
        }
        // x of step c + 3 goes where step c - 1 was, once its y tile has been stored
        if (ok && c + 3 < total) {
          ok = c < 1 || mbar_wait(&s.x_empty[(c - 1) & 3], ((c - 1) >> 2) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_x(c + 3);
          if (ok && c + 6 < total) prefetch_x(c + 6);
        }
      }
      if (*abort_flag) {  // let this CTA's own copies land before its smem is released
        // (within one ring-depth window every slot holds a single chunk)
        #pragma unroll 1
        for (int c = last_x - 3 < 0 ? 0 : last_x - 3; c <= last_x; ++c)
          mbar_wait(&s.full_x[c & 3], (c >> 2) & 1, never, kWaitLimitNs);
        #pragma unroll 1
        for (int c = last_wb - 1 < 0 ? 0 : last_wb - 1; c <= last_wb; ++c)
          mbar_wait(&s.full_wb[c & 1], (c >> 1) & 1, never, kWaitLimitNs);
        #pragma unroll 1
        for (int c = last_c - 1 < 0 ? 0 : last_c - 1; c <= last_c; ++c)
          mbar_wait(&s.full_c[c & 1], (c >> 1) & 1, never, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp walks the loop and forms the descriptors (warp-uniform
    // values); one elected lane issues the MMAs and commits.
    const uint32_t aW = smem_u32(sm + K::oW), aC = smem_u32(sm + K::oC), aB = smem_u32(sm + K::oB);
    const uint32_t aX = smem_u32(sm + K::oX), aH = smem_u32(sm + K::oH);
    constexpr uint32_t id_y = idesc_bf16(64, 128, 0, 1);    // A K-major, B MN-major (2 heads)
    constexpr uint32_t id_s = idesc_bf16(128, 128, 1, 1);   // both MN-major
    #pragma unroll 1
    for (int c = 0; c < total; ++c) {
      const int i = c & 1;
      const uint32_t ph = (c >> 1) & 1;
      bool ok = mbar_wait_warp(&s.full_wb[i], ph, abort_flag, kWaitLimitNs);
      ok = ok && mbar_wait_warp(&s.xp_ready[c & 3], (c >> 2) & 1, abort_flag, kWaitLimitNs);
      if (c >= 2) ok = ok && mbar_wait_warp(&s.acc_free[i], ((c - 2) >> 1) & 1, abort_flag, kWaitLimitNs);
      if (!ok) break;
      tc_fence_after();
      const uint32_t yd = tmem + K::tYd0 + 128 * i;
      const uint32_t st = tmem + K::tS0 + 128 * i;
      // X' of both heads, this chunk; a K step of 16 tokens is 16 rows (2048 B)
      const uint64_t dxp = sw128_desc(aX + (c & 3) * 2 * K::kTile, K::kTile, 1024);
      const uint64_t dw = sw128_desc(aW + i * K::kTile, 16, 1024);  // a K step is 32 B along the row
      const uint64_t db = sw128_desc(aB + i * K::NB * K::kTile, K::kTile, 1024);
      if (elect_one()) {
        // Yd = W' [X'_0 | X'_1]   (K = 64 tokens)
        if (!kStateOnly) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(yd, dw + 2 * kk, dxp + 128 * kk, id_y, kk > 0);
        }
        // S'^T = B^T [X'_0 | X'_1]   (M = 128 states, K = 64 tokens)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(st, db + 128 * kk, dxp + 128 * kk, id_s, kk > 0);
        mma_commit(&s.s_full[i]);
        if (kStateOnly) mma_commit(&s.x_empty[c & 3]);  // X' read: the slot may be refilled
      }
      __syncwarp();
      if (kStateOnly) continue;
      // Yd += C [e^m H_0 | e^m H_1]^T   (K = N)
      ok = mbar_wait_warp(&s.h_ready[i], ph, abort_flag, kWaitLimitNs);
      ok = ok && mbar_wait_warp(&s.full_c[i], ph, abort_flag, kWaitLimitNs);
      if (!ok) break;
      tc_fence_after();
      const uint64_t dc = sw128_desc(aC + i * K::NB * K::kTile, 16, 1024);
      const uint64_t dh = sw128_desc(aH + i * 2 * K::kHTile, K::kHTile, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk)
          mma_bf16_ss(yd, dc + ((kk >> 2) * K::kTile + (kk & 3) * 32) / 16, dh + 128 * kk, id_y, 1);
        mma_commit(&s.mma_done[i]);
      }
      __syncwarp();
    }
    if (elect_one()) {
      mma_commit(&s.drain);
      mbar_wait(&s.drain, 0, never, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ dt scan
    // lanes 0-15 take head h0, lanes 16-31 head h0 + 1; each lane owns 4
    // consecutive tokens, so a chunk needs one 16-lane scan per head.  dt
    // arrives by TMA (a box of 4 heads from the multiple of 4 at or below h0)
    // so that no register load is in flight when the results are released.
    const int j = lane >> 4, l16 = lane & 15;
    int last_dt = -1;
    PairCursor ud, us;
    ud.start(s);
    us.start(s);
    auto issue_dt = [&](int gg) {
      mbar_arrive_expect_tx(&s.full_dt[gg & 7], K::kDtBox);
      tma_load_3d(sm + K::oDt + (gg & 7) * K::kDtBox, &tm_dt, &s.full_dt[gg & 7], s.seg_h0[ud.k] & ~3, ud.c * 64,
                  s.seg_b[ud.k]);
      ud.next(s);
      last_dt = gg;
    };
    if (lane == 0 && !*abort_flag)
      #pragma unroll 1
      for (int c = 0; c < 8 && c < total; ++c) issue_dt(c);
    int cur_seg = -1, col = 0;
    float a2 = 0.f, dsk = 0.f;
    #pragma unroll 1
    for (int g = 0; g < total; ++g, us.next(s)) {
      const int slot = g & 3;
      const int hh = s.seg_h0[us.k];
      if (us.k != cur_seg) {  // a new pair: its heads' A and D
        cur_seg = us.k;
        col = (hh & 3) + j;
        a2 = a.A[hh + j] * kLog2e;
        dsk = a.D ? a.D[hh + j] : 0.f;
      }
      if (g >= 4 && !mbar_wait_warp(&s.scan_empty[slot], ((g - 4) >> 2) & 1, abort_flag, kWaitLimitNs)) break;
      if (!mbar_wait_warp(&s.full_dt[g & 7], (g >> 3) & 1, abort_flag, kWaitLimitNs)) break;
      const float* dts = reinterpret_cast<const float*>(sm + K::oDt + (g & 7) * K::kDtBox);
      const int c = us.c;
      const int nvalid = (int)((int64_t)(c + 1) * 64 <= a.L ? 64 : a.L - (int64_t)c * 64);
      float d[4], cs[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) d[k] = dts[(4 * l16 + k) * 4 + col];
      __syncwarp();
      if (lane == 0 && g + 8 < total) {  // the slot has been read: refill it 8 steps ahead
        fence_proxy_async_smem();
        issue_dt(g + 8);
      }
      cs[0] = d[0] * a2;
#pragma unroll
      for (int k = 1; k < 4; ++k) cs[k] = fmaf(d[k], a2, cs[k - 1]);
      float incl = cs[3];
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o, 16);
        if (l16 >= o) incl += u;
      }
      const float excl = incl - cs[3];
#pragma unroll
      for (int k = 0; k < 4; ++k) cs[k] += excl;
      const int e = nvalid - 1;
      const float mine = (e & 3) == 0 ? cs[0] : (e & 3) == 1 ? cs[1] : (e & 3) == 2 ? cs[2] : cs[3];
      const float cse = __shfl_sync(0xffffffffu, mine, e >> 2, 16);
      float u4[4], v4[4], g4[4];
      bool bad = false;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        u4[k] = exp2f(cs[k]);
        v4[k] = exp2f(-cs[k]) * d[k];
        // D x_t is recovered from X'_t = v_t x_t, so a valid token needs v_t well
        // inside the normal range (the fast division is exact to 2 ulp there)
        g4[k] = dsk != 0.f ? __fdividef(dsk, v4[k]) : 0.f;
        bad |= !(fabsf(cs[k]) <= kRangeLog2) ||
               (dsk != 0.f && 4 * l16 + k < nvalid && !(fabsf(v4[k]) >= 1e-30f && fabsf(v4[k]) <= 1e30f));
      }
      // a chunk the factorised form cannot take: the exact kernel redoes the
      // pair (once, however many chunks or CTAs find it)
      if (__any_sync(0xffffffffu, bad) && lane == 0 && atomicExch(&a.pair_bad[s.seg_pair[us.k]], 1) == 0) {
        const int at = atomicAdd(a.failed_count, 2);
        const int unit = s.seg_b[us.k] * (int)a.H + hh;
        a.failed_list[at] = unit;
        a.failed_list[at + 1] = unit + 1;
      }
      *reinterpret_cast<float4*>(&s.u[slot][j][4 * l16]) = make_float4(u4[0], u4[1], u4[2], u4[3]);
      *reinterpret_cast<float4*>(&s.v[slot][j][4 * l16]) = make_float4(v4[0], v4[1], v4[2], v4[3]);
      *reinterpret_cast<float4*>(&s.g[slot][j][4 * l16]) = make_float4(g4[0], g4[1], g4[2], g4[3]);
      if (l16 == 0) {
        s.sc[slot][j][0] = exp2f(cse);
      }
      mbar_arrive(&s.scan_full[slot]);
    }
    if (lane == 0 && *abort_flag)  // let the dt copies in flight land
      #pragma unroll 1
      for (int c = last_dt - 7 < 0 ? 0 : last_dt - 7; c <= last_dt; ++c)
        mbar_wait(&s.full_dt[c & 7], (c >> 3) & 1, never, kWaitLimitNs);
  } else if (warp == 3) {
    // ------------------------------------------------------------ y stores
    // (the state-only pass stores no y: its MMAs free the x slots)
    if (!kStateOnly && lane == 0) {
      PairCursor uy;
      uy.start(s);
      #pragma unroll 1
      for (int c = 0; c < total; ++c, uy.next(s)) {
        const int sl = c & 3;
        if (!mbar_wait(&s.y_staged[sl], (c >> 2) & 1, abort_flag, kWaitLimitNs)) break;
        for (int j = 0; j < 2; ++j)
          tma_store_3d(&tm_y, sm + K::oX + (sl * 2 + j) * K::kTile, (s.seg_h0[uy.k] + j) * 64, uy.c * 64,
                       s.seg_b[uy.k]);
        bulk_commit_group();
        bulk_wait_read<0>();  // the tiles have been read out: the slot may be refilled
        mbar_arrive(&s.x_empty[sl]);
      }
      bulk_wait<0>();  // stores complete before the CTA's shared memory is released
    }
  } else if (warp < 8) {
    // ------------------------------------------------ epilogue warps (both heads)
    if constexpr (!kStateOnly) {
      const int q = warp & 3;              // TMEM lane quadrant
      const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
      const int te = 16 * q + (lane & 15);   // epilogue row (token) of this thread
      const int half = lane >> 4;            // epilogue columns p in [32 half, 32 half + 32)
      #pragma unroll 1
      for (int c = 1; c <= total; ++c) {
        // ---- epilogue for step c-1, both heads: y = u_t Yd + (D / v_t) X'_t, written over X'
        if (c >= 1) {
          const int ip = (c - 1) & 1, slp = (c - 1) & 3;
          if (!mbar_wait_warp(&s.mma_done[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) break;
          tc_fence_after();
          #pragma unroll 1
          for (int j = 0; j < 2; ++j) {
            uint32_t r[32];
            SSD_TMEM_LD_16x32bx2_X32_HALF32(tq + K::tYd0 + 128 * ip + 64 * j, r);
            SSD_TMEM_WAIT_LD_32(r);
            const float ut = s.u[slp][j][te], gt = s.g[slp][j][te];
            unsigned char* row = sm + K::oX + (slp * 2 + j) * K::kTile + te * 128;
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
          }
          tc_fence_before();
          mbar_arrive(&s.acc_free[ip]);  // this thread's reads of Yd of chunk c-1 are done
          fence_proxy_async_smem();
          mbar_arrive(&s.y_staged[slp]);
          mbar_arrive(&s.scan_empty[slp]);
        }
      }
    }
  } else {
    // ------------------------------------------------ per-head state warps
    const int j = (warp - 8) >> 2;       // head h0 + j of the current pair
    const int q = warp & 3;              // TMEM lane quadrant
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    const int n = 32 * q + lane;         // state row
    const int uw = warp - 8;             // this warp's part of a state hand-over
    const int ut = tid - 256 - 128 * j;  // 0..127 within this head's group
    const int srow = ut >> 1, shalf = ut & 1;
    // X' = diag(v) x for step cc of this head: each thread scales half a
    // 128-byte row in place, at the swizzled positions of its 16-byte columns
    // (the caller has seen scan_full and full_x of step cc; it fences and
    // arrives on xp_ready)
    auto scale_tile = [&](int cc) {
      const int sl = cc & 3;
      const __nv_bfloat162 w2 = __float2bfloat162_rn(s.v[sl][j][srow]);
      unsigned char* row = sm + K::oX + (sl * 2 + j) * K::kTile + srow * 128;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint4* px = reinterpret_cast<uint4*>(row + (((4 * shalf + k) ^ (srow & 7)) << 4));
        uint4 vv = *px;
        __nv_bfloat162* e2 = reinterpret_cast<__nv_bfloat162*>(&vv);
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) e2[q2] = __hmul2(e2[q2], w2);
        *px = vv;
      }
    };
    auto scale_chunk = [&](int cc) -> bool {
      const int sl = cc & 3;
      if (!mbar_wait_warp(&s.scan_full[sl], (cc >> 2) & 1, abort_flag, kWaitLimitNs) ||
          !mbar_wait_warp(&s.full_x[sl], (cc >> 2) & 1, abort_flag, kWaitLimitNs))
        return false;
      scale_tile(cc);
      fence_proxy_async_smem();
      mbar_arrive(&s.xp_ready[sl]);
      return true;
    };
    float H[64];
    float dprod = 1.f;  // state-only pass: the segment's total decay so far
    // state at the start of segment k: h0 (or zero) at a pair's first chunk,
    // otherwise this warp's part of the hand-over the previous CTA wrote, or
    // in split mode h0 carried through the state-only pass's local states of
    // the CTAs before this one (each: H <- decay H + S).  The state-only pass
    // itself starts every segment from zero.
    auto seg_begin = [&](int k) -> bool {
      const int64_t h = s.seg_h0[k] + j, bb = s.seg_b[k];
      if (kStateOnly) {
#pragma unroll
        for (int p = 0; p < 64; ++p) H[p] = 0.f;
        dprod = 1.f;
        return true;
      }
      if (s.seg_c0[k] == 0 || a.split) {
        if (a.h0 && n < a.Nr) {
          const float* src = a.h0 + ((bb * a.H + h) * 64) * a.Nr + n;
#pragma unroll
          for (int p = 0; p < 64; ++p) H[p] = src[p * a.Nr];
        } else {
#pragma unroll
          for (int p = 0; p < 64; ++p) H[p] = 0.f;
        }
        if (s.seg_c0[k] == 0) return true;
        griddep_wait();  // the state-only pass launched before this kernel
        #pragma unroll 1
        for (int ip = s.seg_i0[k]; ip < (int)blockIdx.x; ++ip) {
          const float dd = __ldcg(a.seg_decay + 2 * ip + j);
          const float4* src =
              reinterpret_cast<const float4*>(a.handoff + (size_t)ip * kPairHandoffFloats + ((size_t)j * 128 + n) * 64);
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const float4 v = __ldcg(src + p);
            H[4 * p] = fmaf(dd, H[4 * p], v.x);
            H[4 * p + 1] = fmaf(dd, H[4 * p + 1], v.y);
            H[4 * p + 2] = fmaf(dd, H[4 * p + 2], v.z);
            H[4 * p + 3] = fmaf(dd, H[4 * p + 3], v.w);
          }
        }
        return true;
      }
      const int slot = (int)blockIdx.x - 1;
      bool ok = true;
      if (lane == 0) ok = wait_flag_acquire(a.flags + slot * kPairFlagsPerCta + uw, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) return false;
      const float4* src =
          reinterpret_cast<const float4*>(a.handoff + (size_t)slot * kPairHandoffFloats + ((size_t)j * 128 + n) * 64);
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const float4 v = __ldcg(src + p);
        H[4 * p] = v.x;
        H[4 * p + 1] = v.y;
        H[4 * p + 2] = v.z;
        H[4 * p + 3] = v.w;
      }
      return true;
    };
    // state at the end of segment k: the pair's final state, or the hand-over
    // to the next CTA (data, then this warp's release flag)
    auto seg_end = [&](int k) {
      const int64_t h = s.seg_h0[k] + j, bb = s.seg_b[k];
      if (kStateOnly) {  // the local end state and the total decay, for the CTAs after this one
        float4* dst = reinterpret_cast<float4*>(a.handoff + (size_t)blockIdx.x * kPairHandoffFloats +
                                                ((size_t)j * 128 + n) * 64);
#pragma unroll
        for (int p = 0; p < 16; ++p) __stcg(dst + p, make_float4(H[4 * p], H[4 * p + 1], H[4 * p + 2], H[4 * p + 3]));
        if (n == 0) __stcg(a.seg_decay + 2 * blockIdx.x + j, dprod);
        return;
      }
      if (s.seg_c0[k] + s.seg_len[k] == nc) {
        if (a.final_states && n < a.Nr) {
          float* dst = a.final_states + ((bb * a.H + h) * 64) * a.Nr + n;
#pragma unroll
          for (int p = 0; p < 64; ++p) dst[(int64_t)p * a.Nr] = H[p];
        }
        return;
      }
      if (a.split) return;  // the CTAs after this one start from the state-only pass
      float4* dst = reinterpret_cast<float4*>(a.handoff + (size_t)blockIdx.x * kPairHandoffFloats +
                                              ((size_t)j * 128 + n) * 64);
#pragma unroll
      for (int p = 0; p < 16; ++p) __stcg(dst + p, make_float4(H[4 * p], H[4 * p + 1], H[4 * p + 2], H[4 * p + 3]));
      __threadfence();
      __syncwarp();
      if (lane == 0) store_flag_release(a.flags + (int)blockIdx.x * kPairFlagsPerCta + uw, 1);
    };
    // Steps in order: publish e^m H for step g (the state before g), scale the
    // x tile of step g+1, then fold step g's chunk state into H.
    bool failed = total > 0 && !scale_chunk(0);
    const int nseg = s.nseg;
    #pragma unroll 1
    for (int k = 0; k < nseg && !failed; ++k) {
      if (!seg_begin(k)) {
        failed = true;
        break;
      }
      const int g_end = s.seg_g0[k] + s.seg_len[k];
      #pragma unroll 1
      for (int g = s.seg_g0[k]; g < g_end; ++g) {
        const int i = g & 1, n1 = g + 1, s1 = n1 & 3;
        const bool more = n1 < total;
        // the barriers this step's publish and the next tile's scaling need,
        // probed together (their latencies overlap), then waited for if not yet
        const bool d_ok = kStateOnly || g < 2 || mbar_probe(&s.mma_done[i], ((g - 2) >> 1) & 1);
        const bool v_ok = !more || mbar_probe(&s.scan_full[s1], (n1 >> 2) & 1);
        const bool x_ok = !more || mbar_probe(&s.full_x[s1], (n1 >> 2) & 1);
        if constexpr (!kStateOnly) {
          if (!__all_sync(0xffffffffu, d_ok) &&
              !mbar_wait_warp(&s.mma_done[i], ((g - 2) >> 1) & 1, abort_flag, kWaitLimitNs)) {
            failed = true;
            break;
          }
          {
            unsigned char* base = sm + K::oH + (i * 2 + j) * K::kHTile + (uint32_t)n * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              uint4 vv;
              vv.x = pack_bf16x2(H[8 * kk + 0], H[8 * kk + 1]);
              vv.y = pack_bf16x2(H[8 * kk + 2], H[8 * kk + 3]);
              vv.z = pack_bf16x2(H[8 * kk + 4], H[8 * kk + 5]);
              vv.w = pack_bf16x2(H[8 * kk + 6], H[8 * kk + 7]);
              *reinterpret_cast<uint4*>(base + ((kk ^ (n & 7)) << 4)) = vv;
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(&s.h_ready[i]);
        }
        if (more) {
          if ((!__all_sync(0xffffffffu, v_ok) &&
               !mbar_wait_warp(&s.scan_full[s1], (n1 >> 2) & 1, abort_flag, kWaitLimitNs)) ||
              (!__all_sync(0xffffffffu, x_ok) &&
               !mbar_wait_warp(&s.full_x[s1], (n1 >> 2) & 1, abort_flag, kWaitLimitNs))) {
            failed = true;
            break;
          }
          scale_tile(n1);
          fence_proxy_async_smem();
          mbar_arrive(&s.xp_ready[s1]);
        }
        // ---- state update with step g's chunk state
        if (!mbar_wait_warp(&s.s_full[i], (g >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          break;
        }
        tc_fence_after();
        {
          // H <- d (H + S'), two lanes of fp32 per instruction
          const float dd = s.sc[g & 3][j][0];
          const float2 d2 = make_float2(dd, dd);
          if (kStateOnly) dprod *= dd;
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            uint32_t r[32];
            SSD_TMEM_LD_32x32b_X32(tq + K::tS0 + 128 * i + 64 * j + 32 * hlf, r);
            SSD_TMEM_WAIT_LD_32(r);
#pragma unroll
            for (int kk = 0; kk < 32; kk += 2) {
              const float2 h2 = __fadd2_rn(make_float2(H[32 * hlf + kk], H[32 * hlf + kk + 1]),
                                           make_float2(__uint_as_float(r[kk]), __uint_as_float(r[kk + 1])));
              const float2 o2 = __fmul2_rn(d2, h2);
              H[32 * hlf + kk] = o2.x;
              H[32 * hlf + kk + 1] = o2.y;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&s.acc_free[i]);        // this thread's reads of S of step g are done
        mbar_arrive(&s.scan_empty[g & 3]);  // and of that step's scalars
      }
      if (!failed) seg_end(k);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && *abort_flag) atomicExch(a.err, 1);
  // the state-only pass completes only after the grid before it (the C B^T
  // kernel), so the kernel after it may rely on both once it has waited
  if (kStateOnly && tid == 0) griddep_wait();
  if (warp == 0) tmem_dealloc(tmem, K::kTmemCols);
}

}  // namespace

// (the kernel counts its (pair, chunk) steps in 32-bit integers)
bool tc_pair_shape_ok(const Problem& p) {
  return tc_kernel_n(p) == 128 && p.hpg % 2 == 0 && p.H % 4 == 0 && (p.b * p.H / 2) * p.nc < ((int64_t)1 << 30);
}

// dt is read by TMA, whose base address must be 16-byte aligned
bool tc_pair_supported(const Problem& p) {
  return tc_pair_shape_ok(p) && reinterpret_cast<uintptr_t>(p.dt) % 16 == 0;
}

static int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

// Split when the pairs alone would leave SMs idle and every SM gets at least
// two chunk steps; the state-only pass then costs about a third of a step per
// step, against SMs that would otherwise do nothing.
bool tc_pair_split(const Problem& p) {
  const int sms = sm_count();
  const int64_t npairs = p.b * p.H / 2;
  return sms > 0 && npairs < sms && npairs * p.nc >= 2 * (int64_t)sms;
}

cudaError_t tc_pair_launch(const Problem& p, const TcWorkspace& w, const CUtensorMap& tx, const CUtensorMap& tb,
                           const CUtensorMap& tc_, const CUtensorMap& tw, const CUtensorMap& ty,
                           const CUtensorMap& tdt, const tc::FastArgs& fa, cudaStream_t st) {
  cudaError_t e;
  for (auto* k : {k_ssd_fwd_pair<false>, k_ssd_fwd_pair<true>})
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PairCfg::kSmemBytes)) !=
        cudaSuccess)
      return e;
  const int sms = sm_count();
  if (sms == 0) return cudaErrorInvalidValue;
  tc::FastArgs a = fa;
  a.batch = p.b;
  a.handoff = w.handoff;
  a.flags = w.flags;
  a.pair_bad = w.pair_bad;
  a.seg_decay = w.seg_decay;
  a.split = 0;
  const int64_t npairs = p.b * p.H / 2;
  if (tc_pair_split(p)) {
    // one CTA per SM over equal ranges of the steps, the state-only pass first
    int64_t grid = sms < kPairGridMax ? sms : kPairGridMax;
    a.split = 1;
    if ((e = launch_dependent(k_ssd_fwd_pair<true>, (unsigned)grid, PairCfg::kThreads, PairCfg::kSmemBytes, st, tx,
                              tb, tc_, tw, ty, tdt, a)) != cudaSuccess)
      return e;
    return launch_dependent(k_ssd_fwd_pair<false>, (unsigned)grid, PairCfg::kThreads, PairCfg::kSmemBytes, st, tx,
                            tb, tc_, tw, ty, tdt, a);
  }
  // one CTA per SM over equal ranges of the pair-major steps; if a CTA would
  // touch more pairs than its segment table holds, one CTA per pair instead
  // (whole pairs only: no hand-over)
  int64_t grid = npairs < sms ? npairs : sms;
  if (grid > kPairGridMax) grid = kPairGridMax;
  if ((npairs + grid - 1) / grid + 2 > kPairMaxSeg) grid = npairs;
  return launch_dependent(k_ssd_fwd_pair<false>, (unsigned)grid, PairCfg::kThreads, PairCfg::kSmemBytes, st, tx, tb,
                          tc_, tw, ty, tdt, a);
}

}  // namespace ssd
