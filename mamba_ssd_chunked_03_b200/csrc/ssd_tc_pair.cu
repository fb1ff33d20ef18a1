// Two-head variant of the fast fused SSD forward (see ssd_tc_fast.cu for the
// factorised-decay formulation): one CTA owns two heads (h, h+1) of the same
// batch row and B/C group and walks their chunks together.  The heads share
// the C, B and W' = masked C B^T tiles, and every MMA covers both heads at
// once with M = 128 rows (p of head h, then p of head h+1):
//
//   Yd^T  = X'^T W'^T                 (N = 64 tokens t,  K = 64 tokens s)
//   S     = X'^T B                    (N = 128 states,   K = 64 tokens s)
//   Yd^T += H C^T                     (N = 64 tokens t,  K = N states)
//   y_t   = u_t Yd_t + D x_t,   H <- 2^cs_e (H + S)
//
// per head, with cs_t the in-chunk cumulative sum of dt A (log2 units),
// u_t = 2^cs_t, v_s = 2^-cs_s dt_s and X' = diag(v) x: u_t v_s = exp of the
// decay from s to t times dt_s.  The factors are taken about the chunk's
// first token (ssd_tc_fast.cu takes them about its middle), so the state
// enters the H C^T product as it is, with no per-chunk rescaling; a chunk
// whose total decay exceeds 2^kRangeLog2 sends the pair to the exact kernel.
// The chunked steps are those of "SSM 家族全景图（下）：Mamba-2 与 Jamba"
// section 三.4; the D feed-through is from "从Transformer的二次复杂度困境到Mamba
// 的线性突围" (continuous SSM).
//
// Both A operands live in tensor memory: X'^T (scaled from the x tile through
// 8 x 8 transposing loads) and the bf16 copy of the state.  Shared memory
// carries only the TMA tiles (x, W', B, C, dt), the MMAs' B operands and the
// y tile, which the epilogue writes over x in the same slot before a bulk
// tensor store per head moves it out.  The chunk-to-chunk chain is short: S
// of chunk g lands, the state warps load it, fold it into the fp32 state and
// store the next bf16 state; only then do they scale the x tile of chunk
// g + 2, off that chain, and the next chunk's S and W' products do not wait
// for the state.
//
// Warp roles (896 threads), each a loop over the chunks that only waits on
// the barriers it needs:
//   warp 0      TMA loads (one thread): W', B, C 2 chunks ahead
//   warp 1      MMA issue (descriptors formed by the warp, one elected lane issues)
//   warp 2      dt scan of both heads: u, v and the chunk scalars; it also
//               loads dt by TMA into an 8-deep ring of its own
//   warp 3      y stores and x loads (one thread): an x slot of the 8-slot
//               ring is refilled 8 chunks ahead once its y tile is read out
//   warps 4-11  the epilogue: warp 4 + 4 half + q owns TMEM rows 32q.. (head
//               q/2, p = 32 (q&1) + lane) and tokens [32 half, 32 half + 32)
//   warps 12-27 the state: warp 12 + 4 nq + q owns TMEM rows 32q.. and states
//               n in [32 nq, 32 nq + 32): fp32 state in registers, its bf16
//               copy in TMEM, and tokens [16 nq, 16 nq + 16) of the x scaling
//               into X'^T two chunks ahead
// TMEM (512 columns): Yd^T x2 (64 columns each), S x1 (128), the bf16 state x2
// (64), X'^T x4 (32).  Every wait is bounded; a CTA that times out records the
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
  static constexpr int kThreads = 896;
  static constexpr uint32_t kTile = 8192;
  // ring depths (steps of lead): x tiles (y is staged in place), W' + B, C, dt
  static constexpr int kXSlots = 8, kWbSlots = 2, kCSlots = 2, kDtSlots = 8;
  static constexpr int kWbMax = kWbSlots > 4 ? kWbSlots : 4;  // the state-only pass runs B 4 deep
  static constexpr uint32_t oX = 0;                                // [slots][2 heads] x -> y, in place
  static constexpr uint32_t oW = oX + 2 * kXSlots * kTile;         // [slots] W' tiles
  static constexpr uint32_t oB = oW + kWbSlots * kTile;            // [slots] B, 2 n-blocks each
  static constexpr uint32_t oC = oB + kWbSlots * NB * kTile;       // [slots] C, 2 n-blocks each
  static constexpr uint32_t oDt = oC + kCSlots * NB * kTile;       // [slots] dt boxes: 64 tokens x 4 heads fp32
  static constexpr uint32_t kDtBox = 64 * 16;
  static constexpr uint32_t oEnd = oDt + kDtSlots * kDtBox;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  // TMEM (M = 128 layout, row = lane = 64 j + p for head h0 + j):
  //   Yd^T[2] fp32, 64 columns (t) each;  S fp32, 128 columns (n);
  //   H[2] bf16, 64 columns (two n per column);  X'^T[4] bf16, 32 columns (two s per column)
  static constexpr uint32_t tYd0 = 0, tS = 128, tH0 = 256, tX0 = 384, kTmemCols = 512;
};

constexpr int kPairMaxSeg = 32;  // segments (pairs touched) per CTA, at most

// Slot and phase parity of step c (>= 0) in a ring of n buffers (unsigned
// arithmetic: a mask and a shift when n is a power of two).
template <int n>
__device__ __forceinline__ int ring_slot(int c) {
  return (int)((uint32_t)c % (uint32_t)n);
}
template <int n>
__device__ __forceinline__ uint32_t ring_par(int c) {
  return ((uint32_t)c / (uint32_t)n) & 1u;
}

// Ring barriers are indexed like the buffers they guard, so no barrier can
// complete a second phase before every waiter has seen the first.  A warp
// arrives once (lane 0, after each lane's own wait or fence and a __syncwarp,
// which orders the warp's accesses before that release), so the counts below
// are in warps: 32 times fewer shared-memory atomics than per-thread arrivals.
struct __align__(16) PairSmem {
  uint64_t full_x[PairCfg::kXSlots], x_empty[PairCfg::kXSlots];  // x ring: TMA landed / scaled (state-only pass)
  uint64_t full_dt[PairCfg::kDtSlots];   // dt ring (the scan warp's own)
  uint64_t full_wb[PairCfg::kWbMax];     // W' + B of a chunk landed (state-only pass: B)
  uint64_t wb_free[PairCfg::kWbMax];     // ... and read by its MMAs (state-only pass)
  uint64_t full_c[PairCfg::kCSlots];     // C of a chunk landed
  uint64_t scan_full[4], scan_empty[4];  // scan results of a chunk ready / consumed
  uint64_t xp_ready[4];                  // X'^T of a chunk in TMEM
  uint64_t s_full[2];                    // S of a chunk in TMEM
  uint64_t s_free[2];                    // S of a chunk read out by the state warps
  uint64_t mma_done[2];                  // every MMA of a chunk done: Yd final, C free
  uint64_t h_ready[2];                   // bf16 state for a chunk written to TMEM
  uint64_t acc_free[2];                  // Yd of a chunk read out by the epilogue
  uint64_t y_staged[PairCfg::kXSlots];   // y of a chunk written over its x slot
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
  float sc[4][2][4];  // [0]: d = 2^cs_e, the chunk's total decay; [1]: D of the head
};

static_assert(offsetof(PairSmem, u) % 16 == 0 && offsetof(PairSmem, v) % 16 == 0,
              "scan results are stored as float4");
static_assert(PairCfg::kSmemBytes + sizeof(PairSmem) <= 227 * 1024, "shared memory per CTA");

// Position of one of a CTA's step streams (each role walks its steps in
// order): segment k, chunk c.  next() moves to the following step.  kRev (the
// state-only pass, which has one segment) walks the segment's chunks from its
// last to its first.
template <bool kRev>
struct PairCursor {
  int k, c;
  __device__ __forceinline__ void start(const PairSmem& s) {
    k = 0;
    c = kRev ? s.seg_c0[0] + s.seg_len[0] - 1 : s.seg_c0[0];
  }
  __device__ __forceinline__ void next(const PairSmem& s) {
    if (kRev) {
      --c;
    } else if (++c == s.seg_c0[k] + s.seg_len[k] && k + 1 < s.nseg) {
      ++k;
      c = s.seg_c0[k];
    }
  }
};

// kStateOnly: the state-only pass of split mode.  Each CTA takes only the
// segment of its range that ends inside a pair (there is at most one: the
// head of its last pair), runs it from a zero state with x and B alone (no
// W', C, y) and leaves the end state in handoff and the segment's total decay
// per head in seg_decay.  It walks the segment from its last chunk to its
// first and scales each token's x by its decay to the segment's end (a factor
// of at most one, known as the walk goes: the chunks after it are done), so
// the end state is one MMA accumulation, S += X''^T B, that stays in tensor
// memory until the last chunk; no step waits for the state warps.
template <bool kStateOnly>
__global__ void __launch_bounds__(896, 1)
    k_ssd_fwd_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_dt,
                   const FastArgs a) {
  using K = PairCfg;
  using Cursor = PairCursor<kStateOnly>;
  // B (with W') ring depth.  The state-only pass needs no W' or C: its B ring
  // takes their space and runs 4 steps ahead, since its steps wait on nothing
  // else.
  constexpr int kBR = kStateOnly ? 4 : PairCfg::kWbSlots;
  // (the fused pass refills W', B and C on s_full and mma_done, which are 2 deep)
  static_assert(PairCfg::kWbSlots == 2 && PairCfg::kCSlots == 2, "fused-pass W'/B and C rings");
  static_assert(4 * PairCfg::NB * PairCfg::kTile <= PairCfg::oDt - PairCfg::oW, "state-only B ring");
  constexpr uint32_t oBr = kStateOnly ? PairCfg::oW : PairCfg::oB;
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
    for (int i = 0; i < K::kXSlots; ++i) {
      mbar_init(&s.full_x[i], 1);
      // the state-only pass stores no y: the x scalers (state warps) free the slot
      mbar_init(&s.x_empty[i], 16);
      mbar_init(&s.y_staged[i], 8);
    }
    for (int i = 0; i < K::kDtSlots; ++i) mbar_init(&s.full_dt[i], 1);
    for (int i = 0; i < K::kCSlots; ++i) mbar_init(&s.full_c[i], 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s.scan_full[i], 1);
      // the state warps, and in the fused pass the epilogue warps
      mbar_init(&s.scan_empty[i], kStateOnly ? 16 : 8 + 16);
      mbar_init(&s.xp_ready[i], 16);
    }
    for (int i = 0; i < K::kWbMax; ++i) {
      mbar_init(&s.full_wb[i], 1);
      mbar_init(&s.wb_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_free[i], 16);
      mbar_init(&s.mma_done[i], 1);
      mbar_init(&s.h_ready[i], 16);
      mbar_init(&s.acc_free[i], 8);
    }
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
    // ------------------------------------------------------------ TMA loads: W', B, C
    if (lane == 0) {
      int last_wb = -1, last_c = -1;
      // (the argument is this CTA's step number; each stream has a cursor on
      // its pair and chunk, advanced as the stream issues its steps in order)
      Cursor uwb, uc;
      uwb.start(s);
      uc.start(s);
      auto issue_wb = [&](int gg) {
        const int i = ring_slot<kBR>(gg), bb = s.seg_b[uwb.k], grp = s.seg_grp[uwb.k];
        mbar_arrive_expect_tx(&s.full_wb[i], (kStateOnly ? K::NB : 1 + K::NB) * K::kTile);
        if (!kStateOnly)
          tma_load_3d(sm + K::oW + i * K::kTile, &tm_w, &s.full_wb[i], 0, ((bb * nc + uwb.c) * (int)a.G + grp) * 64,
                      0);
        for (int jb = 0; jb < K::NB; ++jb)
          tma_load_4d(sm + oBr + (i * K::NB + jb) * K::kTile, &tm_b, &s.full_wb[i], 64 * jb, grp, uwb.c * 64, bb);
        uwb.next(s);
        last_wb = gg;
      };
      auto issue_c = [&](int gg) {
        const int i = ring_slot<K::kCSlots>(gg), bb = s.seg_b[uc.k], grp = s.seg_grp[uc.k];
        mbar_arrive_expect_tx(&s.full_c[i], K::NB * K::kTile);
        for (int jb = 0; jb < K::NB; ++jb)
          tma_load_4d(sm + K::oC + (i * K::NB + jb) * K::kTile, &tm_c, &s.full_c[i], 64 * jb, grp, uc.c * 64, bb);
        uc.next(s);
        last_c = gg;
      };
      if (!*abort_flag) {
        if (!kStateOnly) griddep_wait();  // W' comes from the C B^T kernel launched before this one
        #pragma unroll 1
        for (int c = 0; c < kBR && c < total; ++c) issue_wb(c);
        if (!kStateOnly)
          #pragma unroll 1
          for (int c = 0; c < K::kCSlots && c < total; ++c) issue_c(c);
      }
      bool ok = !*abort_flag;
      // each tile is refilled for a later chunk as soon as its MMAs are done:
      // the fused pass takes the two barriers its MMA warp commits anyway (S
      // done frees W' and B, every MMA done frees C: one commit more each on
      // the MMA warp's path measured 3% slower); the state-only pass has
      // barriers of its own for its deeper B ring
      #pragma unroll 1
      for (int c = 0; c < total && ok; ++c) {
        if (c + kBR < total) {
          ok = kStateOnly ? mbar_wait(&s.wb_free[ring_slot<kBR>(c)], ring_par<kBR>(c), abort_flag, kWaitLimitNs)
                          : mbar_wait(&s.s_full[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_wb(c + kBR);
        }
        if (!kStateOnly && ok && c + K::kCSlots < total) {
          ok = mbar_wait(&s.mma_done[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_c(c + K::kCSlots);
        }
      }
      if (*abort_flag) {  // let this CTA's own copies land before its smem is released
        #pragma unroll 1
        for (int c = last_wb - (kBR - 1) < 0 ? 0 : last_wb - (kBR - 1); c <= last_wb; ++c)
          mbar_wait(&s.full_wb[ring_slot<kBR>(c)], ring_par<kBR>(c), never, kWaitLimitNs);
        #pragma unroll 1
        for (int c = last_c - (K::kCSlots - 1) < 0 ? 0 : last_c - (K::kCSlots - 1); c <= last_c; ++c)
          mbar_wait(&s.full_c[ring_slot<K::kCSlots>(c)], ring_par<K::kCSlots>(c), never, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp walks the loop and forms the descriptors (warp-uniform
    // values); one elected lane issues the MMAs and commits.  A step's
    // barriers are probed together with non-blocking tests, whose latencies
    // overlap, and only one not yet complete is then waited for.
    auto need = [&](bool done, uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, done) || mbar_wait_warp(bar, parity, abort_flag, kWaitLimitNs);
    };
    // descriptors of buffer 0; buffer 1 lies a whole number of 8 KB tiles further
    const uint64_t dw0 = sw128_desc(smem_u32(sm + K::oW), 16, 1024);
    const uint64_t db0 = sw128_desc(smem_u32(sm + oBr), K::kTile, 1024);
    const uint64_t dc0 = sw128_desc(smem_u32(sm + K::oC), 16, 1024);
    constexpr uint32_t kTileDesc = K::kTile >> 4;  // an 8 KB tile in descriptor address units
    constexpr uint32_t id_y = idesc_bf16(128, 64, 0, 0);   // A in TMEM, B K-major
    constexpr uint32_t id_s = idesc_bf16(128, 128, 0, 1);  // A in TMEM, B MN-major
    #pragma unroll 1
    for (int c = 0; c < total; ++c) {
      const int i = c & 1, xb = c & 3, ib = ring_slot<kBR>(c), ic = ring_slot<K::kCSlots>(c);
      const uint32_t ph = (c >> 1) & 1, pxp = (c >> 2) & 1, pacc = ((c - 2) >> 1) & 1, psf = ((c - 1) >> 1) & 1;
      const uint32_t pb = ring_par<kBR>(c), pc = ring_par<K::kCSlots>(c);
      // (the state-only pass accumulates S over its whole segment: no S is read out between steps)
      const bool acc = !kStateOnly && c >= 2, sfree = !kStateOnly && c >= 1;
      const bool p_wb = mbar_probe(&s.full_wb[ib], pb);
      const bool p_xp = mbar_probe(&s.xp_ready[xb], pxp);
      const bool p_acc = !acc || mbar_probe(&s.acc_free[i], pacc);
      const bool p_sf = !sfree || mbar_probe(&s.s_free[(c - 1) & 1], psf);
      const bool p_c = kStateOnly || mbar_probe(&s.full_c[ic], pc);
      if (!need(p_wb, &s.full_wb[ib], pb) || !need(p_xp, &s.xp_ready[xb], pxp) ||
          (acc && !need(p_acc, &s.acc_free[i], pacc)))
        break;
      tc_fence_after();
      const uint32_t yd = tmem + K::tYd0 + 64 * i;
      const uint32_t ax = tmem + K::tX0 + 32 * xb;  // X'^T of both heads, this chunk
      const uint64_t dw = dw0 + ib * kTileDesc;
      const uint64_t db = db0 + ib * K::NB * kTileDesc;
      if (!kStateOnly) {
        // Yd^T = X'^T W'^T   (K = 64 tokens s; a K step is 32 bytes along the row)
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_bf16_ts(yd, ax + 8 * kk, dw + 2 * kk, id_y, kk > 0);
        }
        __syncwarp();
      }
      // S = X'^T B   (N = 128 states, K = 64 tokens s; a K step is 16 rows), once
      // the state warps have read out the previous chunk's S
      if (sfree && !need(p_sf, &s.s_free[(c - 1) & 1], psf)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + K::tS, ax + 8 * kk, db + 128 * kk, id_s, kk > 0 || (kStateOnly && c > 0));
        mma_commit(&s.s_full[i]);
        if (kStateOnly) mma_commit(&s.wb_free[ib]);  // the step's B has been read
      }
      __syncwarp();
      if (kStateOnly) continue;
      // Yd^T += H C^T   (K = N states)
      const bool p_h = mbar_probe(&s.h_ready[i], ph);
      if (!need(p_h, &s.h_ready[i], ph) || !need(p_c, &s.full_c[ic], pc)) break;
      tc_fence_after();
      const uint64_t dc = dc0 + ic * K::NB * kTileDesc;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk)
          mma_bf16_ts(yd, tmem + K::tH0 + 64 * i + 8 * kk, dc + ((kk >> 2) * K::kTile + (kk & 3) * 32) / 16, id_y,
                      1);
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
    Cursor ud, us;
    ud.start(s);
    us.start(s);
    auto issue_dt = [&](int gg) {
      const int sl = ring_slot<K::kDtSlots>(gg);
      mbar_arrive_expect_tx(&s.full_dt[sl], K::kDtBox);
      tma_load_3d(sm + K::oDt + sl * K::kDtBox, &tm_dt, &s.full_dt[sl], s.seg_h0[ud.k] & ~3, ud.c * 64,
                  s.seg_b[ud.k]);
      ud.next(s);
      last_dt = gg;
    };
    if (lane == 0 && !*abort_flag)
      #pragma unroll 1
      for (int c = 0; c < K::kDtSlots && c < total; ++c) issue_dt(c);
    int cur_seg = -1, col = 0;
    float a2 = 0.f, dsk = 0.f;
    float suf = 0.f;  // state-only pass: log2 decay from the end of this chunk to the segment's end
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
      if (!mbar_wait_warp(&s.full_dt[ring_slot<K::kDtSlots>(g)], ring_par<K::kDtSlots>(g), abort_flag, kWaitLimitNs))
        break;
      const float* dts = reinterpret_cast<const float*>(sm + K::oDt + ring_slot<K::kDtSlots>(g) * K::kDtBox);
      const int c = us.c;
      const int nvalid = (int)((int64_t)(c + 1) * 64 <= a.L ? 64 : a.L - (int64_t)c * 64);
      float d[4], cs[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) d[k] = dts[(4 * l16 + k) * 4 + col];
      __syncwarp();
      if (lane == 0 && g + K::kDtSlots < total) {  // the slot has been read: refill it
        fence_proxy_async_smem();
        issue_dt(g + K::kDtSlots);
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
      float u4[4], v4[4];
      bool bad = false;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        u4[k] = exp2f(cs[k]);
        // fused pass: v_s = 2^-cs_s dt_s (the chunk's first token as reference);
        // state-only pass: 2^(suf + cs_e - cs_s) dt_s, the decay to the segment's end
        v4[k] = kStateOnly ? exp2f(suf + cse - cs[k]) * d[k] : exp2f(-cs[k]) * d[k];
        bad |= !(fabsf(cs[k]) <= kRangeLog2);
      }
      if (kStateOnly) suf += cse;
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
      if (l16 == 0) {
        s.sc[slot][j][0] = exp2f(cse);
        s.sc[slot][j][1] = dsk;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.scan_full[slot]);
    }
    if (lane == 0 && *abort_flag)  // let the dt copies in flight land
      #pragma unroll 1
      for (int c = last_dt - (K::kDtSlots - 1) < 0 ? 0 : last_dt - (K::kDtSlots - 1); c <= last_dt; ++c)
        mbar_wait(&s.full_dt[ring_slot<K::kDtSlots>(c)], ring_par<K::kDtSlots>(c), never, kWaitLimitNs);
  } else if (warp == 3) {
    // ---------------------------------------------- y stores and x loads
    // An x slot is refilled (8 steps ahead) as soon as the y tile written
    // over it has been read out by its store; in the state-only pass, which
    // stores no y, as soon as the state warps have scaled it.  x comes from
    // HBM: L2 prefetches run 6 steps ahead of the loads (the steps 8-10 after
    // the first x loads are not prefetched).
    if (lane == 0) {
      int last_x = -1, pf = K::kXSlots + 3;  // pf: the step upf is at
      Cursor ux, uy, upf;
      ux.start(s);
      uy.start(s);
      upf.start(s);
      for (int k = 0; k < pf; ++k) upf.next(s);
      auto issue_x = [&](int gg) {
        const int sl = ring_slot<K::kXSlots>(gg), bb = s.seg_b[ux.k], hh = s.seg_h0[ux.k];
        mbar_arrive_expect_tx(&s.full_x[sl], 2 * K::kTile);
        for (int j = 0; j < 2; ++j)
          tma_load_3d(sm + K::oX + (sl * 2 + j) * K::kTile, &tm_x, &s.full_x[sl], (hh + j) * 64, ux.c * 64, bb);
        ux.next(s);
        last_x = gg;
      };
      auto prefetch_x = [&]() {  // step pf, if it is one of this CTA's
        if (pf < total) {
          const int bb = s.seg_b[upf.k], hh = s.seg_h0[upf.k];
          for (int j = 0; j < 2; ++j) tma_prefetch_l2_3d(&tm_x, (hh + j) * 64, upf.c * 64, bb);
        }
        upf.next(s);
        ++pf;
      };
      if (!*abort_flag) {
        #pragma unroll 1
        for (int c = K::kXSlots; c < K::kXSlots + 3 && c < total; ++c) prefetch_x();
        #pragma unroll 1
        for (int c = 0; c < K::kXSlots && c < total; ++c) issue_x(c);  // the ring starts free
      }
      #pragma unroll 1
      for (int c = 0; c < total && !*abort_flag; ++c) {
        const int sl = ring_slot<K::kXSlots>(c);
        if (!kStateOnly) {
          if (!mbar_wait(&s.y_staged[sl], ring_par<K::kXSlots>(c), abort_flag, kWaitLimitNs)) break;
          for (int j = 0; j < 2; ++j)
            tma_store_3d(&tm_y, sm + K::oX + (sl * 2 + j) * K::kTile, (s.seg_h0[uy.k] + j) * 64, uy.c * 64,
                         s.seg_b[uy.k]);
          bulk_commit_group();
          bulk_wait_read<0>();  // the tiles have been read out: the slot may be refilled
          uy.next(s);
        } else if (!mbar_wait(&s.x_empty[sl], ring_par<K::kXSlots>(c), abort_flag, kWaitLimitNs)) {
          break;
        }
        if (c + K::kXSlots < total) {
          issue_x(c + K::kXSlots);
          prefetch_x();
        }
      }
      if (*abort_flag)  // let this CTA's own x copies land before its smem is released
        #pragma unroll 1
        for (int c = last_x - (K::kXSlots - 1) < 0 ? 0 : last_x - (K::kXSlots - 1); c <= last_x; ++c)
          mbar_wait(&s.full_x[ring_slot<K::kXSlots>(c)], ring_par<K::kXSlots>(c), never, kWaitLimitNs);
      bulk_wait<0>();  // stores complete before the CTA's shared memory is released
    }
  } else if (warp < 12) {
    // ------------------------------------------------ epilogue warps (both heads)
    // Warp 4 + 4 half + q reads Yd^T rows 32q.. (head q/2, p = 32 (q&1) + ..)
    // at tokens [32 half, 32 half + 32) with the 16x256b shape, which gives
    // each thread (p, t..t+1) pairs: 8 x 8 blocks in the layout of an 8 x 8
    // transpose.  Per block, x is loaded as (t, p..p+1) and transposed to
    // (p, t..t+1), y = u_t Yd + D x is formed in fp32, and the bf16 result is
    // transposed back and stored where x was read.
    if constexpr (!kStateOnly) {
      const int q = warp & 3;
      const int j = q >> 1;                   // head h0 + j
      const int ch = 32 * ((warp - 4) >> 2);  // first token of this warp's half
      const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
      #pragma unroll 1
      for (int c = 0; c < total; ++c) {
        const int ip = c & 1, sl = ring_slot<K::kXSlots>(c), sc4 = c & 3;
        if (!mbar_wait_warp(&s.mma_done[ip], (c >> 1) & 1, abort_flag, kWaitLimitNs)) break;
        tc_fence_after();
        const float dj = s.sc[sc4][j][1];
        // Both 16-lane Yd loads and the x loads are issued before any y store.
        // x block group G = 2 lh + e (rows p = 32 (q&1) + 16 lh + 8 e + ..) is
        // read with one transposing 4-matrix load, matrix jj holding tokens
        // ch + 8 jj + ..: register jj then pairs with the Yd registers
        // 16 lh + 4 jj + 2 e (+1).  y goes back the same way.
        const uint32_t xt_a = smem_u32(sm + K::oX + (sl * 2 + j) * K::kTile);
        uint32_t r[32];
        uint32_t* r_hi = r + 16;
        SSD_TMEM_LD_16x256b_X4(tq + K::tYd0 + 64 * ip + ch, r);
        SSD_TMEM_LD_16x256b_X4(tq + (16u << 16) + K::tYd0 + 64 * ip + ch, r_hi);
        const uint32_t trow = ch + 8 * (lane >> 3) + (lane & 7);  // the row this thread addresses
        uint32_t xv[4][4];
#pragma unroll
        for (int G = 0; G < 4; ++G)
          ldmatrix_x4_trans(xt_a + sw128(trow * 128 + (32 * (q & 1) + 8 * G) * 2), xv[G]);
        SSD_TMEM_WAIT_LD_32(r);
        const float2 dj2 = make_float2(dj, dj);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float2 u2 = *reinterpret_cast<const float2*>(&s.u[sc4][j][ch + 8 * jj + 2 * (lane & 3)]);
#pragma unroll
          for (int G = 0; G < 4; ++G) {
            // y = u_t Yd + D x_t for the pair (p, t), (p, t+1), two lanes of fp32 per instruction
            const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv[G][jj]));
            const uint32_t* rr = r + 16 * (G >> 1) + 4 * jj + 2 * (G & 1);
            const float2 o2 =
                __ffma2_rn(u2, make_float2(__uint_as_float(rr[0]), __uint_as_float(rr[1])), __fmul2_rn(dj2, x2));
            xv[G][jj] = pack_bf16x2(o2.x, o2.y);
          }
        }
#pragma unroll
        for (int G = 0; G < 4; ++G)
          stmatrix_x4_trans(xt_a + sw128(trow * 128 + (32 * (q & 1) + 8 * G) * 2), xv[G]);
        tc_fence_before();         // this thread's reads of Yd of step c are done
        fence_proxy_async_smem();  // its y stores are visible to the bulk store
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.acc_free[ip]);
          mbar_arrive(&s.y_staged[sl]);
          mbar_arrive(&s.scan_empty[sc4]);
        }
      }
    }
  } else {
    // ------------------------------------------------ state warps
    // The warp holds rows 32q.. (head q/2) and states n in [32 nq, 32 nq + 32)
    // of S and H in the layout of the 16x256b TMEM shape: H[16 m2 + 4 jj + 2 hi + e]
    // is row p = 32 (q&1) + 16 m2 + 8 hi + lane/4, state n = 32 nq + 8 jj +
    // 2 (lane%4) + e.  Each thread then owns (n, n+1) pairs, so a warp's global
    // accesses of a state touch 8 rows x 32 contiguous bytes per instruction.
    const int q = warp & 3;
    const int j = q >> 1;                // head h0 + j
    const int nq = (warp - 12) >> 2;
    const int uw = warp - 12;            // this warp's part of a state hand-over
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    float H[32];
    float dprod = 1.f;  // state-only pass: the segment's total decay so far
    // row p and state n of the pair (H[hk], H[hk + 1]) for m = 2 m2 + hi
    auto st_row = [&](int m) { return 32 * (q & 1) + 16 * (m >> 1) + 8 * (m & 1) + (lane >> 2); };
    auto st_col = [&](int jj) { return 32 * nq + 8 * jj + 2 * (lane & 3); };
    auto st_idx = [&](int m, int jj) { return 16 * (m >> 1) + 4 * jj + 2 * (m & 1); };
    // the bf16 copy of H for step gg (the state before it) into its TMEM buffer
    // (column c holds states 2c, 2c+1); the MMAs that read that buffer two
    // steps earlier are done (every MMA before the last S this warp has seen is)
    auto publish = [&](int gg) {
#pragma unroll
      for (int m2 = 0; m2 < 2; ++m2) {
        uint32_t r[8];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          r[2 * jj] = pack_bf16x2(H[16 * m2 + 4 * jj], H[16 * m2 + 4 * jj + 1]);
          r[2 * jj + 1] = pack_bf16x2(H[16 * m2 + 4 * jj + 2], H[16 * m2 + 4 * jj + 3]);
        }
        SSD_TMEM_ST_16x128b_X4(tq + ((uint32_t)(16 * m2) << 16) + K::tH0 + 64 * (gg & 1) + 16 * nq, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.h_ready[gg & 1]);
    };
    // X'^T of step cc, rows 32q.. (p = 32 (q&1) + ..) and tokens
    // [16 nq, 16 nq + 16), into TMEM in 8 x 8 blocks.  Per half mh (rows
    // 16 mh.. of the warp's 32) one transposing 4-matrix load reads matrix
    // k = 2 e + jj: x at tokens 16 nq + 8 jj + .. and p = 32 (q&1) + 16 mh +
    // 8 e + ..; register k then holds (p, s..s+1), which is scaled by v_s,
    // v_s+1 and stored with the 16x128b shape (two tokens per column, repeat
    // jj, lanes + 8 e).  The X'^T buffer of step cc was last read by the MMAs
    // of step cc - 4, which are done once S of step cc - 2 is.
    auto scale = [&](int cc) -> bool {
      const int sl = ring_slot<K::kXSlots>(cc), xb = cc & 3;
      const bool p_v = mbar_probe(&s.scan_full[cc & 3], (cc >> 2) & 1);
      const bool p_x = mbar_probe(&s.full_x[sl], ring_par<K::kXSlots>(cc));
      if ((!__all_sync(0xffffffffu, p_v) &&
           !mbar_wait_warp(&s.scan_full[cc & 3], (cc >> 2) & 1, abort_flag, kWaitLimitNs)) ||
          (!__all_sync(0xffffffffu, p_x) &&
           !mbar_wait_warp(&s.full_x[sl], ring_par<K::kXSlots>(cc), abort_flag, kWaitLimitNs)))
        return false;
      tc_fence_after();
      const uint32_t xt_a = smem_u32(sm + K::oX + (sl * 2 + j) * K::kTile);
      const int k = lane >> 3;  // the matrix this thread addresses a row of
      const uint32_t srow = 16 * nq + 8 * (k & 1) + (lane & 7);
      __nv_bfloat162 w2[2];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const float2 v2 = *reinterpret_cast<const float2*>(&s.v[cc & 3][j][16 * nq + 8 * jj + 2 * (lane & 3)]);
        w2[jj] = __floats2bfloat162_rn(v2.x, v2.y);
      }
#pragma unroll
      for (int mh = 0; mh < 2; ++mh) {
        uint32_t xv[4];
        ldmatrix_x4_trans(xt_a + sw128(srow * 128 + (32 * (q & 1) + 16 * mh + 8 * (k >> 1)) * 2), xv);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const __nv_bfloat162 x2 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&xv[m]), w2[m & 1]);
          xv[m] = *reinterpret_cast<const uint32_t*>(&x2);
        }
        const uint32_t taddr = tq + ((uint32_t)(16 * mh) << 16) + K::tX0 + 32 * xb + 8 * nq;
        asm volatile("tcgen05.st.sync.aligned.16x128b.x2.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(xv[0]),
                     "r"(xv[2]), "r"(xv[1]), "r"(xv[3])
                     : "memory");
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s.xp_ready[xb]);
        if (kStateOnly) mbar_arrive(&s.x_empty[sl]);  // no epilogue reads this x tile
      }
      return true;
    };
    // state at the start of segment k: h0 (or zero) at a pair's first chunk,
    // otherwise this warp's part of the hand-over the previous CTA wrote, or
    // in split mode h0 carried through the state-only pass's local states of
    // the CTAs before this one (each: H <- decay H + S).  The state-only pass
    // itself starts every segment from zero.
    auto seg_begin = [&](int k) -> bool {
      const int64_t h = s.seg_h0[k] + j, bb = s.seg_b[k];
      if (kStateOnly) {
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) H[kk] = 0.f;
        dprod = 1.f;
        return true;
      }
      if (s.seg_c0[k] == 0 || a.split) {
        if (a.h0 && 32 * nq < a.Nr) {  // (16-byte aligned: the library checks it)
          const float* src = a.h0 + (bb * a.H + h) * 64 * a.Nr;
#pragma unroll
          for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const float2 v = *reinterpret_cast<const float2*>(src + (int64_t)st_row(m) * a.Nr + st_col(jj));
              H[st_idx(m, jj)] = v.x;
              H[st_idx(m, jj) + 1] = v.y;
            }
        } else {
#pragma unroll
          for (int kk = 0; kk < 32; ++kk) H[kk] = 0.f;
        }
        if (s.seg_c0[k] == 0) return true;
        griddep_wait();  // the state-only pass launched before this kernel
        #pragma unroll 1
        for (int ip = s.seg_i0[k]; ip < (int)blockIdx.x; ++ip) {
          const float dd = __ldcg(a.seg_decay + 2 * ip + j);
          const float* src = a.handoff + (size_t)ip * kPairHandoffFloats + (size_t)j * 64 * 128;
#pragma unroll
          for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const float2 v = __ldcg(reinterpret_cast<const float2*>(src + st_row(m) * 128 + st_col(jj)));
              H[st_idx(m, jj)] = fmaf(dd, H[st_idx(m, jj)], v.x);
              H[st_idx(m, jj) + 1] = fmaf(dd, H[st_idx(m, jj) + 1], v.y);
            }
        }
        return true;
      }
      const int slot = (int)blockIdx.x - 1;
      bool ok = true;
      const int* flag = a.flags + (a.stall ? kPairNeverFlag : slot * kPairFlagsPerCta + uw);
      if (lane == 0) ok = wait_flag_acquire(flag, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) return false;
      const float* src = a.handoff + (size_t)slot * kPairHandoffFloats + (size_t)j * 64 * 128;
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(src + st_row(m) * 128 + st_col(jj)));
          H[st_idx(m, jj)] = v.x;
          H[st_idx(m, jj) + 1] = v.y;
        }
      return true;
    };
    // state at the end of segment k: the pair's final state, or the hand-over
    // to the next CTA: the data now, this warp's release flag (after a fence)
    // a few steps later, when the stores have long reached L2 and the fence
    // no longer waits for them.  The next CTA reads the hand-over only at the
    // end of its own range.
    int release_at = -1;  // step after which the pending hand-over flag is released
    auto release = [&]() {
      __threadfence();
      __syncwarp();
      if (lane == 0) store_flag_release(a.flags + (int)blockIdx.x * kPairFlagsPerCta + uw, 1);
      release_at = -1;
    };
    auto seg_end = [&](int k) {
      const int64_t h = s.seg_h0[k] + j, bb = s.seg_b[k];
      float* hand = a.handoff + (size_t)blockIdx.x * kPairHandoffFloats + (size_t)j * 64 * 128;
      auto put_handoff = [&]() {
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            __stcg(reinterpret_cast<float2*>(hand + st_row(m) * 128 + st_col(jj)),
                   make_float2(H[st_idx(m, jj)], H[st_idx(m, jj) + 1]));
      };
      if (kStateOnly) {  // the local end state and the total decay, for the CTAs after this one
        put_handoff();
        if (lane == 0 && nq == 0 && (q & 1) == 0) __stcg(a.seg_decay + 2 * blockIdx.x + j, dprod);
        return;
      }
      if (s.seg_c0[k] + s.seg_len[k] == nc) {
        if (a.final_states && 32 * nq < a.Nr) {  // (16-byte aligned: the library checks it)
          float* dst = a.final_states + (bb * a.H + h) * 64 * a.Nr;
#pragma unroll
          for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              *reinterpret_cast<float2*>(dst + (int64_t)st_row(m) * a.Nr + st_col(jj)) =
                  make_float2(H[st_idx(m, jj)], H[st_idx(m, jj) + 1]);
        }
        return;
      }
      if (a.split) return;  // the CTAs after this one start from the state-only pass
      put_handoff();
      release_at = s.seg_g0[k] + s.seg_len[k] + 2;
    };
    // Per step g: wait for S of g, fold it into H (H <- d (H + S)), publish
    // the bf16 H for step g + 1 unless the segment ends there, then scale the
    // x tile of step g + 2.
    bool failed = false;
    #pragma unroll 1
    for (int c = 0; c < 2 && c < total && !failed; ++c) failed = !scale(c);
    const int nseg = s.nseg;
    #pragma unroll 1
    for (int k = 0; k < nseg && !failed; ++k) {
      if (!seg_begin(k)) {
        failed = true;
        break;
      }
      const int g0 = s.seg_g0[k], g_end = g0 + s.seg_len[k];
      if (!kStateOnly) publish(g0);
      #pragma unroll 1
      for (int g = g0; g < g_end; ++g) {
        const int i = g & 1;
        if (!mbar_wait_warp(&s.s_full[i], (g >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          break;
        }
        tc_fence_after();
        if constexpr (kStateOnly) {
          // S accumulates in TMEM; the wait above only orders the reuse of
          // X'^T buffers (scale below)
          dprod *= s.sc[g & 3][j][0];
        } else {
          uint32_t r[32];
          uint32_t* r_hi = r + 16;
          SSD_TMEM_LD_16x256b_X4(tq + K::tS + 32 * nq, r);
          SSD_TMEM_LD_16x256b_X4(tq + (16u << 16) + K::tS + 32 * nq, r_hi);
          SSD_TMEM_WAIT_LD_32(r);
          tc_fence_before();  // this thread's reads of S of step g are done
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.s_free[i]);
          // H <- d (H + S), two lanes of fp32 per instruction
          const float dd = s.sc[g & 3][j][0];
          const float2 d2 = make_float2(dd, dd);
#pragma unroll
          for (int kk = 0; kk < 32; kk += 2) {
            const float2 h2 = __fadd2_rn(make_float2(H[kk], H[kk + 1]),
                                         make_float2(__uint_as_float(r[kk]), __uint_as_float(r[kk + 1])));
            const float2 o2 = __fmul2_rn(d2, h2);
            H[kk] = o2.x;
            H[kk + 1] = o2.y;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.scan_empty[g & 3]);  // this step's scalars are read
        if (!kStateOnly && g + 1 < g_end) publish(g + 1);
        if (g + 2 < total && !scale(g + 2)) {
          failed = true;
          break;
        }
        if (g == release_at) release();
      }
      if (kStateOnly && !failed && g_end > g0) {
        // the segment's end state: every MMA is done (S of its last step was waited for)
        uint32_t r[32];
        uint32_t* r_hi = r + 16;
        SSD_TMEM_LD_16x256b_X4(tq + K::tS + 32 * nq, r);
        SSD_TMEM_LD_16x256b_X4(tq + (16u << 16) + K::tS + 32 * nq, r_hi);
        SSD_TMEM_WAIT_LD_32(r);
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) H[kk] = __uint_as_float(r[kk]);
      }
      if (!failed) seg_end(k);
    }
    if (release_at >= 0 && !failed) release();
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
