// Fast fused chunked SSD forward on sm_100a (tcgen05 + TMEM + TMA), for the
// common case where every chunk's decay range is moderate.
//
// Three kernels:
//
// k_seq_runs (packed sequences only): lists each sequence as a run (row,
//   first token, length, id), so that every sequence is chunked from its own
//   first token and the two kernels below take it as an independent problem.
//   k_zero_absent then zeroes the final states of ids that no run carries.
//
// k_chunk_cb (one CTA per chunk -- of a batch row, or of a run -- and B/C group): the head-independent
//   part of the intra-chunk "attention",
//       W'[t][s] = C_t . B_s  if s <= t, both tokens valid and in the same
//                             packed sequence, else 0          (bf16, 64 x 64)
//   (the masked C B^T of the dual form, "22 · Mamba 2 — Transformers are
//   SSMs" section 3.2), computed once and shared by all heads of the group.
//
// k_ssd_fwd_fast (one CTA per (batch row, head), or per (run, head), chunks in
//   order, the running state kept on chip).  With cs_t the in-chunk cumulative sum of dt*A (log2
//   units) and m = cs at the chunk's midpoint, the decay between tokens s <= t
//   factorises as exp2(cs_t - cs_s) = u_t v_s / dt_s with
//       u_t = exp2(cs_t - m),   v_s = exp2(m - cs_s) dt_s,
//   both within 2^+-kRangeLog2 when the chunk's cumsum stays that close to m.
//   Then
//       X'  = diag(v) X                                      (one scaling pass)
//       Yd  = (W' + diag(D_h / dt)) X' + C (e^m H_c)^T       (one accumulator)
//       y_t = u_t Yd_t
//       S'  = B^T X',   H_{c+1} = exp2(cs_e) H_c + exp2(cs_e - m) S'
//   which are the four chunked steps of "SSM 家族全景图（下）：Mamba-2 与 Jamba"
//   section 三.4 plus the D skip ("从Transformer的二次复杂度困境到Mamba的线性突围",
//   continuous SSM equations; u_t (D/dt_t) v_t x_t = D x_t since u_t v_t = dt_t):
//   the intra-chunk output (W' X' scaled by u), the chunk state
//   (S'), the state passing (H), and the correction from the chunk's true
//   initial state (the C H^T term, whose per-row factor exp2(cs_t) equals
//   u_t e^m).  A (batch row, head) unit with any chunk out of that range is
//   appended to a list; the exact kernel (ssd_tc.cu), which forms every decay
//   separately, then recomputes those units and overwrites their outputs.
//
// Warp roles (320 threads): warp 0 computes the in-chunk cumulative sums and
// factor vectors two chunks ahead and issues the TMA loads (x in a 3-deep
// ring, scaled in place; W' and C 2-deep; B one tile; each refilled as soon as
// its last reader is done);
// warp 1 issues the MMAs (the whole warp forms the descriptors, one elected
// lane issues); warps 2-9 scale x, update the state and
// write y.  Yd and S are double-buffered in TMEM so chunk c's MMAs
// overlap chunk c-1's state update and epilogue.  Every wait is bounded; a
// CTA that times out records the error, drains its copies and MMAs, frees its
// TMEM and exits.
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

// ============================================================== k_seq_runs
// One CTA lists the runs of equal seq_idx: in row-major token order, a run
// starts at every token whose id differs from the token before it in the same
// row ("Transformers与SSMs的隐藏联系" section 4.2: the decay is cut exactly
// there).  Each run is an independent problem: its state starts from h0 if it
// is its row's first run, else from zero, and its final state is that
// sequence's.  The list is usable when the ids are strictly increasing along
// it and lie in [0, num_seqs) (each id one run); otherwise count = 0 and every
// (row, head) unit is put on the exact kernel's list.
struct SeqRunArgs {
  const int32_t* seq;
  int64_t b, L, H, num_seqs;
  RunList runs;
  int* failed_count;
  int* failed_list;
};

// exclusive prefix sum over the 1024 threads of the block; *total gets the sum
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* total, int64_t* warp_sums) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int64_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int64_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int64_t before = (wid > 0 ? warp_sums[wid - 1] : 0) + incl - v;
  *total = warp_sums[31];
  __syncthreads();  // warp_sums may be reused by the caller's next scan
  return before;
}

__global__ void __launch_bounds__(1024) k_seq_runs(const SeqRunArgs a) {
  __shared__ int64_t warp_sums[32];
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) bad = 0;
  const int64_t total = a.b * a.L;
  // Each warp takes a contiguous range of tokens (a multiple of 32) and reads
  // it 32 consecutive tokens at a time, 16 iterations of loads in flight: a
  // token opens a run at its row's start or where its id differs from the
  // token before (the lane below, or the previous iteration's last lane).
  // Each lane keeps its token's position in the row as a counter.
  const int64_t per_w = ((total + 31) / 32 + 31) / 32 * 32;
  const int64_t wlo = (int64_t)wid * per_w < total ? (int64_t)wid * per_w : total;
  const int64_t whi = wlo + per_w < total ? wlo + per_w : total;
  const int64_t i0 = wlo + lane;
  const int64_t row0 = i0 / a.L, pos0 = i0 - row0 * a.L;
  const int before = wlo > 0 && wlo < total ? a.seq[wlo - 1] : 0;
  constexpr int kBatch = 16;
  // walk the range; visit(base, ballot of starts, is_start, id, row, pos) per 32 tokens
  auto walk = [&](auto&& visit) {
    int64_t pos = pos0, row = row0;
    int carry = before;
    for (int64_t b0 = wlo; b0 < whi; b0 += 32 * kBatch) {
      int cur[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t i = b0 + 32 * u + lane;
        cur[u] = i < whi ? a.seq[i] : 0;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t base = b0 + 32 * u;
        if (base >= whi) break;  // (uniform across the warp)
        int prev = __shfl_up_sync(0xffffffffu, cur[u], 1);
        if (lane == 0) prev = carry;
        const bool st = base + lane < whi && (pos == 0 || cur[u] != prev);
        const uint32_t bal = __ballot_sync(0xffffffffu, st);
        visit(bal, st, cur[u], row, pos);
        carry = __shfl_sync(0xffffffffu, cur[u], 31);
        pos += 32;
        while (pos >= a.L) {
          pos -= a.L;
          ++row;
        }
      }
    }
  };
  int64_t cnt = 0;
  walk([&](uint32_t bal, bool, int, int64_t, int64_t) { cnt += __popc(bal); });
  // warp counts -> each warp's first run index (lane 0 contributes the warp's count)
  int64_t nr = 0;
  const int64_t k0 = block_exclusive_scan(lane == 0 ? cnt : 0, &nr, warp_sums);
  const int64_t kw = __shfl_sync(0xffffffffu, k0, 0);
  const bool fits = nr <= a.num_seqs;
  if (fits) {
    int64_t k = kw;
    walk([&](uint32_t bal, bool st, int id, int64_t row, int64_t pos) {
      if (st) {
        const int64_t at = k + __popc(bal & ((1u << lane) - 1u));
        a.runs.b[at] = (int)row;
        a.runs.t0[at] = (int)pos;
        a.runs.id[at] = id;
      }
      k += __popc(bal);
    });
  }
  __syncthreads();
  // lengths, the id checks and the chunk counts, per block of runs
  const int64_t rper = (nr + 1023) / 1024;
  const int64_t rlo = fits && tid * rper < nr ? tid * rper : nr;
  const int64_t rhi = fits && rlo + rper < nr ? rlo + rper : nr;
  int64_t chunks = 0;
  for (int64_t r = rlo; r < rhi; ++r) {
    const bool last_in_row = r + 1 >= nr || a.runs.b[r + 1] != a.runs.b[r];
    const int len = last_in_row ? (int)(a.L - a.runs.t0[r]) : a.runs.t0[r + 1] - a.runs.t0[r];
    a.runs.len[r] = len;
    const int id = a.runs.id[r];
    if (id < 0 || id >= a.num_seqs || (r > 0 && id <= a.runs.id[r - 1])) bad = 1;
    chunks += (len + 63) / 64;
  }
  int64_t nchunks = 0;
  int64_t c = block_exclusive_scan(chunks, &nchunks, warp_sums);
  for (int64_t r = rlo; r < rhi; ++r) {
    a.runs.c0[r] = (int)c;
    c += (a.runs.len[r] + 63) / 64;
  }
  if (tid == 0 && fits) a.runs.c0[nr] = (int)nchunks;
  __syncthreads();
  if (!fits || bad) {
    for (int64_t u = tid; u < a.b * a.H; u += 1024) a.failed_list[u] = (int)u;
    if (tid == 0) {
      *a.runs.count = 0;
      *a.failed_count = (int)(a.b * a.H);
    }
  } else {
    // the runs longest first: rank = runs with more chunks, or as many and earlier
    if (nr <= kRunSortMax) {
      for (int64_t r = tid; r < nr; r += 1024) {
        const int cr = (a.runs.len[r] + 63) / 64;
        int rank = 0;
        for (int64_t q = 0; q < nr; ++q) {
          const int cq = (a.runs.len[q] + 63) / 64;
          rank += cq > cr || (cq == cr && q < r);
        }
        a.runs.order[rank] = (int)r;
      }
    } else {
      for (int64_t r = tid; r < nr; r += 1024) a.runs.order[r] = (int)r;
    }
    if (tid == 0) *a.runs.count = (int)nr;
  }
}

// ============================================================== k_zero_absent
// The final state of an id that no run carries (an id in [0, num_seqs) that
// never occurs in seq_idx) is zero; the fused kernel writes every run's.  A
// usable list with num_seqs runs carries every id, and the kernel exits after
// one load.  With an unusable list (count 0) every id is zeroed here, and the
// exact kernel, later on the same stream, writes the ids that occur.
constexpr int kZeroSlices = 16;  // blocks' shares of one id's H x P x N floats

__global__ void __launch_bounds__(256) k_zero_absent(const RunList runs, float* final_states, int64_t num_seqs,
                                                     int64_t per_id) {
  const int nr = *runs.count;
  if (nr == num_seqs) return;  // (uniform) every id has its run
  for (int64_t item = blockIdx.x; item < num_seqs * kZeroSlices; item += gridDim.x) {
    const int64_t id = item / kZeroSlices, sl = item % kZeroSlices;
    int lo = 0, hi = nr;  // the runs' ids are strictly increasing: the first >= id
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (runs.id[mid] < id) lo = mid + 1; else hi = mid;
    }
    if (lo < nr && runs.id[lo] == id) continue;  // (uniform) written by the fused kernel
    float* dst = final_states + id * per_id;
    const int64_t a0 = per_id * sl / kZeroSlices, a1 = per_id * (sl + 1) / kZeroSlices;
    for (int64_t i = a0 + threadIdx.x; i < a1; i += blockDim.x) dst[i] = 0.f;
  }
}

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
  griddep_launch_dependents();  // the fused kernel may set up while this grid runs
  // tile r = chunk * G + g; the chunk is (row, 64-token chunk) or, for packed
  // sequences, (run, 64-token chunk of the run)
  const int64_t r = blockIdx.x;
  const int64_t g = r % a.G;
  int64_t b;
  int t0, nvalid;
  if (a.varlen) {
    const int nrun = *a.runs.count;
    const int64_t ch = r / a.G;
    if (nrun == 0 || ch >= a.runs.c0[nrun]) return;  // past the runs' chunks (uniform)
    int lo = 0, hi = nrun - 1;  // the run holding chunk ch: the last with c0 <= ch
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.runs.c0[mid] <= ch) lo = mid; else hi = mid - 1;
    }
    const int c = (int)(ch - a.runs.c0[lo]);
    b = a.runs.b[lo];
    t0 = a.runs.t0[lo] + 64 * c;
    nvalid = a.runs.len[lo] - 64 * c < 64 ? a.runs.len[lo] - 64 * c : 64;
  } else {
    const int64_t c = (r / a.G) % a.nc;
    b = r / (a.G * a.nc);
    t0 = (int)(c * 64);
    nvalid = (int)((c + 1) * 64 <= a.L ? 64 : a.L - t0);
  }
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
      tma_load_4d(sm + K::oC + j * K::kTile, &tm_c, &bar_full, 64 * j, (int)g, t0, (int)b);
      tma_load_4d(sm + K::oB + j * K::kTile, &tm_b, &bar_full, 64 * j, (int)g, t0, (int)b);
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

  // W' = masked C B^T -> bf16, row-major 64 x 64 per (b, c, g)
  const bool ok = mbar_wait_warp(&bar_mma, 0, abort_p, kWaitLimitNs);
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
  static constexpr uint32_t oX = 0;                          // [3] x tiles, scaled in place to X'
  static constexpr uint32_t oW = oX + 3 * kTile;             // [2] W' tiles
  static constexpr uint32_t oB = oW + 2 * kTile;             // B, NB tiles
  static constexpr uint32_t oC = oB + NB * kTile;            // [2] C, NB tiles each
  static constexpr uint32_t oH = oC + 2 * NB * kTile;        // bf16 e^m H, NB tiles
  static constexpr uint32_t oEnd = oH + NB * kTile;
  static constexpr uint32_t kSmemBytes = oEnd + 1024;
  // TMEM columns: Yd[2] (M = 64 layout) then S^T[2] (M = 128 rows per half)
  static constexpr uint32_t tYd0 = 0, tS0 = 128;
  static constexpr uint32_t kSCols = 64 * NH;
  static constexpr uint32_t kTmemCols = NS <= 128 ? 256 : 512;
  static constexpr int kMinBlocks = NS <= 128 ? 2 : 1;
};

struct __align__(8) FastSmem {
  uint64_t full_x[3], x_empty[3], full_w[2], w_empty[2], full_b, b_free, full_c[2], c_free[2];
  // xp_ready is a ring like the x tiles it announces, so it cannot complete a
  // second phase before the MMA thread has seen the first
  uint64_t scan_full[4], scan_empty[4], xp_ready[3], h_ready, h_free;
  uint64_t s_full[2], s_free[2], y_full[2], y_free[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int never;
  int unit_bad;
  float u[4][64];   // per scan slot: exp2(cs_t - m)
  float v[4][64];   // per scan slot: exp2(m - cs_s) dt_s
  float dt[4][64];  // per scan slot: dt (0 past the end of the sequence)
  float sc[4][4];   // per scan slot: E = 2^m, f = 2^(cs_e - m), d = 2^cs_e
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
  griddep_launch_dependents();  // the exact kernel may set up while this grid runs
  // the unit: (batch row, head), or for packed sequences (run, head) -- tokens
  // [t_base, t_base + len) of row b, chunked from t_base
  const int64_t unit = blockIdx.x;
  const int64_t h = unit % a.H;
  int64_t b, out_row, cbase;
  int t_base, len;
  if (a.varlen) {
    const int64_t pos = unit / a.H;
    if (pos >= *a.runs.count) return;  // past the runs (uniform)
    const int64_t ru = a.runs.order[pos];  // the longest runs first
    b = a.runs.b[ru];
    t_base = a.runs.t0[ru];
    len = a.runs.len[ru];
    out_row = a.runs.id[ru];       // final state: the sequence's
    cbase = a.runs.c0[ru];         // W' of the run's chunks
  } else {
    b = unit / a.H;
    t_base = 0;
    len = (int)a.L;
    out_row = b;
    cbase = b * a.nc;
  }
  const bool first = t_base == 0;  // h0 is the state before a row's first token
  const int64_t g = h / a.hpg;
  const int nc = (len + 63) / 64;
  const int64_t rowbase = b * a.L + t_base;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s.scan_full[i], 32);
      mbar_init(&s.scan_empty[i], 256);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&s.full_x[i], 1);
      mbar_init(&s.x_empty[i], 1);
      mbar_init(&s.xp_ready[i], 256);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full_c[i], 1);
      mbar_init(&s.c_free[i], 1);
      mbar_init(&s.full_w[i], 1);
      mbar_init(&s.w_empty[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_free[i], 256);
      mbar_init(&s.y_full[i], 1);
      mbar_init(&s.y_free[i], 256);
    }
    mbar_init(&s.full_b, 1);
    mbar_init(&s.b_free, 1);
    mbar_init(&s.h_ready, 256);
    mbar_init(&s.h_free, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = *reinterpret_cast<volatile int*>(a.err) != 0;
    s.never = 0;
    s.unit_bad = 0;
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
    // ------------------------------------------------ scan + TMA producer warp
    const float a2 = a.A[h] * kLog2e;
    float p0 = 0.f, p1 = 0.f;  // dt of tokens 2*lane, 2*lane+1 of the next chunk to scan
    auto load_dt = [&](int c) {
      const int64_t t = (int64_t)c * 64 + 2 * lane;
      p0 = (c < nc && t < len) ? a.dt[(rowbase + t) * a.H + h] : 0.f;
      p1 = (c < nc && t + 1 < len) ? a.dt[(rowbase + t + 1) * a.H + h] : 0.f;
    };
    load_dt(0);
    int scanned = 0;
    // in-chunk cumulative sum (log2 units), factor vectors and chunk scalars
    auto scan_next = [&]() -> bool {
      const int c = scanned;
      const int slot = c & 3;
      if (c >= 4 && !mbar_wait_warp(&s.scan_empty[slot], ((c - 4) >> 2) & 1, abort_flag, kWaitLimitNs)) return false;
      const float d0 = p0, d1 = p1;
      const float x0 = d0 * a2, x1 = d1 * a2;
      float v = x0 + x1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      const float cs1 = v, cs0 = v - x1;
      const float m = __shfl_sync(0xffffffffu, cs1, 15);  // token 31
      const int nvalid = (c + 1) * 64 <= len ? 64 : len - c * 64;
      const int e = nvalid - 1;
      const float cse = __shfl_sync(0xffffffffu, (e & 1) ? cs1 : cs0, e >> 1);
      float dev = fmaxf(fabsf(cs0 - m), fabsf(cs1 - m));
      // D x_t is carried through u_t v_t = dt_t, which needs dt_t != 0
      if ((2 * lane < nvalid && d0 == 0.f) || (2 * lane + 1 < nvalid && d1 == 0.f)) dev = INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
      if (!(dev <= kRangeLog2) && lane == 0) s.unit_bad = 1;
      s.u[slot][2 * lane] = exp2f(cs0 - m);
      s.u[slot][2 * lane + 1] = exp2f(cs1 - m);
      s.v[slot][2 * lane] = exp2f(m - cs0) * d0;
      s.v[slot][2 * lane + 1] = exp2f(m - cs1) * d1;
      s.dt[slot][2 * lane] = d0;
      s.dt[slot][2 * lane + 1] = d1;
      if (lane == 0) {
        s.sc[slot][0] = exp2f(m);
        s.sc[slot][1] = exp2f(cse - m);
        s.sc[slot][2] = exp2f(cse);
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
      const int sl = c % 3;
      mbar_arrive_expect_tx(&s.full_x[sl], K::kTile);
      tma_load_3d(sm + K::oX + sl * K::kTile, &tm_x, &s.full_x[sl], (int)(h * 64), t_base + c * 64, (int)b);
      last_x = c;
    };
    auto issue_w = [&](int c) {
      mbar_arrive_expect_tx(&s.full_w[c & 1], K::kTile);
      tma_load_3d(sm + K::oW + (c & 1) * K::kTile, &tm_w, &s.full_w[c & 1], 0,
                  (int)(((cbase + c) * a.G + g) * 64), 0);
      last_w = c;
    };
    auto issue_b = [&](int c) {
      mbar_arrive_expect_tx(&s.full_b, K::NB * K::kTile);
      for (int j = 0; j < K::NB; ++j)
        tma_load_4d(sm + K::oB + j * K::kTile, &tm_b, &s.full_b, 64 * j, (int)g, t_base + c * 64, (int)b);
      last_b = c;
    };
    auto issue_c = [&](int c) {
      uint64_t* bar = &s.full_c[c & 1];
      mbar_arrive_expect_tx(bar, K::NB * K::kTile);
      for (int j = 0; j < K::NB; ++j)
        tma_load_4d(sm + K::oC + ((c & 1) * K::NB + j) * K::kTile, &tm_c, bar, 64 * j, (int)g, t_base + c * 64,
                    (int)b);
      last_c = c;
    };
    bool ok = true;
    for (int k = 0; k < 2 && k < nc && ok; ++k) ok = scan_next();
    if (lane == 0 && ok) {
      for (int c = 0; c < 3 && c < nc; ++c) issue_x(c);
      griddep_wait();  // W' comes from the C B^T kernel launched before this one
      for (int c = 0; c < 2 && c < nc; ++c) {
        issue_w(c);
        issue_c(c);
      }
      issue_b(0);
    }
    // each resource of chunk c is refilled for a later chunk as soon as its
    // last reader is done: W' after W' X', B and x (scaled in place) after
    // B^T X', C after C H^T
    for (int c = 0; c < nc && ok; ++c) {
      if (scanned < nc) ok = scan_next();  // chunk c + 2
      if (lane == 0 && ok) {
        if (c + 2 < nc) {
          ok = mbar_wait(&s.w_empty[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_w(c + 2);
        }
        if (ok && c + 1 < nc) {
          ok = mbar_wait(&s.b_free, c & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_b(c + 1);
        }
        if (ok && c + 3 < nc) {
          ok = mbar_wait(&s.x_empty[c % 3], (c / 3) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_x(c + 3);
        }
        if (ok && c + 2 < nc) {
          ok = mbar_wait(&s.c_free[c & 1], (c >> 1) & 1, abort_flag, kWaitLimitNs);
          if (ok) issue_c(c + 2);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
    }
    if (lane == 0 && *abort_flag) {  // let this CTA's own copies land before its smem is released
      if (last_x >= 0) mbar_wait(&s.full_x[last_x % 3], (last_x / 3) & 1, never, kWaitLimitNs);
      if (last_w >= 0) mbar_wait(&s.full_w[last_w & 1], (last_w >> 1) & 1, never, kWaitLimitNs);
      if (last_b >= 0) mbar_wait(&s.full_b, last_b & 1, never, kWaitLimitNs);
      if (last_c >= 0) mbar_wait(&s.full_c[last_c & 1], (last_c >> 1) & 1, never, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop and forms the descriptors (warp-uniform
    // values); one elected lane issues the MMAs and commits.
    const uint32_t aW = smem_u32(sm + K::oW), aC = smem_u32(sm + K::oC), aB = smem_u32(sm + K::oB);
    const uint32_t aX = smem_u32(sm + K::oX), aH = smem_u32(sm + K::oH);
    constexpr uint32_t id_64 = idesc_bf16(64, 64, 0, 1);    // A K-major, B MN-major, M = 64
    constexpr uint32_t id_st = idesc_bf16(128, 64, 1, 1);   // both MN-major, M = 128
    const uint64_t db = sw128_desc(aB, K::kTile, 1024);     // a K step of 16 tokens: 2048 B
    const uint64_t dh = sw128_desc(aH, K::kTile, 1024);
    for (int c = 0; c < nc; ++c) {
      const int i = c & 1;
      const uint32_t ph = (c >> 1) & 1, p1 = c & 1, pp = ((c - 2) >> 1) & 1;
      bool ok = mbar_wait_warp(&s.full_w[i], ph, abort_flag, kWaitLimitNs);
      ok = ok && mbar_wait_warp(&s.xp_ready[c % 3], (c / 3) & 1, abort_flag, kWaitLimitNs);
      if (c >= 2) {
        ok = ok && mbar_wait_warp(&s.y_free[i], pp, abort_flag, kWaitLimitNs);
        ok = ok && mbar_wait_warp(&s.s_free[i], pp, abort_flag, kWaitLimitNs);
      }
      if (!ok) break;
      tc_fence_after();
      const uint32_t yd = tmem + K::tYd0 + 64 * i;
      const uint32_t st = tmem + K::tS0 + K::kSCols * i;
      const uint64_t dx = sw128_desc(aX + (c % 3) * K::kTile, K::kTile, 1024);  // X' of this chunk
      const uint64_t dw = sw128_desc(aW + i * K::kTile, 16, 1024);             // a K step: 32 B
      // Yd = W' X'   (K = 64 tokens)
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(yd, dw + 2 * kk, dx + 128 * kk, id_64, kk > 0);
        mma_commit(&s.w_empty[i]);
      }
      __syncwarp();
      // S'^T = B^T X'   (M = 128 state rows per half, K = 64 tokens)
      if (!mbar_wait_warp(&s.full_b, p1, abort_flag, kWaitLimitNs)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int hf = 0; hf < K::NH; ++hf)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(st + 64 * hf, db + (hf * 2 * K::kTile) / 16 + 128 * kk, dx + 128 * kk, id_st, kk > 0);
        mma_commit(&s.s_full[i]);
        mma_commit(&s.b_free);
        mma_commit(&s.x_empty[c % 3]);
      }
      __syncwarp();
      // Yd += C (e^m H_c)^T   (K = N)
      ok = mbar_wait_warp(&s.h_ready, p1, abort_flag, kWaitLimitNs);
      ok = ok && mbar_wait_warp(&s.full_c[i], ph, abort_flag, kWaitLimitNs);
      if (!ok) break;
      tc_fence_after();
      const uint64_t dc = sw128_desc(aC + i * K::NB * K::kTile, 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk)
          mma_bf16_ss(yd, dc + ((kk >> 2) * K::kTile + (kk & 3) * 32) / 16, dh + 128 * kk, id_64, 1);
        mma_commit(&s.y_full[i]);
        mma_commit(&s.h_free);
        mma_commit(&s.c_free[i]);
      }
      __syncwarp();
    }
    if (elect_one()) {
      mma_commit(&s.drain);
      mbar_wait(&s.drain, 0, never, kWaitLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const int wt = tid - 64;            // 0..255
    const int q = warp & 3;             // TMEM lane quadrant
    const int hq = (warp - 2) >> 2;     // which half of the 64 columns
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    const float dskip = a.D ? a.D[h] : 0.f;
    const int n0 = 32 * q + lane;       // state row(s): n0 (+128)
    const int pc0 = 32 * hq;            // state columns [pc0, pc0 + 32)
    float H[K::NH][32];
#pragma unroll
    for (int hf = 0; hf < K::NH; ++hf)
#pragma unroll
      for (int j = 0; j < 32; ++j)
        H[hf][j] = a.h0 && first && n0 + 128 * hf < a.Nr
                       ? a.h0[((b * a.H + h) * 64 + pc0 + j) * a.Nr + n0 + 128 * hf]
                       : 0.f;
    bool failed = false;

    for (int c = 0; c <= nc; ++c) {
      if (named_barrier_any(2, 256, failed)) {
        failed = true;
        break;
      }
      if (c < nc) {
        // ---- X' = diag(v) x for chunk c (in place), and D folded into W's diagonal
        const int sl = c & 3, ix = c % 3, iw = c & 1;
        if (!mbar_wait_warp(&s.scan_full[sl], (c >> 2) & 1, abort_flag, kWaitLimitNs) ||
            !mbar_wait_warp(&s.full_x[ix], (c / 3) & 1, abort_flag, kWaitLimitNs) ||
            !mbar_wait_warp(&s.full_w[iw], (c >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          continue;
        }
        const int srow = wt >> 2, j4 = wt & 3;
        const __nv_bfloat162 w2 = __float2bfloat162_rn(s.v[sl][srow]);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          uint4* px = reinterpret_cast<uint4*>(sm + K::oX + ix * K::kTile +
                                               sw128((uint32_t)srow * 128 + (2 * j4 + jj) * 16));
          uint4 vv = *px;
          __nv_bfloat162* e2 = reinterpret_cast<__nv_bfloat162*>(&vv);
#pragma unroll
          for (int k = 0; k < 4; ++k) e2[k] = __hmul2(e2[k], w2);
          *px = vv;
        }
        if (wt < 64) {
          // W'[t][t] += D / dt_t, so that u_t (W' X')_t includes D x_t (u_t v_t = dt_t)
          const float dtt = s.dt[sl][wt];
          if (dtt != 0.f && dskip != 0.f) {
            __nv_bfloat16* dg = reinterpret_cast<__nv_bfloat16*>(
                sm + K::oW + iw * K::kTile + sw128((uint32_t)wt * 128 + (wt >> 3) * 16) + (wt & 7) * 2);
            *dg = __float2bfloat16_rn(__bfloat162float(*dg) + dskip / dtt);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&s.xp_ready[ix]);
      }
      // ---- state update for chunk c-1
      if (c >= 1) {
        const int ip = (c - 1) & 1, slp = (c - 1) & 3;
        if (!mbar_wait_warp(&s.s_full[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          continue;
        }
        tc_fence_after();
        const float dd = s.sc[slp][2], ff = s.sc[slp][1];
#pragma unroll
        for (int hf = 0; hf < K::NH; ++hf) {
          uint32_t r[32];
          SSD_TMEM_LD_32x32b_X32(tq + K::tS0 + K::kSCols * ip + 64 * hf + pc0, r);
          SSD_TMEM_WAIT_LD_32(r);
#pragma unroll
          for (int j = 0; j < 32; ++j) H[hf][j] = fmaf(dd, H[hf][j], ff * __uint_as_float(r[j]));
        }
        tc_fence_before();
        mbar_arrive(&s.s_free[ip]);
      }
      // ---- publish e^m H_c (bf16) for chunk c's C H^T product
      if (c < nc) {
        if (c >= 1 && !mbar_wait_warp(&s.h_free, (c - 1) & 1, abort_flag, kWaitLimitNs)) {
          failed = true;
          continue;
        }
        const float E = s.sc[c & 3][0];
#pragma unroll
        for (int hf = 0; hf < K::NH; ++hf) {
          const uint32_t row = (uint32_t)(n0 + 128 * hf);
          unsigned char* base = sm + K::oH + row * 128;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint4 vv;
            vv.x = pack_bf16x2(E * H[hf][8 * jj + 0], E * H[hf][8 * jj + 1]);
            vv.y = pack_bf16x2(E * H[hf][8 * jj + 2], E * H[hf][8 * jj + 3]);
            vv.z = pack_bf16x2(E * H[hf][8 * jj + 4], E * H[hf][8 * jj + 5]);
            vv.w = pack_bf16x2(E * H[hf][8 * jj + 6], E * H[hf][8 * jj + 7]);
            const uint32_t chunk = (uint32_t)(pc0 / 8 + jj);
            *reinterpret_cast<uint4*>(base + ((chunk ^ (row & 7)) << 4)) = vv;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&s.h_ready);
      }
      // ---- epilogue for chunk c-1: y = u_t Yd + D x
      if (c >= 1) {
        const int ip = (c - 1) & 1, slp = (c - 1) & 3;
        const int64_t t0p = (int64_t)(c - 1) * 64;
        const int nvp = c * 64 <= len ? 64 : (int)(len - t0p);
        if (!mbar_wait_warp(&s.y_full[ip], ((c - 1) >> 1) & 1, abort_flag, kWaitLimitNs)) {
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
          const float ut = s.u[slp][t];
          const int64_t yoff = ((rowbase + t0p + t) * a.H + h) * 64 + p0;
          float gz[16];  // the gate: SiLU(z), or 1
          if (a.z) {
            const uint4* zp = reinterpret_cast<const uint4*>(a.z + yoff);
            const uint4 z0 = zp[0], z1 = zp[1];
            const uint32_t zw[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              unpack_bf16x2(zw[j], gz[2 * j], gz[2 * j + 1]);
              gz[2 * j] = silu(gz[2 * j]);
              gz[2 * j + 1] = silu(gz[2 * j + 1]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) gz[j] = 1.f;
          }
          uint32_t packed[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            packed[j] = pack_bf16x2(ut * __uint_as_float(r[2 * j]) * gz[2 * j],
                                    ut * __uint_as_float(r[2 * j + 1]) * gz[2 * j + 1]);
          uint4* dst = reinterpret_cast<uint4*>(a.y + yoff);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        mbar_arrive(&s.scan_empty[slp]);
      }
    }
    if (!failed && a.final_states) {
#pragma unroll
      for (int hf = 0; hf < K::NH; ++hf) {
        if (n0 + 128 * hf >= a.Nr) continue;
        float* dst = a.final_states + ((out_row * a.H + h) * 64 + pc0) * a.Nr + n0 + 128 * hf;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(int64_t)j * a.Nr] = H[hf][j];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    if (*abort_flag) atomicExch(a.err, 1);
    // a chunk's decay range was too wide to factorise: the exact kernel redoes
    // this unit (for packed sequences, the run's whole (row, head), once)
    if (s.unit_bad) {
      const int64_t rowunit = b * a.H + h;
      if (!a.varlen) a.failed_list[atomicAdd(a.failed_count, 1)] = (int)unit;
      else if (atomicExch(&a.unit_bad[rowunit], 1) == 0) a.failed_list[atomicAdd(a.failed_count, 1)] = (int)rowunit;
    }
  }
  if (warp == 0) tmem_dealloc(tmem, K::kTmemCols);
}

// The gate for the two-head kernel, whose epilogue leaves it out: y <- y *
// SiLU(z) in place, 8 bf16 a thread per 16-byte vector (n8 vectors), SiLU as
// the single-head epilogue forms it.  y is rounded to bf16 before the gate
// here, once more after it.
__global__ void __launch_bounds__(256) k_gate_silu(__nv_bfloat16* y, const __nv_bfloat16* z, int64_t n8) {
  uint4* yv = reinterpret_cast<uint4*>(y);
  const uint4* zv = reinterpret_cast<const uint4*>(z);
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += (int64_t)gridDim.x * 256) {
    const uint4 a = yv[i], g = __ldcs(zv + i);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float y0, y1, z0, z1;
      unpack_bf16x2(aw[j], y0, y1);
      unpack_bf16x2(gw[j], z0, z1);
      o[j] = pack_bf16x2(y0 * silu(z0), y1 * silu(z1));
    }
    __stcs(yv + i, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// ev0 / ev1 (optional) are recorded right before and after the fused kernel.
// Packed sequences (seq_idx): the run list first, then W' per run chunk and
// the single-head kernel per (run, head).  A gated call on the two-head
// kernel adds k_gate_silu after it (the exact kernel, which may follow,
// applies the gate itself to the units it redoes).
template <int NS>
cudaError_t launch_fast(const Problem& p, const TcWorkspace& w, cudaStream_t st, cudaEvent_t ev0, cudaEvent_t ev1) {
  const bool varlen = p.seq != nullptr;
  const int64_t chunks = p.b * p.nc + (varlen ? p.num_seqs : 0);  // W' tiles per group, at most
  CUtensorMap tx, tb, tc_, tw;
  if (!make_map_3d(&tx, p.x, p.H * p.P, p.L, p.b) || !make_map_bc(&tb, p.B, p.N, p.G, p.L, p.b) ||
      !make_map_bc(&tc_, p.C, p.N, p.G, p.L, p.b) || !make_map_3d(&tw, w.wp, 64, chunks * p.G * 64, 1))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (varlen) {
    SeqRunArgs sa;
    sa.seq = p.seq;
    sa.b = p.b;
    sa.L = p.L;
    sa.H = p.H;
    sa.num_seqs = p.num_seqs;
    sa.runs = w.runs;
    sa.failed_count = w.failed_count;
    sa.failed_list = w.failed_list;
    k_seq_runs<<<1, 1024, 0, st>>>(sa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.final_states) {
      const int64_t items = p.num_seqs * kZeroSlices;
      k_zero_absent<<<(unsigned)(items < 148 * 8 ? items : 148 * 8), 256, 0, st>>>(
          w.runs, p.final_states, p.num_seqs, p.H * p.P * p.N);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  CbArgs ca{};
  ca.L = p.L;
  ca.G = p.G;
  ca.nc = p.nc;
  ca.seq = nullptr;  // a run never crosses a sequence boundary
  ca.wp = w.wp;
  ca.err = w.err;
  ca.varlen = varlen;
  ca.runs = w.runs;
  e = cudaFuncSetAttribute(k_chunk_cb<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CbCfg<NS>::kSmemBytes);
  if (e != cudaSuccess) return e;
  k_chunk_cb<NS><<<(unsigned)(chunks * p.G), 128, CbCfg<NS>::kSmemBytes, st>>>(tb, tc_, ca);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  FastArgs fa{};
  fa.L = p.L;
  fa.H = p.H;
  fa.G = p.G;
  fa.hpg = p.hpg;
  fa.nc = p.nc;
  fa.dt = p.dt;
  fa.A = p.A;
  fa.D = p.D;
  fa.h0 = p.h0;
  fa.Nr = p.N;
  fa.y = static_cast<__nv_bfloat16*>(p.y);
  fa.final_states = p.final_states;
  fa.failed_count = w.failed_count;
  fa.failed_list = w.failed_list;
  fa.err = w.err;
  fa.batch = p.b;
  fa.handoff = w.handoff;
  fa.flags = w.flags;
  fa.pair_bad = w.pair_bad;
  fa.varlen = varlen;
  fa.z = static_cast<const __nv_bfloat16*>(p.z);
  fa.runs = w.runs;
  fa.unit_bad = w.unit_bad;
  fa.stall = p.stall ? 1 : 0;
  if (!varlen && NS == 128 && tc_pair_supported(p)) {
    CUtensorMap ty, tdt;
    if (!make_map_3d(&ty, p.y, p.H * p.P, p.L, p.b) || !make_map_dt(&tdt, p.dt, p.H, p.L, p.b))
      return cudaErrorInvalidValue;
    if (ev0 && (e = cudaEventRecord(ev0, st)) != cudaSuccess) return e;
    if ((e = tc_pair_launch(p, w, tx, tb, tc_, tw, ty, tdt, fa, st)) != cudaSuccess) return e;
    if (ev1 && (e = cudaEventRecord(ev1, st)) != cudaSuccess) return e;
    if (p.z) {
      const int64_t n8 = p.b * p.L * p.H * p.P / 8;  // P = 64
      const int64_t blocks = (n8 + 255) / 256;
      k_gate_silu<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, st>>>(
          static_cast<__nv_bfloat16*>(p.y), static_cast<const __nv_bfloat16*>(p.z), n8);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(k_ssd_fwd_fast<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)FastCfg<NS>::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (ev0 && (e = cudaEventRecord(ev0, st)) != cudaSuccess) return e;
  const int64_t units = (varlen ? p.num_seqs : p.b) * p.H;  // (run, head): at most num_seqs runs
  e = launch_dependent(k_ssd_fwd_fast<NS>, (unsigned)units, FastCfg<NS>::kThreads, FastCfg<NS>::kSmemBytes, st, tx,
                       tb, tc_, tw, fa);
  if (e != cudaSuccess) return e;
  return ev1 ? cudaEventRecord(ev1, st) : cudaSuccess;
}

}  // namespace

const char* tc_main_kernel(const Problem& p) {
  if (p.seq) return "k_ssd_fwd_fast";  // per (run, head)
  return tc_kernel_n(p) == 128 && tc_pair_supported(tc_tiles(p)) ? "k_ssd_fwd_pair" : "k_ssd_fwd_fast";
}

cudaError_t tc_fast_forward(const Problem& p, const TcWorkspace& w, cudaStream_t st, cudaEvent_t ev0,
                            cudaEvent_t ev1) {
  return tc_kernel_n(p) == 128 ? launch_fast<128>(p, w, st, ev0, ev1) : launch_fast<256>(p, w, st, ev0, ev1);
}

}  // namespace ssd
