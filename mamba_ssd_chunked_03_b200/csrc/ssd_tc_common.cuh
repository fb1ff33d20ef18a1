// Pieces shared by the tensor-core SSD kernels (ssd_tc.cu, ssd_tc_fast.cu,
// ssd_tc_pair.cu):
// constants, kernel argument blocks, the workspace carve-up and TMA tensor
// map creation.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd_internal.h"

namespace ssd {
namespace tc {

constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per bounded wait
// Largest |cs_t - r| (log2 units) for the point r the decay factorisation is
// taken about (the chunk's middle token in ssd_tc_fast.cu, its first in
// ssd_tc_pair.cu): 2^100 stays far inside fp32/bf16.
constexpr float kRangeLog2 = 100.f;

// Packed sequences run one sequence at a time ("runs"): every maximal run of
// equal seq_idx in a batch row is chunked from its own first token, so no chunk
// straddles a boundary and the runs are independent problems.  k_seq_runs
// fills this list in the workspace.
struct RunList {
  int* count;  // runs, or 0 when the ids are not strictly increasing runs in
               // [0, num_seqs) (every unit then goes to the exact kernel)
  int* b;      // [num_seqs] batch row of run r
  int* t0;     // [num_seqs] its first token in the row
  int* len;    // [num_seqs] its tokens
  int* id;     // [num_seqs] its sequence id
  int* c0;     // [num_seqs + 1] its first chunk in the flattened chunk list
  int* order;  // [num_seqs] the runs longest first (by chunks; ties in run order), which
               // the single-head kernel takes in that order so that the long runs do not
               // trail at the end of the grid; run order past kRunSortMax runs
};
constexpr int kRunSortMax = 1024;  // runs k_seq_runs ranks (one per thread)

struct CbArgs {
  int64_t L, G, nc;
  const int32_t* seq;
  __nv_bfloat16* wp;  // (chunks, G, 64, 64) masked C B^T; chunks = b * nc, or the runs' chunks
  int* err;
  int varlen;         // chunks are the runs' chunks (RunList)
  RunList runs;
};

struct FastArgs {
  int64_t L, H, G, hpg, nc, batch;
  int64_t Nr;  // the problem's d_state (<= the kernel's N; rows past it are zero padding)
  const float* dt;
  const float* A;
  const float* D;
  const float* h0;
  __nv_bfloat16* y;
  float* final_states;
  int* failed_count;  // units whose decay range could not be factorised ...
  int* failed_list;   // ... listed here for the exact kernel
  int* err;
  // two-head kernel only: state hand-over between the CTAs that share a pair
  float* handoff;  // [grid][2 heads][128 states][64 p] fp32
  int* flags;      // [grid][kPairFlagsPerCta state warps]: 1 once that warp's part of the hand-over is written
  int* pair_bad;   // [b * H / 2]: 1 once a pair was put on the exact kernel's list
  // split mode (a state-only pass first): the CTA's local end state goes to
  // handoff, its total decay per head to seg_decay [grid][2]
  int split;
  float* seg_decay;
  // single-head kernel, packed sequences: one CTA per (run, head); a unit
  // the factorised form cannot take marks its (row, head) once in unit_bad
  int varlen;
  RunList runs;
  int* unit_bad;
  const __nv_bfloat16* z;  // gate (b, L, H, 64): y * SiLU(z), or null
  int stall;               // two-head kernel: hand-overs wait on the never-set flag (failure-path tests)
};

// persistent grid of the two-head kernel, at most; per-CTA hand-over size
constexpr int kPairGridMax = 256;
constexpr int kPairHandoffFloats = 2 * 128 * 64;
constexpr int kPairFlagsPerCta = 16;  // one per state warp
// the flag after the last CTA's: cleared every call and never set (SSD_FLAG_TEST_STALL)
constexpr int kPairNeverFlag = kPairGridMax * kPairFlagsPerCta;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// the block's gate nonlinearity, SiLU(v) = v / (1 + e^-v)
__device__ __forceinline__ float silu(float v) { return v / (1.f + expf(-v)); }

__device__ __forceinline__ void unpack_bf16x2(uint32_t u, float& lo, float& hi) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  lo = __low2float(v);
  hi = __high2float(v);
}

// 3-D bf16 tensor map over (outer, rows, inner) with a 64 x 64 x 1 box and
// 128-byte swizzle; rows past `rows` read as zeros.
bool make_map_3d(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t outer);
// bf16 tensor map over B or C (b, L, G, N) as 4-D (n, group, token, row) with
// a 64 x 1 x 64 x 1 box and 128-byte swizzle: a box at n = 64 of an N = 64
// tensor lies outside it and reads as zeros, which is how the kernels built
// for N = 128 run N = 64 (the state is zero-padded to 128 rows).
bool make_map_bc(CUtensorMap* m, const void* base, int64_t N, int64_t G, int64_t L, int64_t b);
// fp32 tensor map over dt (b, L, H) with a 4-head x 64-token box, no swizzle;
// needs H * 4 bytes to be a multiple of 16.  Tokens past L read as zeros.
bool make_map_dt(CUtensorMap* m, const float* dt, int64_t H, int64_t L, int64_t b);
// fp32 tensor map over (b, L, H, inner) as 4-D (element, head, token, row) with
// a 32 x 1 x 64 x 1 box (128-byte rows) and 128-byte swizzle, for bulk stores
// of per-chunk gradient tiles; tokens past L are clipped.
bool make_map_f32_tiles(CUtensorMap* m, float* base, int64_t inner, int64_t H, int64_t L, int64_t b);
// fp32 tensor map over units of a rows x inner block each (units, rows, inner
// contiguous) with a 32 x rows x 1 box and 128-byte swizzle: one unit's
// 32-column slice per bulk store.
bool make_map_f32_blocks(CUtensorMap* m, float* base, int64_t inner, int64_t rows, int64_t units);

}  // namespace tc

// Launch `kernel` so that it may start while the previous kernel on the
// stream is still running (programmatic dependent launch): the kernel calls
// griddep_wait() before it reads what that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// The tensor-core kernels work on 64-token chunks.  A chunk of Q = 128 or 256
// tokens is computed as Q/64 consecutive 64-token chunks: the chunked
// decomposition is an exact re-association of the recurrence, so refining
// the chunks changes only the rounding, not the result.  Every tensor-core
// entry point (ssd_tc.cu, ssd_tc_fast.cu) turns the problem into its
// 64-token form first.
// d_state the kernels are built for: 64 runs zero-padded as 128
inline int tc_kernel_n(const Problem& p) { return p.N == 256 ? 256 : 128; }

inline Problem tc_tiles(const Problem& p) {
  Problem t = p;
  t.Q = 64;
  t.nc = (p.L + 63) / 64;
  return t;
}

// Workspace of the tensor-core path, carved from the caller's buffer.
struct TcWorkspace {
  int* err;               // nonzero after a kernel gave up on a bounded wait
  int* failed_count;      // next to err; err .. zero_bytes is cleared by one memset per call
  int* flags;             // two-head kernel: hand-over flags (kPairGridMax x kPairFlagsPerCta), or null
  int* pair_bad;          // two-head kernel: per-pair exact-kernel marks, or null
  size_t zero_bytes;
  __nv_bfloat16* wp;      // masked C B^T per (b, chunk, group)
  int* failed_list;       // (b*H) units for the exact kernel
  float* handoff;         // two-head kernel: kPairGridMax x kPairHandoffFloats, or null
  float* seg_decay;       // two-head kernel: kPairGridMax x 2 total decays (split mode), or null
  tc::RunList runs;       // packed sequences: the run list, else null pointers
  int* unit_bad;          // packed sequences: [b * H] exact-kernel marks (cleared per call), or null
};

// carve the caller's workspace (ws may be null to only size it: *total)
TcWorkspace tc_carve(const Problem& p, void* ws, size_t* total = nullptr);
size_t tc_workspace_need(const Problem& p);
// chunk C B^T kernel, then the fused kernel, bracketed by ev0 / ev1 if given
cudaError_t tc_fast_forward(const Problem& p, const TcWorkspace& w, cudaStream_t st, cudaEvent_t ev0 = nullptr,
                            cudaEvent_t ev1 = nullptr);

// two heads per CTA (ssd_tc_pair.cu): N = 128, an even number of heads per
// group and H a multiple of 4 (shape only) ...
bool tc_pair_shape_ok(const Problem& p);
// ... and a 16-byte aligned dt
bool tc_pair_supported(const Problem& p);
// whether the two-head kernel runs split: a state-only pass over every CTA's
// range first, so that no CTA waits for another (fewer pairs than SMs)
bool tc_pair_split(const Problem& p);
cudaError_t tc_pair_launch(const Problem& p, const TcWorkspace& w, const CUtensorMap& tx, const CUtensorMap& tb,
                           const CUtensorMap& tc_, const CUtensorMap& tw, const CUtensorMap& ty,
                           const CUtensorMap& tdt, const tc::FastArgs& fa, cudaStream_t st);

}  // namespace ssd
