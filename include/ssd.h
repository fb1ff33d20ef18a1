/*
 * ssd.h -- C ABI of libssd, the chunked SSD (structured state space duality)
 * forward for NVIDIA B200 (sm_100a), with its backward (ssd_bwd), the
 * recurrent decode step, the state operations of sequence parallelism and
 * the Mamba-2 block's conv1d + SiLU.
 *
 * What one call computes, per batch row b and head h, with group
 * g = h / (nheads / ngroups) (contiguous heads share B and C):
 *
 *   h_t = a_t h_{t-1} + dt_t x_t B_t^T        state, headdim x dstate
 *   y_t = h_t C_t + D_h x_t                    output, headdim
 *   a_t = exp(dt_t A_h), or 0 at the first token of a new packed sequence
 *
 * with h_{-1} = initial_states[b,h] (or 0).  Sources, by page title:
 *  - "22 · Mamba 2 — Transformers are SSMs" (paper story), section 3.1 (the
 *    scalar-A recurrence), section 3.2 (the dual form Y = (L o C B^T)(dt x)),
 *    section 4.1 (block decomposition into intra- and inter-chunk parts).
 *  - "SSM 家族全景图（下）：Mamba-2 与 Jamba", section 三.4 (the four chunked
 *    steps) and the closing question (a_t = exp(Delta_t A)).
 *  - "从Transformer的二次复杂度困境到Mamba的线性突围", continuous SSM
 *    equations (the D feed-through).
 *  - "Transformers与SSMs的隐藏联系", section 4.2 (packed sequences: the
 *    transition is set to zero at each boundary).
 *
 * The result is computed with the chunked algorithm: an in-chunk cumulative
 * sum of dt*A, the masked decay-weighted C B^T "attention" inside each chunk,
 * per-chunk states, a scan of states across chunks, and an output correction
 * from each chunk's carried state.  Chunking re-associates the same sums, so
 * the result equals the recurrence up to rounding for every chunk size.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them, and keeps no global state, so
 *    calls are re-entrant and may run concurrently on different streams with
 *    different workspaces.
 *  - Tensors are dense and contiguous, row-major in the order given.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL means
 *    the legacy default stream) and the call returns without synchronising.
 *  - Arguments are validated on the host before anything is enqueued; a
 *    rejected call enqueues nothing.  Nothing on the device traps or asserts.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1,  /* null required pointer, bad size, bad alignment, bad enum */
  SSD_ERR_UNSUPPORTED = 2,  /* valid arguments outside the implemented shape set */
  SSD_ERR_WORKSPACE = 3,    /* workspace missing or smaller than ssd_fwd_workspace_size() */
  SSD_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed (see cudaGetLastError) */
  SSD_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up (ssd_fwd_device_status) */
} ssd_status;

/* Element type of x, B, C and y.  dt, A, D, initial_states and final_states
 * are always fp32. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/* flags */
#define SSD_FLAG_GENERIC 1u /* use the generic (CUDA-core, fp32) kernels even where
                               the tensor-core kernels apply; for cross-checks */
#define SSD_FLAG_CHECK_SEQ 2u /* check the seq_idx precondition first: ssd_fwd copies
                                 seq_idx to the host (waiting for `stream`) and
                                 returns ssd_check_seq_idx's verdict if it fails */
#define SSD_FLAG_TEST_STALL 4u /* for tests of the failure path only: the two-head
                                  kernel's state hand-over between CTAs waits on a
                                  flag that nothing sets, so that bounded wait runs
                                  out (after 1 s) and ssd_fwd_device_status reports
                                  SSD_ERR_TIMEOUT; y is then incomplete.  Shapes
                                  without a hand-over are not affected. */

typedef struct {
  /* sizes: b = batch, L = seqlen, H = nheads, P = headdim, N = dstate,
   * G = ngroups (H % G == 0), Q = chunk_size (a power of two, 16..256).
   * L need not be a multiple of Q (the last chunk is short). */
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk_size;
  ssd_dtype dtype;
  uint32_t flags;                 /* SSD_FLAG_* or 0 */

  const void* x;                  /* (b,L,H,P) dtype                                  */
  const float* dt;                /* (b,L,H) fp32, the step size used as given (> 0)  */
  const float* A;                 /* (H) fp32, continuous decay rate (expected < 0)   */
  const void* B;                  /* (b,L,G,N) dtype, input projection ("keys")       */
  const void* C;                  /* (b,L,G,N) dtype, output projection ("queries")   */
  const float* D;                 /* (H) fp32 skip weight, or NULL for D = 0          */
  const float* initial_states;    /* (b,H,P,N) fp32 state before token 0, or NULL = 0.
                                     With seq_idx it applies to each row's first
                                     sequence only.                                  */
  const int32_t* seq_idx;         /* (b,L) int32 packed-sequence ids, or NULL.
                                     Precondition: non-decreasing along each row, ids
                                     in [0, num_seqs), a sequence never spans rows.
                                     A change of id starts a new sequence (a_t = 0).
                                     Ids increasing from row to row (each id one
                                     run) run per sequence on the fast kernels;
                                     other orders on a slower per-(row, head) one. */
  int64_t num_seqs;               /* number of sequence ids; required (> 0) iff seq_idx */

  void* y;                        /* (b,L,H,P) dtype, output                          */
  float* final_states;            /* output or NULL: (b,H,P,N) fp32 state after the
                                     last token; with seq_idx (num_seqs,H,P,N), the
                                     state after each sequence's last token (ids that
                                     do not occur get zeros)                         */

  void* workspace;                /* device scratch of at least
                                     ssd_fwd_workspace_size(args) bytes, 256-byte
                                     aligned; may be NULL when that size is 0.  Its
                                     contents on entry do not matter.                */
  size_t workspace_bytes;

  void* timing_events[2];         /* optional pair of cudaEvent_t (as void*), or NULLs:
                                     recorded on `stream` right before and right after
                                     the main kernel of the call (the fused tensor-core
                                     kernel, or all generic kernels together), so a
                                     caller can time it without a profiler.  Owned by
                                     the caller; both or neither.                    */
  const void* z;                  /* (b,L,H,P) dtype gate, or NULL: y is returned as
                                     y * SiLU(z) (SiLU(v) = v / (1 + e^-v)), the
                                     Mamba-2 block's gate path ("SSM 家族全景图（下）：
                                     Mamba-2 与 Jamba", section 5), multiplied in
                                     where y is formed; on the two-head kernel by a
                                     pass over y right after it (y then rounded to
                                     the output type twice).                        */
} ssd_fwd_args;

/* Bytes of device workspace ssd_fwd needs for these sizes and options (only
 * the size fields, dtype, flags and the presence of seq_idx/final_states are
 * read; pointers may be NULL).  Returns 0 if the sizes are invalid. */
SSD_API size_t ssd_fwd_workspace_size(const ssd_fwd_args* args);

/* Enqueue the SSD forward on `stream`.  Returns SSD_OK once the work is
 * enqueued, or an error code; on error nothing was enqueued except for
 * SSD_ERR_CUDA from a later launch, in which case outputs are undefined. */
SSD_API ssd_status ssd_fwd(const ssd_fwd_args* args, void* stream);

/* ssd_fwd for callers that cannot allocate device memory when they call:
 * identical arguments and results, but the workspace fields are ignored and
 * no memory is allocated or freed.  Meant for code where no device allocator
 * is reachable or allowed once work has started, such as a plugin inside a
 * host runtime that owns all device memory, or a latency-critical loop that
 * must not call cudaMalloc.  The pages describe no such entry point; it has
 * no counterpart there.
 *
 * Scratch comes from one fixed 32 MiB device array inside the library.  Every
 * GPU that loads this part of the library keeps that array until the process
 * exits.  The call takes the kernel path ssd_fwd would take (the tensor-core
 * kernels where they apply, unless SSD_FLAG_GENERIC is set) when that path's
 * workspace fits the array, else the generic CUDA-core kernels; problems
 * whose generic workspace (ssd_fwd_workspace_size with SSD_FLAG_GENERIC) also
 * exceeds 32 MiB are rejected with SSD_ERR_WORKSPACE before anything is
 * enqueued.  SSD_FLAG_CHECK_SEQ is honoured; SSD_FLAG_TEST_STALL is not.
 *  - The array's device address is looked up (cudaGetSymbolAddress) with the
 *    calling device current: on the first call on each device, and again on
 *    every call made outside stream capture, so that a device reset (which
 *    reloads the library's device code) is picked up by the next such call.
 *    A call made while `stream` is capturing uses the address found before;
 *    make the first call on a device before any capture.  A failed lookup
 *    returns SSD_ERR_CUDA.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; each call rewrites every part it reads (and clears what must
 *    start at zero), so sequential calls are independent.  Calls that overlap
 *    on the GPU (other streams, other host threads) race on the array:
 *    serialise them. */
SSD_API ssd_status ssd_fwd_noalloc(const ssd_fwd_args* args, void* stream);

/* ssd_fwd from and to HOST memory, with the copies overlapped: for callers
 * whose inputs live on the host and who want the outputs back there.  The
 * pointer fields of `args` (x, dt, A, B, C, D, z, initial_states, seq_idx, y,
 * final_states) are host addresses, which should be pinned (page-locked,
 * e.g. cudaHostAlloc) for the copies to run asynchronously and overlap; its
 * workspace and timing_events fields are ignored.  The pages describe no such
 * entry point; it has no counterpart there.
 *
 * The work is taken in pieces, alternately on `stream` and `stream2`, each
 * with its own set of device buffers.  rows_per_piece > 0: pieces of that
 * many batch rows.  rows_per_piece < 0: pieces of -rows_per_piece tokens of
 * every row, piece j starting from the state in which piece j - 1 ends (so
 * y and the final states are those of one call), not with seq_idx.
 * rows_per_piece = 0: the library chooses eight pieces: batch / 8 rows each
 * for a batch of 8 or more, else (no seq_idx, rows of 128 tokens or more)
 * whole 64-token chunks of every row, else one piece.  For one piece the call
 * enqueues the copies of its inputs in (one cudaMemcpyAsync per tensor, or
 * one cudaMemcpy2DAsync, a row each, for token pieces), ssd_fwd on them, and
 * the copies of its y and final states out; so a piece's copies in run while
 * the previous piece computes and copies out (on PCIe the two directions run
 * at the same time).  Token pieces hand their state on through two fp32
 * buffers in the workspace, so a piece's ssd_fwd also waits for the previous
 * piece's.  With seq_idx and rows_per_piece = 0, a single row of 128 tokens
 * or more is cut at sequence starts (the first after each eighth of the row,
 * read from the host seq_idx at call time): each piece is then an independent
 * packed problem, and piece j returns the final states of the ids after
 * piece j - 1's last id through its own last id (the last piece through
 * num_seqs - 1), so that ids that never occur still come back as zeros; the
 * two buffer sets are then sized for the whole row.  Ids that are not
 * strictly increasing runs in [0, num_seqs) keep the call in one piece.  Any
 * other call with seq_idx is one piece: final_states is indexed by sequence
 * id, and a call on part of the rows would clear the ids it does not see.
 * `stream2` may be NULL: everything then runs on `stream`, in order.
 *
 * `device_workspace` (256-byte aligned, at least ssd_fwd_host_workspace_size
 * bytes, contents on entry irrelevant) holds the two buffer sets.  The call
 * returns once everything is enqueued; `stream2` first waits for the work
 * enqueued on `stream` before the call, and `stream` waits for `stream2`'s
 * part at the end, so the whole call is ordered on `stream` like a single
 * operation: the host outputs are complete once `stream` reaches that point
 * (e.g. after cudaStreamSynchronize(stream)).  SSD_FLAG_CHECK_SEQ checks the
 * host seq_idx directly, before anything is enqueued.  SSD_ERR_INVALID_ARG
 * for sizes ssd_fwd rejects or a missing pointer, SSD_ERR_WORKSPACE if the
 * workspace is missing or too small (nothing enqueued); otherwise ssd_fwd's
 * verdict on the first piece, in which case the first piece's copies in may
 * have been enqueued, or SSD_ERR_CUDA if a copy, an event or a launch failed.
 * SSD_ERR_INVALID_ARG too for token pieces with seq_idx, or whose row (seqlen
 * x nheads x headdim elements of x) reaches 2^31 bytes, the largest pitch of
 * a strided copy.
 * Outputs are undefined after any error. */
SSD_API size_t ssd_fwd_host_workspace_size(const ssd_fwd_args* args, int64_t rows_per_piece);
SSD_API ssd_status ssd_fwd_host(const ssd_fwd_args* args, int64_t rows_per_piece, void* device_workspace,
                                size_t device_workspace_bytes, void* stream, void* stream2);

/* Number of kernels ssd_fwd enqueues for these arguments (memsets excluded),
 * or 0 if the sizes are invalid. */
SSD_API int ssd_fwd_launch_count(const ssd_fwd_args* args);

/* Name of the kernel path ssd_fwd would take for these arguments
 * ("generic", "tcgen05"), or "invalid". Static string. */
SSD_API const char* ssd_fwd_path(const ssd_fwd_args* args);

/* Name of the fused kernel that dominates the call on the tensor-core path
 * ("k_ssd_fwd_pair": two heads per CTA, N = 128, an even number of heads per
 * group, H a multiple of 4 and dt 16-byte aligned, with a gate z applied to y
 * by a pass of its own after it; "k_ssd_fwd_fast": one head per CTA otherwise,
 * the gate in its epilogue), "generic" on the generic path, or "invalid".  It
 * is the kernel that timing_events bracket.  Static string; no device work. */
SSD_API const char* ssd_fwd_main_kernel(const ssd_fwd_args* args);

/* After an ssd_fwd call with these arguments: waits for `stream`, then reads
 * the error word the tensor-core kernels keep at the start of the workspace.
 * Returns SSD_ERR_TIMEOUT if a bounded device-side wait of that call gave up
 * (every wait is limited to about a second; the call's outputs are then
 * undefined, and the next ssd_fwd on the same workspace clears the word),
 * SSD_OK otherwise; always SSD_OK on the generic path, whose kernels do not
 * wait on one another.  Synchronous; reads 4 bytes; SSD_ERR_CUDA if the
 * synchronisation or the read fails.  No counterpart in the pages. */
SSD_API ssd_status ssd_fwd_device_status(const ssd_fwd_args* args, void* stream);

/* One recurrent step (decode): one new token per batch row against a running
 * state held by the caller, per row b and head h (group g as above):
 *
 *   state[b,h] <- exp(dt[b,h] A_h) state[b,h] + dt[b,h] x[b,h] B[b,g]^T
 *   y[b,h]      = state[b,h] C[b,g] + D_h x[b,h]
 *
 * the recurrent form of the same model ("22 · Mamba 2 — Transformers are
 * SSMs" section 3.1; the D feed-through as above).  It equals ssd_fwd over
 * one token (L = 1) with initial_states = state and final_states written
 * back to state.  Sizes as in ssd_fwd_args with dstate a multiple of 4 and at
 * most 256 (else SSD_ERR_UNSUPPORTED).  All pointers are device pointers
 * owned by the caller; state is read and written in place (16-byte aligned),
 * B and C must be aligned to 4 elements.  Asynchronous on `stream`; nothing
 * is enqueued when the arguments are rejected. */
typedef struct {
  int64_t batch, nheads, headdim, dstate, ngroups;
  ssd_dtype dtype;      /* of x, B, C and y */
  const void* x;        /* (b,H,P) dtype, this step's input                  */
  const float* dt;      /* (b,H) fp32 step sizes                             */
  const float* A;       /* (H) fp32 per-head decay rates                     */
  const void* B;        /* (b,G,N) dtype                                     */
  const void* C;        /* (b,G,N) dtype                                     */
  const float* D;       /* (H) fp32 skip weight, or NULL for D = 0           */
  float* state;         /* (b,H,P,N) fp32, the state before the step; holds
                           the state after it on return                      */
  void* y;              /* (b,H,P) dtype, output                             */
} ssd_step_args;

SSD_API ssd_status ssd_step(const ssd_step_args* args, void* stream);

/* Sequence parallelism: a sequence split over R ranks, rank k holding a
 * contiguous range of the tokens of every row.  The recurrence is affine in
 * the state, so over rank k's range h_out = D_k h_in + S_k, with S_k the
 * range's end state from a zero state (ssd_fwd without initial_states) and
 * D_k its total decay.  Rank r starts from h0 carried through ranks 0..r-1.
 * This is the state passing of "SSM 家族全景图（下）：Mamba-2 与 Jamba"
 * section 三.4 with a rank's range as one chunk.  Packed sequences are not
 * split this way.  Both calls are asynchronous on `stream`; device pointers
 * owned by the caller; nothing is enqueued when the arguments are rejected. */

/* out (b,H) fp32 = exp(A_h * sum_t dt[b,t,h]) over the seqlen tokens of dt
 * (b,L,H) fp32; A (H) fp32.  (The sum is taken in fp64.) */
SSD_API ssd_status ssd_total_decay(const float* dt, const float* A, float* out, int64_t batch, int64_t seqlen,
                                   int64_t nheads, void* stream);

/* out (b,H,P,N) fp32 = initial_states (or 0 when NULL) carried through
 * ranks 0..rank-1: H <- decays[k] * H + states[k] for k = 0..rank-1, with
 * states (R,b,H,P,N) fp32 (S_k) and decays (R,b,H) fp32 (D_k); states and
 * decays may be NULL when rank = 0.  headdim * dstate a multiple of 4
 * (SSD_ERR_UNSUPPORTED otherwise); states, initial_states and out 16-byte
 * aligned.  out must not overlap the inputs. */
SSD_API ssd_status ssd_state_fold(const float* states, const float* decays, const float* initial_states,
                                  float* out, int64_t rank, int64_t batch, int64_t nheads, int64_t headdim,
                                  int64_t dstate, void* stream);

/* The Mamba-2 block's causal depthwise convolution followed by SiLU, the
 * piece before the SSD on its main path ("SSM 家族全景图（下）：Mamba-2 与
 * Jamba", section 5, the block's data flow):
 *
 *   out[b,t,c] = SiLU(bias_c + sum_{k<K} weight[c,k] u[b, t-(K-1)+k, c])
 *
 * with SiLU(v) = v / (1 + e^-v), zeros before the first token and, with
 * seq_idx, no tap reaching into an earlier packed sequence.  K = width,
 * 1..4, and channels a multiple of 4 (else
 * SSD_ERR_UNSUPPORTED); u and out 16-byte aligned and not overlapping.
 * Asynchronous on `stream`; device pointers owned by the caller; nothing is
 * enqueued when the arguments are rejected. */
typedef struct {
  int64_t batch, seqlen, channels, width;
  ssd_dtype dtype;         /* of u and out */
  const void* u;           /* (b,L,channels) dtype                          */
  const float* weight;     /* (channels,width) fp32, tap k multiplies token
                              t-(width-1)+k                                */
  const float* bias;       /* (channels) fp32, or NULL for 0                */
  const int32_t* seq_idx;  /* (b,L) int32 packed-sequence ids, or NULL      */
  void* out;               /* (b,L,channels) dtype                          */
} ssd_conv_args;

SSD_API ssd_status ssd_conv1d_silu(const ssd_conv_args* args, void* stream);

/* The backward of ssd_conv1d_silu: given dout = dLoss/dout, with the
 * pre-activation a (bias + the taps) recomputed and g = dout * SiLU'(a)
 * (SiLU'(v) = s (1 + v (1 - s)), s = 1 / (1 + e^-v)):
 *
 *   du[b,s,c]   = sum over the taps k that reach s from t = s + (K-1) - k
 *                 (same sequence, t < L) of weight[c,k] g[b,t,c]
 *   dweight[c,k] = sum_{b,t} g[b,t,c] u[b, t-(K-1)+k, c]   (taps the forward takes)
 *   dbias[c]     = sum_{b,t} g[b,t,c]
 *
 * Sizes, u, weight, bias and seq_idx as in ssd_conv_args, width 1..4 (else
 * SSD_ERR_UNSUPPORTED).  Gradients are fp32.  dweight and dbias are summed in
 * a fixed order (fp64 over per-strip partials), so results are deterministic.
 * Device pointers owned by the caller; outputs must not overlap the inputs
 * or the workspace.  Asynchronous on `stream`; nothing is enqueued when the
 * arguments are rejected (SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED,
 * SSD_ERR_WORKSPACE as for ssd_bwd). */
typedef struct {
  int64_t batch, seqlen, channels, width;
  ssd_dtype dtype;         /* of u and dout                                  */
  const void* u;           /* (b,L,channels) dtype                           */
  const float* weight;     /* (channels,width) fp32                          */
  const float* bias;       /* (channels) fp32, or NULL for 0                 */
  const int32_t* seq_idx;  /* (b,L) int32 packed-sequence ids, or NULL       */
  const void* dout;        /* (b,L,channels) dtype, dLoss/dout               */
  float* du;               /* (b,L,channels) fp32, output                    */
  float* dweight;          /* (channels,width) fp32, output                  */
  float* dbias;            /* (channels) fp32 output, or NULL to skip        */
  void* workspace;         /* ssd_conv1d_silu_bwd_workspace_size bytes,
                              256-byte aligned; contents on entry do not matter */
  size_t workspace_bytes;
} ssd_conv_bwd_args;

/* Workspace bytes ssd_conv1d_silu_bwd needs (sizes only), or 0 if invalid. */
SSD_API size_t ssd_conv1d_silu_bwd_workspace_size(const ssd_conv_bwd_args* args);

SSD_API ssd_status ssd_conv1d_silu_bwd(const ssd_conv_bwd_args* args, void* stream);

/* The backward pass of ssd_fwd: the gradients of a loss with respect to every
 * input, given dy = dLoss/dy and optionally dfinal = dLoss/dfinal_states.
 * The pages give the forward recurrence (sources above) and say that the
 * backward recomputes the forward's states rather than storing them ("从
 * Transformer的二次复杂度困境到Mamba的线性突围", the hardware-aware algorithm:
 * recomputation); the gradients are the adjoint of that recurrence.  With
 * G_t = dLoss/dh_t, swept from the last token (G_{L-1} also receives dfinal):
 *
 *   G_t   = dy_t C_t^T + a_{t+1} G_{t+1}
 *   dx_t  = dt_t G_t B_t + D_h dy_t
 *   dB_t  = sum over the group's heads of dt_t G_t^T x_t
 *   dC_t  = sum over the group's heads of h_t^T dy_t
 *   ddt_t = <G_t, x_t B_t^T> + A_h a_t <G_t, h_{t-1}>
 *   dA_h  = sum_{b,t} dt_t a_t <G_t, h_{t-1}>
 *   dD_h  = sum_{b,t} <dy_t, x_t>
 *   dinitial_states = a_0 G_0
 *
 * (<.,.> sums over all entries; a token that starts a packed sequence has
 * a_t = 0 and passes no gradient to h_{t-1}, to its decay or to A.)  It is
 * computed chunk by chunk: the states entering each chunk are recomputed, the
 * adjoint state is carried backwards across chunks, and every chunk then
 * forms its gradients from its own tokens and those two states.  All
 * arithmetic is fp32; every gradient is written as fp32, whatever the input
 * dtype.  A_h <= 0 is assumed, as for ssd_fwd: the in-chunk decays
 * exp(cs_t - cs_s) and exp(cs_t) are then at most 1 (with A_h > 0 they can
 * overflow fp32).  Chunking re-associates the same sums, so the result equals the
 * adjoint recurrence up to rounding for every chunk size. */
typedef struct {
  /* sizes as in ssd_fwd_args; headdim and dstate at most 256, and one
   * headdim x dstate state must fit a CTA's shared memory next to an 8-token
   * chunk (so not both 256).  chunk_size is the chunk length of the backward
   * itself, unrelated to the forward's: 0 lets the library choose (64,
   * halved while its shared memory would not fit: 32 for dstate 256 at
   * headdim 64, 16 for 128 x 256), or 1..64 (SSD_ERR_UNSUPPORTED if that
   * does not fit). */
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk_size;
  ssd_dtype dtype;                /* of x, B, C and dy                                */
  const void* x;                  /* (b,L,H,P) dtype                                  */
  const float* dt;                /* (b,L,H) fp32                                     */
  const float* A;                 /* (H) fp32                                         */
  const void* B;                  /* (b,L,G,N) dtype                                  */
  const void* C;                  /* (b,L,G,N) dtype                                  */
  const float* D;                 /* (H) fp32, or NULL for D = 0                      */
  const float* initial_states;    /* (b,H,P,N) fp32, or NULL = 0                      */
  const int32_t* seq_idx;         /* (b,L) int32 packed-sequence ids, or NULL.  Any
                                     change of id between neighbouring tokens starts a
                                     new sequence (a_t = 0 there); ids need not
                                     increase or stay in one row, since the backward
                                     takes no per-sequence final states.              */
  const void* dy;                 /* (b,L,H,P) dtype, dLoss/dy                        */
  const float* dfinal_states;     /* (b,H,P,N) fp32 dLoss/dfinal_states, or NULL = 0.
                                     Not with seq_idx (SSD_ERR_UNSUPPORTED).          */
  float* dx;                      /* (b,L,H,P) fp32, output                           */
  float* ddt;                     /* (b,L,H) fp32, output                             */
  float* dA;                      /* (H) fp32, output                                 */
  float* dB;                      /* (b,L,G,N) fp32, output                           */
  float* dC;                      /* (b,L,G,N) fp32, output                           */
  float* dD;                      /* (H) fp32 output, or NULL to skip                 */
  float* dinitial_states;         /* (b,H,P,N) fp32 output, or NULL to skip (written
                                     also when initial_states is NULL: the gradient
                                     at a zero initial state)                        */
  void* workspace;                /* device scratch of ssd_bwd_workspace_size(args)
                                     bytes, 256-byte aligned; contents on entry do
                                     not matter                                      */
  size_t workspace_bytes;
  void* timing_events[2];         /* optional pair of cudaEvent_t (as void*), or NULLs:
                                     recorded on `stream` right before and right after
                                     k_bwd_chunk, the kernel that dominates the call.
                                     Both or neither.                                */
  const void* z;                  /* (b,L,H,P) dtype gate, or NULL.  With z the forward
                                     returned out = y * SiLU(z) (ssd_fwd_args.z) and dy
                                     is dLoss/dout: the kernels recompute y, write
                                     dz = dy * y * SiLU'(z) and take dy * SiLU(z) as
                                     the gradient of y.                              */
  float* dz;                      /* (b,L,H,P) fp32 output dLoss/dz; required iff z
                                     (unless SSD_BWD_DINITIAL_ONLY)                  */
  uint32_t flags;                 /* SSD_BWD_* or 0                                  */
} ssd_bwd_args;

/* ssd_bwd flags */
#define SSD_BWD_DINITIAL_ONLY 1u /* compute dinitial_states alone (required then; dx, ddt,
                                    dA, dB, dC, dD, dz may be NULL and are not written):
                                    two of the six kernels.  Sequence parallelism needs
                                    only this from its first backward pass.          */

/* Bytes of device workspace ssd_bwd needs (only sizes, chunk_size and dtype
 * are read), or 0 if the sizes are invalid or unsupported. */
SSD_API size_t ssd_bwd_workspace_size(const ssd_bwd_args* args);

/* The chunk length ssd_bwd uses for these arguments (chunk_size, or the
 * library's choice when it is 0), or 0 if the sizes are invalid or
 * unsupported.  Reads only the size fields; no device work. */
SSD_API int64_t ssd_bwd_chunk_size(const ssd_bwd_args* args);

/* The kernels ssd_bwd runs for these arguments: "tcgen05" when the chunk
 * states and the per-chunk gradients are formed on the tensor cores (bf16, no
 * gate, headdim 64, dstate 128, 64-token chunks, x, dy, B, C and dx 16-byte
 * aligned), "generic" when the CUDA-core kernels run, "invalid" for sizes
 * ssd_bwd rejects.  Reads sizes and pointer values only; no device work.
 * Static string. */
SSD_API const char* ssd_bwd_path(const ssd_bwd_args* args);

/* Enqueue the backward on `stream`: five kernels on the tensor-core path, six
 * otherwise (ssd_bwd_path), no allocation, no memset.
 * All pointers are device pointers owned by the caller; outputs must not
 * overlap inputs or the workspace.  Returns SSD_OK once enqueued;
 * SSD_ERR_INVALID_ARG for a null required pointer, a bad size or enum, or a
 * misaligned workspace, a single timing event, z without dz (or dz
 * without z), or an unknown flag; SSD_ERR_UNSUPPORTED as described above;
 * SSD_ERR_WORKSPACE when the workspace is missing or too small; SSD_ERR_CUDA
 * when a launch fails (outputs then undefined). */
SSD_API ssd_status ssd_bwd(const ssd_bwd_args* args, void* stream);

/* The seq_idx precondition, on a HOST copy (b,L) int32: ids in [0, num_seqs),
 * non-decreasing along each row, and no id in two rows.  SSD_OK, or
 * SSD_ERR_INVALID_ARG at the first violation (or for a null pointer or a
 * non-positive size).  Synchronous, host only; ssd_fwd runs it when
 * SSD_FLAG_CHECK_SEQ is set. */
SSD_API ssd_status ssd_check_seq_idx(const int32_t* seq_idx_host, int64_t batch, int64_t seqlen, int64_t num_seqs);

/* Static, human-readable text for a status code. */
SSD_API const char* ssd_status_string(ssd_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
SSD_API int ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
