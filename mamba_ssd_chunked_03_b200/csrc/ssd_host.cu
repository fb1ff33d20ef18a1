// ssd_fwd_host: the SSD forward from and to host memory, its copies
// overlapped with one another and with the compute.
//
// The work is cut into pieces, either of whole batch rows or, for a small
// batch without sequence ids, of a token range of every row.  Piece j runs on
// stream j % 2 with buffer set j % 2 of the device workspace: copies of its
// inputs in, ssd_fwd on them, copies of its y (and final states) out.  A set
// is reused two pieces later on the same stream, after that stream's copies
// out.  Meanwhile the other stream's copies in run beside this stream's
// compute and copies out: on PCIe the two directions move at the same time,
// so a call costs about the larger of its two copy volumes instead of their
// sum.  The tensors are row-major with the batch row outermost, so a row
// piece of each tensor is one contiguous block (one cudaMemcpyAsync), and a
// token piece is one strided block (one cudaMemcpy2DAsync: a row each).
//
// Token pieces carry the state from piece to piece: piece j starts from the
// final state of piece j - 1 (the recurrence's state at its first token, so
// the result is that of one call) and the chain alternates between two fp32
// state buffers.  Piece j's ssd_fwd therefore waits for piece j - 1's; its
// copies in do not.
//
// A single row of packed sequences is cut at sequence starts instead
// (sequence pieces), found on the host ids near each eighth of the row: every
// piece is then an independent packed problem with nothing to hand on.  Its
// final states are computed under the global ids, and piece j copies back
// the ids after piece j - 1's last up to its own last (through num_seqs - 1
// for the last piece), so that every id, occurring or not, comes back from
// exactly one piece.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ssd.h"

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// One buffer set (one piece) and where each tensor sits in it.
struct HostPlan {
  bool tok;        // pieces of `tokens` tokens of every row (else of `rows` rows)
  bool seqp;       // one row of packed sequences, cut at sequence starts at call time
                   // (buffer sets sized for the whole row)
  int64_t rows;    // rows per piece (all of them for token pieces)
  int64_t tokens;  // tokens per piece (the whole row for row pieces)
  int64_t pieces;
  // bytes per token (x, dt, B/C, seq) and per batch row (initial and final states)
  size_t tok_x, tok_dt, tok_bc, tok_seq, row_init, row_final;
  size_t off_x, off_dt, off_B, off_C, off_z, off_init, off_seq, off_y, off_final, off_ws;
  size_t ws_bytes;   // ssd_fwd's workspace for one piece
  size_t set_bytes;  // one buffer set
  size_t off_A, off_D;
  size_t off_state[2];  // token pieces: the fp32 states the pieces hand on
  size_t total;
};

// The piece's arguments as ssd_fwd sees them (device pointers filled in later).
ssd_fwd_args piece_args(const ssd_fwd_args* a, int64_t rows, int64_t tokens) {
  ssd_fwd_args p = *a;
  p.batch = rows;
  p.seqlen = tokens;
  p.flags &= ~SSD_FLAG_CHECK_SEQ;  // checked on the host copy
  p.timing_events[0] = p.timing_events[1] = nullptr;
  p.workspace = nullptr;
  p.workspace_bytes = 0;
  return p;
}

// Pieces the library picks: eight, so that the first piece's copies in and
// the last one's copies out, which nothing overlaps, are an eighth of the call
// each.  Rows when the batch has eight or more, else tokens (in whole 64-token
// chunks) when the rows are long enough and carry no sequence ids, else, for
// a single row with sequence ids, sequence pieces.  (Token and sequence
// pieces are copied with the row as pitch, which must stay below 2^31 bytes.)
constexpr int64_t kAutoPieces = 8;

bool plan(const ssd_fwd_args* a, int64_t rows_per_piece, HostPlan* p) {
  if (!a || a->batch <= 0 || a->seqlen <= 0 || a->nheads <= 0 || a->headdim <= 0 || a->dstate <= 0 ||
      a->ngroups <= 0 || (a->dtype != SSD_F32 && a->dtype != SSD_BF16))
    return false;
  const int64_t b = a->batch, L = a->seqlen, H = a->nheads, P = a->headdim, N = a->dstate, G = a->ngroups;
  if (rows_per_piece < 0 && a->seq_idx) return false;  // token pieces would split sequences
  const size_t es0 = a->dtype == SSD_BF16 ? 2 : 4;
  const bool tok_ok = (size_t)L * (size_t)(H * P) * es0 < ((size_t)1 << 31);
  if (rows_per_piece < 0 && !tok_ok) return false;
  p->tok = false;
  p->seqp = false;
  p->rows = b;
  p->tokens = L;
  if (rows_per_piece < 0) {
    p->tok = true;
    p->tokens = -rows_per_piece < L ? -rows_per_piece : L;
  } else if (rows_per_piece > 0) {
    p->rows = rows_per_piece < b ? rows_per_piece : b;
  } else if (b >= kAutoPieces) {
    p->rows = b / kAutoPieces;
  } else if (!a->seq_idx && L >= 2 * 64 && tok_ok) {
    p->tok = true;
    p->tokens = ((L + kAutoPieces - 1) / kAutoPieces + 63) / 64 * 64;
  } else if (a->seq_idx && b == 1 && L >= 2 * 64 && tok_ok) {
    p->seqp = true;
  }
  if (a->seq_idx) p->rows = b;  // rows of packed sequences: one piece, final states by id
  p->pieces = p->seqp ? kAutoPieces : p->tok ? (L + p->tokens - 1) / p->tokens : (b + p->rows - 1) / p->rows;
  if (p->pieces == 1) p->tok = false;
  const int64_t rows = p->rows, T = p->tokens;
  const size_t es = a->dtype == SSD_BF16 ? 2 : 4;
  p->tok_x = (size_t)(H * P) * es;
  p->tok_dt = (size_t)H * 4;
  p->tok_bc = (size_t)(G * N) * es;
  p->tok_seq = 4;
  p->row_init = (size_t)(H * P * N) * 4;
  p->row_final = (size_t)(H * P * N) * 4;
  ssd_fwd_args pa = piece_args(a, rows, T);
  if (p->tok) pa.initial_states = pa.final_states = reinterpret_cast<float*>(uintptr_t(256));  // (presence only)
  if (ssd_fwd_launch_count(&pa) == 0) return false;  // sizes ssd_fwd rejects
  p->ws_bytes = ssd_fwd_workspace_size(&pa);
  // the last piece may be shorter or have fewer rows: its workspace too
  ssd_fwd_args pl = pa;
  if (p->tok) pl.seqlen = L - (p->pieces - 1) * T;
  else if (!p->seqp) pl.batch = b - (p->pieces - 1) * rows;
  if (ssd_fwd_launch_count(&pl) == 0) return false;
  const size_t wl = ssd_fwd_workspace_size(&pl);
  if (wl > p->ws_bytes) p->ws_bytes = wl;
  const size_t cells = (size_t)(rows * T);  // tokens of one piece, over its rows
  size_t o = 0;
  p->off_x = o;
  o = align_up(o + cells * p->tok_x);
  p->off_dt = o;
  o = align_up(o + cells * p->tok_dt);
  p->off_B = o;
  o = align_up(o + cells * p->tok_bc);
  p->off_C = o;
  o = align_up(o + cells * p->tok_bc);
  p->off_z = o;
  if (a->z) o = align_up(o + cells * p->tok_x);
  p->off_init = o;
  if (a->initial_states && !p->tok) o = align_up(o + rows * p->row_init);
  p->off_seq = o;
  if (a->seq_idx) o = align_up(o + cells * p->tok_seq);
  p->off_y = o;
  o = align_up(o + cells * p->tok_x);
  p->off_final = o;
  if (a->final_states && !p->tok)
    o = align_up(o + (a->seq_idx ? (size_t)a->num_seqs * p->row_final : rows * p->row_final));
  p->off_ws = o;
  o = align_up(o + p->ws_bytes);
  p->set_bytes = o;
  const int64_t sets = p->pieces > 1 ? 2 : 1;
  o = sets * p->set_bytes;
  p->off_A = o;
  o = align_up(o + (size_t)H * 4);
  p->off_D = o;
  if (a->D) o = align_up(o + (size_t)H * 4);
  for (int i = 0; i < 2; ++i) {
    p->off_state[i] = o;
    if (p->tok) o = align_up(o + (size_t)b * p->row_final);
  }
  p->total = o;
  return true;
}

cudaError_t h2d(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s) : cudaSuccess;
}
cudaError_t d2h(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) : cudaSuccess;
}
// tokens [t0, t0 + n) of each of `rows` rows (row stride L tokens of `w` bytes)
// into a packed (rows, n) block, or back
cudaError_t h2d_tok(void* dst, const void* src, size_t w, int64_t L, int64_t t0, int64_t n, int64_t rows,
                    cudaStream_t s) {
  return cudaMemcpy2DAsync(dst, n * w, static_cast<const unsigned char*>(src) + t0 * w, L * w, n * w, rows,
                           cudaMemcpyHostToDevice, s);
}
cudaError_t d2h_tok(void* dst, const void* src, size_t w, int64_t L, int64_t t0, int64_t n, int64_t rows,
                    cudaStream_t s) {
  return cudaMemcpy2DAsync(static_cast<unsigned char*>(dst) + t0 * w, L * w, src, n * w, n * w, rows,
                           cudaMemcpyDeviceToHost, s);
}

// Sequence pieces: the first sequence start at or after each eighth of the
// row, as cut[0] = 0 < cut[1] < .. < cut[n] = L; n, or 0 when the ids are
// not strictly increasing runs in [0, num_seqs) (the call then runs whole).
int64_t seq_cuts(const int32_t* seq, int64_t L, int64_t num_seqs, int64_t cut[kAutoPieces + 1]) {
  int64_t n = 0;
  cut[0] = 0;
  if (seq[0] < 0 || seq[0] >= num_seqs) return 0;
  for (int64_t t = 1; t < L; ++t) {
    if (seq[t] == seq[t - 1]) continue;
    if (seq[t] < seq[t - 1] || seq[t] >= num_seqs) return 0;
    if (n + 1 < kAutoPieces && t >= (n + 1) * L / kAutoPieces) cut[++n] = t;
  }
  cut[++n] = L;
  return n;
}

}  // namespace

extern "C" {

SSD_API size_t ssd_fwd_host_workspace_size(const ssd_fwd_args* args, int64_t rows_per_piece) {
  HostPlan p;
  return plan(args, rows_per_piece, &p) ? p.total : 0;
}

SSD_API ssd_status ssd_fwd_host(const ssd_fwd_args* args, int64_t rows_per_piece, void* device_workspace,
                                size_t device_workspace_bytes, void* stream, void* stream2) {
  HostPlan p;
  if (!args || !plan(args, rows_per_piece, &p)) return SSD_ERR_INVALID_ARG;
  const ssd_fwd_args* a = args;
  if (!a->x || !a->dt || !a->A || !a->B || !a->C || !a->y) return SSD_ERR_INVALID_ARG;
  if (!device_workspace || device_workspace_bytes < p.total) return SSD_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(device_workspace) & (kAlign - 1)) != 0) return SSD_ERR_INVALID_ARG;
  if ((a->flags & SSD_FLAG_CHECK_SEQ) && a->seq_idx) {
    const ssd_status st = ssd_check_seq_idx(a->seq_idx, a->batch, a->seqlen, a->num_seqs);
    if (st != SSD_OK) return st;
  }
  unsigned char* ws = static_cast<unsigned char*>(device_workspace);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  cudaStream_t s1 = stream2 ? static_cast<cudaStream_t>(stream2) : s0;
  int64_t cut[kAutoPieces + 1];
  const int64_t ncut = p.seqp ? seq_cuts(a->seq_idx, a->seqlen, a->num_seqs, cut) : 0;
  const bool seqp = ncut > 1;
  const int64_t pieces = p.seqp ? (seqp ? ncut : 1) : p.pieces;
  const bool two = s1 != s0 && pieces > 1;

  cudaEvent_t fork = nullptr, join = nullptr, done[2] = {nullptr, nullptr};
  auto destroy = [&]() {
    for (cudaEvent_t e : {fork, join, done[0], done[1]})
      if (e) cudaEventDestroy(e);
  };
  if (two && (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
              cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess)) {
    destroy();
    return SSD_ERR_CUDA;
  }
  if (p.tok && two && (cudaEventCreateWithFlags(&done[0], cudaEventDisableTiming) != cudaSuccess ||
                       cudaEventCreateWithFlags(&done[1], cudaEventDisableTiming) != cudaSuccess)) {
    destroy();
    return SSD_ERR_CUDA;
  }
  ssd_status st = SSD_OK;
  auto fail = [&](ssd_status e) {
    if (st == SSD_OK) st = e;
  };
  const int64_t b = a->batch, L = a->seqlen;
  float* state[2] = {reinterpret_cast<float*>(ws + p.off_state[0]), reinterpret_cast<float*>(ws + p.off_state[1])};
  // A and D (per head) once, and for token pieces the initial states (the
  // state before piece 0, in the buffer piece 0 reads), on `stream` before
  // the other stream forks off
  float* dA = reinterpret_cast<float*>(ws + p.off_A);
  float* dD = a->D ? reinterpret_cast<float*>(ws + p.off_D) : nullptr;
  if (h2d(dA, a->A, (size_t)a->nheads * 4, s0) != cudaSuccess) fail(SSD_ERR_CUDA);
  if (dD && h2d(dD, a->D, (size_t)a->nheads * 4, s0) != cudaSuccess) fail(SSD_ERR_CUDA);
  if (p.tok && a->initial_states && h2d(state[1], a->initial_states, (size_t)b * p.row_init, s0) != cudaSuccess)
    fail(SSD_ERR_CUDA);
  if (two && st == SSD_OK &&
      (cudaEventRecord(fork, s0) != cudaSuccess || cudaStreamWaitEvent(s1, fork, 0) != cudaSuccess))
    fail(SSD_ERR_CUDA);

  const unsigned char* hx = static_cast<const unsigned char*>(a->x);
  const unsigned char* hdt = reinterpret_cast<const unsigned char*>(a->dt);
  const unsigned char* hB = static_cast<const unsigned char*>(a->B);
  const unsigned char* hC = static_cast<const unsigned char*>(a->C);
  const unsigned char* hz = static_cast<const unsigned char*>(a->z);
  const unsigned char* hinit = reinterpret_cast<const unsigned char*>(a->initial_states);
  const unsigned char* hseq = reinterpret_cast<const unsigned char*>(a->seq_idx);
  unsigned char* hy = static_cast<unsigned char*>(a->y);
  unsigned char* hfin = reinterpret_cast<unsigned char*>(a->final_states);
  const bool by_tok = p.tok || seqp;  // pieces of tokens of every row
  for (int64_t j = 0; j < pieces && st == SSD_OK; ++j) {
    // row pieces: rows [r0, r0 + nr), every token; token and sequence pieces:
    // every row, tokens [t0, t0 + nt)
    const int64_t r0 = by_tok ? 0 : j * p.rows, nr = by_tok ? b : (b - r0 < p.rows ? b - r0 : p.rows);
    int64_t t0 = 0, nt = L;
    if (p.tok) {
      t0 = j * p.tokens;
      nt = L - t0 < p.tokens ? L - t0 : p.tokens;
    } else if (seqp) {
      t0 = cut[j];
      nt = cut[j + 1] - cut[j];
    }
    cudaStream_t s = (two && (j & 1)) ? s1 : s0;
    unsigned char* set = ws + (two ? (size_t)(j & 1) * p.set_bytes : 0);
    ssd_fwd_args pa = piece_args(a, nr, nt);
    pa.x = set + p.off_x;
    pa.dt = reinterpret_cast<const float*>(set + p.off_dt);
    pa.A = dA;
    pa.B = set + p.off_B;
    pa.C = set + p.off_C;
    pa.D = dD;
    pa.z = a->z ? set + p.off_z : nullptr;
    pa.seq_idx = a->seq_idx ? reinterpret_cast<const int32_t*>(set + p.off_seq) : nullptr;
    pa.y = set + p.off_y;
    if (p.tok) {  // from the state the previous piece left, to the other buffer
      pa.initial_states = (j > 0 || a->initial_states) ? state[(j + 1) & 1] : nullptr;
      pa.final_states = state[j & 1];
    } else {  // (sequence pieces: h0 is the state before the row's first token only)
      pa.initial_states =
          a->initial_states && (!seqp || j == 0) ? reinterpret_cast<const float*>(set + p.off_init) : nullptr;
      pa.final_states = a->final_states ? reinterpret_cast<float*>(set + p.off_final) : nullptr;
    }
    pa.workspace = p.ws_bytes ? set + p.off_ws : nullptr;
    pa.workspace_bytes = p.ws_bytes;
    bool ok;
    if (by_tok) {
      ok = h2d_tok(set + p.off_x, hx, p.tok_x, L, t0, nt, b, s) == cudaSuccess &&
           h2d_tok(set + p.off_dt, hdt, p.tok_dt, L, t0, nt, b, s) == cudaSuccess &&
           h2d_tok(set + p.off_B, hB, p.tok_bc, L, t0, nt, b, s) == cudaSuccess &&
           h2d_tok(set + p.off_C, hC, p.tok_bc, L, t0, nt, b, s) == cudaSuccess &&
           (!hz || h2d_tok(set + p.off_z, hz, p.tok_x, L, t0, nt, b, s) == cudaSuccess) &&
           (!seqp || h2d_tok(set + p.off_seq, hseq, p.tok_seq, L, t0, nt, b, s) == cudaSuccess) &&
           (!seqp || j > 0 || !hinit || h2d(set + p.off_init, hinit, p.row_init, s) == cudaSuccess);
      // piece j's state comes from piece j - 1 (on the other stream)
      if (ok && p.tok && two && j > 0) ok = cudaStreamWaitEvent(s, done[(j - 1) & 1], 0) == cudaSuccess;
    } else {
      const size_t row_x = (size_t)L * p.tok_x, row_dt = (size_t)L * p.tok_dt, row_bc = (size_t)L * p.tok_bc,
                   row_seq = (size_t)L * p.tok_seq;
      ok = h2d(set + p.off_x, hx + r0 * row_x, nr * row_x, s) == cudaSuccess &&
           h2d(set + p.off_dt, hdt + r0 * row_dt, nr * row_dt, s) == cudaSuccess &&
           h2d(set + p.off_B, hB + r0 * row_bc, nr * row_bc, s) == cudaSuccess &&
           h2d(set + p.off_C, hC + r0 * row_bc, nr * row_bc, s) == cudaSuccess &&
           (!hz || h2d(set + p.off_z, hz + r0 * row_x, nr * row_x, s) == cudaSuccess) &&
           (!hinit || h2d(set + p.off_init, hinit + r0 * p.row_init, nr * p.row_init, s) == cudaSuccess) &&
           (!hseq || h2d(set + p.off_seq, hseq + r0 * row_seq, nr * row_seq, s) == cudaSuccess);
    }
    if (!ok) {
      fail(SSD_ERR_CUDA);
      break;
    }
    const ssd_status fs = ssd_fwd(&pa, s);
    if (fs != SSD_OK) {
      fail(fs);
      break;
    }
    if (p.tok && two && cudaEventRecord(done[j & 1], s) != cudaSuccess) {
      fail(SSD_ERR_CUDA);
      break;
    }
    const cudaError_t ey = by_tok ? d2h_tok(hy, set + p.off_y, p.tok_x, L, t0, nt, b, s)
                                  : d2h(hy + r0 * L * p.tok_x, set + p.off_y, nr * L * p.tok_x, s);
    if (ey != cudaSuccess) {
      fail(SSD_ERR_CUDA);
      break;
    }
    if (hfin && seqp) {  // the ids after the previous piece's last, through this piece's last
      const int64_t lo = j == 0 ? 0 : (int64_t)a->seq_idx[cut[j] - 1] + 1;
      const int64_t hi = j == pieces - 1 ? a->num_seqs - 1 : (int64_t)a->seq_idx[cut[j + 1] - 1];
      if (d2h(hfin + lo * p.row_final, set + p.off_final + lo * p.row_final, (size_t)(hi - lo + 1) * p.row_final,
              s) != cudaSuccess) {
        fail(SSD_ERR_CUDA);
        break;
      }
    } else if (hfin && (!p.tok || j == p.pieces - 1)) {  // token pieces: the last piece's end state
      const size_t fb = a->seq_idx ? (size_t)a->num_seqs * p.row_final : nr * p.row_final;
      const void* src = p.tok ? static_cast<const void*>(state[j & 1]) : set + p.off_final;
      if (d2h(hfin + (a->seq_idx ? 0 : r0 * p.row_final), src, fb, s) != cudaSuccess) {
        fail(SSD_ERR_CUDA);
        break;
      }
    }
  }
  if (two) {  // `stream` waits for the other stream's part, also after a failure
    if (cudaEventRecord(join, s1) != cudaSuccess || cudaStreamWaitEvent(s0, join, 0) != cudaSuccess)
      fail(SSD_ERR_CUDA);
  }
  destroy();
  return st;
}

}  // extern "C"
