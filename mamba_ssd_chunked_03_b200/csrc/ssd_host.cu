// ssd_fwd_host: the SSD forward from and to host memory, its copies
// overlapped with one another and with the compute.
//
// The batch is cut into pieces of whole rows.  Piece j runs on stream j % 2
// with buffer set j % 2 of the device workspace: copies of its rows' inputs
// in, ssd_fwd on them, copies of its y (and final states) out.  A set is
// reused two pieces later on the same stream, after that stream's copies out,
// so no piece waits on the other stream.  Meanwhile the other stream's copies
// in run beside this stream's compute and copies out: on PCIe the two
// directions move at the same time, so a call costs about the larger of its
// two copy volumes instead of their sum.  Every copy is one cudaMemcpyAsync
// of a contiguous block: the tensors are row-major with the batch row
// outermost, so a piece's rows of each tensor are one block.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ssd.h"

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// One buffer set (one piece's worth of rows) and where each tensor sits in it.
struct HostPlan {
  int64_t rows;    // rows per piece
  int64_t pieces;  // ceil(batch / rows)
  // bytes per batch row of each per-row tensor, and of the final states
  size_t row_x, row_dt, row_bc, row_init, row_seq, row_final;
  size_t off_x, off_dt, off_B, off_C, off_z, off_init, off_seq, off_y, off_final, off_ws;
  size_t ws_bytes;   // ssd_fwd's workspace for `rows` rows
  size_t set_bytes;  // one buffer set
  size_t off_A, off_D;
  size_t total;
};

// The piece's arguments as ssd_fwd sees them (device pointers filled in later).
ssd_fwd_args piece_args(const ssd_fwd_args* a, int64_t rows) {
  ssd_fwd_args p = *a;
  p.batch = rows;
  p.flags &= ~SSD_FLAG_CHECK_SEQ;  // checked on the host copy
  p.timing_events[0] = p.timing_events[1] = nullptr;
  p.workspace = nullptr;
  p.workspace_bytes = 0;
  return p;
}

bool plan(const ssd_fwd_args* a, int64_t rows_per_piece, HostPlan* p) {
  if (!a || a->batch <= 0 || a->seqlen <= 0 || a->nheads <= 0 || a->headdim <= 0 || a->dstate <= 0 ||
      a->ngroups <= 0 || rows_per_piece < 0 || (a->dtype != SSD_F32 && a->dtype != SSD_BF16))
    return false;
  const int64_t b = a->batch, L = a->seqlen, H = a->nheads, P = a->headdim, N = a->dstate, G = a->ngroups;
  int64_t rows = rows_per_piece > 0 ? rows_per_piece : (b >= 8 ? b / 8 : 1);
  if (rows > b || a->seq_idx) rows = b;  // one piece with sequence ids: final states by id
  p->rows = rows;
  p->pieces = (b + rows - 1) / rows;
  const size_t es = a->dtype == SSD_BF16 ? 2 : 4;
  p->row_x = (size_t)(L * H * P) * es;
  p->row_dt = (size_t)(L * H) * 4;
  p->row_bc = (size_t)(L * G * N) * es;
  p->row_init = (size_t)(H * P * N) * 4;
  p->row_seq = (size_t)L * 4;
  p->row_final = (size_t)(H * P * N) * 4;
  ssd_fwd_args pa = piece_args(a, rows);
  if (ssd_fwd_launch_count(&pa) == 0) return false;  // sizes ssd_fwd rejects
  p->ws_bytes = ssd_fwd_workspace_size(&pa);
  size_t o = 0;
  p->off_x = o;
  o = align_up(o + rows * p->row_x);
  p->off_dt = o;
  o = align_up(o + rows * p->row_dt);
  p->off_B = o;
  o = align_up(o + rows * p->row_bc);
  p->off_C = o;
  o = align_up(o + rows * p->row_bc);
  p->off_z = o;
  if (a->z) o = align_up(o + rows * p->row_x);
  p->off_init = o;
  if (a->initial_states) o = align_up(o + rows * p->row_init);
  p->off_seq = o;
  if (a->seq_idx) o = align_up(o + rows * p->row_seq);
  p->off_y = o;
  o = align_up(o + rows * p->row_x);
  p->off_final = o;
  if (a->final_states) o = align_up(o + (a->seq_idx ? (size_t)a->num_seqs * p->row_final : rows * p->row_final));
  p->off_ws = o;
  o = align_up(o + p->ws_bytes);
  p->set_bytes = o;
  const int64_t sets = p->pieces > 1 ? 2 : 1;
  o = sets * p->set_bytes;
  p->off_A = o;
  o = align_up(o + (size_t)H * 4);
  p->off_D = o;
  if (a->D) o = align_up(o + (size_t)H * 4);
  p->total = o;
  return true;
}

cudaError_t h2d(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s) : cudaSuccess;
}
cudaError_t d2h(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) : cudaSuccess;
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
  const bool two = s1 != s0 && p.pieces > 1;

  cudaEvent_t fork = nullptr, join = nullptr;
  if (two) {
    if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess) return SSD_ERR_CUDA;
    if (cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
      cudaEventDestroy(fork);
      return SSD_ERR_CUDA;
    }
  }
  ssd_status st = SSD_OK;
  auto fail = [&](ssd_status e) {
    if (st == SSD_OK) st = e;
  };
  // A and D (per head) once, on `stream`, before the other stream forks off
  float* dA = reinterpret_cast<float*>(ws + p.off_A);
  float* dD = a->D ? reinterpret_cast<float*>(ws + p.off_D) : nullptr;
  if (h2d(dA, a->A, (size_t)a->nheads * 4, s0) != cudaSuccess) fail(SSD_ERR_CUDA);
  if (dD && h2d(dD, a->D, (size_t)a->nheads * 4, s0) != cudaSuccess) fail(SSD_ERR_CUDA);
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
  for (int64_t j = 0; j < p.pieces && st == SSD_OK; ++j) {
    const int64_t r0 = j * p.rows, nr = a->batch - r0 < p.rows ? a->batch - r0 : p.rows;
    cudaStream_t s = (two && (j & 1)) ? s1 : s0;
    unsigned char* set = ws + (two ? (size_t)(j & 1) * p.set_bytes : 0);
    ssd_fwd_args pa = piece_args(a, nr);
    pa.x = set + p.off_x;
    pa.dt = reinterpret_cast<const float*>(set + p.off_dt);
    pa.A = dA;
    pa.B = set + p.off_B;
    pa.C = set + p.off_C;
    pa.D = dD;
    pa.z = a->z ? set + p.off_z : nullptr;
    pa.initial_states = a->initial_states ? reinterpret_cast<const float*>(set + p.off_init) : nullptr;
    pa.seq_idx = a->seq_idx ? reinterpret_cast<const int32_t*>(set + p.off_seq) : nullptr;
    pa.y = set + p.off_y;
    pa.final_states = a->final_states ? reinterpret_cast<float*>(set + p.off_final) : nullptr;
    pa.workspace = p.ws_bytes ? set + p.off_ws : nullptr;
    pa.workspace_bytes = p.ws_bytes;
    if (h2d(set + p.off_x, hx + r0 * p.row_x, nr * p.row_x, s) != cudaSuccess ||
        h2d(set + p.off_dt, hdt + r0 * p.row_dt, nr * p.row_dt, s) != cudaSuccess ||
        h2d(set + p.off_B, hB + r0 * p.row_bc, nr * p.row_bc, s) != cudaSuccess ||
        h2d(set + p.off_C, hC + r0 * p.row_bc, nr * p.row_bc, s) != cudaSuccess ||
        (hz && h2d(set + p.off_z, hz + r0 * p.row_x, nr * p.row_x, s) != cudaSuccess) ||
        (hinit && h2d(set + p.off_init, hinit + r0 * p.row_init, nr * p.row_init, s) != cudaSuccess) ||
        (hseq && h2d(set + p.off_seq, hseq + r0 * p.row_seq, nr * p.row_seq, s) != cudaSuccess)) {
      fail(SSD_ERR_CUDA);
      break;
    }
    const ssd_status fs = ssd_fwd(&pa, s);
    if (fs != SSD_OK) {
      fail(fs);
      break;
    }
    if (d2h(hy + r0 * p.row_x, set + p.off_y, nr * p.row_x, s) != cudaSuccess) {
      fail(SSD_ERR_CUDA);
      break;
    }
    if (hfin) {
      const size_t fb = a->seq_idx ? (size_t)a->num_seqs * p.row_final : nr * p.row_final;
      if (d2h(hfin + (a->seq_idx ? 0 : r0 * p.row_final), set + p.off_final, fb, s) != cudaSuccess) {
        fail(SSD_ERR_CUDA);
        break;
      }
    }
  }
  if (two) {  // `stream` waits for the other stream's part, also after a failure
    if (cudaEventRecord(join, s1) != cudaSuccess || cudaStreamWaitEvent(s0, join, 0) != cudaSuccess)
      fail(SSD_ERR_CUDA);
    cudaEventDestroy(fork);
    cudaEventDestroy(join);
  }
  return st;
}

}  // extern "C"
