// C ABI of libssd: argument validation, workspace sizing and kernel dispatch.
// The operation and its sources are described in include/ssd.h.
#include <cuda_runtime.h>

#include <vector>

#include "ssd.h"
#include "ssd_internal.h"

namespace ssd {
namespace {

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Size and option checks shared by the workspace query and the forward.
ssd_status check_sizes(const ssd_fwd_args* a) {
  if (!a) return SSD_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->seqlen <= 0 || a->nheads <= 0 || a->headdim <= 0 || a->dstate <= 0 ||
      a->ngroups <= 0 || a->chunk_size <= 0)
    return SSD_ERR_INVALID_ARG;
  if (a->nheads % a->ngroups != 0) return SSD_ERR_INVALID_ARG;
  if (!is_pow2(a->chunk_size) || a->chunk_size < 16 || a->chunk_size > 256) return SSD_ERR_INVALID_ARG;
  if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (a->flags & ~(SSD_FLAG_GENERIC | SSD_FLAG_CHECK_SEQ | SSD_FLAG_TEST_STALL)) return SSD_ERR_INVALID_ARG;
  if (a->seq_idx && a->num_seqs <= 0) return SSD_ERR_INVALID_ARG;
  if (a->seq_idx && a->num_seqs > (int64_t)1 << 31) return SSD_ERR_INVALID_ARG;
  // implemented shape set
  if (a->headdim % 8 != 0 || a->headdim > 256) return SSD_ERR_UNSUPPORTED;
  if (a->dstate % 8 != 0 || a->dstate > 256) return SSD_ERR_UNSUPPORTED;
  if (a->batch > 65535) return SSD_ERR_UNSUPPORTED;
  // keep every flattened index far inside int64 and every grid inside 2^31
  const double tokens = (double)a->batch * (double)a->seqlen;
  if (tokens * (double)a->nheads * (double)(a->headdim > a->dstate ? a->headdim : a->dstate) > 4e18)
    return SSD_ERR_UNSUPPORTED;
  const double chunks = (double)((a->seqlen + a->chunk_size - 1) / a->chunk_size);
  if (chunks * (double)a->nheads * 64.0 > 2.0e9) return SSD_ERR_UNSUPPORTED;
  if (a->seq_idx && (double)a->num_seqs * (double)a->nheads * 64.0 > 2.0e9) return SSD_ERR_UNSUPPORTED;
  if ((a->timing_events[0] == nullptr) != (a->timing_events[1] == nullptr)) return SSD_ERR_INVALID_ARG;
  return SSD_OK;
}

Problem resolve(const ssd_fwd_args* a) {
  Problem p;
  p.b = a->batch;
  p.L = a->seqlen;
  p.H = a->nheads;
  p.P = a->headdim;
  p.N = a->dstate;
  p.G = a->ngroups;
  p.Q = a->chunk_size;
  p.nc = (p.L + p.Q - 1) / p.Q;
  p.hpg = p.H / p.G;
  p.dtype = a->dtype;
  p.x = a->x;
  p.dt = a->dt;
  p.A = a->A;
  p.B = a->B;
  p.C = a->C;
  p.D = a->D;
  p.h0 = a->initial_states;
  p.seq = a->seq_idx;
  p.z = a->z;
  p.num_seqs = a->seq_idx ? a->num_seqs : 0;
  p.y = a->y;
  p.final_states = a->final_states;
  p.stall = (a->flags & SSD_FLAG_TEST_STALL) != 0;
  return p;
}

}  // namespace
}  // namespace ssd

extern "C" {

size_t ssd_fwd_workspace_size(const ssd_fwd_args* args) {
  if (ssd::check_sizes(args) != SSD_OK) return 0;
  const ssd::Problem p = ssd::resolve(args);
  return ssd::tc_supported(p, args->flags) ? ssd::tc_workspace_bytes(p) : ssd::generic_workspace_bytes(p);
}

int ssd_fwd_launch_count(const ssd_fwd_args* args) {
  if (ssd::check_sizes(args) != SSD_OK) return 0;
  const ssd::Problem p = ssd::resolve(args);
  return ssd::tc_supported(p, args->flags) ? ssd::tc_launch_count(p) : ssd::generic_launch_count(p);
}

const char* ssd_fwd_path(const ssd_fwd_args* args) {
  if (ssd::check_sizes(args) != SSD_OK) return "invalid";
  return ssd::tc_supported(ssd::resolve(args), args->flags) ? "tcgen05" : "generic";
}

ssd_status ssd_fwd_device_status(const ssd_fwd_args* args, void* stream) {
  ssd_status st = ssd::check_sizes(args);
  if (st != SSD_OK) return st;
  const ssd::Problem p = ssd::resolve(args);
  if (!ssd::tc_supported(p, args->flags)) return SSD_OK;
  if (!args->workspace) return SSD_ERR_WORKSPACE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SSD_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, ssd::tc_error_word(p, args->workspace), sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SSD_ERR_CUDA;
  return word ? SSD_ERR_TIMEOUT : SSD_OK;
}

const char* ssd_fwd_main_kernel(const ssd_fwd_args* args) {
  if (ssd::check_sizes(args) != SSD_OK) return "invalid";
  const ssd::Problem p = ssd::resolve(args);
  return ssd::tc_supported(p, args->flags) ? ssd::tc_main_kernel(p) : "generic";
}

ssd_status ssd_fwd(const ssd_fwd_args* args, void* stream) {
  ssd_status st = ssd::check_sizes(args);
  if (st != SSD_OK) return st;
  const ssd_fwd_args* a = args;
  if (!a->x || !a->dt || !a->A || !a->B || !a->C || !a->y) return SSD_ERR_INVALID_ARG;
  // 16-byte alignment: vector loads and bulk copies
  if (!ssd::aligned(a->x, 16) || !ssd::aligned(a->B, 16) || !ssd::aligned(a->C, 16) ||
      !ssd::aligned(a->y, 16) || !ssd::aligned(a->dt, 4) || !ssd::aligned(a->A, 4) ||
      !ssd::aligned(a->D, 4) || !ssd::aligned(a->seq_idx, 4) || !ssd::aligned(a->initial_states, 16) ||
      !ssd::aligned(a->final_states, 16))
    return SSD_ERR_INVALID_ARG;
  const ssd::Problem p = ssd::resolve(a);
  const bool tc = ssd::tc_supported(p, a->flags);
  const size_t need = tc ? ssd::tc_workspace_bytes(p) : ssd::generic_workspace_bytes(p);
  if (need > 0 && (!a->workspace || a->workspace_bytes < need)) return SSD_ERR_WORKSPACE;
  if (!ssd::aligned(a->workspace, ssd::kWsAlign)) return SSD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((a->flags & SSD_FLAG_CHECK_SEQ) && a->seq_idx) {
    std::vector<int32_t> host((size_t)(a->batch * a->seqlen));
    if (cudaMemcpyAsync(host.data(), a->seq_idx, host.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return SSD_ERR_CUDA;
    const ssd_status cs = ssd_check_seq_idx(host.data(), a->batch, a->seqlen, a->num_seqs);
    if (cs != SSD_OK) return cs;
  }
  cudaEvent_t ev0 = static_cast<cudaEvent_t>(a->timing_events[0]);
  cudaEvent_t ev1 = static_cast<cudaEvent_t>(a->timing_events[1]);
  if (tc) return ssd::tc_forward(p, a->workspace, s, ev0, ev1) == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
  if (ev0 && cudaEventRecord(ev0, s) != cudaSuccess) return SSD_ERR_CUDA;
  const cudaError_t err = ssd::generic_forward(p, a->workspace, s);
  if (err != cudaSuccess) return SSD_ERR_CUDA;
  if (ev1 && cudaEventRecord(ev1, s) != cudaSuccess) return SSD_ERR_CUDA;
  return SSD_OK;
}

ssd_status ssd_check_seq_idx(const int32_t* seq, int64_t batch, int64_t seqlen, int64_t num_seqs) {
  if (!seq || batch <= 0 || seqlen <= 0 || num_seqs <= 0) return SSD_ERR_INVALID_ARG;
  std::vector<int64_t> row_of((size_t)num_seqs, -1);  // the row each id was seen in
  for (int64_t r = 0; r < batch; ++r) {
    for (int64_t t = 0; t < seqlen; ++t) {
      const int32_t id = seq[r * seqlen + t];
      if (id < 0 || id >= num_seqs) return SSD_ERR_INVALID_ARG;
      if (t > 0 && id < seq[r * seqlen + t - 1]) return SSD_ERR_INVALID_ARG;  // decreasing along the row
      if (row_of[(size_t)id] != -1 && row_of[(size_t)id] != r) return SSD_ERR_INVALID_ARG;  // in two rows
      row_of[(size_t)id] = r;
    }
  }
  return SSD_OK;
}

const char* ssd_status_string(ssd_status s) {
  switch (s) {
    case SSD_OK: return "ok";
    case SSD_ERR_INVALID_ARG: return "invalid argument";
    case SSD_ERR_UNSUPPORTED: return "unsupported shape or option";
    case SSD_ERR_WORKSPACE: return "workspace missing or too small";
    case SSD_ERR_CUDA: return "CUDA error";
    case SSD_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int ssd_version(void) { return 100; }

}  // extern "C"
