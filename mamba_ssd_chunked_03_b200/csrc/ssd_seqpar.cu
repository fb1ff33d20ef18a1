// The two state operations that let a sequence be split over several ranks
// (sequence parallelism): each rank holds a contiguous range of the tokens of
// every row.  The recurrence h_t = a_t h_{t-1} + dt_t x_t B_t^T is affine in
// h, so over a rank's range it is h_out = D h_in + S, with
//     D = prod_t a_t = exp(A_h sum_t dt_t)    (ssd_total_decay)
//     S = the range's end state from h_in = 0 (ssd_fwd without initial_states)
// and rank r starts from h0 carried through ranks 0..r-1 (ssd_state_fold).
// This is the state passing of "SSM 家族全景图（下）：Mamba-2 与 Jamba" section
// 三.4 with a rank's range as one chunk, and the "sequence shortened to 1/Q"
// remark of "22 · Mamba 2 — Transformers are SSMs" section 4.1 one level up.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {
namespace {

// one warp per (row, head): sum of dt over the row's tokens, then exp(A sum)
__global__ void __launch_bounds__(256) k_total_decay(const float* __restrict__ dt, const float* __restrict__ A,
                                                     float* __restrict__ out, int64_t b, int64_t L, int64_t H) {
  const int64_t u = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // b * H + h
  const int lane = threadIdx.x & 31;
  if (u >= b * H) return;
  const int64_t row = u / H, h = u % H;
  double s = 0.0;  // fp64: L may be long, the sum feeds an exponential
  for (int64_t t = lane; t < L; t += 32) s += (double)dt[(row * L + t) * H + h];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) out[u] = (float)exp((double)A[h] * s);
}

// out = h0 (or 0) carried through ranks 0..r-1: H <- D_k H + S_k, elementwise
// over (b, H, P, N); float4 where the state size allows
__global__ void __launch_bounds__(256) k_state_fold(const float* __restrict__ S, const float* __restrict__ Dk,
                                                    const float* __restrict__ h0, float* __restrict__ out,
                                                    int64_t r, int64_t nstate, int64_t per_head,
                                                    int64_t units) {
  const int64_t i4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // index of a float4
  if (4 * i4 >= nstate) return;
  const int64_t u = (4 * i4) / per_head;  // (row, head); per_head is a multiple of 4
  float4 v = h0 ? reinterpret_cast<const float4*>(h0)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t k = 0; k < r; ++k) {
    const float d = Dk[k * units + u];
    const float4 s = reinterpret_cast<const float4*>(S + k * nstate)[i4];
    v = make_float4(fmaf(d, v.x, s.x), fmaf(d, v.y, s.y), fmaf(d, v.z, s.z), fmaf(d, v.w, s.w));
  }
  reinterpret_cast<float4*>(out)[i4] = v;
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

}  // namespace
}  // namespace ssd

extern "C" SSD_API ssd_status ssd_total_decay(const float* dt, const float* A, float* out, int64_t batch,
                                              int64_t seqlen, int64_t nheads, void* stream) {
  if (!dt || !A || !out || batch <= 0 || seqlen <= 0 || nheads <= 0) return SSD_ERR_INVALID_ARG;
  const int64_t units = batch * nheads;
  if ((units + 7) / 8 >= ((int64_t)1 << 31)) return SSD_ERR_UNSUPPORTED;
  ssd::k_total_decay<<<(unsigned)((units + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      dt, A, out, batch, seqlen, nheads);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" SSD_API ssd_status ssd_state_fold(const float* states, const float* decays, const float* initial_states,
                                             float* out, int64_t rank, int64_t batch, int64_t nheads,
                                             int64_t headdim, int64_t dstate, void* stream) {
  if (!out || rank < 0 || batch <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0) return SSD_ERR_INVALID_ARG;
  if (rank > 0 && (!states || !decays)) return SSD_ERR_INVALID_ARG;
  if ((headdim * dstate) % 4 != 0) return SSD_ERR_UNSUPPORTED;
  if (!ssd::aligned16(out) || (states && !ssd::aligned16(states)) ||
      (initial_states && !ssd::aligned16(initial_states)))
    return SSD_ERR_INVALID_ARG;
  const int64_t per_head = headdim * dstate, units = batch * nheads, nstate = units * per_head;
  const int64_t blocks = (nstate / 4 + 255) / 256;
  if (blocks >= ((int64_t)1 << 31)) return SSD_ERR_UNSUPPORTED;
  ssd::k_state_fold<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      states, decays, initial_states, out, rank, nstate, per_head, units);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
