/*
 * Plain fp64 CPU oracle for the SSD (structured state space duality) forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code with the CUDA library.
 *
 * What it computes, per batch row b and head h (group g = h / (H/G)):
 *
 *   S <- initial_states[b,h]  (P x N; zero when absent)          the state h_{-1}
 *   for t = 0 .. L-1:
 *     a_t = exp(dt[b,t,h] * A[h])                                 decay from step size
 *     a_t = 0 instead, where seq_idx[b,t] != seq_idx[b,t-1]       sequence packing reset
 *     S   = a_t * S + dt[b,t,h] * x[b,t,h,:] (outer) B[b,t,g,:]   scalar-A state update
 *     y[b,t,h,:] = S . C[b,t,g,:] + D[h] * x[b,t,h,:]             read-out plus skip
 *   final state = S after the last token (per sequence when packed)
 *
 * Sources (web pages on Mamba-2 / SSD, cited by title and section):
 *  - "22 · Mamba 2 — Transformers are SSMs" (paper story), section 3.1, scalar
 *    A: h_t = a_t h_{t-1} + Delta_t B_t x_t and y_t = C_t^T h_t.
 *  - "SSM 家族全景图（下）：Mamba-2 与 Jamba", closing question on decay: the
 *    transition is a_t = exp(Delta_t A).
 *  - "从Transformer的二次复杂度困境到Mamba的线性突围", continuous-time SSM
 *    equations: the D x(t) feed-through, here one scalar D per head.
 *  - "Transformers与SSMs的隐藏联系", section 4.2 (variable length): packed
 *    sequences are cut apart by setting the transition to zero at each
 *    boundary.  Read as a_t = 0 at the first token of a new sequence; that
 *    token's own input term is kept.
 *
 * Inputs are fp32 arrays (bf16 inputs arrive already widened; both are exact
 * in fp32) and are upcast to double element by element.  Every accumulation is
 * in double, in the plain token order above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One (b, h) unit: the sequential recurrence over all L tokens. */
static void oracle_unit(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                        const float* x, const float* dt, const float* A, const float* Bm,
                        const float* Cm, const float* D, const float* h0, const int32_t* seq_idx,
                        int64_t num_seqs, double* y, double* final_states, double* S) {
  const int64_t g = h / (H / G);
  const double a_log = (double)A[h];
  const double d_skip = D ? (double)D[h] : 0.0;
  if (h0) {
    const float* src = h0 + ((b * H + h) * P) * N;
    for (int64_t i = 0; i < P * N; ++i) S[i] = (double)src[i];
  } else {
    memset(S, 0, sizeof(double) * (size_t)(P * N));
  }
  for (int64_t t = 0; t < L; ++t) {
    const int64_t tok = b * L + t;
    const double dtv = (double)dt[tok * H + h];
    double a = exp(dtv * a_log);
    if (seq_idx && t > 0 && seq_idx[tok] != seq_idx[tok - 1]) a = 0.0;
    const float* xt = x + (tok * H + h) * P;
    const float* Bt = Bm + (tok * G + g) * N;
    const float* Ct = Cm + (tok * G + g) * N;
    double* yt = y + (tok * H + h) * P;
    for (int64_t p = 0; p < P; ++p) {
      const double u = dtv * (double)xt[p];
      double* Sp = S + p * N;
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        Sp[n] = a * Sp[n] + u * (double)Bt[n];
        acc += Sp[n] * (double)Ct[n];
      }
      yt[p] = acc + d_skip * (double)xt[p];
    }
    if (seq_idx && final_states) {
      const int last = (t == L - 1) || (seq_idx[tok + 1] != seq_idx[tok]);
      const int64_t sid = seq_idx[tok];
      if (last && sid >= 0 && sid < num_seqs) {
        double* dst = final_states + ((sid * H + h) * P) * N;
        memcpy(dst, S, sizeof(double) * (size_t)(P * N));
      }
    }
  }
  if (!seq_idx && final_states) {
    double* dst = final_states + ((b * H + h) * P) * N;
    memcpy(dst, S, sizeof(double) * (size_t)(P * N));
  }
}

/*
 * Layouts (all contiguous, row-major):
 *   x (b,L,H,P)  dt (b,L,H)  A (H)  B, C (b,L,G,N)  D (H) or NULL
 *   initial_states (b,H,P,N) or NULL   seq_idx (b,L) or NULL
 *   y (b,L,H,P) double                 final_states (b,H,P,N) or (num_seqs,H,P,N) double, or NULL
 * units: optional list of flattened (b*H + h) units to compute (others are not
 * touched); NULL computes all b*H units.  nthreads <= 0 uses the OpenMP default.
 * Returns 0 on success, -1 on a bad argument, -2 if memory runs out.
 */
int oracle_ssd_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                   int64_t ngroups, const float* x, const float* dt, const float* A, const float* B,
                   const float* C, const float* D, const float* initial_states,
                   const int32_t* seq_idx, int64_t num_seqs, double* y, double* final_states,
                   const int64_t* units, int64_t n_units, int nthreads) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
    return -1;
  if (nheads % ngroups != 0) return -1;
  if (!x || !dt || !A || !B || !C || !y) return -1;
  const int64_t total = units ? n_units : batch * nheads;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * (size_t)(headdim * dstate));
    if (!S) {
#pragma omp atomic write
      err = -2;
    }
    /* every thread reaches the worksharing loop; one without scratch skips */
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < total; ++i) {
      const int64_t u = units ? units[i] : i;
      if (!S || u < 0 || u >= batch * nheads) continue;
      oracle_unit(u / nheads, u % nheads, seqlen, nheads, headdim, dstate, ngroups, x, dt, A, B, C,
                  D, initial_states, seq_idx, num_seqs, y, final_states, S);
    }
    free(S);
  }
  return err;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
