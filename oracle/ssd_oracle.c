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
 * Backward pass: the adjoint of the recurrence above (the pages give no
 * gradient formulas; they are derived in oracle/backward.py, whose numpy code
 * this follows token by token).  Per (b, h) unit, with G_t = dLoss/dh_t:
 *   G_t  = dy_t (outer) C_t + a_{t+1} G_{t+1}      (G_{L-1} also gets dfinal)
 *   dx_t = dt_t G_t B_t + D dy_t
 *   dB_t = dt_t G_t^T x_t,  dC_t = h_t^T dy_t       (per head; summed over the group later)
 *   ddt_t = <G_t, x_t B_t^T> + A a_t <G_t, h_{t-1}>,  dA = sum_t dt_t a_t <G_t, h_{t-1}>
 *   dD = sum_t <dy_t, x_t>,  dh0 = a_0 G_0
 * The states are recomputed: a forward sweep keeps the state before every
 * 64-token block, and the backward sweep rebuilds each block's states from it.
 */
static double step_decay(int64_t tok, int64_t t, int64_t H, int64_t h, const float* dt, double rate,
                         const int32_t* seq_idx) {
  if (seq_idx && t > 0 && seq_idx[tok] != seq_idx[tok - 1]) return 0.0;  /* packed reset */
  return exp((double)dt[tok * H + h] * rate);
}

static void oracle_bwd_unit(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                            const float* x, const float* dt, const float* A, const float* Bm, const float* Cm,
                            const float* D, const float* h0, const int32_t* seq_idx, const float* dy,
                            const float* dfinal, double* dx, double* ddt, double* dA_unit, double* dBh,
                            double* dCh, double* dD_unit, double* dh0, double* ckpt, double* blk, double* Gs,
                            double* dA_abs_unit, double* dD_abs_unit) {
  const int64_t g = h / (H / G), PN = P * N, nb = (L + 63) / 64;
  const double rate = (double)A[h];
  const double skip = D ? (double)D[h] : 0.0;
  /* forward sweep: ckpt[k] = the state before token 64 k */
  double* st = blk; /* scratch for the running state */
  if (h0) {
    for (int64_t i = 0; i < PN; ++i) st[i] = (double)h0[(b * H + h) * PN + i];
  } else {
    memset(st, 0, sizeof(double) * (size_t)PN);
  }
  for (int64_t t = 0; t < L; ++t) {
    const int64_t tok = b * L + t;
    if (t % 64 == 0) memcpy(ckpt + (t / 64) * PN, st, sizeof(double) * (size_t)PN);
    const double decay = step_decay(tok, t, H, h, dt, rate, seq_idx);
    const double step = (double)dt[tok * H + h];
    for (int64_t p = 0; p < P; ++p) {
      const double in = step * (double)x[(tok * H + h) * P + p];
      for (int64_t n = 0; n < N; ++n)
        st[p * N + n] = decay * st[p * N + n] + in * (double)Bm[(tok * G + g) * N + n];
    }
  }
  /* backward sweep */
  if (dfinal) {
    for (int64_t i = 0; i < PN; ++i) Gs[i] = (double)dfinal[(b * H + h) * PN + i];
  } else {
    memset(Gs, 0, sizeof(double) * (size_t)PN);
  }
  double dA_acc = 0.0, dD_acc = 0.0, dA_abs = 0.0, dD_abs = 0.0;
  for (int64_t k = nb - 1; k >= 0; --k) {
    const int64_t t0 = 64 * k, t1 = (t0 + 64 < L) ? t0 + 64 : L;
    /* rebuild the block's states: blk[j] = h_{t0 + j}; the state before t0 is ckpt[k] */
    for (int64_t t = t0; t < t1; ++t) {
      const int64_t tok = b * L + t;
      const double* prev = (t == t0) ? ckpt + k * PN : blk + (t - t0 - 1) * PN;
      double* cur = blk + (t - t0) * PN;
      const double decay = step_decay(tok, t, H, h, dt, rate, seq_idx);
      const double step = (double)dt[tok * H + h];
      for (int64_t p = 0; p < P; ++p) {
        const double in = step * (double)x[(tok * H + h) * P + p];
        for (int64_t n = 0; n < N; ++n) cur[p * N + n] = decay * prev[p * N + n] + in * (double)Bm[(tok * G + g) * N + n];
      }
    }
    for (int64_t t = t1 - 1; t >= t0; --t) {
      const int64_t tok = b * L + t;
      if (t < L - 1) {
        const double next = step_decay(tok + 1, t + 1, H, h, dt, rate, seq_idx);
        for (int64_t i = 0; i < PN; ++i) Gs[i] *= next;
      }
      const float* xt = x + (tok * H + h) * P;
      const float* dyt = dy + (tok * H + h) * P;
      const float* Bt = Bm + (tok * G + g) * N;
      const float* Ct = Cm + (tok * G + g) * N;
      for (int64_t p = 0; p < P; ++p)
        for (int64_t n = 0; n < N; ++n) Gs[p * N + n] += (double)dyt[p] * (double)Ct[n];
      const double* hcur = blk + (t - t0) * PN;
      const double* hprev = (t == t0) ? ckpt + k * PN : blk + (t - t0 - 1) * PN;
      const double step = (double)dt[tok * H + h];
      const double decay = step_decay(tok, t, H, h, dt, rate, seq_idx);
      double g_in = 0.0, g_dec = 0.0;
      for (int64_t p = 0; p < P; ++p) {
        double gb = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          gb += Gs[p * N + n] * (double)Bt[n];
          g_dec += Gs[p * N + n] * hprev[p * N + n];
        }
        dx[(tok * H + h) * P + p] = step * gb + skip * (double)dyt[p];
        g_in += gb * (double)xt[p];
        dD_acc += (double)dyt[p] * (double)xt[p];
        dD_abs += fabs((double)dyt[p] * (double)xt[p]);
      }
      for (int64_t n = 0; n < N; ++n) {
        double gx = 0.0, hy = 0.0;
        for (int64_t p = 0; p < P; ++p) {
          gx += Gs[p * N + n] * (double)xt[p];
          hy += hcur[p * N + n] * (double)dyt[p];
        }
        dBh[(tok * H + h) * N + n] = step * gx;
        dCh[(tok * H + h) * N + n] = hy;
      }
      ddt[tok * H + h] = g_in + rate * decay * g_dec;
      dA_acc += step * decay * g_dec;
      dA_abs += fabs(step * decay * g_dec);
    }
  }
  if (dh0) {
    const double first = step_decay(b * L, 0, H, h, dt, rate, seq_idx);
    for (int64_t i = 0; i < PN; ++i) dh0[(b * H + h) * PN + i] = first * Gs[i];
  }
  *dA_unit = dA_acc;
  *dD_unit = dD_acc;
  if (dA_abs_unit) *dA_abs_unit = dA_abs;
  if (dD_abs_unit) *dD_abs_unit = dD_abs;
}

/*
 * Backward layouts: the forward's inputs, dy (b,L,H,P), dfinal (b,H,P,N) or
 * NULL (not with seq_idx); outputs dx (b,L,H,P), ddt (b,L,H), dBh, dCh
 * (b,L,H,N) per head (the caller sums each group's heads), dA_units and
 * dD_units (b*H) per unit (the caller sums over the batch), dh0 (b,H,P,N) or
 * NULL; dA_abs_units and dD_abs_units (b*H) or NULL: per unit, the sums of
 * the magnitudes of the terms that dA and dD add up (the scale a rounding
 * error in those sums is measured against).  Returns 0, -1 on a bad
 * argument, -2 if memory runs out.
 */
int oracle_ssd_bwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                   int64_t ngroups, const float* x, const float* dt, const float* A, const float* B,
                   const float* C, const float* D, const float* initial_states, const int32_t* seq_idx,
                   const float* dy, const float* dfinal, double* dx, double* ddt, double* dBh, double* dCh,
                   double* dA_units, double* dD_units, double* dh0, int nthreads, double* dA_abs_units,
                   double* dD_abs_units) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0) return -1;
  if (nheads % ngroups != 0 || (seq_idx && dfinal)) return -1;
  if (!x || !dt || !A || !B || !C || !dy || !dx || !ddt || !dBh || !dCh || !dA_units || !dD_units) return -1;
  const int64_t PN = headdim * dstate, nb = (seqlen + 63) / 64;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel
  {
    double* ckpt = (double*)malloc(sizeof(double) * (size_t)(nb * PN));
    double* blk = (double*)malloc(sizeof(double) * (size_t)(64 * PN));
    double* Gs = (double*)malloc(sizeof(double) * (size_t)PN);
    if (!ckpt || !blk || !Gs) {
#pragma omp atomic write
      err = -2;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < batch * nheads; ++u) {
      if (!ckpt || !blk || !Gs) continue;
      oracle_bwd_unit(u / nheads, u % nheads, seqlen, nheads, headdim, dstate, ngroups, x, dt, A, B, C, D,
                      initial_states, seq_idx, dy, dfinal, dx, ddt, dA_units + u, dBh, dCh, dD_units + u,
                      initial_states ? dh0 : NULL, ckpt, blk, Gs, dA_abs_units ? dA_abs_units + u : NULL,
                      dD_abs_units ? dD_abs_units + u : NULL);
    }
    free(ckpt);
    free(blk);
    free(Gs);
  }
  return err;
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
