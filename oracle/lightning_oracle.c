/*
 * lightning_oracle.c -- plain float64 CPU oracle for Lightning Attention.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke entry point and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.  Inputs are the exact values the GPU sees (bf16 bit patterns or
 * fp32 values, upcast losslessly to double); all arithmetic is double.
 *
 * What it computes, for each (b, h) independently (layout [B][H][N][*]):
 *
 *     o_t = sum_{s <= t} exp(-lambda_h * (t - s)) * (q_t . k_s) * v_s
 *
 * Sources: "MiniMax-M1" model entry (archdb), linear/SSM layer configuration
 * field (per-head exponential decay, ALiBi-style slopes, 128x128 state per
 * head) and positional-scheme field (fixed per-head decay, no RoPE);
 * "MiniMax-01" (redeep.blog), "What Makes 1M Context Hard" (linear-complexity
 * variant of attention).  lambda_h is read as a decay rate, gamma = exp(-lambda)
 * as the per-step factor; the sum includes s = t; there is no normaliser.
 *
 * Forms (each a plain restatement, no blocking or reordering beyond the form):
 *   la_oracle_masked     O(N^2 (D+E)) masked sum, the definition itself.
 *   la_oracle_recurrent  O(N D E) recurrence  S_t = gamma S_{t-1} + k_t^T v_t,
 *                        o_t = q_t S_t, optionally from an initial state and
 *                        returning the final state.
 *   la_oracle_blocked    the same sum split into blocks of `blk` tokens: an
 *                        intra-block masked term, an inter-block term through
 *                        the state, and the state carry between blocks.
 *   la_oracle_recurrent_sampled  the recurrence, emitting o_t only at the
 *                        given positions (for sequences too long to store).
 *   la_oracle_decode_step one recurrent step on a given state, in place.
 *
 * Reverse time and gradients (for the backward pass of training; the pages
 * train with 1M-token contexts, abstract and "MiniMax-01" blog):
 *   la_oracle_masked_anticausal / la_oracle_recurrent_anticausal
 *        o_t = sum_{s >= t} exp(-lambda (s - t)) (q_t . k_s) v_s, the same sum
 *        with time reversed (definition, and the recurrence run from t = N-1
 *        down: S_t = gamma S_{t+1} + k_t^T v_t, o_t = q_t S_t).
 *   la_oracle_backward_masked / la_oracle_backward_recurrent
 *        the gradients of L = sum_t dout_t . o_t:
 *          dq_t = sum_{s <= t} g^(t-s) (dout_t . v_s) k_s
 *          dk_s = sum_{t >= s} g^(t-s) (dout_t . v_s) q_t
 *          dv_s = sum_{t >= s} g^(t-s) (q_t . k_s) dout_t      (g = gamma)
 *        (the derivative of the masked sum written out term by term, and the
 *        same sums as recurrences: forward for dq, backward in time for dk, dv).
 *
 * The layer around the operator ("MiniMax-M1" model entry, linear-layer field:
 * SiLU on Q, K, V; RMSNorm on the output; sigmoid gate on the output after the
 * RMSNorm, before the output projection):
 *   la_oracle_fused_layer
 *        y_t = w * RMSNorm(o_t) * sigmoid(g_t), o = the recurrence on
 *        (silu(q), silu(k), silu(v)), RMSNorm over each head's E outputs:
 *        RMSNorm(o_t) = o_t / sqrt(mean_e(o_te^2) + eps); w per channel
 *        (h * E + e); silu(x) = x / (1 + exp(-x)); sigmoid(x) = 1/(1+exp(-x)).
 *        Optionally from an initial state S_0 (nullable, [B][H][D][E]) and
 *        returning the state after the last token (nullable): the layer's
 *        fixed-size recurrent state (same entry, the count of layers with a
 *        fixed-size recurrent state), so that a sequence can continue token by
 *        token (N = 1 is one decode step of the layer).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LA_ORACLE_F32 0
#define LA_ORACLE_BF16 1

/* One input element as double.  bf16 is the top half of an IEEE binary32. */
static inline double in_at(const void* p, int64_t i, int dtype) {
  if (dtype == LA_ORACLE_BF16) {
    uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float*)p)[i];
}

/* Copies n consecutive input elements starting at index i0 into dst. */
static void in_row(double* dst, const void* p, int64_t i0, int64_t n, int dtype) {
  for (int64_t x = 0; x < n; ++x) dst[x] = in_at(p, i0 + x, dtype);
}

static int bad_args(const void* q, const void* k, const void* v, const float* slopes,
                    const void* out, int64_t B, int64_t H, int64_t N, int64_t D, int64_t E) {
  if (!q || !k || !v || !slopes || !out) return 1;
  if (B < 1 || H < 1 || N < 0 || D < 1 || E < 1) return 2;
  return 0;
}

/* Threads for one call: nthreads if positive, else the OpenMP default.  Passed
 * to each parallel loop (num_threads), so one call's choice never changes the
 * next call's default. */
static int pick_threads(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

/* Masked sum: the definition, term by term. */
int la_oracle_masked(const void* q, const void* k, const void* v, int dtype,
                     const float* slopes, double* out,
                     int64_t B, int64_t H, int64_t N, int64_t D, int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double lam = (double)slopes[bh % H];
    double* Q = (double*)malloc(sizeof(double) * (size_t)(N * D + 1));
    double* K = (double*)malloc(sizeof(double) * (size_t)(N * D + 1));
    double* V = (double*)malloc(sizeof(double) * (size_t)(N * E + 1));
    in_row(Q, q, bh * N * D, N * D, dtype);
    in_row(K, k, bh * N * D, N * D, dtype);
    in_row(V, v, bh * N * E, N * E, dtype);
    double* O = out + bh * N * E;
    for (int64_t t = 0; t < N; ++t) {
      for (int64_t e = 0; e < E; ++e) O[t * E + e] = 0.0;
      for (int64_t s = 0; s <= t; ++s) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += Q[t * D + d] * K[s * D + d];
        double w = exp(-lam * (double)(t - s)) * dot;
        for (int64_t e = 0; e < E; ++e) O[t * E + e] += w * V[s * E + e];
      }
    }
    free(Q);
    free(K);
    free(V);
  }
  return 0;
}

/*
 * Recurrence S_t = gamma S_{t-1} + k_t^T v_t (S is D x E, row d, column e),
 * o_t = q_t S_t.  s0 (nullable, [B][H][D][E]) is S_{-1}; zero if NULL.
 * s_final (nullable) receives S_{N-1} (or s0 when N == 0).
 */
int la_oracle_recurrent(const void* q, const void* k, const void* v, int dtype,
                        const float* slopes, const double* s0, double* s_final, double* out,
                        int64_t B, int64_t H, int64_t N, int64_t D, int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double gamma = exp(-(double)slopes[bh % H]);
    double* S = (double*)calloc((size_t)(D * E), sizeof(double));
    double* qt = (double*)malloc(sizeof(double) * (size_t)D);
    double* kt = (double*)malloc(sizeof(double) * (size_t)D);
    double* vt = (double*)malloc(sizeof(double) * (size_t)E);
    if (s0) memcpy(S, s0 + bh * D * E, sizeof(double) * (size_t)(D * E));
    double* O = out + bh * N * E;
    for (int64_t t = 0; t < N; ++t) {
      in_row(qt, q, (bh * N + t) * D, D, dtype);
      in_row(kt, k, (bh * N + t) * D, D, dtype);
      in_row(vt, v, (bh * N + t) * E, E, dtype);
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) S[d * E + e] = gamma * S[d * E + e] + kt[d] * vt[e];
      for (int64_t e = 0; e < E; ++e) O[t * E + e] = 0.0;
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) O[t * E + e] += qt[d] * S[d * E + e];
    }
    if (s_final) memcpy(s_final + bh * D * E, S, sizeof(double) * (size_t)(D * E));
    free(S);
    free(qt);
    free(kt);
    free(vt);
  }
  return 0;
}

/*
 * The recurrence, writing o_t only for t in pos[0..npos) (each 0 <= pos < N,
 * any order) into out[B][H][npos][E].  Same arithmetic as la_oracle_recurrent.
 */
int la_oracle_recurrent_sampled(const void* q, const void* k, const void* v, int dtype,
                                const float* slopes, const int64_t* pos, int64_t npos,
                                double* out, int64_t B, int64_t H, int64_t N, int64_t D,
                                int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  if (npos < 0 || (npos > 0 && !pos)) return 1;
  for (int64_t p = 0; p < npos; ++p)
    if (pos[p] < 0 || pos[p] >= N) return 2;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double gamma = exp(-(double)slopes[bh % H]);
    double* S = (double*)calloc((size_t)(D * E), sizeof(double));
    double* qt = (double*)malloc(sizeof(double) * (size_t)D);
    double* kt = (double*)malloc(sizeof(double) * (size_t)D);
    double* vt = (double*)malloc(sizeof(double) * (size_t)E);
    unsigned char* want = (unsigned char*)calloc((size_t)(N + 1), 1);
    for (int64_t p = 0; p < npos; ++p) want[pos[p]] = 1;
    double* O = out + bh * npos * E;
    for (int64_t t = 0; t < N; ++t) {
      in_row(kt, k, (bh * N + t) * D, D, dtype);
      in_row(vt, v, (bh * N + t) * E, E, dtype);
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) S[d * E + e] = gamma * S[d * E + e] + kt[d] * vt[e];
      if (!want[t]) continue;
      in_row(qt, q, (bh * N + t) * D, D, dtype);
      for (int64_t p = 0; p < npos; ++p) {
        if (pos[p] != t) continue;
        for (int64_t e = 0; e < E; ++e) {
          double acc = 0.0;
          for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[d * E + e];
          O[p * E + e] = acc;
        }
      }
    }
    free(S);
    free(qt);
    free(kt);
    free(vt);
    free(want);
  }
  return 0;
}

/*
 * Blocked form with block size blk >= 1.  For the block [t0, t0 + len):
 *   intra:  o_i += sum_{j <= i in block} exp(-lambda (i - j)) (q_i . k_j) v_j
 *   inter:  o_i += exp(-lambda (i - t0 + 1)) q_i S_prev
 *   carry:  S <- exp(-lambda len) S_prev + sum_j exp(-lambda (t0 + len - 1 - j)) k_j^T v_j
 * Mathematically equal to the masked sum for every blk (blk = 1 is the
 * recurrence, blk >= N the masked sum); only rounding differs.
 */
int la_oracle_blocked(const void* q, const void* k, const void* v, int dtype,
                      const float* slopes, int64_t blk, double* out,
                      int64_t B, int64_t H, int64_t N, int64_t D, int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  if (blk < 1) return 2;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double lam = (double)slopes[bh % H];
    double* S = (double*)calloc((size_t)(D * E), sizeof(double));
    double* Snew = (double*)malloc(sizeof(double) * (size_t)(D * E));
    double* Q = (double*)malloc(sizeof(double) * (size_t)(blk * D));
    double* K = (double*)malloc(sizeof(double) * (size_t)(blk * D));
    double* V = (double*)malloc(sizeof(double) * (size_t)(blk * E));
    double* O = out + bh * N * E;
    for (int64_t t0 = 0; t0 < N; t0 += blk) {
      int64_t len = (N - t0 < blk) ? (N - t0) : blk;
      in_row(Q, q, (bh * N + t0) * D, len * D, dtype);
      in_row(K, k, (bh * N + t0) * D, len * D, dtype);
      in_row(V, v, (bh * N + t0) * E, len * E, dtype);
      for (int64_t i = 0; i < len; ++i) {
        double* o = O + (t0 + i) * E;
        double a = exp(-lam * (double)(i + 1));
        for (int64_t e = 0; e < E; ++e) {
          double acc = 0.0;
          for (int64_t d = 0; d < D; ++d) acc += Q[i * D + d] * S[d * E + e];
          o[e] = a * acc;
        }
        for (int64_t j = 0; j <= i; ++j) {
          double dot = 0.0;
          for (int64_t d = 0; d < D; ++d) dot += Q[i * D + d] * K[j * D + d];
          double p = exp(-lam * (double)(i - j)) * dot;
          for (int64_t e = 0; e < E; ++e) o[e] += p * V[j * E + e];
        }
      }
      double decay = exp(-lam * (double)len);
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) Snew[d * E + e] = decay * S[d * E + e];
      for (int64_t j = 0; j < len; ++j) {
        double w = exp(-lam * (double)(len - 1 - j));
        for (int64_t d = 0; d < D; ++d)
          for (int64_t e = 0; e < E; ++e) Snew[d * E + e] += w * K[j * D + d] * V[j * E + e];
      }
      double* tmp = S;
      S = Snew;
      Snew = tmp;
    }
    free(S);
    free(Snew);
    free(Q);
    free(K);
    free(V);
  }
  return 0;
}

/*
 * One recurrent decode step on state [B][H][D][E] (double, in place):
 *   state <- exp(-lambda_h) state + k^T v ;  out = q . state (updated state).
 * q, k are [B][H][D], v is [B][H][E], out is [B][H][E].
 */
int la_oracle_decode_step(const void* q, const void* k, const void* v, int dtype,
                          const float* slopes, double* state, double* out,
                          int64_t B, int64_t H, int64_t D, int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, 1, D, E);
  if (rc) return rc;
  if (!state) return 1;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 16)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double gamma = exp(-(double)slopes[bh % H]);
    double* S = state + bh * D * E;
    double* o = out + bh * E;
    for (int64_t d = 0; d < D; ++d) {
      double kd = in_at(k, bh * D + d, dtype);
      for (int64_t e = 0; e < E; ++e) S[d * E + e] = gamma * S[d * E + e] + kd * in_at(v, bh * E + e, dtype);
    }
    for (int64_t e = 0; e < E; ++e) o[e] = 0.0;
    for (int64_t d = 0; d < D; ++d) {
      double qd = in_at(q, bh * D + d, dtype);
      for (int64_t e = 0; e < E; ++e) o[e] += qd * S[d * E + e];
    }
  }
  return 0;
}

/* Anti-causal masked sum: the definition with time reversed, term by term. */
int la_oracle_masked_anticausal(const void* q, const void* k, const void* v, int dtype,
                                const float* slopes, double* out, int64_t B, int64_t H, int64_t N,
                                int64_t D, int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double lam = (double)slopes[bh % H];
    double* Q = (double*)malloc(sizeof(double) * (size_t)(N * D + 1));
    double* K = (double*)malloc(sizeof(double) * (size_t)(N * D + 1));
    double* V = (double*)malloc(sizeof(double) * (size_t)(N * E + 1));
    in_row(Q, q, bh * N * D, N * D, dtype);
    in_row(K, k, bh * N * D, N * D, dtype);
    in_row(V, v, bh * N * E, N * E, dtype);
    double* O = out + bh * N * E;
    for (int64_t t = 0; t < N; ++t) {
      for (int64_t e = 0; e < E; ++e) O[t * E + e] = 0.0;
      for (int64_t s = t; s < N; ++s) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += Q[t * D + d] * K[s * D + d];
        double w = exp(-lam * (double)(s - t)) * dot;
        for (int64_t e = 0; e < E; ++e) O[t * E + e] += w * V[s * E + e];
      }
    }
    free(Q);
    free(K);
    free(V);
  }
  return 0;
}

/*
 * Anti-causal recurrence S_t = gamma S_{t+1} + k_t^T v_t for t = N-1 .. 0,
 * o_t = q_t S_t.  s0 (nullable) is S_N (zero if NULL); s_final (nullable)
 * receives S_0 (or s0 when N == 0).
 */
int la_oracle_recurrent_anticausal(const void* q, const void* k, const void* v, int dtype,
                                   const float* slopes, const double* s0, double* s_final,
                                   double* out, int64_t B, int64_t H, int64_t N, int64_t D,
                                   int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double gamma = exp(-(double)slopes[bh % H]);
    double* S = (double*)calloc((size_t)(D * E), sizeof(double));
    double* qt = (double*)malloc(sizeof(double) * (size_t)D);
    double* kt = (double*)malloc(sizeof(double) * (size_t)D);
    double* vt = (double*)malloc(sizeof(double) * (size_t)E);
    if (s0) memcpy(S, s0 + bh * D * E, sizeof(double) * (size_t)(D * E));
    double* O = out + bh * N * E;
    for (int64_t t = N - 1; t >= 0; --t) {
      in_row(qt, q, (bh * N + t) * D, D, dtype);
      in_row(kt, k, (bh * N + t) * D, D, dtype);
      in_row(vt, v, (bh * N + t) * E, E, dtype);
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) S[d * E + e] = gamma * S[d * E + e] + kt[d] * vt[e];
      for (int64_t e = 0; e < E; ++e) O[t * E + e] = 0.0;
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) O[t * E + e] += qt[d] * S[d * E + e];
    }
    if (s_final) memcpy(s_final + bh * D * E, S, sizeof(double) * (size_t)(D * E));
    free(S);
    free(qt);
    free(kt);
    free(vt);
  }
  return 0;
}

static int bad_grads(const void* dout, const double* dq, const double* dk, const double* dv) {
  return (!dout || !dq || !dk || !dv) ? 1 : 0;
}

/* Gradients of L = sum_t dout_t . o_t, each sum written out term by term. */
int la_oracle_backward_masked(const void* q, const void* k, const void* v, const void* dout,
                              int dtype, const float* slopes, double* dq, double* dk, double* dv,
                              int64_t B, int64_t H, int64_t N, int64_t D, int64_t E,
                              int nthreads) {
  int rc = bad_args(q, k, v, slopes, dq, B, H, N, D, E);
  if (rc) return rc;
  if (bad_grads(dout, dq, dk, dv)) return 1;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double lam = (double)slopes[bh % H];
    double* Q = (double*)malloc(sizeof(double) * (size_t)(N * D + 1));
    double* K = (double*)malloc(sizeof(double) * (size_t)(N * D + 1));
    double* V = (double*)malloc(sizeof(double) * (size_t)(N * E + 1));
    double* G = (double*)malloc(sizeof(double) * (size_t)(N * E + 1));
    in_row(Q, q, bh * N * D, N * D, dtype);
    in_row(K, k, bh * N * D, N * D, dtype);
    in_row(V, v, bh * N * E, N * E, dtype);
    in_row(G, dout, bh * N * E, N * E, dtype);
    double* dQ = dq + bh * N * D;
    double* dK = dk + bh * N * D;
    double* dV = dv + bh * N * E;
    for (int64_t x = 0; x < N * D; ++x) dQ[x] = dK[x] = 0.0;
    for (int64_t x = 0; x < N * E; ++x) dV[x] = 0.0;
    for (int64_t t = 0; t < N; ++t)
      for (int64_t s = 0; s <= t; ++s) {
        double w = exp(-lam * (double)(t - s));
        double gv = 0.0, qk = 0.0;
        for (int64_t e = 0; e < E; ++e) gv += G[t * E + e] * V[s * E + e];
        for (int64_t d = 0; d < D; ++d) qk += Q[t * D + d] * K[s * D + d];
        for (int64_t d = 0; d < D; ++d) {
          dQ[t * D + d] += w * gv * K[s * D + d];
          dK[s * D + d] += w * gv * Q[t * D + d];
        }
        for (int64_t e = 0; e < E; ++e) dV[s * E + e] += w * qk * G[t * E + e];
      }
    free(Q);
    free(K);
    free(V);
    free(G);
  }
  return 0;
}

/*
 * The same gradients as recurrences (O(N D E)):
 *   T_t = gamma T_{t-1} + v_t^T k_t (E x D),  dq_t = dout_t T_t        (t up)
 *   U_t = gamma U_{t+1} + dout_t^T q_t (E x D), dk_t = v_t U_t         (t down)
 *   W_t = gamma W_{t+1} + q_t^T dout_t (D x E), dv_t = k_t W_t         (t down)
 */
int la_oracle_backward_recurrent(const void* q, const void* k, const void* v, const void* dout,
                                 int dtype, const float* slopes, double* dq, double* dk,
                                 double* dv, int64_t B, int64_t H, int64_t N, int64_t D,
                                 int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, dq, B, H, N, D, E);
  if (rc) return rc;
  if (bad_grads(dout, dq, dk, dv)) return 1;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    double gamma = exp(-(double)slopes[bh % H]);
    double* T = (double*)calloc((size_t)(E * D), sizeof(double));
    double* qt = (double*)malloc(sizeof(double) * (size_t)D);
    double* kt = (double*)malloc(sizeof(double) * (size_t)D);
    double* vt = (double*)malloc(sizeof(double) * (size_t)E);
    double* gt = (double*)malloc(sizeof(double) * (size_t)E);
    double* dQ = dq + bh * N * D;
    double* dK = dk + bh * N * D;
    double* dV = dv + bh * N * E;
    for (int64_t t = 0; t < N; ++t) {  /* dq, forward in time */
      in_row(kt, k, (bh * N + t) * D, D, dtype);
      in_row(vt, v, (bh * N + t) * E, E, dtype);
      in_row(gt, dout, (bh * N + t) * E, E, dtype);
      for (int64_t e = 0; e < E; ++e)
        for (int64_t d = 0; d < D; ++d) T[e * D + d] = gamma * T[e * D + d] + vt[e] * kt[d];
      for (int64_t d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int64_t e = 0; e < E; ++e) acc += gt[e] * T[e * D + d];
        dQ[t * D + d] = acc;
      }
    }
    double* U = T;  /* E x D, reused */
    double* W = (double*)calloc((size_t)(D * E), sizeof(double));
    for (int64_t x = 0; x < E * D; ++x) U[x] = 0.0;
    for (int64_t t = N - 1; t >= 0; --t) {  /* dk, dv, backward in time */
      in_row(qt, q, (bh * N + t) * D, D, dtype);
      in_row(kt, k, (bh * N + t) * D, D, dtype);
      in_row(vt, v, (bh * N + t) * E, E, dtype);
      in_row(gt, dout, (bh * N + t) * E, E, dtype);
      for (int64_t e = 0; e < E; ++e)
        for (int64_t d = 0; d < D; ++d) U[e * D + d] = gamma * U[e * D + d] + gt[e] * qt[d];
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) W[d * E + e] = gamma * W[d * E + e] + qt[d] * gt[e];
      for (int64_t d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int64_t e = 0; e < E; ++e) acc += vt[e] * U[e * D + d];
        dK[t * D + d] = acc;
      }
      for (int64_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += kt[d] * W[d * E + e];
        dV[t * E + e] = acc;
      }
    }
    free(T);
    free(W);
    free(qt);
    free(kt);
    free(vt);
    free(gt);
  }
  return 0;
}

static double silu(double x) { return x / (1.0 + exp(-x)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

int la_oracle_fused_layer(const void* q, const void* k, const void* v, const void* gate, int dtype,
                          const float* slopes, const float* norm_w, double eps, const double* s0,
                          double* sf, double* out, int64_t B, int64_t H, int64_t N, int64_t D,
                          int64_t E, int nthreads) {
  int rc = bad_args(q, k, v, slopes, out, B, H, N, D, E);
  if (rc) return rc;
  if (!gate || !norm_w || !(eps >= 0.0)) return 1;
  const int nt = pick_threads(nthreads);
  int64_t BH = B * H;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    int64_t h = bh % H;
    double gamma = exp(-(double)slopes[h]);
    double* S = (double*)calloc((size_t)(D * E), sizeof(double));
    double* qt = (double*)malloc(sizeof(double) * (size_t)D);
    double* kt = (double*)malloc(sizeof(double) * (size_t)D);
    double* vt = (double*)malloc(sizeof(double) * (size_t)E);
    double* ot = (double*)malloc(sizeof(double) * (size_t)E);
    double* Y = out + bh * N * E;
    if (s0) memcpy(S, s0 + bh * D * E, sizeof(double) * (size_t)(D * E));
    for (int64_t t = 0; t < N; ++t) {
      in_row(qt, q, (bh * N + t) * D, D, dtype);
      in_row(kt, k, (bh * N + t) * D, D, dtype);
      in_row(vt, v, (bh * N + t) * E, E, dtype);
      for (int64_t d = 0; d < D; ++d) {
        qt[d] = silu(qt[d]);
        kt[d] = silu(kt[d]);
      }
      for (int64_t e = 0; e < E; ++e) vt[e] = silu(vt[e]);
      for (int64_t d = 0; d < D; ++d)
        for (int64_t e = 0; e < E; ++e) S[d * E + e] = gamma * S[d * E + e] + kt[d] * vt[e];
      double ms = 0.0;
      for (int64_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[d * E + e];
        ot[e] = acc;
        ms += acc * acc;
      }
      double rinv = 1.0 / sqrt(ms / (double)E + eps);
      for (int64_t e = 0; e < E; ++e) {
        double g = in_at(gate, (bh * N + t) * E + e, dtype);
        Y[t * E + e] = (double)norm_w[h * E + e] * ot[e] * rinv * sigmoid(g);
      }
    }
    if (sf) memcpy(sf + bh * D * E, S, sizeof(double) * (size_t)(D * E));
    free(S);
    free(qt);
    free(kt);
    free(vt);
    free(ot);
  }
  return 0;
}

/* Number of threads an OpenMP parallel region would use (1 without OpenMP). */
int la_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
