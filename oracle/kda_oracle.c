/*
 * KDA oracle: plain, slow, token-by-token CPU reference in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (Kimi Delta Attention, one head, one sequence):
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t
 * with alpha_t = exp(log_alpha_t) a per-key-channel forget gate.  The state S
 * is d_k x d_v.  Sources:
 *   - "Kimi Linear's 75% KV cache cut comes from making three of every four
 *     layers recurrent" (theclarity.today), third paragraph: each step decays
 *     the state per channel, removes the old state's projection onto the
 *     current key, and writes the new key-value pair; each feature channel has
 *     its own decay scalar.
 *   - "Kimi Linear wlasnie pokonal pelna uwage na wlasnych warunkach"
 *     (remio.ai), section "Jak Kimi Linear wykorzystuje inteligentniejsza
 *     pamiec rekurencyjna": the delta rule replaces the stale key-value
 *     association, the gate is finer-grained than Gated DeltaNet's per-head
 *     decay, and the state has a fixed size.
 * The step is evaluated in the order the first page states it:
 *   (1) decay:  S <- Diag(alpha_t) S                 (row c scaled by alpha_tc)
 *   (2) read:   p = S^T k_t                          (old projection onto k_t)
 *   (3) write:  S <- S + beta_t k_t (v_t - p)^T       (remove p, write v_t)
 *   (4) output: o_t = S^T q_t
 * Expanding (1)-(3) gives exactly (I - beta k k^T) Diag(alpha) S + beta k v^T.
 *
 * Padding ("Transformers Community Reports Kimi Linear Cache Bug", ainews,
 * paragraphs on the reproduction and the follow-up investigation): a padded
 * position must not decay or write the recurrent state.  Here a position with
 * pad_mask == 0 is skipped entirely (the state is untouched) and its output
 * is exactly 0, whatever its gate and input values.
 *
 * Inputs are float32 (bf16 and fp32 values are represented exactly); all
 * arithmetic and all outputs are fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One recurrence step on a dk x dv fp64 state (row-major, dv contiguous). */
static void kda_step(int dk, int dv, double *S, const float *q, const float *k,
                     const float *v, const float *log_alpha, double beta,
                     double *o, double *p) {
  int c, j;
  /* (1) per-channel decay */
  for (c = 0; c < dk; ++c) {
    double a = exp((double)log_alpha[c]);
    double *row = S + (size_t)c * dv;
    for (j = 0; j < dv; ++j) row[j] *= a;
  }
  /* (2) p = S^T k */
  for (j = 0; j < dv; ++j) p[j] = 0.0;
  for (c = 0; c < dk; ++c) {
    double kc = (double)k[c];
    const double *row = S + (size_t)c * dv;
    for (j = 0; j < dv; ++j) p[j] += kc * row[j];
  }
  /* (3) delta-rule write: S += beta k (v - p)^T */
  for (j = 0; j < dv; ++j) p[j] = beta * ((double)v[j] - p[j]);
  for (c = 0; c < dk; ++c) {
    double kc = (double)k[c];
    double *row = S + (size_t)c * dv;
    for (j = 0; j < dv; ++j) row[j] += kc * p[j];
  }
  /* (4) o = S^T q */
  for (j = 0; j < dv; ++j) o[j] = 0.0;
  for (c = 0; c < dk; ++c) {
    double qc = (double)q[c];
    const double *row = S + (size_t)c * dv;
    for (j = 0; j < dv; ++j) o[j] += qc * row[j];
  }
}

/*
 * Prefill over a packed batch.
 *   cu_seqlens [num_seqs+1]: sequence b owns packed positions [cu[b], cu[b+1]).
 *   q, k, log_alpha [N,H,dk]; v [N,H,dv]; beta [N,H]   (N = cu[num_seqs])
 *   pad_mask [N] (1 valid, 0 pad) or NULL (all valid)
 *   init_state [B,H,dk,dv] or NULL (zeros)
 *   o [N,H,dv] fp64 out; final_state [B,H,dk,dv] fp64 out (may be NULL)
 * Returns 0, or -1 on an invalid argument.
 */
int kda_oracle_prefill(int num_seqs, const int32_t *cu_seqlens, int H, int dk,
                       int dv, const float *q, const float *k, const float *v,
                       const float *log_alpha, const float *beta,
                       const uint8_t *pad_mask, const float *init_state,
                       double *o, double *final_state, int nthreads) {
  int b;
  if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !o) return -1;
  for (b = 0; b < num_seqs; ++b)
    if (cu_seqlens[b + 1] < cu_seqlens[b]) return -1;
#ifdef _OPENMP
  /* nthreads > 0 limits this call only; the process-wide default is left alone */
  const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
#endif
  for (long w = 0; w < (long)num_seqs * H; ++w) {
    int bb = (int)(w / H), h = (int)(w % H);
    size_t ssz = (size_t)dk * dv;
    double *S = (double *)calloc(ssz, sizeof(double));
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    int t, j;
    if (init_state) {
      const float *s0 = init_state + ((size_t)bb * H + h) * ssz;
      for (size_t e = 0; e < ssz; ++e) S[e] = (double)s0[e];
    }
    for (t = cu_seqlens[bb]; t < cu_seqlens[bb + 1]; ++t) {
      size_t th = (size_t)t * H + h;
      double *ot = o + th * dv;
      if (pad_mask && pad_mask[t] == 0) {
        for (j = 0; j < dv; ++j) ot[j] = 0.0;
        continue;
      }
      kda_step(dk, dv, S, q + th * dk, k + th * dk, v + th * dv,
               log_alpha + th * dk, (double)beta[th], ot, p);
    }
    if (final_state) memcpy(final_state + ((size_t)bb * H + h) * ssz, S, ssz * sizeof(double));
    free(S);
    free(p);
  }
  return 0;
}

/*
 * One decode step for B independent rows: the same step as above applied to
 * one token per (row, head).  state [B,H,dk,dv] fp64 is updated in place.
 * Rows with mask[b] == 0 leave their state untouched and get o = 0.
 */
int kda_oracle_decode(int B, int H, int dk, int dv, const float *q,
                      const float *k, const float *v, const float *log_alpha,
                      const float *beta, const uint8_t *mask, double *state,
                      double *o, int nthreads) {
  if (B < 0 || H <= 0 || dk <= 0 || dv <= 0 || !state || !o) return -1;
#ifdef _OPENMP
  const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nt)
#endif
  for (long w = 0; w < (long)B * H; ++w) {
    int b = (int)(w / H);
    size_t ssz = (size_t)dk * dv;
    double *ot = o + (size_t)w * dv;
    if (mask && mask[b] == 0) {
      for (int j = 0; j < dv; ++j) ot[j] = 0.0;
      continue;
    }
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    kda_step(dk, dv, state + (size_t)w * ssz, q + (size_t)w * dk,
             k + (size_t)w * dk, v + (size_t)w * dv, log_alpha + (size_t)w * dk,
             (double)beta[w], ot, p);
    free(p);
  }
  return 0;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
