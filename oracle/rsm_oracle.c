/*
 * rsm_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, sequential fp64 CPU restatement of the Raven routing-state-model (RSM) mixer.
 * It exists to check the CUDA library; only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg may load it. It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes, per batch b, head h, token t (one token at a time, no chunking):
 *   1. S_t = the K slots with the largest router logits, ordered by (logit desc, slot index asc).
 *      Raven README (github.com/xiaol/SelectingMemory), "How Raven Works": the router keeps the
 *      TopK of sigmoid(r_proj(x)); sigmoid is monotone, so the order is the order of the logits.
 *      paperlayer.ai summary of "Raven: High-Recall Sequence Modeling with Sparse Memory Routing",
 *      section 4.1: only the top-K entries are kept, the rest are zero.
 *   2. s_i = sigmoid(logit_i) for i in S_t (README, "How Raven Works").
 *   3. decay a_i = exp(s_i * f) with f the per-head (Mamba2) or per-slot (GLA) log-decay
 *      (README, "How Raven Works" and "Model Structure": Mamba2 or GLA decay).
 *   4. for i in S_t: H[i,:] = a_i * H[i,:] + (1 - a_i) * k_i * v ; other rows are not touched
 *      (README, "How Raven Works"; "Raven Part 1 -- Memory as a Set of Slots", "Method": a slot
 *      with zero routing is carried over unchanged).
 *   5. o_t = sum_i q_i * H[i,:], read after the write (README, "How Raven Works").
 *
 * Router variants (rsmo_forward_ex, rsmo_route_ex; the default above is RSMO_SIGMOID):
 *   - softmax scores: s_i = e^{l_i} / sum_{j=1..M} e^{l_j}, over all M slots of the row, in
 *     place of the sigmoid (README, "Model Structure": top-k sigmoid/softmax router; "Usage":
 *     router_score 'sigmoid' or 'softmax'; paperlayer.ai summary, section 6.2.1). The selected
 *     set does not change: softmax, like sigmoid, is monotone in the logit.
 *   - normalised scores: after the TopK cut, s_i = s_i / sum_{j in S_t} s_j, so the selected
 *     weights sum to one (paperlayer.ai summary, section 4.1).
 * Selection counts (rsmo_forward_ex): counts[b,h,i] += number of tokens t with i in S_t, the
 * per-slot count behind the "effective sequence length" analysis (paperlayer.ai summary,
 * section 7.1 and Figure 5: how much each slot processes).
 *
 * Layouts (row-major, contiguous): q, k, logits [B,T,H,M]; v [B,T,H,Dv]; f [B,T,H] (per head)
 * or [B,T,H,M] (per slot); H0, HT [B,H,M,Dv]; o [B,T,H,Dv]; idx, score [B,T,H,K].
 * Inputs are the exact fp32 values the device sees (bf16 inputs are widened exactly beforehand).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Slot a ranks ahead of slot b: larger logit first, the lower index on an exact tie.
 * Comparisons are on the fp32 values (widened to fp64, which preserves order and equality;
 * -0.0 and +0.0 compare equal and fall to the index rule). */
static int rsmo_ahead(const float* row, int a, int b) {
  double xa = (double)row[a], xb = (double)row[b];
  if (xa > xb) return 1;
  if (xa < xb) return 0;
  return a < b;
}

/* TopK by insertion sort of all M slot indices under rsmo_ahead; the first K are kept. */
void rsmo_topk(const float* row, int M, int K, int32_t* idx_out) {
  int* ord = (int*)malloc(sizeof(int) * (size_t)M);
  for (int i = 0; i < M; ++i) {
    int j = i;
    while (j > 0 && rsmo_ahead(row, i, ord[j - 1])) {
      ord[j] = ord[j - 1];
      --j;
    }
    ord[j] = i;
  }
  for (int r = 0; r < K; ++r) idx_out[r] = ord[r];
  free(ord);
}

double rsmo_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

enum { RSMO_SIGMOID = 0, RSMO_SOFTMAX = 1, RSMO_NORMALISE = 2 };

/* Scores of the K selected slots sel[0..K) of one row of M logits, for a router variant. */
void rsmo_scores(const float* row, int M, int K, const int32_t* sel, int router, double* s) {
  if (router & RSMO_SOFTMAX) {
    double mx = (double)row[0];
    for (int j = 1; j < M; ++j)
      if ((double)row[j] > mx) mx = (double)row[j];
    double z = 0.0;
    for (int j = 0; j < M; ++j) z += exp((double)row[j] - mx);
    for (int r = 0; r < K; ++r) s[r] = exp((double)row[sel[r]] - mx) / z;
  } else {
    for (int r = 0; r < K; ++r) s[r] = rsmo_sigmoid((double)row[sel[r]]);
  }
  if (router & RSMO_NORMALISE) {
    double sum = 0.0;
    for (int r = 0; r < K; ++r) sum += s[r];
    for (int r = 0; r < K; ++r) s[r] /= sum;
  }
}

typedef struct {
  int B, T, H, M, K, Dv, per_slot;
  const float *q, *k, *v, *logits, *f;
  const double* H0;
  double *o, *HT;
  int32_t* idx;
  double* score;
  int router;
  int32_t* counts;
  int pair_begin, pair_end; /* range of flattened (b,h) pairs handled by one worker */
} rsmo_job;

/* One (b,h) pair, all T tokens, strictly in order. */
static void rsmo_run_pair(const rsmo_job* J, int pair) {
  const int b = pair / J->H, h = pair % J->H;
  const int M = J->M, K = J->K, Dv = J->Dv, H = J->H, T = J->T;
  double* S = (double*)malloc(sizeof(double) * (size_t)M * (size_t)Dv);
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
  double* sc = (double*)malloc(sizeof(double) * (size_t)K);
  if (J->H0)
    memcpy(S, J->H0 + (size_t)pair * M * Dv, sizeof(double) * (size_t)M * Dv);
  else
    memset(S, 0, sizeof(double) * (size_t)M * Dv);

  for (int t = 0; t < T; ++t) {
    const size_t row = ((size_t)b * T + t) * H + h; /* flattened (b,t,h) */
    const float* q = J->q + row * M;
    const float* k = J->k + row * M;
    const float* lg = J->logits + row * M;
    const float* v = J->v + row * Dv;
    rsmo_topk(lg, M, K, sel);
    rsmo_scores(lg, M, K, sel, J->router, sc);
    for (int r = 0; r < K; ++r) {
      const int i = sel[r];
      const double s = sc[r];
      if (J->counts) J->counts[(size_t)pair * M + i] += 1;
      const double f = J->per_slot ? (double)J->f[row * M + i] : (double)J->f[row];
      const double a = exp(s * f);
      const double wk = (1.0 - a) * (double)k[i];
      double* Si = S + (size_t)i * Dv;
      for (int d = 0; d < Dv; ++d) Si[d] = a * Si[d] + wk * (double)v[d];
      if (J->idx) J->idx[row * K + r] = i;
      if (J->score) J->score[row * K + r] = s;
    }
    if (J->o) {
      double* o = J->o + row * Dv;
      for (int d = 0; d < Dv; ++d) o[d] = 0.0;
      for (int i = 0; i < M; ++i) {
        const double qi = (double)q[i];
        const double* Si = S + (size_t)i * Dv;
        for (int d = 0; d < Dv; ++d) o[d] += qi * Si[d];
      }
    }
  }
  if (J->HT) memcpy(J->HT + (size_t)pair * M * Dv, S, sizeof(double) * (size_t)M * Dv);
  free(sc);
  free(sel);
  free(S);
}

static void* rsmo_worker(void* arg) {
  const rsmo_job* J = (const rsmo_job*)arg;
  for (int p = J->pair_begin; p < J->pair_end; ++p) rsmo_run_pair(J, p);
  return NULL;
}

/* Runs the recurrence over all (b,h) pairs; pairs are independent, so they are split over
 * nthreads POSIX threads (nthreads <= 1 runs inline). `router` is a combination of RSMO_SOFTMAX
 * and RSMO_NORMALISE (0: sigmoid scores); `counts` [B,H,M] (or NULL) is added to.
 * Returns 0 on success, -1 on bad sizes. */
int rsmo_forward_ex(int B, int T, int H, int M, int K, int Dv, int per_slot,
                    const float* q, const float* k, const float* v, const float* logits,
                    const float* f, const double* H0, double* o, double* HT, int32_t* idx,
                    double* score, int router, int32_t* counts, int nthreads) {
  if (B < 0 || T < 0 || H < 0 || M < 1 || K < 1 || K > M || Dv < 1 || router < 0 || router > 3) return -1;
  const int pairs = B * H;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > pairs) nthreads = pairs > 0 ? pairs : 1;
  rsmo_job base = {B, T, H, M, K, Dv, per_slot, q, k, v, logits, f, H0, o, HT, idx, score, router, counts,
                   0, pairs};
  if (nthreads == 1) {
    rsmo_worker(&base);
    return 0;
  }
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  rsmo_job* jobs = (rsmo_job*)malloc(sizeof(rsmo_job) * (size_t)nthreads);
  for (int w = 0; w < nthreads; ++w) {
    jobs[w] = base;
    jobs[w].pair_begin = (int)((long long)pairs * w / nthreads);
    jobs[w].pair_end = (int)((long long)pairs * (w + 1) / nthreads);
    pthread_create(&th[w], NULL, rsmo_worker, &jobs[w]);
  }
  for (int w = 0; w < nthreads; ++w) pthread_join(th[w], NULL);
  free(jobs);
  free(th);
  return 0;
}

/* The default router (sigmoid scores, not normalised), no counts. */
int rsmo_forward(int B, int T, int H, int M, int K, int Dv, int per_slot,
                 const float* q, const float* k, const float* v, const float* logits,
                 const float* f, const double* H0, double* o, double* HT, int32_t* idx,
                 double* score, int nthreads) {
  return rsmo_forward_ex(B, T, H, M, K, Dv, per_slot, q, k, v, logits, f, H0, o, HT, idx, score,
                         RSMO_SIGMOID, NULL, nthreads);
}

/* One generation step: the same update and read for a single token per (b,h), applied in
 * place to the carried state (README, "Model Structure": fused recurrent computation for
 * inference). Layouts: q, k, logits [B,H,M]; v [B,H,Dv]; f [B,H] or [B,H,M];
 * state [B,H,M,Dv] (in/out); o [B,H,Dv]; idx, score [B,H,K]. */
int rsmo_decode_step(int B, int H, int M, int K, int Dv, int per_slot, const float* q,
                     const float* k, const float* v, const float* logits, const float* f,
                     double* state, double* o, int32_t* idx, double* score, int nthreads) {
  /* A step is the T = 1 case of the recurrence with the carried state as both H0 and HT. */
  return rsmo_forward(B, 1, H, M, K, Dv, per_slot, q, k, v, logits, f, state, o, state, idx,
                      score, nthreads);
}

/* ---------------------------------------------------------------------------------------------
 * Gradients of the recurrence (sigmoid router), by reverse-mode differentiation of the forward
 * above taken one token at a time. With G = dL/dH (M x Dv), per token t from the last to the
 * first, selected slots i in S_t, a_i = exp(s_i f), w_i = (1 - a_i) k_i:
 *   read o_t = sum_i q_i H_t[i]:      dq_t[i] = do_t . H_t[i];  G[i] += q_i do_t  (every slot)
 *   write H_t[i] = a_i H_{t-1}[i] + w_i v_t (i in S_t):
 *       dv_t += w_i G[i];  dw_i = G[i] . v_t;  da_i = G[i] . H_{t-1}[i] - k_i dw_i;
 *       dk_{t,i} = (1 - a_i) dw_i;  dlam_i = a_i da_i  (a = e^lam, lam = s f);
 *       df += s_i dlam_i (per head; per slot: df_i = s_i dlam_i);  ds_i = f dlam_i;
 *       dlogit_i = s_i (1 - s_i) ds_i;  then G[i] = a_i G[i]
 *   unselected slots: G[i] passes unchanged; their dk and dlogit are 0 (the TopK cut is
 *   piecewise constant in the logits).
 *   dH0 = G after the first token. H_{t-1} is recovered from H_t by putting back the rows the
 *   token overwrote, kept from a forward sweep ("tape").
 * Inputs as rsmo_forward plus dO [B,T,H,Dv] and dHT [B,H,M,Dv] (NULL = 0); outputs (each may be
 * NULL): dq, dk, dlogits [B,T,H,M]; dv [B,T,H,Dv]; df [B,T,H] or [B,T,H,M]; dH0 [B,H,M,Dv].
 * ------------------------------------------------------------------------------------------- */
typedef struct {
  int B, T, H, M, K, Dv, per_slot;
  const float *q, *k, *v, *logits, *f;
  const double *H0, *dO, *dHT;
  double *dq, *dk, *dv, *dlogits, *df, *dH0;
  int pair_begin, pair_end;
} rsmo_bjob;

static void rsmo_backward_pair(const rsmo_bjob* J, int pair) {
  const int b = pair / J->H, h = pair % J->H;
  const int M = J->M, K = J->K, Dv = J->Dv, H = J->H, T = J->T;
  double* S = (double*)malloc(sizeof(double) * (size_t)M * Dv);
  double* G = (double*)malloc(sizeof(double) * (size_t)M * Dv);
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)T * K);
  double* tape = (double*)malloc(sizeof(double) * (size_t)T * K * Dv); /* H_{t-1} of the rows t overwrote */
  double* sc = (double*)malloc(sizeof(double) * (size_t)K);
  if (J->H0)
    memcpy(S, J->H0 + (size_t)pair * M * Dv, sizeof(double) * (size_t)M * Dv);
  else
    memset(S, 0, sizeof(double) * (size_t)M * Dv);
  /* forward sweep, keeping the overwritten rows */
  for (int t = 0; t < T; ++t) {
    const size_t row = ((size_t)b * T + t) * H + h;
    const float* k = J->k + row * M;
    const float* lg = J->logits + row * M;
    const float* v = J->v + row * Dv;
    int32_t* st = sel + (size_t)t * K;
    rsmo_topk(lg, M, K, st);
    rsmo_scores(lg, M, K, st, 0, sc);
    for (int r = 0; r < K; ++r) {
      const int i = st[r];
      const double f = J->per_slot ? (double)J->f[row * M + i] : (double)J->f[row];
      const double a = exp(sc[r] * f);
      const double wk = (1.0 - a) * (double)k[i];
      double* Si = S + (size_t)i * Dv;
      memcpy(tape + ((size_t)t * K + r) * Dv, Si, sizeof(double) * (size_t)Dv);
      for (int d = 0; d < Dv; ++d) Si[d] = a * Si[d] + wk * (double)v[d];
    }
  }
  /* reverse sweep */
  if (J->dHT)
    memcpy(G, J->dHT + (size_t)pair * M * Dv, sizeof(double) * (size_t)M * Dv);
  else
    memset(G, 0, sizeof(double) * (size_t)M * Dv);
  for (int t = T - 1; t >= 0; --t) {
    const size_t row = ((size_t)b * T + t) * H + h;
    const float* q = J->q + row * M;
    const float* k = J->k + row * M;
    const float* lg = J->logits + row * M;
    const float* v = J->v + row * Dv;
    const double* dO = J->dO ? J->dO + row * Dv : NULL;
    const int32_t* st = sel + (size_t)t * K;
    for (int i = 0; i < M; ++i) {
      double* Gi = G + (size_t)i * Dv;
      const double* Si = S + (size_t)i * Dv;
      double dqi = 0.0;
      if (dO)
        for (int d = 0; d < Dv; ++d) {
          dqi += dO[d] * Si[d];
          Gi[d] += (double)q[i] * dO[d];
        }
      if (J->dq) J->dq[row * M + i] = dqi;
      if (J->dk) J->dk[row * M + i] = 0.0;
      if (J->dlogits) J->dlogits[row * M + i] = 0.0;
      if (J->df && J->per_slot) J->df[row * M + i] = 0.0;
    }
    if (J->dv)
      for (int d = 0; d < Dv; ++d) J->dv[row * Dv + d] = 0.0;
    double dfh = 0.0;
    rsmo_scores(lg, M, K, st, 0, sc);
    for (int r = 0; r < K; ++r) {
      const int i = st[r];
      const double s = sc[r];
      const double f = J->per_slot ? (double)J->f[row * M + i] : (double)J->f[row];
      const double a = exp(s * f);
      const double wk = (1.0 - a) * (double)k[i];
      double* Gi = G + (size_t)i * Dv;
      double* Si = S + (size_t)i * Dv;
      const double* prev = tape + ((size_t)t * K + r) * Dv;
      double dw = 0.0, dap = 0.0;
      for (int d = 0; d < Dv; ++d) {
        dw += Gi[d] * (double)v[d];
        dap += Gi[d] * prev[d];
        if (J->dv) J->dv[row * Dv + d] += wk * Gi[d];
      }
      const double da = dap - (double)k[i] * dw;
      const double dlam = a * da;
      if (J->dk) J->dk[row * M + i] = (1.0 - a) * dw;
      if (J->df) {
        if (J->per_slot) J->df[row * M + i] = s * dlam;
        else dfh += s * dlam;
      }
      if (J->dlogits) J->dlogits[row * M + i] = s * (1.0 - s) * (f * dlam);
      for (int d = 0; d < Dv; ++d) {
        Gi[d] *= a;
        Si[d] = prev[d];
      }
    }
    if (J->df && !J->per_slot) J->df[row] = dfh;
  }
  if (J->dH0) memcpy(J->dH0 + (size_t)pair * M * Dv, G, sizeof(double) * (size_t)M * Dv);
  free(sc);
  free(tape);
  free(sel);
  free(G);
  free(S);
}

static void* rsmo_bworker(void* arg) {
  const rsmo_bjob* J = (const rsmo_bjob*)arg;
  for (int p = J->pair_begin; p < J->pair_end; ++p) rsmo_backward_pair(J, p);
  return NULL;
}

int rsmo_backward(int B, int T, int H, int M, int K, int Dv, int per_slot, const float* q,
                  const float* k, const float* v, const float* logits, const float* f,
                  const double* H0, const double* dO, const double* dHT, double* dq, double* dk,
                  double* dv, double* dlogits, double* df, double* dH0, int nthreads) {
  if (B < 0 || T < 0 || H < 0 || M < 1 || K < 1 || K > M || Dv < 1) return -1;
  const int pairs = B * H;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > pairs) nthreads = pairs > 0 ? pairs : 1;
  rsmo_bjob base = {B, T, H, M, K, Dv, per_slot, q, k, v, logits, f, H0, dO, dHT,
                    dq, dk, dv, dlogits, df, dH0, 0, pairs};
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  rsmo_bjob* jobs = (rsmo_bjob*)malloc(sizeof(rsmo_bjob) * (size_t)nthreads);
  for (int w = 0; w < nthreads; ++w) {
    jobs[w] = base;
    jobs[w].pair_begin = (int)((long long)pairs * w / nthreads);
    jobs[w].pair_end = (int)((long long)pairs * (w + 1) / nthreads);
    if (nthreads == 1) rsmo_bworker(&jobs[w]);
    else pthread_create(&th[w], NULL, rsmo_bworker, &jobs[w]);
  }
  if (nthreads > 1)
    for (int w = 0; w < nthreads; ++w) pthread_join(th[w], NULL);
  free(jobs);
  free(th);
  return 0;
}

/* Standalone routing: TopK indices (rank order) and the router variant's scores, rows [rows, M]. */
int rsmo_route_ex(const float* logits, long long rows, int M, int K, int router, int32_t* idx,
                  double* score) {
  if (rows < 0 || M < 1 || K < 1 || K > M || router < 0 || router > 3) return -1;
  for (long long r = 0; r < rows; ++r) {
    const float* lg = logits + r * M;
    rsmo_topk(lg, M, K, idx + r * K);
    rsmo_scores(lg, M, K, idx + r * K, router, score + r * K);
  }
  return 0;
}

/* Standalone routing with sigmoid scores. */
int rsmo_route(const float* logits, long long rows, int M, int K, int32_t* idx, double* score) {
  return rsmo_route_ex(logits, rows, M, K, RSMO_SIGMOID, idx, score);
}
