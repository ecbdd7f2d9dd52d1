/*
 * nsa_oracle.c -- plain fp64 CPU oracle for Native Sparse Attention (NSA)
 * with mean-pooled compression, as studied in "Sparsity is Cool:
 * Reverse-Engineering MoBA and NSA" and summarised in "DeepSeek's Native
 * Sparse Attention" (section "How Does Native Sparse Attention Work?").
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker of the
 * CUDA library.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it.  The product path never calls it and it
 * shares no code, header or constant with the CUDA sources.
 *
 * Everything is double precision, written as direct loops over the
 * definitions, with no blocking, fusion or reordering beyond them.  OpenMP
 * only splits independent rows (forward) or independent KV groups
 * (backward) across threads; each result is computed by one thread in one
 * fixed order, so results do not depend on the thread count.
 *
 * Layouts (all row-major, contiguous):
 *   q, o_*, out, dq   [B, T, Hq, D]
 *   k, v, dk, dv      [B, T, Hkv, D]
 *   kc, vc            [B, Nc, Hkv, D]      Nc = (T - l) / d + 1 (0 if T < l)
 *   gates, dgates     [B, T, Hq, 3]        branch order (cmp, sel, swa)
 *   lse_*             [B, T, Hq]
 *   score             [B, T, Hkv, Nc]
 *   idx               [B, T, Hkv, topk]    int32, ascending, -1 padded
 * Query head h reads KV head h / (Hq / Hkv).
 *
 * Readings of points the pages leave open (each is applied exactly once,
 * in the function named):
 *   - softmax scale is a parameter (1/sqrt(D) by default)    [all branches]
 *   - compressed block j covers tokens [j*d, j*d + l) and is visible to
 *     query t only when complete: j*d + l - 1 <= t; a query with no
 *     visible block gets output 0, lse -inf, no gradient      [orc_cmp_row]
 *   - compression is the plain mean of the raw rows           [orc_compress]
 *   - block importance = compression softmax probabilities summed over the
 *     query heads of one KV group                              [orc_scores]
 *   - a selection block's importance is the sum of the importances of the
 *     compressed blocks whose tokens overlap it: compressed block i covers
 *     [i*d, i*d + l), selection block j covers [j*l', (j+1)*l'); with
 *     l = d = l' that is compressed block j alone              [orc_topk_row]
 *   - block 0 and the query's own block are always selected and count
 *     toward topk; if a query has at most topk causal blocks it takes all
 *     of them; ties go to the lower block index; the list is ascending and
 *     padded with -1                                           [orc_topk_row]
 *   - keys after the query inside its own block are masked     [orc_sel_row]
 *   - the window holds w keys including the query: [t-w+1, t]  [orc_swa_row]
 *   - gates are post-sigmoid values; out = sum of gate * branch over the
 *     branches enabled by branch_mask                          [orc_combine]
 *   - no gradient flows through the discrete top-k             [backward]
 *   - in a low-precision path the compressed keys/values are stored in that
 *     precision (round-to-nearest-even) before anything reads them, so the
 *     oracle rounds them the same way when asked              [orc_compress]
 *   - likewise the three branch outputs are stored in the path's precision
 *     and the gate gradient dL/dg_i = dO . o_i reads the stored values; the
 *     oracle rounds o_i the same way when asked (the other gradients use
 *     the exact outputs)                                      [orc_backward]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int B, T, Hq, Hkv, D;
  int cmp_block;   /* l  : tokens per compressed block            */
  int cmp_stride;  /* d  : distance between compressed blocks     */
  int sel_block;   /* l' : tokens per selection block             */
  int topk;        /* n  : selection blocks per (query, KV group) */
  int window;      /* w  : sliding-window length                  */
  double scale;    /* softmax scale                               */
  int kv_round;    /* 0 keep fp64, 1 round kc/vc to fp32, 2 to bf16 */
  int branch_mask; /* bit 0 cmp, bit 1 sel, bit 2 swa              */
  int o_round;     /* 0 keep fp64, 1 fp32, 2 bf16: precision in which the
                      branch outputs are stored before the gate gradient
                      reads them (orc_backward only)                 */
} orc_cfg;

#define ORC_CMP 1
#define ORC_SEL 2
#define ORC_SWA 4

/* ------------------------------------------------------------------ */
/* small helpers                                                       */
/* ------------------------------------------------------------------ */

int orc_num_cmp_blocks(const orc_cfg* c) {
  if (c->T < c->cmp_block) return 0;
  return (c->T - c->cmp_block) / c->cmp_stride + 1;
}

int orc_num_sel_blocks(const orc_cfg* c) {
  return (c->T + c->sel_block - 1) / c->sel_block;
}

/* Round a double to the nearest bfloat16 value (8 significant bits),
 * ties to even, by scaling the significand: x = m * 2^e, 0.5 <= |m| < 1,
 * keep round(m * 2^8) / 2^8.  nearbyint uses the default rounding mode,
 * round-half-to-even.  Values here are far from bf16's range limits. */
double orc_round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  double m = frexp(x, &e);
  double r = nearbyint(ldexp(m, 8));
  return ldexp(r, e - 8);
}

static double round_store(double x, int mode) {
  if (mode == 1) return (double)(float)x;
  if (mode == 2) return orc_round_bf16(x);
  return x;
}

static double dot(const double* a, const double* b, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

/* Softmax attention of one query row over an explicit list of key rows.
 * p_out (optional) receives the probabilities in list order.
 * With an empty list the output is 0 and lse = -inf. */
static void attend(const double* qrow, int D, double scale, int n,
                   const double* const* krows, const double* const* vrows,
                   double* out, double* lse, double* p_out) {
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (n == 0) {
    *lse = -INFINITY;
    return;
  }
  double* logit = (double*)malloc(sizeof(double) * (size_t)n);
  double mx = -INFINITY;
  for (int s = 0; s < n; ++s) {
    logit[s] = scale * dot(qrow, krows[s], D);
    if (logit[s] > mx) mx = logit[s];
  }
  double sum = 0.0;
  for (int s = 0; s < n; ++s) {
    logit[s] = exp(logit[s] - mx);
    sum += logit[s];
  }
  for (int s = 0; s < n; ++s) {
    double p = logit[s] / sum;
    if (p_out) p_out[s] = p;
    for (int d = 0; d < D; ++d) out[d] += p * vrows[s][d];
  }
  *lse = mx + log(sum);
  free(logit);
}

/* Backward of `attend` for one row: given dO for this row, accumulate
 * dq (this row), dk and dv (the listed key rows).  Standard softmax
 * calculus: dP_s = dO . v_s, dS_s = P_s (dP_s - dO . o),
 * dq += scale * sum_s dS_s k_s, dk_s += scale * dS_s q, dv_s += P_s dO. */
static void attend_bwd(const double* qrow, int D, double scale, int n,
                       const double* const* krows, const double* const* vrows,
                       const double* dO, double* dq, double* const* dkrows,
                       double* const* dvrows) {
  if (n == 0) return;
  double* p = (double*)malloc(sizeof(double) * (size_t)n);
  double* o = (double*)malloc(sizeof(double) * (size_t)D);
  double lse;
  attend(qrow, D, scale, n, krows, vrows, o, &lse, p);
  double delta = dot(dO, o, D);
  for (int s = 0; s < n; ++s) {
    double dp = dot(dO, vrows[s], D);
    double ds = p[s] * (dp - delta);
    for (int d = 0; d < D; ++d) {
      dq[d] += scale * ds * krows[s][d];
      dkrows[s][d] += scale * ds * qrow[d];
      dvrows[s][d] += p[s] * dO[d];
    }
  }
  free(p);
  free(o);
}

#define QI(c, b, t, h) ((((size_t)(b) * (c)->T + (t)) * (c)->Hq + (h)) * (c)->D)
#define KI(c, b, t, g) ((((size_t)(b) * (c)->T + (t)) * (c)->Hkv + (g)) * (c)->D)
#define CI(c, nc, b, j, g) ((((size_t)(b) * (nc) + (j)) * (c)->Hkv + (g)) * (c)->D)
#define RI(c, b, t, h) (((size_t)(b) * (c)->T + (t)) * (c)->Hq + (h))
#define SI(c, nc, b, t, g) ((((size_t)(b) * (c)->T + (t)) * (c)->Hkv + (g)) * (size_t)(nc))
#define XI(c, b, t, g) ((((size_t)(b) * (c)->T + (t)) * (c)->Hkv + (g)) * (size_t)(c)->topk)

/* ------------------------------------------------------------------ */
/* 1. compression: mean-pool consecutive blocks                        */
/* "Sparsity is Cool", Method and Key claims (mean-pooling instead of  */
/* NSA's MLP); "DeepSeek's Native Sparse Attention", COMPRESSION.       */
/* ------------------------------------------------------------------ */
void orc_compress(const orc_cfg* c, const double* k, const double* v,
                  double* kc, double* vc) {
  const int nc = orc_num_cmp_blocks(c);
  const int l = c->cmp_block, dstr = c->cmp_stride, D = c->D;
  for (int b = 0; b < c->B; ++b)
    for (int j = 0; j < nc; ++j)
      for (int g = 0; g < c->Hkv; ++g)
        for (int d = 0; d < D; ++d) {
          double sk = 0.0, sv = 0.0;
          for (int i = 0; i < l; ++i) {
            sk += k[KI(c, b, j * dstr + i, g) + d];
            sv += v[KI(c, b, j * dstr + i, g) + d];
          }
          kc[CI(c, nc, b, j, g) + d] = round_store(sk / l, c->kv_round);
          vc[CI(c, nc, b, j, g) + d] = round_store(sv / l, c->kv_round);
        }
}

/* number of compressed blocks visible (complete) at query position t */
static int cmp_visible(const orc_cfg* c, int t) {
  const int nc = orc_num_cmp_blocks(c);
  if (t < c->cmp_block - 1) return 0;
  int n = (t - c->cmp_block + 1) / c->cmp_stride + 1;
  return n < nc ? n : nc;
}

/* ------------------------------------------------------------------ */
/* 2. compression-branch attention for one row (b, t, h).              */
/* p_row (optional, length Nc) receives the probabilities, 0 for       */
/* blocks not yet complete.                                            */
/* ------------------------------------------------------------------ */
static void orc_cmp_row(const orc_cfg* c, const double* qrow, const double* kc,
                        const double* vc, int b, int t, int g, double* o,
                        double* lse, double* p_row) {
  const int nc = orc_num_cmp_blocks(c);
  const int n = cmp_visible(c, t);
  const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(n + 1));
  const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(n + 1));
  double* p = (double*)malloc(sizeof(double) * (size_t)(n + 1));
  for (int j = 0; j < n; ++j) {
    kr[j] = kc + CI(c, nc, b, j, g);
    vr[j] = vc + CI(c, nc, b, j, g);
  }
  attend(qrow, c->D, c->scale, n, kr, vr, o, lse, p);
  if (p_row) {
    for (int j = 0; j < nc; ++j) p_row[j] = j < n ? p[j] : 0.0;
  }
  free(kr);
  free(vr);
  free(p);
}

/* ------------------------------------------------------------------ */
/* 3. block importance: the compression probabilities summed over the  */
/* query heads that share KV group g.  "DeepSeek's Native Sparse       */
/* Attention", SELECTION (reuse the compression scores);               */
/* per-GQA-group selection follows the kernel-design paragraph there.  */
/* ------------------------------------------------------------------ */
static void orc_scores_token(const orc_cfg* c, const double* q_tok,
                             const double* kc, const double* vc, int b, int t,
                             double* o_cmp_tok, double* lse_tok,
                             double* score_tok) {
  const int nc = orc_num_cmp_blocks(c);
  const int G = c->Hq / c->Hkv;
  double* p_row = (double*)malloc(sizeof(double) * (size_t)(nc + 1));
  for (int g = 0; g < c->Hkv; ++g)
    for (int j = 0; j < nc; ++j) score_tok[(size_t)g * nc + j] = 0.0;
  for (int h = 0; h < c->Hq; ++h) {
    orc_cmp_row(c, q_tok + (size_t)h * c->D, kc, vc, b, t, h / G,
                o_cmp_tok + (size_t)h * c->D, lse_tok + h, p_row);
    for (int j = 0; j < nc; ++j) score_tok[(size_t)(h / G) * nc + j] += p_row[j];
  }
  free(p_row);
}

/* ------------------------------------------------------------------ */
/* 4. top-k block selection for one (query t, KV group) row.           */
/* "Sparsity is Cool", Method (block 64, top-k 16) and Key claims      */
/* (always include the first block); "DeepSeek's Native Sparse         */
/* Attention", SELECTION.                                              */
/* ------------------------------------------------------------------ */
/* Importance of selection block j for one (token, KV group): the sum of
 * the importances of the compressed blocks whose tokens overlap it
 * (compressed block i covers [i*d, i*d + l), selection block j covers
 * [j*l', (j+1)*l')); blocks not yet complete have importance 0. */
static double sel_block_importance(const orc_cfg* c, const double* cmp_score_row, int j) {
  const int nc = orc_num_cmp_blocks(c);
  const long lo = (long)j * c->sel_block, hi = lo + c->sel_block; /* [lo, hi) */
  double acc = 0.0;
  for (int i = 0; i < nc; ++i) {
    const long clo = (long)i * c->cmp_stride, chi = clo + c->cmp_block;
    if (clo < hi && chi > lo) acc += cmp_score_row[i];
  }
  return acc;
}

/* The selection-block importances of every row: score [B, T, Hkv, Nc] ->
 * out [B, T, Hkv, Nb] (Nb = ceil(T / l')). */
void orc_sel_scores(const orc_cfg* c, const double* score, double* out) {
  const int nc = orc_num_cmp_blocks(c), nb = orc_num_sel_blocks(c);
  const long rows = (long)c->B * c->T * c->Hkv;
  for (long r = 0; r < rows; ++r)
    for (int j = 0; j < nb; ++j)
      out[(size_t)r * nb + j] = sel_block_importance(c, score + (size_t)r * nc, j);
}

static void orc_topk_row(const orc_cfg* c, const double* cmp_score_row, int t,
                         int* idx_row) {
  const int n = c->topk;
  const int cur = t / c->sel_block;
  for (int s = 0; s < n; ++s) idx_row[s] = -1;
  if (cur + 1 <= n) { /* all causal blocks fit */
    for (int j = 0; j <= cur; ++j) idx_row[j] = j;
    return;
  }
  /* selection-block importances from the compressed blocks that overlap
     each selection block (blocks not yet complete have importance 0) */
  double* score_row = (double*)malloc(sizeof(double) * (size_t)(cur + 1));
  for (int j = 0; j <= cur; ++j) score_row[j] = sel_block_importance(c, cmp_score_row, j);
  /* rank the non-forced causal blocks 1..cur-1 by (score desc, index asc)
     with a plain selection sort; keep the first n-2. */
  const int m = cur - 1;
  int* cand = (int*)malloc(sizeof(int) * (size_t)m);
  for (int i = 0; i < m; ++i) cand[i] = i + 1;
  for (int i = 0; i < n - 2; ++i) {
    int best = i;
    for (int r = i + 1; r < m; ++r) {
      double sr = score_row[cand[r]], sb = score_row[cand[best]];
      if (sr > sb || (sr == sb && cand[r] < cand[best])) best = r;
    }
    int tmp = cand[i];
    cand[i] = cand[best];
    cand[best] = tmp;
  }
  /* forced blocks plus the winners, in ascending block order */
  int cnt = 0;
  idx_row[cnt++] = 0;
  for (int i = 0; i < n - 2; ++i) idx_row[cnt++] = cand[i];
  idx_row[cnt++] = cur;
  for (int i = 1; i < cnt; ++i) /* insertion sort */
    for (int r = i; r > 0 && idx_row[r - 1] > idx_row[r]; --r) {
      int tmp = idx_row[r];
      idx_row[r] = idx_row[r - 1];
      idx_row[r - 1] = tmp;
    }
  free(cand);
  free(score_row);
}

/* key positions attended by the selection branch at query t */
static int sel_keys(const orc_cfg* c, const int* idx_row, int t, int* pos) {
  int n = 0;
  for (int s = 0; s < c->topk; ++s) {
    int j = idx_row[s];
    if (j < 0) continue;
    for (int i = 0; i < c->sel_block; ++i) {
      int p = j * c->sel_block + i;
      if (p <= t && p < c->T) pos[n++] = p;
    }
  }
  return n;
}

/* key positions attended by the sliding window at query t */
static int swa_keys(const orc_cfg* c, int t, int* pos) {
  int lo = t - c->window + 1;
  if (lo < 0) lo = 0;
  int n = 0;
  for (int p = lo; p <= t; ++p) pos[n++] = p;
  return n;
}

/* ------------------------------------------------------------------ */
/* 5/6. selection and window attention for one row (b, t, h).          */
/* "DeepSeek's Native Sparse Attention", SELECTION and SLIDING WINDOW; */
/* "Sparsity is Cool", Method (window 512).                            */
/* ------------------------------------------------------------------ */
static void orc_list_row(const orc_cfg* c, const double* qrow, const double* k,
                         const double* v, int b, int g, const int* pos, int n,
                         double* o, double* lse) {
  const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(n + 1));
  const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(n + 1));
  for (int s = 0; s < n; ++s) {
    kr[s] = k + KI(c, b, pos[s], g);
    vr[s] = v + KI(c, b, pos[s], g);
  }
  attend(qrow, c->D, c->scale, n, kr, vr, o, lse, NULL);
  free(kr);
  free(vr);
}

static void orc_sel_row(const orc_cfg* c, const double* qrow, const double* k,
                        const double* v, const int* idx_row, int b, int t,
                        int g, double* o, double* lse) {
  int* pos = (int*)malloc(sizeof(int) * (size_t)(c->topk * c->sel_block + 1));
  int n = sel_keys(c, idx_row, t, pos);
  orc_list_row(c, qrow, k, v, b, g, pos, n, o, lse);
  free(pos);
}

static void orc_swa_row(const orc_cfg* c, const double* qrow, const double* k,
                        const double* v, int b, int t, int g, double* o,
                        double* lse) {
  int* pos = (int*)malloc(sizeof(int) * (size_t)(c->window + 1));
  int n = swa_keys(c, t, pos);
  orc_list_row(c, qrow, k, v, b, g, pos, n, o, lse);
  free(pos);
}

/* ------------------------------------------------------------------ */
/* 7. gated combination.  "DeepSeek's Native Sparse Attention"         */
/* (outputs merged by learned gates); "Sparsity is Cool", TL;DR and    */
/* Key claims (pruning unused branches).                               */
/* ------------------------------------------------------------------ */
static void orc_combine_row(const orc_cfg* c, const double* g3,
                            const double* oc, const double* os,
                            const double* ow, double* out) {
  for (int d = 0; d < c->D; ++d) {
    double acc = 0.0;
    if (c->branch_mask & ORC_CMP) acc += g3[0] * oc[d];
    if (c->branch_mask & ORC_SEL) acc += g3[1] * os[d];
    if (c->branch_mask & ORC_SWA) acc += g3[2] * ow[d];
    out[d] = acc;
  }
}

/* ================================================================== */
/* Whole-tensor entry points (one per library operation)               */
/* ================================================================== */

/* compression branch: o_cmp, lse_cmp and group scores for every row */
void orc_cmp_attn_scores(const orc_cfg* c, const double* q, const double* kc,
                         const double* vc, double* o_cmp, double* lse_cmp,
                         double* score) {
  const int nc = orc_num_cmp_blocks(c);
  const long ntok = (long)c->B * c->T;
#pragma omp parallel for schedule(dynamic, 16)
  for (long bt = 0; bt < ntok; ++bt) {
    int b = (int)(bt / c->T), t = (int)(bt % c->T);
    orc_scores_token(c, q + QI(c, b, t, 0), kc, vc, b, t, o_cmp + QI(c, b, t, 0),
                     lse_cmp + RI(c, b, t, 0), score + SI(c, nc, b, t, 0));
  }
}

void orc_select_topk(const orc_cfg* c, const double* score, int* idx) {
  const int nc = orc_num_cmp_blocks(c);
  const long nrow = (long)c->B * c->T * c->Hkv;
#pragma omp parallel for schedule(static)
  for (long r = 0; r < nrow; ++r) {
    int t = (int)((r / c->Hkv) % c->T);
    orc_topk_row(c, score + (size_t)r * nc, t, idx + (size_t)r * c->topk);
  }
}

void orc_sel_attn_fwd(const orc_cfg* c, const double* q, const double* k,
                      const double* v, const int* idx, double* o_sel,
                      double* lse_sel) {
  const long nrow = (long)c->B * c->T * c->Hq;
  const int G = c->Hq / c->Hkv;
#pragma omp parallel for schedule(dynamic, 64)
  for (long r = 0; r < nrow; ++r) {
    int h = (int)(r % c->Hq);
    int t = (int)((r / c->Hq) % c->T);
    int b = (int)(r / ((long)c->Hq * c->T));
    orc_sel_row(c, q + (size_t)r * c->D, k, v, idx + XI(c, b, t, h / G), b, t,
                h / G, o_sel + (size_t)r * c->D, lse_sel + r);
  }
}

void orc_swa_fwd(const orc_cfg* c, const double* q, const double* k,
                 const double* v, double* o_swa, double* lse_swa) {
  const long nrow = (long)c->B * c->T * c->Hq;
#pragma omp parallel for schedule(dynamic, 64)
  for (long r = 0; r < nrow; ++r) {
    int h = (int)(r % c->Hq);
    int t = (int)((r / c->Hq) % c->T);
    int b = (int)(r / ((long)c->Hq * c->T));
    orc_swa_row(c, q + (size_t)r * c->D, k, v, b, t, h / (c->Hq / c->Hkv),
                o_swa + (size_t)r * c->D, lse_swa + r);
  }
}

void orc_gate_combine(const orc_cfg* c, const double* gates,
                      const double* o_cmp, const double* o_sel,
                      const double* o_swa, double* out) {
  const long nrow = (long)c->B * c->T * c->Hq;
  for (long r = 0; r < nrow; ++r)
    orc_combine_row(c, gates + (size_t)r * 3, o_cmp + (size_t)r * c->D,
                    o_sel + (size_t)r * c->D, o_swa + (size_t)r * c->D,
                    out + (size_t)r * c->D);
}

/* One whole token (all heads, all branches).  kc/vc are the compressed
 * tensors of the full sequence (orc_compress).  Outputs are per token:
 *   o_* / out [Hq, D], lse_* [Hq], score [Hkv, Nc], idx [Hkv, topk]. */
static void orc_token_forward(const orc_cfg* c, const double* q_tok,
                              const double* k, const double* v,
                              const double* kc, const double* vc,
                              const double* gates_tok, int b, int t, double* o_cmp,
                              double* lse_cmp, double* score, int* idx,
                              double* o_sel, double* lse_sel, double* o_swa,
                              double* lse_swa, double* out) {
  const int nc = orc_num_cmp_blocks(c);
  const int G = c->Hq / c->Hkv;
  orc_scores_token(c, q_tok, kc, vc, b, t, o_cmp, lse_cmp, score);
  for (int g = 0; g < c->Hkv; ++g)
    orc_topk_row(c, score + (size_t)g * nc, t, idx + (size_t)g * c->topk);
  for (int h = 0; h < c->Hq; ++h) {
    const double* qrow = q_tok + (size_t)h * c->D;
    orc_sel_row(c, qrow, k, v, idx + (size_t)(h / G) * c->topk, b, t, h / G,
                o_sel + (size_t)h * c->D, lse_sel + h);
    orc_swa_row(c, qrow, k, v, b, t, h / G, o_swa + (size_t)h * c->D,
                lse_swa + h);
    orc_combine_row(c, gates_tok + (size_t)h * 3, o_cmp + (size_t)h * c->D,
                    o_sel + (size_t)h * c->D, o_swa + (size_t)h * c->D,
                    out + (size_t)h * c->D);
  }
}

/* Full forward over every token; every output pointer must be valid. */
void orc_forward(const orc_cfg* c, const double* q, const double* k,
                 const double* v, const double* gates, double* kc, double* vc,
                 double* o_cmp, double* lse_cmp, double* score, int* idx,
                 double* o_sel, double* lse_sel, double* o_swa,
                 double* lse_swa, double* out) {
  const int nc = orc_num_cmp_blocks(c);
  orc_compress(c, k, v, kc, vc);
  const long ntok = (long)c->B * c->T;
#pragma omp parallel for schedule(dynamic, 8)
  for (long bt = 0; bt < ntok; ++bt) {
    int b = (int)(bt / c->T), t = (int)(bt % c->T);
    orc_token_forward(c, q + QI(c, b, t, 0), k, v, kc, vc,
                      gates + RI(c, b, t, 0) * 3, b, t, o_cmp + QI(c, b, t, 0),
                      lse_cmp + RI(c, b, t, 0), score + SI(c, nc, b, t, 0),
                      idx + XI(c, b, t, 0), o_sel + QI(c, b, t, 0),
                      lse_sel + RI(c, b, t, 0), o_swa + QI(c, b, t, 0),
                      lse_swa + RI(c, b, t, 0), out + QI(c, b, t, 0));
  }
}

/* Forward for a sample of tokens only: rows[2*i] = b, rows[2*i+1] = t.
 * kc/vc must already hold orc_compress of the whole input.  Outputs are
 * packed per sampled token: o_* / out [n, Hq, D], lse_* [n, Hq],
 * score [n, Hkv, Nc], idx [n, Hkv, topk]. */
void orc_forward_rows(const orc_cfg* c, const double* q, const double* k,
                      const double* v, const double* gates, const double* kc,
                      const double* vc, int n, const int* rows, double* o_cmp,
                      double* lse_cmp, double* score, int* idx, double* o_sel,
                      double* lse_sel, double* o_swa, double* lse_swa,
                      double* out) {
  const int nc = orc_num_cmp_blocks(c);
  const size_t HD = (size_t)c->Hq * c->D;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n; ++i) {
    int b = rows[2 * i], t = rows[2 * i + 1];
    orc_token_forward(c, q + QI(c, b, t, 0), k, v, kc, vc,
                      gates + RI(c, b, t, 0) * 3, b, t, o_cmp + i * HD, lse_cmp + (size_t)i * c->Hq,
                      score + (size_t)i * c->Hkv * nc,
                      idx + (size_t)i * c->Hkv * c->topk, o_sel + i * HD,
                      lse_sel + (size_t)i * c->Hq, o_swa + i * HD,
                      lse_swa + (size_t)i * c->Hq, out + i * HD);
  }
}

/* ================================================================== */
/* Backward                                                            */
/* ================================================================== */

/* Selection-branch backward given the selection (no gradient through
 * it) and dO_sel = the upstream gradient of o_sel.  dq, dk, dv are
 * ACCUMULATED (+=).  Written as a direct loop over (query, selected key):
 * it follows the chain rule, not the two-pass kernel structure of
 * "Sparsity is Cool", Method. */
void orc_sel_attn_bwd(const orc_cfg* c, const double* q, const double* k,
                      const double* v, const int* idx, const double* dO_sel,
                      double* dq, double* dk, double* dv) {
  const int G = c->Hq / c->Hkv;
  const long ngrp = (long)c->B * c->Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bg = 0; bg < ngrp; ++bg) {
    int b = (int)(bg / c->Hkv), g = (int)(bg % c->Hkv);
    int* pos = (int*)malloc(sizeof(int) * (size_t)(c->topk * c->sel_block + 1));
    const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(c->topk * c->sel_block + 1));
    const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(c->topk * c->sel_block + 1));
    double** dkr = (double**)malloc(sizeof(double*) * (size_t)(c->topk * c->sel_block + 1));
    double** dvr = (double**)malloc(sizeof(double*) * (size_t)(c->topk * c->sel_block + 1));
    for (int t = 0; t < c->T; ++t) {
      int n = sel_keys(c, idx + XI(c, b, t, g), t, pos);
      for (int s = 0; s < n; ++s) {
        kr[s] = k + KI(c, b, pos[s], g);
        vr[s] = v + KI(c, b, pos[s], g);
        dkr[s] = dk + KI(c, b, pos[s], g);
        dvr[s] = dv + KI(c, b, pos[s], g);
      }
      for (int h = g * G; h < (g + 1) * G; ++h)
        attend_bwd(q + QI(c, b, t, h), c->D, c->scale, n, kr, vr,
                   dO_sel + QI(c, b, t, h), dq + QI(c, b, t, h), dkr, dvr);
    }
    free(pos);
    free(kr);
    free(vr);
    free(dkr);
    free(dvr);
  }
}

/* Window-branch backward given dO_swa; accumulates into dq, dk, dv. */
void orc_swa_bwd(const orc_cfg* c, const double* q, const double* k,
                 const double* v, const double* dO_swa, double* dq, double* dk,
                 double* dv) {
  const int G = c->Hq / c->Hkv;
  const long ngrp = (long)c->B * c->Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bg = 0; bg < ngrp; ++bg) {
    int b = (int)(bg / c->Hkv), g = (int)(bg % c->Hkv);
    int* pos = (int*)malloc(sizeof(int) * (size_t)(c->window + 1));
    const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(c->window + 1));
    const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(c->window + 1));
    double** dkr = (double**)malloc(sizeof(double*) * (size_t)(c->window + 1));
    double** dvr = (double**)malloc(sizeof(double*) * (size_t)(c->window + 1));
    for (int t = 0; t < c->T; ++t) {
      int n = swa_keys(c, t, pos);
      for (int s = 0; s < n; ++s) {
        kr[s] = k + KI(c, b, pos[s], g);
        vr[s] = v + KI(c, b, pos[s], g);
        dkr[s] = dk + KI(c, b, pos[s], g);
        dvr[s] = dv + KI(c, b, pos[s], g);
      }
      for (int h = g * G; h < (g + 1) * G; ++h)
        attend_bwd(q + QI(c, b, t, h), c->D, c->scale, n, kr, vr,
                   dO_swa + QI(c, b, t, h), dq + QI(c, b, t, h), dkr, dvr);
    }
    free(pos);
    free(kr);
    free(vr);
    free(dkr);
    free(dvr);
  }
}

/* Compression-branch backward given dO_cmp: gradients reach kc/vc and,
 * through the mean pool, every raw row of each block (d kc_j / d k_t =
 * 1/l for each token t of block j).  Accumulates into dq, dk, dv. */
void orc_cmp_bwd(const orc_cfg* c, const double* q, const double* kc,
                 const double* vc, const double* dO_cmp, double* dq,
                 double* dk, double* dv) {
  const int nc = orc_num_cmp_blocks(c);
  const int G = c->Hq / c->Hkv;
  const int l = c->cmp_block, dstr = c->cmp_stride, D = c->D;
  const long ngrp = (long)c->B * c->Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bg = 0; bg < ngrp; ++bg) {
    int b = (int)(bg / c->Hkv), g = (int)(bg % c->Hkv);
    double* dkc = (double*)calloc((size_t)(nc + 1) * D, sizeof(double));
    double* dvc = (double*)calloc((size_t)(nc + 1) * D, sizeof(double));
    const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    double** dkr = (double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    double** dvr = (double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    for (int j = 0; j < nc; ++j) {
      kr[j] = kc + CI(c, nc, b, j, g);
      vr[j] = vc + CI(c, nc, b, j, g);
      dkr[j] = dkc + (size_t)j * D;
      dvr[j] = dvc + (size_t)j * D;
    }
    for (int t = 0; t < c->T; ++t) {
      int n = cmp_visible(c, t);
      for (int h = g * G; h < (g + 1) * G; ++h)
        attend_bwd(q + QI(c, b, t, h), D, c->scale, n, kr, vr,
                   dO_cmp + QI(c, b, t, h), dq + QI(c, b, t, h), dkr, dvr);
    }
    for (int j = 0; j < nc; ++j)
      for (int i = 0; i < l; ++i)
        for (int d = 0; d < D; ++d) {
          dk[KI(c, b, j * dstr + i, g) + d] += dkc[(size_t)j * D + d] / l;
          dv[KI(c, b, j * dstr + i, g) + d] += dvc[(size_t)j * D + d] / l;
        }
    free(dkc);
    free(dvc);
    free(kr);
    free(vr);
    free(dkr);
    free(dvr);
  }
}

/* The same backward stopped at the compressed keys and values: dq gets the
 * branch's share and dkc, dvc [B, Nc, Hkv, D] the gradient of kc, vc
 * (accumulated).  With a parametric compressor this is what flows into
 * orc_compress_mlp_bwd. */
void orc_cmp_bwd_kc(const orc_cfg* c, const double* q, const double* kc, const double* vc,
                    const double* dO_cmp, double* dq, double* dkc, double* dvc) {
  const int nc = orc_num_cmp_blocks(c);
  const int G = c->Hq / c->Hkv;
  const long ngrp = (long)c->B * c->Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bg = 0; bg < ngrp; ++bg) {
    const int b = (int)(bg / c->Hkv), g = (int)(bg % c->Hkv);
    const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    double** dkr = (double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    double** dvr = (double**)malloc(sizeof(double*) * (size_t)(nc + 1));
    for (int j = 0; j < nc; ++j) {
      kr[j] = kc + CI(c, nc, b, j, g);
      vr[j] = vc + CI(c, nc, b, j, g);
      dkr[j] = dkc + CI(c, nc, b, j, g);
      dvr[j] = dvc + CI(c, nc, b, j, g);
    }
    for (int t = 0; t < c->T; ++t) {
      const int n = cmp_visible(c, t);
      for (int h = g * G; h < (g + 1) * G; ++h)
        attend_bwd(q + QI(c, b, t, h), c->D, c->scale, n, kr, vr, dO_cmp + QI(c, b, t, h),
                   dq + QI(c, b, t, h), dkr, dvr);
    }
    free(kr);
    free(vr);
    free(dkr);
    free(dvr);
  }
}

/* Gradient of the gated combination: dgates[..., i] = dO . o_i for the
 * enabled branches (0 for disabled ones), and dO_i = gate_i * dO. */
void orc_gate_combine_bwd(const orc_cfg* c, const double* gates,
                          const double* dout, const double* o_cmp,
                          const double* o_sel, const double* o_swa,
                          double* dgates, double* dO_cmp, double* dO_sel,
                          double* dO_swa) {
  const long nrow = (long)c->B * c->T * c->Hq;
  const int D = c->D;
  for (long r = 0; r < nrow; ++r) {
    const double* dO = dout + (size_t)r * D;
    const double* ob[3] = {o_cmp + (size_t)r * D, o_sel + (size_t)r * D,
                           o_swa + (size_t)r * D};
    double* dob[3] = {dO_cmp + (size_t)r * D, dO_sel + (size_t)r * D,
                      dO_swa + (size_t)r * D};
    const int bit[3] = {ORC_CMP, ORC_SEL, ORC_SWA};
    for (int i = 0; i < 3; ++i) {
      int on = (c->branch_mask & bit[i]) != 0;
      dgates[(size_t)r * 3 + i] = on ? dot(dO, ob[i], D) : 0.0;
      for (int d = 0; d < D; ++d)
        dob[i][d] = on ? gates[(size_t)r * 3 + i] * dO[d] : 0.0;
    }
  }
}

/* Full backward of out = combine(cmp, sel, swa) with respect to q, k, v
 * and the gates, for a given upstream dout.  The selection idx is taken
 * from a forward pass on the same inputs and held constant.  All gradient
 * outputs are overwritten. */
void orc_backward(const orc_cfg* c, const double* q, const double* k,
                  const double* v, const double* gates, const double* dout,
                  double* dq, double* dk, double* dv, double* dgates) {
  const int nc = orc_num_cmp_blocks(c);
  const size_t nq = (size_t)c->B * c->T * c->Hq * c->D;
  const size_t nk = (size_t)c->B * c->T * c->Hkv * c->D;
  const size_t nkc = (size_t)c->B * (nc + 1) * c->Hkv * c->D;
  const size_t nr = (size_t)c->B * c->T * c->Hq;
  double* kc = (double*)malloc(nkc * sizeof(double));
  double* vc = (double*)malloc(nkc * sizeof(double));
  double* o_cmp = (double*)malloc(nq * sizeof(double));
  double* o_sel = (double*)malloc(nq * sizeof(double));
  double* o_swa = (double*)malloc(nq * sizeof(double));
  double* out = (double*)malloc(nq * sizeof(double));
  double* lse = (double*)malloc(3 * nr * sizeof(double));
  double* score = (double*)malloc(((size_t)c->B * c->T * c->Hkv * nc + 1) * sizeof(double));
  int* idx = (int*)malloc((size_t)c->B * c->T * c->Hkv * c->topk * sizeof(int));
  double* dOb = (double*)malloc(3 * nq * sizeof(double));
  orc_forward(c, q, k, v, gates, kc, vc, o_cmp, lse, score, idx, o_sel,
              lse + nr, o_swa, lse + 2 * nr, out);
  /* the gate gradient reads the branch outputs as stored (reading R15) */
  for (size_t i = 0; i < nq; ++i) {
    o_cmp[i] = round_store(o_cmp[i], c->o_round);
    o_sel[i] = round_store(o_sel[i], c->o_round);
    o_swa[i] = round_store(o_swa[i], c->o_round);
  }
  orc_gate_combine_bwd(c, gates, dout, o_cmp, o_sel, o_swa, dgates, dOb,
                       dOb + nq, dOb + 2 * nq);
  memset(dq, 0, nq * sizeof(double));
  memset(dk, 0, nk * sizeof(double));
  memset(dv, 0, nk * sizeof(double));
  if (c->branch_mask & ORC_CMP) orc_cmp_bwd(c, q, kc, vc, dOb, dq, dk, dv);
  if (c->branch_mask & ORC_SEL)
    orc_sel_attn_bwd(c, q, k, v, idx, dOb + nq, dq, dk, dv);
  if (c->branch_mask & ORC_SWA) orc_swa_bwd(c, q, k, v, dOb + 2 * nq, dq, dk, dv);
  free(kc);
  free(vc);
  free(o_cmp);
  free(o_sel);
  free(o_swa);
  free(out);
  free(lse);
  free(score);
  free(idx);
  free(dOb);
}

/* dq for a sample of query tokens only (dq is local to its row: it needs
 * the row's own forward and upstream gradient).  rows[2*i] = b,
 * rows[2*i+1] = t; kc/vc from orc_compress of the full input;
 * dq_out [n, Hq, D] is overwritten. */
void orc_backward_dq_rows(const orc_cfg* c, const double* q, const double* k,
                          const double* v, const double* gates, const double* dout,
                          const double* kc, const double* vc, int n,
                          const int* rows, double* dq_out) {
  const int nc = orc_num_cmp_blocks(c);
  const int G = c->Hq / c->Hkv;
  const int D = c->D;
  const size_t HD = (size_t)c->Hq * D;
  const int maxk = c->topk * c->sel_block + c->window + nc + 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n; ++i) {
    const int b = rows[2 * i], t = rows[2 * i + 1];
    double* oc = (double*)malloc(HD * sizeof(double));
    double* os = (double*)malloc(HD * sizeof(double));
    double* ow = (double*)malloc(HD * sizeof(double));
    double* out = (double*)malloc(HD * sizeof(double));
    double* lse = (double*)malloc((size_t)3 * c->Hq * sizeof(double));
    double* sc = (double*)malloc(((size_t)c->Hkv * nc + 1) * sizeof(double));
    int* idx = (int*)malloc((size_t)c->Hkv * c->topk * sizeof(int));
    int* pos = (int*)malloc(sizeof(int) * (size_t)maxk);
    const double** kr = (const double**)malloc(sizeof(double*) * (size_t)maxk);
    const double** vr = (const double**)malloc(sizeof(double*) * (size_t)maxk);
    double** dkr = (double**)malloc(sizeof(double*) * (size_t)maxk);
    double** dvr = (double**)malloc(sizeof(double*) * (size_t)maxk);
    double* sink = (double*)calloc((size_t)D, sizeof(double)); /* dk/dv not wanted */
    double* dO = (double*)malloc((size_t)D * sizeof(double));
    orc_token_forward(c, q + QI(c, b, t, 0), k, v, kc, vc, gates + RI(c, b, t, 0) * 3, b, t,
                      oc, lse, sc, idx, os, lse + c->Hq, ow, lse + 2 * c->Hq, out);
    for (int m = 0; m < maxk; ++m) dkr[m] = dvr[m] = sink;
    for (int h = 0; h < c->Hq; ++h) {
      const int g = h / G;
      const double* qrow = q + QI(c, b, t, h);
      const double* g3 = gates + RI(c, b, t, h) * 3;
      const double* dorow = dout + QI(c, b, t, h);
      double* dq = dq_out + (size_t)i * HD + (size_t)h * D;
      for (int d = 0; d < D; ++d) dq[d] = 0.0;
      if (c->branch_mask & ORC_CMP) {
        const int nv = cmp_visible(c, t);
        for (int j = 0; j < nv; ++j) {
          kr[j] = kc + CI(c, nc, b, j, g);
          vr[j] = vc + CI(c, nc, b, j, g);
        }
        for (int d = 0; d < D; ++d) dO[d] = g3[0] * dorow[d];
        attend_bwd(qrow, D, c->scale, nv, kr, vr, dO, dq, dkr, dvr);
      }
      if (c->branch_mask & ORC_SEL) {
        const int nk = sel_keys(c, idx + (size_t)g * c->topk, t, pos);
        for (int m = 0; m < nk; ++m) {
          kr[m] = k + KI(c, b, pos[m], g);
          vr[m] = v + KI(c, b, pos[m], g);
        }
        for (int d = 0; d < D; ++d) dO[d] = g3[1] * dorow[d];
        attend_bwd(qrow, D, c->scale, nk, kr, vr, dO, dq, dkr, dvr);
      }
      if (c->branch_mask & ORC_SWA) {
        const int nk = swa_keys(c, t, pos);
        for (int m = 0; m < nk; ++m) {
          kr[m] = k + KI(c, b, pos[m], g);
          vr[m] = v + KI(c, b, pos[m], g);
        }
        for (int d = 0; d < D; ++d) dO[d] = g3[2] * dorow[d];
        attend_bwd(qrow, D, c->scale, nk, kr, vr, dO, dq, dkr, dvr);
      }
    }
    free(oc); free(os); free(ow); free(out); free(lse); free(sc); free(idx); free(pos);
    free(kr); free(vr); free(dkr); free(dvr); free(sink); free(dO);
  }
}

/* ================================================================== */
/* Decode: one query per sequence at position L-1 against a cache of  */
/* L keys/values (its own already appended) and the compressed cache  */
/* of the same sequence.  Same per-row math as the forward.            */
/* q [B, Hq, D]; kcache/vcache [B, L, Hkv, D]; kc/vc [B, Nc, Hkv, D];  */
/* gates [B, Hq, 3]; out [B, Hq, D]; idx [B, Hkv, topk];               */
/* score_out (optional) [B, Hkv, Nc].                                  */
/* The cfg's T is the cache length L.                                  */
/* ================================================================== */
void orc_decode(const orc_cfg* c, const double* q_last, const double* kcache,
                const double* vcache, const double* kc, const double* vc,
                const double* gates_last, double* out, int* idx_out,
                double* score_out) {
  const int nc = orc_num_cmp_blocks(c);
  const int L = c->T;
  const size_t HD = (size_t)c->Hq * c->D;
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < c->B; ++b) {
    double* oc = (double*)malloc(HD * sizeof(double));
    double* os = (double*)malloc(HD * sizeof(double));
    double* ow = (double*)malloc(HD * sizeof(double));
    double* lse = (double*)malloc((size_t)3 * c->Hq * sizeof(double));
    double* sc = (double*)malloc(((size_t)c->Hkv * nc + 1) * sizeof(double));
    orc_token_forward(c, q_last + (size_t)b * HD, kcache, vcache, kc, vc,
                      gates_last + (size_t)b * c->Hq * 3, b, L - 1, oc, lse, sc,
                      idx_out + (size_t)b * c->Hkv * c->topk, os, lse + c->Hq,
                      ow, lse + 2 * c->Hq, out + (size_t)b * HD);
    if (score_out)
      memcpy(score_out + (size_t)b * c->Hkv * nc, sc, (size_t)c->Hkv * nc * sizeof(double));
    free(oc);
    free(os);
    free(ow);
    free(lse);
    free(sc);
  }
}

/* ================================================================== */
/* MoBA block attention.  "Sparsity is Cool", Method (MoBA with block  */
/* size 512 and top-k 3) and Key claims (MoBA does not always read the */
/* first block; dense below ~1.5k tokens); "DeepSeek's Native Sparse   */
/* Attention" newsletter, MoBA section (blocks, top-k gating that sends */
/* each query to its most relevant blocks, causal protection).          */
/* Readings taken where the pages are silent:                           */
/*   - the gate of block j for query t is q . (mean of block j's keys), */
/*     summed over the query heads of the KV group, so one selection    */
/*     serves the group (as NSA's selection does);                      */
/*   - the query's own block is always selected and counts toward k;    */
/*     the complete past blocks 0 .. cur-1 compete for the other k-1;   */
/*     with at most k causal blocks all are selected; equal gates go to */
/*     the lower block; keys after the query are masked.                */
/* cfg: cmp_block = cmp_stride = sel_block = the MoBA block size L;     */
/* topk = k; kv_round rounds the mean-pooled keys as stored.            */
/* idx [B, T, Hkv, k] MoBA block indices (ascending, -1 padded),        */
/* o [B, T, Hq, D], lse [B, T, Hq].                                     */
/* ================================================================== */
static void orc_moba_select_row(const orc_cfg* c, const double* q, const double* kc, int nc,
                                int b, int t, int g, int* idx_row) {
  const int n = c->topk, G = c->Hq / c->Hkv, D = c->D;
  const int cur = t / c->sel_block;
  for (int s = 0; s < n; ++s) idx_row[s] = -1;
  if (cur + 1 <= n) {
    for (int j = 0; j <= cur; ++j) idx_row[j] = j;
    return;
  }
  /* gates of the complete past blocks */
  double* gate = (double*)malloc(sizeof(double) * (size_t)cur);
  for (int j = 0; j < cur; ++j) {
    double acc = 0.0;
    for (int h = g * G; h < (g + 1) * G; ++h)
      acc += dot(q + QI(c, b, t, h), kc + CI(c, nc, b, j, g), D);
    gate[j] = acc;
  }
  /* the n-1 best of 0 .. cur-1 by (gate desc, index asc), selection sort */
  int* cand = (int*)malloc(sizeof(int) * (size_t)cur);
  for (int i = 0; i < cur; ++i) cand[i] = i;
  for (int i = 0; i < n - 1; ++i) {
    int best = i;
    for (int r = i + 1; r < cur; ++r) {
      const double gr = gate[cand[r]], gb = gate[cand[best]];
      if (gr > gb || (gr == gb && cand[r] < cand[best])) best = r;
    }
    int tmp = cand[i];
    cand[i] = cand[best];
    cand[best] = tmp;
  }
  for (int i = 0; i < n - 1; ++i) idx_row[i] = cand[i];
  idx_row[n - 1] = cur;
  for (int i = 1; i < n; ++i) /* insertion sort, ascending */
    for (int r = i; r > 0 && idx_row[r - 1] > idx_row[r]; --r) {
      int tmp = idx_row[r];
      idx_row[r] = idx_row[r - 1];
      idx_row[r - 1] = tmp;
    }
  free(gate);
  free(cand);
}

void orc_moba_fwd(const orc_cfg* c, const double* q, const double* k, const double* v,
                  int* idx, double* o, double* lse) {
  const int nc = orc_num_cmp_blocks(c);
  const int G = c->Hq / c->Hkv;
  const size_t nkc = (size_t)c->B * (nc + 1) * c->Hkv * c->D;
  double* kc = (double*)malloc(nkc * sizeof(double));
  double* vc = (double*)malloc(nkc * sizeof(double)); /* pooled values: unused */
  orc_compress(c, k, v, kc, vc);
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
  for (int b = 0; b < c->B; ++b)
    for (int t = 0; t < c->T; ++t) {
      int* pos = (int*)malloc(sizeof(int) * (size_t)(c->topk * c->sel_block + 1));
      for (int g = 0; g < c->Hkv; ++g) {
        int* ir = idx + XI(c, b, t, g);
        orc_moba_select_row(c, q, kc, nc, b, t, g, ir);
        const int n = sel_keys(c, ir, t, pos);
        for (int h = g * G; h < (g + 1) * G; ++h)
          orc_list_row(c, q + QI(c, b, t, h), k, v, b, g, pos, n, o + QI(c, b, t, h),
                       lse + RI(c, b, t, h));
      }
      free(pos);
    }
  free(kc);
  free(vc);
}

/* ================================================================== */
/* Parametric compression (the NSA original that "Sparsity is Cool",    */
/* Method and Key claims, replaces with mean-pooling; "DeepSeek's       */
/* Native Sparse Attention", COMPRESSION: a small neural layer          */
/* summarises the block into one key and one value).  Reading taken:    */
/* one linear layer over the block's l rows of D values flattened in    */
/* token order, weights shared by every head and block:                 */
/*   kc[b, j, g, n] = sum_{i<l} sum_{e<D} k[b, j d + i, g, e] Wk[i D + e, n] */
/* (same for vc with Wv).  Mean-pooling is the special case             */
/* W[i D + e, n] = (e == n) / l.  Wk, Wv [l D, D]; kv_round rounds the  */
/* outputs as stored.                                                   */
/* ================================================================== */
void orc_compress_mlp(const orc_cfg* c, const double* k, const double* v, const double* wk,
                      const double* wv, double* kc, double* vc) {
  const int nc = orc_num_cmp_blocks(c);
  const int l = c->cmp_block, dstr = c->cmp_stride, D = c->D;
  for (int b = 0; b < c->B; ++b)
    for (int j = 0; j < nc; ++j)
      for (int g = 0; g < c->Hkv; ++g)
        for (int n = 0; n < D; ++n) {
          double sk = 0.0, sv = 0.0;
          for (int i = 0; i < l; ++i)
            for (int e = 0; e < D; ++e) {
              sk += k[KI(c, b, j * dstr + i, g) + e] * wk[((size_t)i * D + e) * D + n];
              sv += v[KI(c, b, j * dstr + i, g) + e] * wv[((size_t)i * D + e) * D + n];
            }
          kc[CI(c, nc, b, j, g) + n] = round_store(sk, c->kv_round);
          vc[CI(c, nc, b, j, g) + n] = round_store(sv, c->kv_round);
        }
}

/* Its gradient for upstream dkc, dvc [B, Nc, Hkv, D]: the weights'
 *   dWk[i D + e, n] = sum over (b, j, g) of k[b, j d + i, g, e] dkc[b, j, g, n]
 * and the raw rows' dk[b, j d + i, g, e] += sum_n Wk[i D + e, n] dkc[b, j, g, n]
 * summed over every block j whose tokens include the row (same for v).
 * dk, dv, dwk, dwv are overwritten. */
void orc_compress_mlp_bwd(const orc_cfg* c, const double* k, const double* v,
                          const double* wk, const double* wv, const double* dkc,
                          const double* dvc, double* dk, double* dv, double* dwk, double* dwv) {
  const int nc = orc_num_cmp_blocks(c);
  const int l = c->cmp_block, dstr = c->cmp_stride, D = c->D;
  memset(dk, 0, (size_t)c->B * c->T * c->Hkv * D * sizeof(double));
  memset(dv, 0, (size_t)c->B * c->T * c->Hkv * D * sizeof(double));
  memset(dwk, 0, (size_t)l * D * D * sizeof(double));
  memset(dwv, 0, (size_t)l * D * D * sizeof(double));
  for (int b = 0; b < c->B; ++b)
    for (int j = 0; j < nc; ++j)
      for (int g = 0; g < c->Hkv; ++g)
        for (int i = 0; i < l; ++i)
          for (int e = 0; e < D; ++e) {
            const size_t rowi = KI(c, b, j * dstr + i, g) + e;
            double ak = 0.0, av = 0.0;
            for (int n = 0; n < D; ++n) {
              const double gk = dkc[CI(c, nc, b, j, g) + n], gv = dvc[CI(c, nc, b, j, g) + n];
              dwk[((size_t)i * D + e) * D + n] += k[rowi] * gk;
              dwv[((size_t)i * D + e) * D + n] += v[rowi] * gv;
              ak += wk[((size_t)i * D + e) * D + n] * gk;
              av += wv[((size_t)i * D + e) * D + n] * gv;
            }
            dk[rowi] += ak;
            dv[rowi] += av;
          }
}
