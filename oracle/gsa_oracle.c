/*
 * gsa_oracle.c -- plain float64 CPU oracle for Gist Sparse Attention (GSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (long_context_gsa_b200, libgsa.so) never calls it, and the two share no
 * code: no headers, helpers, tables or constants.
 *
 * Sources (web explainers of "Forget, Then Recall: Learnable Compression and
 * Selective Unfolding via Gist Sparse Attention", Mao, Li and Fox):
 *   [ja] gist.science/ja/paper/2604.20920, section 2.1 (basic mechanism,
 *        steps 1-4) and section 2.2 (hierarchical extension, H-GSA)
 *   [ko] gist.science/ko/paper/2604.20920, "2. Methodology"
 *   [nl] gist.science/nl/paper/2604.20920, "Het Proces (Selectieve
 *        Ontvouwing)": Compressie, Scoring (s_{t,m} = q_t^T k_{g_m}),
 *        Selectie (top-k), Selectieve Ontvouwing; "Hierarchische Uitbreiding"
 *
 * What it computes, step by step, in the order the pages give:
 *   1. Scoring   s_m = scale * q . k_gist[m] for every completed gist m
 *                ([nl] Scoring; the 1/sqrt(d) factor is the adopted reading,
 *                a positive factor does not change the ranking).
 *   2. Selection the k highest scores; equal scores go to the lower chunk
 *                index ([nl] Selectie, [ja] 2.1 step 3).
 *   3. Unfolding the attended token set is: for each selected chunk its raw
 *                tokens and its gist token (the SG+SR rule, [ja] 2.1 step 3
 *                and the ablation in section 4); each unselected chunk keeps
 *                its gist token only, or is dropped when `exclude` is set
 *                ([nl] Selectieve Ontvouwing, [ko] 2 hybrid attention); plus
 *                the raw tokens of the query's own unfinished chunk.
 *   4. Attention exact softmax over that set: w_u = exp(z_u - Z) / sum,
 *                z_u = scale * q . k_u, output = sum w_u v_u ([ja] 2.1
 *                step 4, hybrid attention).
 *   H-GSA ([ja] 2.2, [nl] Hierarchische Uitbreiding): meta-gists summarise
 *   groups of g gists; the top meta groups are chosen first, then the top
 *   gists among their children, then the chosen chunks are unfolded.
 *   Prefill: the same steps for every position of a sequence with
 *   interleaved gists; a gist position attends its own chunk's raw tokens
 *   and the gists up to and including itself ([nl] Compressie: the causal
 *   mask lets a gist see only its own block and the preceding gists).
 *
 * Everything is float64 with plain scalar loops; inputs are read from their
 * storage type (float32, or bfloat16 bits) and widened exactly.  A pool of
 * POSIX threads runs independent output rows in parallel.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORC_F32 0
#define ORC_BF16 1

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2

/* Token kinds in the attended-set report. */
#define TOK_RAW 0
#define TOK_GIST 1
#define TOK_META 2
#define TOK_META2 3

/* ------------------------------------------------------------------------ */
/* Argument blocks (mirrored by ctypes in oracle/__init__.py).               */
/* ------------------------------------------------------------------------ */

typedef struct {
  int32_t batch, hq, hkv, d, chunk;
  int32_t n_max, t_max, topk, exclude, dtype;
  double scale;                       /* <= 0 selects 1/sqrt(d) */
  const void *q, *gist_k, *gist_v, *raw_k, *raw_v;
  const int32_t *n_gists, *own_len;   /* [batch] */
  int32_t n_rows;                     /* rows to compute */
  const int32_t *rows;                /* row id b*hq + h; NULL = all rows */
  const int32_t *sel_in;              /* optional forced selection [n_rows][topk] */
  double *out;                        /* [n_rows][d] */
  double *lse;                        /* [n_rows] or NULL */
  int32_t *sel_out;                   /* [n_rows][topk] or NULL */
  double *sel_score;                  /* [n_rows][topk] or NULL */
  double *scores;                     /* [n_rows][n_max] or NULL (NaN past N) */
  int32_t set_cap;                    /* capacity of the set report per row */
  int32_t *set_n, *set_kind, *set_idx;/* [n_rows], [n_rows][set_cap] x2 */
  double *set_w;                      /* [n_rows][set_cap] */
  int32_t n_threads;                  /* 0 = all online cores */
} orc_decode_args;

typedef struct {
  int32_t batch, hq, hkv, d, chunk;
  int32_t n_max, t_max, m_max, topk, exclude, dtype;
  int32_t group, topk_meta;
  double scale;
  const void *q, *meta_k, *meta_v, *gist_k, *gist_v, *raw_k, *raw_v;
  const int32_t *n_gists, *own_len;
  int32_t n_rows;
  const int32_t *rows;
  const int32_t *meta_sel_in;         /* optional [n_rows][topk_meta] */
  const int32_t *sel_in;              /* optional [n_rows][topk] */
  double *out, *lse;
  int32_t *meta_sel_out;              /* [n_rows][topk_meta] or NULL */
  int32_t *sel_out;                   /* [n_rows][topk] or NULL */
  double *meta_scores;                /* [n_rows][m_max] or NULL */
  double *cand_scores;                /* [n_rows][n_max] or NULL: child score by gist id, NaN if not a candidate */
  int32_t set_cap;
  int32_t *set_n, *set_kind, *set_idx;
  double *set_w;
  int32_t n_threads;
} orc_hgsa_args;

/* Gist-position step at chunk completion.  Once the raw tokens of chunk N
 * are complete, its gist token is decoded under the compression mask ([nl]
 * Compressie): the gist query sees the raw tokens of its own chunk and the
 * gists 0..N, the last of which is itself (key / value k_new, v_new, given
 * per kv head).  Afterwards it is the (N+1)-th completed gist. */
typedef struct {
  int32_t batch, hq, hkv, d, chunk, n_max, t_max, dtype;
  double scale;
  const void *q;                      /* [batch][hq][d] gist-position queries */
  const void *k_new, *v_new;          /* [batch][hkv][d] */
  const void *gist_k, *gist_v, *raw_k, *raw_v;
  const int32_t *n_gists, *own_len;   /* [batch] */
  double *out, *lse;                  /* [batch*hq][d], [batch*hq] or NULL */
  int32_t n_threads;
} orc_gist_step_args;

/* Backward of the decode attention for a fixed selection (the top-k choice
 * is piecewise constant, so no gradient flows through the scores). */
typedef struct {
  int32_t batch, hq, hkv, d, chunk;
  int32_t n_max, t_max, topk, exclude, dtype;
  double scale;
  const void *q, *gist_k, *gist_v, *raw_k, *raw_v;
  const int32_t *n_gists, *own_len;
  const int32_t *sel_in;              /* [B*hq][topk] the selection (-1 entries skipped) */
  const double *d_out;                /* [B*hq][d] */
  double *d_q;                        /* [B*hq][d] written */
  double *d_gist_k, *d_gist_v;        /* [B][hkv][n_max][d] accumulated */
  double *d_raw_k, *d_raw_v;          /* [B][hkv][t_max][d] accumulated */
} orc_decode_bwd_args;

/* H-GSA with two meta levels: level-1 meta-gist j summarises gists
 * j*group1 .. +group1-1; level-2 meta-gist i summarises level-1 meta-gists
 * i*group2 .. +group2-1. */
typedef struct {
  int32_t batch, hq, hkv, d, chunk;
  int32_t n_max, t_max, m1_max, m2_max;
  int32_t group1, group2, topk2, topk1, topk, exclude, dtype;
  double scale;
  const void *q, *meta2_k, *meta2_v, *meta_k, *meta_v, *gist_k, *gist_v, *raw_k, *raw_v;
  const int32_t *n_gists, *own_len;
  int32_t n_rows;
  const int32_t *rows;
  const int32_t *meta2_sel_in, *meta_sel_in, *sel_in; /* optional forced selections per level */
  double *out, *lse;
  int32_t *meta2_sel_out, *meta_sel_out, *sel_out;     /* [n_rows][topk2], [topk1], [topk] */
  double *meta2_scores, *meta_cand_scores, *cand_scores;/* [n_rows][m2_max], [m1_max], [n_max]; NaN = not scored */
  int32_t set_cap;
  int32_t *set_n, *set_kind, *set_idx;
  double *set_w;
  int32_t n_threads;
} orc_hgsa2_args;

typedef struct {
  int32_t batch, hq, hkv, d, chunk;
  int32_t n_chunks, topk, exclude, dtype;
  double scale;
  const void *q_raw, *k_raw, *v_raw;     /* [B][H][n_chunks*chunk][d] */
  const void *q_gist, *k_gist, *v_gist;  /* [B][H][n_chunks][d] */
  int32_t n_rows;
  const int64_t *rows;                /* (b*hq + h) * (L + N) + pos; pos < L raw, else gist pos-L */
  const int32_t *sel_in;              /* optional [n_rows][topk] */
  double *out, *lse;
  int32_t *sel_out;
  double *sel_score;
  int32_t set_cap;
  int32_t *set_n, *set_kind, *set_idx;
  double *set_w;
  int32_t n_threads;
} orc_prefill_args;

/* ------------------------------------------------------------------------ */
/* Element access and the two primitives: dot product, ranked order.        */
/* ------------------------------------------------------------------------ */

static double elem(const void *base, size_t i, int dtype) {
  if (dtype == ORC_F32) return (double)((const float *)base)[i];
  uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16; /* bf16 -> f32, exact */
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* q . key, both d-vectors at element offsets qo and ko. */
static double dot(const void *qb, size_t qo, const void *kb, size_t ko, int d, int dtype) {
  double acc = 0.0;
  for (int i = 0; i < d; ++i) acc += elem(qb, qo + i, dtype) * elem(kb, ko + i, dtype);
  return acc;
}

typedef struct {
  double s;
  int32_t m;
} scored_t;

/* Ranking: higher score first; equal scores, lower index first. */
static int cmp_rank(const void *x, const void *y) {
  const scored_t *a = (const scored_t *)x, *b = (const scored_t *)y;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->m < b->m) ? -1 : (a->m > b->m);
}

/* Index order (ascending), for writing a selection out. */
static int cmp_index(const void *x, const void *y) {
  const scored_t *a = (const scored_t *)x, *b = (const scored_t *)y;
  return (a->m > b->m) - (a->m < b->m);
}

/* ------------------------------------------------------------------------ */
/* The attended set and exact softmax attention over it.                    */
/* ------------------------------------------------------------------------ */

typedef struct {
  const void *kb, *vb; /* key / value array */
  size_t off;          /* element offset of the row */
  int32_t kind, idx;   /* report only */
} token_t;

typedef struct {
  token_t *tok;
  int32_t n, cap;
} tokset_t;

static int push(tokset_t *S, const void *kb, const void *vb, size_t off, int kind, int idx) {
  if (S->n == S->cap) {
    int32_t nc = S->cap ? 2 * S->cap : 256;
    token_t *t = (token_t *)realloc(S->tok, (size_t)nc * sizeof(token_t));
    if (!t) return ORC_ENOMEM;
    S->tok = t;
    S->cap = nc;
  }
  token_t *t = &S->tok[S->n++];
  t->kb = kb;
  t->vb = vb;
  t->off = off;
  t->kind = kind;
  t->idx = idx;
  return ORC_OK;
}

/* z_u = scale * q.k_u ; Z = max z ; w_u = exp(z_u - Z) / sum_v exp(z_v - Z) ;
 * out = sum_u w_u v_u ; lse = Z + log(sum_v exp(z_v - Z)).                  */
static int attend(const void *qb, size_t qo, const tokset_t *S, int d, int dtype, double scale,
                  double *out, double *lse, int32_t set_cap, int32_t *set_n, int32_t *set_kind,
                  int32_t *set_idx, double *set_w) {
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  if (S->n == 0) { /* empty set: defined as zero output, lse = -inf */
    if (lse) *lse = -INFINITY;
    if (set_n) *set_n = 0;
    return ORC_OK;
  }
  double *z = (double *)malloc((size_t)S->n * sizeof(double));
  if (!z) return ORC_ENOMEM;
  double Z = -INFINITY;
  for (int u = 0; u < S->n; ++u) {
    z[u] = scale * dot(qb, qo, S->tok[u].kb, S->tok[u].off, d, dtype);
    if (z[u] > Z) Z = z[u];
  }
  double denom = 0.0;
  for (int u = 0; u < S->n; ++u) {
    z[u] = exp(z[u] - Z);
    denom += z[u];
  }
  for (int u = 0; u < S->n; ++u) {
    double w = z[u] / denom;
    for (int i = 0; i < d; ++i) out[i] += w * elem(S->tok[u].vb, S->tok[u].off + i, dtype);
    if (set_w && u < set_cap) {
      set_kind[u] = S->tok[u].kind;
      set_idx[u] = S->tok[u].idx;
      set_w[u] = w;
    }
  }
  if (lse) *lse = Z + log(denom);
  if (set_n) *set_n = S->n;
  free(z);
  return ORC_OK;
}

/* Select min(k, n) of the candidates by the ranking above.  `cand` is
 * reordered in place so that the first min(k, n) entries are the selection
 * in rank order.  Returns the number selected. */
static int32_t select_topk(scored_t *cand, int32_t n, int32_t k) {
  qsort(cand, (size_t)n, sizeof(scored_t), cmp_rank);
  return k < n ? k : n;
}

/* A forced selection (the conditional oracle): the listed indices, in the
 * given order, -1 entries ignored.  Returns the count, or -1 if an index is
 * out of [0, n_valid) or repeated. */
static int32_t forced_selection(const int32_t *in, int32_t k, int32_t n_valid, scored_t *sel,
                                const double *score_of) {
  int32_t n = 0;
  for (int32_t i = 0; i < k; ++i) {
    int32_t m = in[i];
    if (m < 0) continue;
    if (m >= n_valid) return -1;
    for (int32_t j = 0; j < n; ++j)
      if (sel[j].m == m) return -1;
    sel[n].m = m;
    sel[n].s = score_of ? score_of[m] : 0.0;
    ++n;
  }
  return n;
}

/* Step 2 alone, on given scores ([nl] Selectie, [ja] 2.1 step 3): for each
 * row, the min(k, n_valid[row]) highest of scores[row][0 .. n_valid), equal
 * scores to the lower index, written in ascending index order to sel_idx
 * [rows][k] (-1 padded) with their scores in sel_score (NULL allowed; -inf
 * padded).  Scores are compared as given (no rescaling).  Returns ORC_EINVAL
 * for a negative count or one above `stride`. */
int gsa_oracle_topk(const double *scores, const int32_t *n_valid, int64_t rows, int32_t stride, int32_t k,
                    int32_t *sel_idx, double *sel_score) {
  if (rows < 0 || stride < 0 || k < 0) return ORC_EINVAL;
  scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)(stride > 0 ? stride : 1));
  if (!cand) return ORC_ENOMEM;
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t n = n_valid[r];
    if (n < 0 || n > stride) {
      free(cand);
      return ORC_EINVAL;
    }
    for (int32_t m = 0; m < n; ++m) {
      cand[m].s = scores[r * stride + m];
      cand[m].m = m;
    }
    const int32_t ns = select_topk(cand, n, k);
    /* ascending index order: mark, then sweep the indices */
    int32_t *out = sel_idx + r * k;
    double *outs = sel_score ? sel_score + r * k : NULL;
    for (int32_t i = 0; i < k; ++i) {
      out[i] = -1;
      if (outs) outs[i] = -INFINITY;
    }
    for (int32_t i = 0; i < ns; ++i) { /* insertion by index among the chosen */
      int32_t j = i;
      while (j > 0 && out[j - 1] > cand[i].m) {
        out[j] = out[j - 1];
        if (outs) outs[j] = outs[j - 1];
        --j;
      }
      out[j] = cand[i].m;
      if (outs) outs[j] = cand[i].s;
    }
  }
  free(cand);
  return ORC_OK;
}

/* Top-p (nucleus) selection on given scores, the variant the pages compare
 * with top-k ([ja] section 4, "Top-k vs Top-p"; [nl] "Stabiliteit": a fixed
 * probability threshold instead of a fixed chunk budget).  For each row the
 * chunk probabilities are the softmax of scores[row][0 .. n_valid), and the
 * selection is the shortest prefix of the ranking above (score desc, index
 * asc) whose probability mass reaches top_p, at least one chunk when
 * n_valid >= 1 and at most k.  Output as for gsa_oracle_topk, plus the count
 * per row in sel_count and the prefix masses before and at the last chosen
 * entry in mass_lo / mass_hi (NULL allowed), which bound how far top_p is
 * from a boundary. */
int gsa_oracle_topp(const double *scores, const int32_t *n_valid, int64_t rows, int32_t stride, int32_t k,
                    double top_p, int32_t *sel_idx, double *sel_score, int32_t *sel_count, double *mass_lo,
                    double *mass_hi) {
  if (rows < 0 || stride < 0 || k < 0) return ORC_EINVAL;
  scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)(stride > 0 ? stride : 1));
  if (!cand) return ORC_ENOMEM;
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t n = n_valid[r];
    if (n < 0 || n > stride) {
      free(cand);
      return ORC_EINVAL;
    }
    for (int32_t m = 0; m < n; ++m) {
      cand[m].s = scores[r * stride + m];
      cand[m].m = m;
    }
    qsort(cand, (size_t)n, sizeof(scored_t), cmp_rank);
    double z = 0.0;
    for (int32_t m = 0; m < n; ++m) z += exp(cand[m].s - cand[0].s);
    int32_t ns = 0;
    double before = 0.0, mass = 0.0;
    while (ns < n && ns < k) {
      before = mass;
      mass += exp(cand[ns].s - cand[0].s) / z;
      ++ns;
      if (mass >= top_p) break;
    }
    if (sel_count) sel_count[r] = ns;
    if (mass_lo) mass_lo[r] = before;
    if (mass_hi) mass_hi[r] = mass;
    int32_t *out = sel_idx + r * k;
    double *outs = sel_score ? sel_score + r * k : NULL;
    for (int32_t i = 0; i < k; ++i) {
      out[i] = -1;
      if (outs) outs[i] = -INFINITY;
    }
    /* ascending index order: the chosen entries sorted by index */
    qsort(cand, (size_t)ns, sizeof(scored_t), cmp_index);
    for (int32_t i = 0; i < ns; ++i) {
      out[i] = cand[i].m;
      if (outs) outs[i] = cand[i].s;
    }
  }
  free(cand);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Thread pool over output rows.                                             */
/* ------------------------------------------------------------------------ */

typedef int (*row_fn)(const void *args, int64_t row_slot);

typedef struct {
  row_fn fn;
  const void *args;
  int64_t n;
  int64_t next; /* atomic */
  int status;   /* atomic: first error */
} pool_t;

static void *pool_worker(void *p) {
  pool_t *P = (pool_t *)p;
  for (;;) {
    int64_t r = __atomic_fetch_add(&P->next, 1, __ATOMIC_RELAXED);
    if (r >= P->n) break;
    int st = P->fn(P->args, r);
    if (st) {
      int zero = 0;
      __atomic_compare_exchange_n(&P->status, &zero, st, 0, __ATOMIC_RELAXED, __ATOMIC_RELAXED);
    }
  }
  return NULL;
}

int gsa_oracle_default_threads(void) {
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

static int run_pool(row_fn fn, const void *args, int64_t n, int32_t n_threads) {
  pool_t P = {fn, args, n, 0, 0};
  int nt = n_threads > 0 ? n_threads : gsa_oracle_default_threads();
  if (nt > n) nt = (int)(n > 0 ? n : 1);
  if (nt <= 1) {
    pool_worker(&P);
    return P.status;
  }
  pthread_t *th = (pthread_t *)malloc((size_t)nt * sizeof(pthread_t));
  if (!th) return ORC_ENOMEM;
  int started = 0;
  for (int i = 0; i < nt; ++i) {
    if (pthread_create(&th[i], NULL, pool_worker, &P) != 0) break;
    ++started;
  }
  if (started == 0) pool_worker(&P);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  return P.status;
}

static double resolve_scale(double scale, int d) { return scale > 0.0 ? scale : 1.0 / sqrt((double)d); }

/* ------------------------------------------------------------------------ */
/* Flat GSA decode, one (b, h) row.                                          */
/* ------------------------------------------------------------------------ */

/* The attended set of a flat decode row, in interleaved-sequence order:
 * for each selected chunk its raw rows and its gist, the gist of every
 * unselected chunk unless `exclude`, then the own raw rows ([ja] 2.1 steps
 * 3-4, the SG+SR rule). */
static int decode_set(tokset_t *S, const void *raw_k, const void *raw_v, const void *gist_k, const void *gist_v,
                      size_t rbase, size_t gbase, int d, int c, int32_t N, int32_t own, int exclude,
                      const char *chosen) {
  int st = ORC_OK;
  for (int32_t m = 0; m < N && !st; ++m) {
    if (chosen[m]) {
      for (int j = 0; j < c && !st; ++j)
        st = push(S, raw_k, raw_v, (rbase + (size_t)m * c + j) * d, TOK_RAW, m * c + j);
      if (!st) st = push(S, gist_k, gist_v, (gbase + m) * d, TOK_GIST, m);
    } else if (!exclude) {
      st = push(S, gist_k, gist_v, (gbase + m) * d, TOK_GIST, m);
    }
  }
  for (int32_t j = 0; j < own && !st; ++j)
    st = push(S, raw_k, raw_v, (rbase + (size_t)N * c + j) * d, TOK_RAW, N * c + j);
  return st;
}

static int decode_row(const void *pa, int64_t slot) {
  const orc_decode_args *a = (const orc_decode_args *)pa;
  const int32_t row = a->rows ? a->rows[slot] : (int32_t)slot;
  const int b = row / a->hq, h = row % a->hq, kvh = h / (a->hq / a->hkv);
  const int d = a->d, c = a->chunk, dt = a->dtype;
  const double scale = resolve_scale(a->scale, d);
  const int32_t N = a->n_gists[b], own = a->own_len[b];
  const size_t qo = ((size_t)b * a->hq + h) * d;
  const size_t gbase = ((size_t)b * a->hkv + kvh) * a->n_max;
  const size_t rbase = ((size_t)b * a->hkv + kvh) * a->t_max;

  /* 1. scores of every completed gist */
  scored_t *cand = (scored_t *)malloc((size_t)(N > 0 ? N : 1) * sizeof(scored_t));
  double *s = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
  char *chosen = (char *)calloc((size_t)(N > 0 ? N : 1), 1);
  if (!cand || !s || !chosen) return ORC_ENOMEM;
  for (int32_t m = 0; m < N; ++m) {
    s[m] = scale * dot(a->q, qo, a->gist_k, (gbase + m) * d, d, dt);
    cand[m].s = s[m];
    cand[m].m = m;
  }
  if (a->scores) {
    double *sr = a->scores + (size_t)slot * a->n_max;
    for (int32_t m = 0; m < a->n_max; ++m) sr[m] = m < N ? s[m] : NAN;
  }

  /* 2. top-k (or the forced selection) */
  int32_t nsel;
  if (a->sel_in) {
    nsel = forced_selection(a->sel_in + (size_t)slot * a->topk, a->topk, N, cand, s);
    if (nsel < 0) return ORC_EINVAL;
  } else {
    nsel = select_topk(cand, N, a->topk);
  }
  for (int32_t i = 0; i < nsel; ++i) chosen[cand[i].m] = 1;
  if (a->sel_out) {
    int32_t *so = a->sel_out + (size_t)slot * a->topk;
    double *ss = a->sel_score ? a->sel_score + (size_t)slot * a->topk : NULL;
    for (int32_t i = 0; i < a->topk; ++i) {
      so[i] = i < nsel ? cand[i].m : -1;
      if (ss) ss[i] = i < nsel ? cand[i].s : -INFINITY;
    }
  }

  /* 3. the attended set, in interleaved-sequence order */
  tokset_t S = {0};
  int st = decode_set(&S, a->raw_k, a->raw_v, a->gist_k, a->gist_v, rbase, gbase, d, c, N, own, a->exclude, chosen);

  /* 4. exact softmax attention over the set */
  if (!st) {
    const size_t so = (size_t)slot;
    st = attend(a->q, qo, &S, d, dt, scale, a->out + so * d, a->lse ? a->lse + so : NULL, a->set_cap,
                a->set_n ? a->set_n + so : NULL, a->set_kind ? a->set_kind + so * a->set_cap : NULL,
                a->set_idx ? a->set_idx + so * a->set_cap : NULL, a->set_w ? a->set_w + so * a->set_cap : NULL);
  }
  free(S.tok);
  free(cand);
  free(s);
  free(chosen);
  return st;
}

static int check_common(int32_t B, int32_t hq, int32_t hkv, int32_t d, int32_t c, int32_t dtype) {
  if (B <= 0 || hq <= 0 || hkv <= 0 || d <= 0 || c <= 0) return ORC_EINVAL;
  if (hq % hkv) return ORC_EINVAL;
  if (dtype != ORC_F32 && dtype != ORC_BF16) return ORC_EINVAL;
  return ORC_OK;
}

/* Gradients of one decode row.  With w = softmax(z), z_u = scale q.k_u over
 * the attended set, o = sum w_u v_u and g = dL/do:
 *   dL/dv_u = w_u g,  dL/dz_u = w_u (g.v_u - g.o),
 *   dL/dq = scale sum_u dL/dz_u k_u,  dL/dk_u = scale dL/dz_u q. */
static int decode_bwd_row(const orc_decode_bwd_args *a, int32_t row) {
  const int b = row / a->hq, h = row % a->hq;
  const int kvh = h / (a->hq / a->hkv); /* contiguous GQA grouping */
  const int d = a->d, c = a->chunk, dt = a->dtype;
  const double scale = resolve_scale(a->scale, d);
  const int32_t N = a->n_gists[b], own = a->own_len[b];
  const size_t qo = ((size_t)b * a->hq + h) * d;
  const size_t gbase = ((size_t)b * a->hkv + kvh) * a->n_max;
  const size_t rbase = ((size_t)b * a->hkv + kvh) * a->t_max;
  char *chosen = (char *)calloc((size_t)(N > 0 ? N : 1), 1);
  if (!chosen) return ORC_ENOMEM;
  for (int32_t i = 0; i < a->topk; ++i) {
    const int32_t m = a->sel_in[(size_t)row * a->topk + i];
    if (m >= 0 && m < N) chosen[m] = 1;
  }
  tokset_t S = {0};
  int st = decode_set(&S, a->raw_k, a->raw_v, a->gist_k, a->gist_v, rbase, gbase, d, c, N, own, a->exclude, chosen);
  double *dq = a->d_q + (size_t)row * d;
  for (int i = 0; i < d; ++i) dq[i] = 0.0;
  if (!st && S.n > 0) {
    const double *g = a->d_out + (size_t)row * d;
    double *w = (double *)malloc((size_t)S.n * sizeof(double));
    double *gv = (double *)malloc((size_t)S.n * sizeof(double));
    if (!w || !gv) return ORC_ENOMEM;
    double Z = -INFINITY, denom = 0.0;
    for (int u = 0; u < S.n; ++u) {
      w[u] = scale * dot(a->q, qo, S.tok[u].kb, S.tok[u].off, d, dt);
      if (w[u] > Z) Z = w[u];
    }
    for (int u = 0; u < S.n; ++u) {
      w[u] = exp(w[u] - Z);
      denom += w[u];
    }
    double go = 0.0; /* g.o = sum_u w_u g.v_u */
    for (int u = 0; u < S.n; ++u) {
      w[u] /= denom;
      double x = 0.0;
      for (int i = 0; i < d; ++i) x += g[i] * elem(S.tok[u].vb, S.tok[u].off + i, dt);
      gv[u] = x;
      go += w[u] * x;
    }
    for (int u = 0; u < S.n; ++u) {
      const double dz = w[u] * (gv[u] - go);
      const int gist = S.tok[u].kind == TOK_GIST;
      double *dk = (gist ? a->d_gist_k : a->d_raw_k) + S.tok[u].off;
      double *dv = (gist ? a->d_gist_v : a->d_raw_v) + S.tok[u].off;
      for (int i = 0; i < d; ++i) {
        dq[i] += scale * dz * elem(S.tok[u].kb, S.tok[u].off + i, dt);
        dk[i] += scale * dz * elem(a->q, qo + i, dt);
        dv[i] += w[u] * g[i];
      }
    }
    free(w);
    free(gv);
  }
  free(S.tok);
  free(chosen);
  return st;
}

/* Rows run one after another: every row adds into the shared key / value
 * gradients. */
int gsa_oracle_decode_backward(const orc_decode_bwd_args *a) {
  if (!a || check_common(a->batch, a->hq, a->hkv, a->d, a->chunk, a->dtype)) return ORC_EINVAL;
  if (a->topk < 0 || !a->q || !a->gist_k || !a->gist_v || !a->raw_k || !a->raw_v || !a->n_gists || !a->own_len)
    return ORC_EINVAL;
  if ((a->topk > 0 && !a->sel_in) || !a->d_out || !a->d_q || !a->d_gist_k || !a->d_gist_v || !a->d_raw_k ||
      !a->d_raw_v)
    return ORC_EINVAL;
  for (int b = 0; b < a->batch; ++b) {
    int32_t N = a->n_gists[b], own = a->own_len[b];
    if (N < 0 || N > a->n_max || own < 0 || own > a->chunk) return ORC_EINVAL;
    if ((int64_t)N * a->chunk + own > a->t_max) return ORC_EINVAL;
  }
  for (int32_t r = 0; r < a->batch * a->hq; ++r) {
    const int st = decode_bwd_row(a, r);
    if (st) return st;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Gist-position step, one (b, h) row.                                       */
/* ------------------------------------------------------------------------ */

/* The set in interleaved-sequence order: the completed gists 0..N-1, the raw
 * tokens of chunk N (own_len of them; c once the chunk is complete), then
 * the gist token itself. */
static int gist_step_row(const void *pa, int64_t row) {
  const orc_gist_step_args *a = (const orc_gist_step_args *)pa;
  const int b = (int)(row / a->hq), h = (int)(row % a->hq), kvh = h / (a->hq / a->hkv);
  const int d = a->d, c = a->chunk, dt = a->dtype;
  const int32_t N = a->n_gists[b], own = a->own_len[b];
  const size_t gbase = ((size_t)b * a->hkv + kvh) * a->n_max;
  const size_t rbase = ((size_t)b * a->hkv + kvh) * a->t_max;
  tokset_t S = {0};
  int st = ORC_OK;
  for (int32_t m = 0; m < N && !st; ++m) st = push(&S, a->gist_k, a->gist_v, (gbase + m) * d, TOK_GIST, m);
  for (int32_t j = 0; j < own && !st; ++j)
    st = push(&S, a->raw_k, a->raw_v, (rbase + (size_t)N * c + j) * d, TOK_RAW, N * c + j);
  if (!st) st = push(&S, a->k_new, a->v_new, ((size_t)b * a->hkv + kvh) * d, TOK_GIST, N);
  if (!st)
    st = attend(a->q, (size_t)row * d, &S, d, dt, resolve_scale(a->scale, d), a->out + (size_t)row * d,
                a->lse ? a->lse + row : NULL, 0, NULL, NULL, NULL, NULL);
  free(S.tok);
  return st;
}

int gsa_oracle_gist_step(const orc_gist_step_args *a) {
  if (!a || check_common(a->batch, a->hq, a->hkv, a->d, a->chunk, a->dtype)) return ORC_EINVAL;
  if (!a->q || !a->k_new || !a->v_new || !a->gist_k || !a->gist_v || !a->raw_k || !a->raw_v || !a->out)
    return ORC_EINVAL;
  if (!a->n_gists || !a->own_len) return ORC_EINVAL;
  for (int b = 0; b < a->batch; ++b) {
    int32_t N = a->n_gists[b], own = a->own_len[b];
    if (N < 0 || N >= a->n_max || own < 0 || own > a->chunk) return ORC_EINVAL; /* room for the new gist */
    if ((int64_t)N * a->chunk + own > a->t_max) return ORC_EINVAL;
  }
  return run_pool(gist_step_row, a, (int64_t)a->batch * a->hq, a->n_threads);
}

int gsa_oracle_decode(const orc_decode_args *a) {
  if (!a || check_common(a->batch, a->hq, a->hkv, a->d, a->chunk, a->dtype)) return ORC_EINVAL;
  if (a->topk < 0 || !a->q || !a->gist_k || !a->gist_v || !a->raw_k || !a->raw_v || !a->out) return ORC_EINVAL;
  if (!a->n_gists || !a->own_len) return ORC_EINVAL;
  for (int b = 0; b < a->batch; ++b) {
    int32_t N = a->n_gists[b], own = a->own_len[b];
    if (N < 0 || N > a->n_max || own < 0 || own > a->chunk) return ORC_EINVAL;
    if ((int64_t)N * a->chunk + own > a->t_max) return ORC_EINVAL;
  }
  int64_t n = a->rows ? a->n_rows : (int64_t)a->batch * a->hq;
  if (a->rows)
    for (int64_t i = 0; i < n; ++i)
      if (a->rows[i] < 0 || a->rows[i] >= a->batch * a->hq) return ORC_EINVAL;
  return run_pool(decode_row, a, n, a->n_threads);
}

/* ------------------------------------------------------------------------ */
/* H-GSA decode, one (b, h) row: meta level, then gist level, then unfold.  */
/* ------------------------------------------------------------------------ */

static int hgsa_row(const void *pa, int64_t slot) {
  const orc_hgsa_args *a = (const orc_hgsa_args *)pa;
  const int32_t row = a->rows ? a->rows[slot] : (int32_t)slot;
  const int b = row / a->hq, h = row % a->hq, kvh = h / (a->hq / a->hkv);
  const int d = a->d, c = a->chunk, dt = a->dtype, g = a->group;
  const double scale = resolve_scale(a->scale, d);
  const int32_t N = a->n_gists[b], own = a->own_len[b];
  const int32_t M = N / g; /* complete meta groups */
  const size_t qo = ((size_t)b * a->hq + h) * d;
  const size_t gbase = ((size_t)b * a->hkv + kvh) * a->n_max;
  const size_t mbase = ((size_t)b * a->hkv + kvh) * a->m_max;
  const size_t rbase = ((size_t)b * a->hkv + kvh) * a->t_max;
  int st = ORC_OK;

  /* meta level: score the meta-gists, keep the top groups */
  const int32_t Mc = M > 0 ? M : 1, Nc = N > 0 ? N : 1;
  scored_t *mc = (scored_t *)malloc((size_t)Mc * sizeof(scored_t));
  double *ms = (double *)malloc((size_t)Mc * sizeof(double));
  char *meta_chosen = (char *)calloc((size_t)Mc, 1);
  scored_t *gc = (scored_t *)malloc((size_t)Nc * sizeof(scored_t));
  double *gs = (double *)malloc((size_t)Nc * sizeof(double));
  char *is_cand = (char *)calloc((size_t)Nc, 1), *chosen = (char *)calloc((size_t)Nc, 1);
  if (!mc || !ms || !meta_chosen || !gc || !gs || !is_cand || !chosen) return ORC_ENOMEM;

  for (int32_t j = 0; j < M; ++j) {
    ms[j] = scale * dot(a->q, qo, a->meta_k, (mbase + j) * d, d, dt);
    mc[j].s = ms[j];
    mc[j].m = j;
  }
  if (a->meta_scores) {
    double *o = a->meta_scores + (size_t)slot * a->m_max;
    for (int32_t j = 0; j < a->m_max; ++j) o[j] = j < M ? ms[j] : NAN;
  }
  int32_t nmeta;
  if (a->meta_sel_in) {
    nmeta = forced_selection(a->meta_sel_in + (size_t)slot * a->topk_meta, a->topk_meta, M, mc, ms);
    if (nmeta < 0) return ORC_EINVAL;
  } else {
    nmeta = select_topk(mc, M, a->topk_meta);
  }
  for (int32_t i = 0; i < nmeta; ++i) meta_chosen[mc[i].m] = 1;
  if (a->meta_sel_out) {
    int32_t *o = a->meta_sel_out + (size_t)slot * a->topk_meta;
    for (int32_t i = 0; i < a->topk_meta; ++i) o[i] = i < nmeta ? mc[i].m : -1;
  }

  /* gist level: candidates are the children of the chosen groups plus the
   * gists of an incomplete trailing group (no meta-gist summarises them) */
  int32_t ncand = 0;
  for (int32_t m = 0; m < N; ++m) {
    int32_t grp = m / g;
    if (grp >= M || meta_chosen[grp]) {
      is_cand[m] = 1;
      gs[m] = scale * dot(a->q, qo, a->gist_k, (gbase + m) * d, d, dt);
      gc[ncand].s = gs[m];
      gc[ncand].m = m;
      ++ncand;
    }
  }
  if (a->cand_scores) {
    double *o = a->cand_scores + (size_t)slot * a->n_max;
    for (int32_t m = 0; m < a->n_max; ++m) o[m] = (m < N && is_cand[m]) ? gs[m] : NAN;
  }
  int32_t nsel;
  if (a->sel_in) {
    /* forced child selection must name candidates */
    nsel = forced_selection(a->sel_in + (size_t)slot * a->topk, a->topk, N, gc, gs);
    if (nsel < 0) return ORC_EINVAL;
    for (int32_t i = 0; i < nsel; ++i)
      if (!is_cand[gc[i].m]) return ORC_EINVAL;
  } else {
    nsel = select_topk(gc, ncand, a->topk);
  }
  for (int32_t i = 0; i < nsel; ++i) chosen[gc[i].m] = 1;
  if (a->sel_out) {
    int32_t *o = a->sel_out + (size_t)slot * a->topk;
    for (int32_t i = 0; i < a->topk; ++i) o[i] = i < nsel ? gc[i].m : -1;
  }

  /* the attended set: unselected meta-gists, unselected candidate gists,
   * selected chunks (raw + gist), own raw rows */
  tokset_t S = {0};
  if (!a->exclude)
    for (int32_t j = 0; j < M && !st; ++j)
      if (!meta_chosen[j]) st = push(&S, a->meta_k, a->meta_v, (mbase + j) * d, TOK_META, j);
  for (int32_t m = 0; m < N && !st; ++m) {
    if (chosen[m]) {
      for (int j = 0; j < c && !st; ++j)
        st = push(&S, a->raw_k, a->raw_v, (rbase + (size_t)m * c + j) * d, TOK_RAW, m * c + j);
      if (!st) st = push(&S, a->gist_k, a->gist_v, (gbase + m) * d, TOK_GIST, m);
    } else if (is_cand[m] && !a->exclude) {
      st = push(&S, a->gist_k, a->gist_v, (gbase + m) * d, TOK_GIST, m);
    }
  }
  for (int32_t j = 0; j < own && !st; ++j)
    st = push(&S, a->raw_k, a->raw_v, (rbase + (size_t)N * c + j) * d, TOK_RAW, N * c + j);
  if (!st) {
    const size_t so = (size_t)slot;
    st = attend(a->q, qo, &S, d, dt, scale, a->out + so * d, a->lse ? a->lse + so : NULL, a->set_cap,
                a->set_n ? a->set_n + so : NULL, a->set_kind ? a->set_kind + so * a->set_cap : NULL,
                a->set_idx ? a->set_idx + so * a->set_cap : NULL, a->set_w ? a->set_w + so * a->set_cap : NULL);
  }
  free(S.tok);
  free(mc);
  free(ms);
  free(meta_chosen);
  free(gc);
  free(gs);
  free(is_cand);
  free(chosen);
  return st;
}

/* One level of the coarse-to-fine selection: the candidates are the
 * children of the chosen parents plus the entries of an incomplete trailing
 * group (no parent summarises them); they are scored and the top k (or a
 * forced list) chosen.  `chosen_parent` has `n_parents` entries (complete
 * groups); `cand`, `score`, `is_cand`, `chosen` have `n` entries.  Returns
 * the number chosen, or -1 for an invalid forced list. */
static int32_t select_level(const void *q, size_t qo, const void *keys, size_t kbase, int d, int dt, double scale,
                            int32_t n, int32_t group, int32_t n_parents, const char *chosen_parent, int32_t k,
                            const int32_t *forced, scored_t *cand, double *score, char *is_cand, char *chosen) {
  int32_t nc = 0;
  for (int32_t m = 0; m < n; ++m) {
    const int32_t grp = m / group;
    is_cand[m] = 0;
    chosen[m] = 0;
    if (grp >= n_parents || chosen_parent[grp]) {
      is_cand[m] = 1;
      score[m] = scale * dot(q, qo, keys, (kbase + m) * d, d, dt);
      cand[nc].s = score[m];
      cand[nc].m = m;
      ++nc;
    }
  }
  int32_t ns;
  if (forced) {
    ns = forced_selection(forced, k, n, cand, score);
    if (ns < 0) return -1;
    for (int32_t i = 0; i < ns; ++i)
      if (!is_cand[cand[i].m]) return -1;
  } else {
    ns = select_topk(cand, nc, k);
  }
  for (int32_t i = 0; i < ns; ++i) chosen[cand[i].m] = 1;
  return ns;
}

static int hgsa2_row(const void *pa, int64_t slot) {
  const orc_hgsa2_args *a = (const orc_hgsa2_args *)pa;
  const int32_t row = a->rows ? a->rows[slot] : (int32_t)slot;
  const int b = row / a->hq, h = row % a->hq, kvh = h / (a->hq / a->hkv);
  const int d = a->d, c = a->chunk, dt = a->dtype;
  const double scale = resolve_scale(a->scale, d);
  const int32_t N = a->n_gists[b], own = a->own_len[b];
  const int32_t M1 = N / a->group1, M2 = M1 / a->group2; /* complete groups at each level */
  const size_t qo = ((size_t)b * a->hq + h) * d;
  const size_t gbase = ((size_t)b * a->hkv + kvh) * a->n_max;
  const size_t m1base = ((size_t)b * a->hkv + kvh) * a->m1_max;
  const size_t m2base = ((size_t)b * a->hkv + kvh) * a->m2_max;
  const size_t rbase = ((size_t)b * a->hkv + kvh) * a->t_max;
  int st = ORC_OK;
  const int32_t cap = (N > 0 ? N : 1);
  scored_t *cand = (scored_t *)malloc((size_t)cap * sizeof(scored_t));
  double *score2 = (double *)malloc((size_t)(M2 > 0 ? M2 : 1) * sizeof(double));
  double *score1 = (double *)malloc((size_t)(M1 > 0 ? M1 : 1) * sizeof(double));
  double *score0 = (double *)malloc((size_t)cap * sizeof(double));
  char *all2 = (char *)calloc(1, 1);
  char *cand2 = (char *)calloc((size_t)(M2 > 0 ? M2 : 1), 1), *chosen2 = (char *)calloc((size_t)(M2 > 0 ? M2 : 1), 1);
  char *cand1 = (char *)calloc((size_t)(M1 > 0 ? M1 : 1), 1), *chosen1 = (char *)calloc((size_t)(M1 > 0 ? M1 : 1), 1);
  char *cand0 = (char *)calloc((size_t)cap, 1), *chosen0 = (char *)calloc((size_t)cap, 1);
  if (!cand || !score2 || !score1 || !score0 || !all2 || !cand2 || !chosen2 || !cand1 || !chosen1 || !cand0 || !chosen0)
    return ORC_ENOMEM;

  /* level 2: every level-2 meta-gist is a candidate (one group with no parent) */
  const int32_t n2 = select_level(a->q, qo, a->meta2_k, m2base, d, dt, scale, M2, M2 > 0 ? M2 : 1, 0, all2,
                                  a->topk2, a->meta2_sel_in ? a->meta2_sel_in + (size_t)slot * a->topk2 : NULL,
                                  cand, score2, cand2, chosen2);
  if (n2 < 0) return ORC_EINVAL;
  if (a->meta2_sel_out) {
    int32_t *o = a->meta2_sel_out + (size_t)slot * a->topk2;
    for (int32_t i = 0; i < a->topk2; ++i) o[i] = i < n2 ? cand[i].m : -1;
  }
  if (a->meta2_scores) {
    double *o = a->meta2_scores + (size_t)slot * a->m2_max;
    for (int32_t j = 0; j < a->m2_max; ++j) o[j] = j < M2 ? score2[j] : NAN;
  }
  /* level 1: children of the chosen level-2 groups + the trailing level-1 meta-gists */
  const int32_t n1 = select_level(a->q, qo, a->meta_k, m1base, d, dt, scale, M1, a->group2, M2, chosen2, a->topk1,
                                  a->meta_sel_in ? a->meta_sel_in + (size_t)slot * a->topk1 : NULL, cand, score1,
                                  cand1, chosen1);
  if (n1 < 0) return ORC_EINVAL;
  if (a->meta_sel_out) {
    int32_t *o = a->meta_sel_out + (size_t)slot * a->topk1;
    for (int32_t i = 0; i < a->topk1; ++i) o[i] = i < n1 ? cand[i].m : -1;
  }
  if (a->meta_cand_scores) {
    double *o = a->meta_cand_scores + (size_t)slot * a->m1_max;
    for (int32_t j = 0; j < a->m1_max; ++j) o[j] = (j < M1 && cand1[j]) ? score1[j] : NAN;
  }
  /* level 0: children of the chosen level-1 meta-gists + the trailing gists */
  const int32_t n0 = select_level(a->q, qo, a->gist_k, gbase, d, dt, scale, N, a->group1, M1, chosen1, a->topk,
                                  a->sel_in ? a->sel_in + (size_t)slot * a->topk : NULL, cand, score0, cand0,
                                  chosen0);
  if (n0 < 0) return ORC_EINVAL;
  if (a->sel_out) {
    int32_t *o = a->sel_out + (size_t)slot * a->topk;
    for (int32_t i = 0; i < a->topk; ++i) o[i] = i < n0 ? cand[i].m : -1;
  }
  if (a->cand_scores) {
    double *o = a->cand_scores + (size_t)slot * a->n_max;
    for (int32_t m = 0; m < a->n_max; ++m) o[m] = (m < N && cand0[m]) ? score0[m] : NAN;
  }

  /* the attended set at every resolution: unselected level-2 meta-gists,
   * unselected level-1 candidates, unselected gist candidates, the chosen
   * chunks (raw + gist) and the own raw rows */
  tokset_t S = {0};
  if (!a->exclude) {
    for (int32_t i = 0; i < M2 && !st; ++i)
      if (!chosen2[i]) st = push(&S, a->meta2_k, a->meta2_v, (m2base + i) * d, TOK_META2, i);
    for (int32_t j = 0; j < M1 && !st; ++j)
      if (cand1[j] && !chosen1[j]) st = push(&S, a->meta_k, a->meta_v, (m1base + j) * d, TOK_META, j);
  }
  for (int32_t m = 0; m < N && !st; ++m) {
    if (chosen0[m]) {
      for (int j = 0; j < c && !st; ++j)
        st = push(&S, a->raw_k, a->raw_v, (rbase + (size_t)m * c + j) * d, TOK_RAW, m * c + j);
      if (!st) st = push(&S, a->gist_k, a->gist_v, (gbase + m) * d, TOK_GIST, m);
    } else if (cand0[m] && !a->exclude) {
      st = push(&S, a->gist_k, a->gist_v, (gbase + m) * d, TOK_GIST, m);
    }
  }
  for (int32_t j = 0; j < own && !st; ++j)
    st = push(&S, a->raw_k, a->raw_v, (rbase + (size_t)N * c + j) * d, TOK_RAW, N * c + j);
  if (!st) {
    const size_t so = (size_t)slot;
    st = attend(a->q, qo, &S, d, dt, scale, a->out + so * d, a->lse ? a->lse + so : NULL, a->set_cap,
                a->set_n ? a->set_n + so : NULL, a->set_kind ? a->set_kind + so * a->set_cap : NULL,
                a->set_idx ? a->set_idx + so * a->set_cap : NULL, a->set_w ? a->set_w + so * a->set_cap : NULL);
  }
  free(S.tok);
  free(cand);
  free(score2);
  free(score1);
  free(score0);
  free(all2);
  free(cand2);
  free(chosen2);
  free(cand1);
  free(chosen1);
  free(cand0);
  free(chosen0);
  return st;
}

int gsa_oracle_hgsa2(const orc_hgsa2_args *a) {
  if (!a || check_common(a->batch, a->hq, a->hkv, a->d, a->chunk, a->dtype)) return ORC_EINVAL;
  if (a->group1 <= 0 || a->group2 <= 0 || a->topk < 0 || a->topk1 < 0 || a->topk2 < 0) return ORC_EINVAL;
  if (!a->q || !a->meta2_k || !a->meta2_v || !a->meta_k || !a->meta_v || !a->gist_k || !a->gist_v || !a->raw_k ||
      !a->raw_v || !a->out)
    return ORC_EINVAL;
  if (!a->n_gists || !a->own_len) return ORC_EINVAL;
  for (int b = 0; b < a->batch; ++b) {
    int32_t N = a->n_gists[b], own = a->own_len[b];
    if (N < 0 || N > a->n_max || own < 0 || own > a->chunk) return ORC_EINVAL;
    if (N / a->group1 > a->m1_max || N / a->group1 / a->group2 > a->m2_max) return ORC_EINVAL;
    if ((int64_t)N * a->chunk + own > a->t_max) return ORC_EINVAL;
  }
  int64_t n = a->rows ? a->n_rows : (int64_t)a->batch * a->hq;
  if (a->rows)
    for (int64_t i = 0; i < n; ++i)
      if (a->rows[i] < 0 || a->rows[i] >= a->batch * a->hq) return ORC_EINVAL;
  return run_pool(hgsa2_row, a, n, a->n_threads);
}

int gsa_oracle_hgsa(const orc_hgsa_args *a) {
  if (!a || check_common(a->batch, a->hq, a->hkv, a->d, a->chunk, a->dtype)) return ORC_EINVAL;
  if (a->group <= 0 || a->topk < 0 || a->topk_meta < 0) return ORC_EINVAL;
  if (!a->q || !a->meta_k || !a->meta_v || !a->gist_k || !a->gist_v || !a->raw_k || !a->raw_v || !a->out)
    return ORC_EINVAL;
  if (!a->n_gists || !a->own_len) return ORC_EINVAL;
  for (int b = 0; b < a->batch; ++b) {
    int32_t N = a->n_gists[b], own = a->own_len[b];
    if (N < 0 || N > a->n_max || own < 0 || own > a->chunk) return ORC_EINVAL;
    if (N / a->group > a->m_max) return ORC_EINVAL;
    if ((int64_t)N * a->chunk + own > a->t_max) return ORC_EINVAL;
  }
  int64_t n = a->rows ? a->n_rows : (int64_t)a->batch * a->hq;
  if (a->rows)
    for (int64_t i = 0; i < n; ++i)
      if (a->rows[i] < 0 || a->rows[i] >= a->batch * a->hq) return ORC_EINVAL;
  return run_pool(hgsa_row, a, n, a->n_threads);
}

/* ------------------------------------------------------------------------ */
/* Causal prefill with interleaved gists, one (b, h, position) row.          */
/* ------------------------------------------------------------------------ */

static int prefill_row(const void *pa, int64_t slot) {
  const orc_prefill_args *a = (const orc_prefill_args *)pa;
  const int d = a->d, c = a->chunk, dt = a->dtype;
  const int32_t N = a->n_chunks;
  const int64_t L = (int64_t)N * c, P = L + N;
  const int64_t row = a->rows ? a->rows[slot] : slot;
  const int64_t bh = row / P, pos = row % P;
  const int b = (int)(bh / a->hq), h = (int)(bh % a->hq), kvh = h / (a->hq / a->hkv);
  const double scale = resolve_scale(a->scale, d);
  const size_t rb = ((size_t)b * a->hkv + kvh) * (size_t)L;  /* raw rows of this kv head */
  const size_t gb = ((size_t)b * a->hkv + kvh) * (size_t)N;  /* gist rows of this kv head */
  tokset_t S = {0};
  int st = ORC_OK;
  const void *qarr;
  size_t qo;
  int32_t nsel = 0;
  scored_t *cand = NULL;
  double *s = NULL;
  char *chosen = NULL;

  if (pos >= L) {
    /* gist query m: its own chunk's raw tokens and the gists 0..m */
    const int32_t m = (int32_t)(pos - L);
    qarr = a->q_gist;
    qo = (((size_t)b * a->hq + h) * (size_t)N + m) * d;
    for (int j = 0; j < c && !st; ++j) st = push(&S, a->k_raw, a->v_raw, (rb + (size_t)m * c + j) * d, TOK_RAW, m * c + j);
    for (int32_t t = 0; t <= m && !st; ++t) st = push(&S, a->k_gist, a->v_gist, (gb + t) * d, TOK_GIST, t);
  } else {
    /* raw query at position i = m*c + j: completed chunks are 0..m-1 and the
     * own chunk's raw tokens m*c .. i are visible */
    const int32_t m = (int32_t)(pos / c), j = (int32_t)(pos % c);
    qarr = a->q_raw;
    qo = (((size_t)b * a->hq + h) * (size_t)L + pos) * d;
    const int32_t mc = m > 0 ? m : 1;
    cand = (scored_t *)malloc((size_t)mc * sizeof(scored_t));
    s = (double *)malloc((size_t)mc * sizeof(double));
    chosen = (char *)calloc((size_t)mc, 1);
    if (!cand || !s || !chosen) return ORC_ENOMEM;
    for (int32_t t = 0; t < m; ++t) {
      s[t] = scale * dot(qarr, qo, a->k_gist, (gb + t) * d, d, dt);
      cand[t].s = s[t];
      cand[t].m = t;
    }
    if (a->sel_in) {
      nsel = forced_selection(a->sel_in + (size_t)slot * a->topk, a->topk, m, cand, s);
      if (nsel < 0) return ORC_EINVAL;
    } else {
      nsel = select_topk(cand, m, a->topk);
    }
    for (int32_t i = 0; i < nsel; ++i) chosen[cand[i].m] = 1;
    for (int32_t t = 0; t < m && !st; ++t) {
      if (chosen[t]) {
        for (int r = 0; r < c && !st; ++r)
          st = push(&S, a->k_raw, a->v_raw, (rb + (size_t)t * c + r) * d, TOK_RAW, t * c + r);
        if (!st) st = push(&S, a->k_gist, a->v_gist, (gb + t) * d, TOK_GIST, t);
      } else if (!a->exclude) {
        st = push(&S, a->k_gist, a->v_gist, (gb + t) * d, TOK_GIST, t);
      }
    }
    for (int32_t r = 0; r <= j && !st; ++r)
      st = push(&S, a->k_raw, a->v_raw, (rb + (size_t)m * c + r) * d, TOK_RAW, m * c + r);
  }
  if (a->sel_out) {
    int32_t *so = a->sel_out + (size_t)slot * a->topk;
    double *ss = a->sel_score ? a->sel_score + (size_t)slot * a->topk : NULL;
    for (int32_t i = 0; i < a->topk; ++i) {
      so[i] = i < nsel ? cand[i].m : -1;
      if (ss) ss[i] = i < nsel ? cand[i].s : -INFINITY;
    }
  }
  if (!st) {
    const size_t so = (size_t)slot;
    st = attend(qarr, qo, &S, d, dt, scale, a->out + so * d, a->lse ? a->lse + so : NULL, a->set_cap,
                a->set_n ? a->set_n + so : NULL, a->set_kind ? a->set_kind + so * a->set_cap : NULL,
                a->set_idx ? a->set_idx + so * a->set_cap : NULL, a->set_w ? a->set_w + so * a->set_cap : NULL);
  }
  free(S.tok);
  free(cand);
  free(s);
  free(chosen);
  return st;
}

int gsa_oracle_prefill(const orc_prefill_args *a) {
  if (!a || check_common(a->batch, a->hq, a->hkv, a->d, a->chunk, a->dtype)) return ORC_EINVAL;
  if (a->n_chunks < 0 || a->topk < 0) return ORC_EINVAL;
  if (!a->q_raw || !a->k_raw || !a->v_raw || !a->q_gist || !a->k_gist || !a->v_gist || !a->out) return ORC_EINVAL;
  const int64_t P = (int64_t)a->n_chunks * a->chunk + a->n_chunks;
  const int64_t total = (int64_t)a->batch * a->hq * P;
  int64_t n = a->rows ? a->n_rows : total;
  if (a->rows)
    for (int64_t i = 0; i < n; ++i)
      if (a->rows[i] < 0 || a->rows[i] >= total) return ORC_EINVAL;
  return run_pool(prefill_row, a, n, a->n_threads);
}
