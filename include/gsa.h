/*
 * gsa.h -- C ABI of libgsa.so: the Gist Sparse Attention (GSA) hot path on
 * NVIDIA B200 (sm_100a).
 *
 * Method sources (web explainers of "Forget, Then Recall: Learnable
 * Compression and Selective Unfolding via Gist Sparse Attention"):
 *   [nl] gist.science/nl/paper/2604.20920, "Het Proces (Selectieve
 *        Ontvouwing)": Compressie, Scoring (s_{t,m} = q_t^T k_{g_m}),
 *        Selectie (top-k), Selectieve Ontvouwing; "Hierarchische
 *        Uitbreiding (H-GSA)".
 *   [ja] gist.science/ja/paper/2604.20920, section 2.1 (steps 1-4:
 *        gist insertion, relevance scoring, selective unfolding, hybrid
 *        attention) and section 2.2 (H-GSA, coarse-to-fine selection).
 *   [ko] gist.science/ko/paper/2604.20920, "2. Methodology" (hybrid
 *        attention over selected raw tokens plus all, or selected, gists).
 *
 * Conventions for every entry point
 * ---------------------------------
 *  * Pointers named q, *_k, *_v, out*, scores, sel_*, ws, n_gists, own_len
 *    are DEVICE pointers on the current CUDA device, 16-byte aligned,
 *    densely packed in the layouts stated below (row-major, last index
 *    fastest).  The caller allocates and owns all of them; the library
 *    allocates nothing and keeps no per-call state.
 *  * `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call only enqueues work on that stream and returns;
 *    results are ready when the stream is synchronised.
 *  * Argument checks run on the host before anything is enqueued and return
 *    GSA_ERR_INVALID_ARG / GSA_ERR_UNSUPPORTED / GSA_ERR_WORKSPACE without
 *    side effects.  A launch failure returns GSA_ERR_CUDA.  Errors that
 *    only the device can see (an index in sel_idx out of range, a bounded
 *    wait that expired) are recorded as bits in the workspace status word
 *    (gsa_workspace_status) and the offending element is skipped; the
 *    kernels never trap.
 *  * Device-side counts n_gists[b] (completed gists, N) and own_len[b]
 *    (raw tokens of the query's unfinished chunk, 0 <= own <= chunk) are
 *    int32 arrays of length batch.  They must satisfy N <= n_max and
 *    N*chunk + own <= t_max; the kernels clamp to these bounds.
 *  * Query head h reads kv head h / (hq / hkv) (grouped-query layout).
 *  * Scores and logits are scale * q.k with scale = 1/sqrt(d) unless
 *    desc->scale > 0.  All accumulation is fp32.
 *  * Selection per (b, h): the min(topk, N) chunks of highest score, ties
 *    to the lower chunk index ([nl] Selectie); sel_idx rows list the chosen
 *    chunks in ascending chunk order, padded with -1 (sel_score, the
 *    chunk's score, with -inf).
 *  * Attended set per (b, h) ([ja] 2.1 steps 3-4, [nl] Selectieve
 *    Ontvouwing): for each selected chunk its `chunk` raw tokens and its
 *    gist token; each unselected chunk's gist token unless
 *    exclude_unselected; the own chunk's raw tokens.  Output is the exact
 *    softmax average of the values over that set; lse is its natural-log
 *    normaliser (max + log sum exp).
 *  * A workspace `ws` of gsa_workspace_bytes() bytes is passed to every
 *    call.  Calls that consume another call's results (score -> select ->
 *    unfold) must get the same ws.  One ws must not be used by two calls
 *    that may run concurrently.
 */
#ifndef GSA_H
#define GSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gsa_status {
  GSA_OK = 0,
  GSA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or count */
  GSA_ERR_UNSUPPORTED = 2, /* valid but not built: d, dtype, chunk or topk outside the supported set */
  GSA_ERR_WORKSPACE = 3,   /* ws too small (see gsa_workspace_bytes) */
  GSA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  GSA_ERR_TIMEOUT = 5      /* reported by gsa_workspace_status: a bounded device wait expired */
} gsa_status;

typedef enum gsa_dtype { GSA_F32 = 0, GSA_BF16 = 1 } gsa_dtype;

/* Which partial softmax result a producer left in ws for gsa_unfold_attend. */
typedef enum gsa_prior {
  GSA_PRIOR_NONE = 0,  /* nothing: only valid with exclude_unselected = 1 */
  GSA_PRIOR_GISTS = 1, /* gsa_score_gists in default mode: all completed gists */
  GSA_PRIOR_HGSA = 2,  /* hgsa_select: unselected meta-gists + unselected candidate gists */
  GSA_PRIOR_HGSA2 = 3  /* hgsa2_select: the same over two meta levels */
} gsa_prior;

/* Workspace sizing: which call sequence the workspace serves. */
typedef enum gsa_op {
  GSA_OP_DECODE = 0,
  GSA_OP_HGSA = 1,
  GSA_OP_PREFILL = 2,
  GSA_OP_HGSA2 = 3,
  GSA_OP_GIST_STEP = 4,
  GSA_OP_MULTIQUERY = 5
} gsa_op;

/* Device-side status bits (gsa_workspace_status). */
#define GSA_DEVERR_BAD_INDEX 0x1u /* a sel_idx entry >= N was skipped */
#define GSA_DEVERR_TIMEOUT 0x2u   /* an mbarrier wait exceeded its iteration bound */
#define GSA_DEVERR_CAPACITY 0x4u  /* a count exceeded a capacity and was clamped */

typedef struct gsa_desc {
  int32_t batch;              /* B >= 1 */
  int32_t hq, hkv;            /* query heads, kv heads; hq % hkv == 0, hq/hkv <= 16 */
  int32_t d;                  /* head dim: 64 or 128 */
  int32_t chunk;              /* c: raw tokens per chunk, 1..64 */
  int32_t n_max;              /* gist capacity per (b, kv head); prefill: number of chunks N */
  int32_t t_max;              /* raw-row capacity per (b, kv head); prefill: N*chunk */
  int32_t topk;               /* k, 0..1024 */
  int32_t exclude_unselected; /* 0: unselected chunks keep their gist; 1: dropped */
  float scale;                /* <= 0 selects 1/sqrt(d) */
  int32_t dtype;              /* gsa_dtype of q, gist, meta and raw keys/values */
  int32_t out_dtype;          /* gsa_dtype of the attention output */
} gsa_desc;

typedef struct gsa_hdesc {
  int32_t group;     /* g: gists summarised by one meta-gist, >= 1 */
  int32_t topk_meta; /* meta groups kept per (b, h), 1..64, topk_meta*group <= 4096 */
  int32_t m_max;     /* meta capacity per (b, kv head), >= n_max / group */
} gsa_hdesc;

/* H-GSA with two meta levels: level1 groups gists into meta-gists (as
 * gsa_hdesc for hgsa_select); level2 groups level-1 meta-gists into
 * level-2 meta-gists (group = level-1 meta-gists per level-2 meta-gist,
 * topk_meta = level-2 groups kept, m_max = level-2 capacity). */
typedef struct gsa_h2desc {
  gsa_hdesc level1;
  gsa_hdesc level2;
} gsa_h2desc;

/* Human-readable name of a status code (static string). */
const char *gsa_status_string(int32_t status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t gsa_version(void);

/* Bytes of workspace the call sequence `op` needs for these shapes
 * (hdesc only for GSA_OP_HGSA, may be NULL otherwise; for GSA_OP_HGSA2 it
 * points at the two descriptors of a gsa_h2desc, level1 first).  Returns 0
 * if the shapes are invalid. */
size_t gsa_workspace_bytes(const gsa_desc *desc, int32_t op, const gsa_hdesc *hdesc);

/* Zero the workspace on `stream` (cudaMemsetAsync).  Needed once after
 * allocation; every call leaves the workspace reusable afterwards. */
gsa_status gsa_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Synchronise `stream`, copy the workspace status word (GSA_DEVERR_* bits)
 * to *flags_out and clear it.  A nonzero TIMEOUT bit means results of the
 * affected calls are invalid; call gsa_workspace_init before reusing the
 * workspace after any nonzero flag (counters or the ready list may have
 * been left mid-way). */
gsa_status gsa_workspace_status(void *ws, size_t ws_bytes, void *stream, uint32_t *flags_out);

/* ---- Flat GSA decode: three steps ------------------------------------- */

/* Step 1, relevance scoring ([nl] Scoring; [ja] 2.1 step 2).
 *   q       [B, hq, d]
 *   gist_k  [B, hkv, n_max, d]   gist keys; rows >= n_gists[b] are ignored
 *   gist_v  [B, hkv, n_max, d]   gist values; may be NULL when
 *                                exclude_unselected = 1
 *   scores  [B, hq, n_max] fp32  out: scores[b,h,m] for m < n_gists[b];
 *                                entries beyond are not written
 * In default mode the same pass also leaves in ws the softmax partial over
 * all completed gists (every gist is in the attended set, selected or not),
 * consumed by gsa_unfold_attend with prior = GSA_PRIOR_GISTS. */
gsa_status gsa_score_gists(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                           const int32_t *n_gists, float *scores, void *ws, size_t ws_bytes, void *stream);

/* Step 2, top-k chunk selection ([nl] Selectie; [ja] 2.1 step 3).
 *   scores    [B, hq, n_max] fp32; row (b,h) uses its first n_gists[b]
 *   sel_idx   [B, hq, topk] int32 out; sel_score [B, hq, topk] fp32 out
 * Ties go to the lower chunk index.  Also re-arms the per-row counters in
 * ws that gsa_unfold_attend uses. */
gsa_status gsa_topk_select(const gsa_desc *desc, const float *scores, const int32_t *n_gists, int32_t *sel_idx,
                           float *sel_score, void *ws, size_t ws_bytes, void *stream);

/* Step 2, top-p variant: the probability-threshold selection the pages
 * compare with top-k ([ja] section 4 "Top-k vs Top-p"; [nl] Stabiliteit).
 * The chunk probabilities of row (b,h) are the softmax of its first
 * n_gists[b] scores; the selection is the shortest prefix of the ranking
 * (score desc, ties to the lower chunk index) whose probability mass reaches
 * top_p -- at least one chunk (when n_gists[b] >= 1) and at most topk.
 *   scores    [B, hq, n_max] fp32 (as gsa_score_gists writes them)
 *   sel_idx   [B, hq, topk] int32 out, ascending chunk order, -1 padded;
 *   sel_score [B, hq, topk] fp32 out (may be NULL), -inf padded;
 *   sel_count [B, hq] int32 out (may be NULL): chunks selected per row.
 * topk must be 1..256 and n_max <= 16384 (GSA_ERR_UNSUPPORTED otherwise);
 * a NaN top_p is GSA_ERR_INVALID_ARG; top_p >= 1 keeps min(topk, N).  The
 * output feeds gsa_unfold_attend like gsa_topk_select's, and the per-row
 * counters in ws are re-armed the same way. */
gsa_status gsa_topp_select(const gsa_desc *desc, const float *scores, const int32_t *n_gists, float top_p,
                           int32_t *sel_idx, float *sel_score, int32_t *sel_count, void *ws, size_t ws_bytes,
                           void *stream);

/* Step 3, selective unfolding + exact attention ([nl] Selectieve
 * Ontvouwing; [ja] 2.1 steps 3-4).
 *   raw_k, raw_v  [B, hkv, t_max, d]  chunk m occupies rows m*chunk ..
 *                 m*chunk+chunk-1; the own chunk rows N*chunk .. +own-1
 *   gist_v        [B, hkv, n_max, d]  read for selected chunks when
 *                 exclude_unselected = 1 (NULL allowed otherwise)
 *   sel_idx, sel_score  from gsa_topk_select or hgsa_select (the selected
 *                 gist's logit is its score, so gist keys are not re-read)
 *   prior         which partial result ws holds (gsa_prior)
 *   out           [B, hq, d] in out_dtype; lse [B, hq] fp32 or NULL
 * Selected entries that are negative are skipped; entries >= N are skipped
 * and flagged (GSA_DEVERR_BAD_INDEX).  A chunk listed twice is attended
 * twice (the selection calls never list one twice). */
gsa_status gsa_unfold_attend(const gsa_desc *desc, const void *q, const void *raw_k, const void *raw_v,
                             const void *gist_v, const int32_t *n_gists, const int32_t *own_len,
                             const int32_t *sel_idx, const float *sel_score, int32_t prior, void *out, float *lse,
                             void *ws, size_t ws_bytes, void *stream);

/* Steps 1 and 2 ([nl] Scoring + Selectie; [ja] 2.1 steps 2-3), bf16
 * inputs only (GSA_ERR_UNSUPPORTED otherwise): gsa_score_gists and, in the
 * same kernel, the top-k selection of every row -- the last CTAs to finish
 * a (b, kv head) group select for the group's query heads while other
 * groups are still being scored.  Rows longer than 4096 gists (d = 64) or
 * 8192 (d = 128) take gsa_topk_select's kernel after the scoring instead.
 * The selection is the one gsa_topk_select writes (ties to the lower chunk
 * index).
 *   scores    [B, hq, n_max] fp32 out, or NULL (ws holds them)
 *   sel_idx, sel_score  [B, hq, topk] out, or NULL (ws holds them)
 * In default mode ws also receives the gist partial for gsa_unfold_attend
 * with prior = GSA_PRIOR_GISTS. */
gsa_status gsa_score_select(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                            const int32_t *n_gists, float *scores, int32_t *sel_idx, float *sel_score, void *ws,
                            size_t ws_bytes, void *stream);
/* One decode step = score -> select -> unfold on `stream` (bf16: two
 * launches, gsa_score_select then the unfold; fp32: three).  In the bf16
 * form the scoring kernel publishes each selected row in a ready list in
 * ws and the unfold's CTAs take rows as they are published, instead of
 * waiting for the whole scoring kernel.  sel_idx / sel_score ([B, hq,
 * topk]) may be NULL, in which case ws holds them. */
gsa_status gsa_decode(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v, const void *raw_k,
                      const void *raw_v, const int32_t *n_gists, const int32_t *own_len, void *out, float *lse,
                      int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream);

/* Scratch-free decode step.  The paper has no counterpart: this is a
 * deployment variant of gsa_decode for callers that cannot allocate device
 * memory -- for instance a plugin or FFI host that hands over only input
 * and output pointers and exposes no allocator, or a latency-critical
 * caller that must not call cudaMalloc because it may synchronise the
 * device.  It computes exactly what gsa_decode computes, with the same
 * arguments except that there is no `ws`: the workspace is carved from a
 * file-scope device array of GSA_NOALLOC_SCRATCH_BYTES bytes inside
 * libgsa.so, which every GPU that loads the library keeps until the
 * process exits.
 *  * The first call on a device looks up that array's device address
 *    (once per device, with the device current); make that first call
 *    before any stream capture.
 *  * Problems whose workspace (gsa_workspace_bytes(desc, GSA_OP_DECODE,
 *    NULL)) exceeds GSA_NOALLOC_SCRATCH_BYTES are rejected with
 *    GSA_ERR_WORKSPACE before anything is enqueued.
 *  * No cudaMalloc/cudaFree or allocating library routine is called; the
 *    call enqueues a small cudaMemsetAsync that clears the status word and
 *    the per-row and per-group counters, then the decode kernels.
 *  * All calls in the process share the one array and it keeps the last
 *    call's contents: calls whose GPU work may overlap (different streams
 *    without ordering, or several host threads) race and corrupt each
 *    other's results.  Order them on one stream. */
#define GSA_NOALLOC_SCRATCH_BYTES (32u << 20)
gsa_status gsa_decode_noalloc(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                              const void *raw_k, const void *raw_v, const int32_t *n_gists, const int32_t *own_len,
                              void *out, float *lse, int32_t *sel_idx, float *sel_score, void *stream);
/* Device-side status of the last gsa_decode_noalloc call(s) on the current
 * device: synchronises `stream`, copies the GSA_DEVERR_* bits the kernels
 * left in the built-in scratch array to *flags_out and clears them, as
 * gsa_workspace_status does for a caller's workspace (which a scratch-free
 * caller does not have).  Returns GSA_ERR_TIMEOUT when the TIMEOUT bit is
 * set.  Each gsa_decode_noalloc call clears the bits when it starts, so
 * read them after the call whose result you want to check.  Allocates
 * nothing.  The scratch address is looked up once per device; after a
 * device reset (cudaDeviceReset, or a destroyed primary context) it is
 * stale, so neither call may be used across one. */
gsa_status gsa_noalloc_status(void *stream, uint32_t *flags_out);

/* Gist-position step at chunk completion (gist.science/nl/paper/2604.20920,
 * "Het Proces", Compressie: a gist token sees only its own block and the
 * gists before it).  For each sequence b with N = n_gists[b] completed
 * gists and own = own_len[b] raw tokens in chunk N (own = chunk once the
 * chunk is complete):
 *   1. the new gist's key / value (k_new, v_new [B, hkv, d], desc->dtype)
 *      are written at gist row N of gist_k / gist_v;
 *   2. the gist-position query q [B, hq, d] attends the gists 0..N (the
 *      last is itself) and raw rows N*chunk .. N*chunk+own-1 with an exact
 *      softmax: out [B, hq, d] in desc->out_dtype, lse [B, hq] fp32 or NULL;
 *   3. n_gists[b] becomes N+1 and own_len[b] becomes 0 (device-side).
 * desc->topk and desc->exclude_unselected are ignored (the mask has no
 * selection).  Needs N < n_max: a full sequence is flagged
 * (GSA_DEVERR_CAPACITY), attends gists 0..N-1 and the raw rows, and keeps
 * its counts.  Workspace: gsa_workspace_bytes(desc, GSA_OP_GIST_STEP, NULL).
 * gist_k / gist_v / n_gists / own_len are written in place on `stream`. */
gsa_status gsa_gist_step(const gsa_desc *desc, const void *q, const void *k_new, const void *v_new, void *gist_k,
                         void *gist_v, const void *raw_k, const void *raw_v, int32_t *n_gists, int32_t *own_len,
                         void *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* Backward of a decode step for a fixed selection (selective finetuning
 * trains through the path; the top-k choice is piecewise constant, so the
 * gradient flows through the attention over the attended set only).
 * With w = softmax(z), z_u = scale q.k_u over the set, o = sum w_u v_u and
 * g = d_out:  dv_u += w_u g;  dk_u += scale w_u (g.v_u - g.o) q;
 *             d_q += scale sum_u w_u (g.v_u - g.o) k_u.
 *   sel_idx   [B, hq, topk] the forward's selection (negative entries and
 *             entries >= N skipped; no chunk listed twice)
 *   out, lse  the forward's fp32 output [B, hq, d] and lse [B, hq]
 *   d_out     [B, hq, d] fp32
 *   d_q [B, hq, d], d_gist_k / d_gist_v [B, hkv, n_max, d], d_raw_k /
 *   d_raw_v [B, hkv, t_max, d]: fp32, ACCUMULATED (the caller zeroes them;
 *   the heads of a GQA group add into the same key / value rows).
 * Needs no workspace. */
gsa_status gsa_decode_backward(const gsa_desc *desc, const void *q, const void *gist_k, const void *gist_v,
                               const void *raw_k, const void *raw_v, const int32_t *n_gists, const int32_t *own_len,
                               const int32_t *sel_idx, const float *out, const float *lse, const float *d_out,
                               float *d_q, float *d_gist_k, float *d_gist_v, float *d_raw_k, float *d_raw_v,
                               void *stream);

/* ---- H-GSA decode: one meta level ([ja] 2.2; [nl] Hierarchische
 * Uitbreiding) -------------------------------------------------------- */

/* Coarse-to-fine selection.  Meta-gist j (j < M = n_gists[b] / group)
 * summarises gists j*group .. j*group+group-1; gists of an incomplete
 * trailing group have no meta-gist and are always candidates.
 *   meta_k, meta_v  [B, hkv, m_max, d]
 *   meta_idx        [B, hq, topk_meta] int32 out (sorted, -1 padded)
 *   sel_idx         [B, hq, topk] int32 out: chosen chunks (gist ids)
 *   sel_score       [B, hq, topk] fp32 out
 * In default mode ws receives the softmax partial over the unselected
 * meta-gists and all candidate gists (selected candidates' gists are part
 * of the set too), consumed with prior = GSA_PRIOR_HGSA. */
gsa_status hgsa_select(const gsa_desc *desc, const gsa_hdesc *hdesc, const void *q, const void *meta_k,
                       const void *meta_v, const void *gist_k, const void *gist_v, const int32_t *n_gists,
                       int32_t *meta_idx, int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes,
                       void *stream);

/* One H-GSA decode step = hgsa_select -> gsa_unfold_attend.  meta_idx,
 * sel_idx and sel_score may be NULL (ws holds them). */
gsa_status hgsa_decode(const gsa_desc *desc, const gsa_hdesc *hdesc, const void *q, const void *meta_k,
                       const void *meta_v, const void *gist_k, const void *gist_v, const void *raw_k,
                       const void *raw_v, const int32_t *n_gists, const int32_t *own_len, void *out, float *lse,
                       int32_t *meta_idx, int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes,
                       void *stream);

/* ---- H-GSA decode: two meta levels (the recursive gist-of-gist form of
 * [ja] 2.2 / [nl] Hierarchische Uitbreiding) ------------------------------ */

/* Coarse-to-fine over three levels.  With N = n_gists[b], M1 = N / g1
 * level-1 meta-gists and M2 = M1 / g2 level-2 meta-gists (g1 =
 * level1.group, g2 = level2.group): the top level2.topk_meta level-2
 * groups are kept; their level-1 children plus the level-1 meta-gists of an
 * incomplete trailing level-2 group are scored and the top level1.topk_meta
 * kept; their gist children plus the gists of an incomplete trailing
 * level-1 group are scored and the top desc->topk chosen.
 *   meta2_k, meta2_v [B, hkv, level2.m_max, d]; meta_k, meta_v [B, hkv,
 *   level1.m_max, d]; gist and raw arrays as for hgsa_select.
 *   meta2_idx [B, hq, level2.topk_meta], meta_idx [B, hq, level1.topk_meta]
 *   int32 out (ascending, -1 padded); sel_idx / sel_score as hgsa_select.
 * In default mode ws receives the softmax partial over the unselected
 * level-2 meta-gists, the unselected level-1 candidates and all gist
 * candidates, consumed with prior = GSA_PRIOR_HGSA2.  Workspace:
 * gsa_workspace_bytes(desc, GSA_OP_HGSA2, &h2desc.level1). */
gsa_status hgsa2_select(const gsa_desc *desc, const gsa_h2desc *h2desc, const void *q, const void *meta2_k,
                        const void *meta2_v, const void *meta_k, const void *meta_v, const void *gist_k,
                        const void *gist_v, const int32_t *n_gists, int32_t *meta2_idx, int32_t *meta_idx,
                        int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream);

/* One two-level H-GSA decode step = hgsa2_select -> gsa_unfold_attend; the
 * index and score outputs may be NULL (ws holds them). */
gsa_status hgsa2_decode(const gsa_desc *desc, const gsa_h2desc *h2desc, const void *q, const void *meta2_k,
                        const void *meta2_v, const void *meta_k, const void *meta_v, const void *gist_k,
                        const void *gist_v, const void *raw_k, const void *raw_v, const int32_t *n_gists,
                        const int32_t *own_len, void *out, float *lse, int32_t *meta2_idx, int32_t *meta_idx,
                        int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream);

/* ---- Causal prefill with interleaved gists ([nl] Compressie + the
 * decode steps applied at every position) ------------------------------ */

/* Layouts (N = desc->n_max chunks, L = N*chunk = desc->t_max):
 *   q_raw [B, hq, L, d]; k_raw, v_raw [B, hkv, L, d]
 *   q_gist [B, hq, N, d]; k_gist, v_gist [B, hkv, N, d]
 * Raw position i = m*chunk + j sees the completed gists 0..m-1 (top-k
 * selection among them) and its own chunk's raw tokens m*chunk .. i.  Gist
 * position m sees its chunk's raw tokens and gists 0..m (compression mask).
 *
 * Both stages are built for bf16 inputs with d = 64 or 128, topk <= 64
 * and n_max <= 56912 chunks (53760 when topk > 16; GSA_ERR_UNSUPPORTED
 * otherwise), and need t_max = n_max * chunk.
 *
 * Stage 1, scoring + selection (tensor cores).  Every raw row is scored
 * against the gists it can see and keeps the top k; every row (raw and
 * gist) also records its maximum visible score in ws, the softmax
 * reference stage 2 uses.
 *   sel_idx [B, hq, L, topk] int32 out (ascending chunk order, -1 padded),
 *   sel_score [B, hq, L, topk] fp32 out. */
gsa_status gsa_prefill_score(const gsa_desc *desc, const void *q_raw, const void *q_gist, const void *k_gist,
                             int32_t *sel_idx, float *sel_score, void *ws, size_t ws_bytes, void *stream);


/* Multi-query scoring against one shared gist cache (KV reuse: several
 * queries routed over the same document's gists, [ja] section 3 and the
 * KV-cache reuse experiment).  Every query sees all N = desc->n_max gists
 * of its document (the cache is complete), scores them with scale * q.k on
 * the tensor cores (the prefill scoring kernel with the queries placed
 * after the cache) and keeps the top k.
 *   desc: batch = documents; t_max = Q, the queries per (document, query
 *         head); bf16, d = 64 or 128, topk 1..64, n_max <= 56912
 *         (53760 when topk > 16)
 *         (GSA_ERR_UNSUPPORTED otherwise); chunk is ignored.
 *   q       [B, hq, Q, d]; query head h reads kv head h / (hq / hkv)
 *   gist_k  [B, hkv, N, d]
 *   sel_idx [B, hq, Q, topk] int32 out (ascending chunk order),
 *   sel_score [B, hq, Q, topk] fp32 out.
 * Workspace: gsa_workspace_bytes(desc, GSA_OP_MULTIQUERY, NULL). */
gsa_status gsa_multiquery_select(const gsa_desc *desc, const void *q, const void *gist_k, int32_t *sel_idx,
                                 float *sel_score, void *ws, size_t ws_bytes, void *stream);

/* Stage 2, unfolding + attention for every raw and gist position, given
 * stage 1's selection and the row maxima it left in ws (same ws):
 *   out_raw [B, hq, L, d], out_gist [B, hq, N, d] in out_dtype.
 * The dense gist part (all visible gists of a row) runs on the tensor cores
 * with fp16 softmax weights normalised by their own sum; the selected
 * chunks and the own chunk run on the CUDA cores in fp32. */
gsa_status gsa_prefill_attend(const gsa_desc *desc, const void *q_raw, const void *k_raw, const void *v_raw,
                              const void *q_gist, const void *k_gist, const void *v_gist, const int32_t *sel_idx,
                              const float *sel_score, void *out_raw, void *out_gist, void *ws, size_t ws_bytes,
                              void *stream);

/* Both stages.  sel_idx / sel_score may be NULL (ws holds them). */
gsa_status gsa_prefill(const gsa_desc *desc, const void *q_raw, const void *k_raw, const void *v_raw,
                       const void *q_gist, const void *k_gist, const void *v_gist, int32_t *sel_idx,
                       float *sel_score, void *out_raw, void *out_gist, void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GSA_H */
