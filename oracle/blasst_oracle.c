/*
 * blasst_oracle.c - plain, slow, fp64 CPU oracle for blocked attention with
 * softmax thresholding. TEST INFRASTRUCTURE ONLY: the library and its kernels
 * never call it; only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg do.
 *
 * What it follows (citations name the web page and the paragraph on it; the
 * paragraphs of the Telegram post are counted after its headline):
 *
 *   [T] "BLASST: Dynamic BLocked Attention Sparsity via Softmax Thresholding"
 *       (Telegram channel seeallochnaya, post 3655):
 *         para 2  - FlashAttention cuts the sequence into KV blocks and walks
 *                   them left to right; the row max is subtracted before exp
 *                   because softmax does not change under a shift.
 *         para 3  - online softmax: keep the running max, compare each new
 *                   block's local max with it, rescale the earlier partial
 *                   results when it grows; after the last block the result is
 *                   exact.
 *         para 4  - FlashAttention 4 rescales lazily, only when precision is
 *                   at risk; the result is still exact (ref_mode 1 below).
 *         para 5  - BLASST: when a block's max is far below the max of the
 *                   blocks before it, the block is dropped and its V vectors
 *                   take no part in the computation.
 *         para 6  - the figure: the first block is always processed.
 *   [D] "BLASST wins Best Paper at MLSys 2026 ..." (digg.com/ai/al6mgdew),
 *       the authors' announcement: one scalar threshold on the online-softmax
 *       statistics decides the skip.
 *
 * The exact rule: a KV block is skipped when exp(m_blk - m_run) < lambda for
 * every row of the query tile, where m_blk is the row's max score inside the
 * block and m_run the row's running max over the blocks already computed.
 * Readings taken where the pages are silent (listed with reasons in the
 * design notes of the repository):
 *   - scores are s = scale * q.k (natural units); the test is strict;
 *   - a row with no valid key in the block votes "negligible";
 *   - a skipped block adds nothing at all: not to m, not to l, not to O;
 *   - blocks are visited in ascending order; the first visited block of
 *     every query tile (block 0 unless a caller-supplied static block mask
 *     excludes it) and the first block of every decode split are always
 *     computed;
 *   - a block excluded by the static block mask is not visited at all: no
 *     scores, no vote, nothing added (the static block-sparse attention that
 *     a pre-pass selector would feed);
 *   - causal masking is bottom-right aligned: key j is visible from query
 *     row i when j <= i + (Lkv - Lq);
 *   - GQA maps query head hq to KV head hq / (Hq / Hkv);
 *   - decode splits restart the running statistics at each split and are
 *     combined by a log-sum-exp merge.
 *
 * Everything is computed in double. Inputs may be bf16 bit patterns, fp32 or
 * fp64 and are widened exactly.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { OR_BF16 = 0, OR_FP32 = 1, OR_FP64 = 2 };
enum { MASK_COMPUTED = 0, MASK_SKIPPED = 1, MASK_NOT_VISITED = 2 };

static double widen(const void *p, int dtype, int64_t i) {
  if (dtype == OR_BF16) {
    uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
  }
  if (dtype == OR_FP32) return (double)((const float *)p)[i];
  return ((const double *)p)[i];
}

static int resolve_threads(int n) {
  if (n > 0) return n;
  long c = sysconf(_SC_NPROCESSORS_ONLN);
  return c > 0 ? (int)c : 1;
}

/* ------------------------------------------------------------------------ */
/* Prefill: one query tile of Br rows against the KV blocks of its head.     */
/* ------------------------------------------------------------------------ */

typedef struct {
  const void *q, *k, *v;
  int dtype;
  int64_t B, Hq, Hkv, Lq, Lkv, d;
  int causal;
  double lambda;
  int64_t Br, Bc;
  double scale;
  /* Reference point for the exponentials (shift invariance, [T] para 2/4):
   *   0 - the running max itself (plain online softmax);
   *   1 - lazy: the reference is moved to the running max only when the max
   *       has grown past it by more than ref_param;
   *   2 - fixed: the reference is the constant ref_param for the whole pass.
   * The skip test always uses the exact running max. */
  int ref_mode;
  double ref_param;
  const int64_t *items; /* flat tile ids (b*Hq + hq)*nQt + qt, or NULL = all */
  int64_t n_items;
  /* Optional static block mask [B, Hq, nQt, nKt]: nonzero = the (query tile,
   * KV block) pair is excluded before any computation; NULL = none. */
  const uint8_t *static_mask;
  /* Outputs, one slot per listed item (item order):
   *   o      [n_items, Br, d]
   *   lse    [n_items, Br]       natural log; -inf for rows without keys
   *   mask   [n_items, nKt]      0 computed, 1 skipped, 2 not visited
   *   margin [n_items, nKt]      mu = max over rows of (m_blk - m_run),
   *                              natural units; NaN where not visited
   * Rows beyond Lq in a ragged last tile are left at 0. */
  double *o, *lse;
  uint8_t *mask;
  double *margin;
  int nthreads;
} oracle_prefill_args;

typedef struct {
  const oracle_prefill_args *a;
  int64_t next; /* shared work counter */
  pthread_mutex_t mu;
} prefill_ctx;

static void prefill_tile(const oracle_prefill_args *a, int64_t slot,
                         int64_t item, double *qrow, double *kblk,
                         double *vblk, double *s, double *m, double *mref,
                         double *l, double *acc, double *mb) {
  const int64_t d = a->d, Br = a->Br, Bc = a->Bc;
  const int64_t nQt = (a->Lq + Br - 1) / Br, nKt = (a->Lkv + Bc - 1) / Bc;
  const int64_t g = a->Hq / a->Hkv;
  const int64_t qt = item % nQt, bh = item / nQt;
  const int64_t hq = bh % a->Hq, b = bh / a->Hq, hk = hq / g;
  const int64_t r0 = qt * Br;
  const int64_t r1 = r0 + Br < a->Lq ? r0 + Br : a->Lq;
  const int64_t nr = r1 - r0;
  const int64_t off = a->Lkv - a->Lq; /* bottom-right causal alignment */
  const double log_lambda = a->lambda > 0.0 ? log(a->lambda) : -INFINITY;

  /* Last KV block that holds a key visible from some row of the tile. */
  int64_t kt_last = nKt - 1;
  if (a->causal) {
    int64_t last_key = (r1 - 1) + off;
    if (last_key < 0) kt_last = -1;
    else if (last_key / Bc < kt_last) kt_last = last_key / Bc;
  }

  const int64_t qbase = ((b * a->Hq + hq) * a->Lq) * d;
  const int64_t kvbase = ((b * a->Hkv + hk) * a->Lkv) * d;
  for (int64_t r = 0; r < nr; ++r)
    for (int64_t x = 0; x < d; ++x)
      qrow[r * d + x] = widen(a->q, a->dtype, qbase + (r0 + r) * d + x);

  for (int64_t r = 0; r < Br; ++r) {
    m[r] = -INFINITY;
    mref[r] = -INFINITY;
    l[r] = 0.0;
    for (int64_t x = 0; x < d; ++x) acc[r * d + x] = 0.0;
  }

  uint8_t *mask = a->mask ? a->mask + slot * nKt : NULL;
  double *margin = a->margin ? a->margin + slot * nKt : NULL;
  const uint8_t *smask = a->static_mask ? a->static_mask + item * nKt : NULL;
  int visited_before = 0;

  /* [T] para 2: KV blocks are walked left to right. */
  for (int64_t kt = 0; kt < nKt; ++kt) {
    if (kt > kt_last || (smask && smask[kt])) {
      if (mask) mask[kt] = MASK_NOT_VISITED;
      if (margin) margin[kt] = NAN;
      continue;
    }
    const int64_t c0 = kt * Bc;
    const int64_t c1 = c0 + Bc < a->Lkv ? c0 + Bc : a->Lkv;
    const int64_t nc = c1 - c0;
    for (int64_t j = 0; j < nc; ++j)
      for (int64_t x = 0; x < d; ++x) {
        kblk[j * d + x] = widen(a->k, a->dtype, kvbase + (c0 + j) * d + x);
        vblk[j * d + x] = widen(a->v, a->dtype, kvbase + (c0 + j) * d + x);
      }

    /* Scores and the block's row max m_blk (the QK product is always
     * formed: the block max cannot be known otherwise). */
    double mu = -INFINITY;
    for (int64_t r = 0; r < nr; ++r) {
      mb[r] = -INFINITY;
      for (int64_t j = 0; j < nc; ++j) {
        int valid = !a->causal || (c0 + j) <= (r0 + r) + off;
        double sv = -INFINITY;
        if (valid) {
          double dot = 0.0;
          for (int64_t x = 0; x < d; ++x) dot += qrow[r * d + x] * kblk[j * d + x];
          sv = a->scale * dot;
        }
        s[r * Bc + j] = sv;
        if (sv > mb[r]) mb[r] = sv;
      }
      /* Row's distance to its running max; conventions for empty rows:
       * a row with no valid key here votes "negligible" (-inf); a row that
       * has seen no key yet but has one here is "not negligible" (+inf). */
      double dr;
      if (mb[r] == -INFINITY) dr = -INFINITY;
      else if (m[r] == -INFINITY) dr = INFINITY;
      else dr = mb[r] - m[r];
      if (dr > mu) mu = dr;
    }

    /* [T] para 5 + [D]: skip when exp(m_blk - m_run) < lambda on every row,
     * i.e. max_r (m_blk - m_run) < ln(lambda). [T] para 6: never the first
     * visited block. */
    int skip = visited_before && (a->lambda > 0.0) && (mu < log_lambda);
    visited_before = 1;
    if (mask) mask[kt] = skip ? MASK_SKIPPED : MASK_COMPUTED;
    if (margin) margin[kt] = mu;
    if (skip) continue; /* no V, no exp, no update of m, l or O */

    /* [T] para 3: online softmax update with rescaling of earlier partials. */
    for (int64_t r = 0; r < nr; ++r) {
      if (mb[r] == -INFINITY) continue; /* nothing visible in this block */
      double m_new = mb[r] > m[r] ? mb[r] : m[r];
      double ref_new;
      if (a->ref_mode == 2) ref_new = a->ref_param;
      else if (a->ref_mode == 1)
        ref_new = (mref[r] == -INFINITY || m_new > mref[r] + a->ref_param)
                      ? m_new : mref[r];
      else ref_new = m_new;
      double alpha = (mref[r] == -INFINITY) ? 0.0 : exp(mref[r] - ref_new);
      if (mref[r] == ref_new) alpha = 1.0;
      l[r] *= alpha;
      for (int64_t x = 0; x < d; ++x) acc[r * d + x] *= alpha;
      for (int64_t j = 0; j < nc; ++j) {
        double sv = s[r * Bc + j];
        if (sv == -INFINITY) continue;
        double p = exp(sv - ref_new);
        l[r] += p;
        for (int64_t x = 0; x < d; ++x) acc[r * d + x] += p * vblk[j * d + x];
      }
      m[r] = m_new;
      mref[r] = ref_new;
    }
  }

  /* Final normalisation; lse in natural log. */
  for (int64_t r = 0; r < nr; ++r) {
    double *orow = a->o ? a->o + (slot * Br + r) * d : NULL;
    if (l[r] > 0.0) {
      if (orow) for (int64_t x = 0; x < d; ++x) orow[x] = acc[r * d + x] / l[r];
      if (a->lse) a->lse[slot * Br + r] = mref[r] + log(l[r]);
    } else {
      if (orow) for (int64_t x = 0; x < d; ++x) orow[x] = 0.0;
      if (a->lse) a->lse[slot * Br + r] = -INFINITY;
    }
  }
  for (int64_t r = nr; r < Br; ++r) {
    if (a->o) for (int64_t x = 0; x < d; ++x) a->o[(slot * Br + r) * d + x] = 0.0;
    if (a->lse) a->lse[slot * Br + r] = 0.0;
  }
}

static void *prefill_worker(void *p) {
  prefill_ctx *ctx = (prefill_ctx *)p;
  const oracle_prefill_args *a = ctx->a;
  const int64_t d = a->d, Br = a->Br, Bc = a->Bc;
  double *qrow = malloc(sizeof(double) * Br * d);
  double *kblk = malloc(sizeof(double) * Bc * d);
  double *vblk = malloc(sizeof(double) * Bc * d);
  double *s = malloc(sizeof(double) * Br * Bc);
  double *acc = malloc(sizeof(double) * Br * d);
  double *st = malloc(sizeof(double) * Br * 4);
  if (!qrow || !kblk || !vblk || !s || !acc || !st) goto out;
  for (;;) {
    pthread_mutex_lock(&ctx->mu);
    int64_t slot = ctx->next++;
    pthread_mutex_unlock(&ctx->mu);
    if (slot >= a->n_items) break;
    int64_t item = a->items ? a->items[slot] : slot;
    prefill_tile(a, slot, item, qrow, kblk, vblk, s, st, st + Br, st + 2 * Br,
                 acc, st + 3 * Br);
  }
out:
  free(qrow); free(kblk); free(vblk); free(s); free(acc); free(st);
  return NULL;
}

int oracle_prefill(oracle_prefill_args *a) {
  if (!a || a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv ||
      a->Lq <= 0 || a->Lkv <= 0 || a->d <= 0 || a->Br <= 0 || a->Bc <= 0 ||
      a->lambda < 0.0 || a->lambda >= 1.0)
    return -1;
  const int64_t nQt = (a->Lq + a->Br - 1) / a->Br;
  if (!a->items) a->n_items = a->B * a->Hq * nQt;
  prefill_ctx ctx;
  ctx.a = a;
  ctx.next = 0;
  pthread_mutex_init(&ctx.mu, NULL);
  int nt = resolve_threads(a->nthreads);
  if (nt > a->n_items) nt = (int)a->n_items;
  if (nt < 1) nt = 1;
  if (nt > 512) nt = 512;
  pthread_t th[512];
  int ok[512];
  for (int t = 0; t < nt; ++t) ok[t] = pthread_create(&th[t], NULL, prefill_worker, &ctx) == 0;
  for (int t = 0; t < nt; ++t) if (ok[t]) pthread_join(th[t], NULL);
  /* Should every thread creation have failed, run inline. */
  int any = 0;
  for (int t = 0; t < nt; ++t) any |= ok[t];
  if (!any) prefill_worker(&ctx);
  pthread_mutex_destroy(&ctx.mu);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode: one query row per head, KV split into chunks, each chunk a pass   */
/* of its own (running statistics restart), then a log-sum-exp merge.        */
/* ------------------------------------------------------------------------ */

typedef struct {
  const void *q, *k, *v; /* q [B,Hq,1,d]; k, v [B,Hkv,Lkv,d] */
  int dtype;
  int64_t B, Hq, Hkv, Lkv, d;
  double lambda;
  int64_t Bc, num_splits;
  double scale;
  double *o_parts;   /* [B,Hq,S,d] normalised per split (0 for empty splits) */
  double *lse_parts; /* [B,Hq,S] (-inf for empty splits) */
  uint8_t *mask;     /* [B,Hq,nKt] */
  double *margin;    /* [B,Hq,nKt] */
  double *o, *lse;   /* merged: [B,Hq,d], [B,Hq] */
  int nthreads;
} oracle_decode_args;

/* Keys per split: ceil(Lkv / S) rounded up to a whole number of blocks. */
int64_t oracle_split_len(int64_t Lkv, int64_t Bc, int64_t S) {
  int64_t per = (Lkv + S - 1) / S;
  return ((per + Bc - 1) / Bc) * Bc;
}

void oracle_lse_merge(const double *o_parts, const double *lse_parts,
                      int64_t n_rows, int64_t S, int64_t d, double *o,
                      double *lse) {
  for (int64_t r = 0; r < n_rows; ++r) {
    double M = -INFINITY;
    for (int64_t s = 0; s < S; ++s)
      if (lse_parts[r * S + s] > M) M = lse_parts[r * S + s];
    double wsum = 0.0;
    for (int64_t x = 0; x < d; ++x) o[r * d + x] = 0.0;
    if (M == -INFINITY) { lse[r] = -INFINITY; continue; }
    for (int64_t s = 0; s < S; ++s) {
      double ls = lse_parts[r * S + s];
      double w = (ls == -INFINITY) ? 0.0 : exp(ls - M);
      wsum += w;
      for (int64_t x = 0; x < d; ++x) o[r * d + x] += w * o_parts[(r * S + s) * d + x];
    }
    for (int64_t x = 0; x < d; ++x) o[r * d + x] /= wsum;
    lse[r] = M + log(wsum);
  }
}

typedef struct {
  const oracle_decode_args *a;
  int64_t next;
  pthread_mutex_t mu;
} decode_ctx;

static void decode_row_split(const oracle_decode_args *a, int64_t bh, int64_t sp,
                             const double *qv, double *kv_k, double *kv_v,
                             double *s, double *acc) {
  const int64_t d = a->d, Bc = a->Bc, S = a->num_splits;
  const int64_t nKt = (a->Lkv + Bc - 1) / Bc;
  const int64_t g = a->Hq / a->Hkv;
  const int64_t hq = bh % a->Hq, b = bh / a->Hq, hk = hq / g;
  const int64_t Ls = oracle_split_len(a->Lkv, Bc, S);
  const int64_t k0 = sp * Ls;
  const int64_t k1 = k0 + Ls < a->Lkv ? k0 + Ls : a->Lkv;
  const int64_t kvbase = ((b * a->Hkv + hk) * a->Lkv) * d;
  const double log_lambda = a->lambda > 0.0 ? log(a->lambda) : -INFINITY;
  double m = -INFINITY, l = 0.0;
  for (int64_t x = 0; x < d; ++x) acc[x] = 0.0;
  for (int64_t c0 = k0; c0 < k1; c0 += Bc) {
    const int64_t kt = c0 / Bc;
    const int64_t c1 = c0 + Bc < k1 ? c0 + Bc : k1;
    const int64_t nc = c1 - c0;
    double mb = -INFINITY;
    for (int64_t j = 0; j < nc; ++j) {
      double dot = 0.0;
      for (int64_t x = 0; x < d; ++x) {
        kv_k[j * d + x] = widen(a->k, a->dtype, kvbase + (c0 + j) * d + x);
        dot += qv[x] * kv_k[j * d + x];
      }
      s[j] = a->scale * dot;
      if (s[j] > mb) mb = s[j];
    }
    double mu = (m == -INFINITY) ? INFINITY : mb - m;
    /* The first block of every split is always computed: the split starts
     * its own pass with no running max. */
    int skip = (c0 > k0) && (a->lambda > 0.0) && (mu < log_lambda);
    if (a->mask) a->mask[bh * nKt + kt] = skip ? MASK_SKIPPED : MASK_COMPUTED;
    if (a->margin) a->margin[bh * nKt + kt] = mu;
    if (skip) continue;
    for (int64_t j = 0; j < nc; ++j)
      for (int64_t x = 0; x < d; ++x)
        kv_v[j * d + x] = widen(a->v, a->dtype, kvbase + (c0 + j) * d + x);
    double m_new = mb > m ? mb : m;
    double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
    l *= alpha;
    for (int64_t x = 0; x < d; ++x) acc[x] *= alpha;
    for (int64_t j = 0; j < nc; ++j) {
      double p = exp(s[j] - m_new);
      l += p;
      for (int64_t x = 0; x < d; ++x) acc[x] += p * kv_v[j * d + x];
    }
    m = m_new;
  }
  double *op = a->o_parts + (bh * S + sp) * d;
  if (l > 0.0) {
    for (int64_t x = 0; x < d; ++x) op[x] = acc[x] / l;
    a->lse_parts[bh * S + sp] = m + log(l);
  } else {
    for (int64_t x = 0; x < d; ++x) op[x] = 0.0;
    a->lse_parts[bh * S + sp] = -INFINITY;
  }
}

static void *decode_worker(void *p) {
  decode_ctx *ctx = (decode_ctx *)p;
  const oracle_decode_args *a = ctx->a;
  const int64_t d = a->d, Bc = a->Bc, S = a->num_splits;
  double *qv = malloc(sizeof(double) * d);
  double *kk = malloc(sizeof(double) * Bc * d);
  double *vv = malloc(sizeof(double) * Bc * d);
  double *s = malloc(sizeof(double) * Bc);
  double *acc = malloc(sizeof(double) * d);
  const int64_t total = a->B * a->Hq * S;
  if (!qv || !kk || !vv || !s || !acc) goto out;
  for (;;) {
    pthread_mutex_lock(&ctx->mu);
    int64_t job = ctx->next++;
    pthread_mutex_unlock(&ctx->mu);
    if (job >= total) break;
    int64_t bh = job / S, sp = job % S;
    for (int64_t x = 0; x < d; ++x) qv[x] = widen(a->q, a->dtype, bh * d + x);
    decode_row_split(a, bh, sp, qv, kk, vv, s, acc);
  }
out:
  free(qv); free(kk); free(vv); free(s); free(acc);
  return NULL;
}

int oracle_decode(oracle_decode_args *a) {
  if (!a || a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv ||
      a->Lkv <= 0 || a->d <= 0 || a->Bc <= 0 || a->num_splits <= 0 ||
      a->lambda < 0.0 || a->lambda >= 1.0 || !a->o_parts || !a->lse_parts)
    return -1;
  const int64_t nKt = (a->Lkv + a->Bc - 1) / a->Bc;
  if (a->mask) memset(a->mask, MASK_NOT_VISITED, (size_t)(a->B * a->Hq * nKt));
  decode_ctx ctx;
  ctx.a = a;
  ctx.next = 0;
  pthread_mutex_init(&ctx.mu, NULL);
  int64_t total = a->B * a->Hq * a->num_splits;
  int nt = resolve_threads(a->nthreads);
  if (nt > total) nt = (int)total;
  if (nt > 512) nt = 512;
  pthread_t th[512];
  int ok[512], any = 0;
  for (int t = 0; t < nt; ++t) { ok[t] = pthread_create(&th[t], NULL, decode_worker, &ctx) == 0; any |= ok[t]; }
  for (int t = 0; t < nt; ++t) if (ok[t]) pthread_join(th[t], NULL);
  if (!any) decode_worker(&ctx);
  pthread_mutex_destroy(&ctx.mu);
  if (a->o && a->lse)
    oracle_lse_merge(a->o_parts, a->lse_parts, a->B * a->Hq, a->num_splits, a->d,
                     a->o, a->lse);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Backward pass with the forward's decisions held fixed.                    */
/* ------------------------------------------------------------------------ */
/*
 * With the skip decisions of a forward pass held constant, its output is
 * softmax attention over the kept keys of each row ([T] para 5: a dropped
 * block contributes nothing), so the gradient of a loss L(O) is the one of
 * that restricted attention. Written out from the definitions, per query
 * row i with kept key set K_i and s_ij = scale * q_i . k_j:
 *   P_ij  = exp(s_ij - lse_i) for j in K_i, else 0, lse_i = ln sum_K_i exp(s_ij)
 *   O_i   = sum_j P_ij v_j
 *   dP_ij = dO_i . v_j,   D_i = sum_j P_ij dP_ij  (= dO_i . O_i)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i,   dV_j = sum_i P_ij dO_i
 * (summed over the query heads that share a KV head). The kept set comes
 * from a tile mask in the layout of the forward's skip mask: a (query tile,
 * KV block) pair is kept when its entry is 0; NULL keeps every causally
 * visible key. Everything in double.
 */
typedef struct {
  const void *q, *k, *v, *dout;
  int dtype;
  int64_t B, Hq, Hkv, Lq, Lkv, d;
  int causal;
  int64_t Br, Bc;
  double scale;
  const uint8_t *tile_mask; /* [B, Hq, nQt, nKt], 0 = kept; NULL = all visible kept */
  double *dq;               /* [B, Hq, Lq, d] */
  double *dk, *dv;          /* [B, Hkv, Lkv, d] */
  int nthreads;
} oracle_backward_args;

typedef struct {
  const oracle_backward_args *a;
  int64_t next;
  pthread_mutex_t mu;
} backward_ctx;

/* One query row i of head (b, hq): writes dq_i (d values) and adds the
 * row's terms to dk and dv for the keys in [key_lo, key_hi) (dk_acc[j -
 * key_lo], dv_acc[j - key_lo]; NULL adds nothing). Scratch: qi, doi [d];
 * s, p, ds [Lkv]. */
static void backward_row(const oracle_backward_args *a, int64_t b, int64_t hq, int64_t i,
                         double *qi, double *doi, double *s, double *p, double *ds, double *dqi,
                         double *dk_acc, double *dv_acc, int64_t key_lo, int64_t key_hi) {
  const int64_t d = a->d, Lq = a->Lq, Lkv = a->Lkv, g = a->Hq / a->Hkv;
  const int64_t nQt = (Lq + a->Br - 1) / a->Br, nKt = (Lkv + a->Bc - 1) / a->Bc;
  const int64_t off = Lkv - Lq;
  const int64_t hk = hq / g;
  const int64_t kvbase = ((b * a->Hkv + hk) * Lkv) * d;
  const int64_t qbase = ((b * a->Hq + hq) * Lq) * d;
  for (int64_t x = 0; x < d; ++x) {
    qi[x] = widen(a->q, a->dtype, qbase + i * d + x);
    doi[x] = widen(a->dout, a->dtype, qbase + i * d + x);
  }
  const int64_t qt = i / a->Br;
  double mx = -INFINITY;
  for (int64_t j = 0; j < Lkv; ++j) {
    int kept = !a->causal || j <= i + off;
    if (kept && a->tile_mask)
      kept = a->tile_mask[((b * a->Hq + hq) * nQt + qt) * nKt + j / a->Bc] == 0;
    double sv = -INFINITY;
    if (kept) {
      double dot = 0.0;
      for (int64_t x = 0; x < d; ++x) dot += qi[x] * widen(a->k, a->dtype, kvbase + j * d + x);
      sv = a->scale * dot;
    }
    s[j] = sv;
    if (sv > mx) mx = sv;
  }
  for (int64_t x = 0; x < d; ++x) dqi[x] = 0.0;
  if (mx == -INFINITY) return; /* no kept key: O = 0, no gradient */
  double sum = 0.0;
  for (int64_t j = 0; j < Lkv; ++j) sum += s[j] == -INFINITY ? 0.0 : exp(s[j] - mx);
  const double lse = mx + log(sum);
  double D = 0.0;
  for (int64_t j = 0; j < Lkv; ++j) {
    p[j] = s[j] == -INFINITY ? 0.0 : exp(s[j] - lse);
    double dp = 0.0;
    if (p[j] != 0.0)
      for (int64_t x = 0; x < d; ++x) dp += doi[x] * widen(a->v, a->dtype, kvbase + j * d + x);
    ds[j] = dp; /* dP for now */
    D += p[j] * dp;
  }
  for (int64_t j = 0; j < Lkv; ++j) {
    if (p[j] == 0.0) continue;
    const double dsj = p[j] * (ds[j] - D);
    const int in_range = dk_acc && j >= key_lo && j < key_hi;
    double *dkj = in_range ? dk_acc + (j - key_lo) * d : NULL;
    double *dvj = in_range ? dv_acc + (j - key_lo) * d : NULL;
    for (int64_t x = 0; x < d; ++x) {
      dqi[x] += a->scale * dsj * widen(a->k, a->dtype, kvbase + j * d + x);
      if (in_range) {
        dkj[x] += a->scale * dsj * qi[x];
        dvj[x] += p[j] * doi[x];
      }
    }
  }
}

/* One (b, hk) unit: every query head of the group, every row. */
static void backward_unit(const oracle_backward_args *a, int64_t unit, double *qi,
                          double *doi, double *s, double *p, double *ds) {
  const int64_t d = a->d, Lq = a->Lq, Lkv = a->Lkv, g = a->Hq / a->Hkv;
  const int64_t b = unit / a->Hkv, hk = unit % a->Hkv;
  const int64_t kvbase = ((b * a->Hkv + hk) * Lkv) * d;
  for (int64_t hh = 0; hh < g; ++hh) {
    const int64_t hq = hk * g + hh;
    const int64_t qbase = ((b * a->Hq + hq) * Lq) * d;
    for (int64_t i = 0; i < Lq; ++i)
      backward_row(a, b, hq, i, qi, doi, s, p, ds, a->dq + qbase + i * d, a->dk + kvbase,
                   a->dv + kvbase, 0, Lkv);
  }
}

static void *backward_worker(void *vp) {
  backward_ctx *ctx = (backward_ctx *)vp;
  const oracle_backward_args *a = ctx->a;
  double *qi = malloc(sizeof(double) * a->d);
  double *doi = malloc(sizeof(double) * a->d);
  double *s = malloc(sizeof(double) * a->Lkv);
  double *p = malloc(sizeof(double) * a->Lkv);
  double *ds = malloc(sizeof(double) * a->Lkv);
  if (!qi || !doi || !s || !p || !ds) goto out;
  for (;;) {
    pthread_mutex_lock(&ctx->mu);
    int64_t unit = ctx->next++;
    pthread_mutex_unlock(&ctx->mu);
    if (unit >= a->B * a->Hkv) break;
    backward_unit(a, unit, qi, doi, s, p, ds);
  }
out:
  free(qi); free(doi); free(s); free(p); free(ds);
  return NULL;
}

int oracle_backward(oracle_backward_args *a) {
  if (!a || a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv || a->Lq <= 0 ||
      a->Lkv <= 0 || a->d <= 0 || a->Br <= 0 || a->Bc <= 0 || !a->dq || !a->dk || !a->dv)
    return -1;
  memset(a->dk, 0, sizeof(double) * (size_t)(a->B * a->Hkv * a->Lkv * a->d));
  memset(a->dv, 0, sizeof(double) * (size_t)(a->B * a->Hkv * a->Lkv * a->d));
  backward_ctx ctx;
  ctx.a = a;
  ctx.next = 0;
  pthread_mutex_init(&ctx.mu, NULL);
  int64_t total = a->B * a->Hkv;
  int nt = resolve_threads(a->nthreads);
  if (nt > total) nt = (int)total;
  if (nt > 512) nt = 512;
  pthread_t th[512];
  int ok[512], any = 0;
  for (int t = 0; t < nt; ++t) { ok[t] = pthread_create(&th[t], NULL, backward_worker, &ctx) == 0; any |= ok[t]; }
  for (int t = 0; t < nt; ++t) if (ok[t]) pthread_join(th[t], NULL);
  if (!any) backward_worker(&ctx);
  pthread_mutex_destroy(&ctx.mu);
  return 0;
}

/* Sampled rows of the backward pass (for problems too large for the full
 * one): dq of the listed query rows (flat ids (b*Hq + hq)*Lq + i), and the
 * terms those rows add to dk and dv of the keys [key_lo, key_hi) of KV head
 * (kv_b, kv_h). When the listed rows include every row that keeps one of
 * those keys (e.g. the last rows of every head of the group for the last
 * keys under a causal mask), those dk and dv rows are complete. */
typedef struct {
  oracle_backward_args base; /* dq, dk, dv, nthreads of base unused */
  int64_t n_rows;
  const int64_t *rows;
  double *dq_rows;        /* [n_rows, d] */
  int64_t kv_b, kv_h, key_lo, key_hi;
  double *dk_part, *dv_part; /* [key_hi - key_lo, d], overwritten */
  int nthreads;
} oracle_backward_rows_args;

typedef struct {
  const oracle_backward_rows_args *a;
  int64_t next;
  pthread_mutex_t mu;
  double *acc; /* per-thread dk/dv partials: [nt][2][nk * d] */
  int64_t nk;
} rows_ctx;

typedef struct {
  rows_ctx *ctx;
  int t;
} rows_worker_arg;

static void *backward_rows_worker(void *vp) {
  rows_worker_arg *wa = (rows_worker_arg *)vp;
  rows_ctx *ctx = wa->ctx;
  const oracle_backward_rows_args *a = ctx->a;
  const oracle_backward_args *ba = &a->base;
  const int64_t d = ba->d, g = ba->Hq / ba->Hkv;
  double *dk_acc = ctx->acc + (int64_t)wa->t * 2 * ctx->nk * d;
  double *dv_acc = dk_acc + ctx->nk * d;
  double *qi = malloc(sizeof(double) * d);
  double *doi = malloc(sizeof(double) * d);
  double *s = malloc(sizeof(double) * ba->Lkv);
  double *p = malloc(sizeof(double) * ba->Lkv);
  double *ds = malloc(sizeof(double) * ba->Lkv);
  if (!qi || !doi || !s || !p || !ds) goto out;
  for (;;) {
    pthread_mutex_lock(&ctx->mu);
    int64_t r = ctx->next++;
    pthread_mutex_unlock(&ctx->mu);
    if (r >= a->n_rows) break;
    const int64_t id = a->rows[r];
    const int64_t bh = id / ba->Lq, i = id % ba->Lq;
    const int64_t b = bh / ba->Hq, hq = bh % ba->Hq;
    const int mine = ctx->nk > 0 && b == a->kv_b && hq / g == a->kv_h;
    backward_row(ba, b, hq, i, qi, doi, s, p, ds, a->dq_rows + r * d, mine ? dk_acc : NULL,
                 mine ? dv_acc : NULL, a->key_lo, a->key_hi);
  }
out:
  free(qi); free(doi); free(s); free(p); free(ds);
  return NULL;
}

int oracle_backward_rows(oracle_backward_rows_args *a) {
  const oracle_backward_args *ba = a ? &a->base : NULL;
  if (!a || ba->B <= 0 || ba->Hq <= 0 || ba->Hkv <= 0 || ba->Hq % ba->Hkv || ba->Lq <= 0 ||
      ba->Lkv <= 0 || ba->d <= 0 || ba->Br <= 0 || ba->Bc <= 0 || a->n_rows < 0 ||
      (a->n_rows > 0 && (!a->rows || !a->dq_rows)))
    return -1;
  for (int64_t r = 0; r < a->n_rows; ++r)
    if (a->rows[r] < 0 || a->rows[r] >= ba->B * ba->Hq * ba->Lq) return -1;
  int64_t nk = a->key_hi - a->key_lo;
  if (nk < 0 || a->key_lo < 0 || a->key_hi > ba->Lkv) return -1;
  if (nk > 0 && (!a->dk_part || !a->dv_part)) return -1;
  int nt = resolve_threads(a->nthreads);
  if (nt > 512) nt = 512;
  if (a->n_rows > 0 && nt > a->n_rows) nt = (int)a->n_rows;
  if (nt < 1) nt = 1;
  rows_ctx ctx;
  ctx.a = a;
  ctx.next = 0;
  ctx.nk = nk;
  pthread_mutex_init(&ctx.mu, NULL);
  ctx.acc = calloc((size_t)nt * 2 * (size_t)(nk > 0 ? nk : 1) * (size_t)ba->d, sizeof(double));
  if (!ctx.acc) {
    pthread_mutex_destroy(&ctx.mu);
    return -2;
  }
  pthread_t th[512];
  rows_worker_arg wa[512];
  int ok[512], any = 0;
  for (int t = 0; t < nt; ++t) {
    wa[t].ctx = &ctx;
    wa[t].t = t;
    ok[t] = pthread_create(&th[t], NULL, backward_rows_worker, &wa[t]) == 0;
    any |= ok[t];
  }
  for (int t = 0; t < nt; ++t) if (ok[t]) pthread_join(th[t], NULL);
  if (!any) backward_rows_worker(&wa[0]);
  if (nk > 0) {
    const int64_t n = nk * ba->d;
    for (int64_t e = 0; e < n; ++e) {
      double sk = 0.0, sv = 0.0;
      for (int t = 0; t < nt; ++t) {
        sk += ctx.acc[(int64_t)t * 2 * n + e];
        sv += ctx.acc[(int64_t)t * 2 * n + n + e];
      }
      a->dk_part[e] = sk;
      a->dv_part[e] = sv;
    }
  }
  free(ctx.acc);
  pthread_mutex_destroy(&ctx.mu);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Pre-pass block selector (the block-sparse input the forward can take).    */
/* ------------------------------------------------------------------------ */
/*
 * [C] the CRISP review (rit.work, blog/crisp-sparse-attention-long-prefill),
 *     section "What was done" (Что сделали), paragraphs 3-5:
 *       - the selector works from an approximate attention map that is
 *         already computed (FlexPrefill's pooled estimate);
 *       - C_struct is the share of that map on the initial positions and
 *         the local window; it routes each head to the structured
 *         (Vertical-Slash) path or to the pooled path;
 *       - on the structured path the first and the last block are always
 *         kept, the mean background mass is taken over the other blocks and
 *         the blocks above it are selected;
 *       - on the pooled path the cumulative rule stays: blocks are added
 *         until together they cover a given share of the attention.
 * Readings (the page gives no formulas or constants):
 *   - the map is the block-pooled estimate: per head, q_t = mean of the
 *     query rows of tile t, k_j = mean of the keys of block j, and
 *     A[t][j] = softmax over the blocks j visible from tile t of
 *     scale * q_t . k_j (visible: under a causal mask, j up to the block of
 *     the tile's last row, bottom-right aligned);
 *   - "last block" and "local window" = the tile's last visible block;
 *     "initial positions" = block 0;
 *   - C_struct = the mean over the head's tiles of A[t][0] + A[t][last(t)]
 *     (A[t][0] once when the two coincide); structured when C_struct >= tau;
 *   - structured: keep 0 and last(t); background = mean of A[t][j] over the
 *     other visible blocks; keep those with A[t][j] > background (strict);
 *   - pooled: order the visible blocks by A descending (ties by index),
 *     take the shortest prefix whose sum reaches gamma, theta = the last
 *     value taken, keep every visible block with A[t][j] >= theta;
 *   - output: uint8 mask [B, Hq, nQt, nKt], 0 = selected, 1 = not selected
 *     (causally invisible blocks are 1), the static-mask convention.
 */
typedef struct {
  const void *q, *k;
  int dtype;
  int64_t B, Hq, Hkv, Lq, Lkv, d;
  int causal;
  int64_t Br, Bc;
  double scale, tau, gamma;
  uint8_t *mask_out;    /* [B, Hq, nQt, nKt] */
  double *cstruct_out;  /* [B, Hq] or NULL */
  double *amap_out;     /* [B, Hq, nQt, nKt] or NULL; NaN where not visible */
  int nthreads;
} oracle_select_args;

typedef struct {
  const oracle_select_args *a;
  int64_t next;
  pthread_mutex_t mu;
} select_ctx;

static int64_t select_last_block(const oracle_select_args *a, int64_t t) {
  const int64_t nKt = (a->Lkv + a->Bc - 1) / a->Bc;
  if (!a->causal) return nKt - 1;
  int64_t r1 = (t + 1) * a->Br;
  if (r1 > a->Lq) r1 = a->Lq;
  int64_t jl = (r1 - 1 + (a->Lkv - a->Lq)) / a->Bc;
  return jl < nKt - 1 ? jl : nKt - 1;
}

typedef struct {
  double v;
  int64_t j;
} select_item;

static int select_cmp(const void *x, const void *y) {
  const select_item *a = (const select_item *)x, *b = (const select_item *)y;
  if (a->v != b->v) return a->v > b->v ? -1 : 1;
  return a->j < b->j ? -1 : (a->j > b->j ? 1 : 0);
}

/* One (b, hq): the pooled map, C_struct, the route and every tile's blocks. */
static void select_head(const oracle_select_args *a, int64_t bh, double *qbar, double *kbar,
                        double *amap, select_item *order) {
  const int64_t d = a->d, Lq = a->Lq, Lkv = a->Lkv;
  const int64_t nQt = (Lq + a->Br - 1) / a->Br, nKt = (Lkv + a->Bc - 1) / a->Bc;
  const int64_t b = bh / a->Hq, hq = bh % a->Hq, hk = hq / (a->Hq / a->Hkv);
  const int64_t qbase = bh * Lq * d, kbase = (b * a->Hkv + hk) * Lkv * d;
  /* pooled rows */
  for (int64_t t = 0; t < nQt; ++t) {
    const int64_t r0 = t * a->Br, r1 = (t + 1) * a->Br < Lq ? (t + 1) * a->Br : Lq;
    for (int64_t x = 0; x < d; ++x) {
      double acc = 0.0;
      for (int64_t i = r0; i < r1; ++i) acc += widen(a->q, a->dtype, qbase + i * d + x);
      qbar[t * d + x] = acc / (double)(r1 - r0);
    }
  }
  for (int64_t j = 0; j < nKt; ++j) {
    const int64_t c0 = j * a->Bc, c1 = (j + 1) * a->Bc < Lkv ? (j + 1) * a->Bc : Lkv;
    for (int64_t x = 0; x < d; ++x) {
      double acc = 0.0;
      for (int64_t i = c0; i < c1; ++i) acc += widen(a->k, a->dtype, kbase + i * d + x);
      kbar[j * d + x] = acc / (double)(c1 - c0);
    }
  }
  /* the map: softmax over visible blocks of scale * q_t . k_j */
  double cs = 0.0;
  for (int64_t t = 0; t < nQt; ++t) {
    const int64_t jl = select_last_block(a, t);
    double *row = amap + t * nKt;
    double mx = -INFINITY;
    for (int64_t j = 0; j < nKt; ++j) {
      if (j > jl) {
        row[j] = NAN;
        continue;
      }
      double dot = 0.0;
      for (int64_t x = 0; x < d; ++x) dot += qbar[t * d + x] * kbar[j * d + x];
      row[j] = a->scale * dot;
      if (row[j] > mx) mx = row[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j <= jl; ++j) {
      row[j] = exp(row[j] - mx);
      sum += row[j];
    }
    for (int64_t j = 0; j <= jl; ++j) row[j] /= sum;
    cs += row[0] + (jl > 0 ? row[jl] : 0.0);
  }
  cs /= (double)nQt;
  const int structured = cs >= a->tau;
  if (a->cstruct_out) a->cstruct_out[bh] = cs;
  /* per tile */
  for (int64_t t = 0; t < nQt; ++t) {
    const int64_t jl = select_last_block(a, t);
    const double *row = amap + t * nKt;
    uint8_t *m = a->mask_out + (bh * nQt + t) * nKt;
    for (int64_t j = 0; j < nKt; ++j) m[j] = 1;
    if (structured) {
      m[0] = 0;
      m[jl] = 0;
      if (jl >= 2) {
        double bg = 0.0;
        for (int64_t j = 1; j < jl; ++j) bg += row[j];
        bg /= (double)(jl - 1);
        for (int64_t j = 1; j < jl; ++j)
          if (row[j] > bg) m[j] = 0;
      }
    } else {
      /* descending by value, ties by index (library sort) */
      int64_t n = jl + 1;
      for (int64_t j = 0; j < n; ++j) {
        order[j].v = row[j];
        order[j].j = j;
      }
      qsort(order, (size_t)n, sizeof(select_item), select_cmp);
      double cum = 0.0, theta = order[0].v;
      for (int64_t r = 0; r < n; ++r) {
        cum += order[r].v;
        theta = order[r].v;
        if (cum >= a->gamma) break;
      }
      for (int64_t j = 0; j < n; ++j)
        if (row[j] >= theta) m[j] = 0;
    }
  }
  if (a->amap_out) memcpy(a->amap_out + bh * nQt * nKt, amap, sizeof(double) * nQt * nKt);
}

static void *select_worker(void *vp) {
  select_ctx *ctx = (select_ctx *)vp;
  const oracle_select_args *a = ctx->a;
  const int64_t nQt = (a->Lq + a->Br - 1) / a->Br, nKt = (a->Lkv + a->Bc - 1) / a->Bc;
  double *qbar = malloc(sizeof(double) * nQt * a->d);
  double *kbar = malloc(sizeof(double) * nKt * a->d);
  double *amap = malloc(sizeof(double) * nQt * nKt);
  select_item *order = malloc(sizeof(select_item) * nKt);
  if (!qbar || !kbar || !amap || !order) goto out;
  for (;;) {
    pthread_mutex_lock(&ctx->mu);
    int64_t bh = ctx->next++;
    pthread_mutex_unlock(&ctx->mu);
    if (bh >= a->B * a->Hq) break;
    select_head(a, bh, qbar, kbar, amap, order);
  }
out:
  free(qbar); free(kbar); free(amap); free(order);
  return NULL;
}

int oracle_select(oracle_select_args *a) {
  if (!a || a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->Hq % a->Hkv || a->Lq <= 0 ||
      a->Lkv <= 0 || a->d <= 0 || a->Br <= 0 || a->Bc <= 0 || !a->mask_out ||
      (a->causal && a->Lq > a->Lkv) || !(a->gamma > 0.0 && a->gamma <= 1.0))
    return -1;
  select_ctx ctx;
  ctx.a = a;
  ctx.next = 0;
  pthread_mutex_init(&ctx.mu, NULL);
  int64_t total = a->B * a->Hq;
  int nt = resolve_threads(a->nthreads);
  if (nt > total) nt = (int)total;
  if (nt > 512) nt = 512;
  pthread_t th[512];
  int ok[512], any = 0;
  for (int t = 0; t < nt; ++t) { ok[t] = pthread_create(&th[t], NULL, select_worker, &ctx) == 0; any |= ok[t]; }
  for (int t = 0; t < nt; ++t) if (ok[t]) pthread_join(th[t], NULL);
  if (!any) select_worker(&ctx);
  pthread_mutex_destroy(&ctx.mu);
  return 0;
}
