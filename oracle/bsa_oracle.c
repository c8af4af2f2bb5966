/*
 * bsa_oracle.c -- plain, slow, fp64 CPU oracle for block-sparse
 * variable-length attention (forward and backward).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or table with the CUDA library; it reads the raw block index itself.
 *
 * What it computes (every output row independently, so a caller can ask for
 * any sample of rows):
 *
 *   Forward (BlockSparseAttentionGrad README, "Formula": attentionOut =
 *   Softmax(scale * query * key_sparse^T) * value_sparse; BlitzSparseAttention,
 *   "softmax_lse output" and the all-ones worked example, which fixes the LSE
 *   as the natural log of sum exp(scale * q.k)):
 *     J(t)   = { u : u < kvlen_b, floor(u / BKV) is an accepted entry of the
 *                index row of t's query block }
 *     s_u    = scale * sum_d q[t,d] * k[u,d]
 *     lse_t  = m + ln sum_{u in J} exp(s_u - m),   m = max_{u in J} s_u
 *     out_t  = sum_{u in J} exp(s_u - lse_t) * v[u]
 *     J empty -> out_t = 0, lse_t = -inf.
 *   With the causal mask (GenericBlockSparseAttention, "mask" section: the
 *   built-in causal mode; aligned to the end of the kv sequence, our
 *   reading), J(t) also drops every u > t + kvlen_b - qlen_b.
 *
 *   Backward (BlockSparseAttentionGrad README, "Formula"), with out and lse
 *   taken as given inputs:
 *     softmax_grad_t = sum_d dOut[t,d] * out[t,d]
 *     P_tu  = exp(s_u - lse_t)          dP_tu = dOut_t . v_u
 *     dS_tu = P_tu * (dP_tu - softmax_grad_t)
 *     dV_u  = sum_t P_tu dOut_t         (summed over the GQA group's heads)
 *     dQ_t  = scale * sum_u dS_tu k_u
 *     dK_u  = scale * sum_t dS_tu q_t   (summed over the GQA group's heads)
 *
 * Index reading (BlitzSparseAttention, "sabi" section: uint16 entries,
 * 0xFFFF = unused slot, rows ascending): slots are read left to right; 0xFFFF
 * is skipped wherever it appears; an entry >= ceil(kvlen_b / BKV) or <= the
 * previous accepted entry is ignored and raises ORACLE_BAD_INDEX.
 *
 * Addressing:  BNSD q[b][h][t][d]; TND q[cu_q[b] + t][h][d];
 *   PA_BBND (GenericBlockSparseAttention, "Paged Attention"): kv token u of
 *   batch b is cache[block_table[b][u / page]][u % page][h2][d].
 *   kvlen_b = seqused_kv[b] if given, else the stored length.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BNSD 0
#define ORACLE_TND 1
#define ORACLE_PA_BBND 2
#define ORACLE_NO_BLOCK 0xFFFFu

#define ORACLE_BAD_INDEX 1u
#define ORACLE_BAD_SEQLEN 2u
#define ORACLE_BAD_PAGE 4u

typedef struct {
  int32_t layout_q, layout_kv;
  int64_t B, N1, N2, D;
  int64_t Sq, Skv;            /* BNSD stored sequence lengths */
  int64_t Tq, Tkv;            /* TND token rows of q and of k/v */
  int64_t num_pages, page_size, max_pages; /* PA_BBND */
  int64_t BQ, BKV, Hidx, R, W; /* index: BNSD [B,Hidx,R,W]; TND [Hidx,R,W] */
  double scale;
  const double *q, *k, *v;    /* dense, in their own layouts */
  const uint16_t *index;
  const int64_t *cu_q, *cu_kv; /* [B+1] or NULL */
  const int32_t *seqused_kv;   /* [B] or NULL */
  const int32_t *block_table;  /* [B, max_pages] or NULL */
  int32_t causal;              /* 1: u <= t + kvlen_b - qlen_b only */
} oracle_problem;

/* ---------------------------------------------------------------- lengths */
/* query rows of batch b; an inconsistent cu_seqlens gives 0 rows */
static int64_t q_len(const oracle_problem *P, int64_t b, uint32_t *fl) {
  if (P->layout_q != ORACLE_TND) return P->Sq;
  int64_t a = P->cu_q[b], e = P->cu_q[b + 1];
  if (a < 0 || e < a || e > P->Tq) { *fl |= ORACLE_BAD_SEQLEN; return 0; }
  return e - a;
}

static int64_t kv_stored(const oracle_problem *P, int64_t b, uint32_t *fl) {
  if (P->layout_kv == ORACLE_BNSD) return P->Skv;
  if (P->layout_kv == ORACLE_PA_BBND) return P->max_pages * P->page_size;
  int64_t a = P->cu_kv[b], e = P->cu_kv[b + 1];
  if (a < 0 || e < a || e > P->Tkv) { *fl |= ORACLE_BAD_SEQLEN; return 0; }
  return e - a;
}

static int64_t kv_len(const oracle_problem *P, int64_t b, uint32_t *fl) {
  int64_t st = kv_stored(P, b, fl);
  if (!P->seqused_kv) return st;
  int64_t u = P->seqused_kv[b];
  if (u < 0 || u > st) { *fl |= ORACLE_BAD_SEQLEN; return 0; }
  return u;
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* first index row of batch b (TND rows are packed batch after batch) */
static int64_t qblock_offset(const oracle_problem *P, int64_t b) {
  if (P->layout_q != ORACLE_TND) return 0;
  int64_t off = 0;
  uint32_t dummy = 0;
  for (int64_t bb = 0; bb < b; ++bb) off += ceil_div(q_len(P, bb, &dummy), P->BQ);
  return off;
}

/* ------------------------------------------------------------- addressing */
static const double *q_row(const oracle_problem *P, const double *base, int64_t b, int64_t h,
                           int64_t t) {
  if (P->layout_q == ORACLE_TND) return base + ((P->cu_q[b] + t) * P->N1 + h) * P->D;
  return base + ((b * P->N1 + h) * P->Sq + t) * P->D;
}

/* offset (in rows of D) of kv token u of batch b, head h2; -1 if its page is invalid */
static int64_t kv_row_offset(const oracle_problem *P, int64_t b, int64_t h2, int64_t u) {
  if (P->layout_kv == ORACLE_BNSD) return (b * P->N2 + h2) * P->Skv + u;
  if (P->layout_kv == ORACLE_TND) return (P->cu_kv[b] + u) * P->N2 + h2;
  int64_t pg = P->block_table[b * P->max_pages + u / P->page_size];
  if (pg < 0 || pg >= P->num_pages) return -1;
  return (pg * P->page_size + u % P->page_size) * P->N2 + h2;
}

/* lse / softmax_grad arrays: BNSD [B,N1,Sq]; TND [Tq,N1] */
static int64_t row_stat_offset(const oracle_problem *P, int64_t b, int64_t h1, int64_t t) {
  if (P->layout_q == ORACLE_TND) return (P->cu_q[b] + t) * P->N1 + h1;
  return (b * P->N1 + h1) * P->Sq + t;
}

/* ------------------------------------------------------------ index rows */
static int64_t index_head(const oracle_problem *P, int64_t h1) {
  return P->Hidx == P->N1 ? h1 : h1 / (P->N1 / P->N2);
}

/* Accepted kv blocks of query block i of (b, head hi), ascending; returns count. */
static int64_t row_blocks(const oracle_problem *P, int64_t b, int64_t hi, int64_t i,
                          int64_t qboff, int64_t nk, int64_t *blk, uint32_t *fl) {
  const uint16_t *row;
  if (P->layout_q == ORACLE_TND) {
    int64_t r = qboff + i;
    if (r >= P->R) { *fl |= ORACLE_BAD_INDEX; return 0; }
    row = P->index + (hi * P->R + r) * P->W;
  } else {
    row = P->index + ((b * P->Hidx + hi) * P->R + i) * P->W;
  }
  int64_t n = 0, last = -1;
  for (int64_t w = 0; w < P->W; ++w) {
    int64_t e = row[w];
    if (e == ORACLE_NO_BLOCK) continue;
    if (e >= nk || e <= last) { *fl |= ORACLE_BAD_INDEX; continue; }
    blk[n++] = e;
    last = e;
  }
  return n;
}

/* One past the last kv token query row t of batch b may see (causal), or
 * kvlen without the mask. */
static int64_t visible_end(const oracle_problem *P, int64_t t, int64_t kvlen, int64_t qlen) {
  if (!P->causal) return kvlen;
  int64_t e = t + kvlen - qlen + 1;
  return e < 0 ? 0 : (e < kvlen ? e : kvlen);
}

static double dot(const double *a, const double *b, int64_t D) {
  double s = 0.0;
  for (int64_t d = 0; d < D; ++d) s += a[d] * b[d];
  return s;
}

/* ============================================================== forward */
/* rows: nrows triples (b, h1, t).  out_rows: [nrows, D]; lse_rows: [nrows]. */
int oracle_fwd_rows(const oracle_problem *P, const int64_t *rows, int64_t nrows,
                    double *out_rows, double *lse_rows, uint32_t *flags) {
  const int64_t D = P->D, g = P->N1 / P->N2;
  uint32_t fl = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : fl)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t b = rows[3 * r], h1 = rows[3 * r + 1], t = rows[3 * r + 2];
    int64_t h2 = h1 / g, i = t / P->BQ;
    uint32_t f = 0;
    int64_t kvlen = kv_len(P, b, &f);
    int64_t nk = ceil_div(kvlen, P->BKV);
    int64_t *blk = (int64_t *)malloc(sizeof(int64_t) * (P->W + 1));
    int64_t nb = row_blocks(P, b, index_head(P, h1), i, qblock_offset(P, b), nk, blk, &f);
    const int64_t uend = visible_end(P, t, kvlen, q_len(P, b, &f));
    const double *qt = q_row(P, P->q, b, h1, t);
    double *o = out_rows + r * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;

    /* pass 1: the running maximum of the selected scores */
    double m = -INFINITY;
    int64_t count = 0;
    for (int64_t x = 0; x < nb; ++x) {
      int64_t u0 = blk[x] * P->BKV, u1 = u0 + P->BKV < uend ? u0 + P->BKV : uend;
      for (int64_t u = u0; u < u1; ++u) {
        int64_t off = kv_row_offset(P, b, h2, u);
        if (off < 0) { f |= ORACLE_BAD_PAGE; continue; }
        double s = P->scale * dot(qt, P->k + off * D, D);
        if (s > m) m = s;
        ++count;
      }
    }
    if (count == 0) {
      lse_rows[r] = -INFINITY;
    } else {
      /* pass 2: the sum of exponentials and the log-sum-exp */
      double l = 0.0;
      for (int64_t x = 0; x < nb; ++x) {
        int64_t u0 = blk[x] * P->BKV, u1 = u0 + P->BKV < uend ? u0 + P->BKV : uend;
        for (int64_t u = u0; u < u1; ++u) {
          int64_t off = kv_row_offset(P, b, h2, u);
          if (off < 0) continue;
          l += exp(P->scale * dot(qt, P->k + off * D, D) - m);
        }
      }
      double lse = m + log(l);
      lse_rows[r] = lse;
      /* pass 3: out = sum_u softmax_u * v_u */
      for (int64_t x = 0; x < nb; ++x) {
        int64_t u0 = blk[x] * P->BKV, u1 = u0 + P->BKV < uend ? u0 + P->BKV : uend;
        for (int64_t u = u0; u < u1; ++u) {
          int64_t off = kv_row_offset(P, b, h2, u);
          if (off < 0) continue;
          double p = exp(P->scale * dot(qt, P->k + off * D, D) - lse);
          const double *vu = P->v + off * D;
          for (int64_t d = 0; d < D; ++d) o[d] += p * vu[d];
        }
      }
    }
    free(blk);
    fl |= f;
  }
  if (flags) *flags |= fl;
  return 0;
}

/* ============================================================= backward */
/* dQ rows: rows = (b, h1, t) triples; out/dout in q layout; lse in row-stat layout */
int oracle_bwd_dq_rows(const oracle_problem *P, const double *out, const double *dout,
                       const double *lse, const int64_t *rows, int64_t nrows, double *dq_rows,
                       uint32_t *flags) {
  const int64_t D = P->D, g = P->N1 / P->N2;
  uint32_t fl = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : fl)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t b = rows[3 * r], h1 = rows[3 * r + 1], t = rows[3 * r + 2];
    int64_t h2 = h1 / g, i = t / P->BQ;
    uint32_t f = 0;
    int64_t kvlen = kv_len(P, b, &f);
    int64_t nk = ceil_div(kvlen, P->BKV);
    int64_t *blk = (int64_t *)malloc(sizeof(int64_t) * (P->W + 1));
    int64_t nb = row_blocks(P, b, index_head(P, h1), i, qblock_offset(P, b), nk, blk, &f);
    const double *qt = q_row(P, P->q, b, h1, t);
    const double *dOt = q_row(P, dout, b, h1, t);
    const double *ot = q_row(P, out, b, h1, t);
    const int64_t uend = visible_end(P, t, kvlen, q_len(P, b, &f));
    double lt = lse[row_stat_offset(P, b, h1, t)];
    double sg = dot(dOt, ot, D); /* softmax_grad_t */
    double *dq = dq_rows + r * D;
    for (int64_t d = 0; d < D; ++d) dq[d] = 0.0;
    for (int64_t x = 0; x < nb; ++x) {
      int64_t u0 = blk[x] * P->BKV, u1 = u0 + P->BKV < uend ? u0 + P->BKV : uend;
      for (int64_t u = u0; u < u1; ++u) {
        int64_t off = kv_row_offset(P, b, h2, u);
        if (off < 0) { f |= ORACLE_BAD_PAGE; continue; }
        const double *ku = P->k + off * D, *vu = P->v + off * D;
        double p = exp(P->scale * dot(qt, ku, D) - lt);
        double ds = p * (dot(dOt, vu, D) - sg);
        for (int64_t d = 0; d < D; ++d) dq[d] += P->scale * ds * ku[d];
      }
    }
    free(blk);
    fl |= f;
  }
  if (flags) *flags |= fl;
  return 0;
}

/* dK/dV rows: kvrows = (b, h2, u) triples with u a batch-local kv token. */
int oracle_bwd_dkv_rows(const oracle_problem *P, const double *out, const double *dout,
                        const double *lse, const int64_t *kvrows, int64_t nrows, double *dk_rows,
                        double *dv_rows, uint32_t *flags) {
  const int64_t D = P->D, g = P->N1 / P->N2;
  uint32_t fl = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fl)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t b = kvrows[3 * r], h2 = kvrows[3 * r + 1], u = kvrows[3 * r + 2];
    uint32_t f = 0;
    double *dk = dk_rows + r * D, *dv = dv_rows + r * D;
    for (int64_t d = 0; d < D; ++d) dk[d] = dv[d] = 0.0;
    int64_t kvlen = kv_len(P, b, &f), qlen = q_len(P, b, &f);
    int64_t off = u < kvlen ? kv_row_offset(P, b, h2, u) : -1;
    if (off >= 0) {
      int64_t nk = ceil_div(kvlen, P->BKV), j = u / P->BKV;
      int64_t nq = ceil_div(qlen, P->BQ), qboff = qblock_offset(P, b);
      const double *ku = P->k + off * D, *vu = P->v + off * D;
      int64_t *blk = (int64_t *)malloc(sizeof(int64_t) * (P->W + 1));
      for (int64_t h1 = h2 * g; h1 < (h2 + 1) * g; ++h1) {
        for (int64_t i = 0; i < nq; ++i) {
          int64_t nb = row_blocks(P, b, index_head(P, h1), i, qboff, nk, blk, &f);
          int selected = 0;
          for (int64_t x = 0; x < nb; ++x) selected |= (blk[x] == j);
          if (!selected) continue;
          int64_t t1 = (i + 1) * P->BQ < qlen ? (i + 1) * P->BQ : qlen;
          for (int64_t t = i * P->BQ; t < t1; ++t) {
            if (u >= visible_end(P, t, kvlen, qlen)) continue;
            const double *qt = q_row(P, P->q, b, h1, t);
            const double *dOt = q_row(P, dout, b, h1, t);
            const double *ot = q_row(P, out, b, h1, t);
            double p = exp(P->scale * dot(qt, ku, D) - lse[row_stat_offset(P, b, h1, t)]);
            double ds = p * (dot(dOt, vu, D) - dot(dOt, ot, D));
            for (int64_t d = 0; d < D; ++d) {
              dv[d] += p * dOt[d];
              dk[d] += P->scale * ds * qt[d];
            }
          }
        }
      }
      free(blk);
    }
    fl |= f;
  }
  if (flags) *flags |= fl;
  return 0;
}

/* ========================================================= batch lengths */
/* Per batch: query rows, used kv tokens and stored kv rows as the
 * definition reads them (GenericBlockSparseAttention, "dual length"
 * semantics: seqused_kv may not exceed the stored length; a contradictory
 * length counts as 0 and raises ORACLE_BAD_SEQLEN).  The stored rows are
 * those of the batch's own kv storage: BNSD Skv, TND the cu_seqlens_kv
 * difference, PA_BBND the pages that cover the used length. */
int oracle_batch_lengths(const oracle_problem *P, int64_t *qlen, int64_t *kvlen,
                         int64_t *kvstored, uint32_t *flags) {
  uint32_t fl = 0;
  for (int64_t b = 0; b < P->B; ++b) {
    qlen[b] = q_len(P, b, &fl);
    kvlen[b] = kv_len(P, b, &fl);
    if (P->layout_kv == ORACLE_PA_BBND)
      kvstored[b] = ceil_div(kvlen[b], P->page_size) * P->page_size;
    else
      kvstored[b] = kv_stored(P, b, &fl);
  }
  if (flags) *flags |= fl;
  return 0;
}

/* ============================================================ flag scan */
/* Every status bit the inputs raise: each existing index row, each length,
 * each block-table slot covering a used kv token. */
int oracle_scan_flags(const oracle_problem *P, uint32_t *flags) {
  uint32_t fl = 0;
  int64_t *blk = (int64_t *)malloc(sizeof(int64_t) * (P->W + 1));
  int64_t qboff = 0;
  for (int64_t b = 0; b < P->B; ++b) {
    int64_t qlen = q_len(P, b, &fl), kvlen = kv_len(P, b, &fl);
    int64_t nq = ceil_div(qlen, P->BQ), nk = ceil_div(kvlen, P->BKV);
    for (int64_t hi = 0; hi < P->Hidx; ++hi)
      for (int64_t i = 0; i < nq; ++i) row_blocks(P, b, hi, i, qboff, nk, blk, &fl);
    if (P->layout_kv == ORACLE_PA_BBND)
      for (int64_t x = 0; x < ceil_div(kvlen, P->page_size); ++x) {
        int64_t pg = P->block_table[b * P->max_pages + x];
        if (pg < 0 || pg >= P->num_pages) fl |= ORACLE_BAD_PAGE;
      }
    qboff += nq;
  }
  free(blk);
  *flags |= fl;
  return 0;
}

int oracle_abi_version(void) { return 1; }
