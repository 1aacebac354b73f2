/*
 * Ulysses sequence-parallel attention layer -- plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline / reference arm do.  It shares no code, header, table or
 * helper with the CUDA library: the two are compared, never combined.
 *
 * Every routine here is the plain definition of what the method computes,
 * written out with explicit loops and fp64 arithmetic (inputs arrive as fp32,
 * which holds bf16 and fp32 values exactly).  No tiling, no online softmax,
 * no fusion: a reader can check each loop against the pages by eye.
 *
 * Sources (page title, section):
 *  [P1] "Ulysses 序列平行化：突破百萬標記長上下文的訓練瓶頸" (agents-report.net),
 *       section "Ulysses 序列平行化的原理" -- the five steps: shard the
 *       sequence, project QKV, all-to-all so each device holds every position
 *       for a subset of heads, local attention per head, second all-to-all.
 *  [P3] "Paralelismul de Secvență Ulysses: Antrenarea modelelor AI cu
 *       contexte de un milion de token-uri" (world.tibi.club),
 *       section "Mecanismul de funcționare Ulysses", steps 1-6 (rank i holds
 *       tokens [i*n/P, (i+1)*n/P); first all-to-all gives all positions for a
 *       subset of heads; attention heads are independent), and section
 *       "Integrarea cu Accelerate" (losses weighted by each rank's count of
 *       valid tokens).
 *  Attention itself is the standard scaled-dot-product attention the pages
 *  name ("SDPA"): O = softmax(scale * Q K^T + mask) V, scale = 1/sqrt(d).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - GQA: query head q uses KV head floor(q / (H/G)); rank r owns query heads
 *    [r*H/P, (r+1)*H/P) and KV heads [r*G/P, (r+1)*G/P).
 *  - Layouts: seq layout X[P][B][s][Hx][d] (rank-major stack of per-rank
 *    buffers); head layout X[P][B][Hx/P][n][d].
 *  - Causal: key j allowed for query i iff j <= i.  Doc-causal: additionally
 *    doc(j) == doc(i), documents given by cu_seqlens.
 *  - Loss: ignore index given by the caller (-100 in all workloads); a label
 *    outside [0, V) that is not the ignore index is an error and the token is
 *    not counted.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_MASK_NONE 0
#define ORACLE_MASK_CAUSAL 1
#define ORACLE_MASK_DOC_CAUSAL 2

/* ------------------------------------------------------------------------- */
/* Steps 1, 3 and 5: sharding and the two all-to-alls, as explicit loops.     */
/* ------------------------------------------------------------------------- */

/*
 * First all-to-all [P3 "Mecanismul de funcționare Ulysses", steps 1 and 3]:
 * sending rank r holds s = n/P consecutive positions (global t = r*s + tt) for
 * all `heads` heads.  For every receiving rank r2 it sends the heads
 * [r2*hl, (r2+1)*hl), hl = heads/P; rank r2 stores them at global positions
 * [r*s, (r+1)*s) so that afterwards it holds every position for its heads.
 * Rows are `row_bytes` opaque bytes (d elements of any type).
 */
void oracle_seq_to_head(int B, int n, int P, int heads, long row_bytes,
                        const void *src, void *dst) {
  const int s = n / P, hl = heads / P;
  for (int r = 0; r < P; ++r)          /* sending rank   */
    for (int r2 = 0; r2 < P; ++r2)     /* receiving rank */
      for (int b = 0; b < B; ++b)
        for (int hh = 0; hh < hl; ++hh)
          for (int tt = 0; tt < s; ++tt) {
            size_t src_row = (((size_t)r * B + b) * s + tt) * heads + (size_t)r2 * hl + hh;
            size_t dst_row = (((size_t)r2 * B + b) * hl + hh) * n + (size_t)r * s + tt;
            memcpy((char *)dst + dst_row * row_bytes,
                   (const char *)src + src_row * row_bytes, (size_t)row_bytes);
          }
}

/*
 * Second all-to-all [P3 step 5; P1 step 5]: the inverse redistribution.  Rank
 * r2 holds all n positions of its heads; it sends positions [r*s, (r+1)*s) of
 * each head back to rank r, which stores them as heads [r2*hl, (r2+1)*hl) of
 * its local tokens.
 */
void oracle_head_to_seq(int B, int n, int P, int heads, long row_bytes,
                        const void *src, void *dst) {
  const int s = n / P, hl = heads / P;
  for (int r2 = 0; r2 < P; ++r2)       /* sending rank (head owner) */
    for (int r = 0; r < P; ++r)        /* receiving rank (seq owner) */
      for (int b = 0; b < B; ++b)
        for (int hh = 0; hh < hl; ++hh)
          for (int tt = 0; tt < s; ++tt) {
            size_t src_row = (((size_t)r2 * B + b) * hl + hh) * n + (size_t)r * s + tt;
            size_t dst_row = (((size_t)r * B + b) * s + tt) * heads + (size_t)r2 * hl + hh;
            memcpy((char *)dst + dst_row * row_bytes,
                   (const char *)src + src_row * row_bytes, (size_t)row_bytes);
          }
}

/*
 * First all-to-all of K and V when there are fewer KV heads than ranks
 * (G < P, P % G == 0).  The pages require at least as many heads as ranks
 * ("Ulysses 序列平行化", section "與 Ring Attention 的比較": num_heads >=
 * sp_size); with
 * grouped-query attention that bound holds for the H query heads but not for
 * the G KV heads, and the plain reading is that each KV head is sent whole to
 * every rank whose query heads use it.  Rank r2 owns query heads
 * [r2*H/P, (r2+1)*H/P), all of which use KV head floor(r2*G/P); it receives
 * that one KV head for all n positions.  dst: [P][B][1][n][row].
 */
void oracle_kv_replicate_to_head(int B, int n, int P, int G, long row_bytes,
                                 const void *src, void *dst) {
  const int s = n / P;
  for (int r = 0; r < P; ++r)          /* sending rank   */
    for (int r2 = 0; r2 < P; ++r2) {   /* receiving rank */
      const int k = r2 * G / P;        /* the KV head rank r2's query heads use */
      for (int b = 0; b < B; ++b)
        for (int tt = 0; tt < s; ++tt) {
          size_t src_row = (((size_t)r * B + b) * s + tt) * G + (size_t)k;
          size_t dst_row = ((size_t)r2 * B + b) * n + (size_t)r * s + tt;
          memcpy((char *)dst + dst_row * row_bytes,
                 (const char *)src + src_row * row_bytes, (size_t)row_bytes);
        }
    }
}

/*
 * Second all-to-all of dK and dV for replicated KV heads: the gradient of a
 * KV head is the sum of the gradients its copies received on every rank that
 * held one (the copies are the same variable).  src: [P][B][1][n][d] (rank
 * r2's copy of KV head floor(r2*G/P)), dst: seq layout [P][B][n/P][G][d];
 * fp64, summed over the copies in rank order.
 */
void oracle_kv_reduce_to_seq(int B, int n, int P, int G, int d, const double *src,
                             double *dst) {
  const int s = n / P;
  memset(dst, 0, sizeof(double) * (size_t)B * n * G * d);
  for (int r2 = 0; r2 < P; ++r2) {     /* rank holding a copy */
    const int k = r2 * G / P;
    for (int r = 0; r < P; ++r)        /* rank owning the positions */
      for (int b = 0; b < B; ++b)
        for (int tt = 0; tt < s; ++tt) {
          const double *x = src + (((size_t)r2 * B + b) * n + (size_t)r * s + tt) * d;
          double *y = dst + ((((size_t)r * B + b) * s + tt) * G + (size_t)k) * d;
          for (int e = 0; e < d; ++e) y[e] += x[e];
        }
  }
}

/* ------------------------------------------------------------------------- */
/* Label shift for next-token prediction, before the sequence is sharded.     */
/* ------------------------------------------------------------------------- */

/*
 * The label of position t is the token at t+1 (next-token prediction), and the
 * shift has to happen on the whole sequence, before it is split over ranks:
 * the last position of shard r needs the first token of shard r+1 (the
 * SFT trainer's automatic label shift: "Ulysses 序列平行化", section
 * "在 Hugging Face 生態系統中的整合"; padding to a multiple of sp_size and
 * variable-length packed sequences: "Paralelismul de Secvență Ulysses",
 * section "Integrarea cu Transformers Trainer și TRL SFTTrainer").  A position
 * gets ignore_index when t+1 is past the valid tokens (t+1 >= valid_len: the
 * last token and the padding that makes n a multiple of P) or when t+1 starts
 * a new packed document (t+1 is one of cu_seqlens[1..num_docs]).
 * ids: [B][n] in sequence order; labels: seq layout [P][B][n/P].
 */
void oracle_shift_labels(int B, int n, int P, const int *ids, const int *cu_seqlens,
                         int num_docs, int valid_len, int ignore_index, int *labels) {
  const int s = n / P;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < n; ++t) {
      int y = ignore_index;
      if (t + 1 < valid_len) {
        int starts_doc = 0;
        for (int e = 1; e <= num_docs; ++e)
          if (cu_seqlens[e] == t + 1) starts_doc = 1;
        if (!starts_doc) y = ids[(size_t)b * n + t + 1];
      }
      const int r = t / s, tt = t % s;
      labels[((size_t)r * B + b) * s + tt] = y;
    }
}

/* ------------------------------------------------------------------------- */
/* Step 4: scaled-dot-product attention of one head, row by row.             */
/* ------------------------------------------------------------------------- */

typedef struct {
  int n, d, mask;
  const int *cu_seqlens; /* [num_docs+1], mask == doc-causal only */
  int num_docs;
  double scale;
} attn_cfg;

/* Document index of every position (doc-causal mask only). */
static int *doc_index(const attn_cfg *c) {
  int *doc = (int *)malloc(sizeof(int) * (size_t)(c->n > 0 ? c->n : 1));
  for (int t = 0; t < c->n; ++t) doc[t] = -1;
  if (c->mask == ORACLE_MASK_DOC_CAUSAL)
    for (int e = 0; e < c->num_docs; ++e)
      for (int t = c->cu_seqlens[e]; t < c->cu_seqlens[e + 1] && t < c->n; ++t) doc[t] = e;
  return doc;
}

/* Is key j visible to query i? */
static int allowed(const attn_cfg *c, const int *doc, int i, int j) {
  if (c->mask == ORACLE_MASK_NONE) return 1;
  if (j > i) return 0;
  if (c->mask == ORACLE_MASK_CAUSAL) return 1;
  return doc[i] >= 0 && doc[i] == doc[j];
}

/* The set of visible keys of row i is a contiguous range [lo, hi] under all
 * three masks (a document is a contiguous run of positions); hi < lo means
 * no visible key.  Computed from `allowed` so the two cannot disagree. */
static void key_range(const attn_cfg *c, const int *doc, int i, int *lo, int *hi) {
  if (c->mask == ORACLE_MASK_NONE) { *lo = 0; *hi = c->n - 1; return; }
  int l = i;
  while (l > 0 && allowed(c, doc, i, l - 1)) --l;
  if (!allowed(c, doc, i, i)) { *lo = 1; *hi = 0; return; }
  *lo = l; *hi = i;
}

static double dot_f(const float *a, const float *b, int d) {
  double acc = 0.0;
  for (int x = 0; x < d; ++x) acc += (double)a[x] * (double)b[x];
  return acc;
}

/*
 * One query row i of one head: scores s_j = scale * <q_i, k_j> over the
 * visible keys, m = max s_j, l = sum exp(s_j - m), o_i = sum exp(s_j - m) v_j / l,
 * lse_i = m + log l.  A row with no visible key gets o = 0, lse = -inf.
 * `sbuf` is caller scratch of n doubles.
 */
static void attn_row_fwd(const attn_cfg *c, const int *doc, int i,
                         const float *q, long q_rs, const float *k, long k_rs,
                         const float *v, long v_rs, double *sbuf,
                         double *o_row, double *lse) {
  const int d = c->d;
  int lo, hi;
  key_range(c, doc, i, &lo, &hi);
  for (int x = 0; x < d; ++x) o_row[x] = 0.0;
  if (hi < lo) { *lse = -INFINITY; return; }
  const float *qi = q + (size_t)i * q_rs;
  double m = -INFINITY;
  for (int j = lo; j <= hi; ++j) {
    sbuf[j] = c->scale * dot_f(qi, k + (size_t)j * k_rs, d);
    if (sbuf[j] > m) m = sbuf[j];
  }
  double l = 0.0;
  for (int j = lo; j <= hi; ++j) {
    double p = exp(sbuf[j] - m);
    l += p;
    const float *vj = v + (size_t)j * v_rs;
    for (int x = 0; x < d; ++x) o_row[x] += p * (double)vj[x];
  }
  for (int x = 0; x < d; ++x) o_row[x] /= l;
  *lse = m + log(l);
}

/*
 * Backward of one query row i (gradients of sum(O * dO)):
 *   P_ij = exp(s_ij - lse_i), dP_ij = <dO_i, v_j>, D_i = <dO_i, O_i>,
 *   dS_ij = P_ij (dP_ij - D_i),  dQ_i = scale * sum_j dS_ij k_j.
 * Only dQ_i is produced here (it is row-local); the key-side gradients are
 * produced column by column in attn_col_bwd.
 */
static void attn_row_dq(const attn_cfg *c, const int *doc, int i,
                        const float *q, long q_rs, const float *k, long k_rs,
                        const float *v, long v_rs, const float *dout, long do_rs,
                        double lse_i, double D_i, double *dq_row) {
  const int d = c->d;
  int lo, hi;
  key_range(c, doc, i, &lo, &hi);
  for (int x = 0; x < d; ++x) dq_row[x] = 0.0;
  const float *qi = q + (size_t)i * q_rs;
  const float *doi = dout + (size_t)i * do_rs;
  for (int j = lo; j <= hi; ++j) {
    const float *kj = k + (size_t)j * k_rs;
    double p = exp(c->scale * dot_f(qi, kj, d) - lse_i);
    double dp = dot_f(doi, v + (size_t)j * v_rs, d);
    double ds = p * (dp - D_i);
    for (int x = 0; x < d; ++x) dq_row[x] += ds * (double)kj[x];
  }
  for (int x = 0; x < d; ++x) dq_row[x] *= c->scale;
}

/*
 * Key-side backward of one key column j of a KV head, summed over the nq
 * query heads that share it (GQA):
 *   dV_j = sum_heads sum_i P_ij dO_i,   dK_j = scale * sum_heads sum_i dS_ij q_i,
 * over every query row i that sees key j.  lse[hq][i], Dv[hq][i] are the
 * per-row statistics of query head hq.
 */
static void attn_col_bwd(const attn_cfg *c, const int *doc, int j, int nq,
                         const float *const *qs, long q_rs,
                         const float *const *douts, long do_rs,
                         const float *k, long k_rs, const float *v, long v_rs,
                         const double *const *lse, const double *const *Dv,
                         double *dk_row, double *dv_row) {
  const int d = c->d;
  for (int x = 0; x < d; ++x) { dk_row[x] = 0.0; dv_row[x] = 0.0; }
  const float *kj = k + (size_t)j * k_rs;
  const float *vj = v + (size_t)j * v_rs;
  for (int hq = 0; hq < nq; ++hq)
    for (int i = 0; i < c->n; ++i) {
      if (!allowed(c, doc, i, j)) continue;
      const float *qi = qs[hq] + (size_t)i * q_rs;
      const float *doi = douts[hq] + (size_t)i * do_rs;
      double p = exp(c->scale * dot_f(qi, kj, d) - lse[hq][i]);
      double dp = dot_f(doi, vj, d);
      double ds = p * (dp - Dv[hq][i]);
      for (int x = 0; x < d; ++x) {
        dv_row[x] += p * (double)doi[x];
        dk_row[x] += ds * (double)qi[x];
      }
    }
  for (int x = 0; x < d; ++x) dk_row[x] *= c->scale;
}

/* Forward of one head, all rows: o[n][d] (row stride d), lse[n]. */
static void attn_head_fwd(const attn_cfg *c, const int *doc,
                          const float *q, long q_rs, const float *k, long k_rs,
                          const float *v, long v_rs, double *o, long o_rs, double *lse) {
#pragma omp parallel
  {
    double *sbuf = (double *)malloc(sizeof(double) * (size_t)(c->n > 0 ? c->n : 1));
#pragma omp for schedule(dynamic, 16)
    for (int i = 0; i < c->n; ++i)
      attn_row_fwd(c, doc, i, q, q_rs, k, k_rs, v, v_rs, sbuf, o + (size_t)i * o_rs, &lse[i]);
    free(sbuf);
  }
}

/* ------------------------------------------------------------------------- */
/* Plain (non-parallel) multi-head GQA attention on the natural layout        */
/* X[B][n][H][d]: the result Ulysses must reproduce exactly.                  */
/* ------------------------------------------------------------------------- */

static attn_cfg make_cfg(int n, int d, int mask, const int *cu, int ndocs, double scale) {
  attn_cfg c;
  c.n = n; c.d = d; c.mask = mask; c.cu_seqlens = cu; c.num_docs = ndocs;
  c.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)d);
  return c;
}

/* o: [B][n][H][d] (doubles), lse: [B][H][n]. */
void oracle_attention_fwd(int B, int n, int H, int G, int d, int mask,
                          const int *cu_seqlens, int num_docs, double scale,
                          const float *q, const float *k, const float *v,
                          double *o, double *lse) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
  const int group = H / G;
  for (int b = 0; b < B; ++b)
    for (int hq = 0; hq < H; ++hq) {
      const int hk = hq / group;
      attn_head_fwd(&c, doc,
                    q + ((size_t)b * n * H + hq) * d, (long)H * d,
                    k + ((size_t)b * n * G + hk) * d, (long)G * d,
                    v + ((size_t)b * n * G + hk) * d, (long)G * d,
                    o + ((size_t)b * n * H + hq) * d, (long)H * d,
                    lse + ((size_t)b * H + hq) * n);
    }
  free(doc);
}

/* Gradients of sum(O * dO) w.r.t. q, k, v (all on the natural layout). */
void oracle_attention_bwd(int B, int n, int H, int G, int d, int mask,
                          const int *cu_seqlens, int num_docs, double scale,
                          const float *q, const float *k, const float *v,
                          const float *dout, double *dq, double *dk, double *dv) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
  const int group = H / G;
  double *o = (double *)malloc(sizeof(double) * (size_t)n * d);
  double *lse = (double *)malloc(sizeof(double) * (size_t)H * n);
  double *Dv = (double *)malloc(sizeof(double) * (size_t)H * n);
  for (int b = 0; b < B; ++b) {
    /* per query head: O, lse, D = rowsum(dO * O), then dQ row by row */
    for (int hq = 0; hq < H; ++hq) {
      const float *qh = q + ((size_t)b * n * H + hq) * d;
      const float *kh = k + ((size_t)b * n * G + hq / group) * d;
      const float *vh = v + ((size_t)b * n * G + hq / group) * d;
      const float *doh = dout + ((size_t)b * n * H + hq) * d;
      attn_head_fwd(&c, doc, qh, (long)H * d, kh, (long)G * d, vh, (long)G * d,
                    o, d, lse + (size_t)hq * n);
#pragma omp parallel for schedule(dynamic, 16)
      for (int i = 0; i < n; ++i) {
        double D = 0.0;
        for (int x = 0; x < d; ++x) D += (double)doh[(size_t)i * H * d + x] * o[(size_t)i * d + x];
        Dv[(size_t)hq * n + i] = D;
        attn_row_dq(&c, doc, i, qh, (long)H * d, kh, (long)G * d, vh, (long)G * d,
                    doh, (long)H * d, lse[(size_t)hq * n + i], D,
                    dq + (((size_t)b * n + i) * H + hq) * d);
      }
    }
    /* per KV head: dK, dV column by column, summed over its query heads */
    for (int hk = 0; hk < G; ++hk) {
      const float **qs = (const float **)malloc(sizeof(float *) * (size_t)group);
      const float **ds = (const float **)malloc(sizeof(float *) * (size_t)group);
      const double **ls = (const double **)malloc(sizeof(double *) * (size_t)group);
      const double **Ds = (const double **)malloc(sizeof(double *) * (size_t)group);
      for (int e = 0; e < group; ++e) {
        int hq = hk * group + e;
        qs[e] = q + ((size_t)b * n * H + hq) * d;
        ds[e] = dout + ((size_t)b * n * H + hq) * d;
        ls[e] = lse + (size_t)hq * n;
        Ds[e] = Dv + (size_t)hq * n;
      }
      const float *kh = k + ((size_t)b * n * G + hk) * d;
      const float *vh = v + ((size_t)b * n * G + hk) * d;
#pragma omp parallel for schedule(dynamic, 16)
      for (int j = 0; j < n; ++j)
        attn_col_bwd(&c, doc, j, group, qs, (long)H * d, ds, (long)H * d,
                     kh, (long)G * d, vh, (long)G * d, ls, Ds,
                     dk + (((size_t)b * n + j) * G + hk) * d,
                     dv + (((size_t)b * n + j) * G + hk) * d);
      free(qs); free(ds); free(ls); free(Ds);
    }
  }
  free(o); free(lse); free(Dv); free(doc);
}

/* ------------------------------------------------------------------------- */
/* The explicit Ulysses procedure on P emulated ranks.                        */
/* Inputs in seq layout [P][B][s][Hx][d] (fp32), outputs likewise (fp64).     */
/* ------------------------------------------------------------------------- */

static float *to_head_f(int B, int n, int P, int heads, int d, const float *x_seq) {
  float *y = (float *)malloc(sizeof(float) * (size_t)B * n * heads * d);
  oracle_seq_to_head(B, n, P, heads, (long)d * (long)sizeof(float), x_seq, y);
  return y;
}

static float *to_head_rep_f(int B, int n, int P, int G, int d, const float *x_seq) {
  float *y = (float *)malloc(sizeof(float) * (size_t)B * n * P * d);
  oracle_kv_replicate_to_head(B, n, P, G, (long)d * (long)sizeof(float), x_seq, y);
  return y;
}

/*
 * Forward: seq->head all-to-all of Q, K, V; every rank r runs attention on
 * its hl = H/P query heads (KV head of local head hh: hh / (H/G), local to the
 * rank because rank r also owns KV heads [r*G/P, (r+1)*G/P)); head->seq
 * all-to-all of O.  lse_head is left in head layout [P][B][H/P][n].
 * With fewer KV heads than ranks (G < P, P % G == 0) every rank receives a
 * copy of the one KV head its query heads use (oracle_kv_replicate_to_head)
 * and, in the backward, the copies' gradients are summed on the way back
 * (oracle_kv_reduce_to_seq).
 */
void oracle_ulysses_fwd(int B, int n, int P, int H, int G, int d, int mask,
                        const int *cu_seqlens, int num_docs, double scale,
                        const float *q_seq, const float *k_seq, const float *v_seq,
                        double *o_seq, double *lse_head) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
  const int rep = G % P != 0;          /* G < P: one replicated KV head per rank */
  const int hl = H / P, gl = rep ? 1 : G / P, group = hl / gl;
  float *qh = to_head_f(B, n, P, H, d, q_seq);
  float *kh = rep ? to_head_rep_f(B, n, P, G, d, k_seq) : to_head_f(B, n, P, G, d, k_seq);
  float *vh = rep ? to_head_rep_f(B, n, P, G, d, v_seq) : to_head_f(B, n, P, G, d, v_seq);
  double *oh = (double *)malloc(sizeof(double) * (size_t)B * n * H * d);
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b)
      for (int hh = 0; hh < hl; ++hh) {
        const int gg = hh / group;
        const size_t qi = ((size_t)r * B + b) * hl + hh, ki = ((size_t)r * B + b) * gl + gg;
        attn_head_fwd(&c, doc, qh + qi * n * d, d, kh + ki * n * d, d, vh + ki * n * d, d,
                      oh + qi * n * d, d, lse_head + qi * n);
      }
  oracle_head_to_seq(B, n, P, H, (long)d * (long)sizeof(double), oh, o_seq);
  free(qh); free(kh); free(vh); free(oh); free(doc);
}

/*
 * Backward (the adjoint of the forward): dO goes seq->head, every rank runs
 * the attention backward on its heads, dQ/dK/dV go head->seq.
 */
void oracle_ulysses_bwd(int B, int n, int P, int H, int G, int d, int mask,
                        const int *cu_seqlens, int num_docs, double scale,
                        const float *q_seq, const float *k_seq, const float *v_seq,
                        const float *do_seq, double *dq_seq, double *dk_seq, double *dv_seq) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
  const int rep = G % P != 0;          /* G < P: one replicated KV head per rank */
  const int hl = H / P, gl = rep ? 1 : G / P, group = hl / gl;
  float *qh = to_head_f(B, n, P, H, d, q_seq);
  float *kh = rep ? to_head_rep_f(B, n, P, G, d, k_seq) : to_head_f(B, n, P, G, d, k_seq);
  float *vh = rep ? to_head_rep_f(B, n, P, G, d, v_seq) : to_head_f(B, n, P, G, d, v_seq);
  float *doh = to_head_f(B, n, P, H, d, do_seq);
  double *dqh = (double *)malloc(sizeof(double) * (size_t)B * n * H * d);
  double *dkh = (double *)malloc(sizeof(double) * (size_t)B * n * P * gl * d);
  double *dvh = (double *)malloc(sizeof(double) * (size_t)B * n * P * gl * d);
  double *o = (double *)malloc(sizeof(double) * (size_t)n * d);
  double *lse = (double *)malloc(sizeof(double) * (size_t)hl * n);
  double *Dv = (double *)malloc(sizeof(double) * (size_t)hl * n);
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b) {
      for (int hh = 0; hh < hl; ++hh) {
        const size_t qi = ((size_t)r * B + b) * hl + hh;
        const size_t ki = ((size_t)r * B + b) * gl + hh / group;
        const float *qp = qh + qi * n * d, *kp = kh + ki * n * d, *vp = vh + ki * n * d;
        const float *dop = doh + qi * n * d;
        attn_head_fwd(&c, doc, qp, d, kp, d, vp, d, o, d, lse + (size_t)hh * n);
#pragma omp parallel for schedule(dynamic, 16)
        for (int i = 0; i < n; ++i) {
          double D = 0.0;
          for (int x = 0; x < d; ++x) D += (double)dop[(size_t)i * d + x] * o[(size_t)i * d + x];
          Dv[(size_t)hh * n + i] = D;
          attn_row_dq(&c, doc, i, qp, d, kp, d, vp, d, dop, d, lse[(size_t)hh * n + i], D,
                      dqh + (qi * n + i) * d);
        }
      }
      for (int gg = 0; gg < gl; ++gg) {
        const size_t ki = ((size_t)r * B + b) * gl + gg;
        const float **qs = (const float **)malloc(sizeof(float *) * (size_t)group);
        const float **ds = (const float **)malloc(sizeof(float *) * (size_t)group);
        const double **ls = (const double **)malloc(sizeof(double *) * (size_t)group);
        const double **Ds = (const double **)malloc(sizeof(double *) * (size_t)group);
        for (int e = 0; e < group; ++e) {
          const int hh = gg * group + e;
          const size_t qi = ((size_t)r * B + b) * hl + hh;
          qs[e] = qh + qi * n * d;
          ds[e] = doh + qi * n * d;
          ls[e] = lse + (size_t)hh * n;
          Ds[e] = Dv + (size_t)hh * n;
        }
#pragma omp parallel for schedule(dynamic, 16)
        for (int j = 0; j < n; ++j)
          attn_col_bwd(&c, doc, j, group, qs, d, ds, d, kh + ki * n * d, d, vh + ki * n * d, d,
                       ls, Ds, dkh + (ki * n + j) * d, dvh + (ki * n + j) * d);
        free(qs); free(ds); free(ls); free(Ds);
      }
    }
  oracle_head_to_seq(B, n, P, H, (long)d * (long)sizeof(double), dqh, dq_seq);
  if (rep) {
    oracle_kv_reduce_to_seq(B, n, P, G, d, dkh, dk_seq);
    oracle_kv_reduce_to_seq(B, n, P, G, d, dvh, dv_seq);
  } else {
    oracle_head_to_seq(B, n, P, G, (long)d * (long)sizeof(double), dkh, dk_seq);
    oracle_head_to_seq(B, n, P, G, (long)d * (long)sizeof(double), dvh, dv_seq);
  }
  free(qh); free(kh); free(vh); free(doh); free(dqh); free(dkh); free(dvh);
  free(o); free(lse); free(Dv); free(doc);
}

/* ------------------------------------------------------------------------- */
/* Sampled exact values for workloads too large for the full oracle.          */
/* Each output is exact (not an estimate): O_i, lse_i and dQ_i depend only on */
/* row i; dK_j, dV_j need lse and D of every row that sees key j, which are   */
/* computed here for exactly those rows.                                      */
/* ------------------------------------------------------------------------- */

/* One query head (q, dout: [n][d] contiguous), one KV head (k, v: [n][d]).
 * For each listed row: o[r][d], lse[r]; dq[r][d] when dout and dq are given. */
void oracle_head_rows(int n, int d, int mask, const int *cu_seqlens, int num_docs, double scale,
                      const float *q, const float *k, const float *v, const float *dout,
                      const int *rows, int nrows, double *o, double *lse, double *dq) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
#pragma omp parallel
  {
    double *sbuf = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
    for (int e = 0; e < nrows; ++e) {
      const int i = rows[e];
      attn_row_fwd(&c, doc, i, q, d, k, d, v, d, sbuf, o + (size_t)e * d, &lse[e]);
      if (dout && dq) {
        double D = 0.0;
        for (int x = 0; x < d; ++x) D += (double)dout[(size_t)i * d + x] * o[(size_t)e * d + x];
        attn_row_dq(&c, doc, i, q, d, k, d, v, d, dout, d, lse[e], D, dq + (size_t)e * d);
      }
    }
    free(sbuf);
  }
  free(doc);
}

/* One KV head (k, v: [n][d]) and its nq query heads (qs[e], douts[e]: [n][d]).
 * For each listed key column: dk[c][d], dv[c][d], summed over the nq heads. */
void oracle_kv_cols(int n, int d, int mask, const int *cu_seqlens, int num_docs, double scale,
                    int nq, const float *const *qs, const float *const *douts,
                    const float *k, const float *v, const int *cols, int ncols,
                    double *dk, double *dv) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
  /* rows that see at least one of the listed keys */
  char *need = (char *)calloc((size_t)n, 1);
  for (int e = 0; e < ncols; ++e)
    for (int i = 0; i < n; ++i)
      if (allowed(&c, doc, i, cols[e])) need[i] = 1;
  double **lse = (double **)malloc(sizeof(double *) * (size_t)nq);
  double **Dv = (double **)malloc(sizeof(double *) * (size_t)nq);
  for (int h = 0; h < nq; ++h) {
    lse[h] = (double *)malloc(sizeof(double) * (size_t)n);
    Dv[h] = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp parallel
    {
      double *sbuf = (double *)malloc(sizeof(double) * (size_t)n);
      double *orow = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
      for (int i = 0; i < n; ++i) {
        lse[h][i] = -INFINITY;
        Dv[h][i] = 0.0;
        if (!need[i]) continue;
        attn_row_fwd(&c, doc, i, qs[h], d, k, d, v, d, sbuf, orow, &lse[h][i]);
        double D = 0.0;
        for (int x = 0; x < d; ++x) D += (double)douts[h][(size_t)i * d + x] * orow[x];
        Dv[h][i] = D;
      }
      free(sbuf); free(orow);
    }
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < ncols; ++e)
    attn_col_bwd(&c, doc, cols[e], nq, qs, d, douts, d, k, d, v, d,
                 (const double *const *)lse, (const double *const *)Dv,
                 dk + (size_t)e * d, dv + (size_t)e * d);
  for (int h = 0; h < nq; ++h) { free(lse[h]); free(Dv[h]); }
  free(lse); free(Dv); free(need); free(doc);
}

/* The same key columns as oracle_kv_cols, with the per-row statistics
 * lse[h][i] and D[h][i] of every row that sees a listed key supplied by the
 * caller (computed from the definition elsewhere, e.g. with fp64 matrix
 * products for a whole row range); only the column sums are formed here. */
void oracle_kv_cols_stats(int n, int d, int mask, const int *cu_seqlens, int num_docs, double scale,
                          int nq, const float *const *qs, const float *const *douts,
                          const float *k, const float *v, const double *const *lse,
                          const double *const *Dv, const int *cols, int ncols, double *dk, double *dv) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < ncols; ++e)
    attn_col_bwd(&c, doc, cols[e], nq, qs, d, douts, d, k, d, v, d, lse, Dv,
                 dk + (size_t)e * d, dv + (size_t)e * d);
  free(doc);
}

/*
 * Everything one query row i of one head contributes to the layer: O_i,
 * lse_i, dQ_i, and its terms of dK_j = scale * sum_i dS_ij q_i and
 * dV_j = sum_i P_ij dO_i for every visible key j, added into dk, dv ([n][d],
 * zeroed by the caller).  Summed over all rows this is the whole forward and
 * backward of the head; the benchmark times it on a uniform sample of rows.
 * Rows are processed one after another; the key loop of a row runs in
 * parallel (each key j is updated by exactly one thread).
 */
void oracle_head_rows_step(int n, int d, int mask, const int *cu_seqlens, int num_docs, double scale,
                           const float *q, const float *k, const float *v, const float *dout,
                           const int *rows, int nrows, double *o, double *lse, double *dq,
                           double *dk, double *dv) {
  attn_cfg c = make_cfg(n, d, mask, cu_seqlens, num_docs, scale);
  int *doc = doc_index(&c);
  double *p = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double *ds = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int e = 0; e < nrows; ++e) {
    const int i = rows[e];
    int lo, hi;
    key_range(&c, doc, i, &lo, &hi);
    double *oi = o + (size_t)e * d, *dqi = dq + (size_t)e * d;
    for (int x = 0; x < d; ++x) { oi[x] = 0.0; dqi[x] = 0.0; }
    if (hi < lo) { lse[e] = -INFINITY; continue; }
    const float *qi = q + (size_t)i * d, *doi = dout + (size_t)i * d;
#pragma omp parallel for schedule(static)
    for (int j = lo; j <= hi; ++j) p[j] = c.scale * dot_f(qi, k + (size_t)j * d, d);
    double m = -INFINITY;
    for (int j = lo; j <= hi; ++j) if (p[j] > m) m = p[j];
    double l = 0.0;
    for (int j = lo; j <= hi; ++j) { p[j] = exp(p[j] - m); l += p[j]; }
#pragma omp parallel for schedule(static)
    for (int x = 0; x < d; ++x) {
      double acc = 0.0;
      for (int j = lo; j <= hi; ++j) acc += p[j] * (double)v[(size_t)j * d + x];
      oi[x] = acc / l;
    }
    lse[e] = m + log(l);
    double D = 0.0;
    for (int x = 0; x < d; ++x) D += (double)doi[x] * oi[x];
#pragma omp parallel for schedule(static)
    for (int j = lo; j <= hi; ++j) {
      const double P = p[j] / l;
      const double dP = dot_f(doi, v + (size_t)j * d, d);
      ds[j] = P * (dP - D);
      double *dkj = dk + (size_t)j * d, *dvj = dv + (size_t)j * d;
      for (int x = 0; x < d; ++x) {
        dkj[x] += c.scale * ds[j] * (double)qi[x];
        dvj[x] += P * (double)doi[x];
      }
    }
#pragma omp parallel for schedule(static)
    for (int x = 0; x < d; ++x) {
      double acc = 0.0;
      for (int j = lo; j <= hi; ++j) acc += ds[j] * (double)k[(size_t)j * d + x];
      dqi[x] = c.scale * acc;
    }
  }
  free(p); free(ds); free(doc);
}

/* ------------------------------------------------------------------------- */
/* Token-weighted loss aggregation over the P shards.                         */
/* ------------------------------------------------------------------------- */

/*
 * [P3 "Integrarea cu Accelerate"]: every rank computes the loss of its own
 * part of the sequence; the global loss weights each rank by its number of
 * valid tokens, i.e. L = sum_r S_r / sum_r C_r with S_r the sum of per-token
 * cross-entropies and C_r the count of non-ignored tokens of shard r.
 * Per token: l_t = log(sum_v exp(z_tv)) - z_t[y_t] (fp64, max-shifted).
 * logits: [P][T/P][V], labels: [P][T/P].  Returns the number of labels that
 * are neither the ignore index nor in [0, V) (such tokens are not counted).
 * If no token is valid, L is NaN (0/0), like the unsharded mean.
 */
long oracle_loss(int P, long T, int V, const float *logits, const int *labels,
                 int ignore_index, double *shard_sum, long long *shard_count, double *loss) {
  const long per = T / P;
  long bad = 0;
  for (int r = 0; r < P; ++r) { shard_sum[r] = 0.0; shard_count[r] = 0; }
  for (int r = 0; r < P; ++r) {
    double S = 0.0;
    long long C = 0;
    long badr = 0;
#pragma omp parallel for reduction(+ : S, C, badr) schedule(static)
    for (long tt = 0; tt < per; ++tt) {
      const long t = (long)r * per + tt;
      const int y = labels[t];
      if (y == ignore_index) continue;
      if (y < 0 || y >= V) { ++badr; continue; }
      const float *z = logits + (size_t)t * V;
      double m = -INFINITY;
      for (int e = 0; e < V; ++e) if ((double)z[e] > m) m = (double)z[e];
      double acc = 0.0;
      for (int e = 0; e < V; ++e) acc += exp((double)z[e] - m);
      S += (m + log(acc)) - (double)z[y];
      C += 1;
    }
    shard_sum[r] = S;
    shard_count[r] = C;
    bad += badr;
  }
  double Ssum = 0.0;
  long long Csum = 0;
  for (int r = 0; r < P; ++r) { Ssum += shard_sum[r]; Csum += shard_count[r]; }
  *loss = Ssum / (double)Csum;
  return bad;
}

/*
 * Gradient of the aggregated loss with respect to the logits -- the step that
 * follows the aggregation in training.  L = sum_r S_r / sum_r C_r has one
 * denominator for every shard, the global count C = sum_r C_r
 * [P3 "Integrarea cu Accelerate": the loss is weighted by the tokens each rank
 * holds], so for a counted token t:
 *     dL/dz_tv = (softmax(z_t)_v - [v == y_t]) / C,
 * and dL/dz_tv = 0 for an ignored or invalid token.  softmax in fp64 with the
 * maximum subtracted.  logits [T][V] (the shards stacked), labels [T]; writes
 * dlogits [T][V] (fp64) and returns C.  With C = 0 every row is 0.
 */
long long oracle_loss_grad(long T, int V, const float *logits, const int *labels, int ignore_index,
                           double *dlogits) {
  long long C = 0;
  for (long t = 0; t < T; ++t) {
    const int y = labels[t];
    if (y != ignore_index && y >= 0 && y < V) ++C;
  }
#pragma omp parallel for schedule(static)
  for (long t = 0; t < T; ++t) {
    double *g = dlogits + (size_t)t * V;
    const int y = labels[t];
    if (C == 0 || y == ignore_index || y < 0 || y >= V) {
      for (int e = 0; e < V; ++e) g[e] = 0.0;
      continue;
    }
    const float *z = logits + (size_t)t * V;
    double m = -INFINITY;
    for (int e = 0; e < V; ++e) if ((double)z[e] > m) m = (double)z[e];
    double acc = 0.0;
    for (int e = 0; e < V; ++e) acc += exp((double)z[e] - m);
    for (int e = 0; e < V; ++e) g[e] = exp((double)z[e] - m) / acc / (double)C;
    g[y] -= 1.0 / (double)C;
  }
  return C;
}
