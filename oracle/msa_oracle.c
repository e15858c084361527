/*
 * msa_oracle.c -- plain, slow fp64 CPU restatement of the Memory Sparse
 * Attention (MSA) hot path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg call it; the product path never
 * does.  It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (page title, then section):
 *  [EVM]  "Evermind & Shanda Group -- MSA: Memory Sparse Attention for
 *          Efficient End-to-End Memory Model Scaling" (medium summary),
 *          sec. 2 "System architecture", sec. 4B "Memory Parallel & Tiered
 *          Storage", sec. 4C "Memory Interleave".
 *  [BLAB] "MSA: Memory Sparse Attention" (b-lab.team summary), item 1
 *          "Memory-Sparse Attention (MSA) Layer" (Scalable Sparse Attention,
 *          Document-wise RoPE, Global RoPE bullets) and the three-stage
 *          inference pipeline (Global Memory Encoding, Online Routing &
 *          Context Assembly, Sparse Generation).
 *
 * Every value is double; every loop is the definition written out.  The only
 * parallelism is an OpenMP loop over independent outputs (queries, documents,
 * chunks), which does not change any result's arithmetic.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes): chunk scores become a document score by max; cosine per router head,
 * then the mean over heads, then the max over query tokens; RoPE is NeoX
 * rotate-half with base theta; router vectors get no RoPE; token-level RoPE is
 * applied before pooling; a short last chunk is averaged over its own length;
 * ties in top-k go to the lower document id; zero vectors are clamped by eps so
 * their cosine is 0; GQA maps query head h to kv head h / (H_q / H_kv); the
 * softmax scale is 1/sqrt(D); retrieved memory rows come first in rank order
 * and are fully visible, local rows are causal.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EPS 1e-12

/* ---------------------------------------------------------------------------
 * Fixed-length chunking [EVM sec. 2]: document d with tokens [s_d, e_d) is cut
 * into ceil((e_d - s_d) / L) chunks of L tokens; the last one may be short.
 * doc_chunk_off[d] is the index of the first chunk of document d.
 * Returns the total number of chunks, or -1 if a document is empty.
 * ------------------------------------------------------------------------- */
int64_t msa_oracle_doc_chunks(const int64_t *doc_tok_off, int32_t n_docs,
                              int32_t L, int64_t *doc_chunk_off) {
  doc_chunk_off[0] = 0;
  for (int32_t d = 0; d < n_docs; ++d) {
    int64_t len = doc_tok_off[d + 1] - doc_tok_off[d];
    if (len <= 0) return -1;
    doc_chunk_off[d + 1] = doc_chunk_off[d] + (len + L - 1) / L;
  }
  return doc_chunk_off[n_docs];
}

/* ---------------------------------------------------------------------------
 * Rotary position embedding of one head vector x[dim] at position p, NeoX
 * rotate-half form: the pair (x[i], x[i + dim/2]) is rotated by the angle
 * p * theta^(-2i/dim).  Used with document-wise positions for memory keys
 * [BLAB item 1, Document-wise RoPE] and with offset positions for the local
 * query/keys [BLAB item 1, Global RoPE].
 * ------------------------------------------------------------------------- */
static void rope_vec(double *x, int32_t dim, double p, double theta) {
  int32_t half = dim / 2;
  for (int32_t i = 0; i < half; ++i) {
    double freq = pow(theta, -2.0 * (double)i / (double)dim);
    double ang = p * freq;
    double c = cos(ang), s = sin(ang);
    double a = x[i], b = x[i + half];
    x[i] = a * c - b * s;
    x[i + half] = b * c + a * s;
  }
}

/* In place over rows x[n_rows][n_heads][dim], row r at position pos[r]. */
void msa_oracle_rope_rows(double *x, int64_t n_rows, int32_t n_heads,
                          int32_t dim, const int64_t *pos, double theta) {
  for (int64_t r = 0; r < n_rows; ++r)
    for (int32_t h = 0; h < n_heads; ++h)
      rope_vec(x + (r * n_heads + h) * (int64_t)dim, dim, (double)pos[r], theta);
}

/* ---------------------------------------------------------------------------
 * Offline memory encoding [BLAB pipeline stage "Global Memory Encoding";
 * EVM sec. 2 chunk-mean pooling; BLAB item 1 Document-wise RoPE].
 *   K, V   : [n_tok][H_kv][D]   token-major, K before RoPE
 *   Kr     : [n_tok][H_r][d_r]  router keys (no RoPE)
 * For chunk c of document d covering tokens T_c (|T_c| <= L):
 *   Kbar[c]  = (1/|T_c|) sum_{t in T_c} RoPE(K[t], t - s_d)
 *   Vbar[c]  = (1/|T_c|) sum_{t in T_c} V[t]
 *   Krbar[c] = (1/|T_c|) sum_{t in T_c} Kr[t]
 * Token positions restart at 0 in every document.
 * ------------------------------------------------------------------------- */
void msa_oracle_encode(const double *K, const double *V, const double *Kr,
                       const int64_t *doc_tok_off, int32_t n_docs, int32_t L,
                       int32_t H_kv, int32_t D, int32_t H_r, int32_t d_r,
                       double theta, double *Kbar, double *Vbar,
                       double *Krbar) {
  int64_t *doc_chunk_off = (int64_t *)malloc(sizeof(int64_t) * (n_docs + 1));
  msa_oracle_doc_chunks(doc_tok_off, n_docs, L, doc_chunk_off);
  const int64_t wk = (int64_t)H_kv * D, wr = (int64_t)H_r * d_r;
#pragma omp parallel for schedule(dynamic)
  for (int32_t d = 0; d < n_docs; ++d) {
    double *rot = (double *)malloc(sizeof(double) * wk);
    const int64_t s_d = doc_tok_off[d], e_d = doc_tok_off[d + 1];
    for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) {
      const int64_t j = c - doc_chunk_off[d];
      const int64_t t0 = s_d + j * L;
      const int64_t t1 = (t0 + L < e_d) ? t0 + L : e_d;
      const double n = (double)(t1 - t0);
      double *kb = Kbar + c * wk, *vb = Vbar + c * wk, *rb = Krbar + c * wr;
      memset(kb, 0, sizeof(double) * wk);
      memset(vb, 0, sizeof(double) * wk);
      memset(rb, 0, sizeof(double) * wr);
      for (int64_t t = t0; t < t1; ++t) {
        memcpy(rot, K + t * wk, sizeof(double) * wk);
        for (int32_t h = 0; h < H_kv; ++h)
          rope_vec(rot + (int64_t)h * D, D, (double)(t - s_d), theta);
        for (int64_t e = 0; e < wk; ++e) kb[e] += rot[e];
        for (int64_t e = 0; e < wk; ++e) vb[e] += V[t * wk + e];
        for (int64_t e = 0; e < wr; ++e) rb[e] += Kr[t * wr + e];
      }
      for (int64_t e = 0; e < wk; ++e) kb[e] /= n;
      for (int64_t e = 0; e < wk; ++e) vb[e] /= n;
      for (int64_t e = 0; e < wr; ++e) rb[e] /= n;
    }
    free(rot);
  }
  free(doc_chunk_off);
}

/* ---------------------------------------------------------------------------
 * Cosine similarity between two head vectors [EVM sec. 2; BLAB item 1]:
 *   <q, k> / (max(|q|, eps) * max(|k|, eps)).
 * ------------------------------------------------------------------------- */
static double cosine(const double *q, const double *k, int32_t n) {
  double dot = 0.0, qq = 0.0, kk = 0.0;
  for (int32_t i = 0; i < n; ++i) {
    dot += q[i] * k[i];
    qq += q[i] * q[i];
    kk += k[i] * k[i];
  }
  double nq = sqrt(qq), nk = sqrt(kk);
  if (nq < ORACLE_EPS) nq = ORACLE_EPS;
  if (nk < ORACLE_EPS) nk = ORACLE_EPS;
  return dot / (nq * nk);
}

/* Relevance of one query token to one chunk: cosine per router head, then the
 * mean over the router heads [BLAB item 1: per-head mean, then token max]. */
double msa_oracle_chunk_score(const double *qr_tok, const double *krbar_chunk,
                              int32_t H_r, int32_t d_r) {
  double s = 0.0;
  for (int32_t h = 0; h < H_r; ++h)
    s += cosine(qr_tok + (int64_t)h * d_r, krbar_chunk + (int64_t)h * d_r, d_r);
  return s / (double)H_r;
}

/* ---------------------------------------------------------------------------
 * Online routing score [BLAB pipeline stage "Online Routing & Context
 * Assembly"; BLAB item 1].
 *   Qr     : [B][T][H_r][d_r] query router projections (T tokens per query)
 *   Krbar  : [C][H_r][d_r] pooled router keys
 *   doc_score[b][d] <- max(doc_score[b][d],
 *                          max_{t < T} max_{c in chunks(d)} score(Qr[b,t], Krbar[c]))
 * The max-merge into the caller's array is the running state across calls.
 * ------------------------------------------------------------------------- */
void msa_oracle_route(const double *Qr, int32_t B, int32_t T,
                      const double *Krbar, const int64_t *doc_chunk_off,
                      int32_t n_docs, int32_t H_r, int32_t d_r,
                      double *doc_score) {
  const int64_t wr = (int64_t)H_r * d_r;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
  for (int32_t b = 0; b < B; ++b)
    for (int32_t d = 0; d < n_docs; ++d) {
      double best = doc_score[(int64_t)b * n_docs + d];
      for (int32_t t = 0; t < T; ++t) {
        const double *q = Qr + ((int64_t)b * T + t) * wr;
        for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) {
          double s = msa_oracle_chunk_score(q, Krbar + c * wr, H_r, d_r);
          if (s > best) best = s;
        }
      }
      doc_score[(int64_t)b * n_docs + d] = best;
    }
}

/* ---------------------------------------------------------------------------
 * Top-k documents [BLAB item 1 and routing stage; EVM sec. 2]: sort the
 * documents by (score descending, id ascending) and keep the first k.
 * ------------------------------------------------------------------------- */
typedef struct {
  double score;
  int32_t id;
} scored_doc;

static int cmp_scored_doc(const void *pa, const void *pb) {
  const scored_doc *a = (const scored_doc *)pa, *b = (const scored_doc *)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->id > b->id) - (a->id < b->id);
}

void msa_oracle_topk(const double *score, int32_t B, int32_t n_docs, int32_t k,
                     int32_t *ids, double *top_scores) {
#pragma omp parallel for
  for (int32_t b = 0; b < B; ++b) {
    scored_doc *v = (scored_doc *)malloc(sizeof(scored_doc) * n_docs);
    for (int32_t d = 0; d < n_docs; ++d) {
      v[d].score = score[(int64_t)b * n_docs + d];
      v[d].id = d;
    }
    qsort(v, n_docs, sizeof(scored_doc), cmp_scored_doc);
    for (int32_t r = 0; r < k; ++r) {
      ids[(int64_t)b * k + r] = v[r].id;
      if (top_scores) top_scores[(int64_t)b * k + r] = v[r].score;
    }
    free(v);
  }
}

/* ---------------------------------------------------------------------------
 * Sparse generation [BLAB pipeline stage "Sparse Generation"; BLAB item 1
 * Scalable Sparse Attention (concatenate the selected documents' compressed
 * K/V with the query's local K/V) and Global RoPE (the query's positions start
 * at pos_offset, the number k of retrieved blocks)].
 *   Q      : [B][T][H_q][D]        the T new tokens, before RoPE
 *   K_loc, V_loc : [B][L_loc][H_kv][D] every local token so far, K before RoPE;
 *            new token i sits at local index q_start + i
 *   Kbar, Vbar : [C][H_kv][D]      pooled memory (Kbar already rotated per doc)
 *   ids    : [B][k] retrieved documents in rank order
 * For new token i of query b and query head h (kv head g = h / (H_q/H_kv)),
 * j = q_start + i:
 *   context = [Kbar/Vbar rows of chunks of ids[b,0], ..., ids[b,k-1]]
 *             ++ [RoPE(K_loc[b,l,g], pos_offset + l), V_loc[b,l,g]] for l <= j
 *   z = RoPE(Q[b,i,h], pos_offset + j) . key / sqrt(D),  p = softmax(z)
 *   O[b,i,h] = sum p * value;  lse = log sum exp z;  rowsum = sum p.
 * ------------------------------------------------------------------------- */
void msa_oracle_attend(const double *Q, int32_t B, int32_t T, int32_t H_q,
                       const double *K_loc, const double *V_loc, int32_t L_loc,
                       int32_t q_start, const double *Kbar, const double *Vbar,
                       const int64_t *doc_chunk_off, const int32_t *ids,
                       int32_t k, int32_t H_kv, int32_t D, int32_t pos_offset,
                       double theta, double *O, double *lse, double *rowsum) {
  const int32_t group = H_q / H_kv;
  const double scale = 1.0 / sqrt((double)D);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int32_t b = 0; b < B; ++b)
    for (int32_t i = 0; i < T; ++i) {
      const int32_t j = q_start + i;
      int64_t n_mem = 0;
      for (int32_t r = 0; r < k; ++r) {
        int32_t d = ids[(int64_t)b * k + r];
        n_mem += doc_chunk_off[d + 1] - doc_chunk_off[d];
      }
      const int64_t n_ctx = n_mem + (int64_t)j + 1;
      double *z = (double *)malloc(sizeof(double) * n_ctx);
      double *q = (double *)malloc(sizeof(double) * D);
      double *key = (double *)malloc(sizeof(double) * D);
      for (int32_t h = 0; h < H_q; ++h) {
        const int32_t g = h / group;
        memcpy(q, Q + (((int64_t)b * T + i) * H_q + h) * D, sizeof(double) * D);
        rope_vec(q, D, (double)(pos_offset + j), theta);
        /* logits over [memory rows | local rows 0..j] */
        int64_t x = 0;
        for (int32_t r = 0; r < k; ++r) {
          int32_t d = ids[(int64_t)b * k + r];
          for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) {
            const double *kr = Kbar + (c * H_kv + g) * (int64_t)D;
            double dot = 0.0;
            for (int32_t e = 0; e < D; ++e) dot += q[e] * kr[e];
            z[x++] = dot * scale;
          }
        }
        for (int32_t l = 0; l <= j; ++l) {
          memcpy(key, K_loc + (((int64_t)b * L_loc + l) * H_kv + g) * D,
                 sizeof(double) * D);
          rope_vec(key, D, (double)(pos_offset + l), theta);
          double dot = 0.0;
          for (int32_t e = 0; e < D; ++e) dot += q[e] * key[e];
          z[x++] = dot * scale;
        }
        /* softmax */
        double m = -INFINITY;
        for (int64_t y = 0; y < n_ctx; ++y)
          if (z[y] > m) m = z[y];
        double sum = 0.0;
        for (int64_t y = 0; y < n_ctx; ++y) {
          z[y] = exp(z[y] - m);
          sum += z[y];
        }
        double psum = 0.0;
        for (int64_t y = 0; y < n_ctx; ++y) {
          z[y] /= sum;
          psum += z[y];
        }
        /* O = P V */
        double *o = O + (((int64_t)b * T + i) * H_q + h) * D;
        for (int32_t e = 0; e < D; ++e) o[e] = 0.0;
        x = 0;
        for (int32_t r = 0; r < k; ++r) {
          int32_t d = ids[(int64_t)b * k + r];
          for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) {
            const double *vr = Vbar + (c * H_kv + g) * (int64_t)D;
            for (int32_t e = 0; e < D; ++e) o[e] += z[x] * vr[e];
            ++x;
          }
        }
        for (int32_t l = 0; l <= j; ++l) {
          const double *vr = V_loc + (((int64_t)b * L_loc + l) * H_kv + g) * D;
          for (int32_t e = 0; e < D; ++e) o[e] += z[x] * vr[e];
          ++x;
        }
        const int64_t oi = ((int64_t)b * T + i) * H_q + h;
        if (lse) lse[oi] = m + log(sum);
        if (rowsum) rowsum[oi] = psum;
      }
      free(z);
      free(q);
      free(key);
    }
}

/* ---------------------------------------------------------------------------
 * Backward of the routing score, for training the router with an auxiliary
 * routing loss [EVM sec. 4A: the router is supervised with L_aux during
 * continued pre-training].  For one routing call (no carried state):
 *   doc_score[b][d] = max over tokens t and chunks c of d of
 *                     s(b,t,c) = (1/H_r) sum_h cos(Qr[b,t,h], Krbar[c,h]),
 * so, given dL/d doc_score = G[b][d], the gradient flows to the maximising
 * pair (t*, c*) only -- the first in (t ascending, c ascending) order among
 * equal maxima -- and there:
 *   d cos(q, k) / dq = k / (|q| |k|) - cos(q, k) q / |q|^2   (|q|, |k| > eps;
 *   a norm clamped at eps is a constant: its term drops),
 * and symmetrically for k.  dQr and dKrbar are overwritten.
 * ------------------------------------------------------------------------- */
static void cosine_grad(const double *q, const double *k, int32_t n, double g,
                        double *dq, double *dk) {
  double dot = 0.0, qq = 0.0, kk = 0.0;
  for (int32_t i = 0; i < n; ++i) {
    dot += q[i] * k[i];
    qq += q[i] * q[i];
    kk += k[i] * k[i];
  }
  const double rq = sqrt(qq), rk = sqrt(kk);
  const double nq = rq < ORACLE_EPS ? ORACLE_EPS : rq;
  const double nk = rk < ORACLE_EPS ? ORACLE_EPS : rk;
  const double c = dot / (nq * nk);
  for (int32_t i = 0; i < n; ++i) {
    double gq = k[i] / (nq * nk), gk = q[i] / (nq * nk);
    if (rq >= ORACLE_EPS) gq -= c * q[i] / (nq * nq);
    if (rk >= ORACLE_EPS) gk -= c * k[i] / (nk * nk);
    dq[i] += g * gq;
    dk[i] += g * gk;
  }
}

void msa_oracle_route_backward(const double *Qr, int32_t B, int32_t T,
                               const double *Krbar, const int64_t *doc_chunk_off,
                               int32_t n_docs, int32_t H_r, int32_t d_r,
                               const double *G, double *dQr, double *dKrbar) {
  const int64_t wr = (int64_t)H_r * d_r;
  memset(dQr, 0, sizeof(double) * (size_t)B * T * wr);
  memset(dKrbar, 0, sizeof(double) * (size_t)doc_chunk_off[n_docs] * wr);
  for (int32_t b = 0; b < B; ++b)
    for (int32_t d = 0; d < n_docs; ++d) {
      const double g = G[(int64_t)b * n_docs + d];
      if (g == 0.0 || T < 1 || doc_chunk_off[d + 1] == doc_chunk_off[d]) continue;
      double best = -INFINITY;
      int32_t tb = 0;
      int64_t cb = doc_chunk_off[d];
      for (int32_t t = 0; t < T; ++t)
        for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) {
          const double s = msa_oracle_chunk_score(Qr + ((int64_t)b * T + t) * wr,
                                                  Krbar + c * wr, H_r, d_r);
          if (s > best) {
            best = s;
            tb = t;
            cb = c;
          }
        }
      for (int32_t h = 0; h < H_r; ++h)
        cosine_grad(Qr + ((int64_t)b * T + tb) * wr + (int64_t)h * d_r,
                    Krbar + cb * wr + (int64_t)h * d_r, d_r, g / (double)H_r,
                    dQr + ((int64_t)b * T + tb) * wr + (int64_t)h * d_r,
                    dKrbar + cb * wr + (int64_t)h * d_r);
    }
}

/* ---------------------------------------------------------------------------
 * Backward of the sparse attention [BLAB stage "Sparse Generation"; the same
 * context and masking as msa_oracle_attend].  With p = softmax(z) over the
 * context rows y of (b, i, h), z_y = scale * <q', key_y>, q' = RoPE(Q) and
 * O = sum_y p_y value_y, given dO:
 *   dp_y  = <dO, value_y>,        Dv = <dO, O> = sum_y p_y dp_y
 *   dz_y  = p_y (dp_y - Dv)
 *   dq'  += scale dz_y key_y;     dQ = RoPE^-1(dq') (the rotation's transpose)
 *   dkey_y += scale dz_y q';      dvalue_y += p_y dO
 * Memory rows accumulate into dKbar / dVbar [C][H_kv][D] (keys as stored:
 * pooled after document-wise RoPE); local rows into dK_loc / dV_loc
 * [B][L_loc][H_kv][D], dK_loc with respect to the keys BEFORE their RoPE at
 * pos_offset + l (the inputs of msa_oracle_attend).  Every output is
 * overwritten (dKbar / dVbar: n_chunks rows).  Plain loops, no parallelism
 * (outputs are shared).
 * ------------------------------------------------------------------------- */
static void rope_vec_inverse(double *x, int32_t dim, double p, double theta) {
  rope_vec(x, dim, -p, theta);  /* a rotation by -angle is the transpose */
}

void msa_oracle_attend_backward(const double *Q, int32_t B, int32_t T, int32_t H_q,
                                const double *K_loc, const double *V_loc, int32_t L_loc,
                                int32_t q_start, const double *Kbar, const double *Vbar,
                                const int64_t *doc_chunk_off, const int32_t *ids,
                                int32_t k, int32_t H_kv, int32_t D, int32_t pos_offset,
                                double theta, const double *dO, int64_t n_chunks, double *dQ,
                                double *dK_loc, double *dV_loc, double *dKbar, double *dVbar) {
  const int32_t group = H_q / H_kv;
  const double scale = 1.0 / sqrt((double)D);
  memset(dQ, 0, sizeof(double) * (size_t)B * T * H_q * D);
  memset(dK_loc, 0, sizeof(double) * (size_t)B * L_loc * H_kv * D);
  memset(dV_loc, 0, sizeof(double) * (size_t)B * L_loc * H_kv * D);
  memset(dKbar, 0, sizeof(double) * (size_t)n_chunks * H_kv * D);
  memset(dVbar, 0, sizeof(double) * (size_t)n_chunks * H_kv * D);
  for (int32_t b = 0; b < B; ++b)
    for (int32_t i = 0; i < T; ++i) {
      const int32_t j = q_start + i;
      int64_t n_mem = 0;
      for (int32_t r = 0; r < k; ++r) {
        const int32_t d = ids[(int64_t)b * k + r];
        n_mem += doc_chunk_off[d + 1] - doc_chunk_off[d];
      }
      const int64_t n_ctx = n_mem + (int64_t)j + 1;
      double *z = (double *)malloc(sizeof(double) * n_ctx);
      double **key = (double **)malloc(sizeof(double *) * n_ctx);
      double **val = (double **)malloc(sizeof(double *) * n_ctx);
      double **dkey = (double **)malloc(sizeof(double *) * n_ctx);
      double **dval = (double **)malloc(sizeof(double *) * n_ctx);
      double *rot = (double *)malloc(sizeof(double) * ((size_t)j + 1) * D);
      double *drot = (double *)malloc(sizeof(double) * ((size_t)j + 1) * D);
      double *q = (double *)malloc(sizeof(double) * D);
      double *dq = (double *)malloc(sizeof(double) * D);
      double *o = (double *)malloc(sizeof(double) * D);
      for (int32_t h = 0; h < H_q; ++h) {
        const int32_t g = h / group;
        /* the context rows, in the forward's order */
        int64_t x = 0;
        for (int32_t r = 0; r < k; ++r) {
          const int32_t d = ids[(int64_t)b * k + r];
          for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) {
            key[x] = (double *)(Kbar + (c * H_kv + g) * (int64_t)D);
            val[x] = (double *)(Vbar + (c * H_kv + g) * (int64_t)D);
            dkey[x] = dKbar + (c * H_kv + g) * (int64_t)D;
            dval[x] = dVbar + (c * H_kv + g) * (int64_t)D;
            ++x;
          }
        }
        for (int32_t l = 0; l <= j; ++l) {
          double *kr = rot + (int64_t)l * D;
          memcpy(kr, K_loc + (((int64_t)b * L_loc + l) * H_kv + g) * D, sizeof(double) * D);
          rope_vec(kr, D, (double)(pos_offset + l), theta);
          memset(drot + (int64_t)l * D, 0, sizeof(double) * D);
          key[x] = kr;
          val[x] = (double *)(V_loc + (((int64_t)b * L_loc + l) * H_kv + g) * D);
          dkey[x] = drot + (int64_t)l * D;
          dval[x] = dV_loc + (((int64_t)b * L_loc + l) * H_kv + g) * D;
          ++x;
        }
        memcpy(q, Q + (((int64_t)b * T + i) * H_q + h) * D, sizeof(double) * D);
        rope_vec(q, D, (double)(pos_offset + j), theta);
        /* forward: p and O */
        double m = -INFINITY;
        for (int64_t y = 0; y < n_ctx; ++y) {
          double dot = 0.0;
          for (int32_t e = 0; e < D; ++e) dot += q[e] * key[y][e];
          z[y] = dot * scale;
          if (z[y] > m) m = z[y];
        }
        double sum = 0.0;
        for (int64_t y = 0; y < n_ctx; ++y) {
          z[y] = exp(z[y] - m);
          sum += z[y];
        }
        for (int32_t e = 0; e < D; ++e) o[e] = 0.0;
        for (int64_t y = 0; y < n_ctx; ++y) {
          z[y] /= sum;
          for (int32_t e = 0; e < D; ++e) o[e] += z[y] * val[y][e];
        }
        /* backward */
        const double *go = dO + (((int64_t)b * T + i) * H_q + h) * D;
        double Dv = 0.0;
        for (int32_t e = 0; e < D; ++e) Dv += go[e] * o[e];
        for (int32_t e = 0; e < D; ++e) dq[e] = 0.0;
        for (int64_t y = 0; y < n_ctx; ++y) {
          double dp = 0.0;
          for (int32_t e = 0; e < D; ++e) dp += go[e] * val[y][e];
          const double dz = z[y] * (dp - Dv);
          for (int32_t e = 0; e < D; ++e) {
            dq[e] += scale * dz * key[y][e];
            dkey[y][e] += scale * dz * q[e];
            dval[y][e] += z[y] * go[e];
          }
        }
        rope_vec_inverse(dq, D, (double)(pos_offset + j), theta);
        memcpy(dQ + (((int64_t)b * T + i) * H_q + h) * D, dq, sizeof(double) * D);
        /* local keys: back through their RoPE */
        for (int32_t l = 0; l <= j; ++l) {
          double *dr = drot + (int64_t)l * D;
          rope_vec_inverse(dr, D, (double)(pos_offset + l), theta);
          double *dst = dK_loc + (((int64_t)b * L_loc + l) * H_kv + g) * D;
          for (int32_t e = 0; e < D; ++e) dst[e] += dr[e];
        }
      }
      free(z);
      free(key);
      free(val);
      free(dkey);
      free(dval);
      free(rot);
      free(drot);
      free(q);
      free(dq);
      free(o);
    }
}
