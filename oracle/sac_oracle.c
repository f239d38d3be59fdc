/*
 * sac_oracle.c -- fp64 CPU oracle of the DeepSeek-V4 hybrid long-range attention forward
 * (compressor, Lightning Indexer + top-k, shared K=V sparse/sliding attention, per-head sink,
 * partial interleaved RoPE with the inverse rotation of the output).
 *
 * TEST INFRASTRUCTURE. This file is the slow, obviously-correct definition that the CUDA path is
 * checked against. Only the test suite, the package smoke check and the CPU-baseline leg of the
 * benchmark may load it. It shares no code, header, table or helper with the CUDA library.
 *
 * Source: the "DeepSeek-V4" model documentation page of Hugging Face Transformers, sections
 * "Hybrid attention (section 2.3)", "Attention mask layout", "Cache layers" and
 * "DeepseekV4Config". The page names the paper's equations (13-17 indexer, 26 inverse RoPE,
 * 27 sink) but does not print them; every step below that goes beyond the page's prose is a
 * reading and is marked [reading]. Parity status per function is stated in its comment:
 *   - compressor gate formula: parity unpinned (a reading; its special cases are pinned)
 *   - indexer score formula:   parity unpinned (a reading; its special cases are pinned)
 *
 * All arithmetic is IEEE fp64, in the order written; OpenMP only splits independent query rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Attention-relevant hyper-parameters ("DeepseekV4Config" section: head_dim, sliding_window,
 * compress_rates, index_n_heads, index_head_dim, index_topk, rope_theta / compress_rope_theta,
 * partial_rotary_factor). */
typedef struct {
  int B, S, H, D, R;   /* batch, tokens, query heads, head_dim, rope channels (trailing)     */
  double theta;        /* RoPE base for q, window keys and pool entries of this layer         */
  int m, L;            /* compression rate and compressor window length (0, 0 for sliding)   */
  int W;               /* sliding_window                                                      */
  int nI, cI, k;       /* index_n_heads, index_head_dim, index_topk (CSA only)                */
  double scale;        /* softmax scale tau                                                   */
  int64_t pos0;        /* absolute position of token 0                                        */
  int bf16_pools;      /* 1: pools are cached in bf16 (see orc_round_bf16)                     */
  double yarn_factor;  /* YaRN context scale s (<= 1: plain RoPE)                             */
  int yarn_orig;       /* YaRN original context length L                                      */
  double yarn_beta_fast, yarn_beta_slow;  /* YaRN ramp bounds beta (fast) and alpha (slow)    */
} orc_params;

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* [reading] The compressor's pools are cached tensors ("Cache layers": compressor / indexer
 * pool) held in the layer's working dtype. For a bf16 layer each stored pool entry is the fp32
 * value rounded to the nearest bf16, ties to even. The top-k is an integer decision taken from
 * scores of the stored indexer pool, so the oracle scores the same stored values. */
double orc_round_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, sizeof(u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  u &= 0xFFFF0000u;
  memcpy(&f, &u, sizeof(f));
  return (double)f;
}

static void round_pool(const orc_params *p, double *x, size_t n) {
  if (!p->bf16_pools) return;
  for (size_t i = 0; i < n; ++i) x[i] = orc_round_bf16(x[i]);
}

/* ---------------------------------------------------------------------------------------------
 * Partial interleaved-pair RoPE ("Hybrid attention", shared skeleton, partial RoPE bullet):
 * only the trailing R channels of a head rotate; channel pairs are (D-R+2i, D-R+2i+1);
 * pair i turns by angle pos * f_i. A negative pos gives the inverse rotation (the "-i" rotation
 * the page applies to the rope slice of the attention output, eq. 26).
 *
 * Frequencies. Plain RoPE: f_i = theta^(-2i/R). The config pairs compress_rope_theta with a YaRN
 * rope scaling ("DeepseekV4Config") but gives none of its parameters, so they are arguments here
 * ([reading]: factor <= 1 means no scaling). YaRN (Peng et al. 2023, "YaRN:
 * Efficient Context Window Extension of Large Language Models", the "NTK-by-parts"
 * interpolation): with context scale s and original context length L, pair i completes
 * r_i = L / (2 pi / f_i) turns over L tokens; the ramp gamma_i = 0 for r_i < alpha, 1 for
 * r_i > beta and (r_i - alpha) / (beta - alpha) between; the scaled frequency is
 * (1 - gamma_i) * f_i / s + gamma_i * f_i (slow pairs interpolated, fast pairs kept). YaRN's
 * attention temperature multiplies the logits only, so it lives in the softmax scale (an input).
 * ------------------------------------------------------------------------------------------- */
double orc_rope_freq(int i, int R, double theta, double s, int L, double beta_fast,
                     double beta_slow) {
  double f = pow(theta, -2.0 * (double)i / (double)R);
  if (!(s > 1.0)) return f;
  const double pi = 3.14159265358979323846;
  double r = (double)L / (2.0 * pi / f);
  double gamma;
  if (r < beta_slow) gamma = 0.0;
  else if (r > beta_fast) gamma = 1.0;
  else gamma = (r - beta_slow) / (beta_fast - beta_slow);
  return (1.0 - gamma) * f / s + gamma * f;
}

void orc_rope_yarn(double *x, int D, int R, double theta, double s, int L, double beta_fast,
                   double beta_slow, double pos) {
  for (int i = 0; i < R / 2; ++i) {
    double phi = pos * orc_rope_freq(i, R, theta, s, L, beta_fast, beta_slow);
    double c = cos(phi), sn = sin(phi);
    double *p = x + (D - R) + 2 * i;
    double a = p[0], b = p[1];
    p[0] = a * c - b * sn;
    p[1] = a * sn + b * c;
  }
}

void orc_rope(double *x, int D, int R, double theta, double pos) {
  orc_rope_yarn(x, D, R, theta, 1.0, 1, 0.0, 0.0, pos);
}

/* The rotation of a layer: its base and, when yarn_factor > 1, its YaRN frequencies. */
static void layer_rope(const orc_params *p, double *x, double pos) {
  orc_rope_yarn(x, p->D, p->R, p->theta, p->yarn_factor, p->yarn_orig, p->yarn_beta_fast,
                p->yarn_beta_slow, pos);
}

/* ---------------------------------------------------------------------------------------------
 * Compressor ("Hybrid attention": CSA pool with overlapping windows, HCA pool with
 * non-overlapping windows; "Cache layers": buffer / pool / count / overlap state).
 * [reading] Entry w pools the tokens of the window that closes at token (w+1)*m - 1:
 *   window = [(w+1)*m - L, (w+1)*m) clipped to [0, S)   (CSA: L = 2m; HCA: L = m)
 *   offset of token j in the window: o_j = j - (w+1)*m + L  (last token has offset L-1)
 *   gate g_j = <x_j, u> + bias[o_j];  alpha = softmax over the window;  C_w = sum alpha_j x_j
 * The entry count is N = floor(S/m): a trailing window that has not closed yields no entry
 * ("Attention mask layout", HCA paragraph: an entry exists once its source window closed).
 * Parity unpinned for the gate formula; pinned special cases live in the tests.
 * x: [B,S,C], u: [C], bias: [L], out: [B,N,C]. Returns N.
 * ------------------------------------------------------------------------------------------- */
long orc_compress(int B, int S, int C, int m, int L, const double *x, const double *u,
                  const double *bias, double *out) {
  long N = S / m;
  for (int b = 0; b < B; ++b) {
    for (long w = 0; w < N; ++w) {
      long hi = (w + 1) * (long)m;
      long lo = hi - L;
      if (lo < 0) lo = 0;
      long n = hi - lo;
      double *g = (double *)malloc(sizeof(double) * (size_t)n);
      double gmax = -INFINITY;
      for (long j = lo; j < hi; ++j) {
        const double *xj = x + ((size_t)b * S + j) * C;
        double d = 0.0;
        for (int c = 0; c < C; ++c) d += xj[c] * u[c];
        d += bias[j - hi + L];
        g[j - lo] = d;
        if (d > gmax) gmax = d;
      }
      double z = 0.0;
      for (long j = 0; j < n; ++j) { g[j] = exp(g[j] - gmax); z += g[j]; }
      double *cw = out + ((size_t)b * N + w) * C;
      for (int c = 0; c < C; ++c) cw[c] = 0.0;
      for (long j = lo; j < hi; ++j) {
        const double *xj = x + ((size_t)b * S + j) * C;
        double a = g[j - lo] / z;
        for (int c = 0; c < C; ++c) cw[c] += a * xj[c];
      }
      free(g);
    }
  }
  return N;
}

/* Entry visibility ("Attention mask layout", HCA paragraph): query t sees entry w iff
 * w < floor((t+1)/m), i.e. the entry's window closed at or before t. */
static long visible_entries(long t, int m) { return (t + 1) / m; }

/* ---------------------------------------------------------------------------------------------
 * Lightning Indexer score of one query against the first nvis entries of the indexer pool
 * ("Hybrid attention", CSA bullet, eq. 13-17; "DeepseekV4Config": index_n_heads, index_head_dim).
 * [reading] I[t,w] = sum_h wI[t,h] * max(0, <qI[t,h], KI_w>). Entries w >= nvis get -inf.
 * Parity unpinned for the formula; pinned special cases live in the tests.
 * qI_t: [nI, cI], wI_t: [nI], KI: [N, cI], out: [N].
 * ------------------------------------------------------------------------------------------- */
void orc_index_scores(int N, int nI, int cI, const double *qI_t, const double *wI_t,
                      const double *KI, long nvis, double *out) {
  for (long w = 0; w < N; ++w) {
    if (w >= nvis) { out[w] = -INFINITY; continue; }
    double s = 0.0;
    for (int h = 0; h < nI; ++h) {
      double d = 0.0;
      for (int c = 0; c < cI; ++c) d += qI_t[(size_t)h * cI + c] * KI[(size_t)w * cI + c];
      s += wI_t[h] * (d > 0.0 ? d : 0.0);
    }
    out[w] = s;
  }
}

/* Top-k ("Hybrid attention", CSA bullet, eq. 17; "Attention mask layout", CSA paragraph):
 * the k visible entries with the largest score, ordered by score descending with ties going to
 * the lower entry index; slots beyond the visible count hold the sentinel -1. */
typedef struct { double s; long w; } orc_cand;
static int cand_cmp(const void *pa, const void *pb) {
  const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->w < b->w) ? -1 : (a->w > b->w) ? 1 : 0;
}
int orc_topk(const double *scores, long nvis, int k, int32_t *idx) {
  orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)(nvis > 0 ? nvis : 1));
  for (long w = 0; w < nvis; ++w) { c[w].s = scores[w]; c[w].w = w; }
  qsort(c, (size_t)nvis, sizeof(orc_cand), cand_cmp);
  int n = nvis < k ? (int)nvis : k;
  for (int i = 0; i < k; ++i) idx[i] = i < n ? (int32_t)c[i].w : -1;
  free(c);
  return n;
}

/* ---------------------------------------------------------------------------------------------
 * Attention of one query over an explicit key list ("Hybrid attention": shared K=V multi-query
 * attention, one KV head read as both key and value; per-head learnable sink, eq. 27).
 * [reading of eq. 27] the sink is one extra logit per head with a zero value vector:
 *   p_x = exp(l_x) / (exp(sink_h) + sum_y exp(l_y)),  l_x = scale * <q_h, k_x>,  o_h = sum p_x k_x
 * qrot: [H,D] (already rotated), keys: [nk,D] (already rotated), o: [H,D].
 * ------------------------------------------------------------------------------------------- */
void orc_attend(int H, int D, double scale, const double *qrot, long nk, const double *keys,
                const double *sinks, double *o) {
  double *l = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
  for (int h = 0; h < H; ++h) {
    const double *qh = qrot + (size_t)h * D;
    double mx = sinks[h];
    for (long x = 0; x < nk; ++x) {
      double d = 0.0;
      for (int c = 0; c < D; ++c) d += qh[c] * keys[(size_t)x * D + c];
      l[x] = scale * d;
      if (l[x] > mx) mx = l[x];
    }
    double z = exp(sinks[h] - mx);
    for (long x = 0; x < nk; ++x) { l[x] = exp(l[x] - mx); z += l[x]; }
    double *oh = o + (size_t)h * D;
    for (int c = 0; c < D; ++c) oh[c] = 0.0;
    for (long x = 0; x < nk; ++x) {
      double p = l[x] / z;
      for (int c = 0; c < D; ++c) oh[c] += p * keys[(size_t)x * D + c];
    }
  }
  free(l);
}

/* Query side of one row: rotate q at P_t, attend, rotate the output's rope slice by -P_t
 * (eq. 26), so each key contributes as a function of its distance to the query. */
static void attend_row(const orc_params *p, const double *q_t, double pos_t, long nk,
                       const double *keys, const double *sinks, double *o_t) {
  size_t hd = (size_t)p->H * p->D;
  double *qr = (double *)malloc(sizeof(double) * hd);
  memcpy(qr, q_t, sizeof(double) * hd);
  for (int h = 0; h < p->H; ++h) layer_rope(p, qr + (size_t)h * p->D, pos_t);
  orc_attend(p->H, p->D, p->scale, qr, nk, keys, sinks, o_t);
  for (int h = 0; h < p->H; ++h) layer_rope(p, o_t + (size_t)h * p->D, -pos_t);
  free(qr);
}

/* Sliding-window key set of query t ("Hybrid attention", sliding-window branch bullet;
 * "Attention mask layout", sliding-only paragraph): [reading] W tokens including the diagonal,
 * j in (t-W, t]. Returns the first key index. */
static long window_lo(long t, int W) {
  long lo = t - W + 1;
  return lo < 0 ? 0 : lo;
}

/* Copy kv row j of batch b, rotated at its absolute position. */
static void rotated_kv_row(const orc_params *p, const double *kv, int b, long j, double *dst) {
  memcpy(dst, kv + ((size_t)b * p->S + j) * p->D, sizeof(double) * p->D);
  layer_rope(p, dst, (double)(p->pos0 + j));
}

/* [reading] pool entry w is rotated at the first position of the block it stands for,
 * p_w = pos0 + w*m ("entry 0 covers positions 0..7" in the HCA paragraph). */
static double entry_pos(const orc_params *p, long w) { return (double)(p->pos0 + w * (long)p->m); }

/* Rows to compute: rows[i] = b*S + t, or all rows when rows == NULL. The per-row arrays (q, qI,
 * wI, o, topk_out, topk_in) hold the listed rows in list order: entry i belongs to rows[i]. */
static long row_at(const orc_params *p, const int64_t *rows, long i) {
  (void)p;
  return rows ? (long)rows[i] : i;
}

/* ---------------------------------------------------------------------------------------------
 * Full prefill forwards. Inputs are un-rotated. kv: [B,S,D], kI: [B,S,cI]; per-row arrays are
 * [B*S,...] or, with a row list, [nrows,...] in list order: q [.,H,D], qI [.,nI,cI], wI [.,nI],
 * o [.,H,D], topk_out/topk_in [.,k]. pool_out (nullable): rotated pool [B,N,D]. idx_pool_out (nullable): [B,N,cI].
 * topk_out (nullable): [B,S,k]. topk_in (nullable): selections to use instead of the oracle's
 * own (for attention parity on a validated alternative selection inside the tie band).
 * ------------------------------------------------------------------------------------------- */
int orc_swa_forward(const orc_params *p, const double *q, const double *kv, const double *sinks,
                    double *o, const int64_t *rows, long nrows) {
  long total = rows ? nrows : (long)p->B * p->S;
#pragma omp parallel for schedule(dynamic, 1)
  for (long i = 0; i < total; ++i) {
    long r = row_at(p, rows, i);
    int b = (int)(r / p->S);
    long t = r % p->S;
    long lo = window_lo(t, p->W);
    long nk = t - lo + 1;
    double *keys = (double *)malloc(sizeof(double) * (size_t)nk * p->D);
    for (long j = lo; j <= t; ++j) rotated_kv_row(p, kv, b, j, keys + (size_t)(j - lo) * p->D);
    attend_row(p, q + (size_t)i * p->H * p->D, (double)(p->pos0 + t), nk, keys, sinks,
               o + (size_t)i * p->H * p->D);
    free(keys);
  }
  return 0;
}

/* Rotated pool: compress then rotate entry w at p_w. Returns N. */
static long rotated_pool(const orc_params *p, const double *kv, const double *u,
                         const double *bias, double *pool) {
  long N = orc_compress(p->B, p->S, p->D, p->m, p->L, kv, u, bias, pool);
  for (int b = 0; b < p->B; ++b)
    for (long w = 0; w < N; ++w)
      layer_rope(p, pool + ((size_t)b * N + w) * p->D, entry_pos(p, w));
  round_pool(p, pool, (size_t)p->B * N * p->D);
  return N;
}

int orc_hca_forward(const orc_params *p, const double *q, const double *kv, const double *u,
                    const double *bias, const double *sinks, double *o, double *pool_out,
                    const int64_t *rows, long nrows) {
  long N = p->S / p->m;
  double *pool = (double *)malloc(sizeof(double) * ((size_t)p->B * N * p->D + 1));
  rotated_pool(p, kv, u, bias, pool);
  if (pool_out) memcpy(pool_out, pool, sizeof(double) * (size_t)p->B * N * p->D);
  long total = rows ? nrows : (long)p->B * p->S;
#pragma omp parallel for schedule(dynamic, 1)
  for (long i = 0; i < total; ++i) {
    long r = row_at(p, rows, i);
    int b = (int)(r / p->S);
    long t = r % p->S;
    long lo = window_lo(t, p->W);
    long nwin = t - lo + 1;
    long nvis = visible_entries(t, p->m);
    long nk = nwin + nvis;
    double *keys = (double *)malloc(sizeof(double) * (size_t)nk * p->D);
    for (long j = lo; j <= t; ++j) rotated_kv_row(p, kv, b, j, keys + (size_t)(j - lo) * p->D);
    for (long w = 0; w < nvis; ++w)
      memcpy(keys + (size_t)(nwin + w) * p->D, pool + ((size_t)b * N + w) * p->D,
             sizeof(double) * p->D);
    attend_row(p, q + (size_t)i * p->H * p->D, (double)(p->pos0 + t), nk, keys, sinks,
               o + (size_t)i * p->H * p->D);
    free(keys);
  }
  free(pool);
  return 0;
}

int orc_csa_forward(const orc_params *p, const double *q, const double *kv, const double *u,
                    const double *bias, const double *qI, const double *wI, const double *kI,
                    const double *uI, const double *bI, const double *sinks, double *o,
                    int32_t *topk_out, double *pool_out, double *idx_pool_out,
                    const int32_t *topk_in, const int64_t *rows, long nrows) {
  long N = p->S / p->m;
  double *pool = (double *)malloc(sizeof(double) * ((size_t)p->B * N * p->D + 1));
  double *kpool = (double *)malloc(sizeof(double) * ((size_t)p->B * N * p->cI + 1));
  rotated_pool(p, kv, u, bias, pool);
  /* the indexer pool: same windows over the indexer key stream, its own gate, no rotation
   * ("Cache layers": parallel indexer buffer / pool / count / overlap at index_head_dim) */
  orc_compress(p->B, p->S, p->cI, p->m, p->L, kI, uI, bI, kpool);
  round_pool(p, kpool, (size_t)p->B * N * p->cI);
  if (pool_out) memcpy(pool_out, pool, sizeof(double) * (size_t)p->B * N * p->D);
  if (idx_pool_out) memcpy(idx_pool_out, kpool, sizeof(double) * (size_t)p->B * N * p->cI);
  long total = rows ? nrows : (long)p->B * p->S;
#pragma omp parallel for schedule(dynamic, 1)
  for (long i = 0; i < total; ++i) {
    long r = row_at(p, rows, i);
    int b = (int)(r / p->S);
    long t = r % p->S;
    long nvis = visible_entries(t, p->m);
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)p->k);
    if (topk_in) {
      memcpy(sel, topk_in + (size_t)i * p->k, sizeof(int32_t) * (size_t)p->k);
    } else {
      double *sc = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
      orc_index_scores((int)N, p->nI, p->cI, qI + (size_t)i * p->nI * p->cI,
                       wI + (size_t)i * p->nI, kpool + (size_t)b * N * p->cI, nvis, sc);
      orc_topk(sc, nvis, p->k, sel);
      free(sc);
    }
    if (topk_out) memcpy(topk_out + (size_t)i * p->k, sel, sizeof(int32_t) * (size_t)p->k);
    long lo = window_lo(t, p->W);
    long nwin = t - lo + 1;
    long nsel = 0;
    for (int s = 0; s < p->k; ++s) nsel += sel[s] >= 0;
    double *keys = (double *)malloc(sizeof(double) * (size_t)(nwin + nsel) * p->D);
    for (long j = lo; j <= t; ++j) rotated_kv_row(p, kv, b, j, keys + (size_t)(j - lo) * p->D);
    long x = nwin;
    for (int s = 0; s < p->k; ++s) {
      if (sel[s] < 0) continue;
      memcpy(keys + (size_t)x * p->D, pool + ((size_t)b * N + sel[s]) * p->D,
             sizeof(double) * p->D);
      ++x;
    }
    attend_row(p, q + (size_t)i * p->H * p->D, (double)(p->pos0 + t), nwin + nsel, keys, sinks,
               o + (size_t)i * p->H * p->D);
    free(keys);
    free(sel);
  }
  free(pool);
  free(kpool);
  return 0;
}

/* Full-row indexer scores for listed rows (rows[i] = b*S + t): qI [nrows,nI,cI], wI [nrows,nI]
 * in list order, out [nrows, N] with -inf beyond the visible count. Uses the oracle's own
 * indexer pool. */
int orc_csa_index_scores(const orc_params *p, const double *qI, const double *wI,
                         const double *kI, const double *uI, const double *bI,
                         const int64_t *rows, long nrows, double *out) {
  long N = p->S / p->m;
  double *kpool = (double *)malloc(sizeof(double) * ((size_t)p->B * N * p->cI + 1));
  orc_compress(p->B, p->S, p->cI, p->m, p->L, kI, uI, bI, kpool);
  round_pool(p, kpool, (size_t)p->B * N * p->cI);
#pragma omp parallel for schedule(dynamic, 1)
  for (long i = 0; i < nrows; ++i) {
    long r = (long)rows[i];
    int b = (int)(r / p->S);
    long t = r % p->S;
    orc_index_scores((int)N, p->nI, p->cI, qI + (size_t)i * p->nI * p->cI,
                     wI + (size_t)i * p->nI, kpool + (size_t)b * N * p->cI,
                     visible_entries(t, p->m), out + (size_t)i * N);
  }
  free(kpool);
  return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Decode over a paged cache ("Cache layers": sliding-window K=V plus compressor pool per layer).
 * [reading] cache contract: kv pages hold kv already rotated at the token's absolute position,
 * pool pages hold entries already rotated at p_w, indexer pool pages are not rotated. ctx_lens
 * counts the new token, so the query sits at t = ctx-1 and sees floor(ctx/m) entries. Row j of a
 * sequence lives at page block_table[s*max_pages + j/page_size], row j % page_size.
 * q: [nseq,H,D] un-rotated; o: [nseq,H,D]. m = 0 means a sliding-only layer.
 * ------------------------------------------------------------------------------------------- */
static const double *paged_row(const double *pages, const int32_t *bt, int s, int max_pages,
                               int page_size, long j, int width) {
  int page = bt[(size_t)s * max_pages + j / page_size];
  return pages + ((size_t)page * page_size + (size_t)(j % page_size)) * width;
}

int orc_decode(const orc_params *p, int nseq, const double *q, const double *kv_pages,
               const int32_t *kv_bt, int max_pages, const int32_t *ctx_lens, int page_size,
               const double *pool_pages, const double *idx_pool_pages, const int32_t *pool_bt,
               int max_pool_pages, const double *qI, const double *wI, const double *sinks,
               double *o, int32_t *topk_out, const int32_t *topk_in) {
  int is_csa = p->m > 0 && p->k > 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < nseq; ++s) {
    long ctx = ctx_lens[s];
    long t = ctx - 1;
    long lo = window_lo(t, p->W);
    long nwin = t - lo + 1;
    long nvis = p->m > 0 ? visible_entries(t, p->m) : 0;
    int32_t *sel = NULL;
    long npool = nvis;
    if (is_csa) {
      sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)p->k);
      if (topk_in) {
        memcpy(sel, topk_in + (size_t)s * p->k, sizeof(int32_t) * (size_t)p->k);
      } else {
        double *kp = (double *)malloc(sizeof(double) * ((size_t)nvis * p->cI + 1));
        for (long w = 0; w < nvis; ++w)
          memcpy(kp + (size_t)w * p->cI,
                 paged_row(idx_pool_pages, pool_bt, s, max_pool_pages, page_size, w, p->cI),
                 sizeof(double) * p->cI);
        double *sc = (double *)malloc(sizeof(double) * ((size_t)nvis + 1));
        orc_index_scores((int)nvis, p->nI, p->cI, qI + (size_t)s * p->nI * p->cI,
                         wI + (size_t)s * p->nI, kp, nvis, sc);
        orc_topk(sc, nvis, p->k, sel);
        free(sc);
        free(kp);
      }
      if (topk_out) memcpy(topk_out + (size_t)s * p->k, sel, sizeof(int32_t) * (size_t)p->k);
      npool = 0;
      for (int i = 0; i < p->k; ++i) npool += sel[i] >= 0;
    }
    double *keys = (double *)malloc(sizeof(double) * ((size_t)(nwin + npool) * p->D + 1));
    for (long j = lo; j <= t; ++j)
      memcpy(keys + (size_t)(j - lo) * p->D,
             paged_row(kv_pages, kv_bt, s, max_pages, page_size, j, p->D), sizeof(double) * p->D);
    long x = nwin;
    if (is_csa) {
      for (int i = 0; i < p->k; ++i) {
        if (sel[i] < 0) continue;
        memcpy(keys + (size_t)x * p->D,
               paged_row(pool_pages, pool_bt, s, max_pool_pages, page_size, sel[i], p->D),
               sizeof(double) * p->D);
        ++x;
      }
    } else {
      for (long w = 0; w < nvis; ++w, ++x)
        memcpy(keys + (size_t)x * p->D,
               paged_row(pool_pages, pool_bt, s, max_pool_pages, page_size, w, p->D),
               sizeof(double) * p->D);
    }
    attend_row(p, q + (size_t)s * p->H * p->D, (double)(p->pos0 + t), x, keys, sinks,
               o + (size_t)s * p->H * p->D);
    free(keys);
    free(sel);
  }
  return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Grouped low-rank output projection ("Grouped Output Projection" bullet of the architecture
 * overview; config o_groups, o_lora_rank, hidden_size). For each listed token row t:
 *   mid[t, g*rank + i] = sum_c o[t, g*Kg + c] * wa[g, i, c]     (Kg = (H/G)*D features per group)
 *   out[t, j]          = sum_i mid[t, i] * wb[j, i]
 * o [T, H*D], wa [G, rank, Kg], wb [hidden, G*rank], all row-major fp64; mid [n, G*rank] and
 * out [n, hidden] for the n listed rows. [reading] mid is an activation stored in the layer's
 * dtype, so with round_mid it is rounded to bf16 (as orc_round_bf16) before o_b_proj.
 * ------------------------------------------------------------------------------------------- */
void orc_oproj(int H, int D, int G, int rank, int hidden, const double *o, const double *wa,
               const double *wb, int n, const int64_t *rows, int round_mid, double *mid,
               double *out) {
  const int Kg = H / G * D;
  const int M = G * rank;
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r) {
    const double *orow = o + rows[r] * (int64_t)H * D;
    double *m = mid + (int64_t)r * M;
    for (int g = 0; g < G; ++g)
      for (int i = 0; i < rank; ++i) {
        const double *w = wa + ((int64_t)g * rank + i) * Kg;
        const double *x = orow + (int64_t)g * Kg;
        double acc = 0.0;
        for (int c = 0; c < Kg; ++c) acc += x[c] * w[c];
        m[g * rank + i] = round_mid ? orc_round_bf16(acc) : acc;
      }
    double *y = out + (int64_t)r * hidden;
    for (int j = 0; j < hidden; ++j) {
      const double *w = wb + (int64_t)j * M;
      double acc = 0.0;
      for (int i = 0; i < M; ++i) acc += m[i] * w[i];
      y[j] = acc;
    }
  }
}
