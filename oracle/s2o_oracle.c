/*
 * CPU oracle for the S2O prefill path — TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline leg may load this
 * library. It shares no code with the CUDA path; it was written from the method's written
 * definition (the project's definition file, itself a reading of the pages cited below).
 *
 * Sources:
 *   [S2O]  "S2O: Early Stopping for Sparse Attention via Online Permutation" (research card),
 *          Summary ¶2: stripe-level mean pooling, segment-local query ordering, global key/value
 *          ordering, index-driven gather, most-to-least-important block order, early stop at τ.
 *          Key points: the dense local window and Q-perm ablations.
 *   [PBS]  "Sparser Block-Sparse Attention via Token Permutation", lay summary: permutation
 *          within causal segments.
 *   [AB]   "AB-Sparse", Eq. (1) (dense causal attention) and its Figure 2 workflow text
 *          (block score r = q·cᵀ against mean-pooled centroids).
 *
 * Plain, slow, obviously correct: per-element loops, a library sort (qsort) as the only
 * algorithmic primitive, no blocking or reordering beyond what the definition fixes.
 * Index arithmetic follows the definition's rounding rules exactly (fp32 with explicit fmaf,
 * binary64 for weights); attention is evaluated in binary64 with libm exp.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared (see oracle/__init__.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- configuration ---------- */

typedef struct {
  int batch, n_q_heads, n_kv_heads, seq_len, head_dim, segment_len, block_size;
  float tau;
  int query_perm; /* 1: segment-local query ordering (default); 0: identity (Q-perm ablation) */
  int shared_key_order; /* 0: one key ordering per query head (default); 1: per KV head */
  int int4_centroids;   /* 0: fp32 block scores (default); 1: 4-bit key centroids, integer score */
} oracle_config;

/* Optional intermediate values, all per (batch, query head) unless noted; any pointer may be
 * NULL. Sizes: qbar/kbar_top/u [b,Hq,d]; kbar_all [b,Hkv,d]; kappa/rho [b,Hq,N];
 * Qbar/Kbar [b,Hq,nB,d]; r [b,Hq,nB,nB]; n [b,Hq,nSeg,nB] (int32); p [b,Hq,nB,nB] (double). */
typedef struct {
  float *qbar, *kbar_all, *kbar_top, *u, *kappa, *rho, *Qbar, *Kbar, *r;
  int32_t *n;
  double *p;
} oracle_debug;

enum { ORACLE_OK = 0, ORACLE_ERR_UNSUPPORTED = 2, ORACLE_ERR_NOMEM = 9 };

static int check_config(const oracle_config *c) {
  if (c->batch <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->seq_len <= 0) return 0;
  if (c->n_q_heads % c->n_kv_heads) return 0;
  /* The oracle accepts any positive head dim and block size (the hand-worked case uses d = 4,
   * B = 2); the GPU library restricts both to {64, 128}. */
  if (c->head_dim <= 0 || c->block_size <= 0) return 0;
  if (c->segment_len <= 0 || c->segment_len % c->block_size) return 0;
  if (c->seq_len % c->segment_len) return 0;
  if (!(c->tau >= 0.0f) || isinf(c->tau)) return 0;
  return 1;
}

/* ------------------------------------------------------------ arithmetic rules --------- */

static float bf16_to_f32(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, 4);
  return f;
}

/* Score scale: the fp32 value nearest to 1/sqrt(d) (0x1p-3 for d = 64, 0x1.6a09e6p-4 for
 * d = 128; the binary64 quotient is never a binary32 rounding midpoint for these d). */
float oracle_score_scale(int d) { return (float)(1.0 / sqrt((double)d)); }

/* MEAN of a list of `len` rows, each row given by its index into `rows` (a [*, d] bf16 matrix):
 * chunks of `chunk` consecutive list entries summed sequentially from +0, chunk sums added
 * sequentially from +0, then a correctly rounded division by the list length. */
static void list_mean(const uint16_t *rows, int d, const int32_t *list, int len, int chunk,
                      float *out) {
  float *total = calloc((size_t)d, sizeof(float));
  float *part = malloc((size_t)d * sizeof(float));
  for (int c0 = 0; c0 < len; c0 += chunk) {
    for (int t = 0; t < d; ++t) part[t] = 0.0f;
    for (int e = c0; e < c0 + chunk && e < len; ++e) {
      const uint16_t *row = rows + (size_t)list[e] * d;
      for (int t = 0; t < d; ++t) part[t] = part[t] + bf16_to_f32(row[t]);
    }
    for (int t = 0; t < d; ++t) total[t] = total[t] + part[t];
  }
  for (int t = 0; t < d; ++t) out[t] = total[t] / (float)len;
  free(part);
  free(total);
}

/* MEAN of fp32 rows given through bf16 storage is the only mean the definition needs; DOT: */
static float dot_f32(const float *a, const float *b, int d) {
  float acc = 0.0f;
  for (int t = 0; t < d; ++t) acc = fmaf(a[t], b[t], acc);
  return acc;
}

static float dot_f32_bf16(const float *a, const uint16_t *b, int d) {
  float acc = 0.0f;
  for (int t = 0; t < d; ++t) acc = fmaf(a[t], bf16_to_f32(b[t]), acc);
  return acc;
}

/* Sort key: monotone in the value; NaN sorts after every number in a descending order. */
static uint32_t sort_key(float x) {
  if (isnan(x)) return 0u;
  if (x == 0.0f) x = 0.0f; /* -0 -> +0 */
  uint32_t b;
  memcpy(&b, &x, 4);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

typedef struct {
  uint32_t key;
  int32_t idx;
} keyed;

/* Descending key, then ascending index: a stable descending sort. */
static int cmp_keyed_desc(const void *pa, const void *pb) {
  const keyed *a = pa, *b = pb;
  if (a->key != b->key) return a->key > b->key ? -1 : 1;
  return (a->idx > b->idx) - (a->idx < b->idx);
}

typedef struct {
  double p;
  int32_t c;
} scored;

static int cmp_scored_desc(const void *pa, const void *pb) {
  const scored *a = pa, *b = pb;
  if (a->p != b->p) return a->p > b->p ? -1 : 1;
  return (a->c > b->c) - (a->c < b->c);
}

/* exp64: Cody–Waite reduction by ln 2 (two-part constant) and the degree-13 Taylor polynomial
 * of e^t by Horner's rule with fused multiply-adds, scaled by 2^k. Defined for x <= 0. */
double oracle_exp64(double x) {
  static const double INV_LN2 = 0x1.71547652b82fep+0;
  static const double LN2_HI = 0x1.62e42fefa39efp-1;
  static const double LN2_LO = 0x1.abc9e3b39803fp-56;
  if (x < -700.0) return 0.0;
  double k = rint(x * INV_LN2);
  double t = fma(-k, LN2_HI, x);
  t = fma(-k, LN2_LO, t);
  double fact[14];
  fact[0] = 1.0;
  for (int j = 1; j < 14; ++j) fact[j] = fact[j - 1] * (double)j; /* exact up to 13! */
  double P = 1.0 / fact[13];
  for (int j = 12; j >= 0; --j) P = fma(P, t, 1.0 / fact[j]);
  return ldexp(P, (int)k);
}

/* ------------------------------------------------------------ index construction ------- */

/* Everything for one (batch b, query head h). */
static int build_head(const oracle_config *cfg, const uint16_t *q_all, const uint16_t *k_all,
                      int bi, int h, int32_t *perm_q_all, int32_t *perm_k_all,
                      int32_t *sel_cnt_all, int32_t *sel_blk_all, int32_t *local_tiles_all,
                      oracle_debug *dbg) {
  const int N = cfg->seq_len, d = cfg->head_dim, S = cfg->segment_len, B = cfg->block_size;
  const int Hq = cfg->n_q_heads, Hkv = cfg->n_kv_heads, G = Hq / Hkv, g = h / G;
  const int nB = N / B, nSeg = N / S;
  const size_t qh = (size_t)bi * Hq + h; /* flat (batch, query head) */
  const size_t kh = (size_t)bi * Hkv + g; /* flat (batch, kv head)    */
  const uint16_t *Q = q_all + qh * N * d;
  const uint16_t *K = k_all + kh * N * d;
  int32_t *perm_q = perm_q_all + qh * N;
  int32_t *perm_k = perm_k_all + qh * N;
  int32_t *sel_cnt = sel_cnt_all + qh * nB;
  int32_t *sel_blk = sel_blk_all + qh * (size_t)nB * nB;
  int32_t *local_tiles = local_tiles_all + qh * nB;

  int32_t *ident = malloc((size_t)N * sizeof(int32_t));
  float *qbar = malloc((size_t)d * sizeof(float));
  float *kbar_all = malloc((size_t)d * sizeof(float));
  float *kbar_top = malloc((size_t)d * sizeof(float));
  float *u = malloc((size_t)d * sizeof(float));
  float *kappa = malloc((size_t)N * sizeof(float));
  float *rho = malloc((size_t)N * sizeof(float));
  keyed *tmp = malloc((size_t)N * sizeof(keyed));
  float *Qbar = malloc((size_t)nB * d * sizeof(float));
  float *Kbar = malloc((size_t)nB * d * sizeof(float));
  float *r = malloc((size_t)nB * nB * sizeof(float));
  int32_t *n = malloc((size_t)nSeg * nB * sizeof(int32_t));
  double *w = malloc((size_t)nB * sizeof(double));
  scored *chosen = malloc((size_t)nB * sizeof(scored));
  if (!ident || !qbar || !kbar_all || !kbar_top || !u || !kappa || !rho || !tmp || !Qbar ||
      !Kbar || !r || !n || !w || !chosen)
    return ORACLE_ERR_NOMEM;
  for (int i = 0; i < N; ++i) ident[i] = i;

  /* Step 1a — vertical-stripe pooling: mean query, mean key, kappa_j = qbar·k_j. With a
   * shared key ordering kappa uses the group's pooled query: the G heads' mean queries added in
   * head order, divided by G. */
  list_mean(Q, d, ident, N, B, qbar);
  list_mean(K, d, ident, N, B, kbar_all);
  if (cfg->shared_key_order) {
    float *qsum = malloc((size_t)d * sizeof(float));
    float *qh_bar = malloc((size_t)d * sizeof(float));
    if (!qsum || !qh_bar) return ORACLE_ERR_NOMEM;
    for (int t = 0; t < d; ++t) qsum[t] = 0.0f;
    for (int hh = g * G; hh < (g + 1) * G; ++hh) {
      list_mean(q_all + ((size_t)bi * Hq + hh) * N * d, d, ident, N, B, qh_bar);
      for (int t = 0; t < d; ++t) qsum[t] = qsum[t] + qh_bar[t];
    }
    for (int t = 0; t < d; ++t) qsum[t] = qsum[t] / (float)G;
    for (int j = 0; j < N; ++j) kappa[j] = dot_f32_bf16(qsum, K + (size_t)j * d, d);
    free(qsum);
    free(qh_bar);
  } else {
    for (int j = 0; j < N; ++j) kappa[j] = dot_f32_bf16(qbar, K + (size_t)j * d, d);
  }

  /* Step 2a — global key/value ordering: stable descending sort of kappa. */
  for (int j = 0; j < N; ++j) {
    tmp[j].key = sort_key(kappa[j]);
    tmp[j].idx = j;
  }
  qsort(tmp, (size_t)N, sizeof(keyed), cmp_keyed_desc);
  for (int j = 0; j < N; ++j) perm_k[j] = tmp[j].idx;

  /* Step 1b — query score rho_i = q_i·(kbar_top − kbar_all). */
  list_mean(K, d, perm_k, B, B, kbar_top);
  for (int t = 0; t < d; ++t) u[t] = kbar_top[t] - kbar_all[t];
  for (int i = 0; i < N; ++i) rho[i] = dot_f32_bf16(u, Q + (size_t)i * d, d);

  /* Step 2b — segment-local query ordering (identity when the Q-perm ablation is off). */
  for (int s = 0; s < nSeg; ++s) {
    for (int e = 0; e < S; ++e) {
      tmp[e].key = sort_key(rho[s * S + e]);
      tmp[e].idx = s * S + e;
    }
    if (cfg->query_perm) qsort(tmp, (size_t)S, sizeof(keyed), cmp_keyed_desc);
    for (int e = 0; e < S; ++e) perm_q[s * S + e] = tmp[e].idx;
  }

  /* Block means over the permuted blocks and the block scores r = (Qbar_b·Kbar_c)·σ_d. */
  for (int b = 0; b < nB; ++b) {
    list_mean(Q, d, perm_q + (size_t)b * B, B, B, Qbar + (size_t)b * d);
    list_mean(K, d, perm_k + (size_t)b * B, B, B, Kbar + (size_t)b * d);
  }
  const float sigma = oracle_score_scale(d);
  if (!cfg->int4_centroids) {
    for (int b = 0; b < nB; ++b)
      for (int c = 0; c < nB; ++c)
        r[(size_t)b * nB + c] = dot_f32(Qbar + (size_t)b * d, Kbar + (size_t)c * d, d) * sigma;
  } else {
    /* 4-bit key centroids per channel (asymmetric), 8-bit query centroids scaled by the key
     * channel steps (symmetric per block), r from the exact integer product. */
    float *step = malloc((size_t)d * sizeof(float));
    float *lo = malloc((size_t)d * sizeof(float));
    int *qk = malloc((size_t)nB * d * sizeof(int));
    int *qa = malloc((size_t)d * sizeof(int));
    float *a = malloc((size_t)d * sizeof(float));
    if (!step || !lo || !qk || !qa || !a) return ORACLE_ERR_NOMEM;
    for (int t = 0; t < d; ++t) {
      float mn = Kbar[t], mx = Kbar[t];
      for (int c = 1; c < nB; ++c) {
        const float x = Kbar[(size_t)c * d + t];
        if (x < mn) mn = x;
        if (x > mx) mx = x;
      }
      float st = (mx - mn) / 15.0f;
      if (st == 0.0f) st = 1.0f;
      lo[t] = mn;
      step[t] = st;
      for (int c = 0; c < nB; ++c) {
        float code = rintf((Kbar[(size_t)c * d + t] - mn) / st);
        if (code < 0.0f) code = 0.0f;
        if (code > 15.0f) code = 15.0f;
        qk[(size_t)c * d + t] = (int)code;
      }
    }
    for (int b = 0; b < nB; ++b) {
      float m = 0.0f;
      for (int t = 0; t < d; ++t) {
        a[t] = Qbar[(size_t)b * d + t] * step[t];
        if (fabsf(a[t]) > m) m = fabsf(a[t]);
      }
      float sq = m / 127.0f;
      if (sq == 0.0f) sq = 1.0f;
      for (int t = 0; t < d; ++t) {
        float code = rintf(a[t] / sq);
        if (code < -127.0f) code = -127.0f;
        if (code > 127.0f) code = 127.0f;
        qa[t] = (int)code;
      }
      for (int c = 0; c < nB; ++c) {
        long long acc = 0;
        for (int t = 0; t < d; ++t) acc += (long long)qa[t] * qk[(size_t)c * d + t];
        r[(size_t)b * nB + c] = ((float)acc * sq) * sigma;
      }
    }
    free(step); free(lo); free(qk); free(qa); free(a);
  }

  /* Visibility counts n[s][c] = #keys of key block c before the start of segment s. */
  for (int s = 0; s < nSeg; ++s)
    for (int c = 0; c < nB; ++c) {
      int cntv = 0;
      for (int e = 0; e < B; ++e)
        if (perm_k[c * B + e] < s * S) ++cntv;
      n[(size_t)s * nB + c] = cntv;
    }

  /* Step 4 scheduling per query block: local tiles, normalised scores, early stop at τ. */
  const double tau = (double)cfg->tau;
  for (int b = 0; b < nB; ++b) {
    const int s = (b * B) / S;
    int maxi = -1;
    for (int e = 0; e < B; ++e)
      if (perm_q[b * B + e] > maxi) maxi = perm_q[b * B + e];
    local_tiles[b] = (maxi - s * S) / B + 1;

    const int32_t *ns = n + (size_t)s * nB;
    const float *rb = r + (size_t)b * nB;
    int any = 0;
    float M = 0.0f;
    for (int c = 0; c < nB; ++c)
      if (ns[c] > 0 && (!any || rb[c] > M)) {
        M = rb[c];
        any = 1;
      }
    for (int c = 0; c < nB; ++c)
      w[c] = ns[c] > 0 ? (double)ns[c] * oracle_exp64((double)rb[c] - (double)M) : 0.0;
    double Z = 0.0;
    for (int c0 = 0; c0 < nB; c0 += 32) {
      double part = 0.0;
      for (int c = c0; c < c0 + 32 && c < nB; ++c) part = part + w[c];
      Z = Z + part;
    }
    int m = 0;
    for (int c = 0; c < nB; ++c) {
      double p = any ? w[c] / Z : 0.0;
      if (dbg && dbg->p) dbg->p[(qh * nB + b) * nB + c] = ns[c] > 0 ? p : 0.0;
      if (ns[c] > 0 && p >= tau) {
        chosen[m].p = p;
        chosen[m].c = c;
        ++m;
      }
    }
    qsort(chosen, (size_t)m, sizeof(scored), cmp_scored_desc);
    sel_cnt[b] = m;
    for (int e = 0; e < nB; ++e) sel_blk[(size_t)b * nB + e] = e < m ? chosen[e].c : -1;
  }

  if (dbg) {
    if (dbg->qbar) memcpy(dbg->qbar + qh * d, qbar, (size_t)d * sizeof(float));
    if (dbg->kbar_all && h % G == 0) memcpy(dbg->kbar_all + kh * d, kbar_all, (size_t)d * 4);
    if (dbg->kbar_top) memcpy(dbg->kbar_top + qh * d, kbar_top, (size_t)d * sizeof(float));
    if (dbg->u) memcpy(dbg->u + qh * d, u, (size_t)d * sizeof(float));
    if (dbg->kappa) memcpy(dbg->kappa + qh * N, kappa, (size_t)N * sizeof(float));
    if (dbg->rho) memcpy(dbg->rho + qh * N, rho, (size_t)N * sizeof(float));
    if (dbg->Qbar) memcpy(dbg->Qbar + qh * nB * d, Qbar, (size_t)nB * d * sizeof(float));
    if (dbg->Kbar) memcpy(dbg->Kbar + qh * nB * d, Kbar, (size_t)nB * d * sizeof(float));
    if (dbg->r) memcpy(dbg->r + qh * nB * nB, r, (size_t)nB * nB * sizeof(float));
    if (dbg->n) memcpy(dbg->n + qh * nSeg * nB, n, (size_t)nSeg * nB * sizeof(int32_t));
  }
  free(ident); free(qbar); free(kbar_all); free(kbar_top); free(u); free(kappa); free(rho);
  free(tmp); free(Qbar); free(Kbar); free(r); free(n); free(w); free(chosen);
  return ORACLE_OK;
}

/* All index arrays for all (batch, query head): perm_q, perm_k [b,Hq,N]; sel_cnt, local_tiles
 * [b,Hq,nB]; sel_blk [b,Hq,nB,nB] (selected key blocks in processing order, tail -1). */
int oracle_build_indices(const oracle_config *cfg, const uint16_t *q, const uint16_t *k,
                         int32_t *perm_q, int32_t *perm_k, int32_t *sel_cnt, int32_t *sel_blk,
                         int32_t *local_tiles, oracle_debug *dbg, int n_threads) {
  if (!check_config(cfg)) return ORACLE_ERR_UNSUPPORTED;
  const int heads = cfg->batch * cfg->n_q_heads;
  int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
  for (int x = 0; x < heads; ++x) {
    int st = build_head(cfg, q, k, x / cfg->n_q_heads, x % cfg->n_q_heads, perm_q, perm_k,
                        sel_cnt, sel_blk, local_tiles, dbg);
    if (st != ORACLE_OK) {
#pragma omp critical
      status = st;
    }
  }
  return status;
}

/* ------------------------------------------------------------ attention ---------------- */

/* One query row (flat query head qh, original position i), Eq. (1) restricted to the key set
 * K_i of the definition, in binary64. Keys: the local part [sS, i] and, for every selected key
 * block c of the row's query block, the keys of c that lie before the segment. Returns |K_i|. */
static int64_t attend_row(const oracle_config *cfg, const uint16_t *q_all, const uint16_t *k_all,
                          const uint16_t *v_all, const int32_t *perm_k_h, const int32_t *sel_b,
                          int cnt_b, size_t qh, int i, double *z, double *out) {
  const int N = cfg->seq_len, d = cfg->head_dim, S = cfg->segment_len, B = cfg->block_size;
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  const size_t kh = (qh / cfg->n_q_heads) * cfg->n_kv_heads + (qh % cfg->n_q_heads) / G;
  const uint16_t *qi = q_all + (qh * N + i) * d;
  const uint16_t *K = k_all + kh * N * d, *V = v_all + kh * N * d;
  const int s0 = (i / S) * S;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);

  /* Gather the key list: local keys then selected non-local keys. */
  int64_t nk = 0;
  int32_t *keys = malloc(((size_t)S + (size_t)cnt_b * B) * sizeof(int32_t));
  for (int j = s0; j <= i; ++j) keys[nk++] = j;
  for (int e = 0; e < cnt_b; ++e) {
    const int c = sel_b[e];
    for (int x = 0; x < B; ++x) {
      const int j = perm_k_h[c * B + x];
      if (j < s0) keys[nk++] = j;
    }
  }
  double m = -INFINITY;
  for (int64_t a = 0; a < nk; ++a) {
    const uint16_t *kj = K + (size_t)keys[a] * d;
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += (double)bf16_to_f32(qi[t]) * (double)bf16_to_f32(kj[t]);
    z[a] = acc * inv_sqrt_d;
    if (z[a] > m) m = z[a];
  }
  double den = 0.0;
  for (int t = 0; t < d; ++t) out[t] = 0.0;
  for (int64_t a = 0; a < nk; ++a) {
    const double e = exp(z[a] - m);
    const uint16_t *vj = V + (size_t)keys[a] * d;
    den += e;
    for (int t = 0; t < d; ++t) out[t] += e * (double)bf16_to_f32(vj[t]);
  }
  for (int t = 0; t < d; ++t) out[t] /= den;
  free(keys);
  return nk;
}

/* Sparse attention for the rows listed in `rows` (flat indices (batch*Hq + h)*N + i; NULL means
 * every row, in that order). out: [n_rows, d] binary64. pairs: optional Σ|K_i|. */
int oracle_attention(const oracle_config *cfg, const uint16_t *q, const uint16_t *k,
                     const uint16_t *v, const int32_t *perm_q, const int32_t *perm_k,
                     const int32_t *sel_cnt, const int32_t *sel_blk, const int64_t *rows,
                     int64_t n_rows, double *out, int64_t *pairs, int n_threads) {
  if (!check_config(cfg)) return ORACLE_ERR_UNSUPPORTED;
  const int N = cfg->seq_len, d = cfg->head_dim, B = cfg->block_size, nB = N / B;
  const int64_t total = (int64_t)cfg->batch * cfg->n_q_heads * N;
  if (!rows) n_rows = total;
  int64_t pair_sum = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1) reduction(+ : pair_sum)
  {
    int32_t *slot_of = malloc((size_t)N * sizeof(int32_t));
    double *z = malloc(((size_t)N + (size_t)nB * B) * sizeof(double));
    int64_t cached_qh = -1;
#pragma omp for schedule(dynamic, 64)
    for (int64_t x = 0; x < n_rows; ++x) {
      const int64_t flat = rows ? rows[x] : x;
      const size_t qh = (size_t)(flat / N);
      const int i = (int)(flat % N);
      if ((int64_t)qh != cached_qh) { /* inverse of perm_q for this head */
        for (int e = 0; e < N; ++e) slot_of[perm_q[qh * N + e]] = e;
        cached_qh = (int64_t)qh;
      }
      const int b = slot_of[i] / B;
      const int cnt = sel_cnt[qh * nB + b];
      pair_sum += attend_row(cfg, q, k, v, perm_k + qh * N, sel_blk + (qh * nB + b) * nB, cnt,
                             qh, i, z, out + (size_t)x * d);
    }
    free(slot_of);
    free(z);
  }
  if (pairs) *pairs = pair_sum;
  return ORACLE_OK;
}

/* ------------------------------------------------------------ online early stop (variant) */

/* Measured-share early stop (a labelled variant; the definition's D13): for query block b (segment
 * s) with listed blocks c_0..c_{cnt-1} in list order, row i's share of block k is
 *   share_{i,k} = Σ_{j ∈ V_k} e^{z_ij} / Σ_{j ∈ L_i ∪ V_0 ∪ … ∪ V_k} e^{z_ij},
 * L_i = the local keys [sS, i], V_k = the keys of block c_k before sS, z_ij = q_i·k_j/√d. The
 * block's list stops after the first k whose largest share over the block's rows is below τ (block
 * k itself is kept). Writes stop_cnt[qb] (the listed blocks kept) and max_share[qb·nB + k] for
 * every listed k (binary64; libm exp; each row's exponents taken against the row's largest z over
 * its whole list, which leaves every ratio unchanged). */
int oracle_online_stop(const oracle_config *cfg, const uint16_t *q, const uint16_t *k,
                       const int32_t *perm_q, const int32_t *perm_k, const int32_t *sel_cnt,
                       const int32_t *sel_blk, int32_t *stop_cnt, double *max_share,
                       int n_threads) {
  if (!check_config(cfg)) return ORACLE_ERR_UNSUPPORTED;
  const int N = cfg->seq_len, d = cfg->head_dim, S = cfg->segment_len, B = cfg->block_size;
  const int nB = N / B, G = cfg->n_q_heads / cfg->n_kv_heads;
  const int64_t n_qblocks = (int64_t)cfg->batch * cfg->n_q_heads * nB;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  const double tau = (double)cfg->tau;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
  {
    double *zl = malloc((size_t)S * sizeof(double));
    double *zb = malloc((size_t)nB * B * sizeof(double));
    double *ek = malloc((size_t)nB * sizeof(double));
#pragma omp for schedule(dynamic, 4)
    for (int64_t qb = 0; qb < n_qblocks; ++qb) {
      const size_t qh = (size_t)(qb / nB);
      const int b = (int)(qb % nB);
      const int s0 = (b * B / S) * S;
      const size_t kh = (qh / cfg->n_q_heads) * cfg->n_kv_heads + (qh % cfg->n_q_heads) / G;
      const uint16_t *K = k + kh * N * d;
      const int32_t *pk = perm_k + qh * N;
      const int32_t *list = sel_blk + (size_t)qb * nB;
      const int cnt = sel_cnt[qb];
      double *ms = max_share + (size_t)qb * nB;
      for (int x = 0; x < cnt; ++x) ms[x] = 0.0;
      for (int e = 0; e < B; ++e) {
        const int i = perm_q[qh * N + (size_t)b * B + e];
        const uint16_t *qi = q + (qh * N + i) * d;
        double m = -INFINITY;
        int nl = 0;
        for (int j = s0; j <= i; ++j) {
          const uint16_t *kj = K + (size_t)j * d;
          double acc = 0.0;
          for (int t = 0; t < d; ++t) acc += (double)bf16_to_f32(qi[t]) * (double)bf16_to_f32(kj[t]);
          zl[nl] = acc * inv_sqrt_d;
          if (zl[nl] > m) m = zl[nl];
          ++nl;
        }
        for (int x = 0; x < cnt; ++x)
          for (int y = 0; y < B; ++y) {
            const int j = pk[list[x] * B + y];
            double zz = -INFINITY;
            if (j < s0) {
              const uint16_t *kj = K + (size_t)j * d;
              double acc = 0.0;
              for (int t = 0; t < d; ++t)
                acc += (double)bf16_to_f32(qi[t]) * (double)bf16_to_f32(kj[t]);
              zz = acc * inv_sqrt_d;
              if (zz > m) m = zz;
            }
            zb[(size_t)x * B + y] = zz;
          }
        double den = 0.0;
        for (int a = 0; a < nl; ++a) den += exp(zl[a] - m);
        for (int x = 0; x < cnt; ++x) {
          double e_k = 0.0;
          for (int y = 0; y < B; ++y) {
            const double zz = zb[(size_t)x * B + y];
            if (zz != -INFINITY) e_k += exp(zz - m);
          }
          ek[x] = e_k;
        }
        for (int x = 0; x < cnt; ++x) {
          den += ek[x];
          const double share = ek[x] / den;
          if (share > ms[x]) ms[x] = share;
        }
      }
      int kept = cnt;
      for (int x = 0; x < cnt; ++x)
        if (ms[x] < tau) {
          kept = x + 1;
          break;
        }
      stop_cnt[qb] = kept;
    }
    free(zl);
    free(zb);
    free(ek);
  }
  return ORACLE_OK;
}

/* Dense causal attention, Eq. (1) written out in binary64, for listed rows (NULL = all). */
int oracle_dense_causal(const oracle_config *cfg, const uint16_t *q, const uint16_t *k,
                        const uint16_t *v, const int64_t *rows, int64_t n_rows, double *out,
                        int n_threads) {
  if (!check_config(cfg)) return ORACLE_ERR_UNSUPPORTED;
  const int N = cfg->seq_len, d = cfg->head_dim;
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  const int64_t total = (int64_t)cfg->batch * cfg->n_q_heads * N;
  if (!rows) n_rows = total;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
  {
    double *z = malloc((size_t)N * sizeof(double));
#pragma omp for schedule(dynamic, 16)
    for (int64_t x = 0; x < n_rows; ++x) {
      const int64_t flat = rows ? rows[x] : x;
      const size_t qh = (size_t)(flat / N);
      const int i = (int)(flat % N);
      const size_t kh = (qh / cfg->n_q_heads) * cfg->n_kv_heads + (qh % cfg->n_q_heads) / G;
      const uint16_t *qi = q + (qh * N + i) * d;
      double m = -INFINITY;
      for (int j = 0; j <= i; ++j) {
        const uint16_t *kj = k + (kh * N + j) * d;
        double acc = 0.0;
        for (int t = 0; t < d; ++t)
          acc += (double)bf16_to_f32(qi[t]) * (double)bf16_to_f32(kj[t]);
        z[j] = acc * inv_sqrt_d;
        if (z[j] > m) m = z[j];
      }
      double den = 0.0;
      double *o = out + (size_t)x * d;
      for (int t = 0; t < d; ++t) o[t] = 0.0;
      for (int j = 0; j <= i; ++j) {
        const double e = exp(z[j] - m);
        const uint16_t *vj = v + (kh * N + j) * d;
        den += e;
        for (int t = 0; t < d; ++t) o[t] += e * (double)bf16_to_f32(vj[t]);
      }
      for (int t = 0; t < d; ++t) o[t] /= den;
    }
    free(z);
  }
  return ORACLE_OK;
}

/* Σ_i |K_i| over every row, counted from the index arrays alone (pair sparsity numerator). */
int64_t oracle_pair_count(const oracle_config *cfg, const int32_t *perm_q, const int32_t *perm_k,
                          const int32_t *sel_cnt, const int32_t *sel_blk) {
  const int N = cfg->seq_len, S = cfg->segment_len, B = cfg->block_size, nB = N / B;
  const int64_t heads = (int64_t)cfg->batch * cfg->n_q_heads;
  int64_t total = 0;
  for (int64_t qh = 0; qh < heads; ++qh)
    for (int b = 0; b < nB; ++b) {
      const int s0 = (b * B / S) * S;
      int64_t nonlocal = 0;
      for (int e = 0; e < sel_cnt[qh * nB + b]; ++e) {
        const int c = sel_blk[(qh * nB + b) * nB + e];
        for (int x = 0; x < B; ++x)
          if (perm_k[qh * N + c * B + x] < s0) ++nonlocal;
      }
      for (int e = 0; e < B; ++e) {
        const int i = perm_q[qh * N + b * B + e];
        total += (int64_t)(i - s0 + 1) + nonlocal;
      }
    }
  return total;
}
