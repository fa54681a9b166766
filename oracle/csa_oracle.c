/*
 * csa_oracle.c -- plain, slow, fp64 CPU oracle for the Compressed Sparse
 * Attention (CSA) / Heavily Compressed Attention (HCA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Every function computes its definition literally: nested loops, fp64
 * accumulation, exp() in double, inputs decoded from the exact bf16 / fp32
 * bits the GPU receives.  Sources (all prose; the pages never write the
 * equations out, so the formulas below are the plain readings stated at each
 * function):
 *   [A4] "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V",
 *        section "The attention: compress, then select" (CSA and HCA bullets)
 *        and its "three details" (sliding window, sink, QK-norm/RoPE);
 *        section "The skeleton, and what's kept" (single shared KV head,
 *        entry is both key and value).
 *   [E1] "The Exchange Rates of a Million Tokens", section 3 "Rate #2: bytes
 *        buy budget, and spend recall" (two overlapping series under one
 *        joint softmax; ReLU-gated indexer; top-k).
 *   [N3] "DeepSeek V4: How It Made Million-Token AI", section "The Memory
 *        Problem Nobody Wanted to Solve" (learned, not average, pooling;
 *        HCA every 128 tokens; 128-token window).
 *
 * Parallelism: OpenMP over independent outputs only.  Each output element is
 * computed by one thread with a fixed loop order, so results do not depend on
 * the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum {
  ORC_OK = 0,
  ORC_ERR_ARG = -1,     /* bad sizes / dtype / null pointer            */
  ORC_ERR_POS = -2,     /* a query position outside its sequence       */
  ORC_ERR_NAN = -3,     /* a NaN score reached the selector            */
  ORC_ERR_CACHE = -4    /* visible entries exceed the cache rows        */
};

/* ------------------------------------------------------------------ */
/* number formats                                                      */
/* ------------------------------------------------------------------ */

/* Decode element i of a buffer holding fp32 or bf16 (upper 16 bits of an
 * IEEE-754 binary32) values.  Both conversions to double are exact. */
static double ld(const void *p, int dt, size_t i) {
  if (dt == ORC_F32) return (double)((const float *)p)[i];
  uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, directly from the
 * real value (no intermediate fp32 rounding).  bf16 keeps 8 significant bits
 * and the binary32 exponent range; below 2^-126 the spacing is 2^-133. */
static uint16_t bf16_from_double(double v) {
  if (isnan(v)) return (uint16_t)0x7FC0;
  if (isinf(v)) return v > 0 ? (uint16_t)0x7F80 : (uint16_t)0xFF80;
  if (v == 0.0) return signbit(v) ? (uint16_t)0x8000 : (uint16_t)0x0000;
  double a = fabs(v), r;
  int e;
  (void)frexp(a, &e);                   /* a = f * 2^e, 0.5 <= f < 1 */
  int q = e - 8;                        /* weight of the last kept bit */
  if (q < -133) q = -133;               /* subnormal range */
  r = nearbyint(ldexp(a, -q));          /* default rounding: ties to even */
  r = ldexp(r, q);
  float f = (float)r;                   /* exact: r is a bf16 value (or inf) */
  if (r >= 0x1p128) f = INFINITY;
  uint32_t u;
  memcpy(&u, &f, 4);
  uint16_t h = (uint16_t)(u >> 16);
  return v < 0 ? (uint16_t)(h | 0x8000) : h;
}

/* Round n doubles to the output dtype (fp32: C's round-to-nearest-even
 * conversion; bf16: bf16_from_double). */
int orc_round(const double *in, size_t n, int dt, void *out) {
  if (!in || !out) return ORC_ERR_ARG;
  if (dt == ORC_F32) {
    for (size_t i = 0; i < n; ++i) ((float *)out)[i] = (float)in[i];
  } else if (dt == ORC_BF16) {
    for (size_t i = 0; i < n; ++i) ((uint16_t *)out)[i] = bf16_from_double(in[i]);
  } else {
    return ORC_ERR_ARG;
  }
  return ORC_OK;
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static long ceil_div(long a, long b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------ */
/* a1: CSA overlapping compressor                                      */
/* ------------------------------------------------------------------ */
/*
 * [A4] CSA bullet: every 4 tokens become one entry, a learned softmax-
 * weighted pooling of their key-value vectors, per channel, with learned
 * position biases; each entry pools 8 tokens, its own block and the one
 * before.  [E1] section 3: two series C^a / C^b over the overlapping blocks,
 * one joint softmax.  [N3]: learned weights, not average pooling.
 *
 * Reading (the pages do not print the formula):
 *   entry i of sequence b pools slots j = 0..7, token s = 4(i-1) + j;
 *   slots 0..3 (block i-1) use series a, slots 4..7 (block i) series b:
 *     z_s[c] = sum_e x_s[e] * W[e][c] + beta[j][c],  W = Wa (j<4) or Wb,
 *   tokens outside [0, n_b) are masked (no term in the softmax), so entry 0
 *   pools only its own 4 tokens and a trailing partial block pools what
 *   exists; per channel c:
 *     C_i[c] = sum_s softmax_s(z_s[c]) * x_s[c].
 * Output rows i >= ceil(n_b/4) are zero.  out: [B][ceil(n_max/4)][d].
 */
int orc_csa_compress(const void *x, const int32_t *lens, int B, int n_max, int d,
                     const void *Wa, const void *Wb, const void *beta, int dt,
                     double *out) {
  if (!x || !lens || !Wa || !Wb || !beta || !out) return ORC_ERR_ARG;
  if (B < 0 || n_max < 0 || d <= 0 || (dt != ORC_F32 && dt != ORC_BF16)) return ORC_ERR_ARG;
  const long nc_max = ceil_div(n_max, 4);
  for (int b = 0; b < B; ++b)
    if (lens[b] < 0 || lens[b] > n_max) return ORC_ERR_ARG;
  long total = (long)B * nc_max;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 4)
  for (long bi = 0; bi < total; ++bi) {
    const int b = (int)(bi / nc_max);
    const long i = bi % nc_max;
    const long nb = lens[b];
    double *o = out + (size_t)bi * d;
    if (i >= ceil_div(nb, 4)) {
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      continue;
    }
    double *z = (double *)malloc(sizeof(double) * 8 * (size_t)d);
    int valid[8];
    if (!z) { err = ORC_ERR_ARG; continue; }
    for (int j = 0; j < 8; ++j) {
      const long s = 4 * (i - 1) + j;
      valid[j] = (s >= 0 && s < nb);
      if (!valid[j]) continue;
      const void *W = (j < 4) ? Wa : Wb;
      const size_t xrow = ((size_t)b * n_max + (size_t)s) * d;
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += ld(x, dt, xrow + e) * ld(W, dt, (size_t)e * d + c);
        z[j * d + c] = acc + ld(beta, dt, (size_t)j * d + c);
      }
    }
    for (int c = 0; c < d; ++c) {
      double mx = -INFINITY;
      for (int j = 0; j < 8; ++j)
        if (valid[j] && z[j * d + c] > mx) mx = z[j * d + c];
      double den = 0.0, num = 0.0;
      for (int j = 0; j < 8; ++j) {
        if (!valid[j]) continue;
        const long s = 4 * (i - 1) + j;
        const double p = exp(z[j * d + c] - mx);
        den += p;
        num += p * ld(x, dt, ((size_t)b * n_max + (size_t)s) * d + c);
      }
      o[c] = num / den;
    }
    free(z);
  }
  return err;
}

/* ------------------------------------------------------------------ */
/* a2: HCA compressor                                                  */
/* ------------------------------------------------------------------ */
/*
 * [A4] HCA bullet: every m = 128 tokens become one entry, without overlap.
 * [N3]: every 128 tokens collapse into a single KV entry.  Reading: the same
 * softmax-weighted per-channel pooling as CSA with a single series:
 *   z_s[c] = sum_e x_s[e] * W[e][c] + beta[s - m*i][c],  s in block i,
 *   C_i[c] = sum_s softmax_s(z_s[c]) * x_s[c]  (valid s < n_b only).
 * Output rows i >= ceil(n_b/m) are zero.  out: [B][ceil(n_max/m)][d].
 */
int orc_hca_compress(const void *x, const int32_t *lens, int B, int n_max, int d, int m,
                     const void *W, const void *beta, int dt, double *out) {
  if (!x || !lens || !W || !beta || !out) return ORC_ERR_ARG;
  if (B < 0 || n_max < 0 || d <= 0 || m <= 0 || (dt != ORC_F32 && dt != ORC_BF16)) return ORC_ERR_ARG;
  const long nc_max = ceil_div(n_max, m);
  for (int b = 0; b < B; ++b)
    if (lens[b] < 0 || lens[b] > n_max) return ORC_ERR_ARG;
  long total = (long)B * nc_max;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bi = 0; bi < total; ++bi) {
    const int b = (int)(bi / nc_max);
    const long i = bi % nc_max;
    const long nb = lens[b];
    double *o = out + (size_t)bi * d;
    if (i >= ceil_div(nb, m)) {
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      continue;
    }
    long cnt = nb - (long)m * i;
    if (cnt > m) cnt = m;
    double *z = (double *)malloc(sizeof(double) * (size_t)cnt * d);
    if (!z) { err = ORC_ERR_ARG; continue; }
    for (long j = 0; j < cnt; ++j) {
      const size_t xrow = ((size_t)b * n_max + (size_t)(m * i + j)) * d;
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += ld(x, dt, xrow + e) * ld(W, dt, (size_t)e * d + c);
        z[j * d + c] = acc + ld(beta, dt, (size_t)j * d + c);
      }
    }
    for (int c = 0; c < d; ++c) {
      double mx = -INFINITY;
      for (long j = 0; j < cnt; ++j)
        if (z[j * d + c] > mx) mx = z[j * d + c];
      double den = 0.0, num = 0.0;
      for (long j = 0; j < cnt; ++j) {
        const double p = exp(z[j * d + c] - mx);
        den += p;
        num += p * ld(x, dt, ((size_t)b * n_max + (size_t)(m * i + j)) * d + c);
      }
      o[c] = num / den;
    }
    free(z);
  }
  return err;
}

/* ------------------------------------------------------------------ */
/* query positions and visibility                                      */
/* ------------------------------------------------------------------ */
/*
 * [A4] "three details": a compressed entry exists only once its block is
 * complete, so a query at 0-based position t sees entries i < floor((t+1)/m).
 * Position of query (b, tq): q_pos[b][tq] if given, else lens[b] - Tq + tq
 * (the last Tq tokens of the sequence; t = n - 1 for a decode step).
 */
static int query_pos(const int32_t *lens, const int32_t *q_pos, int b, int Tq, int tq, long *t) {
  long v = q_pos ? (long)q_pos[(size_t)b * Tq + tq] : (long)lens[b] - Tq + tq;
  if (v < 0 || v >= lens[b]) return ORC_ERR_POS;
  *t = v;
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* a3: lightning indexer scores                                        */
/* ------------------------------------------------------------------ */
/*
 * [A4] CSA bullet: a small "lightning indexer", 64 heads of 128 dimensions,
 * ranks the compressed blocks for each query.  [E1] section 3: ReLU-gated
 * dot products.  Reading (no scale; a positive global scale does not change
 * the ranking):
 *   I[t,i] = sum_h w[t,h] * max(0, sum_e qI[t,h,e] * kI[i,e]),
 *   for visible i < floor((t+1)/4); invisible entries get -inf.
 * qI: [B][Tq][HI][dI], w: [B][Tq][HI], kI: [B][nc_max][dI],
 * scores: [B][Tq][nc_max] (double).
 */
int orc_index_scores(const void *qI, const void *w, const void *kI, const int32_t *lens,
                     const int32_t *q_pos, int B, int Tq, int HI, int dI, int nc_max,
                     int dt, double *scores) {
  if (!qI || !w || !kI || !lens || !scores) return ORC_ERR_ARG;
  if (B < 0 || Tq < 0 || HI <= 0 || dI <= 0 || nc_max < 0) return ORC_ERR_ARG;
  if (dt != ORC_F32 && dt != ORC_BF16) return ORC_ERR_ARG;
  int err = ORC_OK;
  const long R = (long)B * Tq;
  long *vis = (long *)malloc(sizeof(long) * (size_t)(R > 0 ? R : 1));
  if (!vis) return ORC_ERR_ARG;
  for (long r = 0; r < R; ++r) {
    long t;
    vis[r] = 0;
    if (query_pos(lens, q_pos, (int)(r / Tq), Tq, (int)(r % Tq), &t) != ORC_OK) {
      err = ORC_ERR_POS;
      continue;
    }
    vis[r] = (t + 1) / 4;
    if (vis[r] > nc_max) { err = ORC_ERR_CACHE; vis[r] = 0; }
  }
  /* every score is independent: parallel over (query row, entry) */
  const long total = R * (long)nc_max;
#pragma omp parallel for schedule(static)
  for (long ri = 0; ri < total; ++ri) {
    const long r = ri / nc_max, i = ri % nc_max;
    const int b = (int)(r / Tq);
    if (i >= vis[r]) { scores[ri] = -INFINITY; continue; }
    double acc = 0.0;
    for (int h = 0; h < HI; ++h) {
      double dot = 0.0;
      const size_t qrow = ((size_t)r * HI + h) * dI;
      const size_t krow = ((size_t)b * nc_max + i) * dI;
      for (int e = 0; e < dI; ++e) dot += ld(qI, dt, qrow + e) * ld(kI, dt, krow + e);
      acc += ld(w, dt, (size_t)r * HI + h) * (dot > 0.0 ? dot : 0.0);
    }
    scores[ri] = acc;
  }
  free(vis);
  return err;
}

/* ------------------------------------------------------------------ */
/* a4: per-query top-k                                                 */
/* ------------------------------------------------------------------ */
/*
 * [A4] CSA bullet: each query attends to only the 1,024 (Flash: 512) most
 * relevant entries chosen by the indexer.  Reading: the selected set is the
 * k visible entries that come first in the total order (score descending,
 * index ascending) -- ties go to the lower index, and -0.0 ranks as +0.0
 * (the double comparisons below treat them as equal); every visible entry
 * if fewer than k are visible.  Output: the set in ascending index order,
 * padded with -1.  scores: [R][nc_max], vis: [R], idx: [R][k].
 */
typedef struct { double s; int32_t i; } orc_item;

static int cmp_rank(const void *pa, const void *pb) {
  const orc_item *a = (const orc_item *)pa, *b = (const orc_item *)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int cmp_i32(const void *pa, const void *pb) {
  int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
  return (a > b) - (a < b);
}

int orc_select_topk(const double *scores, const int32_t *vis, long R, int nc_max, int k,
                    int32_t *idx) {
  if (!scores || !vis || !idx || R < 0 || nc_max < 0 || k <= 0) return ORC_ERR_ARG;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < R; ++r) {
    long v = vis[r];
    int32_t *orow = idx + (size_t)r * k;
    for (int j = 0; j < k; ++j) orow[j] = -1;
    if (v < 0 || v > nc_max) { err = ORC_ERR_ARG; continue; }
    orc_item *items = (orc_item *)malloc(sizeof(orc_item) * (size_t)(v > 0 ? v : 1));
    if (!items) { err = ORC_ERR_ARG; continue; }
    int bad = 0;
    for (long i = 0; i < v; ++i) {
      items[i].s = scores[(size_t)r * nc_max + i];
      items[i].i = (int32_t)i;
      if (isnan(items[i].s)) bad = 1;
    }
    if (bad) { err = ORC_ERR_NAN; free(items); continue; }
    qsort(items, (size_t)v, sizeof(orc_item), cmp_rank);
    long take = v < k ? v : k;
    for (long j = 0; j < take; ++j) orow[j] = items[j].i;
    qsort(orow, (size_t)take, sizeof(int32_t), cmp_i32);
    free(items);
  }
  return err;
}

/* Visible-entry counts floor((t+1)/m) per query row, for the selector. */
int orc_visible(const int32_t *lens, const int32_t *q_pos, int B, int Tq, int m, int32_t *vis) {
  if (!lens || !vis || B < 0 || Tq < 0 || m <= 0) return ORC_ERR_ARG;
  int err = ORC_OK;
  for (int b = 0; b < B; ++b)
    for (int tq = 0; tq < Tq; ++tq) {
      long t;
      if (query_pos(lens, q_pos, b, Tq, tq, &t) != ORC_OK) {
        err = ORC_ERR_POS;
        vis[(size_t)b * Tq + tq] = 0;
        continue;
      }
      vis[(size_t)b * Tq + tq] = (int32_t)((t + 1) / m);
    }
  return err;
}

/* ------------------------------------------------------------------ */
/* a5 / a6: attention over selected (CSA) or all (HCA) entries + window */
/* ------------------------------------------------------------------ */
/*
 * [A4] "The skeleton": one key-value head shared by every query head; each
 * cached entry is both the key and the value.  CSA bullet: each query
 * attends to its selected entries.  HCA bullet: queries attend to all
 * entries densely.  "Three details": every CSA and HCA layer also attends to
 * the last 128 tokens directly.  Reading: for each head h,
 *   keys = {C_i : i in S_t} + {x_s : max(0, t-W+1) <= s <= t}, one joint
 *   softmax (no de-duplication), logits l = scale * (q[t,h] . v),
 *   o[t,h] = sum softmax(l) * v.
 * S_t: the entries of idx[b][tq][:] with 0 <= i < floor((t+1)/m) (others,
 * including the -1 padding, contribute nothing); idx == NULL selects every
 * visible entry (HCA).  The window token at position s is row (s mod n_tok)
 * of kv_tok[b] (a ring: it must hold the query's whole window,
 * min(W, t+1) <= n_tok).  scale <= 0 means 1/sqrt(d).
 * [A4] second of the "three details": an attention sink, a learned logit
 * per head whose exponential is added to the softmax denominator (so a
 * head's weights may sum to less than one).  Reading: sink[h] is in the
 * units of the scaled logits l and carries no value:
 *   o[t,h] = sum_j e^{l_j} v_j / (sum_j e^{l_j} + e^{sink[h]});
 * sink == NULL means no sink.
 * q: [B][Tq][H][d], kv_c: [B][nc_max][d], kv_tok: [B][n_tok][d],
 * idx: [B][Tq][k], sink: [H] (double), out: [B][Tq][H][d] (double).
 */
int orc_attend(const void *q, const void *kv_c, const void *kv_tok, int n_tok,
               const int32_t *idx, const int32_t *lens, const int32_t *q_pos, int B, int Tq,
               int H, int d, int nc_max, int k, int window, int m, double scale,
               const double *sink, int dt, double *out) {
  if (!q || !kv_tok || !lens || !out) return ORC_ERR_ARG;
  if (B < 0 || Tq < 0 || H <= 0 || d <= 0 || nc_max < 0 || window <= 0 || m <= 0) return ORC_ERR_ARG;
  if (n_tok <= 0 || (idx && k <= 0) || (nc_max > 0 && !kv_c)) return ORC_ERR_ARG;
  if (dt != ORC_F32 && dt != ORC_BF16) return ORC_ERR_ARG;
  if (!(scale > 0.0)) scale = 1.0 / sqrt((double)d);
  int err = ORC_OK;
  const long R = (long)B * Tq;
#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < R; ++r) {
    const int b = (int)(r / Tq), tq = (int)(r % Tq);
    double *orow = out + (size_t)r * H * d;
    long t;
    if (query_pos(lens, q_pos, b, Tq, tq, &t) != ORC_OK) {
      err = ORC_ERR_POS;
      for (long j = 0; j < (long)H * d; ++j) orow[j] = 0.0;
      continue;
    }
    long vis = (t + 1) / m;
    if (vis > nc_max) {
      err = ORC_ERR_CACHE;
      for (long j = 0; j < (long)H * d; ++j) orow[j] = 0.0;
      continue;
    }
    /* the key list: selected entries (as cache rows), then window tokens */
    long nsel = idx ? k : vis;
    long w0 = t - window + 1;
    if (w0 < 0) w0 = 0;
    long nwin = t - w0 + 1;
    if (nwin > n_tok) {   /* the ring cannot hold this query's window */
      err = ORC_ERR_ARG;
      for (long j = 0; j < (long)H * d; ++j) orow[j] = 0.0;
      continue;
    }
    double *keys = (double *)malloc(sizeof(double) * (size_t)(nsel + nwin) * d);
    if (!keys) { err = ORC_ERR_ARG; continue; }
    long nk = 0;
    for (long j = 0; j < nsel; ++j) {
      long i = idx ? (long)idx[(size_t)r * k + j] : j;
      if (i < 0 || i >= vis) continue;
      for (int e = 0; e < d; ++e) keys[nk * d + e] = ld(kv_c, dt, ((size_t)b * nc_max + i) * d + e);
      ++nk;
    }
    for (long s = w0; s <= t; ++s) {
      const size_t row = (size_t)b * n_tok + (size_t)(s % n_tok);
      for (int e = 0; e < d; ++e) keys[nk * d + e] = ld(kv_tok, dt, row * d + e);
      ++nk;
    }
    double *lg = (double *)malloc(sizeof(double) * (size_t)nk);
    if (!lg) { free(keys); err = ORC_ERR_ARG; continue; }
    for (int h = 0; h < H; ++h) {
      const size_t qrow = ((size_t)r * H + h) * d;
      double mx = -INFINITY;
      for (long j = 0; j < nk; ++j) {
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += ld(q, dt, qrow + e) * keys[j * d + e];
        lg[j] = scale * dot;
        if (lg[j] > mx) mx = lg[j];
      }
      if (sink && sink[h] > mx) mx = sink[h];
      double den = 0.0;
      for (long j = 0; j < nk; ++j) {
        lg[j] = exp(lg[j] - mx);
        den += lg[j];
      }
      if (sink) den += exp(sink[h] - mx);
      for (int e = 0; e < d; ++e) {
        double acc = 0.0;
        for (long j = 0; j < nk; ++j) acc += lg[j] * keys[j * d + e];
        orow[(size_t)h * d + e] = acc / den;
      }
    }
    free(lg);
    free(keys);
  }
  return err;
}

/* ------------------------------------------------------------------ */
/* MXFP4 indexer keys                                                 */
/* ------------------------------------------------------------------ */
/*
 * [A4] "The KV cache, recomputed": the indexer key is 128 numbers in FP4
 * with one one-byte scale per 32 (68 bytes); CSA bullet: the indexer runs in
 * FP4.  Reading (the OCP microscaling format, the pages naming the sizes
 * only): each block of 32 consecutive elements of a key shares a power-of-
 * two scale 2^X stored as the byte X + 127; each element is an E2M1 code
 * (sign bit 3; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7), two per
 * byte, element 2j in the low nibble.  Quantisation: X = floor(log2 amax) - 2
 * (amax the block's largest magnitude; the largest E2M1 magnitude 6 has
 * exponent 2), clamped to [-127, 127], X = -127 for an all-zero block; each
 * element becomes the nearest magnitude of x / 2^X, ties to the even code,
 * saturating at 6.  Dequantised value: sign * magnitude(code) * 2^X.
 * The score of a query against such a key is the indexer score of
 * orc_index_scores against the dequantised key.
 */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* nearest E2M1 magnitude code of y >= 0, ties to the even code */
static int e2m1_code(double y) {
  if (y >= 6.0) return 7;
  int lo = 0;
  while (lo < 7 && kE2M1[lo + 1] <= y) ++lo;
  if (kE2M1[lo] == y || lo == 7) return lo;
  const double dlo = y - kE2M1[lo], dhi = kE2M1[lo + 1] - y;
  if (dlo < dhi) return lo;
  if (dhi < dlo) return lo + 1;
  return (lo % 2 == 0) ? lo : lo + 1;
}

/* k: [rows][dI] (bf16 or fp32), codes: [rows][dI/2], scales: [rows][dI/32] */
int orc_quantize_mxfp4(const void *k, int dt, long rows, int dI, uint8_t *codes, uint8_t *scales) {
  if (!k || !codes || !scales || rows < 0 || dI <= 0 || dI % 32) return ORC_ERR_ARG;
  if (dt != ORC_F32 && dt != ORC_BF16) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (long r = 0; r < rows; ++r) {
    for (int blk = 0; blk < dI / 32; ++blk) {
      double amax = 0.0;
      for (int e = 0; e < 32; ++e) {
        const double x = fabs(ld(k, dt, (size_t)r * dI + blk * 32 + e));
        if (x > amax) amax = x;
      }
      int X = -127;
      if (amax > 0.0) {
        int ex;
        (void)frexp(amax, &ex);  /* amax = f * 2^ex, 0.5 <= f < 1: floor(log2 amax) = ex - 1 */
        X = ex - 1 - 2;
        if (X < -127) X = -127;
        if (X > 127) X = 127;
      }
      scales[(size_t)r * (dI / 32) + blk] = (uint8_t)(X + 127);
      for (int e = 0; e < 32; e += 2) {
        uint8_t byte = 0;
        for (int h = 0; h < 2; ++h) {
          const double x = ld(k, dt, (size_t)r * dI + blk * 32 + e + h);
          int c = e2m1_code(ldexp(fabs(x), -X));
          if (signbit(x)) c |= 8;
          byte |= (uint8_t)(c << (4 * h));
        }
        codes[(size_t)r * (dI / 2) + (blk * 32 + e) / 2] = byte;
      }
    }
  }
  return ORC_OK;
}

/* codes/scales as above -> out [rows][dI] double (exact values) */
int orc_dequant_mxfp4(const uint8_t *codes, const uint8_t *scales, long rows, int dI, double *out) {
  if (!codes || !scales || !out || rows < 0 || dI <= 0 || dI % 32) return ORC_ERR_ARG;
  for (long r = 0; r < rows; ++r)
    for (int e = 0; e < dI; ++e) {
      const int c = (codes[(size_t)r * (dI / 2) + e / 2] >> (4 * (e & 1))) & 15;
      const int X = (int)scales[(size_t)r * (dI / 32) + e / 32] - 127;
      const double v = ldexp(kE2M1[c & 7], X);
      out[(size_t)r * dI + e] = (c & 8) ? -v : v;
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* QK-norm and partial RoPE                                            */
/* ------------------------------------------------------------------ */

/*
 * [A4] "The attention: compress, then select", third detail: queries and
 * compressed entries are RMS-normalised per head, RoPE rotates only the last
 * dims of each vector (64 of 512 there), and since the cached entry is also
 * the value, each output is rotated back by its own query's position so that
 * only relative position remains.  Readings (the pages give no formula):
 *   RMSNorm  y[c] = x[c] / sqrt(mean_c(x^2) + eps) * gamma[c]  (gamma all
 *            ones when NULL), over the d dims of one head;
 *   RoPE     on the last r of the d dims, the adjacent pairs
 *            (d-r+2j, d-r+2j+1), j = 0..r/2-1, rotated by the angle
 *            p * base^(-2j/r):  (a, b) -> (a cos - b sin, a sin + b cos);
 *            the textbook frequencies (base 10000 by default; the pages do
 *            not mention the YaRN extension of the released model);
 *   inverse  the same rotation by the angle -p.
 * Normalisation comes first, then the rotation.
 * x: [R][G][d] (G heads share the position pos[r]); gamma: [d] or NULL;
 * flags: bit 0 normalise, bit 1 rotate, bit 2 rotate by -p instead of +p.
 * out: [R][G][d] double, unrounded.
 */
int orc_norm_rope(const void *x, long R, int G, int d, const int64_t *pos, const void *gamma,
                  double eps, int r, double base, int flags, int dt, double *out) {
  if (!x || !pos || !out || R < 0 || G < 1 || d < 1 || r < 0 || r > d || (r & 1)) return ORC_ERR_ARG;
  if (dt != ORC_F32 && dt != ORC_BF16) return ORC_ERR_ARG;
  if ((flags & 1) && !(eps >= 0.0)) return ORC_ERR_ARG;
  if ((flags & 2) && r > 0 && !(base > 0.0)) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (long row = 0; row < R * G; ++row) {
    const long rr = row / G;
    const size_t o = (size_t)row * d;
    double *y = out + o;
    for (int c = 0; c < d; ++c) y[c] = ld(x, dt, o + c);
    if (flags & 1) {
      double ss = 0.0;
      for (int c = 0; c < d; ++c) ss += y[c] * y[c];
      const double inv = 1.0 / sqrt(ss / d + eps);
      for (int c = 0; c < d; ++c) y[c] = y[c] * inv * (gamma ? ld(gamma, dt, (size_t)c) : 1.0);
    }
    if ((flags & 2) && r > 0) {
      const double p = (flags & 4) ? -(double)pos[rr] : (double)pos[rr];
      for (int j = 0; j < r / 2; ++j) {
        const double ang = p * pow(base, -2.0 * j / r);
        const double cs = cos(ang), sn = sin(ang);
        const int i0 = d - r + 2 * j, i1 = i0 + 1;
        const double a = y[i0], b = y[i1];
        y[i0] = a * cs - b * sn;
        y[i1] = a * sn + b * cs;
      }
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* FP8 cache entries                                                   */
/* ------------------------------------------------------------------ */

/*
 * [A4] "The KV cache, recomputed": an entry keeps its 64 RoPE dimensions in
 * BF16 and the other dimensions in FP8, with one-byte UE8M0 scales (448 FP8
 * numbers and 7 scales: one scale per 64 numbers).  Reading: the FP8 format
 * is E4M3 (sign, 4 exponent bits of bias 7, 3 mantissa bits; subnormals
 * m/8 * 2^-6; largest finite 1.75 * 2^8 = 448; the code S.1111.111 is NaN),
 * the scale rule the one of the MXFP4 keys above: per block of 64 elements
 * X = floor(log2 amax) - 8 (8: the exponent of 448), clamped to
 * [-127, 127], X = -127 for an all-zero block, stored as X + 127; each
 * element becomes the E4M3 value nearest to x / 2^X, ties to the code with
 * an even mantissa, magnitudes above 448 saturate to 448, the sign of -0.0
 * is kept.  The last `r` dims (the rotated ones) are copied unchanged.
 * Layout: fp8 [rows][d - r] codes, scales [rows][(d - r) / 64], rope
 * [rows][r] in the input dtype.  Dequantised value: code value * 2^X.
 */
static double e4m3_value(int code) { /* code 0..126, the sign bit clear */
  const int e = (code >> 3) & 15, m = code & 7;
  return e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
}

/* nearest E4M3 magnitude code of y >= 0 (brute force over the 127 finite
 * codes, ascending in value), ties to the even code, saturating at 448 */
static int e4m3_code(double y) {
  if (y >= 448.0) return 126;
  int best = 0;
  double bd = INFINITY;
  for (int c = 0; c <= 126; ++c) {
    const double dd = fabs(e4m3_value(c) - y);
    if (dd < bd || (dd == bd && (c % 2) == 0)) {
      bd = dd;
      best = c;
    }
  }
  return best;
}

int orc_quantize_fp8_entries(const void *x, int dt, long rows, int d, int r, uint8_t *fp8, uint8_t *scales,
                             void *rope) {
  const int q = d - r;
  if (!x || rows < 0 || d <= 0 || r < 0 || r > d || q % 64) return ORC_ERR_ARG;
  if ((q > 0 && (!fp8 || !scales)) || (r > 0 && !rope)) return ORC_ERR_ARG;
  if (dt != ORC_F32 && dt != ORC_BF16) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (long row = 0; row < rows; ++row) {
    for (int blk = 0; blk < q / 64; ++blk) {
      double amax = 0.0;
      for (int e = 0; e < 64; ++e) {
        const double v = fabs(ld(x, dt, (size_t)row * d + blk * 64 + e));
        if (v > amax) amax = v;
      }
      int X = -127;
      if (amax > 0.0) {
        int ex;
        (void)frexp(amax, &ex); /* floor(log2 amax) = ex - 1 */
        X = ex - 1 - 8;
        if (X < -127) X = -127;
        if (X > 127) X = 127;
      }
      scales[(size_t)row * (q / 64) + blk] = (uint8_t)(X + 127);
      for (int e = 0; e < 64; ++e) {
        const double v = ld(x, dt, (size_t)row * d + blk * 64 + e);
        int c = e4m3_code(ldexp(fabs(v), -X));
        if (signbit(v)) c |= 0x80;
        fp8[(size_t)row * q + blk * 64 + e] = (uint8_t)c;
      }
    }
    for (int e = 0; e < r; ++e) {
      if (dt == ORC_F32)
        ((float *)rope)[(size_t)row * r + e] = ((const float *)x)[(size_t)row * d + q + e];
      else
        ((uint16_t *)rope)[(size_t)row * r + e] = ((const uint16_t *)x)[(size_t)row * d + q + e];
    }
  }
  return ORC_OK;
}

/* fp8 / scales / rope as above -> out [rows][d] double (exact values) */
int orc_dequant_fp8_entries(const uint8_t *fp8, const uint8_t *scales, const void *rope, int dt, long rows,
                            int d, int r, double *out) {
  const int q = d - r;
  if (!out || rows < 0 || d <= 0 || r < 0 || r > d || q % 64) return ORC_ERR_ARG;
  if ((q > 0 && (!fp8 || !scales)) || (r > 0 && !rope)) return ORC_ERR_ARG;
  for (long row = 0; row < rows; ++row) {
    for (int e = 0; e < q; ++e) {
      const int c = fp8[(size_t)row * q + e];
      const int X = (int)scales[(size_t)row * (q / 64) + e / 64] - 127;
      if ((c & 0x7F) == 0x7F) return ORC_ERR_ARG; /* NaN codes are never produced */
      const double v = ldexp(e4m3_value(c & 0x7F), X);
      out[(size_t)row * d + e] = (c & 0x80) ? -v : v;
    }
    for (int e = 0; e < r; ++e) out[(size_t)row * d + q + e] = ld(rope, dt, (size_t)row * r + e);
  }
  return ORC_OK;
}
