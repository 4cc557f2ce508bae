/*
 * sta_oracle.c -- plain fp64 CPU oracle for Sliding Tile Attention (STA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * CUDA product path never calls it, and it shares no code, header or table
 * with that path.
 *
 * What it computes (sources, by page title and section):
 *   "Fast Video Generation with Sliding Tile Attention" -- Abstract:
 *       attention restricted to local 3D spatio-temporal windows, computed
 *       tile by tile rather than token by token.
 *   same page (summary site), Methodology and Novelty:
 *       the video is split into non-overlapping tiles; a query tile attends
 *       densely to whole key tiles inside its window, so no block is partly
 *       masked.
 *   The window placement at the borders is not printed on the pages.  The
 *   reading taken here: the window (w_t, w_h, w_w tiles, clamped to the tile
 *   grid) is centred on the query's tile and shifted inward at the borders
 *   so it always lies fully inside the grid:
 *       start_d = clamp(qtile_d - floor(w_d / 2), 0, G_d - w_d).
 *
 * Everything is fp64.  bf16 inputs are widened exactly (bf16 -> fp32 is a
 * 16-bit shift, fp32 -> fp64 is exact), so the oracle sees the same values as
 * the GPU.  No blocking, no online softmax, no reordering: for every query
 * row the member keys are found from raw token coordinates, the scores are
 * formed, the maximum is subtracted, and the softmax-weighted sum of values
 * is taken, exactly as the definition reads.
 *
 * Geometry array `g` (int32[9]) = {B, Hh, d, T, H, W, tile_t, tile_h, tile_w}.
 * Token layout: raster, token n = (t*H + h)*W + w; tensors are
 * [B][Hh][N][d] with N = T*H*W.  `win` is int32[Hh*3] = (w_t, w_h, w_w) per
 * head, in tiles.
 *
 * Parity status: every function below is pinned by tests/test_oracle.py
 * (brute-force masks, dense attention, closed forms, finite differences).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int B, Hh, d, T, H, W, tt, th, tw;
  int GT, GH, GW;
  long N;
} geom_t;

static int load_geom(const int32_t *g, geom_t *o) {
  o->B = g[0]; o->Hh = g[1]; o->d = g[2];
  o->T = g[3]; o->H = g[4]; o->W = g[5];
  o->tt = g[6]; o->th = g[7]; o->tw = g[8];
  if (o->B < 1 || o->Hh < 1 || o->d < 1 || o->T < 1 || o->H < 1 || o->W < 1) return -1;
  if (o->tt < 1 || o->th < 1 || o->tw < 1) return -1;
  if (o->T % o->tt || o->H % o->th || o->W % o->tw) return -1;
  o->GT = o->T / o->tt; o->GH = o->H / o->th; o->GW = o->W / o->tw;
  o->N = (long)o->T * o->H * o->W;
  return 0;
}

static double widen(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Window start along one dimension (in tiles), window clamped to the grid. */
static int win_start(int qtile, int w, int G) {
  if (w > G) w = G;
  int s = qtile - w / 2;
  if (s < 0) s = 0;
  if (s > G - w) s = G - w;
  return s;
}

static int win_len(int w, int G) { return w > G ? G : w; }

/* Per-query window in TOKEN coordinates: [lo_d, hi_d) for d in t,h,w. */
typedef struct { int lo[3], hi[3]; } box_t;

static void query_box(const geom_t *g, const int32_t *win, int head, long n, box_t *b) {
  int t = (int)(n / ((long)g->H * g->W));
  int h = (int)((n / g->W) % g->H);
  int w = (int)(n % g->W);
  const int32_t *wh = win + 3 * head;
  int st = win_start(t / g->tt, wh[0], g->GT), lt = win_len(wh[0], g->GT);
  int sh = win_start(h / g->th, wh[1], g->GH), lh = win_len(wh[1], g->GH);
  int sw = win_start(w / g->tw, wh[2], g->GW), lw = win_len(wh[2], g->GW);
  b->lo[0] = st * g->tt; b->hi[0] = (st + lt) * g->tt;
  b->lo[1] = sh * g->th; b->hi[1] = (sh + lh) * g->th;
  b->lo[2] = sw * g->tw; b->hi[2] = (sw + lw) * g->tw;
}

/* Membership from raw coordinates: key token kn is in query token qn's
 * window iff, along every dimension, the key's tile lies in
 * [start, start + w). */
static int is_member(const geom_t *g, const int32_t *win, int head, long qn, long kn) {
  int qt = (int)(qn / ((long)g->H * g->W)), qh = (int)((qn / g->W) % g->H), qw = (int)(qn % g->W);
  int kt = (int)(kn / ((long)g->H * g->W)), kh = (int)((kn / g->W) % g->H), kw = (int)(kn % g->W);
  const int32_t *wh = win + 3 * head;
  int s, l;
  s = win_start(qt / g->tt, wh[0], g->GT); l = win_len(wh[0], g->GT);
  if (kt / g->tt < s || kt / g->tt >= s + l) return 0;
  s = win_start(qh / g->th, wh[1], g->GH); l = win_len(wh[1], g->GH);
  if (kh / g->th < s || kh / g->th >= s + l) return 0;
  s = win_start(qw / g->tw, wh[2], g->GW); l = win_len(wh[2], g->GW);
  if (kw / g->tw < s || kw / g->tw >= s + l) return 0;
  return 1;
}

/* List the member keys of query qn in ascending raster order.
 * exhaustive != 0: test every one of the N tokens with is_member().
 * exhaustive == 0: walk the query's token box (the same set, same order). */
static long member_keys(const geom_t *g, const int32_t *win, int head, long qn,
                        int exhaustive, long *out) {
  long cnt = 0;
  if (exhaustive) {
    for (long kn = 0; kn < g->N; ++kn)
      if (is_member(g, win, head, qn, kn)) out[cnt++] = kn;
    return cnt;
  }
  box_t b;
  query_box(g, win, head, qn, &b);
  for (int t = b.lo[0]; t < b.hi[0]; ++t)
    for (int h = b.lo[1]; h < b.hi[1]; ++h)
      for (int w = b.lo[2]; w < b.hi[2]; ++w)
        out[cnt++] = ((long)t * g->H + h) * g->W + w;
  return cnt;
}

/* One query row of the forward pass.  keys/sbuf are scratch of length N.
 * Writes o[d], *lse, and (optionally) the probability of every member key. */
static void forward_row(const geom_t *g, const int32_t *win, double scale,
                        const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        long bh, long qn, int exhaustive, long *keys, double *sbuf,
                        double *o, double *lse, double *probs /* N or NULL */) {
  const int head = (int)(bh % g->Hh);
  const int d = g->d;
  const uint16_t *qrow = q + (bh * g->N + qn) * d;
  long nk = member_keys(g, win, head, qn, exhaustive, keys);
  double m = -INFINITY;
  for (long j = 0; j < nk; ++j) {
    const uint16_t *krow = k + (bh * g->N + keys[j]) * d;
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += widen(qrow[c]) * widen(krow[c]);
    s *= scale;
    sbuf[j] = s;
    if (s > m) m = s;
  }
  double l = 0.0;
  for (long j = 0; j < nk; ++j) {
    sbuf[j] = exp(sbuf[j] - m);
    l += sbuf[j];
  }
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (long j = 0; j < nk; ++j) {
    const double p = sbuf[j] / l;
    const uint16_t *vrow = v + (bh * g->N + keys[j]) * d;
    for (int c = 0; c < d; ++c) o[c] += p * widen(vrow[c]);
    if (probs) probs[keys[j]] = p;
  }
  *lse = m + log(l);
}

/* Forward pass on a list of query rows.
 * rows: int64[nrows] flat indices r = bh*N + n (bh = b*Hh + h, n raster).
 * o: fp64[nrows*d], lse: fp64[nrows].  Returns 0, or -1 on bad geometry. */
int sta_oracle_forward(const int32_t *gdims, const int32_t *win, double scale,
                       const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       long nrows, const int64_t *rows, int exhaustive,
                       double *o, double *lse) {
  geom_t g;
  if (load_geom(gdims, &g)) return -1;
  int bad = 0;
#pragma omp parallel
  {
    long *keys = (long *)malloc(sizeof(long) * g.N);
    double *sbuf = (double *)malloc(sizeof(double) * g.N);
    if (!keys || !sbuf) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (long i = 0; i < nrows; ++i) {
        long bh = rows[i] / g.N, qn = rows[i] % g.N;
        forward_row(&g, win, scale, q, k, v, bh, qn, exhaustive, keys, sbuf,
                    o + i * g.d, lse + i, NULL);
      }
    }
    free(keys);
    free(sbuf);
  }
  return bad ? -2 : 0;
}

/* Attention probabilities of one query row over all N keys (zero for keys
 * outside the window).  probs: fp64[N]. */
int sta_oracle_probs(const int32_t *gdims, const int32_t *win, double scale,
                     const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int64_t row, double *probs) {
  geom_t g;
  if (load_geom(gdims, &g)) return -1;
  long *keys = (long *)malloc(sizeof(long) * g.N);
  double *sbuf = (double *)malloc(sizeof(double) * g.N);
  double *o = (double *)malloc(sizeof(double) * g.d);
  double lse;
  if (!keys || !sbuf || !o) { free(keys); free(sbuf); free(o); return -2; }
  memset(probs, 0, sizeof(double) * g.N);
  forward_row(&g, win, scale, q, k, v, row / g.N, row % g.N, 1, keys, sbuf, o, &lse, probs);
  free(keys); free(sbuf); free(o);
  return 0;
}

/* Membership matrix of one head: mask[i*N + j] = 1 iff key j is in query
 * i's window.  mask: uint8[N*N]. */
int sta_oracle_mask(const int32_t *gdims, const int32_t *win, int head, uint8_t *mask) {
  geom_t g;
  if (load_geom(gdims, &g)) return -1;
  for (long i = 0; i < g.N; ++i)
    for (long j = 0; j < g.N; ++j)
      mask[i * g.N + j] = (uint8_t)is_member(&g, win, head, i, j);
  return 0;
}

/* Backward pass for one (batch, head) slice bh.
 *   D_i   = sum_c dO_ic O_ic
 *   P_ij  = exp(S_ij - LSE_i),  S_ij = scale * q_i . k_j
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 * with i, j ranging only over the pairs where j is in i's window.
 * q_rows / k_rows are token indices n (0..N-1) inside the slice; dq is
 * fp64[nq*d], dk/dv are fp64[nk*d]. */
int sta_oracle_backward(const int32_t *gdims, const int32_t *win, double scale,
                        const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const uint16_t *dout, int64_t bh,
                        long nq, const int64_t *q_rows, long nk, const int64_t *k_rows,
                        double *dq, double *dk, double *dv) {
  geom_t g;
  if (load_geom(gdims, &g)) return -1;
  const int d = g.d;
  const int head = (int)(bh % g.Hh);
  const long N = g.N;

  /* Which queries are needed: the requested dQ rows, plus every query whose
   * window contains one of the requested key rows. */
  uint8_t *need = (uint8_t *)calloc(N, 1);
  double *lse = (double *)malloc(sizeof(double) * N);
  double *dd = (double *)malloc(sizeof(double) * N);
  if (!need || !lse || !dd) { free(need); free(lse); free(dd); return -2; }
  for (long a = 0; a < nq; ++a) need[q_rows[a]] = 1;
  if (nk > 0) {
    uint8_t *ktile = (uint8_t *)calloc((size_t)g.GT * g.GH * g.GW, 1);
    for (long a = 0; a < nk; ++a) {
      long n = k_rows[a];
      int t = (int)(n / ((long)g.H * g.W)), h = (int)((n / g.W) % g.H), w = (int)(n % g.W);
      ktile[((t / g.tt) * g.GH + h / g.th) * g.GW + w / g.tw] = 1;
    }
#pragma omp parallel for schedule(dynamic, 64)
    for (long i = 0; i < N; ++i) {
      box_t b;
      query_box(&g, win, head, i, &b);
      for (int t = b.lo[0] / g.tt; t < b.hi[0] / g.tt && !need[i]; ++t)
        for (int h = b.lo[1] / g.th; h < b.hi[1] / g.th && !need[i]; ++h)
          for (int w = b.lo[2] / g.tw; w < b.hi[2] / g.tw; ++w)
            if (ktile[(t * g.GH + h) * g.GW + w]) { need[i] = 1; break; }
    }
    free(ktile);
  }

  /* Forward statistics of every needed query: LSE_i and D_i. */
  int bad = 0;
#pragma omp parallel
  {
    long *keys = (long *)malloc(sizeof(long) * N);
    double *sbuf = (double *)malloc(sizeof(double) * N);
    double *o = (double *)malloc(sizeof(double) * d);
    if (!keys || !sbuf || !o) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (long i = 0; i < N; ++i) {
        if (!need[i]) continue;
        forward_row(&g, win, scale, q, k, v, bh, i, 0, keys, sbuf, o, &lse[i], NULL);
        const uint16_t *dorow = dout + (bh * N + i) * d;
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += widen(dorow[c]) * o[c];
        dd[i] = s;
      }
    }
    free(keys); free(sbuf); free(o);
  }
  if (bad) { free(need); free(lse); free(dd); return -2; }

  /* dQ rows. */
#pragma omp parallel
  {
    long *keys = (long *)malloc(sizeof(long) * N);
#pragma omp for schedule(dynamic, 4)
    for (long a = 0; a < nq; ++a) {
      const long i = q_rows[a];
      const uint16_t *qrow = q + (bh * N + i) * d;
      const uint16_t *dorow = dout + (bh * N + i) * d;
      double *out = dq + a * d;
      for (int c = 0; c < d; ++c) out[c] = 0.0;
      long cnt = member_keys(&g, win, head, i, 0, keys);
      for (long jj = 0; jj < cnt; ++jj) {
        const uint16_t *krow = k + (bh * N + keys[jj]) * d;
        const uint16_t *vrow = v + (bh * N + keys[jj]) * d;
        double s = 0.0, dp = 0.0;
        for (int c = 0; c < d; ++c) {
          s += widen(qrow[c]) * widen(krow[c]);
          dp += widen(dorow[c]) * widen(vrow[c]);
        }
        const double p = exp(scale * s - lse[i]);
        const double ds = p * (dp - dd[i]);
        for (int c = 0; c < d; ++c) out[c] += scale * ds * widen(krow[c]);
      }
    }
    free(keys);
  }

  /* dK, dV rows: sum over the queries whose window contains the key. */
#pragma omp parallel for schedule(dynamic, 1)
  for (long a = 0; a < nk; ++a) {
    const long j = k_rows[a];
    const uint16_t *krow = k + (bh * N + j) * d;
    const uint16_t *vrow = v + (bh * N + j) * d;
    double *odk = dk + a * d, *odv = dv + a * d;
    for (int c = 0; c < d; ++c) { odk[c] = 0.0; odv[c] = 0.0; }
    for (long i = 0; i < N; ++i) {
      if (!need[i] || !is_member(&g, win, head, i, j)) continue;
      const uint16_t *qrow = q + (bh * N + i) * d;
      const uint16_t *dorow = dout + (bh * N + i) * d;
      double s = 0.0, dp = 0.0;
      for (int c = 0; c < d; ++c) {
        s += widen(qrow[c]) * widen(krow[c]);
        dp += widen(dorow[c]) * widen(vrow[c]);
      }
      const double p = exp(scale * s - lse[i]);
      const double ds = p * (dp - dd[i]);
      for (int c = 0; c < d; ++c) {
        odv[c] += p * widen(dorow[c]);
        odk[c] += scale * ds * widen(qrow[c]);
      }
    }
  }
  free(need); free(lse); free(dd);
  return 0;
}

/* Number of OpenMP threads the oracle will use (1 without OpenMP). */
int sta_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Set the number of OpenMP threads later calls use (n >= 1; no-op without
 * OpenMP).  Only the timing of the oracle uses it; results do not depend on it. */
void sta_oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
