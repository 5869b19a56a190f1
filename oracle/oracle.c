/*
 * oracle.c -- plain, slow, fp64 CPU oracle for packed causal attention with
 * sequence-aware chunking.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg and reference arm call it; the
 * CUDA library never does, and the two share no code.
 *
 * What it computes (SAP/HSAP page, abstract: packing documents into one
 * sequence must not let attention cross documents; "partial attention
 * computation" over chunks of the sequence; the sequence-parallel FAQ of the
 * explainer page states the chunked computation equals the single-device one):
 *
 *   For query head h, key/value head g = floor(h / G), G = hq / hkv, and a
 *   token i of document D = [s_D, e_D):
 *     S_ij  = scale * <Q[i,h,:], K[j,g,:]>            for s_D <= j <= i
 *     LSE_i = log sum_j exp(S_ij)                        (natural log)
 *     O_i   = sum_j exp(S_ij - LSE_i) * V[j,g,:]
 *   Partial over a key range R (a chunk):  the same sums restricted to j in R;
 *   an empty range gives LSE = -inf and O = 0.
 *   Merge of partials b:  LSE = M + log sum_b exp(LSE_b - M), M = max_b LSE_b,
 *                         O   = sum_b exp(LSE_b - LSE) * O_b.
 *   Backward (exact derivative of <dO, O>):
 *     P_ij  = exp(S_ij - LSE_i),  D_i = <dO_i, O_i>
 *     dV[j,g] = sum_{h in g} sum_i P_ij dO_i
 *     dS_ij = P_ij * (<dO_i, V_j> - D_i)
 *     dQ_i  = scale * sum_j dS_ij K_j
 *     dK[j,g] = scale * sum_{h in g} sum_i dS_ij Q_i
 *
 * Tile list: the non-empty (q-tile, kv-tile) pairs of the packed causal mask
 * M[i,j] = (i < N and j < N and doc(i) == doc(j) and j <= i), each tagged
 *   FULL   (0) every pair of the BM x BN box is unmasked,
 *   CAUSAL (1) the diagonal tile (same row and column range) of one document,
 *   MASKED (2) anything else,
 * in canonical order (q-tile ascending, then kv-tile ascending), with
 * q_chunk / kv_chunk the chunk holding the tile's first row / key, chunks being
 * P equal parts of the sequence or explicit contiguous bounds.
 * Balanced chunk bounds: see oracle_balanced_bounds.
 *
 * Layouts: Q, O, dO, dQ are [N][hq][d]; K, V, dK, dV are [N][hkv][d]; LSE is
 * [hq][N].  All floating point is double.
 *
 * Parity status: every function here is pinned by the CPU tests (brute force
 * against a library attention routine, finite differences, closed forms and
 * invariants); see the test files for which pin covers which function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_SEQLENS (-2)
#define ORACLE_ERR_CHUNKS (-3)
#define ORACLE_ERR_CAPACITY (-4)
#define ORACLE_ERR_NOMEM (-5)

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static int check_seqlens(const int32_t* cu, int32_t ndocs, int64_t n) {
  if (ndocs < 0 || cu == NULL) return ORACLE_ERR_ARG;
  if (cu[0] != 0) return ORACLE_ERR_SEQLENS;
  for (int32_t k = 0; k < ndocs; ++k)
    if (cu[k + 1] < cu[k]) return ORACLE_ERR_SEQLENS;
  if ((int64_t)cu[ndocs] != n) return ORACLE_ERR_SEQLENS;
  return ORACLE_OK;
}

/* doc_of[i] = index of the document holding token i; start_of[i] = its first token. */
static void token_docs(const int32_t* cu, int32_t ndocs, int64_t n, int32_t* doc_of, int64_t* start_of,
                       int64_t* end_of) {
  for (int32_t k = 0; k < ndocs; ++k)
    for (int64_t i = cu[k]; i < cu[k + 1]; ++i) {
      if (doc_of) doc_of[i] = k;
      if (start_of) start_of[i] = cu[k];
      if (end_of) end_of[i] = cu[k + 1];
    }
  (void)n;
}

/* ---------------------------------------------------------------- tile list */

/*
 * Chunks are contiguous token ranges [bounds[c], bounds[c+1]): bounds[0] = 0,
 * bounds[nchunks] = n, strictly increasing (except the single empty chunk of
 * an empty batch), interior bounds multiples of both tile sizes.  Equal chunks
 * are bounds[c] = c * n / nchunks.
 */
static int check_bounds(int64_t n, const int64_t* bounds, int32_t nchunks, int32_t bm, int32_t bn) {
  if (bm <= 0 || bn <= 0 || nchunks < 1 || bounds == NULL) return ORACLE_ERR_ARG;
  if (bounds[0] != 0 || bounds[nchunks] != n) return ORACLE_ERR_CHUNKS;
  for (int32_t c = 0; c < nchunks; ++c) {
    if (bounds[c + 1] <= bounds[c] && !(nchunks == 1 && n == 0)) return ORACLE_ERR_CHUNKS;
    if (c > 0 && (bounds[c] % bm != 0 || bounds[c] % bn != 0)) return ORACLE_ERR_CHUNKS;
  }
  return ORACLE_OK;
}

/* The chunk holding token t: the c with bounds[c] <= t < bounds[c+1]. */
static int32_t chunk_of_token(const int64_t* bounds, int32_t nchunks, int64_t t) {
  int32_t c = 0;
  while (c + 1 < nchunks && bounds[c + 1] <= t) ++c;
  return c;
}

int64_t oracle_tile_list_bounds(const int32_t* cu, int32_t ndocs, int64_t n, const int64_t* bounds, int32_t nchunks,
                                int32_t bm, int32_t bn, int exhaustive, int32_t* out, int64_t cap);

/*
 * Equal chunks: bounds[c] = c * n / nchunks, which needs n % nchunks == 0 and
 * a chunk length that is a multiple of both tile sizes (one chunk: any n).
 */
int64_t oracle_tile_list(const int32_t* cu, int32_t ndocs, int64_t n, int32_t nchunks, int32_t bm, int32_t bn,
                         int exhaustive, int32_t* out, int64_t cap) {
  if (bm <= 0 || bn <= 0 || nchunks < 1) return ORACLE_ERR_ARG;
  if (nchunks > 1 && n % nchunks != 0) return ORACLE_ERR_CHUNKS;
  int64_t* bounds = (int64_t*)malloc(sizeof(int64_t) * ((size_t)nchunks + 1));
  if (!bounds) return ORACLE_ERR_NOMEM;
  for (int32_t c = 0; c <= nchunks; ++c) bounds[c] = (int64_t)c * (n / nchunks);
  bounds[nchunks] = n;
  int64_t r = oracle_tile_list_bounds(cu, ndocs, n, bounds, nchunks, bm, bn, exhaustive, out, cap);
  free(bounds);
  return r;
}

/*
 * exhaustive != 0: evaluate M[i,j] on every pair of every candidate box.
 * exhaustive == 0: use, per row, the interval of keys [start(i), i] it may see.
 * Returns the number of items (also when cap is too small, in which case only
 * the first cap items are written and ORACLE_ERR_CAPACITY is not raised: the
 * caller compares the count to cap).
 */
int64_t oracle_tile_list_bounds(const int32_t* cu, int32_t ndocs, int64_t n, const int64_t* bounds, int32_t nchunks,
                                int32_t bm, int32_t bn, int exhaustive, int32_t* out, int64_t cap) {
  int rc = check_seqlens(cu, ndocs, n);
  if (rc) return rc;
  rc = check_bounds(n, bounds, nchunks, bm, bn);
  if (rc) return rc;
  if (n == 0) return 0;
  int32_t* doc_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
  int64_t* start_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
  if (!doc_of || !start_of) {
    free(doc_of);
    free(start_of);
    return ORACLE_ERR_NOMEM;
  }
  token_docs(cu, ndocs, n, doc_of, start_of, NULL);
  int64_t ntq = (n + bm - 1) / bm, ntk = (n + bn - 1) / bn, count = 0;
  for (int64_t qt = 0; qt < ntq; ++qt) {
    int64_t i0 = qt * bm, i1 = i0 + bm; /* nominal rows [i0, i1) */
    for (int64_t kt = 0; kt < ntk; ++kt) {
      int64_t j0 = kt * bn, j1 = j0 + bn;
      int any = 0, all = 1;
      if (exhaustive) {
        for (int64_t i = i0; i < i1; ++i)
          for (int64_t j = j0; j < j1; ++j) {
            int m = (i < n && j < n && doc_of[i] == doc_of[j] && j <= i);
            any |= m;
            all &= m;
          }
      } else {
        for (int64_t i = i0; i < i1; ++i) {
          if (i >= n) {
            all = 0;
            continue;
          }
          int64_t lo = start_of[i], hi = i; /* keys this row may see */
          int64_t a = lo > j0 ? lo : j0, b = hi < j1 - 1 ? hi : j1 - 1;
          if (a <= b) any = 1;
          if (!(lo <= j0 && j1 - 1 <= hi)) all = 0;
        }
      }
      if (!any) continue;
      int tag;
      if (all)
        tag = 0;
      else if (bm == bn && qt == kt && doc_of[i0] == doc_of[(i1 < n ? i1 : n) - 1])
        tag = 1;
      else
        tag = 2;
      if (count < cap && out) {
        int32_t* it = out + 5 * count;
        it[0] = (int32_t)qt;
        it[1] = (int32_t)kt;
        it[2] = chunk_of_token(bounds, nchunks, i0);
        it[3] = chunk_of_token(bounds, nchunks, j0);
        it[4] = tag;
      }
      ++count;
    }
  }
  free(doc_of);
  free(start_of);
  return count;
}

/* ------------------------------------------------------------ balanced cut */

/*
 * Balanced chunk bounds (the load-balancing scheduler of the HSAP method
 * details, read as: cut the sequence into nchunks contiguous, tile-aligned,
 * non-empty parts whose largest work is as small as possible).  Work of a q
 * tile = the number of items (non-empty tiles) in its row of the tile list.
 * Definition:
 *   M* = min over all cuts of max over chunks of the chunk's summed work;
 *   among the cuts reaching M*, the one with the lexicographically largest
 *   bound vector.
 * M* comes from the textbook dynamic program best[k][t] = min over s of
 * max(best[k-1][s], work(s..t)) over cuts of tiles [0, t) into k parts; the
 * bounds are then chosen left to right, each the largest tile index b after
 * the previous bound such that the chunk's work is <= M* and tiles [b, T) can
 * still be cut into the remaining number of parts with work <= M* (a second
 * table, over suffixes).  out_bounds: nchunks + 1 entries, in tokens.
 */
int oracle_balanced_bounds(const int32_t* cu, int32_t ndocs, int64_t n, int32_t nchunks, int32_t block,
                           int64_t* out_bounds) {
  int rc = check_seqlens(cu, ndocs, n);
  if (rc) return rc;
  if (block <= 0 || nchunks < 1 || out_bounds == NULL) return ORACLE_ERR_ARG;
  if (n == 0) {
    if (nchunks != 1) return ORACLE_ERR_CHUNKS;
    out_bounds[0] = out_bounds[1] = 0;
    return ORACLE_OK;
  }
  int64_t T = (n + block - 1) / block;
  if (nchunks > T) return ORACLE_ERR_CHUNKS;
  int64_t cnt = oracle_tile_list(cu, ndocs, n, 1, block, block, 0, NULL, 0);
  if (cnt < 0) return (int)cnt;
  int32_t* items = (int32_t*)malloc(sizeof(int32_t) * 5 * (size_t)(cnt > 0 ? cnt : 1));
  int64_t* pre = (int64_t*)calloc((size_t)T + 1, sizeof(int64_t));   /* pre[t] = work of tiles [0, t) */
  int64_t K = nchunks, W = T + 1;
  int64_t* best = (int64_t*)malloc(sizeof(int64_t) * (size_t)((K + 1) * W));
  int64_t* suf = (int64_t*)malloc(sizeof(int64_t) * (size_t)((K + 1) * W));
  if (!items || !pre || !best || !suf) {
    free(items), free(pre), free(best), free(suf);
    return ORACLE_ERR_NOMEM;
  }
  oracle_tile_list(cu, ndocs, n, 1, block, block, 0, items, cnt);
  for (int64_t e = 0; e < cnt; ++e) pre[items[5 * e] + 1] += 1;
  for (int64_t t = 0; t < T; ++t) pre[t + 1] += pre[t];
  const int64_t INF = INT64_MAX;
  /* best[k][t]: tiles [0, t) in k non-empty parts; suf[m][s]: tiles [s, T) in m non-empty parts */
  for (int64_t i = 0; i < (K + 1) * W; ++i) best[i] = suf[i] = INF;
  best[0 * W + 0] = 0;
  suf[0 * W + T] = 0;
  for (int64_t k = 1; k <= K; ++k)
    for (int64_t t = k; t <= T; ++t)
      for (int64_t s = k - 1; s < t; ++s) {
        int64_t a = best[(k - 1) * W + s];
        if (a == INF) continue;
        int64_t w = pre[t] - pre[s];
        int64_t v = a > w ? a : w;
        if (v < best[k * W + t]) best[k * W + t] = v;
      }
  for (int64_t m = 1; m <= K; ++m)
    for (int64_t s = T - m; s >= 0; --s)
      for (int64_t e = s + 1; e <= T - (m - 1); ++e) {
        int64_t a = suf[(m - 1) * W + e];
        if (a == INF) continue;
        int64_t w = pre[e] - pre[s];
        int64_t v = a > w ? a : w;
        if (v < suf[m * W + s]) suf[m * W + s] = v;
      }
  int64_t mstar = best[K * W + T];
  out_bounds[0] = 0;
  int64_t prev = 0;
  for (int64_t k = 1; k < K; ++k) {
    int64_t chosen = -1;
    for (int64_t b = prev + 1; b <= T - (K - k); ++b)
      if (pre[b] - pre[prev] <= mstar && suf[(K - k) * W + b] <= mstar) chosen = b;
    out_bounds[k] = chosen * block;
    prev = chosen;
  }
  out_bounds[K] = n;
  free(items), free(pre), free(best), free(suf);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ forward */

/*
 * One (row i, head h) of attention over keys j in [lo, hi] (inclusive; empty
 * if lo > hi).  s is scratch of at least hi-lo+1 doubles.
 */
static void row_attention(const double* q, const double* k, const double* v, int32_t hq, int32_t hkv, int32_t d,
                          double scale, int64_t i, int32_t h, int64_t lo, int64_t hi, double* s, double* o_row,
                          double* lse_out) {
  int32_t g = h / (hq / hkv);
  const double* qi = q + ((size_t)i * hq + h) * d;
  for (int32_t c = 0; c < d; ++c) o_row[c] = 0.0;
  if (lo > hi) {
    *lse_out = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int64_t j = lo; j <= hi; ++j) {
    const double* kj = k + ((size_t)j * hkv + g) * d;
    double acc = 0.0;
    for (int32_t c = 0; c < d; ++c) acc += qi[c] * kj[c];
    s[j - lo] = scale * acc;
    if (s[j - lo] > m) m = s[j - lo];
  }
  double sum = 0.0;
  for (int64_t j = lo; j <= hi; ++j) sum += exp(s[j - lo] - m);
  double lse = m + log(sum);
  for (int64_t j = lo; j <= hi; ++j) {
    double p = exp(s[j - lo] - lse);
    const double* vj = v + ((size_t)j * hkv + g) * d;
    for (int32_t c = 0; c < d; ++c) o_row[c] += p * vj[c];
  }
  *lse_out = lse;
}

static int check_heads(int32_t hq, int32_t hkv, int32_t d) {
  if (hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv != 0) return ORACLE_ERR_ARG;
  return ORACLE_OK;
}

/*
 * Forward over keys restricted to [kv_lo, kv_hi) (pass 0, n for the plain,
 * unchunked attention).  o: [n][hq][d], lse: [hq][n].
 */
int oracle_attn_fwd(const double* q, const double* k, const double* v, int64_t n, int32_t hq, int32_t hkv,
                    int32_t d, const int32_t* cu, int32_t ndocs, double scale, int64_t kv_lo, int64_t kv_hi,
                    double* o, double* lse, int nthreads) {
  int rc = check_seqlens(cu, ndocs, n);
  if (rc) return rc;
  if ((rc = check_heads(hq, hkv, d))) return rc;
  if (n == 0) return ORACLE_OK;
  int64_t* start_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
  if (!start_of) return ORACLE_ERR_NOMEM;
  token_docs(cu, ndocs, n, NULL, start_of, NULL);
  int64_t total = n * (int64_t)hq;
  int nt = nthreads > 0 ? nthreads : oracle_max_threads();
  int fail = 0;
#pragma omp parallel num_threads(nt)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    if (!s) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < total; ++t) {
      if (!s) continue;
      int64_t i = t / hq;
      int32_t h = (int32_t)(t % hq);
      int64_t lo = start_of[i] > kv_lo ? start_of[i] : kv_lo;
      int64_t hi = i < kv_hi - 1 ? i : kv_hi - 1;
      row_attention(q, k, v, hq, hkv, d, scale, i, h, lo, hi, s, o + ((size_t)i * hq + h) * d,
                    lse + (size_t)h * n + i);
    }
    free(s);
  }
  free(start_of);
  return fail ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * Exact merge of nparts partial results (o_parts: [nparts][n][hq][d],
 * lse_parts: [nparts][hq][n]) into o [n][hq][d], lse [hq][n].
 */
int oracle_merge(int32_t nparts, const double* o_parts, const double* lse_parts, int64_t n, int32_t hq, int32_t d,
                 double* o, double* lse) {
  if (nparts < 1 || hq <= 0 || d <= 0) return ORACLE_ERR_ARG;
  for (int64_t i = 0; i < n; ++i)
    for (int32_t h = 0; h < hq; ++h) {
      double m = -INFINITY;
      for (int32_t b = 0; b < nparts; ++b) {
        double l = lse_parts[((size_t)b * hq + h) * n + i];
        if (l > m) m = l;
      }
      double* orow = o + ((size_t)i * hq + h) * d;
      for (int32_t c = 0; c < d; ++c) orow[c] = 0.0;
      if (m == -INFINITY) {
        lse[(size_t)h * n + i] = -INFINITY;
        continue;
      }
      double sum = 0.0;
      for (int32_t b = 0; b < nparts; ++b) sum += exp(lse_parts[((size_t)b * hq + h) * n + i] - m);
      double l_all = m + log(sum);
      for (int32_t b = 0; b < nparts; ++b) {
        double w = exp(lse_parts[((size_t)b * hq + h) * n + i] - l_all);
        const double* ob = o_parts + (((size_t)b * n + i) * hq + h) * d;
        for (int32_t c = 0; c < d; ++c) orow[c] += w * ob[c];
      }
      lse[(size_t)h * n + i] = l_all;
    }
  return ORACLE_OK;
}

/*
 * Forward on a sample: (rows[r], heads[t]) for every r < nrows, t < nheads.
 * o_rows: [nrows][nheads][d], lse_rows: [nrows][nheads].  Unchunked.
 */
int oracle_attn_fwd_rows(const double* q, const double* k, const double* v, int64_t n, int32_t hq, int32_t hkv,
                         int32_t d, const int32_t* cu, int32_t ndocs, double scale, const int64_t* rows,
                         int64_t nrows, const int32_t* heads, int32_t nheads, double* o_rows, double* lse_rows,
                         int nthreads) {
  int rc = check_seqlens(cu, ndocs, n);
  if (rc) return rc;
  if ((rc = check_heads(hq, hkv, d))) return rc;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= n) return ORACLE_ERR_ARG;
  for (int32_t t = 0; t < nheads; ++t)
    if (heads[t] < 0 || heads[t] >= hq) return ORACLE_ERR_ARG;
  int64_t* start_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
  if (!start_of) return ORACLE_ERR_NOMEM;
  token_docs(cu, ndocs, n, NULL, start_of, NULL);
  int nt = nthreads > 0 ? nthreads : oracle_max_threads();
  int64_t total = nrows * (int64_t)nheads;
#pragma omp parallel num_threads(nt)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < total; ++t) {
      int64_t r = t / nheads;
      int32_t hh = (int32_t)(t % nheads);
      int64_t i = rows[r];
      row_attention(q, k, v, hq, hkv, d, scale, i, heads[hh], start_of[i], i, s, o_rows + (size_t)t * d,
                    lse_rows + t);
    }
    free(s);
  }
  free(start_of);
  return ORACLE_OK;
}

/* ----------------------------------------------------------------- backward */

static double dot(const double* a, const double* b, int32_t d) {
  double acc = 0.0;
  for (int32_t c = 0; c < d; ++c) acc += a[c] * b[c];
  return acc;
}

/*
 * Full backward.  dq: [n][hq][d], dk, dv: [n][hkv][d] (overwritten).
 * Work is split over (kv head, document) pairs: every such task owns the dQ
 * rows of its document for the heads of its group and the dK/dV rows of its
 * document for its kv head, so tasks never write the same element.
 */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dout, int64_t n, int32_t hq,
                    int32_t hkv, int32_t d, const int32_t* cu, int32_t ndocs, double scale, double* dq, double* dk,
                    double* dv, int nthreads) {
  int rc = check_seqlens(cu, ndocs, n);
  if (rc) return rc;
  if ((rc = check_heads(hq, hkv, d))) return rc;
  memset(dq, 0, sizeof(double) * (size_t)n * hq * d);
  memset(dk, 0, sizeof(double) * (size_t)n * hkv * d);
  memset(dv, 0, sizeof(double) * (size_t)n * hkv * d);
  if (n == 0) return ORACLE_OK;
  int32_t G = hq / hkv;
  int nt = nthreads > 0 ? nthreads : oracle_max_threads();
  int64_t ntask = (int64_t)hkv * ndocs;
#pragma omp parallel num_threads(nt)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    double* orow = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t task = 0; task < ntask; ++task) {
      int32_t g = (int32_t)(task / ndocs);
      int32_t doc = (int32_t)(task % ndocs);
      int64_t s0 = cu[doc], e0 = cu[doc + 1];
      for (int32_t h = g * G; h < (g + 1) * G; ++h)
        for (int64_t i = s0; i < e0; ++i) {
          double lse;
          row_attention(q, k, v, hq, hkv, d, scale, i, h, s0, i, s, orow, &lse);
          const double* qi = q + ((size_t)i * hq + h) * d;
          const double* doi = dout + ((size_t)i * hq + h) * d;
          double* dqi = dq + ((size_t)i * hq + h) * d;
          double Di = dot(doi, orow, d);
          for (int64_t j = s0; j <= i; ++j) {
            const double* kj = k + ((size_t)j * hkv + g) * d;
            const double* vj = v + ((size_t)j * hkv + g) * d;
            double* dkj = dk + ((size_t)j * hkv + g) * d;
            double* dvj = dv + ((size_t)j * hkv + g) * d;
            double p = exp(s[j - s0] - lse);
            double dp = dot(doi, vj, d);
            double ds = p * (dp - Di);
            for (int32_t c = 0; c < d; ++c) {
              dvj[c] += p * doi[c];
              dqi[c] += scale * ds * kj[c];
              dkj[c] += scale * ds * qi[c];
            }
          }
        }
    }
    free(s);
    free(orow);
  }
  return ORACLE_OK;
}

/*
 * Backward on a sample, for the q heads of one kv head g:
 *   dq_rows[r][t][:] = dQ[q_rows[r], g*G + t, :]     (nq x G x d)
 *   dk_rows[r][:]    = dK[kv_rows[r], g, :]          (nk x d)
 *   dv_rows[r][:]    = dV[kv_rows[r], g, :]          (nk x d)
 * Every needed (row, head) forward statistic (LSE_i, D_i) is computed here in
 * fp64 from the inputs.
 */
int oracle_attn_bwd_sampled(const double* q, const double* k, const double* v, const double* dout, int64_t n,
                            int32_t hq, int32_t hkv, int32_t d, const int32_t* cu, int32_t ndocs, double scale,
                            int32_t g, const int64_t* q_rows, int64_t nq, const int64_t* kv_rows, int64_t nk,
                            double* dq_rows, double* dk_rows, double* dv_rows, int nthreads) {
  int rc = check_seqlens(cu, ndocs, n);
  if (rc) return rc;
  if ((rc = check_heads(hq, hkv, d))) return rc;
  if (g < 0 || g >= hkv) return ORACLE_ERR_ARG;
  for (int64_t r = 0; r < nq; ++r)
    if (q_rows[r] < 0 || q_rows[r] >= n) return ORACLE_ERR_ARG;
  for (int64_t r = 0; r < nk; ++r)
    if (kv_rows[r] < 0 || kv_rows[r] >= n) return ORACLE_ERR_ARG;
  int32_t G = hq / hkv;
  int nt = nthreads > 0 ? nthreads : oracle_max_threads();
  int64_t* start_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
  int64_t* end_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
  /* need[i] = 1 if row i's statistics are needed (for every head of the group) */
  char* need = (char*)calloc((size_t)(n > 0 ? n : 1), 1);
  double* lse_all = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * G);
  double* d_all = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * G);
  if (!start_of || !end_of || !need || !lse_all || !d_all) {
    free(start_of), free(end_of), free(need), free(lse_all), free(d_all);
    return ORACLE_ERR_NOMEM;
  }
  token_docs(cu, ndocs, n, NULL, start_of, end_of);
  for (int64_t r = 0; r < nq; ++r) need[q_rows[r]] = 1;
  for (int64_t r = 0; r < nk; ++r)
    for (int64_t i = kv_rows[r]; i < end_of[kv_rows[r]]; ++i) need[i] = 1;
  int64_t total = n * (int64_t)G;
#pragma omp parallel num_threads(nt)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* orow = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
    for (int64_t t = 0; t < total; ++t) {
      int64_t i = t / G;
      int32_t hh = (int32_t)(t % G);
      if (!need[i]) continue;
      int32_t h = g * G + hh;
      double lse;
      row_attention(q, k, v, hq, hkv, d, scale, i, h, start_of[i], i, s, orow, &lse);
      lse_all[(size_t)i * G + hh] = lse;
      d_all[(size_t)i * G + hh] = dot(dout + ((size_t)i * hq + h) * d, orow, d);
    }
    free(s);
    free(orow);
  }
  /* dQ rows */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
  for (int64_t t = 0; t < nq * G; ++t) {
    int64_t r = t / G;
    int32_t hh = (int32_t)(t % G), h = g * G + hh;
    int64_t i = q_rows[r];
    const double* qi = q + ((size_t)i * hq + h) * d;
    const double* doi = dout + ((size_t)i * hq + h) * d;
    double* out = dq_rows + (size_t)t * d;
    for (int32_t c = 0; c < d; ++c) out[c] = 0.0;
    double lse = lse_all[(size_t)i * G + hh], Di = d_all[(size_t)i * G + hh];
    for (int64_t j = start_of[i]; j <= i; ++j) {
      const double* kj = k + ((size_t)j * hkv + g) * d;
      const double* vj = v + ((size_t)j * hkv + g) * d;
      double p = exp(scale * dot(qi, kj, d) - lse);
      double ds = p * (dot(doi, vj, d) - Di);
      for (int32_t c = 0; c < d; ++c) out[c] += scale * ds * kj[c];
    }
  }
  /* dK / dV rows */
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
  for (int64_t r = 0; r < nk; ++r) {
    int64_t j = kv_rows[r];
    const double* kj = k + ((size_t)j * hkv + g) * d;
    const double* vj = v + ((size_t)j * hkv + g) * d;
    double* dkj = dk_rows + (size_t)r * d;
    double* dvj = dv_rows + (size_t)r * d;
    for (int32_t c = 0; c < d; ++c) dkj[c] = dvj[c] = 0.0;
    for (int32_t hh = 0; hh < G; ++hh) {
      int32_t h = g * G + hh;
      for (int64_t i = j; i < end_of[j]; ++i) {
        const double* qi = q + ((size_t)i * hq + h) * d;
        const double* doi = dout + ((size_t)i * hq + h) * d;
        double p = exp(scale * dot(qi, kj, d) - lse_all[(size_t)i * G + hh]);
        double ds = p * (dot(doi, vj, d) - d_all[(size_t)i * G + hh]);
        for (int32_t c = 0; c < d; ++c) {
          dvj[c] += p * doi[c];
          dkj[c] += scale * ds * qi[c];
        }
      }
    }
  }
  free(start_of), free(end_of), free(need), free(lse_all), free(d_all);
  return ORACLE_OK;
}
