/*
 * Plain CPU oracle for column-sparse masked attention (FlashMask encoding).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  The product
 * path (the CUDA library and its Python binding) never calls it, and the two
 * share no code.
 *
 * Source of the definitions: "FlashMask-3 targets masked distributed attention
 * on Hopper GPUs", section "In-depth insight": the mask is column-wise, indexed
 * by key position, and stores four query-axis interval boundaries per key
 * column (LTS, LTE, UTS, UTE).  The exact predicate used here (row i is masked
 * for key j iff LTS[j] <= i < LTE[j] or UTS[j] <= i < UTE[j], half-open
 * intervals) and the forward/backward outputs are the plain definitions of
 * masked softmax attention; the page does not spell them out, so they are
 * written here in their textbook form.  The "clip-shift-max" localisation of
 * a query chunk is named on the same page; its formula max(min(x, b) - a, 0)
 * is the plainest reading of the name.
 *
 * Everything is computed in double precision on inputs that the caller has
 * widened from bf16 (exactly).  No blocking, no online softmax, no fusion.
 * Rows (or key columns) are distributed over OpenMP threads; every output
 * element is produced by exactly one thread, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* The predicate: is query row i masked for key column j? */
static int is_masked(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute, int64_t j,
                     int64_t i) {
  return (lts[j] <= i && i < lte[j]) || (uts[j] <= i && i < ute[j]);
}

static double dot(const double* a, const double* b, int64_t d) {
  double s = 0.0;
  for (int64_t c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

/* Materialises row i of the dense mask: out[j] = 1 if masked. */
void oracle_mask_row(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute, int64_t nk,
                     int64_t i, uint8_t* out) {
  for (int64_t j = 0; j < nk; ++j) out[j] = (uint8_t)is_masked(lts, lte, uts, ute, j, i);
}

/*
 * Row statistics of one query row against all keys of one head:
 * m = max visible logit, l = sum exp(s - m).  Returns the number of visible
 * keys.  s_buf receives the scaled logits (entries of masked keys are unused).
 */
static int64_t row_logits(const double* qi, int64_t row, const double* k, int64_t nk, int64_t d, const int32_t* lts,
                          const int32_t* lte, const int32_t* uts, const int32_t* ute, double scale, double* s_buf,
                          uint8_t* vis, double* m_out, double* l_out) {
  int64_t nvis = 0;
  double m = -INFINITY;
  for (int64_t j = 0; j < nk; ++j) {
    vis[j] = (uint8_t)!is_masked(lts, lte, uts, ute, j, row);
    if (!vis[j]) continue;
    s_buf[j] = scale * dot(qi, k + j * d, d);
    if (s_buf[j] > m) m = s_buf[j];
    ++nvis;
  }
  double l = 0.0;
  for (int64_t j = 0; j < nk; ++j)
    if (vis[j]) l += exp(s_buf[j] - m);
  *m_out = m;
  *l_out = l;
  return nvis;
}

/*
 * Forward for one (batch, q-head): q holds nrows query vectors (row-major,
 * leading dimension d), rows[r] is the sequence position of q row r (NULL:
 * r itself).  k, v are [nk, d] of the KV head, the four vectors are the mask
 * head's [nk] boundaries.
 *   O_i = sum_j softmax_j(s_ij) v_j over visible j,  LSE_i = m + ln(l).
 *   No visible key: O_i = 0, LSE_i = -inf.
 */
void oracle_fwd_head(const double* q, const int64_t* rows, int64_t nrows, const double* k, const double* v,
                     int64_t nk, int64_t d, const int32_t* lts, const int32_t* lte, const int32_t* uts,
                     const int32_t* ute, double scale, double* o, double* lse) {
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    uint8_t* vis = (uint8_t*)malloc((size_t)(nk > 0 ? nk : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
      const int64_t row = rows ? rows[r] : r;
      double m, l;
      double* orow = o + r * d;
      for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
      int64_t nvis = row_logits(q + r * d, row, k, nk, d, lts, lte, uts, ute, scale, s, vis, &m, &l);
      if (nvis == 0) {
        lse[r] = -INFINITY;
        continue;
      }
      for (int64_t j = 0; j < nk; ++j) {
        if (!vis[j]) continue;
        const double p = exp(s[j] - m) / l;
        for (int64_t c = 0; c < d; ++c) orow[c] += p * v[j * d + c];
      }
      lse[r] = m + log(l);
    }
    free(s);
    free(vis);
  }
}

/*
 * Backward, query side, for one (batch, q-head), loss L = sum(O * dO):
 *   P_ij = exp(s_ij - LSE_i) (0 when masked), dP_ij = dO_i . v_j,
 *   D_i = sum_j P_ij dP_ij, dS_ij = P_ij (dP_ij - D_i),
 *   dQ_i = scale * sum_j dS_ij k_j.
 * q and dout hold nrows vectors; rows[r] as in oracle_fwd_head.
 * Row statistics are recomputed here from q, k (never taken from a caller).
 */
void oracle_dq_head(const double* q, const double* dout, const int64_t* rows, int64_t nrows, const double* k,
                    const double* v, int64_t nk, int64_t d, const int32_t* lts, const int32_t* lte,
                    const int32_t* uts, const int32_t* ute, double scale, double* dq) {
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    uint8_t* vis = (uint8_t*)malloc((size_t)(nk > 0 ? nk : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
      const int64_t row = rows ? rows[r] : r;
      double m, l;
      double* g = dq + r * d;
      for (int64_t c = 0; c < d; ++c) g[c] = 0.0;
      int64_t nvis = row_logits(q + r * d, row, k, nk, d, lts, lte, uts, ute, scale, s, vis, &m, &l);
      if (nvis == 0) continue;
      const double lse = m + log(l);
      double D = 0.0;
      for (int64_t j = 0; j < nk; ++j) {
        if (!vis[j]) continue;
        s[j] = exp(s[j] - lse); /* now P_ij */
        dp[j] = dot(dout + r * d, v + j * d, d);
        D += s[j] * dp[j];
      }
      for (int64_t j = 0; j < nk; ++j) {
        if (!vis[j]) continue;
        const double ds = s[j] * (dp[j] - D);
        for (int64_t c = 0; c < d; ++c) g[c] += scale * ds * k[j * d + c];
      }
    }
    free(s);
    free(dp);
    free(vis);
  }
}

/*
 * Backward, key side: contribution of ONE q-head to dK and dV of the listed
 * key columns (the caller sums over the q-heads that share a KV head).
 *   dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i dS_ij q_i.
 * q and dout are the full [nq, d] arrays of the q-head.  The statistics
 * (LSE_i, D_i) of every row that sees at least one listed column are computed
 * first, from scratch, with full passes over that row's keys.
 */
void oracle_dkdv_head(const double* q, const double* dout, int64_t nq, const double* k, const double* v, int64_t nk,
                      int64_t d, const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                      double scale, const int64_t* cols, int64_t ncols, double* dk, double* dv) {
  double* lse = (double*)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1));
  double* Drow = (double*)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1));
  uint8_t* need = (uint8_t*)calloc((size_t)(nq > 0 ? nq : 1), 1);
  for (int64_t i = 0; i < nq; ++i)
    for (int64_t t = 0; t < ncols; ++t)
      if (!is_masked(lts, lte, uts, ute, cols[t], i)) {
        need[i] = 1;
        break;
      }
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    uint8_t* vis = (uint8_t*)malloc((size_t)(nk > 0 ? nk : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t i = 0; i < nq; ++i) {
      lse[i] = -INFINITY;
      Drow[i] = 0.0;
      if (!need[i]) continue;
      double m, l;
      int64_t nvis = row_logits(q + i * d, i, k, nk, d, lts, lte, uts, ute, scale, s, vis, &m, &l);
      if (nvis == 0) continue;
      lse[i] = m + log(l);
      double D = 0.0;
      for (int64_t j = 0; j < nk; ++j) {
        if (!vis[j]) continue;
        D += exp(s[j] - lse[i]) * dot(dout + i * d, v + j * d, d);
      }
      Drow[i] = D;
    }
    free(s);
    free(vis);
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < ncols; ++t) {
    const int64_t j = cols[t];
    double* gk = dk + t * d;
    double* gv = dv + t * d;
    for (int64_t c = 0; c < d; ++c) gk[c] = gv[c] = 0.0;
    for (int64_t i = 0; i < nq; ++i) {
      if (is_masked(lts, lte, uts, ute, j, i)) continue;
      const double p = exp(scale * dot(q + i * d, k + j * d, d) - lse[i]);
      const double dpij = dot(dout + i * d, v + j * d, d);
      const double ds = p * (dpij - Drow[i]);
      for (int64_t c = 0; c < d; ++c) {
        gv[c] += p * dout[i * d + c];
        gk[c] += scale * ds * q[i * d + c];
      }
    }
  }
  free(lse);
  free(Drow);
  free(need);
}

/*
 * Tile classification of one (batch, mask head): for q-tile r (rows
 * [r0, r1), r1 = min(r0 + bm, nq)) and k-tile c (columns [c0, c1),
 * c1 = min(c0 + bn, nk)), with mn_X / mx_X the min / max of vector X over the
 * tile's columns:
 *   skip (0)    if (mx_LTS <= r0 && mn_LTE >= r1) || (mx_UTS <= r0 && mn_UTE >= r1)
 *   full (2)    else if (mn_LTS >= r1 || mx_LTE <= r0 || mn_LTS >= mx_LTE)
 *                    && (mn_UTS >= r1 || mx_UTE <= r0 || mn_UTS >= mx_UTE)
 *   partial (1) otherwise.
 * The minima and maxima are taken here with plain loops over the raw vectors.
 * cls is [nQ][nK] row-major.
 */
void oracle_classify(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute, int64_t nq,
                     int64_t nk, int64_t bm, int64_t bn, uint8_t* cls) {
  const int64_t nqt = (nq + bm - 1) / bm, nkt = (nk + bn - 1) / bn;
  for (int64_t c = 0; c < nkt; ++c) {
    const int64_t c0 = c * bn, c1 = (c0 + bn < nk) ? c0 + bn : nk;
    int64_t mn[4] = {INT64_MAX, INT64_MAX, INT64_MAX, INT64_MAX};
    int64_t mx[4] = {INT64_MIN, INT64_MIN, INT64_MIN, INT64_MIN};
    const int32_t* vec[4] = {lts, lte, uts, ute};
    for (int64_t j = c0; j < c1; ++j)
      for (int t = 0; t < 4; ++t) {
        if (vec[t][j] < mn[t]) mn[t] = vec[t][j];
        if (vec[t][j] > mx[t]) mx[t] = vec[t][j];
      }
    for (int64_t r = 0; r < nqt; ++r) {
      const int64_t r0 = r * bm, r1 = (r0 + bm < nq) ? r0 + bm : nq;
      uint8_t k;
      if ((mx[0] <= r0 && mn[1] >= r1) || (mx[2] <= r0 && mn[3] >= r1))
        k = 0;
      else if ((mn[0] >= r1 || mx[1] <= r0 || mn[0] >= mx[1]) && (mn[2] >= r1 || mx[3] <= r0 || mn[2] >= mx[3]))
        k = 2;
      else
        k = 1;
      cls[r * nkt + c] = k;
    }
  }
}

/* Clip-shift-max localisation of one contiguous query chunk [a, b). */
void oracle_localize(const int32_t* in, int32_t* out, int64_t n, int32_t a, int32_t b) {
  for (int64_t j = 0; j < n; ++j) {
    int32_t x = in[j] < b ? in[j] : b; /* clip to the chunk end   */
    x = x - a;                          /* shift to chunk-local    */
    out[j] = x > 0 ? x : 0;             /* max with zero           */
  }
}

/*
 * Localisation onto several disjoint, increasing chunks [a_k, b_k) that are
 * concatenated in order into one local query sequence: a boundary x maps to
 * the number of chunk rows that lie before x, sum_k (clamp(x, a_k, b_k) - a_k).
 */
void oracle_localize_multi(const int32_t* in, int32_t* out, int64_t n, const int32_t* a, const int32_t* b,
                           int64_t nchunks) {
  for (int64_t j = 0; j < n; ++j) {
    int64_t acc = 0;
    for (int64_t t = 0; t < nchunks; ++t) {
      int64_t x = in[j];
      if (x < a[t]) x = a[t];
      if (x > b[t]) x = b[t];
      acc += x - a[t];
    }
    out[j] = (int32_t)acc;
  }
}

/* Number of unmasked (i, j) pairs of one (batch, mask head), by brute force. */
int64_t oracle_count_unmasked(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                              int64_t nq, int64_t nk) {
  int64_t total = 0;
#pragma omp parallel for reduction(+ : total) schedule(static)
  for (int64_t i = 0; i < nq; ++i) {
    int64_t cnt = 0;
    for (int64_t j = 0; j < nk; ++j) cnt += !is_masked(lts, lte, uts, ute, j, i);
    total += cnt;
  }
  return total;
}

/* Unmasked (i, j) pairs of each bm-row query tile of one (batch, mask head),
 * by brute force: out[t] counts the pairs of rows [t*bm, min((t+1)*bm, nq)). */
void oracle_tile_costs(const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute, int64_t nq,
                       int64_t nk, int64_t bm, int64_t* out) {
  const int64_t nt = (nq + bm - 1) / bm;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < nt; ++t) {
    int64_t cnt = 0;
    const int64_t r1 = (t + 1) * bm < nq ? (t + 1) * bm : nq;
    for (int64_t i = t * bm; i < r1; ++i)
      for (int64_t j = 0; j < nk; ++j) cnt += !is_masked(lts, lte, uts, ute, j, i);
    out[t] = cnt;
  }
}

int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      extern int omp_get_num_threads(void);
      n = omp_get_num_threads();
#endif
    }
  }
  return n;
}
