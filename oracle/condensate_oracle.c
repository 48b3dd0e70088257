/*
 * Condensate attention: plain, slow, double-precision CPU oracle.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file's library.  The CUDA path never
 * calls it and shares no code, header or table with it.
 *
 * What it computes, for one query row i of one (batch, q-head):
 *   t_j   = sum_l q_l k_jl                     (unscaled score, double)
 *   s_j   = t_j / sqrt(d)                      (the scaled score S_ij)
 *   C_i   = {0} U {j : i-W_i+1 <= j <= i} U Top-k_i
 *   o_i   = sum_{j in C_i} e^{s_j - m} v_j / sum_{j in C_i} e^{s_j - m}
 * Sources: "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质", §1.1
 * (attention formula, Q,K,V in R^{n x d}), §2.1 Definition 1 (Condensate
 * Manifold, S = Q K^T / sqrt(d_k)), §2.2.1-§2.2.3 (anchor, local window,
 * dynamic Top-k equations), §2.4 Corollaries 2 and 3 (finite support,
 * adaptive window), §3.2.1 Lemma (excluded scores below the Top-k threshold),
 * §3.2.2 (excluded mass epsilon), §3.2.4 Theorem 4 (output error bound).
 *
 * Readings where the pages leave a step open (each also listed in the
 * design notes):
 *   - Top-k ranks causal candidates outside anchor and window:
 *     cand_i = [1, i - W_i]; m_i = min(k, |cand_i|).  The equation of §2.2.3
 *     ranks over all n positions, which would make |C_i| variable.
 *   - Ties in t go to the lower index.  Selection uses the unscaled t.
 *   - The window is clamped to [0, i]; it then contains the anchor once.
 *   - Masses use the causal denominator (j <= i).
 *   - Theorem 4 is checked with the constant 2 and max_j |v_j|_2 (the exact
 *     identity of the renormalised sparse softmax); the page prints 1.
 *
 * Every function is pinned by the CPU tests to something other than itself:
 * brute-force subset enumeration on tiny integer inputs, a library softmax
 * for the k >= |cand| case, closed forms (two-term softmax, uniform scores),
 * the integers printed in page 1 §4.2 and §4.4, the Lemma, Theorem 4 and
 * planted-needle membership.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Diagnostics written per row (doubles). */
enum {
  DG_M = 0,            /* m_i: number of Top-k entries selected          */
  DG_SIZE,             /* |C_i|                                          */
  DG_ANCHOR_MASS,      /* A_i0 of the full causal softmax (§2.2.1)        */
  DG_WINDOW_MASS,      /* sum over the clamped window (§2.2.2)            */
  DG_TOPK_MASS,        /* sum over the Top-k entries                      */
  DG_EXCLUDED_MASS,    /* epsilon_i = sum over causal j not in C_i (§3.2.2)*/
  DG_COS,              /* cos(o_sparse, o_full) (Theorem 1 as a report)   */
  DG_ERR_L2,           /* |o_sparse - o_full|_2                            */
  DG_VMAX_L2,          /* max_{j<=i} |v_j|_2                                */
  DG_TAU_MIN,          /* t of the m_i-th selected candidate (or -inf)    */
  DG_BEST_UNSEL,       /* t of the best unselected candidate (or -inf)    */
  DG_GAP,              /* TAU_MIN - BEST_UNSEL (+inf if either is absent)  */
  DG_BOUND,            /* fp32 rounding bound beta_i on a score pair       */
  DG_WIN_LO,           /* first window position max(0, i-W_i+1)           */
  DG_LSE,              /* log sum_{j<=i} exp(s_j): the softmax normaliser  */
  DG_COUNT
};

int oracle_diag_count(void) { return DG_COUNT; }

/* t_j = q . k_j for j in [0, nkeys): §2.1 Definition 1 (S = QK^T, unscaled). */
void oracle_scores(const float* q, const float* K, int64_t nkeys, int d,
                   double* t) {
  for (int64_t j = 0; j < nkeys; ++j) {
    const float* kj = K + j * (int64_t)d;
    double acc = 0.0;
    for (int l = 0; l < d; ++l) acc += (double)q[l] * (double)kj[l];
    t[j] = acc;
  }
}

typedef struct {
  double t;
  int64_t j;
} cand_t;

/* Order of §2.2.3 Dynamic Top-k: higher score first, ties to the lower index. */
static int cand_order(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->t > b->t) return -1;
  if (a->t < b->t) return 1;
  if (a->j < b->j) return -1;
  if (a->j > b->j) return 1;
  return 0;
}

/*
 * Dynamic Top-k (§2.2.3) over cand_i = [1, i - W]: sorts the candidates by
 * (t desc, j asc) and writes the first m = min(k, |cand_i|) indices, in rank
 * order, to sel.  Also reports the m-th selected score and the best
 * unselected one.  Returns m.
 */
int64_t oracle_topk(const double* t, int64_t i, int64_t W, int64_t k,
                    int64_t* sel, double* tau_min, double* best_unsel) {
  int64_t hi = i - W; /* last candidate position */
  int64_t ncand = hi >= 1 ? hi : 0;
  int64_t m = k < ncand ? k : ncand;
  *tau_min = -INFINITY;
  *best_unsel = -INFINITY;
  if (ncand == 0) return 0;
  cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)ncand);
  for (int64_t j = 1; j <= hi; ++j) {
    c[j - 1].t = t[j];
    c[j - 1].j = j;
  }
  qsort(c, (size_t)ncand, sizeof(cand_t), cand_order);
  for (int64_t r = 0; r < m; ++r) sel[r] = c[r].j;
  if (m > 0) *tau_min = c[m - 1].t;
  if (m < ncand) *best_unsel = c[m].t;
  free(c);
  return m;
}

static int cmp_i64(const void* pa, const void* pb) {
  int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
  return (a > b) - (a < b);
}

/*
 * Condensate Set of §2.1 Definition 1: {0} U [max(0, i-W+1), i] U sel,
 * written in ascending order without repeats.  Returns |C_i|.
 */
int64_t oracle_condensate_set(int64_t i, int64_t W, const int64_t* sel,
                              int64_t m, int64_t* C) {
  int64_t lo = i - W + 1;
  if (lo < 0) lo = 0;
  int64_t n = 0;
  int64_t* tmp = (int64_t*)malloc(sizeof(int64_t) * (size_t)(m + 1));
  for (int64_t r = 0; r < m; ++r) tmp[r] = sel[r];
  qsort(tmp, (size_t)m, sizeof(int64_t), cmp_i64);
  if (lo > 0) C[n++] = 0; /* anchor, unless the window already holds it */
  for (int64_t r = 0; r < m; ++r) C[n++] = tmp[r];
  for (int64_t j = lo; j <= i; ++j) C[n++] = j;
  free(tmp);
  return n;
}

/*
 * Softmax of s = t / sqrt(d) restricted to the index list C, times V
 * (§2.3 Attention_C; §5.2.2 attention on the subset).  o has d entries.
 */
void oracle_attend(const double* t, const float* V, int d, const int64_t* C,
                   int64_t nC, double* o) {
  double scale = 1.0 / sqrt((double)d);
  double mx = -INFINITY;
  for (int64_t r = 0; r < nC; ++r) {
    double s = t[C[r]] * scale;
    if (s > mx) mx = s;
  }
  double den = 0.0;
  for (int l = 0; l < d; ++l) o[l] = 0.0;
  for (int64_t r = 0; r < nC; ++r) {
    double w = exp(t[C[r]] * scale - mx);
    den += w;
    const float* vj = V + C[r] * (int64_t)d;
    for (int l = 0; l < d; ++l) o[l] += w * (double)vj[l];
  }
  for (int l = 0; l < d; ++l) o[l] /= den;
}

/*
 * One full oracle row: scores, Top-k, set, sparse output, and the reports of
 * §2.2 (masses), §3.2 (epsilon, Lemma threshold) and Theorem 4 against the
 * full causal softmax of §1.1.
 *   q: [d]; K, V: [>= i+1, d] rows of this (batch, kv-head).
 *   C_out: capacity >= min(i+1, 1+W+k) int32 entries; returns |C_i|.
 *   o_sparse: [d]; o_full: [d] or NULL (then masses are skipped);
 *   diag: [DG_COUNT] or NULL.
 */
int64_t oracle_row(const float* q, const float* K, const float* V, int d,
                   int64_t i, int64_t W, int64_t k, int32_t* C_out,
                   double* o_sparse, double* o_full, double* diag) {
  int64_t nkeys = i + 1;
  double* t = (double*)malloc(sizeof(double) * (size_t)nkeys);
  int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (size_t)(k > 0 ? k : 1));
  int64_t cap = 1 + W + k;
  if (cap > nkeys) cap = nkeys;
  int64_t* C = (int64_t*)malloc(sizeof(int64_t) * (size_t)(cap + 1));
  double tau_min, best_unsel;

  oracle_scores(q, K, nkeys, d, t);
  int64_t m = oracle_topk(t, i, W, k, sel, &tau_min, &best_unsel);
  int64_t nC = oracle_condensate_set(i, W, sel, m, C);
  oracle_attend(t, V, d, C, nC, o_sparse);
  for (int64_t r = 0; r < nC; ++r) C_out[r] = (int32_t)C[r];

  if (diag) {
    for (int z = 0; z < DG_COUNT; ++z) diag[z] = 0.0;
    diag[DG_M] = (double)m;
    diag[DG_SIZE] = (double)nC;
    diag[DG_TAU_MIN] = tau_min;
    diag[DG_BEST_UNSEL] = best_unsel;
    diag[DG_GAP] = (m > 0 && isfinite(best_unsel)) ? tau_min - best_unsel
                                                   : INFINITY;
    int64_t lo = i - W + 1;
    diag[DG_WIN_LO] = (double)(lo < 0 ? 0 : lo);
    /* Rounding bound on one fp32 score: gamma_d * sum_l |q_l k_jl| with a
     * unit roundoff of 2^-23 (covers round-to-nearest and truncating fp32
     * accumulation).  beta_i adds the largest bound over the selected set to
     * the largest over the unselected candidates: above it no pair can swap. */
    if (m > 0 && isfinite(best_unsel)) {
      double u = ldexp(1.0, -23);
      double gam = d * u / (1.0 - d * u);
      double amax_sel = 0.0, amax_unsel = 0.0;
      char* in_sel = (char*)calloc((size_t)nkeys, 1);
      for (int64_t r = 0; r < m; ++r) in_sel[sel[r]] = 1;
      for (int64_t j = 1; j <= i - W; ++j) {
        const float* kj = K + j * (int64_t)d;
        double a = 0.0;
        for (int l = 0; l < d; ++l) a += fabs((double)q[l] * (double)kj[l]);
        if (in_sel[j]) {
          if (a > amax_sel) amax_sel = a;
        } else {
          if (a > amax_unsel) amax_unsel = a;
        }
      }
      free(in_sel);
      diag[DG_BOUND] = gam * (amax_sel + amax_unsel);
    } else {
      diag[DG_BOUND] = 0.0;
    }
  }

  if (o_full) {
    /* Full causal softmax over j <= i (§1.1), A_ij for the mass reports. */
    double scale = 1.0 / sqrt((double)d);
    double mx = -INFINITY;
    for (int64_t j = 0; j < nkeys; ++j)
      if (t[j] * scale > mx) mx = t[j] * scale;
    double* A = (double*)malloc(sizeof(double) * (size_t)nkeys);
    double den = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
      A[j] = exp(t[j] * scale - mx);
      den += A[j];
    }
    if (diag) diag[DG_LSE] = mx + log(den);
    for (int l = 0; l < d; ++l) o_full[l] = 0.0;
    double vmax = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
      A[j] /= den;
      const float* vj = V + j * (int64_t)d;
      double vn = 0.0;
      for (int l = 0; l < d; ++l) {
        o_full[l] += A[j] * (double)vj[l];
        vn += (double)vj[l] * (double)vj[l];
      }
      vn = sqrt(vn);
      if (vn > vmax) vmax = vn;
    }
    if (diag) {
      char* inC = (char*)calloc((size_t)nkeys, 1);
      for (int64_t r = 0; r < nC; ++r) inC[C[r]] = 1;
      int64_t lo = i - W + 1;
      if (lo < 0) lo = 0;
      double win = 0.0, excl = 0.0, topm = 0.0;
      for (int64_t j = lo; j <= i; ++j) win += A[j];
      for (int64_t j = 0; j < nkeys; ++j)
        if (!inC[j]) excl += A[j];
      for (int64_t r = 0; r < m; ++r) topm += A[sel[r]];
      double dot = 0.0, na = 0.0, nb = 0.0, e2 = 0.0;
      for (int l = 0; l < d; ++l) {
        dot += o_sparse[l] * o_full[l];
        na += o_sparse[l] * o_sparse[l];
        nb += o_full[l] * o_full[l];
        double e = o_sparse[l] - o_full[l];
        e2 += e * e;
      }
      diag[DG_ANCHOR_MASS] = A[0];
      diag[DG_WINDOW_MASS] = win;
      diag[DG_TOPK_MASS] = topm;
      diag[DG_EXCLUDED_MASS] = excl;
      diag[DG_COS] = (na > 0 && nb > 0) ? dot / sqrt(na * nb) : 1.0;
      diag[DG_ERR_L2] = sqrt(e2);
      diag[DG_VMAX_L2] = vmax;
      free(inC);
    }
    free(A);
  }
  free(t);
  free(sel);
  free(C);
  return nC;
}

/*
 * A batch of independent rows (prefill or decode), one thread per row.
 * Row r is described by:
 *   q_off[r]   element offset of its query in Q
 *   kv_off[r]  element offset of its (batch, kv-head) K and V slab
 *   pos[r]     query position i (keys 0..i are causal)
 *   win[r]     window W_i for this row
 * Outputs: C [rows, C_max] int32 padded with -1, count [rows],
 * o_sparse [rows, d], o_full [rows, d] (may be NULL), diag [rows, DG_COUNT]
 * (may be NULL).  Returns 0, or -1 if some row's set does not fit C_max.
 */
int oracle_rows(const float* Q, const float* K, const float* V, int d, int k,
                const int64_t* q_off, const int64_t* kv_off,
                const int64_t* pos, const int32_t* win, int64_t rows,
                int C_max, int32_t* C, int32_t* count, double* o_sparse,
                double* o_full, double* diag, int threads) {
  int bad = 0;
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#else
  (void)threads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < rows; ++r) {
    int64_t i = pos[r];
    int64_t W = win[r];
    int64_t need = 1 + W + k;
    if (need > i + 1) need = i + 1;
    if (need > C_max) {
      bad |= 1;
      continue;
    }
    int32_t* Cr = C + r * (int64_t)C_max;
    for (int z = 0; z < C_max; ++z) Cr[z] = -1;
    count[r] = (int32_t)oracle_row(
        Q + q_off[r], K + kv_off[r], V + kv_off[r], d, i, W, k, Cr,
        o_sparse + r * (int64_t)d, o_full ? o_full + r * (int64_t)d : NULL,
        diag ? diag + r * (int64_t)DG_COUNT : NULL);
  }
  return bad ? -1 : 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
