/*
 * llsa_oracle.c -- plain CPU oracle for Log-linear Sparse Attention (LLSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg load this library.  The CUDA product path
 * never links, loads or calls it, and it shares no code, header or table with
 * that path.
 *
 * Every routine is written as the method's definition in plain loops with
 * fp64 accumulation: no tiling, no fusion, no reordering of the arithmetic
 * beyond what the definition states.  Each routine works on ONE (batch, head)
 * slice; callers loop over slices.
 *
 * Sources (web pages about the method; cited by page title and section):
 *   [LLSA] "Trainable Log-linear Sparse Attention for Efficient Diffusion
 *          Transformers" (CVPR 2026) -- technical summary page.
 *   [ART]  Popular write-up of arXiv:2512.16615 ("log-linear sparse
 *          attention"), section 三 (hierarchical top-K, KV reweighting) and
 *          section 四 (GPU implementation: sparse index transpose, reordering).
 *
 * Single-slice layouts (all row-major, hierarchical token order unless noted):
 *   x      [N][d]                       level-0 tokens (N = H*W)
 *   pyr    level l = 1..L packed:       [n_l][d] at offset d * sum_{l'<l} n_l'
 *   idx    level l = 1..L packed:       [n_l][K_l] at offset sum_{l'<l} n_l' K_l'
 *   offs   level l = 1..L packed:       [n_l + 1]  at offset sum_{l'<l} (n_l' + 1)
 *   qlist  same packing as idx
 * with n_l = N / B^l, K_L = min(K, n_L), K_l = min(K, K_{l+1} * B) for l < L.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int H, W;               /* image height and width in pixels */
  int d;                  /* head dimension */
  int B;                  /* block size (a perfect square, B = t*t) */
  int L;                  /* number of pooled levels */
  int K;                  /* top-K per level */
  unsigned enrich_mask;   /* bit (l-1) set: level-l coarse KV joins the attention */
  double scale;           /* softmax scale applied to q.k */
} oracle_problem;

/* ---------------------------------------------------------------- sizes */

static int64_t ipow(int64_t b, int e) {
  int64_t r = 1;
  for (int i = 0; i < e; ++i) r *= b;
  return r;
}

static int side_of_block(int B) {
  int t = 0;
  while ((t + 1) * (t + 1) <= B) ++t;
  return (t * t == B) ? t : -1;
}

/* Level sizes n[0..L] and per-level list lengths Kl[1..L] ([LLSA] §三:
 * level l has N / B^l tokens; the coarsest level keeps top-K of all its
 * tokens, every finer level keeps top-K of the K_{l+1}*B children of its
 * parent's picks, or all of them when there are fewer than K).
 * Returns 0, or -1 when the image does not tile into t^L x t^L squares. */
int oracle_levels(const oracle_problem* p, int64_t* n, int64_t* Kl) {
  int t = side_of_block(p->B);
  if (t < 2 || p->L < 1 || p->K < 1) return -1;
  int64_t tl = ipow(t, p->L);
  if (p->H % tl || p->W % tl) return -1;
  int64_t N = (int64_t)p->H * p->W;
  for (int l = 0; l <= p->L; ++l) n[l] = N / ipow(p->B, l);
  Kl[0] = 0;
  Kl[p->L] = n[p->L] < p->K ? n[p->L] : p->K;
  for (int l = p->L - 1; l >= 1; --l) {
    int64_t cand = Kl[l + 1] * p->B;
    Kl[l] = cand < p->K ? cand : p->K;
  }
  return 0;
}

/* ------------------------------------------------------------- reorder */

/* Hierarchical token order for 2-D pixel tokens ([ART] §四, index
 * reordering; [LLSA] §4.2, Fig. 2).  The pages only ask that spatial
 * neighbours stay adjacent after flattening "like a Z-order or Hilbert
 * curve"; the reading used here is recursive t x t tiles (t = sqrt(B)),
 * row-major inside every tile and row-major across the top grid of
 * t^L x t^L squares, so that every aligned run of B^l indices is one
 * t^l x t^l pixel square.
 *   hier(y, x) = (floor(y/t^L) * Gw + floor(x/t^L)) * B^L
 *              + sum_{l=1..L} ((floor(y/t^(l-1)) mod t) * t + floor(x/t^(l-1)) mod t) * B^(l-1)
 * Output: hier_of_raster[y*W + x] = hier(y, x). */
void oracle_reorder_index(const oracle_problem* p, int64_t* hier_of_raster) {
  int t = side_of_block(p->B);
  int64_t tL = ipow(t, p->L), BL = ipow(p->B, p->L);
  int64_t Gw = p->W / tL;
  for (int64_t y = 0; y < p->H; ++y) {
    for (int64_t x = 0; x < p->W; ++x) {
      int64_t h = ((y / tL) * Gw + (x / tL)) * BL;
      int64_t tp = 1, Bp = 1;   /* t^(l-1), B^(l-1) */
      for (int l = 1; l <= p->L; ++l) {
        int64_t ry = (y / tp) % t, rx = (x / tp) % t;
        h += (ry * t + rx) * Bp;
        tp *= t;
        Bp *= p->B;
      }
      hier_of_raster[y * p->W + x] = h;
    }
  }
}

/* Move the rows of one [N][d] slice between raster and hierarchical order. */
void oracle_reorder(const oracle_problem* p, const double* in, double* out, int to_hier) {
  int64_t N = (int64_t)p->H * p->W;
  int64_t* hier = (int64_t*)malloc(sizeof(int64_t) * N);
  oracle_reorder_index(p, hier);
  for (int64_t r = 0; r < N; ++r) {
    const double* src = to_hier ? in + r * p->d : in + hier[r] * p->d;
    double* dst = to_hier ? out + hier[r] * p->d : out + r * p->d;
    for (int c = 0; c < p->d; ++c) dst[c] = src[c];
  }
  free(hier);
}

/* ---------------------------------------------------------------- pool */

/* Hierarchical compression ([LLSA] §三): recursive mean pooling,
 * P_0 = X and P_l[j] = (1/B) * sum_{c<B} P_{l-1}[j*B + c] for l = 1..L.
 * Applied to Q, K and V alike. */
void oracle_pool(const oracle_problem* p, const double* x, double* pyr) {
  int64_t n[64], Kl[64];
  if (oracle_levels(p, n, Kl)) return;
  const double* prev = x;
  double* cur = pyr;
  for (int l = 1; l <= p->L; ++l) {
    for (int64_t j = 0; j < n[l]; ++j) {
      for (int c = 0; c < p->d; ++c) {
        double s = 0.0;
        for (int r = 0; r < p->B; ++r) s += prev[(j * p->B + r) * p->d + c];
        cur[j * p->d + c] = s / p->B;
      }
    }
    prev = cur;
    cur += n[l] * p->d;
  }
}

/* ----------------------------------------------------------- selection */

typedef struct { double s; int32_t id; } scored;

/* higher score first; equal scores: lower index first */
static int by_score_desc(const void* a, const void* b) {
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

static int by_int_asc(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

static int64_t pyr_offset(const int64_t* n, int l, int d) {
  int64_t o = 0;
  for (int i = 1; i < l; ++i) o += n[i] * d;
  return o;
}

static int64_t idx_offset(const int64_t* n, const int64_t* Kl, int l) {
  int64_t o = 0;
  for (int i = 1; i < l; ++i) o += n[i] * Kl[i];
  return o;
}

/* Coarse-to-fine top-K at one level ([LLSA] §三; [ART] §三).
 *   l == L : every level-L query token a scores all n_L level-L key tokens.
 *   l <  L : query a with parent p = floor(a/B) scores only the children
 *            {c*B + r : c in S_{l+1}(p), r < B} of its parent's picks.
 * Score = P^Q_l[a] . P^K_l[c] (the positive softmax scale does not change
 * the ranking).  Keep the K_l best: higher score first, lower index on ties.
 * idx_l receives each kept list sorted ascending.  If R > 0, the R best
 * candidates (descending, ties by lower index) and their scores go to
 * ranked_id / ranked_score (padded with -1 / -INFINITY), so that a test can
 * judge near-ties.
 * pyrQ, pyrK: the single-slice packed pyramids.  idx: the packed index lists;
 * level l+1 must already be filled when l < L. */
void oracle_select_level(const oracle_problem* p, int l, const double* pyrQ, const double* pyrK,
                         int32_t* idx, int R, int32_t* ranked_id, double* ranked_score) {
  int64_t n[64], Kl[64];
  if (oracle_levels(p, n, Kl)) return;
  const int d = p->d;
  const double* q = pyrQ + pyr_offset(n, l, d);
  const double* k = pyrK + pyr_offset(n, l, d);
  int32_t* out = idx + idx_offset(n, Kl, l);
  const int32_t* parent = (l < p->L) ? idx + idx_offset(n, Kl, l + 1) : NULL;
  int64_t ncand = (l == p->L) ? n[l] : Kl[l + 1] * p->B;
  scored* cand = (scored*)malloc(sizeof(scored) * (size_t)ncand);
  for (int64_t a = 0; a < n[l]; ++a) {
    for (int64_t m = 0; m < ncand; ++m) {
      int64_t c;
      if (l == p->L) {
        c = m;
      } else {
        int64_t par = a / p->B;
        c = (int64_t)parent[par * Kl[l + 1] + m / p->B] * p->B + m % p->B;
      }
      double s = 0.0;
      for (int e = 0; e < d; ++e) s += q[a * d + e] * k[c * d + e];
      cand[m].s = s;
      cand[m].id = (int32_t)c;
    }
    qsort(cand, (size_t)ncand, sizeof(scored), by_score_desc);
    for (int64_t m = 0; m < Kl[l]; ++m) out[a * Kl[l] + m] = cand[m].id;
    qsort(out + a * Kl[l], (size_t)Kl[l], sizeof(int32_t), by_int_asc);
    for (int m = 0; m < R; ++m) {
      ranked_id[a * R + m] = m < ncand ? cand[m].id : -1;
      ranked_score[a * R + m] = m < ncand ? cand[m].s : -INFINITY;
    }
  }
  free(cand);
}

/* All levels, coarsest first ([LLSA] §三, Fig. 1). */
void oracle_select(const oracle_problem* p, const double* pyrQ, const double* pyrK, int32_t* idx) {
  for (int l = p->L; l >= 1; --l) oracle_select_level(p, l, pyrQ, pyrK, idx, 0, NULL, NULL);
}

/* ----------------------------------------------------------- attention */

/* The key set of fine query i ([LLSA] §四, hierarchical KV enrichment;
 * [ART] §三, KV reweighting):
 *   fine:   the B tokens of every level-1 block c in S_1(floor(i/B)), logit
 *           scale * q_i . k_j;
 *   coarse: for every enriched level l, the level-l tokens c in
 *           S_l(floor(i/B^l)), logit scale * q_i . P^K_l[c] + ln(B^l), value
 *           P^V_l[c].  The weight W^(l) = B^l multiplies the softmax term of a
 *           coarse token, which is the same as adding ln(B^l) to its logit.
 * Fills key/value pointers and biases; returns the number of keys. */
static int64_t key_set(const oracle_problem* p, const int64_t* n, const int64_t* Kl, int64_t i,
                       const double* k, const double* v, const double* pyrK, const double* pyrV,
                       const int32_t* idx, const double** kp, const double** vp, double* bias,
                       int* level, int64_t* id) {
  const int d = p->d;
  int64_t m = 0;
  const int32_t* s1 = idx + idx_offset(n, Kl, 1) + (i / p->B) * Kl[1];
  for (int64_t u = 0; u < Kl[1]; ++u) {
    for (int r = 0; r < p->B; ++r) {
      int64_t j = (int64_t)s1[u] * p->B + r;
      kp[m] = k + j * d;
      vp[m] = v + j * d;
      bias[m] = 0.0;
      level[m] = 0;
      id[m] = j;
      ++m;
    }
  }
  int64_t Bl = 1;
  for (int l = 1; l <= p->L; ++l) {
    Bl *= p->B;
    if (!((p->enrich_mask >> (l - 1)) & 1u)) continue;
    const int32_t* sl = idx + idx_offset(n, Kl, l) + (i / Bl) * Kl[l];
    const double* kl = pyrK + pyr_offset(n, l, d);
    const double* vl = pyrV + pyr_offset(n, l, d);
    for (int64_t u = 0; u < Kl[l]; ++u) {
      kp[m] = kl + (int64_t)sl[u] * d;
      vp[m] = vl + (int64_t)sl[u] * d;
      bias[m] = log((double)Bl);
      level[m] = l;
      id[m] = sl[u];
      ++m;
    }
  }
  return m;
}

static int64_t max_keys(const oracle_problem* p, const int64_t* Kl) {
  int64_t m = Kl[1] * p->B;
  for (int l = 1; l <= p->L; ++l) m += Kl[l];
  return m;
}

/* Forward for the fine queries listed in rows[0..nrows) (all N when rows is
 * NULL): softmax over the key set above; o_i = sum_j softmax(z)_j v_j and
 * lse_i = log sum_j exp(z_j).  Outputs are indexed by query token i. */
void oracle_attn_fwd_rows(const oracle_problem* p, const double* q, const double* k, const double* v,
                          const double* pyrK, const double* pyrV, const int32_t* idx,
                          const int64_t* rows, int64_t nrows, double* o, double* lse) {
  int64_t n[64], Kl[64];
  if (oracle_levels(p, n, Kl)) return;
  const int d = p->d;
  int64_t mk = max_keys(p, Kl);
  const double** kp = (const double**)malloc(sizeof(double*) * mk);
  const double** vp = (const double**)malloc(sizeof(double*) * mk);
  double* bias = (double*)malloc(sizeof(double) * mk);
  double* z = (double*)malloc(sizeof(double) * mk);
  int* level = (int*)malloc(sizeof(int) * mk);
  int64_t* id = (int64_t*)malloc(sizeof(int64_t) * mk);
  int64_t count = rows ? nrows : n[0];
  for (int64_t r = 0; r < count; ++r) {
    int64_t i = rows ? rows[r] : r;
    int64_t m = key_set(p, n, Kl, i, k, v, pyrK, pyrV, idx, kp, vp, bias, level, id);
    double zmax = -INFINITY;
    for (int64_t j = 0; j < m; ++j) {
      double s = 0.0;
      for (int e = 0; e < d; ++e) s += q[i * d + e] * kp[j][e];
      z[j] = p->scale * s + bias[j];
      if (z[j] > zmax) zmax = z[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < m; ++j) sum += exp(z[j] - zmax);
    for (int e = 0; e < d; ++e) {
      double acc = 0.0;
      for (int64_t j = 0; j < m; ++j) acc += exp(z[j] - zmax) * vp[j][e];
      o[i * d + e] = acc / sum;
    }
    lse[i] = zmax + log(sum);
  }
  free(kp); free(vp); free(bias); free(z); free(level); free(id);
}

void oracle_attn_fwd(const oracle_problem* p, const double* q, const double* k, const double* v,
                     const double* pyrK, const double* pyrV, const int32_t* idx, double* o, double* lse) {
  oracle_attn_fwd_rows(p, q, k, v, pyrK, pyrV, idx, NULL, 0, o, lse);
}

/* Backward with the index lists held fixed ([LLSA] §4.1: the method is
 * trained end to end through the sparse attention; no gradient reaches the
 * selection, whose output is a set of integers).  For every fine query i,
 * with P_j = exp(z_j - lse_i) and D_i = dO_i . o_i:
 *   dz_j  = P_j (dO_i . v_j - D_i)
 *   dq_i += scale * dz_j * k_j
 *   fine j:     dk_j += scale * dz_j * q_i,   dv_j += P_j * dO_i
 *   coarse j:   dPK_l[c] += scale * dz_j * q_i,  dPV_l[c] += P_j * dO_i
 * and the adjoint of mean pooling ([LLSA] §三) sends every pooled gradient
 * back to the B^l tokens it averages: dk_t += dPK_l[floor(t/B^l)] / B^l
 * (the same for v).  Pooled Q is used only for selection, so it receives
 * no gradient.  If dpk/dpv are not NULL they receive the pooled-level
 * gradients (same packing as a pyramid).  With rows != NULL only the listed
 * fine queries contribute (a bounded sample of the work, used to time the
 * oracle); rows == NULL is the complete backward. */
void oracle_attn_bwd_rows(const oracle_problem* p, const double* q, const double* k, const double* v,
                          const double* pyrK, const double* pyrV, const int32_t* idx, const double* dO,
                          const int64_t* rows, int64_t nrows, double* dq, double* dk, double* dv, double* dpk,
                          double* dpv) {
  int64_t n[64], Kl[64];
  if (oracle_levels(p, n, Kl)) return;
  const int d = p->d;
  int64_t pyr_total = pyr_offset(n, p->L + 1, d);
  double* gpk = (double*)calloc((size_t)pyr_total, sizeof(double));
  double* gpv = (double*)calloc((size_t)pyr_total, sizeof(double));
  memset(dq, 0, sizeof(double) * n[0] * d);
  memset(dk, 0, sizeof(double) * n[0] * d);
  memset(dv, 0, sizeof(double) * n[0] * d);
  int64_t mk = max_keys(p, Kl);
  const double** kp = (const double**)malloc(sizeof(double*) * mk);
  const double** vp = (const double**)malloc(sizeof(double*) * mk);
  double* bias = (double*)malloc(sizeof(double) * mk);
  double* z = (double*)malloc(sizeof(double) * mk);
  int* level = (int*)malloc(sizeof(int) * mk);
  int64_t* id = (int64_t*)malloc(sizeof(int64_t) * mk);
  double* o = (double*)malloc(sizeof(double) * d);
  int64_t count = rows ? nrows : n[0];
  for (int64_t r = 0; r < count; ++r) {
    int64_t i = rows ? rows[r] : r;
    int64_t m = key_set(p, n, Kl, i, k, v, pyrK, pyrV, idx, kp, vp, bias, level, id);
    double zmax = -INFINITY;
    for (int64_t j = 0; j < m; ++j) {
      double s = 0.0;
      for (int e = 0; e < d; ++e) s += q[i * d + e] * kp[j][e];
      z[j] = p->scale * s + bias[j];
      if (z[j] > zmax) zmax = z[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < m; ++j) sum += exp(z[j] - zmax);
    double lse = zmax + log(sum);
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int64_t j = 0; j < m; ++j) {
      double P = exp(z[j] - lse);
      for (int e = 0; e < d; ++e) o[e] += P * vp[j][e];
    }
    double D = 0.0;
    for (int e = 0; e < d; ++e) D += dO[i * d + e] * o[e];
    for (int64_t j = 0; j < m; ++j) {
      double P = exp(z[j] - lse);
      double dP = 0.0;
      for (int e = 0; e < d; ++e) dP += dO[i * d + e] * vp[j][e];
      double dz = P * (dP - D);
      for (int e = 0; e < d; ++e) dq[i * d + e] += p->scale * dz * kp[j][e];
      double *gk, *gv;
      if (level[j] == 0) {
        gk = dk + id[j] * d;
        gv = dv + id[j] * d;
      } else {
        gk = gpk + pyr_offset(n, level[j], d) + id[j] * d;
        gv = gpv + pyr_offset(n, level[j], d) + id[j] * d;
      }
      for (int e = 0; e < d; ++e) {
        gk[e] += p->scale * dz * q[i * d + e];
        gv[e] += P * dO[i * d + e];
      }
    }
  }
  /* adjoint of mean pooling */
  for (int64_t t = 0; t < n[0]; ++t) {
    int64_t Bl = 1;
    for (int l = 1; l <= p->L; ++l) {
      Bl *= p->B;
      const double* gk = gpk + pyr_offset(n, l, d) + (t / Bl) * d;
      const double* gv = gpv + pyr_offset(n, l, d) + (t / Bl) * d;
      for (int e = 0; e < d; ++e) {
        dk[t * d + e] += gk[e] / (double)Bl;
        dv[t * d + e] += gv[e] / (double)Bl;
      }
    }
  }
  if (dpk) memcpy(dpk, gpk, sizeof(double) * pyr_total);
  if (dpv) memcpy(dpv, gpv, sizeof(double) * pyr_total);
  free(gpk); free(gpv); free(kp); free(vp); free(bias); free(z); free(level); free(id); free(o);
}

/* The whole backward: every fine query contributes. */
void oracle_attn_bwd(const oracle_problem* p, const double* q, const double* k, const double* v,
                     const double* pyrK, const double* pyrV, const int32_t* idx, const double* dO,
                     double* dq, double* dk, double* dv, double* dpk, double* dpv) {
  oracle_attn_bwd_rows(p, q, k, v, pyrK, pyrV, idx, dO, NULL, 0, dq, dk, dv, dpk, dpv);
}

/* ------------------------------------------------------ index transpose */

/* Sparse index transpose, query-major lists to key-major lists ([ART] §四;
 * [LLSA] §4.1): per level, count how many queries picked each key, take the
 * exclusive prefix sum of the counts as offsets, and place every query id in
 * its key's range.  Within one key's range the query ids are ascending (the
 * pages leave the order open; ascending makes the result unique). */
void oracle_index_transpose(const oracle_problem* p, const int32_t* idx, int32_t* offs, int32_t* qlist) {
  int64_t n[64], Kl[64];
  if (oracle_levels(p, n, Kl)) return;
  int64_t off_base = 0;
  for (int l = 1; l <= p->L; ++l) {
    const int32_t* in = idx + idx_offset(n, Kl, l);
    int32_t* of = offs + off_base;
    int32_t* ql = qlist + idx_offset(n, Kl, l);
    int64_t* count = (int64_t*)calloc((size_t)n[l], sizeof(int64_t));
    for (int64_t a = 0; a < n[l]; ++a)
      for (int64_t u = 0; u < Kl[l]; ++u) count[in[a * Kl[l] + u]] += 1;
    int64_t run = 0;
    for (int64_t j = 0; j < n[l]; ++j) {
      of[j] = (int32_t)run;
      run += count[j];
    }
    of[n[l]] = (int32_t)run;
    int64_t* fill = (int64_t*)calloc((size_t)n[l], sizeof(int64_t));
    for (int64_t a = 0; a < n[l]; ++a) {      /* ascending a, so every range ends up ascending */
      for (int64_t u = 0; u < Kl[l]; ++u) {
        int32_t j = in[a * Kl[l] + u];
        ql[of[j] + fill[j]] = (int32_t)a;
        fill[j] += 1;
      }
    }
    free(count);
    free(fill);
    off_base += n[l] + 1;
  }
}

/* dq for the fine queries listed in rows[0..nrows) only (the same formula as
 * oracle_attn_bwd: dq_i = scale * sum_j P_ij (dO_i . v_j - D_i) k_j); each row
 * needs nothing but its own key set, so it can be computed one by one. */
void oracle_attn_dq_rows(const oracle_problem* p, const double* q, const double* k, const double* v,
                         const double* pyrK, const double* pyrV, const int32_t* idx, const double* dO,
                         const int64_t* rows, int64_t nrows, double* dq) {
  int64_t n[64], Kl[64];
  if (oracle_levels(p, n, Kl)) return;
  const int d = p->d;
  int64_t mk = max_keys(p, Kl);
  const double** kp = (const double**)malloc(sizeof(double*) * mk);
  const double** vp = (const double**)malloc(sizeof(double*) * mk);
  double* bias = (double*)malloc(sizeof(double) * mk);
  double* z = (double*)malloc(sizeof(double) * mk);
  int* level = (int*)malloc(sizeof(int) * mk);
  int64_t* id = (int64_t*)malloc(sizeof(int64_t) * mk);
  double* o = (double*)malloc(sizeof(double) * d);
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t i = rows[r];
    int64_t m = key_set(p, n, Kl, i, k, v, pyrK, pyrV, idx, kp, vp, bias, level, id);
    double zmax = -INFINITY;
    for (int64_t j = 0; j < m; ++j) {
      double s = 0.0;
      for (int e = 0; e < d; ++e) s += q[i * d + e] * kp[j][e];
      z[j] = p->scale * s + bias[j];
      if (z[j] > zmax) zmax = z[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < m; ++j) sum += exp(z[j] - zmax);
    double lse = zmax + log(sum);
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int64_t j = 0; j < m; ++j) {
      double P = exp(z[j] - lse);
      for (int e = 0; e < d; ++e) o[e] += P * vp[j][e];
    }
    double D = 0.0;
    for (int e = 0; e < d; ++e) D += dO[i * d + e] * o[e];
    for (int e = 0; e < d; ++e) dq[i * d + e] = 0.0;
    for (int64_t j = 0; j < m; ++j) {
      double P = exp(z[j] - lse);
      double dP = 0.0;
      for (int e = 0; e < d; ++e) dP += dO[i * d + e] * vp[j][e];
      double dz = P * (dP - D);
      for (int e = 0; e < d; ++e) dq[i * d + e] += p->scale * dz * kp[j][e];
    }
  }
  free(kp); free(vp); free(bias); free(z); free(level); free(id); free(o);
}
