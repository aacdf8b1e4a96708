/*
 * rtp_oracle.c -- plain fp64 CPU oracle of the RTPurbo head-wise sparse attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg load this library.  It shares no code, header or table with the CUDA
 * library; both read the same seeded bf16/fp32 inputs and nothing else.
 *
 * What it computes, for one query head h of one sequence and one query row at absolute
 * position i (the row's own key is already in the cache, so keys j = 0..i are causal):
 *
 *   Local head (Full Attention Strikes Back, P2 section 2 "local heads"; P2 section 8
 *   "window 8192 with 4 attention sinks"):
 *       J = { j <= i : i - j < W }  union  { j <= i : j < S }.
 *
 *   Retrieval head (P2 section 3 "16-dim radar then exact 128-dim attention";
 *   ngjoo digest "low-dimensional pre-RoPE projections ... dynamic top-p"):
 *       qt = Wq_h^T q_i,  kt_j = Wk_h^T k_j      (pre-RoPE, r = 16)
 *       s_j = qt . kt_j,  pi_j = exp(s_j - max s) / sum exp(s - max s)   (j <= i)
 *       order j by (s_j descending, j ascending); J = the shortest prefix of that order
 *       whose cumulative pi is >= p  (P1 insight 3, P2 section 4 "cover p of the
 *       attention mass"; ties go to the lower index; p >= 1 keeps every causal key).
 *
 *   Both classes then run exact attention in the full head dim over J
 *   (P2 section 3 "full 128-dim exact computation on the selected tokens"):
 *       o = sum_{j in J} softmax_j( sm_scale * RoPE(q_i, i) . RoPE(k_j, j) ) v_j.
 *
 *   With a fixed budget k > 0 instead of p (the pages' top-k ablation), J is the first
 *   min(k, i + 1) keys of that order.
 *
 *   With bf16 index-key storage (an option of the layer), every component of kt_j is first
 *   rounded to bf16, ties to even (orc_round_bf16); the query side stays fp64.
 *
 *   RoPE is the rotate-half form: for c < D/2 the pair (c, c + D/2) turns by
 *   angle pos * base^(-2c/D).  The pages lose the formula in extraction; this is the
 *   plainest reading consistent with "low frequencies carry semantics" (P3 finding 2).
 *
 * Everything is fp64; bf16 inputs are widened exactly.  Rows run in parallel with
 * OpenMP; each row is computed independently with plain loops and one library sort.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- scalar helpers */

double orc_bf16(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Rotate-half RoPE of one D-vector at absolute position pos. */
void orc_rope(const double* x, double pos, int D, double base, double* y) {
  int half = D / 2;
  for (int c = 0; c < half; ++c) {
    double theta = pow(base, -2.0 * (double)c / (double)D);
    double a = pos * theta;
    double cs = cos(a), sn = sin(a);
    y[c] = x[c] * cs - x[c + half] * sn;
    y[c + half] = x[c + half] * cs + x[c] * sn;
  }
}

/*
 * x rounded to the nearest bf16 value (8 significant bits), ties to even: the storage of the
 * index keys when the layer keeps them in bf16 (a storage choice the pages leave open; the
 * aitntnews page, finding 2, calls the r = 16 indexer's cost "almost negligible").  Written
 * from the definition: scale the significand to [128, 256), round half to even, scale back.
 */
double orc_round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  double m = frexp(x, &e);        /* x = m * 2^e, 0.5 <= |m| < 1 */
  double t = ldexp(m, 8);         /* |t| in [128, 256): the bf16 significand */
  double f = floor(t);
  double d = t - f;
  if (d > 0.5 || (d == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;
  return ldexp(f, e - 8);
}

/* y[t] = sum_d W[d][t] x[d]: the 16-dim projection (W is [D][r], fp32). */
void orc_index_vec(const double* x, const float* W, int D, int r, double* y) {
  for (int t = 0; t < r; ++t) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += (double)W[(int64_t)d * r + t] * x[d];
    y[t] = acc;
  }
}

/* ---------------------------------------------------------------- top-p selection */

typedef struct {
  double s;
  int64_t j;
} orc_pair;

static int orc_cmp_desc(const void* a, const void* b) {
  const orc_pair* x = (const orc_pair*)a;
  const orc_pair* y = (const orc_pair*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j) ? 1 : 0;
}

/*
 * Top-p over scores s[0..n-1].  Returns K = |J|.  order[0..n-1] receives the key order
 * (s desc, j asc), so order[0..K-1] is J.  pi[j] (optional) receives the softmax mass.
 * mass = cumulative mass of J; pi_t = mass of its last member; cum_prev = cumulative mass
 * of the first K-1 members.
 */
int64_t orc_topp(const double* s, int64_t n, double p, int64_t* order, double* pi, double* mass,
                 double* pi_t, double* cum_prev) {
  if (n <= 0) return 0;
  double m = s[0];
  for (int64_t j = 1; j < n; ++j)
    if (s[j] > m) m = s[j];
  double Z = 0.0;
  for (int64_t j = 0; j < n; ++j) Z += exp(s[j] - m);
  orc_pair* pr = (orc_pair*)malloc(sizeof(orc_pair) * (size_t)n);
  for (int64_t j = 0; j < n; ++j) {
    pr[j].s = s[j];
    pr[j].j = j;
    if (pi) pi[j] = exp(s[j] - m) / Z;
  }
  qsort(pr, (size_t)n, sizeof(orc_pair), orc_cmp_desc);
  int64_t K = n;
  double cum = 0.0, prev = 0.0, last = 0.0;
  for (int64_t k = 0; k < n; ++k) {
    double pk = exp(pr[k].s - m) / Z;
    prev = cum;
    cum += pk;
    last = pk;
    if (p < 1.0 && cum >= p) {
      K = k + 1;
      break;
    }
  }
  for (int64_t k = 0; k < n; ++k) order[k] = pr[k].j;
  if (mass) *mass = cum;
  if (pi_t) *pi_t = last;
  if (cum_prev) *cum_prev = prev;
  free(pr);
  return K;
}

/*
 * Fixed top-k over scores s[0..n-1] (the ablation the techwalker page, section 4 and its
 * Q&A, sets against dynamic top-p: a fixed budget of 4096 or 16384 tokens): J = the first
 * min(k, n) keys of the order (s desc, j asc).  order / pi / mass / pi_t / cum_prev as for
 * orc_topp (the masses are reported, not used for the cut).
 */
int64_t orc_topk(const double* s, int64_t n, int64_t k, int64_t* order, double* pi, double* mass, double* pi_t,
                 double* cum_prev) {
  if (n <= 0) return 0;
  double* pw = (double*)malloc(sizeof(double) * (size_t)n);
  orc_topp(s, n, 1.0, order, pw, NULL, NULL, NULL); /* the full order and every mass */
  int64_t K = k < n ? k : n;
  double cum = 0.0, prev = 0.0, last = 0.0;
  for (int64_t t = 0; t < K; ++t) {
    prev = cum;
    last = pw[order[t]];
    cum += last;
  }
  if (pi) memcpy(pi, pw, sizeof(double) * (size_t)n);
  if (mass) *mass = cum;
  if (pi_t) *pi_t = last;
  if (cum_prev) *cum_prev = prev;
  free(pw);
  return K;
}

static int orc_cmp_i64(const void* a, const void* b) {
  int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return (x < y) ? -1 : (x > y) ? 1 : 0;
}

/* ---------------------------------------------------------------- attention */

/*
 * Exact softmax attention of one query over the keys listed in J.
 * qrot: RoPE'd query (fp64).  krot(j) is either taken from a precomputed table
 * (rows lo..hi) or computed from the bf16 pre-RoPE key.
 */
typedef struct {
  const uint16_t* k;
  const uint16_t* v;
  int64_t stride; /* elements between consecutive positions */
  int D;
  double base;
  int64_t pos_offset;
  const double* rot_tab; /* RoPE'd keys for positions [tab_lo, tab_hi], or NULL */
  int64_t tab_lo, tab_hi;
} orc_kv;

static void orc_key_rot(const orc_kv* kv, int64_t j, double* tmp, double* out) {
  if (kv->rot_tab && j >= kv->tab_lo && j <= kv->tab_hi) {
    memcpy(out, kv->rot_tab + (j - kv->tab_lo) * kv->D, sizeof(double) * (size_t)kv->D);
    return;
  }
  for (int d = 0; d < kv->D; ++d) tmp[d] = orc_bf16(kv->k[j * kv->stride + d]);
  orc_rope(tmp, (double)(j + kv->pos_offset), kv->D, kv->base, out);
}

void orc_attend(const double* qrot, const orc_kv* kv, const int64_t* J, int64_t nJ, double scale,
                double* out) {
  int D = kv->D;
  double* logit = (double*)malloc(sizeof(double) * (size_t)(nJ > 0 ? nJ : 1));
  double* tmp = (double*)malloc(sizeof(double) * (size_t)D);
  double* kr = (double*)malloc(sizeof(double) * (size_t)D);
  double m = -INFINITY;
  for (int64_t t = 0; t < nJ; ++t) {
    orc_key_rot(kv, J[t], tmp, kr);
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += qrot[d] * kr[d];
    logit[t] = scale * acc;
    if (logit[t] > m) m = logit[t];
  }
  double Z = 0.0;
  for (int64_t t = 0; t < nJ; ++t) Z += exp(logit[t] - m);
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int64_t t = 0; t < nJ; ++t) {
    double w = exp(logit[t] - m) / Z;
    const uint16_t* vr = kv->v + J[t] * kv->stride;
    for (int d = 0; d < D; ++d) out[d] += w * orc_bf16(vr[d]);
  }
  free(logit);
  free(tmp);
  free(kr);
}

/* ---------------------------------------------------------------- one head, many rows */

/*
 * k, v: bf16 bits for one sequence, laid out [n_keys][kv_stride]; this head's KV head
 *       starts at element g*D of each position.  q: [nrows][q_stride], row t starts at
 *       q + t*q_stride (pre-RoPE).  pos[t]: absolute position of row t (< n_keys).
 * Outputs (per row t): out[t][D]; sel_count[t] = |J|; sel_mass[t] / pi_t[t] / cum_prev[t]
 * (retrieval heads; local heads report 1, 0, 0); sel_idx[t][0..min(|J|,sel_cap)-1] the
 * members of J ascending (optional); pi_all[t][0..pos] the index-softmax masses
 * (optional, retrieval heads).
 */
int orc_head_rows(const uint16_t* k, const uint16_t* v, int64_t n_keys, int64_t kv_stride, int g,
                  int D, int r, const uint16_t* q, int64_t q_stride, const int64_t* pos,
                  int64_t nrows, int is_retrieval, const float* wq, const float* wk, double top_p,
                  int64_t window, int64_t n_sink, double rope_base, double sm_scale,
                  int64_t pos_offset, double* out, int64_t* sel_count, double* sel_mass,
                  double* pi_t, double* cum_prev, int64_t* sel_idx, int64_t sel_cap,
                  double* pi_all, int64_t pi_stride, int n_threads, int key_bf16, int64_t top_k) {
  if (nrows <= 0) return 0;
  int64_t maxpos = 0, minpos = pos[0];
  for (int64_t t = 0; t < nrows; ++t) {
    if (pos[t] < 0 || pos[t] >= n_keys) return -1;
    if (pos[t] > maxpos) maxpos = pos[t];
    if (pos[t] < minpos) minpos = pos[t];
  }
  orc_kv kv;
  kv.k = k + (int64_t)g * D;
  kv.v = v + (int64_t)g * D;
  kv.stride = kv_stride;
  kv.D = D;
  kv.base = rope_base;
  kv.pos_offset = pos_offset;
  kv.rot_tab = NULL;
  kv.tab_lo = 0;
  kv.tab_hi = -1;

  /* RoPE'd keys for the span the rows can reach, when it fits in memory. */
  int64_t lo = is_retrieval ? 0 : ((minpos - window + 1) > 0 ? (minpos - window + 1) : 0);
  int64_t span = maxpos - lo + 1;
  double* tab = NULL;
  /* a retrieval head's few decode rows touch few keys: RoPE those on demand instead */
  int want_tab = !(is_retrieval && nrows < 32);
  if (want_tab && (double)span * D * 8.0 <= 1.6e9) {
    tab = (double*)malloc(sizeof(double) * (size_t)span * (size_t)D);
    if (tab) {
#pragma omp parallel for schedule(static) num_threads(n_threads)
      for (int64_t j = lo; j <= maxpos; ++j) {
        double x[512];
        for (int d = 0; d < D; ++d) x[d] = orc_bf16(kv.k[j * kv_stride + d]);
        orc_rope(x, (double)(j + pos_offset), D, rope_base, tab + (j - lo) * D);
      }
      kv.rot_tab = tab;
      kv.tab_lo = lo;
      kv.tab_hi = maxpos;
    }
  }

  /* Pre-RoPE 16-dim index keys for every causal position (retrieval heads). */
  double* kt = NULL;
  if (is_retrieval) {
    kt = (double*)malloc(sizeof(double) * (size_t)(maxpos + 1) * (size_t)r);
#pragma omp parallel for schedule(static) num_threads(n_threads)
    for (int64_t j = 0; j <= maxpos; ++j) {
      double x[512];
      for (int d = 0; d < D; ++d) x[d] = orc_bf16(kv.k[j * kv_stride + d]);
      orc_index_vec(x, wk, D, r, kt + j * r);
      if (key_bf16)
        for (int c = 0; c < r; ++c) kt[j * r + c] = orc_round_bf16(kt[j * r + c]);
    }
  }

#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t i = pos[t];
    double qv[512], qr[512];
    for (int d = 0; d < D; ++d) qv[d] = orc_bf16(q[t * q_stride + d]);
    orc_rope(qv, (double)(i + pos_offset), D, rope_base, qr);
    int64_t* J = NULL;
    int64_t nJ = 0;
    if (is_retrieval) {
      int64_t n = i + 1;
      double qt[64];
      orc_index_vec(qv, wq, D, r, qt);
      double* s = (double*)malloc(sizeof(double) * (size_t)n);
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int c = 0; c < r; ++c) acc += qt[c] * kt[j * r + c];
        s[j] = acc;
      }
      J = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
      double ms = 0, pt = 0, cp = 0;
      if (top_k > 0)
        nJ = orc_topk(s, n, top_k, J, pi_all ? pi_all + t * pi_stride : NULL, &ms, &pt, &cp);
      else
        nJ = orc_topp(s, n, top_p, J, pi_all ? pi_all + t * pi_stride : NULL, &ms, &pt, &cp);
      sel_mass[t] = ms;
      pi_t[t] = pt;
      cum_prev[t] = cp;
      free(s);
      qsort(J, (size_t)nJ, sizeof(int64_t), orc_cmp_i64);
    } else {
      J = (int64_t*)malloc(sizeof(int64_t) * (size_t)(window + n_sink + 1));
      /* sinks: j < S (and j <= i) */
      for (int64_t j = 0; j < n_sink && j <= i; ++j) J[nJ++] = j;
      /* window: i - j < W, skipping positions already taken as sinks */
      int64_t w0 = i - window + 1;
      if (w0 < n_sink) w0 = n_sink;
      for (int64_t j = w0; j <= i; ++j) J[nJ++] = j;
      sel_mass[t] = 1.0;
      pi_t[t] = 0.0;
      cum_prev[t] = 0.0;
    }
    sel_count[t] = nJ;
    if (sel_idx) {
      int64_t m = nJ < sel_cap ? nJ : sel_cap;
      for (int64_t a = 0; a < m; ++a) sel_idx[t * sel_cap + a] = J[a];
    }
    orc_attend(qr, &kv, J, nJ, sm_scale, out + t * D);
    free(J);
  }
  free(tab);
  free(kt);
  return 0;
}

/*
 * Exact attention of one query row (bf16 bits q, pre-RoPE, at absolute position pos) over a
 * given key set J: the final step of both head classes on its own, for comparing a result
 * whose set legitimately differs from the oracle's (a cut exactly at the mass boundary).
 */
void orc_attend_set(const uint16_t* k, const uint16_t* v, int64_t kv_stride, int g, int D,
                    const uint16_t* q, int64_t pos, double rope_base, double sm_scale,
                    int64_t pos_offset, const int64_t* J, int64_t nJ, double* out) {
  orc_kv kv;
  kv.k = k + (int64_t)g * D;
  kv.v = v + (int64_t)g * D;
  kv.stride = kv_stride;
  kv.D = D;
  kv.base = rope_base;
  kv.pos_offset = pos_offset;
  kv.rot_tab = NULL;
  kv.tab_lo = 0;
  kv.tab_hi = -1;
  double qv[512], qr[512];
  for (int d = 0; d < D; ++d) qv[d] = orc_bf16(q[d]);
  orc_rope(qv, (double)(pos + pos_offset), D, rope_base, qr);
  orc_attend(qr, &kv, J, nJ, sm_scale, out);
}

/* Index scores s_j = (Wq^T q).(Wk^T k_j) for j < n (pre-RoPE), fp64; with key_bf16 each
 * index-key component is first rounded to bf16 (the stored keys). */
void orc_index_scores(const uint16_t* k, int64_t n, int64_t kv_stride, int g, int D, int r,
                      const uint16_t* q, const float* wq, const float* wk, double* s, int key_bf16) {
  double qv[512], qt[64], x[512], kt[64];
  for (int d = 0; d < D; ++d) qv[d] = orc_bf16(q[d]);
  orc_index_vec(qv, wq, D, r, qt);
  for (int64_t j = 0; j < n; ++j) {
    const uint16_t* kr = k + j * kv_stride + (int64_t)g * D;
    for (int d = 0; d < D; ++d) x[d] = orc_bf16(kr[d]);
    orc_index_vec(x, wk, D, r, kt);
    if (key_bf16)
      for (int c = 0; c < r; ++c) kt[c] = orc_round_bf16(kt[c]);
    double acc = 0.0;
    for (int c = 0; c < r; ++c) acc += qt[c] * kt[c];
    s[j] = acc;
  }
}

/* ---------------------------------------------------------------- K-cache clustering
 *
 * The RTPurboV2 two-level funnel (aitntnews page, finding 3): the N cached tokens of a
 * retrieval head are grouped into K semantic clusters in the r = 16 index space, a query is
 * matched against the K cluster centres first, and exact attention then runs only over the
 * tokens of the clusters it hits.  The page fixes none of the steps; the readings taken here:
 *   - the clustered vectors are the stored bf16 index keys kt_j (the layer's bf16 option),
 *     put on the fixed-point grid 2^-27 (xq = rint(kt * 2^27)) so that centre sums are exact
 *     integers, whatever their order;
 *   - Lloyd's k-means: centres start at the keys j_k = floor((2k + 1) n / (2K)); each pass
 *     assigns every key to the centre of least squared distance (fp64, the 16 terms summed
 *     in dimension order with fused multiply-adds; ties to the lower centre), then moves every
 *     non-empty centre to the mean of its keys (integer sum / count * 2^-27); an empty
 *     cluster keeps its centre; a final assignment follows the last pass;
 *   - the coarse match: centre score c_k = qt . mu_k; a cluster weighs n_k exp(c_k - max c)
 *     (its key count times the softmax weight of its centre: the mass its keys would carry if
 *     they sat at the centre); clusters ordered by (c_k desc, k asc), the shortest prefix whose
 *     weight reaches p of the total is hit (p >= 1: every non-empty cluster);
 *   - keys cached after the clustering are always kept; the fine step is exact attention over
 *     the hit clusters' keys and those. */

#define ORC_CL_SCALE 134217728.0 /* 2^27 */

/* kt_j = Wk^T k_j for j < n, each component rounded to bf16 (the stored keys). */
void orc_index_keys_bf16(const uint16_t* k, int64_t n, int64_t kv_stride, int g, int D, int r,
                         const float* wk, double* kt) {
  double x[512];
  for (int64_t j = 0; j < n; ++j) {
    const uint16_t* kr = k + j * kv_stride + (int64_t)g * D;
    for (int d = 0; d < D; ++d) x[d] = orc_bf16(kr[d]);
    orc_index_vec(x, wk, D, r, kt + j * r);
    for (int c = 0; c < r; ++c) kt[j * r + c] = orc_round_bf16(kt[j * r + c]);
  }
}

static double orc_sqdist(const double* x, const double* mu, int r) {
  double acc = 0.0;
  for (int c = 0; c < r; ++c) {
    const double d = x[c] - mu[c];
    acc = fma(d, d, acc);
  }
  return acc;
}

/* qt = Wq^T q for one bf16 query (the index query, fp64). */
void orc_index_query(const uint16_t* q, int D, int r, const float* wq, double* qt) {
  double qv[512];
  for (int d = 0; d < D; ++d) qv[d] = orc_bf16(q[d]);
  orc_index_vec(qv, wq, D, r, qt);
}

/* Lloyd's k-means of the n keys kt[n][r] into K clusters (K <= n) with `iters` passes.
 * cent[K][r] receives the centres, counts[K] the cluster sizes and assign[n] each key's
 * cluster, all after the final assignment. */
void orc_kmeans(const double* kt, int64_t n, int r, int K, int iters, double* cent, int64_t* counts,
                int32_t* assign) {
  double* xq = (double*)malloc(sizeof(double) * (size_t)n * (size_t)r);
  int64_t* qi = (int64_t*)malloc(sizeof(int64_t) * (size_t)n * (size_t)r);
  int64_t* sums = (int64_t*)malloc(sizeof(int64_t) * (size_t)K * (size_t)r);
  for (int64_t i = 0; i < n * r; ++i) {
    qi[i] = (int64_t)rint(kt[i] * ORC_CL_SCALE);
    xq[i] = (double)qi[i] / ORC_CL_SCALE;
  }
  for (int k = 0; k < K; ++k) {
    const int64_t j = ((int64_t)(2 * k + 1) * n) / (2 * (int64_t)K);
    for (int c = 0; c < r; ++c) cent[(int64_t)k * r + c] = xq[j * r + c];
  }
  for (int it = 0; it <= iters; ++it) {
    for (int64_t j = 0; j < n; ++j) {
      int best = 0;
      double bd = orc_sqdist(xq + j * r, cent, r);
      for (int k = 1; k < K; ++k) {
        const double d = orc_sqdist(xq + j * r, cent + (int64_t)k * r, r);
        if (d < bd) {
          bd = d;
          best = k;
        }
      }
      assign[j] = best;
    }
    for (int k = 0; k < K; ++k) counts[k] = 0;
    for (int64_t i = 0; i < (int64_t)K * r; ++i) sums[i] = 0;
    for (int64_t j = 0; j < n; ++j) {
      counts[assign[j]] += 1;
      for (int c = 0; c < r; ++c) sums[(int64_t)assign[j] * r + c] += qi[j * r + c];
    }
    if (it == iters) break; /* the final assignment: centres stay */
    for (int k = 0; k < K; ++k)
      if (counts[k] > 0)
        for (int c = 0; c < r; ++c)
          cent[(int64_t)k * r + c] = (double)sums[(int64_t)k * r + c] / (double)counts[k] / ORC_CL_SCALE;
  }
  free(xq);
  free(qi);
  free(sums);
}

typedef struct {
  double c;
  int k;
} orc_cl;

static int orc_cmp_cl(const void* a, const void* b) {
  const orc_cl* x = (const orc_cl*)a;
  const orc_cl* y = (const orc_cl*)b;
  if (x->c > y->c) return -1;
  if (x->c < y->c) return 1;
  return x->k - y->k;
}

/* The coarse match of one index query qt[r] against K centres: hit[k] = 1 for the clusters
 * taken.  w[k] (optional) receives each cluster's weight fraction; returns the number hit and
 * *w_t the weight fraction of the last cluster taken. */
int orc_cluster_select(const double* qt, const double* cent, const int64_t* counts, int K, int r, double p,
                       int32_t* hit, double* w, double* w_t) {
  orc_cl* o = (orc_cl*)malloc(sizeof(orc_cl) * (size_t)K);
  int m = 0;
  double cmax = -INFINITY;
  for (int k = 0; k < K; ++k) {
    hit[k] = 0;
    if (w) w[k] = 0.0;
    if (counts[k] <= 0) continue;
    double acc = 0.0;
    for (int c = 0; c < r; ++c) acc += qt[c] * cent[(int64_t)k * r + c];
    o[m].c = acc;
    o[m].k = k;
    if (acc > cmax) cmax = acc;
    ++m;
  }
  double tot = 0.0;
  for (int i = 0; i < m; ++i) tot += (double)counts[o[i].k] * exp(o[i].c - cmax);
  qsort(o, (size_t)m, sizeof(orc_cl), orc_cmp_cl);
  double cum = 0.0, last = 0.0;
  int taken = 0;
  for (int i = 0; i < m; ++i) {
    const double f = (double)counts[o[i].k] * exp(o[i].c - cmax) / tot;
    if (w) w[o[i].k] = f;
    if (taken == i && (p >= 1.0 || cum < p)) {
      hit[o[i].k] = 1;
      cum += f;
      last = f;
      taken = i + 1;
    }
  }
  if (w_t) *w_t = last;
  free(o);
  return taken;
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
