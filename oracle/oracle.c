/*
 * Plain fp64 CPU oracle of the routed atomic-expert branch of an OmniMoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the test suite, the graft smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code with the CUDA library.
 *
 * Every quantity is computed in double precision from the exact values of the
 * stored inputs (fp32, or bf16 widened exactly).  Loops follow the order in
 * which the method is described; OpenMP is used only over iterations that are
 * independent (tokens, tasks, output columns), so the result does not depend
 * on the thread count.
 *
 * Sources (web pages about OmniMoE, cited by title and section):
 *  [NL 2.1]  "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at
 *            Scale" (gist.science, Dutch), Technisch Overzicht, section 2.1
 *            "Kerncomponenten van de Architectuur": an atomic expert is a
 *            vector pair (w_in, w_out) computing E_i(x) = sigma(x w_in^T) w_out;
 *            all N experts live in two global matrices W, V.
 *  [NL 2.2]  same page, section 2.2 "Algoritmische Innovaties": the Cartesian
 *            Product Router splits the expert index space into an Nr x Nc grid
 *            and scores experts from row and column logits; Expert-Centric
 *            Scheduling flattens the routing decisions into tasks, groups them
 *            by expert and sorts by token inside each group.
 *  [MS router]  OmniMoE explainer (omnimoeexpl, manus.space), Cartesian
 *            product router section: experts are grid coordinates (i, j);
 *            p(i,j|x) ~ pr(i|x) pc(j|x), so in log space S_ij = pr[i] + pc[j]
 *            and no N-wide score vector is needed; at N = 16K the router costs
 *            1.56% of a flat router.
 *  [MS sched]  same page, Expert-Centric Scheduling steps: flatten all
 *            (token, expert, weight) triples into M = L*K tasks; collect the
 *            unique active experts, sort them by id and cut every B into a
 *            group; sort tasks by group id (primary) then token id
 *            (secondary); each group loads its expert parameters once.  Memory
 *            traffic: token-centric D = 2d*L*K, expert-centric D = 2d*|E_active|.
 *
 * Readings where the pages are silent (each also listed with the design notes):
 *  - expert id of grid cell (i, j) is e = i*Nc + j;
 *  - the per-axis "distributions" are log-softmax of the axis logits;
 *  - top-k per axis, then the k x k joint scores, then top-K of those, then
 *    the gate is the softmax of the K selected joint scores;
 *  - sigma is the scalar SiLU, z / (1 + exp(-z));
 *  - every ordering breaks ties by the smaller index/id; the K outputs of a
 *    token are ordered by (score desc, id asc);
 *  - inside a (group, token) the tasks are ordered by expert id.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int64_t L, d, Nr, Nc, k, K, B;
  int32_t dtype; /* 0 = fp32 storage, 1 = bf16 storage (uint16 bits) */
  int32_t pad;
} or_dims;

/* Exact value of element i of a stored fp32 or bf16 array. */
static double elem(const void* p, int32_t dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)p)[i];
  uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Widen one stored row of length d to double. */
static void load_row(const void* base, int32_t dtype, int64_t row, int64_t d, double* out) {
  for (int64_t m = 0; m < d; ++m) out[m] = elem(base, dtype, row * d + m);
}

static double dot(const double* a, const double* b, int64_t n) {
  double s = 0.0;
  for (int64_t m = 0; m < n; ++m) s += a[m] * b[m];
  return s;
}

/* sigma of an atomic expert: scalar SiLU [NL 2.1] (SwiGLU named, one vector pair given). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------------- */
/* Router                                                                    */
/* ------------------------------------------------------------------------- */

/* Axis logits of one token: z[i] = x[t] . Wa[i] + bias[i]   [NL 2.2] */
static void axis_logits(const void* x, const void* Wa, const float* bias, int32_t dtype,
                        int64_t t, int64_t d, int64_t n_axis, double* xrow, double* wrow,
                        double* z) {
  load_row(x, dtype, t, d, xrow);
  for (int64_t i = 0; i < n_axis; ++i) {
    load_row(Wa, dtype, i, d, wrow);
    z[i] = dot(xrow, wrow, d) + (bias ? (double)bias[i] : 0.0);
  }
}

/* log-softmax in place: z[i] - log(sum_j exp(z[j])), max-shifted. */
static void log_softmax(double* z, int64_t n) {
  double mx = z[0];
  for (int64_t i = 1; i < n; ++i)
    if (z[i] > mx) mx = z[i];
  double s = 0.0;
  for (int64_t i = 0; i < n; ++i) s += exp(z[i] - mx);
  double lse = mx + log(s);
  for (int64_t i = 0; i < n; ++i) z[i] -= lse;
}

/* Row-wise log-softmax of rows x n logits, in place (for callers that start
 * from their own axis logits). */
int oracle_log_softmax(double* z, int64_t rows, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) log_softmax(z + r * n, n);
  return 0;
}

typedef struct {
  double v;
  int64_t id;
} scored;

/* order: larger value first, then smaller id */
static int cmp_scored(const void* pa, const void* pb) {
  const scored* a = (const scored*)pa;
  const scored* b = (const scored*)pb;
  if (a->v > b->v) return -1;
  if (a->v < b->v) return 1;
  return (a->id < b->id) ? -1 : (a->id > b->id);
}

/* top-k of one axis: ids and values, ordered by (value desc, id asc) */
static void axis_topk(const double* lz, int64_t n, int64_t k, scored* tmp, int64_t* ids,
                      double* vals) {
  for (int64_t i = 0; i < n; ++i) {
    tmp[i].v = lz[i];
    tmp[i].id = i;
  }
  qsort(tmp, (size_t)n, sizeof(scored), cmp_scored);
  for (int64_t a = 0; a < k; ++a) {
    ids[a] = tmp[a].id;
    vals[a] = tmp[a].v;
  }
}

/* Raw axis logits of the listed tokens: zr [nt x Nr], zc [nt x Nc]  [NL 2.2] */
int oracle_axis_logits(const or_dims* D, const void* x, const void* Wr, const void* Wc,
                       const float* bias_r, const float* bias_c, const int64_t* tok, int64_t nt,
                       double* zr, double* zc) {
  const int64_t d = D->d, Nr = D->Nr, Nc = D->Nc;
#pragma omp parallel
  {
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* wrow = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nt; ++r) {
      axis_logits(x, Wr, bias_r, D->dtype, tok[r], d, Nr, xrow, wrow, zr + r * Nr);
      axis_logits(x, Wc, bias_c, D->dtype, tok[r], d, Nc, xrow, wrow, zc + r * Nc);
    }
    free(xrow);
    free(wrow);
  }
  return 0;
}

/* Per-axis log-softmax logits of the listed tokens: lr [nt x Nr], lc [nt x Nc]. */
int oracle_axis_logprobs(const or_dims* D, const void* x, const void* Wr, const void* Wc,
                         const float* bias_r, const float* bias_c, const int64_t* tok,
                         int64_t nt, double* lr, double* lc) {
  const int64_t d = D->d, Nr = D->Nr, Nc = D->Nc;
#pragma omp parallel
  {
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* wrow = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nt; ++r) {
      axis_logits(x, Wr, bias_r, D->dtype, tok[r], d, Nr, xrow, wrow, lr + r * Nr);
      axis_logits(x, Wc, bias_c, D->dtype, tok[r], d, Nc, xrow, wrow, lc + r * Nc);
      log_softmax(lr + r * Nr, Nr);
      log_softmax(lc + r * Nc, Nc);
    }
    free(xrow);
    free(wrow);
  }
  return 0;
}

/*
 * Selection from per-axis log-probabilities (the Cartesian Product Router
 * after its two projections) [NL 2.2], [MS router]:
 *   R = top-k rows of lr, C = top-k columns of lc;
 *   joint score of every (i, j) in R x C: S = lr[i] + lc[j], id e = i*Nc + j;
 *   the K best by (S desc, e asc);
 *   gate = softmax of those K joint scores.
 * No N-wide score vector is formed.
 */
int oracle_select(const or_dims* D, const double* lr, const double* lc, int64_t nt,
                  int32_t* idx, double* gate, double* score) {
  const int64_t Nr = D->Nr, Nc = D->Nc, k = D->k, K = D->K;
  if (k > Nr || k > Nc || K > k * k || K < 1) return 1;
#pragma omp parallel
  {
    int64_t nmax = Nr > Nc ? Nr : Nc;
    scored* tmp = (scored*)malloc(sizeof(scored) * (nmax > k * k ? nmax : k * k));
    int64_t* ri = (int64_t*)malloc(sizeof(int64_t) * k);
    int64_t* ci = (int64_t*)malloc(sizeof(int64_t) * k);
    double* rv = (double*)malloc(sizeof(double) * k);
    double* cv = (double*)malloc(sizeof(double) * k);
#pragma omp for schedule(dynamic, 8)
    for (int64_t r = 0; r < nt; ++r) {
      axis_topk(lr + r * Nr, Nr, k, tmp, ri, rv);
      axis_topk(lc + r * Nc, Nc, k, tmp, ci, cv);
      int64_t c = 0;
      for (int64_t a = 0; a < k; ++a)
        for (int64_t b = 0; b < k; ++b) {
          tmp[c].v = rv[a] + cv[b];
          tmp[c].id = ri[a] * Nc + ci[b];
          ++c;
        }
      qsort(tmp, (size_t)c, sizeof(scored), cmp_scored);
      double mx = tmp[0].v, s = 0.0;
      for (int64_t q = 0; q < K; ++q) s += exp(tmp[q].v - mx);
      for (int64_t q = 0; q < K; ++q) {
        idx[r * K + q] = (int32_t)tmp[q].id;
        score[r * K + q] = tmp[q].v;
        gate[r * K + q] = exp(tmp[q].v - mx) / s;
      }
    }
    free(tmp);
    free(ri);
    free(ci);
    free(rv);
    free(cv);
  }
  return 0;
}

/*
 * Brute force over the full N-way product: every expert e = i*Nc + j gets
 * S[e] = lr[i] + lc[j]; the K best by (S desc, e asc), their softmax gate,
 * and the (K+1)-th best score (-inf when K = N), used to flag near-ties.
 * This is the flat scoring the router avoids; it serves only as a check.
 */
int oracle_select_bruteforce(const or_dims* D, const double* lr, const double* lc, int64_t nt,
                             int32_t* idx, double* gate, double* score, double* next) {
  const int64_t Nr = D->Nr, Nc = D->Nc, K = D->K, N = Nr * Nc;
  if (K < 1 || K > N) return 1;
  const int64_t keep = (K < N) ? K + 1 : K;
#pragma omp parallel
  {
    scored* best = (scored*)malloc(sizeof(scored) * (keep + 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nt; ++r) {
      int64_t nb = 0; /* best[0..nb) kept sorted by cmp_scored */
      for (int64_t e = 0; e < N; ++e) {
        scored s;
        s.v = lr[r * Nr + e / Nc] + lc[r * Nc + e % Nc];
        s.id = e;
        if (nb == keep && cmp_scored(&s, &best[nb - 1]) >= 0) continue;
        int64_t p = (nb < keep) ? nb++ : nb - 1;
        while (p > 0 && cmp_scored(&s, &best[p - 1]) < 0) {
          best[p] = best[p - 1];
          --p;
        }
        best[p] = s;
      }
      double mx = best[0].v, sum = 0.0;
      for (int64_t q = 0; q < K; ++q) sum += exp(best[q].v - mx);
      for (int64_t q = 0; q < K; ++q) {
        idx[r * K + q] = (int32_t)best[q].id;
        score[r * K + q] = best[q].v;
        gate[r * K + q] = exp(best[q].v - mx) / sum;
      }
      next[r] = (K < N) ? best[K].v : -INFINITY;
    }
    free(best);
  }
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Expert-Centric Scheduling [NL 2.2], [MS sched]                            */
/* ------------------------------------------------------------------------- */

typedef struct {
  int64_t g, t, e;
  double gate;
} task;

static int cmp_task(const void* pa, const void* pb) {
  const task* a = (const task*)pa;
  const task* b = (const task*)pb;
  if (a->g != b->g) return (a->g < b->g) ? -1 : 1;
  if (a->t != b->t) return (a->t < b->t) ? -1 : 1;
  return (a->e < b->e) ? -1 : (a->e > b->e);
}

/*
 * Tasks are the (token, expert, gate) triples of the listed tokens (row r of
 * idx/gate belongs to token tok[r]).  U = sorted unique experts; the group of
 * expert e is (position of e in U) / B; tasks are sorted by (group, token,
 * expert).  group_off[g] is the first task of group g, group_off[G] = M.
 * Outputs are sized by the caller: M = nt*K tasks, uniq[min(N, M)],
 * group_off[ceil(min(N,M)/B) + 1].
 */
int oracle_schedule(const or_dims* D, const int64_t* tok, int64_t nt, const int32_t* idx,
                    const double* gate, int32_t* task_token, int32_t* task_expert,
                    double* task_gate, int32_t* uniq, int32_t* group_off, int64_t* n_active,
                    int64_t* n_groups) {
  const int64_t N = D->Nr * D->Nc, K = D->K, B = D->B, M = nt * K;
  if (B < 1) return 1;
  /* step 1: collect the unique active experts, sorted by id */
  unsigned char* active = (unsigned char*)calloc((size_t)N, 1);
  for (int64_t q = 0; q < M; ++q) {
    if (idx[q] < 0 || idx[q] >= N) {
      free(active);
      return 2;
    }
    active[idx[q]] = 1;
  }
  int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * N);
  int64_t nu = 0;
  for (int64_t e = 0; e < N; ++e) {
    pos[e] = -1;
    if (active[e]) {
      uniq[nu] = (int32_t)e;
      pos[e] = nu++;
    }
  }
  /* step 2: every B of them form a group */
  const int64_t G = (nu + B - 1) / B;
  /* step 3: flatten into tasks and sort by (group, token, expert) */
  task* ts = (task*)malloc(sizeof(task) * (M > 0 ? M : 1));
  for (int64_t r = 0; r < nt; ++r)
    for (int64_t q = 0; q < K; ++q) {
      task* p = &ts[r * K + q];
      p->e = idx[r * K + q];
      p->t = tok[r];
      p->g = pos[p->e] / B;
      p->gate = gate[r * K + q];
    }
  qsort(ts, (size_t)M, sizeof(task), cmp_task);
  for (int64_t q = 0; q < M; ++q) {
    task_token[q] = (int32_t)ts[q].t;
    task_expert[q] = (int32_t)ts[q].e;
    task_gate[q] = ts[q].gate;
  }
  /* step 4: group boundaries */
  int64_t q = 0;
  for (int64_t g = 0; g < G; ++g) {
    while (q < M && ts[q].g < g) ++q;
    group_off[g] = (int32_t)q;
  }
  group_off[G] = (int32_t)M;
  *n_active = nu;
  *n_groups = G;
  free(ts);
  free(pos);
  free(active);
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Execution                                                                 */
/* ------------------------------------------------------------------------- */

/* local slot of expert e among uniq[u0 .. u0+nb) (sorted): binary search */
static int64_t slot_of(const int32_t* uniq, int64_t u0, int64_t nb, int32_t e) {
  int64_t lo = 0, hi = nb - 1;
  while (lo < hi) {
    int64_t mid = (lo + hi) / 2;
    if (uniq[u0 + mid] < e)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

/*
 * Expert-centric order [MS sched]: group by group, the rows W[e], V[e] of the
 * group's experts uniq[g*B .. min((g+1)*B, n_active)) are loaded once; then
 * every task (t, e, gate) of the group, in (token, expert) order, adds
 * gate * h * V[e] to y[t]   [NL 2.1], [NL 2.2], with h = SiLU(x[t] . W[e]).
 * With U != NULL the expert is gated (SwiGLU, named by the OmniMoE explainer's
 * Atomic Expert section; the pages give only the pair (w_in, w_out), and the
 * gated form taken here adds a third global matrix U [N x d]):
 * h = SiLU(x[t] . W[e]) * (x[t] . U[e]).
 * y rows are indexed by out_row[t] (the caller's row of token t).
 * rows_loaded[0] / [1] count rows of W / V brought in (|E_active| each).
 *
 * The work is split in two loops over the same groups: first the scalar
 * c = gate * SiLU(x[t] . W[e]) of every task (groups are independent), then
 * the accumulation y[t] += c * V[e] (output columns split across threads, so
 * each y element receives its terms in the single-threaded order).
 */
int oracle_forward_expert(const or_dims* D, const void* x, const void* W, const void* U,
                          const void* V, const int32_t* task_token, const int32_t* task_expert,
                          const double* task_gate, const int32_t* uniq,
                          const int32_t* group_off, int64_t n_active, int64_t n_groups,
                          const int64_t* out_row, double* y, int64_t y_rows,
                          int64_t* rows_loaded) {
  const int64_t d = D->d, B = D->B;
  const int64_t M = n_groups > 0 ? group_off[n_groups] : 0;
  memset(y, 0, sizeof(double) * y_rows * d);
  double* c = (double*)malloc(sizeof(double) * (M > 0 ? M : 1));
  int64_t wloaded = 0, vloaded = 0;
#pragma omp parallel reduction(+ : wloaded)
  {
    double* wg = (double*)malloc(sizeof(double) * B * d);
    double* ug = (double*)malloc(sizeof(double) * B * d);
    double* xrow = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t g = 0; g < n_groups; ++g) {
      const int64_t u0 = g * B, nb = (n_active - u0 < B) ? n_active - u0 : B;
      for (int64_t j = 0; j < nb; ++j) load_row(W, D->dtype, uniq[u0 + j], d, wg + j * d);
      if (U)
        for (int64_t j = 0; j < nb; ++j) load_row(U, D->dtype, uniq[u0 + j], d, ug + j * d);
      wloaded += nb;
      for (int64_t q = group_off[g]; q < group_off[g + 1]; ++q) {
        const int64_t j = slot_of(uniq, u0, nb, task_expert[q]);
        load_row(x, D->dtype, task_token[q], d, xrow);
        c[q] = task_gate[q] * silu(dot(xrow, wg + j * d, d));
        if (U) c[q] *= dot(xrow, ug + j * d, d);
      }
    }
    free(wg);
    free(ug);
    free(xrow);
  }
  int nth_used = 1;
#pragma omp parallel reduction(+ : vloaded)
  {
    int tid = 0, nth = 1;
#ifdef _OPENMP
    tid = omp_get_thread_num();
    nth = omp_get_num_threads();
#endif
    const int64_t c0 = d * tid / nth, c1 = d * (tid + 1) / nth, w = c1 - c0;
    double* vg = (double*)malloc(sizeof(double) * B * (w > 0 ? w : 1));
    for (int64_t g = 0; g < n_groups; ++g) {
      const int64_t u0 = g * B, nb = (n_active - u0 < B) ? n_active - u0 : B;
      for (int64_t j = 0; j < nb; ++j)
        for (int64_t m = c0; m < c1; ++m)
          vg[j * w + (m - c0)] = elem(V, D->dtype, (int64_t)uniq[u0 + j] * d + m);
      if (tid == 0) vloaded += nb; /* every thread loads a slice of the same rows */
      for (int64_t q = group_off[g]; q < group_off[g + 1]; ++q) {
        const int64_t j = slot_of(uniq, u0, nb, task_expert[q]);
        double* yr = y + out_row[task_token[q]] * d;
        for (int64_t m = c0; m < c1; ++m) yr[m] += c[q] * vg[j * w + (m - c0)];
      }
    }
    if (tid == 0) nth_used = nth;
    free(vg);
  }
  (void)nth_used;
  rows_loaded[0] = wloaded;
  rows_loaded[1] = vloaded;
  free(c);
  return 0;
}

/*
 * Token-centric order (the execution the scheduling replaces) [NL 2.2],
 * [MS sched]: every token fetches the rows of each of its K experts itself,
 * y[t] = sum_k gate[t,k] * SiLU(x[t] . W[e_k]) * V[e_k], times
 * (x[t] . U[e_k]) for the gated expert (U != NULL, as oracle_forward_expert).
 * Row r of idx/gate belongs to token tok[r]; y row r is written.
 * rows_loaded[0] / [1] count rows of W / V fetched (L*K each).
 */
int oracle_forward_token(const or_dims* D, const void* x, const void* W, const void* U,
                         const void* V,
                         const int64_t* tok, int64_t nt, const int32_t* idx, const double* gate,
                         double* y, int64_t* rows_loaded) {
  const int64_t d = D->d, K = D->K;
  int64_t fetched = 0;
#pragma omp parallel reduction(+ : fetched)
  {
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* wrow = (double*)malloc(sizeof(double) * d);
    double* vrow = (double*)malloc(sizeof(double) * d);
    double* urow = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nt; ++r) {
      double* yr = y + r * d;
      for (int64_t m = 0; m < d; ++m) yr[m] = 0.0;
      load_row(x, D->dtype, tok[r], d, xrow);
      for (int64_t q = 0; q < K; ++q) {
        const int64_t e = idx[r * K + q];
        load_row(W, D->dtype, e, d, wrow);
        load_row(V, D->dtype, e, d, vrow);
        fetched += 1;
        double cq = gate[r * K + q] * silu(dot(xrow, wrow, d));
        if (U) {
          load_row(U, D->dtype, e, d, urow);
          cq *= dot(xrow, urow, d);
        }
        for (int64_t m = 0; m < d; ++m) yr[m] += cq * vrow[m];
      }
    }
    free(xrow);
    free(wrow);
    free(vrow);
    free(urow);
  }
  rows_loaded[0] = fetched;
  rows_loaded[1] = fetched;
  return 0;
}

/*
 * Shared dense MLP branch [NL 2.1]: an always-on dense MLP beside the routed
 * experts, y = MLP(x) + routed(x) (the explainer's ablation table removes it
 * as "w/o shared MLP").  The pages give neither its width nor its
 * activation; the reading taken is one hidden layer of F units with the same
 * scalar SiLU as the atomic experts:
 *   h[f] = SiLU(x[t] . W1[f]),  f < F;   mlp[t, j] = h . W2[j],  j < d,
 * with W1 [F x d] and W2 [d x F] in the storage type (row j of W2 holds the
 * F weights of output j).  Row r of y (fp64, d values) is token tok[r].
 */
int oracle_shared_mlp(const or_dims* D, int64_t F, const void* x, const void* W1, const void* W2,
                      const int64_t* tok, int64_t nt, double* y) {
  const int64_t d = D->d;
  if (F < 1) return 1;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * d);
    double* h = (double*)malloc(sizeof(double) * F);
    double* w1 = (double*)malloc(sizeof(double) * d);
    double* w2 = (double*)malloc(sizeof(double) * F);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nt; ++r) {
      load_row(x, D->dtype, tok[r], d, xt);
      for (int64_t f = 0; f < F; ++f) {
        load_row(W1, D->dtype, f, d, w1);
        h[f] = silu(dot(xt, w1, d));
      }
      for (int64_t j = 0; j < d; ++j) {
        load_row(W2, D->dtype, j, F, w2);
        y[r * d + j] = dot(h, w2, F);
      }
    }
    free(xt);
    free(h);
    free(w1);
    free(w2);
  }
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Backward of the routed branch                                             */
/* ------------------------------------------------------------------------- */

/* d SiLU / dz = sig(z) * (1 + z * (1 - sig(z))), sig the logistic function. */
static double silu_grad(double z) {
  const double sg = 1.0 / (1.0 + exp(-z));
  return sg * (1.0 + z * (1.0 - sg));
}

/*
 * Gradients of the routed branch (the pages train the model [NL 4]; this is
 * the forward differentiated by the chain rule).  With the forward's routing
 * fixed (idx: the K experts chosen for each token, gate: the softmax of their
 * joint scores) and the loss l = sum over t of dy[t] . y[t]:
 *
 *   forward, per token t and selected expert e_k = idx[t,k] (i_k = e_k / Nc,
 *   j_k = e_k % Nc):
 *     zr = x[t] . Wr^T + br,  zc = x[t] . Wc^T + bc          [NL 2.2]
 *     lr = zr - LSE(zr),      lc = zc - LSE(zc)              (per-axis log-softmax)
 *     S_k = lr[i_k] + lc[j_k],  gate_k = exp(S_k) / sum_q exp(S_q)
 *     a_k = x[t] . W[e_k],  h_k = SiLU(a_k),  y[t] = sum_k gate_k h_k V[e_k]
 *
 *   backward, in the reverse order:
 *     s_k = dy[t] . V[e_k]
 *     dV[e_k]  += gate_k h_k dy[t]
 *     dgate_k   = h_k s_k
 *     da_k      = gate_k s_k SiLU'(a_k)
 *     dW[e_k]  += da_k x[t],   dx[t] += da_k W[e_k]
 *     dS_k      = gate_k (dgate_k - sum_q gate_q dgate_q)     (softmax)
 *     dlr[i_k] += dS_k,        dlc[j_k] += dS_k
 *     dzr = dlr - softmax(zr) sum_i dlr[i]                     (log-softmax; same for c)
 *     dWr[i] += dzr[i] x[t],   dbr[i] += dzr[i],   dx[t] += dzr[i] Wr[i]   (same for c)
 *
 * The choice of the top-k rows, columns and pairs is piecewise constant in
 * the inputs: no gradient flows through it.
 * Row r of idx/gate/dy/dx belongs to token tok[r].  dx [nt x d] is
 * overwritten; dW, dV [N x d], dWr [Nr x d], dWc [Nc x d], dbr [Nr], dbc [Nc]
 * are added to.  Parameter gradients are summed token by token in order
 * (each output column by one thread), so they do not depend on the thread
 * count.
 */
int oracle_backward(const or_dims* D, const void* x, const void* Wr, const void* Wc,
                    const float* br, const float* bc, const void* W, const void* V,
                    const int64_t* tok, int64_t nt, const int32_t* idx, const double* gate,
                    const double* dy, double* dx, double* dW, double* dV, double* dWr,
                    double* dWc, double* dbr, double* dbc) {
  const int64_t d = D->d, K = D->K, Nr = D->Nr, Nc = D->Nc;
  const int64_t M = nt * K;
  double* h = (double*)malloc(sizeof(double) * (size_t)M);
  double* da = (double*)malloc(sizeof(double) * (size_t)M);
  double* dzr = (double*)calloc((size_t)(nt * Nr), sizeof(double));
  double* dzc = (double*)calloc((size_t)(nt * Nc), sizeof(double));
  if (!h || !da || !dzr || !dzc) {
    free(h); free(da); free(dzr); free(dzc);
    return 1;
  }
  /* per token: the scalars of its tasks, the logit gradients, dx */
#pragma omp parallel
  {
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* wrow = (double*)malloc(sizeof(double) * d);
    double* vrow = (double*)malloc(sizeof(double) * d);
    double* zr = (double*)malloc(sizeof(double) * Nr);
    double* zc = (double*)malloc(sizeof(double) * Nc);
    double* dg = (double*)malloc(sizeof(double) * K);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nt; ++r) {
      const int64_t t = tok[r];
      const double* dyr = dy + r * d;
      double* dxr = dx + r * d;
      for (int64_t m = 0; m < d; ++m) dxr[m] = 0.0;
      load_row(x, D->dtype, t, d, xrow);
      /* experts */
      for (int64_t q = 0; q < K; ++q) {
        const int64_t e = idx[r * K + q];
        load_row(V, D->dtype, e, d, vrow);
        load_row(W, D->dtype, e, d, wrow);
        const double sk = dot(dyr, vrow, d);
        const double a = dot(xrow, wrow, d);
        h[r * K + q] = silu(a);
        dg[q] = h[r * K + q] * sk;
        da[r * K + q] = gate[r * K + q] * sk * silu_grad(a);
        for (int64_t m = 0; m < d; ++m) dxr[m] += da[r * K + q] * wrow[m];
      }
      /* gate = softmax of the selected joint scores */
      double gdg = 0.0;
      for (int64_t q = 0; q < K; ++q) gdg += gate[r * K + q] * dg[q];
      double* dlr = dzr + r * Nr;
      double* dlc = dzc + r * Nc;
      for (int64_t q = 0; q < K; ++q) {
        const int64_t e = idx[r * K + q];
        const double dS = gate[r * K + q] * (dg[q] - gdg);
        dlr[e / Nc] += dS;
        dlc[e % Nc] += dS;
      }
      /* per-axis log-softmax, then the projections */
      axis_logits(x, Wr, br, D->dtype, t, d, Nr, xrow, wrow, zr);
      axis_logits(x, Wc, bc, D->dtype, t, d, Nc, xrow, wrow, zc);
      log_softmax(zr, Nr);
      log_softmax(zc, Nc);
      double sr = 0.0, sc = 0.0;
      for (int64_t i = 0; i < Nr; ++i) sr += dlr[i];
      for (int64_t j = 0; j < Nc; ++j) sc += dlc[j];
      for (int64_t i = 0; i < Nr; ++i) dlr[i] -= exp(zr[i]) * sr;
      for (int64_t j = 0; j < Nc; ++j) dlc[j] -= exp(zc[j]) * sc;
      load_row(x, D->dtype, t, d, xrow);
      for (int64_t i = 0; i < Nr; ++i) {
        load_row(Wr, D->dtype, i, d, wrow);
        for (int64_t m = 0; m < d; ++m) dxr[m] += dlr[i] * wrow[m];
      }
      for (int64_t j = 0; j < Nc; ++j) {
        load_row(Wc, D->dtype, j, d, wrow);
        for (int64_t m = 0; m < d; ++m) dxr[m] += dlc[j] * wrow[m];
      }
    }
    free(xrow); free(wrow); free(vrow); free(zr); free(zc); free(dg);
  }
  /* parameter gradients, token by token in order; one thread per column */
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < d; ++m) {
    for (int64_t r = 0; r < nt; ++r) {
      const double xm = elem(x, D->dtype, tok[r] * d + m);
      const double dym = dy[r * d + m];
      for (int64_t q = 0; q < K; ++q) {
        const int64_t e = idx[r * K + q];
        dV[e * d + m] += gate[r * K + q] * h[r * K + q] * dym;
        dW[e * d + m] += da[r * K + q] * xm;
      }
      for (int64_t i = 0; i < Nr; ++i) dWr[i * d + m] += dzr[r * Nr + i] * xm;
      for (int64_t j = 0; j < Nc; ++j) dWc[j * d + m] += dzc[r * Nc + j] * xm;
    }
  }
  for (int64_t r = 0; r < nt; ++r) {
    if (dbr)
      for (int64_t i = 0; i < Nr; ++i) dbr[i] += dzr[r * Nr + i];
    if (dbc)
      for (int64_t j = 0; j < Nc; ++j) dbc[j] += dzc[r * Nc + j];
  }
  free(h); free(da); free(dzr); free(dzc);
  return 0;
}

/* Threads an OpenMP region of this library uses (for reporting). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Sets the threads of later OpenMP regions (n >= 1); timing only, the results
   do not depend on it. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
