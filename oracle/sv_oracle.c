/*
 * sv_oracle.c -- float64 CPU oracle for batched speculative-sampling verification.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header, table or constant with that path.
 *
 * Every quantity is computed the plain way, in float64, one request or row at
 * a time, with sequential sums in vocabulary order.  bf16 and fp32 inputs are
 * widened to float64 exactly.  Nothing is blocked, fused or reordered.
 *
 * Sources (the pages these functions restate):
 *  [SD]   "基于推测性解码的强化学习训练" (ReSpec blog, beipo.top), section
 *         "推测解码 Speculative Decoding（SD）": draft k tokens, one target
 *         forward, compare target and draft logits, resample the first bad
 *         token, else sample one more token from the target.
 *  [ACC]  "ReSpec: Towards Optimizing Speculative Decoding in Reinforcement
 *         Learning Systems" (reading notes), section 2 "背景速查", "SD
 *         acceptance test (one-shot)": accept with min(1, p/q); on rejection
 *         resample from r(x) = max(0, p-q) / sum max(0, p-q); the marginal is
 *         the target's (Leviathan et al. 2023).  The equation body itself was
 *         lost from the page; min(1, p(x)/q(x)) is the named textbook rule.
 *  [TREE] same notes, section 3 "G1 解法": EAGLE candidate trees (s, t, n).
 *  [MSS]  the pages name the trees but no rule for verifying them by
 *         sampling; the rule restated here is the multi-step speculative
 *         sampling of SpecInfer (Miao et al., "SpecInfer: Accelerating Large
 *         Language Model Serving with Tree-based Speculative Inference and
 *         Verification"), the recursive rejection sampling EAGLE adopts: it
 *         keeps the target's distribution when every node's children are
 *         drawn independently from that node's draft distribution.
 *  [TOPK] same notes, section 4 "G2 解法", worked example: keep the top-K=32
 *         target log-probs of the V=151936 row; KD target KL(softmax(log p) || q).
 *  [RWKD] ReSpec blog, section "奖励加权的适应机制": L_KD = w(r) * sum_t
 *         KL(p~ || q_theta); reading notes section 5 "G3 解法": w(r) = r by
 *         default, normalised and clipped in practice; GRPO group example.
 *
 * Readings where the pages are silent, each the plainest one the rest supports:
 *  - accept iff u*q(x) < p(x), u in [0,1) (strict: p(x)=0 always rejects);
 *  - one uniform per draft position (column i < k) plus one uniform (column k)
 *    for the single resample-or-bonus draw;
 *  - inverse-CDF sampling in ascending vocabulary order: the smallest j with
 *    u*W < C_j = sum_{l<=j} w_l;
 *  - a zero residual mass at a rejection (impossible in exact arithmetic for
 *    inputs where x ~ q) falls back to sampling the target row;
 *  - the same temperature T scales target and draft logits; draft
 *    probabilities are used as given;
 *  - argmax and top-K ties go to the lowest vocabulary index;
 *  - top-K log-probs are full-vocabulary log-softmax values; the KD target
 *    p~ renormalises them over the K kept entries;
 *  - the KD loss sums the accepted draft positions i < n_acc (optionally the
 *    first rejected position as well).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1 };
enum { OR_DRAFT_LOGITS = 0, OR_DRAFT_PROBS = 1 };
enum { OR_W_RAW = 0, OR_W_GROUP_NORM = 1 };
enum {
  OR_OK = 0,
  OR_BAD_ARG = -1,
  OR_BAD_TOKEN = -2,
  OR_NO_FINITE = -3,
  OR_BAD_TREE = -4,
  OR_NOMEM = -5
};

/* A deliberate mistake can be compiled in (-DOR_PLANT=n) so that the tests
 * can show that their pins catch it.  The default build plants nothing. */
#ifndef OR_PLANT
#define OR_PLANT 0
#endif

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Exact widening of element i of an fp32 or bf16 array to float64. */
static double load_value(const void* base, int dtype, size_t i) {
  if (dtype == OR_F32) return (double)((const float*)base)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Temperature softmax of one row:  a_j = z_j / T,  m = max_j a_j,
 * S = sum_j exp(a_j - m),  p_j = exp(a_j - m) / S.
 * Writes p (may be NULL) and returns the log-partition m + log S, or NAN when
 * the row has no finite logit. */
static double softmax_row(const void* base, int dtype, size_t off, int V, double T,
                          double* p) {
  double m = -INFINITY;
  for (int j = 0; j < V; ++j) {
    double a = load_value(base, dtype, off + (size_t)j) / T;
    if (a > m) m = a;
  }
  if (!isfinite(m)) return NAN;
  double S = 0.0;
  for (int j = 0; j < V; ++j) {
    double e = exp(load_value(base, dtype, off + (size_t)j) / T - m);
    if (p) p[j] = e;
    S += e;
  }
  if (p)
    for (int j = 0; j < V; ++j) p[j] /= S;
  return m + log(S);
}

/* Index of the largest value of a row; ties go to the lowest index. */
static int argmax_row(const void* base, int dtype, size_t off, int V) {
  int best = 0;
  double bv = load_value(base, dtype, off);
  for (int j = 1; j < V; ++j) {
    double v = load_value(base, dtype, off + (size_t)j);
    if (v > bv) {
      bv = v;
      best = j;
    }
  }
  return best;
}

/* Inverse-CDF draw from non-negative weights w (not necessarily normalised):
 * W = sum_j w_j, C_j = sum_{l<=j} w_l, result = smallest j with u*W < C_j.
 * *margin receives min_j |u - C_j / W|, the distance of the uniform to the
 * nearest CDF boundary (used by the tests to flag near-tie draws).
 * Returns -1 when W == 0. */
static int inverse_cdf(const double* w, int V, double u, double* margin) {
  double W = 0.0;
  for (int j = 0; j < V; ++j) W += w[j];
  if (!(W > 0.0)) {
    if (margin) *margin = 0.0;
    return -1;
  }
  double target = u * W, C = 0.0, best_gap = INFINITY;
  int pick = -1, last_positive = -1;
  for (int j = 0; j < V; ++j) {
    C += w[j];
    if (w[j] > 0.0) last_positive = j;
    double gap = fabs(u - C / W);
    if (gap < best_gap) best_gap = gap;
    if (pick < 0 && target < C) pick = j;
  }
  if (pick < 0) pick = last_positive; /* only reachable through rounding */
  if (margin) *margin = best_gap;
  return pick;
}

/* ------------------------------------------------------------------------ */
/* Chain verification ([SD], [ACC]).                                          */
/*                                                                            */
/* target [B, k+1, V], draft [B, k, V] (logits or probabilities),             */
/* draft_tokens [B, k], u [B, k+1].  Outputs accepted_len [B] and             */
/* out_tokens [B, k+1] (drafts[0..n) ++ [resample or bonus] ++ -1 padding).   */
/* Diagnostics (may be NULL): p_x, q_x [B, k] (NAN where the row was not      */
/* tested), cdf_margin [B], sample_row [B] (the row whose distribution was    */
/* sampled), fallback [B] (1 when the residual mass was zero).                */
/* T == 0 selects greedy verification.                                        */
/* ------------------------------------------------------------------------ */
/* draft_len [B] (may be NULL: k for every request): request b drafted
 * k_b <= k tokens; it uses target rows 0..k_b, draft rows 0..k_b-1, the
 * uniforms 0..k_b-1 for the tests and uniform k_b for the draw.  active [B]
 * (may be NULL: all active): an inactive request verifies nothing,
 * accepted_len = 0 and every out_token -1 (no token is emitted).          */
int oracle_verify_chain(const void* target, int t_dtype, const void* draft, int d_dtype,
                        int d_kind, const int32_t* draft_tokens, const float* u, int B,
                        int k, int V, double T, const int32_t* draft_len, const int32_t* active,
                        int32_t* accepted_len, int32_t* out_tokens, double* p_x, double* q_x,
                        double* cdf_margin, int32_t* sample_row, int32_t* fallback,
                        int nthreads) {
  if (B < 0 || k < 1 || V < 1 || !(T >= 0.0) || !target || !draft_tokens || !accepted_len ||
      !out_tokens)
    return OR_BAD_ARG;
  if (T > 0.0 && (!draft || !u)) return OR_BAD_ARG;
  for (int b = 0; b < B; ++b) {
    const int kb = draft_len ? draft_len[b] : k;
    if (kb < 0 || kb > k) return OR_BAD_ARG;
    if (active && !active[b]) continue;
    for (int i = 0; i < kb; ++i) {
      const int32_t t = draft_tokens[(size_t)b * k + i];
      if (t < 0 || t >= V) return OR_BAD_TOKEN;
    }
  }
  set_threads(nthreads);
  const int P = k + 1;
  int err = OR_OK;

#pragma omp parallel
  {
    double* p = (double*)malloc(sizeof(double) * (size_t)V);
    double* q = (double*)malloc(sizeof(double) * (size_t)V);
    double* r = (double*)malloc(sizeof(double) * (size_t)V);
    if (!p || !q || !r) {
#pragma omp atomic write
      err = OR_NOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
      if (!p || !q || !r) continue;
      const int32_t* x = draft_tokens + (size_t)b * k;
      int32_t* out = out_tokens + (size_t)b * P;
      for (int i = 0; i < P; ++i) out[i] = -1;
      if (p_x)
        for (int i = 0; i < k; ++i) p_x[(size_t)b * k + i] = q_x[(size_t)b * k + i] = NAN;
      if (cdf_margin) cdf_margin[b] = INFINITY;
      if (fallback) fallback[b] = 0;
      if (active && !active[b]) {  /* nothing verified, nothing emitted */
        accepted_len[b] = 0;
        if (sample_row) sample_row[b] = -1;
        continue;
      }
      const int kb = draft_len ? draft_len[b] : k;

      if (T == 0.0) {
        /* Greedy: accept x_i iff it equals the target argmax at row i; emit
         * the target argmax at the first mismatch, or at row k. */
        int n = kb, emit = -1;
        for (int i = 0; i < kb; ++i) {
          int g = argmax_row(target, t_dtype, ((size_t)b * P + i) * (size_t)V, V);
          if (x[i] != g) {
            n = i;
            emit = g;
            break;
          }
        }
        if (n == kb) emit = argmax_row(target, t_dtype, ((size_t)b * P + kb) * (size_t)V, V);
        for (int i = 0; i < n; ++i) out[i] = x[i];
        out[n] = emit;
        accepted_len[b] = n;
        if (sample_row) sample_row[b] = n;
        continue;
      }

      int n = kb, emit = -1, bad = 0;
      for (int i = 0; i < kb; ++i) {
        size_t trow = ((size_t)b * P + i) * (size_t)V;
        size_t drow = ((size_t)b * k + i) * (size_t)V;
        if (isnan(softmax_row(target, t_dtype, trow, V, T, p))) {
          bad = 1;
          break;
        }
        if (d_kind == OR_DRAFT_LOGITS) {
          if (isnan(softmax_row(draft, d_dtype, drow, V, T, q))) {
            bad = 1;
            break;
          }
        } else {
          for (int j = 0; j < V; ++j) q[j] = load_value(draft, d_dtype, drow + (size_t)j);
        }
        double px = p[x[i]], qx = q[x[i]];
        if (p_x) {
          p_x[(size_t)b * k + i] = px;
          q_x[(size_t)b * k + i] = qx;
        }
        double ub = (double)u[(size_t)b * P + i];
#if OR_PLANT == 2
        int accept = ub * px < qx; /* planted mistake: ratio inverted */
#else
        int accept = ub * qx < px; /* accept with probability min(1, p/q) */
#endif
        if (accept) continue;
        /* First rejection: draw from the residual max(0, p - q). */
        n = i;
        for (int j = 0; j < V; ++j) {
#if OR_PLANT == 1
          double d = q[j] - p[j]; /* planted mistake: residual sign flipped */
#else
          double d = p[j] - q[j];
#endif
          r[j] = d > 0.0 ? d : 0.0;
        }
        double mg;
        emit = inverse_cdf(r, V, (double)u[(size_t)b * P + kb], &mg);
        if (emit < 0) {
          /* Zero residual mass: sample the target row itself. */
          emit = inverse_cdf(p, V, (double)u[(size_t)b * P + kb], &mg);
          if (fallback) fallback[b] = 1;
        }
        if (cdf_margin) cdf_margin[b] = mg;
        break;
      }
      if (bad) {
        accepted_len[b] = -1;
#pragma omp atomic write
        err = OR_NO_FINITE;
        continue;
      }
      if (n == kb) {
        /* Every draft accepted: one bonus token from the target row k_b. */
#if OR_PLANT == 3
        size_t trow = ((size_t)b * P + k) * (size_t)V;
#else
        size_t trow = ((size_t)b * P + kb) * (size_t)V;
#endif
        if (isnan(softmax_row(target, t_dtype, trow, V, T, p))) {
          accepted_len[b] = -1;
#pragma omp atomic write
          err = OR_NO_FINITE;
          continue;
        }
        double mg;
        emit = inverse_cdf(p, V, (double)u[(size_t)b * P + kb], &mg);
        if (cdf_margin) cdf_margin[b] = mg;
      }
      for (int i = 0; i < n; ++i) out[i] = x[i];
      out[n] = emit;
      accepted_len[b] = n;
      if (sample_row) sample_row[b] = n;
    }
    free(p);
    free(q);
    free(r);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* Greedy tree verification ([TREE]).                                         */
/*                                                                            */
/* logits [B, n, V]: the target distribution after each candidate node.       */
/* node_tokens [B, n], parents [B, n] with parents[0] = -1 (node 0 is the     */
/* root, always accepted) and 0 <= parents[j] < j.  Node j >= 1 is accepted   */
/* iff its parent is accepted and its token equals the argmax of the parent's */
/* row.  The deepest accepted node wins (lowest index on ties).  Outputs:     */
/* accepted_len [B] = its depth; accepted_nodes [B, max_depth+1] = the path   */
/* root..best; out_tokens [B, max_depth+1] = the path's tokens (root          */
/* excluded) followed by the argmax of the best node's row; -1 padding.       */
/* ------------------------------------------------------------------------ */
int oracle_tree_greedy(const void* logits, int dtype, const int32_t* node_tokens,
                       const int32_t* parents, int B, int n, int V, int max_depth,
                       int32_t* accepted_len, int32_t* out_tokens, int32_t* accepted_nodes,
                       int nthreads) {
  if (B < 0 || n < 1 || V < 1 || max_depth < 0 || !logits || !node_tokens || !parents ||
      !accepted_len || !out_tokens || !accepted_nodes)
    return OR_BAD_ARG;
  for (int b = 0; b < B; ++b) {
    const int32_t* par = parents + (size_t)b * n;
    if (par[0] != -1) return OR_BAD_TREE;
    int* depth = (int*)malloc(sizeof(int) * (size_t)n);
    if (!depth) return OR_NOMEM;
    depth[0] = 0;
    int ok = 1;
    for (int j = 1; j < n && ok; ++j) {
      if (par[j] < 0 || par[j] >= j) ok = 0;
      else {
        depth[j] = depth[par[j]] + 1;
        if (depth[j] > max_depth) ok = 0;
      }
      if (node_tokens[(size_t)b * n + j] < 0 || node_tokens[(size_t)b * n + j] >= V) ok = 0;
    }
    free(depth);
    if (!ok) return OR_BAD_TREE;
  }
  set_threads(nthreads);
  const int W = max_depth + 1;
  int err = OR_OK;
#pragma omp parallel
  {
    int* g = (int*)malloc(sizeof(int) * (size_t)n);
    int* depth = (int*)malloc(sizeof(int) * (size_t)n);
    char* acc = (char*)malloc((size_t)n);
    if (!g || !depth || !acc) {
#pragma omp atomic write
      err = OR_NOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
      if (!g || !depth || !acc) continue;
      const int32_t* par = parents + (size_t)b * n;
      const int32_t* tok = node_tokens + (size_t)b * n;
      for (int j = 0; j < n; ++j) g[j] = argmax_row(logits, dtype, ((size_t)b * n + j) * (size_t)V, V);
      acc[0] = 1;
      depth[0] = 0;
      int best = 0;
      for (int j = 1; j < n; ++j) {
        depth[j] = depth[par[j]] + 1;
        acc[j] = acc[par[j]] && tok[j] == g[par[j]];
        if (acc[j] && depth[j] > depth[best]) best = j;
      }
      int L = depth[best];
      int32_t* on = accepted_nodes + (size_t)b * W;
      int32_t* ot = out_tokens + (size_t)b * W;
      for (int d = 0; d < W; ++d) on[d] = ot[d] = -1;
      for (int j = best, d = L; d >= 0; j = par[j], --d) on[d] = j;
      for (int d = 0; d < L; ++d) ot[d] = tok[on[d + 1]];
      ot[L] = g[best];
      accepted_len[b] = L;
    }
    free(g);
    free(depth);
    free(acc);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* Sampling tree verification ([TREE] for the trees; [MSS] for the rule).     */
/*                                                                            */
/* target [B, n, V]: the target distribution after each node; draft [B, n, V] */
/* (logits or probabilities): the draft distribution the node's children     */
/* were drawn from; node_tokens, parents as in oracle_tree_greedy; u [B, n]:  */
/* column j >= 1 tests node j, column 0 drives the one final draw.            */
/* Multi-step speculative sampling walks from the root.  At node v, r = p_v;  */
/* its children are tried in ascending index order: child c with token x is   */
/* accepted iff u_c * q_v(x) < r(x) (probability min(1, r(x)/q_v(x))), and    */
/* the walk moves to c; otherwise r becomes max(0, r - q_v) / sum max(0,      */
/* r - q_v) and the next child is tried.  When no child is accepted (or v is  */
/* a leaf) one token is drawn from r by inverse CDF with u_0.  A zero         */
/* residual mass (probability zero when the children are drawn from q_v)      */
/* ends the tests at v and draws from p_v.  Outputs as oracle_tree_greedy;    */
/* diagnostics (may be NULL): test_margin [B] = min over the tests of         */
/* |u_c - r(x)/q_v(x)| (q_v(x) > 0; +inf without such a test), cdf_margin     */
/* [B], fallback [B], n_tests [B].                                            */
/* ------------------------------------------------------------------------ */
int oracle_tree_sample(const void* target, int t_dtype, const void* draft, int d_dtype,
                       int d_kind, const int32_t* node_tokens, const int32_t* parents,
                       const float* u, int B, int n, int V, double T, int max_depth,
                       int32_t* accepted_len, int32_t* out_tokens, int32_t* accepted_nodes,
                       double* test_margin, double* cdf_margin, int32_t* fallback,
                       int32_t* n_tests, int nthreads) {
  if (B < 0 || n < 1 || V < 1 || max_depth < 0 || !(T > 0.0) || !target || !draft ||
      !node_tokens || !parents || !u || !accepted_len || !out_tokens || !accepted_nodes)
    return OR_BAD_ARG;
  for (int b = 0; b < B; ++b) {
    const int32_t* par = parents + (size_t)b * n;
    if (par[0] != -1) return OR_BAD_TREE;
    int* depth = (int*)malloc(sizeof(int) * (size_t)n);
    if (!depth) return OR_NOMEM;
    depth[0] = 0;
    int ok = 1;
    for (int j = 1; j < n && ok; ++j) {
      if (par[j] < 0 || par[j] >= j) ok = 0;
      else {
        depth[j] = depth[par[j]] + 1;
        if (depth[j] > max_depth) ok = 0;
      }
      if (node_tokens[(size_t)b * n + j] < 0 || node_tokens[(size_t)b * n + j] >= V) ok = 0;
    }
    free(depth);
    if (!ok) return OR_BAD_TREE;
  }
  set_threads(nthreads);
  const int W = max_depth + 1;
  int err = OR_OK;
#pragma omp parallel
  {
    double* p = (double*)malloc(sizeof(double) * (size_t)V);
    double* q = (double*)malloc(sizeof(double) * (size_t)V);
    double* r = (double*)malloc(sizeof(double) * (size_t)V);
    if (!p || !q || !r) {
#pragma omp atomic write
      err = OR_NOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
      if (!p || !q || !r) continue;
      const int32_t* par = parents + (size_t)b * n;
      const int32_t* tok = node_tokens + (size_t)b * n;
      const float* ub = u + (size_t)b * n;
      int32_t* on = accepted_nodes + (size_t)b * W;
      int32_t* ot = out_tokens + (size_t)b * W;
      for (int d = 0; d < W; ++d) on[d] = ot[d] = -1;
      double tm = INFINITY, mg = INFINITY;
      int fb = 0, tests = 0, depth = 0, v = 0, emit = -1, bad = 0;
      on[0] = 0;
      for (;;) {
        const size_t row = ((size_t)b * n + v) * (size_t)V;
        if (isnan(softmax_row(target, t_dtype, row, V, T, p))) {
          bad = 1;
          break;
        }
        if (d_kind == OR_DRAFT_LOGITS) {
          if (isnan(softmax_row(draft, d_dtype, row, V, T, q))) {
            bad = 1;
            break;
          }
        } else {
          for (int j = 0; j < V; ++j) q[j] = load_value(draft, d_dtype, row + (size_t)j);
        }
        memcpy(r, p, sizeof(double) * (size_t)V);
        int next = -1;
        for (int c = v + 1; c < n; ++c) {
          if (par[c] != v) continue;
          const int x = tok[c];
          const double uc = (double)ub[c];
          ++tests;
#if OR_PLANT == 4
          const double rx = p[x]; /* planted mistake: siblings tested against p, not the residual */
#else
          const double rx = r[x];
#endif
          if (q[x] > 0.0) {
            const double gap = fabs(uc - rx / q[x]);
            if (gap < tm) tm = gap;
          }
          if (uc * q[x] < rx) { /* accept with probability min(1, r(x) / q(x)) */
            next = c;
            break;
          }
          double s = 0.0;
          for (int j = 0; j < V; ++j) {
            const double d = r[j] - q[j];
            r[j] = d > 0.0 ? d : 0.0;
            s += r[j];
          }
          if (!(s > 0.0)) { /* zero residual mass: draw from the target row */
            memcpy(r, p, sizeof(double) * (size_t)V);
            fb = 1;
            break;
          }
          for (int j = 0; j < V; ++j) r[j] /= s;
        }
        if (next >= 0) {
          ++depth;
          on[depth] = next;
          ot[depth - 1] = tok[next];
          v = next;
          continue;
        }
        emit = inverse_cdf(r, V, (double)ub[0], &mg);
        break;
      }
      if (bad || emit < 0) {
        for (int d = 0; d < W; ++d) on[d] = ot[d] = -1;
        accepted_len[b] = -1;
#pragma omp atomic write
        err = OR_NO_FINITE;
      } else {
        ot[depth] = emit;
        accepted_len[b] = depth;
      }
      if (test_margin) test_margin[b] = tm;
      if (cdf_margin) cdf_margin[b] = mg;
      if (fallback) fallback[b] = fb;
      if (n_tests) n_tests[b] = tests;
    }
    free(p);
    free(q);
    free(r);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* Top-K extraction ([TOPK]).                                                 */
/*                                                                            */
/* For each of `rows` rows of V logits: lse = log sum_j exp(z_j / T); the K   */
/* kept entries are the first K of a full sort by (z desc, index asc);        */
/* topk_logp = z_j / T - lse (full-vocabulary log-softmax).                   */
/* ------------------------------------------------------------------------ */
typedef struct {
  double z;
  int idx;
} zi_t;

static int cmp_value_desc_index_asc(const void* a, const void* b) {
  const zi_t* x = (const zi_t*)a;
  const zi_t* y = (const zi_t*)b;
  if (x->z > y->z) return -1;
  if (x->z < y->z) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

int oracle_topk(const void* logits, int dtype, int rows, int V, int K, double T,
                double* topk_logp, int32_t* topk_idx, double* lse, int nthreads) {
  if (rows < 0 || V < 1 || K < 1 || K > V || !(T > 0.0) || !logits || !topk_logp ||
      !topk_idx || !lse)
    return OR_BAD_ARG;
  set_threads(nthreads);
  int err = OR_OK;
#pragma omp parallel
  {
    zi_t* buf = (zi_t*)malloc(sizeof(zi_t) * (size_t)V);
    if (!buf) {
#pragma omp atomic write
      err = OR_NOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
      if (!buf) continue;
      size_t off = (size_t)r * V;
      double L = softmax_row(logits, dtype, off, V, T, NULL);
      lse[r] = L;
      if (isnan(L)) {
#pragma omp atomic write
        err = OR_NO_FINITE;
        continue;
      }
      for (int j = 0; j < V; ++j) {
        buf[j].z = load_value(logits, dtype, off + (size_t)j);
        buf[j].idx = j;
      }
      qsort(buf, (size_t)V, sizeof(zi_t), cmp_value_desc_index_asc);
      for (int t = 0; t < K; ++t) {
        topk_idx[(size_t)r * K + t] = buf[t].idx;
        topk_logp[(size_t)r * K + t] = buf[t].z / T - L;
      }
    }
    free(buf);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* KD divergence per draft position ([TOPK], [RWKD]).                         */
/*                                                                            */
/* topk_logp / topk_idx [B, k+1, K] hold the target's kept log-probs; draft   */
/* row (b, i < k) is paired with target row (b, i).  p~_j = exp(lp_j -        */
/* logsumexp_K(lp)); log q_j = z_d,j / T - lse_d (logits) or log q_j (probs). */
/* KL = sum_j p~_j (log p~_j - log q_j), with 0 log 0 = 0.                    */
/* scale [B, k] (may be NULL) receives sum_j p~_j |log q_j|, the magnitude    */
/* that sets how many digits of KL survive rounding.                          */
/* ------------------------------------------------------------------------ */
int oracle_kl(const double* topk_logp, const int32_t* topk_idx, int B, int k, int K,
              const void* draft, int d_dtype, int d_kind, int V, double T, double* kl,
              double* scale, int nthreads) {
  if (B < 0 || k < 1 || K < 1 || K > V || !(T > 0.0) || !topk_logp || !topk_idx || !draft ||
      !kl)
    return OR_BAD_ARG;
  set_threads(nthreads);
  const int P = k + 1;
  int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int row = 0; row < B * k; ++row) {
    int b = row / k, i = row % k;
    const double* lp = topk_logp + ((size_t)b * P + i) * K;
    const int32_t* ix = topk_idx + ((size_t)b * P + i) * K;
    size_t drow = ((size_t)b * k + i) * (size_t)V;
    double lse_d = 0.0;
    if (d_kind == OR_DRAFT_LOGITS) {
      lse_d = softmax_row(draft, d_dtype, drow, V, T, NULL);
      if (isnan(lse_d)) {
#pragma omp atomic write
        err = OR_NO_FINITE;
        kl[row] = NAN;
        continue;
      }
    }
    double mk = -INFINITY;
    for (int t = 0; t < K; ++t)
      if (lp[t] > mk) mk = lp[t];
    double sk = 0.0;
    for (int t = 0; t < K; ++t) sk += exp(lp[t] - mk);
    double lse_k = mk + log(sk);
    double acc = 0.0, mag = 0.0;
    for (int t = 0; t < K; ++t) {
      int j = ix[t];
      if (j < 0 || j >= V) {
#pragma omp atomic write
        err = OR_BAD_TOKEN;
        continue;
      }
      double log_pt = lp[t] - lse_k;
      double pt = exp(log_pt);
      if (pt == 0.0) continue;
      double log_q = d_kind == OR_DRAFT_LOGITS
                         ? load_value(draft, d_dtype, drow + (size_t)j) / T - lse_d
                         : log(load_value(draft, d_dtype, drow + (size_t)j));
      acc += pt * (log_pt - log_q);
      mag += pt * fabs(log_q);
    }
    kl[row] = acc;
    if (scale) scale[row] = mag;
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* Reward-weighted reduction ([RWKD]).                                        */
/*                                                                            */
/* w_b = r_b (RAW) or r_b / sum_{b' in group(b)} r_b' (GROUP_NORM, groups of  */
/* `group` consecutive requests; a zero group sum gives w = 0); clip > 0      */
/* clamps w to [-clip, clip].  loss_b = w_b * sum_{i < m_b} kl[b, i] (0 when  */
/* w_b == 0: a zero-weight sample contributes nothing); total = sum_b loss_b. */
/* m_b = accepted_len[b] (positions = 0: the accepted drafts), or, with       */
/* positions = 1, one more when a draft was rejected (n < k): the first       */
/* rejected position too, as drafters that learn from their rejected          */
/* proposals do ("Draft-OPD" page).                                           */
/* Ragged batches: draft_len [B] (may be NULL: k) moves the "rejected" test   */
/* to n < k_b; a request with active[b] == 0 (active may be NULL) has         */
/* loss_b = 0.                                                                */
/* ------------------------------------------------------------------------ */
int oracle_reward_loss(const double* kl, const int32_t* accepted_len, const double* reward,
                       int B, int k, int mode, int group, double clip, int positions,
                       const int32_t* draft_len, const int32_t* active, double* w,
                       double* loss, double* total) {
  if (B < 0 || k < 1 || !kl || !accepted_len || !reward || !loss || !total) return OR_BAD_ARG;
  if (mode == OR_W_GROUP_NORM && (group < 1 || B % group != 0)) return OR_BAD_ARG;
  double sum = 0.0;
  for (int b = 0; b < B; ++b) {
    double wb = reward[b];
    if (mode == OR_W_GROUP_NORM) {
      int g0 = (b / group) * group;
      double gs = 0.0;
      for (int t = g0; t < g0 + group; ++t) gs += reward[t];
      wb = gs == 0.0 ? 0.0 : reward[b] / gs;
    }
    if (clip > 0.0) wb = wb > clip ? clip : (wb < -clip ? -clip : wb);
    if (w) w[b] = wb;
    const int kb = draft_len ? draft_len[b] : k;
    int n = accepted_len[b];
    if (kb < 0 || kb > k || n < 0 || n > kb) return OR_BAD_ARG;
    int m = (positions && n < kb) ? n + 1 : n;
    double s = 0.0;
    for (int i = 0; i < m; ++i) s += kl[(size_t)b * k + i];
    loss[b] = (wb == 0.0 || (active && !active[b])) ? 0.0 : wb * s;
    sum += loss[b];
  }
  *total = sum;
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Gradient of the reward-weighted KD loss with respect to the draft logits   */
/* ([RWKD]; reading notes section 4, Algorithm 1 step 3: the drafter's        */
/* gradient flows into the current q_theta only, never into the stored       */
/* log q).  From d log q_j / d z_l = (delta_jl - q_l) / T and sum_j p~_j = 1:  */
/*   d loss_b / d z_d[b, i, l] = w_b [i < n_b] (q_il - p~_il [l in K]) / T.    */
/* Logit drafts only; w_b and the positions i < m_b as in oracle_reward_loss. */
/* ------------------------------------------------------------------------ */
int oracle_kd_grad(const double* topk_logp, const int32_t* topk_idx, int B, int k, int K,
                   const void* draft, int d_dtype, int V, double T,
                   const int32_t* accepted_len, const double* reward, int mode, int group,
                   double clip, int positions, double* grad, int nthreads) {
  if (B < 0 || k < 1 || K < 1 || K > V || !(T > 0.0) || !topk_logp || !topk_idx || !draft ||
      !accepted_len || !reward || !grad)
    return OR_BAD_ARG;
  if (mode == OR_W_GROUP_NORM && (group < 1 || B % group != 0)) return OR_BAD_ARG;
  set_threads(nthreads);
  const int P = k + 1;
  int err = OR_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int row = 0; row < B * k; ++row) {
    int b = row / k, i = row % k;
    double* g = grad + (size_t)row * V;
    for (int j = 0; j < V; ++j) g[j] = 0.0;
    double wb = reward[b];
    if (mode == OR_W_GROUP_NORM) {
      int g0 = (b / group) * group;
      double gs = 0.0;
      for (int t = g0; t < g0 + group; ++t) gs += reward[t];
      wb = gs == 0.0 ? 0.0 : reward[b] / gs;
    }
    if (clip > 0.0) wb = wb > clip ? clip : (wb < -clip ? -clip : wb);
    int n = accepted_len[b];
    if (n < 0 || n > k) {
#pragma omp atomic write
      err = OR_BAD_ARG;
      continue;
    }
    int m = (positions && n < k) ? n + 1 : n;
    if (i >= m || wb == 0.0) continue;
    size_t drow = (size_t)row * (size_t)V;
    double lse_d = softmax_row(draft, d_dtype, drow, V, T, NULL);
    if (isnan(lse_d)) {
#pragma omp atomic write
      err = OR_NO_FINITE;
      continue;
    }
    for (int j = 0; j < V; ++j) g[j] = wb * exp(load_value(draft, d_dtype, drow + (size_t)j) / T - lse_d) / T;
    const double* lp = topk_logp + ((size_t)b * P + i) * K;
    const int32_t* ix = topk_idx + ((size_t)b * P + i) * K;
    double mk = -INFINITY;
    for (int t = 0; t < K; ++t)
      if (lp[t] > mk) mk = lp[t];
    double sk = 0.0;
    for (int t = 0; t < K; ++t) sk += exp(lp[t] - mk);
    double lse_k = mk + log(sk);
    for (int t = 0; t < K; ++t) {
      int j = ix[t];
      if (j < 0 || j >= V) {
#pragma omp atomic write
        err = OR_BAD_TOKEN;
        continue;
      }
      g[j] -= wb * exp(lp[t] - lse_k) / T;
    }
  }
  return err;
}

/* Temperature softmax of `rows` rows (exposed so that the tests can compare
 * the oracle's normalisation against an independent library routine). */
int oracle_softmax(const void* logits, int dtype, int rows, int V, double T, double* p,
                   double* log_partition) {
  if (rows < 0 || V < 1 || !(T > 0.0) || !logits || !p) return OR_BAD_ARG;
  for (int r = 0; r < rows; ++r) {
    double L = softmax_row(logits, dtype, (size_t)r * V, V, T, p + (size_t)r * V);
    if (log_partition) log_partition[r] = L;
    if (isnan(L)) return OR_NO_FINITE;
  }
  return OR_OK;
}
