/*
 * psispec_oracle.c -- plain fp64 CPU oracle of the Psi-Spec verification step.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the benchmark's
 * CPU-baseline leg, never by the product path. It shares no code with the CUDA library.
 *
 * The method is the rejection-correction step of "Unlocking Lossless Speedups in LLMs via
 * Discrete Diffusion" (arXiv 2609.04010), as stated on the long-form review page
 * (vibe-research.pages.dev, 2026-09-09), section 3.3 "Psi-Spec": accept draft token i with
 * probability min(1, p_AR(x_i)/p_draft(x_i)), keep the longest prefix before the first
 * rejection, resample the rejected position from the normalised residual [p_AR - p_draft]_+,
 * and draw one extra token from the last verifier row when the whole block is accepted.
 * Temperature and top-p are the sampling controls listed by the project's README (inference
 * example, "--temperature --top-p"). Section 3.4 names the tree sampler; its acceptance rule
 * is not printed on the pages, and the reading implemented here is recursive rejection
 * sampling over the children of a node, in index order, with the proposal the children came
 * from: drawn from q without replacement (the default), fixed in advance (the candidate trie
 * of top-k tokens and best prefixes that section 3.4 describes, built by oracle_build_tree),
 * or drawn from q independently.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - top-p keeps every token whose logit is >= tau, where tau is the largest logit value
 *     whose tie-inclusive upper-tail probability reaches top_p; it is applied after the
 *     temperature, to the verifier row and to the draft row separately;
 *   - top-k (listed among the README's common controls, "--top-k", and defined nowhere on
 *     the pages) keeps every token whose logit is >= the k-th largest logit of the row (ties
 *     with it kept together); it acts after the temperature and before top-p, which then
 *     works on the renormalised top-k set; k <= 0 or k >= V is off, and it is a no-op at
 *     temperature 0;
 *   - temperature 0 is greedy: a point mass on the lowest-index maximum;
 *   - an inverse-CDF draw walks the vocabulary in index order and returns the first v with
 *     C(v) > u * Z (strict, inclusive prefix), so a zero-mass token is never drawn;
 *   - "accept with probability min(1, p/q)" is the test u * q < p with u in [0, 1);
 *   - an all-zero residual (reachable only by rounding) leaves the previous distribution.
 *
 * Everything below is straight fp64 loops over the vocabulary; no blocking or reordering.
 */
#include "psispec_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static double dmin(double a, double b) { return a < b ? a : b; }

/* Keeps the smallest band of a path and the kind of decision (E1, E2, E3) it belongs to. */
static void note_band(double* band, int* kind, double b, int k) {
  if (b < *band) {
    *band = b;
    *kind = k;
  }
}

static int cmp_desc(const void* a, const void* b) {
  double x = *(const double*)a, y = *(const double*)b;
  return (x < y) - (x > y);
}

int oracle_row_dist_k(const double* l, int V, double T, double top_p, int top_k, double* out, double* band) {
  *band = INFINITY;
  if (V <= 0 || !(T >= 0)) return -1;
  int any_finite = 0;
  for (int v = 0; v < V; ++v) {
    if (isnan(l[v]) || l[v] == INFINITY) return -1;
    if (isfinite(l[v])) any_finite = 1;
  }
  if (!any_finite) return -1;

  /* row maximum, lowest index on ties */
  double m = -INFINITY;
  int amax = -1;
  for (int v = 0; v < V; ++v)
    if (l[v] > m) { m = l[v]; amax = v; }

  if (T == 0.0) {
    for (int v = 0; v < V; ++v) out[v] = 0.0;
    out[amax] = 1.0;
    return 0;
  }

  /* softmax(l / T) numerator and total, in vocabulary order */
  double S = 0.0;
  for (int v = 0; v < V; ++v) {
    out[v] = exp((l[v] - m) / T);
    S += out[v];
  }

  double tau = -INFINITY, S_kept = S;
  const int use_k = top_k > 0 && top_k < V;
  if (use_k || top_p < 1.0) {
    double* vals = (double*)malloc(sizeof(double) * (size_t)V);
    memcpy(vals, l, sizeof(double) * (size_t)V);
    qsort(vals, (size_t)V, sizeof(double), cmp_desc);
    if (use_k) {
      /* top-k: the k-th largest value, every token at or above it kept */
      tau = vals[top_k - 1];
      S_kept = 0.0;
      for (int v = 0; v < V; ++v)
        if (l[v] >= tau) S_kept += out[v];
    }
    if (top_p < 1.0) {
      /* walk the distinct logit values of the kept set from the top; stop at the first value
         whose tie-inclusive tail mass reaches top_p of the kept set's total */
      const double floor_v = tau, total = S_kept;
      double tail = 0.0;
      int found = 0;
      for (int i = 0; i < V && vals[i] >= floor_v;) {
        double t = vals[i], group = 0.0;
        int j = i;
        while (j < V && vals[j] == t) { group += exp((t - m) / T); ++j; }
        double above = tail;
        tail += group;
        if (tail >= top_p * total) {
          tau = t;
          S_kept = tail;
          *band = dmin(fabs(tail / total - top_p), fabs(above / total - top_p));
          found = 1;
          break;
        }
        i = j;
      }
      if (!found) *band = 0.0;  /* rounding only: the whole kept set stays */
    }
    free(vals);
  }
  for (int v = 0; v < V; ++v) out[v] = (l[v] >= tau) ? out[v] / S_kept : 0.0;
  return 0;
}

int oracle_row_dist(const double* l, int V, double T, double top_p, double* out, double* band) {
  return oracle_row_dist_k(l, V, T, top_p, 0, out, band);
}

int oracle_inverse_cdf(const double* r, int V, double u, double* band) {
  double Z = 0.0;
  for (int v = 0; v < V; ++v) Z += r[v];
  if (!(Z > 0.0)) { *band = 0.0; return -1; }
  double target = u * Z, C = 0.0;
  int last = -1;
  for (int v = 0; v < V; ++v) {
    double before = C;
    C += r[v];
    if (r[v] > 0.0) last = v;
    if (C > target) {
      *band = dmin(fabs(before / Z - u), fabs(C / Z - u));
      return v;
    }
  }
  *band = 0.0;
  return last;
}

int oracle_sample_draft(const double* draft, int rows, int V, const int* row_req,
                        const double* temperature, const double* top_p, const int* top_k, const double* u,
                        int* tokens, double* q_at, double* band, int* band_kind) {
  if (rows < 0 || V <= 0) return ORACLE_BAD_ARG;
  double* q = (double*)malloc(sizeof(double) * (size_t)V);
  for (int i = 0; i < rows; ++i) {
    int b = row_req[i];
    double b3 = INFINITY, b2 = INFINITY;
    tokens[i] = -1;
    q_at[i] = -1.0;
    band[i] = INFINITY;
    if (band_kind) band_kind[i] = ORACLE_BAND_NONE;
    if (oracle_row_dist_k(draft + (size_t)i * V, V, temperature[b], top_p[b], top_k ? top_k[b] : 0, q, &b3) != 0)
      continue;
    int y = oracle_inverse_cdf(q, V, u[i], &b2);
    tokens[i] = y;
    q_at[i] = y >= 0 ? q[y] : -1.0;
    int kind = ORACLE_BAND_NONE;
    double bi = INFINITY;
    note_band(&bi, &kind, b3, ORACLE_BAND_E3);
    note_band(&bi, &kind, b2, ORACLE_BAND_E2);
    band[i] = bi;
    if (band_kind) band_kind[i] = kind;
  }
  free(q);
  return ORACLE_OK;
}

int oracle_verify_linear(const double* target, const double* draft, int B, int K, int V,
                         const int* draft_tokens, const double* u_accept, const double* u_resid,
                         const double* temperature, const double* top_p, const int* top_k,
                         int* out_tokens, int* accept_len, double* out_p, double* out_q,
                         double* band, double* pq_band, int* band_kind) {
  if (B < 0 || K < 0 || V <= 0) return ORACLE_BAD_ARG;
  double* p = (double*)malloc(sizeof(double) * (size_t)V);
  double* q = (double*)malloc(sizeof(double) * (size_t)V);
  double* res = (double*)malloc(sizeof(double) * (size_t)V);
  for (int b = 0; b < B; ++b) {
    const double T = temperature[b], tp = top_p[b];
    const int tk = top_k ? top_k[b] : 0;
    const double* tgt = target + (size_t)b * (K + 1) * V;
    const double* drf = draft + (size_t)b * K * V;
    int* toks = out_tokens + (size_t)b * (K + 1);
    int bad = 0, j = K, y = -1, path_kind = ORACLE_BAND_NONE;
    double path_band = INFINITY;
    for (int i = 0; i <= K; ++i) toks[i] = -1;
    for (int i = 0; i < K; ++i) pq_band[(size_t)b * K + i] = INFINITY;

    for (int i = 0; i < K && !bad; ++i) {
      double bp = INFINITY, bq = INFINITY;
      int x = draft_tokens[(size_t)b * K + i];
      if (x < 0 || x >= V) { bad = 1; break; }
      if (oracle_row_dist_k(tgt + (size_t)i * V, V, T, tp, tk, p, &bp) != 0) { bad = 1; break; }
      if (oracle_row_dist_k(drf + (size_t)i * V, V, T, tp, tk, q, &bq) != 0) { bad = 1; break; }
      out_p[(size_t)b * K + i] = p[x];
      out_q[(size_t)b * K + i] = q[x];
      pq_band[(size_t)b * K + i] = dmin(bp, bq);
      if (i > j) continue; /* past the first rejection: probabilities only */
      double u = u_accept[(size_t)b * K + i];
      note_band(&path_band, &path_kind, dmin(bp, bq), ORACLE_BAND_E3);
      if (q[x] > 0.0) note_band(&path_band, &path_kind, fabs(u - p[x] / q[x]), ORACLE_BAND_E1);
      if (u * q[x] < p[x]) continue; /* accepted */
      /* first rejection: draw from the normalised residual [p - q]_+ */
      j = i;
      double Z = 0.0;
      for (int v = 0; v < V; ++v) {
        res[v] = p[v] > q[v] ? p[v] - q[v] : 0.0;
        Z += res[v];
      }
      double b2 = INFINITY;
      y = oracle_inverse_cdf(Z > 0.0 ? res : p, V, u_resid[(size_t)b * (K + 1) + i], &b2);
      note_band(&path_band, &path_kind, b2, ORACLE_BAND_E2);
    }
    if (!bad) {
      double bp = INFINITY;
      if (oracle_row_dist_k(tgt + (size_t)K * V, V, T, tp, tk, p, &bp) != 0) bad = 1;
      if (!bad && j == K) { /* whole block accepted: bonus draw from the last verifier row */
        double b2 = INFINITY;
        y = oracle_inverse_cdf(p, V, u_resid[(size_t)b * (K + 1) + K], &b2);
        note_band(&path_band, &path_kind, bp, ORACLE_BAND_E3);
        note_band(&path_band, &path_kind, b2, ORACLE_BAND_E2);
      }
    }
    if (bad) {
      accept_len[b] = -1;
      for (int i = 0; i < K; ++i) { out_p[(size_t)b * K + i] = -1.0; out_q[(size_t)b * K + i] = -1.0; }
      band[b] = INFINITY;
      if (band_kind) band_kind[b] = ORACLE_BAND_NONE;
      continue;
    }
    accept_len[b] = j;
    for (int i = 0; i < j; ++i) toks[i] = draft_tokens[(size_t)b * K + i];
    toks[j] = y;
    band[b] = path_band;
    if (band_kind) band_kind[b] = path_kind;
  }
  free(p);
  free(q);
  free(res);
  return ORACLE_OK;
}

int oracle_verify_tree(const double* target, const double* draft, int B, int V,
                       const int* node_offsets, const int* parent, const int* tokens,
                       const double* u_accept, const double* u_resid,
                       const double* temperature, const double* top_p, const int* top_k, int max_depth,
                       int* out_path, int* out_tokens, int* accept_len, double* band, int* band_kind) {
  return oracle_verify_tree_rule(target, draft, B, V, node_offsets, parent, tokens, u_accept, u_resid, temperature,
                                 top_p, top_k, max_depth, ORACLE_TREE_SAMPLED_WOR, out_path, out_tokens, accept_len,
                                 band, band_kind);
}

/* Tree verification under one of three candidate rules, the same walk for each: at the
 * current node the children are tested in index order with their own uniforms; an accepted
 * child becomes the current node; when every child is rejected (or the node is a leaf) the
 * final token is drawn from the node's current residual r with the node's u_resid.
 *   ORACLE_TREE_SAMPLED_WOR    children drawn from q one after another without replacement:
 *                              accept t iff u q~(t) < r(t); on rejection r <- norm([r - q~]_+)
 *                              and q~ <- q~ without t, renormalised (R7);
 *   ORACLE_TREE_DETERMINISTIC  children fixed in advance (a candidate tree from top-k and best
 *                              prefixes): each is the point mass delta_t, so the same step with
 *                              q~ = delta_t reads: accept t iff u < r(t); on rejection
 *                              r <- [r - delta_t]_+ renormalised, i.e. r without t;
 *   ORACLE_TREE_SAMPLED_WR     children drawn independently from q (with replacement): accept t
 *                              iff u q(t) < r(t); on rejection r <- norm([r - q]_+), q unchanged.
 * Each is recursive rejection sampling with the proposal its children were drawn from, so the
 * emitted tokens follow the verifier's law whenever the children were produced that way. */
int oracle_verify_tree_rule(const double* target, const double* draft, int B, int V,
                            const int* node_offsets, const int* parent, const int* tokens,
                            const double* u_accept, const double* u_resid,
                            const double* temperature, const double* top_p, const int* top_k, int max_depth,
                            int rule, int* out_path, int* out_tokens, int* accept_len, double* band,
                            int* band_kind) {
  if (B < 0 || V <= 0 || max_depth < 0) return ORACLE_BAD_ARG;
  if (rule != ORACLE_TREE_SAMPLED_WOR && rule != ORACLE_TREE_DETERMINISTIC && rule != ORACLE_TREE_SAMPLED_WR)
    return ORACLE_BAD_ARG;
  double* r = (double*)malloc(sizeof(double) * (size_t)V);
  double* qt = (double*)malloc(sizeof(double) * (size_t)V);
  double* res = (double*)malloc(sizeof(double) * (size_t)V);
  for (int b = 0; b < B; ++b) {
    const int n0 = node_offsets[b], n = node_offsets[b + 1] - node_offsets[b];
    const double T = temperature[b], tp = top_p[b];
    const int tk = top_k ? top_k[b] : 0;
    int* path = out_path + (size_t)b * max_depth;
    int* toks = out_tokens + (size_t)b * (max_depth + 1);
    for (int i = 0; i < max_depth; ++i) path[i] = -1;
    for (int i = 0; i <= max_depth; ++i) toks[i] = -1;
    accept_len[b] = -1;
    band[b] = INFINITY;
    if (band_kind) band_kind[b] = ORACLE_BAND_NONE;

    /* structure checks: root first, parents precede children, depth within max_depth */
    int bad = n <= 0 || parent[n0] != -1;
    int* depth = (int*)calloc((size_t)(n > 0 ? n : 1), sizeof(int));
    for (int c = 1; c < n && !bad; ++c) {
      int pa = parent[n0 + c], t = tokens[n0 + c];
      if (pa < 0 || pa >= c || t < 0 || t >= V) { bad = 1; break; }
      depth[c] = depth[pa] + 1;
      if (depth[c] > max_depth) bad = 1;
    }
    free(depth);
    if (bad) continue;

    double path_band = INFINITY;
    int cur = 0, len = 0, y = -1, path_kind = ORACLE_BAND_NONE;
    for (;;) {
      double b3 = INFINITY;
      if (oracle_row_dist_k(target + (size_t)(n0 + cur) * V, V, T, tp, tk, r, &b3) != 0) { bad = 1; break; }
      note_band(&path_band, &path_kind, b3, ORACLE_BAND_E3);
      int has_child = 0;
      for (int c = cur + 1; c < n; ++c) has_child |= parent[n0 + c] == cur;
      if (has_child && T > 0.0 && rule != ORACLE_TREE_DETERMINISTIC) {
        if (oracle_row_dist_k(draft + (size_t)(n0 + cur) * V, V, T, tp, tk, qt, &b3) != 0) { bad = 1; break; }
        note_band(&path_band, &path_kind, b3, ORACLE_BAND_E3);
      }
      int next = -1;
      for (int c = cur + 1; c < n && next < 0; ++c) {
        if (parent[n0 + c] != cur) continue;
        int t = tokens[n0 + c];
        if (T == 0.0) { /* greedy: the child carrying the verifier's argmax is accepted */
          if (r[t] > 0.0) next = c;
          continue;
        }
        if (rule == ORACLE_TREE_DETERMINISTIC) {
          const double ud = u_accept[n0 + c];
          note_band(&path_band, &path_kind, fabs(ud - r[t]), ORACLE_BAND_E1);
          if (ud < r[t]) { next = c; break; }
          /* rejected: [r - delta_t]_+ is r without t; renormalise */
          r[t] = 0.0;
          double Zr = 0.0;
          for (int v = 0; v < V; ++v) Zr += r[v];
          if (Zr > 0.0)
            for (int v = 0; v < V; ++v) r[v] /= Zr;
          continue;
        }
        double qmass = 0.0;
        for (int v = 0; v < V; ++v) qmass += qt[v];
        if (!(qmass > 0.0)) break; /* draft mass exhausted: remaining siblings skipped */
        double u = u_accept[n0 + c];
        if (qt[t] > 0.0) note_band(&path_band, &path_kind, fabs(u - r[t] / qt[t]), ORACLE_BAND_E1);
        if (u * qt[t] < r[t]) { next = c; break; }
        /* rejected: r <- norm([r - qt]_+), then remove t from the draft and renormalise */
        double Z = 0.0;
        for (int v = 0; v < V; ++v) {
          res[v] = r[v] > qt[v] ? r[v] - qt[v] : 0.0;
          Z += res[v];
        }
        if (Z > 0.0)
          for (int v = 0; v < V; ++v) r[v] = res[v] / Z;
        if (rule == ORACLE_TREE_SAMPLED_WOR) {
          qt[t] = 0.0;
          double Zq = 0.0;
          for (int v = 0; v < V; ++v) Zq += qt[v];
          if (Zq > 0.0)
            for (int v = 0; v < V; ++v) qt[v] /= Zq;
        }
      }
      if (next >= 0) {
        path[len] = next;
        toks[len] = tokens[n0 + next];
        ++len;
        cur = next;
        continue;
      }
      double b2 = INFINITY;
      y = oracle_inverse_cdf(r, V, u_resid[n0 + cur], &b2);
      note_band(&path_band, &path_kind, b2, ORACLE_BAND_E2);
      break;
    }
    if (bad) {
      for (int i = 0; i < max_depth; ++i) path[i] = -1;
      for (int i = 0; i <= max_depth; ++i) toks[i] = -1;
      continue;
    }
    toks[len] = y;
    accept_len[b] = len;
    band[b] = path_band;
    if (band_kind) band_kind[b] = path_kind;
  }
  free(r);
  free(qt);
  free(res);
  return ORACLE_OK;
}

/* Candidate trie of the tree sampler. Review page, section 3.4 ("Tree Sampler"): at every
 * position of the block take the top-K tokens, then keep the V most probable prefixes and
 * verify them together with tree attention; the README's tree example sets the two sizes by
 * flags (a tree candidate top-k and a tree verify size). Readings where the page is silent:
 *   - the per-position distributions are the draft's q_i (after the sampling controls, as
 *     everywhere); a prefix's probability is the product of q_i over its tokens;
 *   - candidates at position i are the cand_k tokens of largest q_i with q_i > 0 (ties to the
 *     lower token index); prefixes have length 1..K;
 *   - "the V most probable prefixes" are taken in decreasing probability, ties to the shorter
 *     prefix, then to the lexicographically smaller sequence of candidate ranks; a prefix is
 *     never less probable than its parent, so the kept set is closed under taking prefixes and
 *     forms a trie;
 *   - probabilities are compared exactly where that is possible: two prefixes of the same
 *     length share their positions, hence their normalisers, so the more probable one is the
 *     one with the larger sum of logits (exact in fp64 for bf16 and ordinary fp32 logits;
 *     logits on the bf16 grid make equal sums, i.e. exact ties, common). Prefixes of different
 *     lengths are compared by their fp64 probabilities.
 * They are found best-first: the frontier starts with the first position's candidates; the
 * best frontier prefix is kept and its extensions by the next position's candidates join the
 * frontier. Kept prefixes become nodes in the order kept (node 0 is the root, the empty
 * prefix), so parents precede children and siblings are in decreasing probability.
 * draft[K*V]: the draft rows of positions 0..K-1. Outputs (n_prefixes + 1 entries): parent,
 * tokens (-1 at the root), depth (number of tokens of the prefix), score (its probability);
 * *n_nodes = 1 + the number of kept prefixes (fewer than n_prefixes when the candidates run
 * out). Returns ORACLE_OK, ORACLE_BAD_ARG, or -1 for a bad draft row. */
int oracle_build_tree(const double* draft, int K, int V, double T, double top_p, int top_k, int cand_k,
                      int n_prefixes, int* parent, int* tokens, int* depth, double* score, int* n_nodes) {
  if (K < 0 || V <= 0 || cand_k < 0 || n_prefixes < 0) return ORACLE_BAD_ARG;
  double* q = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * V);
  int* cand = (int*)malloc(sizeof(int) * (size_t)(K > 0 ? K : 1) * (cand_k > 0 ? cand_k : 1));
  int* ncand = (int*)calloc((size_t)(K > 0 ? K : 1), sizeof(int));
  int rc = ORACLE_OK;
  for (int i = 0; i < K && rc == ORACLE_OK; ++i) {
    double b3;
    double* qi = q + (size_t)i * V;
    if (oracle_row_dist_k(draft + (size_t)i * V, V, T, top_p, top_k, qi, &b3) != 0) { rc = -1; break; }
    /* the cand_k most probable tokens, one selection pass each */
    for (int r = 0; r < cand_k; ++r) {
      int best = -1;
      for (int v = 0; v < V; ++v) {
        if (!(qi[v] > 0.0)) continue;
        int taken = 0;
        for (int j = 0; j < r && !taken; ++j) taken = cand[i * cand_k + j] == v;
        if (taken) continue;
        if (best < 0 || qi[v] > qi[best]) best = v;
      }
      if (best < 0) break;
      cand[i * cand_k + r] = best;
      ncand[i] = r + 1;
    }
  }
  if (rc != ORACLE_OK) {
    free(q);
    free(cand);
    free(ncand);
    return rc;
  }
  /* kept prefixes: rank path of every node (its candidate rank at each position) */
  const int cap = n_prefixes + 1;
  int* ranks = (int*)calloc((size_t)cap * (K > 0 ? K : 1), sizeof(int));
  double* lsum = (double*)calloc((size_t)cap, sizeof(double)); /* sum of the prefix's logits */
  /* frontier entries: (parent node, candidate rank at the parent's depth) */
  const int fcap = cand_k * cap + 1;
  int* f_par = (int*)malloc(sizeof(int) * (size_t)fcap);
  int* f_rank = (int*)malloc(sizeof(int) * (size_t)fcap);
  int nf = 0;
  parent[0] = -1;
  tokens[0] = -1;
  depth[0] = 0;
  score[0] = 1.0;
  int nn = 1;
  if (K > 0)
    for (int r = 0; r < ncand[0]; ++r) { f_par[nf] = 0; f_rank[nf] = r; ++nf; }
  while (nn < cap && nf > 0) {
    /* the best frontier entry: highest probability, then shorter, then smaller rank path */
    int bi = 0;
    for (int e = 1; e < nf; ++e) {
      const int pa = f_par[e], pb = f_par[bi];
      const int da = depth[pa], db = depth[pb];
      const int ta = cand[da * cand_k + f_rank[e]], tb = cand[db * cand_k + f_rank[bi]];
      int better;
      if (da != db) {
        const double sa = score[pa] * q[(size_t)da * V + ta];
        const double sb = score[pb] * q[(size_t)db * V + tb];
        better = sa > sb || (sa == sb && da < db);
      } else {
        const double la = lsum[pa] + draft[(size_t)da * V + ta];
        const double lb = lsum[pb] + draft[(size_t)db * V + tb];
        better = la > lb;
        if (la == lb) {
          int cmp = 0;
          for (int j = 0; j < da && cmp == 0; ++j)
            cmp = (ranks[(size_t)pa * K + j] > ranks[(size_t)pb * K + j]) -
                  (ranks[(size_t)pa * K + j] < ranks[(size_t)pb * K + j]);
          better = cmp < 0 || (cmp == 0 && f_rank[e] < f_rank[bi]);
        }
      }
      if (better) bi = e;
    }
    const int pa = f_par[bi], ra = f_rank[bi], d = depth[pa];
    f_par[bi] = f_par[nf - 1];
    f_rank[bi] = f_rank[nf - 1];
    --nf;
    parent[nn] = pa;
    tokens[nn] = cand[d * cand_k + ra];
    depth[nn] = d + 1;
    score[nn] = score[pa] * q[(size_t)d * V + tokens[nn]];
    lsum[nn] = lsum[pa] + draft[(size_t)d * V + tokens[nn]];
    for (int j = 0; j < d; ++j) ranks[(size_t)nn * K + j] = ranks[(size_t)pa * K + j];
    ranks[(size_t)nn * K + d] = ra;
    if (d + 1 < K)
      for (int r = 0; r < ncand[d + 1]; ++r) { f_par[nf] = nn; f_rank[nf] = r; ++nf; }
    ++nn;
  }
  *n_nodes = nn;
  free(q);
  free(cand);
  free(ncand);
  free(ranks);
  free(lsum);
  free(f_par);
  free(f_rank);
  return ORACLE_OK;
}
