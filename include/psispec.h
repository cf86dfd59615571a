/*
 * psispec.h -- C ABI of the B200 (sm_100a) Psi-Spec verification library, libpsispec.so.
 *
 * The operation is the lossless rejection-correction step of Uno's Psi-Spec sampler,
 * "Unlocking Lossless Speedups in LLMs via Discrete Diffusion" (arXiv 2609.04010). The
 * long-form review page (vibe-research.pages.dev, 2026-09-09) states it in section 3.3: the
 * diffusion path drafts a token block; the AR (target) path scores every drafted position;
 * draft token i is accepted with probability min(1, p_AR(x_i) / p_draft(x_i)); the longest
 * prefix before the first rejection is kept; a rejected position is resampled from the
 * normalised residual [p_AR - p_draft]_+; when the whole block is accepted, one extra token is
 * drawn from the last verifier row. Section 3.4 names the linear sampler (one candidate per
 * position) and the tree sampler (several candidate prefixes verified together). The
 * project README's inference example lists the sampling controls --temperature and --top-p.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named *_logits, u_*, temperature, top_p, draft_tokens, node_*, parent, tokens,
 *    out_*, row_stats and workspace are DEVICE pointers owned by the caller. The library
 *    allocates no memory and keeps no state between calls (psispec_verify_linear_static
 *    excepted: it uses one library-owned scratch array per device); it only enqueues kernels
 *    on `stream` (a cudaStream_t; NULL selects the legacy default stream). Calls are
 *    asynchronous: outputs are valid once the stream reaches that point.
 *  - Logit rows are contiguous: row r of a [rows, V] tensor starts at element r * V. dtype is
 *    PSISPEC_F32 or PSISPEC_BF16. Any V >= 1 is accepted; V up to 2^24.
 *  - Temperature T (per request): T == 0 means greedy (a point mass on the lowest-index
 *    maximum); T > 0 divides the logits by T before the softmax over the whole vocabulary.
 *    T < 0, NaN or inf is a per-request data error.
 *  - top_p (per request): in (0, 1); values >= 1 (and NaN) switch the filter off, values <= 0
 *    keep only the maximum's value (with its ties). The kept set is every
 *    token whose logit is >= tau, where tau is the largest logit value whose tie-inclusive
 *    upper-tail probability is >= top_p; the distribution is renormalised over the kept set.
 *    It is applied after the temperature, to the verifier row and to the draft row
 *    separately, and it is a no-op at T == 0. (The pages leave top-p's definition open.)
 *  - top_k (per request, the *_k entry points only; NULL for all requests off): the project
 *    README lists it among the common sampling controls without defining it. Read plainly:
 *    keep every token whose logit is >= the k-th largest logit of the row (ties with it kept
 *    together), after the temperature and before top-p, which then acts on the renormalised
 *    top-k set. k <= 0 or k >= V switches it off; it is a no-op at T == 0.
 *  - Uniforms u are floats in [0, 1) supplied by the caller; the library draws no random
 *    numbers. An inverse-CDF draw with uniform u over weights r returns the first index v, in
 *    vocabulary order, with C(v) > u * Z (C inclusive prefix sum, Z = sum of r), so a token of
 *    zero probability is never returned.
 *  - The accept test for a draft token x is u * q(x) < p(x); with q(x) > 0 this is
 *    u < p(x)/q(x), i.e. acceptance with probability min(1, p/q).
 *  - Data errors found on the device (a NaN or +inf logit, a row with no finite logit, a draft
 *    token outside [0, V), a malformed trie, a bad temperature) affect only the request they
 *    occur in: its accept length is written as -1 and its token outputs as -1.
 *  - Host-side argument errors are returned as a status before anything is enqueued.
 *  - workspace: device scratch of at least psispec_workspace_size(...) bytes, 256-byte
 *    aligned. Its contents need no initialisation and are not meaningful after the call. Two
 *    calls in flight at the same time must not share one workspace.
 */
#ifndef PSISPEC_H
#define PSISPEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PSISPEC_OK = 0,
  PSISPEC_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad dtype, misaligned pointer */
  PSISPEC_ERR_UNSUPPORTED = 2, /* a size beyond the documented limits */
  PSISPEC_ERR_CUDA = 3,        /* a kernel launch failed (cudaGetLastError after the launch) */
  PSISPEC_ERR_WORKSPACE = 4    /* workspace null, too small or not 256-byte aligned */
} psispec_status;

typedef enum { PSISPEC_F32 = 0, PSISPEC_BF16 = 1 } psispec_dtype;

typedef enum {
  PSISPEC_OP_SAMPLE_DRAFT = 0,
  PSISPEC_OP_VERIFY_LINEAR = 1,
  PSISPEC_OP_VERIFY_TREE = 2,
  PSISPEC_OP_ROW_STATS = 3,
  PSISPEC_OP_BUILD_TREE = 4 /* a = B, b = K, c = V */
} psispec_op;

/* Bytes of one per-row statistics record (psispec_sample_draft's out_row_stats,
 * psispec_row_stats' output, psispec_verify_linear's draft_row_stats). Layout, in order:
 *   float m       row maximum of the logits
 *   float c       log2(e) / T (0 for a greedy row)
 *   float s       sum over the row of 2^((l - m) c)
 *   float s_kept  the same sum over the top-p kept set (= s without a cut)
 *   uint32 tau    kept <=> key(l) >= tau, key the order-preserving map of the fp32 bits b
 *                 of l (b | 0x80000000 when the sign bit is clear, ~b when it is set, -0
 *                 taken as +0); tau = 0 keeps every token
 *   int32 amax    lowest index of the maximum (greedy rows), -1 otherwise
 *   int32 status  0, or 1 for a data error in the row
 *   int32 pad
 * so a kept token's probability is 2^((l - m) c) / s_kept. */
#define PSISPEC_ROW_STATS_BYTES 32

/* Human-readable name of a status code (static string, never NULL). */
const char* psispec_status_string(int status);

/* Library ABI version: 100 * major + minor. */
int psispec_version(void);

/* Workspace bytes needed by one call of `op` with these sizes (an upper bound).
 *   SAMPLE_DRAFT:  a = B, b = K (rows = B*K), c = V
 *   VERIFY_LINEAR: a = B, b = K, c = V
 *   VERIFY_TREE:   a = B, b = N (total nodes), c = V
 *   ROW_STATS:     a = B, b = K (rows = B*K), c = V
 * Returns 0 for invalid sizes. */
size_t psispec_workspace_size(int op, int64_t a, int64_t b, int64_t c);

/*
 * psispec_sample_draft -- draw each drafted token from its draft distribution q.
 * Section 3.3 of the review page: the drafted block is a sample of the diffusion path's
 * distribution, after the sampling controls (temperature, top-p).
 *
 *   draft_logits  [B, K, V] dtype   draft (diffusion-path) logits, row i of request b at
 *                                   element (b*K + i) * V
 *   temperature   [B] float, top_p [B] float
 *   u             [B, K] float in [0, 1)     one uniform per drafted position
 *   out_tokens    [B, K] int32      drawn token (-1 on a data error in that row)
 *   out_q         [B, K] float      q(token) after temperature/top-p; may be NULL
 *   out_row_stats [B, K] records of PSISPEC_ROW_STATS_BYTES; may be NULL. When given, they
 *                 can be passed to psispec_verify_linear (draft_row_stats) for the same
 *                 draft logits, temperature and top-p, so that the verifier does not re-read
 *                 the whole draft tensor.
 * Limits: B, K >= 1, B*K <= 2^26, V <= 2^24.
 */
psispec_status psispec_sample_draft(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                    const float* temperature, const float* top_p, const float* u,
                                    int32_t* out_tokens, float* out_q, void* out_row_stats,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * psispec_sample_draft_k -- psispec_sample_draft with a per-request top-k (see the
 * conventions above): top_k [B] int32 device array, or NULL (off for every request). Row
 * statistics records written here carry the top-k threshold and can be passed to
 * psispec_verify_linear_k with the same top_k.
 */
psispec_status psispec_sample_draft_k(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                      const float* temperature, const float* top_p, const int32_t* top_k,
                                      const float* u, int32_t* out_tokens, float* out_q, void* out_row_stats,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * psispec_row_stats -- the per-row statistics of the sampling distribution softmax(l / T)
 * after top-p over the full vocabulary (review page, section 3.3: both distributions of the
 * rule are taken after the sampling controls): row maximum, normaliser, top-p threshold and
 * kept mass, or the argmax of a greedy row. These are the records psispec_sample_draft
 * writes, without the draw; psispec_verify_linear accepts them as draft_row_stats.
 *
 *   logits        [B, K, V] dtype   row i of request b at element (b*K + i) * V
 *   temperature   [B] float, top_p [B] float
 *   out_row_stats [B, K] records of PSISPEC_ROW_STATS_BYTES (16-byte aligned); a row with a
 *                 data error (NaN/+inf logit, no finite logit, bad temperature) gets a
 *                 record whose status field is nonzero
 * Workspace: psispec_workspace_size(PSISPEC_OP_ROW_STATS, B, K, V) bytes.
 * Limits: B, K >= 1, B*K <= 2^26, V <= 2^24.
 */
psispec_status psispec_row_stats(const void* logits, int dtype, int32_t B, int32_t K, int32_t V,
                                 const float* temperature, const float* top_p, void* out_row_stats,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * psispec_row_stats_k -- psispec_row_stats with a per-request top-k (see the conventions
 * above): top_k [B] int32 device array, or NULL (off for every request). The records carry the
 * top-k (then top-p) threshold and serve psispec_verify_linear_k with the same top_k.
 */
psispec_status psispec_row_stats_k(const void* logits, int dtype, int32_t B, int32_t K, int32_t V,
                                   const float* temperature, const float* top_p, const int32_t* top_k,
                                   void* out_row_stats, void* workspace, size_t workspace_bytes, void* stream);

/*
 * psispec_verify_linear -- Psi-Spec linear verification (review page, section 3.3; linear
 * sampler of section 3.4).
 *
 * For request b and drafted position i < K: p_i = verifier distribution of target row i,
 * q_i = draft distribution of draft row i (both after temperature/top-p); x_i =
 * draft_tokens[b, i]. Position i is accepted iff u_accept[b, i] * q_i(x_i) < p_i(x_i). With j
 * the first rejected position (j = K if none), the call emits x_0 .. x_{j-1} and then one
 * more token y: for j < K, y is drawn with u_resid[b, j] from max(0, p_j - q_j) (from p_j if
 * that residual is zero everywhere); for j = K it is the bonus token drawn with
 * u_resid[b, K] from p_K. At T == 0 this reduces to exact argmax matching.
 *
 *   target_logits   [B, K+1, V] dtype    verifier rows (row K is the bonus row)
 *   draft_logits    [B, K, V] dtype      draft rows (only the rejected row is read in full
 *                                        when draft_row_stats is given)
 *   draft_tokens    [B, K] int32
 *   draft_row_stats [B, K] records from psispec_sample_draft over the same draft logits and
 *                   controls, or NULL to recompute them here
 *   u_accept [B, K] float, u_resid [B, K+1] float, temperature [B] float, top_p [B] float
 *   out_tokens      [B, K+1] int32    accepted prefix, then y, then -1 padding
 *   out_accept_len  [B] int32         j, or -1 on a data error
 *   out_p, out_q    [B, K] float      p_i(x_i) and q_i(x_i) for every position; may be NULL
 * Limits: B >= 1, 1 <= K <= 64, B*(K+1) <= 2^26, V <= 2^24.
 */
psispec_status psispec_verify_linear(const void* target_logits, const void* draft_logits, int dtype,
                                     int32_t B, int32_t K, int32_t V, const int32_t* draft_tokens,
                                     const void* draft_row_stats, const float* u_accept,
                                     const float* u_resid, const float* temperature, const float* top_p,
                                     int32_t* out_tokens, int32_t* out_accept_len, float* out_p,
                                     float* out_q, void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * psispec_verify_linear_k -- psispec_verify_linear with a per-request top-k applied to the
 * verifier rows and the draft rows alike: top_k [B] int32 device array, or NULL (off for
 * every request). draft_row_stats, when given, must come from psispec_sample_draft_k with
 * the same top_k. Same workspace size, limits and errors as psispec_verify_linear.
 */
psispec_status psispec_verify_linear_k(const void* target_logits, const void* draft_logits, int dtype,
                                       int32_t B, int32_t K, int32_t V, const int32_t* draft_tokens,
                                       const void* draft_row_stats, const float* u_accept,
                                       const float* u_resid, const float* temperature, const float* top_p,
                                       const int32_t* top_k, int32_t* out_tokens, int32_t* out_accept_len,
                                       float* out_p, float* out_q, void* workspace, size_t workspace_bytes,
                                       void* stream);

/*
 * psispec_verify_tree -- Psi-Spec tree verification (tree sampler of the review page's
 * section 3.4; the pages give no acceptance rule for it, so this is the plainest lossless
 * reading: recursive rejection sampling without replacement over each node's children).
 *
 * Request b owns nodes node_offsets[b] .. node_offsets[b+1]-1; the first one is its root.
 * Every node n has a verifier row target[n] and a draft row draft[n], both distributions of
 * the token that follows the prefix ending at n. The children of n (nodes whose parent is n)
 * carry distinct tokens drawn without replacement from n's draft distribution. The walk
 * starts at the root with r = p_root and q~ = q_root and tries the children in increasing
 * node order: child c with token t is accepted iff u_accept[c] * q~(t) < r(t); then the walk
 * moves to c. On rejection r <- normalise(max(0, r - q~)) (unchanged if that is zero) and
 * q~ <- q~ with t removed, renormalised (when no draft mass is left the remaining children
 * are skipped). When no child is accepted the final token is drawn from r with
 * u_resid[current node]. At T == 0 the child whose token is the verifier's argmax is
 * accepted and the final token is that argmax. With one child per node this is exactly
 * psispec_verify_linear.
 *
 *   target_logits, draft_logits  [N, V] dtype
 *   node_offsets [B+1] int32 (node_offsets[0] = 0, node_offsets[B] = N)
 *   parent       [N] int32   request-local index of the parent, -1 at the root, otherwise
 *                            smaller than the node's own local index
 *   tokens       [N] int32   token appended by each node (ignored at the root)
 *   u_accept [N] float, u_resid [N] float, temperature [B] float, top_p [B] float
 *   max_depth    path-length limit; a trie deeper than this is a data error
 *   out_path       [B, max_depth] int32   local node ids of the accepted path, -1 padded
 *   out_tokens     [B, max_depth+1] int32 accepted tokens, then the final token, -1 padded
 *   out_accept_len [B] int32              number of accepted nodes, -1 on a data error
 * Limits: B >= 1, N >= B, N <= 2^26, 1 <= max_depth <= 64, V <= 2^24. A request with more
 * than 1024 nodes, or a node with more than 64 children, is reported as a data error (-1).
 */
psispec_status psispec_verify_tree(const void* target_logits, const void* draft_logits, int dtype,
                                   int32_t B, int32_t N, int32_t V, const int32_t* node_offsets,
                                   const int32_t* parent, const int32_t* tokens, const float* u_accept,
                                   const float* u_resid, const float* temperature, const float* top_p,
                                   int32_t max_depth, int32_t* out_path, int32_t* out_tokens,
                                   int32_t* out_accept_len, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * psispec_verify_tree_k -- psispec_verify_tree with a per-request top-k applied to every
 * node's verifier and draft rows: top_k [B] int32 device array, or NULL (off for every
 * request). Same workspace size, limits and errors as psispec_verify_tree.
 */
psispec_status psispec_verify_tree_k(const void* target_logits, const void* draft_logits, int dtype,
                                     int32_t B, int32_t N, int32_t V, const int32_t* node_offsets,
                                     const int32_t* parent, const int32_t* tokens, const float* u_accept,
                                     const float* u_resid, const float* temperature, const float* top_p,
                                     const int32_t* top_k, int32_t max_depth, int32_t* out_path,
                                     int32_t* out_tokens, int32_t* out_accept_len, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * psispec_build_tree -- candidate trie of the tree sampler (review page, section 3.4: at every
 * position the top-K tokens, then the V most probable prefixes; the README's tree flags set
 * the two sizes). Readings: position i's distribution is draft row i's q after temperature,
 * top-k and top-p; its candidates are the cand_k kept tokens of largest q (ties to the lower
 * index, q > 0); a prefix's probability is the product of its tokens' q (fp64); the
 * n_prefixes most probable prefixes are kept, ties to the shorter prefix and then to the
 * smaller sequence of candidate ranks, numbered in the order kept (node 0 = the empty prefix,
 * so parents precede children and siblings follow in decreasing probability).
 *
 *   draft_logits  [B, K, V] dtype   draft rows of the K drafted positions of each request
 *   temperature [B] float, top_p [B] float, top_k [B] int32 or NULL
 *   out_parent, out_tokens, out_depth  [B, n_prefixes + 1] int32 (root: -1, -1, 0; slots
 *                 beyond the node count: -1)
 *   out_score     [B, n_prefixes + 1] double, prefix probabilities; may be NULL
 *   out_nodes     [B] int32 node count (1 + kept prefixes), or -1 when a draft row of the
 *                 request has a data error
 * Workspace: psispec_workspace_size(PSISPEC_OP_BUILD_TREE, B, K, V) bytes.
 * Limits: 1 <= K <= 16, 1 <= cand_k <= 32, 1 <= n_prefixes <= 64, B*K <= 2^26, V <= 2^24.
 * The trie's node arrays plug into psispec_verify_tree (node_offsets b*(n_prefixes+1) with
 * the unused slots trimmed by the caller).
 */
psispec_status psispec_build_tree(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                  const float* temperature, const float* top_p, const int32_t* top_k,
                                  int32_t cand_k, int32_t n_prefixes, int32_t* out_parent, int32_t* out_tokens,
                                  int32_t* out_depth, double* out_score, int32_t* out_nodes, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * psispec_verify_tree_det -- tree verification of a trie whose children were fixed in advance
 * (the candidate trie of psispec_build_tree): rejection sampling with point-mass proposals.
 * At a node with verifier distribution p (after temperature, top-k, top-p), child t (in node
 * order) is accepted iff u_accept[t] < r(t), r = p without the siblings rejected before it,
 * renormalised; where the walk stops the final token is drawn from that r with the node's
 * u_resid (-1 if the rejected siblings held all of p's mass). No draft rows are read.
 * Arguments, outputs, limits and errors as psispec_verify_tree (top_k may be NULL).
 */
psispec_status psispec_verify_tree_det(const void* target_logits, int dtype, int32_t B, int32_t N, int32_t V,
                                       const int32_t* node_offsets, const int32_t* parent, const int32_t* tokens,
                                       const float* u_accept, const float* u_resid, const float* temperature,
                                       const float* top_p, const int32_t* top_k, int32_t max_depth,
                                       int32_t* out_path, int32_t* out_tokens, int32_t* out_accept_len,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * psispec_verify_linear_static -- psispec_verify_linear without a caller workspace.
 *
 * The pages have no counterpart to this call: it is an integration convenience. It runs
 * exactly psispec_verify_linear, with its scratch in one file-scope device array of
 * PSISPEC_STATIC_WORKSPACE_BYTES bytes inside the library instead of a caller buffer. It
 * allocates nothing: no cudaMalloc, no cudaFree. It serves callers that cannot allocate
 * device memory on the calling path, e.g. a host program that links only this library and
 * has no device allocator of its own, or a serving loop that must not let cudaMalloc or
 * cudaFree synchronise the device between steps.
 *
 * Set-up: the first call on a device looks up the array's device address with
 * cudaGetSymbolAddress (this may load the library's device code) and caches it for that
 * device. Make that first call, on every device used, before any stream capture begins.
 * Nothing in the array needs to start at zero: the call's first kernel clears the per-request
 * arrival counters, and everything else is written before it is read.
 *
 * The array is shared by every call on one device: two calls whose executions overlap (on
 * different streams, or from different threads) race on it and give undefined results. Calls
 * on one stream run one after another and are safe.
 *
 * Arguments, outputs and limits as for psispec_verify_linear. In addition, a size whose
 * psispec_workspace_size(PSISPEC_OP_VERIFY_LINEAR, B, K, V) exceeds
 * PSISPEC_STATIC_WORKSPACE_BYTES is rejected with PSISPEC_ERR_UNSUPPORTED before anything
 * is enqueued (e.g. B = 64, K = 8, V = 151936 needs about 3 MB; B = 512, K = 16 does not fit).
 * If the device address cannot be obtained the call returns PSISPEC_ERR_CUDA.
 */
#define PSISPEC_STATIC_WORKSPACE_BYTES (16u << 20)

psispec_status psispec_verify_linear_static(const void* target_logits, const void* draft_logits, int dtype,
                                            int32_t B, int32_t K, int32_t V, const int32_t* draft_tokens,
                                            const void* draft_row_stats, const float* u_accept,
                                            const float* u_resid, const float* temperature,
                                            const float* top_p, int32_t* out_tokens, int32_t* out_accept_len,
                                            float* out_p, float* out_q, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* PSISPEC_H */
