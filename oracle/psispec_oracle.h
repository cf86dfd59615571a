/*
 * psispec_oracle.h -- plain, slow fp64 CPU oracle of the Psi-Spec verification step.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library. It shares no code, header, table or constant with the CUDA
 * library; neither side includes or links the other.
 *
 * Source of the method: "Unlocking Lossless Speedups in LLMs via Discrete Diffusion"
 * (arXiv 2609.04010), long-form review page (vibe-research.pages.dev, silicon-writer,
 * 2026-09-09), section 3.3 "Psi-Spec": draft block sampled from the diffusion path; accept
 * draft token i with probability min(1, p_AR(x_i)/p_draft(x_i)); keep the longest prefix
 * before the first rejection; on rejection resample from the normalised residual
 * [p_AR - p_draft]_+; if the whole block is accepted, draw one more token from the last
 * verifier row. Section 3.4 names the linear and tree samplers (the tree rule itself is not
 * stated on the pages; the reading used here is recursive rejection without replacement
 * over the sibling candidates).
 *
 * All randomness is an explicit input: every uniform u is a double in [0, 1).
 * Logits are passed as doubles (bf16 and fp32 inputs convert to double exactly).
 *
 * "band" outputs: for every request (or draft row) the smallest distance, over the decisions
 * on the oracle's own path, between a uniform and the quantity it is compared against:
 *   E1 |u - p/q|               for each accept test (q > 0),
 *   E2 |C(y-1)/Z - u|, |C(y)/Z - u|   for each inverse-CDF draw,
 *   E3 |tail(tau)/S - top_p|, |tail(tau+)/S - top_p|   for each top-p threshold used.
 * A comparison whose band is below the agreed tolerance may legitimately differ between
 * two correct implementations with different rounding. The optional band_kind outputs (NULL:
 * not wanted) name the kind of the decision that gives the band: ORACLE_BAND_E1, _E2 or _E3,
 * or ORACLE_BAND_NONE when the path holds no decision (or on a data error).
 */
#ifndef PSISPEC_ORACLE_H
#define PSISPEC_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. Per-request data errors are reported through accept_len = -1 instead. */
#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* Kinds of decision behind a band (band_kind outputs). */
#define ORACLE_BAND_NONE 0
#define ORACLE_BAND_E1 1 /* accept test |u - p/q| */
#define ORACLE_BAND_E2 2 /* inverse-CDF draw edge */
#define ORACLE_BAND_E3 3 /* top-p tail against top_p */

/* One row's distribution after temperature T and top-p.
 * l[V] logits; T == 0 means greedy (a point mass on the lowest-index maximum).
 * top_p >= 1 disables the filter. out[V] receives probabilities (sum 1).
 * *band receives the E3 margin (+inf when the filter is off).
 * Returns 0, or -1 for a bad row (NaN or +inf logit, or no finite logit). */
int oracle_row_dist(const double* l, int V, double T, double top_p, double* out, double* band);

/* oracle_row_dist with top-k first: the tokens whose logit is >= the k-th largest logit of the
 * row (ties kept together) stay, then top-p acts on that renormalised set (its E3 margin
 * relative to the set's mass). top_k <= 0 or >= V is off; a no-op at T == 0. */
int oracle_row_dist_k(const double* l, int V, double T, double top_p, int top_k, double* out, double* band);

/* Inverse-CDF draw in vocabulary order: y = min{v : C(v) > u * Z}, C inclusive.
 * r[V] >= 0 need not be normalised. If no index qualifies (rounding), y is the last v with
 * r[v] > 0. Returns y, or -1 when Z == 0. *band receives the E2 margin. */
int oracle_inverse_cdf(const double* r, int V, double u, double* band);

/* Draft sampling, one draw per row.
 * draft[rows*V]; row_req[rows] maps a row to its request for temperature[]/top_p[]/top_k[]
 * (top_k may be NULL: off for every request);
 * u[rows]. Outputs: tokens[rows] (-1 on a bad row), q_at[rows] = q(token), band[rows],
 * band_kind[rows] (nullable). */
int oracle_sample_draft(const double* draft, int rows, int V, const int* row_req,
                        const double* temperature, const double* top_p, const int* top_k, const double* u,
                        int* tokens, double* q_at, double* band, int* band_kind);

/* Linear verification.
 * target[B*(K+1)*V], draft[B*K*V], draft_tokens[B*K], u_accept[B*K], u_resid[B*(K+1)],
 * temperature[B], top_p[B], top_k[B] or NULL (top-k off).
 * Outputs: out_tokens[B*(K+1)] (accepted prefix, then the resampled or bonus token, then -1),
 * accept_len[B] (-1 on a data error), out_p[B*K] = p_i(x_i), out_q[B*K] = q_i(x_i),
 * band[B] = smallest E1/E2/E3 margin on the request's path,
 * pq_band[B*K] = E3 margin of the two rows behind out_p/out_q at that position,
 * band_kind[B] (nullable) = the kind of decision that gives band[b]. */
int oracle_verify_linear(const double* target, const double* draft, int B, int K, int V,
                         const int* draft_tokens, const double* u_accept, const double* u_resid,
                         const double* temperature, const double* top_p, const int* top_k,
                         int* out_tokens, int* accept_len, double* out_p, double* out_q,
                         double* band, double* pq_band, int* band_kind);

/* Tree verification (recursive rejection without replacement over siblings).
 * node_offsets[B+1]: request b owns nodes [node_offsets[b], node_offsets[b+1]); the first is
 * its root. parent[N]: local index of the parent (-1 at the root, otherwise < own local
 * index). tokens[N]: token that node appends (root's ignored). target[N*V], draft[N*V]:
 * the next-token rows at each node. u_accept[N] is consumed when a node is tested as a
 * candidate child; u_resid[N] when the final draw happens at that node.
 * Outputs: out_path[B*max_depth] local node ids of the accepted path (-1 padded),
 * out_tokens[B*(max_depth+1)], accept_len[B] (-1 on a data error), band[B], band_kind[B]
 * (nullable). */
int oracle_verify_tree(const double* target, const double* draft, int B, int V,
                       const int* node_offsets, const int* parent, const int* tokens,
                       const double* u_accept, const double* u_resid,
                       const double* temperature, const double* top_p, const int* top_k, int max_depth,
                       int* out_path, int* out_tokens, int* accept_len, double* band, int* band_kind);

/* Candidate rules of tree verification (oracle_verify_tree_rule). */
#define ORACLE_TREE_SAMPLED_WOR 0    /* children drawn from q without replacement (R7) */
#define ORACLE_TREE_DETERMINISTIC 1  /* children fixed in advance (top-k / best prefixes) */
#define ORACLE_TREE_SAMPLED_WR 2     /* children drawn from q independently, with replacement */

/* Tree verification under a candidate rule: ORACLE_TREE_SAMPLED_WOR is oracle_verify_tree;
 * ORACLE_TREE_DETERMINISTIC tests child t with u < r(t) and on rejection removes t from r and
 * renormalises (the draft rows are not read); ORACLE_TREE_SAMPLED_WR tests u q(t) < r(t) and
 * on rejection sets r <- norm([r - q]_+) with q unchanged. Same arguments and outputs as
 * oracle_verify_tree; an unknown rule is ORACLE_BAD_ARG. */
int oracle_verify_tree_rule(const double* target, const double* draft, int B, int V,
                            const int* node_offsets, const int* parent, const int* tokens,
                            const double* u_accept, const double* u_resid,
                            const double* temperature, const double* top_p, const int* top_k, int max_depth,
                            int rule, int* out_path, int* out_tokens, int* accept_len, double* band,
                            int* band_kind);

/* Candidate trie of the tree sampler from the draft rows of K positions (draft[K*V], after
 * temperature/top-p/top-k): the cand_k most probable tokens per position, then the n_prefixes
 * most probable prefixes (product of the q_i; ties to the shorter prefix, then to the smaller
 * candidate ranks), as a trie whose node 0 is the empty prefix and whose nodes follow in the
 * order kept. Outputs have room for n_prefixes + 1 nodes: parent (-1 at the root), tokens (-1
 * at the root), depth, score (prefix probability); *n_nodes receives the node count. Returns
 * ORACLE_OK, ORACLE_BAD_ARG, or -1 for a bad draft row. */
int oracle_build_tree(const double* draft, int K, int V, double T, double top_p, int top_k, int cand_k,
                      int n_prefixes, int* parent, int* tokens, int* depth, double* score, int* n_nodes);

#ifdef __cplusplus
}
#endif
#endif
