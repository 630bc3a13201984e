/*
 * ckv_oracle.h -- CPU oracle for CommunityKV's per-step community-retrieval
 * sparse decode and its prefill top-kappa graph.
 *
 * TEST INFRASTRUCTURE ONLY. This is the plain, slow, single-threaded
 * statement of what the method computes, used to check the CUDA library.
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may call it. It shares no code, header, table or constant with the CUDA
 * library, and the library never calls it.
 *
 * Source: "CommunityKV: Efficient Long-Context Decoding via Graph
 * Partitioning" -- the abstract (local update rule, query-group graphs),
 * Figure 1's caption (steps (1) graph construction, (2) initial
 * partitioning with one centroid per community, (3) incremental update) and
 * Table 1 (O(d) per-step update, O(sqrt(n) d) retrieval).  The pages leave
 * many steps open; each function below states the reading it implements.
 *
 * Precision: the pages fix none.  Values are computed in double; a value
 * that decides an integer (a ranking, an argmax) is rounded to the float
 * the CUDA kernels rank in, and the ranking is taken on that float.  The
 * community centroids are stored as float (their storage type) and every
 * update of them is computed in double and rounded once.
 *
 * Parity pins: every function here is pinned by a test in tests/ against
 * brute force, a closed form or a library routine (see test_oracle_*.py).
 */
#ifndef CKV_ORACLE_H
#define CKV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { CKVO_F32 = 0, CKVO_BF16 = 1 };
enum { CKVO_KMAX = 64 };   /* largest kappa the oracle accepts */

typedef struct ckvo_graph ckvo_graph;   /* one graph's community state */

/* Result record of one decode step, with the cutoff gaps the parity checker
 * uses to recognise a near-tie (relative gap = |a-b| / max(|a|,|b|)). */
typedef struct {
    int32_t C;            /* communities selected                           */
    int32_t T;            /* member tokens selected                         */
    float   cut_gap_lo;   /* score gap: last kept vs first dropped (+inf if none dropped) */
    float   cut_gap_hi;   /* score gap: first dropped vs the next one (+inf if none)      */
    int32_t n_edges;      /* min(kappa, T)                                  */
    int32_t edge_col[CKVO_KMAX];   /* token ids, rank order                 */
    float   edge_w[CKVO_KMAX];     /* aggregated attention probability      */
    int32_t edge_comm[CKVO_KMAX];  /* community of each edge token          */
    float   edge_gap;     /* w gap at rank kappa-1 vs kappa (+inf if T <= kappa) */
    int32_t assigned;     /* community the new token joined                 */
    double  vote_gap;     /* relative gap between best and second vote (+inf if one) */
    double  m[CKVO_KMAX]; /* per-head softmax max of z (for the checker)     */
    double  l[CKVO_KMAX]; /* per-head softmax denominator sum exp(z - m)    */
} ckvo_step_info;

/* ---- graph state ------------------------------------------------------ */
ckvo_graph* ckvo_graph_new(int n_comm, int head_dim, int n_max);
void        ckvo_graph_free(ckvo_graph* g);
int         ckvo_graph_ntok(const ckvo_graph* g);      /* tokens assigned + sinks */

/* Initial partition (Figure 1, step (2)): members of community c are the
 * positions j >= S with labels[j] == c, ascending; centroid = mean of member
 * keys.  Returns 0, or -1 on a label outside [0, n_comm). */
int ckvo_init(ckvo_graph* g, int n, int n_sinks, const int32_t* labels,
              const void* K, int kv_dtype);

/* Read-out of the state (host buffers). members: all members, community by
 * community in id order, ascending within a community; returns their count. */
void ckvo_get_centroids(const ckvo_graph* g, float* mu /* [Nc][D] */);
void ckvo_get_sizes(const ckvo_graph* g, int32_t* size /* [Nc] */);
int  ckvo_get_members(const ckvo_graph* g, int32_t* members);
/* Overwrite the state from the same interchange form (used by the checker
 * to re-synchronise after an exempt near-tie). Returns 0 or -1. */
int  ckvo_set_state(ckvo_graph* g, int n_tok, const float* mu, const int32_t* size,
                    const int32_t* members);

/* ---- decode step pieces (Figure 1, step (3)) -------------------------- */
/* a1: s_c = sum over the graph's heads of q_h . mu_c (double, rounded to
 * float); empty communities score -inf. */
void ckvo_score(const ckvo_graph* g, int n_heads, const void* q, int q_dtype,
                float* s /* [Nc] */);
/* a2: order non-empty communities by (s desc, id asc) and keep the longest
 * prefix whose sizes sum to <= budget, at least one.  Writes the kept ids in
 * that order to sel; returns C and the two cutoff gaps. */
int  ckvo_select(int n_comm, const float* s, const int32_t* size, int budget,
                 int32_t* sel, float* gap_lo, float* gap_hi);
/* a3: exact softmax attention of n_heads queries over the rows listed in
 * `rows` (token positions into K, V; row stride D).  out [H][D] float.
 * If p is not NULL it receives the probabilities [H][R] (double);
 * m, l receive the per-head max and denominator. */
void ckvo_attend(int n_heads, int D, const void* q, int q_dtype,
                 const void* K, const void* V, int kv_dtype,
                 const int32_t* rows, int R, float* out, double* p,
                 double* m, double* l);
/* a4: top-kappa of the candidates by (w desc, token asc), w = float(sum_h p). */
int  ckvo_topk(int R, const float* w, const int32_t* tok, int kappa,
               int32_t* out_idx /* indices into the candidate arrays */, float* gap);
/* a5: weighted plurality over the edges in rank order; ties to lower id. */
int  ckvo_vote(int n_edges, const int32_t* edge_comm, const float* edge_w,
               double* gap);
/* a6: running-mean centroid update and member append for token t. */
int  ckvo_update(ckvo_graph* g, int c, int t, const void* k_t, int kv_dtype);

/* The whole step for one graph: cache length n (new token at t = n-1, its
 * K/V already in the cache).  q [H][D]; K, V rows [0, n) of the graph's KV
 * head; out [H][D].  sel receives the selected community ids (>= Nc slots).
 * Returns 0, or -1 if n != tokens assigned + sinks + 1. */
int  ckvo_decode_step(ckvo_graph* g, int n_heads, int n_sinks, int kappa, int budget,
                      int n, const void* q, const void* K, const void* V, int dtype,
                      float* out, int32_t* sel, ckvo_step_info* info);

/* ---- prefill graph (Figure 1, step (1)) ------------------------------- */
/* Closed-form CSR degree of row i: min(kappa, max(0, i - S)). */
int64_t ckvo_row_ptr(int64_t i, int n_sinks, int kappa);
/* For each listed row i of one head: z_ij = q_i.k_j / sqrt(D), softmax over
 * j in [0, i]; edges = top-kappa of j in [S, i-1] by (float z desc, j asc),
 * weight p_ij.  col/w are [n_rows][kappa]; deg[r] edges are valid; gap[r] is
 * the relative z gap at the cutoff (+inf when all candidates are kept). */
void ckvo_prefill_rows(int n, int D, int n_sinks, int kappa, const void* Q, const void* K,
                       int dtype, const int32_t* rows, int n_rows,
                       int32_t* col, float* w, int32_t* deg, float* gap);

/* Dense softmax statistics over every position [0, n) of K, per head (the
 * denominator of the attention-mass recall; see ckv_oracle.c). */
void ckvo_dense_stats(int n_heads, int D, const void* q, int q_dtype, const void* K, int kv_dtype, int n,
                      double* m_out, double* l_out);

/* Query-group aggregated prefill rows: the group's nh heads (Q [nh][n][D])
 * share one graph over K [n][D]; w_ij = sum_h p_hij, top-kappa of j in
 * [S, i-1] by (w desc, j asc).  Outputs as ckvo_prefill_rows. */
void ckvo_prefill_rows_grouped(int n, int D, int n_sinks, int kappa, int nh, const void* Q, const void* K,
                               int dtype, const int32_t* rows, int n_rows,
                               int32_t* col, float* w, int32_t* deg, float* gap);

/* Leiden partition of a top-kappa token graph (leiden_oracle.c): the
 * directed CSR (row_ptr [n+1], col, w) read as an undirected weighted graph;
 * modularity quality with resolution gamma; the deterministic variant
 * described in leiden_oracle.c.  labels [n] get community ids 0..C-1 by
 * first appearance; returns C. */
int ckvo_leiden(int n, const int64_t* row_ptr, const int32_t* col, const float* w, double gamma, int max_levels,
                int32_t* labels);
/* Modularity with resolution gamma of a labelling of the same graph:
 * (in - gamma sum_c K_c^2 / (4m)) / m. */
double ckvo_modularity(int n, const int64_t* row_ptr, const int32_t* col, const float* w, const int32_t* labels,
                       double gamma);

#ifdef __cplusplus
}
#endif
#endif
