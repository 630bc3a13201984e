/*
 * ckv.h -- C ABI of libckv: CommunityKV community-retrieval sparse decode
 * attention and prefill top-kappa graph construction for NVIDIA B200
 * (sm_100a).
 *
 * Method: "CommunityKV: Efficient Long-Context Decoding via Graph
 * Partitioning".  Figure 1's caption gives the three stages: (1) during
 * prefill each query connects to its top-kappa keys of the attention matrix,
 * sinks excluded; (2) the token graph is partitioned into communities (the
 * Leiden partition arrives here as a label array) and each community gets a
 * centroid; (3) at each decode step the query is scored against the
 * centroids, the best communities up to a token budget are retrieved, exact
 * attention runs over them plus the sink tokens, and the new token's
 * top-kappa keys become its edges and assign it to a community in constant
 * time (abstract: "a local update rule").  Table 1 gives the costs: O(d)
 * update, O(sqrt(n) d) retrieval.
 *
 * Conventions for every call:
 *  - Pointers named "host" are host memory; all other data pointers are
 *    device memory on the context's device.  The caller owns every buffer it
 *    passes; the context owns the community state and its scratch.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous on it unless stated otherwise.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns CKV_ERR_INVALID_ARG and launches nothing.
 *  - Errors found on the device (label out of range, community storage
 *    exhausted) set the context's error word.  They surface at the next
 *    ckv_last_error(), and every later call of that context then returns
 *    the same error until ckv_init_communities() or ckv_import_state().
 *  - No call aborts, traps or prints.
 *  - Calls that allocate device memory (ckv_create, ckv_init_communities,
 *    ckv_import_state, ckv_refresh, ckv_graph_modularity) allocate before
 *    they change the context, so CKV_ERR_OOM leaves its state as it was.
 *    For tests of that path, CKV_FAULT_ALLOC=k in the environment makes the
 *    k-th device allocation inside each such call fail as out of memory.
 *  - A context is not thread-safe; use one context per host thread.
 */
#ifndef CKV_H
#define CKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CKV_OK = 0,
    CKV_ERR_INVALID_ARG = 1,  /* a pointer, size or configuration is out of range        */
    CKV_ERR_CAPACITY = 2,     /* community member storage of a graph is exhausted        */
    CKV_ERR_OOM = 3,          /* device or host allocation failed                        */
    CKV_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, copy, sync)         */
    CKV_ERR_TIMEOUT = 5,      /* a bounded device wait ran out                           */
    CKV_ERR_STATE = 6         /* call out of order (e.g. step before init, wrong n)      */
} ckv_status;

typedef enum { CKV_F32 = 0, CKV_BF16 = 1 } ckv_dtype;

/* Graph aggregation (abstract: "one graph per query head" versus
 * "query-group graph aggregation").  PER_HEAD: one graph per (batch, query
 * head).  QUERY_GROUP: one graph per (batch, KV head), shared by the query
 * heads of its group; the group's scores and edge weights are sums over
 * its heads. */
typedef enum { CKV_PER_HEAD = 0, CKV_QUERY_GROUP = 1 } ckv_graph_mode;

typedef struct {
    int batch;            /* B >= 1                                                   */
    int n_q_heads;        /* H_q >= 1                                                 */
    int n_kv_heads;       /* H_kv >= 1, H_q % H_kv == 0; QUERY_GROUP: H_q/H_kv in {1,2,4,8} */
    int head_dim;         /* D; must be 128                                           */
    int n_max;            /* rows of the caller's K/V caches per (batch, KV head)     */
    int max_communities;  /* most communities a graph may have (1 .. 16384; the
                             selection keeps one graph's scores in shared memory)    */
    int n_sinks;          /* S >= 0: positions [0, S) are always attended            */
    int kappa;            /* edges per new token, 1..32 (the pages default to 8)      */
    int budget;           /* token budget T_b >= 1 for the retrieved communities     */
    int slack;            /* spare member slots given to each community at init      */
    ckv_dtype kv_dtype;   /* element type of q, K and V                                */
    ckv_graph_mode mode;
    int device;           /* CUDA device ordinal of every device pointer              */
    int pool_capacity;    /* member slots per graph; 0 = automatic, enough for any
                             sequence of steps up to n_max: 5*n_max +
                             max_communities*(slack+32).  A smaller value bounds
                             memory; running out is reported as CKV_ERR_CAPACITY.  */
} ckv_config;

typedef struct ckv_ctx ckv_ctx;   /* opaque; owns all community state and scratch */

/* Number of graphs G of a configuration: B*H_kv (QUERY_GROUP) or B*H_q
 * (PER_HEAD).  Returns -1 for an invalid mode. */
int ckv_graph_count(const ckv_config* cfg);

/* Allocate a context and all its device state for cfg (synchronous).
 * Errors: CKV_ERR_INVALID_ARG (cfg out of range), CKV_ERR_OOM, CKV_ERR_CUDA. */
ckv_status ckv_create(const ckv_config* cfg, ckv_ctx** out);

/* Free a context (synchronises its device first).  NULL is ignored. */
void ckv_destroy(ckv_ctx* ctx);

/* Prefill graph construction -- Figure 1, step (1): for each head and each
 * causal query row i of Q, z_ij = q_i.k_j / sqrt(D) for j <= i; the row's
 * edges are its top-kappa keys j in [S, i-1] (sinks and self excluded) by
 * (z desc, j asc), weighted by the softmax probability over j in [0, i].
 * Q, K: [n_heads][n][D] bf16 (dtype must be CKV_BF16, D = 128), device.
 * Outputs (caller-allocated, device):
 *   row_ptr [n_heads][n+1] int64: offsets of row i within its head's edges,
 *           row i holding min(kappa, max(0, i - S)) edges (closed form);
 *   col     [n_heads][E] int32 and w [n_heads][E] float, E = row_ptr[h][n],
 *           each row's edges in rank order.
 * The n x n score matrix is never stored.  Stateless, asynchronous.
 * Errors: CKV_ERR_INVALID_ARG, CKV_ERR_CUDA. */
ckv_status ckv_build_graph(int n_heads, int n, int head_dim, int n_sinks, int kappa,
                           ckv_dtype dtype, const void* Q, const void* K,
                           int64_t* row_ptr, int32_t* col, float* w, void* stream);

/* Query-group aggregated prefill graph -- the abstract's query-group graph
 * aggregation applied to Figure 1, step (1): one graph per KV head, shared
 * by its `group` query heads.  For row i every head h of the group has its
 * own causal softmax p_hij over j in [0, i] (z_hij = q_hi.k_j / sqrt(D));
 * the edge weight is w_ij = sum_h p_hij and the row's edges are its
 * top-kappa j in [S, i-1] by (w desc, j asc).  With group = 1 this is
 * ckv_build_graph with the weights ranked instead of the scores.
 * Q: [n_kv_heads * group][n][D] bf16 (query heads u*group .. u*group+group-1
 * belong to KV head u), K: [n_kv_heads][n][D] bf16, device.  group is 1, 2
 * or 4.  workspace: device scratch of ckv_build_graph_grouped_workspace()
 * bytes, 16-byte aligned, owned by the caller (per-head row statistics of
 * the first pass; undefined afterwards).  Outputs as ckv_build_graph, per
 * KV head: row_ptr [n_kv_heads][n+1], col and w [n_kv_heads][E].  Two
 * kernels (row statistics, then the grouped graph on the tensor cores); the
 * n x n matrices are never stored.  Asynchronous.  A bounded wait that runs
 * out marks row_ptr[u][0] = -1.
 * Errors: CKV_ERR_INVALID_ARG, CKV_ERR_CUDA. */
size_t ckv_build_graph_grouped_workspace(int n_kv_heads, int group, int n);
ckv_status ckv_build_graph_grouped(int n_kv_heads, int group, int n, int head_dim, int n_sinks, int kappa,
                                   ckv_dtype dtype, const void* Q, const void* K, void* workspace,
                                   int64_t* row_ptr, int32_t* col, float* w, void* stream);

/* Leiden partition of a prefill token graph -- Figure 1, step (2) ("the
 * token graph is partitioned with Leiden"), run on the host as the pages
 * do.  Input: one graph of ckv_build_graph's output copied to host memory
 * (row_ptr_host [n+1], col_host and w_host [row_ptr_host[n]]), read as an
 * undirected weighted graph: an edge i -> j of weight w adds w between i
 * and j.  Quality: modularity with resolution gamma > 0.  The algorithm is
 * Leiden's local moving, refinement and aggregation, repeated from its own
 * result until it no longer changes, with every choice deterministic:
 *   - nodes go through the queue and the refinement in ascending id;
 *   - a node moves to the neighbouring community of largest gain, ties to
 *     staying, then to the lower id;
 *   - the refinement takes the largest positive gain (zero randomness);
 *   - all sums are taken in a fixed order.
 * Output: labels_host [n], community ids 0..C-1 by first appearance, and
 * *n_communities = C; the labels feed ckv_init_communities (sinks' labels
 * are ignored there).  Synchronous, host only.
 * Errors: CKV_ERR_INVALID_ARG (n < 1, gamma not finite and positive,
 * row_ptr not monotone, a column outside [0, n), a weight not finite and
 * non-negative), CKV_ERR_OOM. */
ckv_status ckv_leiden(int n, const int64_t* row_ptr_host, const int32_t* col_host, const float* w_host,
                      double gamma, int32_t* labels_host, int* n_communities);

/* Modularity of a partition of that graph -- Figure 3 (left) tracks it over
 * generation.  Q = (in - gamma * sum_c K_c^2 / (4m)) / m over the graph read
 * as in ckv_leiden: m is the total edge weight, in the weight of edges
 * whose ends share a label, K_c the summed degree of community c.
 * row_ptr, col, w, labels [n] (each in [0, n_communities)) are device
 * memory; workspace: ckv_modularity_workspace(n_communities) bytes of
 * device scratch, 8-byte aligned.  Computed on the device in double; the
 * call synchronises `stream` and writes Q to *q_host.
 * Errors: CKV_ERR_INVALID_ARG (including a label or column out of range,
 * found on the device), CKV_ERR_CUDA. */
size_t ckv_modularity_workspace(int n_communities);
ckv_status ckv_modularity(int n, const int64_t* row_ptr, const int32_t* col, const float* w,
                          const int32_t* labels, int n_communities, double gamma, void* workspace,
                          double* q_host, void* stream);

/* Token graph of the context, for refresh and modularity.  Registers each
 * graph's token graph over positions [0, n) on the host (copied): the
 * prefill graph in the layout of ckv_build_graph, row_ptr_host [G][n+1]
 * (each starting at 0) and col_host, w_host [G][E] with E = row_ptr_host[n]
 * (graph 0's count, the stride of every graph).  Allowed right after
 * ckv_init_communities(..., n) and before any decode step (n must be the
 * init's n).  Synchronous, host only.
 * Errors: CKV_ERR_INVALID_ARG (layout, a column outside [0, n), a weight
 * not finite and non-negative), CKV_ERR_STATE. */
ckv_status ckv_set_token_graph(ckv_ctx* ctx, const int64_t* row_ptr_host, const int32_t* col_host,
                               const float* w_host, int n);

/* Refresh -- Tables 8-9 compare periodic re-partitioning with the
 * incremental update of step (3).  Each graph's token graph is extended by
 * the decode-time rows the context recorded since the last init (the new
 * tokens' top-kappa edges).  It is then partitioned again with ckv_leiden
 * (gamma; the graphs on parallel host threads), and the communities are
 * re-initialised from the new labels over [0, n_tok) with the keys K, as
 * ckv_init_communities does.  Decoding continues with the next n.
 * n_communities_host [G] (may be NULL) gets each graph's count.  Requires a
 * registered token graph covering [0, n_init) (ckv_set_token_graph, or the
 * previous refresh).  Synchronous.
 * Errors: CKV_ERR_INVALID_ARG, CKV_ERR_STATE (no token graph, a step half
 * done), CKV_ERR_CAPACITY (more communities than max_communities: the state
 * is kept), CKV_ERR_OOM, CKV_ERR_CUDA, sticky device errors. */
ckv_status ckv_refresh(ckv_ctx* ctx, const void* K, double gamma, int32_t* n_communities_host, void* stream);

/* Modularity (ckv_modularity, on the device) of each graph's current
 * partition on its current token graph: the registered rows plus the
 * decode-time rows, with the community of every position the incremental
 * update gave it (sinks alone).  q_host [G].  Synchronous (allocates and
 * frees device scratch).
 * Errors: as ckv_refresh, CKV_ERR_CUDA. */
ckv_status ckv_graph_modularity(ckv_ctx* ctx, double gamma, double* q_host, void* stream);

/* Initial partition -- Figure 1, step (2): community c of graph g holds the
 * positions j in [S, n) with labels[g][j] == c (ascending); its centroid is
 * the mean of those keys (float, summed in double).  labels: int32
 * [G][n] (graph-major), host (labels_on_device = 0) or device memory.
 * K: the caller's key cache [B][H_kv][n_max][D] with rows [0, n) filled.
 * Resets the context: previous state, pending steps and errors are dropped.
 * Synchronous (returns after the device work has finished).
 * Errors: CKV_ERR_INVALID_ARG (a label outside [0, n_communities), n, or
 * n_communities out of range), CKV_ERR_CAPACITY, CKV_ERR_OOM, CKV_ERR_CUDA. */
ckv_status ckv_init_communities(ckv_ctx* ctx, const int32_t* labels, int labels_on_device,
                                int n_communities, const void* K, int n, void* stream);

/* Decode step -- Figure 1, step (3): for every graph, score the query
 * against every community centroid (QUERY_GROUP: summed over the group's
 * heads), keep communities in (score desc, id asc) order while their sizes
 * fit the budget (at least one), run exact softmax attention of each query
 * head over the sinks, the kept members and the new token; then (Figure 1,
 * step (3) end, and Table 1's O(d) update) rank the kept members by their
 * attention weight summed over the graph's heads, record the top kappa as
 * the new token's edges, assign the token to the community with the largest
 * summed edge weight (ties to the lower id) and update that centroid's
 * running mean mu + (k - mu) / (m + 1), k being row n-1 of K.
 * q: [B][H_q][D] (kv_dtype); K, V: caches [B][H_kv][n_max][D] whose row
 * n-1 already holds the new token; n: cache length including the new token;
 * it must be one more than after the previous step (or init).
 * out: [B][H_q][D] float32, device.  Asynchronous.
 * Errors: CKV_ERR_INVALID_ARG, CKV_ERR_STATE (no init, wrong n, or the
 * previous step's ckv_assign_update missing), sticky device errors;
 * community storage exhaustion is reported by the next ckv_last_error() as
 * CKV_ERR_CAPACITY and leaves that graph's state as it was before the
 * step. */
ckv_status ckv_decode_step(ckv_ctx* ctx, const void* q, const void* K, const void* V, int n,
                           float* out, void* stream);

/* Closes the decode step begun by ckv_decode_step with the same n: the new
 * token's top-kappa edges over the kept members, its community by the
 * weighted vote of their communities, and the centroid update and append
 * (Figure 1 caption, step (3); abstract, "a local update rule").  Launches
 * one kernel (one CTA per graph) on `stream` at the lowest stream priority;
 * it reads the new token's key from row n-1 of K and what the step's
 * attention kernel left.  The step's output needs none of it, so a caller
 * may run this call on a second stream, overlapping the next layer's work;
 * it must then make the context's next ckv_decode_step wait for it (an
 * event recorded on that stream after this call).  With CKV_STEP=fused or
 * CKV_UPDATE=inline in the environment at ckv_create, the step's last
 * kernel already did this work and the call launches nothing.
 * Errors: CKV_ERR_INVALID_ARG, CKV_ERR_STATE (no preceding decode step),
 * CKV_ERR_CUDA; a step that failed on the device changes no state here. */
ckv_status ckv_assign_update(ckv_ctx* ctx, const void* K, int n, void* stream);

/* One whole decode step from host memory: copies the new token's key and
 * value (k_new_host, v_new_host: [B][H_kv][D]) into row n-1 of the device
 * caches K and V, copies q_host ([B][H_q][D]) to the device, runs
 * ckv_decode_step, copies the output to out_host ([B][H_q][D] float32),
 * launches ckv_assign_update's kernel and returns once the output has
 * arrived; the update finishes on `stream` behind it (the next call on the
 * stream is ordered after it; its device errors surface at the next
 * ckv_last_error).  Host buffers should be page-locked for the copies to
 * be asynchronous; all of them may be reused on return.
 * Errors: as the two calls above, plus CKV_ERR_CUDA. */
ckv_status ckv_decode_host(ckv_ctx* ctx, const void* q_host, const void* k_new_host,
                           const void* v_new_host, void* K, void* V, int n, float* out_host,
                           void* stream);

/* Synchronise the context's device work and return its error word
 * (CKV_OK if none). */
ckv_status ckv_last_error(ckv_ctx* ctx);

/* Kernel launches of one decode step (ckv_decode_step plus
 * ckv_assign_update) of this context: 4 by default (scoring, selection,
 * attention, then edges/assignment/update), 3 with CKV_UPDATE=inline (the
 * attention kernel also runs the last part), 1 when CKV_STEP=fused (one
 * persistent kernel); the environment variables are read at ckv_create.
 * -1 for NULL. */
int ckv_step_launches(const ckv_ctx* ctx);

/* Failure detection: the bound of the fused step's cross-CTA waits (a
 * selection waiting for its graph's score items, an attention item for its
 * graph's selection, a finish for its graph's attention items), in polls
 * of about 64 ns each; 0 restores the default (2^22 polls).  A wait that runs out
 * stops the step and sets CKV_ERR_TIMEOUT in the error word (read by
 * ckv_last_error); the context is then failed until ckv_init_communities()
 * or ckv_import_state().  A limit of 1 poll makes any step whose selection
 * is not already published time out, which is how the tests drive it.
 * Errors: CKV_ERR_INVALID_ARG (NULL). */
ckv_status ckv_set_wait_limit(ckv_ctx* ctx, unsigned polls);

/* Read back the last completed step's decisions into host buffers (any may
 * be NULL).  n_sel [G]; sel [G][max_communities] (kept community ids of
 * each graph, ascending id); n_tok_sel [G] (member tokens kept); n_edges
 * [G]; edges [G][kappa] (token ids, rank order); edge_w [G][kappa];
 * assigned [G].  Synchronous. */
ckv_status ckv_get_step_debug(ckv_ctx* ctx, int32_t* n_sel, int32_t* sel, int32_t* n_tok_sel,
                              int32_t* n_edges, int32_t* edges, float* edge_w, int32_t* assigned);

/* Attention-mass recall of the last decode step -- Figure 3 (right), the
 * share of the full attention mass that the retrieved set captures.  Per
 * query head: the dense softmax of q over every position [0, n) of K,
 * summed over the rows that step attended (sinks, kept members, the new
 * token); computed as l_sel * exp(m_sel - m) / l from the step's own
 * softmax max and sum over its attended rows (left by ckv_decode_step) and
 * the dense max and sum over [0, n) (one pass over K here).
 * q, K: the query and key cache the step with this n was given (q
 * [B][H_q][D], K [B][H_kv][n_max][D], kv_dtype).  recall: [B][H_q] float32,
 * device.  Valid after ckv_decode_step(n), before or after its
 * ckv_assign_update, until the next decode step.  Reads K once; allocates
 * nothing.  Asynchronous.  Supported for H_q/H_kv <= 32 (bf16) or <= 8
 * (float32).
 * Errors: CKV_ERR_INVALID_ARG, CKV_ERR_STATE (no decode step with this n
 * since init or import), sticky device errors, CKV_ERR_CUDA. */
ckv_status ckv_step_recall(ckv_ctx* ctx, const void* q, const void* K, int n, float* recall, void* stream);

/* Dense decode attention, the comparator for the sparse step: every query
 * head attends over every position [0, n) of its KV head,
 * out = softmax(q K^T / sqrt(D)) V and lse = m + ln(l) per head.
 * q, K, V as in ckv_decode_step; out [B][H_q][D] float32 and lse [B][H_q]
 * float32 (may be NULL), device.  Uses the context's dimensions and
 * scratch only (no community state; allowed before init).  Asynchronous.
 * Supported for H_q/H_kv <= 8.
 * Errors: CKV_ERR_INVALID_ARG (bad pointer, n outside [1, n_max], group
 * too large), CKV_ERR_CUDA. */
ckv_status ckv_dense_decode(ckv_ctx* ctx, const void* q, const void* K, const void* V, int n, float* out,
                            float* lse, void* stream);

/* Per-kernel device time of the decode steps, in the spirit of the pages'
 * Table 10 split of a step into retrieval and attention.  After
 * ckv_profile_begin, every ckv_decode_step / ckv_assign_update records CUDA
 * events on its stream around each of its kernels; ckv_profile_end
 * synchronises, writes the summed milliseconds of ms[0] centroid scoring,
 * ms[1] community selection, ms[2] gather + attention + output (with
 * CKV_UPDATE=inline also the edges, assignment and update) and ms[3]
 * ckv_assign_update's edges + assignment + update kernel (0 when it
 * launches nothing); with CKV_STEP=fused ms[0] is the whole step.  Also
 * the number of steps they cover; stops recording.  Both are host calls; begin is not
 * allowed while a step is half done.  Errors: CKV_ERR_INVALID_ARG,
 * CKV_ERR_STATE, CKV_ERR_CUDA. */
ckv_status ckv_profile_begin(ckv_ctx* ctx);
ckv_status ckv_profile_end(ckv_ctx* ctx, float* ms /* [4] */, int* steps);

/* Checkpoint of the community state in a layout-free host format:
 *   int32 header[9] = {0x31564B43 ("CKV1"), 1, G, n_communities, D, n_tok,
 *                      S, kappa, n_init}
 *   float   centroids [G][n_communities][D]
 *   int32   sizes     [G][n_communities]
 *   int32   members   [G][n_tok - S]  (community by community, ascending)
 *   int32   deg       [G][n_tok - n_init]          decode-time edges of
 *   int32   col       [G][n_tok - n_init][kappa]   positions n_init .. n_tok-1
 *   float   w         [G][n_tok - n_init][kappa]
 * n_tok = positions covered (sinks + assigned tokens).  Export: pass
 * host_buf = NULL to get the size in *bytes; otherwise *bytes is the
 * buffer's capacity on entry and the bytes written on return.  Import
 * validates the record against the context (dimensions; sizes summing to
 * n_tok - S; every position in [S, n_tok) a member exactly once, ascending
 * within its community; edge degrees in [0, kappa] and columns in
 * [0, n_tok); finite centroids; finite non-negative edge weights) and
 * replaces the state.
 * Both are synchronous.  Errors: CKV_ERR_INVALID_ARG, CKV_ERR_STATE (no
 * state yet), CKV_ERR_OOM, CKV_ERR_CUDA. */
ckv_status ckv_export_state(ckv_ctx* ctx, void* host_buf, size_t* bytes);
ckv_status ckv_import_state(ckv_ctx* ctx, const void* host_buf, size_t bytes);

/* Exact softmax attention with sinks over caller-chosen rows, without any
 * device allocation.  The paper has no counterpart: this entry point exists
 * for hosts that cannot call cudaMalloc where the attention runs (for
 * example an inference engine's custom-op execute path that forbids device
 * allocation after set-up and gives the op no workspace), so it needs no
 * context.  For every graph g of cfg (only batch, heads, head_dim, n_max,
 * n_sinks, kv_dtype, mode and device are read), each of the graph's query
 * heads attends over the sinks [0, S), the positions rows_host[g][0 ..
 * n_rows_host[g]) and the new token n-1 -- the attention of ckv_decode_step
 * with the kept rows given instead of selected.  q, K, V, out as in
 * ckv_decode_step (device); rows_host [G][max_rows] and n_rows_host [G] are
 * host memory, each row in [S, n-1).
 * Scratch: a 16 MiB file-scope device array that every GPU loading the
 * library keeps until exit; a call needs about max_rows * (4 + 4 * heads
 * per graph) bytes plus its split partials, so max_rows up to about 800,000
 * for a group of 4 heads; a larger max_rows returns CKV_ERR_CAPACITY.
 * Every call shares the array, so calls from different host threads race;
 * serialise them.  The call runs on `stream` and is synchronous: it copies
 * the row lists in, launches one kernel, reads the kernel's error word back
 * and waits for the stream, so rows_host and n_rows_host (pageable or
 * page-locked) may be reused on return, and the call cannot be captured
 * into a CUDA graph.  The caller's current device is restored on return.
 * Errors: CKV_ERR_INVALID_ARG (bad pointer, size, row or device),
 * CKV_ERR_CAPACITY (max_rows too large for the array), CKV_ERR_STATE (the
 * kernel found a row outside the cache), CKV_ERR_TIMEOUT (a bounded wait
 * inside the kernel ran out), CKV_ERR_CUDA. */
ckv_status ckv_attend_rows_static(const ckv_config* cfg, const void* q, const void* K, const void* V,
                                  int n, const int32_t* rows_host, const int32_t* n_rows_host,
                                  int max_rows, float* out, void* stream);

/* Auxiliary storage of the context (centroids, community index, member
 * pool, decode-time edges; scratch excluded) and, for comparison, the bytes
 * of the K and V caches it serves. */
ckv_status ckv_aux_bytes(const ckv_ctx* ctx, size_t* aux_bytes, size_t* kv_bytes);

/* Static description of a status code. */
const char* ckv_status_string(ckv_status s);

#ifdef __cplusplus
}
#endif
#endif
