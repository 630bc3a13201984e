// ckv_internal.cuh -- context layout and kernel launchers of libckv.
//
// Device memory of one context (G graphs, Nc = max_communities, D = 128,
// NM = n_max rows, HG = query heads per graph):
//   mu        float [G][Nc][D]     centroids (Figure 1, step (2): one per community)
//   csize     int32 [G][Nc]        members per community
//   coff,ccap int32 [G][Nc]        segment of the community in the member pool
//   pool      int32 [G][P]         member positions, ascending within a segment
//   pool_top  int32 [G]            first free pool slot (segments move up when full)
//   tok_comm  int32 [G][NM]        community of each position (-1: sink / none)
//   edges     int32/float [G][NM-n_init][kappa] + deg  decode-time token graph rows
// Per-step scratch (reused every step; KC = CTAs of the attention grid):
//   score     float [G][Nc]        centroid scores
//   sel       int32 [G][Nc]        kept communities (ascending id)
//   meta      int32 [G][META]      C, T, rows, edges, assigned of the step
//   rtok,rcomm int32 [G][NM]       token / community of each kept member row
//   zrow      float [G][NM][HG]    logits of the kept members (for the edges)
//   part_ml   float [G][KC][HG][2] per-CTA softmax max and sum per head
//   part_o    float [G][KC][HG][D] per-CTA P.V per head, relative to its max
//   bar       uint  [G][2]         arrivals of a graph's slices (slot 0)
//   e_*       [G][kappa]           the step's edges (rank order) for the update
//   srange    uint  [G][4]         score range keys and total size of the step (k_score -> k_select)
//   sel_ml    float [B][Hq][2]     softmax max and sum of each query head over the
//                                  step's attended rows (for the attention-mass recall)
// Dense statistics scratch (k_dense.cu; U = B*Hkv units):
//   dense_part float [U + grid][..] per-piece (m, l[, o]) of each unit's heads
//   dense_cnt  uint  [U]           arrivals of a unit's pieces
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ckv.h"

namespace ckv {

constexpr int kD = 128;          // head_dim the kernels are written for
constexpr int kMaxKappa = 32;
constexpr int kSelBins = 2048;   // bucket count of the selection passes
constexpr int kAttWarps = 8;     // warps of an attention CTA

// meta slots per graph
enum { M_C = 0, M_T = 1, M_ROWS = 2, M_NEDGE = 3, M_ASSIGNED = 4, M_COUNT = 8 };

struct DevState {
    float* mu;
    int32_t* csize;
    int32_t* coff;
    int32_t* ccap;
    int32_t* pool;
    int32_t* pool_top;
    int32_t* tok_comm;
    int32_t* edge_col;
    float* edge_w;
    int32_t* edge_deg;
    // scratch
    float* score;
    int32_t* sel;
    int32_t* meta;
    int32_t* rtok;
    int32_t* rcomm;
    float* zrow;
    float* part_ml;
    float* part_o;
    unsigned int* bar;
    int32_t* e_tok;
    float* e_w;
    int32_t* e_comm;
    float* sel_ml;           // may be null (then the attention kernel does not write it)
    uint32_t* srange;        // [G][4] min and max score key of the non-empty communities, their total
                             // size, pad: accumulated by the scoring, read and reset by the selection
    // fused step kernel (k_step.cu)
    unsigned* step_ctr;      // [2] queue head and CTAs done; reset by the last CTA to leave
    unsigned* gcnt;          // [G][4] score items done, selection done, attention items done, pad
    unsigned* shist;         // [G][step_hist_bins()] sizes per coarse score bin, filled by the score
                             // items, read and cleared by the selection
    int32_t* sel_row;        // [G][3 (Nc + 1)] kept list (ids, row starts, segments) when it
                             // does not fit shared memory
    int32_t* kinfo;          // [G][Nc][4] each kept community's id, row start, size, segment start
    unsigned* smax;          // [G][nsu] each 16-community slot's largest score key (0: all empty)
    const int32_t* rows_T;   // [G] kept rows of each graph when the rows are given (else null)
    int* err;                // sticky device error word (ckv_status)
};

struct Dims {
    int B, Hq, Hkv, Gq, G, HG, Nc, NM, S, kappa, budget, mode, bf16;
    int64_t P;               // pool capacity per graph
    int nCTA;                // CTAs of the (co-resident) attention grid
    int nSM;                 // multiprocessors of the device
    int n_comm;              // communities in use (set at init)
    int n_init;              // first decode position (edge store row 0)
    int defer_update;        // edges, assignment and update run in k_update (ckv_assign_update)
    int att_cluster;         // the attention runs as one cluster of 4 CTAs per graph (merge in shared memory)
    int fuse_assign;         // the attention kernel also assigns the new token and updates
    int att_aligned;         // attention CTAs split graph by graph (else the rows evenly)
    int pdl;                 // programmatic dependent launch: 0 off, 1 trigger at kernel start, 2 after the main work
    // fused step kernel (k_step.cu)
    int spg;                 // score items per graph
    int api;                 // attention items per graph
    int rows_given;          // attention over given rows: no scoring, selection, edges or update
    unsigned wait_polls;     // polls of an attention item's wait for its graph's selection
    int nStep;               // CTAs of the step grid (co-resident)
    int rtok_stride;         // entries per graph of the kept-row list rtok (n_max, or the given rows' capacity)
    int n_workers;           // CTAs of the step grid that run the selections and finishes
    int nsu;                 // 16-community slots per graph (max_communities / 16, rounded up)
    int fused;               // ckv_decode_step runs the fused kernel (else the three kernels)
};

// kernel launchers (k_decode.cu)
cudaError_t launch_score(const DevState& s, const Dims& d, const void* q, cudaStream_t st);
cudaError_t launch_select(const DevState& s, const Dims& d, cudaStream_t st);
// attention and output, then (unless d.defer_update) the edges and (with
// d.fuse_assign) the assignment and update of the step
cudaError_t launch_attend(const DevState& s, const Dims& d, const void* q, const void* K,
                          const void* V, int n, float* out, cudaStream_t st);
// the step's edges, assignment and update when d.defer_update (one CTA per
// graph, at the lowest stream priority)
cudaError_t launch_update(const DevState& s, const Dims& d, const void* K, int n, cudaStream_t st);
size_t select_smem_bytes(int n_comm, int budget);
// sets the kernels' shared-memory limits on the current device; then the
// number of co-resident CTAs of the attention kernel (0 on error)
cudaError_t prepare_kernels(const Dims& d);
int attend_grid(const Dims& d, int sms);
bool attend_on_clusters(const Dims& d, int sms);
constexpr int kMaxCommunities = 16384;   // k_select holds 16 of a graph's communities per thread

// the fused step (k_step.cu): scoring, selection, attention, edges, vote
// and update of every graph in one persistent cooperative launch
int step_cpi();                                  // communities per score item
int step_hist_bins();                            // coarse score bins per graph
int step_api(int S, int rows);                   // attention items for up to `rows` kept rows
cudaError_t prepare_step(const Dims& d, int sms, int* grid);
cudaError_t launch_step(const DevState& s, const Dims& d, const void* q, const void* K, const void* V, int n,
                        float* out, cudaStream_t st);
constexpr unsigned kStepWaitPolls = 1u << 22;    // default bound of a cross-CTA wait (polls with 64 ns naps)
constexpr int kStepWorkers = 8;                  // selection / finish CTAs of the step grid, at most

// dense decode statistics over a whole cache (k_dense.cu): with V, the dense
// attention output and log-sum-exp per query head; with sel_ml, the
// attention-mass recall of the attended rows
struct DenseIO {
    float* out;              // [B][Hq][D] (with V)
    float* lse;              // [B][Hq] or null
    const float* sel_ml;     // [B][Hq][2] or null
    float* recall;           // [B][Hq] or null (needs sel_ml)
};
constexpr int kDenseMaxCtasPerSM = 4;
bool dense_supported(const Dims& d, bool with_v);
size_t dense_part_floats(const Dims& d);
cudaError_t launch_dense(const Dims& d, const void* q, const void* K, const void* V, int n, float* part,
                         unsigned* cnt, const DenseIO& io, cudaStream_t st);

// init kernels (k_init.cu)
cudaError_t launch_init_count(const DevState& s, const Dims& d, const int32_t* labels, int n,
                              cudaStream_t st);
cudaError_t launch_init_layout(const DevState& s, const Dims& d, int slack, cudaStream_t st);
cudaError_t launch_init_fill(const DevState& s, const Dims& d, const int32_t* labels, int n,
                             cudaStream_t st);
cudaError_t launch_init_centroids(const DevState& s, const Dims& d, const void* K,
                                  cudaStream_t st);

// prefill (k_prefill.cu)
cudaError_t launch_build_graph(int H, int n, int S, int kappa, const void* Q, const void* K,
                               int64_t* row_ptr, int32_t* col, float* w, cudaStream_t st);
// query-group aggregated prefill graph: per-head row statistics into stats
// (build_graph_grouped_stats_floats floats), then one graph per KV head
size_t build_graph_grouped_stats_floats(int Hkv, int group, int n);
cudaError_t launch_build_graph_grouped(int Hkv, int group, int n, int S, int kappa, const void* Q, const void* K,
                                       float* stats, int64_t* row_ptr, int32_t* col, float* w, cudaStream_t st);

// device error word: first error wins
__device__ __forceinline__ void set_error(int* err, int code) { atomicCAS(err, 0, code); }

// Range checks of the debug build (libckv_debug.so, compiled with
// -DCKV_DEBUG_BOUNDS): CKV_IN_RANGE(i, lo, hi, err) is true when lo <= i <
// hi and otherwise sets CKV_ERR_STATE in the error word and is false, so the
// caller skips the access or redirects it in bounds.  They cover the
// community segments (offset + size inside the member pool) wherever a
// kernel reads or moves one, and the community an update writes.  In the
// release build they compile to `true`.  Gathered token rows are checked in
// both builds.
__device__ __forceinline__ bool in_range_or_flag(int64_t i, int64_t lo, int64_t hi, int* err)
{
    if (i >= lo && i < hi) return true;
    set_error(err, CKV_ERR_STATE);
    return false;
}
#ifdef CKV_DEBUG_BOUNDS
#define CKV_IN_RANGE(i, lo, hi, err) ::ckv::in_range_or_flag((int64_t)(i), (int64_t)(lo), (int64_t)(hi), (err))
#else
#define CKV_IN_RANGE(i, lo, hi, err) true
#endif

}  // namespace ckv
