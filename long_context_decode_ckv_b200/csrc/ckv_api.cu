// ckv_api.cu -- the C ABI of libckv (declared in include/ckv.h).
//
// Host side of "CommunityKV: Efficient Long-Context Decoding via Graph
// Partitioning": argument checks, the context's device memory, the launch
// order of one decode step (Figure 1 caption, step (3)), the initial
// partition (step (2)), checkpoint export/import and the host-buffer step
// used for end-to-end timing.  Every step of the method runs in the CUDA
// kernels of k_decode.cu, k_init.cu and k_prefill.cu.
#include <cuda_runtime.h>
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <array>
#include <new>
#include <thread>
#include <vector>

#include "ckv_internal.cuh"
#include "leiden.h"
#ifdef CKV_DEBUG_BOUNDS
#include "ckv_debug.h"
#endif

#define CKV_API extern "C" __attribute__((visibility("default")))

using ckv::DevState;
using ckv::Dims;

struct ckv_ctx {
    ckv_config cfg;
    Dims d;
    DevState s;
    std::vector<void*> allocs;   // everything cudaMalloc'd for this context
    void* edge_alloc[3];         // edge store, sized at init
    int64_t edge_rows;
    void* stage;                 // staging for ckv_decode_host: q | k_new | v_new | out
    size_t stage_bytes;
    int initialized;
    int n_tok;                   // positions covered: sinks + assigned tokens
    int pending;                 // a decode step awaits its assign/update
    int pending_n;
    int last_n;                  // n of the last decode step (0: none since init)
    float* dense_part;           // k_dense piece slots
    unsigned* dense_cnt;         // k_dense arrivals per unit
    ckv_status sticky;
    // profiling: one event per kernel boundary of each profiled step
    int profiling;
    std::vector<cudaEvent_t> ev_pool;   // all events ever created (reused)
    cudaEvent_t host_done;              // ckv_decode_host: its output has reached the host
    size_t ev_used;
    std::vector<std::array<cudaEvent_t, 6>> ev_steps;
    // token graph of every graph on the host (rows [0, tg_rows)): the
    // prefill graph the caller registered, extended by decode-time rows at
    // each refresh
    struct TokenGraph {
        std::vector<int64_t> rp;
        std::vector<int32_t> col;
        std::vector<float> w;
    };
    std::vector<TokenGraph> tg;
    int tg_rows;
};

namespace {

constexpr uint32_t kMagic = 0x31564B43u;   // "CKV1"

// a resolution is a finite positive number; an edge weight a finite
// non-negative one (NaN fails both comparisons)
bool valid_gamma(double g) { return g > 0.0 && g <= DBL_MAX; }
bool valid_weight(float w) { return w >= 0.0f && w <= FLT_MAX; }

ckv_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return CKV_OK;
    if (e == cudaErrorMemoryAllocation) return CKV_ERR_OOM;
    if (e == cudaErrorInvalidValue) return CKV_ERR_INVALID_ARG;
    return CKV_ERR_CUDA;
}

// Forced allocation failure for the failure-handling tests: with
// CKV_FAULT_ALLOC=k in the environment, the k-th device allocation made
// inside one library call fails as if the device were out of memory.  Each
// call that allocates arms the count on entry (FaultScope); dev_malloc is
// the only allocator of the context code.
thread_local int t_fault_left = 0;

struct FaultScope {
    FaultScope()
    {
        const char* v = getenv("CKV_FAULT_ALLOC");
        t_fault_left = v ? atoi(v) : 0;
    }
    ~FaultScope() { t_fault_left = 0; }
};

cudaError_t dev_malloc(void** p, size_t bytes)
{
    *p = nullptr;
    if (t_fault_left > 0 && --t_fault_left == 0) return cudaErrorMemoryAllocation;
    return cudaMalloc(p, bytes);
}

#define CKV_CUDA(call)                                      \
    do {                                                    \
        cudaError_t e_ = (call);                            \
        if (e_ != cudaSuccess) return cuda_status(e_);      \
    } while (0)

int graph_count(const ckv_config* c)
{
    if (c->mode == CKV_QUERY_GROUP) return c->batch * c->n_kv_heads;
    if (c->mode == CKV_PER_HEAD) return c->batch * c->n_q_heads;
    return -1;
}

size_t elem_bytes(ckv_dtype t) { return t == CKV_BF16 ? 2 : 4; }

bool valid_config(const ckv_config* c)
{
    if (!c) return false;
    if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1) return false;
    if (c->n_q_heads % c->n_kv_heads) return false;
    if (c->head_dim != ckv::kD) return false;
    if (c->n_max < 1 || c->max_communities < 1 || c->max_communities > ckv::kMaxCommunities) return false;
    if (c->n_sinks < 0 || c->n_sinks >= c->n_max) return false;
    if (c->kappa < 1 || c->kappa > ckv::kMaxKappa) return false;
    if (c->budget < 1 || c->slack < 0 || c->slack > (1 << 20)) return false;
    if (c->kv_dtype != CKV_F32 && c->kv_dtype != CKV_BF16) return false;
    if (c->mode != CKV_PER_HEAD && c->mode != CKV_QUERY_GROUP) return false;
    const int gq = c->n_q_heads / c->n_kv_heads;
    if (c->mode == CKV_QUERY_GROUP && gq != 1 && gq != 2 && gq != 4 && gq != 8) return false;
    if (c->device < 0) return false;
    // sizes that must fit the kernels' 32-bit indices
    const int64_t G = graph_count(c);
    if (c->pool_capacity < 0) return false;
    if ((int64_t)c->n_max * 5 + (int64_t)c->max_communities * (c->slack + 32) > INT32_MAX) return false;
    if (G * c->max_communities > INT32_MAX) return false;
    return true;
}

template <typename T>
cudaError_t dalloc(ckv_ctx* x, T** p, size_t count)
{
    void* v = nullptr;
    cudaError_t e = dev_malloc(&v, count * sizeof(T) + 16);
    if (e != cudaSuccess) return e;
    x->allocs.push_back(v);
    *p = static_cast<T*>(v);
    return cudaSuccess;
}

ckv_status check_ctx(ckv_ctx* x)
{
    if (!x) return CKV_ERR_INVALID_ARG;
    if (x->sticky != CKV_OK) return x->sticky;
    return CKV_OK;
}

void free_edges(ckv_ctx* x)
{
    for (void*& p : x->edge_alloc) {
        if (p) cudaFree(p);
        p = nullptr;
    }
    x->edge_rows = 0;
    x->s.edge_col = nullptr;
    x->s.edge_w = nullptr;
    x->s.edge_deg = nullptr;
}

// a new edge store for `rows` decode rows per graph, allocated before the
// old one is released: on failure the context keeps its store
struct EdgeStore {
    void* p[3] = {nullptr, nullptr, nullptr};
    int64_t rows = 0;
    void release()
    {
        for (void*& q : p) {
            if (q) cudaFree(q);
            q = nullptr;
        }
    }
};

cudaError_t new_edges(const ckv_ctx* x, int64_t rows, EdgeStore& es)
{
    const int64_t G = x->d.G, k = x->d.kappa;
    const int64_t r = rows > 0 ? rows : 1;
    cudaError_t e;
    es.rows = rows;
    if ((e = dev_malloc(&es.p[0], (size_t)(G * r * k) * 4)) == cudaSuccess &&
        (e = dev_malloc(&es.p[1], (size_t)(G * r * k) * 4)) == cudaSuccess &&
        (e = dev_malloc(&es.p[2], (size_t)(G * r) * 4)) == cudaSuccess)
        return cudaSuccess;
    es.release();
    return e;
}

void install_edges(ckv_ctx* x, EdgeStore& es)
{
    free_edges(x);
    for (int i = 0; i < 3; ++i) x->edge_alloc[i] = es.p[i];
    x->s.edge_col = static_cast<int32_t*>(x->edge_alloc[0]);
    x->s.edge_w = static_cast<float*>(x->edge_alloc[1]);
    x->s.edge_deg = static_cast<int32_t*>(x->edge_alloc[2]);
    x->edge_rows = es.rows;
    es = EdgeStore{};
}

// empty score range and zero total size for every graph (k_score accumulates
// into it, k_select resets it after reading)
cudaError_t reset_srange(ckv_ctx* x, cudaStream_t st)
{
    std::vector<uint32_t> h((size_t)x->d.G * 4, 0u);
    for (size_t g = 0; g < (size_t)x->d.G; ++g) h[4 * g] = 0xffffffffu;
    cudaError_t e = cudaMemcpyAsync(x->s.srange, h.data(), h.size() * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

ckv_status read_device_error(ckv_ctx* x)
{
    int err = 0;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaDeviceSynchronize());
    CKV_CUDA(cudaMemcpy(&err, x->s.err, sizeof(int), cudaMemcpyDeviceToHost));
    return (ckv_status)err;
}

// host-side layout of the community state (used by export/import)
struct HostState {
    std::vector<float> mu;          // [G][Nc_used][D]
    std::vector<int32_t> size;      // [G][Nc_used]
    std::vector<int32_t> members;   // [G][n_tok - S]
    std::vector<int32_t> deg, col;  // edges of decode rows
    std::vector<float> w;
};

cudaError_t next_event(ckv_ctx* x, cudaEvent_t* e)
{
    if (x->ev_used == x->ev_pool.size()) {
        cudaEvent_t ne;
        cudaError_t r = cudaEventCreate(&ne);
        if (r != cudaSuccess) return r;
        x->ev_pool.push_back(ne);
    }
    *e = x->ev_pool[x->ev_used++];
    return cudaSuccess;
}

// record the event of kernel boundary `slot` of the current profiled step
cudaError_t prof_mark(ckv_ctx* x, int slot, cudaStream_t st)
{
    if (!x->profiling) return cudaSuccess;
    if (slot == 0) x->ev_steps.emplace_back();
    cudaEvent_t e;
    cudaError_t r = next_event(x, &e);
    if (r != cudaSuccess) return r;
    x->ev_steps.back()[slot] = e;
    // under stream capture an external record becomes an event-record node
    // whose timestamps stay usable for cudaEventElapsedTime; the flag is
    // only accepted while the stream is capturing
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    r = cudaStreamIsCapturing(st, &cap);
    if (r != cudaSuccess) return r;
    if (cap == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    return cudaEventRecord(e, st);
}

}  // namespace

// ------------------------------------------------------------------ API
CKV_API int ckv_graph_count(const ckv_config* cfg) { return cfg ? graph_count(cfg) : -1; }

CKV_API const char* ckv_status_string(ckv_status s)
{
    switch (s) {
        case CKV_OK: return "ok";
        case CKV_ERR_INVALID_ARG: return "invalid argument";
        case CKV_ERR_CAPACITY: return "community storage exhausted";
        case CKV_ERR_OOM: return "out of memory";
        case CKV_ERR_CUDA: return "CUDA error";
        case CKV_ERR_TIMEOUT: return "device wait timed out";
        case CKV_ERR_STATE: return "call out of order";
    }
    return "unknown status";
}

CKV_API void ckv_destroy(ckv_ctx* x)
{
    if (!x) return;
    cudaSetDevice(x->cfg.device);
    cudaDeviceSynchronize();
    for (cudaEvent_t e : x->ev_pool) cudaEventDestroy(e);
    if (x->host_done) cudaEventDestroy(x->host_done);
    free_edges(x);
    for (void* p : x->allocs) cudaFree(p);
    if (x->stage) cudaFree(x->stage);
    delete x;
}

CKV_API ckv_status ckv_create(const ckv_config* cfg, ckv_ctx** out)
{
    FaultScope fault;
    if (!out) return CKV_ERR_INVALID_ARG;
    *out = nullptr;
    if (!valid_config(cfg)) return CKV_ERR_INVALID_ARG;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || cfg->device >= ndev) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(cfg->device));
    int sms = 0;
    CKV_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, cfg->device));

    ckv_ctx* x = new (std::nothrow) ckv_ctx();
    if (!x) return CKV_ERR_OOM;
    x->cfg = *cfg;
    Dims& d = x->d;
    d.B = cfg->batch;
    d.Hq = cfg->n_q_heads;
    d.Hkv = cfg->n_kv_heads;
    d.Gq = d.Hq / d.Hkv;
    d.G = graph_count(cfg);
    d.HG = (cfg->mode == CKV_QUERY_GROUP) ? d.Gq : 1;
    d.Nc = cfg->max_communities;
    d.NM = cfg->n_max;
    d.S = cfg->n_sinks;
    d.kappa = cfg->kappa;
    d.budget = cfg->budget;
    d.mode = cfg->mode;
    d.bf16 = cfg->kv_dtype == CKV_BF16;
    // A community that grows from its initial segment by doubling allocates
    // at most 4 * (final size) + 32 slots after it, so this automatic size
    // can never run out before n_max.
    d.P = cfg->pool_capacity > 0 ? (int64_t)cfg->pool_capacity
                                 : (int64_t)cfg->n_max * 5 + (int64_t)cfg->max_communities * (cfg->slack + 32);
    // the attention grid: as many CTAs as can be co-resident
    d.nSM = sms;
    d.fuse_assign = 1;
    {   // attention split: graph by graph unless CKV_ATT_SPLIT=rows
        const char* v = getenv("CKV_ATT_SPLIT");
        d.att_aligned = !(v && v[0] == 'r');
    }
    {   // programmatic dependent launch between the decode kernels: off unless
        // CKV_PDL is 1 (each kernel lets the next one launch at its start) or
        // 2 (after its main work)
        const char* v = getenv("CKV_PDL");
        d.pdl = (v && (v[0] == '1' || v[0] == '2')) ? v[0] - '0' : 0;
    }
    {   // the decode step: three kernels (scoring, selection, attention)
        // unless CKV_STEP=fused (one persistent kernel)
        const char* v = getenv("CKV_STEP");
        d.fused = v && v[0] == 'f';
    }
    {   // the three-kernel step leaves the edges, assignment and update to
        // ckv_assign_update's own kernel, unless CKV_UPDATE=inline (then the
        // attention kernel's last slice of each graph runs them)
        const char* v = getenv("CKV_UPDATE");
        d.defer_update = !d.fused && !(v && v[0] == 'i');
    }
    {   // with the deferred update and at most a quarter as many graphs as
        // SMs, the attention runs as one cluster of four CTAs per graph
        // whose slices merge in distributed shared memory, unless
        // CKV_ATT_CLUSTER=0
        const char* v = getenv("CKV_ATT_CLUSTER");
        d.att_cluster = !(v && v[0] == '0') && !d.fused && ckv::attend_on_clusters(d, sms);
    }
    d.nCTA = ckv::attend_grid(d, sms);
    if (d.nCTA < 1) { delete x; return CKV_ERR_CUDA; }
    d.api = ckv::step_api(d.S, d.budget);
    d.spg = 1;
    d.rows_given = 0;
    d.rtok_stride = d.NM;
    d.nsu = (d.Nc + 15) / 16;
    d.wait_polls = ckv::kStepWaitPolls;
    if (ckv::prepare_step(d, sms, &d.nStep) != cudaSuccess || d.nStep < 2) { delete x; return CKV_ERR_CUDA; }
    {   // worker CTAs of the fused step (CKV_STEP_WORKERS overrides the default, for measurements)
        const char* v = getenv("CKV_STEP_WORKERS");
        const int want = (v && atoi(v) > 0) ? atoi(v) : ckv::kStepWorkers;
        d.n_workers = std::min(std::min(d.G, want), d.nStep / 2);
    }
    d.n_comm = 0;
    d.n_init = 0;

    const size_t G = d.G, Nc = d.Nc, NM = d.NM, HG = d.HG;
    DevState& s = x->s;
    cudaError_t e = cudaSuccess;
#define ALLOC(ptr, n) if (e == cudaSuccess) e = dalloc(x, &s.ptr, (n))
    ALLOC(mu, G * Nc * ckv::kD);
    ALLOC(csize, G * Nc);
    ALLOC(coff, G * Nc);
    ALLOC(ccap, G * Nc);
    ALLOC(pool, G * (size_t)d.P);
    ALLOC(pool_top, G);
    ALLOC(tok_comm, G * NM);
    const size_t KC = std::max(d.nCTA, d.api), kap = d.kappa;
    ALLOC(score, G * Nc);
    ALLOC(sel, G * Nc);
    ALLOC(meta, G * ckv::M_COUNT);
    ALLOC(rtok, G * NM);
    ALLOC(rcomm, G * NM);
    ALLOC(zrow, G * NM * HG);
    ALLOC(part_ml, G * KC * HG * 2);
    ALLOC(part_o, G * KC * HG * ckv::kD);
    ALLOC(bar, G * 2);
    ALLOC(e_tok, G * kap);
    ALLOC(e_w, G * kap);
    ALLOC(e_comm, G * kap);
    ALLOC(sel_ml, (size_t)d.B * d.Hq * 2);
    ALLOC(srange, G * 4);
    ALLOC(step_ctr, 2);
    ALLOC(gcnt, G * 4);
    ALLOC(shist, G * ckv::step_hist_bins());
    ALLOC(sel_row, G * 3 * (Nc + 1));
    ALLOC(kinfo, G * Nc * 4);
    ALLOC(smax, G * ((Nc + 15) / 16));
    ALLOC(err, 1);
#undef ALLOC
    s.rows_T = nullptr;
    if (e == cudaSuccess) e = cudaMemset(s.step_ctr, 0, 2 * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(s.gcnt, 0, G * 4 * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(s.shist, 0, G * ckv::step_hist_bins() * sizeof(unsigned));
    if (e == cudaSuccess) e = dalloc(x, &x->dense_part, ckv::dense_part_floats(d));
    if (e == cudaSuccess) e = dalloc(x, &x->dense_cnt, (size_t)d.B * d.Hkv);
    if (e == cudaSuccess) e = cudaMemset(x->dense_cnt, 0, (size_t)d.B * d.Hkv * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(s.bar, 0, G * 2 * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(s.err, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(s.meta, 0, G * ckv::M_COUNT * sizeof(int32_t));
    if (e == cudaSuccess) e = reset_srange(x, 0);
    const size_t qb = (size_t)d.B * d.Hq * ckv::kD;
    x->stage_bytes = qb * elem_bytes(cfg->kv_dtype) + 2 * (size_t)d.B * d.Hkv * ckv::kD * elem_bytes(cfg->kv_dtype) +
                     qb * sizeof(float) + 64;
    if (e == cudaSuccess) e = dev_malloc(&x->stage, x->stage_bytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        ckv_status st = cuda_status(e);
        ckv_destroy(x);
        return st == CKV_ERR_INVALID_ARG ? CKV_ERR_CUDA : st;
    }
    x->sticky = CKV_OK;
    *out = x;
    return CKV_OK;
}

CKV_API ckv_status ckv_init_communities(ckv_ctx* x, const int32_t* labels, int labels_on_device,
                                        int n_communities, const void* K, int n, void* stream)
{
    if (!x || !labels || !K) return CKV_ERR_INVALID_ARG;
    if (n < x->d.S || n > x->d.NM || n_communities < 1 || n_communities > x->d.Nc)
        return CKV_ERR_INVALID_ARG;
    FaultScope fault;
    cudaStream_t st = (cudaStream_t)stream;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaStreamSynchronize(st));
    // everything the call allocates comes first: when an allocation fails
    // the context keeps its state
    EdgeStore es;
    void* tmp = nullptr;
    {
        cudaError_t ea = new_edges(x, (int64_t)x->d.NM - n, es);
        if (ea == cudaSuccess && !labels_on_device) ea = dev_malloc(&tmp, x->d.G * (size_t)n * sizeof(int32_t) + 16);
        if (ea != cudaSuccess) {
            es.release();
            return cuda_status(ea);
        }
    }
    x->initialized = 0;
    x->pending = 0;
    x->last_n = 0;
    x->sticky = CKV_OK;
    Dims& d = x->d;
    DevState& s = x->s;
    d.n_comm = n_communities;
    d.spg = (n_communities + ckv::step_cpi() - 1) / ckv::step_cpi();
    d.n_init = n;
    const size_t G = d.G;
    const int32_t* dlabels = labels;
    if (!labels_on_device) {
        cudaError_t e = cudaMemcpyAsync(tmp, labels, G * (size_t)n * sizeof(int32_t), cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) { cudaFree(tmp); es.release(); return cuda_status(e); }
        dlabels = static_cast<const int32_t*>(tmp);
    }
    cudaError_t e = cudaSuccess;
    auto step = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
    step(cudaMemsetAsync(s.err, 0, sizeof(int), st));
    step(cudaMemsetAsync(s.csize, 0, G * d.Nc * sizeof(int32_t), st));
    step(cudaMemsetAsync(s.coff, 0, G * d.Nc * sizeof(int32_t), st));
    step(cudaMemsetAsync(s.ccap, 0, G * d.Nc * sizeof(int32_t), st));
    step(cudaMemsetAsync(s.tok_comm, 0xff, G * d.NM * sizeof(int32_t), st));
    step(cudaMemsetAsync(s.bar, 0, G * 2 * sizeof(unsigned), st));
    step(cudaMemsetAsync(s.step_ctr, 0, 2 * sizeof(unsigned), st));
    step(cudaMemsetAsync(s.gcnt, 0, G * 4 * sizeof(unsigned), st));
    step(cudaMemsetAsync(s.shist, 0, G * ckv::step_hist_bins() * sizeof(unsigned), st));
    step(cudaMemsetAsync(s.mu, 0, G * d.Nc * ckv::kD * sizeof(float), st));
    step(reset_srange(x, st));
    step(ckv::launch_init_count(s, d, dlabels, n, st));
    int err = 0;
    step(cudaMemcpyAsync(&err, s.err, sizeof(int), cudaMemcpyDeviceToHost, st));
    step(cudaStreamSynchronize(st));
    if (e == cudaSuccess && err == 0) {
        step(ckv::launch_init_layout(s, d, x->cfg.slack, st));
        step(cudaMemsetAsync(s.csize, 0, G * d.Nc * sizeof(int32_t), st));
        step(ckv::launch_init_fill(s, d, dlabels, n, st));
        step(ckv::launch_init_centroids(s, d, K, st));
        step(cudaMemcpyAsync(&err, s.err, sizeof(int), cudaMemcpyDeviceToHost, st));
        step(cudaStreamSynchronize(st));
    }
    if (tmp) cudaFree(tmp);
    if (e != cudaSuccess) { es.release(); return cuda_status(e); }
    if (err != 0) {
        es.release();
        cudaMemset(s.err, 0, sizeof(int));
        return (ckv_status)err;
    }
    install_edges(x, es);
    x->n_tok = n;
    x->initialized = 1;
    return CKV_OK;
}

CKV_API ckv_status ckv_decode_step(ckv_ctx* x, const void* q, const void* K, const void* V, int n,
                                   float* out, void* stream)
{
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!q || !K || !V || !out) return CKV_ERR_INVALID_ARG;
    if (!x->initialized || x->pending) return CKV_ERR_STATE;
    if (n != x->n_tok + 1 || n > x->d.NM) return CKV_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(prof_mark(x, 0, st));
    if (x->d.fused) {
        CKV_CUDA(ckv::launch_step(x->s, x->d, q, K, V, n, out, st));
        CKV_CUDA(prof_mark(x, 1, st));
        CKV_CUDA(prof_mark(x, 2, st));
    } else {
        CKV_CUDA(ckv::launch_score(x->s, x->d, q, st));
        CKV_CUDA(prof_mark(x, 1, st));
        CKV_CUDA(ckv::launch_select(x->s, x->d, st));
        CKV_CUDA(prof_mark(x, 2, st));
        CKV_CUDA(ckv::launch_attend(x->s, x->d, q, K, V, n, out, st));
    }
    CKV_CUDA(prof_mark(x, 3, st));
    x->pending = 1;
    x->pending_n = n;
    x->last_n = n;
    return CKV_OK;
}

CKV_API ckv_status ckv_assign_update(ckv_ctx* x, const void* K, int n, void* stream)
{
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!K) return CKV_ERR_INVALID_ARG;
    if (!x->pending || n != x->pending_n) return CKV_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    // the edges, assignment and update: their own kernel, or already done by
    // the step's last kernel (the fused step, or CKV_UPDATE=inline)
    CKV_CUDA(prof_mark(x, 4, st));
    if (x->d.defer_update) CKV_CUDA(ckv::launch_update(x->s, x->d, K, n, st));
    CKV_CUDA(prof_mark(x, 5, st));
    x->pending = 0;
    x->n_tok = n;
    return CKV_OK;
}

namespace ckv {
cudaError_t launch_append_rows(const Dims& d, const void* knew, const void* vnew, void* K, void* V,
                               int row, cudaStream_t st);
}

CKV_API ckv_status ckv_decode_host(ckv_ctx* x, const void* q_host, const void* k_new_host,
                                   const void* v_new_host, void* K, void* V, int n, float* out_host,
                                   void* stream)
{
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!q_host || !k_new_host || !v_new_host || !K || !V || !out_host) return CKV_ERR_INVALID_ARG;
    if (!x->initialized || x->pending) return CKV_ERR_STATE;
    if (n != x->n_tok + 1 || n > x->d.NM) return CKV_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    const Dims& d = x->d;
    const size_t eb = elem_bytes(x->cfg.kv_dtype);
    const size_t qb = (size_t)d.B * d.Hq * ckv::kD * eb;
    const size_t kb = (size_t)d.B * d.Hkv * ckv::kD * eb;
    char* stg = static_cast<char*>(x->stage);
    char* dq = stg;
    char* dk = stg + qb;
    char* dv = dk + kb;
    float* dout = reinterpret_cast<float*>(((uintptr_t)(dv + kb) + 15) & ~(uintptr_t)15);
    CKV_CUDA(cudaMemcpyAsync(dq, q_host, qb, cudaMemcpyHostToDevice, st));
    CKV_CUDA(cudaMemcpyAsync(dk, k_new_host, kb, cudaMemcpyHostToDevice, st));
    CKV_CUDA(cudaMemcpyAsync(dv, v_new_host, kb, cudaMemcpyHostToDevice, st));
    CKV_CUDA(ckv::launch_append_rows(d, dk, dv, K, V, n - 1, st));
    cs = ckv_decode_step(x, dq, K, V, n, dout, stream);
    if (cs != CKV_OK) return cs;
    // the output goes back first; the call returns when it has arrived, and
    // the update kernel finishes behind it on the stream
    CKV_CUDA(cudaMemcpyAsync(out_host, dout, (size_t)d.B * d.Hq * ckv::kD * sizeof(float),
                             cudaMemcpyDeviceToHost, st));
    if (!x->host_done) CKV_CUDA(cudaEventCreateWithFlags(&x->host_done, cudaEventDisableTiming));
    CKV_CUDA(cudaEventRecord(x->host_done, st));
    cs = ckv_assign_update(x, K, n, stream);
    if (cs != CKV_OK) return cs;
    CKV_CUDA(cudaEventSynchronize(x->host_done));
    return CKV_OK;
}

CKV_API ckv_status ckv_step_recall(ckv_ctx* x, const void* q, const void* K, int n, float* recall, void* stream)
{
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!q || !K || !recall) return CKV_ERR_INVALID_ARG;
    if (!ckv::dense_supported(x->d, false)) return CKV_ERR_INVALID_ARG;
    if (!x->initialized || x->last_n == 0 || n != x->last_n) return CKV_ERR_STATE;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    const ckv::DenseIO io{nullptr, nullptr, x->s.sel_ml, recall};
    CKV_CUDA(ckv::launch_dense(x->d, q, K, nullptr, n, x->dense_part, x->dense_cnt, io, (cudaStream_t)stream));
    return CKV_OK;
}

CKV_API ckv_status ckv_dense_decode(ckv_ctx* x, const void* q, const void* K, const void* V, int n, float* out,
                                    float* lse, void* stream)
{
    if (!x) return CKV_ERR_INVALID_ARG;
    if (!q || !K || !V || !out) return CKV_ERR_INVALID_ARG;
    if (n < 1 || n > x->d.NM || !ckv::dense_supported(x->d, true)) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    const ckv::DenseIO io{out, lse, nullptr, nullptr};
    CKV_CUDA(ckv::launch_dense(x->d, q, K, V, n, x->dense_part, x->dense_cnt, io, (cudaStream_t)stream));
    return CKV_OK;
}

CKV_API ckv_status ckv_last_error(ckv_ctx* x)
{
    if (!x) return CKV_ERR_INVALID_ARG;
    if (x->sticky != CKV_OK) return x->sticky;
    ckv_status e = read_device_error(x);
    if (e != CKV_OK) x->sticky = e;
    return e;
}

CKV_API int ckv_step_launches(const ckv_ctx* x)
{
    return x ? (x->d.fused ? 1 : 3 + (x->d.defer_update ? 1 : 0)) : -1;
}

CKV_API ckv_status ckv_set_wait_limit(ckv_ctx* x, unsigned polls)
{
    if (!x) return CKV_ERR_INVALID_ARG;
    x->d.wait_polls = polls ? polls : ckv::kStepWaitPolls;
    return CKV_OK;
}

CKV_API ckv_status ckv_profile_begin(ckv_ctx* x)
{
    if (!x) return CKV_ERR_INVALID_ARG;
    if (x->pending) return CKV_ERR_STATE;
    x->ev_steps.clear();
    x->ev_used = 0;
    x->profiling = 1;
    return CKV_OK;
}

CKV_API ckv_status ckv_profile_end(ckv_ctx* x, float* ms, int* steps)
{
    if (!x || !ms || !steps) return CKV_ERR_INVALID_ARG;
    if (!x->profiling || x->pending) return CKV_ERR_STATE;
    x->profiling = 0;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    double tot[4] = {0, 0, 0, 0};
    static const int from[4] = {0, 1, 2, 4}, to[4] = {1, 2, 3, 5};
    for (const auto& ev : x->ev_steps) {
        CKV_CUDA(cudaEventSynchronize(ev[5]));
        for (int k = 0; k < 4; ++k) {
            float t = 0.f;
            CKV_CUDA(cudaEventElapsedTime(&t, ev[from[k]], ev[to[k]]));
            tot[k] += t;
        }
    }
    for (int k = 0; k < 4; ++k) ms[k] = (float)tot[k];
    *steps = (int)x->ev_steps.size();
    x->ev_steps.clear();
    x->ev_used = 0;
    return CKV_OK;
}

CKV_API ckv_status ckv_get_step_debug(ckv_ctx* x, int32_t* n_sel, int32_t* sel, int32_t* n_tok_sel,
                                      int32_t* n_edges, int32_t* edges, float* edge_w, int32_t* assigned)
{
    if (!x) return CKV_ERR_INVALID_ARG;
    if (!x->initialized) return CKV_ERR_STATE;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaDeviceSynchronize());
    const Dims& d = x->d;
    std::vector<int32_t> meta((size_t)d.G * ckv::M_COUNT);
    CKV_CUDA(cudaMemcpy(meta.data(), x->s.meta, meta.size() * 4, cudaMemcpyDeviceToHost));
    for (int g = 0; g < d.G; ++g) {
        const int32_t* m = &meta[(size_t)g * ckv::M_COUNT];
        if (n_sel) n_sel[g] = m[ckv::M_C];
        if (n_tok_sel) n_tok_sel[g] = m[ckv::M_T];
        if (n_edges) n_edges[g] = m[ckv::M_NEDGE];
        if (assigned) assigned[g] = m[ckv::M_ASSIGNED];
    }
    if (sel) CKV_CUDA(cudaMemcpy(sel, x->s.sel, (size_t)d.G * d.Nc * 4, cudaMemcpyDeviceToHost));
    if (edges) CKV_CUDA(cudaMemcpy(edges, x->s.e_tok, (size_t)d.G * d.kappa * 4, cudaMemcpyDeviceToHost));
    if (edge_w) CKV_CUDA(cudaMemcpy(edge_w, x->s.e_w, (size_t)d.G * d.kappa * 4, cudaMemcpyDeviceToHost));
    return CKV_OK;
}

CKV_API ckv_status ckv_export_state(ckv_ctx* x, void* host_buf, size_t* bytes)
{
    if (!x || !bytes) return CKV_ERR_INVALID_ARG;
    if (!x->initialized) return CKV_ERR_STATE;
    const Dims& d = x->d;
    const size_t G = d.G, Nc = d.n_comm, D = ckv::kD;
    const size_t nmem = (size_t)(x->n_tok - d.S);
    const size_t rows = (size_t)(x->n_tok - d.n_init);
    const size_t need = 9 * 4 + G * Nc * D * 4 + G * Nc * 4 + G * nmem * 4 + G * rows * 4 +
                        2 * G * rows * d.kappa * 4;
    if (!host_buf) { *bytes = need; return CKV_OK; }
    if (*bytes < need) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaDeviceSynchronize());
    std::vector<float> mu(G * d.Nc * D);
    std::vector<int32_t> size(G * d.Nc), off(G * d.Nc), pool(G * (size_t)d.P);
    CKV_CUDA(cudaMemcpy(mu.data(), x->s.mu, mu.size() * 4, cudaMemcpyDeviceToHost));
    CKV_CUDA(cudaMemcpy(size.data(), x->s.csize, size.size() * 4, cudaMemcpyDeviceToHost));
    CKV_CUDA(cudaMemcpy(off.data(), x->s.coff, off.size() * 4, cudaMemcpyDeviceToHost));
    CKV_CUDA(cudaMemcpy(pool.data(), x->s.pool, pool.size() * 4, cudaMemcpyDeviceToHost));
    char* p = static_cast<char*>(host_buf);
    const int32_t hdr[9] = {(int32_t)kMagic, 1, d.G, d.n_comm, ckv::kD, x->n_tok, d.S, d.kappa, d.n_init};
    memcpy(p, hdr, sizeof hdr);
    p += sizeof hdr;
    for (size_t g = 0; g < G; ++g) {
        memcpy(p, &mu[g * d.Nc * D], Nc * D * 4);
        p += Nc * D * 4;
    }
    for (size_t g = 0; g < G; ++g) {
        memcpy(p, &size[g * d.Nc], Nc * 4);
        p += Nc * 4;
    }
    for (size_t g = 0; g < G; ++g) {
        size_t k = 0;
        for (size_t c = 0; c < Nc; ++c) {
            const int32_t sz = size[g * d.Nc + c], o = off[g * d.Nc + c];
            // the segment read back must lie inside the pool before host code reads it
            if (sz < 0 || o < 0 || (int64_t)o + sz > d.P || k + sz > nmem) return CKV_ERR_STATE;
            memcpy(p + (k * 4), &pool[g * d.P + o], (size_t)sz * 4);
            k += sz;
        }
        if (k != nmem) return CKV_ERR_STATE;
        p += nmem * 4;
    }
    if (rows) {
        std::vector<int32_t> deg(G * x->edge_rows), col(G * x->edge_rows * d.kappa);
        std::vector<float> w(G * x->edge_rows * d.kappa);
        CKV_CUDA(cudaMemcpy(deg.data(), x->s.edge_deg, deg.size() * 4, cudaMemcpyDeviceToHost));
        CKV_CUDA(cudaMemcpy(col.data(), x->s.edge_col, col.size() * 4, cudaMemcpyDeviceToHost));
        CKV_CUDA(cudaMemcpy(w.data(), x->s.edge_w, w.size() * 4, cudaMemcpyDeviceToHost));
        for (size_t g = 0; g < G; ++g) { memcpy(p, &deg[g * x->edge_rows], rows * 4); p += rows * 4; }
        for (size_t g = 0; g < G; ++g) {
            memcpy(p, &col[g * x->edge_rows * d.kappa], rows * d.kappa * 4);
            p += rows * d.kappa * 4;
        }
        for (size_t g = 0; g < G; ++g) {
            memcpy(p, &w[g * x->edge_rows * d.kappa], rows * d.kappa * 4);
            p += rows * d.kappa * 4;
        }
    }
    *bytes = need;
    return CKV_OK;
}

CKV_API ckv_status ckv_import_state(ckv_ctx* x, const void* host_buf, size_t bytes)
{
    FaultScope fault;
    if (!x || !host_buf || bytes < 36) return CKV_ERR_INVALID_ARG;
    int32_t hdr[9];
    memcpy(hdr, host_buf, sizeof hdr);
    Dims& d = x->d;
    if ((uint32_t)hdr[0] != kMagic || hdr[1] != 1 || hdr[2] != d.G || hdr[3] < 1 || hdr[3] > d.Nc ||
        hdr[4] != ckv::kD || hdr[6] != d.S || hdr[7] != d.kappa)
        return CKV_ERR_INVALID_ARG;
    const int Nc = hdr[3], n_tok = hdr[5], n_init = hdr[8];
    if (n_tok < d.S || n_tok > d.NM || n_init < d.S || n_init > n_tok) return CKV_ERR_INVALID_ARG;
    const size_t G = d.G, D = ckv::kD;
    const size_t nmem = (size_t)(n_tok - d.S), rows = (size_t)(n_tok - n_init);
    const size_t need = 36 + G * Nc * D * 4 + G * Nc * 4 + G * nmem * 4 + G * rows * 4 + 2 * G * rows * d.kappa * 4;
    if (bytes < need) return CKV_ERR_INVALID_ARG;
    const char* p = static_cast<const char*>(host_buf) + 36;
    const float* mu_in = reinterpret_cast<const float*>(p);
    p += G * Nc * D * 4;
    const int32_t* size_in = reinterpret_cast<const int32_t*>(p);
    p += G * Nc * 4;
    const int32_t* mem_in = reinterpret_cast<const int32_t*>(p);
    p += G * nmem * 4;
    const int32_t* deg_in = reinterpret_cast<const int32_t*>(p);
    p += G * rows * 4;
    const int32_t* col_in = reinterpret_cast<const int32_t*>(p);
    p += G * rows * d.kappa * 4;
    const float* w_in = reinterpret_cast<const float*>(p);
    // validate and lay out on the host
    std::vector<int32_t> size(G * d.Nc, 0), off(G * d.Nc, 0), cap(G * d.Nc, 0), top(G, 0);
    std::vector<int32_t> pool(G * (size_t)d.P, 0), tokc(G * (size_t)d.NM, -1);
    std::vector<float> mu(G * d.Nc * D, 0.f);
    std::vector<unsigned char> seen((size_t)n_tok);
    for (size_t g = 0; g < G; ++g) {
        std::fill(seen.begin(), seen.end(), 0);
        int64_t total = 0, o = 0;
        size_t k = 0;
        for (int c = 0; c < Nc; ++c) {
            const int32_t sz = size_in[g * Nc + c];
            if (sz < 0 || total + sz > (int64_t)nmem) return CKV_ERR_INVALID_ARG;
            total += sz;
            const int64_t cp = (int64_t)sz + x->cfg.slack;
            if (o + cp > d.P) return CKV_ERR_CAPACITY;
            size[g * d.Nc + c] = sz;
            off[g * d.Nc + c] = (int32_t)o;
            cap[g * d.Nc + c] = (int32_t)cp;
            for (int32_t r = 0; r < sz; ++r, ++k) {
                const int32_t j = mem_in[g * nmem + k];
                if (j < d.S || j >= n_tok || seen[j] || (r > 0 && j <= mem_in[g * nmem + k - 1]))
                    return CKV_ERR_INVALID_ARG;
                seen[j] = 1;
                pool[g * d.P + o + r] = j;
                tokc[g * d.NM + j] = c;
            }
            o += cp;
        }
        if (total != (int64_t)nmem) return CKV_ERR_INVALID_ARG;
        top[g] = (int32_t)o;
        memcpy(&mu[g * d.Nc * D], &mu_in[g * Nc * D], (size_t)Nc * D * 4);
        for (size_t i = 0; i < (size_t)Nc * D; ++i)
            if (!(std::fabs(mu_in[g * Nc * D + i]) <= FLT_MAX)) return CKV_ERR_INVALID_ARG;   // finite centroids
        for (size_t r = 0; r < rows; ++r) {
            const int32_t dg = deg_in[g * rows + r];
            if (dg < 0 || dg > d.kappa) return CKV_ERR_INVALID_ARG;
            // the token at n_init + r links to earlier ordinary positions
            for (int e = 0; e < dg; ++e) {
                const int32_t c = col_in[(g * rows + r) * d.kappa + e];
                if (c < d.S || c >= n_init + (int64_t)r || !valid_weight(w_in[(g * rows + r) * d.kappa + e]))
                    return CKV_ERR_INVALID_ARG;
            }
        }
    }
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaDeviceSynchronize());
    {
        EdgeStore es;
        const cudaError_t e = new_edges(x, (int64_t)d.NM - n_init, es);
        if (e != cudaSuccess) return cuda_status(e);   // the context keeps its state
        install_edges(x, es);
    }
    DevState& s = x->s;
    CKV_CUDA(cudaMemcpy(s.mu, mu.data(), mu.size() * 4, cudaMemcpyHostToDevice));
    CKV_CUDA(cudaMemcpy(s.csize, size.data(), size.size() * 4, cudaMemcpyHostToDevice));
    CKV_CUDA(cudaMemcpy(s.coff, off.data(), off.size() * 4, cudaMemcpyHostToDevice));
    CKV_CUDA(cudaMemcpy(s.ccap, cap.data(), cap.size() * 4, cudaMemcpyHostToDevice));
    CKV_CUDA(cudaMemcpy(s.pool, pool.data(), pool.size() * 4, cudaMemcpyHostToDevice));
    CKV_CUDA(cudaMemcpy(s.pool_top, top.data(), top.size() * 4, cudaMemcpyHostToDevice));
    CKV_CUDA(cudaMemcpy(s.tok_comm, tokc.data(), tokc.size() * 4, cudaMemcpyHostToDevice));
    if (rows) {
        const size_t er = (size_t)x->edge_rows;
        for (size_t g = 0; g < G; ++g) {
            CKV_CUDA(cudaMemcpy(s.edge_deg + g * er, deg_in + g * rows, rows * 4, cudaMemcpyHostToDevice));
            CKV_CUDA(cudaMemcpy(s.edge_col + g * er * d.kappa, col_in + g * rows * d.kappa, rows * d.kappa * 4,
                                cudaMemcpyHostToDevice));
            CKV_CUDA(cudaMemcpy(s.edge_w + g * er * d.kappa, w_in + g * rows * d.kappa, rows * d.kappa * 4,
                                cudaMemcpyHostToDevice));
        }
    }
    CKV_CUDA(cudaMemset(s.err, 0, sizeof(int)));
    CKV_CUDA(cudaMemset(s.bar, 0, G * 2 * sizeof(unsigned)));
    CKV_CUDA(cudaMemset(s.step_ctr, 0, 2 * sizeof(unsigned)));
    CKV_CUDA(cudaMemset(s.gcnt, 0, G * 4 * sizeof(unsigned)));
    CKV_CUDA(cudaMemset(s.shist, 0, G * ckv::step_hist_bins() * sizeof(unsigned)));
    CKV_CUDA(reset_srange(x, 0));
    CKV_CUDA(cudaDeviceSynchronize());
    d.n_comm = Nc;
    d.spg = (Nc + ckv::step_cpi() - 1) / ckv::step_cpi();
    d.n_init = n_init;
    x->n_tok = n_tok;
    x->pending = 0;
    x->last_n = 0;
    x->sticky = CKV_OK;
    x->initialized = 1;
    return CKV_OK;
}

#ifdef CKV_DEBUG_BOUNDS
// Fault injection of the debug build only: overwrite one int32 of the
// device community state, bypassing every host check, so that a test can
// show the kernels' range checks turning a corrupt entry into CKV_ERR_STATE.
CKV_API ckv_status ckv_debug_poke(ckv_ctx* x, int what, int g, int c, int r, int32_t value)
{
    if (!x || !x->initialized || g < 0 || g >= x->d.G || c < 0 || c >= x->d.n_comm) return CKV_ERR_INVALID_ARG;
    if (what != 0 && what != 1) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaDeviceSynchronize());
    const int64_t gi = (int64_t)g * x->d.Nc + c;
    if (what == 1) {
        CKV_CUDA(cudaMemcpy(x->s.coff + gi, &value, sizeof value, cudaMemcpyHostToDevice));
        return CKV_OK;
    }
    int32_t size = 0, off = 0;
    CKV_CUDA(cudaMemcpy(&size, x->s.csize + gi, sizeof size, cudaMemcpyDeviceToHost));
    CKV_CUDA(cudaMemcpy(&off, x->s.coff + gi, sizeof off, cudaMemcpyDeviceToHost));
    if (r < 0 || r >= size || off < 0 || (int64_t)off + r >= x->d.P) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaMemcpy(x->s.pool + (int64_t)g * x->d.P + off + r, &value, sizeof value, cudaMemcpyHostToDevice));
    return CKV_OK;
}
#endif

CKV_API ckv_status ckv_aux_bytes(const ckv_ctx* x, size_t* aux_bytes, size_t* kv_bytes)
{
    if (!x || !aux_bytes || !kv_bytes) return CKV_ERR_INVALID_ARG;
    const Dims& d = x->d;
    const size_t G = d.G, Nc = d.n_comm ? d.n_comm : d.Nc;
    *aux_bytes = G * Nc * ckv::kD * 4 + G * Nc * 12 + G * (size_t)d.P * 4 + G * (size_t)d.NM * 4 +
                 G * (size_t)x->edge_rows * (2 * (size_t)d.kappa + 1) * 4;
    *kv_bytes = 2 * (size_t)d.B * d.Hkv * d.NM * ckv::kD * elem_bytes(x->cfg.kv_dtype);
    return CKV_OK;
}

CKV_API ckv_status ckv_build_graph(int n_heads, int n, int head_dim, int n_sinks, int kappa, ckv_dtype dtype,
                                   const void* Q, const void* K, int64_t* row_ptr, int32_t* col, float* w,
                                   void* stream)
{
    if (n_heads < 1 || n < 1 || head_dim != ckv::kD || n_sinks < 0 || kappa < 1 || kappa > ckv::kMaxKappa ||
        dtype != CKV_BF16 || !Q || !K || !row_ptr || !col || !w)
        return CKV_ERR_INVALID_ARG;
    if ((int64_t)n_heads * n > INT32_MAX) return CKV_ERR_INVALID_ARG;
    cudaPointerAttributes a;
    CKV_CUDA(cudaPointerGetAttributes(&a, Q));
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(a.device));
    CKV_CUDA(ckv::launch_build_graph(n_heads, n, n_sinks, kappa, Q, K, row_ptr, col, w, (cudaStream_t)stream));
    return CKV_OK;
}

CKV_API ckv_status ckv_leiden(int n, const int64_t* row_ptr_host, const int32_t* col_host, const float* w_host,
                              double gamma, int32_t* labels_host, int* n_communities)
{
    if (n < 1 || !row_ptr_host || !labels_host || !n_communities || !valid_gamma(gamma)) return CKV_ERR_INVALID_ARG;
    if (row_ptr_host[0] != 0) return CKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (row_ptr_host[i + 1] < row_ptr_host[i]) return CKV_ERR_INVALID_ARG;
    const int64_t E = row_ptr_host[n];
    if (E > 0 && (!col_host || !w_host)) return CKV_ERR_INVALID_ARG;
    for (int64_t e = 0; e < E; ++e)
        if (col_host[e] < 0 || col_host[e] >= n || !valid_weight(w_host[e])) return CKV_ERR_INVALID_ARG;
    try {
        *n_communities = ckv::leiden_partition(n, row_ptr_host, col_host, w_host, gamma, 64, labels_host);
    } catch (...) {
        return CKV_ERR_OOM;
    }
    return CKV_OK;
}

CKV_API size_t ckv_modularity_workspace(int n_communities)
{
    return n_communities < 1 ? 0 : ckv::modularity_scratch_doubles(n_communities) * sizeof(double) + sizeof(double);
}

CKV_API ckv_status ckv_modularity(int n, const int64_t* row_ptr, const int32_t* col, const float* w,
                                  const int32_t* labels, int n_communities, double gamma, void* workspace,
                                  double* q_host, void* stream)
{
    if (n < 1 || n_communities < 1 || !row_ptr || !labels || !workspace || !q_host || !valid_gamma(gamma))
        return CKV_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 7) return CKV_ERR_INVALID_ARG;
    cudaPointerAttributes a;
    CKV_CUDA(cudaPointerGetAttributes(&a, row_ptr));
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(a.device));
    double* scratch = static_cast<double*>(workspace);
    double* q_dev = scratch + ckv::modularity_scratch_doubles(n_communities);
    cudaStream_t st = (cudaStream_t)stream;
    CKV_CUDA(ckv::launch_modularity(n, row_ptr, col, w, labels, n_communities, gamma, scratch, q_dev, st));
    CKV_CUDA(cudaMemcpyAsync(q_host, q_dev, sizeof(double), cudaMemcpyDeviceToHost, st));
    CKV_CUDA(cudaStreamSynchronize(st));
    if (*q_host != *q_host) return CKV_ERR_INVALID_ARG;   // a label or column out of range
    return CKV_OK;
}

// ---------------------------------------------------------------- refresh
CKV_API ckv_status ckv_set_token_graph(ckv_ctx* x, const int64_t* row_ptr_host, const int32_t* col_host,
                                       const float* w_host, int n)
{
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!row_ptr_host || !col_host || !w_host) return CKV_ERR_INVALID_ARG;
    if (!x->initialized || x->pending || n != x->d.n_init || n != x->n_tok) return CKV_ERR_STATE;
    const int G = x->d.G;
    const int64_t E = row_ptr_host[n];                         // edge stride of every graph
    std::vector<ckv_ctx::TokenGraph> tg((size_t)G);
    for (int g = 0; g < G; ++g) {
        const int64_t* rp = row_ptr_host + (size_t)g * (n + 1);
        if (rp[0] != 0 || rp[n] > E) return CKV_ERR_INVALID_ARG;
        for (int i = 0; i < n; ++i)
            if (rp[i + 1] < rp[i]) return CKV_ERR_INVALID_ARG;
        const int32_t* col = col_host + (size_t)g * E;
        const float* w = w_host + (size_t)g * E;
        for (int64_t e = 0; e < rp[n]; ++e)
            if (col[e] < 0 || col[e] >= n || !valid_weight(w[e])) return CKV_ERR_INVALID_ARG;
        tg[(size_t)g].rp.assign(rp, rp + n + 1);
        tg[(size_t)g].col.assign(col, col + rp[n]);
        tg[(size_t)g].w.assign(w, w + rp[n]);
    }
    x->tg.swap(tg);
    x->tg_rows = n;
    return CKV_OK;
}

namespace {

// the decode-time rows [n_init, n_tok) of every graph, from the device
cudaError_t fetch_decode_rows(ckv_ctx* x, std::vector<int32_t>& deg, std::vector<int32_t>& col,
                              std::vector<float>& w)
{
    const Dims& d = x->d;
    const size_t rows = (size_t)(x->n_tok - d.n_init), G = d.G, er = (size_t)x->edge_rows;
    deg.assign(G * rows, 0);
    col.assign(G * rows * d.kappa, 0);
    w.assign(G * rows * d.kappa, 0.f);
    if (!rows) return cudaSuccess;
    cudaError_t e;
    for (size_t g = 0; g < G; ++g) {
        if ((e = cudaMemcpy(&deg[g * rows], x->s.edge_deg + g * er, rows * 4, cudaMemcpyDeviceToHost)) != cudaSuccess)
            return e;
        if ((e = cudaMemcpy(&col[g * rows * d.kappa], x->s.edge_col + g * er * d.kappa, rows * d.kappa * 4,
                            cudaMemcpyDeviceToHost)) != cudaSuccess)
            return e;
        if ((e = cudaMemcpy(&w[g * rows * d.kappa], x->s.edge_w + g * er * d.kappa, rows * d.kappa * 4,
                            cudaMemcpyDeviceToHost)) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

// graph g's token graph over [0, n_tok): the host rows, then the decode rows
// the decode-time rows read back from the device are well formed: degrees
// in [0, kappa], the row of position n_init + r linking only to ordinary
// positions in [S, n_init + r), finite non-negative weights (host code
// indexes by them)
bool valid_decode_rows(const ckv_ctx* x, const std::vector<int32_t>& deg, const std::vector<int32_t>& col,
                       const std::vector<float>& w)
{
    const int kap = x->d.kappa;
    const size_t rows = (size_t)(x->n_tok - x->d.n_init);
    for (size_t i0 = 0; i0 < deg.size(); ++i0) {
        if (deg[i0] < 0 || deg[i0] > kap) return false;
        const int64_t hi = (int64_t)x->d.n_init + (int64_t)(rows ? i0 % rows : 0);
        for (int k = 0; k < deg[i0]; ++k) {
            const size_t i = i0 * (size_t)kap + (size_t)k;
            if (col[i] < x->d.S || col[i] >= hi || !valid_weight(w[i])) return false;
        }
    }
    return true;
}

ckv_ctx::TokenGraph combined_graph(const ckv_ctx* x, int g, const std::vector<int32_t>& deg,
                                   const std::vector<int32_t>& col, const std::vector<float>& w)
{
    const Dims& d = x->d;
    const size_t rows = (size_t)(x->n_tok - d.n_init);
    ckv_ctx::TokenGraph t = x->tg[(size_t)g];
    for (size_t r = 0; r < rows; ++r) {
        const int nd = deg[(size_t)g * rows + r];
        for (int k = 0; k < nd; ++k) {
            t.col.push_back(col[((size_t)g * rows + r) * d.kappa + k]);
            t.w.push_back(w[((size_t)g * rows + r) * d.kappa + k]);
        }
        t.rp.push_back((int64_t)t.col.size());
    }
    return t;
}

}  // namespace

CKV_API ckv_status ckv_refresh(ckv_ctx* x, const void* K, double gamma, int32_t* n_communities_host, void* stream)
{
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!K || !valid_gamma(gamma)) return CKV_ERR_INVALID_ARG;
    if (!x->initialized || x->pending || x->tg.empty() || x->tg_rows != x->d.n_init) return CKV_ERR_STATE;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    cs = read_device_error(x);
    if (cs != CKV_OK) { x->sticky = cs; return cs; }
    std::vector<int32_t> deg, col;
    std::vector<float> w;
    CKV_CUDA(fetch_decode_rows(x, deg, col, w));
    if (!valid_decode_rows(x, deg, col, w)) return CKV_ERR_STATE;
    const int G = x->d.G, n = x->n_tok;
    std::vector<ckv_ctx::TokenGraph> next((size_t)G);
    std::vector<int32_t> labels((size_t)G * n), counts((size_t)G, 0);
    // the graphs are independent: partition them on several host threads
    const int nthr = std::max(1, std::min(G, (int)std::thread::hardware_concurrency()));
    std::vector<std::thread> pool;
    std::vector<char> failed((size_t)nthr + 1, 0);
    auto work = [&](int t) {
        try {
            for (int g = t; g < G; g += nthr) {
                next[(size_t)g] = combined_graph(x, g, deg, col, w);
                counts[(size_t)g] = ckv::leiden_partition(n, next[(size_t)g].rp.data(), next[(size_t)g].col.data(),
                                                          next[(size_t)g].w.data(), gamma, 64, &labels[(size_t)g * n]);
            }
        } catch (...) {
            failed[(size_t)t] = 1;
        }
    };
    try {
        for (int t = 1; t < nthr; ++t) pool.emplace_back(work, t);
    } catch (...) {
        failed[(size_t)nthr] = 1;   // fewer threads: this one still covers its own share below
    }
    work(0);
    for (auto& th : pool) th.join();
    if (failed[(size_t)nthr]) {     // a thread could not start: finish its graphs here
        for (int t = (int)pool.size() + 1; t < nthr; ++t) work(t);
    }
    for (int t = 0; t < nthr; ++t)
        if (failed[(size_t)t]) return CKV_ERR_OOM;
    const int nc = *std::max_element(counts.begin(), counts.end());
    if (nc > x->d.Nc) return CKV_ERR_CAPACITY;   // the state is unchanged
    cs = ckv_init_communities(x, labels.data(), 0, nc, K, n, stream);
    if (cs != CKV_OK) return cs;
    x->tg.swap(next);
    x->tg_rows = n;
    if (n_communities_host)
        for (int g = 0; g < G; ++g) n_communities_host[g] = counts[(size_t)g];
    return CKV_OK;
}

CKV_API ckv_status ckv_graph_modularity(ckv_ctx* x, double gamma, double* q_host, void* stream)
{
    FaultScope fault;
    ckv_status cs = check_ctx(x);
    if (cs != CKV_OK) return cs;
    if (!q_host || !valid_gamma(gamma)) return CKV_ERR_INVALID_ARG;
    if (!x->initialized || x->pending || x->tg.empty() || x->tg_rows != x->d.n_init) return CKV_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    CKV_CUDA(cudaSetDevice(x->cfg.device));
    CKV_CUDA(cudaStreamSynchronize(st));
    std::vector<int32_t> deg, col;
    std::vector<float> w;
    CKV_CUDA(fetch_decode_rows(x, deg, col, w));
    if (!valid_decode_rows(x, deg, col, w)) return CKV_ERR_STATE;
    const Dims& d = x->d;
    const int n = x->n_tok;
    std::vector<int32_t> lab((size_t)n);
    for (int g = 0; g < d.G; ++g) {
        const ckv_ctx::TokenGraph t = combined_graph(x, g, deg, col, w);
        CKV_CUDA(cudaMemcpy(lab.data(), x->s.tok_comm + (size_t)g * d.NM, (size_t)n * 4, cudaMemcpyDeviceToHost));
        for (int32_t& l : lab) l = (l < 0) ? d.n_comm : l;      // sinks (no edges): one extra label
        const size_t E = t.col.size();
        void* buf = nullptr;
        const size_t bytes = (size_t)(n + 1) * 8 + E * 8 + (size_t)n * 4 + ckv_modularity_workspace(d.n_comm + 1) + 64;
        CKV_CUDA(dev_malloc(&buf, bytes));
        char* p = static_cast<char*>(buf);
        int64_t* drp = reinterpret_cast<int64_t*>(p);
        int32_t* dcol = reinterpret_cast<int32_t*>(p + (size_t)(n + 1) * 8);
        float* dw = reinterpret_cast<float*>(p + (size_t)(n + 1) * 8 + E * 4);
        int32_t* dlab = reinterpret_cast<int32_t*>(p + (size_t)(n + 1) * 8 + E * 8);
        void* ws = reinterpret_cast<void*>(((uintptr_t)(p + (size_t)(n + 1) * 8 + E * 8 + (size_t)n * 4) + 15) & ~(uintptr_t)15);
        cudaError_t e = cudaMemcpy(drp, t.rp.data(), (size_t)(n + 1) * 8, cudaMemcpyHostToDevice);
        if (e == cudaSuccess && E) e = cudaMemcpy(dcol, t.col.data(), E * 4, cudaMemcpyHostToDevice);
        if (e == cudaSuccess && E) e = cudaMemcpy(dw, t.w.data(), E * 4, cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemcpy(dlab, lab.data(), (size_t)n * 4, cudaMemcpyHostToDevice);
        ckv_status r = (e == cudaSuccess) ? ckv_modularity(n, drp, dcol, dw, dlab, d.n_comm + 1, gamma, ws,
                                                           &q_host[g], stream)
                                          : CKV_ERR_CUDA;
        cudaFree(buf);
        if (r != CKV_OK) return r;
    }
    return CKV_OK;
}

CKV_API size_t ckv_build_graph_grouped_workspace(int n_kv_heads, int group, int n)
{
    if (n_kv_heads < 1 || group < 1 || n < 1) return 0;
    return ckv::build_graph_grouped_stats_floats(n_kv_heads, group, n) * sizeof(float);
}

CKV_API ckv_status ckv_build_graph_grouped(int n_kv_heads, int group, int n, int head_dim, int n_sinks, int kappa,
                                           ckv_dtype dtype, const void* Q, const void* K, void* workspace,
                                           int64_t* row_ptr, int32_t* col, float* w, void* stream)
{
    if (n_kv_heads < 1 || (group != 1 && group != 2 && group != 4) || n < 1 || head_dim != ckv::kD ||
        n_sinks < 0 || kappa < 1 || kappa > ckv::kMaxKappa || dtype != CKV_BF16 || !Q || !K || !workspace ||
        !row_ptr || !col || !w)
        return CKV_ERR_INVALID_ARG;
    if ((int64_t)n_kv_heads * group * n > INT32_MAX / 2) return CKV_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15) return CKV_ERR_INVALID_ARG;
    cudaPointerAttributes a;
    CKV_CUDA(cudaPointerGetAttributes(&a, Q));
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return CKV_ERR_INVALID_ARG;
    CKV_CUDA(cudaSetDevice(a.device));
    CKV_CUDA(ckv::launch_build_graph_grouped(n_kv_heads, group, n, n_sinks, kappa, Q, K,
                                             static_cast<float*>(workspace), row_ptr, col, w,
                                             (cudaStream_t)stream));
    return CKV_OK;
}
