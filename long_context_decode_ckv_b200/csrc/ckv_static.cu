// ckv_static.cu -- sparse decode attention over caller-chosen rows with no
// device allocation.
//
// Some hosts cannot call cudaMalloc where this runs: plugin-style
// integrations (an inference engine's custom-op execute path, for example)
// that forbid device allocation after set-up and hand the op no workspace.
// For them ckv_attend_rows_static runs the attention items of the library's
// fused decode kernel (the gather, the tensor-core contractions and the
// merge of the partials that ckv_decode_step uses) with its scratch -- the
// row lists, per-item softmax statistics and P.V partials, the queue and
// arrival counters -- in the file-scope device array below instead of
// memory from a context.
//
// The array is kStaticScratchBytes per device and stays resident on every
// GPU that loads the library until the process exits.  Every call shares
// it: the call clears the counters it needs, copies the row lists in,
// launches on `stream`, reads the kernel's error word back and waits for
// the stream, so it is synchronous and cannot be captured into a graph;
// calls from different host threads race on the array and must be
// serialised by the caller.  The first call on a device looks up the
// array's device address and sets the kernel's launch attributes.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "ckv_internal.cuh"

#define CKV_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct DeviceSetup {
    void* addr;     // device address of g_static_scratch
    int sms;
};
std::mutex g_setup_mutex;
DeviceSetup g_setup[kMaxDevices];

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Restores the caller's current device when the call returns.
struct DeviceGuard {
    int prev = -1;
    cudaError_t enter(int dev)
    {
        cudaError_t e = cudaGetDevice(&prev);
        if (e != cudaSuccess) { prev = -1; return e; }
        return prev == dev ? cudaSuccess : cudaSetDevice(dev);
    }
    ~DeviceGuard()
    {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

}  // namespace

CKV_API ckv_status ckv_attend_rows_static(const ckv_config* cfg, const void* q, const void* K, const void* V,
                                          int n, const int32_t* rows_host, const int32_t* n_rows_host,
                                          int max_rows, float* out, void* stream)
{
    using ckv::kD;
    if (!cfg || !q || !K || !V || !out || !rows_host || !n_rows_host) return CKV_ERR_INVALID_ARG;
    if (cfg->batch < 1 || cfg->n_q_heads < 1 || cfg->n_kv_heads < 1 || cfg->n_q_heads % cfg->n_kv_heads ||
        cfg->head_dim != kD || cfg->n_max < 1 || cfg->n_sinks < 0 || cfg->device < 0 ||
        (cfg->kv_dtype != CKV_F32 && cfg->kv_dtype != CKV_BF16) ||
        (cfg->mode != CKV_PER_HEAD && cfg->mode != CKV_QUERY_GROUP))
        return CKV_ERR_INVALID_ARG;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || cfg->device >= ndev || cfg->device >= kMaxDevices)
        return CKV_ERR_INVALID_ARG;
    const int Gq = cfg->n_q_heads / cfg->n_kv_heads;
    const int HG = cfg->mode == CKV_QUERY_GROUP ? Gq : 1;
    if (HG != 1 && HG != 2 && HG != 4 && HG != 8) return CKV_ERR_INVALID_ARG;
    if (n < cfg->n_sinks + 1 || n > cfg->n_max || max_rows < 0) return CKV_ERR_INVALID_ARG;
    const int64_t G64 = cfg->mode == CKV_QUERY_GROUP ? (int64_t)cfg->batch * cfg->n_kv_heads
                                                     : (int64_t)cfg->batch * cfg->n_q_heads;
    if (G64 > (1 << 20)) return CKV_ERR_INVALID_ARG;
    const int G = (int)G64;
    // every row must be an ordinary past position: not a sink, not the new token
    for (int g = 0; g < G; ++g) {
        const int T = n_rows_host[g];
        if (T < 0 || T > max_rows) return CKV_ERR_INVALID_ARG;
        for (int r = 0; r < T; ++r) {
            const int32_t j = rows_host[(int64_t)g * max_rows + r];
            if (j < cfg->n_sinks || j >= n - 1) return CKV_ERR_INVALID_ARG;
        }
    }

    ckv::Dims d{};
    d.B = cfg->batch;
    d.Hq = cfg->n_q_heads;
    d.Hkv = cfg->n_kv_heads;
    d.Gq = Gq;
    d.G = G;
    d.HG = HG;
    d.NM = cfg->n_max;
    d.S = cfg->n_sinks;
    d.kappa = 1;
    d.mode = cfg->mode;
    d.bf16 = cfg->kv_dtype == CKV_BF16;
    d.rows_given = 1;
    d.rtok_stride = max_rows;
    d.api = ckv::step_api(d.S, max_rows);
    d.wait_polls = ckv::kStepWaitPolls;
    // scratch layout: counters (queue head, CTAs done, error word, pad,
    // graphs' arrivals) | kept-row counts | row lists | partials
    const size_t A = (size_t)d.api;
    size_t off = 0;
    const size_t o_ctr = off;   off = align256(off + (4 + 4 * (size_t)G) * 4);
    const size_t o_rT = off;    off = align256(off + (size_t)G * 4);
    const size_t o_rtok = off;  off = align256(off + (size_t)G * max_rows * 4);
    const size_t o_pml = off;   off = align256(off + (size_t)G * A * HG * 2 * 4);
    const size_t o_po = off;    off = align256(off + (size_t)G * A * HG * kD * 4);
    if (off > kStaticScratchBytes) return CKV_ERR_CAPACITY;   // the rows and partials do not fit the array

    DeviceGuard guard;
    if (guard.enter(cfg->device) != cudaSuccess) return CKV_ERR_CUDA;
    DeviceSetup su;
    {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        DeviceSetup& ds = g_setup[cfg->device];
        if (!ds.addr) {
            // the host-side name g_static_scratch is only a stand-in: a
            // kernel must be given the address this returns
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return CKV_ERR_CUDA;
            if (cudaDeviceGetAttribute(&ds.sms, cudaDevAttrMultiProcessorCount, cfg->device) != cudaSuccess)
                return CKV_ERR_CUDA;
            ds.addr = p;
        }
        su = ds;
    }
    int grid = 0;
    if (ckv::prepare_step(d, su.sms, &grid) != cudaSuccess || grid < 1) return CKV_ERR_CUDA;
    d.nStep = grid;
    d.n_workers = G < ckv::kStepWorkers ? G : ckv::kStepWorkers;
    if (d.n_workers > grid / 2) d.n_workers = grid / 2;
    unsigned char* sb = static_cast<unsigned char*>(su.addr);
    ckv::DevState s{};
    s.step_ctr = reinterpret_cast<unsigned*>(sb + o_ctr);
    s.err = reinterpret_cast<int*>(sb + o_ctr + 8);
    s.gcnt = reinterpret_cast<unsigned*>(sb + o_ctr + 16);
    s.rows_T = reinterpret_cast<const int32_t*>(sb + o_rT);
    s.rtok = reinterpret_cast<int32_t*>(sb + o_rtok);
    s.part_ml = reinterpret_cast<float*>(sb + o_pml);
    s.part_o = reinterpret_cast<float*>(sb + o_po);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(sb + o_ctr, 0, (4 + 4 * (size_t)G) * 4, st);
    // host -> device copies straight from the caller's buffers; the call
    // waits for the stream before it returns, so the buffers (pageable or
    // page-locked) may be reused as soon as it does
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(sb + o_rT, n_rows_host, (size_t)G * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && max_rows > 0)
        e = cudaMemcpyAsync(sb + o_rtok, rows_host, (size_t)G * max_rows * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = ckv::launch_step(s, d, q, K, V, n, out, st);
    // the kernel's own checks (a row outside the cache, a wait that ran
    // out) land in the error word
    int err = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&err, s.err, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return CKV_ERR_CUDA;
    return err ? (ckv_status)err : CKV_OK;
}
