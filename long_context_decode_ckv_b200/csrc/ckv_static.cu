// ckv_static.cu -- sparse decode attention over caller-chosen rows with no
// device allocation.
//
// Some hosts cannot call cudaMalloc where this runs: plugin-style
// integrations (an inference engine's custom-op execute path, for example)
// that forbid device allocation after set-up and hand the op no workspace.
// For them ckv_attend_rows_static runs the library's gather-attention
// kernel (the one ckv_decode_step uses) with its scratch -- row list,
// logits, per-CTA softmax statistics and P.V partials, arrival counter,
// edge ranking -- in the file-scope device array below instead of memory
// from a context.
//
// The array is kStaticScratchBytes per device and stays resident on every
// GPU that loads the library until the process exits.  Every call shares
// it: the call clears the counter and error word it needs, copies its row
// list in, and launches on `stream`; calls whose work overlaps on the GPU
// (different streams, or different host threads) race on it and must be
// serialised by the caller.  The first call on a device looks up the
// array's device address; make that first call before any stream capture.
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

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];   // device address of g_static_scratch, per device

// Device address of the scratch array on `dev` (the current device).  The
// host-side name g_static_scratch is only a stand-in; a kernel must get the
// address returned by cudaGetSymbolAddress.
cudaError_t scratch_address(int dev, void** out)
{
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

CKV_API ckv_status ckv_attend_rows_static(const ckv_config* cfg, const void* q, const void* K, const void* V,
                                          int n, const int32_t* rows_host, const int32_t* n_rows_host,
                                          int max_rows, float* out, void* stream)
{
    using ckv::kD;
    if (!cfg || !q || !K || !V || !out || !rows_host || !n_rows_host) return CKV_ERR_INVALID_ARG;
    if (cfg->batch < 1 || cfg->n_q_heads < 1 || cfg->n_kv_heads < 1 || cfg->n_q_heads % cfg->n_kv_heads ||
        cfg->head_dim != kD || cfg->n_max < 1 || cfg->n_sinks < 0 || cfg->device < 0 ||
        cfg->device >= kMaxDevices || (cfg->kv_dtype != CKV_F32 && cfg->kv_dtype != CKV_BF16) ||
        (cfg->mode != CKV_PER_HEAD && cfg->mode != CKV_QUERY_GROUP))
        return CKV_ERR_INVALID_ARG;
    const int Gq = cfg->n_q_heads / cfg->n_kv_heads;
    const int HG = cfg->mode == CKV_QUERY_GROUP ? Gq : 1;
    if (HG != 1 && HG != 2 && HG != 4 && HG != 8) return CKV_ERR_INVALID_ARG;
    if (n < cfg->n_sinks + 1 || n > cfg->n_max || max_rows < 0) return CKV_ERR_INVALID_ARG;
    const int G = cfg->mode == CKV_QUERY_GROUP ? cfg->batch * cfg->n_kv_heads : cfg->batch * cfg->n_q_heads;
    // every row must be an ordinary past position: not a sink, not the new token
    for (int g = 0; g < G; ++g) {
        const int T = n_rows_host[g];
        if (T < 0 || T > max_rows) return CKV_ERR_INVALID_ARG;
        for (int r = 0; r < T; ++r) {
            const int32_t j = rows_host[(int64_t)g * max_rows + r];
            if (j < cfg->n_sinks || j >= n - 1) return CKV_ERR_INVALID_ARG;
        }
    }
    int sms = 0;
    cudaError_t e = cudaSetDevice(cfg->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, cfg->device);
    void* base = nullptr;
    if (e == cudaSuccess) e = scratch_address(cfg->device, &base);
    if (e != cudaSuccess) return CKV_ERR_CUDA;

    // one graph per launch, so the scratch holds a single graph's rows
    ckv::Dims d{};
    d.B = 1;
    d.Hkv = 1;
    d.Hq = HG;
    d.Gq = HG;
    d.G = 1;
    d.HG = HG;
    d.NM = cfg->n_max;
    d.S = cfg->n_sinks;
    d.kappa = 1;          // the kernel also ranks one edge; this call discards it
    d.mode = CKV_QUERY_GROUP;
    d.bf16 = cfg->kv_dtype == CKV_BF16;
    const int grid = ckv::attend_grid(d, sms);
    if (grid < 1) return CKV_ERR_CUDA;
    // at most one CTA per 64 rows of the largest graph
    const int64_t rows_max = (int64_t)d.S + max_rows + 1;
    d.nCTA = (int)((rows_max + 63) / 64 < grid ? (rows_max + 63) / 64 : grid);
    // scratch layout: meta | bar | err | edges | row list | logits | partials
    const size_t KC = d.nCTA;
    size_t off = 0;
    const size_t o_meta = off;  off = align256(off + ckv::M_COUNT * 4);
    const size_t o_bar = off;   off = align256(off + 2 * 4);
    const size_t o_err = off;   off = align256(off + 4);
    const size_t o_e = off;     off = align256(off + 3 * 4);
    // (graph index 0 in every launch: the row list holds max_rows entries and
    // the spill logits rows_max rows, whatever the cache length)
    const size_t o_rtok = off;  off = align256(off + (size_t)max_rows * 4);
    const size_t o_zrow = off;  off = align256(off + (size_t)rows_max * HG * 4);
    const size_t o_pml = off;   off = align256(off + KC * HG * 2 * 4);
    const size_t o_po = off;    off = align256(off + KC * HG * kD * 4);
    if (off > kStaticScratchBytes) return CKV_ERR_CAPACITY;   // max_rows too large for the array
    unsigned char* sb = static_cast<unsigned char*>(base);
    ckv::DevState s{};
    s.meta = reinterpret_cast<int32_t*>(sb + o_meta);
    s.bar = reinterpret_cast<unsigned int*>(sb + o_bar);
    s.err = reinterpret_cast<int*>(sb + o_err);
    s.e_tok = reinterpret_cast<int32_t*>(sb + o_e);
    s.e_w = reinterpret_cast<float*>(sb + o_e + 4);
    s.e_comm = reinterpret_cast<int32_t*>(sb + o_e + 8);
    s.rtok = reinterpret_cast<int32_t*>(sb + o_rtok);
    s.rcomm = s.rtok;     // community of a row: only read for the edges, which this call discards
    s.zrow = reinterpret_cast<float*>(sb + o_zrow);
    s.part_ml = reinterpret_cast<float*>(sb + o_pml);
    s.part_o = reinterpret_cast<float*>(sb + o_po);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t eb = d.bf16 ? 2 : 4;
    for (int g = 0; g < G; ++g) {
        int b, h0, kvh;
        if (cfg->mode == CKV_QUERY_GROUP) { b = g / cfg->n_kv_heads; kvh = g % cfg->n_kv_heads; h0 = kvh * Gq; }
        else { b = g / cfg->n_q_heads; h0 = g % cfg->n_q_heads; kvh = h0 / Gq; }
        const int T = n_rows_host[g];
        int32_t meta[ckv::M_COUNT] = {0};
        meta[ckv::M_T] = T;
        meta[ckv::M_ROWS] = d.S + T + 1;
        const char* qg = static_cast<const char*>(q) + ((int64_t)b * cfg->n_q_heads + h0) * kD * eb;
        const char* Kg = static_cast<const char*>(K) + ((int64_t)b * cfg->n_kv_heads + kvh) * cfg->n_max * kD * eb;
        const char* Vg = static_cast<const char*>(V) + ((int64_t)b * cfg->n_kv_heads + kvh) * cfg->n_max * kD * eb;
        float* og = out + ((int64_t)b * cfg->n_q_heads + h0) * kD;
        e = cudaMemcpyAsync(s.meta, meta, sizeof meta, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess && T > 0)
            e = cudaMemcpyAsync(s.rtok, rows_host + (int64_t)g * max_rows, (size_t)T * 4, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(sb + o_bar, 0, 256 + 256, st);   // arrival counters, error word
        if (e == cudaSuccess) e = ckv::launch_attend(s, d, qg, Kg, Vg, n, og, st);
        if (e != cudaSuccess) return CKV_ERR_CUDA;
    }
    return CKV_OK;
}
