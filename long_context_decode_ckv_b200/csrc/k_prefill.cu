// k_prefill.cu -- prefill top-kappa token graph on the sm_100a tensor cores.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 1 caption, step (1) Graph Construction: during prefill each query
// is connected to its top-kappa keys of the attention matrix, sink tokens
// excluded from the pool; Table 10 times this "fused top-kappa selection"
// inside prefill.  Here: for each head and causal row i, z_ij = q_i.k_j /
// sqrt(D) over j <= i; edges = top-kappa of j in [S, i-1] by (z desc, j asc)
// with weight softmax_j(z)_ij over [0, i].  The n x n matrix never leaves
// the SM: a 128 x 128 tile of Q K^T lives in tensor memory only.
//
// One CTA per (head, 128-row query block), heaviest (longest causal row
// range) blocks first.  Warp roles:
//   warp 0      TMA producer: Q block once, then K tiles through a 3-stage
//               ring (128-byte swizzled, the layout tcgen05 reads).
//   warp 1      allocates 256 TMEM columns (two 128 x 128 fp32
//               accumulators) and issues tcgen05.mma (kind::f16, bf16 in,
//               fp32 accumulate, M = N = 128, K = 16 x 8) from one thread.
//   warps 2..17 epilogue, four warps per TMEM lane quarter: thread = one
//               query row (its TMEM lane) and one 32-column chunk of every
//               tile; it reads the chunk with tcgen05.ld and keeps the
//               online softmax (max, sum of exp2) and a sorted register
//               top-KM list; the four parts of a row merge at the end.
//               Four warps per quarter keep more independent rows in
//               flight: the per-row work is a chain of dependent steps.
// Every mbarrier wait is bounded; a wait that runs out marks row_ptr[h][0]
// = -1 (an impossible offset), every role leaves its loop, and the TMEM is
// freed before the CTA exits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stddef.h>
#include <stdint.h>

#include "ckv_internal.cuh"

namespace ckv {

namespace {

constexpr int kBM = 128, kBN = 128;
constexpr int kStages = 4;                           // K ring of the grouped kernel
constexpr int kThreads = 192;                        // the grouped kernel: producer, MMA, 4 epilogue warps
constexpr int kStagesH = 3;                          // K ring of the per-head kernel
constexpr int kParts = 4;                            // per-head kernel: epilogue warps per TMEM lane quarter
constexpr int kEpiWarps = 4 * kParts;
constexpr int kThreadsH = 64 + 32 * kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kMaxKM = 32;
constexpr int kHalfBytes = kBM * 64 * 2;            // one 64-column half of a 128-row tile
constexpr int kTileBytes = 2 * kHalfBytes;           // 32 KB
constexpr float kLog2eOverSqrtD = 0.12751743082459868f;   // log2(e) / sqrt(128)

struct __align__(1024) PrefillSmem {
    unsigned char q[kTileBytes];
    unsigned char k[kStagesH][kTileBytes];
    unsigned long long bar_q;
    unsigned long long bar_kfull[kStagesH];
    unsigned long long bar_kempty[kStagesH];
    unsigned long long bar_afull[2];
    unsigned long long bar_aempty[2];
    uint32_t tmem_base;
    int abort;
    // each part's current KM-th best score of each row (a lower bound of the
    // row's final KM-th: every part gates its candidates by the largest)
    float thr[kBM][kParts];
    // a part's row state, merged into part 0's at the end
    float xm[kBM][2];
    union {
        float stage[32 * kEpiThreads];   // during the loop: a gated chunk's values, column k of thread e at [k * kEpiThreads + e]
        struct {
            float v[kBM][kMaxKM];
            int i[kBM][kMaxKM];
        } x;                             // at the end: a part's top-KM list per row
    } u;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(unsigned long long* b, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long* b, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

// bounded wait for the phase with the given parity to complete.  Each poll
// may suspend the thread for up to kSuspendNs (it wakes as soon as the phase
// completes), so a waiting role issues few instructions; at most
// kWaitPolls polls, about a second, before the CTA gives up.
constexpr unsigned kSuspendNs = 4000;
constexpr unsigned kWaitPolls = 1u << 18;
__device__ __forceinline__ bool mbar_wait(unsigned long long* b, unsigned parity, volatile int* abort)
{
    const uint32_t a = smem_u32(b);
    for (unsigned it = 0; it < kWaitPolls; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity), "r"(kSuspendNs)
            : "memory");
        if (done) return true;
        if ((it & 63) == 63 && *abort) return false;
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, unsigned long long* bar,
                                            int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// UMMA shared-memory descriptor of a K-major, 128-byte-swizzled bf16 tile:
// rows 128 B apart, 8-row groups 1024 B apart (SBO), version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
    d |= (uint64_t)(16 >> 4) << 16;                   // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset
    d |= (uint64_t)1 << 46;                           // descriptor version
    d |= (uint64_t)2 << 61;                           // layout: SWIZZLE_128B
    return d;
}

// instruction descriptor: D f32, A and B bf16, both K-major, M = 128, N = n
constexpr uint32_t idesc_n(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}
constexpr uint32_t kIdesc = idesc_n(kBN);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accum,
                                          uint32_t idesc = kIdesc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

__device__ __forceinline__ void umma_commit(unsigned long long* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

// 32 columns of this warp's TMEM lanes, without waiting (tmem_wait_tie does)
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// waits for this thread's outstanding tcgen05.ld and ties r to the wait, so
// that no use of r is scheduled before it
__device__ __forceinline__ void tmem_wait_tie(uint32_t (&r)[32], bool wait)
{
    if (wait) asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                   "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                   "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// Insert the chunk's candidates (columns j0 + k, k in the bit mask) into the
// sorted top-KM list.  Candidates are rare after a row's first columns, so
// the loop over them stays rolled and only one copy of the insertion
// network is emitted (an unrolled copy per column thrashed the
// instruction cache).  Ties keep the earlier column ahead.
template <int KM>
__device__ __forceinline__ void insert_candidates(unsigned cm, const float (&v)[32], int j0, float (&vals)[KM],
                                                  int (&idx)[KM])
{
#pragma unroll 1
    while (cm) {
        const int k = __ffs(cm) - 1;
        cm &= cm - 1;
        float a = v[0];
#pragma unroll
        for (int kk = 1; kk < 32; ++kk) a = (k == kk) ? v[kk] : a;
        if (!(a > vals[KM - 1])) continue;      // the list rose past it since the mask was taken
        const int j = j0 + k;
#pragma unroll
        for (int p = KM - 1; p > 0; --p) {
            const float up = vals[p - 1];
            const int upi = idx[p - 1];
            const bool shift = up < a;
            const bool land = !shift && vals[p] < a;
            vals[p] = shift ? up : (land ? a : vals[p]);
            idx[p] = shift ? upi : (land ? j : idx[p]);
        }
        if (vals[0] < a) { vals[0] = a; idx[0] = j; }
    }
}

// The same with the chunk's values staged in shared memory (column k of
// this thread at stage[k * stride]): a candidate is one load instead of a
// select over 32 registers.
template <int KM>
__device__ __forceinline__ void insert_staged(unsigned cm, const float* stage, int stride, int j0, float (&vals)[KM],
                                              int (&idx)[KM])
{
#pragma unroll 1
    while (cm) {
        const int k = __ffs(cm) - 1;
        cm &= cm - 1;
        const float a = stage[k * stride];
        if (!(a > vals[KM - 1])) continue;      // the list rose past it since the mask was taken
        const int j = j0 + k;
#pragma unroll
        for (int p = KM - 1; p > 0; --p) {
            const float up = vals[p - 1];
            const int upi = idx[p - 1];
            const bool shift = up < a;
            const bool land = !shift && vals[p] < a;
            vals[p] = shift ? up : (land ? a : vals[p]);
            idx[p] = shift ? upi : (land ? j : idx[p]);
        }
        if (vals[0] < a) { vals[0] = a; idx[0] = j; }
    }
}

// Insert one candidate (value a, column j) into the sorted top-KM list
// (callers know a ranks above the list's last entry).
template <int KM>
__device__ __forceinline__ void insert_one(float a, int j, float (&vals)[KM], int (&idx)[KM])
{
#pragma unroll
    for (int p = KM - 1; p > 0; --p) {
        const float up = vals[p - 1];
        const int upi = idx[p - 1];
        const bool shift = up < a;
        const bool land = !shift && vals[p] < a;
        vals[p] = shift ? up : (land ? a : vals[p]);
        idx[p] = shift ? upi : (land ? j : idx[p]);
    }
    if (vals[0] < a) { vals[0] = a; idx[0] = j; }
}

// barrier 1 among the per-head kernel's epilogue warps only
__device__ __forceinline__ void epi_sync()
{
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kEpiWarps) : "memory");
}

// the largest float below x (x finite or -inf): "v >= x" is "v > below(x)"
__device__ __forceinline__ float below(float x)
{
    if (x == -INFINITY) return x;
    const int b = __float_as_int(x);
    if (x > 0.f) return __int_as_float(b - 1);
    if (x < 0.f) return __int_as_float(b + 1);
    return -1.4e-45f;   // below +-0: the negative subnormal of least magnitude
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// edges before row i: rows S+1 .. S+kappa have 1 .. kappa edges, later rows kappa
__device__ __forceinline__ int64_t row_offset(int64_t i, int S, int kappa)
{
    const int64_t a = max((int64_t)0, min(i, (int64_t)S + kappa + 1) - S - 1);
    return a * (a + 1) / 2 + max((int64_t)0, i - (S + kappa + 1)) * kappa;
}

// STATS: no edges; each row's (max of z log2(e), sum of 2^(z log2(e) - max))
// go to stats[h][i][2] instead (the first pass of the query-group graph),
// and a bounded wait that runs out sets the int word after them.
// group: query heads per KV head (the K rows of head h are those of h / group).
static_assert(sizeof(PrefillSmem) + 1024 <= 227 * 1024, "the per-head kernel's shared memory fits one CTA");
static_assert(kParts == 4, "the gate reads a row's four part thresholds");

template <int KM, bool STATS>
__global__ void __launch_bounds__(kThreadsH, 1)
k_prefill_topk(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int H, int n,
               int S, int kappa, int group, int64_t* __restrict__ row_ptr, int32_t* __restrict__ col,
               float* __restrict__ w, float* __restrict__ stats)
{
    extern __shared__ unsigned char smem_raw[];
    PrefillSmem& sm = *reinterpret_cast<PrefillSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = (n + kBM - 1) / kBM;
    const int qb = nqb - 1 - (int)(blockIdx.x / H);    // heaviest blocks first
    const int h = (int)(blockIdx.x % H);
    const int i0 = qb * kBM;
    const int ntiles = qb + 1;
    const int64_t E = row_offset(n, S, kappa);

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < kStagesH; ++s) { mbar_init(&sm.bar_kfull[s], 1); mbar_init(&sm.bar_kempty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&sm.bar_afull[b], 1); mbar_init(&sm.bar_aempty[b], kEpiWarps); }
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;"
                     ::"r"(smem_u32(&sm.tmem_base)) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort = &sm.abort;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(&sm.bar_q, kTileBytes);
            tma_load_3d(sm.q, &tmQ, &sm.bar_q, 0, i0, h);
            tma_load_3d(sm.q + kHalfBytes, &tmQ, &sm.bar_q, 64, i0, h);
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kStagesH;
                if (!mbar_wait(&sm.bar_kempty[s], ((t / kStagesH) & 1) ^ 1, abort)) break;
                mbar_expect_tx(&sm.bar_kfull[s], kTileBytes);
                tma_load_3d(sm.k[s], &tmK, &sm.bar_kfull[s], 0, t * kBN, h / group);
                tma_load_3d(sm.k[s] + kHalfBytes, &tmK, &sm.bar_kfull[s], 64, t * kBN, h / group);
                issued = t + 1;
            }
            // do not leave with copies in flight: the last load of every stage has landed
            for (int t = max(0, issued - kStagesH); t < issued; ++t)
                mbar_wait(&sm.bar_kfull[t % kStagesH], (t / kStagesH) & 1, abort);
            mbar_wait(&sm.bar_q, 0, abort);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA
        if (lane == 0) {
            int committed = 0;
            if (mbar_wait(&sm.bar_q, 0, abort)) {
                const uint32_t qa = smem_u32(sm.q);
                for (int t = 0; t < ntiles; ++t) {
                    const int s = t % kStagesH, b = t & 1;
                    if (!mbar_wait(&sm.bar_kfull[s], (t / kStagesH) & 1, abort)) break;
                    if (!mbar_wait(&sm.bar_aempty[b], ((t >> 1) & 1) ^ 1, abort)) break;
                    tc_fence_after();
                    const uint32_t ka = smem_u32(sm.k[s]);
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t off = c * kHalfBytes + k * 32;
                            umma_bf16(tmem + b * kBN, umma_desc(qa + off), umma_desc(ka + off), (c | k) != 0);
                        }
                    umma_commit(&sm.bar_kempty[s]);
                    umma_commit(&sm.bar_afull[b]);
                    committed = t + 1;
                }
            }
            // the tensor core has finished every issued tile before TMEM is freed
            if (committed > 0) {
                const int t = committed - 1;
                mbar_wait(&sm.bar_afull[t & 1], (t >> 1) & 1, abort);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        // kParts warps per TMEM lane quarter: thread = one row, part = the
        // 32-column chunk of every tile it takes
        const int quarter = warp & 3;                 // TMEM lanes this warp may read
        const int part = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const int i = i0 + r;
        const bool row_ok = i < n;
        float m2 = -INFINITY, l = 0.f;                // running max of z*log2e and sum of 2^(.)
        float vals[KM];
        int idx[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k) { vals[k] = -INFINITY; idx[k] = -1; }
        // a gated chunk's values, column k of epilogue thread e at stage[k * kEpiThreads + e]; the
        // merge scratch is free until the loop ends
        float* stage = sm.u.stage + (threadIdx.x - 64);
        volatile float* thr_row = &sm.thr[r][0];   // the parts of row r (read while others write)
        thr_row[part] = -INFINITY;
        epi_sync();
        auto chunk = [&](const uint32_t (&rv)[32], int j0, bool diag) {
            // causal mask: only the diagonal tile reaches past i
            float v[32];
            // four independent chains for the max and the sum (latency, not issue, bounds a single chain)
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (diag) {
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    v[k] = (j0 + k > i) ? -INFINITY : __uint_as_float(rv[k]);
                    mq[k & 3] = fmaxf(mq[k & 3], v[k]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    v[k] = __uint_as_float(rv[k]);
                    mq[k & 3] = fmaxf(mq[k & 3], v[k]);
                }
            }
            const float mc = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            if (!row_ok || mc == -INFINITY) return;   // no column of this chunk is at or before i
            const float mcs = mc * kLog2eOverSqrtD;
            if (mcs > m2) {
                l *= ex2(m2 - mcs);
                m2 = mcs;
            }
            float pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 32; ++k) pq[k & 3] += ex2(fmaf(v[k], kLog2eOverSqrtD, -m2));
            l += (pq[0] + pq[1]) + (pq[2] + pq[3]);
            if constexpr (!STATS) {
                // top-KM candidates j in [S, i-1], ranked by the raw score:
                // above this part's KM-th (a later column loses a tie) and not
                // below another part's KM-th (KM scores of the row rank at
                // least that high already; a tie there may still win on j)
                const float own = vals[KM - 1];
                const float gate = fmaxf(fmaxf(thr_row[0], thr_row[1]), fmaxf(thr_row[2], thr_row[3]));
                const float thr = gate > own ? below(gate) : own;
                if (mc > thr) {   // some column may enter the list
                    unsigned cm = 0u;
                    if (diag || j0 < S) {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            cm |= (v[k] > thr && j0 + k >= S && j0 + k < i) ? (1u << k) : 0u;
                    } else {   // every column is in [S, i-1]
#pragma unroll
                        for (int k = 0; k < 32; ++k) cm |= (v[k] > thr) ? (1u << k) : 0u;
                    }
                    if (__popc(cm) > 1) {
#pragma unroll
                        for (int k = 0; k < 32; ++k) stage[k * kEpiThreads] = v[k];
                        insert_staged<KM>(cm, stage, kEpiThreads, j0, vals, idx);
                    } else if (cm) {
                        if (diag || j0 < S)   // the max may be a masked column (a sink, i itself)
                            insert_candidates<KM>(cm, v, j0, vals, idx);
                        else                  // every column is a candidate: the one is the max
                            insert_one<KM>(mc, j0 + __ffs(cm) - 1, vals, idx);
                    }
                    thr_row[part] = vals[KM - 1];
                }
            }
        };
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            if (!mbar_wait(&sm.bar_afull[b], (t >> 1) & 1, abort)) break;
            tc_fence_after();
            uint32_t ra[32];
            __syncwarp();   // tcgen05.ld is warp-collective
            tmem_ld32_async(lane_addr + b * kBN + part * 32, ra);
            tmem_wait_tie(ra, true);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.bar_aempty[b]);   // the accumulator is read: the MMA may refill it
            const bool diag = t == ntiles - 1;      // the tile holding the block's diagonal
            chunk(ra, t * kBN + part * 32, diag);
        }
        // parts 1 .. kParts-1 hand their row state to part 0 in turn
        for (int src = 1; src < kParts; ++src) {
            epi_sync();   // the staging area (first round) or the previous hand-off is free
            if (part == src) {
                sm.xm[r][0] = m2;
                sm.xm[r][1] = l;
                if constexpr (!STATS) {
#pragma unroll
                    for (int k = 0; k < KM; ++k) { sm.u.x.v[r][k] = vals[k]; sm.u.x.i[r][k] = idx[k]; }
                }
            }
            epi_sync();
            if (part != 0) continue;
            const float mo = sm.xm[r][0], lo = sm.xm[r][1];
            const float mn = fmaxf(m2, mo);
            if (mn != -INFINITY) {
                l = (m2 == -INFINITY ? 0.f : l * ex2(m2 - mn)) + (mo == -INFINITY ? 0.f : lo * ex2(mo - mn));
                m2 = mn;
            }
            if constexpr (!STATS) {
                // insert the other part's list, ranked by (score desc, j asc)
                auto before = [](float a, int ja, float b, int jb) { return a > b || (a == b && ja < jb); };
#pragma unroll 1
                for (int k = 0; k < KM; ++k) {
                    const float a = sm.u.x.v[r][k];
                    const int j = sm.u.x.i[r][k];
                    if (j < 0 || !before(a, j, vals[KM - 1], idx[KM - 1])) break;   // the rest rank lower
#pragma unroll
                    for (int p = KM - 1; p > 0; --p) {
                        const float up = vals[p - 1];
                        const int upi = idx[p - 1];
                        const bool shift = before(a, j, up, upi);
                        const bool land = !shift && before(a, j, vals[p], idx[p]);
                        vals[p] = shift ? up : (land ? a : vals[p]);
                        idx[p] = shift ? upi : (land ? j : idx[p]);
                    }
                    if (before(a, j, vals[0], idx[0])) { vals[0] = a; idx[0] = j; }
                }
            }
        }
        if (part == 0) {
            if (STATS && row_ok && !*abort) {
                stats[((int64_t)h * n + i) * 2] = m2;
                stats[((int64_t)h * n + i) * 2 + 1] = l;
            } else if (row_ok && !*abort) {
                const int64_t base = (int64_t)h * E + row_offset(i, S, kappa);
                const int deg = (int)min((int64_t)kappa, max((int64_t)0, (int64_t)i - S));
                const float inv_l = 1.f / l;
#pragma unroll
                for (int k = 0; k < KM; ++k) {
                    if (k < deg) {
                        col[base + k] = idx[k];
                        w[base + k] = ex2(fmaf(vals[k], kLog2eOverSqrtD, -m2)) * inv_l;
                    }
                }
                row_ptr[(int64_t)h * (n + 1) + i] = row_offset(i, S, kappa);
                if (i == n - 1) row_ptr[(int64_t)h * (n + 1) + n] = E;
            }
        }
    }
    __syncthreads();
    if (*abort && threadIdx.x == 0) {
        // the grouped pass reads the failure word after the statistics
        if (STATS) atomicExch(reinterpret_cast<int*>(stats + (int64_t)H * n * 2), 1);
        else row_ptr[(int64_t)h * (n + 1)] = -1;
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
    }
}

// ---- query-group aggregated graph, second pass --------------------------
// One CTA per (KV head u, 128-row query block), heaviest blocks first.  The
// group's NH query blocks stay in shared memory; every K tile (BN rows)
// feeds NH MMAs, one TMEM accumulator per head, double buffered
// (2 x NH x BN <= 512 columns).  Epilogue thread = one row: it adds the
// heads' probabilities 2^(z log2(e) - c_h), c_h = max_h + log2(sum_h) from
// the first pass, and keeps the row's top-KM by that sum.
template <int NH>
struct __align__(1024) GroupSmem {
    static constexpr int BN = (NH >= 4) ? 64 : 128;            // K rows per tile
    static constexpr int KT = BN * 256;                         // one K tile (two 64-column halves)
    unsigned char q[NH][kTileBytes];
    unsigned char k[kStages][KT];
    unsigned long long bar_q;
    unsigned long long bar_kfull[kStages];
    unsigned long long bar_kempty[kStages];
    unsigned long long bar_afull[2];
    unsigned long long bar_aempty[2];
    uint32_t tmem_base;
    int abort;
};

template <int KM, int NH>
__global__ void __launch_bounds__(kThreads, 1)
k_prefill_group(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int Hkv, int n,
                int S, int kappa, const float* __restrict__ stats, int64_t* __restrict__ row_ptr,
                int32_t* __restrict__ col, float* __restrict__ w)
{
    using GS = GroupSmem<NH>;
    constexpr int BN = GS::BN, KT = GS::KT, KH = BN * 128;
    constexpr uint32_t TCOLS = (2 * NH * BN <= 256) ? 256u : 512u;
    constexpr uint32_t IDESC = idesc_n(BN);
    static_assert(2 * NH * BN <= 512, "accumulators must fit the tensor memory");
    extern __shared__ unsigned char smem_raw[];
    GS& sm = *reinterpret_cast<GS*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nqb = (n + kBM - 1) / kBM;
    const int qb = nqb - 1 - (int)(blockIdx.x / Hkv);
    const int u = (int)(blockIdx.x % Hkv);
    const int i0 = qb * kBM;
    const int ntiles = min(i0 + kBM - 1, n - 1) / BN + 1;       // tiles holding a column <= the block's last row
    const int64_t E = row_offset(n, S, kappa);
    const int Hq = Hkv * NH;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < kStages; ++s) { mbar_init(&sm.bar_kfull[s], 1); mbar_init(&sm.bar_kempty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&sm.bar_afull[b], 1); mbar_init(&sm.bar_aempty[b], 4); }
        // a first pass that gave up leaves its failure word set
        sm.abort = *reinterpret_cast<const volatile int*>(stats + (int64_t)Hq * n * 2) != 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&sm.tmem_base)), "r"(TCOLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort = &sm.abort;
    const bool failed = *abort != 0;

    if (failed) {
        // nothing to do: the cleanup below reports the failure
    } else if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(&sm.bar_q, NH * kTileBytes);
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                tma_load_3d(sm.q[h], &tmQ, &sm.bar_q, 0, i0, u * NH + h);
                tma_load_3d(sm.q[h] + kHalfBytes, &tmQ, &sm.bar_q, 64, i0, u * NH + h);
            }
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kStages;
                if (!mbar_wait(&sm.bar_kempty[s], ((t / kStages) & 1) ^ 1, abort)) break;
                mbar_expect_tx(&sm.bar_kfull[s], KT);
                tma_load_3d(sm.k[s], &tmK, &sm.bar_kfull[s], 0, t * BN, u);
                tma_load_3d(sm.k[s] + KH, &tmK, &sm.bar_kfull[s], 64, t * BN, u);
                issued = t + 1;
            }
            for (int t = max(0, issued - kStages); t < issued; ++t)
                mbar_wait(&sm.bar_kfull[t % kStages], (t / kStages) & 1, abort);
            mbar_wait(&sm.bar_q, 0, abort);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA
        if (lane == 0) {
            int committed = 0;
            if (mbar_wait(&sm.bar_q, 0, abort)) {
                for (int t = 0; t < ntiles; ++t) {
                    const int s = t % kStages, b = t & 1;
                    if (!mbar_wait(&sm.bar_kfull[s], (t / kStages) & 1, abort)) break;
                    if (!mbar_wait(&sm.bar_aempty[b], ((t >> 1) & 1) ^ 1, abort)) break;
                    tc_fence_after();
                    const uint32_t ka = smem_u32(sm.k[s]);
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const uint32_t qa = smem_u32(sm.q[h]);
#pragma unroll
                        for (int c = 0; c < 2; ++c)
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                umma_bf16(tmem + (uint32_t)((b * NH + h) * BN), umma_desc(qa + c * kHalfBytes + k * 32),
                                          umma_desc(ka + c * KH + k * 32), (c | k) != 0, IDESC);
                    }
                    umma_commit(&sm.bar_kempty[s]);
                    umma_commit(&sm.bar_afull[b]);
                    committed = t + 1;
                }
            }
            if (committed > 0) {
                const int t = committed - 1;
                mbar_wait(&sm.bar_afull[t & 1], (t >> 1) & 1, abort);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int i = i0 + r;
        const bool row_ok = i < n;
        float ch[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            ch[h] = 0.f;
            if (row_ok) {
                const float2 ml = *reinterpret_cast<const float2*>(stats + ((int64_t)(u * NH + h) * n + i) * 2);
                ch[h] = ml.x + __log2f(ml.y);
            }
        }
        float vals[KM];
        int idx[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k) { vals[k] = -INFINITY; idx[k] = -1; }
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            if (!mbar_wait(&sm.bar_afull[b], (t >> 1) & 1, abort)) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                float ws[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) ws[k] = 0.f;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    float v[32];
                    __syncwarp();   // tcgen05.ld is warp-collective
                    tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((b * NH + h) * BN + cc * 32), v);
#pragma unroll
                    for (int k = 0; k < 32; ++k) ws[k] += ex2(fmaf(v[k], kLog2eOverSqrtD, -ch[h]));
                }
                if (!row_ok) continue;
                const int j0 = t * BN + cc * 32;
                // top-KM candidates j in [S, i-1] by the summed probability
                const float thr = vals[KM - 1];
                float mq[4] = {ws[0], ws[1], ws[2], ws[3]};
#pragma unroll
                for (int k = 4; k < 32; ++k) mq[k & 3] = fmaxf(mq[k & 3], ws[k]);
                const float mc = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
                if (mc > thr) {   // some column may enter the list
                    unsigned cm = 0u;
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        cm |= (ws[k] > thr && j0 + k >= S && j0 + k < i) ? (1u << k) : 0u;
                    insert_candidates<KM>(cm, ws, j0, vals, idx);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.bar_aempty[b]);
        }
        if (row_ok && !*abort) {
            const int64_t base = (int64_t)u * E + row_offset(i, S, kappa);
            const int deg = (int)min((int64_t)kappa, max((int64_t)0, (int64_t)i - S));
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                if (k < deg) {
                    col[base + k] = idx[k];
                    w[base + k] = vals[k];
                }
            }
            row_ptr[(int64_t)u * (n + 1) + i] = row_offset(i, S, kappa);
            if (i == n - 1) row_ptr[(int64_t)u * (n + 1) + n] = E;
        }
    }
    __syncthreads();
    if (*abort && threadIdx.x == 0) row_ptr[(int64_t)u * (n + 1)] = -1;
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS) : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [H][n][128] bf16 viewed as a 3-D tensor, box = 64 columns x box_rows rows x 1 head
bool make_map(CUtensorMap* m, const void* base, int H, int n, int box_rows = 128)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)n, (cuuint64_t)H};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)n * 128 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KM, bool STATS>
cudaError_t launch_km(const CUtensorMap& mq, const CUtensorMap& mk, int H, int n, int S, int kappa, int group,
                      int64_t* row_ptr, int32_t* col, float* w, float* stats, cudaStream_t st)
{
    const size_t smem = sizeof(PrefillSmem) + 1024;
    auto kern = k_prefill_topk<KM, STATS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nqb = (n + kBM - 1) / kBM;
    kern<<<H * nqb, kThreadsH, smem, st>>>(mq, mk, H, n, S, kappa, group, row_ptr, col, w, stats);
    return cudaGetLastError();
}

template <int KM, int NH>
cudaError_t launch_group(const CUtensorMap& mq, const CUtensorMap& mk, int Hkv, int n, int S, int kappa,
                         const float* stats, int64_t* row_ptr, int32_t* col, float* w, cudaStream_t st)
{
    const size_t smem = sizeof(GroupSmem<NH>) + 1024;
    auto kern = k_prefill_group<KM, NH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nqb = (n + kBM - 1) / kBM;
    kern<<<Hkv * nqb, kThreads, smem, st>>>(mq, mk, Hkv, n, S, kappa, stats, row_ptr, col, w);
    return cudaGetLastError();
}

template <int KM>
cudaError_t launch_group_nh(int nh, const CUtensorMap& mq, const CUtensorMap& mk, int Hkv, int n, int S, int kappa,
                            const float* stats, int64_t* row_ptr, int32_t* col, float* w, cudaStream_t st)
{
    switch (nh) {
        case 1: return launch_group<KM, 1>(mq, mk, Hkv, n, S, kappa, stats, row_ptr, col, w, st);
        case 2: return launch_group<KM, 2>(mq, mk, Hkv, n, S, kappa, stats, row_ptr, col, w, st);
        case 4: return launch_group<KM, 4>(mq, mk, Hkv, n, S, kappa, stats, row_ptr, col, w, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_build_graph(int H, int n, int S, int kappa, const void* Q, const void* K, int64_t* row_ptr,
                               int32_t* col, float* w, cudaStream_t st)
{
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) & 15) return cudaErrorInvalidValue;
    CUtensorMap mq, mk;
    if (!make_map(&mq, Q, H, n) || !make_map(&mk, K, H, n)) return cudaErrorInvalidValue;
    if (kappa <= 8) return launch_km<8, false>(mq, mk, H, n, S, kappa, 1, row_ptr, col, w, nullptr, st);
    if (kappa <= 16) return launch_km<16, false>(mq, mk, H, n, S, kappa, 1, row_ptr, col, w, nullptr, st);
    return launch_km<32, false>(mq, mk, H, n, S, kappa, 1, row_ptr, col, w, nullptr, st);
}

size_t build_graph_grouped_stats_floats(int Hkv, int group, int n)
{
    return (size_t)Hkv * group * n * 2 + 4;   // (max, sum) per query head and row, then the failure word
}

cudaError_t launch_build_graph_grouped(int Hkv, int group, int n, int S, int kappa, const void* Q, const void* K,
                                       float* stats, int64_t* row_ptr, int32_t* col, float* w, cudaStream_t st)
{
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) & 15) return cudaErrorInvalidValue;
    if (group != 1 && group != 2 && group != 4) return cudaErrorInvalidValue;
    const int Hq = Hkv * group;
    const int bn = (group >= 4) ? 64 : 128;
    CUtensorMap mq, mk, mkg;
    if (!make_map(&mq, Q, Hq, n) || !make_map(&mk, K, Hkv, n) || !make_map(&mkg, K, Hkv, n, bn))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(stats + (size_t)Hq * n * 2, 0, 4 * sizeof(float), st);
    if (e != cudaSuccess) return e;
    // first pass: every query head's row statistics
    e = launch_km<8, true>(mq, mk, Hq, n, S, kappa, group, row_ptr, col, w, stats, st);
    if (e != cudaSuccess) return e;
    // second pass: one graph per KV head, ranked by the summed probabilities
    if (kappa <= 8) return launch_group_nh<8>(group, mq, mkg, Hkv, n, S, kappa, stats, row_ptr, col, w, st);
    if (kappa <= 16) return launch_group_nh<16>(group, mq, mkg, Hkv, n, S, kappa, stats, row_ptr, col, w, st);
    return launch_group_nh<32>(group, mq, mkg, Hkv, n, S, kappa, stats, row_ptr, col, w, st);
}

}  // namespace ckv
