// k_decode.cu -- the per-step decode kernels of CommunityKV on sm_100a.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 1 caption, step (3): score the query against the community
// centroids, retrieve a candidate subset, run exact attention over it plus
// the sink tokens, take the top-kappa keys as the new token's edges and
// assign it to a community in constant time; Table 1: O(sqrt(n) d)
// retrieval, O(d) update.
//
// Four kernels per step:
//   k_score   centroid GEMV (HBM-bound): a persistent TMA ring of 16 KB
//             units (32 communities), lane = 4 dims, the 32 partial dots
//             reduced by a butterfly transpose.
//   k_select  one CTA per graph, each thread's communities in registers:
//             exact budgeted top-C by a size-weighted histogram linear in
//             the score (radix passes over (score bits, id) only when the
//             boundary bin is crowded) and an exact rank of the boundary
//             bin; writes the kept list and the kept rows.
//   k_attend  the graphs' rows split evenly over one CTA per SM; every warp
//             gathers its own run of K and V rows (16-byte cp.async) and,
//             for bf16, runs both contractions on the tensor cores
//             (mma.sync) with an online softmax; the last slice of a graph
//             to finish merges the (m, l, o) partials into the output and
//             each head's (m, l).
//   k_update  (ckv_assign_update, lowest priority) one CTA per graph ranks
//             the kept members' edge weights, assigns the new token by
//             weighted plurality and updates that community's running
//             mean.  With d.defer_update off, k_attend's last slice runs
//             the same code instead.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>
#include <utility>

#include "ckv_internal.cuh"
#include "dev_async.cuh"
#include "warp_mma.cuh"

namespace ckv {

namespace {

template <bool BF16>
__device__ __forceinline__ float elem(const void* p, int64_t i)
{
    if (BF16) return __uint_as_float((uint32_t)(((const uint16_t*)p)[i]) << 16);
    return ((const float*)p)[i];
}

__device__ __forceinline__ void graph_heads(const Dims& d, int g, int& b, int& h0, int& kvh)
{
    if (d.mode == CKV_QUERY_GROUP) {
        b = g / d.Hkv;
        kvh = g % d.Hkv;
        h0 = kvh * d.Gq;
    } else {
        b = g / d.Hq;
        h0 = g % d.Hq;
        kvh = h0 / d.Gq;
    }
}

// order-preserving map of a float to an unsigned (larger float -> larger)
__device__ __forceinline__ uint32_t ord_u(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- k_score
// Work unit = 32 consecutive communities of one graph (16 KB of centroids,
// one bulk copy).  Each CTA owns a contiguous run of units in graph-major
// order; its producer lane streams them through a ring, consumer warp c
// takes local units c, c + 8, ...: lane = 4 dims, 32 partial dots reduced
// by a butterfly transpose so lane r ends with row r's score.
constexpr int kScoreCW = 8;
constexpr int kScoreThreads = 32 * (1 + kScoreCW);
constexpr int kScoreNST = 8;
constexpr int kScoreStage = 32 * kD * 4;
// unit u goes through slot u % kScoreNST and is read by warp u % kScoreCW:
// every slot must belong to one consumer warp, so that its mbarrier phases
// complete in the order that warp waits for them (a parity wait on a phase
// two generations ahead would pass at once)
static_assert(kScoreNST % kScoreCW == 0, "each ring slot is read by a single consumer warp");

struct ScoreSmem {
    unsigned char ring[kScoreNST][kScoreStage];
    unsigned long long full[kScoreNST];
    unsigned long long empty[kScoreNST];
    int abort;
};

// whether the step already failed, read once for the whole CTA (every
// thread then takes the same branch; another CTA may set the word meanwhile)
__device__ __forceinline__ bool step_failed(const int* err)
{
    __shared__ int e;
    __syncthreads();
    if (threadIdx.x == 0) e = *(volatile const int*)err;
    __syncthreads();
    return e != 0;
}

template <bool BF16>
__global__ void __launch_bounds__(kScoreThreads, 1) k_score(DevState s, Dims d, const void* __restrict__ q)
{
    pdl_wait();
    if (d.pdl) pdl_trigger();
    if (step_failed(s.err)) return;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int upg = (d.n_comm + 31) / 32;                    // units per graph
    const int64_t NU = (int64_t)d.G * upg;
    const int64_t u0 = (int64_t)blockIdx.x * NU / gridDim.x, u1 = (int64_t)(blockIdx.x + 1) * NU / gridDim.x;
    const int nu = (int)(u1 - u0);
    if (tid == 0) {
        for (int i = 0; i < kScoreNST; ++i) { mbar_init(&sm.full[i], 1); mbar_init(&sm.empty[i], 1); }
        sm.abort = 0;
        mbar_fence_init();
    }
    __syncthreads();
    volatile int* abort_flag = &sm.abort;
    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();   // the centroids are streamed once per step
            int issued = 0;
            for (int u = 0; u < nu; ++u) {
                const int st = u % kScoreNST;
                if (!mbar_wait(&sm.empty[st], ((u / kScoreNST) & 1) ^ 1, abort_flag)) break;
                const int64_t gu = u0 + u;
                const int g = (int)(gu / upg), c0 = (int)(gu % upg) * 32;
                const int rows = min(32, d.n_comm - c0);
                mbar_expect_tx(&sm.full[st], rows * kD * 4);
                bulk_g2s_hint(sm.ring[st], s.mu + ((int64_t)g * d.Nc + c0) * kD, rows * kD * 4, &sm.full[st], pol);
                issued = u + 1;
            }
            // nothing may still be landing when the CTA exits
            for (int u = max(0, issued - kScoreNST); u < issued; ++u)
                mbar_wait(&sm.full[u % kScoreNST], (u / kScoreNST) & 1, abort_flag);
        }
        return;
    }
    const int c = warp - 1;
    int gq = -1;
    float qs[4] = {0.f, 0.f, 0.f, 0.f};
    // the graph's score range over its non-empty communities and their
    // total size, for the selection: each lane keeps its own while the warp
    // stays on one graph, then one reduction and three atomics per graph
    uint32_t rmin = 0xffffffffu, rmax = 0u;
    int rsum = 0;
    auto flush_range = [&](int gf) {
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            rmin = min(rmin, __shfl_xor_sync(kFull, rmin, o));
            rmax = max(rmax, __shfl_xor_sync(kFull, rmax, o));
            rsum += __shfl_xor_sync(kFull, rsum, o);
        }
        if (lane == 0 && gf >= 0 && rmax != 0u) {
            atomicMin(s.srange + 4 * gf, rmin);
            atomicMax(s.srange + 4 * gf + 1, rmax);
            atomicAdd(s.srange + 4 * gf + 2, (unsigned)rsum);
        }
        rmin = 0xffffffffu;
        rmax = 0u;
        rsum = 0;
    };
    for (int u = c; u < nu; u += kScoreCW) {
        const int64_t gu = u0 + u;
        const int g = (int)(gu / upg), c0 = (int)(gu % upg) * 32;
        if (g != gq) {   // sum of the graph's query heads, this lane's 4 dims
            flush_range(gq);
            int b, h0, kvh;
            graph_heads(d, g, b, h0, kvh);
#pragma unroll
            for (int k = 0; k < 4; ++k) qs[k] = 0.f;
            for (int h = 0; h < d.HG; ++h) {
                const int64_t base = ((int64_t)b * d.Hq + h0 + h) * kD + 4 * lane;
#pragma unroll
                for (int k = 0; k < 4; ++k) qs[k] += elem<BF16>(q, base + k);
            }
            gq = g;
        }
        const int st = u % kScoreNST;
        const int64_t gi = (int64_t)g * d.Nc + c0 + lane;
        const int sz = (c0 + lane < d.n_comm) ? s.csize[gi] : 0;
        if (!mbar_wait(&sm.full[st], (u / kScoreNST) & 1, abort_flag)) break;
        const int rows = min(32, d.n_comm - c0);
        const float4* mu = reinterpret_cast<const float4*>(sm.ring[st]);
        float part[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            const float4 v = (r < rows) ? mu[r * (kD / 4) + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
            part[r] = fmaf(qs[3], v.w, fmaf(qs[2], v.z, fmaf(qs[1], v.y, qs[0] * v.x)));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
        // butterfly transpose-reduce: afterwards lane L holds row c0 + L
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const bool up = (lane & off) != 0;
#pragma unroll
            for (int i = 0; i < off; ++i) {
                const float send = up ? part[i] : part[i + off];
                const float keep = up ? part[i + off] : part[i];
                part[i] = keep + __shfl_xor_sync(kFull, send, off);
            }
        }
        if (lane < rows) s.score[gi] = (sz > 0) ? part[0] : -INFINITY;
        if (lane < rows && sz > 0) {   // this lane's running range and size (order-preserving keys; +0 for -0)
            const uint32_t k = ord_u(part[0] + 0.0f);
            rmin = min(rmin, k);
            rmax = max(rmax, k);
            rsum += sz;
        }
    }
    flush_range(gq);
    if (*abort_flag && c == 0 && lane == 0) set_error(s.err, CKV_ERR_TIMEOUT);
}

// --------------------------------------------------------------- k_select
// One CTA of 1024 threads per graph.  Thread t owns communities t, t + 1024,
// ... (E of them, scores and sizes in registers, their status in register
// bit masks).  Exact budgeted top-C in (score desc, id asc) order:
//   1. one round of loads; the score range and the total size come from
//      k_score (order-preserving keys reduced by atomics per graph);
//   2. a size-weighted histogram over kSelBins bins, linear in the score
//      (bins are monotone in the score, so every community of a higher bin
//      ranks before every one of a lower bin); the boundary bin is where the
//      size summed from the top first exceeds the budget;
//   3. while the boundary bin holds more than kSelCand communities, radix
//      passes over the composite key (score bits, inverted id) of those
//      communities narrow it by 11 bits a pass;
//   4. the boundary bin's communities are ranked exactly: each counts the
//      size of the better ones, and is kept iff the sizes through it fit;
//   5. the kept ids in ascending order with the prefix of their sizes, by
//      ballots per 32 ids and one scan over the (round, warp) counts;
//   6. warps copy the kept communities' member segments into the row list,
//      eight communities' loads in flight per warp.
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelCand = 1024;     // boundary-bin communities ranked exactly

// asks L2 to fetch n ints from p on (one prefetch per 128-byte line)
__device__ __forceinline__ void prefetch_l2_range(const int32_t* pool, int off, int n, int64_t P)
{
#ifdef CKV_DEBUG_BOUNDS
    if (off < 0 || (int64_t)off + n > P) return;   // a bad segment: the row copy reports it
#endif
    const int32_t* p = pool + off;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p) & ~(uintptr_t)127;
    const uintptr_t a1 = reinterpret_cast<uintptr_t>(p + n);
    for (uintptr_t a = a0; a < a1; a += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
}

// key of a community: (order-preserving score bits, inverted id): larger = kept first
__device__ __forceinline__ unsigned long long sel_key(float sc, int c)
{
    // -0 and +0 are the same score (adding +0 turns -0 into +0)
    return ((unsigned long long)ord_u(sc + 0.0f) << 32) | (unsigned long long)(~(uint32_t)c);
}

// inclusive prefix sum over the warp
__device__ __forceinline__ int warp_incl(int x, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

template <int E>
__global__ void __launch_bounds__(kSelThreads, 1) k_select(DevState s, Dims d)
{
    pdl_wait();
    if (d.pdl == 1) pdl_trigger();
    if (step_failed(s.err)) return;
    extern __shared__ __align__(16) unsigned char smem_sel[];
    __shared__ int r_w[kSelWarps];
    __shared__ unsigned long long r_kmin[kSelWarps], r_kmax[kSelWarps];
    __shared__ int off_c[E][kSelWarps], off_w[E][kSelWarps];
    __shared__ int sh_b, sh_above, sh_n, sh_C, sh_T, sh_bn, sh_bt;
    const int g = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Nc = d.n_comm, budget = d.budget;

    // ---- 1. scores and sizes (one round of loads), range and total size
    const float* gsc = s.score + (int64_t)g * d.Nc;
    const int32_t* gsz = s.csize + (int64_t)g * d.Nc;
    const int32_t* gco = s.coff + (int64_t)g * d.Nc;
    const int32_t* gpool = s.pool + (int64_t)g * d.P;
    float v[E];
    int w[E], co[E];   // score, size, segment start
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int c = i * kSelThreads + tid;
        w[i] = (c < Nc) ? gsz[c] : 0;
        v[i] = (c < Nc) ? gsc[c] : 0.f;
        co[i] = (c < Nc) ? gco[c] : 0;
    }
    // the score range and the total size, left by k_score
    const uint4 rg = __ldcg(reinterpret_cast<const uint4*>(s.srange + 4 * g));
    // status of the thread's communities as bit masks: still a candidate
    // (cmask), surely kept (imask)
    unsigned cmask = 0u, imask = 0u;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        if (w[i] > 0) cmask |= 1u << i;
        else w[i] = 0;
    }
    auto from_ord = [](uint32_t u) { return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u); };
    const bool any = rg.y != 0u;
    const float lo = any ? from_ord(rg.x) : INFINITY, hi = any ? from_ord(rg.y) : -INFINITY;
    const int wsum = (int)rg.z;
    if (tid == 0) { sh_n = 0; sh_above = 0; sh_bn = 0; sh_bt = 0; }
    __syncthreads();
    if (tid == 0) *reinterpret_cast<uint4*>(s.srange + 4 * g) = make_uint4(0xffffffffu, 0u, 0u, 0u);   // for the next step

    // shared memory: the passes' histogram and boundary candidates, later
    // (same bytes) the kept list
    unsigned char* ub = smem_sel;
    unsigned long long* ckey = reinterpret_cast<unsigned long long*>(ub);    // [kSelCand]
    int* hist = reinterpret_cast<int*>(ckey + kSelCand);                      // [kSelBins]
    int* cwt = hist + kSelBins;                                               // [kSelCand]
    int* ccof = cwt + kSelCand;                                               // [kSelCand]
    for (int i = tid; i < kSelBins; i += kSelThreads) hist[i] = 0;

    if (wsum <= budget) {   // every community fits: keep them all
        imask = cmask;
        cmask = 0u;
#pragma unroll
        for (int i = 0; i < E; ++i)
            if (imask & (1u << i)) prefetch_l2_range(gpool, co[i], w[i], d.P);
    } else {
        // ---- 2./3. bucket passes until the boundary bin is small
        const float scale = (hi > lo) ? (float)kSelBins / (hi - lo) : 0.f;
        int above = 0;      // size of the communities known to be kept
        int shift = -1;     // -1: linear in the score; else radix window of the key
        int m = 0;
        __syncthreads();    // hist zeroed
        for (int pass = 0;; ++pass) {
            if (pass == 8) {   // 64 key bits take at most 6 radix passes: unreachable
                if (tid == 0) set_error(s.err, CKV_ERR_STATE);
                return;
            }
            auto bin_of = [&](int i, int c) -> int {
                if (shift < 0) return min(kSelBins - 1, (int)((v[i] - lo) * scale));
                return (int)((sel_key(v[i], c) >> shift) & (unsigned long long)(kSelBins - 1));
            };
#pragma unroll
            for (int i = 0; i < E; ++i)
                if (cmask & (1u << i)) atomicAdd(&hist[bin_of(i, i * kSelThreads + tid)], w[i]);
            __syncthreads();
            // boundary bin: the size summed from the top bin down first exceeds the budget
            const int b0 = kSelBins - 1 - 2 * tid, b1 = b0 - 1;
            const int h0 = hist[b0], h1 = hist[b1];
            const int x = h0 + h1;
            const int incl = warp_incl(x, lane);
            if (lane == 31) r_w[warp] = incl;
            __syncthreads();
            const int rw = r_w[lane];   // kSelWarps == 32
            const int wpre = __shfl_sync(kFull, warp_incl(rw, lane) - rw, warp);
            const int bef = above + wpre + incl - x;
            if (bef <= budget && bef + h0 > budget) { sh_b = b0; sh_above = bef; }
            else if (bef + h0 <= budget && bef + h0 + h1 > budget) { sh_b = b1; sh_above = bef + h0; }
            __syncthreads();
            const int bs = sh_b;
            above = sh_above;
            hist[b0] = 0;
            hist[b1] = 0;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                if (!(cmask & (1u << i))) continue;
                const int c = i * kSelThreads + tid;
                const int b = bin_of(i, c);
                if (b > bs) {
                    imask |= 1u << i;
                    cmask &= ~(1u << i);
                    prefetch_l2_range(gpool, co[i], w[i], d.P);   // its members, for the row copy
                } else if (b < bs) {
                    cmask &= ~(1u << i);
                } else {
                    const int slot = atomicAdd(&sh_n, 1);
                    if (slot < kSelCand) { ckey[slot] = sel_key(v[i], c); cwt[slot] = w[i]; ccof[slot] = co[i]; }
                    if (shift < 0) prefetch_l2_range(gpool, co[i], w[i], d.P);   // likely kept too
                }
            }
            __syncthreads();
            m = sh_n;
            if (m <= kSelCand) break;                      // uniform
            // crowded boundary bin: the key range of its communities
            unsigned long long kmn = ~0ull, kmx = 0ull;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                if (!(cmask & (1u << i))) continue;
                const unsigned long long k = sel_key(v[i], i * kSelThreads + tid);
                kmn = min(kmn, k);
                kmx = max(kmx, k);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                kmn = min(kmn, __shfl_xor_sync(kFull, kmn, o));
                kmx = max(kmx, __shfl_xor_sync(kFull, kmx, o));
            }
            if (lane == 0) { r_kmin[warp] = kmn; r_kmax[warp] = kmx; }
            __syncthreads();
            kmn = r_kmin[lane];
            kmx = r_kmax[lane];
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                kmn = min(kmn, __shfl_xor_sync(kFull, kmn, o));
                kmx = max(kmx, __shfl_xor_sync(kFull, kmx, o));
            }
            // the candidates share every key bit above the highest differing one
            shift = max(0, 63 - __clzll((long long)(kmn ^ kmx)) - 10);
            __syncthreads();                               // sh_n read by all
            if (tid == 0) sh_n = 0;
        }
    }
    // ---- 4./5. in one phase: the boundary bin's communities ranked exactly
    // (each counts the better ones and their sizes; kept iff the sizes
    // through it fit), and the surely kept ids placed in ascending order by
    // ballots per 32 ids plus one scan over the (round, warp) totals.  The
    // kept boundary communities follow the surely kept ones, in rank order.
    const int m = (wsum <= budget) ? 0 : min(sh_n, kSelCand);
    unsigned long long bkey = 0ull;
    int brank = 0, bpre = 0, bw = 0, bco = 0;
    bool bkeep = false;
    if (tid < m) {
        bkey = ckey[tid];
        bw = cwt[tid];
        bco = ccof[tid];
        for (int t = 0; t < m; ++t) {
            const bool better = ckey[t] > bkey;
            brank += better ? 1 : 0;
            bpre += better ? cwt[t] : 0;
        }
        bkeep = (sh_above + bpre + bw <= budget) || (sh_above == 0 && bpre == 0);
        if (bkeep) { atomicAdd(&sh_bn, 1); atomicAdd(&sh_bt, bw); }
    }
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const bool kept = (imask >> i) & 1u;
        const unsigned bal = __ballot_sync(kFull, kept);
        const int wt = bal ? (int)__reduce_add_sync(kFull, kept ? (unsigned)w[i] : 0u) : 0;
        if (lane == 0) { off_c[i][warp] = __popc(bal); off_w[i][warp] = wt; }
    }
    __syncthreads();
    if (warp == 0) {   // exclusive offsets in (round, warp) order; lane owns E consecutive entries
        int sc = 0, sw = 0;
        for (int j = 0; j < E; ++j) {
            const int e = lane * E + j;
            sc += off_c[e / kSelWarps][e % kSelWarps];
            sw += off_w[e / kSelWarps][e % kSelWarps];
        }
        const int ic = warp_incl(sc, lane), iw = warp_incl(sw, lane);
        int pc = ic - sc, pw = iw - sw;
        for (int j = 0; j < E; ++j) {
            const int e = lane * E + j;
            const int a = off_c[e / kSelWarps][e % kSelWarps], b = off_w[e / kSelWarps][e % kSelWarps];
            off_c[e / kSelWarps][e % kSelWarps] = pc;
            off_w[e / kSelWarps][e % kSelWarps] = pw;
            pc += a;
            pw += b;
        }
        if (lane == 31) { sh_C = ic; sh_T = iw; }
    }
    __syncthreads();
    const int C0 = sh_C, T0 = sh_T;                // surely kept
    const int C = C0 + sh_bn, T = T0 + sh_bt;
    // the kept list (overlays the passes' arrays): row start, id, segment start
    int* pre = reinterpret_cast<int*>(ub);       // [C + 1]
    int* cid = pre + C + 1;                      // [C]
    int* cof = cid + C;                          // [C]
    int32_t* gsel = s.sel + (int64_t)g * d.Nc;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int c = i * kSelThreads + tid;
        const bool kept = (imask >> i) & 1u;
        const unsigned bal = __ballot_sync(kFull, kept);
        if (bal == 0u) continue;                                   // warp-uniform
        const int wk = kept ? w[i] : 0;
        const int wx = (bal & (bal - 1u)) ? warp_incl(wk, lane) - wk : 0;   // exclusive prefix
        if (kept) {
            const int pos = off_c[i][warp] + __popc(bal & ((1u << lane) - 1u));
            pre[pos] = off_w[i][warp] + wx;
            cid[pos] = c;
            cof[pos] = co[i];
            gsel[pos] = c;
        }
    }
    if (bkeep) {
        const int pos = C0 + brank, c = (int)~(uint32_t)(bkey & 0xffffffffull);
        pre[pos] = T0 + bpre;
        cid[pos] = c;
        cof[pos] = bco;
        gsel[pos] = c;
    }
    if (tid == 0) {
        pre[C] = T;
        int32_t* meta = s.meta + (int64_t)g * M_COUNT;
        meta[M_C] = C;
        meta[M_T] = T;
        meta[M_ROWS] = d.S + T + 1;
    }
    if (d.pdl == 2) pdl_trigger();
    __syncthreads();
    // ---- 6. the kept members' rows: warp k copies kept communities k,
    // k + 32, ... (contiguous segments, eight communities' loads in flight)
    const int32_t* pool = s.pool + (int64_t)g * d.P;
    int32_t* rtok = s.rtok + (int64_t)g * d.NM;
    int32_t* rcomm = s.rcomm + (int64_t)g * d.NM;
    for (int k0 = warp; k0 < C; k0 += 8 * kSelWarps) {
        int tk[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int k = k0 + u * kSelWarps;
            const int sz = k < C ? pre[k + 1] - pre[k] : 0;
            // the segment inside the pool (debug build; a bad one reads token 0)
            const bool in = k < C && CKV_IN_RANGE(cof[k], 0, (int64_t)d.P - sz + 1, s.err);
            tk[u] = (in && lane < sz) ? pool[cof[k] + lane] : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int k = k0 + u * kSelWarps;
            if (k >= C) break;
            const int r0 = pre[k], sz = pre[k + 1] - r0, cc = cid[k];
            const bool in = CKV_IN_RANGE(cof[k], 0, (int64_t)d.P - sz + 1, s.err);
            if (lane < sz) { rtok[r0 + lane] = tk[u]; rcomm[r0 + lane] = cc; }
            for (int j = 32 + lane; j < sz; j += 32) {   // communities longer than a warp
                rtok[r0 + j] = in ? pool[cof[k] + j] : 0;
                rcomm[r0 + j] = cc;
            }
        }
    }
}

// --------------------------------------------------------------- k_attend
// One CTA per SM, each a slice of one graph's rows (or whole graphs when
// there are more graphs than CTAs).  Every warp owns a contiguous run of the
// slice's rows and streams it through its own 3-batch shared-memory
// pipeline, K and V rows of a batch gathered together with 16-byte cp.async
// (the LSU gather path; one bulk copy per 256-byte row is far slower).
//
// bf16 caches: a batch is 16 rows and both contractions run on the tensor
// cores (mma.sync m16n8k16, fp32 accumulate): S^T = K_tile . Q^T with the
// graph's heads as the 8 columns, then O^T += V_tile^T . P^T with P split
// into a bf16 high and low part (two MMAs) so the weights keep ~16 bits.
// Rows sit in shared memory with their 16-byte chunks XOR-swizzled by
// (row mod 8), which makes every ldmatrix conflict-free.  fp32 caches:
// 4-row batches on the CUDA cores (partial dots reduced by a butterfly).
//
// Each warp keeps an online softmax (running max and sum per head) and
// spills the kept members' logits to L2.  The CTA combines its warps into
// one (m, l, o) partial per head, publishes it and counts itself in on the
// graph's arrival counter; no CTA waits.  The slice that arrives last
// finishes the graph (finish_graph):
// - it merges the partials into the output and the softmax statistics;
// - it ranks the kept members' edge weights w_j into the top-kappa edges;
// - it votes on the new token's community and updates that community.
constexpr int kAttNBuf = 3;        // batches per warp pipeline

template <bool BF16, int HG>
struct AttLayout {
    static constexpr int NB = BF16 ? 16 : 4;                     // rows per warp batch
    static constexpr int RB = kD * (BF16 ? 2 : 4);               // bytes per K or V row
    static constexpr int BATCH = NB * 2 * RB;                    // K rows, then V rows
    static constexpr int WBUF = kAttNBuf * BATCH;                // one warp's pipeline
    static constexpr int TOKW = 128;                             // row tokens a warp keeps at once
    static constexpr int off_buf = 0;
    static constexpr int off_pz = off_buf + kAttWarps * WBUF;    // fp32: [warps][NB*HG] z / p exchange
    static constexpr int off_tokw = off_pz + (BF16 ? 0 : kAttWarps * NB * HG * 4);   // [warps][TOKW]
    static constexpr int off_misc = off_tokw + kAttWarps * TOKW * 4;
    static constexpr int bytes = off_misc + 1280;
    // end-of-slice reduction [warps][HG][RSTR] reuses the pipelines; a row is
    // acc[0..D), m, l, padded to a multiple of 16 bytes for float4 access
    static constexpr int RSTR = kD + 4;
    static_assert(kAttWarps * HG * RSTR * 4 <= kAttWarps * WBUF, "reduction must fit");
    static_assert(kAttWarps * 6 * (kMaxKappa + 128) * 4 <= kAttWarps * WBUF, "edge lists must fit");
};

// HG logits of one kept-member row (16-, 8- or 4-byte aligned by HG)
template <int HG>
__device__ __forceinline__ void load_logits(const float* p, float (&z)[HG])
{
    if constexpr (HG % 4 == 0) {
#pragma unroll
        for (int h = 0; h < HG; h += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(p + h));
            z[h] = v.x; z[h + 1] = v.y; z[h + 2] = v.z; z[h + 3] = v.w;
        }
    } else if constexpr (HG == 2) {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(p));
        z[0] = v.x; z[1] = v.y;
    } else {
        z[0] = __ldcg(p);
    }
}

// Edge ranking of one graph by a whole CTA.  The kept members go by in
// rounds of FR rows per thread (one round of loads each); the running top
// kappa (w desc, token asc) sits in shared memory and joins every round as
// extra entries of threads 0 .. kappa-1.  Per round: tau = the kappa-th
// best of the threads' best entries is a lower bound of the answer, and
// only the kappa threads whose best reaches tau can hold entries at least
// that good, so at most kappa * (FR + 1) entries are compacted and ranked
// by counting.
constexpr int kFinMaxRows = 16;                                  // rows per thread and round
constexpr int kFinCand = kAttWarps * kMaxKappa * (kFinMaxRows + 1);   // compacted entries, at most

// 64-bit order-preserving key of an edge candidate: larger = ranked first
// (w desc, token asc; w >= 0); 0 marks an empty slot
__device__ __forceinline__ unsigned long long edge_key(float w, int t)
{
    return ((unsigned long long)__float_as_uint(w) << 32) | (unsigned long long)(~(uint32_t)t);
}
__device__ __forceinline__ float key_w(unsigned long long k) { return __uint_as_float((uint32_t)(k >> 32)); }
__device__ __forceinline__ int key_t(unsigned long long k) { return (int)~(uint32_t)(k & 0xffffffffull); }

struct EdgeScratch {
    unsigned long long lk[kMaxKappa];            // running list (rank order)
    int lx[kMaxKappa];                           // kept-member row of each entry
    int lc[kMaxKappa], lsz[kMaxKappa], lcap[kMaxKappa], loff[kMaxKappa];   // its community and counters
    unsigned long long wk[kAttWarps][kMaxKappa]; // each warp's best lane-bests
    int m;                                       // compacted entries
    unsigned long long ck[kFinCand];
    int cx[kFinCand];
};

template <int HG>
struct EdgeRows {
    static constexpr int FR = (64 / HG < kFinMaxRows) ? 64 / HG : kFinMaxRows;   // rows per thread and round
    float z[FR][HG];
    int t[FR];
};

// one round's logits and tokens of this thread: rows j0 + tid + u * NT
template <int HG>
__device__ __forceinline__ void edges_load(const Dims& d, const float* __restrict__ zrow,
                                           const int32_t* __restrict__ rtok, int T, int j0, EdgeRows<HG>& r)
{
    constexpr int NT = kAttWarps * 32;
#pragma unroll
    for (int u = 0; u < EdgeRows<HG>::FR; ++u) {
        const int j = j0 + threadIdx.x + u * NT;
        r.t[u] = 0;
        if (j < T) {
            load_logits<HG>(zrow + (int64_t)(d.S + j) * HG, r.z[u]);
            r.t[u] = __ldcg(rtok + j);
        }
    }
}

// r holds round 0 (edges_load with j0 = 0) on entry.  With `counters`,
// each ranked entry also fetches its community (rcomm) and that
// community's size, capacity and segment start for the assignment.
template <int HG>
__device__ __forceinline__ void cta_edges(const DevState& st, const Dims& d, int g, const float* __restrict__ zrow,
                                          const int32_t* __restrict__ rtok, int T, const float* sM,
                                          const float* sL, EdgeScratch& e, EdgeRows<HG>& r, bool counters)
{
    constexpr int NT = kAttWarps * 32;
    constexpr int FR = EdgeRows<HG>::FR;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kappa = d.kappa;
    if (tid < kMaxKappa) { e.lk[tid] = 0ull; e.lx[tid] = -1; }
    for (int j0 = 0; j0 < max(T, 1); j0 += FR * NT) {
        if (j0 > 0) edges_load<HG>(d, zrow, rtok, T, j0, r);
        unsigned long long key[FR + 1];
#pragma unroll
        for (int u = 0; u < FR; ++u) {
            const int j = j0 + tid + u * NT;
            float sw = 0.f;
#pragma unroll
            for (int h = 0; h < HG; ++h) sw += __expf(r.z[u][h] - sM[h]) * sL[h];
            key[u] = (j < T) ? edge_key(sw, r.t[u]) : 0ull;
        }
        if (j0 > 0) __syncthreads();   // the running list is complete (round 0: each thread cleared its own)
        // the running list's entry `tid` joins as the thread's extra entry
        key[FR] = (tid < kappa) ? e.lk[tid] : 0ull;
        const int xl = (tid < kappa) ? e.lx[tid] : -1;
        unsigned long long best = 0ull;
#pragma unroll
        for (int u = 0; u <= FR; ++u) best = max(best, key[u]);
        // tau: every warp's kappa-th best lane-best is a lower bound of the
        // answer (that warp holds kappa keys at least as good); their max
        // bounds it best.  Entries >= tau come from at most kappa lanes per
        // warp.
        int rank = 0;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) rank += (__shfl_sync(kFull, best, i) > best) ? 1 : 0;
        const unsigned tb = __ballot_sync(kFull, best != 0ull && rank == kappa - 1);
        const unsigned long long tw = tb ? __shfl_sync(kFull, best, __ffs(tb) - 1) : 1ull;   // tb is warp-uniform
        if (lane == 0) e.wk[warp][0] = tw;
        if (tid == 0) e.m = 0;
        __syncthreads();
        unsigned long long tk = 1ull;
#pragma unroll
        for (int wi = 0; wi < kAttWarps; ++wi) tk = max(tk, e.wk[wi][0]);
        // compact the entries at least as good as tau
#pragma unroll
        for (int u = 0; u <= FR; ++u) {
            if (key[u] && key[u] >= tk) {
                const int slot = atomicAdd(&e.m, 1);
                if (slot < kFinCand) {
                    e.ck[slot] = key[u];
                    e.cx[slot] = (u < FR) ? j0 + tid + u * NT : xl;
                }
            }
        }
        __syncthreads();
        // rank them; the first kappa become the running list
        const int m = min(e.m, kFinCand);
        for (int i = tid; i < m; i += NT) {
            const unsigned long long mk = e.ck[i];
            const int x = e.cx[i];
            int rr = 0;
#pragma unroll 8
            for (int j = 0; j < m; ++j) rr += (e.ck[j] > mk) ? 1 : 0;
            if (rr < kappa) {
                e.lk[rr] = mk;
                e.lx[rr] = x;
                if (counters && j0 + FR * NT >= T) {   // last round: prefetch for the vote
                    const int cm = __ldcg(st.rcomm + (int64_t)g * d.NM + x);
                    const int64_t gi = (int64_t)g * d.Nc + cm;
                    e.lc[rr] = cm;
                    e.lsz[rr] = st.csize[gi];
                    e.lcap[rr] = st.ccap[gi];
                    e.loff[rr] = st.coff[gi];
                }
            }
        }
        for (int i = m + tid; i < kappa; i += NT) { e.lk[i] = 0ull; e.lx[i] = -1; }
    }
    __syncthreads();
}

// Rows of one warp: [a0, a1) in the graph's row numbering (sinks, kept
// members, the new token).
struct WarpRows {
    const char* Kb;          // this (batch, KV head)'s K cache
    const char* Vb;
    const int32_t* rtok;     // token of each kept-member row
    float* zrow;             // logits of the kept members, [row][HG]
    int* err;                // the step's error word
    int a0, a1, S, T, R, t_new;
};

__device__ __forceinline__ int row_token(const WarpRows& a, int r)
{
    if (r < a.S) return r;
    if (r == a.R - 1) return a.t_new;
    return a.rtok[r - a.S];
}

// tokens of rows r .. r + TOKW - 1 of this warp into its smem window (a
// token outside [0, n) -- a corrupt row list -- sets the error word and
// gathers row 0 instead, so no address outside the cache is formed)
template <int TOKW>
__device__ __forceinline__ void tokens_from(const WarpRows& a, int r, int* tokw, int lane)
{
    __syncwarp();
#pragma unroll
    for (int i = 0; i < TOKW / 32; ++i) {
        const int rr = r + 32 * i + lane;
        int t = (rr < a.a1) ? row_token(a, rr) : 0;
        if ((unsigned)t > (unsigned)a.t_new) {
            set_error(a.err, CKV_ERR_STATE);
            t = 0;
        }
        tokw[32 * i + lane] = t;
    }
    __syncwarp();
}

// bf16 rows on the tensor cores; leaves the warp's (acc, m, l) per head in
// red[warp][h][RSTR] (after a CTA barrier, as red overlays the pipelines)
template <int HG>
__device__ __forceinline__ void warp_rows_mma(const WarpRows& a, const uint32_t* __restrict__ q2,
                                              unsigned char* wbuf, int* tokw, float* red)
{
    using L = AttLayout<true, HG>;
    constexpr int NB = L::NB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    // B operand Q^T (dims x heads): lane holds head gid, dims 16ks + 2tig (+1, +8, +9)
    uint32_t qf[8][2];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        qf[ks][0] = (gid < HG) ? q2[(gid * kD + 16 * ks + 2 * tig) / 2] : 0u;
        qf[ks][1] = (gid < HG) ? q2[(gid * kD + 16 * ks + 2 * tig + 8) / 2] : 0u;
    }
    const int nb = (a.a1 - a.a0 + NB - 1) / NB;
    const uint64_t pol = l2_evict_first();   // gathered rows are read once per step
    int tok_base = -L::TOKW;
    auto issue = [&](int bb) {
        if (bb < nb) {
            const uint32_t dst = smem_u32(wbuf + (bb % kAttNBuf) * L::BATCH);
            const int rbase = a.a0 + bb * NB;
            if (rbase + NB > tok_base + L::TOKW) {
                tokens_from<L::TOKW>(a, rbase, tokw, lane);
                tok_base = rbase;
            }
            const int ch = lane & 15;
#pragma unroll
            for (int i = 0; i < NB / 2; ++i) {
                const int row = 2 * i + (lane >> 4);
                const bool ok = rbase + row < a.a1;
                const int64_t src = ok ? (int64_t)tokw[rbase - tok_base + row] * 256 + ch * 16 : 0;
                const uint32_t so = row * 256 + ((ch ^ (row & 7)) << 4);
                cp_async16z_ef(dst + so, a.Kb + src, ok, pol);
                cp_async16z_ef(dst + NB * 256 + so, a.Vb + src, ok, pol);
            }
        }
        cp_async_commit();
    };

    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
    // ldmatrix row addresses of this lane: K tiles (A of S^T) and V tiles (A of O^T, transposed)
    const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, khi = lane >> 4;
    const int vrow = (lane & 7) + (lane >> 4) * 8, vhi = (lane >> 3) & 1;
    const bool h0ok = 2 * tig < HG, h1ok = 2 * tig + 1 < HG;

    issue(0);
    issue(1);
    for (int bb = 0; bb < nb; ++bb) {
        issue(bb + 2);
        cp_async_wait<kAttNBuf - 1>();
        __syncwarp();
        const uint32_t kt = smem_u32(wbuf + (bb % kAttNBuf) * L::BATCH), vt = kt + NB * 256;
        const int rbase = a.a0 + bb * NB;
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t fa[4];
            ldsm4(kt + krow * 256 + (((2 * ks + khi) ^ (krow & 7)) << 4), fa);
            mma_bf16(sc, fa, qf[ks][0], qf[ks][1]);
        }
        // logits of rows gid and gid + 8, heads 2tig and 2tig + 1
        const int ra = rbase + gid, rb = ra + 8;
        const bool va = ra < a.a1, vb = rb < a.a1;
        const float kScale = 0.08838834764831845f;   // 1 / sqrt(128)
        float z[4];
        z[0] = (va && h0ok) ? sc[0] * kScale : -INFINITY;
        z[1] = (va && h1ok) ? sc[1] * kScale : -INFINITY;
        z[2] = (vb && h0ok) ? sc[2] * kScale : -INFINITY;
        z[3] = (vb && h1ok) ? sc[3] * kScale : -INFINITY;
        if (h0ok) {   // the kept members' logits, for the edge ranking
            const bool ma = va && ra >= a.S && ra < a.S + a.T, mb = vb && rb >= a.S && rb < a.S + a.T;
            if (HG == 1) {
                if (ma) a.zrow[ra] = z[0];
                if (mb) a.zrow[rb] = z[2];
            } else {
                if (ma) *reinterpret_cast<float2*>(a.zrow + (int64_t)ra * HG + 2 * tig) = make_float2(z[0], z[1]);
                if (mb) *reinterpret_cast<float2*>(a.zrow + (int64_t)rb * HG + 2 * tig) = make_float2(z[2], z[3]);
            }
        }
        // online softmax per head; the max is shared by the 8 lanes of a head column
        float p[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float t = fmaxf(z[j], z[2 + j]);
            t = fmaxf(t, __shfl_xor_sync(kFull, t, 4));
            t = fmaxf(t, __shfl_xor_sync(kFull, t, 8));
            t = fmaxf(t, __shfl_xor_sync(kFull, t, 16));
            const float mn = fmaxf(m[j], t);
            const float al = (m[j] == -INFINITY) ? 0.f : __expf(m[j] - mn);
            p[j] = (z[j] == -INFINITY) ? 0.f : __expf(z[j] - mn);
            p[2 + j] = (z[2 + j] == -INFINITY) ? 0.f : __expf(z[2 + j] - mn);
            l[j] = fmaf(l[j], al, p[j] + p[2 + j]);
            m[j] = mn;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                acc[mt][j] *= al;
                acc[mt][2 + j] *= al;
            }
        }
        // P^T as the B operand, split into bf16 high + low parts
        const uint32_t h01 = pack_bf16(p[0], p[1]), h23 = pack_bf16(p[2], p[3]);
        const uint32_t l01 = pack_bf16(p[0] - bf_lo(h01), p[1] - bf_hi(h01));
        const uint32_t l23 = pack_bf16(p[2] - bf_lo(h23), p[3] - bf_hi(h23));
        const uint32_t bh0 = movtrans(h01), bh1 = movtrans(h23);
        const uint32_t bl0 = movtrans(l01), bl1 = movtrans(l23);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t fv[4];
            ldsm4t(vt + vrow * 256 + (((2 * mt + vhi) ^ (vrow & 7)) << 4), fv);
            mma_bf16(acc[mt], fv, bh0, bh1);
            mma_bf16(acc[mt], fv, bl0, bl1);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        l[j] += __shfl_xor_sync(kFull, l[j], 4);
        l[j] += __shfl_xor_sync(kFull, l[j], 8);
        l[j] += __shfl_xor_sync(kFull, l[j], 16);
    }
    __syncthreads();   // every warp is done with its pipeline: red overlays them
    float* rw = red + warp * HG * L::RSTR;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int h = 2 * tig + j;
        if (h < HG) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                rw[h * L::RSTR + 16 * mt + gid] = acc[mt][j];
                rw[h * L::RSTR + 16 * mt + gid + 8] = acc[mt][2 + j];
            }
            if (gid == 0) { rw[h * L::RSTR + kD] = m[j]; rw[h * L::RSTR + kD + 1] = l[j]; }
        }
    }
}

// fp32 rows on the CUDA cores: 4-row batches, lane = 4 dims
template <int HG>
__device__ __forceinline__ void warp_rows_fma(const WarpRows& a, const float* __restrict__ qg,
                                              unsigned char* wbuf, int* tokw, float* pz, float* red)
{
    using L = AttLayout<false, HG>;
    constexpr int NB = L::NB, RB = L::RB, NV = 4 * HG;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float qv[HG][4];
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) qv[h][j] = qg[h * kD + 4 * lane + j];
    const int nb = (a.a1 - a.a0 + NB - 1) / NB;
    int tok_base = -L::TOKW;
    auto issue = [&](int bb) {
        if (bb < nb) {
            unsigned char* dst = wbuf + (bb % kAttNBuf) * L::BATCH;
            const int rbase = a.a0 + bb * NB;
            if (rbase + NB > tok_base + L::TOKW) {
                tokens_from<L::TOKW>(a, rbase, tokw, lane);
                tok_base = rbase;
            }
            constexpr int NCH = RB / 16;   // 16-byte chunks per row
#pragma unroll
            for (int j = 0; j < NB * NCH / 32; ++j) {
                const int e = j * 32 + lane;
                const int row = e / NCH, ch = e % NCH;
                if (rbase + row < a.a1) {
                    const int tk = tokw[rbase - tok_base + row];
                    cp_async16(dst + row * RB + ch * 16, a.Kb + (int64_t)tk * RB + ch * 16);
                    cp_async16(dst + (NB + row) * RB + ch * 16, a.Vb + (int64_t)tk * RB + ch * 16);
                }
            }
        }
        cp_async_commit();
    };
    float m_run[HG], l_run[HG], acc[HG][4];
#pragma unroll
    for (int h = 0; h < HG; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
    }
    issue(0);
    issue(1);
    for (int bb = 0; bb < nb; ++bb) {
        issue(bb + 2);
        cp_async_wait<kAttNBuf - 1>();
        __syncwarp();
        const unsigned char* kt = wbuf + (bb % kAttNBuf) * L::BATCH;
        const unsigned char* vt = kt + NB * RB;
        const int rbase = a.a0 + bb * NB;
        const int rows_in = min(NB, a.a1 - rbase);
        {   // logits of the 4 rows: one butterfly
            float v[NV];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float x[4] = {0.f, 0.f, 0.f, 0.f};
                if (r < rows_in) {
                    const float4 w = *reinterpret_cast<const float4*>(kt + r * RB + 16 * lane);
                    x[0] = w.x; x[1] = w.y; x[2] = w.z; x[3] = w.w;
                }
#pragma unroll
                for (int h = 0; h < HG; ++h)
                    v[r * HG + h] = fmaf(qv[h][3], x[3], fmaf(qv[h][2], x[2], fmaf(qv[h][1], x[1], qv[h][0] * x[0])));
            }
            const float z = transpose_reduce<NV>(v, lane) * 0.08838834764831845f;   // 1 / sqrt(128)
            const int idx = tr_index<NV>(lane);
            constexpr int lowmask = (NV >= 32) ? 0 : (32 / NV) - 1;
            if ((lane & lowmask) == 0) {
                const int rr = idx / HG;
                pz[rr * HG + idx % HG] = (rr < rows_in) ? z : -INFINITY;
                const int r = rbase + rr;
                if (rr < rows_in && r >= a.S && r < a.S + a.T) a.zrow[(int64_t)r * HG + idx % HG] = z;
            }
        }
        __syncwarp();
        float pb[NB][HG];
#pragma unroll
        for (int r = 0; r < NB; ++r)
#pragma unroll
            for (int h = 0; h < HG; ++h) pb[r][h] = pz[r * HG + h];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            float mb = pb[0][h];
#pragma unroll
            for (int r = 1; r < NB; ++r) mb = fmaxf(mb, pb[r][h]);
            const float m_new = fmaxf(m_run[h], mb);
            const float sc = (m_run[h] == -INFINITY) ? 0.f : __expf(m_run[h] - m_new);
            l_run[h] *= sc;
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[h][e] *= sc;
            m_run[h] = m_new;
#pragma unroll
            for (int r = 0; r < NB; ++r) {
                pb[r][h] = (pb[r][h] == -INFINITY) ? 0.f : __expf(pb[r][h] - m_new);
                l_run[h] += pb[r][h];
            }
        }
#pragma unroll
        for (int r = 0; r < NB; ++r) {
            if (r >= rows_in) break;
            const float4 w = *reinterpret_cast<const float4*>(vt + r * RB + 16 * lane);
            const float x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < HG; ++h)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h][e] = fmaf(pb[r][h], x[e], acc[h][e]);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    __syncthreads();   // every warp is done with its pipeline: red overlays them
#pragma unroll
    for (int h = 0; h < HG; ++h) {
        float* rw = red + (warp * HG + h) * L::RSTR;
        *reinterpret_cast<float4*>(rw + 4 * lane) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
        if (lane == 0) { rw[kD] = m_run[h]; rw[kD + 1] = l_run[h]; }
    }
}

// The new token's edges (the top kappa of w = sum_h exp(z - M_h) / L_h over
// the kept members), its assignment and the community update, for graph g
// of the step whose output merge left sM (max) and sL (1 / sum) per head.
// er: the first round of kept members' logits, loaded by the caller; kv:
// this thread's value of the new token's key (threads < D).
template <int HG>
__device__ __forceinline__ void edges_assign_update(const DevState& s, const Dims& d, int g, int T, int n, float kv,
                                                    EdgeRows<HG>& er, unsigned char* scratch, const float* sM,
                                                    const float* sL, int* sflag)
{
    constexpr int NT = kAttWarps * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t* rtok = s.rtok + (int64_t)g * d.NM;
    const float* zrow = s.zrow + (int64_t)g * d.NM * HG;
    EdgeScratch& es = *reinterpret_cast<EdgeScratch*>(scratch);
    cta_edges<HG>(s, d, g, zrow, rtok, T, sM, sL, es, er, d.fuse_assign != 0);
    if (warp == 0) {
        const unsigned long long lk = (lane < d.kappa) ? es.lk[lane] : 0ull;
        const bool real = lk != 0ull;
        const int ne = __popc(__ballot_sync(kFull, real));
        const float lw = key_w(lk);
        const int cm = !real ? 0 : d.fuse_assign ? es.lc[lane] : __ldcg(s.rcomm + (int64_t)g * d.NM + es.lx[lane]);
        if (real) {
            s.e_w[(int64_t)g * d.kappa + lane] = lw;
            s.e_tok[(int64_t)g * d.kappa + lane] = key_t(lk);
            s.e_comm[(int64_t)g * d.kappa + lane] = cm;
        }
        if (lane == 0) s.meta[(int64_t)g * M_COUNT + M_NEDGE] = ne;
        if (d.fuse_assign) {
            // weighted plurality of the edges' communities: each lane sums
            // its community's weights in rank order (double), ties to the
            // lower id
            double v = 0.0;
            for (int e = 0; e < ne; ++e) {
                const int ce = __shfl_sync(kFull, cm, e);
                const float we = __shfl_sync(kFull, lw, e);
                if (ce == cm) v += (double)we;
            }
            double bv = real ? v : -1.0;
            int bc = real ? cm : 0x7fffffff;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const double v2 = __shfl_xor_sync(kFull, bv, o);
                const int c2 = __shfl_xor_sync(kFull, bc, o);
                if (v2 > bv || (v2 == bv && c2 < bc)) { bv = v2; bc = c2; }
            }
            if (lane == 0) {
                // the winner's counters were fetched with the ranking (no
                // edges: community 0)
                const int c = (ne == 0) ? 0 : bc;
                int src = 0;
                while (src < ne - 1 && es.lc[src] != c) ++src;
                const int64_t gi = (int64_t)g * d.Nc + c;
                const int size = ne ? es.lsz[src] : s.csize[gi];
                const int cp = ne ? es.lcap[src] : s.ccap[gi];
                const int off0 = ne ? es.loff[src] : s.coff[gi];
                const int top = s.pool_top[g];
                int ok = 1, off = off0;
                // the community and its segment inside the pool (debug build)
                if (!CKV_IN_RANGE(c, 0, d.Nc, s.err) || !CKV_IN_RANGE(size, 0, (int64_t)cp + 1, s.err) ||
                    !CKV_IN_RANGE(off0, 0, d.P - cp + 1, s.err))
                    ok = -1;
                if (ok > 0 && size == cp) {   // segment full: move it to the pool top with twice the room
                    const int ncap = max(16, 2 * cp);
                    if ((int64_t)top + ncap > d.P) ok = 0;
                    else { s.pool_top[g] = top + ncap; off = top; }
                }
                if (!ok) set_error(s.err, CKV_ERR_CAPACITY);
                sflag[0] = c; sflag[1] = ok > 0; sflag[2] = off; sflag[3] = size; sflag[4] = off0; sflag[5] = ne;
            }
        }
    }
    if (!d.fuse_assign) return;
    __syncthreads();
    if (!sflag[1]) return;
    const int c = sflag[0], off = sflag[2], size = sflag[3], old_off = sflag[4], ne = sflag[5];
    const int t = n - 1;
    int32_t* pool = s.pool + (int64_t)g * d.P;
    if (off != old_off)
        for (int i = tid; i < size; i += NT) pool[off + i] = pool[old_off + i];
    // running-mean update of the assigned centroid, double math rounded once
    if (tid < kD) {
        float* mu = s.mu + ((int64_t)g * d.Nc + c) * kD;
        const double mv = (double)mu[tid];
        mu[tid] = __double2float_rn(__dadd_rn(mv, __ddiv_rn(__dsub_rn((double)kv, mv), (double)(size + 1))));
    }
    __syncthreads();   // the segment copy is complete before the append
    const int64_t row = (int64_t)g * (d.NM - d.n_init) + (t - d.n_init);
    if (tid == 0) {
        if (off != old_off) {
            s.coff[(int64_t)g * d.Nc + c] = off;
            s.ccap[(int64_t)g * d.Nc + c] = max(16, 2 * s.ccap[(int64_t)g * d.Nc + c]);
        }
        pool[off + size] = t;
        s.csize[(int64_t)g * d.Nc + c] = size + 1;
        s.tok_comm[(int64_t)g * d.NM + t] = c;
        s.meta[(int64_t)g * M_COUNT + M_ASSIGNED] = c;
        s.edge_deg[row] = ne;
    }
    if (tid < ne) {
        s.edge_col[row * d.kappa + tid] = s.e_tok[(int64_t)g * d.kappa + tid];
        s.edge_w[row * d.kappa + tid] = s.e_w[(int64_t)g * d.kappa + tid];
    }
}


// A graph's last slice to finish: merge the slices' partials into the
// output and each head's (m, l); with UPD also rank the edges, assign the
// new token and update its community.  Runs with the whole CTA; red / smem
// scratch is free.
template <int HG, bool UPD>
__device__ __forceinline__ void finish_graph(const DevState& s, const Dims& d, int g, int nc, int R,
                                             const void* __restrict__ K, int n, float* __restrict__ out,
                                             unsigned char* scratch, float* sM, float* sL, int* sflag)
{
    constexpr int NT = kAttWarps * 32;
    const int tid = threadIdx.x;
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    const int T = R - d.S - 1;
    const int32_t* rtok = s.rtok + (int64_t)g * d.NM;
    const float* zrow = s.zrow + (int64_t)g * d.NM * HG;
    const float* pmg = s.part_ml + (int64_t)g * d.nCTA * HG * 2;
    const float* pog = s.part_o + (int64_t)g * d.nCTA * HG * kD;

    // inline update (UPD): the first round of kept members and the new
    // token's key are loaded under the output merge (else k_update runs it)
    EdgeRows<HG> er;
    float kv = 0.f;
    if constexpr (UPD) {
        edges_load<HG>(d, zrow, rtok, T, 0, er);
        if (d.fuse_assign && tid < kD) {
            const int64_t krow = (((int64_t)b * d.Hkv + kvh) * d.NM + (n - 1)) * kD;
            kv = d.bf16 ? elem<true>(K, krow + tid) : elem<false>(K, krow + tid);
        }
    }
    // ---- output: every value merged online over the slices; the thread of
    // a head's first value also leaves that head's max and 1 / sum.  A
    // thread's IPT values take their loads of a batch of slices together.
    {
        constexpr int IPT = (HG * kD + NT - 1) / NT;              // values per thread
        constexpr int U = (8 / IPT > 1) ? 8 / IPT : 2;            // slices per batch
        float M[IPT], Ls[IPT], o[IPT];
#pragma unroll
        for (int it = 0; it < IPT; ++it) { M[it] = -INFINITY; Ls[it] = 0.f; o[it] = 0.f; }
        for (int j0 = 0; j0 < nc; j0 += U) {
            float2 mj[IPT][U];
            float oj[IPT][U];
#pragma unroll
            for (int it = 0; it < IPT; ++it) {
                const int i = tid + it * NT;
                const int h = i / kD;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const bool ok = j0 + u < nc && i < HG * kD;
                    mj[it][u] = ok ? __ldcg(reinterpret_cast<const float2*>(pmg + ((int64_t)(j0 + u) * HG + h) * 2))
                                   : make_float2(-INFINITY, 0.f);
                    oj[it][u] = ok ? __ldcg(pog + (int64_t)(j0 + u) * HG * kD + i) : 0.f;
                }
            }
#pragma unroll
            for (int it = 0; it < IPT; ++it)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (mj[it][u].x == -INFINITY) continue;
                    const float mn = fmaxf(M[it], mj[it][u].x);
                    const float a = (M[it] == -INFINITY) ? 0.f : __expf(M[it] - mn), c = __expf(mj[it][u].x - mn);
                    o[it] = o[it] * a + oj[it][u] * c;
                    Ls[it] = Ls[it] * a + mj[it][u].y * c;
                    M[it] = mn;
                }
        }
#pragma unroll
        for (int it = 0; it < IPT; ++it) {
            const int i = tid + it * NT;
            if (i >= HG * kD) continue;
            const int h = i / kD;
            out[((int64_t)b * d.Hq + h0 + h) * kD + i % kD] = o[it] / Ls[it];
            if (i % kD == 0) {
                sM[h] = M[it];
                sL[h] = 1.f / Ls[it];
                if (s.sel_ml)
                    *reinterpret_cast<float2*>(s.sel_ml + 2 * ((int64_t)b * d.Hq + h0 + h)) = make_float2(M[it], Ls[it]);
            }
        }
    }
    __syncthreads();
    if constexpr (UPD) edges_assign_update<HG>(s, d, g, T, n, kv, er, scratch, sM, sL, sflag);
}

// CTA work: the graphs' rows laid end to end (graph-major, each graph's
// rows in its own order) are split evenly over the CTAs; a CTA's share is
// one or more pieces, each a contiguous run of one graph's rows.
struct Piece {
    int g, r0, r1;     // graph and its rows [r0, r1)
    int k, nc;         // slice index of the piece among the graph's nc slices
    int R;             // the graph's rows
};
constexpr int kMaxPieces = 32;

// the CTA whose share holds global row x: shares are [lo(i), lo(i+1)) with
// lo(i) = floor(i * tot / P), so the last i with lo(i) <= x
__device__ __forceinline__ int share_of(long long x, long long tot, int P)
{
    return (int)(((x + 1) * P - 1) / tot);
}

// kAttCluster CTAs per graph, one thread-block cluster, when CL: each CTA
// leaves its slice's partial in its own shared memory and the cluster's
// rank 0 merges the four through distributed shared memory (no partials in
// global memory, no arrival counter)
constexpr int kAttCluster = 4;
constexpr int kAttClPart = 64 * 1024;   // the cluster partial's offset in the (free) pipeline area

template <bool BF16, int HG, bool UPD, bool CL>
__global__ void __launch_bounds__(kAttWarps * 32, 1) k_attend(DevState s, Dims d, const void* __restrict__ q,
                                                             const void* __restrict__ K,
                                                             const void* __restrict__ V, int n,
                                                             float* __restrict__ out)
{
    using L = AttLayout<BF16, HG>;
    constexpr int RB = L::RB;
    constexpr int NT = kAttWarps * 32;
    pdl_wait();
    if (d.pdl == 1) pdl_trigger();
    extern __shared__ __align__(128) unsigned char smem[];
    float* sM = reinterpret_cast<float*>(smem + L::off_misc);          // [8] graph max per head
    float* sL = sM + 8;                                                // [8] 1 / graph sum per head
    int* sflag = reinterpret_cast<int*>(sL + 8);                       // [8]
    int* snp = sflag + 8;                                              // [1] pieces of this CTA
    int* snf = snp + 1;                                                // [1] graphs it finishes
    Piece* sp = reinterpret_cast<Piece*>(snp + 4);                     // [kMaxPieces]
    int* sfin = reinterpret_cast<int*>(sp + kMaxPieces);               // [kMaxPieces] their pieces
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = d.G;
    unsigned char* wbuf = smem + L::off_buf + warp * L::WBUF;
    int* tokw = reinterpret_cast<int*>(smem + L::off_tokw) + warp * L::TOKW;
    float* red = reinterpret_cast<float*>(smem + L::off_buf);          // [warps][HG][RSTR]

    // ---- this CTA's pieces.  Graph-aligned split (at least as many CTAs as
    // graphs): graph g owns CTAs [g P / G, (g + 1) P / G), each one slice of
    // its rows, so a CTA needs only its own graph's row count.  Otherwise the
    // graphs' rows laid end to end are split evenly: all graphs' row counts
    // and the error word in one round of loads, then warp 0 lists the pieces,
    // kMaxPieces at a time (a later round reloads the rows: the staging area
    // is reused).
    const bool aligned = d.att_aligned && (int)gridDim.x >= G;
    int* sR = reinterpret_cast<int*>(smem + L::off_buf);
    __shared__ int s_failed;   // the step already failed (read with the row count: one round trip)
    if (aligned) {
        if (tid == 0) {
            const int failed = *(volatile const int*)s.err;
            const int Pa = (int)gridDim.x;
            const int g = CL ? (int)blockIdx.x / kAttCluster : (int)(((long long)(blockIdx.x + 1) * G - 1) / Pa);
            const int fa = CL ? g * kAttCluster : (int)((long long)g * Pa / G);
            const int fb = CL ? fa + kAttCluster : (int)((long long)(g + 1) * Pa / G);
            Piece pc;
            pc.g = g;
            pc.k = (int)blockIdx.x - fa;
            pc.nc = fb - fa;
            pc.R = __ldcg(s.meta + (int64_t)g * M_COUNT + M_ROWS);
            pc.r0 = (int)((int64_t)pc.k * pc.R / pc.nc);
            pc.r1 = (int)((int64_t)(pc.k + 1) * pc.R / pc.nc);
            sp[0] = pc;
            *snp = 1;
            *snf = 0;
            s_failed = failed;
        }
    } else {
        if (tid == 0) s_failed = *(volatile const int*)s.err;
        for (int g = tid; g < G; g += NT) sR[g] = s.meta[(int64_t)g * M_COUNT + M_ROWS];
    }
    __syncthreads();
    // (CL: no early exit -- every CTA of a cluster must reach its barriers;
    // a failed step's rows are checked tokens of a consistent row list)
    if (!CL && s_failed) return;
    for (int done = 0;; done += kMaxPieces) {
        if (!aligned && warp == 0) {
            auto rows_of = [&](int g) -> int {
                return done == 0 ? sR[g] : __ldcg(s.meta + (int64_t)g * M_COUNT + M_ROWS);
            };
            long long tot = 0;
            for (int g0 = 0; g0 < G; g0 += 32) tot += (g0 + lane < G) ? rows_of(g0 + lane) : 0;
#pragma unroll
            for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(kFull, tot, o);
            const int P = (int)min((long long)gridDim.x, tot);
            const long long A = (long long)blockIdx.x * tot / P, B = (long long)(blockIdx.x + 1) * tot / P;
            int np = 0;                            // pieces seen so far
            long long carry = 0;
            for (int g0 = 0; g0 < G && (int)blockIdx.x < P; g0 += 32) {
                const int g = g0 + lane;
                const int R = (g < G) ? rows_of(g) : 0;
                long long incl = R;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long t = __shfl_up_sync(kFull, incl, o);
                    if (lane >= o) incl += t;
                }
                const long long Pg = carry + incl - R;
                const bool mine = g < G && Pg < B && Pg + R > A;
                const unsigned bal = __ballot_sync(kFull, mine);
                if (mine) {
                    const int slot = np + __popc(bal & ((1u << lane) - 1u)) - done;
                    if (slot >= 0 && slot < kMaxPieces) {
                        Piece pc;
                        pc.g = g;
                        pc.r0 = (int)(max(A, Pg) - Pg);
                        pc.r1 = (int)(min(B, Pg + R) - Pg);
                        const int f = share_of(Pg, tot, P);
                        pc.k = (int)blockIdx.x - f;
                        pc.nc = share_of(Pg + R - 1, tot, P) - f + 1;
                        pc.R = R;
                        sp[slot] = pc;
                    }
                }
                np += __popc(bal);
                carry += __shfl_sync(kFull, incl, 31);
            }
            if (lane == 0) { *snp = max(0, min(np - done, kMaxPieces)); *snf = 0; }
        }
        __syncthreads();
        const int npieces = *snp;
        for (int pi = 0; pi < npieces; ++pi) {
            const Piece pc = sp[pi];
            const int g = pc.g, k = pc.k, nc = pc.nc, R = pc.R;
            int b, h0, kvh;
            graph_heads(d, g, b, h0, kvh);
            const int T = R - d.S - 1;
            const int nrows = pc.r1 - pc.r0;
            const int64_t kvbase = ((int64_t)b * d.Hkv + kvh) * d.NM;
            WarpRows a;
            a.Kb = reinterpret_cast<const char*>(K) + kvbase * RB;
            a.Vb = reinterpret_cast<const char*>(V) + kvbase * RB;
            a.rtok = s.rtok + (int64_t)g * d.NM;
            a.zrow = s.zrow + (int64_t)g * d.NM * HG;
            a.err = s.err;
            a.a0 = pc.r0 + (int)((int64_t)warp * nrows / kAttWarps);
            a.a1 = pc.r0 + (int)((int64_t)(warp + 1) * nrows / kAttWarps);
            a.S = d.S;
            a.T = T;
            a.R = R;
            a.t_new = n - 1;
            __syncthreads();   // the previous piece of this CTA is done with the buffers
            if constexpr (BF16) {
                const uint32_t* q2 = reinterpret_cast<const uint32_t*>(q) + ((int64_t)b * d.Hq + h0) * kD / 2;
                warp_rows_mma<HG>(a, q2, wbuf, tokw, red);
            } else {
                const float* qg = reinterpret_cast<const float*>(q) + ((int64_t)b * d.Hq + h0) * kD;
                float* pz = reinterpret_cast<float*>(smem + L::off_pz) + warp * L::NB * HG;
                warp_rows_fma<HG>(a, qg, wbuf, tokw, pz, red);
            }
            __syncthreads();
            // combine the warps: (m, l, acc) -> this slice's partial per head
            // (CL: into this CTA's shared memory, past the reduction area)
            float* po = CL ? reinterpret_cast<float*>(smem + L::off_buf + kAttClPart)
                           : s.part_o + ((int64_t)g * d.nCTA + k) * HG * kD;
            float* pm = CL ? po + HG * kD : s.part_ml + ((int64_t)g * d.nCTA + k) * HG * 2;
            for (int i = tid; i < HG * kD; i += NT) {
                const int h = i / kD, dd = i % kD;
                float mw[kAttWarps];
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kAttWarps; ++w) {
                    mw[w] = red[(w * HG + h) * L::RSTR + kD];
                    M = fmaxf(M, mw[w]);
                }
                float o = 0.f, l = 0.f;
#pragma unroll
                for (int w = 0; w < kAttWarps; ++w) {
                    const float* rw = red + (w * HG + h) * L::RSTR;
                    const float f = (mw[w] == -INFINITY) ? 0.f : __expf(mw[w] - M);
                    o = fmaf(rw[dd], f, o);
                    l = fmaf(rw[kD + 1], f, l);
                }
                po[i] = o;
                if (dd == 0) *reinterpret_cast<float2*>(pm + h * 2) = make_float2(M, l);
            }
            if constexpr (CL) {
                static_assert(kAttWarps * HG * L::RSTR * 4 <= kAttClPart &&
                                  kAttClPart + (HG * kD + 2 * HG) * 4 <= kAttWarps * L::WBUF,
                              "the cluster partial lies in the pipelines, past the reduction");
                // ---- the cluster's four partials merged by its rank 0
                namespace cg = cooperative_groups;
                cg::cluster_group cl = cg::this_cluster();
                cl.sync();                                   // every slice's partial is in place
                if (cl.block_rank() == 0) {
                    int b, h0, kvh;
                    graph_heads(d, g, b, h0, kvh);
                    for (int i = tid; i < HG * kD; i += NT) {
                        const int h = i / kD;
                        float mr[kAttCluster], orr[kAttCluster], lr[kAttCluster];
                        float M = -INFINITY;
#pragma unroll
                        for (int r = 0; r < kAttCluster; ++r) {
                            const float* pr = cl.map_shared_rank(po, r);
                            const float2 ml = *reinterpret_cast<const float2*>(pr + HG * kD + h * 2);
                            mr[r] = ml.x;
                            lr[r] = ml.y;
                            orr[r] = pr[i];
                            M = fmaxf(M, mr[r]);
                        }
                        float o = 0.f, l = 0.f;
#pragma unroll
                        for (int r = 0; r < kAttCluster; ++r) {
                            const float f = (mr[r] == -INFINITY) ? 0.f : __expf(mr[r] - M);
                            o = fmaf(orr[r], f, o);
                            l = fmaf(lr[r], f, l);
                        }
                        out[((int64_t)b * d.Hq + h0 + h) * kD + i % kD] = o / l;
                        if (i % kD == 0 && s.sel_ml)
                            *reinterpret_cast<float2*>(s.sel_ml + 2 * ((int64_t)b * d.Hq + h0 + h)) = make_float2(M, l);
                    }
                }
                cl.sync();                                   // no slice leaves before rank 0 has read it
                return;
            }
            // ---- the last slice of a graph to arrive finishes it
            __threadfence();
            __syncthreads();
            if (tid == 0 && atomicAdd(&s.bar[g * 2], 1u) == (unsigned)nc - 1) sfin[(*snf)++] = pi;
        }
        // ---- graphs whose last slice this CTA was: finish them (after all
        // of this CTA's pieces, so none of its slices waits behind a finish)
        __syncthreads();
        const int nfin = *snf;
        if (nfin) __threadfence();
        if (d.pdl == 2) pdl_trigger();
        for (int f = 0; f < nfin; ++f) {
            const Piece pc = sp[sfin[f]];
            __syncthreads();   // the scratch is free
            finish_graph<HG, UPD>(s, d, pc.g, pc.nc, pc.R, K, n, out, smem + L::off_buf, sM, sL, sflag);
            if (tid == 0) s.bar[pc.g * 2] = 0u;
        }
        if (npieces < kMaxPieces) break;
        __syncthreads();   // every thread is done with this round's list
    }
}

// The deferred part of a decode step, launched by ckv_assign_update: one CTA
// per graph computes the new token's edges, assignment and community update
// from what the step's attention kernel left -- each head's softmax max and
// sum over the attended rows (sel_ml), the kept members' logits (zrow) and
// rows (rtok, rcomm).  A step that already failed changes no state.  It
// runs beside the next step's scan: at most 96 registers a thread, so that
// one update CTA (two warps per SM sub-partition) and one scan CTA (three
// warps on one sub-partition) fit in a sub-partition's 16 K registers.
template <int HG>
__global__ void __maxnreg__(96) k_update(DevState s, Dims d, const void* __restrict__ K, int n)
{
    extern __shared__ __align__(128) unsigned char smem[];
    float* sM = reinterpret_cast<float*>(smem + sizeof(EdgeScratch));   // [8]
    float* sL = sM + 8;                                                  // [8]
    int* sflag = reinterpret_cast<int*>(sL + 8);                         // [8]
    const int g = blockIdx.x, tid = threadIdx.x;
    if (step_failed(s.err)) return;
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    const int T = __ldcg(s.meta + (int64_t)g * M_COUNT + M_ROWS) - d.S - 1;
    EdgeRows<HG> er;
    edges_load<HG>(d, s.zrow + (int64_t)g * d.NM * HG, s.rtok + (int64_t)g * d.NM, T, 0, er);
    float kv = 0.f;
    if (tid < kD) {
        const int64_t krow = (((int64_t)b * d.Hkv + kvh) * d.NM + (n - 1)) * kD;
        kv = d.bf16 ? elem<true>(K, krow + tid) : elem<false>(K, krow + tid);
    }
    if (tid < HG) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(s.sel_ml) + ((int64_t)b * d.Hq + h0 + tid));
        sM[tid] = ml.x;
        sL[tid] = 1.f / ml.y;
    }
    __syncthreads();
    edges_assign_update<HG>(s, d, g, T, n, kv, er, smem, sM, sL, sflag);
}

constexpr size_t kUpdateSmem = sizeof(EdgeScratch) + 24 * 4;
static_assert(sizeof(ScoreSmem) + kUpdateSmem + 2 * 1024 <= 228 * 1024, "a scan CTA and an update CTA share an SM");

// new token's K and V rows: staging [B][H_kv][D] -> cache row `row`
__global__ void k_append(const uint32_t* __restrict__ knew, const uint32_t* __restrict__ vnew,
                         uint32_t* __restrict__ K, uint32_t* __restrict__ V, int64_t NM, int row, int words)
{
    const int bh = blockIdx.x;
    const int64_t dst = ((int64_t)bh * NM + row) * words;
    for (int i = threadIdx.x; i < words; i += blockDim.x) {
        K[dst + i] = knew[(int64_t)bh * words + i];
        V[dst + i] = vnew[(int64_t)bh * words + i];
    }
}

// the stream priority range {lowest, highest} (the same on every device)
struct PriorityRange {
    int lo = 0, hi = 0;
    PriorityRange()
    {
        if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) lo = hi = 0;
    }
};
inline void priority_range(int& lo, int& hi)
{
    static const PriorityRange r;   // fetched once, on first use
    lo = r.lo;
    hi = r.hi;
}

// The decode kernels run at the highest priority (the step's output waits
// on them; the deferred update runs at the lowest), with programmatic
// stream serialization when d.pdl: the kernel may begin launching while
// the previous kernel of the stream finishes; every decode kernel starts
// with pdl_wait.
template <typename... P, typename... A>
cudaError_t launch_ex(const Dims& d, void (*fn)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      A&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    int lo = 0, hi = 0;
    priority_range(lo, hi);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributePriority;
    attr[0].val.priority = hi;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = d.pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, fn, std::forward<A>(args)...);
}

template <typename F>
cudaError_t dispatch_hg(int hg, F&& f)
{
    switch (hg) {
        case 1: return f(std::integral_constant<int, 1>{});
        case 2: return f(std::integral_constant<int, 2>{});
        case 4: return f(std::integral_constant<int, 4>{});
        case 8: return f(std::integral_constant<int, 8>{});
        default: return cudaErrorInvalidValue;
    }
}

// the attention kernel of a context: fp32 or bf16 rows, HG heads per graph,
// with the edges, assignment and update inline or left to k_update
template <int HG>
void* attend_fn(const Dims& d)
{
    if (d.att_cluster)
        return d.bf16 ? reinterpret_cast<void*>(k_attend<true, HG, false, true>)
                      : reinterpret_cast<void*>(k_attend<false, HG, false, true>);
    if (d.bf16)
        return d.defer_update ? reinterpret_cast<void*>(k_attend<true, HG, false, false>)
                              : reinterpret_cast<void*>(k_attend<true, HG, true, false>);
    return d.defer_update ? reinterpret_cast<void*>(k_attend<false, HG, false, false>)
                          : reinterpret_cast<void*>(k_attend<false, HG, true, false>);
}

template <int HG>
void* update_fn()
{
    return reinterpret_cast<void*>(k_update<HG>);
}

}  // namespace

size_t select_smem_bytes(int n_comm, int budget)
{
    // the larger of the passes' arrays and the kept list
    const size_t kept_cap = (size_t)std::min(n_comm, budget + 1);
    const size_t passes = (size_t)8 * kSelCand + 4 * kSelBins + 8 * kSelCand;
    return std::max(passes, 4 * (3 * kept_cap + 1));
}

template <int E>
static cudaError_t launch_select_e(const DevState& s, const Dims& d, cudaStream_t st)
{
    return launch_ex(d, k_select<E>, dim3(d.G), dim3(kSelThreads), select_smem_bytes(d.n_comm, d.budget), st, s, d);
}cudaError_t launch_score(const DevState& s, const Dims& d, const void* q, cudaStream_t st)
{
    const int units = d.G * ((d.n_comm + 31) / 32);
    const int grid = units < d.nSM ? units : d.nSM;   // persistent: one CTA per SM
    const size_t smem = sizeof(ScoreSmem);
    return launch_ex(d, d.bf16 ? k_score<true> : k_score<false>, dim3(grid), dim3(kScoreThreads), smem, st, s, d, q);
}

cudaError_t launch_select(const DevState& s, const Dims& d, cudaStream_t st)
{
    switch ((d.n_comm + kSelThreads - 1) / kSelThreads) {
        case 0:
        case 1: return launch_select_e<1>(s, d, st);
        case 2: return launch_select_e<2>(s, d, st);
        case 3: return launch_select_e<3>(s, d, st);
        case 4: return launch_select_e<4>(s, d, st);
        case 5: return launch_select_e<5>(s, d, st);
        case 6: return launch_select_e<6>(s, d, st);
        case 7: return launch_select_e<7>(s, d, st);
        case 8: return launch_select_e<8>(s, d, st);
        case 9: return launch_select_e<9>(s, d, st);
        case 10: return launch_select_e<10>(s, d, st);
        case 11: return launch_select_e<11>(s, d, st);
        case 12: return launch_select_e<12>(s, d, st);
        case 13: return launch_select_e<13>(s, d, st);
        case 14: return launch_select_e<14>(s, d, st);
        case 15: return launch_select_e<15>(s, d, st);
        default: return launch_select_e<16>(s, d, st);
    }
}

cudaError_t prepare_kernels(const Dims& d)
{
    // shared-memory limits are set once per device, before any launch (and
    // so outside any stream capture)
    const int sel_bytes = (int)select_smem_bytes(kMaxCommunities, kMaxCommunities);
    cudaError_t e = cudaSuccess;
    const void* sel_fns[] = {(const void*)k_select<1>,  (const void*)k_select<2>,  (const void*)k_select<3>,
                             (const void*)k_select<4>,  (const void*)k_select<5>,  (const void*)k_select<6>,
                             (const void*)k_select<7>,  (const void*)k_select<8>,  (const void*)k_select<9>,
                             (const void*)k_select<10>, (const void*)k_select<11>, (const void*)k_select<12>,
                             (const void*)k_select<13>, (const void*)k_select<14>, (const void*)k_select<15>,
                             (const void*)k_select<16>};
    for (const void* f : sel_fns)
        if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, sel_bytes);
    // the scan and the update kernel (side stream) share SMs: both ask for
    // the largest shared-memory carveout, so that a scan CTA never waits
    // for an SM's update CTA to leave (their registers fit together too)
    for (const void* f : {(const void*)k_score<true>, (const void*)k_score<false>}) {
        if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(ScoreSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    }
    if (e != cudaSuccess) return e;
    return dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        void* fn = attend_fn<HG>(d);
        const int bytes = d.bf16 ? AttLayout<true, HG>::bytes : AttLayout<false, HG>::bytes;
        cudaError_t e2 = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e2 == cudaSuccess)
            e2 = cudaFuncSetAttribute(update_fn<HG>(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kUpdateSmem);
        if (e2 == cudaSuccess)
            e2 = cudaFuncSetAttribute(update_fn<HG>(), cudaFuncAttributePreferredSharedMemoryCarveout,
                                      cudaSharedmemCarveoutMaxShared);
        return e2;
    });
}

bool attend_on_clusters(const Dims& d, int sms)
{
    return d.defer_update && d.att_aligned && (int64_t)d.G * kAttCluster <= sms;
}

int attend_grid(const Dims& d, int sms)
{
    int occ = 0;
    cudaError_t e = prepare_kernels(d);
    if (e == cudaSuccess)
        e = dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
            constexpr int HG = decltype(hgc)::value;
            void* fn = attend_fn<HG>(d);
            const int bytes = d.bf16 ? AttLayout<true, HG>::bytes : AttLayout<false, HG>::bytes;
            return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kAttWarps * 32, bytes);
        });
    if (e != cudaSuccess || occ < 1) return 0;
    return occ * sms;
}

cudaError_t launch_attend(const DevState& s, const Dims& d, const void* q, const void* K, const void* V, int n,
                          float* out, cudaStream_t st)
{
    return dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        const int bytes = d.bf16 ? AttLayout<true, HG>::bytes : AttLayout<false, HG>::bytes;
        if (d.att_cluster) {   // kAttCluster CTAs per graph in one cluster
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(d.G * kAttCluster);
            cfg.blockDim = dim3(kAttWarps * 32);
            cfg.dynamicSmemBytes = bytes;
            cfg.stream = st;
            int lo = 0, hi = 0;
            priority_range(lo, hi);
            cudaLaunchAttribute attr[2];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = kAttCluster;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            attr[1].id = cudaLaunchAttributePriority;
            attr[1].val.priority = hi;
            cfg.attrs = attr;
            cfg.numAttrs = 2;
            if (d.bf16) return cudaLaunchKernelEx(&cfg, k_attend<true, HG, false, true>, s, d, q, K, V, n, out);
            return cudaLaunchKernelEx(&cfg, k_attend<false, HG, false, true>, s, d, q, K, V, n, out);
        }
        if (d.bf16) {
            if (d.defer_update)
                return launch_ex(d, k_attend<true, HG, false, false>, dim3(d.nCTA), dim3(kAttWarps * 32), bytes, st,
                                 s, d, q, K, V, n, out);
            return launch_ex(d, k_attend<true, HG, true, false>, dim3(d.nCTA), dim3(kAttWarps * 32), bytes, st, s,
                             d, q, K, V, n, out);
        }
        if (d.defer_update)
            return launch_ex(d, k_attend<false, HG, false, false>, dim3(d.nCTA), dim3(kAttWarps * 32), bytes, st, s,
                             d, q, K, V, n, out);
        return launch_ex(d, k_attend<false, HG, true, false>, dim3(d.nCTA), dim3(kAttWarps * 32), bytes, st, s, d, q,
                         K, V, n, out);
    });
}

cudaError_t launch_update(const DevState& s, const Dims& d, const void* K, int n, cudaStream_t st)
{
    return dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        // the lowest stream priority: where it shares the GPU with the next
        // step's kernels, those get the SMs first
        int lo = 0, hi = 0;
        priority_range(lo, hi);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(d.G);
        cfg.blockDim = dim3(kAttWarps * 32);
        cfg.dynamicSmemBytes = kUpdateSmem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributePriority;
        attr[0].val.priority = lo;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, k_update<HG>, s, d, K, n);
    });
}

cudaError_t launch_append_rows(const Dims& d, const void* knew, const void* vnew, void* K, void* V, int row,
                               cudaStream_t st)
{
    const int words = kD * (d.bf16 ? 2 : 4) / 4;
    k_append<<<d.B * d.Hkv, 64, 0, st>>>(static_cast<const uint32_t*>(knew), static_cast<const uint32_t*>(vnew),
                                         static_cast<uint32_t*>(K), static_cast<uint32_t*>(V), d.NM, row, words);
    return cudaGetLastError();
}

}  // namespace ckv
