// k_step.cu -- one CommunityKV decode step as a single persistent kernel on
// sm_100a.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 1 caption, step (3): score the query against the community
// centroids, retrieve the best communities up to the token budget, run exact
// attention over them plus the sink tokens, take the top-kappa keys as the
// new token's edges and assign it to a community in constant time; Table 1:
// O(sqrt(n) d) retrieval, O(d) update.
//
// The work of a step, for every graph g (one per (batch, KV head) or per
// (batch, query head)), is cut into items of one queue:
//   score item S(g, p)   centroids of communities [256p, 256p + 256) of g
//                        against g's summed query: an HBM stream of 1-D bulk
//                        copies (TMA engine) through per-warp rings;
//   attention item A(g,k) slice k of g's attended rows (sinks, kept members,
//                        new token): 16-byte cp.async gathers of K and V,
//                        both contractions on the tensor cores (mma.sync),
//                        an online softmax; leaves (m, l, o) per head.
// Every score item comes before every attention item, graph by graph.
// CTAs claim items in queue order from one atomic counter.  Two more pieces
// of work run where their inputs complete, on the CTA that completes them:
//   selection of g       after g's last score item: the exact budgeted
//                        top-C (histogram over the score range, radix
//                        refinement of a crowded boundary bin, exact rank of
//                        the boundary) and g's kept rows;
//   finish of g          after g's last attention item: merge the partials
//                        into the output, rank the kept members' summed
//                        attention weights into the top-kappa edges, vote
//                        the new token's community, update that centroid's
//                        running mean and append the token.
// An attention item waits (bounded) for its graph's selection.  All score
// items were claimed before any attention item by CTAs that are running
// (the launch is cooperative, so the grid is co-resident) and none of them
// waits for anything, so the wait ends.  Two CTAs share each SM: while one
// runs a latency-bound phase (the ramp-up of its rings, a selection, a
// finish) the other keeps the SM's loads in flight.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "ckv_internal.cuh"
#include "dev_async.cuh"
#include "warp_mma.cuh"

namespace ckv {

namespace {

constexpr int kW = 4;                           // warps of a streaming half
constexpr int kT = 32 * kW;                     // threads of a streaming half
constexpr int kWW = 2 * kW;                     // warps of a CTA (a worker uses them all)
constexpr int kWT = 32 * kWW;                   // threads of a CTA
constexpr int kSlot = 8192;                     // bytes of one pipeline slot
constexpr int kNSlot = 3;                       // slots per warp
constexpr int kRing = kW * kNSlot * kSlot;      // a half's rings, 96 KB
constexpr int kSubC = 16;                       // communities per score slot (8 KB)
constexpr int kSubPW = 4;                       // score slots per warp and item
constexpr int kCPI = kW * kSubPW * kSubC;       // communities per score item
constexpr int kRPI = 264;                       // target rows per attention item
constexpr int kMaxApi = 64;                     // attention items per graph, at most
constexpr int kTokW = 128;                      // row tokens a warp keeps at once
constexpr int kCoarseShift = 20;                // coarse bin of a score: the top 12 bits of its key
constexpr int kCoarse = 1 << (32 - kCoarseShift);

struct Misc {
    int item;                  // the half's next item (its thread 0 -> all)
    int flag;                  // a broadcast decision
    int abort[kW];             // per warp: a bounded wait ran out
    float sM[8], sL[8];        // finish: each head's max and 1 / sum
    int sflag[8];              // finish: the assignment's decisions
    int scan_i[4 * kWW];       // block scans (workers)
    unsigned long long red_k[2 * kWW];
};

// shared memory: two halves, each rings | row-token windows | mbarriers |
// Misc.  A worker CTA uses half 0's rings for its staging and half 1's
// rings for the selection's bitmaps and lists, with half 0's Misc.
constexpr int kHOffTok = kRing;
constexpr int kHOffBar = kHOffTok + kW * kTokW * 4;
constexpr int kHOffMisc = kHOffBar + ((kW * kNSlot * 8 + 127) / 128) * 128;
constexpr int kHalf = kHOffMisc + ((int)sizeof(Misc) + 127) / 128 * 128;
constexpr int kSmemBytes = 2 * kHalf;
constexpr int kOffX = kHalf;                    // the selection's bitmaps and lists (in half 1's rings)
constexpr int kXS = kRing;
static_assert(kSmemBytes <= 232448, "the CTA's shared memory must fit");

// barrier of the calling thread's half (4 warps): named barrier 1 + half
__device__ __forceinline__ void hsync()
{
    asm volatile("bar.sync %0, %1;" ::"r"(1 + (int)(threadIdx.x >> 7)), "r"(kT) : "memory");
}

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
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// selection key of a community: (order-preserving score bits, inverted id),
// larger = kept first; -0 and +0 are the same score
__device__ __forceinline__ unsigned long long sel_key(float sc, int c)
{
    return ((unsigned long long)ord_u(sc + 0.0f) << 32) | (unsigned long long)(~(uint32_t)c);
}

// 4-byte asynchronous copy global -> shared (for rows that are not 16-byte aligned)
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem) : "memory");
}

__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

// exclusive prefix sum over the CTA in thread order; *tot gets the total.
// Contains two barriers.
__device__ __forceinline__ int cta_excl(int x, int* scan, int* tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_incl(x, lane);
    __syncthreads();                       // scan[] free
    if (lane == 31) scan[warp] = incl;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kWW; ++w) {
        const int v = scan[w];
        before += (w < warp) ? v : 0;
        all += v;
    }
    *tot = all;
    return before + incl - x;
}

// bounded spin of thread 0 until a counter other CTAs advance reaches
// `target`; gives up at once when the step already failed
__device__ __forceinline__ bool wait_count(const unsigned* ctr, unsigned target, const int* err, unsigned polls)
{
    for (unsigned it = 0; it < polls; ++it) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
        if (*(volatile const int*)err) return false;
        __nanosleep(64);
    }
    return false;
}

// bounded wait for a bulk copy still in flight after a wait ran out, so
// that nothing lands after the item
__device__ __forceinline__ void mbar_drain(unsigned long long* b, unsigned parity)
{
    const uint32_t a = smem_u32(b);
    for (unsigned it = 0; it < kWaitLimit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return;
    }
}

__device__ __forceinline__ void set_flag(unsigned* flag)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(1u) : "memory");
}

// ------------------------------------------------------------ score item
// Warp w takes the item's slots w, w + 4, w + 8, w + 12 (16 communities,
// 8 KB each) through its own 3-slot ring: lane = 4 dims, the 16 partial dots
// reduced by a butterfly transpose so lane 2r holds community r's score.
// Every non-empty community also adds its size to bin (key >> 20) of the
// graph's coarse histogram in global memory (key: the order-preserving bits
// of its score, so the bins order the communities by score and need no
// score range), and each slot publishes its largest key: the selection
// starts from the histogram and looks only at slots that reach its
// boundary.
template <bool BF16>
__device__ __forceinline__ void score_item(const DevState& s, const Dims& d, const void* __restrict__ q, int g,
                                           int p, unsigned char* smem, unsigned long long* bars, unsigned& fills,
                                           Misc& mi)
{
    const int lane = threadIdx.x & 31, warp = (threadIdx.x >> 5) & (kW - 1);
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    unsigned char* ring = smem + warp * (kNSlot * kSlot);
    unsigned long long* fb = bars + warp * kNSlot;
    const int cbase = p * kCPI;
    int nsub = 0;   // this warp's slots in the item (a prefix of j = 0..kSubPW-1)
#pragma unroll
    for (int j = 0; j < kSubPW; ++j)
        if (cbase + kSubC * (warp + kW * j) < d.n_comm) nsub = j + 1;
    const float* mu_g = s.mu + (int64_t)g * d.Nc * kD;
    const uint64_t pol = l2_evict_first();   // the centroids are streamed once per step
    auto issue = [&](int j) {
        const int c0 = cbase + kSubC * (warp + kW * j);
        const int rows = min(kSubC, d.n_comm - c0);
        const int slot = (int)((fills + j) % kNSlot);
        mbar_expect_tx(&fb[slot], rows * kD * 4);
        bulk_g2s_hint(ring + slot * kSlot, mu_g + (int64_t)c0 * kD, rows * kD * 4, &fb[slot], pol);
    };
    if (lane == 0) {
        fence_proxy_async();   // the ring's earlier generic reads before the copies' writes
        for (int j = 0; j < min(nsub, kNSlot); ++j) issue(j);
    }
    // the graph's query heads summed, this lane's 4 dims
    float qs[4] = {0.f, 0.f, 0.f, 0.f};
    for (int h = 0; h < d.HG; ++h) {
        const int64_t base = ((int64_t)b * d.Hq + h0 + h) * kD + 4 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) qs[k] += elem<BF16>(q, base + k);
    }
    unsigned* hist = s.shist + (int64_t)g * kCoarse;
    int j = 0;
    for (; j < nsub; ++j) {
        const int c0 = cbase + kSubC * (warp + kW * j);
        const int rows = min(kSubC, d.n_comm - c0);
        const int row = lane >> 1;
        const int64_t gi = (int64_t)g * d.Nc + c0 + row;
        const int sz = (row < rows) ? s.csize[gi] : 0;
        const unsigned f = fills + j;
        const int slot = (int)(f % kNSlot);
        if (!mbar_wait(&fb[slot], (f / kNSlot) & 1, (volatile int*)&mi.abort[warp])) break;
        const float4* mu = reinterpret_cast<const float4*>(ring + slot * kSlot);
        float part[kSubC];
#pragma unroll
        for (int r = 0; r < kSubC; ++r) {
            const float4 v = (r < rows) ? mu[r * (kD / 4) + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
            part[r] = fmaf(qs[3], v.w, fmaf(qs[2], v.z, fmaf(qs[1], v.y, qs[0] * v.x)));
        }
        __syncwarp();
        if (lane == 0 && j + kNSlot < nsub) {
            fence_proxy_async();
            issue(j + kNSlot);
        }
        const float v = transpose_reduce<kSubC>(part, lane);   // lane 2r: community c0 + r
        const bool live = (lane & 1) == 0 && row < rows && sz > 0;
        if ((lane & 1) == 0 && row < rows) {
            s.score[gi] = (sz > 0) ? v : -INFINITY;
            if (sz > 0) atomicAdd(hist + (ord_u(v + 0.0f) >> kCoarseShift), (unsigned)sz);
        }
        // the slot's largest key (0: no non-empty community), for the selection
        const unsigned smk = __reduce_max_sync(kFull, live ? ord_u(v + 0.0f) : 0u);
        if (lane == 0) s.smax[(int64_t)g * d.nsu + c0 / kSubC] = smk;
    }
    if (j < nsub) {
        // a copy never completed: report it, and wait (bounded) for the
        // copies still in flight so that none lands after the item
        if (lane == 0) set_error(s.err, CKV_ERR_TIMEOUT);
        for (int jj = j; jj < min(nsub, j + kNSlot); ++jj) {
            const unsigned f = fills + jj;
            mbar_drain(&fb[f % kNSlot], (f / kNSlot) & 1);
        }
    }
    fills += nsub;
}

// ------------------------------------------------------------- selection
// Exact budgeted top-C of graph g by the whole CTA, in (score desc, id asc)
// order: keep the longest prefix whose sizes sum to at most the budget, at
// least one community.  Two dependent rounds of global loads: the scores,
// sizes and segment starts staged into the rings' shared memory by
// cp.async together with the coarse histogram (into registers), then the
// kept members' pool entries.  The loops give each thread several
// independent chains (one warp per scheduler leaves no other latency
// hiding).
constexpr int kSelCache = 8192;    // communities staged in shared memory (the rest read from L2)
constexpr int kSelB = 1024;        // bins of a refinement pass
constexpr int kSelCap = 256;       // boundary communities ranked exactly
constexpr int kSelCapW = 64;       // boundary communities each warp lists
constexpr int kKeepCap = (kSelCache - 1) / 3;   // kept-list entries in the scores' bytes

struct SelSmem {                   // in the rings
    float cs[kSelCache];           // scores, then the kept list: ids | row starts | segment starts
    int cz[kSelCache];             // sizes, then the row -> kept-community map (16-bit)
    int co[kSelCache];             // segment starts
};
static_assert(sizeof(SelSmem) <= kRing, "selection staging must fit the rings");
struct SelX {                      // in the region after the rings
    int hist[kSelB];
    unsigned long long wkey[kWW * kSelCapW];    // boundary candidates: per warp, or (refinement) flat
    int ww[kWW * kSelCapW];
    unsigned keep[kMaxCommunities / 32];       // kept bitmap
    unsigned cand[kMaxCommunities / 32];       // still-a-candidate bitmap
    int nw[kWW];                                // candidates each warp listed
    int n_cand, b_bin, b_above;
};
static_assert(kWW * kSelCapW >= kSelCap, "the flat candidate list must fit");
static_assert(sizeof(SelX) <= kXS, "the selection's lists must fit half 1's rings");

// Boundary of a histogram of NB bins held top-first, PB = NB / kWT bins per
// thread (thread t: bins NB-1-PB t .. NB-PB(t+1)): the bin where `above`
// plus the sizes summed from the top first exceeds the budget, and the sizes
// above it, set only when above plus the whole histogram exceeds the
// budget.  Returns the histogram's total.
template <int PB>
__device__ __forceinline__ int sel_boundary(const int (&loc)[PB], SelX& x, Misc& mi, int above, int budget)
{
    constexpr int NB = PB * kWT;
    const int t = threadIdx.x;
    int tsum = 0;
#pragma unroll
    for (int k = 0; k < PB; ++k) tsum += loc[k];
    int tot;
    int acc = above + cta_excl(tsum, mi.scan_i, &tot);
#pragma unroll
    for (int k = 0; k < PB; ++k) {
        if (acc <= budget && acc + loc[k] > budget) {
            x.b_bin = NB - 1 - (PB * t + k);
            x.b_above = acc;
        }
        acc += loc[k];
    }
    __syncthreads();
    return tot;   // the histogram's total
}

__device__ void select_graph(const DevState& s, const Dims& d, int g, SelSmem& sm, SelX& x, Misc& mi)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const int Nc = d.n_comm, budget = d.budget;
    const float* gsc = s.score + (int64_t)g * d.Nc;
    const int32_t* gsz = s.csize + (int64_t)g * d.Nc;
    const int32_t* gco = s.coff + (int64_t)g * d.Nc;
    const int32_t* gpool = s.pool + (int64_t)g * d.P;
    auto bin_of = [](float v) { return (int)(ord_u(v + 0.0f) >> kCoarseShift); };
    const int NWd = (Nc + 31) / 32;
    const int NS = min(Nc, kSelCache);            // staged communities
    // ---- round 1: the coarse histogram (this thread's 32 bins, top first;
    // cleared for the next step) and the staged scores, sizes and segment
    // starts (16-byte copies when each graph's rows are 16-byte aligned)
    constexpr int PB = kCoarse / kWT;
    int loc[PB];
    {
        uint4* gh = reinterpret_cast<uint4*>(s.shist + (int64_t)g * kCoarse) + (kCoarse - PB * (tid + 1)) / 4;
        uint4 h4[PB / 4];
#pragma unroll
        for (int i = 0; i < PB / 4; ++i) h4[i] = __ldcg(gh + i);
        if ((d.Nc & 3) == 0) {
            const int nch = (NS + 3) / 4;
            for (int i = tid; i < nch; i += kWT) {
                cp_async16(sm.cs + 4 * i, gsc + 4 * i);
                cp_async16(sm.cz + 4 * i, gsz + 4 * i);
                cp_async16(sm.co + 4 * i, gco + 4 * i);
            }
        } else {
            for (int c = tid; c < NS; c += kWT) {
                cp_async4(sm.cs + c, gsc + c);
                cp_async4(sm.cz + c, gsz + c);
                cp_async4(sm.co + c, gco + c);
            }
        }
        cp_async_commit();
#pragma unroll
        for (int i = 0; i < PB / 4; ++i) {
            gh[i] = make_uint4(0u, 0u, 0u, 0u);
            // h4[i] holds bins base + 4i .. 4i+3; loc[k] is bin NB-1-(PB t + k)
            loc[PB - 1 - 4 * i] = (int)h4[i].x;
            loc[PB - 2 - 4 * i] = (int)h4[i].y;
            loc[PB - 3 - 4 * i] = (int)h4[i].z;
            loc[PB - 4 - 4 * i] = (int)h4[i].w;
        }
    }
    // the slots' largest keys (this thread: slots tid + kWT j)
    constexpr int SJ = (kMaxCommunities / kSubC + kWT - 1) / kWT;
    static_assert(SJ * kWW <= 4 * kWW && kMaxCommunities / kSubC <= kSelB, "live-slot scan and list sizes");
    const int NSU = (Nc + kSubC - 1) / kSubC;
    unsigned smk[SJ];
#pragma unroll
    for (int j = 0; j < SJ; ++j) {
        const int su = tid + kWT * j;
        smk[j] = (su < NSU) ? __ldcg(s.smax + (int64_t)g * d.nsu + su) : 0u;
    }
    for (int i = tid; i < NWd; i += kWT) { x.cand[i] = 0u; x.keep[i] = 0u; }
    // ---- the boundary bin, and from the same scan the total size: when
    // everything fits there is no boundary
    const int wsum = sel_boundary<PB>(loc, x, mi, 0, budget);
    const bool all = wsum <= budget;
    int above = 0, b0 = -1;
    if (!all) {
        b0 = x.b_bin;
        above = x.b_above;
    }
    cp_async_wait<0>();
    __syncthreads();
    auto get = [&](int c, float& v, int& w) {
        if (c < kSelCache) { v = sm.cs[c]; w = sm.cz[c]; }
        else { v = __ldcg(gsc + c); w = gsz[c]; }
    };
    // ---- the live slots: those whose largest key reaches the boundary bin
    // (with everything kept, every slot with a non-empty community), listed
    // in ascending order (slot tid + kWT j goes j-major, warp by warp)
    int* lsl = reinterpret_cast<int*>(x.hist);   // the live slots (the refinement's bins come later)
    {
        unsigned bl[SJ];
        int cntw = 0;
#pragma unroll
        for (int j = 0; j < SJ; ++j) {
            const bool lv = smk[j] != 0u && (all || (int)(smk[j] >> kCoarseShift) >= b0);
            bl[j] = __ballot_sync(kFull, lv);
            if (lane == 0) mi.scan_i[j * kWW + warp] = __popc(bl[j]);
            cntw += __popc(bl[j]);
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < SJ; ++j) {
            int base = 0;
            for (int q = 0; q < j * kWW + warp; ++q) base += mi.scan_i[q];
            if ((bl[j] >> lane) & 1u) lsl[base + __popc(bl[j] & lt)] = tid + kWT * j;
        }
        int nl = 0;
        for (int q = 0; q < SJ * kWW; ++q) nl += mi.scan_i[q];
        __syncthreads();
        if (tid == 0) x.n_cand = nl;   // (the live count, kept until the ranking resets it)
        __syncthreads();
    }
    const int NLV = x.n_cand;
    // ---- classify the live slots, one 16-byte chunk (4 communities) a
    // thread: above the boundary bin kept, in it a candidate.  The 4 chunks
    // of a slot sit in 4 consecutive lanes, which assemble its 16 bits; each
    // warp lists its candidates by ballot prefix.
    int ncw = 0;   // candidates this warp has met (uniform in the warp)
    for (int t0 = 0; t0 < 4 * NLV; t0 += kWT) {
        const int t = t0 + tid;
        const bool on = t < 4 * NLV;
        const int su = on ? lsl[t >> 2] : 0, qc = t & 3;
        const int i = 4 * su + qc;   // chunk
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        int4 w = make_int4(0, 0, 0, 0);
        if (on) {
            if (4 * i < kSelCache) {
                v = reinterpret_cast<const float4*>(sm.cs)[i];
                w = reinterpret_cast<const int4*>(sm.cz)[i];
            } else {   // beyond the staged communities: from L2
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * i + e;
                    (&v.x)[e] = (c < Nc) ? __ldcg(gsc + c) : 0.f;
                    (&w.x)[e] = (c < Nc) ? gsz[c] : 0;
                }
            }
        }
        unsigned kb = 0u, cb = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int bn = ((&w.x)[e] <= 0 || 4 * i + e >= Nc) ? -1 : all ? kCoarse : bin_of((&v.x)[e]);
            kb |= (bn > b0 ? 1u : 0u) << e;
            cb |= (bn == b0 ? 1u : 0u) << e;
        }
        unsigned kw = kb << (4 * qc), cw = cb << (4 * qc);
        kw |= __shfl_xor_sync(kFull, kw, 1);
        cw |= __shfl_xor_sync(kFull, cw, 1);
        kw |= __shfl_xor_sync(kFull, kw, 2);
        cw |= __shfl_xor_sync(kFull, cw, 2);
        if (on && qc == 0) {
            if (kw) atomicOr(&x.keep[su >> 1], kw << (16 * (su & 1)));
            if (cw) atomicOr(&x.cand[su >> 1], cw << (16 * (su & 1)));
        }
        if (__any_sync(kFull, cb != 0u)) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const unsigned me = __ballot_sync(kFull, (cb >> e) & 1u);
                if ((cb >> e) & 1u) {
                    const int slot = ncw + __popc(me & lt);
                    if (slot < kSelCapW) {
                        x.wkey[warp * kSelCapW + slot] = sel_key((&v.x)[e], 4 * i + e);
                        x.ww[warp * kSelCapW + slot] = (&w.x)[e];
                    }
                }
                ncw += __popc(me);
            }
        }
    }
    if (lane == 0) x.nw[warp] = ncw;
    __syncthreads();
    if (!all) {
        int nwl[kWW], m = 0;
        bool over = false;
#pragma unroll
        for (int w = 0; w < kWW; ++w) {
            nwl[w] = x.nw[w];
            m += nwl[w];
            over |= nwl[w] > kSelCapW;
        }
        if (over || m > kSelCap) {
            // ---- a crowded boundary bin (ties or a narrow score range):
            // radix passes over the candidates' keys, 10 bits below their
            // highest differing bit each time; the final candidates end in
            // the flat list
            for (int w = 0; w < kWW; ++w) nwl[w] = 0;
            for (int pass = 0; m > kSelCap || over; ++pass) {
                over = false;
                if (pass == 8) {   // 64 key bits take at most 7 passes: unreachable
                    if (tid == 0) set_error(s.err, CKV_ERR_STATE);
                    return;
                }
                unsigned long long kmn = ~0ull, kmx = 0ull;
                for (int i = tid; i < NWd; i += kWT) {
                    unsigned bits = x.cand[i];
                    while (bits) {
                        const int c = 32 * i + __ffs(bits) - 1;
                        bits &= bits - 1u;
                        float v;
                        int w;
                        get(c, v, w);
                        const unsigned long long k = sel_key(v, c);
                        kmn = min(kmn, k);
                        kmx = max(kmx, k);
                    }
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    kmn = min(kmn, __shfl_xor_sync(kFull, kmn, o));
                    kmx = max(kmx, __shfl_xor_sync(kFull, kmx, o));
                }
                if (lane == 0) { mi.red_k[warp] = kmn; mi.red_k[kWW + warp] = kmx; }
                for (int i = tid; i < kSelB; i += kWT) x.hist[i] = 0;
                __syncthreads();
                kmn = mi.red_k[0];
                kmx = mi.red_k[kWW];
#pragma unroll
                for (int w = 1; w < kWW; ++w) {
                    kmn = min(kmn, mi.red_k[w]);
                    kmx = max(kmx, mi.red_k[kWW + w]);
                }
                const int shift = max(0, 63 - __clzll((long long)(kmn ^ kmx)) - 9);
                auto digit = [&](unsigned long long k) { return (int)((k >> shift) & (unsigned long long)(kSelB - 1)); };
                for (int i = tid; i < NWd; i += kWT) {
                    unsigned bits = x.cand[i];
                    while (bits) {
                        const int c = 32 * i + __ffs(bits) - 1;
                        bits &= bits - 1u;
                        float v;
                        int w;
                        get(c, v, w);
                        atomicAdd(&x.hist[digit(sel_key(v, c))], w);
                    }
                }
                __syncthreads();
                {
                    constexpr int RB = kSelB / kWT;
                    int rl[RB];
#pragma unroll
                    for (int k = 0; k < RB; ++k) rl[k] = x.hist[kSelB - 1 - (RB * tid + k)];
                    sel_boundary<RB>(rl, x, mi, above, budget);
                }
                const int d0 = x.b_bin;
                above = x.b_above;
                if (tid == 0) x.n_cand = 0;
                __syncthreads();
                for (int i = tid; i < NWd; i += kWT) {
                    unsigned bits = x.cand[i], nc = 0u, nk = 0u;
                    while (bits) {
                        const int bit = __ffs(bits) - 1;
                        const int c = 32 * i + bit;
                        bits &= bits - 1u;
                        float v;
                        int w;
                        get(c, v, w);
                        const unsigned long long k = sel_key(v, c);
                        const int dg = digit(k);
                        if (dg > d0) nk |= 1u << bit;
                        else if (dg == d0) {
                            nc |= 1u << bit;
                            const int slot = atomicAdd(&x.n_cand, 1);
                            if (slot < kSelCap) { x.wkey[slot] = k; x.ww[slot] = w; }
                        }
                    }
                    x.cand[i] = nc;
                    x.keep[i] |= nk;
                }
                __syncthreads();
                m = x.n_cand;
            }
            nwl[0] = m;   // one flat list
        }
        // ---- the boundary communities ranked exactly: each sums the sizes
        // of the better ones and is kept iff the sizes through it fit
        // the lists made one (in the refinement bins' bytes), then thread i
        // ranks candidate i against all of them
        unsigned long long* fk = reinterpret_cast<unsigned long long*>(x.hist);   // [kSelCap]
        int* fw = reinterpret_cast<int*>(fk + kSelCap);                          // [kSelCap]
        static_assert(kSelCap * 12 <= (int)sizeof(x.hist), "the flat candidates must fit the bins");
        {
            int base = 0;
#pragma unroll
            for (int l = 0; l < kWW; ++l) base += (l < warp) ? nwl[l] : 0;
            for (int t = lane; t < nwl[warp]; t += 32) {
                fk[base + t] = x.wkey[warp * kSelCapW + t];
                fw[base + t] = x.ww[warp * kSelCapW + t];
            }
        }
        __syncthreads();
        for (int i = tid; i < m; i += kWT) {
            const unsigned long long k = fk[i];
            const int w = fw[i];
            int bp[4] = {0, 0, 0, 0};
            int t = 0;
            for (; t + 4 <= m; t += 4) {
#pragma unroll
                for (int q = 0; q < 4; ++q) bp[q] += (fk[t + q] > k) ? fw[t + q] : 0;
            }
            for (; t < m; ++t) bp[0] += (fk[t] > k) ? fw[t] : 0;
            const int bpre = bp[0] + bp[1] + bp[2] + bp[3];
            if (above + bpre + w <= budget || (above == 0 && bpre == 0)) {
                const int c = (int)~(uint32_t)(k & 0xffffffffull);
                atomicOr(&x.keep[c >> 5], 1u << (c & 31));
            }
        }
        __syncthreads();
    }
    // ---- the kept ids in ascending order with their row starts: thread t
    // owns the bitmap words [t WPT, (t + 1) WPT); one scan of (count, sizes)
    auto size_of = [&](int c) { return (c < kSelCache) ? sm.cz[c] : gsz[c]; };
    auto off_of = [&](int c) { return (c < kSelCache) ? sm.co[c] : gco[c]; };
    const int WPT = (NWd + kWT - 1) / kWT;
    const int wa = min(NWd, tid * WPT), wb = min(NWd, (tid + 1) * WPT);
    int cnt = 0, tsz = 0;
    for (int i = wa; i < wb; ++i) {
        unsigned bits = x.keep[i];
        cnt += __popc(bits);
        while (bits) {
            tsz += size_of(32 * i + __ffs(bits) - 1);
            bits &= bits - 1u;
        }
    }
    int C, T;
    int pos, row;
    {
        const int ic = warp_incl(cnt, lane), is = warp_incl(tsz, lane);
        __syncthreads();
        if (lane == 31) { mi.scan_i[warp] = ic; mi.scan_i[kWW + warp] = is; }
        __syncthreads();
        int bc = 0, bs = 0;
        C = 0;
        T = 0;
#pragma unroll
        for (int w = 0; w < kWW; ++w) {
            const int vc = mi.scan_i[w], vs = mi.scan_i[kWW + w];
            bc += (w < warp) ? vc : 0;
            bs += (w < warp) ? vs : 0;
            C += vc;
            T += vs;
        }
        pos = bc + ic - cnt;
        row = bs + is - tsz;
    }
    // the kept list (ids | row starts | segment starts) in the scores'
    // bytes when it fits (the scores are no longer read), else in the
    // graph's global scratch; the same code through generic pointers.  The
    // finish reads it as kinfo[k] = (id, row start, size, segment start).
    const bool in_smem = C <= kKeepCap;
    int* kc = in_smem ? reinterpret_cast<int*>(sm.cs) : s.sel_row + (int64_t)g * (d.Nc + 1) * 3;
    int* krow = kc + (in_smem ? kKeepCap : d.Nc + 1);
    int* koff = krow + (in_smem ? kKeepCap + 1 : d.Nc + 1);
    int32_t* gsel = s.sel + (int64_t)g * d.Nc;
    int4* kinfo = reinterpret_cast<int4*>(s.kinfo) + (int64_t)g * d.Nc;
    for (int i = wa; i < wb; ++i) {
        unsigned bits = x.keep[i];
        while (bits) {
            const int c = 32 * i + __ffs(bits) - 1;
            bits &= bits - 1u;
            const int sz = size_of(c), o = off_of(c);
            kc[pos] = c;
            krow[pos] = row;
            koff[pos] = o;
            gsel[pos] = c;
            kinfo[pos] = make_int4(c, row, sz, o);
            ++pos;
            row += sz;
        }
    }
    if (tid == 0) {
        krow[C] = T;
        int32_t* meta = s.meta + (int64_t)g * M_COUNT;
        meta[M_C] = C;
        meta[M_T] = T;
        meta[M_ROWS] = d.S + T + 1;
    }
    __syncthreads();   // the kept list is complete
    // ---- round 2: the kept members' rows.  Warp w copies kept communities
    // w, w + 8, ... (lane = member), 32 communities' loads in flight.
    int32_t* rtok = s.rtok + (int64_t)g * d.rtok_stride;
    constexpr int KU = 32;
    for (int k0 = warp; k0 < C; k0 += KU * kWW) {
        int rs[KU], sz[KU], of[KU], tk[KU];
#pragma unroll
        for (int u = 0; u < KU; ++u) {
            const int k = k0 + u * kWW;
            const bool on = k < C;
            rs[u] = on ? krow[k] : 0;
            sz[u] = on ? krow[k + 1] - rs[u] : 0;
            of[u] = on ? koff[k] : 0;
            if (of[u] < 0 || (int64_t)of[u] + sz[u] > d.P) sz[u] = -1;   // a corrupt segment: read nothing
        }
#pragma unroll
        for (int u = 0; u < KU; ++u) tk[u] = (lane < sz[u]) ? gpool[of[u] + lane] : 0;
#pragma unroll
        for (int u = 0; u < KU; ++u) {
            if (lane < sz[u]) rtok[rs[u] + lane] = tk[u];
            if (sz[u] < 0 && lane == 0) set_error(s.err, CKV_ERR_STATE);
        }
#pragma unroll
        for (int u = 0; u < KU; ++u)   // communities longer than a warp: the rest
            for (int r = 32 + lane; r < sz[u]; r += 32) rtok[rs[u] + r] = gpool[of[u] + r];
    }
}

// ---------------------------------------------------------- attention item
template <bool BF16, int HG>
struct AttL {
    static constexpr int NB = BF16 ? 16 : 4;          // rows per warp batch
    static constexpr int RB = kD * (BF16 ? 2 : 4);    // bytes per K or V row
    static constexpr int BATCH = NB * 2 * RB;         // K rows, then V rows
    static constexpr int RSTR = kD + 4;               // reduction row: acc[D], m, l, pad
    static_assert(BATCH <= kSlot, "a batch fills at most one slot");
    static_assert(kW * HG * RSTR * 4 <= kRing, "the reduction must fit the rings");
};

// Rows of one warp: [a0, a1) in the graph's row numbering (sinks, kept
// members, the new token).
struct WarpRows {
    const char* Kb;          // this (batch, KV head)'s K cache
    const char* Vb;
    const int32_t* rtok;     // token of each kept-member row
    float* zrow;             // logits of the kept members, [row][HG] (null: not kept)
    int* err;                // the step's error word
    int a0, a1, S, T, R, t_new;
};

__device__ __forceinline__ int row_token(const WarpRows& a, int r)
{
    if (r < a.S) return r;
    if (r == a.R - 1) return a.t_new;
    return __ldcg(a.rtok + (r - a.S));
}

// tokens of rows r .. r + kTokW - 1 of this warp into its window
// (a token outside [0, n) -- a corrupt row list -- sets the error word and
// gathers row 0 instead, so no address outside the cache is formed)
__device__ __forceinline__ void tokens_from(const WarpRows& a, int r, int* tokw, int lane)
{
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kTokW / 32; ++i) {
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

// bf16 rows on the tensor cores (mma.sync m16n8k16, fp32 accumulate):
// S^T = K_tile . Q^T with the graph's heads as the 8 columns, then
// O^T += V_tile^T . P^T with P split into bf16 high and low parts (two MMAs,
// ~16 bits).  Rows sit in shared memory with their 16-byte chunks
// XOR-swizzled by (row mod 8), so every ldmatrix is conflict-free.  Leaves
// the warp's (acc, m, l) per head in red[warp][h][RSTR] (after a CTA
// barrier: red overlays the rings).
template <int HG>
__device__ __forceinline__ void warp_rows_mma(const WarpRows& a, const uint32_t* __restrict__ q2,
                                              unsigned char* wbuf, int* tokw, float* red)
{
    using L = AttL<true, HG>;
    constexpr int NB = L::NB;
    const int lane = threadIdx.x & 31, warp = (threadIdx.x >> 5) & (kW - 1);
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
    int tok_base = -kTokW;
    auto issue = [&](int bb) {
        if (bb < nb) {
            const uint32_t dst = smem_u32(wbuf + (bb % kNSlot) * kSlot);
            const int rbase = a.a0 + bb * NB;
            if (rbase + NB > tok_base + kTokW) {
                tokens_from(a, rbase, tokw, lane);
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
        cp_async_wait<kNSlot - 1>();
        __syncwarp();
        const uint32_t kt = smem_u32(wbuf + (bb % kNSlot) * kSlot), vt = kt + NB * 256;
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
        if (a.zrow && h0ok) {   // the kept members' logits, for the edge ranking
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
        for (int jj = 0; jj < 2; ++jj) {
            float t = fmaxf(z[jj], z[2 + jj]);
            t = fmaxf(t, __shfl_xor_sync(kFull, t, 4));
            t = fmaxf(t, __shfl_xor_sync(kFull, t, 8));
            t = fmaxf(t, __shfl_xor_sync(kFull, t, 16));
            const float mn = fmaxf(m[jj], t);
            const float al = (m[jj] == -INFINITY) ? 0.f : __expf(m[jj] - mn);
            p[jj] = (z[jj] == -INFINITY) ? 0.f : __expf(z[jj] - mn);
            p[2 + jj] = (z[2 + jj] == -INFINITY) ? 0.f : __expf(z[2 + jj] - mn);
            l[jj] = fmaf(l[jj], al, p[jj] + p[2 + jj]);
            m[jj] = mn;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                acc[mt][jj] *= al;
                acc[mt][2 + jj] *= al;
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
    for (int jj = 0; jj < 2; ++jj) {
        l[jj] += __shfl_xor_sync(kFull, l[jj], 4);
        l[jj] += __shfl_xor_sync(kFull, l[jj], 8);
        l[jj] += __shfl_xor_sync(kFull, l[jj], 16);
    }
    hsync();   // every warp of the half is done with its pipeline: red overlays them
    float* rw = red + warp * HG * L::RSTR;
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
        const int h = 2 * tig + jj;
        if (h < HG) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                rw[h * L::RSTR + 16 * mt + gid] = acc[mt][jj];
                rw[h * L::RSTR + 16 * mt + gid + 8] = acc[mt][2 + jj];
            }
            if (gid == 0) { rw[h * L::RSTR + kD] = m[jj]; rw[h * L::RSTR + kD + 1] = l[jj]; }
        }
    }
}

// fp32 rows on the CUDA cores: 4-row batches, lane = 4 dims, the row dots
// reduced by a butterfly; the z / p exchange sits after the batch in its slot
template <int HG>
__device__ __forceinline__ void warp_rows_fma(const WarpRows& a, const float* __restrict__ qg, unsigned char* wbuf,
                                              int* tokw, float* red)
{
    using L = AttL<false, HG>;
    constexpr int NB = L::NB, RB = L::RB, NV = 4 * HG;
    static_assert(L::BATCH + NB * HG * 4 <= kSlot, "batch and exchange must fit a slot");
    const int lane = threadIdx.x & 31, warp = (threadIdx.x >> 5) & (kW - 1);
    float qv[HG][4];
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) qv[h][jj] = qg[h * kD + 4 * lane + jj];
    const int nb = (a.a1 - a.a0 + NB - 1) / NB;
    int tok_base = -kTokW;
    auto issue = [&](int bb) {
        if (bb < nb) {
            unsigned char* dst = wbuf + (bb % kNSlot) * kSlot;
            const int rbase = a.a0 + bb * NB;
            if (rbase + NB > tok_base + kTokW) {
                tokens_from(a, rbase, tokw, lane);
                tok_base = rbase;
            }
            constexpr int NCH = RB / 16;   // 16-byte chunks per row
#pragma unroll
            for (int jj = 0; jj < NB * NCH / 32; ++jj) {
                const int e = jj * 32 + lane;
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
        cp_async_wait<kNSlot - 1>();
        __syncwarp();
        unsigned char* slot = wbuf + (bb % kNSlot) * kSlot;
        const unsigned char* kt = slot;
        const unsigned char* vt = kt + NB * RB;
        float* pz = reinterpret_cast<float*>(slot + L::BATCH);
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
                if (a.zrow && rr < rows_in && r >= a.S && r < a.S + a.T) a.zrow[(int64_t)r * HG + idx % HG] = z;
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
    hsync();   // every warp of the half is done with its pipeline: red overlays them
#pragma unroll
    for (int h = 0; h < HG; ++h) {
        float* rw = red + (warp * HG + h) * L::RSTR;
        *reinterpret_cast<float4*>(rw + 4 * lane) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
        if (lane == 0) { rw[kD] = m_run[h]; rw[kD + 1] = l_run[h]; }
    }
}

// ------------------------------------------------------------------ edges
// Edge ranking of one graph by the whole CTA.  The kept members go by in
// rounds of FR rows per thread (r holds round 0 on entry); the running top
// kappa (w desc, token asc) sits in shared memory and joins every round as
// extra entries of threads 0 .. kappa-1.  Per round: tau = the kappa-th
// best of each warp's lane-bests is a lower bound of the answer (that warp
// holds kappa keys at least as good), so only entries >= the largest such
// tau -- at most kWW * kappa * (FR + 1), the capacity of ck / cx -- are
// compacted and ranked by counting.  The list keeps each entry's kept-member
// row for the assignment.
constexpr int kFinMaxRows = 16;                                 // rows per thread and round
constexpr int kFinCand = kWW * kMaxKappa * (kFinMaxRows + 1);    // compacted entries, at most

// An edge weight (a sum of at most 8 probabilities, so below 8, with every
// vote's total below 8 too) as fixed point in units of 2^-59: exact for
// weights of at least 2^-36, and sums of them exact.  The votes are then
// exact sums; a double-precision sum in any order differs from them by at
// most a few units of 2^-53 relative.
__device__ __forceinline__ unsigned long long weight_fix(float w)
{
    const uint32_t b = __float_as_uint(w);
    const int e = (int)((b >> 23) & 255u);
    if (e == 0) return 0ull;                         // zero (and subnormals, far below 2^-36)
    const unsigned long long m = (unsigned long long)((b & 0x7fffffu) | 0x800000u);
    const int sh = e - 127 - 23 + 59;                // value = m 2^(e - 127 - 23)
    return sh >= 0 ? (m << sh) : (sh > -64 ? (m >> -sh) : 0ull);
}

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
    unsigned long long wk[kWW];                   // each warp's tau
    int m;                                       // compacted entries
};
// the finish's shared memory: half 0's rings hold the staged logits,
// tokens and kept-community table (when they fit); half 1's rings the item
// weights, the edge scratch and the compaction slots (keys, then rows)
constexpr int kFinWgt = 0;                       // [nc][HG] floats, nc <= kMaxApi
constexpr int kFinScr = kMaxApi * 8 * 4;
constexpr int kFinCk = kFinScr + ((int)sizeof(EdgeScratch) + 127) / 128 * 128;
static_assert(kFinCk + kFinCand * 12 <= kRing, "edge scratch must fit the rings");

template <int HG>
struct EdgeRows {
    static constexpr int FR = (64 / HG < kFinMaxRows) ? 64 / HG : kFinMaxRows;   // rows per thread and round
    float z[FR][HG];
    int t[FR];
};

// where a graph's kept-member logits (row j at z[j * HG]), tokens (t[j])
// and kept-community table (ki[k] = id, row start, size, segment start) are
// read: staged in shared memory, or in global memory (read through L2:
// other CTAs wrote them during this launch)
struct EdgeSrc {
    const float* z;
    const int32_t* t;
    const int4* ki;
    bool staged;
};

// HG logits of one kept-member row (16-, 8- or 4-byte aligned by HG)
template <int HG, bool GLOBAL>
__device__ __forceinline__ void load_logits(const float* p, float (&z)[HG])
{
    if constexpr (HG % 4 == 0) {
#pragma unroll
        for (int h = 0; h < HG; h += 4) {
            const float4 v = GLOBAL ? __ldcg(reinterpret_cast<const float4*>(p + h)) : *reinterpret_cast<const float4*>(p + h);
            z[h] = v.x; z[h + 1] = v.y; z[h + 2] = v.z; z[h + 3] = v.w;
        }
    } else if constexpr (HG == 2) {
        const float2 v = GLOBAL ? __ldcg(reinterpret_cast<const float2*>(p)) : *reinterpret_cast<const float2*>(p);
        z[0] = v.x; z[1] = v.y;
    } else {
        z[0] = GLOBAL ? __ldcg(p) : *p;
    }
}

// one round's logits and tokens of this thread: rows j0 + tid + u * kWT
template <int HG>
__device__ __forceinline__ void edges_load(const EdgeSrc& src, int T, int j0, EdgeRows<HG>& r)
{
#pragma unroll
    for (int u = 0; u < EdgeRows<HG>::FR; ++u) {
        const int j = j0 + threadIdx.x + u * kWT;
        r.t[u] = 0;
        if (j < T) {
            if (src.staged) {
                load_logits<HG, false>(src.z + (int64_t)j * HG, r.z[u]);
                r.t[u] = src.t[j];
            } else {
                load_logits<HG, true>(src.z + (int64_t)j * HG, r.z[u]);
                r.t[u] = __ldcg(src.t + j);
            }
        }
    }
}

template <int HG>
__device__ __forceinline__ void cta_edges(const Dims& d, const EdgeSrc& src, int T, const float* sM,
                                          const float* sL, EdgeScratch& e, unsigned long long* ck, int* cx,
                                          EdgeRows<HG>& r)
{
    constexpr int FR = EdgeRows<HG>::FR;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kappa = d.kappa;
    const int cap = kWW * kappa * (FR + 1);
    if (tid < kMaxKappa) { e.lk[tid] = 0ull; e.lx[tid] = -1; }
    for (int j0 = 0; j0 < max(T, 1); j0 += FR * kWT) {
        if (j0 > 0) edges_load<HG>(src, T, j0, r);
        unsigned long long key[FR + 1];
#pragma unroll
        for (int u = 0; u < FR; ++u) {
            const int j = j0 + tid + u * kWT;
            float sw = 0.f;
#pragma unroll
            for (int h = 0; h < HG; ++h) sw += __expf(r.z[u][h] - sM[h]) * sL[h];
            key[u] = (j < T) ? edge_key(sw, r.t[u]) : 0ull;
        }
        if (j0 > 0) __syncthreads();   // the running list is complete (round 0: each thread cleared its own)
        key[FR] = (tid < kappa) ? e.lk[tid] : 0ull;
        const int xl = (tid < kappa) ? e.lx[tid] : -1;
        unsigned long long best = 0ull;
#pragma unroll
        for (int u = 0; u <= FR; ++u) best = max(best, key[u]);
        int rank = 0;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) rank += (__shfl_sync(kFull, best, i) > best) ? 1 : 0;
        const unsigned tb = __ballot_sync(kFull, best != 0ull && rank == kappa - 1);
        const unsigned long long tw = tb ? __shfl_sync(kFull, best, __ffs(tb) - 1) : 1ull;   // tb is warp-uniform
        if (lane == 0) e.wk[warp] = tw;
        if (tid == 0) e.m = 0;
        __syncthreads();
        unsigned long long tk = 1ull;
#pragma unroll
        for (int wi = 0; wi < kWW; ++wi) tk = max(tk, e.wk[wi]);
#pragma unroll
        for (int u = 0; u <= FR; ++u) {
            if (key[u] && key[u] >= tk) {
                const int slot = atomicAdd(&e.m, 1);
                if (slot < cap) {
                    ck[slot] = key[u];
                    cx[slot] = (u < FR) ? j0 + tid + u * kWT : xl;
                }
            }
        }
        __syncthreads();
        // rank them; the first kappa become the running list
        const int m = min(e.m, cap);
        for (int i = tid; i < m; i += kWT) {
            const unsigned long long mk = ck[i];
            int rr = 0;
#pragma unroll 8
            for (int jx = 0; jx < m; ++jx) rr += (ck[jx] > mk) ? 1 : 0;
            if (rr < kappa) {
                e.lk[rr] = mk;
                e.lx[rr] = cx[i];
            }
        }
        for (int i = m + tid; i < kappa; i += kWT) { e.lk[i] = 0ull; e.lx[i] = -1; }
    }
    __syncthreads();
}

// ----------------------------------------------------------------- finish
// The CTA that completed a graph's last attention item: merge the items'
// partials into the output (every value merged with each item's weight
// exp(m_k - M) / L), rank the edges, assign the new token by weighted
// plurality and update that community.  With rows given (no community
// state) only the output.  Two dependent rounds of global loads: the
// items' partials with the kept members' logits, tokens and the kept
// communities staged into shared memory, then the winner's centroid row,
// capacity and the pool top.
template <int HG>
__device__ void finish_graph(const DevState& s, const Dims& d, int g, int R, const void* __restrict__ K, int n,
                             float* __restrict__ out, unsigned char* scratch, Misc& mi)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    const int T = R - d.S - 1;
    const int nc = d.api;
    const bool full = !d.rows_given;
    const float* pmg = s.part_ml + (int64_t)g * nc * HG * 2;
    const float* pog = s.part_o + (int64_t)g * nc * HG * kD;
    unsigned char* scratch1 = scratch + kHalf;
    float* wgt = reinterpret_cast<float*>(scratch1 + kFinWgt);   // [nc][HG] item weights
    int C = 0;
    EdgeSrc src;
    unsigned long long* ck = nullptr;
    int* cx = nullptr;
    if (full) {
        // the kept members' logits (rows S .. S+T-1 of zrow), tokens and the
        // kept-community table, staged by 16-byte copies when they fit next
        // to the compaction slots (each copy starts at the 16-byte boundary
        // at or below its first element); read from global memory otherwise
        C = __ldcg(s.meta + (int64_t)g * M_COUNT + M_C);
        const int64_t ze = ((int64_t)g * d.NM + d.S) * HG, te = (int64_t)g * d.rtok_stride;
        const int zpad = (int)(ze & 3), tpad = (int)(te & 3);
        const int zc = (zpad + T * HG + 3) & ~3, tc = (tpad + T + 3) & ~3;   // elements copied
        const int cap = kWW * d.kappa * (EdgeRows<HG>::FR + 1);
        const int4* kig = reinterpret_cast<const int4*>(s.kinfo) + (int64_t)g * d.Nc;
        src.staged = 4 * ((int64_t)zc + tc) + 16 * (int64_t)C <= kRing;
        if (src.staged) {
            float* zs = reinterpret_cast<float*>(scratch);
            int32_t* ts = reinterpret_cast<int32_t*>(zs + zc);
            int4* ks = reinterpret_cast<int4*>(ts + tc);
            const float* zg = s.zrow + (ze - zpad);
            const int32_t* tg = s.rtok + (te - tpad);
            for (int i = tid; i < zc / 4; i += kWT) cp_async16(zs + 4 * i, zg + 4 * i);
            for (int i = tid; i < tc / 4; i += kWT) cp_async16(ts + 4 * i, tg + 4 * i);
            for (int i = tid; i < C; i += kWT) cp_async16(ks + i, kig + i);
            cp_async_commit();
            src.z = zs + zpad;
            src.t = ts + tpad;
            src.ki = ks;
        } else {
            src.z = s.zrow + ze;
            src.t = s.rtok + te;
            src.ki = kig;
        }
        ck = reinterpret_cast<unsigned long long*>(scratch1 + kFinCk);
        cx = reinterpret_cast<int*>(ck + cap);
    }
    EdgeRows<HG> er;   // the first round of kept members
    float kv = 0.f;    // the new token's key, for the update
    if (full && tid < kD) {
        const int64_t krow = (((int64_t)b * d.Hkv + kvh) * d.NM + (n - 1)) * kD;
        kv = d.bf16 ? elem<true>(K, krow + tid) : elem<false>(K, krow + tid);
    }
    constexpr bool kPre = HG * (kD / 4) <= kWT;
    const bool pre = kPre && nc <= 16;
    float4 ov[kPre ? 16 : 1];
    if constexpr (kPre) {
        if (pre) {
            const int h = tid / (kD / 4), d4 = tid % (kD / 4);
#pragma unroll
            for (int u = 0; u < 16; ++u)
                ov[u] = (u < nc && tid < HG * (kD / 4))
                            ? __ldcg(reinterpret_cast<const float4*>(pog + ((int64_t)u * HG + h) * kD) + d4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if (full && !src.staged) edges_load<HG>(src, T, 0, er);
    // ---- the heads' max and sum over the items: warp h % kWW takes head h
    for (int h = warp; h < HG; h += kWW) {
        float M = -INFINITY, Lsum = 0.f;
        for (int k0 = 0; k0 < nc; k0 += 32) {
            const int k = k0 + lane;
            const float2 ml = (k < nc) ? __ldcg(reinterpret_cast<const float2*>(pmg + ((int64_t)k * HG + h) * 2))
                                       : make_float2(-INFINITY, 0.f);
            float mm = ml.x;
#pragma unroll
            for (int o = 16; o; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(kFull, mm, o));
            const float Mn = fmaxf(M, mm);
            float ls = (ml.x == -INFINITY) ? 0.f : ml.y * __expf(ml.x - Mn);
#pragma unroll
            for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(kFull, ls, o);
            Lsum = ((M == -INFINITY) ? 0.f : Lsum * __expf(M - Mn)) + ls;
            M = Mn;
            if (k < nc) wgt[k * HG + h] = ml.x;   // the item's max, turned into its weight below
        }
        __syncwarp();
        for (int k = lane; k < nc; k += 32) {
            const float mk = wgt[k * HG + h];
            wgt[k * HG + h] = (mk == -INFINITY) ? 0.f : __expf(mk - M) / Lsum;
        }
        if (lane == 0) {
            mi.sM[h] = M;
            mi.sL[h] = 1.f / Lsum;
            if (full && s.sel_ml)
                *reinterpret_cast<float2*>(s.sel_ml + 2 * ((int64_t)b * d.Hq + h0 + h)) = make_float2(M, Lsum);
        }
    }
    __syncthreads();
    // ---- the output: thread t takes 4 consecutive dims of a head; all the
    // items' values of those dims are loaded together (for up to 4 heads and
    // 16 items, before the heads' statistics are merged above)
    if (pre) {
        if (tid < HG * (kD / 4)) {
            const int h = tid / (kD / 4), d4 = tid % (kD / 4);
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float f = (u < nc) ? wgt[u * HG + h] : 0.f;
                o.x = fmaf(ov[u].x, f, o.x);
                o.y = fmaf(ov[u].y, f, o.y);
                o.z = fmaf(ov[u].z, f, o.z);
                o.w = fmaf(ov[u].w, f, o.w);
            }
            *reinterpret_cast<float4*>(out + ((int64_t)b * d.Hq + h0 + h) * kD + 4 * d4) = o;
        }
    } else for (int i4 = tid; i4 < HG * (kD / 4); i4 += kWT) {
        const int h = i4 / (kD / 4), d4 = i4 % (kD / 4);
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k0 = 0; k0 < nc; k0 += 16) {
            float4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                v[u] = (k0 + u < nc) ? __ldcg(reinterpret_cast<const float4*>(pog + ((int64_t)(k0 + u) * HG + h) * kD) + d4)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float f = (k0 + u < nc) ? wgt[(k0 + u) * HG + h] : 0.f;
                o.x = fmaf(v[u].x, f, o.x);
                o.y = fmaf(v[u].y, f, o.y);
                o.z = fmaf(v[u].z, f, o.z);
                o.w = fmaf(v[u].w, f, o.w);
            }
        }
        *reinterpret_cast<float4*>(out + ((int64_t)b * d.Hq + h0 + h) * kD + 4 * d4) = o;
    }
    if (!full) return;
    // ---- edges: the top kappa of w = sum_h exp(z - M_h) / L_h over the kept members
    if (src.staged) {
        cp_async_wait<0>();
        __syncthreads();
        edges_load<HG>(src, T, 0, er);
    }
    EdgeScratch& es = *reinterpret_cast<EdgeScratch*>(scratch1 + kFinScr);
    cta_edges<HG>(d, src, T, mi.sM, mi.sL, es, ck, cx, er);
    // ---- the assignment: each edge's kept community (the last with row
    // start <= its row), then the weighted plurality of their ids
    if (warp == 0) {
        const unsigned long long lk = (lane < d.kappa) ? es.lk[lane] : 0ull;
        const bool real = lk != 0ull;
        const int ne = __popc(__ballot_sync(kFull, real));
        const float lw = key_w(lk);
        int cm = 0, csz = 0, coff = 0;
        if (real) {
            const int j = es.lx[lane];
            int a = 0, z = C - 1;
            while (a < z) {
                const int mid = (a + z + 1) >> 1;
                const int rs = src.staged ? src.ki[mid].y : __ldcg(&src.ki[mid].y);
                if (rs <= j) a = mid;
                else z = mid - 1;
            }
            const int4 ki = src.staged ? src.ki[a] : __ldcg(src.ki + a);
            cm = ki.x;
            csz = ki.z;
            coff = ki.w;
            if (cm < 0 || cm >= d.n_comm) {   // corrupt state: report, assign nothing real
                set_error(s.err, CKV_ERR_STATE);
                cm = 0;
            }
            s.e_w[(int64_t)g * d.kappa + lane] = lw;
            s.e_tok[(int64_t)g * d.kappa + lane] = key_t(lk);
            s.e_comm[(int64_t)g * d.kappa + lane] = cm;
        }
        if (lane == 0) s.meta[(int64_t)g * M_COUNT + M_NEDGE] = ne;
        // each lane sums its community's weights exactly, in fixed point
        // (the order of the sum does not matter then); the largest sum wins,
        // ties to the lower id
        const unsigned long long fw = real ? weight_fix(lw) : 0ull;
        unsigned long long v = 0ull;
#pragma unroll 8
        for (int e = 0; e < ne; ++e) {
            const int ce = __shfl_sync(kFull, cm, e);
            const unsigned long long we = __shfl_sync(kFull, fw, e);
            v += (ce == cm) ? we : 0ull;
        }
        // (vote + 1, inverted id): the largest key is the winner; no edge: 0
        unsigned long long bv = real ? v + 1ull : 0ull;
        int bc = real ? cm : 0x7fffffff;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const unsigned long long v2 = __shfl_xor_sync(kFull, bv, o);
            const int c2 = __shfl_xor_sync(kFull, bc, o);
            if (v2 > bv || (v2 == bv && c2 < bc)) { bv = v2; bc = c2; }
        }
        // the winner's size and segment from its first edge (no edges:
        // community 0, read below)
        const unsigned wm = __ballot_sync(kFull, real && cm == bc);
        const int src_l = wm ? __ffs(wm) - 1 : 0;
        const int wsz = __shfl_sync(kFull, csz, src_l), woff = __shfl_sync(kFull, coff, src_l);
        if (lane == 0) {
            mi.sflag[0] = (ne == 0) ? 0 : bc;
            mi.sflag[3] = ne ? wsz : -1;
            mi.sflag[4] = ne ? woff : -1;
            mi.sflag[5] = ne;
        }
    }
    __syncthreads();
    // ---- round 2: the winner's centroid row, capacity (and, with no edges,
    // size and segment) and the pool top
    const int c = mi.sflag[0], ne = mi.sflag[5];
    const int64_t gi = (int64_t)g * d.Nc + c;
    float* mu = s.mu + gi * kD;
    const float mval = (tid < kD) ? mu[tid] : 0.f;
    if (tid == 0) {
        const int cp = s.ccap[gi];
        const int top = s.pool_top[g];
        const int size = ne ? mi.sflag[3] : s.csize[gi];
        const int off0 = ne ? mi.sflag[4] : s.coff[gi];
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
        mi.sflag[1] = ok > 0; mi.sflag[2] = off; mi.sflag[3] = size; mi.sflag[4] = off0; mi.sflag[6] = cp;
    }
    __syncthreads();
    if (!mi.sflag[1]) return;
    const int off = mi.sflag[2], size = mi.sflag[3], old_off = mi.sflag[4], cp = mi.sflag[6];
    const int t = n - 1;
    int32_t* pool = s.pool + (int64_t)g * d.P;
    if (off != old_off)
        for (int i = tid; i < size; i += kWT) pool[off + i] = pool[old_off + i];
    // running-mean update of the assigned centroid, double math rounded once
    if (tid < kD) {
        const double mv = (double)mval;
        mu[tid] = __double2float_rn(__dadd_rn(mv, __ddiv_rn(__dsub_rn((double)kv, mv), (double)(size + 1))));
    }
    __syncthreads();   // the segment copy is complete before the append
    const int64_t row = (int64_t)g * (d.NM - d.n_init) + (t - d.n_init);
    if (tid == 0) {
        if (off != old_off) {
            s.coff[gi] = off;
            s.ccap[gi] = max(16, 2 * cp);
        }
        pool[off + size] = t;
        s.csize[gi] = size + 1;
        s.tok_comm[(int64_t)g * d.NM + t] = c;
        s.meta[(int64_t)g * M_COUNT + M_ASSIGNED] = c;
        s.edge_deg[row] = ne;
    }
    if (tid < ne) {
        s.edge_col[row * d.kappa + tid] = key_t(es.lk[tid]);
        s.edge_w[row * d.kappa + tid] = key_w(es.lk[tid]);
    }
}

// ------------------------------------------------------------ the kernel
// One CTA of 256 threads per SM.  The first n_workers CTAs are workers:
// all 8 warps run every selection and then every finish, graph g on worker
// g mod n_workers (two warps per scheduler hide each other's latency in
// that serial code).  Every other CTA runs as two independent halves of 4
// warps, each with its own rings, barriers and named barrier, streaming
// items from the queue: while one half waits (a ring ramping up, a
// selection not yet published) the other keeps the SM's loads in flight.
template <bool BF16, int HG>
__global__ void __launch_bounds__(kWT, 1) k_step(DevState s, Dims d, const void* __restrict__ q,
                                                 const void* __restrict__ K, const void* __restrict__ V, int n,
                                                 float* __restrict__ out)
{
    using L = AttL<BF16, HG>;
    extern __shared__ __align__(128) unsigned char smem[];
    const int half = threadIdx.x >> 7, ht = threadIdx.x & (kT - 1), hwarp = ht >> 5;
    unsigned char* hb = smem + half * kHalf;
    Misc& mh = *reinterpret_cast<Misc*>(hb + kHOffMisc);
    unsigned long long* bars = reinterpret_cast<unsigned long long*>(hb + kHOffBar);
    int* tokw = reinterpret_cast<int*>(hb + kHOffTok) + hwarp * kTokW;
    float* red = reinterpret_cast<float*>(hb);
    const int NS = d.rows_given ? 0 : d.G * d.spg;
    const int total = NS + d.G * d.api;
    unsigned* qctr = s.step_ctr;
    const int NWk = d.n_workers;
    const bool worker = (int)blockIdx.x < NWk;
    if (ht == 0) {
        for (int i = 0; i < kW * kNSlot; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
        mh.item = (worker || *(volatile int*)s.err) ? total : (int)atomicAdd(qctr, 1u);
    }
    if (ht < kW) mh.abort[ht] = 0;
    __syncthreads();
    if (worker) {
        Misc& mw = *reinterpret_cast<Misc*>(smem + kHOffMisc);   // half 0's
        bool ok = true;
        for (int g = blockIdx.x; ok && !d.rows_given && g < d.G; g += NWk) {
            // ---------------- selection of g once its score items are done
            if (threadIdx.x == 0) mw.flag = wait_count(s.gcnt + 4 * g, (unsigned)d.spg, s.err, d.wait_polls);
            __syncthreads();
            ok = mw.flag;
            if (!ok) break;
            __threadfence();
            select_graph(s, d, g, *reinterpret_cast<SelSmem*>(smem), *reinterpret_cast<SelX*>(smem + kOffX), mw);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) set_flag(s.gcnt + 4 * g + 1);
        }
        for (int g = blockIdx.x; ok && g < d.G; g += NWk) {
            // ---------------- finish of g once its attention items are done
            if (threadIdx.x == 0) mw.flag = wait_count(s.gcnt + 4 * g + 2, (unsigned)d.api, s.err, d.wait_polls);
            __syncthreads();
            ok = mw.flag;
            if (!ok) break;
            __threadfence();
            const int R = d.rows_given ? d.S + s.rows_T[g] + 1 : __ldcg(s.meta + (int64_t)g * M_COUNT + M_ROWS);
            finish_graph<HG>(s, d, g, R, K, n, out, smem, mw);
            __syncthreads();
        }
        if (!ok && threadIdx.x == 0) set_error(s.err, CKV_ERR_TIMEOUT);
    } else {
        int item = mh.item;
        unsigned fills = 0;   // score slots this warp has used (uniform in the warp)
        while (item < total) {
            if (item < NS) {
                // ---------------- score item
                const int g = item / d.spg, p = item % d.spg;
                score_item<BF16>(s, d, q, g, p, hb, bars, fills, mh);
                __threadfence();
                hsync();
                if (ht == 0) atomicAdd(s.gcnt + 4 * g, 1u);
            } else {
                // ---------------- attention item
                const int j = item - NS;
                const int g = j / d.api, k = j % d.api;
                if (!d.rows_given) {
                    if (ht == 0) mh.flag = wait_count(s.gcnt + 4 * g + 1, 1u, s.err, d.wait_polls);
                    hsync();
                    if (!mh.flag) {
                        if (ht == 0) set_error(s.err, CKV_ERR_TIMEOUT);
                        break;
                    }
                }
                int b, h0, kvh;
                graph_heads(d, g, b, h0, kvh);
                const int R = d.rows_given ? d.S + s.rows_T[g] + 1 : __ldcg(s.meta + (int64_t)g * M_COUNT + M_ROWS);
                const int r0 = (int)((int64_t)k * R / d.api), r1 = (int)((int64_t)(k + 1) * R / d.api);
                const int nrows = r1 - r0;
                const int64_t kvbase = ((int64_t)b * d.Hkv + kvh) * d.NM;
                WarpRows a;
                a.Kb = reinterpret_cast<const char*>(K) + kvbase * L::RB;
                a.Vb = reinterpret_cast<const char*>(V) + kvbase * L::RB;
                a.rtok = s.rtok + (int64_t)g * d.rtok_stride;
                a.zrow = d.rows_given ? nullptr : s.zrow + (int64_t)g * d.NM * HG;
                a.a0 = r0 + (int)((int64_t)hwarp * nrows / kW);
                a.a1 = r0 + (int)((int64_t)(hwarp + 1) * nrows / kW);
                a.S = d.S;
                a.T = R - d.S - 1;
                a.R = R;
                a.t_new = n - 1;
                a.err = s.err;
                unsigned char* wbuf = hb + hwarp * (kNSlot * kSlot);
                if constexpr (BF16) {
                    const uint32_t* q2 = reinterpret_cast<const uint32_t*>(q) + ((int64_t)b * d.Hq + h0) * kD / 2;
                    warp_rows_mma<HG>(a, q2, wbuf, tokw, red);
                } else {
                    const float* qg = reinterpret_cast<const float*>(q) + ((int64_t)b * d.Hq + h0) * kD;
                    warp_rows_fma<HG>(a, qg, wbuf, tokw, red);
                }
                hsync();
                // combine the warps: (m, l, acc) -> this item's partial per head
                float* po = s.part_o + ((int64_t)g * d.api + k) * HG * kD;
                float* pm = s.part_ml + ((int64_t)g * d.api + k) * HG * 2;
                for (int i = ht; i < HG * kD; i += kT) {
                    const int h = i / kD, dd = i % kD;
                    float mwv[kW];
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kW; ++w) {
                        mwv[w] = red[(w * HG + h) * L::RSTR + kD];
                        M = fmaxf(M, mwv[w]);
                    }
                    float o = 0.f, l = 0.f;
#pragma unroll
                    for (int w = 0; w < kW; ++w) {
                        const float* rw = red + (w * HG + h) * L::RSTR;
                        const float f = (mwv[w] == -INFINITY) ? 0.f : __expf(mwv[w] - M);
                        o = fmaf(rw[dd], f, o);
                        l = fmaf(rw[kD + 1], f, l);
                    }
                    po[i] = o;
                    if (dd == 0) *reinterpret_cast<float2*>(pm + h * 2) = make_float2(M, l);
                }
                __threadfence();
                hsync();
                if (ht == 0) atomicAdd(s.gcnt + 4 * g + 2, 1u);
            }
            hsync();
            if (ht == 0) mh.item = (*(volatile int*)s.err) ? total : (int)atomicAdd(qctr, 1u);
            hsync();
            item = mh.item;
        }
    }
    // ---- the last CTA to leave resets the queue and the graphs' counters
    // for the next step
    Misc& m0 = *reinterpret_cast<Misc*>(smem + kHOffMisc);
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        m0.flag = (atomicAdd(qctr + 1, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (m0.flag) {
        __threadfence();
        for (int i = threadIdx.x; i < 4 * d.G; i += kWT) s.gcnt[i] = 0u;
        if (threadIdx.x == 0) { qctr[0] = 0u; qctr[1] = 0u; }
    }
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

template <bool BF16, int HG>
const void* step_fn()
{
    return reinterpret_cast<const void*>(k_step<BF16, HG>);
}

}  // namespace

int step_cpi() { return kCPI; }

int step_hist_bins() { return kCoarse; }

int step_api(int S, int rows)
{
    const int64_t r = (int64_t)S + rows + 1;
    const int64_t a = (r + kRPI - 1) / kRPI;
    return (int)(a < 1 ? 1 : a > kMaxApi ? kMaxApi : a);
}

size_t step_kept_scratch_ints(int Nc) { return (size_t)3 * (Nc + 1); }

cudaError_t prepare_step(const Dims& d, int sms, int* grid)
{
    *grid = 0;
    int occ = 0;
    cudaError_t e = dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        const void* fn = d.bf16 ? step_fn<true, HG>() : step_fn<false, HG>();
        cudaError_t r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        // the CTA's ~197 KB need the largest shared-memory share of the L1
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (r != cudaSuccess) return r;
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kWT, kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorLaunchOutOfResources;
    *grid = occ * sms;
    return cudaSuccess;
}

cudaError_t launch_step(const DevState& s, const Dims& d, const void* q, const void* K, const void* V, int n,
                        float* out, cudaStream_t st)
{
    return dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(d.nStep);
        cfg.blockDim = dim3(kWT);
        cfg.dynamicSmemBytes = kSmemBytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;   // the grid is co-resident: the waits end
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (d.bf16) return cudaLaunchKernelEx(&cfg, k_step<true, HG>, s, d, q, K, V, n, out);
        return cudaLaunchKernelEx(&cfg, k_step<false, HG>, s, d, q, K, V, n, out);
    });
}

}  // namespace ckv
