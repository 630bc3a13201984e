// k_decode.cu -- the per-step decode kernels of CommunityKV on sm_100a.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 1 caption, step (3): score the query against the community
// centroids, retrieve a candidate subset, run exact attention over it plus
// the sink tokens, take the top-kappa keys as the new token's edges and
// assign it to a community in constant time; Table 1: O(sqrt(n) d)
// retrieval, O(d) update.
//
// Four kernels per step, all memory-bound:
//   k_score   centroid GEMV, one warp per 32 communities, lane = 4 dims,
//             32 partial dots reduced by a butterfly transpose (31 shuffles
//             for 32 rows).
//   k_select  one CTA per graph: exact budgeted top-C by bucket passes over
//             the scores (a monotone linear bucketing, then radix windows of
//             the order-preserving score bits, then of the id) and a final
//             bitonic sort of <= 1024 candidates; writes the kept list, its
//             size prefix and the kept member rows.
//   k_attend  split-K gather attention: each CTA streams 32-row tiles of K
//             and V (16-byte cp.async into an XOR-swizzled shared layout,
//             double-buffered), all query heads of a graph share one gather;
//             the last CTA of a graph merges the (m, l, o) partials.
//   k_assign  one CTA per graph: edge weights from the logits, top-kappa,
//             weighted-plurality vote, running-mean update, member append.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "ckv_internal.cuh"

namespace ckv {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kTile = 32;          // rows per attention tile
constexpr int kAttThreads = 256;
constexpr int kSelThreads = 1024;
constexpr int kAsgThreads = 256;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

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
template <bool BF16>
__global__ void __launch_bounds__(256) k_score(DevState s, Dims d, const void* __restrict__ q)
{
    if (*(volatile int*)s.err) return;
    const int g = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * 256 + warp * 32;
    if (c0 >= d.n_comm) return;
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    const int hg = d.HG;
    // Sum of the graph's query heads, 4 dims per lane (a group's score is
    // the sum of its heads' scores).
    float qs[4] = {0.f, 0.f, 0.f, 0.f};
    for (int h = 0; h < hg; ++h) {
        const int64_t base = ((int64_t)b * d.Hq + h0 + h) * kD + 4 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) qs[k] += elem<BF16>(q, base + k);
    }
    const float4* mu = reinterpret_cast<const float4*>(s.mu + (int64_t)g * d.Nc * kD);
    float part[32];
#pragma unroll
    for (int rb = 0; rb < 32; rb += 8) {
        float4 v[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int c = c0 + rb + r;
            v[r] = (c < d.n_comm) ? __ldcs(mu + (int64_t)c * (kD / 4) + lane)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
            part[rb + r] = fmaf(qs[3], v[r].w, fmaf(qs[2], v[r].z, fmaf(qs[1], v[r].y, qs[0] * v[r].x)));
    }
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
    const int c = c0 + lane;
    if (c < d.n_comm) {
        const int64_t gi = (int64_t)g * d.Nc + c;
        s.score[gi] = (s.csize[gi] > 0) ? part[0] : -INFINITY;
    }
}

// -------------------------------------------------------- block utilities
// inclusive block scan of an int (kSelThreads threads); returns the block total
__device__ __forceinline__ int block_scan_incl(int v, int* warp_sums, int& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += t;
        }
        warp_sums[lane] = w;
    }
    __syncthreads();
    const int add = warp ? warp_sums[warp - 1] : 0;
    total = warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();
    return v + add;
}

__device__ __forceinline__ float block_reduce_max(float v, float* red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = -INFINITY;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r = fmaxf(r, red[i]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ uint32_t block_reduce_or_u(uint32_t v, uint32_t* red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o; o >>= 1) v |= __shfl_xor_sync(kFull, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t r = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r |= red[i];
    __syncthreads();
    return r;
}

// --------------------------------------------------------------- k_select
// Status of a community during selection.
enum : int8_t { ST_OUT = 0, ST_IN = 1, ST_CAND = 2 };

struct SelShared {
    int hist[kSelBins];
    unsigned long long key[kSortCap];
    int wt[kSortCap];
    int warp_sums[32];
    float redf[32];
    uint32_t redu[32];
    int bstar;          // boundary bin
    int w_above;        // weight already kept
    int n_cand;
    int done;
};

// key of a candidate: (order-preserving score bits, inverted id): larger = kept first
__device__ __forceinline__ unsigned long long sel_key(float sc, int c)
{
    return ((unsigned long long)ord_u(sc) << 32) | (unsigned long long)(~(uint32_t)c);
}

__global__ void __launch_bounds__(kSelThreads) k_select(DevState s, Dims d, int n)
{
    if (*(volatile int*)s.err) return;
    __shared__ SelShared sh;
    const int g = blockIdx.x;
    const int tid = threadIdx.x;
    const int Nc = d.n_comm;
    const float* sc = s.score + (int64_t)g * d.Nc;
    const int32_t* csz = s.csize + (int64_t)g * d.Nc;
    int8_t* stat = s.cstat + (int64_t)g * d.Nc;
    // ---- pass 0: all non-empty communities are candidates
    int wsum_local = 0;
    for (int c = tid; c < Nc; c += kSelThreads) {
        const int w = csz[c];
        stat[c] = (w > 0) ? ST_CAND : ST_OUT;
        wsum_local += (w > 0) ? w : 0;
    }
    int total_w;
    block_scan_incl(wsum_local, sh.warp_sums, total_w);
    if (tid == 0) { sh.w_above = 0; sh.done = (total_w <= d.budget) ? 1 : 0; }
    __syncthreads();
    if (sh.done) {   // every community fits the budget: keep them all
        for (int c = tid; c < Nc; c += kSelThreads)
            if (stat[c] == ST_CAND) stat[c] = ST_IN;
        __syncthreads();
    }

    // ---- bucket passes until <= kSortCap candidates remain
    // pass kinds: 0 = linear in the float score over [lo, hi]; 1 = radix window
    // of ord_u(score); 2 = radix window of the inverted id.
    int kind = 0;
    for (int pass = 0; pass < 12 && !sh.done; ++pass) {
        // candidate statistics
        float lo = INFINITY, hi = -INFINITY;
        uint32_t uor = 0, uand = 0xffffffffu, ior = 0, iand = 0xffffffffu;
        int cnt = 0;
        for (int c = tid; c < Nc; c += kSelThreads) {
            if (stat[c] != ST_CAND) continue;
            const float v = sc[c];
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
            const uint32_t u = ord_u(v), iv = ~(uint32_t)c;
            uor |= u; uand &= u; ior |= iv; iand &= iv;
            ++cnt;
        }
        int ncand;
        block_scan_incl(cnt, sh.warp_sums, ncand);
        if (ncand <= kSortCap) break;
        const float glo = -block_reduce_max(-lo, sh.redf);
        const float ghi = block_reduce_max(hi, sh.redf);
        // bits that differ among the candidates: OR of all & ~(AND of all)
        const uint32_t udiff = block_reduce_or_u(uor, sh.redu) & block_reduce_or_u(~uand, sh.redu);
        const uint32_t idiff = block_reduce_or_u(ior, sh.redu) & block_reduce_or_u(~iand, sh.redu);
        int shift = 0;
        if (kind == 0 && !(glo < ghi)) kind = 1;
        if (kind == 1 && udiff == 0) kind = 2;
        if (kind == 1) { const int top = 31 - __clz(udiff); shift = max(0, top - 10); }
        if (kind == 2) { const int top = 31 - __clz(idiff); shift = max(0, top - 10); }
        const double dlo = (double)glo, dscale = (double)kSelBins / ((double)ghi - (double)glo);
        for (int i = tid; i < kSelBins; i += kSelThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int c = tid; c < Nc; c += kSelThreads) {
            if (stat[c] != ST_CAND) continue;
            const float v = sc[c];
            int bin;
            if (kind == 0) bin = max(0, min(kSelBins - 1, (int)(((double)v - dlo) * dscale)));
            else if (kind == 1) bin = (int)((ord_u(v) >> shift) & (kSelBins - 1));
            else bin = (int)((~(uint32_t)c >> shift) & (kSelBins - 1));
            atomicAdd(&sh.hist[bin], csz[c]);
        }
        __syncthreads();
        // boundary bin, scanning from the top bin down (2 bins per thread)
        const int rb0 = kSelBins - 1 - 2 * tid, rb1 = rb0 - 1;
        const int h0v = sh.hist[rb0], h1v = sh.hist[rb1];
        int tot;
        const int incl = block_scan_incl(h0v + h1v, sh.warp_sums, tot);
        const int before = sh.w_above + incl - (h0v + h1v);
        if (tid == 0) sh.bstar = -1;
        __syncthreads();
        if (before <= d.budget && before + h0v > d.budget) sh.bstar = rb0;
        else if (before + h0v <= d.budget && before + h0v + h1v > d.budget) sh.bstar = rb1;
        __syncthreads();
        const int bstar = sh.bstar;
        // weight strictly above the boundary bin
        int above_local = 0;
        if (bstar >= 0) {
            if (rb0 > bstar) above_local += h0v;
            if (rb1 > bstar) above_local += h1v;
        }
        int above;
        block_scan_incl(above_local, sh.warp_sums, above);
        for (int c = tid; c < Nc; c += kSelThreads) {
            if (stat[c] != ST_CAND) continue;
            if (bstar < 0) { stat[c] = ST_IN; continue; }
            const float v = sc[c];
            int bin;
            if (kind == 0) bin = max(0, min(kSelBins - 1, (int)(((double)v - dlo) * dscale)));
            else if (kind == 1) bin = (int)((ord_u(v) >> shift) & (kSelBins - 1));
            else bin = (int)((~(uint32_t)c >> shift) & (kSelBins - 1));
            stat[c] = (bin > bstar) ? ST_IN : (bin < bstar ? ST_OUT : ST_CAND);
        }
        __syncthreads();
        if (tid == 0) {
            if (bstar < 0) sh.done = 1;
            else sh.w_above += above;
        }
        if (kind == 0) kind = 1;   // the linear pass runs once, radix windows after
        __syncthreads();
    }

    // ---- final exact pass: sort the remaining candidates by key
    if (!sh.done) {
        if (tid == 0) sh.n_cand = 0;
        __syncthreads();
        for (int c = tid; c < Nc; c += kSelThreads) {
            if (stat[c] != ST_CAND) continue;
            const int slot = atomicAdd(&sh.n_cand, 1);
            if (slot < kSortCap) { sh.key[slot] = sel_key(sc[c], c); sh.wt[slot] = csz[c]; }
        }
        __syncthreads();
        const int m = min(sh.n_cand, kSortCap);
        int m2 = 1;
        while (m2 < m) m2 <<= 1;
        for (int i = m + tid; i < m2; i += kSelThreads) { sh.key[i] = 0ull; sh.wt[i] = 0; }
        __syncthreads();
        // bitonic sort, descending keys
        for (int k = 2; k <= m2; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = tid; i < m2; i += kSelThreads) {
                    const int p = i ^ j;
                    if (p > i) {
                        const bool desc = ((i & k) == 0);
                        const unsigned long long a = sh.key[i], bb = sh.key[p];
                        if (desc ? (a < bb) : (a > bb)) {
                            sh.key[i] = bb; sh.key[p] = a;
                            const int t = sh.wt[i]; sh.wt[i] = sh.wt[p]; sh.wt[p] = t;
                        }
                    }
                }
                __syncthreads();
            }
        }
        // keep the prefix that fits (forced first when nothing is kept yet)
        const int w_above = sh.w_above;
        int local = (tid < m) ? sh.wt[tid] : 0;
        int tot;
        const int incl = block_scan_incl(local, sh.warp_sums, tot);
        if (tid < m) {
            const bool keep = (w_above + incl <= d.budget) || (w_above == 0 && tid == 0);
            const int c = (int)(~(uint32_t)(sh.key[tid] & 0xffffffffull));
            stat[c] = keep ? ST_IN : ST_OUT;
        }
        __syncthreads();
    }

    // ---- compaction in ascending id, prefix of sizes
    int32_t* sel = s.sel + (int64_t)g * d.Nc;
    int32_t* pre = s.sel_pre + (int64_t)g * (d.Nc + 1);
    int carry_c = 0, carry_t = 0;
    for (int base = 0; base < Nc; base += kSelThreads) {
        const int c = base + tid;
        const bool in = (c < Nc) && stat[c] == ST_IN;
        const int w = in ? csz[c] : 0;
        int tc, tw;
        const int ic = block_scan_incl(in ? 1 : 0, sh.warp_sums, tc);
        const int iw = block_scan_incl(w, sh.warp_sums, tw);
        if (in) {
            sel[carry_c + ic - 1] = c;
            pre[carry_c + ic - 1] = carry_t + iw - w;
        }
        carry_c += tc;
        carry_t += tw;
    }
    if (tid == 0) {
        pre[carry_c] = carry_t;
        int32_t* meta = s.meta + (int64_t)g * M_COUNT;
        meta[M_C] = carry_c;
        meta[M_T] = carry_t;
        meta[M_ROWS] = d.S + carry_t + 1;
    }
    __syncthreads();
    // ---- materialise the kept member rows: token and community of row r
    const int32_t* coff = s.coff + (int64_t)g * d.Nc;
    const int32_t* pool = s.pool + (int64_t)g * d.P;
    int32_t* rtok = s.rtok + (int64_t)g * d.NM;
    int32_t* rcomm = s.rcomm + (int64_t)g * d.NM;
    const int lane = tid & 31, warp = tid >> 5;
    for (int k = warp; k < carry_c; k += kSelThreads / 32) {
        const int c = sel[k];
        const int off = coff[c];
        const int sz = csz[c];
        const int p0 = pre[k];
        for (int i = lane; i < sz; i += 32) {
            rtok[p0 + i] = pool[off + i];
            rcomm[p0 + i] = c;
        }
    }
    (void)n;
}

// --------------------------------------------------------------- k_attend
// shared layout: q[HG][128] f32 | tok[2][32] | K[2][32][RB] | V[2][32][RB] |
//                zp[8][HG][32] | p[32][HG] | alpha[HG] | misc
template <bool BF16, int HG>
struct AttLayout {
    static constexpr int RB = kD * (BF16 ? 2 : 4);       // bytes per K/V row
    static constexpr int NCH = RB / 16;                  // 16-byte chunks per row
    static constexpr int off_q = 0;
    static constexpr int off_tok = off_q + HG * kD * 4;
    static constexpr int off_k = off_tok + 2 * kTile * 4;
    static constexpr int off_v = off_k + 2 * kTile * RB;
    static constexpr int off_zp = off_v + 2 * kTile * RB;
    static constexpr int off_p = off_zp + 8 * HG * kTile * 4;
    static constexpr int off_alpha = off_p + kTile * HG * 4;
    static constexpr int bytes_loop = off_alpha + 64;
    // end-of-CTA reduction buffer (reuses the K/V region): [16][HG][128] f32
    static constexpr int bytes_red = off_k + 16 * HG * kD * 4;
    static constexpr int bytes = bytes_loop > bytes_red ? bytes_loop : bytes_red;
};

__device__ __forceinline__ int swz(int row, int ch) { return (ch & ~7) | ((ch ^ row) & 7); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

template <bool BF16, int HG>
__global__ void __launch_bounds__(kAttThreads) k_attend(DevState s, Dims d, const void* __restrict__ q,
                                                       const void* __restrict__ K,
                                                       const void* __restrict__ V, int n,
                                                       float* __restrict__ out)
{
    using L = AttLayout<BF16, HG>;
    if (*(volatile int*)s.err) return;
    extern __shared__ __align__(128) unsigned char smem[];
    float* qf = reinterpret_cast<float*>(smem + L::off_q);
    int* tok = reinterpret_cast<int*>(smem + L::off_tok);
    unsigned char* Ks = smem + L::off_k;
    unsigned char* Vs = smem + L::off_v;
    float* zp = reinterpret_cast<float*>(smem + L::off_zp);
    float* pt = reinterpret_cast<float*>(smem + L::off_p);
    float* alpha = reinterpret_cast<float*>(smem + L::off_alpha);
    __shared__ int s_last;

    const int g = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    const int R = s.meta[(int64_t)g * M_COUNT + M_ROWS];
    const int T = R - d.S - 1;
    const int per = (R + gridDim.x - 1) / gridDim.x;
    const int r0 = min(R, split * per), r1 = min(R, r0 + per);
    const int ntiles = (r1 - r0 + kTile - 1) / kTile;
    const int t_new = n - 1;
    const int64_t kvbase = ((int64_t)b * d.Hkv + kvh) * d.NM;     // row index base
    const char* Kb = reinterpret_cast<const char*>(K) + kvbase * L::RB;
    const char* Vb = reinterpret_cast<const char*>(V) + kvbase * L::RB;
    const int32_t* rtok = s.rtok + (int64_t)g * d.NM;
    float* zrow = s.zrow + (int64_t)g * d.NM * HG;

    for (int i = tid; i < HG * kD; i += kAttThreads) {
        const int h = i / kD, dd = i % kD;
        qf[i] = elem<BF16>(q, ((int64_t)b * d.Hq + h0 + h) * kD + dd);
    }

    auto row_token = [&](int r) -> int {
        if (r < d.S) return r;
        if (r == R - 1) return t_new;
        return rtok[r - d.S];
    };
    auto issue = [&](int tile) {
        const int buf = tile & 1;
        const int rbase = r0 + tile * kTile;
        if (tid < kTile) {
            const int r = rbase + tid;
            tok[buf * kTile + tid] = (r < r1) ? row_token(r) : -1;
        }
        __syncthreads();
        // K and V: kTile rows x NCH chunks each
        for (int i = tid; i < kTile * L::NCH; i += kAttThreads) {
            const int row = i / L::NCH, ch = i % L::NCH;
            const int tk = tok[buf * kTile + row];
            if (tk < 0) continue;
            const int dst = (buf * kTile + row) * L::RB + swz(row, ch) * 16;
            cp_async16(Ks + dst, Kb + (int64_t)tk * L::RB + ch * 16);
            cp_async16(Vs + dst, Vb + (int64_t)tk * L::RB + ch * 16);
        }
        cp_async_commit();
    };

    // running softmax state, kept by warp h for head h
    float m_run = -INFINITY, l_run = 0.f;
    // PV accumulators: thread = (row group rg = tid/16, chunk c8 = tid%16): 8 dims x HG heads
    const int c8 = tid & 15, rg = tid >> 4;
    float acc[HG][8];
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[h][j] = 0.f;

    const float scale = 0.08838834764831845f;   // 1 / sqrt(128), correctly rounded
    if (ntiles > 0) issue(0);
    for (int tile = 0; tile < ntiles; ++tile) {
        const int buf = tile & 1;
        if (tile + 1 < ntiles) { issue(tile + 1); cp_async_wait<1>(); }
        else cp_async_wait<0>();
        __syncthreads();
        // ---- logits: warp e = dims [16e, 16e+16), lane = row
        {
            const int e = warp, r = lane;
            float a[HG][8];
#pragma unroll
            for (int h = 0; h < HG; ++h)
#pragma unroll
                for (int j = 0; j < 8; ++j) a[h][j] = 0.f;
            const unsigned char* krow = Ks + (buf * kTile + r) * L::RB;
            if (BF16) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int ch = 2 * e + cc;
                    const uint4 w = *reinterpret_cast<const uint4*>(krow + swz(r, ch) * 16);
                    float kv[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                                   bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
                    for (int h = 0; h < HG; ++h) {
                        const float4 qa = *reinterpret_cast<const float4*>(qf + h * kD + ch * 8);
                        const float4 qb = *reinterpret_cast<const float4*>(qf + h * kD + ch * 8 + 4);
                        a[h][0] = fmaf(qa.x, kv[0], a[h][0]);
                        a[h][1] = fmaf(qa.y, kv[1], a[h][1]);
                        a[h][2] = fmaf(qa.z, kv[2], a[h][2]);
                        a[h][3] = fmaf(qa.w, kv[3], a[h][3]);
                        a[h][4] = fmaf(qb.x, kv[4], a[h][4]);
                        a[h][5] = fmaf(qb.y, kv[5], a[h][5]);
                        a[h][6] = fmaf(qb.z, kv[6], a[h][6]);
                        a[h][7] = fmaf(qb.w, kv[7], a[h][7]);
                    }
                }
            } else {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int ch = 4 * e + cc;
                    const float4 w = *reinterpret_cast<const float4*>(krow + swz(r, ch) * 16);
#pragma unroll
                    for (int h = 0; h < HG; ++h) {
                        const float4 qa = *reinterpret_cast<const float4*>(qf + h * kD + ch * 4);
                        const int j0 = (cc & 1) * 4;
                        a[h][j0 + 0] = fmaf(qa.x, w.x, a[h][j0 + 0]);
                        a[h][j0 + 1] = fmaf(qa.y, w.y, a[h][j0 + 1]);
                        a[h][j0 + 2] = fmaf(qa.z, w.z, a[h][j0 + 2]);
                        a[h][j0 + 3] = fmaf(qa.w, w.w, a[h][j0 + 3]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < HG; ++h)
                zp[(e * HG + h) * kTile + r] =
                    ((a[h][0] + a[h][1]) + (a[h][2] + a[h][3])) + ((a[h][4] + a[h][5]) + (a[h][6] + a[h][7]));
        }
        __syncthreads();
        // ---- softmax of the tile: warp h handles head h, lane = row
        if (warp < HG) {
            const int h = warp, r = lane;
            const int gr = r0 + tile * kTile + r;
            float z = -INFINITY;
            if (gr < r1) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = zp[(e * HG + h) * kTile + r];
                z = (((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]))) * scale;
                if (gr >= d.S && gr < d.S + T) zrow[(int64_t)(gr - d.S) * HG + h] = z;
            }
            float mt = z;
#pragma unroll
            for (int o = 16; o; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, o));
            const float m_new = fmaxf(m_run, mt);
            const float p = (gr < r1) ? __expf(z - m_new) : 0.f;
            float ps = p;
#pragma unroll
            for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(kFull, ps, o);
            const float al = (m_run == -INFINITY) ? 0.f : __expf(m_run - m_new);
            l_run = l_run * al + ps;
            m_run = m_new;
            pt[r * HG + h] = p;
            if (lane == 0) alpha[h] = al;
        }
        __syncthreads();
        // ---- PV: rows rg and rg + 16 of the tile (rows past the CTA's end
        // hold stale shared memory and are skipped)
        {
            const int nvalid = min(kTile, r1 - (r0 + tile * kTile));
            float al[HG];
#pragma unroll
            for (int h = 0; h < HG; ++h) al[h] = alpha[h];
#pragma unroll
            for (int h = 0; h < HG; ++h)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[h][j] *= al[h];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = rg + 16 * rr;
                if (r >= nvalid) continue;
                const unsigned char* vrow = Vs + (buf * kTile + r) * L::RB;
                float vv[8];
                if (BF16) {
                    const uint4 w = *reinterpret_cast<const uint4*>(vrow + swz(r, c8) * 16);
                    vv[0] = bf_lo(w.x); vv[1] = bf_hi(w.x); vv[2] = bf_lo(w.y); vv[3] = bf_hi(w.y);
                    vv[4] = bf_lo(w.z); vv[5] = bf_hi(w.z); vv[6] = bf_lo(w.w); vv[7] = bf_hi(w.w);
                } else {
                    const float4 w0 = *reinterpret_cast<const float4*>(vrow + swz(r, 2 * c8) * 16);
                    const float4 w1 = *reinterpret_cast<const float4*>(vrow + swz(r, 2 * c8 + 1) * 16);
                    vv[0] = w0.x; vv[1] = w0.y; vv[2] = w0.z; vv[3] = w0.w;
                    vv[4] = w1.x; vv[5] = w1.y; vv[6] = w1.z; vv[7] = w1.w;
                }
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    const float p = pt[r * HG + h];
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[h][j] = fmaf(p, vv[j], acc[h][j]);
                }
            }
        }
        __syncthreads();
    }

    // ---- reduce the 16 row groups and write this CTA's partial
    float* red = reinterpret_cast<float*>(smem + L::off_k);
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[(rg * HG + h) * kD + c8 * 8 + j] = acc[h][j];
    __syncthreads();
    float* part = s.part + ((int64_t)g * gridDim.x + split) * HG * (kD + 2);
    for (int i = tid; i < HG * kD; i += kAttThreads) {
        const int h = i / kD, dd = i % kD;
        float o = 0.f;
        for (int k = 0; k < 16; ++k) o += red[(k * HG + h) * kD + dd];
        part[h * (kD + 2) + 2 + dd] = o;
    }
    if (warp < HG && lane == 0) {
        part[warp * (kD + 2) + 0] = m_run;
        part[warp * (kD + 2) + 1] = l_run;
    }
    // ---- last CTA of the graph merges
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&s.counter[g], 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int ns = gridDim.x;
    const float* pg = s.part + (int64_t)g * ns * HG * (kD + 2);
    float* ml = s.ml + (int64_t)g * HG * 2;
    float* wgt = reinterpret_cast<float*>(smem + L::off_k);   // [ns][HG] merge weights
    __shared__ float sM[8], sL[8];
    if (warp < HG) {
        const int h = warp;
        float M = -INFINITY;
        for (int k = lane; k < ns; k += 32) M = fmaxf(M, __ldcg(pg + ((int64_t)k * HG + h) * (kD + 2)));
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
        float Lsum = 0.f;
        for (int k = lane; k < ns; k += 32) {
            const float mk = __ldcg(pg + ((int64_t)k * HG + h) * (kD + 2));
            const float lk = __ldcg(pg + ((int64_t)k * HG + h) * (kD + 2) + 1);
            const float wk = (mk == -INFINITY) ? 0.f : __expf(mk - M);
            if ((int64_t)ns * HG * 4 <= (int64_t)(L::bytes - L::off_k)) wgt[k * HG + h] = wk;
            Lsum += lk * wk;
        }
        // fixed-order sum over lanes
#pragma unroll
        for (int o = 16; o; o >>= 1) Lsum += __shfl_xor_sync(kFull, Lsum, o);
        if (lane == 0) { sM[h] = M; sL[h] = Lsum; ml[h * 2] = M; ml[h * 2 + 1] = Lsum; }
    }
    __syncthreads();
    const bool wgt_in_smem = (int64_t)ns * HG * 4 <= (int64_t)(L::bytes - L::off_k);
    for (int i = tid; i < HG * kD; i += kAttThreads) {
        const int h = i / kD, dd = i % kD;
        float o = 0.f;
        for (int k = 0; k < ns; ++k) {
            float wk;
            if (wgt_in_smem) wk = wgt[k * HG + h];
            else {
                const float mk = __ldcg(pg + ((int64_t)k * HG + h) * (kD + 2));
                wk = (mk == -INFINITY) ? 0.f : __expf(mk - sM[h]);
            }
            if (wk != 0.f) o = fmaf(__ldcg(pg + ((int64_t)k * HG + h) * (kD + 2) + 2 + dd), wk, o);
        }
        out[((int64_t)b * d.Hq + h0 + h) * kD + dd] = o / sL[h];
    }
    if (tid == 0) s.counter[g] = 0u;
}

// --------------------------------------------------------------- k_assign
template <bool BF16, int HG>
__global__ void __launch_bounds__(kAsgThreads) k_assign(DevState s, Dims d, const void* __restrict__ K,
                                                       int n)
{
    if (*(volatile int*)s.err) return;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float redw[32];
    __shared__ int redt[32], redi[32];
    __shared__ int e_tok[kMaxKappa], e_idx[kMaxKappa];
    __shared__ float e_w[kMaxKappa];
    __shared__ int s_c, s_ok, s_off, s_size;

    const int g = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int b, h0, kvh;
    graph_heads(d, g, b, h0, kvh);
    const int32_t* meta = s.meta + (int64_t)g * M_COUNT;
    const int T = meta[M_T];
    const int t = n - 1;
    const float* zrow = s.zrow + (int64_t)g * d.NM * HG;
    const int32_t* rtok = s.rtok + (int64_t)g * d.NM;
    const int32_t* rcomm = s.rcomm + (int64_t)g * d.NM;
    float M[HG], invL[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) {
        M[h] = s.ml[((int64_t)g * HG + h) * 2];
        invL[h] = 1.f / s.ml[((int64_t)g * HG + h) * 2 + 1];
    }
    // edge weights w_j = sum_h p_hj of the kept members (cached in shared
    // memory when they fit, else recomputed per round)
    float* ws = reinterpret_cast<float*>(smem);
    int* ts = reinterpret_cast<int*>(smem) + kSortCap * 4;
    const bool cached = (T <= kSortCap * 4);
    auto weight = [&](int i) -> float {
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < HG; ++h) acc += expf(zrow[(int64_t)i * HG + h] - M[h]) * invL[h];
        return acc;
    };
    if (cached) {
        for (int i = tid; i < T; i += kAsgThreads) { ws[i] = weight(i); ts[i] = rtok[i]; }
        __syncthreads();
    }
    // ---- top-kappa by (w desc, token asc): kappa rounds of block argmax
    // below the previous winner's key
    const int E = min(d.kappa, T);
    float pw = INFINITY;
    int ptk = -1;
    for (int k = 0; k < E; ++k) {
        float bw = -INFINITY;
        int bt = 0x7fffffff, bi = -1;
        for (int i = tid; i < T; i += kAsgThreads) {
            const float w = cached ? ws[i] : weight(i);
            const int tk = cached ? ts[i] : rtok[i];
            const bool below = (w < pw) || (w == pw && tk > ptk);
            const bool better = (w > bw) || (w == bw && tk < bt);
            if (below && better) { bw = w; bt = tk; bi = i; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ow = __shfl_xor_sync(kFull, bw, o);
            const int ot = __shfl_xor_sync(kFull, bt, o);
            const int oi = __shfl_xor_sync(kFull, bi, o);
            if (ow > bw || (ow == bw && ot < bt)) { bw = ow; bt = ot; bi = oi; }
        }
        if (lane == 0) { redw[warp] = bw; redt[warp] = bt; redi[warp] = bi; }
        __syncthreads();
        if (warp == 0) {
            const int nw = kAsgThreads / 32;
            bw = (lane < nw) ? redw[lane] : -INFINITY;
            bt = (lane < nw) ? redt[lane] : 0x7fffffff;
            bi = (lane < nw) ? redi[lane] : -1;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ow = __shfl_xor_sync(kFull, bw, o);
                const int ot = __shfl_xor_sync(kFull, bt, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                if (ow > bw || (ow == bw && ot < bt)) { bw = ow; bt = ot; bi = oi; }
            }
            if (lane == 0) { e_w[k] = bw; e_tok[k] = bt; e_idx[k] = bi; }
        }
        __syncthreads();
        pw = e_w[k];
        ptk = e_tok[k];
    }
    // ---- vote and capacity check (thread 0)
    const int32_t* csz = s.csize + (int64_t)g * d.Nc;
    int32_t* coff = s.coff + (int64_t)g * d.Nc;
    int32_t* ccap = s.ccap + (int64_t)g * d.Nc;
    if (tid == 0) {
        int ids[kMaxKappa];
        double v[kMaxKappa];
        int nd = 0;
        for (int e = 0; e < E; ++e) {
            const int c = rcomm[e_idx[e]];
            int k = 0;
            while (k < nd && ids[k] != c) ++k;
            if (k == nd) { ids[nd] = c; v[nd] = 0.0; ++nd; }
            v[k] += (double)e_w[e];
        }
        int best = -1;
        for (int k = 0; k < nd; ++k)
            if (best < 0 || v[k] > v[best] || (v[k] == v[best] && ids[k] < ids[best])) best = k;
        const int c = (best < 0) ? 0 : ids[best];
        const int size = csz[c], cp = ccap[c];
        int ok = 1, off = coff[c];
        if (size == cp) {
            const int ncap = max(16, 2 * cp);
            const int top = s.pool_top[g];
            if ((int64_t)top + ncap > d.P) ok = 0;
            else { s.pool_top[g] = top + ncap; off = top; }
        }
        s_c = c; s_ok = ok; s_off = off; s_size = size;
        if (!ok) set_error(s.err, CKV_ERR_CAPACITY);
    }
    __syncthreads();
    if (!s_ok) return;
    const int c = s_c, size = s_size, off = s_off;
    int32_t* pool = s.pool + (int64_t)g * d.P;
    const int old_off = coff[c];
    if (off != old_off) {   // relocate the full segment
        for (int i = tid; i < size; i += kAsgThreads) pool[off + i] = pool[old_off + i];
    }
    // running-mean update of the assigned centroid, double math rounded once
    const int64_t krow = (((int64_t)b * d.Hkv + kvh) * d.NM + t) * kD;
    float* mu = s.mu + ((int64_t)g * d.Nc + c) * kD;
    const double m1 = (double)(size + 1);
    for (int i = tid; i < kD; i += kAsgThreads) {
        const double mv = (double)mu[i];
        const double kv = (double)elem<BF16>(K, krow + i);
        mu[i] = __double2float_rn(__dadd_rn(mv, __ddiv_rn(__dsub_rn(kv, mv), m1)));
    }
    __syncthreads();
    if (tid == 0) {
        if (off != old_off) { coff[c] = off; ccap[c] = max(16, 2 * ccap[c]); }
        pool[off + size] = t;
        s.csize[(int64_t)g * d.Nc + c] = size + 1;
        s.tok_comm[(int64_t)g * d.NM + t] = c;
        int32_t* m = s.meta + (int64_t)g * M_COUNT;
        m[M_NEDGE] = E;
        m[M_ASSIGNED] = c;
        const int64_t row = (int64_t)g * (d.NM - d.n_init) + (t - d.n_init);
        s.edge_deg[row] = E;
        for (int e = 0; e < E; ++e) {
            s.edge_col[row * d.kappa + e] = e_tok[e];
            s.edge_w[row * d.kappa + e] = e_w[e];
            s.dbg_edges[(int64_t)g * d.kappa + e] = e_tok[e];
            s.dbg_w[(int64_t)g * d.kappa + e] = e_w[e];
        }
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

}  // namespace

size_t select_smem_bytes() { return sizeof(SelShared); }

cudaError_t launch_append_rows(const Dims& d, const void* knew, const void* vnew, void* K, void* V,
                               int row, cudaStream_t st)
{
    const int words = kD * (d.bf16 ? 2 : 4) / 4;
    k_append<<<d.B * d.Hkv, 64, 0, st>>>(static_cast<const uint32_t*>(knew), static_cast<const uint32_t*>(vnew),
                                         static_cast<uint32_t*>(K), static_cast<uint32_t*>(V), d.NM, row, words);
    return cudaGetLastError();
}

cudaError_t launch_score(const DevState& s, const Dims& d, const void* q, cudaStream_t st)
{
    dim3 grid((d.n_comm + 255) / 256, d.G);
    if (d.bf16) k_score<true><<<grid, 256, 0, st>>>(s, d, q);
    else k_score<false><<<grid, 256, 0, st>>>(s, d, q);
    return cudaGetLastError();
}

cudaError_t launch_select(const DevState& s, const Dims& d, int n, cudaStream_t st)
{
    k_select<<<d.G, kSelThreads, 0, st>>>(s, d, n);
    return cudaGetLastError();
}

cudaError_t launch_attend(const DevState& s, const Dims& d, const void* q, const void* K,
                          const void* V, int n, float* out, cudaStream_t st)
{
    return dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        dim3 grid(d.splits, d.G);
        if (d.bf16) {
            using L = AttLayout<true, HG>;
            auto kern = k_attend<true, HG>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes);
            if (e != cudaSuccess) return e;
            kern<<<grid, kAttThreads, L::bytes, st>>>(s, d, q, K, V, n, out);
        } else {
            using L = AttLayout<false, HG>;
            auto kern = k_attend<false, HG>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes);
            if (e != cudaSuccess) return e;
            kern<<<grid, kAttThreads, L::bytes, st>>>(s, d, q, K, V, n, out);
        }
        return cudaGetLastError();
    });
}

cudaError_t launch_assign(const DevState& s, const Dims& d, const void* K, int n, cudaStream_t st)
{
    const size_t smem = (size_t)kSortCap * 4 * 8;   // w (float) + token (int) of up to 4096 rows
    return dispatch_hg(d.HG, [&](auto hgc) -> cudaError_t {
        constexpr int HG = decltype(hgc)::value;
        auto kern = d.bf16 ? k_assign<true, HG> : k_assign<false, HG>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<d.G, kAsgThreads, smem, st>>>(s, d, K, n);
        return cudaGetLastError();
    });
}

}  // namespace ckv
