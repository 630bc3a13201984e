// k_dense.cu -- dense decode attention statistics over a whole KV cache.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 3 (right): the attention-mass recall of the retrieved set, i.e.
// per query head the share of the dense softmax mass over every cached
// position that falls on the rows a decode step attended.  The decode
// step's attention kernel leaves (m, l) of its attended rows per head; this
// kernel supplies the dense (m, l) over [0, n) and divides:
//     recall = l_sel * exp(m_sel - m) / l.
// With V it is also a plain dense decode attention (o / l and the
// log-sum-exp per head), the comparator the sparse step is timed against.
//
// Work split: one unit per (batch, KV head), streamed once for all the
// query heads of its group.  The units' tiles (4 KB of K: 16 bf16 rows or
// 8 fp32 rows) are laid end to end and split evenly over a co-resident
// grid; a CTA's share is one or more pieces (a run of one unit's tiles).
// Every warp streams every 8th tile of the piece through its own 16-byte
// cp.async ring; bf16 logits come from mma.sync (the K tile as A, the
// unit's queries as B, fp32 accumulation), fp32 logits from FMAs and a
// butterfly transpose-reduce.  A piece's (m, l[, o]) per head goes to a
// slot of its own; the unit's last piece to arrive merges the slots.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ckv_internal.cuh"
#include "dev_async.cuh"
#include "warp_mma.cuh"

namespace ckv {

namespace {

constexpr int kDnWarps = 8;
constexpr int kDnThreads = kDnWarps * 32;
constexpr int kDnBuf = 3;          // tiles in flight per warp ring
constexpr int kTileBytes = 4096;   // bytes of K (and of V) per tile
constexpr float kScale = 0.08838834764831845f;   // 1 / sqrt(128)

struct DenseArgs {
    const void* q;         // [B][Hq][D]
    const char* K;         // [B][Hkv][NM][D]
    const char* V;         // same layout, or null (statistics only)
    int n, B, Hq, Hkv, NH, NM;
    int TU;                // tiles per unit
    long long TT;          // tiles of all units
    float* part;           // [U + grid][NH][PSTR] piece slots
    unsigned* cnt;         // [U] arrivals (reset by the last piece)
    float* out;            // [B][Hq][D] o / l (with V)
    float* lse;            // [B][Hq] m + log l, or null
    const float* sel_ml;   // [B][Hq][2] (m, l) of the step's attended rows, or null
    float* recall;         // [B][Hq], or null
};

// the CTA whose share [lo(p), lo(p+1)), lo(p) = p * TT / P, holds tile x
__device__ __forceinline__ int owner_of(long long x, long long TT, int P)
{
    return (int)(((x + 1) * (long long)P - 1) / TT);
}

// merge (m2, l2) into (m, l); -inf marks an empty side
__device__ __forceinline__ void ml_merge(float& m, float& l, float m2, float l2)
{
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) { m = m2; l = l2; return; }
    const float mn = fmaxf(m, m2);
    l = l * __expf(m - mn) + l2 * __expf(m2 - mn);
    m = mn;
}

// ---- bf16: 16-row tiles on the tensor cores -----------------------------
// Lane (gid, tig) holds the logits of rows gid and gid + 8 of a tile for
// heads 8 ht + 2 tig and + 1.  Without V each lane keeps its own running
// (m, l) per head; with V (one head tile) the max is shared by the 8 lanes
// of a head column so that P can feed the P.V contraction.
template <int NHT, bool WV>
__device__ __forceinline__ void warp_tiles_bf16(const char* __restrict__ Kb, const char* __restrict__ Vb, int n,
                                                int t0, int t1, const uint32_t (&qf)[NHT][8][2],
                                                unsigned char* wbuf, float (&m)[NHT][2], float (&l)[NHT][2],
                                                float (&acc)[8][4])
{
    constexpr int STAGE = WV ? 2 * kTileBytes : kTileBytes;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gid = lane >> 2;
    const int first = t0 + warp;
    const int nb = (t1 > first) ? (t1 - first + kDnWarps - 1) / kDnWarps : 0;
    const uint64_t pol = l2_evict_first();   // the cache is streamed once
    auto issue = [&](int bb) {
        if (bb < nb) {
            const uint32_t dst = smem_u32(wbuf + (bb % kDnBuf) * STAGE);
            const int rbase = 16 * (first + bb * kDnWarps);
            const int ch = lane & 15;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = 2 * i + (lane >> 4);
                const bool ok = rbase + row < n;
                const int64_t src = ok ? (int64_t)(rbase + row) * 256 + ch * 16 : 0;
                const uint32_t so = row * 256 + ((ch ^ (row & 7)) << 4);
                cp_async16z_ef(dst + so, Kb + src, ok, pol);
                if (WV) cp_async16z_ef(dst + kTileBytes + so, Vb + src, ok, pol);
            }
        }
        cp_async_commit();
    };
    const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, khi = lane >> 4;
    const int vrow = (lane & 7) + (lane >> 4) * 8, vhi = (lane >> 3) & 1;
#pragma unroll
    for (int i = 0; i < kDnBuf - 1; ++i) issue(i);
    for (int bb = 0; bb < nb; ++bb) {
        issue(bb + kDnBuf - 1);
        cp_async_wait<kDnBuf - 1>();
        __syncwarp();
        const uint32_t kt = smem_u32(wbuf + (bb % kDnBuf) * STAGE);
        const int rbase = 16 * (first + bb * kDnWarps);
        float sc[NHT][4];
#pragma unroll
        for (int ht = 0; ht < NHT; ++ht)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[ht][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t fa[4];
            ldsm4(kt + krow * 256 + (((2 * ks + khi) ^ (krow & 7)) << 4), fa);
#pragma unroll
            for (int ht = 0; ht < NHT; ++ht) mma_bf16(sc[ht], fa, qf[ht][ks][0], qf[ht][ks][1]);
        }
        const bool va = rbase + gid < n, vb = rbase + gid + 8 < n;
        if constexpr (!WV) {
#pragma unroll
            for (int ht = 0; ht < NHT; ++ht)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float za = va ? sc[ht][j] * kScale : -INFINITY;
                    const float zb = vb ? sc[ht][2 + j] * kScale : -INFINITY;
                    const float mn = fmaxf(m[ht][j], fmaxf(za, zb));
                    if (mn == -INFINITY) continue;
                    const float al = (m[ht][j] == -INFINITY) ? 0.f : __expf(m[ht][j] - mn);
                    const float pa = (za == -INFINITY) ? 0.f : __expf(za - mn);
                    const float pb = (zb == -INFINITY) ? 0.f : __expf(zb - mn);
                    l[ht][j] = fmaf(l[ht][j], al, pa + pb);
                    m[ht][j] = mn;
                }
        } else {
            float z[4], p[4];
            z[0] = va ? sc[0][0] * kScale : -INFINITY;
            z[1] = va ? sc[0][1] * kScale : -INFINITY;
            z[2] = vb ? sc[0][2] * kScale : -INFINITY;
            z[3] = vb ? sc[0][3] * kScale : -INFINITY;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float t = fmaxf(z[j], z[2 + j]);
                t = fmaxf(t, __shfl_xor_sync(kFull, t, 4));
                t = fmaxf(t, __shfl_xor_sync(kFull, t, 8));
                t = fmaxf(t, __shfl_xor_sync(kFull, t, 16));
                const float mn = fmaxf(m[0][j], t);   // finite: a tile has a valid row
                const float al = (m[0][j] == -INFINITY) ? 0.f : __expf(m[0][j] - mn);
                p[j] = (z[j] == -INFINITY) ? 0.f : __expf(z[j] - mn);
                p[2 + j] = (z[2 + j] == -INFINITY) ? 0.f : __expf(z[2 + j] - mn);
                l[0][j] = fmaf(l[0][j], al, p[j] + p[2 + j]);
                m[0][j] = mn;
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
            const uint32_t vt = kt + kTileBytes;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t fv[4];
                ldsm4t(vt + vrow * 256 + (((2 * mt + vhi) ^ (vrow & 7)) << 4), fv);
                mma_bf16(acc[mt], fv, bh0, bh1);
                mma_bf16(acc[mt], fv, bl0, bl1);
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    __syncwarp();
}

// ---- fp32: 8-row tiles on the CUDA cores --------------------------------
// Lane = 4 dims.  Each half tile's 4 rows x NHP heads partial dots are
// summed by one transpose-reduce; the logits go through the warp's pz
// window so that every lane holds every row's logit and the per-head
// running (m, l) is the same in all lanes.
template <int NHP, bool WV>
__device__ __forceinline__ void warp_tiles_f32(const char* __restrict__ Kb, const char* __restrict__ Vb, int n,
                                               int t0, int t1, const float (&qv)[NHP][4], unsigned char* wbuf,
                                               float* pz, float (&m)[NHP], float (&l)[NHP], float (&acc)[NHP][4])
{
    constexpr int STAGE = WV ? 2 * kTileBytes : kTileBytes;
    constexpr int NV = 4 * NHP;
    constexpr int lowmask = (NV >= 32) ? 0 : (32 / NV) - 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int first = t0 + warp;
    const int nb = (t1 > first) ? (t1 - first + kDnWarps - 1) / kDnWarps : 0;
    const uint64_t pol = l2_evict_first();   // the cache is streamed once
    auto issue = [&](int bb) {
        if (bb < nb) {
            const uint32_t dst = smem_u32(wbuf + (bb % kDnBuf) * STAGE);
            const int rbase = 8 * (first + bb * kDnWarps);
#pragma unroll
            for (int row = 0; row < 8; ++row) {
                const bool ok = rbase + row < n;
                const int64_t src = ok ? (int64_t)(rbase + row) * 512 + lane * 16 : 0;
                cp_async16z_ef(dst + row * 512 + lane * 16, Kb + src, ok, pol);
                if (WV) cp_async16z_ef(dst + kTileBytes + row * 512 + lane * 16, Vb + src, ok, pol);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < kDnBuf - 1; ++i) issue(i);
    for (int bb = 0; bb < nb; ++bb) {
        issue(bb + kDnBuf - 1);
        cp_async_wait<kDnBuf - 1>();
        __syncwarp();
        const unsigned char* kt = wbuf + (bb % kDnBuf) * STAGE;
        const int rbase = 8 * (first + bb * kDnWarps);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[NV];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float4 w = *reinterpret_cast<const float4*>(kt + (4 * half + r) * 512 + 16 * lane);
#pragma unroll
                for (int h = 0; h < NHP; ++h)
                    v[r * NHP + h] = fmaf(qv[h][3], w.w, fmaf(qv[h][2], w.z, fmaf(qv[h][1], w.y, qv[h][0] * w.x)));
            }
            const float z = transpose_reduce<NV>(v, lane) * kScale;
            const int idx = tr_index<NV>(lane);
            if ((lane & lowmask) == 0) {
                const int r = 4 * half + idx / NHP;
                pz[r * NHP + idx % NHP] = (rbase + r < n) ? z : -INFINITY;
            }
        }
        __syncwarp();
        float pb[8][NHP];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int h = 0; h < NHP; ++h) pb[r][h] = pz[r * NHP + h];
#pragma unroll
        for (int h = 0; h < NHP; ++h) {
            float mb = pb[0][h];   // row 0 of a tile is always valid
#pragma unroll
            for (int r = 1; r < 8; ++r) mb = fmaxf(mb, pb[r][h]);
            const float mn = fmaxf(m[h], mb);
            const float al = (m[h] == -INFINITY) ? 0.f : __expf(m[h] - mn);
            l[h] *= al;
            if (WV)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h][e] *= al;
            m[h] = mn;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                pb[r][h] = (pb[r][h] == -INFINITY) ? 0.f : __expf(pb[r][h] - mn);
                l[h] += pb[r][h];
            }
        }
        if (WV) {
            const unsigned char* vt = kt + kTileBytes;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float4 w = *reinterpret_cast<const float4*>(vt + r * 512 + 16 * lane);
#pragma unroll
                for (int h = 0; h < NHP; ++h) {
                    acc[h][0] = fmaf(pb[r][h], w.x, acc[h][0]);
                    acc[h][1] = fmaf(pb[r][h], w.y, acc[h][1]);
                    acc[h][2] = fmaf(pb[r][h], w.z, acc[h][2]);
                    acc[h][3] = fmaf(pb[r][h], w.w, acc[h][3]);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    __syncwarp();
}

// ---- the kernel ----------------------------------------------------------
// NHX: head tiles of 8 (bf16) or padded heads (fp32) held per unit.
template <bool BF16, int NHX, bool WV>
struct DenseLayout {
    static constexpr int STAGE = WV ? 2 * kTileBytes : kTileBytes;
    static constexpr int WBUF = kDnBuf * STAGE;                  // one warp's ring
    static constexpr int NHMAX = BF16 ? 8 * NHX : NHX;          // heads per unit, padded
    static constexpr int RSTR = WV ? kD + 4 : 2;                 // warp result row: [o[D],] m, l
    static constexpr int off_pz = kDnWarps * WBUF;               // fp32 logits window [warps][64]
    static constexpr int off_flag = off_pz + kDnWarps * 64 * 4;
    static constexpr int bytes = off_flag + 16;
    static_assert(kDnWarps * NHMAX * RSTR * 4 <= kDnWarps * WBUF, "warp results must fit the rings");
};

template <bool BF16, int NHX, bool WV>
__global__ void __launch_bounds__(kDnThreads, WV ? 1 : 2) k_dense(DenseArgs a)
{
    using L = DenseLayout<BF16, NHX, WV>;
    constexpr int NHMAX = L::NHMAX, RSTR = L::RSTR;
    constexpr int PSTR = WV ? 2 + kD : 2;                        // slot row per head: m, l[, o[D]]
    constexpr int MOFF = WV ? kD : 0;                            // m, l in a warp result row
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    unsigned char* wbuf = smem + warp * L::WBUF;
    float* pz = reinterpret_cast<float*>(smem + L::off_pz) + warp * 64;
    int* sflag = reinterpret_cast<int*>(smem + L::off_flag);
    float* red = reinterpret_cast<float*>(smem);                 // overlays the rings after a barrier
    const int P = gridDim.x, p = blockIdx.x;
    const long long lo = (long long)p * a.TT / P, hi = (long long)(p + 1) * a.TT / P;
    constexpr int ESZ = BF16 ? 2 : 4;

    for (long long x = lo; x < hi;) {
        // ---- one piece: tiles [t0, t1) of unit u
        const int u = (int)(x / a.TU);
        const long long ue = (long long)(u + 1) * a.TU;
        const long long xe = hi < ue ? hi : ue;
        const int t0 = (int)(x - (long long)u * a.TU), t1 = (int)(xe - (long long)u * a.TU);
        x = xe;
        const int b = u / a.Hkv, kvh = u % a.Hkv;
        const int64_t ubase = (int64_t)u * a.NM * kD * ESZ;      // u = b * Hkv + kvh
        const char* Kb = a.K + ubase;
        const char* Vb = WV ? a.V + ubase : nullptr;
        const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * a.NH;   // the unit's first query head

        if constexpr (BF16) {
            uint32_t qf[NHX][8][2];
            const uint32_t* q2 = static_cast<const uint32_t*>(a.q);
#pragma unroll
            for (int ht = 0; ht < NHX; ++ht) {
                const int h = 8 * ht + gid;
                const bool ok = h < a.NH;
                const int64_t base = (qrow0 + h) * kD;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    qf[ht][ks][0] = ok ? q2[(base + 16 * ks + 2 * tig) / 2] : 0u;
                    qf[ht][ks][1] = ok ? q2[(base + 16 * ks + 2 * tig + 8) / 2] : 0u;
                }
            }
            float m[NHX][2], l[NHX][2], acc[8][4];
#pragma unroll
            for (int ht = 0; ht < NHX; ++ht) { m[ht][0] = m[ht][1] = -INFINITY; l[ht][0] = l[ht][1] = 0.f; }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
            warp_tiles_bf16<NHX, WV>(Kb, Vb, a.n, t0, t1, qf, wbuf, m, l, acc);
            // the 8 lanes of a head column -> one (m, l) per head
#pragma unroll
            for (int ht = 0; ht < NHX; ++ht)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int off = 4; off <= 16; off <<= 1) {
                        const float m2 = __shfl_xor_sync(kFull, m[ht][j], off);
                        const float l2 = __shfl_xor_sync(kFull, l[ht][j], off);
                        if (WV) l[ht][j] += l2;                  // the max is already shared
                        else ml_merge(m[ht][j], l[ht][j], m2, l2);
                    }
                }
            __syncthreads();   // every ring is drained: red overlays them
#pragma unroll
            for (int ht = 0; ht < NHX; ++ht)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = 8 * ht + 2 * tig + j;
                    float* rw = red + (warp * NHMAX + h) * RSTR;
                    if (WV) {
#pragma unroll
                        for (int mt = 0; mt < 8; ++mt) {
                            rw[16 * mt + gid] = acc[mt][j];
                            rw[16 * mt + gid + 8] = acc[mt][2 + j];
                        }
                    }
                    if (gid == 0) { rw[MOFF] = m[ht][j]; rw[MOFF + 1] = l[ht][j]; }
                }
        } else {
            float qv[NHX][4];
            const float* qf = static_cast<const float*>(a.q);
#pragma unroll
            for (int h = 0; h < NHX; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j) qv[h][j] = (h < a.NH) ? qf[(qrow0 + h) * kD + 4 * lane + j] : 0.f;
            float m[NHX], l[NHX], acc[NHX][4];
#pragma unroll
            for (int h = 0; h < NHX; ++h) {
                m[h] = -INFINITY;
                l[h] = 0.f;
                acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
            }
            warp_tiles_f32<NHX, WV>(Kb, Vb, a.n, t0, t1, qv, wbuf, pz, m, l, acc);
            __syncthreads();   // every ring is drained: red overlays them
#pragma unroll
            for (int h = 0; h < NHX; ++h) {
                float* rw = red + (warp * NHMAX + h) * RSTR;
                if (WV) *reinterpret_cast<float4*>(rw + 4 * lane) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
                if (lane == 0) { rw[MOFF] = m[h]; rw[MOFF + 1] = l[h]; }
            }
        }
        __syncthreads();
        // ---- the piece's slot: the 8 warps merged per head
        float* slot = a.part + (int64_t)(u + p) * a.NH * PSTR;
        if (!WV) {
            for (int h = tid; h < a.NH; h += kDnThreads) {
                float M = -INFINITY, Ls = 0.f;
#pragma unroll
                for (int w = 0; w < kDnWarps; ++w) ml_merge(M, Ls, red[(w * NHMAX + h) * RSTR + MOFF], red[(w * NHMAX + h) * RSTR + MOFF + 1]);
                slot[h * PSTR] = M;
                slot[h * PSTR + 1] = Ls;
            }
        } else {
            for (int i = tid; i < a.NH * kD; i += kDnThreads) {
                const int h = i / kD, dd = i % kD;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kDnWarps; ++w) M = fmaxf(M, red[(w * NHMAX + h) * RSTR + kD]);
                float o = 0.f, Ls = 0.f;
#pragma unroll
                for (int w = 0; w < kDnWarps; ++w) {
                    const float* rw = red + (w * NHMAX + h) * RSTR;
                    if (rw[kD] == -INFINITY) continue;           // a warp without tiles
                    const float c = __expf(rw[kD] - M);
                    o = fmaf(rw[dd], c, o);
                    Ls = fmaf(rw[kD + 1], c, Ls);
                }
                slot[h * PSTR + 2 + dd] = o;
                if (dd == 0) { slot[h * PSTR] = M; slot[h * PSTR + 1] = Ls; }
            }
        }
        __threadfence();
        __syncthreads();
        // ---- arrival; the unit's last piece merges every slot
        const int pf = owner_of((long long)u * a.TU, a.TT, P), pl = owner_of(ue - 1, a.TT, P);
        if (tid == 0) {
            const unsigned old = atomicAdd(a.cnt + u, 1u);
            sflag[0] = (old == (unsigned)(pl - pf)) ? 1 : 0;
        }
        __syncthreads();
        if (sflag[0]) {
            __threadfence();
            const int ns = pl - pf + 1;
            const float* s0 = a.part + (int64_t)(u + pf) * a.NH * PSTR;   // slots u+pf .. u+pl
            if (!WV) {
                for (int h = warp; h < a.NH; h += kDnWarps) {
                    float M = -INFINITY, Ls = 0.f;
                    for (int j = lane; j < ns; j += 32) {
                        const float2 v = __ldcg(reinterpret_cast<const float2*>(s0 + ((int64_t)j * a.NH + h) * PSTR));
                        ml_merge(M, Ls, v.x, v.y);
                    }
#pragma unroll
                    for (int off = 16; off; off >>= 1) {
                        const float m2 = __shfl_xor_sync(kFull, M, off), l2 = __shfl_xor_sync(kFull, Ls, off);
                        ml_merge(M, Ls, m2, l2);
                    }
                    if (lane == 0) {
                        const int64_t hq = qrow0 + h;
                        if (a.lse) a.lse[hq] = M + logf(Ls);
                        if (a.recall) a.recall[hq] = a.sel_ml[2 * hq + 1] * expf(a.sel_ml[2 * hq] - M) / Ls;
                    }
                }
            } else {
                for (int i = tid; i < a.NH * kD; i += kDnThreads) {
                    const int h = i / kD, dd = i % kD;
                    float M = -INFINITY, Ls = 0.f, o = 0.f;
                    for (int j = 0; j < ns; ++j) {
                        const float* sj = s0 + ((int64_t)j * a.NH + h) * PSTR;
                        const float mj = __ldcg(sj), lj = __ldcg(sj + 1), oj = __ldcg(sj + 2 + dd);
                        if (mj == -INFINITY) continue;
                        const float mn = fmaxf(M, mj);
                        const float al = (M == -INFINITY) ? 0.f : __expf(M - mn), c = __expf(mj - mn);
                        o = o * al + oj * c;
                        Ls = Ls * al + lj * c;
                        M = mn;
                    }
                    const int64_t hq = qrow0 + h;
                    a.out[hq * kD + dd] = o / Ls;
                    if (dd == 0) {
                        if (a.lse) a.lse[hq] = M + logf(Ls);
                        if (a.recall) a.recall[hq] = a.sel_ml[2 * hq + 1] * expf(a.sel_ml[2 * hq] - M) / Ls;
                    }
                }
            }
            if (tid == 0) a.cnt[u] = 0;
        }
        __syncthreads();   // sflag and red are reused by the next piece
    }
}

template <bool BF16, int NHX, bool WV>
cudaError_t launch_dense_t(DenseArgs a, int max_ctas, cudaStream_t st)
{
    using L = DenseLayout<BF16, NHX, WV>;
    auto fn = k_dense<BF16, NHX, WV>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes);
    if (e != cudaSuccess) return e;
    int per_sm = 0, dev = 0, sms = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kDnThreads, L::bytes)) != cudaSuccess) return e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long P = (long long)per_sm * sms;
    if (P > max_ctas) P = max_ctas;
    if (P > a.TT) P = a.TT;
    fn<<<(unsigned)P, kDnThreads, L::bytes, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool dense_supported(const Dims& d, bool with_v)
{
    const int NH = d.Gq;
    if (with_v) return NH <= 8;
    return d.bf16 ? NH <= 32 : NH <= 8;
}

size_t dense_part_floats(const Dims& d)
{
    const size_t U = (size_t)d.B * d.Hkv, NH = d.Gq;
    const size_t per_slot = NH <= 8 ? NH * (2 + kD) : NH * 2;
    return (U + (size_t)kDenseMaxCtasPerSM * d.nSM) * per_slot;
}

cudaError_t launch_dense(const Dims& d, const void* q, const void* K, const void* V, int n, float* part,
                         unsigned* cnt, const DenseIO& io, cudaStream_t st)
{
    if (!dense_supported(d, V != nullptr) || n < 1 || n > d.NM) return cudaErrorInvalidValue;
    DenseArgs a;
    a.q = q;
    a.K = static_cast<const char*>(K);
    a.V = static_cast<const char*>(V);
    a.n = n;
    a.B = d.B;
    a.Hq = d.Hq;
    a.Hkv = d.Hkv;
    a.NH = d.Gq;
    a.NM = d.NM;
    a.TU = d.bf16 ? (n + 15) / 16 : (n + 7) / 8;
    a.TT = (long long)d.B * d.Hkv * a.TU;
    a.part = part;
    a.cnt = cnt;
    a.out = io.out;
    a.lse = io.lse;
    a.sel_ml = io.sel_ml;
    a.recall = io.recall;
    const int maxc = kDenseMaxCtasPerSM * d.nSM;
    const int NH = d.Gq;
    const bool wv = V != nullptr;
    if (d.bf16) {
        if (wv) return launch_dense_t<true, 1, true>(a, maxc, st);
        if (NH <= 8) return launch_dense_t<true, 1, false>(a, maxc, st);
        if (NH <= 16) return launch_dense_t<true, 2, false>(a, maxc, st);
        return launch_dense_t<true, 4, false>(a, maxc, st);
    }
    if (NH <= 1) return wv ? launch_dense_t<false, 1, true>(a, maxc, st) : launch_dense_t<false, 1, false>(a, maxc, st);
    if (NH <= 2) return wv ? launch_dense_t<false, 2, true>(a, maxc, st) : launch_dense_t<false, 2, false>(a, maxc, st);
    if (NH <= 4) return wv ? launch_dense_t<false, 4, true>(a, maxc, st) : launch_dense_t<false, 4, false>(a, maxc, st);
    return wv ? launch_dense_t<false, 8, true>(a, maxc, st) : launch_dense_t<false, 8, false>(a, maxc, st);
}

}  // namespace ckv
