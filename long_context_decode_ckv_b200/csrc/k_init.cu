// k_init.cu -- initial community state from a partition label array.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 1 caption, step (2) Initial Partitioning: the token graph is
// partitioned into communities and a centroid is computed per community.
// Here the partition arrives as one label per position; sinks (positions
// [0, S)) belong to no community.  Members are stored ascending in a
// per-graph pool with `slack` spare slots per community; each centroid is
// the mean of its members' keys, summed in double in ascending position
// order and rounded once to float.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ckv_internal.cuh"

namespace ckv {

namespace {

constexpr unsigned kFull = 0xffffffffu;

// sizes and the position -> community map; rejects labels out of range
__global__ void k_init_count(DevState s, Dims d, const int32_t* __restrict__ labels, int n)
{
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)d.G * n) return;
    const int g = (int)(idx / n), j = (int)(idx % n);
    if (j < d.S) return;
    const int c = labels[idx];
    if (c < 0 || c >= d.n_comm) {
        set_error(s.err, CKV_ERR_INVALID_ARG);
        return;
    }
    atomicAdd(&s.csize[(int64_t)g * d.Nc + c], 1);
    s.tok_comm[(int64_t)g * d.NM + j] = c;
}

// segment layout: capacity = size + slack, offsets by exclusive scan in id order
__global__ void __launch_bounds__(1024) k_init_layout(DevState s, Dims d, int slack)
{
    __shared__ int warp_sums[32];
    __shared__ long long carry;
    const int g = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < d.n_comm; base += 1024) {
        const int c = base + tid;
        const int cap = (c < d.n_comm) ? s.csize[(int64_t)g * d.Nc + c] + slack : 0;
        int v = cap;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(kFull, v, o);
            if (lane >= o) v += t;
        }
        if (lane == 31) warp_sums[warp] = v;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(kFull, w, o);
                if (lane >= o) w += t;
            }
            warp_sums[lane] = w;
        }
        __syncthreads();
        const long long excl = carry + (warp ? warp_sums[warp - 1] : 0) + v - cap;
        if (c < d.n_comm) {
            s.coff[(int64_t)g * d.Nc + c] = (int32_t)excl;
            s.ccap[(int64_t)g * d.Nc + c] = cap;
        }
        __syncthreads();
        if (tid == 0) carry += warp_sums[31];
        __syncthreads();
    }
    if (tid == 0) {
        if (carry > d.P) set_error(s.err, CKV_ERR_CAPACITY);
        s.pool_top[g] = (int32_t)(carry > d.P ? d.P : carry);
    }
}

// members in ascending position: one warp per graph walks the positions in
// order, 32 at a time; lanes with the same label get consecutive slots
__global__ void k_init_fill(DevState s, Dims d, const int32_t* __restrict__ labels, int n)
{
    const int g = blockIdx.x, lane = threadIdx.x;
    int32_t* csz = s.csize + (int64_t)g * d.Nc;      // reused as the fill counter
    const int32_t* coff = s.coff + (int64_t)g * d.Nc;
    int32_t* pool = s.pool + (int64_t)g * d.P;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = d.S; base < n; base += 32) {
        const int j = base + lane;
        const int c = (j < n) ? labels[(int64_t)g * n + j] : -1;
        const unsigned grp = __match_any_sync(kFull, c);
        const int leader = __ffs(grp) - 1;
        const int rank = __popc(grp & lt);
        int have = 0;
        if (lane == leader && c >= 0) have = csz[c];
        const int first = __shfl_sync(kFull, have, leader);
        if (c >= 0) {
            pool[coff[c] + first + rank] = j;
            if (lane == leader) csz[c] = first + __popc(grp);
        }
        __syncwarp();
    }
}

// centroid = mean of member keys: one warp per community, 4 dims per lane
template <bool BF16>
__global__ void __launch_bounds__(256) k_init_centroids(DevState s, Dims d, const void* __restrict__ K)
{
    const int g = blockIdx.y;
    const int c = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (c >= d.n_comm) return;
    int b, kvh;
    if (d.mode == CKV_QUERY_GROUP) { b = g / d.Hkv; kvh = g % d.Hkv; }
    else { b = g / d.Hq; kvh = (g % d.Hq) / d.Gq; }
    const int64_t gi = (int64_t)g * d.Nc + c;
    const int size = s.csize[gi];
    const int off = s.coff[gi];
    const int32_t* pool = s.pool + (int64_t)g * d.P;
    const int64_t rowbase = ((int64_t)b * d.Hkv + kvh) * d.NM;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int r = 0; r < size; ++r) {
        const int64_t j = pool[off + r];
        const int64_t e = (rowbase + j) * kD + 4 * lane;
        if (BF16) {
            const uint2 w = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(K) + e);
            acc[0] = __dadd_rn(acc[0], (double)__uint_as_float(w.x << 16));
            acc[1] = __dadd_rn(acc[1], (double)__uint_as_float(w.x & 0xffff0000u));
            acc[2] = __dadd_rn(acc[2], (double)__uint_as_float(w.y << 16));
            acc[3] = __dadd_rn(acc[3], (double)__uint_as_float(w.y & 0xffff0000u));
        } else {
            const float4 w = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(K) + e);
            acc[0] = __dadd_rn(acc[0], (double)w.x);
            acc[1] = __dadd_rn(acc[1], (double)w.y);
            acc[2] = __dadd_rn(acc[2], (double)w.z);
            acc[3] = __dadd_rn(acc[3], (double)w.w);
        }
    }
    float4 m;
    if (size > 0) {
        const double sz = (double)size;
        m = make_float4(__double2float_rn(__ddiv_rn(acc[0], sz)), __double2float_rn(__ddiv_rn(acc[1], sz)),
                        __double2float_rn(__ddiv_rn(acc[2], sz)), __double2float_rn(__ddiv_rn(acc[3], sz)));
    } else {
        m = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    reinterpret_cast<float4*>(s.mu + gi * kD)[lane] = m;
}

}  // namespace

cudaError_t launch_init_count(const DevState& s, const Dims& d, const int32_t* labels, int n,
                              cudaStream_t st)
{
    const int64_t total = (int64_t)d.G * n;
    if (total == 0) return cudaSuccess;
    k_init_count<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(s, d, labels, n);
    return cudaGetLastError();
}

cudaError_t launch_init_layout(const DevState& s, const Dims& d, int slack, cudaStream_t st)
{
    k_init_layout<<<d.G, 1024, 0, st>>>(s, d, slack);
    return cudaGetLastError();
}

cudaError_t launch_init_fill(const DevState& s, const Dims& d, const int32_t* labels, int n,
                             cudaStream_t st)
{
    k_init_fill<<<d.G, 32, 0, st>>>(s, d, labels, n);
    return cudaGetLastError();
}

cudaError_t launch_init_centroids(const DevState& s, const Dims& d, const void* K, cudaStream_t st)
{
    dim3 grid((d.n_comm + 7) / 8, d.G);
    if (d.bf16) k_init_centroids<true><<<grid, 256, 0, st>>>(s, d, K);
    else k_init_centroids<false><<<grid, 256, 0, st>>>(s, d, K);
    return cudaGetLastError();
}

}  // namespace ckv
