// k_modularity.cu -- modularity of a partition of the token graph, on the
// device.
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 3 (left): the graph modularity Q of the partition, tracked while
// tokens are generated.  The graph is the directed top-kappa CSR read as
// undirected (an edge i -> j of weight w adds w between i and j);
// Q = (in - gamma sum_c K_c^2 / (4m)) / m with m the total edge weight, in
// the weight of edges inside a community and K_c the summed degree of c.
// One pass over the edges (one thread per row, double atomics per
// community degree, block sums of m and in), then one CTA sums K_c^2 and
// writes Q.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "leiden.h"

namespace ckv {

namespace {

constexpr int kModThreads = 256;

__device__ __forceinline__ double block_sum(double x, double* red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) red[warp] = x;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0)
        for (int i = 0; i < kModThreads / 32; ++i) s += red[i];
    __syncthreads();
    return s;   // valid in thread 0
}

// scratch: [0] m, [1] in, [2] bad entries, [3 ..] K_c.  A label outside
// [0, nc) or a column outside [0, n) is counted as bad and skipped.
__global__ void __launch_bounds__(kModThreads) k_mod_edges(int n, int nc, const int64_t* __restrict__ row_ptr,
                                                           const int32_t* __restrict__ col,
                                                           const float* __restrict__ w,
                                                           const int32_t* __restrict__ labels, double* scratch)
{
    __shared__ double red[kModThreads / 32];
    double m = 0.0, in = 0.0;
    for (int i = blockIdx.x * kModThreads + threadIdx.x; i < n; i += gridDim.x * kModThreads) {
        const int li = labels[i];
        if (li < 0 || li >= nc) { atomicAdd(scratch + 2, 1.0); continue; }
        double ki = 0.0;
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
            const int j = col[e];
            if (j < 0 || j >= n) { atomicAdd(scratch + 2, 1.0); continue; }
            const double x = (double)w[e];
            const int lj = labels[j];
            if (lj < 0 || lj >= nc) { atomicAdd(scratch + 2, 1.0); continue; }
            m += x;
            ki += x;
            atomicAdd(scratch + 3 + lj, x);
            if (lj == li) in += x;
        }
        if (ki != 0.0) atomicAdd(scratch + 3 + li, ki);
    }
    const double bm = block_sum(m, red);
    const double bi = block_sum(in, red);
    if (threadIdx.x == 0) {
        atomicAdd(scratch, bm);
        atomicAdd(scratch + 1, bi);
    }
}

__global__ void __launch_bounds__(kModThreads) k_mod_final(int nc, double gamma, const double* __restrict__ scratch,
                                                           double* q_out)
{
    __shared__ double red[kModThreads / 32];
    double kk = 0.0;
    for (int c = threadIdx.x; c < nc; c += kModThreads) kk += scratch[3 + c] * scratch[3 + c];
    const double s = block_sum(kk, red);
    if (threadIdx.x == 0) {
        const double m = scratch[0];
        // a bad label or column makes the result NaN
        *q_out = (scratch[2] != 0.0) ? __longlong_as_double(0x7ff8000000000000ll)
                                     : (m > 0.0) ? (scratch[1] - gamma * s / (4.0 * m)) / m : 0.0;
    }
}

}  // namespace

size_t modularity_scratch_doubles(int n_communities) { return (size_t)n_communities + 4; }

cudaError_t launch_modularity(int n, const int64_t* row_ptr, const int32_t* col, const float* w,
                              const int32_t* labels, int n_communities, double gamma, double* scratch,
                              double* q_out, cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(scratch, 0, modularity_scratch_doubles(n_communities) * sizeof(double), st);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int blocks = std::max(1, std::min(4 * sms, (n + kModThreads - 1) / kModThreads));
    k_mod_edges<<<blocks, kModThreads, 0, st>>>(n, n_communities, row_ptr, col, w, labels, scratch);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_mod_final<<<1, kModThreads, 0, st>>>(n_communities, gamma, scratch, q_out);
    return cudaGetLastError();
}

}  // namespace ckv
