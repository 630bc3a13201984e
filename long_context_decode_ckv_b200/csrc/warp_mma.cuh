// warp_mma.cuh -- warp-level sm_100a helpers shared by the decode-step and
// dense-statistics kernels: 16-byte asynchronous copies into shared memory,
// ldmatrix / movmatrix, the bf16 m16n8k16 tensor-core MMA with fp32
// accumulation, bf16 packing, and a butterfly transpose-reduce.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dev_async.cuh"

namespace ckv {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
// 16 bytes, or 16 zero bytes when !valid (nothing is read then)
__device__ __forceinline__ void cp_async16z(uint32_t dst, const void* src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
// L2 policy "evict first" for data read once per step from a stream far
// larger than L2 (centroids, gathered K/V rows): those lines go first, so
// the stream does not push out what the step reuses (its scratch, the
// community index, the kernels' own code)
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
    return p;
}
__device__ __forceinline__ void cp_async16z_ef(uint32_t dst, const void* src, bool valid, uint64_t pol)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// four 8x8 b16 matrices; lanes 8i..8i+7 give the row addresses of matrix i
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// c += a . b  (16x16 bf16, row-major) x (16x8 bf16, column-major), fp32
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// transpose of the warp's 8x8 b16 matrix held in fragment layout
__device__ __forceinline__ uint32_t movtrans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}
// (lo, hi) -> bf16 pair, round to nearest even; lo in the low half
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Butterfly transpose-reduce of NV values per lane (NV a power of two
// <= 32): afterwards every lane holds the warp-wide sum of value index
// tr_index<NV>(lane); lanes that differ only in the bits below the last
// halving offset hold the same value.
template <int NV>
__device__ __forceinline__ int tr_index(int lane)
{
    int idx = 0;
#pragma unroll
    for (int s = 0, len = NV; len > 1; ++s, len >>= 1)
        idx += ((lane >> (4 - s)) & 1) * (len >> 1);
    return idx;
}

template <int NV>
__device__ __forceinline__ float transpose_reduce(float (&v)[NV], int lane)
{
#pragma unroll
    for (int s = 0, len = NV; len > 1; ++s, len >>= 1) {
        const int off = 16 >> s;
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < (len >> 1); ++i) {
            const float send = up ? v[i] : v[i + (len >> 1)];
            const float keep = up ? v[i + (len >> 1)] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, off);
        }
    }
    float r = v[0];
    constexpr int levels = (NV >= 32) ? 5 : (NV >= 16) ? 4 : (NV >= 8) ? 3 : (NV >= 4) ? 2 : (NV >= 2) ? 1 : 0;
#pragma unroll
    for (int off = 16 >> levels; off >= 1 && levels < 5; off >>= 1) r += __shfl_xor_sync(kFull, r, off);
    return r;
}

}  // namespace ckv
