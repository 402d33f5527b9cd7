// summaries.cu -- per-block element-wise max / min of permuted tokens.
//
// "Adaptive tiling (SPADE)", The idea, step 3: each block of `block`
// consecutive tokens (one tile after the permutation) is summarised by its
// per-channel maximum and minimum.  Results are exact selections of inputs.
//
// One CTA per (bh, block).  Lanes own 16-byte column chunks; row groups walk
// the block's rows with 128-bit loads, then reduce through shared memory.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

constexpr int kThreads = 256;

template <typename T>
struct Vec;  // 16 bytes of T with element-wise max / min

template <>
struct Vec<__nv_bfloat16> {
    __nv_bfloat162 v[4];
    __device__ static Vec load(const void *p) {
        Vec r;
        *reinterpret_cast<uint4 *>(r.v) = __ldcs(reinterpret_cast<const uint4 *>(p));
        return r;
    }
    __device__ void store(void *p) const { *reinterpret_cast<uint4 *>(p) = *reinterpret_cast<const uint4 *>(v); }
    __device__ void vmax(const Vec &o) {
        #pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __hmax2(v[i], o.v[i]);
    }
    __device__ void vmin(const Vec &o) {
        #pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __hmin2(v[i], o.v[i]);
    }
};

template <>
struct Vec<float> {
    float v[4];
    __device__ static Vec load(const void *p) {
        Vec r;
        *reinterpret_cast<float4 *>(r.v) = __ldcs(reinterpret_cast<const float4 *>(p));
        return r;
    }
    __device__ void store(void *p) const { *reinterpret_cast<float4 *>(p) = *reinterpret_cast<const float4 *>(v); }
    __device__ void vmax(const Vec &o) {
        #pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = fmaxf(v[i], o.v[i]);
    }
    __device__ void vmin(const Vec &o) {
        #pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = fminf(v[i], o.v[i]);
    }
};

template <typename T, int CPR>
__global__ void __launch_bounds__(kThreads) summaries_kernel(const uint8_t *__restrict__ x, int S, int block, int nb,
                                                             uint8_t *__restrict__ xmax, uint8_t *__restrict__ xmin) {
    constexpr int RG = kThreads / CPR;  // row groups
    __shared__ uint4 smax[RG][CPR];
    __shared__ uint4 smin[RG][CPR];
    const int blk = blockIdx.x, bh = blockIdx.y;
    const int chunk = threadIdx.x % CPR, rg = threadIdx.x / CPR;
    const size_t row0 = static_cast<size_t>(bh) * S + static_cast<size_t>(blk) * block;
    const uint8_t *base = x + row0 * CPR * 16 + chunk * 16;
    Vec<T> mx, mn;
    if (rg < block) {
        mx = Vec<T>::load(base + static_cast<size_t>(rg) * CPR * 16);
        mn = mx;
        #pragma unroll 4
        for (int r = rg + RG; r < block; r += RG) {
            const Vec<T> v = Vec<T>::load(base + static_cast<size_t>(r) * CPR * 16);
            mx.vmax(v);
            mn.vmin(v);
        }
        mx.store(&smax[rg][chunk]);
        mn.store(&smin[rg][chunk]);
    }
    __syncthreads();
    if (rg == 0) {
        #pragma unroll 4
        for (int g = 1; g < RG && g < block; ++g) {
            mx.vmax(*reinterpret_cast<const Vec<T> *>(&smax[g][chunk]));
            mn.vmin(*reinterpret_cast<const Vec<T> *>(&smin[g][chunk]));
        }
        const size_t o = (static_cast<size_t>(bh) * nb + blk) * CPR * 16 + chunk * 16;
        mx.store(xmax + o);
        mn.store(xmin + o);
    }
}

}  // namespace

cudaError_t launch_summaries(const void *x, int esize, int BH, int S, int D, int block, void *xmax, void *xmin,
                             cudaStream_t st) {
    const int nb = S / block;
    const int cpr = D * esize / 16;
    dim3 grid(nb, BH);
    const uint8_t *xi = static_cast<const uint8_t *>(x);
    uint8_t *mx = static_cast<uint8_t *>(xmax), *mn = static_cast<uint8_t *>(xmin);
    if (esize == 2) {
        if (cpr == 8) summaries_kernel<__nv_bfloat16, 8><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn);
        else summaries_kernel<__nv_bfloat16, 16><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn);
    } else {
        if (cpr == 16) summaries_kernel<float, 16><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn);
        else summaries_kernel<float, 32><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn);
    }
    return cudaGetLastError();
}

}  // namespace vsa
