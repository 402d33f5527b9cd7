// scores.cu -- SPADE min/max block scores.
//
// "Adaptive tiling (SPADE)", The idea, step 3 and minmax_block_scores:
//   score(i, j) = max(a_i . k_max_j, a_i . k_min_j),  a_i = q_max_i + q_min_i.
// a_i is formed in fp32 (exact for bf16 summaries whose exponents differ by
// less than 2^16, and for every small-integer-valued input); the dot products
// accumulate in fp32 with FMA.  64 x 64 output tile per CTA, D staged through
// shared memory in chunks of 32 channels, 4 x 4 outputs per thread.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

constexpr int TI = 64, TJ = 64, DK = 32, PAD = TI + 4;

template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
    #pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
    }
}

template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(256) scores_kernel(const T *__restrict__ qmax, const T *__restrict__ qmin,
                                                    const T *__restrict__ kmax, const T *__restrict__ kmin, int nb,
                                                    int D, float *__restrict__ out) {
    __shared__ __align__(16) float sA[DK][PAD];
    __shared__ __align__(16) float sX[DK][PAD];
    __shared__ __align__(16) float sN[DK][PAD];
    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * TI, j0 = blockIdx.x * TJ;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const size_t head = static_cast<size_t>(bh) * nb * D;
    float acc_x[4][4] = {}, acc_n[4][4] = {};
    const int lrow = threadIdx.x / 4, ld = (threadIdx.x % 4) * 8;  // loader: row, first channel
    for (int d0 = 0; d0 < D; d0 += DK) {
        {
            float a[8], b[8];
            const int i = i0 + lrow, j = j0 + lrow;
            if (i < nb) {
                load8<T>(qmax + head + static_cast<size_t>(i) * D + d0 + ld, a);
                load8<T>(qmin + head + static_cast<size_t>(i) * D + d0 + ld, b);
            } else {
                #pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.f;
            }
            #pragma unroll
            for (int e = 0; e < 8; ++e) sA[ld + e][lrow] = a[e] + b[e];
            if (j < nb) {
                load8<T>(kmax + head + static_cast<size_t>(j) * D + d0 + ld, a);
                load8<T>(kmin + head + static_cast<size_t>(j) * D + d0 + ld, b);
            } else {
                #pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.f;
            }
            #pragma unroll
            for (int e = 0; e < 8; ++e) {
                sX[ld + e][lrow] = a[e];
                sN[ld + e][lrow] = b[e];
            }
        }
        __syncthreads();
        #pragma unroll 8
        for (int d = 0; d < DK; ++d) {
            const float4 a4 = *reinterpret_cast<const float4 *>(&sA[d][ty * 4]);
            const float4 x4 = *reinterpret_cast<const float4 *>(&sX[d][tx * 4]);
            const float4 n4 = *reinterpret_cast<const float4 *>(&sN[d][tx * 4]);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
            const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
            const float nv[4] = {n4.x, n4.y, n4.z, n4.w};
            #pragma unroll
            for (int r = 0; r < 4; ++r)
                #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc_x[r][c] = fmaf(av[r], xv[c], acc_x[r][c]);
                    acc_n[r][c] = fmaf(av[r], nv[c], acc_n[r][c]);
                }
        }
        __syncthreads();
    }
    float *o = out + static_cast<size_t>(bh) * nb * nb;
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = i0 + ty * 4 + r;
        if (i >= nb) continue;
        #pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = j0 + tx * 4 + c;
            if (j < nb) o[static_cast<size_t>(i) * nb + j] = fmaxf(acc_x[r][c], acc_n[r][c]);
        }
    }
}

}  // namespace

cudaError_t launch_scores(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int esize, int BH,
                          int nb, int D, float *scores, cudaStream_t st) {
    dim3 grid((nb + TJ - 1) / TJ, (nb + TI - 1) / TI, BH);
    if (esize == 2)
        scores_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(qmax), static_cast<const __nv_bfloat16 *>(qmin),
            static_cast<const __nv_bfloat16 *>(kmax), static_cast<const __nv_bfloat16 *>(kmin), nb, D, scores);
    else
        scores_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(qmax), static_cast<const float *>(qmin),
                                                   static_cast<const float *>(kmax), static_cast<const float *>(kmin),
                                                   nb, D, scores);
    return cudaGetLastError();
}

}  // namespace vsa
