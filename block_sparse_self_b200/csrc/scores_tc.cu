// scores_tc.cu -- SPADE min/max block scores on tcgen05 tensor cores (bf16).
//
// "Adaptive tiling (SPADE)", The idea, step 3 and minmax_block_scores:
//   score(i, j) = max((q_max_i + q_min_i) . k_max_j, (q_max_i + q_min_i) . k_min_j).
// Each dot product is taken as q_max . k + q_min . k: both are accumulated in
// fp32 on the tensor cores from exact bf16 x bf16 products (one 128 x 128
// accumulator for k_max, one for k_min, 2 x 8 MMAs of K = 16 each), so the
// result is exact on small-integer-valued summaries and otherwise within
// fp32 accumulation error.  One CTA computes a 128 x 128 tile of one head's
// score matrix: TMA loads the four 128-block summary tiles (rows past nb read
// as zero), one thread issues the MMAs, four warps take the max of the two
// accumulators row by row and store the fp32 scores.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

template <int D>
struct ScCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;
    static constexpr int TILE = SLAB * KSLABS;             // one 128-row summary tile
    static constexpr int SMEM = 1024 + 4 * TILE + 64;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
scores_tc_kernel(const __grid_constant__ CUtensorMap tmQX, const __grid_constant__ CUtensorMap tmQN,
                 const __grid_constant__ CUtensorMap tmKX, const __grid_constant__ CUtensorMap tmKN, int nb,
                 int vec4, float *__restrict__ out, int *status) {
    using C = ScCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQX = base, *sQN = base + C::TILE, *sKX = base + 2 * C::TILE, *sKN = base + 3 * C::TILE;
    uint64_t *full = reinterpret_cast<uint64_t *>(base + 4 * C::TILE);
    uint64_t *done = full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = blockIdx.x * 128, i0 = blockIdx.y * 128, bh = blockIdx.z;

    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmQX);
        mbar_arrive_expect_tx(full, 4 * C::TILE);
        for (int s = 0; s < C::KSLABS; ++s) {
            tma_load_3d(sQX + s * C::SLAB, &tmQX, full, s * 64, i0, bh);
            tma_load_3d(sQN + s * C::SLAB, &tmQN, full, s * 64, i0, bh);
            tma_load_3d(sKX + s * C::SLAB, &tmKX, full, s * 64, j0, bh);
            tma_load_3d(sKN + s * C::SLAB, &tmKN, full, s * 64, j0, bh);
        }
        ok = mbar_wait(full, 0, nullptr);
        if (ok) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
            const uint64_t dQX = sdesc_sw128(smem_u32(sQX), 16, 1024), dQN = sdesc_sw128(smem_u32(sQN), 16, 1024);
            const uint64_t dKX = sdesc_sw128(smem_u32(sKX), 16, 1024), dKN = sdesc_sw128(smem_u32(sKN), 16, 1024);
            #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                umma_bf16(tmem, dQX + off, dKX + off, idesc, kk > 0 ? 1u : 0u);        // q_max . k_max
                umma_bf16(tmem + 128, dQX + off, dKN + off, idesc, kk > 0 ? 1u : 0u);  // q_max . k_min
            }
            #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                umma_bf16(tmem, dQN + off, dKX + off, idesc, 1u);        // + q_min . k_max
                umma_bf16(tmem + 128, dQN + off, dKN + off, idesc, 1u);  // + q_min . k_min
            }
        }
        umma_commit(done);
        if (!ok) report(status, DEV_TIMEOUT);
    }
    __syncwarp();
    // epilogue: row r = lane of warp's quadrant; max of the two accumulators
    const int r = warp * 32 + lane;
    const int i = i0 + r;
    const bool waited = mbar_wait(done, 0, nullptr);
    if (!waited && threadIdx.x == 0) report(status, DEV_TIMEOUT);
    tc_fence_after();
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float *orow = out + (static_cast<size_t>(bh) * nb + (i < nb ? i : 0)) * nb;
    #pragma unroll 1
    for (int c = 0; c < 128; c += 32) {
        uint32_t x[32], n[32];
        tmem_ld32(t_lane + c, x);
        tmem_ld32(t_lane + 128 + c, n);
        tmem_ld_wait();
        if (i < nb && waited) {
            const int j = j0 + c;
            if (vec4 && j + 32 <= nb) {  // rows start 16-byte aligned only when nb % 4 == 0
                float4 *dst = reinterpret_cast<float4 *>(orow + j);
                #pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(fmaxf(__uint_as_float(x[4 * e]), __uint_as_float(n[4 * e])),
                                         fmaxf(__uint_as_float(x[4 * e + 1]), __uint_as_float(n[4 * e + 1])),
                                         fmaxf(__uint_as_float(x[4 * e + 2]), __uint_as_float(n[4 * e + 2])),
                                         fmaxf(__uint_as_float(x[4 * e + 3]), __uint_as_float(n[4 * e + 3])));
            } else {
                #pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (j + e < nb) orow[j + e] = fmaxf(__uint_as_float(x[e]), __uint_as_float(n[e]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <int D>
cudaError_t run_scores_tc(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int BH, int nb,
                          float *scores, int *status, cudaStream_t st) {
    using C = ScCfg<D>;
    CUtensorMap mqx, mqn, mkx, mkn;
    if (!make_tile_map(&mqx, qmax, D, nb, BH, 128) || !make_tile_map(&mqn, qmin, D, nb, BH, 128) ||
        !make_tile_map(&mkx, kmax, D, nb, BH, 128) || !make_tile_map(&mkn, kmin, D, nb, BH, 128))
        return cudaErrorInvalidValue;
    auto kern = scores_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int nt = (nb + 127) / 128;
    dim3 grid(nt, nt, BH);
    const int vec4 = (nb % 4 == 0 && (reinterpret_cast<uintptr_t>(scores) & 15u) == 0) ? 1 : 0;
    kern<<<grid, 128, C::SMEM, st>>>(mqx, mqn, mkx, mkn, nb, vec4, scores, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scores_tc(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int BH, int nb,
                             int D, float *scores, int *status, cudaStream_t st) {
    return D == 128 ? run_scores_tc<128>(qmax, qmin, kmax, kmin, BH, nb, scores, status, st)
                    : run_scores_tc<64>(qmax, qmin, kmax, kmin, BH, nb, scores, status, st);
}

}  // namespace vsa
