// scores_tc.cu -- SPADE min/max block scores on tcgen05 tensor cores (bf16).
//
// "Adaptive tiling (SPADE)", The idea, step 3 and minmax_block_scores:
//   score(i, j) = max((q_max_i + q_min_i) . k_max_j, (q_max_i + q_min_i) . k_min_j).
// Each dot product is taken as q_max . k + q_min . k: both are accumulated in
// fp32 on the tensor cores from exact bf16 x bf16 products (one 128 x 128
// accumulator for k_max, one for k_min, 2 x 8 MMAs of K = 16 each), so the
// result is exact on small-integer-valued summaries and otherwise within
// fp32 accumulation error.  TMA loads 128-block summary tiles (rows past nb
// read as zero), one thread issues the MMAs, four warps take the max of the
// two accumulators row by row and store the fp32 scores.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

int sm_count_here() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int D>
struct ScCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;
    static constexpr int TILE = SLAB * KSLABS;             // one 128-row summary tile
    static constexpr int STAGE = 128 * 128;                // 32 score columns x 128 rows fp32
    // Q_max, Q_min, two slots of (K_max, K_min), two staging buffers for the
    // TMA stores; at least half the SM's shared memory, so one CTA (which
    // takes all 512 TMEM columns) per SM
    static constexpr int NEED = 1024 + 6 * TILE + 2 * STAGE + 16 * 8 + 64;
    static constexpr int SMEM = NEED > 120 * 1024 ? NEED : 120 * 1024;
};

constexpr int kScThreads = 160;  // warps 0-3: epilogue (thread = score row), warp 4: loads and MMAs

// One CTA owns 128 query blocks (rows i0 .. i0+127) of one head and a run of
// 128-wide key-block tiles; Q_max/Q_min stay in shared memory, (K_max, K_min)
// tiles are double-buffered, and the two accumulators of a tile (q.k_max and
// q.k_min, 128 TMEM columns each) are double-buffered in TMEM so that the MMAs
// of tile u+1 run while the epilogue warps store tile u.
// With TMA (scores rows 16-byte aligned) each 32-column slab of a tile is
// staged in shared memory (128-byte swizzled rows, so the row-per-thread
// writes spread over the banks) and written by one tensor store; otherwise
// each thread stores its row directly.
template <int D, bool TMA>
__global__ void __launch_bounds__(kScThreads, 1)
scores_tc_kernel(const __grid_constant__ CUtensorMap tmQX, const __grid_constant__ CUtensorMap tmQN,
                 const __grid_constant__ CUtensorMap tmKX, const __grid_constant__ CUtensorMap tmKN,
                 const __grid_constant__ CUtensorMap tmOut, int nb, int tiles_per_cta, int vec4,
                 float *__restrict__ out, int *status) {
    using C = ScCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQX = base, *sQN = base + C::TILE;
    uint8_t *sK = base + 2 * C::TILE;  // slot s: K_max at sK + 2 s TILE, K_min right after
    uint8_t *stage = base + 6 * C::TILE;  // [2][STAGE]
    uint64_t *q_full = reinterpret_cast<uint64_t *>(stage + 2 * C::STAGE);
    uint64_t *k_full = q_full + 1;     // [2]
    uint64_t *k_empty = k_full + 2;    // [2]
    uint64_t *acc_full = k_empty + 2;  // [2]
    uint64_t *acc_empty = acc_full + 2;  // [2]
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * 128, bh = blockIdx.y;
    const int n_jt = (nb + 127) / 128;
    const int jt0 = blockIdx.z * tiles_per_cta;
    const int n = max(0, min(jt0 + tiles_per_cta, n_jt) - jt0);  // tiles of this CTA

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tmQX);
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
            const uint64_t dQX = sdesc_sw128(smem_u32(sQX), 16, 1024), dQN = sdesc_sw128(smem_u32(sQN), 16, 1024);
            const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
            constexpr uint64_t kTile16 = C::TILE >> 4;
            auto load_k = [&](int u) {
                const int s = u & 1, j0 = (jt0 + u) * 128;
                uint8_t *kx = sK + (2 * s) * C::TILE, *kn = kx + C::TILE;
                mbar_arrive_expect_tx(&k_full[s], 2 * C::TILE);
                for (int sl = 0; sl < C::KSLABS; ++sl) {
                    tma_load_3d(kx + sl * C::SLAB, &tmKX, &k_full[s], sl * 64, j0, bh);
                    tma_load_3d(kn + sl * C::SLAB, &tmKN, &k_full[s], sl * 64, j0, bh);
                }
            };
            mbar_arrive_expect_tx(q_full, 2 * C::TILE);
            for (int sl = 0; sl < C::KSLABS; ++sl) {
                tma_load_3d(sQX + sl * C::SLAB, &tmQX, q_full, sl * 64, i0, bh);
                tma_load_3d(sQN + sl * C::SLAB, &tmQN, q_full, sl * 64, i0, bh);
            }
            load_k(0);
            int loaded = 1;  // K tiles issued
            bool ok = mbar_wait(q_full, 0, abort_flag);
            for (int u = 0; ok && u < n; ++u) {
                const int s = u & 1;
                // refill the other slot once the MMAs of tile u - 1 (its last reader) are done
                if (u + 1 < n) {
                    if (u >= 1 && !mbar_wait(&k_empty[s ^ 1], ((u - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    load_k(u + 1);
                    loaded = u + 2;
                }
                if (!mbar_wait(&k_full[s], (u >> 1) & 1, abort_flag)) { ok = false; break; }
                // the epilogue must have read this accumulator buffer (tile u - 2)
                if (u >= 2 && !mbar_wait(&acc_empty[s], ((u - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint64_t kx = dK + (2 * s) * kTile16, kn = kx + kTile16;
                const uint32_t d = tmem + s * 256;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(d, dQX + off, kx + off, idesc, kk > 0 ? 1u : 0u);        // q_max . k_max
                    umma_bf16(d + 128, dQX + off, kn + off, idesc, kk > 0 ? 1u : 0u);  // q_max . k_min
                }
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(d, dQN + off, kx + off, idesc, 1u);        // + q_min . k_max
                    umma_bf16(d + 128, dQN + off, kn + off, idesc, 1u);  // + q_min . k_min
                }
                umma_commit(&k_empty[s]);
                umma_commit(&acc_full[s]);
            }
            if (!ok) {
                if (!*abort_flag) { report(status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the loads already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                for (int u = max(0, loaded - 2); u < loaded; ++u) mbar_wait(&k_full[u & 1], (u >> 1) & 1, nullptr);
            }
            // every MMA issued has finished before TMEM is released
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else {
        // epilogue: row r = lane of the warp's quadrant; max of the two accumulators
        const int r = warp * 32 + lane;
        const int i = i0 + r;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        float *orow = out + (static_cast<size_t>(bh) * nb + (i < nb ? i : 0)) * nb;
        // The four warps run every slab's named barriers in every case (bar.sync
        // has no time limit); a warp whose wait gave up only skips its work.
        bool alive = true;
        for (int u = 0; u < n; ++u) {
            const int s = u & 1;
            if (alive) alive = __all_sync(0xffffffffu, mbar_wait(&acc_full[s], (u >> 1) & 1, abort_flag));
            if (!alive && lane == 0 && !*abort_flag) { report(status, DEV_TIMEOUT); *abort_flag = 1; }
            if (!TMA && !alive) break;
            tc_fence_after();
            const int jb = (jt0 + u) * 128;
            #pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
                uint32_t x[32], y[32];
                if (alive) {
                    tmem_ld32(t_lane + s * 256 + c, x);
                    tmem_ld32(t_lane + s * 256 + 128 + c, y);
                    tmem_ld_wait();
                }
                if constexpr (TMA) {
                    const int g = u * 4 + (c >> 5);  // slab counter: staging buffer g & 1
                    uint8_t *buf = stage + (g & 1) * C::STAGE;
                    // the store issued from this buffer two slabs ago has read it
                    if (threadIdx.x == 0) bulk_wait_read<1>();
                    named_barrier(1, 128);
                    uint8_t *rowp = buf + r * 128;
                    if (alive) {
                        #pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<float4 *>(rowp + ((k ^ (r & 7)) << 4)) =
                                make_float4(fmaxf(__uint_as_float(x[4 * k]), __uint_as_float(y[4 * k])),
                                            fmaxf(__uint_as_float(x[4 * k + 1]), __uint_as_float(y[4 * k + 1])),
                                            fmaxf(__uint_as_float(x[4 * k + 2]), __uint_as_float(y[4 * k + 2])),
                                            fmaxf(__uint_as_float(x[4 * k + 3]), __uint_as_float(y[4 * k + 3])));
                    }
                    fence_proxy_async_smem();
                    named_barrier(1, 128);
                    // rows and columns past nb are clipped by the tensor store
                    if (threadIdx.x == 0) {
                        tma_store_3d(&tmOut, buf, jb + c, i0, bh);
                        bulk_commit();
                    }
                } else if (i < nb) {
                    const int j = jb + c;
                    if (vec4 && j + 32 <= nb) {  // rows start 16-byte aligned only when nb % 4 == 0
                        float4 *dst = reinterpret_cast<float4 *>(orow + j);
                        #pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(fmaxf(__uint_as_float(x[4 * e]), __uint_as_float(y[4 * e])),
                                                 fmaxf(__uint_as_float(x[4 * e + 1]), __uint_as_float(y[4 * e + 1])),
                                                 fmaxf(__uint_as_float(x[4 * e + 2]), __uint_as_float(y[4 * e + 2])),
                                                 fmaxf(__uint_as_float(x[4 * e + 3]), __uint_as_float(y[4 * e + 3])));
                    } else {
                        #pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j + e < nb) orow[j + e] = fmaxf(__uint_as_float(x[e]), __uint_as_float(y[e]));
                    }
                }
            }
            if (alive) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[s]);
            }
        }
        if (TMA && threadIdx.x == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
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
    CUtensorMap mout;
    const bool tma = nb % 4 == 0 && (reinterpret_cast<uintptr_t>(scores) & 15u) == 0 &&
                     make_scores_store_map(&mout, scores, nb, BH);
    if (!tma) mout = mqx;  // unused
    auto kern = tma ? scores_tc_kernel<D, true> : scores_tc_kernel<D, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int nt = (nb + 127) / 128;
    // split the key-block tiles over enough CTAs to give every SM about two
    const long long base_ctas = static_cast<long long>(nt) * BH;
    int split = static_cast<int>((2LL * sm_count_here() + base_ctas - 1) / base_ctas);
    split = max(1, min(split, nt));
    const int per = (nt + split - 1) / split;
    split = (nt + per - 1) / per;
    dim3 grid(nt, BH, split);
    const int vec4 = (nb % 4 == 0 && (reinterpret_cast<uintptr_t>(scores) & 15u) == 0) ? 1 : 0;
    kern<<<grid, kScThreads, C::SMEM, st>>>(mqx, mqn, mkx, mkn, mout, nb, per, vec4, scores, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scores_tc(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int BH, int nb,
                             int D, float *scores, int *status, cudaStream_t st) {
    return D == 128 ? run_scores_tc<128>(qmax, qmin, kmax, kmin, BH, nb, scores, status, st)
                    : run_scores_tc<64>(qmax, qmin, kmax, kmin, BH, nb, scores, status, st);
}

}  // namespace vsa
