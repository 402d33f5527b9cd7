// scores_topk.cu -- SPADE min/max block scores and the top-k lists in one
// kernel: the nb x nb score matrix never reaches global memory.
//
// "Adaptive tiling (SPADE)", The idea, steps 3 and 4 (min/max block scores,
// fixed per-row budget plus sink and diagonal blocks), and Dense by design (a
// fused estimator).  The scores are those of vsa_block_scores,
//   score(i, j) = max((q_max_i + q_min_i) . k_max_j, (q_max_i + q_min_i) . k_min_j),
// each dot product accumulated in fp32 on the tensor cores as q_max . k +
// q_min . k from exact bf16 products; the lists are those of
// vsa_topk_block_mask (topk_row.cuh).
//
// One CTA per 16 query blocks of one head, two CTAs per SM.  The MMAs take the
// key summaries as the 128-row operand and the CTA's 16 query summaries as
// the N = 16 operand, so tensor memory holds, per 128-key tile, a 16-column
// accumulator for k_max and one for k_min (32 columns a tile; nb <= 1024
// fills 256 columns).  Eight warps (two per lane quadrant) read the
// accumulators back lane by lane (lane = key), take the max of the pair and
// write the 16 score rows into shared memory (over the ring the key tiles
// came through, which the MMAs no longer read); then each of the sixteen
// warps makes one row's list.  The lists are instruction bound, so the
// second CTA on the SM keeps the issue slots busy while one loads and
// multiplies.
#include "common.cuh"
#include "internal.h"
#include "topk_row.cuh"

namespace vsa {

namespace {

constexpr int kFuWarps = 16;       // 0-3, 8-11: accumulators -> rows, 4: TMA, 5: MMA and TMEM; all: lists
constexpr int kFuRows = 16;        // query blocks per CTA (the MMA's N)
constexpr int kFuMaxBlocks = 1024; // blocks per head (8 key tiles x 32 TMEM columns)

template <int D>
struct FuCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int QSLAB = kFuRows * 128;   // 16 rows x 128 bytes
    static constexpr int QTILE = QSLAB * KSLABS;  // Q_max (or Q_min) rows of the CTA
    static constexpr int KSLAB = 128 * 128;
    static constexpr int KTILE = KSLAB * KSLABS;  // one 128-key summary tile
    static constexpr int NST = 2;                 // ring stages: K_max and K_min of one tile
    static constexpr int RING = NST * KTILE;
    static constexpr int ROWS = kFuRows * kFuMaxBlocks * 4;  // score rows, over the ring
    static constexpr int BIG = RING > ROWS ? RING : ROWS;
    static constexpr int N_BARS = 1 + 2 * NST + 1;
    static constexpr int SMEM = 1024 + 2 * QTILE + BIG + N_BARS * 8 + 64 + kFuWarps * kTopkCand * 4;
    static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};

template <int D, int NPL>
__global__ void __launch_bounds__(kFuWarps * 32, 2)
scores_topk_kernel(const __grid_constant__ CUtensorMap tmQX, const __grid_constant__ CUtensorMap tmQN,
                   const __grid_constant__ CUtensorMap tmKX, const __grid_constant__ CUtensorMap tmKN, int nb, int k,
                   int n_sink, int diag_hw, int32_t *__restrict__ idx, int32_t *__restrict__ cnt, int cap,
                   uint32_t tmem_cols, int *status) {
    using C = FuCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQX = base, *sQN = base + C::QTILE;
    uint8_t *sK = base + 2 * C::QTILE;                       // [NST][KTILE], later the score rows
    float *rows = reinterpret_cast<float *>(sK);              // [16][nct * 128]
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sK + C::BIG);
    uint64_t *k_full = q_full + 1;     // [NST]
    uint64_t *k_empty = k_full + C::NST;
    uint64_t *mma_done = k_empty + C::NST;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint32_t *cand = reinterpret_cast<uint32_t *>(tmem_slot + 16);  // [kFuWarps][kTopkCand]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * kFuRows, bh = blockIdx.y;
    const int nct = (nb + 127) / 128;   // key tiles
    const int rstride = nct * 128;      // floats per score row in shared memory

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ================= TMA producer =================
        // Q_max, Q_min rows; then per key tile t: K_max(t), K_min(t) through the ring
        if (lane == 0) {
            tma_prefetch_desc(&tmKX);
            tma_prefetch_desc(&tmKN);
            mbar_arrive_expect_tx(q_full, 2 * C::QTILE);
            for (int sl = 0; sl < C::KSLABS; ++sl) {
                tma_load_3d(sQX + sl * C::QSLAB, &tmQX, q_full, sl * 64, r0, bh);
                tma_load_3d(sQN + sl * C::QSLAB, &tmQN, q_full, sl * 64, r0, bh);
            }
            int u = 0;
            bool ok = true;
            for (; u < 2 * nct; ++u) {
                const int s = u % C::NST;
                if (u >= C::NST && !mbar_wait(&k_empty[s], ((u / C::NST) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&k_full[s], C::KTILE);
                for (int sl = 0; sl < C::KSLABS; ++sl)
                    tma_load_3d(sK + s * C::KTILE + sl * C::KSLAB, (u & 1) ? &tmKN : &tmKX, &k_full[s], sl * 64,
                                (u >> 1) * 128, bh);
            }
            if (!ok) {
                if (!*abort_flag) { report(status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the loads already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                for (int v = u > C::NST ? u - C::NST : 0; v < u; ++v) mbar_wait(&k_full[v % C::NST], (v / C::NST) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ================= MMA issuer =================
        // accumulator of tile t at columns 32 t (k_max) and 32 t + 16 (k_min):
        // q_max . k first, then + q_min . k, 16 channels per MMA
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, kFuRows, false);
            const uint64_t dQX = sdesc_sw128(smem_u32(sQX), 16, 1024), dQN = sdesc_sw128(smem_u32(sQN), 16, 1024);
            const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
            constexpr uint64_t kTile16 = C::KTILE >> 4;
            bool ok = mbar_wait(q_full, 0, abort_flag);
            for (int t = 0; ok && t < nct; ++t) {
                const int u0 = 2 * t, u1 = 2 * t + 1, s0 = u0 % C::NST, s1 = u1 % C::NST;
                ok = mbar_wait(&k_full[s0], (u0 / C::NST) & 1, abort_flag) &&
                     mbar_wait(&k_full[s1], (u1 / C::NST) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint64_t kx = dK + s0 * kTile16, kn = dK + s1 * kTile16;
                const uint32_t d = tmem + t * 32;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ok_ = static_cast<uint64_t>(((kk >> 2) * C::KSLAB + (kk & 3) * 32) >> 4);
                    const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * C::QSLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(d, kx + ok_, dQX + oq, idesc, kk > 0 ? 1u : 0u);        // k_max . q_max
                    umma_bf16(d + 16, kn + ok_, dQX + oq, idesc, kk > 0 ? 1u : 0u);   // k_min . q_max
                }
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ok_ = static_cast<uint64_t>(((kk >> 2) * C::KSLAB + (kk & 3) * 32) >> 4);
                    const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * C::QSLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(d, kx + ok_, dQN + oq, idesc, 1u);        // + k_max . q_min
                    umma_bf16(d + 16, kn + ok_, dQN + oq, idesc, 1u);   // + k_min . q_min
                }
                umma_commit(&k_empty[s0]);
                umma_commit(&k_empty[s1]);
            }
            if (!ok && !*abort_flag) { report(status, DEV_TIMEOUT); *abort_flag = 1; }
            // every MMA issued has finished before the rows overwrite the ring
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else if ((warp & 4) == 0) {
        // ================= accumulators -> score rows (warps 0-3, 8-11) =================
        // lane = key 128 t + 32 (warp % 4) + lane, column c = query block r0 + c;
        // warps 0-3 take the even key tiles, warps 8-11 the odd ones
        const int wq = warp & 3;
        const bool alive = __all_sync(0xffffffffu, mbar_wait(mma_done, 0, abort_flag));
        if (alive) {
            tc_fence_after();
            const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
            for (int t = warp >> 3; t < nct; t += 2) {
                uint32_t mx[kFuRows], mn[kFuRows];
                tmem_ld16(t_lane + t * 32, mx);
                tmem_ld16(t_lane + t * 32 + 16, mn);
                tmem_ld_wait();
                const int j = t * 128 + wq * 32 + lane;
                #pragma unroll
                for (int c = 0; c < kFuRows; ++c)
                    rows[c * rstride + j] = fmaxf(__uint_as_float(mx[c]), __uint_as_float(mn[c]));
            }
        } else if (lane == 0 && !*abort_flag) {
            report(status, DEV_TIMEOUT);
            *abort_flag = 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
    if (*abort_flag) return;  // a wait gave up: the lists of this CTA are not written
    // ================= the lists: rows warp, warp + 8, ... =================
    for (int c = warp; c < kFuRows; c += kFuWarps) {
        const int i = r0 + c;
        if (i >= nb) break;
        const float *row = rows + c * rstride;
        uint32_t key[NPL];
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const int j = lane + 32 * t;
            key[t] = j < nb ? order_key(row[j]) : 0u;
        }
        const size_t r = static_cast<size_t>(bh) * nb + i;
        topk_row<NPL>(key, nb, k, i, n_sink, diag_hw, idx + r * cap, cnt + r, cap, cand + warp * kTopkCand);
    }
}

template <int D, int NPL>
cudaError_t run_scores_topk(const CUtensorMap (&m)[4], int BH, int nb, int k, int n_sink, int diag_hw, int32_t *idx,
                            int32_t *cnt, int cap, int *status, cudaStream_t st) {
    using C = FuCfg<D>;
    auto kern = scores_topk_kernel<D, NPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int nct = (nb + 127) / 128;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(nct * 32)) cols <<= 1;
    dim3 grid((nb + kFuRows - 1) / kFuRows, BH);
    kern<<<grid, kFuWarps * 32, C::SMEM, st>>>(m[0], m[1], m[2], m[3], nb, k, n_sink, diag_hw, idx, cnt, cap, cols,
                                               status);
    return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_scores_topk(const CUtensorMap (&m)[4], int BH, int nb, int k, int n_sink, int diag_hw,
                                 int32_t *idx, int32_t *cnt, int cap, int *status, cudaStream_t st) {
    const int npl = (nb + 31) / 32;
#define VSA_FU(N) return run_scores_topk<D, N>(m, BH, nb, k, n_sink, diag_hw, idx, cnt, cap, status, st)
    if (npl <= 2) VSA_FU(2);
    if (npl <= 4) VSA_FU(4);
    if (npl <= 8) VSA_FU(8);
    if (npl <= 16) VSA_FU(16);
    if (npl <= 30) VSA_FU(30);
    VSA_FU(32);
#undef VSA_FU
}

}  // namespace

int scores_topk_max_blocks() { return kFuMaxBlocks; }

cudaError_t launch_scores_topk(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int BH, int nb,
                               int D, int k, int n_sink, int diag_hw, int32_t *idx, int32_t *cnt, int cap, int *status,
                               cudaStream_t st) {
    CUtensorMap m[4];
    if (!make_tile_map(&m[0], qmax, D, nb, BH, kFuRows) || !make_tile_map(&m[1], qmin, D, nb, BH, kFuRows) ||
        !make_tile_map(&m[2], kmax, D, nb, BH, 128) || !make_tile_map(&m[3], kmin, D, nb, BH, 128))
        return cudaErrorInvalidValue;
    return D == 128 ? dispatch_scores_topk<128>(m, BH, nb, k, n_sink, diag_hw, idx, cnt, cap, status, st)
                    : dispatch_scores_topk<64>(m, BH, nb, k, n_sink, diag_hw, idx, cnt, cap, status, st);
}

}  // namespace vsa
