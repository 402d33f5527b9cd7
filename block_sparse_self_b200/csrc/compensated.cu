// compensated.cu -- block-sparse attention whose skipped key blocks take part
// through their centroids ("Adaptive tiling (SPADE)", Recipe: the attention
// call centroid_compensated_attention(q, k, v, q_labels, k_labels,
// block_mask); its recipe note names dropping the skipped blocks as the
// alternative).  The pages give the call and its arguments only.  The reading
// taken here: query i attends exactly to the keys of its kept blocks, and
// every skipped key block b of n_b keys takes part as one key, its mean key
// kbar_b, with value its mean value vbar_b and weight n_b:
//   o_i = (sum_kept e^{s(q_i, k_t)} v_t + sum_skipped n_b e^{s(q_i, kbar_b)} vbar_b)
//       / (sum_kept e^{s(q_i, k_t)}     + sum_skipped n_b e^{s(q_i, kbar_b)}).
// Blocks are the 128-position blocks of the tile-contiguous order (labels =
// position / 128), the kept blocks of query block i are its list.
//
// Three launches:
//   1. centroid_kernel: per key block, the fp32 mean of its keys and values,
//      each stored as a pair of bf16 (hi = bf16(mean), lo = bf16(mean - hi)),
//      so that the tensor cores see the centroids to about 16 bits.
//   2. the block-sparse attention kernel over the kept blocks, writing its
//      normalised output in fp32 and each row's softmax state (m, l).
//   3. comp_pair_kernel: per pair of query tiles, S = Q kbar^T (hi and lo
//      MMAs) over all centroids, kept blocks masked, an online softmax with
//      the same lazy running max as the attention kernel, O = P vbar (hi and
//      lo MMAs); then the two partial softmaxes are merged exactly:
//        o = (l1 2^(m1-M) o1 + n_b 2^(m2-M) O2) / (l1 2^(m1-M) + n_b l2 2^(m2-M)),
//      M = max(m1, m2), and written in the output dtype.
// Tiled mode takes q, k, v and o in T-major order, as the tiled attention
// does: each head's blocks are those of its own tiling, the centroid kernel
// and the pass read a block's rows where the tiling puts them (Q as 5-D TMA
// boxes), and every output row goes to its T-major token.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

constexpr int kBlock = 128;        // tokens per block (and per centroid tile)
constexpr int kMaxCentroidTiles = 64;  // nb <= 64 * 128 = 8192 blocks per head

// Tiled mode: each head's tiling (candidate choice[bh], tiling 0 without a
// choice); position p of its tile-contiguous order is T-major token
// tile_token_fast(p, divs[c]), and query tile qt is the 128-token box at
// part qt % m of tile qt / m (m = volume / 128, bt = tile.t / m frames).
struct CompTiling {
    int n;
    const int32_t *choice;
    TileDivs divs[kMaxTiles];
    FastDiv m[kMaxTiles], nthw[kMaxTiles], ntw[kMaxTiles];
    int bt[kMaxTiles], th[kMaxTiles], tw[kMaxTiles];
};

// the head's tiling, or -1 for a choice out of range (the head is left unwritten)
__device__ __forceinline__ int comp_tiling(const CompTiling &tl, int bh) {
    const int c = tl.choice ? __ldg(tl.choice + bh) : 0;
    return (c < 0 || c >= tl.n) ? -1 : c;
}

// ---------------------------------------------------------------------------
// 1. centroids
// ---------------------------------------------------------------------------
// One CTA per (key block, bh), 256 threads: thread t sums 16-byte chunk
// t % (D / 8) of every (256 / (D / 8))-th row of the block, for K and V.
template <int D, bool TILED>
__global__ void __launch_bounds__(256) centroid_kernel(const __nv_bfloat16 *__restrict__ k,
                                                       const __nv_bfloat16 *__restrict__ v, int S, int nb,
                                                       __nv_bfloat16 *__restrict__ khi, __nv_bfloat16 *__restrict__ klo,
                                                       __nv_bfloat16 *__restrict__ vhi, __nv_bfloat16 *__restrict__ vlo,
                                                       const CompTiling tl) {
    constexpr int CPR = D / 8;            // 16-byte chunks per row
    constexpr int G = 256 / CPR;          // row groups
    __shared__ float red[2][G][D];
    const int b = blockIdx.x, bh = blockIdx.y;
    const int chunk = threadIdx.x % CPR, g = threadIdx.x / CPR;
    const uint4 *kr = reinterpret_cast<const uint4 *>(k + static_cast<size_t>(bh) * S * D);
    const uint4 *vr = reinterpret_cast<const uint4 *>(v + static_cast<size_t>(bh) * S * D);
    int c = 0;
    if constexpr (TILED) {
        c = comp_tiling(tl, bh);
        if (c < 0) c = 0;  // the head is left unwritten downstream; read tiling 0 in bounds
    }
    float ak[8] = {}, av[8] = {};
    #pragma unroll 4
    for (int r = g; r < kBlock; r += G) {
        const uint32_t p = static_cast<uint32_t>(b * kBlock + r);
        const size_t row = TILED ? tile_token_fast(p, tl.divs[c]) : p;
        const uint4 xk = __ldg(kr + row * CPR + chunk), xv = __ldg(vr + row * CPR + chunk);
        const __nv_bfloat162 *pk = reinterpret_cast<const __nv_bfloat162 *>(&xk);
        const __nv_bfloat162 *pv = reinterpret_cast<const __nv_bfloat162 *>(&xv);
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 fk = __bfloat1622float2(pk[e]), fv = __bfloat1622float2(pv[e]);
            ak[2 * e] += fk.x;
            ak[2 * e + 1] += fk.y;
            av[2 * e] += fv.x;
            av[2 * e + 1] += fv.y;
        }
    }
    #pragma unroll
    for (int e = 0; e < 8; ++e) {
        red[0][g][chunk * 8 + e] = ak[e];
        red[1][g][chunk * 8 + e] = av[e];
    }
    __syncthreads();
    if (threadIdx.x < 2 * D) {
        const int which = threadIdx.x / D, d = threadIdx.x % D;
        float sum = 0.f;
        #pragma unroll
        for (int i = 0; i < G; ++i) sum += red[which][i][d];
        const float mean = sum * (1.0f / kBlock);  // an exact scaling by a power of two
        const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
        const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
        const size_t o = (static_cast<size_t>(bh) * nb + b) * D + d;
        if (which == 0) {
            khi[o] = hi;
            klo[o] = lo;
        } else {
            vhi[o] = hi;
            vlo[o] = lo;
        }
    }
}

// ---------------------------------------------------------------------------
// 3. the centroid pass and the merge
// ---------------------------------------------------------------------------
// Two query tiles per CTA, as in the block-sparse attention kernel: warps 0-3
// run tile A's softmax and merge, warps 4-7 tile B's, warp 8 the TMA loads,
// warp 9 the MMAs and the tensor memory.  Both tiles walk every centroid tile
// of the head, so each centroid tile (its kbar hi and lo parts, its vbar hi
// and lo parts) is loaded once for the two of them; a tile's kept blocks and
// the blocks past nb are masked.  Tensor memory: S_A, S_B (128 columns
// each), O_A, O_B (D each); P is written over the first 64 columns of its S.
// The MMAs go in the order QK_A(0) QK_B(0) | PV_A(c) QK_A(c+1) PV_B(c)
// QK_B(c+1) | c = 0, 1, ..., so one tile's softmax runs while the other's
// products do.
template <int D>
struct PairCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;            // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = SLAB * KSLABS;  // one 128-row operand tile
    static constexpr int O_COL = 256;                 // S_A, S_B at 0 and 128; O_A, O_B at 256 and 256 + D
    static constexpr int N_BARS = 1 + 4 + 3 * 2 + 1;
    static constexpr int MASK_WORDS = kMaxCentroidTiles * 4;  // per tile: bit j set when block j is kept
    // Q_A, Q_B, kbar hi, kbar lo, vbar hi, vbar lo
    static constexpr int SMEM = 1024 + 6 * TILE_BYTES + N_BARS * 8 + 64 + 2 * MASK_WORDS * 4;
    static_assert(SMEM <= 232448, "shared memory");
};
constexpr int kPairThreads = 320;
constexpr float kCompMaxRowSum = 16777216.0f;

struct CompArgs {
    int S, nb, nct, nq;        // positions per head, blocks per head, centroid tiles, query tiles
    const int32_t *idx, *cnt;
    int cap, list_per_head;
    float scale_log2;
    float weight;              // n_b: keys per skipped block
    const float2 *stats;       // main pass (m, l) per row
    const float *o1;           // main pass normalised output, fp32 [BH, S, D]
    void *out;
    int out_f32;
    int *status;
};

struct CompMaps {
    CUtensorMap q[kMaxTiles];  // slot 0 only, or one per candidate tiling in tiled mode
    CUtensorMap khi, klo, vhi, vlo;
};

template <int D, bool TILED>
__global__ void __launch_bounds__(kPairThreads, 1)
comp_pair_kernel(const __grid_constant__ CompMaps maps, const CompArgs a, const CompTiling tl) {
    using C = PairCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                               // [2][TILE]
    uint8_t *sKh = sQ + 2 * C::TILE_BYTES;
    uint8_t *sKl = sKh + C::TILE_BYTES;
    uint8_t *sVh = sKl + C::TILE_BYTES;
    uint8_t *sVl = sVh + C::TILE_BYTES;
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sVl + C::TILE_BYTES);
    uint64_t *k_full = q_full + 1;
    uint64_t *k_empty = k_full + 1;
    uint64_t *v_full = k_empty + 1;
    uint64_t *v_empty = v_full + 1;
    uint64_t *s_full = v_empty + 1;   // [2]
    uint64_t *p_full = s_full + 2;    // [2]
    uint64_t *pv_done = p_full + 2;   // [2]
    uint64_t *mma_done = pv_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *list_ok = reinterpret_cast<int *>(tmem_slot + 2);          // [2]
    uint32_t *kept = reinterpret_cast<uint32_t *>(tmem_slot + 16);  // [2][MASK_WORDS]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    int tc = 0;  // tiled mode: this head's tiling (out of range: the head is left unwritten)
    if constexpr (TILED) tc = comp_tiling(tl, bh);
    int qt[2];
    const int32_t *list[2] = {nullptr, nullptr};
    int cnt[2] = {0, 0};
    bool valid[2];
    for (int t = 0; t < 2; ++t) {
        qt[t] = 2 * blockIdx.x + t;
        valid[t] = qt[t] < a.nq && tc >= 0;
        if (valid[t]) {
            const size_t lrow = (a.list_per_head ? static_cast<size_t>(bh) * a.nb : 0) + qt[t];
            list[t] = a.idx + lrow * a.cap;
            cnt[t] = __ldg(a.cnt + lrow);
        }
    }

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(k_full, 1);
        mbar_init(k_empty, 1);
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);
            mbar_init(&pv_done[t], 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (tc < 0 && threadIdx.x == 0) report(a.status, DEV_RUNTIME);
    if (tc < 0) tc = 0;
    for (int i = threadIdx.x; i < 2 * C::MASK_WORDS; i += blockDim.x) kept[i] = 0u;
    if (warp < 2) {  // warp t validates tile t's list as the attention kernel does
        const int t = warp;
        bool ok = valid[t] && cnt[t] >= 1 && cnt[t] <= a.cap;
        if (ok) {
            for (int j = lane; j < cnt[t]; j += 32) {
                const int b = __ldg(list[t] + j);
                ok = ok && b >= 0 && b < a.nb && (j == 0 || __ldg(list[t] + j - 1) < b);
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (lane == 0) list_ok[t] = ok ? 1 : 0;
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    __syncthreads();
    bool act[2];
    for (int t = 0; t < 2; ++t) {
        act[t] = valid[t] && list_ok[t];
        if (valid[t] && !list_ok[t] && threadIdx.x == 0) report(a.status, DEV_RUNTIME);
        if (act[t])
            for (int j = threadIdx.x; j < cnt[t]; j += blockDim.x) {
                const int b = __ldg(list[t] + j);
                atomicOr(&kept[t * C::MASK_WORDS + (b >> 5)], 1u << (b & 31));
            }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nct = a.nct;
    const bool any = act[0] || act[1];
    const int last = act[1] ? 1 : 0;  // the tile whose MMAs are the last readers of a centroid tile

    if (warp == 8) {
        // ================= TMA producer =================
        if (lane == 0 && any) {
            tma_prefetch_desc(&maps.khi);
            tma_prefetch_desc(&maps.vhi);
            mbar_arrive_expect_tx(q_full, (act[0] + act[1]) * C::TILE_BYTES);
            for (int t = 0; t < 2; ++t) {
                if (!act[t]) continue;
                if constexpr (TILED) {  // the 128-token box of query tile qt in this head's tiling
                    const uint32_t tile = fdiv(static_cast<uint32_t>(qt[t]), tl.m[tc]);
                    const uint32_t part = static_cast<uint32_t>(qt[t]) - tile * tl.m[tc].d;
                    const uint32_t ct = fdiv(tile, tl.nthw[tc]), rem = tile - ct * tl.nthw[tc].d;
                    const uint32_t ch = fdiv(rem, tl.ntw[tc]), cw = rem - ch * tl.ntw[tc].d;
                    const int bw = static_cast<int>(cw) * tl.tw[tc], bhh = static_cast<int>(ch) * tl.th[tc];
                    const int bt = static_cast<int>(ct * tl.m[tc].d + part) * tl.bt[tc];
                    for (int s = 0; s < C::KSLABS; ++s)
                        tma_load_5d(sQ + t * C::TILE_BYTES + s * C::SLAB, &maps.q[tc], q_full, s * 64, bw, bhh, bt, bh);
                } else {
                    for (int s = 0; s < C::KSLABS; ++s)
                        tma_load_3d(sQ + t * C::TILE_BYTES + s * C::SLAB, &maps.q[0], q_full, s * 64, qt[t] * kBlock, bh);
                }
            }
            int kl = 0, vl = 0;  // centroid tiles whose K, V parts were issued
            bool ok = true;
            for (int c = 0; ok && c < nct; ++c) {
                if (c > 0 && !mbar_wait(k_empty, (c - 1) & 1, abort_flag)) { ok = false; break; }
                mbar_arrive_expect_tx(k_full, 2 * C::TILE_BYTES);
                for (int s = 0; s < C::KSLABS; ++s) {
                    tma_load_3d(sKh + s * C::SLAB, &maps.khi, k_full, s * 64, c * kBlock, bh);
                    tma_load_3d(sKl + s * C::SLAB, &maps.klo, k_full, s * 64, c * kBlock, bh);
                }
                ++kl;
                if (c > 0 && !mbar_wait(v_empty, (c - 1) & 1, abort_flag)) { ok = false; break; }
                mbar_arrive_expect_tx(v_full, 2 * C::TILE_BYTES);
                for (int s = 0; s < C::KSLABS; ++s) {
                    tma_load_3d(sVh + s * C::SLAB, &maps.vhi, v_full, s * 64, c * kBlock, bh);
                    tma_load_3d(sVl + s * C::SLAB, &maps.vlo, v_full, s * 64, c * kBlock, bh);
                }
                ++vl;
            }
            if (!ok) {
                if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the loads already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                if (kl > 0) mbar_wait(k_full, (kl - 1) & 1, nullptr);
                if (vl > 0) mbar_wait(v_full, (vl - 1) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ================= MMA issuer =================
        if (lane == 0 && any) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBlock, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dKh = sdesc_sw128(smem_u32(sKh), 16, 1024), dKl = sdesc_sw128(smem_u32(sKl), 16, 1024);
            const uint64_t dVh = sdesc_sw128(smem_u32(sVh), C::SLAB, 1024), dVl = sdesc_sw128(smem_u32(sVl), C::SLAB, 1024);
            constexpr uint64_t kTile16 = C::TILE_BYTES >> 4;
            // S_t = Q_t kbar_hi^T + Q_t kbar_lo^T, once PV_t(c - 1) has read the P over S_t
            auto qk = [&](int t, int c) -> bool {
                if (!mbar_wait(k_full, c & 1, abort_flag)) return false;
                if (c > 0 && !mbar_wait(&pv_done[t], (c - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t q0 = dQ + t * kTile16;
                const uint32_t d = tmem + t * 128;
                #pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t k0 = part == 0 ? dKh : dKl;
                    #pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                        umma_bf16(d, q0 + off, k0 + off, idesc_qk, (part > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&s_full[t]);
                if (t == last) umma_commit(k_empty);
                return true;
            };
            // O_t += P_t vbar_hi + P_t vbar_lo
            auto pv = [&](int t, int c) -> bool {
                if (!mbar_wait(&p_full[t], c & 1, abort_flag)) return false;
                if (!mbar_wait(v_full, c & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t d = tmem + C::O_COL + t * D, pa = tmem + t * 128;
                #pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t v0 = part == 0 ? dVh : dVl;
                    #pragma unroll
                    for (int kk = 0; kk < kBlock / 16; ++kk)
                        umma_bf16_ts(d, pa + kk * 8, v0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                                     (c > 0 || part > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&pv_done[t]);
                if (t == last) umma_commit(v_empty);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, abort_flag);
            for (int t = 0; ok && t < 2; ++t)
                if (act[t]) ok = qk(t, 0);
            for (int c = 0; ok && c < nct; ++c)
                for (int t = 0; ok && t < 2; ++t)
                    if (act[t]) {
                        ok = pv(t, c);
                        if (ok && c + 1 < nct) ok = qk(t, c + 1);
                    }
            if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ================= softmax over the centroids, then the merge (warps 0-7) =================
        const int t = warp >> 2, wq = warp & 3, row = wq * 32 + lane;
        const int rg = (valid[t] ? qt[t] : 0) * kBlock + row;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t s_col = t * 128, o_col = C::O_COL + t * D;
        const uint32_t *kept_t = kept + t * C::MASK_WORDS;
        const float sl2 = a.scale_log2;
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        const int n = act[t] ? nct : 0;
        for (int c = 0; c < n; ++c) {
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], c & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            uint32_t x[kBlock];
            #pragma unroll
            for (int u = 0; u < kBlock / 32; ++u)
                tmem_ld32(t_lane + s_col + 32 * u, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * u]));
            tmem_ld_wait();
            // a centroid takes part iff its block exists and is not kept
            uint32_t skip[4];
            #pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int b0 = c * kBlock + w * 32;
                const int nv = a.nb - b0 >= 32 ? 32 : (a.nb - b0 > 0 ? a.nb - b0 : 0);
                const uint32_t vm = nv == 32 ? ~0u : ((1u << nv) - 1u);
                skip[w] = ~kept_t[c * 4 + w] & vm;
            }
            // per 32 columns, a branch the whole tile takes alike (the mask
            // is the query tile's): most words skip every centroid
            auto apply_mask = [&]() {
                #pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (skip[w] != ~0u) {
                        #pragma unroll
                        for (int u = 0; u < 32; ++u)
                            if (!((skip[w] >> u) & 1u)) x[32 * w + u] = __float_as_uint(-INFINITY);
                    }
                }
            };
            apply_mask();
            auto exp_pass = [&](float m_use) -> float {
                const uint64_t sl2x2 = f32x2(sl2, sl2), nmx2 = f32x2(-m_use, -m_use);
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
                #pragma unroll
                for (int q = 0; q < kBlock / 2; ++q) {
                    float a0, a1;
                    f32x2_split(fma_f32x2(f32x2(__uint_as_float(x[2 * q]), __uint_as_float(x[2 * q + 1])), sl2x2, nmx2),
                                a0, a1);
                    const uint32_t pk = pack_bf16x2(ex2_approx(a0), ex2_approx(a1));
                    if (q & 1) add_bf16x2_f32(pk, s2, s3);
                    else add_bf16x2_f32(pk, s0, s1);
                    x[q] = pk;
                }
                return (s0 + s2) + (s1 + s3);
            };
            auto raw_max = [&]() -> float {
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                #pragma unroll
                for (int u = 0; u < kBlock; u += 8) {
                    #pragma unroll
                    for (int e = 0; e < 4; ++e)
                        m4[e] = fmax3(m4[e], __uint_as_float(x[u + 2 * e]), __uint_as_float(x[u + 2 * e + 1]));
                }
                return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            };
            if (m_ref == -INFINITY) m_ref = raw_max() * sl2;  // may stay -inf (every centroid of the tile kept)
            float rs = 0.f;
            #pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                rs = exp_pass(m_ref == -INFINITY ? 0.f : m_ref);
                const bool need = !(rs <= kCompMaxRowSum);
                if (pass == 1 || !__any_sync(0xffffffffu, need)) break;
                #pragma unroll
                for (int u = 0; u < kBlock / 32; ++u)
                    tmem_ld32(t_lane + s_col + 32 * u, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * u]));
                tmem_ld_wait();
                apply_mask();
                const float m_new = need ? fmaxf(m_ref, raw_max() * sl2) : m_ref;
                if (c > 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[t], (c - 1) & 1, abort_flag))) {
                        ok = false;
                    } else {
                        tc_fence_after();
                        const float alpha = (m_new > m_ref && m_ref != -INFINITY) ? ex2_approx(m_ref - m_new) : 1.f;
                        #pragma unroll 1
                        for (int u = 0; u < D / 8; ++u) {
                            uint32_t o[8];
                            tmem_ld8(t_lane + o_col + 8 * u, o);
                            tmem_ld_wait();
                            #pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st8(t_lane + o_col + 8 * u, o);
                        }
                        tmem_st_wait();
                        l_sum *= alpha;
                    }
                }
                if (!__all_sync(0xffffffffu, ok)) break;
                m_ref = m_new;
            }
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            l_sum += rs;
            tmem_st32(t_lane + s_col, *reinterpret_cast<const uint32_t(*)[32]>(&x[0]));
            tmem_st32(t_lane + s_col + 32, *reinterpret_cast<const uint32_t(*)[32]>(&x[32]));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t]);
        }
        if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
        bool have_c = ok && n > 0;
        if (have_c && !__all_sync(0xffffffffu, mbar_wait(&pv_done[t], (n - 1) & 1, abort_flag))) {
            have_c = false;
            if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
        }
        if (have_c) tc_fence_after();
        if (valid[t]) {
            // ---- merge with the main pass and write the row ----
            // main pass: o1 (normalised) with state (m1, l1); centroids: O2 (not
            // normalised) with state (m2, l2), each centroid weighted by n_b
            const size_t prow = static_cast<size_t>(bh) * a.S + rg;  // the row's state: permuted position
            // o1 and the output: the permuted row, or its T-major token in tiled mode
            const size_t orow = TILED ? static_cast<size_t>(bh) * a.S + tile_token_fast(static_cast<uint32_t>(rg), tl.divs[tc])
                                      : prow;
            const float2 st = a.stats[prow];
            const float m2 = have_c ? m_ref : -INFINITY;
            const float M = fmaxf(st.x, m2);
            const float f1 = st.x == -INFINITY ? 0.f : ex2_approx(st.x - M);
            const float f2 = m2 == -INFINITY ? 0.f : a.weight * ex2_approx(m2 - M);
            const float w1 = st.y * f1;
            const float den = w1 + f2 * (have_c ? l_sum : 0.f);
            const float c1 = den > 0.f ? w1 / den : 0.f, c2 = den > 0.f ? f2 / den : 0.f;
            const float *o1 = a.o1 + orow * D;
            #pragma unroll 1
            for (int u = 0; u < D / 8; ++u) {
                uint32_t o2[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if (have_c) {
                    tmem_ld8(t_lane + o_col + 8 * u, o2);
                    tmem_ld_wait();
                }
                const float4 fa = reinterpret_cast<const float4 *>(o1 + 8 * u)[0];
                const float4 fb = reinterpret_cast<const float4 *>(o1 + 8 * u)[1];
                const float r0 = c1 * fa.x + c2 * __uint_as_float(o2[0]), r1 = c1 * fa.y + c2 * __uint_as_float(o2[1]);
                const float r2 = c1 * fa.z + c2 * __uint_as_float(o2[2]), r3 = c1 * fa.w + c2 * __uint_as_float(o2[3]);
                const float r4 = c1 * fb.x + c2 * __uint_as_float(o2[4]), r5 = c1 * fb.y + c2 * __uint_as_float(o2[5]);
                const float r6 = c1 * fb.z + c2 * __uint_as_float(o2[6]), r7 = c1 * fb.w + c2 * __uint_as_float(o2[7]);
                if (a.out_f32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + orow * D + 8 * u);
                    dst[0] = make_float4(r0, r1, r2, r3);
                    dst[1] = make_float4(r4, r5, r6, r7);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + orow * D + 8 * u);
                    *dst = make_uint4(pack_bf16x2(r0, r1), pack_bf16x2(r2, r3), pack_bf16x2(r4, r5), pack_bf16x2(r6, r7));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

struct CompLayout {
    size_t khi, klo, vhi, vlo, stats, o32, total;
};

CompLayout comp_layout(int BH, int S, int D, int out_f32) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t nb = static_cast<size_t>(S) / kBlock;
    const size_t cent = up(static_cast<size_t>(BH) * nb * D * 2);
    CompLayout L;
    L.khi = 0;
    L.klo = L.khi + cent;
    L.vhi = L.klo + cent;
    L.vlo = L.vhi + cent;
    L.stats = L.vlo + cent;
    L.o32 = L.stats + up(static_cast<size_t>(BH) * S * 8);
    L.total = L.o32 + (out_f32 ? 0 : up(static_cast<size_t>(BH) * S * D * 4));
    return L;
}

template <int D, bool TILED>
vsa_status run_compensated(const AttnLaunch &L, void *workspace, int *status, cudaStream_t st) {
    using C = PairCfg<D>;
    const int nb = L.S / kBlock;
    const CompLayout lay = comp_layout(L.BH, L.S, D, L.out_f32);
    char *ws = static_cast<char *>(workspace);
    auto *khi = reinterpret_cast<__nv_bfloat16 *>(ws + lay.khi);
    auto *klo = reinterpret_cast<__nv_bfloat16 *>(ws + lay.klo);
    auto *vhi = reinterpret_cast<__nv_bfloat16 *>(ws + lay.vhi);
    auto *vlo = reinterpret_cast<__nv_bfloat16 *>(ws + lay.vlo);
    auto *stats = reinterpret_cast<float2 *>(ws + lay.stats);
    float *o1 = L.out_f32 ? static_cast<float *>(L.o) : reinterpret_cast<float *>(ws + lay.o32);

    CompTiling tl = {};
    tl.n = TILED ? L.tiles.n : 1;
    tl.choice = TILED ? L.choice : nullptr;
    for (int c = 0; c < kMaxTiles; ++c) {
        if (TILED && c < L.tiles.n) {
            const int tt = L.tiles.t[c], th = L.tiles.h[c], tw = L.tiles.w[c];
            const int m = tt * th * tw / kBlock;
            tl.divs[c] = make_tile_divs(L.Hg, L.Wg, tt, th, tw);
            tl.m[c] = make_fastdiv(static_cast<uint32_t>(m));
            tl.nthw[c] = make_fastdiv(static_cast<uint32_t>((L.Hg / th) * (L.Wg / tw)));
            tl.ntw[c] = make_fastdiv(static_cast<uint32_t>(L.Wg / tw));
            tl.bt[c] = tt / m;
            tl.th[c] = th;
            tl.tw[c] = tw;
        } else {
            tl.divs[c] = make_tile_divs(1, 1, 1, 1, 1);
            tl.m[c] = tl.nthw[c] = tl.ntw[c] = make_fastdiv(1);
            tl.bt[c] = tl.th[c] = tl.tw[c] = 1;
        }
    }
    centroid_kernel<D, TILED><<<dim3(nb, L.BH), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(L.k),
                                                               static_cast<const __nv_bfloat16 *>(L.v), L.S, nb, khi,
                                                               klo, vhi, vlo, tl);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return check_cuda(e, "centroid launch");

    AttnLaunch m = L;  // the kept blocks: normalised fp32 output and the row states
    m.o = o1;
    m.out_f32 = 1;
    m.stats = stats;
    const vsa_status s = launch_attention(m, status, st);
    if (s != VSA_OK) return s;

    CompMaps maps = {};
    bool ok = make_tile_map(&maps.khi, khi, D, nb, L.BH, 128) && make_tile_map(&maps.klo, klo, D, nb, L.BH, 128) &&
              make_tile_map(&maps.vhi, vhi, D, nb, L.BH, 128) && make_tile_map(&maps.vlo, vlo, D, nb, L.BH, 128);
    if (TILED) {
        for (int c = 0; ok && c < L.tiles.n; ++c)
            ok = make_box_map(&maps.q[c], L.q, D, L.T, L.Hg, L.Wg, L.BH, tl.bt[c], tl.th[c], tl.tw[c]);
    } else {
        ok = ok && make_tile_map(&maps.q[0], L.q, D, L.S, L.BH, 128);
    }
    if (!ok) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
    auto kern = comp_pair_kernel<D, TILED>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(compensation pass)");
    CompArgs a;
    a.S = L.S;
    a.nb = nb;
    a.nct = (nb + kBlock - 1) / kBlock;
    a.nq = nb;
    a.idx = L.idx;
    a.cnt = L.cnt;
    a.cap = L.cap;
    a.list_per_head = L.list_per_head;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.weight = static_cast<float>(kBlock);
    a.stats = stats;
    a.o1 = o1;
    a.out = L.o;
    a.out_f32 = L.out_f32;
    a.status = status;
    kern<<<dim3((nb + 1) / 2, L.BH), kPairThreads, C::SMEM, st>>>(maps, a, tl);
    return check_cuda(cudaGetLastError(), "compensation pass launch");
}

}  // namespace

size_t compensated_workspace_bytes(int BH, int S, int D, int out_f32) {
    return comp_layout(BH, S, D, out_f32).total;
}

vsa_status launch_compensated(const AttnLaunch &L, void *workspace, int *status, cudaStream_t st) {
    if (L.S / kBlock > kMaxCentroidTiles * kBlock)
        return fail(VSA_ERR_UNSUPPORTED, "compensated attention supports at most %d blocks per head",
                    kMaxCentroidTiles * kBlock);
    if (L.tiled)
        return L.D == 128 ? run_compensated<128, true>(L, workspace, status, st)
                          : run_compensated<64, true>(L, workspace, status, st);
    return L.D == 128 ? run_compensated<128, false>(L, workspace, status, st)
                      : run_compensated<64, false>(L, workspace, status, st);
}

}  // namespace vsa
