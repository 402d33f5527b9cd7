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
//   3. comp_pass_kernel: per query tile, S = Q kbar^T (hi and lo MMAs) over
//      all centroids, kept blocks masked, an online softmax with the same
//      lazy running max as the attention kernel, O = P vbar (hi and lo MMAs);
//      then the two partial softmaxes are merged exactly:
//        o = (l1 2^(m1-M) o1 + n_b 2^(m2-M) O2) / (l1 2^(m1-M) + n_b l2 2^(m2-M)),
//      M = max(m1, m2), and written in the output dtype.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

constexpr int kBlock = 128;        // tokens per block (and per centroid tile)
constexpr int kMaxCentroidTiles = 64;  // nb <= 64 * 128 = 8192 blocks per head

// ---------------------------------------------------------------------------
// 1. centroids
// ---------------------------------------------------------------------------
// One CTA per (key block, bh), 256 threads: thread t sums 16-byte chunk
// t % (D / 8) of every (256 / (D / 8))-th row of the block, for K and V.
template <int D>
__global__ void __launch_bounds__(256) centroid_kernel(const __nv_bfloat16 *__restrict__ k,
                                                       const __nv_bfloat16 *__restrict__ v, int S, int nb,
                                                       __nv_bfloat16 *__restrict__ khi, __nv_bfloat16 *__restrict__ klo,
                                                       __nv_bfloat16 *__restrict__ vhi, __nv_bfloat16 *__restrict__ vlo) {
    constexpr int CPR = D / 8;            // 16-byte chunks per row
    constexpr int G = 256 / CPR;          // row groups
    __shared__ float red[2][G][D];
    const int b = blockIdx.x, bh = blockIdx.y;
    const int chunk = threadIdx.x % CPR, g = threadIdx.x / CPR;
    const size_t base = (static_cast<size_t>(bh) * S + static_cast<size_t>(b) * kBlock) * D;
    const uint4 *kr = reinterpret_cast<const uint4 *>(k + base);
    const uint4 *vr = reinterpret_cast<const uint4 *>(v + base);
    float ak[8] = {}, av[8] = {};
    #pragma unroll 4
    for (int r = g; r < kBlock; r += G) {
        const uint4 xk = __ldg(kr + r * CPR + chunk), xv = __ldg(vr + r * CPR + chunk);
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
template <int D>
struct CompCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;            // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = SLAB * KSLABS;  // one 128-row operand tile
    static constexpr int NR = 2;                      // operand ring depth
    static constexpr int O_COL = 128;                 // S at column 0, O after it
    static constexpr int TMEM_COLS = 256;
    static constexpr int N_BARS = 1 + 2 * NR + 1 + 1 + 1 + 1;
    static constexpr int MASK_WORDS = kMaxCentroidTiles * 4;
    static constexpr int SMEM = 1024 + (1 + NR) * TILE_BYTES + N_BARS * 8 + 64 + MASK_WORDS * 4 + kMaxCentroidTiles * 4;
    static_assert(O_COL + D <= TMEM_COLS, "tensor memory");
    static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};
constexpr int kCompThreads = 192;  // warps 0-3 softmax/merge, 4 TMA producer, 5 MMA issuer and TMEM owner
constexpr float kCompMaxRowSum = 16777216.0f;

struct CompArgs {
    int S, nb, nct;            // positions per head, blocks per head, centroid tiles (ceil(nb / 128))
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
    CUtensorMap q, khi, klo, vhi, vlo;
};

template <int D>
__global__ void __launch_bounds__(kCompThreads, 2)
comp_pass_kernel(const __grid_constant__ CompMaps maps, const CompArgs a) {
    using C = CompCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sR = sQ + C::TILE_BYTES;  // [NR][TILE]
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sR + C::NR * C::TILE_BYTES);
    uint64_t *r_full = q_full + 1;
    uint64_t *r_empty = r_full + C::NR;
    uint64_t *s_full = r_empty + C::NR;
    uint64_t *p_full = s_full + 1;
    uint64_t *pv_done = p_full + 1;
    uint64_t *mma_done = pv_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *n_sched = reinterpret_cast<int *>(tmem_slot + 2);
    int *list_ok = reinterpret_cast<int *>(tmem_slot + 3);
    uint32_t *kept = reinterpret_cast<uint32_t *>(tmem_slot + 16);  // [MASK_WORDS] bit j: block j kept
    int *sched = reinterpret_cast<int *>(kept + C::MASK_WORDS);     // centroid tiles with a skipped block

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, bh = blockIdx.y;
    const size_t lrow = (a.list_per_head ? static_cast<size_t>(bh) * a.nb : 0) + qt;
    const int32_t *list = a.idx + lrow * a.cap;
    const int cnt = __ldg(a.cnt + lrow);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NR; ++s) {
            mbar_init(&r_full[s], 1);
            mbar_init(&r_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < C::MASK_WORDS; i += blockDim.x) kept[i] = 0u;
    if (warp == 0) {  // validate the list as the attention kernel does
        bool ok = cnt >= 1 && cnt <= a.cap;
        if (ok) {
            for (int j = lane; j < cnt; j += 32) {
                const int b = __ldg(list + j);
                ok = ok && b >= 0 && b < a.nb && (j == 0 || __ldg(list + j - 1) < b);
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (lane == 0) *list_ok = ok ? 1 : 0;
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();
    if (*list_ok) {
        for (int j = threadIdx.x; j < cnt; j += blockDim.x) {
            const int b = __ldg(list + j);
            atomicOr(&kept[b >> 5], 1u << (b & 31));
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // the centroid tiles that hold at least one skipped block (none if the
        // list is invalid: the output then keeps the main pass's zeros)
        int n = 0;
        if (*list_ok) {
            for (int c = 0; c < a.nct; ++c) {
                bool any = false;
                for (int w = 0; w < 4; ++w) {
                    const int b0 = c * kBlock + w * 32;
                    if (b0 >= a.nb) break;
                    const int valid = a.nb - b0 >= 32 ? 32 : a.nb - b0;
                    const uint32_t vm = valid == 32 ? ~0u : ((1u << valid) - 1u);
                    any = any || ((~kept[c * 4 + w]) & vm) != 0u;
                }
                if (any) sched[n++] = c;
            }
        } else {
            report(a.status, DEV_RUNTIME);
        }
        *n_sched = n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n = *n_sched;

    if (warp == 4) {
        // ================= TMA producer =================
        // per scheduled centroid tile: kbar hi, kbar lo (for QK), vbar hi, vbar lo (for PV)
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&maps.q);
            mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
            for (int s = 0; s < C::KSLABS; ++s)
                tma_load_3d(sQ + s * C::SLAB, &maps.q, q_full, s * 64, qt * kBlock, bh);
            const CUtensorMap *ops[4] = {&maps.khi, &maps.klo, &maps.vhi, &maps.vlo};
            uint32_t lc = 0;
            bool ok = true;
            for (int j = 0; ok && j < n; ++j) {
                const int c = sched[j];
                for (int op = 0; ok && op < 4; ++op, ++lc) {
                    const int slot = lc % C::NR;
                    if (lc >= static_cast<uint32_t>(C::NR) &&
                        !mbar_wait(&r_empty[slot], ((lc / C::NR) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&r_full[slot], C::TILE_BYTES);
                    for (int s = 0; s < C::KSLABS; ++s)
                        tma_load_3d(sR + slot * C::TILE_BYTES + s * C::SLAB, ops[op], &r_full[slot], s * 64,
                                    c * kBlock, bh);
                }
            }
            if (!ok) {
                if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the loads already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                for (uint32_t c = lc > static_cast<uint32_t>(C::NR) ? lc - C::NR : 0; c < lc; ++c)
                    mbar_wait(&r_full[c % C::NR], (c / C::NR) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ================= MMA issuer =================
        // per tile j: QK(j) = Q khi^T + Q klo^T into S (after PV(j-1) has read
        // the P over S), then PV(j) = P vhi + P vlo into O once P is written
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBlock, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dRk = sdesc_sw128(smem_u32(sR), 16, 1024);
            const uint64_t dRv = sdesc_sw128(smem_u32(sR), C::SLAB, 1024);
            constexpr uint64_t kTile16 = C::TILE_BYTES >> 4;
            uint32_t lc = 0;
            bool ok = mbar_wait(q_full, 0, abort_flag);
            for (int j = 0; ok && j < n; ++j) {
                // QK(j)
                const int s0 = lc % C::NR, s1 = (lc + 1) % C::NR;
                ok = mbar_wait(&r_full[s0], (lc / C::NR) & 1, abort_flag) &&
                     mbar_wait(&r_full[s1], ((lc + 1) / C::NR) & 1, abort_flag) &&
                     (j == 0 || mbar_wait(pv_done, (j - 1) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                #pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t k0 = dRk + ((part == 0 ? s0 : s1) * kTile16);
                    #pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                        umma_bf16(tmem, dQ + off, k0 + off, idesc_qk, (part > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(s_full);
                umma_commit(&r_empty[s0]);
                umma_commit(&r_empty[s1]);
                lc += 2;
                // PV(j)
                const int s2 = lc % C::NR, s3 = (lc + 1) % C::NR;
                ok = mbar_wait(p_full, j & 1, abort_flag) &&
                     mbar_wait(&r_full[s2], (lc / C::NR) & 1, abort_flag) &&
                     mbar_wait(&r_full[s3], ((lc + 1) / C::NR) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                #pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t v0 = dRv + ((part == 0 ? s2 : s3) * kTile16);
                    #pragma unroll
                    for (int kk = 0; kk < kBlock / 16; ++kk)
                        umma_bf16_ts(tmem + C::O_COL, tmem + kk * 8, v0 + static_cast<uint64_t>((kk * 2048) >> 4),
                                     idesc_pv, (j > 0 || part > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(pv_done);
                umma_commit(&r_empty[s2]);
                umma_commit(&r_empty[s3]);
                lc += 2;
            }
            if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ================= softmax over the centroids, then the merge (warps 0-3) =================
        const int wq = warp, row = wq * 32 + lane;
        const int rg = qt * kBlock + row;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const float sl2 = a.scale_log2;
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int c = sched[j];
            if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            uint32_t x[kBlock];
            #pragma unroll
            for (int u = 0; u < kBlock / 32; ++u)
                tmem_ld32(t_lane + 32 * u, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * u]));
            tmem_ld_wait();
            // a centroid takes part iff its block exists and is not kept
            uint32_t skip[4];
            #pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int b0 = c * kBlock + w * 32;
                const int valid = a.nb - b0 >= 32 ? 32 : (a.nb - b0 > 0 ? a.nb - b0 : 0);
                const uint32_t vm = valid == 32 ? ~0u : ((1u << valid) - 1u);
                skip[w] = ~kept[c * 4 + w] & vm;
            }
            // per 32 columns, a branch the whole CTA takes alike (the mask
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
            if (m_ref == -INFINITY) m_ref = raw_max() * sl2;
            float rs = 0.f;
            #pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                rs = exp_pass(m_ref == -INFINITY ? 0.f : m_ref);
                const bool need = !(rs <= kCompMaxRowSum);
                if (pass == 1 || !__any_sync(0xffffffffu, need)) break;
                #pragma unroll
                for (int u = 0; u < kBlock / 32; ++u)
                    tmem_ld32(t_lane + 32 * u, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * u]));
                tmem_ld_wait();
                apply_mask();
                const float m_new = need ? fmaxf(m_ref, raw_max() * sl2) : m_ref;
                if (j > 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1, abort_flag))) {
                        ok = false;
                    } else {
                        tc_fence_after();
                        const float alpha = (m_new > m_ref && m_ref != -INFINITY) ? ex2_approx(m_ref - m_new) : 1.f;
                        #pragma unroll 1
                        for (int u = 0; u < D / 8; ++u) {
                            uint32_t o[8];
                            tmem_ld8(t_lane + C::O_COL + 8 * u, o);
                            tmem_ld_wait();
                            #pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st8(t_lane + C::O_COL + 8 * u, o);
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
            tmem_st32(t_lane, *reinterpret_cast<const uint32_t(*)[32]>(&x[0]));
            tmem_st32(t_lane + 32, *reinterpret_cast<const uint32_t(*)[32]>(&x[32]));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
        bool have_c = ok && n > 0;
        if (have_c && !__all_sync(0xffffffffu, mbar_wait(pv_done, (n - 1) & 1, abort_flag))) {
            have_c = false;
            if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
        }
        if (have_c) tc_fence_after();
        // ---- merge with the main pass and write the row ----
        // main pass: o1 (normalised) with state (m1, l1); centroids: O2 (not
        // normalised) with state (m2, l2), each centroid weighted by n_b
        const size_t prow = static_cast<size_t>(bh) * a.S + rg;
        const float2 st = a.stats[prow];
        const float m2 = have_c ? m_ref : -INFINITY;
        const float M = fmaxf(st.x, m2);
        const float f1 = st.x == -INFINITY ? 0.f : ex2_approx(st.x - M);
        const float f2 = m2 == -INFINITY ? 0.f : a.weight * ex2_approx(m2 - M);
        const float w1 = st.y * f1;
        const float den = w1 + f2 * (have_c ? l_sum : 0.f);
        const float c1 = den > 0.f ? w1 / den : 0.f, c2 = den > 0.f ? f2 / den : 0.f;
        const float *o1 = a.o1 + prow * D;
        #pragma unroll 1
        for (int u = 0; u < D / 8; ++u) {
            uint32_t o2[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (have_c) {
                tmem_ld8(t_lane + C::O_COL + 8 * u, o2);
                tmem_ld_wait();
            }
            const float4 fa = reinterpret_cast<const float4 *>(o1 + 8 * u)[0];
            const float4 fb = reinterpret_cast<const float4 *>(o1 + 8 * u)[1];
            const float r0 = c1 * fa.x + c2 * __uint_as_float(o2[0]), r1 = c1 * fa.y + c2 * __uint_as_float(o2[1]);
            const float r2 = c1 * fa.z + c2 * __uint_as_float(o2[2]), r3 = c1 * fa.w + c2 * __uint_as_float(o2[3]);
            const float r4 = c1 * fb.x + c2 * __uint_as_float(o2[4]), r5 = c1 * fb.y + c2 * __uint_as_float(o2[5]);
            const float r6 = c1 * fb.z + c2 * __uint_as_float(o2[6]), r7 = c1 * fb.w + c2 * __uint_as_float(o2[7]);
            if (a.out_f32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + prow * D + 8 * u);
                dst[0] = make_float4(r0, r1, r2, r3);
                dst[1] = make_float4(r4, r5, r6, r7);
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + prow * D + 8 * u);
                *dst = make_uint4(pack_bf16x2(r0, r1), pack_bf16x2(r2, r3), pack_bf16x2(r4, r5), pack_bf16x2(r6, r7));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
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

template <int D>
vsa_status run_compensated(const AttnLaunch &L, void *workspace, int *status, cudaStream_t st) {
    using C = CompCfg<D>;
    const int nb = L.S / kBlock;
    const CompLayout lay = comp_layout(L.BH, L.S, D, L.out_f32);
    char *ws = static_cast<char *>(workspace);
    auto *khi = reinterpret_cast<__nv_bfloat16 *>(ws + lay.khi);
    auto *klo = reinterpret_cast<__nv_bfloat16 *>(ws + lay.klo);
    auto *vhi = reinterpret_cast<__nv_bfloat16 *>(ws + lay.vhi);
    auto *vlo = reinterpret_cast<__nv_bfloat16 *>(ws + lay.vlo);
    auto *stats = reinterpret_cast<float2 *>(ws + lay.stats);
    float *o1 = L.out_f32 ? static_cast<float *>(L.o) : reinterpret_cast<float *>(ws + lay.o32);

    centroid_kernel<D><<<dim3(nb, L.BH), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(L.k),
                                                        static_cast<const __nv_bfloat16 *>(L.v), L.S, nb, khi, klo,
                                                        vhi, vlo);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return check_cuda(e, "centroid launch");

    AttnLaunch m = L;  // the kept blocks: normalised fp32 output and the row states
    m.o = o1;
    m.out_f32 = 1;
    m.stats = stats;
    const vsa_status s = launch_attention(m, status, st);
    if (s != VSA_OK) return s;

    CompMaps maps = {};
    const bool ok = make_tile_map(&maps.q, L.q, D, L.S, L.BH, 128) && make_tile_map(&maps.khi, khi, D, nb, L.BH, 128) &&
                    make_tile_map(&maps.klo, klo, D, nb, L.BH, 128) && make_tile_map(&maps.vhi, vhi, D, nb, L.BH, 128) &&
                    make_tile_map(&maps.vlo, vlo, D, nb, L.BH, 128);
    if (!ok) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
    auto kern = comp_pass_kernel<D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(compensation pass)");
    CompArgs a;
    a.S = L.S;
    a.nb = nb;
    a.nct = (nb + kBlock - 1) / kBlock;
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
    kern<<<dim3(nb, L.BH), kCompThreads, C::SMEM, st>>>(maps, a);
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
    return L.D == 128 ? run_compensated<128>(L, workspace, status, st) : run_compensated<64>(L, workspace, status, st);
}

}  // namespace vsa
