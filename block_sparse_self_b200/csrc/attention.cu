// attention.cu -- block-sparse and sliding-window attention on tcgen05 tensor
// cores (sm_100a).
//
// Semantics: "Adaptive tiling (SPADE)", Recipe and recipe note (block mask
// expanded to tokens, skipped blocks dropped, softmax attention over the kept
// keys); "fastvideo/mlx_runtime/windowed_attention.py", Window policy and
// _key_ranges_for_block (work only on the key blocks the window or the sinks
// reach).
//
// One CTA computes one 128-row query tile of one (batch, head).  Warps:
//   0-3  softmax + epilogue: thread t owns query row t (TMEM lane t);
//   4    TMA producer: Q once, then K/V tiles of each listed key block;
//   5    MMA issuer (one elected thread) and TMEM owner.
// Per key block j:  S_j = Q K_j^T  -> TMEM (double-buffered, fp32);
//                   P_j = exp2(scale*log2e*S_j - m) -> bf16 in shared memory;
//                   O  += P_j V_j  -> TMEM (fp32).
// The running max m is only raised (and O, l rescaled) when a row's max grows
// by more than 2^8; the final O / l is exact either way because O and l always
// share the same reference.  All waits are bounded (see common.cuh).
//
// Tiled mode (TILED): Q, K, V and O stay in T-major order and each (b, head)
// uses its chosen tiling; a block of BN tokens is one 5-D TMA box of whole
// (h, w) planes of its tile, which lands in shared memory as BN rows in
// tile-contiguous order, and the epilogue writes each row to its token.  On a
// zero-padded grid (PAD; "Adaptive tiling (SPADE)", Deviations and notes) the
// boxes read zeros past the real tensors, keys there are masked in the blocks
// that cross the edge, rows there are not written and query blocks wholly in
// the padding are skipped.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

struct AttnArgs {
    int S, BH, nq;   // S: positions per head (tiled mode: of the padded grid)
    int S_out;       // rows per head of o (tiled mode: real tokens)
    // block-list mode
    const int32_t *idx, *cnt;
    int cap, list_per_head, group, nb;
    // window mode
    int half, sink, dense;
    float scale_log2;
    void *out;
    int out_f32;
    int *status;
    // tiled mode
    int H, W;  // the padded grid's frame
    RealGrid real;
    TileSet tiles;
    const int32_t *choice;
    struct BoxGeom {
        FastDiv m, nthw, ntw;  // m = volume / BN, tiles per frame, tiles per tile row
        FastDiv bhw, bw;       // box frame (th * tw) and row (tw): key column -> (dt, dh, dw)
        int bt;                // frames of one BN-token box
    } geom[kMaxTiles];
};

// Tensor maps: slot 0 only, or one per candidate tiling in tiled mode.
struct AttnMaps {
    CUtensorMap q[kMaxTiles], k[kMaxTiles], v[kMaxTiles];
};
static_assert(sizeof(AttnMaps) + sizeof(AttnArgs) <= 4096, "kernel parameters");

// Block b of a head in tiled mode: the TMA coordinates (w, h, t) of its box.
struct BoxAt {
    int w, h, t;
};
__device__ __forceinline__ BoxAt box_at(uint32_t b, const AttnArgs::BoxGeom &g, int th, int tw) {
    const uint32_t tile = fdiv(b, g.m), part = b - tile * g.m.d;
    const uint32_t ct = fdiv(tile, g.nthw), rem = tile - ct * g.nthw.d;
    const uint32_t ch = fdiv(rem, g.ntw), cw = rem - ch * g.ntw.d;
    return BoxAt{static_cast<int>(cw) * tw, static_cast<int>(ch) * th, static_cast<int>(ct * g.m.d + part) * g.bt};
}

template <int D, int BN>
struct Cfg {
    static constexpr int BM = 128;
    static constexpr int KSLABS = D / 64;           // 128-byte slabs along D
    static constexpr int PSLABS = (BN + 63) / 64;   // 128-byte slabs along the keys of P
    static constexpr int SLAB_Q = BM * 128;         // one slab of 128 rows
    static constexpr int Q_BYTES = SLAB_Q * KSLABS;
    static constexpr int K_BYTES = BN * 128 * KSLABS;
    static constexpr int V_BYTES = BN * 128 * KSLABS;
    static constexpr int P_BYTES = BM * 128 * PSLABS;
    static constexpr int BUDGET = 200 * 1024;
    static constexpr int NS = (Q_BYTES + 4 * (K_BYTES + V_BYTES) + P_BYTES <= BUDGET)   ? 4
                              : (Q_BYTES + 3 * (K_BYTES + V_BYTES) + P_BYTES <= BUDGET) ? 3
                                                                                       : 2;
    static constexpr int O_COL = 2 * BN;
    static constexpr int COLS_USED = 2 * BN + D;
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                     : COLS_USED <= 256 ? 256 : 512;
    static constexpr int N_BARS = 1 + 3 * NS + 2 + 2 + 1 + 1 + 1;
    static constexpr int SMEM = 1024 + Q_BYTES + NS * (K_BYTES + V_BYTES) + P_BYTES + N_BARS * 8 + 64;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BN == 32 || BN == 64 || BN == 128, "block");
    static_assert(COLS_USED <= 512, "tensor memory");
};

constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8

template <int D, int BN, bool WINDOW, bool TILED, bool PAD>
__global__ void __launch_bounds__(192, 1)
attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
    using C = Cfg<D, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sK = sQ + C::Q_BYTES;
    uint8_t *sV = sK + C::NS * C::K_BYTES;
    uint8_t *sP = sV + C::NS * C::V_BYTES;
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sP + C::P_BYTES);
    uint64_t *k_full = q_full + 1;
    uint64_t *v_full = k_full + C::NS;
    uint64_t *kv_empty = v_full + C::NS;
    uint64_t *s_full = kv_empty + C::NS;
    uint64_t *s_empty = s_full + 2;
    uint64_t *p_full = s_empty + 2;
    uint64_t *pv_done = p_full + 1;
    uint64_t *mma_done = pv_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *list_ok = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = blockIdx.x, bh = blockIdx.y;
    const int q_row0 = qt * BN;
    const int S = a.S;

    // ---- the key-block schedule of this query tile ----------------------
    int n_kb = 0;
    int r0_len = 0, r1_start = 0;  // window: blocks [0, r0_len) then [r1_start, ...)
    const int32_t *list = nullptr;
    if constexpr (WINDOW) {
        if (a.dense) {
            r0_len = (S + BN - 1) / BN;
            n_kb = r0_len;
        } else {
            const int qe = min(q_row0 + BN, S);
            const int lo = max(0, q_row0 - a.half), hi = min(S, qe + a.half);
            const int lb0 = lo / BN, lb1 = (hi + BN - 1) / BN;
            const int sb = (a.sink + BN - 1) / BN;
            if (sb == 0) {
                r0_len = 0; r1_start = lb0; n_kb = lb1 - lb0;
            } else if (lb0 <= sb) {
                r0_len = max(lb1, sb); n_kb = r0_len;
            } else {
                r0_len = sb; r1_start = lb0; n_kb = sb + (lb1 - lb0);
            }
        }
    } else {
        const size_t lrow = (a.list_per_head ? static_cast<size_t>(bh) * a.nb : 0) + qt;
        list = a.idx + lrow * a.cap;
        n_kb = __ldg(a.cnt + lrow);
    }
    auto kblock = [&](int j) -> int {
        if constexpr (WINDOW) return j < r0_len ? j : r1_start + (j - r0_len);
        else return __ldg(list + j);
    };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        *list_ok = 1;
        fence_mbar_init();
    }
    if constexpr (!WINDOW) {
        if (warp == 0) {  // validate the list: 1 <= cnt <= cap, strictly ascending, in [0, nb)
            bool ok = n_kb >= 1 && n_kb <= a.cap;
            if (ok) {
                for (int j = lane; j < n_kb; j += 32) {
                    const int v = __ldg(list + j);
                    ok = ok && v >= 0 && v < a.nb && (j == 0 || __ldg(list + j - 1) < v);
                }
            }
            ok = __all_sync(0xffffffffu, ok);
            if (lane == 0 && !ok) *list_ok = 0;
        }
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool list_valid = true;
    if constexpr (!WINDOW) {
        list_valid = *list_ok != 0;
        if (!list_valid) {
            if (threadIdx.x == 0) report(a.status, DEV_RUNTIME);
            n_kb = 0;
        }
    }
    int tc = 0;             // tiled mode: this head's tiling
    bool q_skip = false;    // tiled mode: the query block has no row to write
    if constexpr (TILED) {
        if (a.choice) tc = __ldg(a.choice + bh);
        if (tc < 0 || tc >= a.tiles.n) {  // the head is left unwritten
            if (threadIdx.x == 0) report(a.status, DEV_RUNTIME);
            tc = 0;
            n_kb = 0;
            q_skip = true;
        }
        if constexpr (PAD) {
            const BoxAt qb = box_at(static_cast<uint32_t>(qt), a.geom[tc], a.tiles.h[tc], a.tiles.w[tc]);
            if (qb.t >= a.real.T || qb.h >= a.real.H || qb.w >= a.real.W) {  // wholly in the padding
                n_kb = 0;
                q_skip = true;
            }
        }
    }
    const int th = a.tiles.h[tc], tw = a.tiles.w[tc];
    const CUtensorMap *tmQ = &maps.q[tc], *tmK = &maps.k[tc], *tmV = &maps.v[tc];
    // block b's BN rows of Q, K or V into dst (slabs of 64 columns, `slab` bytes apart)
    auto load_block = [&](uint8_t *dst, int slab, const CUtensorMap *map, uint64_t *bar, int b) {
        if constexpr (TILED) {
            const BoxAt c = box_at(static_cast<uint32_t>(b), a.geom[tc], th, tw);
            for (int s = 0; s < C::KSLABS; ++s) tma_load_5d(dst + s * slab, map, bar, s * 64, c.w, c.h, c.t, bh);
        } else {
            for (int s = 0; s < C::KSLABS; ++s) tma_load_3d(dst + s * slab, map, bar, s * 64, b * BN, bh);
        }
    };

    if (warp == 4) {
        // ================= TMA producer =================
        if (lane == 0 && n_kb > 0) {
            tma_prefetch_desc(tmQ);
            tma_prefetch_desc(tmK);
            tma_prefetch_desc(tmV);
            mbar_arrive_expect_tx(q_full, BN * 128 * C::KSLABS);
            load_block(sQ, C::SLAB_Q, tmQ, q_full, qt);
            int issued = 0;
            for (int j = 0; j < n_kb; ++j) {
                const int st = j % C::NS;
                if (j >= C::NS && !mbar_wait(&kv_empty[st], ((j / C::NS) - 1) & 1, abort_flag)) {
                    if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                    break;
                }
                const int kb = kblock(j);
                mbar_arrive_expect_tx(&k_full[st], C::K_BYTES);
                load_block(sK + st * C::K_BYTES, BN * 128, tmK, &k_full[st], kb);
                mbar_arrive_expect_tx(&v_full[st], C::V_BYTES);
                load_block(sV + st * C::V_BYTES, BN * 128, tmV, &v_full[st], kb);
                issued = j + 1;
            }
            if (*abort_flag) {
                // let every load already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                for (int j = max(0, issued - C::NS); j < issued; ++j) {
                    mbar_wait(&k_full[j % C::NS], (j / C::NS) & 1, nullptr);
                    mbar_wait(&v_full[j % C::NS], (j / C::NS) & 1, nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            bool ok = true;
            auto issue_qk = [&](int j) -> bool {
                const int st = j % C::NS, b = j & 1;
                if (!mbar_wait(&k_full[st], (j / C::NS) & 1, abort_flag)) return false;
                if (j >= 2 && !mbar_wait(&s_empty[b], ((j >> 1) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t d = tmem + b * BN;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    const uint64_t da = sdesc_sw128(aQ + (kk >> 2) * C::SLAB_Q + koff, 16, 1024);
                    const uint64_t db = sdesc_sw128(aK + st * C::K_BYTES + (kk >> 2) * (BN * 128) + koff, 16, 1024);
                    umma_bf16(d, da, db, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[b]);
                return true;
            };
            if (n_kb > 0) {
                ok = mbar_wait(q_full, 0, abort_flag);
                if (ok) ok = issue_qk(0);
                for (int j = 0; ok && j < n_kb; ++j) {
                    if (j + 1 < n_kb && !issue_qk(j + 1)) { ok = false; break; }
                    const int st = j % C::NS;
                    if (!mbar_wait(p_full, j & 1, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&v_full[st], (j / C::NS) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    #pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        const uint64_t da = sdesc_sw128(aP + (kk >> 2) * (C::BM * 128) + (kk & 3) * 32, 16, 1024);
                        const uint64_t db = sdesc_sw128(aV + st * C::V_BYTES + kk * 2048, BN * 128, 1024);
                        umma_bf16(tmem + C::O_COL, da, db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(pv_done);
                    umma_commit(&kv_empty[st]);
                }
                if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
            }
            // every MMA issued so far completes before TMEM is released
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ================= softmax + epilogue (warps 0-3) =================
        const int row = threadIdx.x;                 // 0..127: TMEM lane = query row in the tile
        const int rows_valid = BN;                   // rows of the tile that exist
        const bool warp_valid = warp * 32 < rows_valid;
        const int rg = q_row0 + row;                 // position in the head
        bool row_valid = warp_valid && row < rows_valid && rg < S && !q_skip;
        // output row: the position itself, or its T-major token in tiled mode
        int orow_in_head = rg;
        if constexpr (TILED) {
            int pt, ph, pw;
            tile_coords(row_valid ? rg : 0, a.H, a.W, a.tiles.t[tc], th, tw, pt, ph, pw);
            if constexpr (PAD) {
                const int tok = real_token(pt, ph, pw, a.real);
                row_valid = row_valid && tok >= 0;
                orow_in_head = tok < 0 ? 0 : tok;
            } else {
                orow_in_head = (pt * a.H + ph) * a.W + pw;
            }
        }
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = a.scale_log2;
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kb; ++j) {
            const int b = j & 1;
            if (!mbar_wait(&s_full[b], (j >> 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t raw[BN];
            if (warp_valid) {
                #pragma unroll
                for (int c = 0; c < BN / 32; ++c)
                    tmem_ld32(t_lane + b * BN + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&raw[32 * c]));
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[b]);

            bool waited_pv = (j == 0);
            if (warp_valid) {
                float *x = reinterpret_cast<float *>(raw);  // scores, then probabilities, in place
                const int kb = kblock(j);
                const int ks = kb * BN;
                bool full;
                if constexpr (WINDOW) {
                    const int qe = min(q_row0 + BN, S);
                    full = (ks + BN <= S) &&
                           (a.dense || ks + BN <= a.sink || max(qe - 1 - ks, ks + BN - 1 - q_row0) <= a.half);
                    if (!full) {
                        #pragma unroll
                        for (int c = 0; c < BN; ++c) {
                            const int kc = ks + c;
                            const int dd = rg > kc ? rg - kc : kc - rg;
                            const bool vis = kc < S && (a.dense || kc < a.sink || dd <= a.half);
                            if (!vis) x[c] = -INFINITY;
                        }
                    }
                } else {
                    full = a.group <= 0;
                    if (!full) {
                        // key ks + c is in the row's group iff it lies in [g0, g0 + group)
                        const int g0 = (rg / a.group) * a.group - ks;
                        #pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (c < g0 || c >= g0 + a.group) x[c] = -INFINITY;
                    }
                    if constexpr (PAD) {
                        // a key box crossing the real grid's edge: mask its padding columns
                        // (column u * 32 + lane is bit lane of kv[u])
                        const AttnArgs::BoxGeom &g = a.geom[tc];
                        const BoxAt c = box_at(static_cast<uint32_t>(kb), g, th, tw);
                        if (c.t + g.bt > a.real.T || c.h + th > a.real.H || c.w + tw > a.real.W) {
                            uint32_t kv[BN / 32];
                            #pragma unroll
                            for (int u = 0; u < BN / 32; ++u) {
                                const uint32_t col = static_cast<uint32_t>(u * 32 + lane);
                                const uint32_t dt = fdiv(col, g.bhw), r2 = col - dt * g.bhw.d;
                                const uint32_t dh = fdiv(r2, g.bw), dw = r2 - dh * g.bw.d;
                                kv[u] = __ballot_sync(0xffffffffu, c.t + static_cast<int>(dt) < a.real.T &&
                                                                       c.h + static_cast<int>(dh) < a.real.H &&
                                                                       c.w + static_cast<int>(dw) < a.real.W);
                            }
                            #pragma unroll
                            for (int cc = 0; cc < BN; ++cc)
                                if (!((kv[cc >> 5] >> (cc & 31)) & 1u)) x[cc] = -INFINITY;
                        }
                    }
                }
                float mb = -INFINITY;
                #pragma unroll
                for (int c = 0; c < BN; ++c) mb = fmaxf(mb, x[c]);
                mb *= sl2;
                const float m_new = fmaxf(m_ref, mb);
                const bool need = m_new > m_ref + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    if (j > 0) {
                        if (!mbar_wait(pv_done, (j - 1) & 1, abort_flag)) {
                            ok = false;
                        } else {
                            waited_pv = true;
                            tc_fence_after();
                            const float alpha = (need && m_ref != -INFINITY) ? ex2_approx(m_ref - m_new) : 1.f;
                            #pragma unroll
                            for (int c = 0; c < D / 32; ++c) {
                                uint32_t o[32];
                                tmem_ld32(t_lane + C::O_COL + 32 * c, o);
                                tmem_ld_wait();
                                #pragma unroll
                                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                                tmem_st32(t_lane + C::O_COL + 32 * c, o);
                            }
                            tmem_st_wait();
                            l_sum *= alpha;
                        }
                    }
                    if (need) m_ref = m_new;
                }
                if (!__all_sync(0xffffffffu, ok)) ok = false;
                if (!ok) break;
                const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
                // the row sum adds the bf16-rounded P that the PV MMA multiplies
                float s0 = 0.f, s1 = 0.f;
                #pragma unroll
                for (int c = 0; c < BN; c += 2) {
                    const uint32_t pk = pack_bf16x2(ex2_approx(fmaf(x[c], sl2, -m_use)),
                                                    ex2_approx(fmaf(x[c + 1], sl2, -m_use)));
                    raw[c >> 1] = pk;
                    add_bf16x2_f32(pk, s0, s1);
                }
                l_sum += s0 + s1;
            } else {
                #pragma unroll
                for (int c = 0; c < BN / 2; ++c) raw[c] = 0u;
            }
            if (!waited_pv) {
                if (!mbar_wait(pv_done, (j - 1) & 1, abort_flag)) { ok = false; break; }
            }
            // P row -> shared memory, 128-byte swizzle, K-major (keys along the row)
            #pragma unroll
            for (int cc = 0; cc < BN / 8; ++cc) {
                const int slab = cc >> 3, cpos = (cc & 7) ^ (row & 7);
                uint4 v = make_uint4(raw[4 * cc], raw[4 * cc + 1], raw[4 * cc + 2], raw[4 * cc + 3]);
                *reinterpret_cast<uint4 *>(sP + slab * (C::BM * 128) + row * 128 + cpos * 16) = v;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }

        // ---- epilogue: O / l -> global ----
        const size_t orow = static_cast<size_t>(bh) * a.S_out + orow_in_head;
        bool have_o = ok && n_kb > 0;
        if (have_o) {
            if (!mbar_wait(pv_done, (n_kb - 1) & 1, abort_flag)) {
                have_o = false;
                if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
            }
        }
        if (have_o && warp_valid) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(t_lane + C::O_COL + 32 * c, o);
                tmem_ld_wait();
                if (row_valid) {
                    if (a.out_f32) {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + orow * D + 32 * c);
                        #pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                                 __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
                    } else {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + orow * D + 32 * c);
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t *u = &o[8 * e];
                            dst[e] = make_uint4(pack_bf16x2(__uint_as_float(u[0]) * inv, __uint_as_float(u[1]) * inv),
                                                pack_bf16x2(__uint_as_float(u[2]) * inv, __uint_as_float(u[3]) * inv),
                                                pack_bf16x2(__uint_as_float(u[4]) * inv, __uint_as_float(u[5]) * inv),
                                                pack_bf16x2(__uint_as_float(u[6]) * inv, __uint_as_float(u[7]) * inv));
                        }
                    }
                }
            }
            if (row_valid && l_sum <= 0.f) report(a.status, DEV_RUNTIME);  // empty key set
        } else if (row_valid && !list_valid) {
            // invalid list: the row is written as zeros
            if (a.out_f32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + orow * D);
                for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + orow * D);
                for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
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

template <int D, int BN, bool WINDOW, bool TILED = false, bool PAD = false>
vsa_status run(const AttnLaunch &L, int *status, cudaStream_t st) {
    using C = Cfg<D, BN>;
    AttnMaps maps = {};  // copied into the launch parameters
    bool ok = true;
    if constexpr (TILED) {
        for (int c = 0; c < L.tiles.n; ++c) {
            const int m = L.tiles.t[c] * L.tiles.h[c] * L.tiles.w[c] / BN;
            const int bt = L.tiles.t[c] / m, bhh = L.tiles.h[c], bw = L.tiles.w[c];
            // the real tensors: boxes reaching past them read zeros
            ok = ok && make_box_map(&maps.q[c], L.q, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw) &&
                 make_box_map(&maps.k[c], L.k, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw) &&
                 make_box_map(&maps.v[c], L.v, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw);
        }
    } else {
        ok = make_tile_map(&maps.q[0], L.q, D, L.S, L.BH, BN) && make_tile_map(&maps.k[0], L.k, D, L.S, L.BH, BN) &&
             make_tile_map(&maps.v[0], L.v, D, L.S, L.BH, BN);
    }
    if (!ok) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
    auto kern = attn_kernel<D, BN, WINDOW, TILED, PAD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(attention)");
    AttnArgs a;
    const int positions = TILED ? L.Tp * L.Hp * L.Wp : L.S;
    a.S = positions;
    a.S_out = L.S;
    a.BH = L.BH;
    a.nq = (positions + BN - 1) / BN;
    a.idx = L.idx;
    a.cnt = L.cnt;
    a.cap = L.cap;
    a.list_per_head = L.list_per_head;
    a.group = L.group;
    a.nb = L.nb;
    a.half = L.half;
    a.sink = L.sink;
    a.dense = L.dense;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.out = L.o;
    a.out_f32 = L.out_f32;
    a.status = status;
    a.H = TILED ? L.Hp : L.Hg;
    a.W = TILED ? L.Wp : L.Wg;
    a.real = RealGrid{L.T, L.Hg, L.Wg};
    a.tiles = L.tiles;
    a.choice = L.choice;
    if (!TILED) a.tiles.n = 1;
    for (int c = 0; c < kMaxTiles; ++c) {
        auto &g = a.geom[c];
        if (TILED && c < L.tiles.n) {
            const int tt = L.tiles.t[c], th = L.tiles.h[c], tw = L.tiles.w[c];
            const int m = tt * th * tw / BN;
            g.m = make_fastdiv(m);
            g.nthw = make_fastdiv((L.Hp / th) * (L.Wp / tw));
            g.ntw = make_fastdiv(L.Wp / tw);
            g.bhw = make_fastdiv(th * tw);
            g.bw = make_fastdiv(tw);
            g.bt = tt / m;
        } else {
            g.m = g.nthw = g.ntw = g.bhw = g.bw = make_fastdiv(1);
            g.bt = 1;
        }
    }
    dim3 grid(a.nq, L.BH);
    kern<<<grid, 192, C::SMEM, st>>>(maps, a);
    return check_cuda(cudaGetLastError(), "attention launch");
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [BH, S, D] bf16 viewed as a 3-D tensor (D, S, BH); box (64, rows, 1), 128-byte swizzle.
bool make_tile_map(CUtensorMap *m, const void *ptr, int D, int S, int BH, int rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


bool make_scores_store_map(CUtensorMap *m, float *ptr, int nb, int BH) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(nb), static_cast<cuuint64_t>(nb), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(nb) * 4, static_cast<cuuint64_t>(nb) * nb * 4};
    cuuint32_t box[3] = {32, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_box_map(CUtensorMap *m, const void *ptr, int D, int T, int H, int W, int BH, int bt, int bh, int bw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t e = 2;  // bf16
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[4] = {static_cast<cuuint64_t>(D) * e, static_cast<cuuint64_t>(W) * D * e,
                             static_cast<cuuint64_t>(H) * W * D * e, static_cast<cuuint64_t>(T) * H * W * D * e};
    cuuint32_t box[5] = {64, static_cast<cuuint32_t>(bw), static_cast<cuuint32_t>(bh), static_cast<cuuint32_t>(bt), 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

vsa_status launch_attention(const AttnLaunch &L, int *status, cudaStream_t st) {
    if (L.block == 128) return launch_attention_pp(L, status, st);  // two query tiles per CTA
    if (L.tiled) {
        const bool pad = L.Tp * L.Hp * L.Wp != L.S;
        if (L.D == 128) {
            if (L.block == 64) return pad ? run<128, 64, false, true, true>(L, status, st) : run<128, 64, false, true>(L, status, st);
            return pad ? run<128, 32, false, true, true>(L, status, st) : run<128, 32, false, true>(L, status, st);
        }
        if (L.block == 64) return pad ? run<64, 64, false, true, true>(L, status, st) : run<64, 64, false, true>(L, status, st);
        return pad ? run<64, 32, false, true, true>(L, status, st) : run<64, 32, false, true>(L, status, st);
    }
    // 32- and 64-token blocks in permuted order (windows always use 128-token tiles)
    if (L.D == 128) return L.block == 64 ? run<128, 64, false>(L, status, st) : run<128, 32, false>(L, status, st);
    return L.block == 64 ? run<64, 64, false>(L, status, st) : run<64, 32, false>(L, status, st);
}

}  // namespace vsa
