// attention_pp.cu -- block-sparse and sliding-window attention on tcgen05 tensor
// cores, two query tiles per CTA ("ping-pong") for 128-token blocks.
//
// Semantics are those of attention.cu ("Adaptive tiling (SPADE)", Recipe and
// recipe note; "fastvideo/mlx_runtime/windowed_attention.py", Window policy
// and _key_ranges_for_block).  This variant keeps the tensor pipe busy while a
// softmax runs: each CTA owns two 128-row query tiles A and B, and while one
// tile's softmax warpgroup turns S into P, the MMA warp runs the other tile's
// QK^T and PV.
//
// Warps: 0-3 softmax/epilogue of tile A, 4-7 of tile B (thread = query row =
// TMEM lane), 8 TMA producer, 9 MMA issuer and TMEM owner.  Three warps share
// some SM sub-partitions, so a thread has at most 168 registers: the softmax
// keeps one block's 128 scores in registers and rescales O in 8-column steps.
// Tensor memory (512 columns): S_A, S_B (128 fp32 columns each), O_A, O_B
// (D columns each).  P (bf16, 64 columns) is written over the first half of
// its tile's S and is the TMEM operand of the PV MMA, so shared memory only
// holds Q_A, Q_B, a ring of K tiles and a ring of V tiles.  The producer loads
// and the MMA warp issues in one fixed program order:
//   QK_A(0) QK_B(0) | PV_A(j) QK_A(j+1) PV_B(j) QK_B(j+1) | j = 0, 1, ...
// An MMA only orders behind an earlier one with the same accumulator, so
// QK_t(j+1), which overwrites the P_t(j) that PV_t(j) reads, first waits for
// PV_t(j) to complete.
//
// Tiled mode on a zero-padded grid ("Adaptive tiling (SPADE)", Deviations
// and notes): block lists count blocks of the padded grid, the TMA boxes read
// the real tensors and fill the part past their edge with zeros, keys there
// are masked in the blocks that cross the edge, rows there are not written,
// and query tiles wholly past the edge are skipped.
//
// Softmax: after a row's first visible block the exponentials use the running
// row max without taking the block's max at all; only if the block's P would
// sum above 2^24 (the max grew, rare) is the running max raised, O and l
// rescaled and the block redone from S, which is still intact in TMEM.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

struct PPArgs {
    int S, nq;        // positions per head (tiled mode: of the padded grid), query tiles
    int items;        // one-block kernel: query tiles of all heads, nq * BH
    FastDiv nqdiv;    // one-block kernel: item -> (bh, query tile)
    int S_out;        // rows per head of o (tiled mode: real tokens)
    const int32_t *idx, *cnt;
    int cap, list_per_head, group, nb;
    int gstride;  // > 1: keys share a row's group iff their positions agree with it mod gstride (a power of two)
    int half, sink, dense;
    float scale_log2;
    void *out;
    int out_f32;
    float2 *stats;  // optional per-row (m, l), see AttnLaunch
    int *status;
    // tiled mode: T-major tensors, per-head tiling (all of volume 128 * m)
    int H, W;         // the padded grid's frame (equal to the real one when nothing is padded)
    RealGrid real;
    TileSet tiles;
    const int32_t *choice;
    struct BoxGeom {
        FastDiv m, nthw, ntw;  // m = volume / 128, tiles per frame, tiles per tile row
        FastDiv bhw, bw;       // box frame (th * tw) and row (tw): key column -> (dt, dh, dw)
        int bt;                // frames of one 128-token box: tile.t / m
    } geom[kMaxTiles];
};

// Tensor maps: slot 0 only, or one per candidate tiling in tiled mode.
struct MapSet {
    CUtensorMap q[kMaxTiles], k[kMaxTiles], v[kMaxTiles];
};
static_assert(sizeof(MapSet) + sizeof(PPArgs) <= 4096, "kernel parameters");

// In tiled mode, block b of a head whose tiling is (tt, th, tw) is the
// 128-token box (tt/m, th, tw) at part b % m of tile b / m (m = volume/128):
// its TMA coordinates in the (D, W, H, T, BH) tensor.
struct BoxCoord {
    int w, h, t;
};
__device__ __forceinline__ BoxCoord box_of(uint32_t b, const PPArgs::BoxGeom &g, int th, int tw) {
    const uint32_t tile = fdiv(b, g.m), part = b - tile * g.m.d;
    const uint32_t ct = fdiv(tile, g.nthw), rem = tile - ct * g.nthw.d;
    const uint32_t ch = fdiv(rem, g.ntw), cw = rem - ch * g.ntw.d;
    return BoxCoord{static_cast<int>(cw) * tw, static_cast<int>(ch) * th,
                    static_cast<int>(ct * g.m.d + part) * g.bt};
}

template <int D>
struct PPCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;         // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = SLAB * KSLABS;  // Q, K or V tile of 128 rows
    static constexpr int NK = D == 128 ? 3 : 4;    // K ring depth
    static constexpr int NV = D == 128 ? 2 : 4;    // V ring depth
    static constexpr int O_COL = 256;              // O_A at 256, O_B at 256 + D
    static constexpr int N_BARS = 1 + 2 * NK + 2 * NV + 2 + 2 + 2 + 1;
    static constexpr int SMEM = 1024 + (2 + NK + NV) * TILE_BYTES + N_BARS * 8 + 64;
    static_assert(SMEM <= 232448, "shared memory");
};

constexpr int kThreads = 320;
// The running row max is only raised when a block's P would sum above 2^24:
// every P then stays in (0, 2^24] (bf16 has the range) and O, l stay far below
// fp32 overflow for any key count a list can name, while redos are rare.
constexpr float kMaxRowSum = 16777216.0f;


struct TileSched {
    int qt;       // query tile index, -1 if this CTA has no such tile
    int n;        // key blocks
    int r0_len, r1_start;
    const int32_t *list;
};

template <bool WINDOW>
__device__ __forceinline__ TileSched make_sched(const PPArgs &a, int qt, int bh) {
    TileSched t{};
    t.qt = qt;
    if (qt < 0 || qt >= a.nq) {
        t.qt = -1;
        return t;
    }
    const int S = a.S, BN = 128;
    if constexpr (WINDOW) {
        const int q0 = qt * BN;
        if (a.dense) {
            t.r0_len = (S + BN - 1) / BN;
            t.n = t.r0_len;
        } else {
            const int qe = min(q0 + BN, S);
            const int lo = max(0, q0 - a.half), hi = min(S, qe + a.half);
            const int lb0 = lo / BN, lb1 = (hi + BN - 1) / BN;
            const int sb = (a.sink + BN - 1) / BN;
            if (sb == 0) {
                t.r0_len = 0; t.r1_start = lb0; t.n = lb1 - lb0;
            } else if (lb0 <= sb) {
                t.r0_len = max(lb1, sb); t.n = t.r0_len;
            } else {
                t.r0_len = sb; t.r1_start = lb0; t.n = sb + (lb1 - lb0);
            }
        }
    } else {
        const size_t lrow = (a.list_per_head ? static_cast<size_t>(bh) * a.nb : 0) + qt;
        t.list = a.idx + lrow * a.cap;
        t.n = __ldg(a.cnt + lrow);
    }
    return t;
}

template <bool WINDOW>
__device__ __forceinline__ int kblock_of(const TileSched &t, int j) {
    if constexpr (WINDOW) return j < t.r0_len ? j : t.r1_start + (j - t.r0_len);
    else return __ldg(t.list + j);
}

// PAD (tiled mode only): the grid is zero-padded, so padding rows and keys need
// handling; a separate instantiation keeps that code out of the common case.
template <int D, bool WINDOW, bool TILED, bool PAD>
__global__ void __launch_bounds__(kThreads, 1)
attn_pp_kernel(const __grid_constant__ MapSet maps, const PPArgs a) {
    using C = PPCfg<D>;
    constexpr int BN = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                                  // [2][TILE]
    uint8_t *sK = sQ + 2 * C::TILE_BYTES;                // [NK][TILE]
    uint8_t *sV = sK + C::NK * C::TILE_BYTES;            // [NV][TILE]
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sV + C::NV * C::TILE_BYTES);
    uint64_t *k_full = q_full + 1;
    uint64_t *k_empty = k_full + C::NK;
    uint64_t *v_full = k_empty + C::NK;
    uint64_t *v_empty = v_full + C::NV;
    uint64_t *s_full = v_empty + C::NV;   // [2]
    uint64_t *p_full = s_full + 2;        // [2]
    uint64_t *pv_done = p_full + 2;       // [2]
    uint64_t *mma_done = pv_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *list_ok = reinterpret_cast<int *>(tmem_slot + 2);  // [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int S = a.S;
    TileSched ts[2] = {make_sched<WINDOW>(a, 2 * blockIdx.x, bh), make_sched<WINDOW>(a, 2 * blockIdx.x + 1, bh)};

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);
            mbar_init(&pv_done[t], 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if constexpr (!WINDOW) {
        if (warp < 2) {  // warp t validates tile t's list
            const TileSched &t = ts[warp];
            if (t.qt >= 0) {
                bool ok = t.n >= 1 && t.n <= a.cap;
                if (ok) {
                    for (int j = lane; j < t.n; j += 32) {
                        const int v = __ldg(t.list + j);
                        ok = ok && v >= 0 && v < a.nb && (j == 0 || __ldg(t.list + j - 1) < v);
                    }
                }
                ok = __all_sync(0xffffffffu, ok);
                // written only here (read after the barrier below): an initial
                // value set by another thread could land after this store
                if (lane == 0) list_ok[warp] = ok ? 1 : 0;
            }
        }
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool bad[2] = {false, false};
    for (int t = 0; t < 2; ++t) {
        if (ts[t].qt < 0) ts[t].n = 0;
        if constexpr (!WINDOW) {
            if (ts[t].qt >= 0 && !list_ok[t]) {
                bad[t] = true;
                ts[t].n = 0;
                if (threadIdx.x == 0) report(a.status, DEV_RUNTIME);
            }
        }
    }
    int tc = 0;  // tiled mode: this head's tiling
    if constexpr (TILED) {
        if (a.choice) tc = __ldg(a.choice + bh);
        if (tc < 0 || tc >= a.tiles.n) {  // the head is left unwritten
            if (threadIdx.x == 0) report(a.status, DEV_RUNTIME);
            ts[0].n = ts[1].n = 0;
            ts[0].qt = ts[1].qt = -1;
            tc = 0;
        }
    }
    const int tt = a.tiles.t[tc], th = a.tiles.h[tc], tw = a.tiles.w[tc];
    if constexpr (PAD) {
        {  // a query box wholly in the padding has no row to write
            for (int t = 0; t < 2; ++t) {
                if (ts[t].qt < 0) continue;
                const BoxCoord c = box_of(static_cast<uint32_t>(ts[t].qt), a.geom[tc], th, tw);
                if (c.t >= a.real.T || c.h >= a.real.H || c.w >= a.real.W) {
                    ts[t].qt = -1;
                    ts[t].n = 0;
                }
            }
        }
    }
    const CUtensorMap *tmQ = &maps.q[tc], *tmK = &maps.k[tc], *tmV = &maps.v[tc];
    // one 128-row tile of Q, K or V: block b of this head
    auto load_tile = [&](uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int b) {
        if constexpr (TILED) {
            const BoxCoord c = box_of(static_cast<uint32_t>(b), a.geom[tc], th, tw);
            for (int s = 0; s < C::KSLABS; ++s) tma_load_5d(dst + s * C::SLAB, map, bar, s * 64, c.w, c.h, c.t, bh);
        } else {
            for (int s = 0; s < C::KSLABS; ++s) tma_load_3d(dst + s * C::SLAB, map, bar, s * 64, b * BN, bh);
        }
    };
    const int nA = ts[0].n, nB = ts[1].n;
    const int nmax = max(nA, nB);


    if (warp == 8) {
        // ================= TMA producer =================
        if (lane == 0 && nmax > 0) {
            tma_prefetch_desc(tmQ);
            tma_prefetch_desc(tmK);
            tma_prefetch_desc(tmV);
            const int nq_loaded = (nA > 0) + (nB > 0);
            mbar_arrive_expect_tx(q_full, nq_loaded * C::TILE_BYTES);
            for (int t = 0; t < 2; ++t)
                if (ts[t].n > 0) load_tile(sQ + t * C::TILE_BYTES, tmQ, q_full, ts[t].qt);
            uint32_t kc = 0, vc = 0;
            bool ok = true;
            auto load = [&](bool is_k, int t, int j) -> bool {
                uint32_t &c = is_k ? kc : vc;
                const int depth = is_k ? C::NK : C::NV;
                const int slot = c % depth;
                uint64_t *full = is_k ? &k_full[slot] : &v_full[slot];
                uint64_t *empty = is_k ? &k_empty[slot] : &v_empty[slot];
                if (c >= static_cast<uint32_t>(depth) && !mbar_wait(empty, ((c / depth) - 1) & 1, abort_flag))
                    return false;
                uint8_t *dst = (is_k ? sK : sV) + slot * C::TILE_BYTES;
                const int kb = kblock_of<WINDOW>(ts[t], j);
                mbar_arrive_expect_tx(full, C::TILE_BYTES);
                load_tile(dst, is_k ? tmK : tmV, full, kb);
                ++c;
                return true;
            };
            if (nA > 0) ok = ok && load(true, 0, 0);
            if (nB > 0) ok = ok && load(true, 1, 0);
            for (int j = 0; ok && j < nmax; ++j)
                for (int t = 0; ok && t < 2; ++t)
                    if (j < ts[t].n) {
                        ok = load(false, t, j);
                        if (ok && j + 1 < ts[t].n) ok = load(true, t, j + 1);
                    }
            if (!ok) {
                if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the loads already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                for (uint32_t c = kc > static_cast<uint32_t>(C::NK) ? kc - C::NK : 0; c < kc; ++c)
                    mbar_wait(&k_full[c % C::NK], (c / C::NK) & 1, nullptr);
                for (uint32_t c = vc > static_cast<uint32_t>(C::NV) ? vc - C::NV : 0; c < vc; ++c)
                    mbar_wait(&v_full[c % C::NV], (c / C::NV) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            // Descriptor bases, built once.  The start-address field holds
            // addr >> 4 in 14 bits and every shared address here is < 256 KB,
            // so advancing a descriptor by a byte offset is a plain add of
            // offset >> 4 with no carry out of the field.
            const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dV = sdesc_sw128(smem_u32(sV), C::SLAB, 1024);
            constexpr uint64_t kTile16 = C::TILE_BYTES >> 4;
            uint32_t kc = 0, vc = 0;
            bool ok = true;
            auto qk = [&](int t, int j) -> bool {
                const int slot = kc % C::NK;
                if (!mbar_wait(&k_full[slot], (kc / C::NK) & 1, abort_flag)) return false;
                if (j > 0 && !mbar_wait(&pv_done[t], (j - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t q0 = dQ + t * kTile16, k0 = dK + slot * kTile16;
                const uint32_t d = tmem + t * 128;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(d, q0 + off, k0 + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[t]);
                umma_commit(&k_empty[slot]);
                ++kc;
                return true;
            };
            auto pv = [&](int t, int j) -> bool {
                const int slot = vc % C::NV;
                if (!mbar_wait(&p_full[t], j & 1, abort_flag)) return false;
                if (!mbar_wait(&v_full[slot], (vc / C::NV) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t v0 = dV + slot * kTile16;
                const uint32_t d = tmem + C::O_COL + t * D, pa = tmem + t * 128;
                const uint32_t acc0 = j > 0 ? 1u : 0u;
                #pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_bf16_ts(d, pa + kk * 8, v0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                                 kk > 0 ? 1u : acc0);
                umma_commit(&pv_done[t]);
                umma_commit(&v_empty[slot]);
                ++vc;
                return true;
            };
            if (nmax > 0) {
                ok = mbar_wait(q_full, 0, abort_flag);
                if (ok && nA > 0) ok = qk(0, 0);
                if (ok && nB > 0) ok = qk(1, 0);
                for (int j = 0; ok && j < nmax; ++j)
                    for (int t = 0; ok && t < 2; ++t)
                        if (j < ts[t].n) {
                            ok = pv(t, j);
                            if (ok && j + 1 < ts[t].n) ok = qk(t, j + 1);
                        }
                if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
            }
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ================= softmax + epilogue (warps 0-7) =================
        const int t = warp >> 2;                  // tile
        const int wq = warp & 3;                  // TMEM lane quadrant
        const int row = wq * 32 + lane;           // row of the tile
        const TileSched &sc = ts[t];
        const int n = sc.n;
        const int q0 = (sc.qt < 0 ? 0 : sc.qt) * BN;
        const int rg = q0 + row;
        bool row_valid = sc.qt >= 0 && rg < S;
        // output row: the permuted position itself, or its T-major token in tiled mode
        uint32_t orow_in_head = rg;
        if constexpr (PAD) {
            int pt, ph, pw;
            tile_coords(rg, a.H, a.W, tt, th, tw, pt, ph, pw);
            const int tok = real_token(pt, ph, pw, a.real);
            row_valid = row_valid && tok >= 0;
            orow_in_head = tok < 0 ? 0u : static_cast<uint32_t>(tok);
        } else if constexpr (TILED) {
            orow_in_head = tile_token(rg, a.H, a.W, tt, th, tw);
        }
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t s_col = t * 128, o_col = C::O_COL + t * D;
        const float sl2 = a.scale_log2;
        float m_ref = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            uint32_t x[BN];
            #pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tmem_ld32(t_lane + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * c]));
            tmem_ld_wait();
            // padded grid: which of the key block's 128 columns are real tokens
            // (column u * 32 + lane in bit lane of kv[u]); all ones off the edge
            uint32_t kv[4] = {~0u, ~0u, ~0u, ~0u};
            bool key_edge = false;
            if constexpr (PAD) {
                {
                    const PPArgs::BoxGeom &g = a.geom[tc];
                    const BoxCoord c = box_of(static_cast<uint32_t>(kblock_of<WINDOW>(sc, j)), g, th, tw);
                    key_edge = c.t + g.bt > a.real.T || c.h + th > a.real.H || c.w + tw > a.real.W;
                    if (key_edge) {
                        #pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t col = static_cast<uint32_t>(u * 32 + lane);
                            const uint32_t dt = fdiv(col, g.bhw), r2 = col - dt * g.bhw.d;
                            const uint32_t dh = fdiv(r2, g.bw), dw = r2 - dh * g.bw.d;
                            kv[u] = __ballot_sync(0xffffffffu, c.t + static_cast<int>(dt) < a.real.T &&
                                                                   c.h + static_cast<int>(dh) < a.real.H &&
                                                                   c.w + static_cast<int>(dw) < a.real.W);
                        }
                    }
                }
            }
            auto apply_mask = [&]() {
                if constexpr (WINDOW) {
                    const int ks = kblock_of<WINDOW>(sc, j) * BN;
                    const int qe = min(q0 + BN, S);
                    const bool full = (ks + BN <= S) &&
                                      (a.dense || ks + BN <= a.sink || max(qe - 1 - ks, ks + BN - 1 - q0) <= a.half);
                    if (!full) {
                        #pragma unroll
                        for (int c = 0; c < BN; ++c) {
                            const int kc2 = ks + c;
                            const int dd = rg > kc2 ? rg - kc2 : kc2 - rg;
                            if (!(kc2 < S && (a.dense || kc2 < a.sink || dd <= a.half)))
                                x[c] = __float_as_uint(-INFINITY);
                        }
                    }
                } else {
                    if (a.group > 0) {
                        const int ks = kblock_of<WINDOW>(sc, j) * BN;
                        // key ks + c is in the row's group iff it lies in [g0, g0 + group)
                        const int g0 = (rg / a.group) * a.group - ks;
                        #pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (c < g0 || c >= g0 + a.group) x[c] = __float_as_uint(-INFINITY);
                    } else if (a.gstride > 1) {
                        const int ks = kblock_of<WINDOW>(sc, j) * BN;
                        // key ks + c is in the row's group iff (ks + c - rg) is a multiple of gstride
                        const int r0 = (rg - ks) & (a.gstride - 1);
                        #pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if ((c & (a.gstride - 1)) != r0) x[c] = __float_as_uint(-INFINITY);
                    }
                    if (key_edge) {
                        #pragma unroll
                        for (int c = 0; c < BN; ++c)
                            if (!((kv[c >> 5] >> (c & 31)) & 1u)) x[c] = __float_as_uint(-INFINITY);
                    }
                }
            };
            apply_mask();
            // P = 2^(scale*log2e*S - m_use) in place (bf16 pairs), returns the row sum
            // The arguments use two-wide fp32 instructions: the exponentials are
            // bound by the exponential unit, and fewer issue slots here leave more
            // to the other tile's warp on the sub-partition.  The row sum adds the
            // bf16-rounded P that the PV MMA multiplies, so O / l is a convex
            // combination of V rows: a row held by a few keys then carries no
            // rounding error in its weights' total.  The mixed-precision adds take
            // each half of the packed pair as it is; unpacking the pair first for
            // two-wide adds measured a few percent slower.
            auto exp_pass = [&](float m_use) -> float {
                const uint64_t sl2x2 = f32x2(sl2, sl2), nmx2 = f32x2(-m_use, -m_use);
                float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
                #pragma unroll
                for (int q = 0; q < BN / 2; ++q) {
                    float a0, a1;
                    f32x2_split(fma_f32x2(f32x2(__uint_as_float(x[2 * q]), __uint_as_float(x[2 * q + 1])), sl2x2, nmx2),
                                a0, a1);
                    const uint32_t pk = pack_bf16x2(ex2_approx(a0), ex2_approx(a1));
                    if (q & 1) add_bf16x2_f32(pk, s2, s3);
                    else add_bf16x2_f32(pk, s0, s1);
                    x[q] = pk;   // P, packed in place (q <= 2q)
                }
                return (s0 + s2) + (s1 + s3);
            };
            auto raw_max = [&]() -> float {
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                #pragma unroll
                for (int c = 0; c < BN; c += 8) {
                    #pragma unroll
                    for (int u = 0; u < 4; ++u)
                        m4[u] = fmax3(m4[u], __uint_as_float(x[c + 2 * u]), __uint_as_float(x[c + 2 * u + 1]));
                }
                return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            };
            // first visible keys of this row: take the block max before the exponentials
            if (m_ref == -INFINITY) m_ref = raw_max() * sl2;  // may stay -inf
            // The running max is lazy: every P is at most the row sum, so a sum
            // above kMaxRowSum (or inf) means the row's max grew; then O and l are
            // rescaled and the block is redone from S, still intact in TMEM.
            float rs = 0.f;
            #pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                rs = exp_pass(m_ref == -INFINITY ? 0.f : m_ref);
                const bool need = !(rs <= kMaxRowSum);
                if (pass == 1 || !__any_sync(0xffffffffu, need)) break;
                #pragma unroll
                for (int c = 0; c < BN / 32; ++c)
                    tmem_ld32(t_lane + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * c]));
                tmem_ld_wait();
                apply_mask();
                const float m_new = need ? fmaxf(m_ref, raw_max() * sl2) : m_ref;
                if (j > 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[t], (j - 1) & 1, abort_flag))) {
                        ok = false;
                    } else {
                        tc_fence_after();
                        const float alpha = (m_new > m_ref && m_ref != -INFINITY) ? ex2_approx(m_ref - m_new) : 1.f;
                        #pragma unroll 1
                        for (int c = 0; c < D / 8; ++c) {
                            uint32_t o[8];
                            tmem_ld8(t_lane + o_col + 8 * c, o);
                            tmem_ld_wait();
                            #pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st8(t_lane + o_col + 8 * c, o);
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
            // P over the first 64 columns of this tile's S
            tmem_st32(t_lane + s_col, *reinterpret_cast<const uint32_t(*)[32]>(&x[0]));
            tmem_st32(t_lane + s_col + 32, *reinterpret_cast<const uint32_t(*)[32]>(&x[32]));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t]);
        }
        if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }

        // ---- epilogue: O / l -> global ----
        const size_t orow = static_cast<size_t>(bh) * a.S_out + orow_in_head;
        bool have_o = ok && n > 0;
        if (have_o && !__all_sync(0xffffffffu, mbar_wait(&pv_done[t], (n - 1) & 1, abort_flag))) {
            have_o = false;
            if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
        }
        if (have_o) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(t_lane + o_col + 32 * c, o);
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
            if (row_valid && l_sum <= 0.f) report(a.status, DEV_RUNTIME);
            if (a.stats && row_valid) a.stats[static_cast<size_t>(bh) * a.S + rg] = make_float2(m_ref, l_sum);
        } else if (row_valid && bad[t]) {
            if (a.stats) a.stats[static_cast<size_t>(bh) * a.S + rg] = make_float2(-INFINITY, 0.f);
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
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool WINDOW, bool TILED, bool PAD = false>
vsa_status run_pp(const AttnLaunch &L, int *status, cudaStream_t st) {
    using C = PPCfg<D>;
    MapSet maps = {};  // copied into the launch parameters
    bool ok = true;
    if constexpr (TILED) {
        for (int c = 0; c < L.tiles.n; ++c) {
            const int m = L.tiles.t[c] * L.tiles.h[c] * L.tiles.w[c] / 128;
            const int bt = L.tiles.t[c] / m, bhh = L.tiles.h[c], bw = L.tiles.w[c];
            // the real tensors: boxes reaching past them read zeros
            ok = ok && make_box_map(&maps.q[c], L.q, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw) &&
                 make_box_map(&maps.k[c], L.k, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw) &&
                 make_box_map(&maps.v[c], L.v, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw);
        }
    } else {
        ok = make_tile_map(&maps.q[0], L.q, D, L.S, L.BH, 128) && make_tile_map(&maps.k[0], L.k, D, L.S, L.BH, 128) &&
             make_tile_map(&maps.v[0], L.v, D, L.S, L.BH, 128);
    }
    if (!ok) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
    auto kern = attn_pp_kernel<D, WINDOW, TILED, PAD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(attention, two tiles)");
    PPArgs a;
    const int positions = TILED ? L.Tp * L.Hp * L.Wp : L.S;
    a.S = positions;
    a.S_out = L.S;
    a.nq = (positions + 127) / 128;
    a.items = a.nq * L.BH;
    a.nqdiv = make_fastdiv(static_cast<uint32_t>(a.nq));
    a.idx = L.idx;
    a.cnt = L.cnt;
    a.cap = L.cap;
    a.list_per_head = L.list_per_head;
    a.group = L.group;
    a.gstride = L.gstride;
    a.nb = L.nb;
    a.half = L.half;
    a.sink = L.sink;
    a.dense = L.dense;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.out = L.o;
    a.out_f32 = L.out_f32;
    a.stats = L.stats;
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
            const int m = tt * th * tw / 128;
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
    dim3 grid((a.nq + 1) / 2, L.BH);
    kern<<<grid, kThreads, C::SMEM, st>>>(maps, a);
    return check_cuda(cudaGetLastError(), "attention launch (two tiles)");
}

// Lists of one key block (such as the temporal-only mask's diagonal): the
// work is HBM bound (Q, K and V read and O written once per query tile), so
// what matters is keeping loads in flight.  Persistent CTAs, two per SM, take
// query tiles in turn; a CTA holds one Q, K and V tile (96 KB at D = 128) and
// one S and one O in 256 tensor-memory columns.  The next tile's Q and K load
// as soon as the current QK^T completes and its V as soon as the current PV
// completes, and the next QK^T runs while the epilogue reads O out, so a CTA
// pays its set-up once rather than per 128 rows.  Every role walks the same
// tiles and derives the same per-tile decision (list valid, tiling, padding)
// from global memory; the barriers advance once per tile with work.
template <int D>
struct OneCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;            // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = SLAB * KSLABS;  // Q, K or V tile of 128 rows
    static constexpr int O_COL = 128;                 // S at column 0, O after it
    static constexpr int N_BARS = 8;
    static constexpr int SMEM = 1024 + 3 * TILE_BYTES + N_BARS * 8 + 64;
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr int TMEM_COLS = 256;
    static_assert(O_COL + D <= TMEM_COLS, "tensor memory");
    static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};
constexpr int kOneThreads = 192;  // warps 0-3 softmax/epilogue, 4 TMA producer, 5 MMA issuer and TMEM owner

// At most 160 registers a thread, so that two CTAs (12 warps) fit in the
// SM's register file beside each other.
template <int D, bool WINDOW, bool TILED, bool PAD>
__global__ void __maxnreg__(160)
attn_one_kernel(const __grid_constant__ MapSet maps, const PPArgs a) {
    static_assert(!WINDOW, "window attention always takes the two-tile kernel");
    using C = OneCfg<D>;
    constexpr int BN = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sK = sQ + C::TILE_BYTES;
    uint8_t *sV = sK + C::TILE_BYTES;
    uint64_t *qk_full = reinterpret_cast<uint64_t *>(sV + C::TILE_BYTES);  // Q and K of a tile landed
    uint64_t *v_full = qk_full + 1;     // V landed
    uint64_t *s_full = v_full + 1;      // QK^T complete (S in tensor memory)
    uint64_t *qk_empty = s_full + 1;    // QK^T complete: sQ and sK free
    uint64_t *p_full = qk_empty + 1;    // P written (four warps)
    uint64_t *pv_done = p_full + 1;     // PV complete: sV free, O final, S/P free
    uint64_t *o_free = pv_done + 1;     // O read out by the epilogue (four warps)
    uint64_t *mma_done = o_free + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.S;
    if (threadIdx.x == 0) {
        mbar_init(qk_full, 1);
        mbar_init(v_full, 1);
        mbar_init(s_full, 1);
        mbar_init(qk_empty, 1);
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(o_free, 4);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // One query tile: its head, schedule and tiling, identical in every role.
    // n = 0: nothing to compute (bad = its list is invalid: its rows get zeros).
    struct Tile {
        int bh, tc;
        TileSched sc;
        bool bad, bad_choice;
    };
    auto tile_of = [&](int it) -> Tile {
        Tile T{};
        T.bh = static_cast<int>(fdiv(static_cast<uint32_t>(it), a.nqdiv));
        const int qt = it - T.bh * a.nq;
        T.sc = make_sched<false>(a, qt, T.bh);
        if (T.sc.qt < 0) {
            T.sc.n = 0;
        } else {
            bool ok = T.sc.n >= 1 && T.sc.n <= a.cap;
            for (int j = 0; ok && j < T.sc.n; ++j) {
                const int v = __ldg(T.sc.list + j);
                ok = v >= 0 && v < a.nb && (j == 0 || __ldg(T.sc.list + j - 1) < v);
            }
            if (!ok) {
                T.bad = true;
                T.sc.n = 0;
            }
        }
        T.tc = 0;
        if constexpr (TILED) {
            if (a.choice) T.tc = __ldg(a.choice + T.bh);
            if (T.tc < 0 || T.tc >= a.tiles.n) {  // the head is left unwritten
                T.bad_choice = true;
                T.bad = false;
                T.sc.n = 0;
                T.sc.qt = -1;
                T.tc = 0;
            }
        }
        if constexpr (PAD) {
            if (T.sc.qt >= 0) {  // a query box wholly in the padding has no row to write
                const BoxCoord c = box_of(static_cast<uint32_t>(T.sc.qt), a.geom[T.tc], a.tiles.h[T.tc], a.tiles.w[T.tc]);
                if (c.t >= a.real.T || c.h >= a.real.H || c.w >= a.real.W) {
                    T.sc.qt = -1;
                    T.sc.n = 0;
                }
            }
        }
        return T;
    };
    // one 128-row tile of Q, K or V: block b of head bh in tiling tc
    auto load_tile = [&](uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int b, int bh, int tc) {
        if constexpr (TILED) {
            const BoxCoord c = box_of(static_cast<uint32_t>(b), a.geom[tc], a.tiles.h[tc], a.tiles.w[tc]);
            for (int s = 0; s < C::KSLABS; ++s) tma_load_5d(dst + s * C::SLAB, map, bar, s * 64, c.w, c.h, c.t, bh);
        } else {
            for (int s = 0; s < C::KSLABS; ++s) tma_load_3d(dst + s * C::SLAB, map, bar, s * 64, b * BN, bh);
        }
    };

    if (warp == 4) {
        // ================= TMA producer =================
        if (lane == 0) {
            for (int c = 0; c < a.tiles.n; ++c) {
                tma_prefetch_desc(&maps.q[c]);
                tma_prefetch_desc(&maps.k[c]);
                tma_prefetch_desc(&maps.v[c]);
            }
            int n_qk = 0, n_v = 0;  // tiles whose Q and K, and whose V, were issued
            bool ok = true;
            for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x) {
                const Tile T = tile_of(it);
                if (T.sc.n == 0) continue;
                const int kb = kblock_of<false>(T.sc, 0);
                if (n_qk >= 1 && !mbar_wait(qk_empty, (n_qk - 1) & 1, abort_flag)) { ok = false; break; }
                mbar_arrive_expect_tx(qk_full, 2 * C::TILE_BYTES);
                load_tile(sQ, &maps.q[T.tc], qk_full, T.sc.qt, T.bh, T.tc);
                load_tile(sK, &maps.k[T.tc], qk_full, kb, T.bh, T.tc);
                ++n_qk;
                if (n_v >= 1 && !mbar_wait(pv_done, (n_v - 1) & 1, abort_flag)) { ok = false; break; }
                mbar_arrive_expect_tx(v_full, C::TILE_BYTES);
                load_tile(sV, &maps.v[T.tc], v_full, kb, T.bh, T.tc);
                ++n_v;
            }
            if (!ok) {
                if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the last loads issued land before the CTA exits (earlier ones
                // were consumed before these were issued)
                if (n_qk > 0) mbar_wait(qk_full, (n_qk - 1) & 1, nullptr);
                if (n_v > 0) mbar_wait(v_full, (n_v - 1) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ================= MMA issuer =================
        // per tile w: [wait PV(w-1)] QK(w) | [wait P(w), V(w), O read out of w-1] PV(w)
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
            // descriptor bases (start-address field addr >> 4; every address here
            // is below 256 KB, so byte offsets add without a carry out of the field)
            const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dV = sdesc_sw128(smem_u32(sV), C::SLAB, 1024);
            int w = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x) {
                const Tile T = tile_of(it);
                if (T.sc.n == 0) continue;
                const uint32_t ph = w & 1, prev = (w - 1) & 1;
                // QK^T overwrites the P that PV(w-1) reads
                if (!mbar_wait(qk_full, ph, abort_flag) || (w >= 1 && !mbar_wait(pv_done, prev, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(tmem, dQ + off, dK + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full);
                umma_commit(qk_empty);
                // PV overwrites the O that the epilogue of w-1 reads
                if (!mbar_wait(p_full, ph, abort_flag) || !mbar_wait(v_full, ph, abort_flag) ||
                    (w >= 1 && !mbar_wait(o_free, prev, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                #pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_bf16_ts(tmem + C::O_COL, tmem + kk * 8, dV + static_cast<uint64_t>((kk * 2048) >> 4),
                                 idesc_pv, kk > 0 ? 1u : 0u);
                umma_commit(pv_done);
                ++w;
            }
            if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ================= softmax + epilogue (warps 0-3) =================
        const int wq = warp;                      // TMEM lane quadrant
        const int row = wq * 32 + lane;           // row of the tile
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const float sl2 = a.scale_log2;
        int w = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x) {
            const Tile T = tile_of(it);
            const TileSched &sc = T.sc;
            const int bh = T.bh, tc = T.tc;
            const int tt = a.tiles.t[tc], th = a.tiles.h[tc], tw = a.tiles.w[tc];
            if ((T.bad || T.bad_choice) && threadIdx.x == 0) report(a.status, DEV_RUNTIME);
            const int q0 = (sc.qt < 0 ? 0 : sc.qt) * BN;
            const int rg = q0 + row;
            bool row_valid = sc.qt >= 0 && rg < S;
            // output row: the permuted position itself, or its T-major token in tiled mode
            uint32_t orow_in_head = rg;
            if constexpr (PAD) {
                int pt, ph, pw;
                tile_coords(rg, a.H, a.W, tt, th, tw, pt, ph, pw);
                const int tok = real_token(pt, ph, pw, a.real);
                row_valid = row_valid && tok >= 0;
                orow_in_head = tok < 0 ? 0u : static_cast<uint32_t>(tok);
            } else if constexpr (TILED) {
                orow_in_head = tile_token(rg, a.H, a.W, tt, th, tw);
            }
            const size_t orow = static_cast<size_t>(bh) * a.S_out + orow_in_head;
            if (sc.n == 0) {
                if (row_valid && T.bad) {
                    if (a.stats) a.stats[static_cast<size_t>(bh) * a.S + rg] = make_float2(-INFINITY, 0.f);
                    if (a.out_f32) {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + orow * D);
                        for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
                    } else {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + orow * D);
                        for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                continue;
            }
            const uint32_t ph = w & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(s_full, ph, abort_flag))) { ok = false; break; }
            tc_fence_after();
            uint32_t x[BN];
            #pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tmem_ld32(t_lane + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * c]));
            tmem_ld_wait();
            const int ks = kblock_of<false>(sc, 0) * BN;
            // padded grid: the key block's columns past the real grid are masked
            if constexpr (PAD) {
                const PPArgs::BoxGeom &g = a.geom[tc];
                const BoxCoord c = box_of(static_cast<uint32_t>(kblock_of<false>(sc, 0)), g, th, tw);
                if (c.t + g.bt > a.real.T || c.h + th > a.real.H || c.w + tw > a.real.W) {
                    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t col = static_cast<uint32_t>(u * 32 + lane);
                        const uint32_t dt = fdiv(col, g.bhw), r2 = col - dt * g.bhw.d;
                        const uint32_t dh = fdiv(r2, g.bw), dw = r2 - dh * g.bw.d;
                        const uint32_t kv = __ballot_sync(0xffffffffu, c.t + static_cast<int>(dt) < a.real.T &&
                                                                           c.h + static_cast<int>(dh) < a.real.H &&
                                                                           c.w + static_cast<int>(dw) < a.real.W);
                        #pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (!((kv >> e) & 1u)) x[u * 32 + e] = __float_as_uint(-INFINITY);
                    }
                }
            }
            if (a.group > 0) {
                // key ks + c is in the row's group iff it lies in [g0, g0 + group)
                const int g0 = (rg / a.group) * a.group - ks;
                #pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c < g0 || c >= g0 + a.group) x[c] = __float_as_uint(-INFINITY);
            } else if (a.gstride > 1) {
                // key ks + c is in the row's group iff (ks + c - rg) is a multiple of gstride
                const int r0 = (rg - ks) & (a.gstride - 1);
                #pragma unroll
                for (int c = 0; c < BN; ++c)
                    if ((c & (a.gstride - 1)) != r0) x[c] = __float_as_uint(-INFINITY);
            }
            // The row's only block: its max is the row max, so every P <= 1 and
            // no rescaling is ever needed.  P = 2^(scale*log2e*S - m) in place
            // (bf16 pairs, two-wide arguments), and l adds the bf16-rounded P
            // that the PV MMA multiplies, as in the two-tile kernel.
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            #pragma unroll
            for (int c = 0; c < BN; c += 8) {
                #pragma unroll
                for (int u = 0; u < 4; ++u)
                    m4[u] = fmax3(m4[u], __uint_as_float(x[c + 2 * u]), __uint_as_float(x[c + 2 * u + 1]));
            }
            const float m_ref = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;  // may be -inf
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
            const uint64_t sl2x2 = f32x2(sl2, sl2), nmx2 = f32x2(-m_use, -m_use);
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            #pragma unroll
            for (int q = 0; q < BN / 2; ++q) {
                float a0, a1;
                f32x2_split(fma_f32x2(f32x2(__uint_as_float(x[2 * q]), __uint_as_float(x[2 * q + 1])), sl2x2, nmx2),
                            a0, a1);
                const uint32_t pk = pack_bf16x2(ex2_approx(a0), ex2_approx(a1));
                if (q & 1) add_bf16x2_f32(pk, s2, s3);
                else add_bf16x2_f32(pk, s0, s1);
                x[q] = pk;   // P, packed in place (q <= 2q)
            }
            // P over the first 64 columns of S
            tmem_st32(t_lane, *reinterpret_cast<const uint32_t(*)[32]>(&x[0]));
            tmem_st32(t_lane + 32, *reinterpret_cast<const uint32_t(*)[32]>(&x[32]));
            const float l_sum = (s0 + s2) + (s1 + s3);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);

            // ---- epilogue: O / l -> global ----
            if (!__all_sync(0xffffffffu, mbar_wait(pv_done, ph, abort_flag))) { ok = false; break; }
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(t_lane + C::O_COL + 32 * c, o);
                tmem_ld_wait();
                if (c == D / 32 - 1) {  // every O column is in registers: PV of the next tile may start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(o_free);
                }
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
            if (row_valid && l_sum <= 0.f) report(a.status, DEV_RUNTIME);
            if (a.stats && row_valid) a.stats[static_cast<size_t>(bh) * a.S + rg] = make_float2(m_ref, l_sum);
            ++w;
        }
        if (!ok && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool TILED, bool PAD = false>
vsa_status run_one(const AttnLaunch &L, int *status, cudaStream_t st) {
    constexpr bool WINDOW = false;
    using C = OneCfg<D>;
    // with one S buffer, QK(1) would wait for PV(0), which is issued after it:
    // lists of more than one block belong to the two-tile kernel
    if (L.cap != 1) return fail(VSA_ERR_UNSUPPORTED, "the one-key-block kernel takes lists of one block");
    MapSet maps = {};  // copied into the launch parameters
    bool ok = true;
    if constexpr (TILED) {
        for (int c = 0; c < L.tiles.n; ++c) {
            const int m = L.tiles.t[c] * L.tiles.h[c] * L.tiles.w[c] / 128;
            const int bt = L.tiles.t[c] / m, bhh = L.tiles.h[c], bw = L.tiles.w[c];
            // the real tensors: boxes reaching past them read zeros
            ok = ok && make_box_map(&maps.q[c], L.q, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw) &&
                 make_box_map(&maps.k[c], L.k, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw) &&
                 make_box_map(&maps.v[c], L.v, D, L.T, L.Hg, L.Wg, L.BH, bt, bhh, bw);
        }
    } else {
        ok = make_tile_map(&maps.q[0], L.q, D, L.S, L.BH, 128) && make_tile_map(&maps.k[0], L.k, D, L.S, L.BH, 128) &&
             make_tile_map(&maps.v[0], L.v, D, L.S, L.BH, 128);
    }
    if (!ok) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
    auto kern = attn_one_kernel<D, WINDOW, TILED, PAD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(attention, one key block)");
    PPArgs a;
    const int positions = TILED ? L.Tp * L.Hp * L.Wp : L.S;
    a.S = positions;
    a.S_out = L.S;
    a.nq = (positions + 127) / 128;
    a.items = a.nq * L.BH;
    a.nqdiv = make_fastdiv(static_cast<uint32_t>(a.nq));
    a.idx = L.idx;
    a.cnt = L.cnt;
    a.cap = L.cap;
    a.list_per_head = L.list_per_head;
    a.group = L.group;
    a.gstride = L.gstride;
    a.nb = L.nb;
    a.half = L.half;
    a.sink = L.sink;
    a.dense = L.dense;
    a.scale_log2 = L.scale * 1.4426950408889634f;
    a.out = L.o;
    a.out_f32 = L.out_f32;
    a.stats = L.stats;
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
            const int m = tt * th * tw / 128;
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
    // persistent CTAs: as many as can be resident at once, from the kernel's
    // registers and shared memory (two per SM: 160 registers a thread and
    // ~100 KB each, with the largest shared-memory carveout)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncSetAttribute(attention, one key block, carveout)");
    int dev = 0, sms = 148, regs_sm = 65536, smem_sm = 233472, smem_res = 1024;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&smem_res, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    }
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return check_cuda(e, "cudaFuncGetAttributes(attention, one key block)");
    const int warp_regs = (fa.numRegs * 32 + 255) / 256 * 256;  // registers are allocated per warp, 256 at a time
    const int by_regs = regs_sm / (warp_regs * (kOneThreads / 32));
    const int by_smem = smem_sm / (C::SMEM + smem_res);
    int per_sm = by_regs < by_smem ? by_regs : by_smem;
    per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);
    const int grid = a.items < per_sm * sms ? a.items : per_sm * sms;
    kern<<<grid, kOneThreads, C::SMEM, st>>>(maps, a);
    return check_cuda(cudaGetLastError(), "attention launch (one key block)");
}

}  // namespace

vsa_status launch_attention_pp(const AttnLaunch &L, int *status, cudaStream_t st) {
    if (L.window) return L.D == 128 ? run_pp<128, true, false>(L, status, st) : run_pp<64, true, false>(L, status, st);
    if (L.cap == 1) {  // lists of one key block
        if (L.tiled) {
            if (L.Tp * L.Hp * L.Wp != L.S)
                return L.D == 128 ? run_one<128, true, true>(L, status, st) : run_one<64, true, true>(L, status, st);
            return L.D == 128 ? run_one<128, true>(L, status, st) : run_one<64, true>(L, status, st);
        }
        return L.D == 128 ? run_one<128, false>(L, status, st) : run_one<64, false>(L, status, st);
    }
    if (L.tiled) {
        if (L.Tp * L.Hp * L.Wp != L.S)  // a zero-padded grid
            return L.D == 128 ? run_pp<128, false, true, true>(L, status, st) : run_pp<64, false, true, true>(L, status, st);
        return L.D == 128 ? run_pp<128, false, true>(L, status, st) : run_pp<64, false, true>(L, status, st);
    }
    return L.D == 128 ? run_pp<128, false, false>(L, status, st) : run_pp<64, false, false>(L, status, st);
}

}  // namespace vsa
