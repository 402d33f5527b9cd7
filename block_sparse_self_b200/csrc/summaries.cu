// summaries.cu -- per-block element-wise max / min of permuted tokens.
//
// "Adaptive tiling (SPADE)", The idea, step 3: each block of `block`
// consecutive tokens (one tile after the permutation) is summarised by its
// per-channel maximum and minimum.  Results are exact selections of inputs.
//
// One CTA per (bh, block).  Lanes own 16-byte column chunks; row groups walk
// the block's rows with 128-bit loads, then reduce through shared memory.
//
// Tiled variant: x stays in T-major token order and the block's rows are read
// where the head's chosen tiling puts them (position p of the tile-contiguous
// order is token tile_token(p)), which gives the same result as permuting
// first without writing the permuted copy.  On a zero-padded grid ("Adaptive
// tiling (SPADE)", Deviations and notes) the positions cover the padded grid
// and a padding position counts as a zero row.
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

struct TiledArgs {
    TileSet tiles;
    TileDivs divs[kMaxTiles];  // per candidate tiling, over the (padded) grid
    RealGrid real;             // PAD: the real grid
    const int32_t *choice;
    int *status;
};

template <typename T, int CPR, bool TILED, bool PAD>
__global__ void __launch_bounds__(kThreads) summaries_kernel(const uint8_t *__restrict__ x, int S, int block, int nb,
                                                             uint8_t *__restrict__ xmax, uint8_t *__restrict__ xmin,
                                                             const TiledArgs ta) {
    constexpr int RG = kThreads / CPR;  // row groups
    __shared__ uint4 smax[RG][CPR];
    __shared__ uint4 smin[RG][CPR];
    __shared__ int rowtok[TILED ? 256 : 1];  // tiled mode: the token of each row of the block (-1: padding)
    const int blk = blockIdx.x, bh = blockIdx.y;
    const int chunk = threadIdx.x % CPR, rg = threadIdx.x / CPR;
    const size_t head = static_cast<size_t>(bh) * S;
    int c = 0;
    uint32_t origin = 0, rr0 = 0;  // tiled mode, block within one tile: the tile's first token, block offset
    uint32_t ot = 0, oh = 0, ow = 0;  // PAD: the tile's first coordinates
    bool one_tile = false;
    if constexpr (TILED) {
        c = ta.choice ? __ldg(ta.choice + bh) : 0;
        if (c < 0 || c >= ta.tiles.n) {  // the head's summaries are left unwritten (uniform over the CTA)
            if (threadIdx.x == 0) report(ta.status, DEV_RUNTIME);
            return;
        }
        const TileDivs &d = ta.divs[c];
        const uint32_t p0 = static_cast<uint32_t>(blk * block);
        one_tile = static_cast<uint32_t>(block) <= d.vol.d;  // then block divides the volume
        if (one_tile) {
            const uint32_t tile = fdiv(p0, d.vol);
            rr0 = p0 - tile * d.vol.d;
            if constexpr (PAD) tile_coords_fast(tile * d.vol.d, d, ot, oh, ow);
            else origin = tile_token_fast(tile * d.vol.d, d);
        }
    }
    // token of the block's r-th row (PAD: -1 for padding)
    auto row_token = [&](int r) -> int {
        uint32_t tok = static_cast<uint32_t>(blk * block + r);
        if constexpr (TILED) {
            const TileDivs &d = ta.divs[c];
            if constexpr (PAD) {
                uint32_t t, h, w;
                if (one_tile) {
                    const uint32_t rr = rr0 + static_cast<uint32_t>(r);
                    const uint32_t dt = fdiv(rr, d.thw), r2 = rr - dt * d.thw.d;
                    const uint32_t dh = fdiv(r2, d.tw), dw = r2 - dh * d.tw.d;
                    t = ot + dt;
                    h = oh + dh;
                    w = ow + dw;
                } else {
                    tile_coords_fast(tok, d, t, h, w);
                }
                return real_token(t, h, w, ta.real);
            } else if (one_tile) {
                const uint32_t rr = rr0 + static_cast<uint32_t>(r);
                const uint32_t dt = fdiv(rr, d.thw), r2 = rr - dt * d.thw.d;
                const uint32_t dh = fdiv(r2, d.tw), dw = r2 - dh * d.tw.d;
                tok = origin + (dt * d.H + dh) * d.W + dw;
            } else {
                tok = tile_token_fast(tok, d);
            }
        }
        return static_cast<int>(tok);
    };
    // Every row is read by CPR threads (one 16-byte chunk each), so its token is
    // worked out once per CTA, not once per thread.
    if constexpr (TILED) {
        for (int r = threadIdx.x; r < block; r += kThreads) rowtok[r] = row_token(r);
        __syncthreads();
    }
    auto load_row = [&](int r) -> Vec<T> {
        const int tok = TILED ? rowtok[r] : blk * block + r;
        if constexpr (PAD) {
            if (tok < 0) {
                Vec<T> z;
                *reinterpret_cast<uint4 *>(&z) = make_uint4(0u, 0u, 0u, 0u);  // +0.0 in every element
                return z;
            }
        }
        return Vec<T>::load(x + (head + static_cast<size_t>(tok)) * CPR * 16 + chunk * 16);
    };
    Vec<T> mx, mn;
    if (rg < block) {
        mx = load_row(rg);
        mn = mx;
        #pragma unroll 4
        for (int r = rg + RG; r < block; r += RG) {
            const Vec<T> v = load_row(r);
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

// S: tokens per head of x; Sp: positions per head (the padded grid's tokens, or S)
template <bool TILED, bool PAD>
cudaError_t run_summaries(const void *x, int esize, int BH, int S, int Sp, int D, int block, void *xmax, void *xmin,
                          const TiledArgs &ta, cudaStream_t st) {
    const int nb = Sp / block;
    const int cpr = D * esize / 16;
    dim3 grid(nb, BH);
    const uint8_t *xi = static_cast<const uint8_t *>(x);
    uint8_t *mx = static_cast<uint8_t *>(xmax), *mn = static_cast<uint8_t *>(xmin);
    if (esize == 2) {
        if (cpr == 8) summaries_kernel<__nv_bfloat16, 8, TILED, PAD><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn, ta);
        else summaries_kernel<__nv_bfloat16, 16, TILED, PAD><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn, ta);
    } else {
        if (cpr == 16) summaries_kernel<float, 16, TILED, PAD><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn, ta);
        else summaries_kernel<float, 32, TILED, PAD><<<grid, kThreads, 0, st>>>(xi, S, block, nb, mx, mn, ta);
    }
    return cudaGetLastError();
}


// ---------------------------------------------------------------------------
// Tiled bf16 summaries of 128-token blocks through TMA (the adaptive path)
// ---------------------------------------------------------------------------
// When every candidate's 128-token block is a box of whole (h, w) planes (as
// for the tiled attention), a block is one 5-D TMA box and arrives in shared
// memory as 128 rows of 128-byte slabs in tile-contiguous order; a box that
// reaches past the real grid reads zeros there, which are the padding rows.
// Persistent CTAs, two per SM, stream blocks through kSumStages stages: one
// producer thread issues the boxes, eight consumer warps take each column's
// max and min out of shared memory with warp shuffles.  HBM sees only long
// bulk reads, and no thread spends instructions on addresses.
constexpr int kSumStages = 3;
constexpr int kSumWarps = 8;  // consumer warps

struct SumBoxGeom {
    FastDiv m, nthw, ntw;  // m = volume / 128, tiles per frame, tiles per tile row (padded grid)
    int bt;                // frames of one 128-token box
};
struct SumTmaArgs {
    int nb, items;  // blocks per head, B * heads * nb
    FastDiv nbdiv;
    TileSet tiles;
    SumBoxGeom geom[kMaxTiles];
    const int32_t *choice;
    int *status;
    uint8_t *xmax, *xmin;
};
struct SumMaps {
    CUtensorMap x[kMaxTiles];
};

template <int D>
__global__ void __launch_bounds__((kSumWarps + 1) * 32) summaries_tma_kernel(const __grid_constant__ SumMaps maps,
                                                                           const SumTmaArgs a) {
    constexpr int KSLABS = D / 64, SLAB = 128 * 128, STAGE = SLAB * KSLABS;
    constexpr int CPR = D / 8;              // 16-byte chunks per row
    constexpr int CPW = CPR / kSumWarps;    // chunks per consumer warp
    constexpr int LPC = 32 / CPW;           // lanes per chunk
    constexpr int RPL = 128 / LPC;          // rows per lane
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stage = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(stage + kSumStages * STAGE);
    uint64_t *empty = full + kSumStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kSumStages);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSumStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSumWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    auto tiling_of = [&](int bh) -> int {  // -1: out of range (the head is left unwritten)
        const int c = a.choice ? __ldg(a.choice + bh) : 0;
        return (c < 0 || c >= a.tiles.n) ? -1 : c;
    };

    if (warp == kSumWarps) {
        // ---- producer: one box per block ----
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < a.items; item += gridDim.x, ++it) {
                const int s = it % kSumStages;
                if (it >= kSumStages && !mbar_wait(&empty[s], ((it / kSumStages) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(item), a.nbdiv));
                const uint32_t blk = static_cast<uint32_t>(item - bh * a.nb);
                const int c = tiling_of(bh);
                if (c < 0) {
                    mbar_arrive(&full[s]);
                    continue;
                }
                const SumBoxGeom &g = a.geom[c];
                const uint32_t tile = fdiv(blk, g.m), part = blk - tile * g.m.d;
                const uint32_t ct = fdiv(tile, g.nthw), rem = tile - ct * g.nthw.d;
                const uint32_t ch = fdiv(rem, g.ntw), cw = rem - ch * g.ntw.d;
                const int bw = static_cast<int>(cw) * a.tiles.w[c], bhh = static_cast<int>(ch) * a.tiles.h[c];
                const int bt = static_cast<int>(ct * g.m.d + part) * g.bt;
                mbar_arrive_expect_tx(&full[s], STAGE);
                for (int sl = 0; sl < KSLABS; ++sl)
                    tma_load_5d(stage + s * STAGE + sl * SLAB, &maps.x[c], &full[s], sl * 64, bw, bhh, bt, bh);
            }
            if (!ok && !*abort_flag) {
                report(a.status, DEV_TIMEOUT);
                *abort_flag = 1;
            }
            // stay until every box issued has landed (the CTA's shared memory must outlive them)
            const int first = it > kSumStages ? it - kSumStages : 0;
            for (int q = first; q < it; ++q) mbar_wait(&full[q % kSumStages], (q / kSumStages) & 1, nullptr);
        }
        return;
    }

    // ---- consumers: warp w owns chunks w*CPW .. w*CPW+CPW-1 of every row ----
    const int q = warp * CPW + lane / LPC;  // this lane's chunk
    const int r0 = lane % LPC;              // first row; then every LPC-th
    const int sl = q / 8, c8 = q % 8;
    int it = 0;
    for (int item = blockIdx.x; item < a.items; item += gridDim.x, ++it) {
        const int s = it % kSumStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / kSumStages) & 1, abort_flag))) {
            if (lane == 0 && !*abort_flag) {
                report(a.status, DEV_TIMEOUT);
                *abort_flag = 1;
            }
            break;
        }
        const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(item), a.nbdiv));
        const bool valid = tiling_of(bh) >= 0;
        __nv_bfloat162 mx[4], mn[4];
        if (valid) {
            const uint8_t *src = stage + s * STAGE + sl * SLAB;
            #pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int r = r0 + LPC * i;  // 128-byte swizzle: chunk c8 of row r sits at c8 ^ (r % 8)
                const uint4 v = *reinterpret_cast<const uint4 *>(src + r * 128 + ((c8 ^ (r & 7)) << 4));
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    mx[e] = i == 0 ? h[e] : __hmax2(mx[e], h[e]);
                    mn[e] = i == 0 ? h[e] : __hmin2(mn[e], h[e]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp's reads of the stage are done
        if (valid) {
            #pragma unroll
            for (int off = LPC / 2; off > 0; off >>= 1) {
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t ux = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t *>(&mx[e]), off);
                    const uint32_t un = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t *>(&mn[e]), off);
                    mx[e] = __hmax2(mx[e], *reinterpret_cast<const __nv_bfloat162 *>(&ux));
                    mn[e] = __hmin2(mn[e], *reinterpret_cast<const __nv_bfloat162 *>(&un));
                }
            }
            if (r0 == 0) {
                const size_t o = (static_cast<size_t>(item) * CPR + q) * 16;
                *reinterpret_cast<uint4 *>(a.xmax + o) = *reinterpret_cast<const uint4 *>(mx);
                *reinterpret_cast<uint4 *>(a.xmin + o) = *reinterpret_cast<const uint4 *>(mn);
            }
        } else if (lane == 0 && warp == 0) {
            report(a.status, DEV_RUNTIME);
        }
    }
}

template <int D>
cudaError_t run_summaries_tma(const void *x, int BH, int T, int H, int W, int Hp, int Wp, int nb,
                              const TileSet &tiles, const int32_t *choice, void *xmax, void *xmin, int *status,
                              cudaStream_t st) {
    SumMaps maps = {};
    SumTmaArgs a;
    a.nb = nb;
    a.items = BH * nb;
    a.nbdiv = make_fastdiv(static_cast<uint32_t>(nb));
    a.tiles = tiles;
    for (int c = 0; c < kMaxTiles; ++c) {
        SumBoxGeom &g = a.geom[c];
        if (c < tiles.n) {
            const int m = tiles.t[c] * tiles.h[c] * tiles.w[c] / 128;
            g.m = make_fastdiv(static_cast<uint32_t>(m));
            g.nthw = make_fastdiv(static_cast<uint32_t>((Hp / tiles.h[c]) * (Wp / tiles.w[c])));
            g.ntw = make_fastdiv(static_cast<uint32_t>(Wp / tiles.w[c]));
            g.bt = tiles.t[c] / m;
            if (!make_box_map(&maps.x[c], x, D, T, H, W, BH, g.bt, tiles.h[c], tiles.w[c]))
                return cudaErrorInvalidValue;
        } else {
            g.m = g.nthw = g.ntw = make_fastdiv(1);
            g.bt = 1;
        }
    }
    a.choice = choice;
    a.status = status;
    a.xmax = static_cast<uint8_t *>(xmax);
    a.xmin = static_cast<uint8_t *>(xmin);
    constexpr int kStage = 128 * 128 * (D / 64);
    const int smem = 1024 + kSumStages * kStage + 2 * kSumStages * 8 + 16;
    auto kern = summaries_tma_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = a.items < 2 * sms ? a.items : 2 * sms;
    kern<<<grid, (kSumWarps + 1) * 32, smem, st>>>(maps, a);
    return cudaGetLastError();
}

// Whether the TMA path covers these tilings: bf16, 128-token blocks, every
// candidate of one volume V (a multiple of 128) with tile.t divisible by V/128,
// and every box inside the real grid.
bool summaries_tma_ok(int esize, int D, int block, int T, int H, int W, const TileSet &tiles) {
    if (esize != 2 || block != 128 || (D != 64 && D != 128)) return false;
    const int vol = tiles.t[0] * tiles.h[0] * tiles.w[0];
    if (vol % 128 != 0) return false;
    for (int c = 0; c < tiles.n; ++c) {
        const int m = vol / 128;
        if (tiles.t[c] * tiles.h[c] * tiles.w[c] != vol || tiles.t[c] % m != 0) return false;
        if (tiles.t[c] / m > T || tiles.h[c] > H || tiles.w[c] > W) return false;
    }
    return true;
}
}  // namespace

cudaError_t launch_summaries(const void *x, int esize, int BH, int S, int D, int block, void *xmax, void *xmin,
                             cudaStream_t st) {
    TiledArgs ta{};
    return run_summaries<false, false>(x, esize, BH, S, S, D, block, xmax, xmin, ta, st);
}

cudaError_t launch_summaries_tiled(const void *x, int esize, int BH, int D, int T, int H, int W, int Tp, int Hp,
                                   int Wp, const TileSet &tiles, const int32_t *choice, void *xmax, void *xmin,
                                   int *status, cudaStream_t st, int block) {
    TiledArgs ta;
    ta.tiles = tiles;
    for (int c = 0; c < kMaxTiles; ++c)
        ta.divs[c] = c < tiles.n ? make_tile_divs(Hp, Wp, tiles.t[c], tiles.h[c], tiles.w[c]) : make_tile_divs(1, 1, 1, 1, 1);
    ta.real = RealGrid{T, H, W};
    ta.choice = choice;
    ta.status = status;
    const int S = T * H * W, Sp = Tp * Hp * Wp;
    if (summaries_tma_ok(esize, D, block, T, H, W, tiles) && (reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
        return D == 128 ? run_summaries_tma<128>(x, BH, T, H, W, Hp, Wp, Sp / block, tiles, choice, xmax, xmin, status, st)
                        : run_summaries_tma<64>(x, BH, T, H, W, Hp, Wp, Sp / block, tiles, choice, xmax, xmin, status, st);
    }
    if (Sp != S) return run_summaries<true, true>(x, esize, BH, S, Sp, D, block, xmax, xmin, ta, st);
    return run_summaries<true, false>(x, esize, BH, S, S, D, block, xmax, xmin, ta, st);
}

}  // namespace vsa
