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
    // byte address of chunk `chunk` of the block's r-th row (PAD: nullptr for padding)
    auto row_ptr = [&](int r) -> const uint8_t * {
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
                const int rt = real_token(t, h, w, ta.real);
                if (rt < 0) return nullptr;
                tok = static_cast<uint32_t>(rt);
            } else if (one_tile) {
                const uint32_t rr = rr0 + static_cast<uint32_t>(r);
                const uint32_t dt = fdiv(rr, d.thw), r2 = rr - dt * d.thw.d;
                const uint32_t dh = fdiv(r2, d.tw), dw = r2 - dh * d.tw.d;
                tok = origin + (dt * d.H + dh) * d.W + dw;
            } else {
                tok = tile_token_fast(tok, d);
            }
        }
        return x + (head + tok) * CPR * 16 + chunk * 16;
    };
    auto load_row = [&](int r) -> Vec<T> {
        if constexpr (PAD) {
            const uint8_t *ptr = row_ptr(r);
            if (!ptr) {
                Vec<T> z;
                *reinterpret_cast<uint4 *>(&z) = make_uint4(0u, 0u, 0u, 0u);  // +0.0 in every element
                return z;
            }
            return Vec<T>::load(ptr);
        } else {
            return Vec<T>::load(row_ptr(r));
        }
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
    if (Sp != S) return run_summaries<true, true>(x, esize, BH, S, Sp, D, block, xmax, xmin, ta, st);
    return run_summaries<true, false>(x, esize, BH, S, S, D, block, xmax, xmin, ta, st);
}

}  // namespace vsa
