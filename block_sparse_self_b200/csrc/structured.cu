// structured.cu -- structured static masks as block lists.
//
// "ADR-0001: Sparse-attention roadmap for video DiTs", step 1
// (spatial_only_mask, temporal_only_mask, sliding_tile_block_mask,
// sliding_tile_centered_mask).  Every one of them is a tile neighbourhood:
// query and key tokens see each other iff their tiles' coordinates differ by
// at most the radius along each axis, clipped at the grid border.  The
// centred form keeps min(2r + 1, n) tiles per axis instead, the window moved
// inside the grid at the border.  In the tile-contiguous order of that tile,
// when a tile is a whole number of blocks, query block i lists every block of
// every neighbouring tile in ascending order.  When a block is made of several
// radius-0 tiles, query block i lists only itself (the attention kernel then
// applies the tile-volume group mask inside the block).
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

// Key tiles [lo, hi] of query tile c along an axis of n tiles.
__device__ __forceinline__ int2 axis_window(int c, int r, int n, bool centered) {
    if (!centered) return make_int2(max(0, c - r), min(n - 1, c + r));
    const int w = min(2 * r + 1, n);
    const int lo = max(0, min(c - r, n - w));
    return make_int2(lo, lo + w - 1);
}

__global__ void neighbourhood_kernel(int T, int H, int W, int tt, int th, int tw, int rt, int rh, int rw, bool centered,
                                     int block, int nb, int32_t *__restrict__ idx, int32_t *__restrict__ cnt,
                                     int cap) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nb) return;
    const int vol = tt * th * tw;
    const int bpt = vol / block;  // blocks per tile
    const int ntt = T / tt, nth = H / th, ntw = W / tw;
    const int tile = i / bpt;
    const int ct = tile / (nth * ntw), ch = (tile / ntw) % nth, cw = tile % ntw;
    int32_t *out = idx + static_cast<size_t>(i) * cap;
    const int2 wt = axis_window(ct, rt, ntt, centered), wh = axis_window(ch, rh, nth, centered),
               ww = axis_window(cw, rw, ntw, centered);
    int c = 0;
    for (int at = wt.x; at <= wt.y; ++at)
        for (int ah = wh.x; ah <= wh.y; ++ah)
            for (int aw = ww.x; aw <= ww.y; ++aw) {
                const int nt = (at * nth + ah) * ntw + aw;
                for (int q = 0; q < bpt; ++q) {
                    if (c < cap) out[c] = nt * bpt + q;
                    ++c;
                }
            }
    for (int s = c; s < cap; ++s) out[s] = -1;
    cnt[i] = c;
}

__global__ void self_list_kernel(int nb, int32_t *__restrict__ idx, int32_t *__restrict__ cnt, int cap) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nb) return;
    int32_t *out = idx + static_cast<size_t>(i) * cap;
    out[0] = i;
    for (int s = 1; s < cap; ++s) out[s] = -1;
    cnt[i] = 1;
}

}  // namespace

cudaError_t launch_structured(int T, int H, int W, int tt, int th, int tw, int rt, int rh, int rw, bool centered,
                              int block, int32_t *idx, int32_t *cnt, int cap, cudaStream_t st) {
    const int nb = T * H * W / block;
    const int vol = tt * th * tw;
    const int grid = (nb + 127) / 128;
    if (vol % block == 0)
        neighbourhood_kernel<<<grid, 128, 0, st>>>(T, H, W, tt, th, tw, rt, rh, rw, centered, block, nb, idx, cnt,
                                                    cap);
    else
        self_list_kernel<<<grid, 128, 0, st>>>(nb, idx, cnt, cap);
    return cudaGetLastError();
}

}  // namespace vsa
