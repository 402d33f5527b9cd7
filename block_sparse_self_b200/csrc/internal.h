// internal.h -- host-side declarations shared by the libvsa translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/vsa.h"

namespace vsa {

// Record a message for vsa_last_error() and return `s`.
vsa_status fail(vsa_status s, const char *fmt, ...);
// Map a CUDA error to VSA_ERR_CUDA (with its message), or VSA_OK.
vsa_status check_cuda(cudaError_t e, const char *what);
// Per-device cache of a __device__ symbol's address (see cached_symbol_address).
struct SymbolCache {
    static constexpr int kDevices = 128;
    std::mutex mu;
    void *addr[kDevices] = {};
};
// Device address of a file-scope __device__ symbol on the current device.
// `lookup` calls cudaGetSymbolAddress in the symbol's own file.  It runs on
// every call whose stream is not capturing; during a capture the address
// cached by the last such call on the device is used.
vsa_status cached_symbol_address(SymbolCache &cache, cudaStream_t st, cudaError_t (*lookup)(void **), void **out);
// Device address of the status word of the current device (nullptr on error).
int *device_status_word(cudaStream_t st);

constexpr int kMaxTiles = 8;
struct TileSet {
    int n;
    int t[kMaxTiles], h[kMaxTiles], w[kMaxTiles];
};

// Launchers (arguments already validated by the C ABI layer).
// (T, H, W): the real grid (T-major side); (Tp, Hp, Wp): the grid the tiles
// cut, equal to it or zero-padded (permuted side).
cudaError_t launch_permute(const void *src, void *dst, int esize, int BH, int D, int T, int H, int W, int Tp, int Hp,
                           int Wp, const TileSet &tiles, const int32_t *choice, bool inverse, int *status,
                           cudaStream_t st);
cudaError_t launch_cast_f32_bf16(const float *x, void *y, int64_t n, cudaStream_t st);
cudaError_t launch_summaries(const void *x, int esize, int BH, int S, int D, int block, void *xmax, void *xmin,
                             cudaStream_t st);
// Summaries of the blocks of a T-major x taken in each head's tile-contiguous order.
// (T, H, W) real grid, (Tp, Hp, Wp) padded grid: padding rows are zero vectors.
cudaError_t launch_summaries_tiled(const void *x, int esize, int BH, int D, int T, int H, int W, int Tp, int Hp,
                                   int Wp, const TileSet &tiles, const int32_t *choice, void *xmax, void *xmin,
                                   int *status, cudaStream_t st, int block);
cudaError_t launch_scores(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int esize, int BH,
                          int nb, int D, float *scores, cudaStream_t st);
// bf16 summaries on tcgen05 (D in {64, 128})
cudaError_t launch_scores_tc(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int BH, int nb,
                             int D, float *scores, int *status, cudaStream_t st);
cudaError_t launch_topk(const float *scores, int BH, int nb, int k, int n_sink, int diag_hw, int32_t *idx,
                        int32_t *cnt, int cap, cudaStream_t st);
// Scores and top-k lists in one kernel (bf16 summaries, nb <= scores_topk_max_blocks()).
int scores_topk_max_blocks();
cudaError_t launch_scores_topk(const void *qmax, const void *qmin, const void *kmax, const void *kmin, int BH, int nb,
                               int D, int k, int n_sink, int diag_hw, int32_t *idx, int32_t *cnt, int cap, int *status,
                               cudaStream_t st);
cudaError_t launch_topp(const float *scores, int BH, int nb, float p, float scale, int n_sink, int diag_hw,
                        int32_t *idx, int32_t *cnt, int cap, cudaStream_t st);
cudaError_t launch_structured(int T, int H, int W, int tt, int th, int tw, int rt, int rh, int rw, bool centered,
                              int block, int32_t *idx, int32_t *cnt, int cap, cudaStream_t st);

struct SelectGeom {
    int Rt, Rh, Rw;   // region = per-axis lcm of the candidate tiles
    int Ct, Ch, Cw;   // cell = per-axis gcd of the candidate tiles
    int n_regions;    // regions per (b, head) of the padded grid
    int cells;        // cells per region
};
// (Tp, Hp, Wp): the padded grid (every axis a multiple of the region's).
bool select_geometry(int Tp, int Hp, int Wp, const TileSet &tiles, SelectGeom *g);
// Per region and candidate: the sum of SICS over its tiles that hold a non-zero
// query, and the number of such tiles (two floats each).
cudaError_t launch_select_tiling(const void *q, int esize, int BH, int D, int T, int H, int W, int Tp, int Hp, int Wp,
                                 const TileSet &tiles, const SelectGeom &g, int32_t *choice, float *sics,
                                 float *partial, int *status, cudaStream_t st);

struct AttnLaunch {
    const void *q, *k, *v;
    void *o;
    int out_f32;
    int BH, S, D;
    int block;          // rows per query tile = keys per key tile
    bool window;
    // block-list mode
    const int32_t *idx, *cnt;
    int cap, list_per_head, group, nb;
    // window mode
    int half, sink, dense;
    float scale;
    // tiled mode: q, k, v, o in T-major order; each (b, head) uses its chosen
    // tiling and the kernel permutes through its TMA boxes and epilogue
    bool tiled;
    int gstride;  // tiled mode: strided groups (0 = none)
    int T, Hg, Wg;      // tiled mode: the real grid (S = T * Hg * Wg tokens in q, k, v, o)
    int Tp, Hp, Wp;     // tiled mode: the padded grid the tiles cut (block lists over its positions)
    TileSet tiles;
    const int32_t *choice;
    // optional: per row (position p of head bh at stats[bh * positions + p])
    // the softmax state behind the normalised output, in the log2 domain:
    // (m, l) with l = sum over the visible keys of 2^(scale log2e q.k - m)
    float2 *stats;
};
vsa_status launch_attention(const AttnLaunch &a, int *status, cudaStream_t st);
// Two query tiles per CTA (128-token blocks only); launch_attention routes to it.
vsa_status launch_attention_pp(const AttnLaunch &a, int *status, cudaStream_t st);
// [BH, S, D] bf16 as a 3-D TMA tensor map (D, S, BH), box (64, rows, 1), 128-byte swizzle.
bool make_tile_map(CUtensorMap *m, const void *ptr, int D, int S, int BH, int rows);
// [BH, T, H, W, D] bf16 as a 5-D TMA tensor map (D, W, H, T, BH), box
// (64, bw, bh, bt, 1), 128-byte swizzle: a (bt, bh, bw) token box lands as
// rows of 128 bytes in (t, h, w) row-major order.
bool make_box_map(CUtensorMap *m, const void *ptr, int D, int T, int H, int W, int BH, int bt, int bh, int bw);
// [BH, nb, nb] fp32 scores as a 3-D tensor (nb, nb, BH), box (32, 128, 1), 128-byte swizzle, for TMA stores
// (needs nb % 4 == 0 and a 16-byte aligned base).
bool make_scores_store_map(CUtensorMap *m, float *ptr, int nb, int BH);

cudaError_t launch_wait_timeout(uint64_t limit_ns, int *status, cudaStream_t st);

// Head profile (profile.cu): CTAs per head over the key tiles, and the scratch
// (gathered sample tiles, then per-part row partials) that launch needs.
int profile_split(int BH, int S);
size_t profile_workspace_bytes(int BH, int S, int D);
cudaError_t launch_head_profile(const void *q, const void *k, int BH, int S, int D, int HW, const int32_t *rows,
                                int R, float scale, int rule, void *workspace, float *masses, int32_t *kind,
                                int *status, cudaStream_t st);

// Skipped key blocks compensated by their centroids (compensated.cu).
size_t compensated_workspace_bytes(int BH, int S, int D, int out_f32);
vsa_status launch_compensated(const AttnLaunch &a, void *workspace, int *status, cudaStream_t st);

// Address and size of the file-scope scratch array that
// vsa_select_tiling_noalloc uses (see cached_symbol_address).
vsa_status select_static_scratch(float **ptr, size_t *bytes, cudaStream_t st);

}  // namespace vsa
