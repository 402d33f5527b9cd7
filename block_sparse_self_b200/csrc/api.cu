// api.cu -- the C ABI of libvsa: argument validation (before any launch),
// error reporting and dispatch to the kernels.
//
// Validation follows the pages' rules ("fastvideo/mlx_runtime/
// windowed_attention.py": _validate_qkv, windowed_attention argument checks,
// _default_scale; "Adaptive tiling (SPADE)", Deviations and notes: a grid
// the candidates do not divide is zero-padded) and the limits of this
// implementation.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {
thread_local std::string g_last_error;
__device__ int g_status_word = 0;  // first device-side failure (see common.cuh)
}  // namespace

vsa_status fail(vsa_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

vsa_status check_cuda(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return VSA_OK;
    return fail(VSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

vsa_status cached_symbol_address(SymbolCache &cache, cudaStream_t st, cudaError_t (*lookup)(void **), void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetDevice");
    if (dev < 0 || dev >= SymbolCache::kDevices) return fail(VSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    // Outside a capture the address is looked up again, so a context that was
    // torn down and created anew (cudaDeviceReset, a released primary
    // context) is never served a stale address.  During a capture the lookup
    // is skipped (it may have to load the module) and the last address seen
    // on the device is used.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const bool capturing = cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
    std::lock_guard<std::mutex> lock(cache.mu);
    if (!capturing || !cache.addr[dev]) {
        void *p = nullptr;
        e = lookup(&p);
        if (e != cudaSuccess) return check_cuda(e, "cudaGetSymbolAddress");
        cache.addr[dev] = p;
    }
    *out = cache.addr[dev];
    return VSA_OK;
}

namespace {
cudaError_t status_word_lookup(void **p) { return cudaGetSymbolAddress(p, g_status_word); }
}  // namespace

int *device_status_word(cudaStream_t st) {
    static SymbolCache cache;
    void *p = nullptr;
    if (cached_symbol_address(cache, st, status_word_lookup, &p) != VSA_OK) return nullptr;
    return static_cast<int *>(p);
}

}  // namespace vsa

using namespace vsa;

namespace {

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
int esize_of(vsa_dtype d) { return d == VSA_BF16 ? 2 : d == VSA_F32 ? 4 : 0; }
cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

#define VSA_REQUIRE(cond, ...)                                   \
    do {                                                         \
        if (!(cond)) return fail(VSA_ERR_INVALID_ARGUMENT, __VA_ARGS__); \
    } while (0)

vsa_status check_grid(vsa_dims3 grid, int S) {
    VSA_REQUIRE(grid.t > 0 && grid.h > 0 && grid.w > 0, "grid dimensions must be positive, got (%d, %d, %d)",
                grid.t, grid.h, grid.w);
    VSA_REQUIRE(static_cast<long long>(grid.t) * grid.h * grid.w == S,
                "grid (%d, %d, %d) has %lld tokens but S = %d", grid.t, grid.h, grid.w,
                static_cast<long long>(grid.t) * grid.h * grid.w, S);
    return VSA_OK;
}

long long lcm_ll(long long a, long long b) {
    long long x = a, y = b;
    while (y) { const long long r = x % y; x = y; y = r; }
    return a / x * b;
}

// Candidate tiles need not divide the grid: the grid is then zero-padded on
// each axis to the next multiple of the candidates' lcm ("Adaptive tiling
// (SPADE)", Deviations and notes); *padded receives that grid.
vsa_status check_tiles(vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, TileSet *ts, vsa_dims3 *padded = nullptr) {
    VSA_REQUIRE(tiles != nullptr, "tiles must not be NULL");
    VSA_REQUIRE(n_tiles >= 1 && n_tiles <= 8, "n_tiles must be in [1, 8], got %d", n_tiles);
    ts->n = n_tiles;
    long long l[3] = {1, 1, 1};
    for (int c = 0; c < n_tiles; ++c) {
        const vsa_dims3 t = tiles[c];
        VSA_REQUIRE(t.t > 0 && t.h > 0 && t.w > 0, "tile %d must be positive, got (%d, %d, %d)", c, t.t, t.h, t.w);
        ts->t[c] = t.t;
        ts->h[c] = t.h;
        ts->w[c] = t.w;
        l[0] = lcm_ll(l[0], t.t);
        l[1] = lcm_ll(l[1], t.h);
        l[2] = lcm_ll(l[2], t.w);
        VSA_REQUIRE(l[0] <= (1 << 20) && l[1] <= (1 << 20) && l[2] <= (1 << 20), "the candidate tiles' lcm is too large");
    }
    for (int c = n_tiles; c < 8; ++c) ts->t[c] = ts->h[c] = ts->w[c] = 1;
    const long long pt = (grid.t + l[0] - 1) / l[0] * l[0], ph = (grid.h + l[1] - 1) / l[1] * l[1],
                    pw = (grid.w + l[2] - 1) / l[2] * l[2];
    VSA_REQUIRE(pt * ph * pw <= 0x7fffffffLL, "the padded grid (%lld, %lld, %lld) has too many tokens", pt, ph, pw);
    if (padded) *padded = vsa_dims3{static_cast<int32_t>(pt), static_cast<int32_t>(ph), static_cast<int32_t>(pw)};
    return VSA_OK;
}


vsa_status check_bhsd(int B, int n_heads, int S, int D) {
    VSA_REQUIRE(B >= 1 && n_heads >= 1, "B and n_heads must be >= 1, got %d, %d", B, n_heads);
    VSA_REQUIRE(S >= 1, "sequence length S must be > 0, got %d", S);
    VSA_REQUIRE(D >= 1, "head dim D must be > 0, got %d", D);
    VSA_REQUIRE(static_cast<long long>(B) * n_heads <= 65535, "B * n_heads must be <= 65535");
    return VSA_OK;
}

vsa_status check_d(int D) {
    if (D != 64 && D != 128) return fail(VSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128, got %d", D);
    return VSA_OK;
}

// [a, a + na) and [b, b + nb) share a byte
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

#define VSA_TRY(expr)                     \
    do {                                  \
        vsa_status _s = (expr);           \
        if (_s != VSA_OK) return _s;      \
    } while (0)

int *status_or_null(void *stream) { return device_status_word(as_stream(stream)); }

}  // namespace

extern "C" {

const char *vsa_last_error(void) { return g_last_error.c_str(); }

vsa_status vsa_padded_grid(vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, vsa_dims3 *padded) {
    VSA_REQUIRE(grid.t > 0 && grid.h > 0 && grid.w > 0, "grid dimensions must be positive, got (%d, %d, %d)",
                grid.t, grid.h, grid.w);
    VSA_REQUIRE(padded != nullptr, "padded must not be NULL");
    TileSet ts;
    return check_tiles(grid, tiles, n_tiles, &ts, padded);
}

vsa_status vsa_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return check_cuda(e, "cudaStreamSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int));
    if (e != cudaSuccess) return check_cuda(e, "reading the device status word");
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int));
    if (e != cudaSuccess) return check_cuda(e, "clearing the device status word");
    if (v == DEV_RUNTIME) return fail(VSA_ERR_RUNTIME, "a device-side check failed (invalid block list, choice or empty key set)");
    if (v == DEV_TIMEOUT) return fail(VSA_ERR_TIMEOUT, "a bounded wait inside a kernel gave up");
    if (v != 0) return fail(VSA_ERR_RUNTIME, "device status word holds %d", v);
    return VSA_OK;
}

size_t vsa_select_tiling_workspace_size(int B, int n_heads, vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles) {
    TileSet ts;
    vsa_dims3 pg;
    if (B < 1 || n_heads < 1 || grid.t < 1 || grid.h < 1 || grid.w < 1) return 0;
    if (check_tiles(grid, tiles, n_tiles, &ts, &pg) != VSA_OK) return 0;
    SelectGeom g;
    if (!select_geometry(pg.t, pg.h, pg.w, ts, &g)) return 0;
    // per region and candidate: a SICS sum and a tile count
    const size_t bytes = static_cast<size_t>(B) * n_heads * g.n_regions * 2 * n_tiles * sizeof(float);
    return (bytes + 255) & ~static_cast<size_t>(255);
}

vsa_status vsa_select_tiling(const void *q, vsa_dtype dtype, int B, int n_heads, int S, int D, vsa_dims3 grid,
                             const vsa_dims3 *tiles, int n_tiles, int32_t *choice, float *sics, void *workspace,
                             size_t workspace_bytes, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(aligned16(q), "q must be a non-NULL 16-byte aligned device pointer");
    VSA_REQUIRE(aligned4(choice), "choice must be a non-NULL 4-byte aligned device pointer");
    VSA_REQUIRE(sics == nullptr || aligned4(sics), "sics must be NULL or 4-byte aligned");
    VSA_TRY(check_grid(grid, S));
    TileSet ts;
    vsa_dims3 pg;
    VSA_TRY(check_tiles(grid, tiles, n_tiles, &ts, &pg));
    SelectGeom g;
    if (!select_geometry(pg.t, pg.h, pg.w, ts, &g))
        return fail(VSA_ERR_UNSUPPORTED,
                    "the candidate tiles' lcm region holds %d cells of their gcd tile (at most 256 supported)",
                    g.cells);
    const size_t need = vsa_select_tiling_workspace_size(B, n_heads, grid, tiles, n_tiles);
    VSA_REQUIRE(aligned16(workspace), "workspace must be a non-NULL 16-byte aligned device pointer");
    VSA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
    return check_cuda(launch_select_tiling(q, esize_of(dtype), B * n_heads, D, grid.t, grid.h, grid.w, pg.t, pg.h,
                                           pg.w, ts, g, choice, sics, static_cast<float *>(workspace),
                                           status_or_null(stream), as_stream(stream)),
                      "select_tiling launch");
}

vsa_status vsa_select_tiling_noalloc(const void *q, vsa_dtype dtype, int B, int n_heads, int S, int D,
                                     vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, int32_t *choice,
                                     float *sics, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(aligned16(q), "q must be a non-NULL 16-byte aligned device pointer");
    VSA_REQUIRE(aligned4(choice), "choice must be a non-NULL 4-byte aligned device pointer");
    VSA_REQUIRE(sics == nullptr || aligned4(sics), "sics must be NULL or 4-byte aligned");
    VSA_TRY(check_grid(grid, S));
    TileSet ts;
    vsa_dims3 pg;
    VSA_TRY(check_tiles(grid, tiles, n_tiles, &ts, &pg));
    SelectGeom g;
    if (!select_geometry(pg.t, pg.h, pg.w, ts, &g))
        return fail(VSA_ERR_UNSUPPORTED,
                    "the candidate tiles' lcm region holds %d cells of their gcd tile (at most 256 supported)",
                    g.cells);
    const size_t need = vsa_select_tiling_workspace_size(B, n_heads, grid, tiles, n_tiles);
    VSA_REQUIRE(need <= VSA_SELECT_TILING_NOALLOC_MAX_BYTES,
                "this call needs %zu bytes of scratch; the allocation-free variant holds at most %d bytes "
                "(use vsa_select_tiling with a workspace instead)",
                need, VSA_SELECT_TILING_NOALLOC_MAX_BYTES);
    float *scratch = nullptr;
    size_t scratch_bytes = 0;
    VSA_TRY(select_static_scratch(&scratch, &scratch_bytes, as_stream(stream)));
    return check_cuda(launch_select_tiling(q, esize_of(dtype), B * n_heads, D, grid.t, grid.h, grid.w, pg.t, pg.h,
                                           pg.w, ts, g, choice, sics, scratch, status_or_null(stream), as_stream(stream)),
                      "select_tiling (no-alloc) launch");
}

static vsa_status permute_common(const void *src, void *dst, vsa_dtype dtype, int B, int n_heads, int S, int D,
                                 vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, const int32_t *choice,
                                 bool inverse, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(aligned16(src) && aligned16(dst), "x and y must be non-NULL 16-byte aligned device pointers");
    VSA_REQUIRE(choice == nullptr || aligned4(choice), "choice must be NULL or 4-byte aligned");
    VSA_TRY(check_grid(grid, S));
    TileSet ts;
    vsa_dims3 pg;
    VSA_TRY(check_tiles(grid, tiles, n_tiles, &ts, &pg));
    const long long Sp = static_cast<long long>(pg.t) * pg.h * pg.w;
    VSA_REQUIRE(static_cast<long long>(B) * n_heads * Sp <= 0x7fffffffLL, "B * n_heads * padded tokens too large");
    const size_t row = static_cast<size_t>(D) * esize_of(dtype);
    const size_t tbytes = static_cast<size_t>(B) * n_heads * S * row, pbytes = static_cast<size_t>(B) * n_heads * Sp * row;
    VSA_REQUIRE(!overlaps(src, inverse ? pbytes : tbytes, dst, inverse ? tbytes : pbytes), "x and y must not overlap");
    return check_cuda(launch_permute(src, dst, esize_of(dtype), B * n_heads, D, grid.t, grid.h, grid.w, pg.t, pg.h,
                                     pg.w, ts, choice, inverse, status_or_null(stream), as_stream(stream)),
                      inverse ? "unpermute launch" : "permute launch");
}

vsa_status vsa_permute(const void *x, void *y, vsa_dtype dtype, int B, int n_heads, int S, int D, vsa_dims3 grid,
                       const vsa_dims3 *tiles, int n_tiles, const int32_t *choice, void *stream) {
    return permute_common(x, y, dtype, B, n_heads, S, D, grid, tiles, n_tiles, choice, false, stream);
}

vsa_status vsa_unpermute(const void *y, void *x, vsa_dtype dtype, int B, int n_heads, int S, int D, vsa_dims3 grid,
                         const vsa_dims3 *tiles, int n_tiles, const int32_t *choice, void *stream) {
    return permute_common(y, x, dtype, B, n_heads, S, D, grid, tiles, n_tiles, choice, true, stream);
}

vsa_status vsa_block_summaries(const void *x_perm, vsa_dtype dtype, int B, int n_heads, int S, int D, int block,
                               void *x_max, void *x_min, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(block == 16 || block == 32 || block == 64 || block == 128 || block == 256,
                "block must be one of 16, 32, 64, 128, 256, got %d", block);
    VSA_REQUIRE(S % block == 0, "block (%d) must divide S (%d)", block, S);
    VSA_REQUIRE(aligned16(x_perm) && aligned16(x_max) && aligned16(x_min),
                "x_perm, x_max and x_min must be non-NULL 16-byte aligned device pointers");
    return check_cuda(launch_summaries(x_perm, esize_of(dtype), B * n_heads, S, D, block, x_max, x_min,
                                       as_stream(stream)),
                      "block_summaries launch");
}

vsa_status vsa_block_summaries_tiled(const void *x, vsa_dtype dtype, int B, int n_heads, int S, int D,
                                     vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, const int32_t *choice,
                                     int block, void *x_max, void *x_min, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(block == 16 || block == 32 || block == 64 || block == 128 || block == 256,
                "block must be one of 16, 32, 64, 128, 256, got %d", block);
    VSA_REQUIRE(aligned16(x) && aligned16(x_max) && aligned16(x_min),
                "x, x_max and x_min must be non-NULL 16-byte aligned device pointers");
    VSA_REQUIRE(choice == nullptr || aligned4(choice), "choice must be NULL or 4-byte aligned");
    VSA_TRY(check_grid(grid, S));
    TileSet ts;
    vsa_dims3 pg;
    VSA_TRY(check_tiles(grid, tiles, n_tiles, &ts, &pg));
    const long long Sp = static_cast<long long>(pg.t) * pg.h * pg.w;
    VSA_REQUIRE(Sp % block == 0, "block (%d) must divide the padded token count (%lld)", block, Sp);
    VSA_REQUIRE(Sp / block <= 0x7fffffffLL && static_cast<long long>(B) * n_heads <= 65535,
                "too many blocks or heads");
    return check_cuda(launch_summaries_tiled(x, esize_of(dtype), B * n_heads, D, grid.t, grid.h, grid.w, pg.t, pg.h,
                                             pg.w, ts, choice, x_max, x_min, status_or_null(stream), as_stream(stream),
                                             block),
                      "block_summaries_tiled launch");
}

vsa_status vsa_block_scores(const void *q_max, const void *q_min, const void *k_max, const void *k_min,
                            vsa_dtype dtype, int B, int n_heads, int nb, int D, float *scores, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, nb, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(aligned16(q_max) && aligned16(q_min) && aligned16(k_max) && aligned16(k_min),
                "summaries must be non-NULL 16-byte aligned device pointers");
    VSA_REQUIRE(aligned4(scores), "scores must be a non-NULL 4-byte aligned device pointer");
    VSA_REQUIRE(static_cast<long long>(nb) <= 65535LL * 64, "nb too large");
    if (dtype == VSA_BF16)  // tensor cores: exact bf16 products, fp32 accumulation
        return check_cuda(launch_scores_tc(q_max, q_min, k_max, k_min, B * n_heads, nb, D, scores, status_or_null(stream),
                                           as_stream(stream)),
                          "block_scores launch");
    return check_cuda(launch_scores(q_max, q_min, k_max, k_min, esize_of(dtype), B * n_heads, nb, D, scores,
                                    as_stream(stream)),
                      "block_scores launch");
}

vsa_status vsa_topk_block_mask(const float *scores, int B, int n_heads, int nb, int k, int n_sink_blocks,
                               int diag_halfwidth, int32_t *idx, int32_t *cnt, int cap, void *stream) {
    VSA_REQUIRE(B >= 1 && n_heads >= 1, "B and n_heads must be >= 1");
    VSA_REQUIRE(nb >= 1, "nb must be >= 1, got %d", nb);
    VSA_REQUIRE(k >= 1 && k <= nb, "k must be in [1, nb] = [1, %d], got %d", nb, k);
    VSA_REQUIRE(n_sink_blocks >= 0 && n_sink_blocks <= nb, "n_sink_blocks must be in [0, nb], got %d",
                n_sink_blocks);
    VSA_REQUIRE(diag_halfwidth >= -1, "diag_halfwidth must be >= -1 (-1 = no diagonal), got %d", diag_halfwidth);
    long long most = static_cast<long long>(k) + n_sink_blocks + (diag_halfwidth >= 0 ? 2LL * diag_halfwidth + 1 : 0);
    if (most > nb) most = nb;
    VSA_REQUIRE(cap >= most, "cap (%d) must be >= min(nb, k + n_sink + 2*diag_halfwidth + 1) = %lld", cap, most);
    VSA_REQUIRE(aligned4(scores) && aligned4(idx) && aligned4(cnt),
                "scores, idx and cnt must be non-NULL 4-byte aligned device pointers");
    return check_cuda(launch_topk(scores, B * n_heads, nb, k, n_sink_blocks, diag_halfwidth, idx, cnt, cap,
                                  as_stream(stream)),
                      "topk launch");
}

vsa_status vsa_block_scores_topk(const void *q_max, const void *q_min, const void *k_max, const void *k_min,
                                 vsa_dtype dtype, int B, int n_heads, int nb, int D, int k, int n_sink_blocks,
                                 int diag_halfwidth, int32_t *idx, int32_t *cnt, int cap, void *stream) {
    VSA_REQUIRE(esize_of(dtype) != 0, "dtype must be VSA_BF16 or VSA_F32");
    VSA_TRY(check_bhsd(B, n_heads, nb, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(k >= 1 && k <= nb, "k must be in [1, nb] = [1, %d], got %d", nb, k);
    VSA_REQUIRE(n_sink_blocks >= 0 && n_sink_blocks <= nb, "n_sink_blocks must be in [0, nb], got %d",
                n_sink_blocks);
    VSA_REQUIRE(diag_halfwidth >= -1, "diag_halfwidth must be >= -1 (-1 = no diagonal), got %d", diag_halfwidth);
    long long most = static_cast<long long>(k) + n_sink_blocks + (diag_halfwidth >= 0 ? 2LL * diag_halfwidth + 1 : 0);
    if (most > nb) most = nb;
    VSA_REQUIRE(cap >= most, "cap (%d) must be >= min(nb, k + n_sink + 2*diag_halfwidth + 1) = %lld", cap, most);
    VSA_REQUIRE(aligned16(q_max) && aligned16(q_min) && aligned16(k_max) && aligned16(k_min),
                "summaries must be non-NULL 16-byte aligned device pointers");
    VSA_REQUIRE(aligned4(idx) && aligned4(cnt), "idx and cnt must be non-NULL 4-byte aligned device pointers");
    if (dtype != VSA_BF16) return fail(VSA_ERR_UNSUPPORTED, "the fused scores and lists take bf16 summaries");
    if (nb > scores_topk_max_blocks())
        return fail(VSA_ERR_UNSUPPORTED, "the fused scores and lists take rows of at most %d blocks, got %d",
                    scores_topk_max_blocks(), nb);
    return check_cuda(launch_scores_topk(q_max, q_min, k_max, k_min, B * n_heads, nb, D, k, n_sink_blocks,
                                         diag_halfwidth, idx, cnt, cap, status_or_null(stream), as_stream(stream)),
                      "scores_topk launch");
}

vsa_status vsa_topp_block_mask(const float *scores, int B, int n_heads, int nb, float p, float scale,
                               int n_sink_blocks, int diag_halfwidth, int32_t *idx, int32_t *cnt, int cap,
                               void *stream) {
    VSA_REQUIRE(B >= 1 && n_heads >= 1, "B and n_heads must be >= 1");
    VSA_REQUIRE(nb >= 1, "nb must be >= 1, got %d", nb);
    VSA_REQUIRE(p > 0.f && p <= 1.f, "p must be in (0, 1], got %g", static_cast<double>(p));
    VSA_REQUIRE(scale >= 0.f && scale < 3.0e38f, "scale must be finite and >= 0, got %g", static_cast<double>(scale));
    VSA_REQUIRE(n_sink_blocks >= 0 && n_sink_blocks <= nb, "n_sink_blocks must be in [0, nb], got %d",
                n_sink_blocks);
    VSA_REQUIRE(diag_halfwidth >= -1, "diag_halfwidth must be >= -1 (-1 = no diagonal), got %d", diag_halfwidth);
    VSA_REQUIRE(cap >= nb, "cap (%d) must be >= nb (%d): a top-p list can hold every block", cap, nb);
    VSA_REQUIRE(aligned4(scores) && aligned4(idx) && aligned4(cnt),
                "scores, idx and cnt must be non-NULL 4-byte aligned device pointers");
    if (nb > 1024) return fail(VSA_ERR_UNSUPPORTED, "top-p lists support rows of at most 1024 blocks, got %d", nb);
    return check_cuda(launch_topp(scores, B * n_heads, nb, p, scale, n_sink_blocks, diag_halfwidth, idx, cnt, cap,
                                  as_stream(stream)),
                      "topp launch");
}

vsa_status vsa_structured_block_list(vsa_mask_kind kind, vsa_dims3 grid, vsa_dims3 tile, vsa_dims3 radius, int block,
                                     int32_t *idx, int32_t *cnt, int cap, int *group_size_out, void *stream) {
    VSA_REQUIRE(grid.t > 0 && grid.h > 0 && grid.w > 0, "grid dimensions must be positive");
    const long long S = static_cast<long long>(grid.t) * grid.h * grid.w;
    VSA_REQUIRE(S < (1LL << 31), "grid too large");
    if (kind == VSA_MASK_SPATIAL) {
        tile = vsa_dims3{1, grid.h, grid.w};
        radius = vsa_dims3{0, 0, 0};
    } else if (kind == VSA_MASK_TEMPORAL) {
        tile = vsa_dims3{grid.t, 1, 1};
        radius = vsa_dims3{0, 0, 0};
    } else {
        VSA_REQUIRE(kind == VSA_MASK_SLIDING_TILE || kind == VSA_MASK_SLIDING_TILE_CENTERED, "unknown mask kind %d",
                    static_cast<int>(kind));
    }
    VSA_REQUIRE(tile.t > 0 && tile.h > 0 && tile.w > 0, "tile must be positive");
    VSA_REQUIRE(grid.t % tile.t == 0 && grid.h % tile.h == 0 && grid.w % tile.w == 0,
                "tile (%d, %d, %d) does not divide the grid (%d, %d, %d)", tile.t, tile.h, tile.w, grid.t, grid.h,
                grid.w);
    VSA_REQUIRE(radius.t >= 0 && radius.h >= 0 && radius.w >= 0, "radius must be >= 0");
    VSA_REQUIRE(block == 32 || block == 64 || block == 128, "block must be 32, 64 or 128, got %d", block);
    VSA_REQUIRE(S % block == 0, "block (%d) must divide S (%lld)", block, S);
    VSA_REQUIRE(aligned4(idx) && aligned4(cnt), "idx and cnt must be non-NULL 4-byte aligned device pointers");
    VSA_REQUIRE(group_size_out != nullptr, "group_size_out must not be NULL");
    const long long vol = static_cast<long long>(tile.t) * tile.h * tile.w;
    long long longest;
    int group;
    if (vol % block == 0) {
        const long long nt[3] = {grid.t / tile.t, grid.h / tile.h, grid.w / tile.w};
        const long long r[3] = {radius.t, radius.h, radius.w};
        longest = vol / block;
        for (int a = 0; a < 3; ++a) longest *= (2 * r[a] + 1 < nt[a] ? 2 * r[a] + 1 : nt[a]);
        group = 0;
    } else if (block % vol == 0 && radius.t == 0 && radius.h == 0 && radius.w == 0) {
        longest = 1;
        group = static_cast<int>(vol);
    } else {
        return fail(VSA_ERR_UNSUPPORTED,
                    "tile volume %lld and block %d: need a tile that is a whole number of blocks, or radius 0 and "
                    "a block that is a whole number of tiles",
                    vol, block);
    }
    VSA_REQUIRE(cap >= longest, "cap (%d) must be >= the longest list (%lld)", cap, longest);
    *group_size_out = group;
    // A radius of n - 1 tiles already spans an axis of n tiles in both forms;
    // clamping keeps the kernel's c +- r and 2r + 1 within int.
    radius.t = radius.t < grid.t / tile.t ? radius.t : grid.t / tile.t - 1;
    radius.h = radius.h < grid.h / tile.h ? radius.h : grid.h / tile.h - 1;
    radius.w = radius.w < grid.w / tile.w ? radius.w : grid.w / tile.w - 1;
    return check_cuda(launch_structured(grid.t, grid.h, grid.w, tile.t, tile.h, tile.w, radius.t, radius.h,
                                        radius.w, kind == VSA_MASK_SLIDING_TILE_CENTERED, block, idx, cnt, cap,
                                        as_stream(stream)),
                      "structured_block_list launch");
}

size_t vsa_head_profile_workspace_size(int B, int n_heads, int S, int D) {
    if (B < 1 || n_heads < 1 || S < 1 || (D != 64 && D != 128)) return 0;
    return vsa::profile_workspace_bytes(B * n_heads, S, D);
}

vsa_status vsa_head_profile(const void *q, const void *k, int B, int n_heads, int S, int D, vsa_dims3 grid,
                            const int32_t *rows, int R, float scale, vsa_profile_rule rule, float *masses,
                            int32_t *kind, void *workspace, size_t workspace_bytes, void *stream) {
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(S < (1 << 30), "S must be < 2^30, got %d", S);
    VSA_TRY(check_grid(grid, S));
    VSA_REQUIRE(aligned16(q) && aligned16(k), "q and k must be non-NULL 16-byte aligned device pointers");
    VSA_REQUIRE(R >= 1 && R <= 128, "R (sampled rows) must be in [1, 128], got %d", R);
    VSA_REQUIRE(aligned4(rows), "rows must be a non-NULL 4-byte aligned device pointer");
    VSA_REQUIRE(aligned4(masses) && aligned4(kind), "masses and kind must be non-NULL 4-byte aligned device pointers");
    VSA_REQUIRE(scale == scale && scale < 3.0e38f, "scale must be finite");
    VSA_REQUIRE(rule == VSA_PROFILE_MASS || rule == VSA_PROFILE_MASS_PER_KEY, "unknown profile rule %d",
                static_cast<int>(rule));
    const size_t need = vsa_head_profile_workspace_size(B, n_heads, S, D);
    VSA_REQUIRE(aligned16(workspace), "workspace must be a non-NULL 16-byte aligned device pointer");
    VSA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
    return check_cuda(launch_head_profile(q, k, B * n_heads, S, D, grid.h * grid.w, rows, R, sc, static_cast<int>(rule),
                                          workspace, masses, kind, status_or_null(stream), as_stream(stream)),
                      "head_profile launch");
}

static vsa_status check_attention_common(const void *q, const void *k, const void *v, void *o, vsa_dtype out_dtype,
                                         int B, int n_heads, int S, int D, float scale) {
    VSA_TRY(check_bhsd(B, n_heads, S, D));
    VSA_TRY(check_d(D));
    VSA_REQUIRE(out_dtype == VSA_BF16 || out_dtype == VSA_F32, "out_dtype must be VSA_BF16 or VSA_F32");
    VSA_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(o),
                "q, k, v and o must be non-NULL 16-byte aligned device pointers");
    const size_t obytes = static_cast<size_t>(B) * n_heads * S * D * esize_of(out_dtype);
    const size_t ibytes = static_cast<size_t>(B) * n_heads * S * D * 2;
    VSA_REQUIRE(!overlaps(o, obytes, q, ibytes) && !overlaps(o, obytes, k, ibytes) && !overlaps(o, obytes, v, ibytes),
                "o must not overlap q, k or v");
    VSA_REQUIRE(scale == scale && scale < 3.0e38f, "scale must be finite");
    return VSA_OK;
}

vsa_status vsa_block_sparse_attention(const void *q, const void *k, const void *v, void *o, vsa_dtype out_dtype,
                                      int B, int n_heads, int S, int D, int block, const int32_t *idx,
                                      const int32_t *cnt, int cap, int list_per_head, int group_size, float scale,
                                      void *stream) {
    VSA_TRY(check_attention_common(q, k, v, o, out_dtype, B, n_heads, S, D, scale));
    VSA_REQUIRE(block == 32 || block == 64 || block == 128, "block must be 32, 64 or 128, got %d", block);
    VSA_REQUIRE(S % block == 0, "block (%d) must divide S (%d)", block, S);
    VSA_REQUIRE(aligned4(idx) && aligned4(cnt), "idx and cnt must be non-NULL 4-byte aligned device pointers");
    VSA_REQUIRE(cap >= 1, "cap must be >= 1, got %d", cap);
    VSA_REQUIRE(group_size >= 0, "group_size must be >= 0, got %d", group_size);
    AttnLaunch L{};
    L.q = q; L.k = k; L.v = v; L.o = o;
    L.out_f32 = out_dtype == VSA_F32;
    L.BH = B * n_heads; L.S = S; L.D = D;
    L.block = block;
    L.window = false;
    L.idx = idx; L.cnt = cnt; L.cap = cap; L.list_per_head = list_per_head ? 1 : 0;
    L.group = group_size; L.nb = S / block;
    L.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
    return launch_attention(L, status_or_null(stream), as_stream(stream));
}

vsa_status vsa_block_sparse_attention_tiled(const void *q, const void *k, const void *v, void *o,
                                            vsa_dtype out_dtype, int B, int n_heads, int S, int D, vsa_dims3 grid,
                                            const vsa_dims3 *tiles, int n_tiles, const int32_t *choice,
                                            const int32_t *idx, const int32_t *cnt, int cap, int list_per_head,
                                            int group_stride, float scale, void *stream) {
    VSA_TRY(check_attention_common(q, k, v, o, out_dtype, B, n_heads, S, D, scale));
    VSA_REQUIRE(group_stride == 0 || (group_stride >= 2 && group_stride <= 128 && (group_stride & (group_stride - 1)) == 0),
                "group_stride must be 0 or a power of two in [2, 128], got %d", group_stride);
    VSA_REQUIRE(aligned4(idx) && aligned4(cnt), "idx and cnt must be non-NULL 4-byte aligned device pointers");
    VSA_REQUIRE(cap >= 1, "cap must be >= 1, got %d", cap);
    VSA_REQUIRE(choice == nullptr || aligned4(choice), "choice must be NULL or 4-byte aligned");
    VSA_TRY(check_grid(grid, S));
    TileSet ts;
    vsa_dims3 pg;
    VSA_TRY(check_tiles(grid, tiles, n_tiles, &ts, &pg));
    const long long Sp = static_cast<long long>(pg.t) * pg.h * pg.w;
    const int vol = ts.t[0] * ts.h[0] * ts.w[0];
    // blocks: the tile itself for volumes 32, 64 and 128, else 128-token parts of it
    VSA_REQUIRE(vol == 32 || vol == 64 || vol % 128 == 0, "tile volume (%d) must be 32, 64 or a multiple of 128", vol);
    const int blk = vol < 128 ? vol : 128;
    if (group_stride != 0 && blk != 128)
        return fail(VSA_ERR_UNSUPPORTED, "group_stride needs 128-token blocks; the tiles hold %d tokens", vol);
    for (int c = 0; c < n_tiles; ++c) {
        VSA_REQUIRE(ts.t[c] * ts.h[c] * ts.w[c] == vol, "every tile must have the volume of tile 0 (%d); tile %d has %d",
                    vol, c, ts.t[c] * ts.h[c] * ts.w[c]);
        VSA_REQUIRE(ts.t[c] % (vol / blk) == 0,
                    "tile %d: tile.t (%d) must be divisible by volume / %d (%d) so each %d-token block is whole "
                    "(h, w) planes",
                    c, ts.t[c], blk, vol / blk, blk);
        // a TMA box (one block) must fit inside the real tensor
        if (ts.t[c] / (vol / blk) > grid.t || ts.h[c] > grid.h || ts.w[c] > grid.w)
            return fail(VSA_ERR_UNSUPPORTED, "tile %d: its %d-token box (%d, %d, %d) is larger than the grid (%d, %d, %d)",
                        c, blk, ts.t[c] / (vol / blk), ts.h[c], ts.w[c], grid.t, grid.h, grid.w);
    }
    AttnLaunch L{};
    L.q = q; L.k = k; L.v = v; L.o = o;
    L.out_f32 = out_dtype == VSA_F32;
    L.BH = B * n_heads; L.S = S; L.D = D;
    L.block = blk;
    L.window = false;
    L.idx = idx; L.cnt = cnt; L.cap = cap; L.list_per_head = list_per_head ? 1 : 0;
    L.group = 0; L.nb = static_cast<int>(Sp / blk);
    L.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
    L.tiled = true;
    L.gstride = group_stride;
    L.T = grid.t; L.Hg = grid.h; L.Wg = grid.w;
    L.Tp = pg.t; L.Hp = pg.h; L.Wp = pg.w;
    L.tiles = ts;
    L.choice = choice;
    return launch_attention(L, status_or_null(stream), as_stream(stream));
}

size_t vsa_centroid_compensated_attention_workspace_size(int B, int n_heads, int S, int D, vsa_dtype out_dtype) {
    if (B < 1 || n_heads < 1 || S < 128 || S % 128 != 0 || (D != 64 && D != 128)) return 0;
    if (out_dtype != VSA_BF16 && out_dtype != VSA_F32) return 0;
    return compensated_workspace_bytes(B * n_heads, S, D, out_dtype == VSA_F32);
}

vsa_status vsa_centroid_compensated_attention(const void *q, const void *k, const void *v, void *o,
                                              vsa_dtype out_dtype, int B, int n_heads, int S, int D, int block,
                                              const int32_t *idx, const int32_t *cnt, int cap, int list_per_head,
                                              float scale, void *workspace, size_t workspace_bytes, void *stream) {
    VSA_TRY(check_attention_common(q, k, v, o, out_dtype, B, n_heads, S, D, scale));
    if (block != 128) return fail(VSA_ERR_UNSUPPORTED, "compensated attention takes 128-token blocks, got %d", block);
    VSA_REQUIRE(S % block == 0, "block (%d) must divide S (%d)", block, S);
    VSA_REQUIRE(aligned4(idx) && aligned4(cnt), "idx and cnt must be non-NULL 4-byte aligned device pointers");
    VSA_REQUIRE(cap >= 1, "cap must be >= 1, got %d", cap);
    if (S / block > 8192) return fail(VSA_ERR_UNSUPPORTED, "compensated attention supports at most 8192 blocks per head");
    const size_t need = vsa_centroid_compensated_attention_workspace_size(B, n_heads, S, D, out_dtype);
    VSA_REQUIRE(workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0,
                "workspace must be a non-NULL 256-byte aligned device pointer");
    VSA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
    const size_t in_bytes = static_cast<size_t>(B) * n_heads * S * D * 2;
    VSA_REQUIRE(!overlaps(workspace, need, o, static_cast<size_t>(B) * n_heads * S * D * esize_of(out_dtype)) &&
                    !overlaps(workspace, need, q, in_bytes) && !overlaps(workspace, need, k, in_bytes) &&
                    !overlaps(workspace, need, v, in_bytes),
                "workspace must not overlap q, k, v or o");
    AttnLaunch L{};
    L.q = q; L.k = k; L.v = v; L.o = o;
    L.out_f32 = out_dtype == VSA_F32;
    L.BH = B * n_heads; L.S = S; L.D = D;
    L.block = block;
    L.window = false;
    L.idx = idx; L.cnt = cnt; L.cap = cap; L.list_per_head = list_per_head ? 1 : 0;
    L.group = 0; L.nb = S / block;
    L.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
    return launch_compensated(L, workspace, status_or_null(stream), as_stream(stream));
}

vsa_status vsa_centroid_compensated_attention_tiled(const void *q, const void *k, const void *v, void *o,
                                                    vsa_dtype out_dtype, int B, int n_heads, int S, int D,
                                                    vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles,
                                                    const int32_t *choice, const int32_t *idx, const int32_t *cnt,
                                                    int cap, int list_per_head, float scale, void *workspace,
                                                    size_t workspace_bytes, void *stream) {
    VSA_TRY(check_attention_common(q, k, v, o, out_dtype, B, n_heads, S, D, scale));
    VSA_REQUIRE(aligned4(idx) && aligned4(cnt), "idx and cnt must be non-NULL 4-byte aligned device pointers");
    VSA_REQUIRE(cap >= 1, "cap must be >= 1, got %d", cap);
    VSA_REQUIRE(choice == nullptr || aligned4(choice), "choice must be NULL or 4-byte aligned");
    VSA_TRY(check_grid(grid, S));
    TileSet ts;
    vsa_dims3 pg;
    VSA_TRY(check_tiles(grid, tiles, n_tiles, &ts, &pg));
    if (pg.t != grid.t || pg.h != grid.h || pg.w != grid.w)
        return fail(VSA_ERR_UNSUPPORTED, "compensated attention in tiled mode needs a grid every tile divides");
    const int vol = ts.t[0] * ts.h[0] * ts.w[0];
    if (vol % 128 != 0)
        return fail(VSA_ERR_UNSUPPORTED, "compensated attention takes 128-token blocks; the tiles hold %d tokens", vol);
    for (int c = 0; c < n_tiles; ++c) {
        VSA_REQUIRE(ts.t[c] * ts.h[c] * ts.w[c] == vol, "every tile must have the volume of tile 0 (%d); tile %d has %d",
                    vol, c, ts.t[c] * ts.h[c] * ts.w[c]);
        VSA_REQUIRE(ts.t[c] % (vol / 128) == 0,
                    "tile %d: tile.t (%d) must be divisible by volume / 128 (%d) so each 128-token block is whole "
                    "(h, w) planes",
                    c, ts.t[c], vol / 128);
        if (ts.t[c] / (vol / 128) > grid.t || ts.h[c] > grid.h || ts.w[c] > grid.w)
            return fail(VSA_ERR_UNSUPPORTED, "tile %d: its 128-token box is larger than the grid", c);
    }
    if (S / 128 > 8192) return fail(VSA_ERR_UNSUPPORTED, "compensated attention supports at most 8192 blocks per head");
    const size_t need = vsa_centroid_compensated_attention_workspace_size(B, n_heads, S, D, out_dtype);
    VSA_REQUIRE(workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0,
                "workspace must be a non-NULL 256-byte aligned device pointer");
    VSA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
    const size_t in_bytes = static_cast<size_t>(B) * n_heads * S * D * 2;
    VSA_REQUIRE(!overlaps(workspace, need, o, static_cast<size_t>(B) * n_heads * S * D * esize_of(out_dtype)) &&
                    !overlaps(workspace, need, q, in_bytes) && !overlaps(workspace, need, k, in_bytes) &&
                    !overlaps(workspace, need, v, in_bytes),
                "workspace must not overlap q, k, v or o");
    AttnLaunch L{};
    L.q = q; L.k = k; L.v = v; L.o = o;
    L.out_f32 = out_dtype == VSA_F32;
    L.BH = B * n_heads; L.S = S; L.D = D;
    L.block = 128;
    L.window = false;
    L.idx = idx; L.cnt = cnt; L.cap = cap; L.list_per_head = list_per_head ? 1 : 0;
    L.group = 0; L.nb = S / 128;
    L.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
    L.tiled = true;
    L.gstride = 0;
    L.T = grid.t; L.Hg = grid.h; L.Wg = grid.w;
    L.Tp = pg.t; L.Hp = pg.h; L.Wp = pg.w;
    L.tiles = ts;
    L.choice = choice;
    return launch_compensated(L, workspace, status_or_null(stream), as_stream(stream));
}

vsa_status vsa_window_attention(const void *q, const void *k, const void *v, void *o, vsa_dtype out_dtype, int B,
                                int n_heads, int S, int D, int window, int sink, float scale, int chunk,
                                void *stream) {
    VSA_TRY(check_attention_common(q, k, v, o, out_dtype, B, n_heads, S, D, scale));
    VSA_REQUIRE(window >= 1, "window must be >= 1, got %d", window);
    VSA_REQUIRE(sink >= 0, "sink must be >= 0, got %d", sink);
    VSA_REQUIRE(sink <= S, "sink (%d) cannot exceed sequence length (%d)", sink, S);
    VSA_REQUIRE(chunk >= 0, "chunk_size must be >= 1 (or 0 for the default), got %d", chunk);
    AttnLaunch L{};
    L.q = q; L.k = k; L.v = v; L.o = o;
    L.out_f32 = out_dtype == VSA_F32;
    L.BH = B * n_heads; L.S = S; L.D = D;
    L.block = 128;
    L.window = true;
    L.dense = window >= S ? 1 : 0;
    L.half = window / 2;
    L.sink = sink;
    L.scale = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
    return launch_attention(L, status_or_null(stream), as_stream(stream));
}

vsa_status vsa_cast_f32_to_bf16(const float *x, void *y, int64_t n, void *stream) {
    VSA_REQUIRE(n >= 0, "n must be >= 0");
    if (n == 0) return VSA_OK;
    VSA_REQUIRE(aligned16(x), "x must be a non-NULL 16-byte aligned device pointer");
    VSA_REQUIRE(y != nullptr && (reinterpret_cast<uintptr_t>(y) & 7u) == 0, "y must be a non-NULL 8-byte aligned device pointer");
    return check_cuda(launch_cast_f32_bf16(x, y, n, as_stream(stream)), "cast launch");
}

vsa_status vsa_debug_wait_timeout(int64_t timeout_ns, void *stream) {
    VSA_REQUIRE(timeout_ns >= 0 && timeout_ns <= 10000000000LL, "timeout_ns must be in [0, 1e10]");
    return check_cuda(launch_wait_timeout(static_cast<uint64_t>(timeout_ns), status_or_null(stream), as_stream(stream)),
                      "wait_timeout launch");
}

}  // extern "C"
