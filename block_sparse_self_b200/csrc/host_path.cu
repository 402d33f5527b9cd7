// host_path.cu -- the whole SPADE path for Q, K, V and O in host memory.
//
// "Adaptive tiling (SPADE)", Recipe: per head, choose the tiling, order the
// tokens tile by tile, score key blocks with the min/max summaries, keep the
// top-k blocks plus the sink and diagonal blocks, attend, and return to the
// T-major order.  The device steps are the library's own entry points
// (vsa_select_tiling, vsa_block_summaries_tiled, vsa_block_scores,
// vsa_topk_block_mask, vsa_block_sparse_attention_tiled), run on groups of
// (b, head) rows staged through a caller-provided device workspace.  Copies
// in and out run on two streams of their own, so the copies of one group
// overlap the kernels of another; every (b, head) is independent, so the
// result equals the device path on the whole batch bit for bit.
#include <string.h>

#include "internal.h"

using namespace vsa;

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Sizes of one group of at most R (b, head) rows, and where each buffer sits
// in the workspace.
struct HostPlan {
    int R;                 // rows per group (the largest group)
    int n_groups;
    int block, nb, cap;
    size_t in_bytes;       // one of q, k, v for R rows
    size_t out_bytes;      // o for R rows
    size_t sel_bytes;      // select_tiling workspace for R rows
    // offsets
    size_t in_off[2][3], out_off[2], choice_off, sel_off, summ_off[4], scores_off, idx_off, cnt_off, total;
};

vsa_status plan_host(int B, int n_heads, int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, int k,
                     int n_sink, int diag_hw, int out_esize, int groups, HostPlan *p) {
    if (B < 1 || n_heads < 1 || S < 1 || D < 1) return fail(VSA_ERR_INVALID_ARGUMENT, "B, n_heads, S and D must be >= 1");
    if (groups < 1) return fail(VSA_ERR_INVALID_ARGUMENT, "groups must be >= 1, got %d", groups);
    if (tiles == nullptr || n_tiles < 1 || n_tiles > kMaxTiles)
        return fail(VSA_ERR_INVALID_ARGUMENT, "n_tiles must be in [1, %d] with a non-NULL tiles array", kMaxTiles);
    const long long BH = static_cast<long long>(B) * n_heads;
    vsa_dims3 pg;
    const vsa_status st = vsa_padded_grid(grid, tiles, n_tiles, &pg);
    if (st != VSA_OK) return st;
    const int vol = tiles[0].t * tiles[0].h * tiles[0].w;
    for (int c = 1; c < n_tiles; ++c)
        if (tiles[c].t * tiles[c].h * tiles[c].w != vol)
            return fail(VSA_ERR_INVALID_ARGUMENT, "every candidate tile must have the volume of tile 0 (%d)", vol);
    if (!(vol == 32 || vol == 64 || vol % 128 == 0))
        return fail(VSA_ERR_UNSUPPORTED, "tile volume %d: the host path runs tiles of 32, 64 or a multiple of 128 tokens",
                    vol);
    p->block = vol < 128 ? vol : 128;
    const long long Sp = static_cast<long long>(pg.t) * pg.h * pg.w;
    if (Sp % p->block) return fail(VSA_ERR_INVALID_ARGUMENT, "block does not divide the padded grid");
    p->nb = static_cast<int>(Sp / p->block);
    if (k < 1 || k > p->nb) return fail(VSA_ERR_INVALID_ARGUMENT, "k must be in [1, nb] = [1, %d], got %d", p->nb, k);
    long long cap = static_cast<long long>(k) + n_sink + (diag_hw >= 0 ? 2LL * diag_hw + 1 : 0);
    p->cap = static_cast<int>(cap < p->nb ? cap : p->nb);
    p->n_groups = static_cast<int>(groups < BH ? groups : BH);
    p->R = static_cast<int>((BH + p->n_groups - 1) / p->n_groups);
    p->in_bytes = static_cast<size_t>(p->R) * S * D * 2;
    p->out_bytes = static_cast<size_t>(p->R) * S * D * out_esize;
    p->sel_bytes = n_tiles > 1 ? vsa_select_tiling_workspace_size(1, p->R, grid, tiles, n_tiles) : 0;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    for (int s = 0; s < 2; ++s)
        for (int t = 0; t < 3; ++t) p->in_off[s][t] = take(p->in_bytes);
    for (int s = 0; s < 2; ++s) p->out_off[s] = take(p->out_bytes);
    p->choice_off = take(static_cast<size_t>(p->R) * 4);
    p->sel_off = take(p->sel_bytes > 0 ? p->sel_bytes : 256);
    for (int t = 0; t < 4; ++t) p->summ_off[t] = take(static_cast<size_t>(p->R) * p->nb * D * 2);
    p->scores_off = take(static_cast<size_t>(p->R) * p->nb * p->nb * 4);
    p->idx_off = take(static_cast<size_t>(p->R) * p->nb * p->cap * 4);
    p->cnt_off = take(static_cast<size_t>(p->R) * p->nb * 4);
    p->total = off;
    return VSA_OK;
}

// Streams and events of one call, released at the end of it (a stream or an
// event destroyed with work pending is released once that work completes).
struct HostStreams {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, ready[2] = {}, done[2] = {}, copied[2] = {}, last = nullptr;
    ~HostStreams() {
        for (cudaEvent_t e : {start, ready[0], ready[1], done[0], done[1], copied[0], copied[1], last})
            if (e) cudaEventDestroy(e);
        if (h2d) cudaStreamDestroy(h2d);
        if (d2h) cudaStreamDestroy(d2h);
    }
    cudaError_t create() {
        cudaError_t e = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking);
        for (cudaEvent_t *ev : {&start, &ready[0], &ready[1], &done[0], &done[1], &copied[0], &copied[1], &last})
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        return e;
    }
};

}  // namespace

extern "C" {

size_t vsa_spade_attention_host_workspace_size(int B, int n_heads, int S, int D, vsa_dims3 grid,
                                               const vsa_dims3 *tiles, int n_tiles, int k, int n_sink_blocks,
                                               int diag_halfwidth, vsa_dtype out_dtype, int groups) {
    HostPlan p;
    const int oes = out_dtype == VSA_F32 ? 4 : 2;
    if (plan_host(B, n_heads, S, D, grid, tiles, n_tiles, k, n_sink_blocks, diag_halfwidth, oes, groups, &p) != VSA_OK)
        return 0;
    return p.total;
}

vsa_status vsa_spade_attention_host(const void *q, const void *k, const void *v, void *o, vsa_dtype out_dtype,
                                    int B, int n_heads, int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles,
                                    int n_tiles, int topk, int n_sink_blocks, int diag_halfwidth, float scale,
                                    int groups, void *workspace, size_t workspace_bytes, void *stream) {
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
        return fail(VSA_ERR_INVALID_ARGUMENT, "q, k, v and o must be non-NULL host pointers");
    if (out_dtype != VSA_BF16 && out_dtype != VSA_F32)
        return fail(VSA_ERR_INVALID_ARGUMENT, "out_dtype must be VSA_BF16 or VSA_F32");
    if (static_cast<long long>(B) * n_heads > 65535) return fail(VSA_ERR_INVALID_ARGUMENT, "B * n_heads must be <= 65535");
    const int oes = out_dtype == VSA_F32 ? 4 : 2;
    HostPlan p;
    vsa_status st = plan_host(B, n_heads, S, D, grid, tiles, n_tiles, topk, n_sink_blocks, diag_halfwidth, oes,
                              groups, &p);
    if (st != VSA_OK) return st;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(VSA_ERR_INVALID_ARGUMENT, "workspace must be a non-NULL 256-byte aligned device pointer");
    if (workspace_bytes < p.total)
        return fail(VSA_ERR_INVALID_ARGUMENT, "workspace holds %zu bytes, %zu needed", workspace_bytes, p.total);
    // the device steps check their arguments again; these checks make the
    // common errors come back before any copy is issued
    if (static_cast<long long>(grid.t) * grid.h * grid.w != S)
        return fail(VSA_ERR_INVALID_ARGUMENT, "grid (%d, %d, %d) does not hold S = %d tokens", grid.t, grid.h, grid.w, S);
    if (D != 64 && D != 128) return fail(VSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128, got %d", D);
    if (n_sink_blocks < 0 || n_sink_blocks > p.nb)
        return fail(VSA_ERR_INVALID_ARGUMENT, "n_sink_blocks must be in [0, nb], got %d", n_sink_blocks);
    if (diag_halfwidth < -1) return fail(VSA_ERR_INVALID_ARGUMENT, "diag_halfwidth must be >= -1, got %d", diag_halfwidth);
    if (!(scale == scale && scale < 3.0e38f)) return fail(VSA_ERR_INVALID_ARGUMENT, "scale must be finite");
    for (int c = 0; c < n_tiles; ++c) {
        const int per = tiles[c].t * tiles[c].h * tiles[c].w / p.block;  // blocks per tile
        if (tiles[c].t % per != 0 || tiles[c].t / per > grid.t || tiles[c].h > grid.h || tiles[c].w > grid.w)
            return fail(VSA_ERR_UNSUPPORTED,
                        "tile %d: its %d-token blocks must be whole (h, w) planes of the tile and fit in the grid", c,
                        p.block);
    }
    char *ws = static_cast<char *>(workspace);
    const cudaStream_t comp = static_cast<cudaStream_t>(stream);
    const long long BH = static_cast<long long>(B) * n_heads;
    const size_t row_in = static_cast<size_t>(S) * D * 2, row_out = static_cast<size_t>(S) * D * oes;

    HostStreams hs;
    cudaError_t ce = hs.create();
    if (ce != cudaSuccess) return check_cuda(ce, "creating the copy streams");
    // the copy streams start behind the work already queued on `stream`
    // (an earlier call may still be using the workspace)
    ce = cudaEventRecord(hs.start, comp);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(hs.h2d, hs.start, 0);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(hs.d2h, hs.start, 0);
    if (ce != cudaSuccess) return check_cuda(ce, "ordering the copy streams");

    const char *src[3] = {static_cast<const char *>(q), static_cast<const char *>(k), static_cast<const char *>(v)};
    int32_t *choice = reinterpret_cast<int32_t *>(ws + p.choice_off);
    void *summ[4];
    for (int t = 0; t < 4; ++t) summ[t] = ws + p.summ_off[t];
    float *scores = reinterpret_cast<float *>(ws + p.scores_off);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + p.idx_off);
    int32_t *cnt = reinterpret_cast<int32_t *>(ws + p.cnt_off);

    for (int g = 0; g < p.n_groups && st == VSA_OK; ++g) {
        const long long a = BH * g / p.n_groups, b = BH * (g + 1) / p.n_groups;
        const int n = static_cast<int>(b - a), slot = g & 1;
        // inputs: wait until the attention of group g - 2 is done with the slot
        if (g >= 2) ce = cudaStreamWaitEvent(hs.h2d, hs.done[slot], 0);
        for (int t = 0; t < 3 && ce == cudaSuccess; ++t)
            ce = cudaMemcpyAsync(ws + p.in_off[slot][t], src[t] + a * row_in, n * row_in, cudaMemcpyHostToDevice,
                                 hs.h2d);
        if (ce == cudaSuccess) ce = cudaEventRecord(hs.ready[slot], hs.h2d);
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(comp, hs.ready[slot], 0);
        // the output slot: wait until group g - 2's copy back has read it
        if (ce == cudaSuccess && g >= 2) ce = cudaStreamWaitEvent(comp, hs.copied[slot], 0);
        if (ce != cudaSuccess) {
            st = check_cuda(ce, "staging a group of heads");
            break;
        }
        const void *qd = ws + p.in_off[slot][0], *kd = ws + p.in_off[slot][1], *vd = ws + p.in_off[slot][2];
        void *od = ws + p.out_off[slot];
        const int32_t *ch = nullptr;
        if (n_tiles > 1) {
            st = vsa_select_tiling(qd, VSA_BF16, 1, n, S, D, grid, tiles, n_tiles, choice, nullptr, ws + p.sel_off,
                                   p.sel_bytes, stream);
            ch = choice;
        }
        if (st == VSA_OK)
            st = vsa_block_summaries_tiled(qd, VSA_BF16, 1, n, S, D, grid, tiles, n_tiles, ch, p.block, summ[0],
                                           summ[1], stream);
        if (st == VSA_OK)
            st = vsa_block_summaries_tiled(kd, VSA_BF16, 1, n, S, D, grid, tiles, n_tiles, ch, p.block, summ[2],
                                           summ[3], stream);
        if (st == VSA_OK)
            st = vsa_block_scores(summ[0], summ[1], summ[2], summ[3], VSA_BF16, 1, n, p.nb, D, scores, stream);
        if (st == VSA_OK)
            st = vsa_topk_block_mask(scores, 1, n, p.nb, topk, n_sink_blocks, diag_halfwidth, idx, cnt, p.cap, stream);
        if (st == VSA_OK)
            st = vsa_block_sparse_attention_tiled(qd, kd, vd, od, out_dtype, 1, n, S, D, grid, tiles, n_tiles, ch, idx,
                                                  cnt, p.cap, 1, 0, scale, stream);
        if (st != VSA_OK) break;
        ce = cudaEventRecord(hs.done[slot], comp);
        if (ce == cudaSuccess) ce = cudaStreamWaitEvent(hs.d2h, hs.done[slot], 0);
        if (ce == cudaSuccess)
            ce = cudaMemcpyAsync(static_cast<char *>(o) + a * row_out, od, n * row_out, cudaMemcpyDeviceToHost, hs.d2h);
        if (ce == cudaSuccess) ce = cudaEventRecord(hs.copied[slot], hs.d2h);
        if (ce != cudaSuccess) st = check_cuda(ce, "copying a group of outputs back");
    }
    // whatever happened, `stream` ends behind both copy streams, so the
    // workspace and the host output are settled once it reaches this point
    cudaError_t e1 = cudaEventRecord(hs.last, hs.h2d);
    if (e1 == cudaSuccess) e1 = cudaStreamWaitEvent(comp, hs.last, 0);
    cudaError_t e2 = cudaEventRecord(hs.copied[0], hs.d2h);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(comp, hs.copied[0], 0);
    if (st != VSA_OK) return st;
    if (e1 != cudaSuccess) return check_cuda(e1, "joining the input copies");
    return check_cuda(e2, "joining the output copies");
}

}  // extern "C"
