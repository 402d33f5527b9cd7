/*
 * vsa.h -- C ABI of libvsa: structured and input-adaptive block-sparse
 * self-attention over a video DiT's T-major spatiotemporal token sequence,
 * for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Token order is T-major: token (t, h, w) of a (T, Hg, Wg) latent grid is
 *   at index (t*Hg + h)*Wg + w, S = T*Hg*Wg ("ADR-0001: Sparse-attention
 *   roadmap for video DiTs", Conventions).
 * - Tensors are dense row-major device arrays.  Q/K/V/O are [B, n_heads, S, D];
 *   (b, h) pairs are flattened as bh = b*n_heads + h.
 * - Every pointer argument is a DEVICE pointer unless stated, 16-byte aligned.
 *   The caller owns every buffer; the library allocates no device memory.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *   call only enqueues work on it and returns without synchronising.
 * - Argument errors are detected on the host before anything is launched
 *   and return VSA_ERR_INVALID_ARGUMENT (the pages raise ValueError for
 *   these, "ADR-0001", Conventions: Validation).  Violations that only the
 *   device can see (a block index out of range, an empty key set) set a
 *   device status word that vsa_device_status() returns (the pages'
 *   RuntimeError).  A CUDA launch failure returns VSA_ERR_CUDA.
 * - vsa_last_error() gives a readable message for the last non-OK status
 *   returned on the calling host thread.
 */
#ifndef VSA_H
#define VSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARGUMENT = 1, /* bad shape, size or option (ValueError)      */
    VSA_ERR_RUNTIME = 2,          /* violated invariant seen on the device        */
    VSA_ERR_CUDA = 3,             /* CUDA runtime / launch failure                */
    VSA_ERR_UNSUPPORTED = 4,      /* valid request the library does not implement */
    VSA_ERR_TIMEOUT = 5           /* a bounded on-device wait gave up             */
} vsa_status;

typedef enum { VSA_BF16 = 0, VSA_F32 = 1 } vsa_dtype;

/* A (t, h, w) triple: a latent grid (T, Hg, Wg), a tile (tt, th, tw) or a
 * neighbourhood radius (rt, rh, rw).                                        */
typedef struct { int32_t t, h, w; } vsa_dims3;

typedef enum {
    VSA_MASK_SPATIAL = 0,      /* same frame: tile (1, Hg, Wg), radius 0      */
    VSA_MASK_TEMPORAL = 1,     /* same (h, w): tile (T, 1, 1), radius 0       */
    VSA_MASK_SLIDING_TILE = 2, /* tiles whose coordinates differ by <= radius */
    VSA_MASK_SLIDING_TILE_CENTERED = 3 /* 2 radius + 1 tiles per axis, shifted
                                          inside the grid at the border     */
} vsa_mask_kind;

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char *vsa_last_error(void);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: VSA_OK, VSA_ERR_RUNTIME (a device-side check failed)
 * or VSA_ERR_TIMEOUT (a bounded wait inside a kernel gave up).  Meant for
 * tests and debugging; the compute calls never synchronise.               */
vsa_status vsa_device_status(void *stream);

/* ------------------------------------------------------------------------ */
/* Grids the candidate tiles do not divide.  "Adaptive tiling (SPADE)",
 * Deviations and notes: the grid is padded with zero tokens until every
 * candidate tiles it, the padding takes no part in the cohesion, and padded
 * keys are masked.  Here each axis is rounded up to the next multiple of the
 * least common multiple of the candidates' extents on that axis:
 *   padded = (ceil(T / lt) lt, ceil(Hg / lh) lh, ceil(Wg / lw) lw).
 * Every call that takes (grid, tiles) works on that padded grid: tilings,
 * permuted positions and block indices refer to it (Sp = padded.t * padded.h
 * * padded.w positions per head), while the T-major tensors it reads or
 * writes hold the S = T*Hg*Wg real tokens only.  With a grid every
 * candidate divides, padded == grid and Sp == S.
 * Returns VSA_ERR_INVALID_ARGUMENT for a non-positive grid or tile, an lcm
 * above 2^20 or a padded grid of 2^31 tokens or more.                      */
vsa_status vsa_padded_grid(vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles,
                           vsa_dims3 *padded);

/* ------------------------------------------------------------------------ */
/* Adaptive tiling: per-(b, head) choice of the most cohesive tiling.
 * "Adaptive tiling (SPADE)", The idea, step 1, and the function table
 * (block_self_similarity, select_tiling), "Deviations and notes" (selection
 * statistic; zero-padded grids).
 *
 * For every (b, head) and candidate c, the cohesion is the mean over the
 * tiles of tiling c (of the padded grid, see vsa_padded_grid) that hold at
 * least one non-zero-norm query of the tile's SICS: the mean cosine
 * similarity over the distinct pairs of its non-zero-norm queries, computed
 * as (|sum of unit queries|^2 - m) / (m (m - 1)) (a tile with m < 2 scores
 * 0).  choice[bh] = argmax_c cohesion, ties to the lower c.
 *
 *   q        [B, n_heads, S, D] in `dtype` (VSA_BF16 or VSA_F32)
 *   grid     (T, Hg, Wg) with T*Hg*Wg == S (padded as vsa_padded_grid says)
 *   tiles    HOST array of n_tiles candidate tiles (1 <= n_tiles <= 8)
 *   choice   [B*n_heads] int32 output
 *   sics     [B*n_heads, n_tiles] fp32 output, or NULL
 *   workspace, workspace_bytes: device scratch of at least
 *            vsa_select_tiling_workspace_size(...) bytes, 16-byte aligned;
 *            its contents need not be initialised and are overwritten.
 * Limits: D in {64, 128}; the lcm of the candidate tiles (per axis) may
 * hold at most 256 cells of gcd-tile size (VSA_ERR_UNSUPPORTED otherwise).
 * Cohesion is accumulated in fp32: candidates whose cohesion differs by
 * less than about 1e-5 may be ranked either way.                          */
size_t vsa_select_tiling_workspace_size(int B, int n_heads, vsa_dims3 grid,
                                        const vsa_dims3 *tiles, int n_tiles);
vsa_status vsa_select_tiling(const void *q, vsa_dtype dtype, int B, int n_heads,
                             int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles,
                             int n_tiles, int32_t *choice, float *sics,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Allocation-free variant of vsa_select_tiling.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory, or pass a workspace, at the point where they choose the
 * tilings -- for example code that runs inside a memory pool or allocator,
 * a process whose device memory is entirely reserved by another framework's
 * pool, or a plugin interface that hands over inputs and outputs but no
 * allocator and no workspace argument.
 *
 * Same arguments and results as vsa_select_tiling, without the workspace.
 * The scratch lives in a file-scope device array of
 * VSA_SELECT_TILING_NOALLOC_MAX_BYTES bytes that every GPU loading the
 * library holds until the process exits; a request whose scratch
 * (vsa_select_tiling_workspace_size) exceeds it returns
 * VSA_ERR_INVALID_ARGUMENT without launching anything.  The call allocates
 * nothing.  A call whose stream is not capturing looks the array's device
 * address up (cudaGetSymbolAddress, with that device current), so a context
 * that was torn down and created anew on the device is never handed an old
 * address; a call whose stream is capturing uses the address that the last
 * such call on the device found, so make one call on the device before any
 * stream capture.  All calls share the one array:
 * every scratch entry a call reads is written earlier in the same call, so
 * nothing has to start at zero, but calls whose work overlaps on the GPU
 * (different streams, or different host threads on one device) race on it
 * and must be serialised by the caller.                                   */
#define VSA_SELECT_TILING_NOALLOC_MAX_BYTES (1 << 20)
vsa_status vsa_select_tiling_noalloc(const void *q, vsa_dtype dtype, int B, int n_heads,
                                     int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles,
                                     int n_tiles, int32_t *choice, float *sics, void *stream);

/* ------------------------------------------------------------------------ */
/* Tile-contiguous permutation and its inverse.
 * "ADR-0001", step 6 (block_contiguous_permutation, invert_permutation);
 * "Adaptive tiling (SPADE)", The idea, step 2, and the Recipe (argsort of
 * tile_labels; take(..., argsort(order)) to return to T-major order).
 *
 * perm_c lists the tiles of tiling c in row-major tile order and, inside a
 * tile, its tokens in T-major order (a stable argsort of the tile labels).
 *   vsa_permute:   y[bh, p, :] = x[bh, perm_{c(bh)}[p], :]
 *   vsa_unpermute: x[bh, perm_{c(bh)}[p], :] = y[bh, p, :]
 * where c(bh) = choice[bh] (device int32 [B*n_heads]), or 0 if choice is NULL.
 * x is [B, n_heads, S, D] (T-major, S = T*Hg*Wg) and y [B, n_heads, Sp, D]
 * (Sp of vsa_padded_grid; Sp == S when the tiles divide grid), both in
 * `dtype`, not overlapping.  On a padded grid perm runs over the padded
 * grid's tokens: vsa_permute writes zero rows at padding positions and
 * vsa_unpermute ignores them.  tiles is a HOST array of n_tiles (1..8)
 * tiles; a device choice outside [0, n_tiles) sets VSA_ERR_RUNTIME and that
 * head is left unwritten.  The copy is exact (bit for bit).               */
vsa_status vsa_permute(const void *x, void *y, vsa_dtype dtype, int B, int n_heads,
                       int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles,
                       int n_tiles, const int32_t *choice, void *stream);
vsa_status vsa_unpermute(const void *y, void *x, vsa_dtype dtype, int B, int n_heads,
                         int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles,
                         int n_tiles, const int32_t *choice, void *stream);

/* ------------------------------------------------------------------------ */
/* Per-block element-wise summaries.  "Adaptive tiling (SPADE)", The idea,
 * step 3 (element-wise max/min summaries).
 *   x_max[bh, i, d] = max_{r < block} x_perm[bh, i*block + r, d], x_min likewise.
 * x_perm [B, n_heads, S, D]; x_max, x_min [B, n_heads, S/block, D], all in
 * `dtype`.  block in {16, 32, 64, 128, 256}, S % block == 0, D in {64, 128}.
 * The result is an exact selection of input values.                       */
vsa_status vsa_block_summaries(const void *x_perm, vsa_dtype dtype, int B, int n_heads,
                               int S, int D, int block, void *x_max, void *x_min,
                               void *stream);

/* The same summaries read from a T-major x, with no permuted copy: block i of
 * (b, head) covers positions [i*block, (i+1)*block) of that head's
 * tile-contiguous order under tiles[choice[bh]] (the order vsa_permute
 * writes).  The result equals vsa_permute followed by vsa_block_summaries,
 * bit for bit.
 *   x      [B, n_heads, S, D] in `dtype`, T-major (S = grid.t*grid.h*grid.w)
 *   tiles, n_tiles, choice  as for vsa_permute (choice NULL: tile 0)
 *   x_max, x_min  [B, n_heads, Sp/block, D] in `dtype` (Sp of
 *          vsa_padded_grid, a multiple of block); padding positions count
 *          as zero rows, as in the output of vsa_permute
 * A choice outside [0, n_tiles) leaves that head's summaries unwritten and
 * sets VSA_ERR_RUNTIME (read with vsa_device_status).                      */
vsa_status vsa_block_summaries_tiled(const void *x, vsa_dtype dtype, int B, int n_heads,
                                     int S, int D, vsa_dims3 grid, const vsa_dims3 *tiles,
                                     int n_tiles, const int32_t *choice, int block,
                                     void *x_max, void *x_min, void *stream);

/* ------------------------------------------------------------------------ */
/* Block scores.  "Adaptive tiling (SPADE)", The idea, step 3, and the
 * function table (minmax_block_scores).
 *   scores[bh, i, j] = max((q_max_i + q_min_i) . k_max_j, (q_max_i + q_min_i) . k_min_j)
 * unscaled, accumulated in fp32 as q_max.k + q_min.k, so every product of
 * bf16 inputs is exact; on small-integer-valued inputs the scores are exact.
 * Summaries are [B, n_heads, nb, D] in `dtype`; scores [B, n_heads, nb, nb]
 * fp32.  D in {64, 128}, 1 <= nb.                                          */
vsa_status vsa_block_scores(const void *q_max, const void *q_min, const void *k_max,
                            const void *k_min, vsa_dtype dtype, int B, int n_heads,
                            int nb, int D, float *scores, void *stream);

/* ------------------------------------------------------------------------ */
/* Top-k key blocks plus static sink and diagonal blocks, as a compact list.
 * "Adaptive tiling (SPADE)", The idea, step 4 (fixed per-row budget plus
 * static sink and diagonal blocks), function table (top_k_block_mask), the
 * Recipe (k = max(1, floor(budget * n_blocks))) and the recipe note (OR the
 * sink and diagonal blocks into the top-k mask).
 *
 * Row i of every (b, head) keeps the k highest scores (equal scores: lower
 * block index first), then adds the blocks j < n_sink_blocks and
 * |j - i| <= diag_halfwidth (diag_halfwidth = -1: none).  The kept block
 * indices are written in ascending order to idx[bh, i, 0 .. cnt[bh, i]),
 * the remaining slots get -1.
 *   scores [B, n_heads, nb, nb] fp32 (NaN not allowed; -0 equals +0)
 *   idx    [B, n_heads, nb, cap] int32,  cnt [B, n_heads, nb] int32
 * 1 <= k <= nb, 0 <= n_sink_blocks <= nb, cap >= min(nb, k + n_sink_blocks
 * + 2*diag_halfwidth + 1).  Integer output: bit-exact by construction.   */
vsa_status vsa_topk_block_mask(const float *scores, int B, int n_heads, int nb, int k,
                               int n_sink_blocks, int diag_halfwidth, int32_t *idx,
                               int32_t *cnt, int cap, void *stream);

/* vsa_block_scores followed by vsa_topk_block_mask in one kernel: the
 * scores of a row stay on the chip and are never written ("Adaptive tiling
 * (SPADE)", Dense by design: its speed comes from a fused estimator).  The
 * arguments and the lists (idx, cnt, cap) are those of the two calls; the
 * scores are the same fp32 sums of exact bf16 products, so on
 * small-integer-valued summaries the lists equal the two calls' bit for bit
 * (elsewhere fp32 rounding may order near-equal scores differently).
 * bf16 summaries only and nb <= 1024 (VSA_ERR_UNSUPPORTED otherwise); D in
 * {64, 128}.                                                              */
vsa_status vsa_block_scores_topk(const void *q_max, const void *q_min, const void *k_max,
                                 const void *k_min, vsa_dtype dtype, int B, int n_heads, int nb,
                                 int D, int k, int n_sink_blocks, int diag_halfwidth, int32_t *idx,
                                 int32_t *cnt, int cap, void *stream);

/* Top-p (mass budget) key-block lists.  "Adaptive tiling (SPADE)" names
 * top_p_block_mask among the functions its recipe composes with but does not
 * define it; this is the reading used here.  For each row (b, head, i):
 * probabilities softmax_j(scale * scores[bh, i, j]); the kept blocks are the
 * shortest prefix of the row in descending score order (equal scores: lower
 * index first) whose probabilities sum to at least p; then, as for
 * vsa_topk_block_mask, blocks j < n_sink_blocks and |j - i| <= diag_halfwidth
 * (-1: none) are ORed in, and the list is written in ascending order with
 * -1 in unused slots.
 *   scores  [B, n_heads, nb, nb] fp32 (vsa_block_scores)
 *   p       in (0, 1]; scale >= 0 (0 makes every block equally likely, so the
 *           list is the top-k list with k = ceil(p * nb))
 *   idx     [B, n_heads, nb, cap] int32 with cap >= nb; cnt [B, n_heads, nb]
 * Masses are accumulated in fp32: a block whose inclusion changes the
 * prefix mass across p by less than about 1e-6 * (row mass) may be taken or
 * left.  Rows of more than 1024 blocks return VSA_ERR_UNSUPPORTED.          */
vsa_status vsa_topp_block_mask(const float *scores, int B, int n_heads, int nb, float p, float scale,
                               int n_sink_blocks, int diag_halfwidth, int32_t *idx, int32_t *cnt, int cap,
                               void *stream);

/* ------------------------------------------------------------------------ */
/* Structured static masks as block lists.  "ADR-0001", step 1
 * (spatial_only_mask, temporal_only_mask, sliding_tile_block_mask,
 * sliding_tile_centered_mask).
 *
 * The mask is a tile neighbourhood: token i sees token j iff the coordinates
 * of their tiles differ by at most the radius along (t, h, w), clipped at the
 * grid border.  SPATIAL uses tile (1, Hg, Wg) and radius 0 (same frame);
 * TEMPORAL uses tile (T, 1, 1) and radius 0 (same (h, w)); SLIDING_TILE uses
 * the given tile and radius.  SLIDING_TILE_CENTERED keeps the window's size
 * instead of clipping it: along an axis of n tiles, query tile c sees the
 * w = min(2 r + 1, n) tiles from start min(max(c - r, 0), n - w) on, so every
 * query sees the same number of tiles and the mask is not symmetric at the
 * border (the source names this mask only; this is the reading taken).
 * `tile` and `radius` are ignored for SPATIAL and TEMPORAL.  The list is expressed in the tile-contiguous order of that
 * tile (use vsa_permute with the same tile):
 *   - tile volume a multiple of block: query block i lists every block of
 *     every neighbouring tile, ascending; *group_size_out = 0;
 *   - block a multiple of the tile volume and radius 0: query block i lists
 *     itself and a key is visible iff it lies in the query's group of
 *     tile-volume tokens; *group_size_out = tile volume.
 * idx [S/block, cap] int32 (-1 padded), cnt [S/block] int32 (the same list
 * serves every batch entry and head); group_size_out is a HOST int.       */
vsa_status vsa_structured_block_list(vsa_mask_kind kind, vsa_dims3 grid, vsa_dims3 tile,
                                     vsa_dims3 radius, int block, int32_t *idx,
                                     int32_t *cnt, int cap, int *group_size_out,
                                     void *stream);

/* ------------------------------------------------------------------------ */
/* Block-sparse attention on tcgen05 tensor cores.  "Adaptive tiling (SPADE)",
 * Recipe and recipe note (skipped blocks are dropped: the block mask is
 * expanded to tokens and softmax attention runs over the kept keys).
 *
 * For query row p of query block i = p / block (tile-contiguous order):
 *   o[p] = sum_j softmax_j(scale * q[p] . k[j]) v[j]
 * over the keys j of the blocks idx[.., i, 0 .. cnt[.., i]) that are also in
 * p's group of group_size tokens when group_size > 0.  QK^T and PV run in
 * bf16 with fp32 accumulation, the online softmax in fp32.
 *   q, k, v  [B, n_heads, S, D] bf16;  o [B, n_heads, S, D] in out_dtype
 *   idx/cnt  [B, n_heads, nb, cap] / [B, n_heads, nb] if list_per_head,
 *            else [nb, cap] / [nb] shared by every (b, head)
 *   scale    softmax scale; <= 0 selects 1/sqrt(D) (_default_scale)
 * block in {32, 64, 128}, S % block == 0, D in {64, 128}.  Each list must be
 * strictly ascending with entries in [0, nb) and 1 <= cnt <= cap; rows whose
 * list breaks this are written as zeros and set VSA_ERR_RUNTIME.  Every one
 * of the S rows is a key here: for a zero-padded grid, whose padding keys
 * must be masked, use vsa_block_sparse_attention_tiled.                   */
vsa_status vsa_block_sparse_attention(const void *q, const void *k, const void *v,
                                      void *o, vsa_dtype out_dtype, int B, int n_heads,
                                      int S, int D, int block, const int32_t *idx,
                                      const int32_t *cnt, int cap, int list_per_head,
                                      int group_size, float scale, void *stream);

/* Block-sparse attention with centroid compensation.  "Adaptive tiling
 * (SPADE)", Recipe: the attention call centroid_compensated_attention(q, k,
 * v, q_labels, k_labels, block_mask), with dropping the skipped blocks named
 * as the alternative in its recipe note.  The pages give the call and its
 * arguments only; the reading taken here: query i attends exactly to the
 * keys of the blocks its list names, and every other key block b (n_b keys)
 * takes part as one key, the mean kbar_b of its keys, with value the mean
 * vbar_b of its values and weight n_b:
 *   o_i = (sum_kept e^{s(q_i,k_t)} v_t + sum_skipped n_b e^{s(q_i,kbar_b)} vbar_b)
 *       / (sum_kept e^{s(q_i,k_t)}     + sum_skipped n_b e^{s(q_i,kbar_b)}),
 * s(q, k) = scale q . k.  Blocks are those of the tile-contiguous order
 * (labels = position / block), so a block whose keys are all equal
 * contributes exactly what it would if kept.
 *   q, k, v  [B, n_heads, S, D] bf16 (tile-contiguous order); o in out_dtype
 *   idx/cnt  block lists as for vsa_block_sparse_attention (list_per_head)
 *   block    128 (S % 128 == 0); at most 8192 blocks per head
 *   workspace DEVICE scratch of vsa_centroid_compensated_attention_workspace_size
 *            bytes, 256-byte aligned, not overlapping q, k, v or o: the centroids (as
 *            bf16 pairs hi + lo, about 16 significant bits), each row's
 *            softmax state over its kept keys and, for a bf16 output, the
 *            fp32 output of the kept keys
 * The kept keys run on the block-sparse attention kernel; a second tcgen05
 * pass attends each query tile to the centroids its list skips and merges
 * the two softmaxes exactly.  Lists are checked as for
 * vsa_block_sparse_attention (rows of an invalid list are written as zeros,
 * VSA_ERR_RUNTIME).  A bf16 output is the fp32 result rounded once.  D in
 * {64, 128}.                                                               */
size_t vsa_centroid_compensated_attention_workspace_size(int B, int n_heads, int S, int D,
                                                         vsa_dtype out_dtype);
vsa_status vsa_centroid_compensated_attention(const void *q, const void *k, const void *v, void *o,
                                              vsa_dtype out_dtype, int B, int n_heads, int S,
                                              int D, int block, const int32_t *idx,
                                              const int32_t *cnt, int cap, int list_per_head,
                                              float scale, void *workspace, size_t workspace_bytes,
                                              void *stream);

/* The same in tiled mode: q, k, v and o in T-major order over `grid`, each
 * (b, head)'s blocks those of tiles[choice[bh]] (choice NULL: tile 0), as in
 * vsa_block_sparse_attention_tiled: the result equals vsa_permute of q, k, v,
 * vsa_centroid_compensated_attention and vsa_unpermute of o, bit for bit,
 * with no permuted copies.  Every tile has one volume, a multiple of 128,
 * with tile.t divisible by volume / 128; the tiles must divide the grid (no
 * padding).  A choice out of range leaves that head unwritten and sets
 * VSA_ERR_RUNTIME.  Workspace, lists and errors as above.                     */
vsa_status vsa_centroid_compensated_attention_tiled(const void *q, const void *k, const void *v, void *o,
                                                    vsa_dtype out_dtype, int B, int n_heads, int S, int D,
                                                    vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles,
                                                    const int32_t *choice, const int32_t *idx,
                                                    const int32_t *cnt, int cap, int list_per_head,
                                                    float scale, void *workspace, size_t workspace_bytes,
                                                    void *stream);

/* Block-sparse attention on T-major q, k, v and o, with each (b, head) in its
 * own tiling and no permuted copies ("Adaptive tiling (SPADE)", Recipe: the
 * permutation, attention and inverse permutation in one pass).  Block i of
 * (b, head) is positions [128 i, 128 i + 128) of the head's tile-contiguous
 * order under tiles[choice[bh]]; idx/cnt list blocks in that numbering, as
 * vsa_topk_block_mask writes them.  The result equals vsa_permute of q, k and
 * v, vsa_block_sparse_attention with block 128 and group_size 0, then
 * vsa_unpermute of o, bit for bit, when the tiles divide the grid.  On a
 * grid they do not divide (vsa_padded_grid), positions and blocks refer to
 * the padded grid (nb = Sp/128), keys at padding positions are masked out
 * (the zero-padding recipe of "Adaptive tiling (SPADE)", Deviations and
 * notes) and only the S real rows of o are written.
 *   q, k, v  [B, n_heads, S, D] bf16, o [B, n_heads, S, D] in out_dtype, T-major
 *   tiles    every candidate of the same volume V: 32 or 64 (a block is the
 *            tile), or a multiple of 128 with tile.t divisible by V/128 (a
 *            128-token block is tile.t*128/V whole (h, w) planes of the tile);
 *            a block's box must fit inside the real grid (VSA_ERR_UNSUPPORTED
 *            otherwise).  Lists count blocks of min(V, 128) tokens.
 *   choice   [B, n_heads] int32 or NULL (tile 0 for every head)
 *   group_stride  0, or (128-token blocks only) a power of two s in [2, 128]: a key is then visible
 *            to a query only if their positions (tile-contiguous order)
 *            differ by a multiple of s.  With tile (T, 1, 128 / T) and the
 *            diagonal list this is the temporal-only mask ("ADR-0001", step 1):
 *            position t * s + w of a block holds frame t of column w.
 * Lists are checked as for vsa_block_sparse_attention; a choice outside
 * [0, n_tiles) leaves the head unwritten and sets VSA_ERR_RUNTIME.         */
vsa_status vsa_block_sparse_attention_tiled(const void *q, const void *k, const void *v,
                                            void *o, vsa_dtype out_dtype, int B,
                                            int n_heads, int S, int D, vsa_dims3 grid,
                                            const vsa_dims3 *tiles, int n_tiles,
                                            const int32_t *choice, const int32_t *idx,
                                            const int32_t *cnt, int cap, int list_per_head,
                                            int group_stride, float scale, void *stream);

/* ------------------------------------------------------------------------ */
/* Symmetric sliding-window attention with global sinks.
 * "fastvideo/mlx_runtime/windowed_attention.py": module docstring (Window
 * policy), windowed_attention, _key_ranges_for_block, _default_scale.
 *
 * Key j is visible to query i iff j < sink or |i - j| <= window / 2; when
 * window >= S every key is visible (dense attention, as the page does).
 * Work is restricted to the 128x128 tiles that meet the window or the sinks.
 *   q, k, v [B, n_heads, S, D] bf16 (any S >= 1); o in out_dtype
 *   window >= 1, 0 <= sink <= S, scale <= 0 selects 1/sqrt(D)
 *   chunk    the page's query chunk size; results do not depend on it.
 *            0 selects min(window, 512); otherwise it must be >= 1.
 * D in {64, 128}.                                                          */
vsa_status vsa_window_attention(const void *q, const void *k, const void *v, void *o,
                                vsa_dtype out_dtype, int B, int n_heads, int S, int D,
                                int window, int sink, float scale, int chunk,
                                void *stream);

/* ------------------------------------------------------------------------ */
/* Head profile: spatial or temporal pattern per head.  "ADR-0001", step 2
 * (classify_heads_from_qk, classify_heads_from_probs, classify: the profiler
 * consumes Q and K only) and "SVG implementation for LTX 2", overview (each
 * head is profiled on query tokens and given the spatial or the temporal
 * attention pattern).  The pages give the names and that purpose only; the
 * reading taken here:
 *   for each sampled query row i (T-major position rows[r]) of a (b, head),
 *   p_ij = softmax_j(scale * q_i . k_j) over all S keys;
 *   mass_spatial(i)  = sum of p_ij over the keys of i's frame
 *                      (the spatial_only mask),
 *   mass_temporal(i) = sum of p_ij over the keys at i's (h, w)
 *                      (the temporal_only mask);
 *   masses[bh] = (mean_i mass_spatial, mean_i mass_temporal);
 *   kind[bh]   = 1 (temporal) if the temporal pattern wins under `rule`,
 *                else 0 (spatial; ties too):
 *     VSA_PROFILE_MASS          the larger mean mass;
 *     VSA_PROFILE_MASS_PER_KEY  the larger mean mass per key of the pattern,
 *                               mass_spatial / (Hg Wg) against
 *                               mass_temporal / T (a frame holds many more
 *                               keys than a pixel's T frames, so raw mass
 *                               favours the spatial pattern at large frames).
 * QK^T runs on the tensor cores (bf16 inputs, fp32 accumulation); the
 * softmax sums are fp32, so masses are within about 1e-5 of exact and heads
 * whose two masses differ by less than that may take either kind.
 *   q, k      [B, n_heads, S, D] bf16, T-major over grid (T, Hg, Wg)
 *   rows      [R] int32 device array of query positions in [0, S), shared
 *             by every (b, head); 1 <= R <= 128 (the sample is an input:
 *             callers draw it).  A position out of range sets
 *             VSA_ERR_RUNTIME in the device status word (that row is
 *             profiled as a zero query).
 *   scale     softmax scale; <= 0 selects 1/sqrt(D)
 *   rule      VSA_PROFILE_MASS or VSA_PROFILE_MASS_PER_KEY (the kind only)
 *   masses    [B*n_heads, 2] fp32 output;  kind [B*n_heads] int32 output
 *   workspace device scratch of vsa_head_profile_workspace_size(...) bytes,
 *             16-byte aligned; contents need not be initialised.
 * D in {64, 128}; S < 2^30.                                                */
typedef enum { VSA_PROFILE_MASS = 0, VSA_PROFILE_MASS_PER_KEY = 1 } vsa_profile_rule;
size_t vsa_head_profile_workspace_size(int B, int n_heads, int S, int D);
vsa_status vsa_head_profile(const void *q, const void *k, int B, int n_heads, int S, int D,
                            vsa_dims3 grid, const int32_t *rows, int R, float scale,
                            vsa_profile_rule rule, float *masses, int32_t *kind, void *workspace,
                            size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* The whole SPADE path for Q, K, V and O in HOST memory.  "Adaptive tiling
 * (SPADE)", Recipe: per (b, head) the tiling choice (skipped with one
 * candidate), the tile-contiguous order, the min/max block scores, the top-k
 * lists with the sink and diagonal blocks, block-sparse attention and the
 * return to T-major order -- the composition of vsa_select_tiling,
 * vsa_block_summaries_tiled, vsa_block_scores, vsa_topk_block_mask and
 * vsa_block_sparse_attention_tiled, whose result it equals bit for bit.
 *
 * The (b, head) rows are taken in `groups` groups (at most B*n_heads).  Each
 * group's Q, K, V are copied into the workspace, its steps run on `stream`,
 * and its O is copied back, with the copies on two streams of the call's own:
 * the copies of one group overlap the kernels of another.  Host buffers
 * should be page-locked (cudaHostAlloc / cudaHostRegister); pageable memory
 * works but its copies do not overlap.
 *   q, k, v  HOST [B, n_heads, S, D] bf16, T-major over grid (S = T*Hg*Wg)
 *   o        HOST [B, n_heads, S, D] in out_dtype (VSA_BF16 or VSA_F32)
 *   tiles    HOST array of n_tiles (1..8) candidate tiles of one volume V:
 *            32 or 64 (a block is the tile) or a multiple of 128 whose blocks
 *            are whole (h, w) planes (the conditions of
 *            vsa_block_sparse_attention_tiled); grids the tiles do not divide
 *            are padded as vsa_padded_grid says
 *   topk     k key blocks per query block, 1 <= k <= nb (nb = padded tokens
 *            / block); n_sink_blocks, diag_halfwidth as for
 *            vsa_topk_block_mask; scale <= 0 selects 1/sqrt(D)
 *   workspace DEVICE scratch of vsa_spade_attention_host_workspace_size(...)
 *            bytes (same arguments), 256-byte aligned, owned by the caller
 * The call enqueues its work and returns: `stream` reaches the end of the
 * call once every copy into o has landed, so synchronise `stream` before
 * reading o, and do not reuse the workspace on another stream before then.
 * Argument errors return before any copy is issued; an error that a device
 * step reports for a group stops the call there (earlier groups' copies
 * have been issued) and is returned.  D in {64, 128}.                      */
size_t vsa_spade_attention_host_workspace_size(int B, int n_heads, int S, int D, vsa_dims3 grid,
                                               const vsa_dims3 *tiles, int n_tiles, int topk,
                                               int n_sink_blocks, int diag_halfwidth,
                                               vsa_dtype out_dtype, int groups);
vsa_status vsa_spade_attention_host(const void *q, const void *k, const void *v, void *o,
                                    vsa_dtype out_dtype, int B, int n_heads, int S, int D,
                                    vsa_dims3 grid, const vsa_dims3 *tiles, int n_tiles, int topk,
                                    int n_sink_blocks, int diag_halfwidth, float scale, int groups,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Round-to-nearest-even fp32 -> bf16 conversion of n elements (x, y device).
 * Used to feed fp32 tensors to the bf16 attention calls.                  */
vsa_status vsa_cast_f32_to_bf16(const float *x, void *y, int64_t n, void *stream);

/* Test hook for the bounded-wait machinery: launches one tiny kernel that
 * waits on an mbarrier nothing will complete, gives up after timeout_ns of
 * device time, records VSA_ERR_TIMEOUT in the device status word and
 * returns.  vsa_device_status() then reports VSA_ERR_TIMEOUT.             */
vsa_status vsa_debug_wait_timeout(int64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H */
