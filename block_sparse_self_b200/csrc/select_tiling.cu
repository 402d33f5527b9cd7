// select_tiling.cu -- per-(batch, head) choice of the most cohesive tiling.
//
// "Adaptive tiling (SPADE)", The idea, step 1 and select_tiling /
// block_self_similarity: the cohesion of a tiling is the mean over its tiles
// of the tile's SICS, the mean cosine over distinct pairs of its non-zero
// queries, (|sum of unit queries|^2 - m) / (m (m - 1)); the choice is the
// most cohesive candidate, ties to the lower index.
//
// Q is read once for all candidates.  The grid is cut into regions of the
// per-axis lcm of the candidate tiles (every candidate tiles a region
// exactly) and each region into cells of the per-axis gcd (every tile is a
// union of cells).  Pass 1: one CTA per (region, bh) normalises each query
// once, sums unit vectors per cell, then per candidate tile sums its cells
// and turns the norm into the tile's SICS; it writes per-candidate sums of
// tile SICS for its region.  Pass 2: one warp per bh adds the regions in a
// fixed order, divides by the tile count and takes the argmax.
//
// A grid the candidates do not divide is zero-padded per axis to a multiple of
// the region ("Adaptive tiling (SPADE)", Deviations and notes).  Padding
// tokens have zero norm, so they are never loaded: cells past the real grid
// are skipped and cells across its edge test each token.  The mean is taken
// over the tiles that hold at least one non-zero query, so every region
// reports its SICS sum and the number of such tiles.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

// acc_lo += lo * lo, acc_hi += hi * hi for the two bf16 halves of pk: sm_100
// mixed-precision FMAs (the product of two bf16 values is exact in fp32, so
// each is one rounding, as an fp32 FMA on the widened values would give).
__device__ __forceinline__ void sq_bf16x2_f32(uint32_t pk, float &acc_lo, float &acc_hi) {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "fma.rn.f32.bf16 %0, lo, lo, %0;\n\tfma.rn.f32.bf16 %1, hi, hi, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi)
        : "r"(pk));
}

// 16 bytes from global memory read once: no L1 allocation, and the L2 fetches
// the whole 256-byte line around it (a token row of D = 128 bf16 values).
__device__ __forceinline__ uint4 ld_stream_l2_256(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCells = 256;

int gcd(int a, int b) { return b == 0 ? a : gcd(b, a % b); }
int lcm(int a, int b) { return a / gcd(a, b) * b; }

struct SelArgs {
    const uint8_t *q;
    int S, T, H, W, D, esize;  // S = T * H * W real tokens per head
    TileSet tiles;
    int Rt, Rh, Rw, Ct, Ch, Cw;
    int nrt, nrh, nrw;  // regions per axis of the padded grid
    int cells, items;
    FastDiv cell_hw, cell_w;  // Ch * Cw and Cw: token of a cell -> (dt, dh, dw)
    FastDiv reg_hw, reg_w;    // nrh * nrw and nrw: region -> (rt, rh, rw)
    FastDiv cel_hw, cel_w;    // nch * ncw and ncw: cell -> (ct, ch, cw)
    int nch, ncw;             // cells of a region along h and w
    int tpr_t[kMaxTiles], tpr_h[kMaxTiles], tpr_w[kMaxTiles];  // candidate c: its tiles per region axis
    int cpt_t[kMaxTiles], cpt_h[kMaxTiles], cpt_w[kMaxTiles];  // candidate c: cells per tile axis
    int item_first[kMaxTiles + 1];                             // candidate c's first item in a region
    float *partial;     // [BH][n_regions][2][tiles.n]: SICS sums, then counts of tiles with a query
};

// Candidate tiles inside one region, candidate by candidate (the same item
// layout in every region, precomputed on the host): warp w takes items w,
// w + kWarps, ...; it sums the tile's cells, four channels per lane, and turns
// |sum|^2 into the tile's SICS.  cell_sum is [cells][D], cell_cnt [cells].
__device__ void region_tile_pass(const SelArgs &a, const float *cell_sum, const float *cell_cnt, float *tile_val,
                                 float *tile_used, int warp, int lane) {
    int item = 0;
    for (int c = 0; c < a.tiles.n; ++c) {
        const int kt = a.cpt_t[c], kh = a.cpt_h[c], kw = a.cpt_w[c];
        for (int at = 0; at < a.tpr_t[c]; ++at)
            for (int ah = 0; ah < a.tpr_h[c]; ++ah)
                for (int aw = 0; aw < a.tpr_w[c]; ++aw, ++item) {
                    if (item % kWarps != warp) continue;  // warp-uniform
                    float sq = 0.f, m = 0.f;
                    for (int d4 = lane; d4 < a.D / 4; d4 += 32) {
                        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int x = 0; x < kt; ++x)
                            for (int y = 0; y < kh; ++y) {
                                const int row = ((at * kt + x) * a.nch + ah * kh + y) * a.ncw + aw * kw;
                                for (int z = 0; z < kw; ++z) {
                                    const float4 v = reinterpret_cast<const float4 *>(cell_sum + (row + z) * a.D)[d4];
                                    sum.x += v.x;
                                    sum.y += v.y;
                                    sum.z += v.z;
                                    sum.w += v.w;
                                }
                            }
                        sq = fmaf(sum.x, sum.x, sq);
                        sq = fmaf(sum.y, sum.y, sq);
                        sq = fmaf(sum.z, sum.z, sq);
                        sq = fmaf(sum.w, sum.w, sq);
                    }
                    for (int x = 0; x < kt; ++x)
                        for (int y = 0; y < kh; ++y) {
                            const int row = ((at * kt + x) * a.nch + ah * kh + y) * a.ncw + aw * kw;
                            for (int z = 0; z < kw; ++z) m += cell_cnt[row + z];
                        }
                    #pragma unroll
                    for (int off = 16; off > 0; off >>= 1) sq += __shfl_down_sync(0xffffffffu, sq, off);
                    if (lane == 0) {
                        tile_val[item] = m >= 2.f ? (sq - m) / (m * (m - 1.f)) : 0.f;
                        tile_used[item] = m >= 1.f ? 1.f : 0.f;
                    }
                }
    }
}

// Candidate c's sum of tile SICS over this region and its count of tiles that
// hold a non-zero query, into the [BH][n_regions][2][n_tiles] partials.
__device__ void region_write(const SelArgs &a, const float *tile_val, const float *tile_used, int region, int bh,
                             int c) {
    const int first = a.item_first[c], n = a.item_first[c + 1] - first;
    float s = 0.f, used = 0.f;
    for (int i = 0; i < n; ++i) {
        s += tile_val[first + i];
        used += tile_used[first + i];
    }
    const int n_regions = a.nrt * a.nrh * a.nrw;
    float *out = a.partial + (static_cast<size_t>(bh) * n_regions + region) * 2 * a.tiles.n;
    out[c] = s;
    out[a.tiles.n + c] = used;
}

// LPT lanes share a query row; each lane takes CPL of the row's 16-byte chunks,
// chunk lt + LPT u (lt = lane % LPT), so one load instruction reads LPT
// consecutive chunks of every row it touches.  Four CTAs per SM (64
// registers, a few bytes spilled outside the token loop) measured 5 % faster
// than three at 80 registers.
template <typename T, int LPT, int CPL>
__global__ void __launch_bounds__(kThreads, 4) sics_partial_kernel(const SelArgs a) {
    constexpr int EPC = 16 / sizeof(T);  // elements per chunk
    constexpr int EPL = EPC * CPL;       // elements per lane
    constexpr int TPI = 32 / LPT;        // query rows per warp pass
    constexpr int CPR = LPT * CPL;       // 16-byte chunks per query row
    extern __shared__ float sm[];
    float *cell_sum = sm;                               // [cells][D]
    float *cell_cnt = cell_sum + a.cells * a.D;         // [cells]
    float *tile_val = cell_cnt + a.cells;               // [items]
    float *tile_used = tile_val + a.items;              // [items]: 1 if the tile holds a non-zero query
    int *cell_off = reinterpret_cast<int *>(tile_used + a.items);  // [cvol]: token offset inside a cell
    const int region = blockIdx.x, bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lt = lane % LPT;
    // multiply-shift divisions: a runtime division per coordinate cost about 5 %
    const int rt = static_cast<int>(fdiv(static_cast<uint32_t>(region), a.reg_hw));
    const int r_hw = region - rt * static_cast<int>(a.reg_hw.d);
    const int rh = static_cast<int>(fdiv(static_cast<uint32_t>(r_hw), a.reg_w)), rw = r_hw - rh * a.nrw;
    const int t0 = rt * a.Rt, h0 = rh * a.Rh, w0 = rw * a.Rw;
    const int cvol = a.Ct * a.Ch * a.Cw;
    const size_t head = static_cast<size_t>(bh) * a.S;
    // every cell has the same shape: offsets of its tokens from its first one, once per CTA
    for (int tk = threadIdx.x; tk < cvol; tk += kThreads) {
        const int dt = static_cast<int>(fdiv(static_cast<uint32_t>(tk), a.cell_hw));
        const int r2 = tk - dt * (a.Ch * a.Cw);
        const int dh = static_cast<int>(fdiv(static_cast<uint32_t>(r2), a.cell_w)), dw = r2 - dh * a.Cw;
        cell_off[tk] = (dt * a.H + dh) * a.W + dw;
    }
    __syncthreads();
    const uint4 *q4 = reinterpret_cast<const uint4 *>(a.q);

    for (int cell = warp; cell < a.cells; cell += kWarps) {
        const int ct = static_cast<int>(fdiv(static_cast<uint32_t>(cell), a.cel_hw));
        const int c_hw = cell - ct * static_cast<int>(a.cel_hw.d);
        const int ch = static_cast<int>(fdiv(static_cast<uint32_t>(c_hw), a.cel_w)), cw = c_hw - ch * a.ncw;
        const int tb = t0 + ct * a.Ct, hb = h0 + ch * a.Ch, wb = w0 + cw * a.Cw;
        // padded grids: a cell wholly past the real grid holds only zero tokens
        // (no loads), one across its edge tests each token (warp-uniform flags)
        const bool outside = tb >= a.T || hb >= a.H || wb >= a.W;
        const bool interior = tb + a.Ct <= a.T && hb + a.Ch <= a.H && wb + a.Cw <= a.W;
        const int n_tok = outside ? 0 : cvol;
        float acc[EPL];
        #pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        float m = 0.f;
        // chunk lt of the cell's first token; each token adds cell_off * CPR chunks
        const uint4 *cell_q = q4 + (head + static_cast<size_t>((tb * a.H + hb) * a.W + wb)) * CPR + lt;
        // NB passes' loads are issued before any of them is used
        constexpr int NB = sizeof(T) == 2 ? 4 : 2;
        #pragma unroll 1
        for (int tok_b = 0; tok_b < n_tok; tok_b += NB * TPI) {  // uniform trip count: shuffles below
            uint4 raw[NB][CPL];
            #pragma unroll
            for (int pb = 0; pb < NB; ++pb) {
                const int tok = tok_b + pb * TPI + lane / LPT;
                bool valid = tok < cvol;
                if (!interior && valid) {
                    const int dt = static_cast<int>(fdiv(static_cast<uint32_t>(tok), a.cell_hw));
                    const int r2 = tok - dt * (a.Ch * a.Cw);
                    const int dh = static_cast<int>(fdiv(static_cast<uint32_t>(r2), a.cell_w)), dw = r2 - dh * a.Cw;
                    valid = tb + dt < a.T && hb + dh < a.H && wb + dw < a.W;
                }
                const uint4 *row = cell_q + static_cast<size_t>(cell_off[valid ? tok : 0]) * CPR;
                #pragma unroll
                for (int u = 0; u < CPL; ++u)
                    raw[pb][u] = valid ? ld_stream_l2_256(row + LPT * u) : make_uint4(0u, 0u, 0u, 0u);
            }
            #pragma unroll
            for (int pb = 0; pb < NB; ++pb) {
                float x[EPL];
                #pragma unroll
                for (int u = 0; u < CPL; ++u) {
                    if constexpr (sizeof(T) == 2) {
                        // bf16 -> fp32 is the bf16 bits in the high half of the word
                        const uint32_t w[4] = {raw[pb][u].x, raw[pb][u].y, raw[pb][u].z, raw[pb][u].w};
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            x[u * EPC + 2 * e] = __uint_as_float(w[e] << 16);
                            x[u * EPC + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                        }
                    } else {
                        const float *fv = reinterpret_cast<const float *>(&raw[pb][u]);
                        #pragma unroll
                        for (int e = 0; e < EPC; ++e) x[u * EPC + e] = fv[e];
                    }
                }
                // the sum of squares in two interleaved partial sums; bf16
                // rows square their packed pairs with mixed-precision FMAs, so
                // the norm does not wait for the unpacking (2 % faster)
                float ss_lo = 0.f, ss_hi = 0.f;
                if constexpr (sizeof(T) == 2) {
                    #pragma unroll
                    for (int u = 0; u < CPL; ++u) {
                        sq_bf16x2_f32(raw[pb][u].x, ss_lo, ss_hi);
                        sq_bf16x2_f32(raw[pb][u].y, ss_lo, ss_hi);
                        sq_bf16x2_f32(raw[pb][u].z, ss_lo, ss_hi);
                        sq_bf16x2_f32(raw[pb][u].w, ss_lo, ss_hi);
                    }
                } else {
                    uint64_t ss2 = f32x2(0.f, 0.f);
                    #pragma unroll
                    for (int e = 0; e < EPL / 2; ++e) {
                        const uint64_t xe = f32x2(x[2 * e], x[2 * e + 1]);
                        ss2 = fma_f32x2(xe, xe, ss2);
                    }
                    f32x2_split(ss2, ss_lo, ss_hi);
                }
                float ss = ss_lo + ss_hi;
                #pragma unroll
                for (int off = LPT / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                if (ss > 0.f) {
                    const float inv = rsqrtf(ss);
                    const uint64_t inv2 = f32x2(inv, inv);
                    #pragma unroll
                    for (int e = 0; e < EPL / 2; ++e)
                        f32x2_split(fma_f32x2(f32x2(x[2 * e], x[2 * e + 1]), inv2, f32x2(acc[2 * e], acc[2 * e + 1])),
                                    acc[2 * e], acc[2 * e + 1]);
                    m += 1.f;
                }
            }
        }
        // add the rows of the warp's token slots (lanes with the same lt)
        #pragma unroll
        for (int off = LPT; off < 32; off <<= 1) {
            #pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
            m += __shfl_xor_sync(0xffffffffu, m, off);
        }
        if (lane < LPT) {
            #pragma unroll
            for (int u = 0; u < CPL; ++u)
                #pragma unroll
                for (int e = 0; e < EPC; ++e) cell_sum[cell * a.D + (lane + LPT * u) * EPC + e] = acc[u * EPC + e];
        }
        if (lane == 0) cell_cnt[cell] = m;
    }
    __syncthreads();

    region_tile_pass(a, cell_sum, cell_cnt, tile_val, tile_used, warp, lane);
    __syncthreads();
    if (threadIdx.x < a.tiles.n) region_write(a, tile_val, tile_used, region, bh, threadIdx.x);
}

struct FinalArgs {
    const float *partial;
    int BH, n_regions, n_tiles;
    int32_t *choice;
    float *sics;
};

__global__ void sics_final_kernel(const FinalArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * (blockDim.x / 32) + warp;
    if (bh >= a.BH) return;
    float best = 0.f;
    int best_c = 0;
    for (int c = 0; c < a.n_tiles; ++c) {
        float s = 0.f, used = 0.f;  // tile counts are exact in fp32 (far below 2^24)
        for (int r = lane; r < a.n_regions; r += 32) {
            const float *p = a.partial + (static_cast<size_t>(bh) * a.n_regions + r) * 2 * a.n_tiles;
            s += p[c];
            used += p[a.n_tiles + c];
        }
        #pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            s += __shfl_down_sync(0xffffffffu, s, off);
            used += __shfl_down_sync(0xffffffffu, used, off);
        }
        s = __shfl_sync(0xffffffffu, s, 0);
        used = __shfl_sync(0xffffffffu, used, 0);
        const float mean = used > 0.f ? s / used : 0.f;
        if (c == 0 || mean > best) {
            best = mean;
            best_c = c;
        }
        if (lane == 0 && a.sics) a.sics[static_cast<size_t>(bh) * a.n_tiles + c] = mean;
    }
    if (lane == 0) a.choice[bh] = best_c;
}

cudaError_t launch_sics_final(const float *partial, int BH, int n_regions, int n_tiles, int32_t *choice, float *sics,
                              cudaStream_t st) {
    FinalArgs f;
    f.partial = partial;
    f.BH = BH;
    f.n_regions = n_regions;
    f.n_tiles = n_tiles;
    f.choice = choice;
    f.sics = sics;
    sics_final_kernel<<<(BH + 7) / 8, 256, 0, st>>>(f);
    return cudaGetLastError();
}

}  // namespace

bool select_geometry(int Tp, int Hp, int Wp, const TileSet &tiles, SelectGeom *g) {
    int Rt = 1, Rh = 1, Rw = 1, Ct = tiles.t[0], Ch = tiles.h[0], Cw = tiles.w[0];
    for (int c = 0; c < tiles.n; ++c) {
        Rt = lcm(Rt, tiles.t[c]);
        Rh = lcm(Rh, tiles.h[c]);
        Rw = lcm(Rw, tiles.w[c]);
        Ct = gcd(Ct, tiles.t[c]);
        Ch = gcd(Ch, tiles.h[c]);
        Cw = gcd(Cw, tiles.w[c]);
    }
    g->Rt = Rt; g->Rh = Rh; g->Rw = Rw;
    g->Ct = Ct; g->Ch = Ch; g->Cw = Cw;
    if (Tp % Rt || Hp % Rh || Wp % Rw) return false;
    g->n_regions = (Tp / Rt) * (Hp / Rh) * (Wp / Rw);
    g->cells = (Rt / Ct) * (Rh / Ch) * (Rw / Cw);
    return g->cells <= kMaxCells;
}

cudaError_t launch_select_tiling(const void *q, int esize, int BH, int D, int T, int H, int W, int Tp, int Hp, int Wp,
                                 const TileSet &tiles, const SelectGeom &g, int32_t *choice, float *sics,
                                 float *partial, int *status, cudaStream_t st) {
    (void)status;
    SelArgs a;
    a.q = static_cast<const uint8_t *>(q);
    a.S = T * H * W; a.T = T; a.H = H; a.W = W; a.D = D; a.esize = esize;
    a.tiles = tiles;
    a.Rt = g.Rt; a.Rh = g.Rh; a.Rw = g.Rw;
    a.Ct = g.Ct; a.Ch = g.Ch; a.Cw = g.Cw;
    a.nrt = Tp / g.Rt; a.nrh = Hp / g.Rh; a.nrw = Wp / g.Rw;
    a.cells = g.cells;
    a.cell_hw = make_fastdiv(static_cast<uint32_t>(g.Ch * g.Cw));
    a.cell_w = make_fastdiv(static_cast<uint32_t>(g.Cw));
    a.partial = partial;
    int items = 0;
    for (int c = 0; c < tiles.n; ++c)
        items += (g.Rt / tiles.t[c]) * (g.Rh / tiles.h[c]) * (g.Rw / tiles.w[c]);
    a.items = items;
    a.nch = g.Rh / g.Ch;
    a.ncw = g.Rw / g.Cw;
    a.reg_hw = make_fastdiv(static_cast<uint32_t>(a.nrh * a.nrw));
    a.reg_w = make_fastdiv(static_cast<uint32_t>(a.nrw));
    a.cel_hw = make_fastdiv(static_cast<uint32_t>(a.nch * a.ncw));
    a.cel_w = make_fastdiv(static_cast<uint32_t>(a.ncw));
    a.item_first[0] = 0;
    for (int c = 0; c < kMaxTiles; ++c) {
        const bool on = c < tiles.n;
        a.tpr_t[c] = on ? g.Rt / tiles.t[c] : 0;
        a.tpr_h[c] = on ? g.Rh / tiles.h[c] : 0;
        a.tpr_w[c] = on ? g.Rw / tiles.w[c] : 0;
        a.cpt_t[c] = on ? tiles.t[c] / g.Ct : 0;
        a.cpt_h[c] = on ? tiles.h[c] / g.Ch : 0;
        a.cpt_w[c] = on ? tiles.w[c] / g.Cw : 0;
        a.item_first[c + 1] = a.item_first[c] + a.tpr_t[c] * a.tpr_h[c] * a.tpr_w[c];
    }
    cudaError_t e = cudaSuccess;
    const size_t cvol = static_cast<size_t>(g.Ct) * g.Ch * g.Cw;
    const size_t smem = (static_cast<size_t>(g.cells) * D + g.cells + 2 * items) * sizeof(float) + cvol * sizeof(int);
    dim3 grid(g.n_regions, BH);
    const int lpt = D * esize / 16;
#define VSA_SICS_LAUNCH(TYPE, L, C)                                                                           \
    do {                                                                                                      \
        e = cudaFuncSetAttribute(sics_partial_kernel<TYPE, L, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                 static_cast<int>(smem));                                                     \
        if (e != cudaSuccess) return e;                                                                       \
        sics_partial_kernel<TYPE, L, C><<<grid, kThreads, smem, st>>>(a);                                     \
    } while (0)
    // chunks per row = lpt (bf16 D=64: 8, bf16 D=128 and fp32 D=64: 16, fp32 D=128: 32);
    // two chunks per lane measured fastest (bf16 D=128: 8 x 2 ahead of 16 x 1 and 4 x 4)
    if (esize == 2) {
        if (lpt == 8) VSA_SICS_LAUNCH(__nv_bfloat16, 4, 2);
        else VSA_SICS_LAUNCH(__nv_bfloat16, 8, 2);
    } else {
        if (lpt == 16) VSA_SICS_LAUNCH(float, 8, 2);
        else VSA_SICS_LAUNCH(float, 16, 2);
    }
#undef VSA_SICS_LAUNCH
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_sics_final(partial, BH, g.n_regions, tiles.n, choice, sics, st);
}

}  // namespace vsa

// ---------------------------------------------------------------------------
// Scratch for vsa_select_tiling_noalloc: a file-scope device array, so that
// callers who cannot allocate device memory need not pass a workspace.  Every
// GPU that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kStaticScratchBytes = VSA_SELECT_TILING_NOALLOC_MAX_BYTES;
static __device__ __align__(256) float g_select_scratch[kStaticScratchBytes / sizeof(float)];
}  // namespace

namespace vsa {

// Device address of g_select_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, by cached_symbol_address.
namespace {
cudaError_t select_scratch_lookup(void **p) { return cudaGetSymbolAddress(p, g_select_scratch); }
}  // namespace

vsa_status select_static_scratch(float **ptr, size_t *bytes, cudaStream_t st) {
    static SymbolCache cache;
    void *p = nullptr;
    const vsa_status s = cached_symbol_address(cache, st, select_scratch_lookup, &p);
    if (s != VSA_OK) return s;
    *ptr = static_cast<float *>(p);
    *bytes = kStaticScratchBytes;
    return VSA_OK;
}

}  // namespace vsa

