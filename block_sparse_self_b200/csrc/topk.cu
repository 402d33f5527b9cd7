// topk.cu -- fixed-budget top-k key blocks plus sink and diagonal blocks,
// emitted as a compact ascending index list per query block.
//
// "Adaptive tiling (SPADE)", The idea, step 4 (fixed per-row budget, static
// sink and diagonal blocks), top_k_block_mask, and the recipe note (OR the
// static blocks into the top-k mask).  Equal scores rank the lower block
// index first, so the result is unique and bit-exact.
//
// One warp per row.  Scores map to order-preserving uint32 keys; a 4-pass
// 8-bit radix select finds the k-th largest key T and how many keys equal to
// T are taken (lowest indices first); a final ordered pass ranks the ties,
// ORs in the static blocks and compacts the kept indices with ballots.  Rows
// of up to 1024 blocks keep their keys in registers and find the threshold by
// bisection instead (below); longer rows use the radix select, re-reading the
// row (from L1/L2) on each pass.
#include "common.cuh"
#include "internal.h"
#include "topk_row.cuh"

namespace vsa {

namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) topk_kernel(const float *__restrict__ scores, long long rows, int nb,
                                                          int k, int n_sink, int diag_hw, int32_t *__restrict__ idx,
                                                          int32_t *__restrict__ cnt, int cap) {
    __shared__ uint32_t hist[kWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t *h = hist[warp];
    for (long long row = static_cast<long long>(blockIdx.x) * kWarps + warp; row < rows;
         row += static_cast<long long>(gridDim.x) * kWarps) {
        const float *s = scores + row * nb;
        const int i = static_cast<int>(row % nb);  // query block of this row
        uint32_t prefix = 0u, pmask = 0u;
        int need = k;  // rank of the threshold among the keys still matching the prefix
        #pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int b = lane; b < 256; b += 32) h[b] = 0u;
            __syncwarp();
            for (int j0 = 0; j0 < nb; j0 += 32) {
                const int j = j0 + lane;
                const bool in = j < nb;
                const uint32_t key = in ? order_key(__ldg(s + j)) : 0u;
                const bool match = in && (key & pmask) == prefix;
                const uint32_t digit = (key >> shift) & 255u;
                const uint32_t active = __ballot_sync(0xffffffffu, match);
                if (match) {
                    const uint32_t same = __match_any_sync(active, digit);
                    if (lane == __ffs(same) - 1) atomicAdd(&h[digit], __popc(same));
                }
            }
            __syncwarp();
            // lane L owns digits 255-8L .. 248-8L (highest digits first)
            uint32_t local[8];
            uint32_t tot = 0;
            #pragma unroll
            for (int e = 0; e < 8; ++e) {
                local[e] = h[255 - 8 * lane - e];
                tot += local[e];
            }
            uint32_t incl = tot;
            #pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const uint32_t excl = incl - tot;
            const bool mine = excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl;
            const uint32_t owner = __ballot_sync(0xffffffffu, mine);
            const int src = __ffs(owner) - 1;
            uint32_t digit = 0, above = 0;
            if (lane == src) {
                uint32_t run = excl;
                #pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (run + local[e] >= static_cast<uint32_t>(need)) {
                        digit = 255u - 8u * lane - e;
                        above = run;
                        break;
                    }
                    run += local[e];
                }
            }
            digit = __shfl_sync(0xffffffffu, digit, src);
            above = __shfl_sync(0xffffffffu, above, src);
            need -= static_cast<int>(above);
            prefix |= digit << shift;
            pmask |= 255u << shift;
            __syncwarp();
        }
        // prefix = the k-th largest key; take every larger key and the first
        // `need` keys equal to it, then OR in the static blocks.
        int32_t *out = idx + row * cap;
        int taken_eq = 0, written = 0;
        for (int j0 = 0; j0 < nb; j0 += 32) {
            const int j = j0 + lane;
            const bool in = j < nb;
            const uint32_t key = in ? order_key(__ldg(s + j)) : 0u;
            const bool eq = in && key == prefix;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rank = taken_eq + __popc(eqm & ((1u << lane) - 1u));
            const int dd = j > i ? j - i : i - j;
            const bool keep = in && (key > prefix || (eq && rank < need) || j < n_sink || dd <= diag_hw);
            const uint32_t km = __ballot_sync(0xffffffffu, keep);
            const int pos = written + __popc(km & ((1u << lane) - 1u));
            if (keep && pos < cap) out[pos] = j;
            taken_eq += __popc(eqm);
            written += __popc(km);
        }
        for (int p = written + lane; p < cap; p += 32) out[p] = -1;
        if (lane == 0) cnt[row] = written;
    }
}

// Rows of up to 32 * NPL blocks: the keys stay in registers and the list is
// made by topk_row (topk_row.cuh).
template <int NPL>
__global__ void __launch_bounds__(kWarps * 32, 4) topk_reg_kernel(const float *__restrict__ scores, long long rows,
                                                              int nb, int k, int n_sink, int diag_hw,
                                                              int32_t *__restrict__ idx, int32_t *__restrict__ cnt,
                                                              int cap) {
    __shared__ uint32_t cand_buf[kWarps][kTopkCand];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (long long row = static_cast<long long>(blockIdx.x) * kWarps + warp; row < rows;
         row += static_cast<long long>(gridDim.x) * kWarps) {
        const float *s = scores + row * nb;
        uint32_t key[NPL];  // 0 marks a slot past the row (every finite score maps above 0)
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const int j = lane + 32 * t;
            key[t] = j < nb ? order_key(__ldg(s + j)) : 0u;
        }
        topk_row<NPL>(key, nb, k, static_cast<int>(row % nb), n_sink, diag_hw, idx + row * cap, cnt + row, cap,
                      cand_buf[warp]);
    }
}

// Top-p (mass budget) lists ("Adaptive tiling (SPADE)" names top_p_block_mask
// among the functions its recipe composes with; no definition is given).  Per
// row: probabilities softmax(scale * s); the kept blocks are the shortest
// prefix in descending score order (equal scores: lower index first) whose
// mass reaches p; sink and diagonal blocks are ORed in.  With e_j =
// 2^(scale log2e (s_j - max)) and Z their sum, the threshold key T is the
// largest t with mass(key >= t) >= p Z, found by the same bisection as the
// top-k threshold with masses for counts (each a sum of non-negative terms in
// a fixed order, so monotone in t); then every key above T is kept and the
// first `need` keys equal to T, need = ceil((p Z - mass(key > T)) / e_T).
template <int NPL>
__device__ __forceinline__ float mass_ge(const uint32_t (&key)[NPL], const float (&e)[NPL], uint32_t t) {
    float m[2] = {0.f, 0.f};
    #pragma unroll
    for (int i = 0; i < NPL; ++i) m[i & 1] += key[i] >= t ? e[i] : 0.f;
    float v = m[0] + m[1];
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int NPL>
__global__ void __launch_bounds__(kWarps * 32, 1) topp_reg_kernel(const float *__restrict__ scores, long long rows,
                                                              int nb, float p, float scale_log2, int n_sink,
                                                              int diag_hw, int32_t *__restrict__ idx,
                                                              int32_t *__restrict__ cnt, int cap) {
    const int lane = threadIdx.x & 31;
    for (long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5); row < rows;
         row += static_cast<long long>(gridDim.x) * kWarps) {
        const float *s = scores + row * nb;
        const int i = static_cast<int>(row % nb);
        uint32_t key[NPL];
        float x[NPL], e[NPL];
        float mx = -INFINITY;
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const int j = lane + 32 * t;
            x[t] = j < nb ? __ldg(s + j) : -INFINITY;
            key[t] = j < nb ? order_key(x[t]) : 0u;
            mx = fmaxf(mx, x[t]);
        }
        #pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const int j = lane + 32 * t;
            e[t] = j < nb ? ex2_approx(scale_log2 * (x[t] - mx)) : 0.f;
        }
        const float target = p * mass_ge<NPL>(key, e, 0u);
        uint32_t thr = 0u;
        #pragma unroll 1
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t cand = thr | (1u << bit);
            if (mass_ge<NPL>(key, e, cand) >= target) thr = cand;
        }
        // T = thr; its probability weight (every key equal to T has the same
        // score) and how many keys share it
        float e_t = 0.f;
        int n_eq = 0;
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const bool eq = lane + 32 * t < nb && key[t] == thr;
            e_t = eq ? e[t] : e_t;
            n_eq += __popc(__ballot_sync(0xffffffffu, eq));
        }
        // non-negative floats order as their bits: the max picks the shared value
        e_t = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(e_t)));
        const float above = thr == 0xffffffffu ? 0.f : mass_ge<NPL>(key, e, thr + 1u);
        int need = e_t > 0.f ? static_cast<int>(ceilf((target - above) / e_t)) : n_eq;
        need = need < 1 ? 1 : (need > n_eq ? n_eq : need);
        int32_t *out = idx + row * cap;
        int taken_eq = 0, written = 0;
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const int j = lane + 32 * t;
            const bool in = j < nb;
            const bool eq = in && key[t] == thr;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rank = taken_eq + __popc(eqm & ((1u << lane) - 1u));
            const int dd = j > i ? j - i : i - j;
            const bool keep = in && (key[t] > thr || (eq && rank < need) || j < n_sink || dd <= diag_hw);
            const uint32_t km = __ballot_sync(0xffffffffu, keep);
            const int pos = written + __popc(km & ((1u << lane) - 1u));
            if (keep && pos < cap) out[pos] = j;
            taken_eq += __popc(eqm);
            written += __popc(km);
        }
        for (int q = written + lane; q < cap; q += 32) out[q] = -1;
        if (lane == 0) cnt[row] = written;
    }
}

}  // namespace

cudaError_t launch_topp(const float *scores, int BH, int nb, float p, float scale, int n_sink, int diag_hw,
                        int32_t *idx, int32_t *cnt, int cap, cudaStream_t st) {
    const long long rows = static_cast<long long>(BH) * nb;
    long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    const int grid = static_cast<int>(blocks);
    const int npl = (nb + 31) / 32;
    const float sl2 = scale * 1.4426950408889634f;
#define VSA_TOPP_REG(N) topp_reg_kernel<N><<<grid, kWarps * 32, 0, st>>>(scores, rows, nb, p, sl2, n_sink, diag_hw, idx, cnt, cap)
    if (npl <= 1) VSA_TOPP_REG(1);
    else if (npl <= 2) VSA_TOPP_REG(2);
    else if (npl <= 4) VSA_TOPP_REG(4);
    else if (npl <= 8) VSA_TOPP_REG(8);
    else if (npl <= 16) VSA_TOPP_REG(16);
    else if (npl <= 30) VSA_TOPP_REG(30);
    else if (npl <= 32) VSA_TOPP_REG(32);
    else return cudaErrorInvalidValue;
#undef VSA_TOPP_REG
    return cudaGetLastError();
}

cudaError_t launch_topk(const float *scores, int BH, int nb, int k, int n_sink, int diag_hw, int32_t *idx,
                        int32_t *cnt, int cap, cudaStream_t st) {
    const long long rows = static_cast<long long>(BH) * nb;
    long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    const int grid = static_cast<int>(blocks);
    const int npl = (nb + 31) / 32;
    // every counting pass costs a compare per slot, so the slot count follows
    // the row closely (960 blocks: 30 slots, 11 % faster than 32)
#define VSA_TOPK_REG(N) topk_reg_kernel<N><<<grid, kWarps * 32, 0, st>>>(scores, rows, nb, k, n_sink, diag_hw, idx, cnt, cap)
    if (npl <= 1) VSA_TOPK_REG(1);
    else if (npl <= 2) VSA_TOPK_REG(2);
    else if (npl <= 4) VSA_TOPK_REG(4);
    else if (npl <= 6) VSA_TOPK_REG(6);
    else if (npl <= 8) VSA_TOPK_REG(8);
    else if (npl <= 12) VSA_TOPK_REG(12);
    else if (npl <= 16) VSA_TOPK_REG(16);
    else if (npl <= 20) VSA_TOPK_REG(20);
    else if (npl <= 28) VSA_TOPK_REG(28);
    else if (npl <= 30) VSA_TOPK_REG(30);
    else if (npl <= 32) VSA_TOPK_REG(32);
    else topk_kernel<<<grid, kWarps * 32, 0, st>>>(scores, rows, nb, k, n_sink, diag_hw, idx, cnt, cap);
#undef VSA_TOPK_REG
    return cudaGetLastError();
}

}  // namespace vsa
