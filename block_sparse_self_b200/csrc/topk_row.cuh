// topk_row.cuh -- one warp's top-k list of one score row whose keys are in
// registers: the k highest scores (equal scores: lower block index first),
// then the sink blocks j < n_sink and the diagonal |j - i| <= diag_hw ORed in,
// written in ascending order ("Adaptive tiling (SPADE)", The idea, step 4,
// top_k_block_mask, and the recipe note).  Shared by the top-k kernel and the
// fused score/top-k kernel.
#pragma once

#include "common.cuh"

namespace vsa {

// Order-preserving map of a float to uint32: a larger float gives a larger
// key, and -0 the same key as +0.  Every finite score maps above 0, so 0 can
// mark an empty slot.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0u) u = 0u;              // -0 ranks equal to +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // larger float -> larger key
}

template <int NPL>
__device__ __forceinline__ int count_ge(const uint32_t (&key)[NPL], uint32_t t) {
    uint32_t c[4] = {0u, 0u, 0u, 0u};
    #pragma unroll
    for (int i = 0; i < NPL; ++i) c[i & 3] += key[i] >= t ? 1u : 0u;
    return static_cast<int>(__reduce_add_sync(0xffffffffu, (c[0] + c[1]) + (c[2] + c[3])));
}

// Once the threshold's leading bits are fixed, only the keys that share them
// (the candidates) can still move the count; when at most kTopkCand remain
// they are gathered, two per lane, and the low bits are decided on those alone.
constexpr int kTopkCand = 64;

// key[t]: order key of block lane + 32 t of row i (0 for a slot past nb).
// The k-th largest key T is found by bisection on its bits: T is the largest
// value with count(key >= T) >= k, each count a per-lane compare-and-add plus
// a warp sum.  out[0 .. cap) receives the list (-1 padded), *cnt_out its
// length; cand is a warp-private shared buffer of kTopkCand words.
template <int NPL>
__device__ __forceinline__ void topk_row(const uint32_t (&key)[NPL], int nb, int k, int i, int n_sink, int diag_hw,
                                         int32_t *out, int32_t *cnt_out, int cap, uint32_t *cand) {
    const int lane = threadIdx.x & 31;
    // bisection on the bits of T, high to low; after bit b is decided every
    // key >= T + 2^b (c_hi of them) is above T and the candidates are the
    // keys in [T, T + 2^b)
    uint32_t thr = 0u;
    int c_lo = 32 * NPL, c_hi = 0;  // count_ge(T), count_ge(T + 2^b)
    int bit = 31;
    #pragma unroll 1
    for (; bit >= 0; --bit) {
        const uint32_t cnd = thr | (1u << bit);
        const int c = count_ge<NPL>(key, cnd);
        if (c >= k) {
            thr = cnd;
            c_lo = c;
        } else {
            c_hi = c;
        }
        if (c_lo - c_hi <= kTopkCand) break;
    }
    int need;
    if (bit > 0) {
        // gather the candidates of [thr, thr + 2^bit), then decide bits bit-1 .. 0 on them
        const uint64_t top = static_cast<uint64_t>(thr) + (uint64_t{1} << bit);
        int n_c = 0;
        #pragma unroll
        for (int t = 0; t < NPL; ++t) {
            const bool in = key[t] >= thr && static_cast<uint64_t>(key[t]) < top;
            const uint32_t m = __ballot_sync(0xffffffffu, in);
            const int pos = n_c + __popc(m & ((1u << lane) - 1u));
            if (in) cand[pos] = key[t];
            n_c += __popc(m);
        }
        __syncwarp();
        const uint32_t k0 = lane < n_c ? cand[lane] : 0u;
        const uint32_t k1 = lane + 32 < n_c ? cand[lane + 32] : 0u;
        __syncwarp();  // the buffer is reused by this warp's next row
        auto count_c = [&](uint32_t t) -> int {
            return c_hi + static_cast<int>(__reduce_add_sync(0xffffffffu, (k0 >= t ? 1u : 0u) + (k1 >= t ? 1u : 0u)));
        };
        #pragma unroll 1
        for (int b2 = bit - 1; b2 >= 0; --b2) {
            const uint32_t cnd = thr | (1u << b2);
            if (count_c(cnd) >= k) thr = cnd;
        }
        need = k - (thr == 0xffffffffu ? c_hi : count_c(thr + 1u));
    } else {
        need = k - (thr == 0xffffffffu ? 0 : count_ge<NPL>(key, thr + 1u));
    }
    // thr = the k-th largest key; `need` keys equal to it are taken, lowest index first
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
    for (int p = written + lane; p < cap; p += 32) out[p] = -1;
    if (lane == 0) *cnt_out = written;
}

}  // namespace vsa
