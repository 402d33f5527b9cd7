// profile.cu -- per-head spatial/temporal attention mass on sampled queries.
//
// "ADR-0001: Sparse-attention roadmap for video DiTs", step 2 (the head
// profiler: classify_heads_from_qk / classify_heads_from_probs / classify,
// consuming Q and K only) and "SVG implementation for LTX 2", overview (each
// head is profiled on query tokens and given the spatial or the temporal
// pattern).  For sampled query rows i of a head, with p_ij =
// softmax_j(scale q_i . k_j) over all S keys:
//   mass_spatial(i)  = sum of p_ij over the keys of i's frame,
//   mass_temporal(i) = sum of p_ij over the keys at i's (h, w),
// averaged over the sampled rows; the head's kind is the pattern with the
// larger mean mass (ties: spatial).
//
// Three launches:
//   1. gather: the sampled rows of each (b, head) into one 128-row bf16 tile;
//   2. profile (tcgen05): each CTA streams a run of 128-key tiles of one head
//      through TMA, one thread issues S = Q_s K^T into TMEM (three 128-column
//      accumulators, so the MMAs of the next tiles overlap the reads of this
//      one), and sixteen warps (four per TMEM lane quadrant, 32 columns each)
//      keep for their row an online max and two exponential sums -- all
//      keys, the frame's keys -- written as one partial per (column quarter,
//      CTA).  The sums are latency bound per warp, so four warps share each
//      sub-partition;
//      meanwhile one more warp takes the logits of the T keys at each sampled
//      row's (h, w) directly (T x D products) for the temporal sum;
//   3. finish: partials combined per row, masses averaged per head, kind.
// The kernel reads K once (HBM bound for 128 sampled rows: 2 x 128 flops per
// key element against 2 bytes).
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

template <int D>
struct PrCfg {
    static constexpr int KSLABS = D / 64;
    static constexpr int SLAB = 128 * 128;         // 128 rows x 64 bf16 (128 bytes, swizzled)
    static constexpr int TILE = SLAB * KSLABS;     // one 128-row tile of Q samples or keys
    static constexpr int NSTAGE = D == 128 ? 4 : 8;  // key tiles in flight
    static constexpr int SMEM = 1024 + (1 + NSTAGE) * TILE + 256;
};

constexpr int kPrSumWarps = 16;  // thread = sampled row, a quarter of each tile's columns
constexpr int kPrCols = 128 / (kPrSumWarps / 4);
// + warp 16: TMA loads and MMAs; warp 17: the logits of the keys at each
// sampled row's (h, w), taken directly (testing every key for that pattern in
// the sums cost a fifth of the kernel's time)
constexpr int kPrThreads = 32 * (kPrSumWarps + 2);
// 128-column fp32 accumulators in tensor memory: the MMAs run up to two tiles
// ahead of the sums
constexpr int kPrAcc = 3;
constexpr int kPrTmemCols = 512;

struct PrArgs {
    int S, HW;                 // keys per head; tokens per frame
    int R;                     // sampled rows (<= 128)
    int tiles_per_cta, nparts;
    float cf;                  // scale * log2(e)
    const int32_t *rows;       // [R] T-major query positions
    const __nv_bfloat16 *qs;   // [BH][128][D] gathered sample rows
    const __nv_bfloat16 *k;    // [BH][S][D]
    float2 *tpart;             // [BH][128]: (max, sum) over the row's (h, w) keys, base-2 domain
    float4 *partial;           // [BH][nparts][128]: (max, sum, frame sum, unused), base-2 domain
    int *status;
};

__global__ void gather_rows_kernel(const __nv_bfloat16 *__restrict__ q, int S, int D, const int32_t *__restrict__ rows,
                                   int R, __nv_bfloat16 *__restrict__ qs, int *status) {
    const int bh = blockIdx.x;
    const int vpr = D / 8;  // 16-byte vectors per row
    const uint4 *src = reinterpret_cast<const uint4 *>(q + static_cast<size_t>(bh) * S * D);
    uint4 *dst = reinterpret_cast<uint4 *>(qs + static_cast<size_t>(bh) * 128 * D);
    for (int e = threadIdx.x; e < 128 * vpr; e += blockDim.x) {
        const int r = e / vpr, c = e - r * vpr;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < R) {
            const int p = rows[r];
            if (p >= 0 && p < S)
                v = src[static_cast<size_t>(p) * vpr + c];
            else if (c == 0)
                report(status, DEV_RUNTIME);
        }
        dst[e] = v;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// q . k for two bf16 rows of D elements, fp32 accumulation.
template <int D>
__device__ __forceinline__ float dot_bf16(const uint4 *__restrict__ a, const uint4 *__restrict__ b) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll 4
    for (int c = 0; c < D / 8; ++c) {
        const uint4 x = a[c], y = b[c];
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xs[i]));
            const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ys[i]));
            acc[i] = fmaf(xf.x, yf.x, acc[i]);
            acc[i] = fmaf(xf.y, yf.y, acc[i]);
        }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// One warp's W logits x of a key tile (keys jc .. jc+W-1, the first nvalid
// of them real) folded into its row's running maximum m (base 2) and sums:
// l over all keys, lsp over the keys of the frame [f0, f0 + HW).  A chunk
// wholly inside the frame adds its whole sum; only a chunk that a frame edge
// cuts (none when HW is a multiple of W) sums its probabilities again over
// the part inside.
template <int W, bool MASKED>
__device__ __forceinline__ void profile_chunk(const uint32_t (&x)[W], int jc, int nvalid, float cf, int HW, int f0,
                                              float &m, float &l, float &lsp) {
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll
    for (int e = 0; e < W; ++e)
        if (!MASKED || e < nvalid) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(x[e]));
    // cf > 0, so the largest logit gives the largest scaled logit
    const float mn = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * cf);
    if (mn > m) {  // rescale the sums to the new maximum (the first chunk scales zeros)
        const float f = ex2_approx(m - mn);
        l *= f;
        lsp *= f;
        m = mn;
    }
    float p[W];
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
    for (int e = 0; e < W; ++e) {
        p[e] = ex2_approx(fmaf(__uint_as_float(x[e]), cf, -m));
        if (MASKED && e >= nvalid) p[e] = 0.f;
        s4[e & 3] += p[e];
    }
    const float cs = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    l += cs;
    const int lo = f0 - jc, hi = lo + HW;  // the frame covers the chunk's entries [lo, hi)
    if (lo <= 0 && hi >= W) {
        lsp += cs;
    } else if (lo < W && hi > 0) {
        float ps = 0.f;
        #pragma unroll
        for (int e = 0; e < W; ++e) ps += (e >= lo && e < hi) ? p[e] : 0.f;
        lsp += ps;
    }
}

template <int D>
__global__ void __launch_bounds__(kPrThreads, 1)
profile_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, PrArgs a) {
    using C = PrCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sK = base + C::TILE;  // [NSTAGE][TILE]
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sK + C::NSTAGE * C::TILE);
    uint64_t *k_full = q_full + 1;              // [NSTAGE]
    uint64_t *k_empty = k_full + C::NSTAGE;     // [NSTAGE]
    uint64_t *acc_full = k_empty + C::NSTAGE;   // [kPrAcc]
    uint64_t *acc_empty = acc_full + kPrAcc;    // [kPrAcc]
    uint64_t *mma_done = acc_empty + kPrAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int n_kt = (a.S + 127) / 128;
    const int kt0 = blockIdx.x * a.tiles_per_cta;
    const int n = max(0, min(kt0 + a.tiles_per_cta, n_kt) - kt0);  // key tiles of this CTA

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kPrAcc; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], kPrSumWarps);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kPrSumWarps) {
        tmem_alloc(tmem_slot, kPrTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kPrSumWarps) {
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tmK);
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
            const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
            constexpr uint64_t kTile16 = C::TILE >> 4;
            auto load_k = [&](int u) {
                const int s = u % C::NSTAGE;
                mbar_arrive_expect_tx(&k_full[s], C::TILE);
                for (int sl = 0; sl < C::KSLABS; ++sl)
                    tma_load_3d(sK + s * C::TILE + sl * C::SLAB, &tmK, &k_full[s], sl * 64, (kt0 + u) * 128, bh);
            };
            mbar_arrive_expect_tx(q_full, C::TILE);
            for (int sl = 0; sl < C::KSLABS; ++sl) tma_load_3d(sQ + sl * C::SLAB, &tmQ, q_full, sl * 64, 0, bh);
            const int pre = min(n, C::NSTAGE);
            for (int u = 0; u < pre; ++u) load_k(u);
            int loaded = pre;  // key tiles issued
            bool ok = mbar_wait(q_full, 0, abort_flag);
            for (int u = 0; ok && u < n; ++u) {
                // refill the slot of tile u - 1 once its MMAs (its only reader) are done
                if (u >= 1 && u - 1 + C::NSTAGE < n) {
                    const int sp = (u - 1) % C::NSTAGE;
                    if (!mbar_wait(&k_empty[sp], ((u - 1) / C::NSTAGE) & 1, abort_flag)) { ok = false; break; }
                    load_k(u - 1 + C::NSTAGE);
                    loaded = u - 1 + C::NSTAGE + 1;
                }
                const int s = u % C::NSTAGE, acc = u % kPrAcc;
                if (!mbar_wait(&k_full[s], (u / C::NSTAGE) & 1, abort_flag)) { ok = false; break; }
                // the sum warps must have read this accumulator (tile u - kPrAcc)
                if (u >= kPrAcc && !mbar_wait(&acc_empty[acc], ((u - kPrAcc) / kPrAcc) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t kd = dK + s * kTile16;
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::SLAB + (kk & 3) * 32) >> 4);
                    umma_bf16(tmem + acc * 128, dQ + off, kd + off, idesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&k_empty[s]);
                umma_commit(&acc_full[acc]);
            }
            if (!ok) {
                if (!*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                // let the loads already issued land before the CTA exits
                mbar_wait(q_full, 0, nullptr);
                for (int u = max(0, loaded - C::NSTAGE); u < loaded; ++u)
                    mbar_wait(&k_full[u % C::NSTAGE], (u / C::NSTAGE) & 1, nullptr);
            }
            // every MMA issued has finished before TMEM is released
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, nullptr);
        }
        __syncwarp();
    } else if (warp < kPrSumWarps) {
        const int quad = warp & 3, part = warp >> 2;
        const int r = quad * 32 + lane;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const int pos = r < a.R ? a.rows[r] : 0;
        const int posc = (pos >= 0 && pos < a.S) ? pos : 0;  // the gather reported a bad position
        const int f0 = posc - posc % a.HW;  // first key of the query's frame
        float m = -INFINITY, l = 0.f, lsp = 0.f;
        bool alive = true;
        for (int u = 0; u < n && alive; ++u) {
            const int acc = u % kPrAcc;
            alive = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (u / kPrAcc) & 1, abort_flag));
            if (!alive) {
                if (lane == 0 && !*abort_flag) { report(a.status, DEV_TIMEOUT); *abort_flag = 1; }
                break;
            }
            tc_fence_after();
            static_assert(kPrCols == 32, "one 32-column TMEM load per warp and tile");
            uint32_t x[32];
            tmem_ld32(t_lane + acc * 128 + part * kPrCols, x);
            tmem_ld_wait();
            // the logits are in registers: hand the accumulator back to the MMA thread
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            const int jc = (kt0 + u) * 128 + part * kPrCols;
            const int nvalid = a.S - jc;  // keys past S were zero-filled
            if (nvalid >= kPrCols)
                profile_chunk<kPrCols, false>(x, jc, nvalid, a.cf, a.HW, f0, m, l, lsp);
            else
                profile_chunk<kPrCols, true>(x, jc, nvalid, a.cf, a.HW, f0, m, l, lsp);
        }
        a.partial[(static_cast<size_t>(bh) * a.nparts + blockIdx.x * (kPrSumWarps / 4) + part) * 128 + r] =
            make_float4(m, l, lsp, 0.f);
    } else {
        // rows blockIdx.x, blockIdx.x + gridDim.x, ... of this head: lane t takes
        // keys hw + t HW, t = lane, lane + 32, ... (an online max and sum), then
        // the warp merges them
        const int T = a.S / a.HW;
        for (int r = blockIdx.x; r < a.R; r += gridDim.x) {
            const int pos = a.rows[r];
            const int hw = (pos >= 0 && pos < a.S) ? pos % a.HW : 0;  // the gather reported a bad position
            const uint4 *qr = reinterpret_cast<const uint4 *>(a.qs + (static_cast<size_t>(bh) * 128 + r) * D);
            float tm = -INFINITY, tl = 0.f;
            for (int t = lane; t < T; t += 32) {
                const uint4 *kr = reinterpret_cast<const uint4 *>(
                    a.k + (static_cast<size_t>(bh) * a.S + hw + static_cast<size_t>(t) * a.HW) * D);
                const float x = dot_bf16<D>(qr, kr) * a.cf;
                if (x > tm) {
                    tl *= ex2_approx(tm - x);
                    tm = x;
                }
                tl += ex2_approx(x - tm);
            }
            const float wm = warp_max(tm);
            tl = warp_sum(tm == -INFINITY ? 0.f : tl * ex2_approx(tm - wm));
            if (lane == 0) a.tpart[static_cast<size_t>(bh) * 128 + r] = make_float2(wm, tl);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kPrSumWarps) {
        tc_fence_after();
        tmem_dealloc(tmem, kPrTmemCols);
    }
}

// One CTA per (b, head), thread r = sampled row: the row's maximum M and
// sums over all keys and its frame from the partials, its (h, w) sum brought
// to M, the two mass fractions; then their means over the rows and the kind.
// The kind compares w_sp * spatial mass with w_tp * temporal mass (both 1
// for the mass rule; 1 / (H W) and 1 / T for the mass-per-key rule).
__global__ void profile_finish_kernel(const float4 *__restrict__ partial, int nparts, const float2 *__restrict__ tpart,
                                      int R, float w_sp, float w_tp, float *__restrict__ masses,
                                      int32_t *__restrict__ kind) {
    __shared__ float red[2][4];
    const int bh = blockIdx.x, r = threadIdx.x;
    float fsp = 0.f, ftp = 0.f;
    if (r < R) {
        const float4 *pr = partial + static_cast<size_t>(bh) * nparts * 128 + r;
        float mx = -INFINITY;
        for (int p = 0; p < nparts; ++p) mx = fmaxf(mx, pr[p * 128].x);
        float l = 0.f, lsp = 0.f;
        for (int p = 0; p < nparts; ++p) {
            const float4 v = pr[p * 128];
            if (v.x == -INFINITY) continue;  // a part that saw no key
            const float f = ex2_approx(v.x - mx);
            l += v.y * f;
            lsp += v.z * f;
        }
        const float2 t = tpart[static_cast<size_t>(bh) * 128 + r];
        // l is 0 only when every part of the row gave up on a wait (the
        // status word then holds VSA_ERR_TIMEOUT): the row adds nothing
        // rather than a NaN
        if (l > 0.f) {
            fsp = lsp / l;
            ftp = t.y * ex2_approx(t.x - mx) / l;
        }
    }
    fsp = warp_sum(fsp);
    ftp = warp_sum(ftp);
    if ((r & 31) == 0) {
        red[0][r >> 5] = fsp;
        red[1][r >> 5] = ftp;
    }
    __syncthreads();
    if (r == 0) {
        const float sp = ((red[0][0] + red[0][1]) + (red[0][2] + red[0][3])) / R;
        const float tp = ((red[1][0] + red[1][1]) + (red[1][2] + red[1][3])) / R;
        masses[2 * bh] = sp;
        masses[2 * bh + 1] = tp;
        kind[bh] = tp * w_tp > sp * w_sp ? 1 : 0;
    }
}

int sm_count_now() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int D>
cudaError_t run_profile(const void *k, const __nv_bfloat16 *qs, int BH, int S, int HW, const int32_t *rows, int R,
                        float scale, int split, float4 *partial, float2 *tpart, int *status, cudaStream_t st) {
    using C = PrCfg<D>;
    CUtensorMap mq, mk;
    if (!make_tile_map(&mq, qs, D, 128, BH, 128) || !make_tile_map(&mk, k, D, S, BH, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(profile_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int n_kt = (S + 127) / 128;
    PrArgs a;
    a.S = S;
    a.HW = HW;
    a.R = R;
    a.tiles_per_cta = (n_kt + split - 1) / split;
    a.nparts = (kPrSumWarps / 4) * split;
    a.cf = scale * 1.4426950408889634f;  // log2(e)
    a.rows = rows;
    a.qs = qs;
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.tpart = tpart;
    a.partial = partial;
    a.status = status;
    profile_kernel<D><<<dim3(split, BH), kPrThreads, C::SMEM, st>>>(mq, mk, a);
    return cudaGetLastError();
}

}  // namespace

int profile_split(int BH, int S) {
    const int n_kt = (S + 127) / 128;
    const int sms = sm_count_now();
    int split = BH >= sms ? 1 : sms / BH;
    split = max(1, min(split, n_kt));
    // every CTA gets at least one key tile
    const int per = (n_kt + split - 1) / split;
    return (n_kt + per - 1) / per;
}

// Scratch: the gathered sample tiles [BH][128][D] bf16, the partials
// [BH][nparts][128] float4, the rows' (h, w) partials [BH][128] float2.
size_t profile_workspace_bytes(int BH, int S, int D) {
    const size_t qs = (static_cast<size_t>(BH) * 128 * D * 2 + 255) & ~static_cast<size_t>(255);
    const size_t part = static_cast<size_t>(BH) * (kPrSumWarps / 4) * profile_split(BH, S) * 128 * sizeof(float4);
    return qs + part + static_cast<size_t>(BH) * 128 * sizeof(float2);
}

cudaError_t launch_head_profile(const void *q, const void *k, int BH, int S, int D, int HW, const int32_t *rows,
                                int R, float scale, int rule, void *workspace, float *masses, int32_t *kind,
                                int *status, cudaStream_t st) {
    const int split = profile_split(BH, S);
    __nv_bfloat16 *qs = static_cast<__nv_bfloat16 *>(workspace);
    const size_t qs_bytes = (static_cast<size_t>(BH) * 128 * D * 2 + 255) & ~static_cast<size_t>(255);
    float4 *partial = reinterpret_cast<float4 *>(static_cast<uint8_t *>(workspace) + qs_bytes);
    const int nparts = (kPrSumWarps / 4) * split;
    float2 *tpart = reinterpret_cast<float2 *>(partial + static_cast<size_t>(BH) * nparts * 128);
    gather_rows_kernel<<<BH, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(q), S, D, rows, R, qs, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = D == 128 ? run_profile<128>(k, qs, BH, S, HW, rows, R, scale, split, partial, tpart, status, st)
                 : run_profile<64>(k, qs, BH, S, HW, rows, R, scale, split, partial, tpart, status, st);
    if (e != cudaSuccess) return e;
    const float w_sp = rule == VSA_PROFILE_MASS_PER_KEY ? 1.0f / static_cast<float>(HW) : 1.0f;
    const float w_tp = rule == VSA_PROFILE_MASS_PER_KEY ? static_cast<float>(HW) / static_cast<float>(S) : 1.0f;
    profile_finish_kernel<<<BH, 128, 0, st>>>(partial, nparts, tpart, R, w_sp, w_tp, masses, kind);
    return cudaGetLastError();
}

}  // namespace vsa
