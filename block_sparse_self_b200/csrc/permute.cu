// permute.cu -- tile-contiguous gather/scatter of token rows, fp32->bf16
// cast, and the bounded-wait test kernel.
//
// "ADR-0001: Sparse-attention roadmap for video DiTs", step 6
// (block_contiguous_permutation / invert_permutation) and "Adaptive tiling
// (SPADE)", Recipe (argsort of tile_labels; argsort(order) to go back).
// Position p of the tile-contiguous order holds token perm(p): tiles in
// row-major tile order, tokens of a tile in T-major order.  perm is computed
// arithmetically from (grid, tile); the chosen tiling of each (b, head) is
// read on the device.  On a zero-padded grid ("Adaptive tiling (SPADE)",
// Deviations and notes) the permuted order covers the padded grid: padding
// positions are written as zero rows, and going back writes real tokens only.
#include "common.cuh"
#include "internal.h"

namespace vsa {

namespace {

struct PermArgs {
    const uint8_t *src;
    uint8_t *dst;
    int S, Sp, BH;             // tokens per head: real (T-major side), padded (permuted side)
    RealGrid real;
    int padded;                // Sp != S
    TileSet tiles;
    TileDivs divs[kMaxTiles];  // per candidate tiling, over the padded grid
    const int32_t *choice;
    int inverse;
    int *status;
};

constexpr int kRowsPerItem = 128;  // permuted rows handled per work item
constexpr int kThreads = 256;

// CPR = 16-byte chunks per row.  Each work item is (bh, 128 consecutive
// permuted positions); lanes move 16-byte chunks, 4 rows in flight per lane.
template <int CPR>
__global__ void __launch_bounds__(kThreads) permute_kernel(const PermArgs a) {
    constexpr int RPP = kThreads / CPR;  // rows per pass
    constexpr int UNROLL = 4;
    const int items_per_head = (a.Sp + kRowsPerItem - 1) / kRowsPerItem;
    const long long n_items = static_cast<long long>(items_per_head) * a.BH;
    const int chunk = threadIdx.x % CPR;
    const int rsub = threadIdx.x / CPR;
    for (long long it = blockIdx.x; it < n_items; it += gridDim.x) {
        const int bh = static_cast<int>(it / items_per_head);
        const int p0 = static_cast<int>(it - static_cast<long long>(bh) * items_per_head) * kRowsPerItem;
        int c = 0;
        if (a.choice) {
            c = __ldg(a.choice + bh);
            if (c < 0 || c >= a.tiles.n) {
                if (threadIdx.x == 0) report(a.status, DEV_RUNTIME);
                continue;
            }
        }
        const TileDivs dv = a.divs[c];
        const size_t head_t = static_cast<size_t>(bh) * a.S, head_p = static_cast<size_t>(bh) * a.Sp;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.src);
        uint4 *dst = reinterpret_cast<uint4 *>(a.dst);
        #pragma unroll 1
        for (int r0 = 0; r0 < kRowsPerItem; r0 += RPP * UNROLL) {
            uint4 v[UNROLL];
            size_t drow[UNROLL];
            bool ok[UNROLL];
            #pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int p = p0 + r0 + u * RPP + rsub;
                ok[u] = (r0 + u * RPP + rsub) < kRowsPerItem && p < a.Sp;
                if (ok[u]) {
                    int tok;
                    if (a.padded) {
                        uint32_t t, h, w;
                        tile_coords_fast(static_cast<uint32_t>(p), dv, t, h, w);
                        tok = real_token(t, h, w, a.real);
                    } else {
                        tok = static_cast<int>(tile_token_fast(static_cast<uint32_t>(p), dv));
                    }
                    if (a.inverse) {  // padding positions have no token to go back to
                        ok[u] = tok >= 0;
                        drow[u] = head_t + tok;
                        if (ok[u]) v[u] = __ldcs(src + (head_p + p) * CPR + chunk);
                    } else {          // padding positions become zero rows
                        drow[u] = head_p + p;
                        v[u] = tok >= 0 ? __ldcs(src + (head_t + tok) * CPR + chunk) : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            #pragma unroll
            for (int u = 0; u < UNROLL; ++u)
                if (ok[u]) dst[drow[u] * CPR + chunk] = v[u];
        }
    }
}

__global__ void cast_kernel(const float *__restrict__ x, __nv_bfloat16 *__restrict__ y, int64_t n) {
    const int64_t n4 = n / 4;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
        const float4 v = reinterpret_cast<const float4 *>(x)[i];
        uint2 o;
        o.x = pack_bf16x2(v.x, v.y);
        o.y = pack_bf16x2(v.z, v.w);
        reinterpret_cast<uint2 *>(y)[i] = o;
    }
    for (int64_t i = n4 * 4 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
        y[i] = __float2bfloat16_rn(x[i]);
}

__global__ void wait_timeout_kernel(uint64_t limit_ns, int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: the wait must give up after limit_ns.
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, nullptr, limit_ns)) report(status, DEV_TIMEOUT);
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace

cudaError_t launch_permute(const void *src, void *dst, int esize, int BH, int D, int T, int H, int W, int Tp, int Hp,
                           int Wp, const TileSet &tiles, const int32_t *choice, bool inverse, int *status,
                           cudaStream_t st) {
    PermArgs a;
    a.src = static_cast<const uint8_t *>(src);
    a.dst = static_cast<uint8_t *>(dst);
    a.S = T * H * W;
    a.Sp = Tp * Hp * Wp;
    a.real = RealGrid{T, H, W};
    a.padded = a.Sp != a.S;
    a.BH = BH;
    a.tiles = tiles;
    for (int c = 0; c < kMaxTiles; ++c)
        a.divs[c] = c < tiles.n ? make_tile_divs(Hp, Wp, tiles.t[c], tiles.h[c], tiles.w[c]) : make_tile_divs(1, 1, 1, 1, 1);
    a.choice = choice;
    a.inverse = inverse ? 1 : 0;
    a.status = status;
    const int cpr = D * esize / 16;
    const long long items = static_cast<long long>((a.Sp + kRowsPerItem - 1) / kRowsPerItem) * BH;
    const int grid = static_cast<int>(items < 16LL * sm_count() ? items : 16LL * sm_count());
    switch (cpr) {
        case 8: permute_kernel<8><<<grid, kThreads, 0, st>>>(a); break;
        case 16: permute_kernel<16><<<grid, kThreads, 0, st>>>(a); break;
        case 32: permute_kernel<32><<<grid, kThreads, 0, st>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_cast_f32_bf16(const float *x, void *y, int64_t n, cudaStream_t st) {
    const int64_t blocks = (n / 4 + 255) / 256 + 1;
    const int grid = static_cast<int>(blocks < 8LL * sm_count() ? blocks : 8LL * sm_count());
    cast_kernel<<<grid, 256, 0, st>>>(x, static_cast<__nv_bfloat16 *>(y), n);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout(uint64_t limit_ns, int *status, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(limit_ns, status);
    return cudaGetLastError();
}

}  // namespace vsa
