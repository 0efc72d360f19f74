// pool.cu -- key pyramid (close reading §04 4.1, Eq.(3)-(4)).
//
// pool_leaves_kernel: one CTA per 16 consecutive leaves of one (b, kv-head).
// Warps stream the raw keys once with 16-byte loads, reduce each leaf to its
// fp32 mean, and finish the CTA's subtree (levels 2..5) in shared memory, so K
// is read exactly once. pool_top_kernel: one CTA per head finishes the few
// levels above (each node the mean of its existing children).
#include "pisa_internal.h"

namespace pisa {

constexpr int kLeavesPerCta = 16;  // the CTA subtree spans levels 1..5

__device__ __forceinline__ int64_t keys_of(const PoolParams& p, int64_t b) {
    if (!p.len) return p.N;
    int64_t n = p.len[b];
    return n < 0 ? 0 : (n > p.k_rows ? p.k_rows : n);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) pool_leaves_kernel(const T* __restrict__ K, float* __restrict__ pyr,
                                                          PoolParams p) {
    constexpr int E = Ld16<T>::E;   // elements per 16-byte load
    constexpr int TPR = D / E;      // lanes per row
    constexpr int RPW = 32 / TPR;   // rows per warp step
    constexpr int LPC = kLeavesPerCta;
    __shared__ __align__(16) float sm[2][LPC][D];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t bh = blockIdx.y;
    const int64_t len = keys_of(p, bh / p.Hkv);
    const int C = p.C;
    const T* Kh = K + bh * p.k_rows * D;
    float* P = pyr + bh * p.geom.rows * D;
    const int64_t leaf0 = (int64_t)blockIdx.x * LPC;
    const int64_t live_leaves = (len + C - 1) / C;
    const int rsub = lane / TPR, col = (lane % TPR) * E;

    for (int li = warp; li < LPC; li += 8) {
        const int64_t leaf = leaf0 + li;
        if (leaf >= live_leaves) break;
        const int64_t lo = leaf * C, hi = min(lo + C, len);
        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        int64_t r = lo + rsub;
        for (; r + 3 * RPW < hi; r += 4 * RPW) {
            float x0[E], x1[E], x2[E], x3[E];
            Ld16<T>::run(Kh + r * D + col, x0);
            Ld16<T>::run(Kh + (r + RPW) * D + col, x1);
            Ld16<T>::run(Kh + (r + 2 * RPW) * D + col, x2);
            Ld16<T>::run(Kh + (r + 3 * RPW) * D + col, x3);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += (x0[e] + x1[e]) + (x2[e] + x3[e]);
        }
        for (; r < hi; r += RPW) {
            float x[E];
            Ld16<T>::run(Kh + r * D + col, x);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += x[e];
        }
#pragma unroll
        for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += __shfl_xor_sync(kFull, acc[e], o);
        const float inv = 1.f / (float)(hi - lo);
        if (rsub == 0) {
            float* dst = P + (p.geom.off[1] + leaf) * D + col;
#pragma unroll
            for (int e = 0; e < E; e += 4) {
                const float4 v = make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
                *reinterpret_cast<float4*>(dst + e) = v;
                *reinterpret_cast<float4*>(&sm[0][li][col + e]) = v;
            }
        }
    }
    __syncthreads();

    int cur = 0;
    for (int l = 2, nodes = LPC / 2; l <= p.geom.L && nodes >= 1; ++l, nodes >>= 1) {
        const int64_t span = (int64_t)C << (l - 1), cspan = span >> 1;
        const int64_t node0 = (int64_t)blockIdx.x * nodes;
        for (int i = threadIdx.x; i < nodes * D; i += blockDim.x) {
            const int nl = i / D, e = i - nl * D;
            const int64_t node = node0 + nl;
            if (node * span >= len) continue;
            float a = sm[cur][2 * nl][e];
            if ((2 * node + 1) * cspan < len) a = (a + sm[cur][2 * nl + 1][e]) * 0.5f;
            sm[cur ^ 1][nl][e] = a;
            P[(p.geom.off[l] + node) * D + e] = a;
        }
        __syncthreads();
        cur ^= 1;
    }
}

// levels first_level..L of one (b, kv-head), each node the mean of its
// existing children one level down (already written).
__global__ void __launch_bounds__(512) pool_top_kernel(float* __restrict__ pyr, PoolParams p, int D,
                                                       int first_level) {
    const int64_t bh = blockIdx.x;
    const int64_t len = keys_of(p, bh / p.Hkv);
    float* P = pyr + bh * p.geom.rows * D;
    for (int l = first_level; l <= p.geom.L; ++l) {
        const int64_t span = (int64_t)p.C << (l - 1), cspan = span >> 1;
        const int64_t n = p.geom.M[l] * D;
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
            const int64_t node = i / D;
            const int e = (int)(i - node * D);
            if (node * span >= len) continue;
            float a = P[(p.geom.off[l - 1] + 2 * node) * D + e];
            if ((2 * node + 1) * cspan < len) a = (a + P[(p.geom.off[l - 1] + 2 * node + 1) * D + e]) * 0.5f;
            P[(p.geom.off[l] + node) * D + e] = a;
        }
        __syncthreads();
    }
}

template <typename T, int D>
static cudaError_t launch_pool_t(const void* K, float* pyr, const PoolParams& p, cudaStream_t st) {
    const int64_t M1 = p.geom.M[1];
    dim3 grid((unsigned)((M1 + kLeavesPerCta - 1) / kLeavesPerCta), (unsigned)(p.B * p.Hkv));
    pool_leaves_kernel<T, D><<<grid, 256, 0, st>>>((const T*)K, pyr, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int first = 2 + 4;  // log2(kLeavesPerCta) = 4 levels above the leaves done in-CTA
    if (p.geom.L >= first) {
        pool_top_kernel<<<(unsigned)(p.B * p.Hkv), 512, 0, st>>>(pyr, p, D, first);
        e = cudaGetLastError();
    }
    return e;
}

// Pyramid cache growth (close reading §5.3, decode cache: the capacity grows by
// a fixed ratio). Row r of the new layout (level l, node i) takes old row
// (l, i) when that node exists in the old layout; node 0 of a level above the
// old root takes the old root (its second child starts past the old capacity,
// so at any length the old layout can hold it is the mean of one node: the
// old root); every other row is zero until tokens reach it. One warp per row.
__global__ void __launch_bounds__(256) pyramid_grow_kernel(const float* __restrict__ old_pyr,
                                                           float* __restrict__ new_pyr, int64_t units, int d,
                                                           Geom go, Geom gn) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= units * gn.rows) return;
    const int64_t u = row / gn.rows, r = row - u * gn.rows;
    int l = 1;
    while (l < gn.L && r >= gn.off[l + 1]) ++l;
    const int64_t i = r - gn.off[l];
    int64_t src = -1;
    if (l <= go.L && i < go.M[l]) src = go.off[l] + i;
    else if (l > go.L && i == 0) src = go.off[go.L];
    const float* from = old_pyr + (u * go.rows + (src < 0 ? 0 : src)) * d;
    float* to = new_pyr + row * d;
    for (int e = lane; e < d; e += 32) to[e] = src >= 0 ? from[e] : 0.f;
}

cudaError_t launch_pyramid_grow(const float* old_pyr, float* new_pyr, int64_t units, int d, const Geom& go,
                                const Geom& gn, cudaStream_t st) {
    const int64_t rows = units * gn.rows;
    pyramid_grow_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(old_pyr, new_pyr, units, d, go, gn);
    return cudaGetLastError();
}

// K or V cache rows into a cache of a larger capacity: per (b, kv-head) unit,
// rows [0, rows_old) are copied and rows [rows_old, rows_new) are zeroed; one
// 16-byte chunk per thread and step of a grid-stride loop.
__global__ void __launch_bounds__(256) cache_grow_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         int64_t units, int64_t rows_old, int64_t rows_new,
                                                         int chunks) {
    const int64_t total = units * rows_new * chunks;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = i % chunks, r = (i / chunks) % rows_new, u = i / (chunks * rows_new);
        dst[i] = r < rows_old ? src[(u * rows_old + r) * chunks + c] : make_uint4(0u, 0u, 0u, 0u);
    }
}

cudaError_t launch_cache_grow(const void* src, void* dst, int64_t units, int64_t rows_old, int64_t rows_new,
                              int row_bytes, cudaStream_t st) {
    const int chunks = row_bytes / 16;
    const int64_t total = units * rows_new * chunks;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + 255) / 256, cap = (int64_t)sms * 16;
    cache_grow_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, st>>>((const uint4*)src, (uint4*)dst, units,
                                                                          rows_old, rows_new, chunks);
    return cudaGetLastError();
}

cudaError_t launch_pool(int dtype, int d, const void* K, float* pyr, const PoolParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_pool_t<__nv_bfloat16, 128>(K, pyr, p, st);
        if (d == 64) return launch_pool_t<__nv_bfloat16, 64>(K, pyr, p, st);
    } else {
        if (d == 128) return launch_pool_t<float, 128>(K, pyr, p, st);
        if (d == 64) return launch_pool_t<float, 64>(K, pyr, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
