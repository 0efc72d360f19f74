// bsa.cu -- flat block selection (close reading §02, Eq.(1)): the quadratic
// comparison that scores every eligible leaf's mean summary per query.
//
// One warp per (b, kv-head, t). Leaves are scored 32/G at a time from level 1
// of the pyramid (reduce-scatter with slot = leaf * G + head, then a sum over
// the G heads); a running Top-K sits sorted in lanes 0..K-1 and a batch is
// merged (two bitonic sorts) only when one of its leaves beats the current
// K-th key. Forced leaves enter with key +inf and count against K, as in the
// pyramid walk; ties rank the lower leaf first.
#include "pisa_internal.h"
#include "pisa_walk.cuh"

namespace pisa {

template <typename T, int D, int G>
__global__ void __launch_bounds__(256) bsa_kernel(const T* __restrict__ Q, const float* __restrict__ pyr,
                                                  int32_t* __restrict__ idx, SelectParams p) {
    constexpr int RB = 32 / G;
    const int lane = threadIdx.x & 31;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    if (unit >= units) return;
    const int64_t bh = unit / p.N;
    const int64_t t = unit - bh * p.N;
    const int64_t b = bh / p.Hkv;
    const int kvh = (int)(bh - b * p.Hkv);

    Walk<T, D, G> w;
    {
        const T* qrow[G];
#pragma unroll
        for (int h = 0; h < G; ++h) qrow[h] = Q + (((b * p.Hq + (int64_t)kvh * G + h) * p.N) + t) * D;
        w.load_q(qrow, p.qscale, lane);
    }
    const float* leaves = pyr + bh * p.geom.rows * D;  // level 1 starts at row 0
    const Forced F(t, p.C, p.causal, p.forced_mask);
    const int64_t M1 = p.geom.M[1];
    const int64_t n_elig = p.causal ? min(M1, t / p.C + 1) : M1;

    // running list: lanes 0..K-1 hold the best (key, leaf) pairs, sorted
    float key = -INFINITY;
    int id = 0x7fffffff;
    {
        // forced leaves first (key +inf)
        const int f = lane == 0 ? F.f0 : lane == 1 ? F.f1 : lane == 2 ? F.f2 : -1;
        bool dup = false;
        if (lane == 1) dup = F.f1 == F.f0;
        if (lane == 2) dup = F.f2 == F.f0 || F.f2 == F.f1;
        if (lane < 3 && f >= 0 && !dup && f < n_elig) { key = INFINITY; id = f; }
        warp_sort_desc(key, id, lane);
        if (lane >= p.K) { key = -INFINITY; id = 0x7fffffff; }
    }
    for (int64_t base = 0; base < n_elig; base += RB) {
        float v[32];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int64_t leaf = base + r;
            w.dots_into(v, r, leaves + leaf * D, leaf < n_elig, lane);
        }
        float s = reduce_scatter32(v, lane);
#pragma unroll
        for (int o = 1; o < G; o <<= 1) s += __shfl_xor_sync(kFull, s, o);
        const int64_t leaf = base + lane / G;
        const bool ok = (lane % G) == 0 && leaf < n_elig && !F.has((int)leaf, 1);
        float ck = ok ? s : -INFINITY;
        int ci = ok ? (int)leaf : 0x7fffffff;
        const float kth = __shfl_sync(kFull, key, p.K - 1);
        const int kthi = __shfl_sync(kFull, id, p.K - 1);
        if (__ballot_sync(kFull, ok && ranks_before(ck, ci, kth, kthi)) == 0u) continue;
        warp_sort_desc(ck, ci, lane);  // best of the batch in lanes 0..K-1
        const float mk = __shfl_sync(kFull, ck, (lane - p.K) & 31);
        const int mi = __shfl_sync(kFull, ci, (lane - p.K) & 31);
        if (lane >= p.K) {
            key = lane < 2 * p.K ? mk : -INFINITY;
            id = lane < 2 * p.K ? mi : 0x7fffffff;
        }
        warp_sort_desc(key, id, lane);
        if (lane >= p.K) { key = -INFINITY; id = 0x7fffffff; }
    }
    int v = (lane < p.K && key != -INFINITY) ? id : 0x7fffffff;
    warp_sort_asc(v, lane);
    if (lane < p.K) idx[unit * p.K + lane] = v == 0x7fffffff ? -1 : v;
}

template <typename T, int D, int G>
static cudaError_t launch_bsa_t(const void* Q, const float* pyr, int32_t* idx, const SelectParams& p,
                                cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    bsa_kernel<T, D, G><<<(unsigned)((units + 7) / 8), 256, 0, st>>>((const T*)Q, pyr, idx, p);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_bsa_d(const void* Q, const float* pyr, int32_t* idx, const SelectParams& p,
                                cudaStream_t st) {
    switch (p.Hq / p.Hkv) {
        case 1: return launch_bsa_t<T, D, 1>(Q, pyr, idx, p, st);
        case 2: return launch_bsa_t<T, D, 2>(Q, pyr, idx, p, st);
        case 4: return launch_bsa_t<T, D, 4>(Q, pyr, idx, p, st);
        case 8: return launch_bsa_t<T, D, 8>(Q, pyr, idx, p, st);
        case 16: return launch_bsa_t<T, D, 16>(Q, pyr, idx, p, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_bsa(int dtype, int d, const void* Q, const float* pyr, int32_t* idx, const SelectParams& p,
                       cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_bsa_d<__nv_bfloat16, 128>(Q, pyr, idx, p, st);
        if (d == 64) return launch_bsa_d<__nv_bfloat16, 64>(Q, pyr, idx, p, st);
    } else {
        if (d == 128) return launch_bsa_d<float, 128>(Q, pyr, idx, p, st);
        if (d == 64) return launch_bsa_d<float, 64>(Q, pyr, idx, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
