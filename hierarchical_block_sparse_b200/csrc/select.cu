// select.cu -- pyramid Top-K selection, one warp per (b, kv-head, query t).
//
// close reading §04 4.2-4.4 (Eq.(5)-(7), (11)) and §5.3: starting from the
// root, each level keeps all eligible candidates when there are at most K,
// else the forced ones plus the best-scoring others; the kept nodes' children
// become the next level's candidates; the kept leaves are written sorted
// ascending and padded with -1.
#include "pisa_internal.h"
#include "pisa_walk.cuh"

namespace pisa {

template <typename T, int D, int G>
__global__ void __launch_bounds__(256) select_kernel(const T* __restrict__ Q, const T* __restrict__ Kmat,
                                                     const float* __restrict__ pyr,
                                                     int32_t* __restrict__ idx, SelectParams p) {
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
    const T* Kh = Kmat + bh * p.N * D;
    const float* P = pyr + bh * p.geom.rows * D;
    const Forced F(t, p.C, p.causal, p.forced_mask);

    int cand = lane == 0 ? 0 : -1;
    for (int l = p.geom.L; l >= 1; --l) {
        const LevelState s = level_state(cand, l, p.C, p.N, t, p.causal, F);
        float score = -INFINITY;
        if (s.n > p.K) {
            const unsigned fmask = __ballot_sync(kFull, s.forced);
            if (__popc(fmask) < p.K) {
                const unsigned need = s.vmask & ~fmask;
                if (l >= 2)
                    score = w.score_internal(cand, need, P + p.geom.off[l - 1] * D,
                                             (int64_t)p.C << (l - 2), p.N, lane, p.variant);
                else
                    score = w.score_leaves(cand, need, Kh, p.C, p.N, lane, p.variant);
            }
        }
        int id = cand;
        const int kept = keep_topk(id, score, s, p.K, lane);
        if (l > 1) {
            const int parent = __shfl_sync(kFull, id, lane >> 1);
            cand = lane < 2 * kept ? 2 * parent + (lane & 1) : -1;
        } else {
            int v = lane < kept ? id : 0x7fffffff;
            warp_sort_asc(v, lane);
            if (lane < p.K) idx[unit * p.K + lane] = v == 0x7fffffff ? -1 : v;
        }
    }
}

template <typename T, int D, int G>
static cudaError_t launch_select_t(const void* Q, const void* K, const float* pyr, int32_t* idx,
                                   const SelectParams& p, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    const int64_t blocks = (units + 7) / 8;
    select_kernel<T, D, G><<<(unsigned)blocks, 256, 0, st>>>((const T*)Q, (const T*)K, pyr, idx, p);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_select_d(const void* Q, const void* K, const float* pyr, int32_t* idx,
                                   const SelectParams& p, cudaStream_t st) {
    switch (p.Hq / p.Hkv) {
        case 1: return launch_select_t<T, D, 1>(Q, K, pyr, idx, p, st);
        case 2: return launch_select_t<T, D, 2>(Q, K, pyr, idx, p, st);
        case 4: return launch_select_t<T, D, 4>(Q, K, pyr, idx, p, st);
        case 8: return launch_select_t<T, D, 8>(Q, K, pyr, idx, p, st);
        case 16: return launch_select_t<T, D, 16>(Q, K, pyr, idx, p, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_select(int dtype, int d, const void* Q, const void* K, const float* pyr, int32_t* idx,
                          const SelectParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_select_d<__nv_bfloat16, 128>(Q, K, pyr, idx, p, st);
        if (d == 64) return launch_select_d<__nv_bfloat16, 64>(Q, K, pyr, idx, p, st);
    } else {
        if (d == 128) return launch_select_d<float, 128>(Q, K, pyr, idx, p, st);
        if (d == 64) return launch_select_d<float, 64>(Q, K, pyr, idx, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
