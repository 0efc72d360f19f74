// attn.cu -- attention over the selected leaf blocks (close reading §02,
// Eq.(2); §5.3 causal mask inside the block), one warp per (b, kv-head, t)
// serving the G query heads that share the selection.
//
// The per-warp online softmax lives in pisa_attn.cuh; this file maps warps
// to query rows and writes the normalised output.
#include "pisa_internal.h"
#include "pisa_attn.cuh"

namespace pisa {

template <typename T, int D, int G>
__global__ void __launch_bounds__(256) attn_kernel(const T* __restrict__ Q, const T* __restrict__ Kmat,
                                                   const T* __restrict__ Vmat, const int32_t* __restrict__ idx,
                                                   T* __restrict__ O, AttnParams p) {
    constexpr int VD = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t unit = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    if (unit >= units) return;
    const int64_t bh = unit / p.N;
    const int64_t t = unit - bh * p.N;
    const int64_t b = bh / p.Hkv;
    const int kvh = (int)(bh - b * p.Hkv);

    Walk<T, D, G> w;
    const T* qrow[G];
#pragma unroll
    for (int h = 0; h < G; ++h) qrow[h] = Q + (((b * p.Hq + (int64_t)kvh * G + h) * p.N) + t) * D;
    w.load_q(qrow, p.qscale, lane);
    const T* Kh = Kmat + bh * p.N * D;
    const T* Vh = Vmat + bh * p.N * D;

    const int my_blk = lane < p.K ? idx[unit * p.K + lane] : -1;
    AttnAcc<T, D, G> acc;
    acc.init();
    for (int k = 0; k < p.K; ++k) {
        const int blk = __shfl_sync(kFull, my_blk, k);
        if (blk < 0) continue;
        const int64_t lo = (int64_t)blk * p.C;
        int64_t hi = min(lo + p.C, (int64_t)p.N);
        if (p.causal) hi = min(hi, t + 1);
        if (lo >= hi) continue;
        acc.block(w, Kh, Vh, lo, hi, lane);
    }
    acc.finish(lane);
#pragma unroll
    for (int h = 0; h < G; ++h) {
        T* dst = O + (((b * p.Hq + (int64_t)kvh * G + h) * p.N) + t) * D + lane * VD;
        store_vec<T, VD>(dst, acc.o[h]);
    }
}

template <typename T, int D, int G>
static cudaError_t launch_attn_t(const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                                 const AttnParams& p, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Hkv * p.N;
    attn_kernel<T, D, G><<<(unsigned)((units + 7) / 8), 256, 0, st>>>((const T*)Q, (const T*)K, (const T*)V,
                                                                        idx, (T*)O, p);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_attn_d(const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                                 const AttnParams& p, cudaStream_t st) {
    switch (p.Hq / p.Hkv) {
        case 1: return launch_attn_t<T, D, 1>(Q, K, V, idx, O, p, st);
        case 2: return launch_attn_t<T, D, 2>(Q, K, V, idx, O, p, st);
        case 4: return launch_attn_t<T, D, 4>(Q, K, V, idx, O, p, st);
        case 8: return launch_attn_t<T, D, 8>(Q, K, V, idx, O, p, st);
        case 16: return launch_attn_t<T, D, 16>(Q, K, V, idx, O, p, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn(int dtype, int d, const void* Q, const void* K, const void* V, const int32_t* idx,
                        void* O, const AttnParams& p, cudaStream_t st) {
    if (dtype == 1) {
        if (d == 128) return launch_attn_d<__nv_bfloat16, 128>(Q, K, V, idx, O, p, st);
        if (d == 64) return launch_attn_d<__nv_bfloat16, 64>(Q, K, V, idx, O, p, st);
    } else {
        if (d == 128) return launch_attn_d<float, 128>(Q, K, V, idx, O, p, st);
        if (d == 64) return launch_attn_d<float, 64>(Q, K, V, idx, O, p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pisa
